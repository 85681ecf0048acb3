// Host-side helpers shared by the translation units of libpa.so.
#pragma once

#include <cstdarg>
#include <cstdint>

#include "pa.h"

namespace pa {

// Record a message for pa_last_error_string() and return `status`.
int fail(int status, const char* fmt, ...);

// Return PA_OK after clearing nothing (the last message stays until the
// next failure, like errno).
inline int ok() { return PA_OK; }

// Device address of the device error word on the current device (set up
// once per device).  Returns nullptr and records a message on failure.
int32_t* device_error_word();

// Where a kernel may store its output: device (or managed) memory, or
// page-locked host memory that the device addresses at the same pointer
// (cudaHostAlloc / cudaHostRegister under unified addressing), which the
// kernels then write across PCIe as each result is final.  Pageable host
// memory and pointers CUDA does not know are refused with PA_ERR_INVALID
// (a kernel store there would fault).  `who` names the call in the message.
int check_output_pointer(const void* out, const char* who);

// Streaming multiprocessor count of the current device (cached).
int sm_count();

// Opt a kernel into `bytes` of dynamic shared memory on the current device.
int set_smem_attr(const void* kernel, int bytes);

// Encode a tiled TMA descriptor through the driver entry point.
// Writes 128 bytes into `desc` (64-byte aligned).  Returns PA_OK or
// PA_ERR_CUDA with a message.
int encode_tensor_map(void* desc, int rank, void* base, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box, int swizzle_128b);

}  // namespace pa

#define PA_CUDA_TRY(expr)                                                            \
  do {                                                                               \
    cudaError_t pa_e_ = (expr);                                                      \
    if (pa_e_ != cudaSuccess)                                                        \
      return ::pa::fail(PA_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(pa_e_));    \
  } while (0)
