// Library-wide runtime pieces: error reporting, the device error word,
// per-device caches, the TMA descriptor encoder and the bounded-wait
// self-test.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>
#include <vector>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {
thread_local char g_last_error[512] = "no error";
constexpr int kMaxDevices = 64;
int32_t* g_err_word[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
}  // namespace

// OR of PA_DEVERR_* bits raised by any kernel of this library on a device.
__device__ int32_t g_device_error_word = 0;

int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return status;
}

int check_output_pointer(const void* out, const char* who) {
  cudaPointerAttributes at;
  const cudaError_t e = cudaPointerGetAttributes(&at, out);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(PA_ERR_INVALID, "%s: out is not a CUDA-visible pointer (%s)", who, cudaGetErrorString(e));
  }
  switch (at.type) {
    case cudaMemoryTypeDevice:
    case cudaMemoryTypeManaged:
      return PA_OK;
    case cudaMemoryTypeHost:
      if (at.devicePointer == out) return PA_OK;
      return fail(PA_ERR_INVALID, "%s: out is pinned host memory mapped at another device address", who);
    default:
      return fail(PA_ERR_INVALID, "%s: out is pageable host memory; pass device or pinned host memory", who);
  }
}

static int current_device(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) {
    fail(PA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  if (*dev < 0 || *dev >= kMaxDevices) {
    fail(PA_ERR_UNSUPPORTED, "device ordinal %d beyond %d", *dev, kMaxDevices);
    return PA_ERR_UNSUPPORTED;
  }
  return PA_OK;
}

int32_t* device_error_word() {
  int dev;
  if (current_device(&dev) != PA_OK) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_err_word[dev] == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_device_error_word);
    if (e != cudaSuccess) {
      fail(PA_ERR_CUDA, "cudaGetSymbolAddress(error word): %s", cudaGetErrorString(e));
      return nullptr;
    }
    g_err_word[dev] = static_cast<int32_t*>(p);
  }
  return g_err_word[dev];
}

int sm_count() {
  int dev;
  if (current_device(&dev) != PA_OK) return 0;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_sm_count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 0;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

// The attribute is set once per (kernel, device) and raised only when a
// launch needs more, so steady-state launches (and launches recorded into a
// CUDA graph after a first eager call) make no attribute calls.
int set_smem_attr(const void* kernel, int bytes) {
  struct Entry {
    const void* kernel;
    int device;
    int bytes;
  };
  static std::vector<Entry> done;
  int dev;
  if (current_device(&dev) != PA_OK) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  for (Entry& e : done)
    if (e.kernel == kernel && e.device == dev && e.bytes >= bytes) return PA_OK;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess)
    return fail(PA_ERR_CUDA, "cudaFuncSetAttribute(%d bytes smem): %s", bytes,
                cudaGetErrorString(e));
  bool found = false;
  for (Entry& x : done)
    if (x.kernel == kernel && x.device == dev) {
      x.bytes = bytes;
      found = true;
    }
  if (!found) done.push_back({kernel, dev, bytes});
  return PA_OK;
}

// L2 fetch granularity of the TMA loads (build-time tuning; the decode
// boxes read 128-byte halves of 256-byte rows, so 256-byte promotion brings
// the other half into L2 with the first).
#ifndef PA_TMA_L2_PROMOTION
#define PA_TMA_L2_PROMOTION CU_TENSOR_MAP_L2_PROMOTION_L2_256B
#endif

int encode_tensor_map(void* desc, int rank, void* base, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box, int swizzle_128b) {
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
      if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr)
        return fail(PA_ERR_CUDA, "driver entry point cuTensorMapEncodeTiled unavailable");
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  cuuint64_t d[5];
  cuuint64_t s[4];
  cuuint32_t b[5];
  cuuint32_t es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) s[i] = strides_bytes[i];
  }
  CUresult r = g_encode(static_cast<CUtensorMap*>(desc), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        static_cast<cuuint32_t>(rank), base, d, s, b, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle_128b ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        PA_TMA_L2_PROMOTION, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return PA_OK;
}

// One thread waits on a barrier phase that nothing completes.
__global__ void selftest_wait_timeout_kernel(uint64_t limit_ns, int32_t* err) {
  __shared__ alignas(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
    if (!mbar_wait_bounded(smem_u32(&bar), 0, limit_ns)) flag_error(err, PA_DEVERR_WAIT_TIMEOUT);
  }
}

}  // namespace pa

extern "C" {

int pa_version(void) { return 100; }

const char* pa_last_error_string(void) { return pa::g_last_error; }

int pa_device_error(int32_t* code_out, int clear) {
  if (code_out == nullptr) return pa::fail(PA_ERR_INVALID, "pa_device_error: code_out is NULL");
  if (pa::device_error_word() == nullptr) return PA_ERR_CUDA;
  PA_CUDA_TRY(cudaDeviceSynchronize());
  int32_t v = 0;
  PA_CUDA_TRY(cudaMemcpyFromSymbol(&v, pa::g_device_error_word, sizeof(v)));
  if (clear) {
    const int32_t zero = 0;
    PA_CUDA_TRY(cudaMemcpyToSymbol(pa::g_device_error_word, &zero, sizeof(zero)));
  }
  *code_out = v;
  return PA_OK;
}

int pa_selftest_wait_timeout(int64_t limit_ns, void* stream) {
  if (limit_ns <= 0 || limit_ns > 5000000000ll)
    return pa::fail(PA_ERR_INVALID, "limit_ns must be in (0, 5e9], got %lld", (long long)limit_ns);
  int32_t* err = pa::device_error_word();
  if (err == nullptr) return PA_ERR_CUDA;
  pa::selftest_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_ns), err);
  PA_CUDA_TRY(cudaGetLastError());
  return PA_OK;
}

}  // extern "C"
