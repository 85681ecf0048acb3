// pa_decode_noalloc: pa_decode with its split-K scratch in a fixed array
// compiled into the library, for callers that cannot allocate device memory
// (a plugin inside a host program that owns the GPU memory budget, or a
// decode loop that cannot afford cudaMalloc's implicit synchronisation).
//
// The array is a file-scope __device__ variable: its name in host code is
// only a stand-in, so the device address is looked up once per device with
// cudaGetSymbolAddress (on the first call, that device current) and passed
// to the kernels as the workspace pointer.
#include <cuda_runtime.h>

#include <mutex>

#include "pa_internal.h"

namespace pa {
namespace {

constexpr size_t kScratchBytes = PA_NOALLOC_SCRATCH_BYTES;

// Split-K partials of every pa_decode_noalloc call on this device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

int scratch_address(void** out) {
  int dev = -1;
  PA_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices)
    return fail(PA_ERR_UNSUPPORTED, "pa_decode_noalloc: device ordinal %d beyond %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(PA_ERR_CUDA, "pa_decode_noalloc: cudaGetSymbolAddress(scratch): %s",
                  cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return PA_OK;
}

}  // namespace
}  // namespace pa

extern "C" int pa_decode_noalloc(pa_bf16* out, const pa_bf16* q, const pa_bf16* kv_pool,
                                 const int32_t* block_tables, const int32_t* seq_lens, int batch,
                                 int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                 int num_blocks, int max_blocks_per_seq, int max_seq_len,
                                 float scale, void* stream) {
  size_t need = 0;
  int parts = 0;
  int rc = pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, block_size,
                                    max_seq_len, &need, &parts);
  if (rc != PA_OK) return rc;
  if (need > pa::kScratchBytes)
    return pa::fail(PA_ERR_UNSUPPORTED,
                    "pa_decode_noalloc: this call needs %zu bytes of split-K scratch, above the "
                    "built-in %zu; use pa_decode with a caller workspace",
                    need, pa::kScratchBytes);
  void* scratch = nullptr;
  rc = pa::scratch_address(&scratch);
  if (rc != PA_OK) return rc;
  return pa_decode(out, q, kv_pool, block_tables, seq_lens, batch, num_q_heads, num_kv_heads,
                   head_dim, block_size, num_blocks, max_blocks_per_seq, max_seq_len, scale, scratch,
                   pa::kScratchBytes, stream);
}
