// pa_reshape_and_cache and pa_copy_blocks: bit-exact data movement into and
// within the paged KV pool, with 16-byte vector loads and stores.
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

// One thread moves one 16-byte chunk of one (token, k/v, head) row.  Thread
// order is (token, head, k/v, chunk) with the chunk fastest, so a warp moves
// whole contiguous rows on both sides.
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4* __restrict__ key, const uint4* __restrict__ value, uint4* __restrict__ pool,
    const int64_t* __restrict__ slot_mapping, int64_t total, int num_kv_heads, int block_size,
    int chunks, int64_t num_slots, int32_t* err) {
  pdl_trigger();
  pdl_wait();
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int chunk = static_cast<int>(idx % chunks);
  int64_t row = idx / chunks;
  const int kv = static_cast<int>(row & 1);
  row >>= 1;
  const int head = static_cast<int>(row % num_kv_heads);
  const int64_t token = row / num_kv_heads;
  const int64_t slot = __ldg(slot_mapping + token);
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (chunk == 0 && kv == 0 && head == 0) flag_error(err, PA_DEVERR_SLOT);
    return;
  }
  const int64_t block = slot / block_size;
  const int64_t offset = slot - block * block_size;
  const uint4* src = (kv ? value : key) + (token * num_kv_heads + head) * chunks + chunk;
  const int64_t dst_row = ((block * 2 + kv) * num_kv_heads + head) * block_size + offset;
  pool[dst_row * chunks + chunk] = __ldg(src);
}

// grid.x = pair, grid.y = slice of the block; each thread copies kUnroll
// 16-byte vectors with all loads issued before the stores.
constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(
    uint4* __restrict__ pool, const int32_t* __restrict__ pairs, int num_blocks,
    int64_t vecs_per_block, int32_t* err) {
  pdl_trigger();
  pdl_wait();
  const int src = __ldg(pairs + 2 * blockIdx.x);
  const int dst = __ldg(pairs + 2 * blockIdx.x + 1);
  if (static_cast<unsigned>(src) >= static_cast<unsigned>(num_blocks) ||
      static_cast<unsigned>(dst) >= static_cast<unsigned>(num_blocks)) {
    if (blockIdx.y == 0 && threadIdx.x == 0) flag_error(err, PA_DEVERR_COPY_PAIR);
    return;
  }
  const uint4* s = pool + src * vecs_per_block;
  uint4* d = pool + dst * vecs_per_block;
  const int64_t base =
      static_cast<int64_t>(blockIdx.y) * kCopyThreads * kCopyUnroll + threadIdx.x;
  uint4 v[kCopyUnroll];
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u) {
    const int64_t i = base + static_cast<int64_t>(u) * kCopyThreads;
    if (i < vecs_per_block) v[u] = s[i];
  }
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u) {
    const int64_t i = base + static_cast<int64_t>(u) * kCopyThreads;
    if (i < vecs_per_block) d[i] = v[u];
  }
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace pa

extern "C" {

int pa_reshape_and_cache(const pa_bf16* key, const pa_bf16* value, pa_bf16* kv_pool,
                         const int64_t* slot_mapping, int num_tokens, int num_blocks,
                         int num_kv_heads, int block_size, int head_dim, void* stream) {
  using namespace pa;
  if (num_tokens < 0 || num_blocks <= 0 || num_kv_heads <= 0 || block_size <= 0 || head_dim <= 0)
    return fail(PA_ERR_INVALID, "pa_reshape_and_cache: non-positive size");
  if (head_dim % 8 != 0)
    return fail(PA_ERR_INVALID, "pa_reshape_and_cache: head_dim %d not a multiple of 8", head_dim);
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !kv_pool || !slot_mapping)
    return fail(PA_ERR_INVALID, "pa_reshape_and_cache: NULL pointer");
  if (!aligned16(key) || !aligned16(value) || !aligned16(kv_pool) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return fail(PA_ERR_INVALID, "pa_reshape_and_cache: misaligned pointer");
  int32_t* err = device_error_word();
  if (err == nullptr) return PA_ERR_CUDA;
  const int chunks = head_dim / 8;
  const int64_t total = static_cast<int64_t>(num_tokens) * num_kv_heads * 2 * chunks;
  const int64_t grid = (total + 255) / 256;
  if (grid > 0x7fffffffll) return fail(PA_ERR_INVALID, "pa_reshape_and_cache: too many tokens");
  PA_CUDA_TRY(launch_pdl(reshape_and_cache_kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0,
                         static_cast<cudaStream_t>(stream), reinterpret_cast<const uint4*>(key),
                         reinterpret_cast<const uint4*>(value), reinterpret_cast<uint4*>(kv_pool),
                         slot_mapping, total, num_kv_heads, block_size, chunks,
                         static_cast<int64_t>(num_blocks) * block_size, err));
  return PA_OK;
}

int pa_copy_blocks(pa_bf16* kv_pool, const int32_t* block_pairs, int num_pairs, int num_blocks,
                   int num_kv_heads, int block_size, int head_dim, void* stream) {
  using namespace pa;
  if (num_pairs < 0 || num_blocks <= 0 || num_kv_heads <= 0 || block_size <= 0 || head_dim <= 0)
    return fail(PA_ERR_INVALID, "pa_copy_blocks: non-positive size");
  if (head_dim % 8 != 0)
    return fail(PA_ERR_INVALID, "pa_copy_blocks: head_dim %d not a multiple of 8", head_dim);
  if (num_pairs == 0) return PA_OK;
  if (!kv_pool || !block_pairs) return fail(PA_ERR_INVALID, "pa_copy_blocks: NULL pointer");
  if (!aligned16(kv_pool) || (reinterpret_cast<uintptr_t>(block_pairs) & 3u))
    return fail(PA_ERR_INVALID, "pa_copy_blocks: misaligned pointer");
  if (num_pairs > 0x7fffffff) return fail(PA_ERR_INVALID, "pa_copy_blocks: too many pairs");
  int32_t* err = device_error_word();
  if (err == nullptr) return PA_ERR_CUDA;
  const int64_t vecs = static_cast<int64_t>(2) * num_kv_heads * block_size * head_dim / 8;
  const int64_t per_cta = static_cast<int64_t>(kCopyThreads) * kCopyUnroll;
  const int64_t slices = (vecs + per_cta - 1) / per_cta;
  if (slices > 65535) return fail(PA_ERR_UNSUPPORTED, "pa_copy_blocks: block too large");
  dim3 grid(static_cast<unsigned>(num_pairs), static_cast<unsigned>(slices));
  PA_CUDA_TRY(launch_pdl(copy_blocks_kernel, grid, dim3(kCopyThreads), 0,
                         static_cast<cudaStream_t>(stream), reinterpret_cast<uint4*>(kv_pool),
                         block_pairs, num_blocks, vecs, err));
  return PA_OK;
}

}  // extern "C"
