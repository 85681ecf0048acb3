// Pieces shared by the decode kernels: the argument block, the device-side
// length checks, the balanced schedule's unit arithmetic and the per-request
// block-count prefix sums.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "pa_device.cuh"

namespace pa {

constexpr unsigned kFullMask = 0xffffffffu;

struct DecodeArgs {
  __nv_bfloat16* out;
  const __nv_bfloat16* q;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  float* part_o;  // [B*Hq][max_parts][D]
  float* part_m;  // [B*Hq][max_parts]
  float* part_l;  // [B*Hq][max_parts]
  int32_t* err;
  int num_q_heads, num_kv_heads, group;
  int num_blocks, max_blocks_per_seq;
  int len_cap;  // > 0: the longest length the table row holds (else max_blocks_per_seq * bs)
  int part_blocks, max_parts;
  float scale_log2;  // scale * log2(e)
  int* stream_prefix;  // balanced schedule: per-request block-count prefix sums [B+1]
  int qtok;            // query tokens per request (1 = single-token decode)
  int cols;            // group * qtok: (token, head) columns per KV head
  // fused cache write (pa_decode_append): request b's newest token, at
  // position seq_lens[b] - 1, has keys/values new_k/new_v [B][Hkv][D] and
  // slot new_slots[b] (< 0: nothing to write); null when not fused
  const uint4* new_k;
  const uint4* new_v;
  const int64_t* new_slots;
  uint4* pool_w;       // the pool, for the fused cache write (merge kernel, or the tcgen05 decode kernel)
  // balanced schedule: virtual work units added to every (request, KV head)
  // that has blocks, so a CTA covering many short ones takes fewer real
  // blocks (per-segment costs); they carry no data and are skipped
  int seg_extra;
};

// Tokens of request b the kernels attend over, after the device-side checks
// (both kernels use this, so they agree on the partition count).
__device__ __forceinline__ int effective_len(int raw, int bs, const DecodeArgs& a, bool report) {
  int len = raw < 0 ? 0 : raw;
  const int cap_table = a.len_cap > 0 ? a.len_cap : a.max_blocks_per_seq * bs;
  const long long cap_grid = static_cast<long long>(a.max_parts) * a.part_blocks * bs;
  if (len > cap_table || len > cap_grid || raw < 0) {
    if (report) flag_error(a.err, PA_DEVERR_SEQ_LEN);
    len = min(len, cap_table);
    len = static_cast<int>(min(static_cast<long long>(len), cap_grid));
  }
  return len;
}

// First unit of the CTA range that contains unit u: the largest c with
// floor(total * c / ctas) <= u.
__device__ __forceinline__ long long stream_begin(long long total, int c, int ctas) {
  return total * c / ctas;
}
__device__ __forceinline__ int stream_cta_of(long long total, long long u, int ctas) {
  return static_cast<int>((static_cast<long long>(ctas) * (u + 1) + total - 1) / total - 1);
}

// (b, h, k) of unit u, from the block-count prefix sums (b with no blocks
// are skipped because the largest b with hkv*prefix[b] <= u is taken).
__device__ __forceinline__ void stream_locate(const int* prefix, int batch, int hkv, long long u,
                                              int& b, int& h, int& k) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (static_cast<long long>(hkv) * prefix[mid] <= u) lo = mid;
    else hi = mid - 1;
  }
  b = lo;
  const int nb = prefix[b + 1] - prefix[b];
  const long long r = u - static_cast<long long>(hkv) * prefix[b];
  h = static_cast<int>(r / nb);
  k = static_cast<int>(r - static_cast<long long>(h) * nb);
}

__device__ __forceinline__ void stream_next(const int* prefix, int batch, int hkv, int& b, int& h,
                                            int& k) {
  k = 0;
  if (++h == hkv) {
    h = 0;
    do {
      ++b;
    } while (b < batch && prefix[b + 1] == prefix[b]);
  }
}

// prefix[b] = sum_{b' < b} units(b') for b in [0, batch], units(b) =
// ceil(L_b / bs) (+ seg_extra when that is > 0); all NT threads of the CTA;
// scan holds NT + 1 ints.
template <int BS, int NT>
__device__ __forceinline__ void block_count_prefix(int* prefix, int* scan, int batch,
                                                   const DecodeArgs& a, bool report) {
  constexpr int kThreads = NT;
  const int t = threadIdx.x;
  const int per = (batch + kThreads - 1) / kThreads;
  const int lo = min(batch, t * per);
  const int hi = min(batch, lo + per);
  int sum = 0;
  for (int i = lo; i < hi; ++i) {
    const int len = effective_len(__ldg(a.seq_lens + i), BS, a, report);
    const int nb = (len + BS - 1) / BS;
    const int units = nb > 0 ? nb + a.seg_extra : 0;
    prefix[i] = units;
    sum += units;
  }
  scan[t] = sum;
  __syncthreads();
  if (t < 32) {  // exclusive scan of the kThreads partial sums by one warp
    constexpr int kPer = (kThreads + 31) / 32;
    int v[kPer];
    int run = 0;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const int idx = t * kPer + e;
      v[e] = idx < kThreads ? scan[idx] : 0;
      run += v[e];
    }
    int incl = run;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(kFullMask, incl, off);
      if (t >= off) incl += y;
    }
    int excl = incl - run;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const int idx = t * kPer + e;
      if (idx < kThreads) scan[idx] = excl;
      excl += v[e];
    }
    if (t == 31) scan[kThreads] = incl;  // grand total
  }
  __syncthreads();
  int run = scan[t];
  for (int i = lo; i < hi; ++i) {
    const int nb = prefix[i];
    prefix[i] = run;
    run += nb;
  }
  if (t == 0) prefix[batch] = scan[kThreads];
  __syncthreads();
}

// Fused cache write: part p of request b's newest key / value row of KV
// head h (p < D/8: 16 bytes of the key, else of the value) into its slot of
// a pool of PBS-token blocks.  A slot past the pool is flagged and skipped.
template <int D, int PBS>
__device__ __forceinline__ void store_new_part(const DecodeArgs& a, long long slot, int b, int h, int p,
                                               uint4 v) {
  if (slot >= static_cast<long long>(a.num_blocks) * PBS) {
    flag_error(a.err, PA_DEVERR_SLOT);
    return;
  }
  const int kv = p / (D / 8), chunk = p % (D / 8);
  const long long blk = slot / PBS, off = slot - blk * PBS;
  a.pool_w[(((blk * 2 + kv) * a.num_kv_heads + h) * PBS + off) * (D / 8) + chunk] = v;
}

// Fused cache write of the requests with no block to attend over (no CTA's
// range holds them): CTA 0 stores their rows; `prefix` is the balanced
// schedule's unit prefix table (equal neighbours: no blocks).
template <int D, int PBS, int NT>
__device__ __forceinline__ void store_new_rows_of_empty(const DecodeArgs& a, const int* prefix, int batch) {
  if (a.new_k == nullptr || blockIdx.x != 0) return;
  const int hkv = a.num_kv_heads;
  for (int b = threadIdx.x; b < batch; b += NT) {
    const long long slot = prefix[b + 1] == prefix[b] ? __ldg(a.new_slots + b) : -1;
    if (slot < 0) continue;
    for (int h = 0; h < hkv; ++h)
      for (int p = 0; p < 2 * (D / 8); ++p) {
        const uint4* src = (p < D / 8 ? a.new_k : a.new_v) + (static_cast<size_t>(b) * hkv + h) * (D / 8) + p % (D / 8);
        store_new_part<D, PBS>(a, slot, b, h, p, __ldg(src));
      }
  }
}

// Host side of the balanced schedule, shared by the decode translation units.
// The merge kernel of the balanced schedule for `ctas` persistent CTAs
// (defined with the mma.sync kernels).
int launch_stream_merge(int d, int bs, const DecodeArgs& a, int batch, int ctas, cudaStream_t st);
// The tcgen05 consumer (pa_decode_tc.cu): 1 <= cols <= 32, head_dim 64/128,
// block_size 16/32; launches the decode kernel and the merge.
int tc_decode_supported(int d, int bs, int cols);
// Virtual units per (request, KV head) the tcgen05 consumer's split adds.
int tc_decode_segment_extra(int bs, int cols);
int launch_tc_decode(const DecodeArgs& a, const void* kv_pool, int batch, int d, int bs, int num_blocks,
                     int ctas, cudaStream_t st);

}  // namespace pa
