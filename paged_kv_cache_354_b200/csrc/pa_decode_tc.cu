// Balanced paged decode with a tcgen05 (tensor memory) consumer, for wide
// column counts: GQA groups of 9..32 query heads per KV head, or several
// query tokens per request (columns = query tokens x group, up to 32).
// Columns come in halves of 16: up to 16 columns one half, 17..32 two on
// every loaded tile.  The MMAs cover all halves at once (N = 16 or 32);
// every tensor-memory access is 16 columns wide and every P tile (one per
// half) 32 bytes wide, the second reached through the descriptor's leading
// byte offset.
//
// What it computes is pa_decode's (quiz page "PagedAttention (vLLM)", code
// sketch "Conceptual: PagedAttention block lookup": keys and values of
// position pos come from block block_table[pos / bs], row pos % bs, then
// scaled-dot-product attention); the work is split exactly like the
// mma.sync balanced kernel -- units (request, KV head, block), an equal
// contiguous share per CTA, cut (request, head) pairs merged by the same
// log-sum-exp merge kernel.  What changes is the tile and who does the math:
//
//  * a tile is 128 consecutive tokens of one (request, KV head): 8 blocks of
//    16 or 4 of 32.  The producer warp loads each block's keys and values
//    with one TMA box each through a 5-D view of the pool that writes every
//    block as [8-row group][64-dim slab][row][64 dims] (128-byte swizzle), so
//    in the tile the 8-token groups of every slab sit at one uniform stride
//    and the tile is a canonical tensor-core operand;
//  * one thread issues S^T = K Q^T (M = 128 tokens, N = the columns held,
//    K = head dim) into tensor memory, then O^T += V^T P^T (M = head dim,
//    N = the columns held, K = the tile's tokens) into a tensor-memory
//    accumulator that stays there for the whole (request, head) segment;
//  * four softmax warps per half each own 32 token rows of S^T (one row per
//    thread, the half's 16 columns in registers): mask, online max with a
//    lagging kept max, probabilities rounded to bf16 into shared memory (the
//    MN-major B operand of the next MMA); at the end of a segment the same
//    warps read the half's O^T (one head-dim row per thread) and write the
//    output or the fp32 partial.
//
// The running max of a column may lag the true one by up to 2^8 (exp2
// domain), as in the mma.sync kernel: only when some logit of the tile
// exceeds kept max + 8 do the softmax warps form exact column maxima
// (shuffles + shared memory) and rescale the sums and, in tensor memory, O.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "pa_decode_common.cuh"
#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_tcgen05.cuh"

namespace pa {
namespace {

// Tokens per tile (build-time tuning).  The MMA is always M = 128 rows of
// S^T; with shorter tiles the rows past the tile read whatever follows in
// shared memory and are masked, and the ring holds more, smaller stages.
#ifndef PA_TC_TILE_TOKENS
#define PA_TC_TILE_TOKENS 128
#endif
// warp 0 producer, warp 1 MMA, then four softmax / epilogue warps per
// 16-column half (one per TMEM lane quadrant)
constexpr int kTcSoftmax = 128;      // softmax / epilogue threads of one half
template <int NH>
__host__ __device__ constexpr int tc_threads() { return 64 + kTcSoftmax * NH; }
constexpr int kTcTileTokens = PA_TC_TILE_TOKENS;
constexpr int kTcRows = 128;         // M of S^T = K Q^T
constexpr int kTcRingBytes = 196608; // K and V tiles in flight
static_assert(kTcTileTokens % 32 == 0 && kTcTileTokens <= kTcRows, "tile of 32, 64, 96 or 128 tokens");
constexpr float kTcSlack = 8.f;      // log2 units: probabilities stay <= 256
constexpr int kTcHalf = 16;          // columns per half: per TMEM access, per P tile, per softmax group
constexpr int kTcMaxCols = 32;       // (token, head) columns per KV head: two halves

template <int D, int BS, int NH>
struct TcGeo {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(BS == 16 || BS == 32, "block_size 16 or 32");
  static_assert(NH == 1 || NH == 2, "one or two 16-column halves");
  static constexpr int kCols = kTcHalf * NH;                 // columns the CTA holds per KV head
  static constexpr int kSlabs = D / 64;
  static constexpr int kTileBlocks = kTcTileTokens / BS;
  static constexpr int kChunk = (32 / kTileBlocks) * kTileBlocks;  // table entries per warp load
  static constexpr int kBlockBytes = BS * D * 2;             // keys (or values) of one block and head
  static constexpr int kTileBytes = kTcTileTokens * D * 2;
  static constexpr int kStages = kTcRingBytes / (2 * kTileBytes);  // 3 (D128) or 6 (D64)
  static constexpr int kGroupStride = kSlabs * 1024;         // between 8-token groups of a tile
  static constexpr int kQSlab = kCols * 128;                 // one 64-dim slab of Q (kCols rows)
  static constexpr int kQBytes = kSlabs * kQSlab;
  static constexpr int kPRow = kTcHalf * 2;                  // one token's probabilities in a half
  static constexpr int kPHalf = kTcRows * kPRow;             // the P tile of one half
  static constexpr int kPBytes = NH * kPHalf;
  static constexpr int kK = 0;
  static constexpr int kV = kStages * kTileBytes;
  static constexpr int kQ = 2 * kStages * kTileBytes;
  static constexpr int kP = kQ + 2 * kQBytes;
  static constexpr int kBar = kP + 2 * kPBytes;
  // tile records: the producer writes tile j's once S^T(j - S) is done, by
  // which time every tile <= j - S - 2 has left the softmax: S + 3 slots do
  static constexpr int kInfoSlots = kStages + 3 <= 8 ? 8 : 16;
  // k_full[S], v_full[S], k_empty[S], v_empty[S], q_full[2], q_empty[2], s_full[2], p_full[2],
  // pv_done[2], drain, info_full[kInfoSlots]
  static constexpr int kNumBars = 4 * kStages + 11 + kInfoSlots;
  static constexpr int kInfo = (kBar + 8 * kNumBars + 15) & ~15;  // TileInfo[kInfoSlots]
  static constexpr int kMisc = kInfo + 32 * kInfoSlots;  // tmem base, abort, last_k[S], last_v[S], last_q[2]
  static constexpr int kRedMax = (kMisc + 8 + 8 * kStages + 8 + 15) & ~15;  // float [4][kCols]
  static constexpr int kRedSum = kRedMax + 4 * kCols * 4;                 // float [4][kCols]
  static constexpr int kTotal = kRedSum + 4 * kCols * 4;
  static constexpr int kDynamic = kTotal + 1024;  // 1024-byte alignment slack
  static_assert(kDynamic <= 232448, "shared memory per CTA");
  static_assert(kQSlab % 1024 == 0 && kPBytes % 1024 == 0 && kTileBytes % 1024 == 0, "swizzle atoms");
  // the last K tile's M = 128 rows may run (kTcRows - kTcTileTokens) rows into the V ring
  static_assert(kV - kTileBytes + kTcRows * D * 2 <= kTotal, "S^T rows past the tile stay in shared memory");
  // S^T double buffer (2 kCols) + O^T (kCols): columns [0, 3 kCols)
  static constexpr uint32_t kTmemCols = 128;
  static_assert(3 * kCols <= static_cast<int>(kTmemCols), "tensor memory columns");
};

// Published by the producer for every tile it loads, read by the MMA and
// softmax warps once the tile's barrier completes.
struct TileInfo {
  int b, h;     // request, KV head
  int pos0;     // position of the tile's first token in the request
  int nblk;     // blocks in the tile
  int len;      // the request's length after the device checks
  int flags;
  int seg;      // segment ordinal within the CTA (counting segments of virtual units only)
  int qseg;     // ordinal of the segments that load a query tile: buffer qseg & 1
};
constexpr int kFirst = 1;     // first tile of a segment
constexpr int kLast = 2;      // last tile of a segment
constexpr int kComplete = 4;  // the segment covers its whole (request, head)
constexpr int kFinal = 8;     // last tile of the CTA

// Named barrier `id` (1 + half) over the 128 softmax threads of one half.
__device__ __forceinline__ bool softmax_any(bool pred, uint32_t id) {
  __syncwarp();  // an aligned barrier: the warp arrives converged
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void softmax_sync(uint32_t id) {
  __syncwarp();
  asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}

// Warp-wide TMEM accesses of 16 columns.  They are .sync.aligned: the warp
// reconverges first (the bounded mbarrier waits before them let lanes leave
// their spin loops at different iterations), and a load returns only after
// its wait.
__device__ __forceinline__ void tmem_load16(uint32_t taddr, uint32_t (&r)[kTcHalf]) {
  __syncwarp();
  tc::tmem_ld_x16(taddr, r);
  tc::wait_ld_x16(r);
}
__device__ __forceinline__ void tmem_store16(uint32_t taddr, const uint32_t (&r)[kTcHalf]) {
  __syncwarp();
  tc::tmem_st_x16(taddr, r);
  tc::wait_st();
}

// Column-wise reduction of 16 columns v[0..16) across the warp's 32 lanes:
// afterwards lane c holds the result for column c mod 16.  The lanes l and
// l + 16 first combine every column, then each step halves the columns a
// lane keeps and hands the other half to its partner.
template <bool kMax>
__device__ __forceinline__ float warp_columns(float (&v)[kTcHalf], int lane) {
#pragma unroll
  for (int c = 0; c < kTcHalf; ++c) {
    const float o = __shfl_xor_sync(kFullMask, v[c], 16);
    v[c] = kMax ? fmaxf(v[c], o) : v[c] + o;
  }
#pragma unroll
  for (int off = kTcHalf / 2; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int c = 0; c < off; ++c) {
      const float give = upper ? v[c] : v[c + off];
      const float keep = upper ? v[c + off] : v[c];
      const float o = __shfl_xor_sync(kFullMask, give, off);
      v[c] = kMax ? fmaxf(keep, o) : keep + o;
    }
  }
  return v[0];
}

template <int D, int BS, int NH>
__global__ void __launch_bounds__(tc_threads<NH>(), 1)
    paged_decode_tc_kernel(const __grid_constant__ CUtensorMap kv_map, const __grid_constant__ CUtensorMap q_map,
                           const DecodeArgs a, int batch) {
  using G = TcGeo<D, BS, NH>;
  constexpr int S = G::kStages;
  constexpr int NC = G::kCols;  // columns held: 16 per half
  constexpr int H16 = kTcHalf;
  constexpr int kThreads = tc_threads<NH>();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t pad = ((raw_base + 1023u) & ~1023u) - raw_base;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_base + pad;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = a.group;
  const int cols = a.cols;
  const int hkv = a.num_kv_heads;
  const int ctas = gridDim.x;

  auto bar = [&](int i) -> uint32_t { return sbase + G::kBar + 8 * i; };
  auto k_full = [&](int s) { return bar(s); };
  auto v_full = [&](int s) { return bar(S + s); };
  // keys and values of a stage are released separately: the keys once
  // S^T is done, the values once P.V is
  auto k_empty = [&](int s) { return bar(2 * S + s); };
  auto v_empty = [&](int s) { return bar(3 * S + s); };
  auto q_full = [&](int j) { return bar(4 * S + j); };
  auto q_empty = [&](int j) { return bar(4 * S + 2 + j); };
  auto s_full = [&](int j) { return bar(4 * S + 4 + j); };
  auto p_full = [&](int j) { return bar(4 * S + 6 + j); };
  // P.V of tile i completes pv_done[i & 1]: a wait for tile i then never
  // meets a barrier two phases behind (P.V of tile i - 2 has finished once
  // the softmax holds tile i's S^T), which a parity wait could not tell apart
  auto pv_done = [&](int j) { return bar(4 * S + 8 + j); };
  const uint32_t drain = bar(4 * S + 10);
  // tile record j is published on info_full[j % slots] (the softmax warps
  // cannot use k_full for that: with the keys released early, k_full of a
  // stage may run two phases ahead of them)
  auto info_full = [&](int j) { return bar(4 * S + 11 + j); };
  TileInfo* info = reinterpret_cast<TileInfo*>(smem + G::kInfo);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + G::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + G::kMisc + 4);
  int* last_k = reinterpret_cast<int*>(smem + G::kMisc + 8);  // last issued round of a stage's keys
  int* last_v = last_k + S;                                     // ... and values
  int* last_q = last_v + S;

  if (threadIdx.x == 0) {  // shared memory only: may overlap the previous grid
    for (int s = 0; s < S; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_empty(s), 1);
      last_k[s] = -1;
      last_v[s] = -1;
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(q_full(j), 1);
      mbar_init(q_empty(j), 1);
      mbar_init(s_full(j), 1);
      mbar_init(p_full(j), kTcSoftmax * NH);
      last_q[j] = -1;
    }
    mbar_init(pv_done(0), 1);
    mbar_init(pv_done(1), 1);
    mbar_init(drain, 1);
    for (int j = 0; j < G::kInfoSlots; ++j) mbar_init(info_full(j), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    __syncwarp();
    tc::tmem_alloc(smem_u32(tmem_slot), G::kTmemCols);
    tc::tmem_relinquish();
  }
  pdl_wait();  // every global access below comes after the previous grid
  pdl_trigger();  // after the wait: the merge reads inputs before its own

  // per-request block-count prefix sums, in the still idle K ring
  int* prefix = reinterpret_cast<int*>(smem + G::kK);
  int* scan = prefix + ((batch + 1 + 3) & ~3);
  block_count_prefix<BS, kThreads>(prefix, scan, batch, a, blockIdx.x == 0);
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i <= batch; i += kThreads) a.stream_prefix[i] = prefix[i];
  const long long total = static_cast<long long>(hkv) * prefix[batch];
  const long long u_begin = stream_begin(total, blockIdx.x, ctas);
  const long long u_end = stream_begin(total, blockIdx.x + 1, ctas);
  int b0 = 0, h0 = 0, k0 = 0;
  if (u_begin < u_end) stream_locate(prefix, batch, hkv, u_begin, b0, h0, k0);
  // the CTA's last unit that holds a real block (units past a (b, h)'s
  // blocks are the split's virtual ones); -1: the range holds none
  long long u_last = -1;
  for (long long v = u_end - 1; v >= u_begin;) {
    int bb, hh, kk;
    stream_locate(prefix, batch, hkv, v, bb, hh, kk);
    const int nreal = prefix[bb + 1] - prefix[bb] - a.seg_extra;
    if (kk < nreal) {
      u_last = v;
      break;
    }
    v -= kk - nreal + 1;  // the last real block of this (b, h)
  }
  // fused cache write for requests with no block to attend over (nothing
  // reads their rows here)
  store_new_rows_of_empty<D, BS, kThreads>(a, prefix, batch);
  fence_proxy_async_smem();  // the ring's generic writes above, TMA writes below
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (u_last >= 0) {
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0) {
        prefetch_tensor_map(&kv_map);
        prefetch_tensor_map(&q_map);
      }
      int b = b0, h = h0, k = k0;
      int len = effective_len(__ldg(a.seq_lens + b), BS, a, false);
      int nb = (len + BS - 1) / BS;  // real blocks; the (b, h) spans nb + seg_extra units
      long long u = u_begin;
      int i = 0, seg = 0, qseg = 0;
      bool stop = false;
      while (u <= u_last && !stop) {
        const int cnt_u = static_cast<int>(min(static_cast<long long>(nb + a.seg_extra - k), u_end - u));
        const int cnt = max(0, min(k + cnt_u, nb) - k);  // real blocks of this segment
        const bool complete = (k == 0 && cnt == nb);
        int failed = 0;
        if (cnt > 0) {
        // this segment's query rows: (token t, head h*g + j) for t < qtok, j < g
        if (lane == 0) {
          const int qb = qseg & 1;
          if (!mbar_wait(q_empty(qb), ((qseg >> 1) & 1) ^ 1)) {
            failed = 1;
          } else {
            mbar_arrive_expect_tx(q_full(qb), G::kSlabs * 128 * cols);
#pragma unroll
            for (int x = 0; x < G::kSlabs; ++x)
              tma_load_4d(sbase + G::kQ + qb * G::kQBytes + x * G::kQSlab, &q_map, q_full(qb), 0, h * g,
                          b * a.qtok, x);
            last_q[qb] = qseg >> 1;
          }
        }
        if (__shfl_sync(kFullMask, failed, 0)) {
          if (lane == 0) {
            flag_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
            *abort_flag = 1;
          }
          break;
        }
        // fused cache write: the CTA that streams this (b, h)'s last block
        // stores the newest token's key and value rows into their slot just
        // before that block's TMA load (only this CTA reads the block's rows
        // of head h); lane p fetches part p now
        const bool writes_new = a.new_k != nullptr && k + cnt == nb;
        const long long new_slot = writes_new ? __ldg(a.new_slots + b) : -1;
        uint4 new_part = make_uint4(0u, 0u, 0u, 0u);
        if (new_slot >= 0 && lane < 2 * (D / 8))
          new_part = __ldg((lane < D / 8 ? a.new_k : a.new_v) + (static_cast<size_t>(b) * hkv + h) * (D / 8) +
                           lane % (D / 8));
        const int32_t* trow = a.block_tables + static_cast<size_t>(b) * a.max_blocks_per_seq + k;
        for (int base = 0; base < cnt && !stop; base += G::kChunk) {
          int phys = 0;
          if (lane < G::kChunk && base + lane < cnt) {
            phys = __ldg(trow + base + lane);
            if (static_cast<unsigned>(phys) >= static_cast<unsigned>(a.num_blocks)) {
              flag_error(a.err, PA_DEVERR_BLOCK_ID);
              phys = a.num_blocks;  // past the tensor map: TMA fills the tile with zeros
            }
          }
          const int n32 = min(G::kChunk, cnt - base);
          for (int t0 = 0; t0 < n32; t0 += G::kTileBlocks) {
            const int nblk = min(G::kTileBlocks, n32 - t0);
            int pb[G::kTileBlocks];
#pragma unroll
            for (int j = 0; j < G::kTileBlocks; ++j) pb[j] = __shfl_sync(kFullMask, phys, (t0 + j) & 31);
            if (new_slot >= 0 && base + t0 + nblk == cnt) {  // the tile with the last block
              if (lane < 2 * (D / 8)) {
                store_new_part<D, BS>(a, new_slot, b, h, lane, new_part);
                fence_proxy_async_global();  // before lane 0's TMA load of the block
              }
              __syncwarp();
            }
            failed = 0;
            if (lane == 0) {
              const int s = i % S;
              const int round = i / S;
              if (!mbar_wait(k_empty(s), (round & 1) ^ 1)) {
                failed = 1;
              } else {
                TileInfo t;
                t.b = b;
                t.h = h;
                t.pos0 = (k + base + t0) * BS;
                t.nblk = nblk;
                t.len = len;
                t.flags = (base + t0 == 0 ? kFirst : 0) | (base + t0 + nblk == cnt ? kLast : 0) |
                          (complete ? kComplete : 0) | (u + base + t0 + nblk - 1 == u_last ? kFinal : 0);
                t.seg = seg;
                t.qseg = qseg;
                info[i % G::kInfoSlots] = t;
                mbar_arrive(info_full(i % G::kInfoSlots));  // release: the record is visible
                const uint32_t kt = sbase + G::kK + s * G::kTileBytes;
                const uint32_t vt = sbase + G::kV + s * G::kTileBytes;
                mbar_arrive_expect_tx(k_full(s), nblk * G::kBlockBytes);
#pragma unroll
                for (int j = 0; j < G::kTileBlocks; ++j)
                  if (j < nblk) tma_load_5d(kt + j * G::kBlockBytes, &kv_map, k_full(s), 0, 0, 0, h * (BS / 8), 2 * pb[j]);
                last_k[s] = round;
                if (!mbar_wait(v_empty(s), (round & 1) ^ 1)) {
                  failed = 1;
                } else {
                  mbar_arrive_expect_tx(v_full(s), nblk * G::kBlockBytes);
#pragma unroll
                  for (int j = 0; j < G::kTileBlocks; ++j)
                    if (j < nblk)
                      tma_load_5d(vt + j * G::kBlockBytes, &kv_map, v_full(s), 0, 0, 0, h * (BS / 8), 2 * pb[j] + 1);
                  last_v[s] = round;
                }
              }
            }
            if (__shfl_sync(kFullMask, failed, 0)) {
              if (lane == 0) {
                flag_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
                *abort_flag = 1;
              }
              stop = true;
              break;
            }
            ++i;
          }
        }
        ++qseg;
        }  // cnt > 0 (a segment of virtual units only is skipped)
        u += cnt_u;
        ++seg;
        k = 0;
        if (++h == hkv) {  // next request with at least one block
          h = 0;
          do {
            ++b;
            if (b >= batch) break;
            len = effective_len(__ldg(a.seq_lens + b), BS, a, false);
            nb = (len + BS - 1) / BS;
          } while (nb == 0);
        }
      }
    } else if (warp == 1) {
      // --------------------------------------------------------- MMA issue
      if (lane == 0) {
        constexpr uint32_t kIdSW = tc::idesc_bf16(128, NC, false, false);
        constexpr uint32_t kIdOW = tc::idesc_bf16(128, NC, true, true);
        // S^T (tile i) = K Q^T over the head dim, 16 dims per instruction;
        // half h2's columns land in TMEM columns [16 h2, 16 h2 + 16) of the
        // tile's buffer
        auto issue_s = [&](int i, const TileInfo& t) {
          const uint32_t kt = sbase + G::kK + (i % S) * G::kTileBytes;
          const uint32_t qt = sbase + G::kQ + (t.qseg & 1) * G::kQBytes;
          const uint32_t d = tmem + (i & 1) * NC;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const int x = ks >> 2, kk = ks & 3;
            const uint64_t ad = tc::smem_desc(kt + x * 1024 + kk * 32, 16, G::kGroupStride, tc::kSwizzle128B);
            // all NC rows of Q in one MMA of N = NC
            const uint64_t bd = tc::smem_desc(qt + x * G::kQSlab + kk * 32, 16, 1024, tc::kSwizzle128B);
            tc::mma_bf16(d, ad, bd, kIdSW, ks > 0 ? 1u : 0u);
          }
        };
        // O^T += V^T P^T over the tile's real tokens, 16 per instruction;
        // head dim 64 makes rows 64..127 repeat rows 0..63 (unused)
        auto issue_pv = [&](int i, const TileInfo& t) {
          const uint32_t vt = sbase + G::kV + (i % S) * G::kTileBytes;
          const uint32_t pt = sbase + G::kP + (i & 1) * G::kPBytes;
          const int steps = t.nblk * (BS / 16);
          for (int kk = 0; kk < steps; ++kk) {
            const uint64_t ad =
                tc::smem_desc(vt + 2 * kk * G::kGroupStride, D == 128 ? 1024 : 0, G::kGroupStride, tc::kSwizzle128B);
            // both halves' P tiles in one MMA of N = NC: the second 16 columns
            // sit one P tile further on (the leading byte offset)
            const uint64_t bd = tc::smem_desc(pt + kk * 16 * G::kPRow, NH == 2 ? G::kPHalf : 8192, 8 * G::kPRow,
                                              tc::kSwizzle32B);
            tc::mma_bf16(tmem + 2 * NC, ad, bd, kIdOW, ((t.flags & kFirst) && kk == 0) ? 0u : 1u);
          }
        };
        auto give_up = [&]() {
          flag_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
          *abort_flag = 1;
        };
        // Issue S^T of the next tile and P.V of the oldest one independently,
        // each as soon as its inputs are ready (tested without blocking), so
        // a tile's P.V -- and with it the stage's release -- never waits for
        // the next tile's keys to arrive.  S^T(j) goes into the buffer of
        // tile j-2, free once P.V(j-2) was issued (after the softmax of tile
        // j-2 arrived): hence j <= pv_next + 1.  Every S^T commit then also
        // covers P.V(j-2), which is what the softmax warps rely on.
        int s_next = 0, pv_next = 0;
        int final_idx = 0x7fffffff;
        int q_commits0 = 0, q_commits1 = 0;  // q_empty commits per query buffer
        TileInfo ti0, ti1;  // tiles pv_next and pv_next + 1 (by parity), kept in registers
        uint64_t idle_since = 0;
        while (pv_next <= final_idx) {
          bool progress = false;
          if (s_next <= final_idx && s_next <= pv_next + 1 &&
              mbar_test_wait(k_full(s_next % S), (s_next / S) & 1)) {
            const TileInfo t = info[s_next % G::kInfoSlots];
            if (!(t.flags & kFirst) || mbar_test_wait(q_full(t.qseg & 1), (t.qseg >> 1) & 1)) {
              tc::fence_after_sync();
              issue_s(s_next, t);
              tc::commit(k_empty(s_next % S));  // the keys go back to the producer
              if (t.flags & kLast) {
                tc::commit(q_empty(t.qseg & 1));
                if (t.qseg & 1) ++q_commits1;
                else ++q_commits0;
              }
              tc::commit(s_full(s_next & 1));
              if (s_next & 1) ti1 = t;
              else ti0 = t;
              if (t.flags & kFinal) final_idx = s_next;
              ++s_next;
              progress = true;
            }
          }
          if (pv_next < s_next && mbar_test_wait(p_full(pv_next & 1), (pv_next >> 1) & 1) &&
              mbar_test_wait(v_full(pv_next % S), (pv_next / S) & 1)) {
            tc::fence_after_sync();
            issue_pv(pv_next, (pv_next & 1) ? ti1 : ti0);
            tc::commit(pv_done(pv_next & 1));
            tc::commit(v_empty(pv_next % S));  // the values go back to the producer
            ++pv_next;
            progress = true;
          }
          if (progress) {
            idle_since = 0;
          } else {
            if (*abort_flag) break;
            const uint64_t now = globaltimer_ns();
            if (idle_since == 0) {
              idle_since = now;
            } else if (now - idle_since > kWaitLimitNs) {
              give_up();
              break;
            }
          }
        }
        // every issued MMA has finished before tensor memory is released,
        // and every commit's arrival has landed before shared memory goes
        // away (nothing else waits for the last releases of each barrier)
        tc::commit(drain);
        mbar_wait_bounded(drain, 0, kWaitLimitNs);
        auto wait_last = [&](uint32_t b, int commits) {
          if (commits > 0) mbar_wait_bounded(b, (commits - 1) & 1, kWaitLimitNs);
        };
        for (int st = 0; st < S; ++st) {
          wait_last(k_empty(st), s_next > st ? (s_next - st + S - 1) / S : 0);
          wait_last(v_empty(st), pv_next > st ? (pv_next - st + S - 1) / S : 0);
        }
        for (int j = 0; j < 2; ++j) wait_last(pv_done(j), pv_next > j ? (pv_next - j + 1) / 2 : 0);
        wait_last(q_empty(0), q_commits0);
        wait_last(q_empty(1), q_commits1);
      }
      __syncwarp();
    } else {
      // ---------------------------------------------- softmax and epilogue
      // four warps per half: half h2 owns columns [16 h2, 16 h2 + 16), its
      // S^T and O^T columns in TMEM and its P tile
      const int h2 = (warp - 2) >> 2;
      const uint32_t bar_id = 1 + h2;   // the half's named barrier
      const int c0 = h2 * H16;          // its first column
      const int qd = warp & 3;          // TMEM lane quadrant of this warp
      const int row = 32 * qd + lane;   // token row of S^T, head-dim row of O^T
      float* red_max = reinterpret_cast<float*>(smem + G::kRedMax);
      float* red_sum = reinterpret_cast<float*>(smem + G::kRedSum);
      const size_t q_tok_heads = static_cast<size_t>(a.num_q_heads);
      float m[H16], l[H16];  // this half's columns
      int i = 0;
      bool bad = false;  // a wait of this thread ran out; checked uniformly at the next tile
      while (true) {
        const int s = i % S;
        if (!bad) bad = !mbar_wait(info_full(i % G::kInfoSlots), (i / G::kInfoSlots) & 1);
        if (!bad) bad = !mbar_wait(s_full(i & 1), (i >> 1) & 1);
        if (softmax_any(bad || *abort_flag != 0, bar_id)) {  // uniform: the half's four warps leave together
          if (bad) {
            flag_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
            *abort_flag = 1;
          }
          break;
        }
        const TileInfo t = info[i % G::kInfoSlots];
        tc::fence_after_sync();
        uint32_t sr[H16];
        tmem_load16(tc::tmem_addr(tmem, 32 * qd, (i & 1) * NC + c0), sr);
        if (t.flags & kFirst) {
#pragma unroll
          for (int c = 0; c < H16; ++c) {
            m[c] = -INFINITY;
            l[c] = 0.f;
          }
        }
        // column c = (query token c / g, head c % g) sees positions <= len - qtok + c / g
        const int pos = t.pos0 + row;
        const bool real = row < t.nblk * BS;
        const int cmin = real ? max(0, g * (pos - (t.len - a.qtok))) : NC;
        float sv[H16];
        bool over = false;
#pragma unroll
        for (int c = 0; c < H16; ++c) {
          const bool vis = c0 + c >= cmin && c0 + c < cols;
          sv[c] = vis ? __uint_as_float(sr[c]) * a.scale_log2 : -INFINITY;
          over |= sv[c] > m[c] + kTcSlack;  // true while m = -inf
        }
        if (softmax_any(over, bar_id)) {
          // exact column maxima over the tile's 128 rows
          float mx[H16];
#pragma unroll
          for (int c = 0; c < H16; ++c) mx[c] = sv[c];
          const float wmax = warp_columns<true>(mx, lane);
          if (lane < H16) red_max[qd * NC + c0 + lane] = wmax;
          softmax_sync(bar_id);
          bool rescale = false;
          float alpha[H16];
#pragma unroll
          for (int c = 0; c < H16; ++c) {
            const float mn = fmaxf(fmaxf(m[c], fmaxf(red_max[c0 + c], red_max[NC + c0 + c])),
                                   fmaxf(red_max[2 * NC + c0 + c], red_max[3 * NC + c0 + c]));
            alpha[c] = (m[c] == -INFINITY) ? 0.f : exp2f(m[c] - mn);
            rescale |= (m[c] != -INFINITY) && (mn != m[c]);
            l[c] *= alpha[c];
            m[c] = mn;
          }
          softmax_sync(bar_id);  // red_max is read; it may be written again
          if (rescale && !(t.flags & kFirst)) {
            // O^T holds the sum through tile i-1: rescale it in place
            if (!bad) bad = !mbar_wait(pv_done((i - 1) & 1), ((i - 1) >> 1) & 1);
            tc::fence_after_sync();
            uint32_t o[H16];
            const uint32_t oaddr = tc::tmem_addr(tmem, 32 * qd, 2 * NC + c0);
            tmem_load16(oaddr, o);
#pragma unroll
            for (int c = 0; c < H16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha[c]);
            tmem_store16(oaddr, o);
          }
        }
        // probabilities (bf16) -> this half's P row of this token (32 bytes);
        // the sums take the rounded values the MMA multiplies
        const uint32_t prow = sbase + G::kP + (i & 1) * G::kPBytes + h2 * G::kPHalf + row * G::kPRow;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = ch * 8 + 2 * e;
            const float m0 = m[c] == -INFINITY ? 0.f : m[c];
            const float m1 = m[c + 1] == -INFINITY ? 0.f : m[c + 1];
            w[e] = pack_bf16x2(exp2f(sv[c] - m0), exp2f(sv[c + 1] - m1));
            l[c] += bf16lo_to_f32(w[e]);
            l[c + 1] += bf16hi_to_f32(w[e]);
          }
          const int sw = ch ^ ((row >> 2) & 1);  // 32-byte swizzle
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(prow + sw * 16), "r"(w[0]), "r"(w[1]),
                       "r"(w[2]), "r"(w[3])
                       : "memory");
        }
        // rows past the request's end inside its last block may hold NaN:
        // zero their values so P = 0 there contributes exactly 0 (the first
        // half's warps; the P.V of every half waits for all of them)
        if (h2 == 0 && real && pos >= t.len) {
          if (!bad) bad = !mbar_wait(v_full(s), (i / S) & 1);
          const uint32_t vrow = sbase + G::kV + s * G::kTileBytes + (row >> 3) * G::kGroupStride + (row & 7) * 128;
#pragma unroll
          for (int x = 0; x < G::kSlabs; ++x)
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
              asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vrow + x * 1024 + ch * 16), "r"(0u)
                           : "memory");
        }
        fence_proxy_async_smem();  // P and the zeroed rows are read by the MMA (async proxy)
        tc::fence_before_sync();
        mbar_arrive(p_full(i & 1));

        if (t.flags & kLast) {
          // ---- segment epilogue: column sums over the 128 rows, then O^T
          float lv[H16];
#pragma unroll
          for (int c = 0; c < H16; ++c) lv[c] = l[c];
          const float wsum = warp_columns<false>(lv, lane);
          if (lane < H16) red_sum[qd * NC + c0 + lane] = wsum;
          softmax_sync(bar_id);
          const int cl = c0 + (lane & (H16 - 1));  // lane c: the half's column c mod 16
          const float lsum = red_sum[cl] + red_sum[NC + cl] + red_sum[2 * NC + cl] + red_sum[3 * NC + cl];
          softmax_sync(bar_id);  // red_sum is read
          if (!bad) bad = !mbar_wait(pv_done(i & 1), (i >> 1) & 1);
          tc::fence_after_sync();
          uint32_t o[H16];
          tmem_load16(tc::tmem_addr(tmem, 32 * qd, 2 * NC + c0), o);
          tc::fence_before_sync();  // the next segment's first MMA overwrites O^T
          const size_t qrow0 = static_cast<size_t>(t.b) * a.qtok * q_tok_heads + static_cast<size_t>(t.h) * g;
          if (t.flags & kComplete) {
            const float inv_l = lsum > 0.f ? 1.f / lsum : 0.f;  // a token that sees nothing gets 0
            int tt = c0 / g, j = c0 - (c0 / g) * g;  // (query token, head) of column c0
#pragma unroll
            for (int c = 0; c < H16; ++c) {
              const float inv = __shfl_sync(kFullMask, inv_l, c);
              if (c0 + c < cols && row < D)
                a.out[(qrow0 + tt * q_tok_heads + j) * D + row] = __float2bfloat16_rn(__uint_as_float(o[c]) * inv);
              if (++j == g) {
                j = 0;
                ++tt;
              }
            }
          } else {
            const size_t prow_part = (static_cast<size_t>(blockIdx.x) * 2 + (t.seg == 0 ? 0 : 1)) * cols;
#pragma unroll
            for (int c = 0; c < H16; ++c)
              if (c0 + c < cols && row < D) a.part_o[(prow_part + c0 + c) * D + row] = __uint_as_float(o[c]);
            if (qd == 0 && lane < H16 && c0 + lane < cols) {
              float mc = m[0];
#pragma unroll
              for (int c = 1; c < H16; ++c) mc = (lane == c) ? m[c] : mc;
              a.part_m[prow_part + c0 + lane] = mc;
              a.part_l[prow_part + c0 + lane] = lsum;
            }
          }
        }
        if (t.flags & kFinal) {
          if (bad) {
            flag_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
            *abort_flag = 1;
          }
          break;
        }
        ++i;
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // unwind: let every issued tile and query load land before the CTA's memory goes away
    for (int s = 0; s < S; ++s) {
      if (last_k[s] >= 0) mbar_wait_bounded(k_full(s), last_k[s] & 1, kWaitLimitNs);
      if (last_v[s] >= 0) mbar_wait_bounded(v_full(s), last_v[s] & 1, kWaitLimitNs);
    }
    for (int j = 0; j < 2; ++j)
      if (last_q[j] >= 0) mbar_wait_bounded(q_full(j), last_q[j] & 1, kWaitLimitNs);
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc(tmem, G::kTmemCols);
  }
}

template <int D, int BS, int NH>
int launch_tc(const CUtensorMap& kv_map, const CUtensorMap& q_map, const DecodeArgs& a, int batch, int ctas,
              cudaStream_t st) {
  using G = TcGeo<D, BS, NH>;
  auto kern = paged_decode_tc_kernel<D, BS, NH>;
  int rc = set_smem_attr(reinterpret_cast<const void*>(kern), G::kDynamic);
  if (rc != PA_OK) return rc;
  PA_CUDA_TRY(launch_pdl(kern, dim3(static_cast<unsigned>(ctas)), dim3(tc_threads<NH>()), G::kDynamic, st, kv_map,
                         q_map, a, batch));
  return PA_OK;
}

// Up to 16 (token, head) columns: one half; 17..32: two halves sharing
// every loaded tile.
template <int D, int BS>
int launch_tc_cols(const CUtensorMap& kv_map, const CUtensorMap& q_map, const DecodeArgs& a, int batch, int ctas,
                   cudaStream_t st) {
  if (a.cols <= kTcHalf) return launch_tc<D, BS, 1>(kv_map, q_map, a, batch, ctas, st);
  return launch_tc<D, BS, 2>(kv_map, q_map, a, batch, ctas, st);
}

}  // namespace

// Per-segment cost of this kernel (a partial last tile, the epilogue) in
// tokens' worth of streaming: the split adds this many virtual tokens to
// every (request, KV head) so CTAs covering many short requests are not the
// last to finish (build-time tuning).
#ifndef PA_TC_SEG_EXTRA_TOKENS
#define PA_TC_SEG_EXTRA_TOKENS 192
#endif
// ... and with two 16-column halves (an epilogue per half, twice the MMA
// columns): group 32 at the llama8b lengths, 192 / 256 / 320 / 384 tokens:
// 122.4 / 120.5 / 120.6 / 121.2 us (decode + merge)
#ifndef PA_TC_SEG_EXTRA_TOKENS_TWO_HALVES
#define PA_TC_SEG_EXTRA_TOKENS_TWO_HALVES 256
#endif

int tc_decode_segment_extra(int bs, int cols) {
  return (cols > kTcHalf ? PA_TC_SEG_EXTRA_TOKENS_TWO_HALVES : PA_TC_SEG_EXTRA_TOKENS) / bs;
}

int tc_decode_supported(int d, int bs, int cols) {
  return (d == 64 || d == 128) && (bs == 16 || bs == 32) && cols >= 1 && cols <= kTcMaxCols;
}

int launch_tc_decode(const DecodeArgs& a, const void* kv_pool, int batch, int d, int bs, int num_blocks, int ctas,
                     cudaStream_t st) {
  if (!tc_decode_supported(d, bs, a.cols))
    return fail(PA_ERR_UNSUPPORTED, "tcgen05 decode: head_dim %d, block_size %d, %d columns", d, bs, a.cols);
  // the prefix table and its scan scratch are built in the (still idle) tile ring
  if (((batch + 1 + 3) & ~3) + tc_threads<2>() + 1 > kTcRingBytes / 4)
    return fail(PA_ERR_UNSUPPORTED, "tcgen05 decode: batch %d too large for the prefix table", batch);
  const int hkv = a.num_kv_heads;
  const int hq = a.num_q_heads;
  // Pool view, 5-D: x = dim within a 64-dim slab, y = row within an 8-row
  // group, z = slab, w = (KV head, 8-row group), v = 2*block + (0 keys | 1
  // values).  A box (64, 8, D/64, bs/8, 1) lands in shared memory as
  // [group][slab][row][64], the layout the tile's MMA descriptors expect.
  alignas(64) CUtensorMap kv_map;
  {
    const uint64_t dims[5] = {64, 8, static_cast<uint64_t>(d / 64), static_cast<uint64_t>(hkv) * bs / 8,
                              2ull * static_cast<uint64_t>(num_blocks)};
    const uint64_t strides[4] = {static_cast<uint64_t>(d) * 2, 128, 16ull * d,
                                 static_cast<uint64_t>(hkv) * bs * d * 2};
    const uint32_t box[5] = {64, 8, static_cast<uint32_t>(d / 64), static_cast<uint32_t>(bs / 8), 1};
    int rc = encode_tensor_map(&kv_map, 5, const_cast<void*>(kv_pool), dims, strides, box, 1);
    if (rc != PA_OK) return rc;
  }
  // Query view, 4-D over q [B][T][Hq][D]: x = dim within a slab, y = query
  // head, z = (request, token), w = slab.  A box (64, g, T, 1) brings one
  // slab of a (request, KV head)'s columns c = t * g + j, row c of the tile.
  alignas(64) CUtensorMap q_map;
  {
    const uint64_t dims[4] = {64, static_cast<uint64_t>(hq), static_cast<uint64_t>(batch) * a.qtok,
                              static_cast<uint64_t>(d / 64)};
    const uint64_t strides[3] = {static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(hq) * d * 2, 128};
    const uint32_t box[4] = {64, static_cast<uint32_t>(a.group), static_cast<uint32_t>(a.qtok), 1};
    int rc = encode_tensor_map(&q_map, 4, const_cast<__nv_bfloat16*>(a.q), dims, strides, box, 1);
    if (rc != PA_OK) return rc;
  }
  int rc;
  if (d == 128) rc = bs == 16 ? launch_tc_cols<128, 16>(kv_map, q_map, a, batch, ctas, st)
                              : launch_tc_cols<128, 32>(kv_map, q_map, a, batch, ctas, st);
  else rc = bs == 16 ? launch_tc_cols<64, 16>(kv_map, q_map, a, batch, ctas, st)
                     : launch_tc_cols<64, 32>(kv_map, q_map, a, batch, ctas, st);
  if (rc != PA_OK) return rc;
  DecodeArgs m = a;
  m.new_k = m.new_v = nullptr;  // the decode kernel stored the new rows already
  m.new_slots = nullptr;
  return launch_stream_merge(d, bs, m, batch, ctas, st);
}

}  // namespace pa
