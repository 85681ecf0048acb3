// pa_decode: single-token decode attention over the paged KV pool.
//
// What it computes is the quiz page's sketch ("Conceptual: PagedAttention
// block lookup"): for each request b and query head j, keys and values of
// logical position pos come from physical block block_table[b][pos / bs],
// row pos % bs, followed by scaled-dot-product attention.  The sketch notes
// that real kernels fold the gather into the inner tiling loop; here the
// gather *is* the tiling loop: one tile = one physical block of one KV head.
//
// Design for sm_100a (one CTA per (request, KV head, sequence partition)):
//  * a producer warp reads the partition's block-table entries and issues
//    one TMA tile load per physical block and 64-dim slab (box 64 x bs x 2
//    covers the K rows and the V rows of that block and head), into a
//    multi-stage shared-memory ring with 128-byte swizzle, completion on
//    mbarriers;
//  * four consumer warps each own every fourth block and keep their own
//    online-softmax state; the query heads of a GQA group share every loaded
//    tile;
//  * consumer math: by default bf16 mma.sync with
//    fp32 accumulate in a transposed form, S^T = K Q^T then O^T += V^T P^T,
//    so the 16-row side of the MMA is the token / head-dim axis and the
//    group of g <= 8 query heads fills the 8-wide side; P^T is formed from
//    the S^T accumulators in registers with movmatrix.  On request, for
//    groups 1, 2 and 4, fp32 FMA on CUDA cores;
//  * the warps' partial states merge through shared memory; a sequence cut
//    into several partitions writes fp32 partials (O, running max, sum) and
//    a second kernel merges them with the log-sum-exp rule.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "pa_decode_common.cuh"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxGroup = 8;
// The widest column count the default variant gives to the tcgen05 consumer.
constexpr int kTcAutoMaxCols = 32;
constexpr float kRescaleSlack = 8.f;  // log2 units: probabilities stay <= 256
constexpr unsigned kFull = 0xffffffffu;

enum Variant { kCudaCore = 1, kMma = 2, kTc = 3 };

template <int D, int BS>
struct Geo {
  static_assert(D % 64 == 0, "head_dim must be a multiple of 64");
  static_assert(BS % 16 == 0, "block_size must be a multiple of 16");
  static constexpr int kRegions = D / 64;                  // 64-dim slabs of a row
  static constexpr int kRegionBytes = 2 * BS * 128;        // K rows then V rows of one slab
  static constexpr int kStageBytes = kRegions * kRegionBytes;  // one block of one head
  static constexpr int kStages = (kStageBytes <= 8192) ? 8 : 4;
  static constexpr int kStageSmem = kStages * kStageBytes;
  // stage s must always go to warp s % warps (see StreamSmem::kStages)
  static_assert(kStages % kConsumerWarps == 0, "stage s must always go to warp s % warps");
  // epilogue scratch aliased on the stage ring; head rows padded by 4
  // floats so the tensor-core store pattern hits 32 distinct banks
  static constexpr int kOStride = D + 4;
  static constexpr int kEpiO = kConsumerWarps * kMaxGroup * kOStride * 4;
  static constexpr int kEpiBytes = kEpiO + 2 * kConsumerWarps * kMaxGroup * 4;
  static_assert(kEpiBytes <= kStageSmem, "epilogue scratch must fit in the stage ring");
};

// Shared-memory carve-up after the 1024-byte aligned stage ring.
template <int D, int BS, int G>
struct Smem {
  using geo = Geo<D, BS>;
  static constexpr int kBar = geo::kStageSmem;                          // full[S], empty[S]
  static constexpr int kMisc = kBar + 16 * geo::kStages;                // last_round[S], abort
  static constexpr int kPbuf = (kMisc + 4 * geo::kStages + 4 + 15) & ~15;  // CUDA-core p tiles
  static constexpr int kPbufBytes = kConsumerWarps * BS * (G > 0 ? G : 1) * 4;
  static constexpr int kFw = kPbuf + kPbufBytes;                        // merge factors
  static constexpr int kTotal = kFw + (kConsumerWarps * kMaxGroup + 2 * kMaxGroup) * 4;
  static constexpr int kDynamic = kTotal + 1024;                        // alignment slack
};

// --------------------------------------------------------------------------
// Tensor-core consumer: state and per-block step.
//
// The 8*NT columns of S^T are (query token, query head) pairs: column
// c = t * g + j is head j of the KV head's group for query token t, which
// may attend to positions <= lim(c) = len - T + t (T = 1: the whole request).
// Columns past g * T are padding (zero query, never stored).
// --------------------------------------------------------------------------
template <int D, int BS, int NT>
struct MmaConsumer {
  using geo = Geo<D, BS>;
  static constexpr int kDT = D / 16;   // 16-dim tiles of the head dim
  static constexpr int kTT = BS / 16;  // 16-token tiles of a block
  uint32_t qb[NT][kDT][2];             // Q^T as the B operand of S^T = K Q^T
  float o[kDT][NT][4];                 // O^T accumulators
  float m[NT][2], l[NT][2];            // two columns per n-tile of this thread
  int lim[NT][2];                      // last position each of those columns sees

  // qbase: Q row of (token 0, head 0) of this KV head's group; consecutive
  // tokens are q_tok_stride elements apart, heads D apart.
  // col0: the first of the warp's 8 * NT columns (a warp pair splits 16).
  __device__ __forceinline__ void init(const __nv_bfloat16* qbase, int cols, int group, int qtok,
                                       size_t q_tok_stride, int len, int lane, int col0 = 0) {
    const int c = 2 * (lane & 3);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int col = col0 + nt * 8 + (lane >> 2);  // B-operand column of this thread
      const bool real = col < cols;
      const int t = real ? col / group : 0;
      const __nv_bfloat16* qr = qbase + t * q_tok_stride + (col - t * group) * D + c;
#pragma unroll
      for (int ks = 0; ks < kDT; ++ks) {
        qb[nt][ks][0] = real ? *reinterpret_cast<const uint32_t*>(qr + 16 * ks) : 0u;
        qb[nt][ks][1] = real ? *reinterpret_cast<const uint32_t*>(qr + 16 * ks + 8) : 0u;
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int cc = col0 + nt * 8 + c + e;  // accumulator column of this thread
        lim[nt][e] = cc < cols ? len - qtok + cc / group : len - 1;
        m[nt][e] = -INFINITY;
        l[nt][e] = 0.f;
      }
#pragma unroll
      for (int dt = 0; dt < kDT; ++dt) o[dt][nt][0] = o[dt][nt][1] = o[dt][nt][2] = o[dt][nt][3] = 0.f;
    }
  }

  // sb: staged block; pos0: position of its row 0 in the request; the
  // stage goes back to the producer (arrive on empty_bar) once this warp has
  // read it.  With one 16-token tile per block and one 8-column tile, V^T is
  // read into registers right after S^T = K Q^T, so the stage is free for the
  // next TMA load while the softmax and O^T += V^T P^T run (wider tiles keep
  // V^T in shared memory: the extra 32 registers would spill).
  __device__ __forceinline__ void step(uint32_t sb, int pos0, float scale_log2, int lane,
                                       uint32_t empty_bar) {
    const int mat = lane >> 3;
    const int r8 = lane & 7;
    // ---- S^T = K Q^T : rows = tokens of the block, cols = (token, head)
    // two independent accumulation chains over the head dim (even / odd
    // 16-dim steps), summed at the end: half the dependent MMA latency
    float s[kTT][NT][4];
#pragma unroll
    for (int mt = 0; mt < kTT; ++mt) {
      float s2[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        s[mt][nt][0] = s[mt][nt][1] = s[mt][nt][2] = s[mt][nt][3] = 0.f;
        s2[nt][0] = s2[nt][1] = s2[nt][2] = s2[nt][3] = 0.f;
      }
      const int tok = 16 * mt + ((mat & 1) << 3) + r8;
#pragma unroll
      for (int ks = 0; ks < kDT; ++ks) {
        const int chunk = (2 * (ks & 3) + (mat >> 1)) ^ r8;
        const uint32_t addr = sb + (ks >> 2) * geo::kRegionBytes + tok * 128 + chunk * 16;
        uint32_t a0, a1, a2, a3;
        ldsm_x4(addr, a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (ks & 1) mma_bf16_16816(s2[nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
          else mma_bf16_16816(s[mt][nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
        }
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[mt][nt][e] += s2[nt][e];
    }
    constexpr bool kEarly = (kTT == 1 && NT == 1);
    uint32_t vf[kEarly ? kDT : 1][4];
    if constexpr (kEarly) {
      const int row = BS + ((mat >> 1) << 3) + r8;
#pragma unroll
      for (int dt = 0; dt < kDT; ++dt) {
        const int chunk = (2 * (dt & 3) + (mat & 1)) ^ r8;
        ldsm_x4_trans(sb + (dt >> 2) * geo::kRegionBytes + row * 128 + chunk * 16, vf[dt][0], vf[dt][1],
                      vf[dt][2], vf[dt][3]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar);
    }
    // ---- scale, mask positions each column may not see, local max
    float mx[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mx[nt][0] = mx[nt][1] = -INFINITY;
#pragma unroll
    for (int mt = 0; mt < kTT; ++mt) {
      const int p0 = pos0 + 16 * mt + (lane >> 2);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          s[mt][nt][e] = p0 <= lim[nt][e] ? s[mt][nt][e] * scale_log2 : -INFINITY;
          s[mt][nt][e + 2] = p0 + 8 <= lim[nt][e] ? s[mt][nt][e + 2] * scale_log2 : -INFINITY;
          mx[nt][e] = fmaxf(mx[nt][e], fmaxf(s[mt][nt][e], s[mt][nt][e + 2]));
        }
      }
    }
    // The kept max m may lag the true running max by up to kRescaleSlack
    // (log2 units): p = 2^(s - m) then stays <= 2^kRescaleSlack, which bf16 P
    // and the fp32 sums hold with the same relative precision, and the final
    // normalisation divides by a sum taken against the same m.  Each thread
    // checks its own logits against that bound; only when one exceeds it
    // (always on a column's first visible block) does the warp form the exact
    // column max with shuffles and rescale the accumulators.
    bool over = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) over |= mx[nt][e] > m[nt][e] + kRescaleSlack;  // true while m = -inf
    if (__any_sync(kFull, over)) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
#pragma unroll
          for (int off = 4; off < 32; off <<= 1)
            mx[nt][e] = fmaxf(mx[nt][e], __shfl_xor_sync(kFull, mx[nt][e], off));
          const float mnew = fmaxf(m[nt][e], mx[nt][e]);
          const float a = (m[nt][e] == -INFINITY) ? 0.f : exp2f(m[nt][e] - mnew);
#pragma unroll
          for (int dt = 0; dt < kDT; ++dt) {
            o[dt][nt][e] *= a;
            o[dt][nt][e + 2] *= a;
          }
          l[nt][e] *= a;
          m[nt][e] = mnew;
        }
    }
    // ---- P (bf16) -> P^T fragments; O^T += V^T P^T.  A column that has seen
    // no visible position yet keeps m = -inf: its p must be 0, not NaN.
    float msafe[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) msafe[nt][e] = m[nt][e] == -INFINITY ? 0.f : m[nt][e];
#pragma unroll
    for (int mt = 0; mt < kTT; ++mt) {
      uint32_t b0[NT], b1[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t pa = pack_bf16x2(exp2f(s[mt][nt][0] - msafe[nt][0]), exp2f(s[mt][nt][1] - msafe[nt][1]));
        const uint32_t pb = pack_bf16x2(exp2f(s[mt][nt][2] - msafe[nt][0]), exp2f(s[mt][nt][3] - msafe[nt][1]));
        l[nt][0] += bf16lo_to_f32(pa) + bf16lo_to_f32(pb);
        l[nt][1] += bf16hi_to_f32(pa) + bf16hi_to_f32(pb);
        b0[nt] = movmatrix_trans(pa);
        b1[nt] = movmatrix_trans(pb);
      }
      if constexpr (kEarly) {
#pragma unroll
        for (int dt = 0; dt < kDT; ++dt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_bf16_16816(o[dt][nt], vf[dt][0], vf[dt][1], vf[dt][2], vf[dt][3], b0[nt], b1[nt]);
      } else {
        const int row = BS + 16 * mt + ((mat >> 1) << 3) + r8;
#pragma unroll
        for (int dt = 0; dt < kDT; ++dt) {
          const int chunk = (2 * (dt & 3) + (mat & 1)) ^ r8;
          const uint32_t addr = sb + (dt >> 2) * geo::kRegionBytes + row * 128 + chunk * 16;
          uint32_t a0, a1, a2, a3;
          ldsm_x4_trans(addr, a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(o[dt][nt], a0, a1, a2, a3, b0[nt], b1[nt]);
        }
      }
    }
    if constexpr (!kEarly) {
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar);
    }
  }

  // Write this warp's unnormalised O, running max and sum to the epilogue
  // scratch: o_s[column][dim] (row stride kOStride), m_s[column], l_s[column].
  __device__ __forceinline__ void store(float* o_s, float* m_s, float* l_s, int rows, int lane) {
    const int c = 2 * (lane & 3);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float le = l[nt][e];
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) le += __shfl_xor_sync(kFull, le, off);
        l[nt][e] = le;
      }
      const int c0 = nt * 8 + c;
      if (c0 >= rows) continue;  // columns past the call's (even) column count
#pragma unroll
      for (int dt = 0; dt < kDT; ++dt) {
        const int d = 16 * dt + (lane >> 2);
        constexpr int S = geo::kOStride;
        o_s[c0 * S + d] = o[dt][nt][0];
        o_s[(c0 + 1) * S + d] = o[dt][nt][1];
        o_s[c0 * S + d + 8] = o[dt][nt][2];
        o_s[(c0 + 1) * S + d + 8] = o[dt][nt][3];
      }
      if (lane < 4) {
        m_s[c0] = m[nt][0];
        m_s[c0 + 1] = m[nt][1];
        l_s[c0] = l[nt][0];
        l_s[c0 + 1] = l[nt][1];
      }
    }
  }
};

// --------------------------------------------------------------------------
// CUDA-core consumer for narrow groups (G query heads per KV head).
// QK: a quad of 4 lanes per token, 8 tokens per pass, the quad splits the
//     head dim; PV: each lane owns D/32 consecutive output dims.
// --------------------------------------------------------------------------
template <int D, int BS, int G>
struct CudaCoreConsumer {
  using geo = Geo<D, BS>;
  static constexpr int kQD = D / 4;     // dims per lane in QK
  static constexpr int kPass = BS / 8;  // token passes per block
  static constexpr int kOD = D / 32;    // output dims per lane in PV
  float qf[G][kQD];
  float o[G][kOD];
  float m[G], l[G];

  __device__ __forceinline__ void init(const __nv_bfloat16* qrow_base, int lane) {
    const int qq = lane & 3;
#pragma unroll
    for (int j = 0; j < G; ++j) {
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
          const int d0 = x * 64 + (qq + 4 * hi) * 8;
          const uint4 raw = *reinterpret_cast<const uint4*>(qrow_base + j * D + d0);
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            qf[j][(x * 2 + hi) * 8 + 2 * e] = bf16lo_to_f32(w[e]);
            qf[j][(x * 2 + hi) * 8 + 2 * e + 1] = bf16hi_to_f32(w[e]);
          }
        }
#pragma unroll
      for (int e = 0; e < kOD; ++e) o[j][e] = 0.f;
      m[j] = -INFINITY;
      l[j] = 0.f;
    }
  }

  __device__ __forceinline__ void step(uint32_t sb, float* pbuf, int valid, float scale_log2,
                                       int lane) {
    const int qq = lane & 3;
    const int qd = lane >> 2;
    float s[kPass][G];
#pragma unroll
    for (int ps = 0; ps < kPass; ++ps) {
      // quads (2k, 2k+1) take tokens (k, k+4): conflict-free 16-byte reads
      const int tok = ps * 8 + ((qd & 1) << 2) + (qd >> 1);
      float dot[G];
#pragma unroll
      for (int j = 0; j < G; ++j) dot[j] = 0.f;
#pragma unroll
      for (int x = 0; x < D / 64; ++x)
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
          const int chunk = (qq + 4 * hi) ^ (tok & 7);
          uint4 raw;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(raw.x), "=r"(raw.y), "=r"(raw.z), "=r"(raw.w)
                       : "r"(sb + x * geo::kRegionBytes + tok * 128 + chunk * 16));
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float k0 = bf16lo_to_f32(w[e]), k1 = bf16hi_to_f32(w[e]);
#pragma unroll
            for (int j = 0; j < G; ++j) {
              dot[j] = fmaf(k0, qf[j][(x * 2 + hi) * 8 + 2 * e], dot[j]);
              dot[j] = fmaf(k1, qf[j][(x * 2 + hi) * 8 + 2 * e + 1], dot[j]);
            }
          }
        }
#pragma unroll
      for (int j = 0; j < G; ++j) {
        dot[j] += __shfl_xor_sync(kFull, dot[j], 1);
        dot[j] += __shfl_xor_sync(kFull, dot[j], 2);
        s[ps][j] = tok < valid ? dot[j] * scale_log2 : -INFINITY;
      }
    }
    float mx[G];
    bool moved = false;
#pragma unroll
    for (int j = 0; j < G; ++j) {
      mx[j] = s[0][j];
#pragma unroll
      for (int ps = 1; ps < kPass; ++ps) mx[j] = fmaxf(mx[j], s[ps][j]);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) mx[j] = fmaxf(mx[j], __shfl_xor_sync(kFull, mx[j], off));
      mx[j] = fmaxf(mx[j], m[j]);
      moved |= mx[j] > m[j];
    }
    if (__any_sync(kFull, moved)) {  // values are warp-uniform; the vote keeps it explicit
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float a = (m[j] == -INFINITY) ? 0.f : exp2f(m[j] - mx[j]);
#pragma unroll
        for (int e = 0; e < kOD; ++e) o[j][e] *= a;
        l[j] *= a;
        m[j] = mx[j];
      }
    }
#pragma unroll
    for (int ps = 0; ps < kPass; ++ps) {
      const int tok = ps * 8 + ((qd & 1) << 2) + (qd >> 1);
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float p = exp2f(s[ps][j] - m[j]);
        l[j] += p;
        if (qq == 0) pbuf[tok * G + j] = p;
      }
    }
    __syncwarp();
    // ---- PV over the valid rows only (rows past the end may hold NaN)
    const int x = (D == 128) ? (lane >> 4) : 0;
    const int c = (D == 128) ? ((lane & 15) >> 1) : (lane >> 2);
    const int sub = (D == 128) ? (lane & 1) * 8 : (lane & 3) * 4;
#pragma unroll 4
    for (int tok = 0; tok < valid; ++tok) {
      const uint32_t addr =
          sb + x * geo::kRegionBytes + (BS + tok) * 128 + ((c ^ (tok & 7)) << 4) + sub;
      float v[kOD];
      if constexpr (kOD == 4) {
        uint32_t w0, w1;
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(addr));
        v[0] = bf16lo_to_f32(w0);
        v[1] = bf16hi_to_f32(w0);
        v[2] = bf16lo_to_f32(w1);
        v[3] = bf16hi_to_f32(w1);
      } else {
        uint32_t w0;
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w0) : "r"(addr));
        v[0] = bf16lo_to_f32(w0);
        v[1] = bf16hi_to_f32(w0);
      }
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float p = pbuf[tok * G + j];
#pragma unroll
        for (int e = 0; e < kOD; ++e) o[j][e] = fmaf(p, v[e], o[j][e]);
      }
    }
  }

  __device__ __forceinline__ void store(float* o_s, float* m_s, float* l_s, int lane) {
#pragma unroll
    for (int j = 0; j < G; ++j) {
      float lj = l[j];
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) lj += __shfl_xor_sync(kFull, lj, off);
#pragma unroll
      for (int e = 0; e < kOD; ++e) o_s[j * geo::kOStride + lane * kOD + e] = o[j][e];
      if (lane == 0) {
        m_s[j] = m[j];
        l_s[j] = lj;
      }
    }
  }
};

// --------------------------------------------------------------------------
// One consumer warp's work on one staged block (shared by both schedules),
// ending with the stage handed back to the producer.
// --------------------------------------------------------------------------
template <int D, int BS, int VAR, int G, int NT>
__device__ __forceinline__ void consume_block(MmaConsumer<D, BS, NT>& mc,
                                              CudaCoreConsumer<D, BS, (G > 0 ? G : 1)>& cc,
                                              uint32_t sb, float* pbuf, int valid, int pos0,
                                              float scale_log2, int lane, uint32_t empty_bar) {
  using geo = Geo<D, BS>;
  if constexpr (VAR == kMma) {
    if (valid < BS) {
      // rows past the end may hold anything, even NaN: zero their V so that
      // P = 0 there contributes exactly 0
      const int rows = BS - valid;
      for (int t = lane; t < rows * geo::kRegions * 8; t += 32) {
        const int r = valid + t / (geo::kRegions * 8);
        const int x = (t / 8) % geo::kRegions;
        const int ch = t % 8;
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(
                         sb + x * geo::kRegionBytes + (BS + r) * 128 + ch * 16),
                     "r"(0u)
                     : "memory");
      }
      // order these generic writes before the next TMA refill of the stage
      fence_proxy_async_smem();
      __syncwarp();
    }
    mc.step(sb, pos0, scale_log2, lane, empty_bar);
  } else {
    cc.step(sb, pbuf, valid, scale_log2, lane);
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar);
  }
}

// --------------------------------------------------------------------------
// The decode kernel.  grid = (max_parts, num_kv_heads, batch).
// --------------------------------------------------------------------------
template <int D, int BS, int VAR, int G>
__global__ void __launch_bounds__(kThreads, (VAR == kMma || G <= 2) ? 3 : 2)
    paged_decode_kernel(const __grid_constant__ CUtensorMap kv_map, const DecodeArgs a) {
  using geo = Geo<D, BS>;
  using sm = Smem<D, BS, G>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t pad = ((raw_base + 1023u) & ~1023u) - raw_base;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_base + pad;

  const int part = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = a.group;

  pdl_trigger();
  pdl_wait();  // every global access below comes after the previous grid
  const int len = effective_len(__ldg(a.seq_lens + b), BS, a, part == 0 && threadIdx.x == 0);
  const int nblk = (len + BS - 1) / BS;
  const int nparts = (nblk + a.part_blocks - 1) / a.part_blocks;
  const size_t head0 = static_cast<size_t>(b) * a.num_q_heads + static_cast<size_t>(kvh) * g;
  if (len == 0) {  // nothing to attend over: output is zero
    if (part == 0)
      for (int i = threadIdx.x; i < g * D; i += kThreads)
        a.out[head0 * D + i] = __float2bfloat16_rn(0.f);
    return;
  }
  if (part >= nparts) return;
  const int blk0 = part * a.part_blocks;
  const int n = min(a.part_blocks, nblk - blk0);
  const int last_valid = len - (nblk - 1) * BS;  // rows of the request's final block

  const uint32_t bar_full = sbase + sm::kBar;
  const uint32_t bar_empty = bar_full + 8 * geo::kStages;
  int* last_round = reinterpret_cast<int*>(smem + sm::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + sm::kMisc + 4 * geo::kStages);

  if (threadIdx.x == 0) {
    for (int s = 0; s < geo::kStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
      last_round[s] = -1;
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  [[maybe_unused]] MmaConsumer<D, BS, 1> mc;
  [[maybe_unused]] CudaCoreConsumer<D, BS, (G > 0 ? G : 1)> cc;
  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) prefetch_tensor_map(&kv_map);
    const int32_t* trow =
        a.block_tables + static_cast<size_t>(b) * a.max_blocks_per_seq + blk0;
    bool stop = false;
    for (int base = 0; base < n && !stop; base += 32) {
      int phys = 0;
      if (base + lane < n) {
        phys = __ldg(trow + base + lane);
        if (static_cast<unsigned>(phys) >= static_cast<unsigned>(a.num_blocks)) {
          flag_error(a.err, PA_DEVERR_BLOCK_ID);
          phys = a.num_blocks;  // past the tensor map: TMA fills the tile with zeros
        }
      }
      const int cnt = min(32, n - base);
      for (int j = 0; j < cnt; ++j) {
        const int pb = __shfl_sync(kFull, phys, j);
        int failed = 0;
        if (lane == 0) {
          const int i = base + j;
          const int s = i % geo::kStages;
          const int round = i / geo::kStages;
          if (!mbar_wait(bar_empty + 8 * s, (round & 1) ^ 1)) {
            flag_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
            *abort_flag = 1;
            failed = 1;
          } else {
            const uint32_t fb = bar_full + 8 * s;
            mbar_arrive_expect_tx(fb, geo::kStageBytes);
            const uint32_t dst = sbase + s * geo::kStageBytes;
#pragma unroll
            for (int x = 0; x < geo::kRegions; ++x)
              tma_load_3d(dst + x * geo::kRegionBytes, &kv_map, fb, x * 64, kvh * BS, 2 * pb);
            last_round[s] = round;
          }
        }
        if (__shfl_sync(kFull, failed, 0)) {
          stop = true;
          break;
        }
      }
    }
  } else {
    // ----------------------------------------------------------- consumers
    const __nv_bfloat16* qrow = a.q + head0 * D;
    float* pbuf = reinterpret_cast<float*>(smem + sm::kPbuf) + warp * BS * (G > 0 ? G : 1);
    if constexpr (VAR == kMma)
      mc.init(qrow, g, g, 1, static_cast<size_t>(a.num_q_heads) * D, len, lane);
    else
      cc.init(qrow, lane);
    for (int i = warp; i < n; i += kConsumerWarps) {
      if (*abort_flag) break;
      const int s = i % geo::kStages;
      if (!mbar_wait(bar_full + 8 * s, (i / geo::kStages) & 1)) {
        if (lane == 0) {
          flag_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      const uint32_t sb = sbase + s * geo::kStageBytes;
      const int valid = (blk0 + i == nblk - 1) ? last_valid : BS;
      consume_block<D, BS, VAR, G, 1>(mc, cc, sb, pbuf, valid, (blk0 + i) * BS, a.scale_log2, lane,
                                      bar_empty + 8 * s);
    }
  }
  __syncthreads();  // (A) the stage ring is idle; it becomes epilogue scratch
  if (warp < kConsumerWarps && *abort_flag == 0) {
    float* o_s = reinterpret_cast<float*>(smem) + warp * kMaxGroup * geo::kOStride;
    float* m_s = reinterpret_cast<float*>(smem + geo::kEpiO) + warp * kMaxGroup;
    float* l_s = m_s + kConsumerWarps * kMaxGroup;
    if constexpr (VAR == kMma) mc.store(o_s, m_s, l_s, kMaxGroup, lane);
    else cc.store(o_s, m_s, l_s, lane);
  }
  __syncthreads();  // (B) epilogue scratch written

  if (*abort_flag) {
    // unwind: let every issued tile land before the CTA's memory goes away
    if (threadIdx.x == 0)
      for (int s = 0; s < geo::kStages; ++s)
        if (last_round[s] >= 0) mbar_wait_bounded(bar_full + 8 * s, last_round[s] & 1, kWaitLimitNs);
    return;
  }

  // ---------------------------------------------------------- merge warps
  const float* o_all = reinterpret_cast<const float*>(smem);
  const float* m_all = reinterpret_cast<const float*>(smem + geo::kEpiO);
  const float* l_all = m_all + kConsumerWarps * kMaxGroup;
  float* fw = reinterpret_cast<float*>(smem + sm::kFw);  // [warp][head]
  float* mrow = fw + kConsumerWarps * kMaxGroup;         // [head]
  float* lrow = mrow + kMaxGroup;                        // [head]
  const bool single = (nparts == 1);
  if (threadIdx.x < g) {
    const int j = threadIdx.x;
    float mm = -INFINITY;
    for (int w = 0; w < kConsumerWarps; ++w) mm = fmaxf(mm, m_all[w * kMaxGroup + j]);
    float f[kConsumerWarps];
    float ll = 0.f;
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float mw = m_all[w * kMaxGroup + j];
      f[w] = (mw == -INFINITY) ? 0.f : exp2f(mw - mm);
      ll += f[w] * l_all[w * kMaxGroup + j];
    }
    const float inv = single ? 1.f / ll : 1.f;
    for (int w = 0; w < kConsumerWarps; ++w) fw[w * kMaxGroup + j] = f[w] * inv;
    mrow[j] = mm;
    lrow[j] = ll;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < g * D / 2; idx += kThreads) {
    const int j = (2 * idx) / D;
    const int d = (2 * idx) % D;
    float v0 = 0.f, v1 = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float f = fw[w * kMaxGroup + j];
      const float* ow = o_all + (w * kMaxGroup + j) * geo::kOStride + d;
      v0 = fmaf(f, ow[0], v0);
      v1 = fmaf(f, ow[1], v1);
    }
    if (single) {
      *reinterpret_cast<__nv_bfloat162*>(a.out + (head0 + j) * D + d) =
          __floats2bfloat162_rn(v0, v1);
    } else {
      const size_t row = (head0 + j) * a.max_parts + part;
      *reinterpret_cast<float2*>(a.part_o + row * D + d) = make_float2(v0, v1);
      if (d == 0) {
        a.part_m[row] = mrow[j];
        a.part_l[row] = lrow[j];
      }
    }
  }
}

// --------------------------------------------------------------------------
// Balanced ("stream") schedule.
//
// Work units are (request b, KV head h, block k) in that order; there are
// U = Hkv * sum_b ceil(L_b / bs) of them.  A fixed grid of C CTAs (two per
// SM) gives CTA c the contiguous units [floor(U c / C), floor(U (c+1) / C)),
// so every CTA streams the same number of blocks and the whole batch runs in
// one wave with no tail.  A CTA walks its range as segments of constant
// (b, h): a segment that covers all of its (b, h) writes the bf16 output; a
// segment cut by the CTA's range start or end (only the first and the last
// can be) writes an fp32 partial into slot 0 (first) or 1 (last) of the CTA,
// merged afterwards by paged_decode_stream_merge_kernel.
// --------------------------------------------------------------------------
// Build-time tuning of the balanced schedule: CTAs per SM and bytes of TMA
// ring per CTA (the stage count is the ring size over one block's bytes).
#ifndef PA_STREAM_CTAS_PER_SM
#define PA_STREAM_CTAS_PER_SM 2
#endif
#ifndef PA_STREAM_RING_BYTES
#define PA_STREAM_RING_BYTES 65536
#endif
constexpr int kStreamCtasPerSm = PA_STREAM_CTAS_PER_SM;
// Per-segment cost of the balanced kernel (segment epilogue, a pipeline
// drain at the segment's end) in tokens' worth of streaming: the split
// counts this many virtual tokens for every (request, KV head) so the CTAs
// covering many short requests finish with the others.
#ifndef PA_STREAM_SEG_EXTRA_TOKENS
#define PA_STREAM_SEG_EXTRA_TOKENS 64
#endif
constexpr int kStreamSegExtraTokens = PA_STREAM_SEG_EXTRA_TOKENS;
constexpr int kStreamMaxBatch = 4096;  // the prefix table lives in shared memory
// The tcgen05 consumer builds its prefix table in its idle tile ring at the
// start, so it takes larger batches: more than 8 columns above
// kStreamMaxBatch requests run there whatever the head dim.
constexpr int kTcMaxBatch = 32768;

// Consumer groups of the balanced kernel: with up to 8 (token, head) columns
// each consumer warp takes every fourth block alone; with up to 16 (two
// 8-wide MMA tiles) the warps pair up, both warps of a pair take every other
// block and each computes 8 of the columns; with up to 32 all four warps take
// every block, 8 columns each.  No warp carries more than one tile's
// registers, and a group keeps kStages / kGroups stages in flight.
template <int NT>
struct StreamGroups {
  static_assert(NT == 1 || NT == 2 || NT == 4, "1, 2 or 4 tiles of 8 columns");
  static constexpr int kPerGroup = NT;                         // warps sharing a block
  static constexpr int kGroups = kConsumerWarps / kPerGroup;  // block streams per CTA
};

template <int D, int BS, int G, int NT>
struct StreamSmem {
  using geo = Geo<D, BS>;
  static constexpr int kCols = 8;  // epilogue rows per warp: its (token, head) columns
  // Stage s must always be consumed by group s % kGroups: a group then takes
  // a stage's rounds one after the other, so a parity wait (which only tells
  // the current phase from the previous one) never runs two rounds ahead.
  // Hence a whole multiple of the consumer group count.
  static constexpr int kGroups = StreamGroups<NT>::kGroups;
  static constexpr int kRingStages = (PA_STREAM_RING_BYTES / geo::kStageBytes) / kGroups * kGroups;
  static constexpr int kStages = kRingStages > kGroups ? kRingStages : kGroups;
  static_assert(kStages >= kGroups && kStages % kGroups == 0,
                "stages must be a positive multiple of the consumer groups");
  static constexpr int kBar = kStages * geo::kStageBytes;         // full[S], empty[S]
  static constexpr int kMisc = kBar + 16 * kStages;               // last_round[S], abort
  static constexpr int kScan = (kMisc + 4 * kStages + 4 + 15) & ~15;  // scan scratch
  static constexpr int kPbuf = kScan + (kThreads + 4) * 4;       // CUDA-core p tiles
  static constexpr int kPbufBytes = kConsumerWarps * BS * (G > 0 ? G : 1) * 4;
  static constexpr int kEpi = (kPbuf + kPbufBytes + 15) & ~15;   // per-warp O, m, l
  // the epilogue holds only the columns a call uses (group * query tokens,
  // rounded up to a pair), so narrow groups leave room for a deeper ring
  static __host__ __device__ constexpr int epi_rows(int cols) {
    return cols + (cols & 1) < kCols ? cols + (cols & 1) : kCols;
  }
  static __host__ __device__ constexpr int epi_o_bytes(int cols) {
    return kConsumerWarps * epi_rows(cols) * geo::kOStride * 4;
  }
  static __host__ __device__ constexpr int prefix_offset(int cols) {
    return kEpi + epi_o_bytes(cols) + 2 * kConsumerWarps * epi_rows(cols) * 4;  // int32 [batch+1]
  }
  static constexpr int dynamic_bytes(int batch, int cols) {
    return prefix_offset(cols) + 4 * (batch + 1) + 1024;
  }
};

__device__ __forceinline__ void consumer_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

// Where a (request, KV head, block) tile lives.  kPaged: the pool
// [NB][2][Hkv][bs][D] through the block table.  kContiguous: one reserved
// run per request, [B][2][Hkv][max_len][D], block k being rows
// [k bs, (k+1) bs) -- no table; the naive layout paging replaces.
// kPagedPairs: the pool of 16-token blocks with head dim 64, taken two
// table entries per 32-token tile (each block's 2 KiB K and V planes
// would otherwise make stages too small for the per-stage costs).
enum Layout { kPaged = 0, kContiguous = 1, kPagedPairs = 2 };

template <int D, int BS, int VAR, int G, int NT, int LAYOUT = kPaged>
__global__ void __launch_bounds__(kThreads, kStreamCtasPerSm)
    paged_decode_stream_kernel(const __grid_constant__ CUtensorMap kv_map, const DecodeArgs a,
                               int batch) {
  using geo = Geo<D, BS>;
  using sm = StreamSmem<D, BS, G, NT>;
  using grp = StreamGroups<NT>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t pad = ((raw_base + 1023u) & ~1023u) - raw_base;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw_base + pad;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = a.group;
  const int hkv = a.num_kv_heads;
  const int ctas = gridDim.x;
  const uint32_t bar_full = sbase + sm::kBar;
  const uint32_t bar_empty = bar_full + 8 * sm::kStages;
  int* last_round = reinterpret_cast<int*>(smem + sm::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + sm::kMisc + 4 * sm::kStages);
  int* prefix = reinterpret_cast<int*>(smem + sm::prefix_offset(a.cols));

  if (threadIdx.x == 0) {  // shared memory only: may overlap the previous grid
    for (int s = 0; s < sm::kStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, grp::kPerGroup);
      last_round[s] = -1;
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  pdl_wait();  // every global access below comes after the previous grid
  pdl_trigger();  // after the wait: the merge reads inputs before its own
  block_count_prefix<BS, kThreads>(prefix, reinterpret_cast<int*>(smem + sm::kScan), batch, a,
                         blockIdx.x == 0);
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i <= batch; i += kThreads) a.stream_prefix[i] = prefix[i];
  const long long total = static_cast<long long>(hkv) * prefix[batch];
  const long long u_begin = stream_begin(total, blockIdx.x, ctas);
  const long long u_end = stream_begin(total, blockIdx.x + 1, ctas);
  // fused cache write where the consumers cannot patch the staged tile (warp
  // groups share it; a block-pair tile holds two blocks): the producer
  // stores the newest row into its slot just before the TMA load of the
  // (b, h)'s last tile, and CTA 0 stores the rows of requests with no block
  constexpr bool kStoreNew = NT > 1 || LAYOUT == kPagedPairs;
  constexpr int kPoolBs = LAYOUT == kPagedPairs ? BS / 2 : BS;  // block size of the pool
  if constexpr (kStoreNew) store_new_rows_of_empty<D, kPoolBs, kThreads>(a, prefix, batch);
  if (u_begin >= u_end) return;  // uniform: this CTA has no units

  [[maybe_unused]] MmaConsumer<D, BS, 1> mc;  // one 8-column tile per warp
  [[maybe_unused]] CudaCoreConsumer<D, BS, (G > 0 ? G : 1)> cc;
  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) prefetch_tensor_map(&kv_map);
    int b, h, k;
    stream_locate(prefix, batch, hkv, u_begin, b, h, k);
    long long u = u_begin;
    int i = 0;  // running block index in this CTA
    bool stop = false;
    while (u < u_end && !stop) {
      // the (b, h) spans nbu units: nb real tiles, then a.seg_extra virtual
      // ones of the overhead-weighted split (no data, skipped)
      const int nbu = prefix[b + 1] - prefix[b];
      const int nb = nbu - a.seg_extra;
      const int cnt_u = static_cast<int>(min(static_cast<long long>(nbu - k), u_end - u));
      const int cnt = max(0, min(k + cnt_u, nb) - k);  // real tiles of this segment
      constexpr int kPerFetch = LAYOUT == kPagedPairs ? 16 : 32;  // tiles per table fetch
      // physical blocks of request b (the pair layout's last tile may hold one)
      const int nphys = LAYOUT == kPagedPairs
                            ? (effective_len(__ldg(a.seq_lens + b), BS, a, false) + BS / 2 - 1) / (BS / 2)
                            : 0;
      // fused cache write (kStoreNew): lane p fetches part p of the new row now
      long long new_slot = -1;
      uint4 new_part = make_uint4(0u, 0u, 0u, 0u);
      if constexpr (kStoreNew) {
        if (a.new_k != nullptr && cnt > 0 && k + cnt == nb) {
          new_slot = __ldg(a.new_slots + b);
          if (new_slot >= 0 && lane < 2 * (D / 8))
            new_part = __ldg((lane < D / 8 ? a.new_k : a.new_v) + (static_cast<size_t>(b) * hkv + h) * (D / 8) +
                             lane % (D / 8));
        }
      }
      for (int base = 0; base < cnt && !stop; base += kPerFetch) {
        int phys = 0;
        if constexpr (LAYOUT == kPaged || LAYOUT == kPagedPairs) {
          const int32_t* trow = a.block_tables + static_cast<size_t>(b) * a.max_blocks_per_seq;
          // kPaged: entry k + base + lane; pairs: entry 2 (k + base) + lane
          const int e = LAYOUT == kPaged ? k + base + lane : 2 * (k + base) + lane;
          const bool in = LAYOUT == kPaged ? base + lane < cnt : (e < 2 * (k + cnt) && e < nphys);
          phys = -1;
          if (in) {
            phys = __ldg(trow + e);
            if (static_cast<unsigned>(phys) >= static_cast<unsigned>(a.num_blocks)) {
              flag_error(a.err, PA_DEVERR_BLOCK_ID);
              phys = a.num_blocks;  // past the tensor map: TMA fills the tile with zeros
            }
          }
        }
        const int n32 = min(kPerFetch, cnt - base);
        for (int j = 0; j < n32; ++j) {
          const int pb = (LAYOUT == kPaged) ? __shfl_sync(kFull, phys, j)
                                            : (LAYOUT == kPagedPairs ? __shfl_sync(kFull, phys, 2 * j) : 0);
          const int pb1 = (LAYOUT == kPagedPairs) ? __shfl_sync(kFull, phys, 2 * j + 1) : -1;
          if constexpr (kStoreNew) {
            if (new_slot >= 0 && base + j == cnt - 1) {  // the (b, h)'s last tile
              if (lane < 2 * (D / 8)) {
                store_new_part<D, kPoolBs>(a, new_slot, b, h, lane, new_part);
                fence_proxy_async_global();  // before lane 0's TMA load of the tile
              }
              __syncwarp();
            }
          }
          int failed = 0;
          if (lane == 0) {
            const int ii = i + base + j;
            const int s = ii % sm::kStages;
            const int round = ii / sm::kStages;
            if (!mbar_wait(bar_empty + 8 * s, (round & 1) ^ 1)) {
              flag_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
              *abort_flag = 1;
              failed = 1;
            } else {
              const uint32_t fb = bar_full + 8 * s;
              const uint32_t dst = sbase + s * geo::kStageBytes;
              if constexpr (LAYOUT == kPagedPairs) {
                // K then V rows of the tile's first block, the second block's
                // below them (16 rows = 2 KiB each); a missing second block
                // leaves rows 16..31 stale, which the consumer masks
                static_assert(D == 64 && BS == 32, "pairs of 16-token blocks, head dim 64");
                mbar_arrive_expect_tx(fb, pb1 >= 0 ? geo::kStageBytes : geo::kStageBytes / 2);
                tma_load_3d(dst, &kv_map, fb, 0, h * (BS / 2), 2 * pb);
                tma_load_3d(dst + BS * 128, &kv_map, fb, 0, h * (BS / 2), 2 * pb + 1);
                if (pb1 >= 0) {
                  tma_load_3d(dst + (BS / 2) * 128, &kv_map, fb, 0, h * (BS / 2), 2 * pb1);
                  tma_load_3d(dst + (BS + BS / 2) * 128, &kv_map, fb, 0, h * (BS / 2), 2 * pb1 + 1);
                }
              } else {
                mbar_arrive_expect_tx(fb, geo::kStageBytes);
              }
              if constexpr (LAYOUT == kPaged) {
#pragma unroll
                for (int x = 0; x < geo::kRegions; ++x)
                  tma_load_3d(dst + x * geo::kRegionBytes, &kv_map, fb, x * 64, h * BS, 2 * pb);
              } else if constexpr (LAYOUT == kContiguous) {  // rows of block k + base + j of request b
#pragma unroll
                for (int x = 0; x < geo::kRegions; ++x)
                  tma_load_4d(dst + x * geo::kRegionBytes, &kv_map, fb, x * 64, (k + base + j) * BS, h, 2 * b);
              }
              last_round[s] = round;
            }
          }
          if (__shfl_sync(kFull, failed, 0)) stop = true;
          if (stop) break;
        }
      }
      i += cnt;
      u += cnt_u;
      stream_next(prefix, batch, hkv, b, h, k);
    }
  } else {
    // ----------------------------------------------------------- consumers
    float* pbuf = reinterpret_cast<float*>(smem + sm::kPbuf) + warp * BS * (G > 0 ? G : 1);
    const int kC = sm::epi_rows(a.cols);  // epilogue rows per warp
    float* o_all = reinterpret_cast<float*>(smem + sm::kEpi);
    float* m_all = reinterpret_cast<float*>(smem + sm::kEpi + sm::epi_o_bytes(a.cols));
    float* l_all = m_all + kConsumerWarps * kC;
    const int cols = a.cols;
    const size_t q_tok_stride = static_cast<size_t>(a.num_q_heads) * D;
    const int grp_id = warp / grp::kPerGroup;  // block stream of this warp
    const int sub = warp % grp::kPerGroup;     // its 8 columns within the group's
    int b, h, k;
    stream_locate(prefix, batch, hkv, u_begin, b, h, k);
    long long u = u_begin;
    int i = 0;
    int seg = 0;
    while (u < u_end) {
      const int nbu = prefix[b + 1] - prefix[b];  // units: nb real tiles + the split's virtual ones
      const int nb = nbu - a.seg_extra;
      const int cnt_u = static_cast<int>(min(static_cast<long long>(nbu - k), u_end - u));
      const int cnt = max(0, min(k + cnt_u, nb) - k);  // real tiles of this segment
      if (cnt > 0) {  // (uniform over the consumer warps: a virtual-only segment is skipped)
      const bool complete = (k == 0 && cnt == nb);
      // Q row of (token 0, head 0) of this KV head's group; out rows alike
      const size_t qrow0 = static_cast<size_t>(b) * a.qtok * a.num_q_heads + static_cast<size_t>(h) * g;
      const int len = effective_len(__ldg(a.seq_lens + b), BS, a, false);
      const int last_valid = len - (nb - 1) * BS;
      const __nv_bfloat16* qbase = a.q + qrow0 * D;
      if constexpr (VAR == kMma) mc.init(qbase, cols, g, a.qtok, q_tok_stride, len, lane, 8 * sub);
      else cc.init(qbase, lane);
      // fused cache write: the warp that takes this (b, h)'s last block
      // fetches the new K/V row now and patches it into the staged tile
      const int last_ii = i + cnt - 1;
      bool patch = false;
      uint4 new_row = make_uint4(0u, 0u, 0u, 0u);
      // (warp groups and block pairs: the producer stores the row instead)
      if (!kStoreNew && a.new_k != nullptr && k + cnt == nb && last_ii % kConsumerWarps == warp) {
        patch = __ldg(a.new_slots + b) >= 0;
        if (patch && lane < 2 * (D / 8)) {
          const uint4* src = (lane < D / 8 ? a.new_k : a.new_v) +
                             (static_cast<size_t>(b) * hkv + h) * (D / 8) + lane % (D / 8);
          new_row = __ldg(src);
        }
      }
      // this warp's blocks of the segment: running indices i..i+cnt-1 that are
      // congruent to its group number
      for (int ii = i + ((grp_id - i % grp::kGroups + grp::kGroups) % grp::kGroups); ii < i + cnt;
           ii += grp::kGroups) {
        if (*abort_flag) break;
        const int s = ii % sm::kStages;
        if (!mbar_wait(bar_full + 8 * s, (ii / sm::kStages) & 1)) {
          if (lane == 0) {
            flag_error(a.err, PA_DEVERR_WAIT_TIMEOUT);
            *abort_flag = 1;
          }
          break;
        }
        const uint32_t sb = sbase + s * geo::kStageBytes;
        const int blk = k + (ii - i);
        const int valid = (blk == nb - 1) ? last_valid : BS;
        if (patch && ii == last_ii) {
          // row of position len - 1: K row in the K half, V row in the V half
          if (lane < 2 * (D / 8)) {
            const int kv = lane / (D / 8);
            const int chunk = lane % (D / 8);
            const int r = valid - 1;
            const uint32_t addr = sb + (chunk >> 3) * geo::kRegionBytes + (kv * BS + r) * 128 +
                                  (((chunk & 7) ^ (r & 7)) << 4);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(new_row.x),
                         "r"(new_row.y), "r"(new_row.z), "r"(new_row.w)
                         : "memory");
          }
          fence_proxy_async_smem();  // the stage goes back to TMA later
          __syncwarp();
        }
        consume_block<D, BS, VAR, G, 1>(mc, cc, sb, pbuf, valid, blk * BS, a.scale_log2, lane,
                                        bar_empty + 8 * s);
      }
      // ---- segment epilogue: merge the warps' states (column c lives in the
      // scratch rows of the group members that computed it)
      {
        float* o_s = o_all + warp * kC * geo::kOStride;
        if constexpr (VAR == kMma) mc.store(o_s, m_all + warp * kC, l_all + warp * kC, kC, lane);
        else cc.store(o_s, m_all + warp * kC, l_all + warp * kC, lane);
      }
      consumer_bar();
      if (*abort_flag == 0) {
        const int slot = (seg == 0) ? 0 : 1;
        const size_t prow = (static_cast<size_t>(blockIdx.x) * 2 + slot) * cols;
        for (int idx = threadIdx.x; idx < cols * D / 2; idx += kConsumerWarps * 32) {
          const int c = (2 * idx) / D;  // column: token c / g, head c % g
          const int d = (2 * idx) % D;
          const int csub = grp::kPerGroup > 1 ? (c >> 3) : 0;  // which member of a group
          const int cr = c - 8 * csub;                           // row in that member's scratch
          float mm = -INFINITY;
#pragma unroll
          for (int gi = 0; gi < grp::kGroups; ++gi)
            mm = fmaxf(mm, m_all[(gi * grp::kPerGroup + csub) * kC + cr]);
          float ll = 0.f, v0 = 0.f, v1 = 0.f;
#pragma unroll
          for (int gi = 0; gi < grp::kGroups; ++gi) {
            const int w = gi * grp::kPerGroup + csub;
            const float mw = m_all[w * kC + cr];
            const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - mm);
            const float* ow = o_all + (w * kC + cr) * geo::kOStride + d;
            ll = fmaf(f, l_all[w * kC + cr], ll);
            v0 = fmaf(f, ow[0], v0);
            v1 = fmaf(f, ow[1], v1);
          }
          if (complete) {
            // a query token that sees no position (len < T) gets 0
            const float inv = ll > 0.f ? 1.f / ll : 0.f;
            const int t = c / g;
            *reinterpret_cast<__nv_bfloat162*>(a.out + (qrow0 + t * a.num_q_heads + (c - t * g)) * D + d) =
                __floats2bfloat162_rn(v0 * inv, v1 * inv);
          } else {
            *reinterpret_cast<float2*>(a.part_o + (prow + c) * D + d) = make_float2(v0, v1);
            if (d == 0) {
              a.part_m[prow + c] = mm;
              a.part_l[prow + c] = ll;
            }
          }
        }
      }
      consumer_bar();  // the scratch is free for the next segment
      }  // cnt > 0
      i += cnt;
      u += cnt_u;
      ++seg;
      stream_next(prefix, batch, hkv, b, h, k);
    }
  }
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // unwind: let every issued tile land before the CTA's memory goes away
    for (int s = 0; s < sm::kStages; ++s)
      if (last_round[s] >= 0) mbar_wait_bounded(bar_full + 8 * s, last_round[s] & 1, kWaitLimitNs);
  }
}

// Merge for the balanced schedule: one warp per (request, query token, query head).  A
// (b, h) covered by a single CTA was written directly; a (b, h) split across
// CTAs c_first..c_last is merged from their partial slots (slot 0 when the
// (b, h) is the CTA's first segment, else slot 1).  CTAs with an empty range
// (more CTAs than units) wrote nothing and are skipped.  Requests of length
// 0 get zeros here.
//
// What does not depend on the decode kernel's output is done before the
// grid dependency wait, while the decode still streams: up to
// kMergeLocalPrefix requests, the block-count prefix sums (from the lengths,
// with the decode kernel's own arithmetic), and the loads of the new
// tokens' K/V rows of the fused cache write.  Those are inputs no kernel of
// the call writes, and the decode kernel lets this grid launch only after
// its own wait, so whatever wrote them has finished.  After the wait one
// dependent memory round per warp is left: (m, l) and the O row slice of up
// to 8 covering CTAs at once (larger batches first read the decode kernel's
// copy of the prefix sums).
constexpr int kMergeLocalPrefix = 512;

template <int D, int BS>
__global__ void __launch_bounds__(128) paged_decode_stream_merge_kernel(const DecodeArgs a,
                                                                        int batch, int ctas) {
  constexpr int kPer = D / 32;
  constexpr int kUnroll = 8;
  __shared__ int s_prefix[kMergeLocalPrefix + 1];
  __shared__ int s_scan[128 + 1];
  pdl_trigger();
  const bool local = batch <= kMergeLocalPrefix;  // uniform
  if (local) block_count_prefix<BS, 128>(s_prefix, s_scan, batch, a, false);
  const int gw = blockIdx.x * 4 + (threadIdx.x >> 5);  // (request, token, query head)
  const int lane = threadIdx.x & 31;
  const int hkv = a.num_kv_heads;
  const int g = a.group;
  const int per_req = a.qtok * a.num_q_heads;
  const bool live = gw < batch * per_req;
  const int b = live ? gw / per_req : 0;
  const int t = (gw - b * per_req) / a.num_q_heads;
  const int qh = gw - b * per_req - t * a.num_q_heads;  // query head
  const int h = qh / g;                                 // its KV head
  const int j = t * g + (qh - h * g);                   // its column in the (token, head) tile
  const int cols = a.cols;
  // fused cache write: lane p of the KV head's first warp fetches part p of
  // request b's new K/V row now and stores it once the decode kernel has
  // finished reading the pool
  const bool writer = live && a.new_k != nullptr && t == 0 && qh == h * g && lane < 2 * (D / 8);
  long long new_slot = -1;
  uint4 new_part = make_uint4(0u, 0u, 0u, 0u);
  if (writer) {
    new_slot = __ldg(a.new_slots + b);
    new_part = __ldg((lane < D / 8 ? a.new_k : a.new_v) + (static_cast<size_t>(b) * hkv + h) * (D / 8) +
                     lane % (D / 8));
  }
  pdl_wait();
  if (!live) return;
  if (writer) {
    const long long nslots = static_cast<long long>(a.num_blocks) * BS;
    if (new_slot >= nslots) {
      if (lane == 0) flag_error(a.err, PA_DEVERR_SLOT);
    } else if (new_slot >= 0) {
      const int kv = lane / (D / 8);
      const int chunk = lane % (D / 8);
      const long long blk = new_slot / BS;
      const long long off = new_slot - blk * BS;
      a.pool_w[(((blk * 2 + kv) * hkv + h) * BS + off) * (D / 8) + chunk] = new_part;
    }
  }
  const int* prefix = local ? s_prefix : a.stream_prefix;
  const int pb0 = prefix[b], pb1 = prefix[b + 1], pall = prefix[batch];
  const int nbu = pb1 - pb0;                          // work units of each (b, h)
  const int nb = nbu > 0 ? nbu - a.seg_extra : 0;     // of which real blocks
  __nv_bfloat16* o = a.out + static_cast<size_t>(gw) * D + lane * kPer;
  if (nb == 0) {
#pragma unroll
    for (int e = 0; e < kPer; e += 2)
      *reinterpret_cast<__nv_bfloat162*>(o + e) = __floats2bfloat162_rn(0.f, 0.f);
    return;
  }
  const long long total = static_cast<long long>(hkv) * pall;
  const long long us = static_cast<long long>(hkv) * pb0 + static_cast<long long>(h) * nbu;
  const int c0 = stream_cta_of(total, us, ctas);
  const int c1 = stream_cta_of(total, us + nb - 1, ctas);
  if (c0 == c1) return;  // one CTA held the whole (b, h) and wrote the output
  // partial row of CTA c for this (b, h) and column j, or -1 if c holds no units
  auto row_of = [&](int c) -> long long {
    const long long cb = stream_begin(total, c, ctas);
    if (stream_begin(total, c + 1, ctas) <= cb) return -1;
    return (static_cast<long long>(c) * 2 + (cb >= us ? 0 : 1)) * cols + j;
  };
  // every lane loads (m, l) and its slice of the O row of up to 8 covering
  // CTAs at once: a (b, h) split over at most 8 CTAs takes one round of loads
  float mm = -INFINITY, den = 0.f;
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
#pragma unroll 1
  for (int cu = c0; cu <= c1; cu += kUnroll) {
    float w[kUnroll], lw[kUnroll], v[kUnroll][kPer];
#pragma unroll
    for (int q = 0; q < kUnroll; ++q) {
      const int c = cu + q;
      const long long r = c <= c1 ? row_of(c) : -1;
      w[q] = -INFINITY;
      lw[q] = 0.f;
#pragma unroll
      for (int e = 0; e < kPer; ++e) v[q][e] = 0.f;
      if (r >= 0) {
        w[q] = a.part_m[r];
        lw[q] = a.part_l[r];
        const float* op = a.part_o + r * D + lane * kPer;
        if constexpr (kPer == 4) {
          const float4 x = *reinterpret_cast<const float4*>(op);
          v[q][0] = x.x;
          v[q][1] = x.y;
          v[q][2] = x.z;
          v[q][3] = x.w;
        } else {
          const float2 x = *reinterpret_cast<const float2*>(op);
          v[q][0] = x.x;
          v[q][1] = x.y;
        }
      }
    }
    float mnew = mm;
#pragma unroll
    for (int q = 0; q < kUnroll; ++q) mnew = fmaxf(mnew, w[q]);
    if (mnew == -INFINITY) continue;  // no position seen yet by this column
    const float f = (mm == -INFINITY) ? 0.f : exp2f(mm - mnew);
    den *= f;
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] *= f;
#pragma unroll
    for (int q = 0; q < kUnroll; ++q) {
      // a partial whose column saw no position has m = -inf and O = 0
      if (w[q] != -INFINITY) {
        const float wq = exp2f(w[q] - mnew);
        den = fmaf(wq, lw[q], den);
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[e] = fmaf(wq, v[q][e], acc[e]);
      }
    }
    mm = mnew;
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;  // a token that sees nothing gets 0
#pragma unroll
  for (int e = 0; e < kPer; e += 2)
    *reinterpret_cast<__nv_bfloat162*>(o + e) = __floats2bfloat162_rn(acc[e] * inv, acc[e + 1] * inv);
}

// --------------------------------------------------------------------------
// Log-sum-exp merge of the sequence partitions: one warp per (request, head).
//   M = max_p m_p;  out = sum_p 2^(m_p - M) O_p / sum_p 2^(m_p - M) l_p
// (m in the log2 domain; O_p unnormalised w.r.t. its own m_p).  The lanes
// read the partitions' (m, l) in parallel, then the O rows are read eight
// partitions at a time with all loads in flight: two or three dependent
// memory round trips per warp instead of one per partition.
// --------------------------------------------------------------------------
template <int D, int BS>
__global__ void __launch_bounds__(128) paged_decode_reduce_kernel(const DecodeArgs a, int batch) {
  constexpr int kPer = D / 32;
  constexpr int kUnroll = 8;
  pdl_trigger();
  pdl_wait();
  const int gw = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= batch * a.num_q_heads) return;
  const int b = gw / a.num_q_heads;
  const int len = effective_len(__ldg(a.seq_lens + b), BS, a, false);
  const int nblk = (len + BS - 1) / BS;
  const int nparts = (nblk + a.part_blocks - 1) / a.part_blocks;
  if (nparts <= 1) return;  // the main kernel wrote this output directly
  const size_t base = static_cast<size_t>(gw) * a.max_parts;
  const float* pm = a.part_m + base;
  const float* pl = a.part_l + base;
  float mm = -INFINITY;
  for (int p = lane; p < nparts; p += 32) mm = fmaxf(mm, pm[p]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mm = fmaxf(mm, __shfl_xor_sync(kFull, mm, off));
  float den = 0.f;
  for (int p = lane; p < nparts; p += 32) den = fmaf(exp2f(pm[p] - mm), pl[p], den);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(kFull, den, off);
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  const float* po = a.part_o + base * D + lane * kPer;
#pragma unroll 1
  for (int p0 = 0; p0 < nparts; p0 += kUnroll) {
    float v[kUnroll][kPer];
    float w[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int p = p0 + u;
      w[u] = 0.f;
#pragma unroll
      for (int e = 0; e < kPer; ++e) v[u][e] = 0.f;
      if (p < nparts) {
        w[u] = pm[p];
        if constexpr (kPer == 4) {
          const float4 x = *reinterpret_cast<const float4*>(po + static_cast<size_t>(p) * D);
          v[u][0] = x.x;
          v[u][1] = x.y;
          v[u][2] = x.z;
          v[u][3] = x.w;
        } else {
          const float2 x = *reinterpret_cast<const float2*>(po + static_cast<size_t>(p) * D);
          v[u][0] = x.x;
          v[u][1] = x.y;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (p0 + u < nparts) {
        const float wu = exp2f(w[u] - mm);
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[e] = fmaf(wu, v[u][e], acc[e]);
      }
    }
  }
  const float inv = 1.f / den;
  __nv_bfloat16* o = a.out + static_cast<size_t>(gw) * D + lane * kPer;
#pragma unroll
  for (int e = 0; e < kPer; e += 2)
    *reinterpret_cast<__nv_bfloat162*>(o + e) = __floats2bfloat162_rn(acc[e] * inv, acc[e + 1] * inv);
}

// --------------------------------------------------------------------------
// Host side
// --------------------------------------------------------------------------
struct Plan {
  bool stream = false;  // balanced schedule (else the per-partition grid)
  int part_blocks = 1;
  int max_parts = 1;
  int ctas = 0;  // stream: persistent CTAs
  size_t off_m = 0, off_l = 0, off_prefix = 0, bytes = 0;
};

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// partition_tokens: 0 = choose (balanced when the batch fits and has enough
// work), kForceBalanced = balanced, > 0 = per-partition grid with
// partitions of that many tokens.
constexpr int kForceBalanced = -1;
// Tokens per tile of the balanced schedule: one block, or two blocks for
// 16-token blocks of head dim 64 (kPagedPairs).
static int stream_tile(int d, int bs) { return (d == 64 && bs == 16) ? 2 * bs : bs; }

static int make_plan(int batch, int hq, int hkv, int d, int bs, int max_seq_len,
                     int partition_tokens, Plan* plan, int qtok = 1) {
  const int nblk_max = max_seq_len > 0 ? (max_seq_len + bs - 1) / bs : 1;
  const int group = hq / hkv;
  if (qtok > 1 && partition_tokens > 0)
    return fail(PA_ERR_UNSUPPORTED, "multi-token decode runs on the balanced schedule only");
  // more than 8 (token, head) columns: two or four MMA tiles on grouped
  // warps, which only the balanced kernel has
  if (group * qtok > kMaxGroup && partition_tokens > 0)
    return fail(PA_ERR_UNSUPPORTED, "groups above %d run on the balanced schedule only", kMaxGroup);
  if (qtok > 1 || group * qtok > kMaxGroup) partition_tokens = kForceBalanced;
  const int sms = sm_count() > 0 ? sm_count() : 148;
  // the balanced schedule pays when there are at least a few tiles per
  // persistent CTA; tiny batches (launch-bound anyway) take the grid
  const int tile = stream_tile(d, bs);
  const long long units_max =
      static_cast<long long>(batch) * hkv * (max_seq_len > 0 ? (max_seq_len + tile - 1) / tile : 1);
  const bool tc_only = group * qtok > kMaxGroup && batch > kStreamMaxBatch;  // only the tcgen05 consumer fits
  if (tc_only && (batch > kTcMaxBatch || !tc_decode_supported(d, bs, group * qtok)))
    return fail(PA_ERR_UNSUPPORTED, "balanced schedule: batch %d above %d", batch, kTcMaxBatch);
  if (partition_tokens == kForceBalanced && batch > kStreamMaxBatch && !tc_only)
    return fail(PA_ERR_UNSUPPORTED, "balanced schedule: batch %d above %d", batch, kStreamMaxBatch);
  if (partition_tokens == kForceBalanced ||
      (partition_tokens == 0 && batch <= kStreamMaxBatch &&
       units_max >= 2ll * sms * kStreamCtasPerSm)) {
    plan->stream = true;
    plan->ctas = sms * kStreamCtasPerSm;
    plan->part_blocks = 1;  // set per call from max_blocks_per_seq
    plan->max_parts = 1;
    const size_t rows = static_cast<size_t>(plan->ctas) * 2 * group * qtok;
    plan->off_m = align256(rows * d * sizeof(float));
    plan->off_l = plan->off_m + align256(rows * sizeof(float));
    plan->off_prefix = plan->off_l + align256(rows * sizeof(float));
    plan->bytes = plan->off_prefix + align256((static_cast<size_t>(batch) + 1) * sizeof(int));
    return PA_OK;
  }
  int pb;
  if (partition_tokens > 0) {
    if (partition_tokens % bs != 0)
      return fail(PA_ERR_INVALID, "partition_tokens %d not a multiple of block_size %d",
                  partition_tokens, bs);
    pb = partition_tokens / bs;
  } else {
    // batches above the stream limit, or too little work for it: 512-token
    // partitions, halved while the grid would leave the SMs short of work
    pb = 512 / bs;
    const long long pairs = static_cast<long long>(batch) * hkv;
    while (pb > 4 && pairs * ((nblk_max + pb - 1) / pb) < 4ll * sms) pb /= 2;
  }
  pb = pb < 1 ? 1 : pb;
  plan->stream = false;
  plan->part_blocks = pb;
  plan->max_parts = (nblk_max + pb - 1) / pb;
  if (plan->max_parts > 1) {
    const size_t rows = static_cast<size_t>(batch) * hq * plan->max_parts;
    plan->off_m = align256(rows * d * sizeof(float));
    plan->off_l = plan->off_m + align256(rows * sizeof(float));
    plan->bytes = plan->off_l + align256(rows * sizeof(float));
  } else {
    plan->off_m = plan->off_l = plan->bytes = 0;
  }
  return PA_OK;
}

static int check_shape(int batch, int hq, int hkv, int d, int bs, int max_seq_len) {
  if (batch < 0 || hq <= 0 || hkv <= 0 || max_seq_len < 0)
    return fail(PA_ERR_INVALID, "pa_decode: bad sizes (batch %d, heads %d/%d, max_seq_len %d)",
                batch, hq, hkv, max_seq_len);
  if (hq % hkv != 0)
    return fail(PA_ERR_INVALID, "pa_decode: num_q_heads %d not a multiple of num_kv_heads %d", hq, hkv);
  if (hq / hkv > 4 * kMaxGroup)
    return fail(PA_ERR_UNSUPPORTED, "pa_decode: group size %d above %d", hq / hkv, 4 * kMaxGroup);
  if (d != 64 && d != 128) return fail(PA_ERR_UNSUPPORTED, "pa_decode: head_dim %d not in {64,128}", d);
  if (bs != 16 && bs != 32)
    return fail(PA_ERR_UNSUPPORTED, "pa_decode: block_size %d not in {16,32}", bs);
  if (batch > 65535 || hkv > 65535)
    return fail(PA_ERR_UNSUPPORTED, "pa_decode: batch or num_kv_heads above 65535");
  return PA_OK;
}

template <int D, int BS, int VAR, int G>
static int launch_main(const CUtensorMap& map, const DecodeArgs& a, int batch, cudaStream_t st) {
  using sm = Smem<D, BS, G>;
  auto kern = paged_decode_kernel<D, BS, VAR, G>;
  int rc = set_smem_attr(reinterpret_cast<const void*>(kern), sm::kDynamic);
  if (rc != PA_OK) return rc;
  dim3 grid(static_cast<unsigned>(a.max_parts), static_cast<unsigned>(a.num_kv_heads),
            static_cast<unsigned>(batch));
  PA_CUDA_TRY(launch_pdl(kern, grid, dim3(kThreads), sm::kDynamic, st, map, a));
  return PA_OK;
}

template <int D, int BS, int VAR, int G, int NT = 1, int LAYOUT = kPaged>
static int launch_stream(const CUtensorMap& map, const DecodeArgs& a, int batch, int ctas,
                         cudaStream_t st) {
  using sm = StreamSmem<D, BS, G, NT>;
  auto kern = paged_decode_stream_kernel<D, BS, VAR, G, NT, LAYOUT>;
  const int smem = sm::dynamic_bytes(batch, a.cols);
  int rc = set_smem_attr(reinterpret_cast<const void*>(kern), smem);
  if (rc != PA_OK) return rc;
  PA_CUDA_TRY(launch_pdl(kern, dim3(static_cast<unsigned>(ctas)), dim3(kThreads), smem, st, map, a, batch));
  const int warps = batch * a.qtok * a.num_q_heads;
  DecodeArgs m = a;
  if (NT > 1 || LAYOUT == kPagedPairs) {  // the decode kernel stored the new rows already
    m.new_k = m.new_v = nullptr;
    m.new_slots = nullptr;
  }
  PA_CUDA_TRY(launch_pdl(paged_decode_stream_merge_kernel<D, BS>, dim3((warps + 3) / 4), dim3(128), 0, st,
                         m, batch, ctas));
  return PA_OK;
}

int launch_stream_merge(int d, int bs, const DecodeArgs& a, int batch, int ctas, cudaStream_t st) {
  const int warps = batch * a.qtok * a.num_q_heads;
  const dim3 grid((warps + 3) / 4);
  cudaError_t e;
  if (d == 64) e = bs == 16 ? launch_pdl(paged_decode_stream_merge_kernel<64, 16>, grid, dim3(128), 0, st, a, batch, ctas)
                            : launch_pdl(paged_decode_stream_merge_kernel<64, 32>, grid, dim3(128), 0, st, a, batch, ctas);
  else e = bs == 16 ? launch_pdl(paged_decode_stream_merge_kernel<128, 16>, grid, dim3(128), 0, st, a, batch, ctas)
                    : launch_pdl(paged_decode_stream_merge_kernel<128, 32>, grid, dim3(128), 0, st, a, batch, ctas);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "merge launch: %s", cudaGetErrorString(e));
  return PA_OK;
}

template <int D, int BS>
static int dispatch(const CUtensorMap& map, const DecodeArgs& a, int batch, int variant,
                    const Plan& plan, cudaStream_t st) {
  if (plan.stream) {
    if (variant == kMma && a.cols > 16) return launch_stream<D, BS, kMma, 0, 4>(map, a, batch, plan.ctas, st);
    if (variant == kMma && a.cols > 8) return launch_stream<D, BS, kMma, 0, 2>(map, a, batch, plan.ctas, st);
    if (variant == kMma) return launch_stream<D, BS, kMma, 0, 1>(map, a, batch, plan.ctas, st);
    switch (a.group) {
      case 1: return launch_stream<D, BS, kCudaCore, 1>(map, a, batch, plan.ctas, st);
      case 2: return launch_stream<D, BS, kCudaCore, 2>(map, a, batch, plan.ctas, st);
      case 4: return launch_stream<D, BS, kCudaCore, 4>(map, a, batch, plan.ctas, st);
      default:
        return fail(PA_ERR_UNSUPPORTED, "pa_decode: CUDA-core variant has no group size %d", a.group);
    }
  }
  int rc;
  if (variant == kMma) {
    rc = launch_main<D, BS, kMma, 0>(map, a, batch, st);
  } else {
    switch (a.group) {
      case 1: rc = launch_main<D, BS, kCudaCore, 1>(map, a, batch, st); break;
      case 2: rc = launch_main<D, BS, kCudaCore, 2>(map, a, batch, st); break;
      case 4: rc = launch_main<D, BS, kCudaCore, 4>(map, a, batch, st); break;
      default:
        return fail(PA_ERR_UNSUPPORTED, "pa_decode: CUDA-core variant has no group size %d", a.group);
    }
  }
  if (rc != PA_OK) return rc;
  if (a.max_parts > 1) {
    const int warps = batch * a.num_q_heads;
    PA_CUDA_TRY(launch_pdl(paged_decode_reduce_kernel<D, BS>, dim3((warps + 3) / 4), dim3(128), 0, st,
                           a, batch));
  }
  return PA_OK;
}

// Balanced schedule on a pool of 16-token blocks with head dim 64: 32-token
// tiles of two blocks each (kPagedPairs).
static int dispatch_pairs(const CUtensorMap& map, const DecodeArgs& a, int batch, int variant, int ctas,
                          cudaStream_t st) {
  if (variant == kMma && a.cols > 16) return launch_stream<64, 32, kMma, 0, 4, kPagedPairs>(map, a, batch, ctas, st);
  if (variant == kMma && a.cols > 8) return launch_stream<64, 32, kMma, 0, 2, kPagedPairs>(map, a, batch, ctas, st);
  if (variant == kMma) return launch_stream<64, 32, kMma, 0, 1, kPagedPairs>(map, a, batch, ctas, st);
  switch (a.group) {
    case 1: return launch_stream<64, 32, kCudaCore, 1, 1, kPagedPairs>(map, a, batch, ctas, st);
    case 2: return launch_stream<64, 32, kCudaCore, 2, 1, kPagedPairs>(map, a, batch, ctas, st);
    case 4: return launch_stream<64, 32, kCudaCore, 4, 1, kPagedPairs>(map, a, batch, ctas, st);
    default:
      return fail(PA_ERR_UNSUPPORTED, "pa_decode: CUDA-core variant has no group size %d", a.group);
  }
}

static int decode_impl(pa_bf16* out, const pa_bf16* q, const pa_bf16* kv_pool,
                       const int32_t* block_tables, const int32_t* seq_lens, int batch, int hq,
                       int hkv, int d, int bs, int num_blocks, int max_blocks, int max_seq_len,
                       float scale, void* workspace, size_t ws_bytes, int variant,
                       int partition_tokens, void* stream, int qtok = 1,
                       const pa_bf16* new_k = nullptr, const pa_bf16* new_v = nullptr,
                       const int64_t* new_slots = nullptr) {
  int rc = check_shape(batch, hq, hkv, d, bs, max_seq_len);
  if (rc != PA_OK) return rc;
  if (num_blocks <= 0 || max_blocks <= 0)
    return fail(PA_ERR_INVALID, "pa_decode: num_blocks and max_blocks_per_seq must be positive");
  if (partition_tokens < kForceBalanced)
    return fail(PA_ERR_INVALID, "pa_decode: partition_tokens %d below -1", partition_tokens);
  if (!std::isfinite(scale)) return fail(PA_ERR_INVALID, "pa_decode: scale is not finite");
  if (batch == 0) return PA_OK;
  if (!out || !q || !kv_pool || !block_tables || !seq_lens)
    return fail(PA_ERR_INVALID, "pa_decode: NULL pointer");
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(out) || !a16(q) || !a16(kv_pool) || (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return fail(PA_ERR_INVALID, "pa_decode: misaligned pointer");
  rc = check_output_pointer(out, "pa_decode");
  if (rc != PA_OK) return rc;
  bool fused = new_k != nullptr;
  if (fused) {
    if (!new_v || !new_slots) return fail(PA_ERR_INVALID, "pa_decode_append: NULL new_v or slot_mapping");
    if (!a16(new_k) || !a16(new_v) || (reinterpret_cast<uintptr_t>(new_slots) & 7u))
      return fail(PA_ERR_INVALID, "pa_decode_append: misaligned pointer");
    if (qtok != 1) return fail(PA_ERR_UNSUPPORTED, "pa_decode_append: one new token per request");
  }
  const int group = hq / hkv;
  if (qtok < 1) return fail(PA_ERR_INVALID, "num_query_tokens %d below 1", qtok);
  if (group * qtok > 4 * kMaxGroup)
    return fail(PA_ERR_UNSUPPORTED, "group %d x query tokens %d above %d columns", group, qtok,
                4 * kMaxGroup);
  if (qtok > 1 && variant == kCudaCore)
    return fail(PA_ERR_UNSUPPORTED, "multi-token decode has the tensor-core variants only");
  // tensor cores for every group: at scale mma.sync beats the CUDA-core
  // consumer even where the group leaves most of the 8-wide tile empty
  // (g = 1, 2); from 9 to kTcAutoMaxCols columns of head dim 128 the tcgen05
  // consumer takes over (at head dim 64 its 128-token tiles carry half the
  // bytes for the same per-tile work, and mma.sync stays faster)
  if (variant == PA_DECODE_AUTO)
    variant = (group * qtok > kMaxGroup && group * qtok <= kTcAutoMaxCols &&
               (d == 128 || batch > kStreamMaxBatch) && tc_decode_supported(d, bs, group * qtok)) ? kTc : kMma;
  if (group * qtok > kMaxGroup && batch > kStreamMaxBatch && variant != kTc)
    return fail(PA_ERR_UNSUPPORTED, "pa_decode: more than %d columns with batch %d above %d: the tcgen05 variant only",
                kMaxGroup, batch, kStreamMaxBatch);
  if (variant == kCudaCore && group != 1 && group != 2 && group != 4)
    return fail(PA_ERR_UNSUPPORTED, "pa_decode: CUDA-core variant has no group size %d", group);
  if (variant != kCudaCore && variant != kMma && variant != kTc)
    return fail(PA_ERR_INVALID, "pa_decode: unknown variant %d", variant);
  if (variant == kTc) {  // the tcgen05 consumer exists on the balanced schedule only
    if (!tc_decode_supported(d, bs, group * qtok))
      return fail(PA_ERR_UNSUPPORTED, "pa_decode: the tcgen05 variant takes 1..32 columns, not %d", group * qtok);
    if (partition_tokens > 0)
      return fail(PA_ERR_UNSUPPORTED, "pa_decode: the tcgen05 variant runs on the balanced schedule only");
    partition_tokens = kForceBalanced;
  }

  Plan plan;
  rc = make_plan(batch, hq, hkv, d, bs, max_seq_len, partition_tokens, &plan, qtok);
  if (rc != PA_OK) return rc;
  if (plan.bytes > 0) {
    if (workspace == nullptr || ws_bytes < plan.bytes)
      return fail(PA_ERR_INVALID, "pa_decode: workspace of %zu bytes needed, %zu given",
                  plan.bytes, workspace ? ws_bytes : static_cast<size_t>(0));
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
      return fail(PA_ERR_INVALID, "pa_decode: workspace not 256-byte aligned");
  }
  int32_t* err = device_error_word();
  if (err == nullptr) return PA_ERR_CUDA;
  const bool tc = variant == kTc;
  const bool pairs = !tc && plan.stream && stream_tile(d, bs) != bs;

  // TMA view of the pool: x = head dim, y = (kv head, row) of one K or V
  // plane of a block, z = 2*block + (0 keys | 1 values); a box brings both
  // planes, or (block pairs) one plane at a time.
  // (the tcgen05 consumer encodes views of its own)
  alignas(64) CUtensorMap map;
  if (!tc) {
    const uint64_t dims[3] = {static_cast<uint64_t>(d), static_cast<uint64_t>(hkv) * bs,
                              2ull * static_cast<uint64_t>(num_blocks)};
    const uint64_t strides[2] = {static_cast<uint64_t>(d) * 2,
                                 static_cast<uint64_t>(hkv) * bs * d * 2};
    const uint32_t box[3] = {64u, static_cast<uint32_t>(bs), pairs ? 1u : 2u};
    rc = encode_tensor_map(&map, 3, const_cast<pa_bf16*>(kv_pool), dims, strides, box, 1);
    if (rc != PA_OK) return rc;
  }

  DecodeArgs a;
  a.out = reinterpret_cast<__nv_bfloat16*>(out);
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.block_tables = block_tables;
  a.seq_lens = seq_lens;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.part_o = plan.bytes ? reinterpret_cast<float*>(ws) : nullptr;
  a.part_m = plan.bytes ? reinterpret_cast<float*>(ws + plan.off_m) : nullptr;
  a.part_l = plan.bytes ? reinterpret_cast<float*>(ws + plan.off_l) : nullptr;
  a.err = err;
  a.num_q_heads = hq;
  a.num_kv_heads = hkv;
  a.group = group;
  a.num_blocks = num_blocks;
  a.max_blocks_per_seq = max_blocks;
  a.len_cap = pairs ? max_blocks * bs : 0;
  a.part_blocks = plan.stream ? (pairs ? (max_blocks + 1) / 2 : max_blocks) : plan.part_blocks;
  a.max_parts = plan.max_parts;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.stream_prefix = plan.stream ? reinterpret_cast<int*>(ws + plan.off_prefix) : nullptr;
  a.qtok = qtok;
  a.cols = group * qtok;
  a.new_k = nullptr;
  a.new_v = nullptr;
  a.new_slots = nullptr;
  a.pool_w = reinterpret_cast<uint4*>(const_cast<pa_bf16*>(kv_pool));
  // overhead-weighted split of the balanced schedule (virtual units per
  // (request, KV head), in the kernel's tiles)
  a.seg_extra = tc ? tc_decode_segment_extra(bs, a.cols) : (plan.stream ? kStreamSegExtraTokens / stream_tile(d, bs) : 0);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (fused) {
    // mma.sync, one warp per block: the decode kernel patches the staged
    // tile, the merge kernel stores the row; tcgen05, warp groups, block
    // pairs: the decode kernel's producer stores the row before the TMA
    // load of its tile; the per-partition grid runs the cache write first
    if (plan.stream) {
      a.new_k = reinterpret_cast<const uint4*>(new_k);
      a.new_v = reinterpret_cast<const uint4*>(new_v);
      a.new_slots = new_slots;
    } else {  // per-partition grid: the cache write runs first, on its own
      rc = pa_reshape_and_cache(new_k, new_v, const_cast<pa_bf16*>(kv_pool), new_slots, batch,
                                num_blocks, hkv, bs, d, stream);
      if (rc != PA_OK) return rc;
    }
  }

  if (tc) return launch_tc_decode(a, kv_pool, batch, d, bs, num_blocks, sm_count() > 0 ? sm_count() : 148, st);
  if (pairs) return dispatch_pairs(map, a, batch, variant, plan.ctas, st);
  if (d == 64 && bs == 16) return dispatch<64, 16>(map, a, batch, variant, plan, st);
  if (d == 64 && bs == 32) return dispatch<64, 32>(map, a, batch, variant, plan, st);
  if (d == 128 && bs == 16) return dispatch<128, 16>(map, a, batch, variant, plan, st);
  return dispatch<128, 32>(map, a, batch, variant, plan, st);
}

// Decode over a contiguous per-request cache [B][2][Hkv][max_len][D]: the
// balanced kernel with the table gather replaced by direct row addressing
// (16-row tiles), so the two layouts run the same schedule and arithmetic.
constexpr int kContiguousTile = 16;

template <int D>
static int dispatch_contiguous(const CUtensorMap& map, const DecodeArgs& a, int batch, int variant,
                               int ctas, cudaStream_t st) {
  constexpr int T = kContiguousTile;
  if (variant == kMma && a.cols > 16) return launch_stream<D, T, kMma, 0, 4, kContiguous>(map, a, batch, ctas, st);
  if (variant == kMma && a.cols > 8) return launch_stream<D, T, kMma, 0, 2, kContiguous>(map, a, batch, ctas, st);
  if (variant == kMma) return launch_stream<D, T, kMma, 0, 1, kContiguous>(map, a, batch, ctas, st);
  switch (a.group) {
    case 1: return launch_stream<D, T, kCudaCore, 1, 1, kContiguous>(map, a, batch, ctas, st);
    case 2: return launch_stream<D, T, kCudaCore, 2, 1, kContiguous>(map, a, batch, ctas, st);
    case 4: return launch_stream<D, T, kCudaCore, 4, 1, kContiguous>(map, a, batch, ctas, st);
    default:
      return fail(PA_ERR_UNSUPPORTED, "pa_decode_contiguous: CUDA-core variant has no group size %d", a.group);
  }
}

static int contiguous_plan(int batch, int hq, int hkv, int d, int max_len, Plan* plan) {
  int rc = check_shape(batch, hq, hkv, d, kContiguousTile, max_len);
  if (rc != PA_OK) return rc;
  if (max_len <= 0 || max_len % kContiguousTile != 0)
    return fail(PA_ERR_INVALID, "pa_decode_contiguous: max_len %d not a positive multiple of %d", max_len,
                kContiguousTile);
  if (hq / hkv > 4 * kMaxGroup)
    return fail(PA_ERR_UNSUPPORTED, "pa_decode_contiguous: group size %d above %d", hq / hkv, 4 * kMaxGroup);
  if (batch > kStreamMaxBatch)
    return fail(PA_ERR_UNSUPPORTED, "pa_decode_contiguous: batch %d above %d", batch, kStreamMaxBatch);
  // (above 8 query heads per KV head: the mma.sync kernel's grouped warps,
  // as pa_decode on request, so the two layouts still compare kernel for kernel)
  return make_plan(batch, hq, hkv, d, kContiguousTile, max_len, kForceBalanced, plan);
}

static int decode_contiguous_impl(pa_bf16* out, const pa_bf16* q, const pa_bf16* kv_cache,
                                  const int32_t* seq_lens, int batch, int hq, int hkv, int d,
                                  int max_len, float scale, void* workspace, size_t ws_bytes,
                                  int variant, void* stream) {
  Plan plan;
  int rc = contiguous_plan(batch, hq, hkv, d, max_len, &plan);
  if (rc != PA_OK) return rc;
  if (!std::isfinite(scale)) return fail(PA_ERR_INVALID, "pa_decode_contiguous: scale is not finite");
  if (batch == 0) return PA_OK;
  if (!out || !q || !kv_cache || !seq_lens) return fail(PA_ERR_INVALID, "pa_decode_contiguous: NULL pointer");
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(out) || !a16(q) || !a16(kv_cache) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return fail(PA_ERR_INVALID, "pa_decode_contiguous: misaligned pointer");
  rc = check_output_pointer(out, "pa_decode_contiguous");
  if (rc != PA_OK) return rc;
  const int group = hq / hkv;
  if (variant == PA_DECODE_AUTO) variant = kMma;
  if (variant != kCudaCore && variant != kMma)
    return fail(PA_ERR_INVALID, "pa_decode_contiguous: unknown variant %d", variant);
  if (variant == kCudaCore && group != 1 && group != 2 && group != 4)
    return fail(PA_ERR_UNSUPPORTED, "pa_decode_contiguous: CUDA-core variant has no group size %d", group);
  if (workspace == nullptr || ws_bytes < plan.bytes)
    return fail(PA_ERR_INVALID, "pa_decode_contiguous: workspace of %zu bytes needed, %zu given", plan.bytes,
                workspace ? ws_bytes : static_cast<size_t>(0));
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(PA_ERR_INVALID, "pa_decode_contiguous: workspace not 256-byte aligned");
  int32_t* err = device_error_word();
  if (err == nullptr) return PA_ERR_CUDA;

  // TMA view: x = head dim, y = row (position), z = KV head, w = 2*request +
  // (0 keys | 1 values); a box of 2 along w brings a tile's keys and values.
  alignas(64) CUtensorMap map;
  const uint64_t dims[4] = {static_cast<uint64_t>(d), static_cast<uint64_t>(max_len),
                            static_cast<uint64_t>(hkv), 2ull * static_cast<uint64_t>(batch)};
  const uint64_t strides[3] = {static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(max_len) * d * 2,
                               static_cast<uint64_t>(hkv) * max_len * d * 2};
  const uint32_t box[4] = {64u, static_cast<uint32_t>(kContiguousTile), 1u, 2u};
  rc = encode_tensor_map(&map, 4, const_cast<pa_bf16*>(kv_cache), dims, strides, box, 1);
  if (rc != PA_OK) return rc;

  DecodeArgs a{};
  a.out = reinterpret_cast<__nv_bfloat16*>(out);
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.block_tables = nullptr;
  a.seq_lens = seq_lens;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.part_o = reinterpret_cast<float*>(ws);
  a.part_m = reinterpret_cast<float*>(ws + plan.off_m);
  a.part_l = reinterpret_cast<float*>(ws + plan.off_l);
  a.err = err;
  a.num_q_heads = hq;
  a.num_kv_heads = hkv;
  a.group = group;
  a.num_blocks = 0;
  a.max_blocks_per_seq = max_len / kContiguousTile;  // lengths above max_len are flagged and clamped
  a.part_blocks = a.max_blocks_per_seq;
  a.max_parts = 1;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.stream_prefix = reinterpret_cast<int*>(ws + plan.off_prefix);
  a.qtok = 1;
  a.cols = group;
  a.new_k = nullptr;
  a.new_v = nullptr;
  a.new_slots = nullptr;
  a.pool_w = nullptr;
  // the paged kernel's split, so that at equal lengths both layouts cut the
  // same (request, head) pairs and merge them in the same order
  a.seg_extra = kStreamSegExtraTokens / kContiguousTile;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 64) return dispatch_contiguous<64>(map, a, batch, variant, plan.ctas, st);
  return dispatch_contiguous<128>(map, a, batch, variant, plan.ctas, st);
}

}  // namespace pa

extern "C" {

int pa_decode_workspace_size_ex(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                int block_size, int max_seq_len, int partition_tokens,
                                size_t* bytes_out, int* num_partitions_out, int* balanced_out) {
  using namespace pa;
  if (bytes_out == nullptr) return fail(PA_ERR_INVALID, "pa_decode_workspace_size: NULL bytes_out");
  int rc = check_shape(batch, num_q_heads, num_kv_heads, head_dim, block_size, max_seq_len);
  if (rc != PA_OK) return rc;
  if (partition_tokens < kForceBalanced)
    return fail(PA_ERR_INVALID, "partition_tokens %d below -1", partition_tokens);
  Plan plan;
  rc = make_plan(batch, num_q_heads, num_kv_heads, head_dim, block_size, max_seq_len,
                 partition_tokens, &plan);
  if (rc != PA_OK) return rc;
  *bytes_out = plan.bytes;
  if (num_partitions_out) *num_partitions_out = plan.stream ? plan.ctas : plan.max_parts;
  if (balanced_out) *balanced_out = plan.stream ? 1 : 0;
  return PA_OK;
}

int pa_decode_multi_workspace_size(int batch, int num_query_tokens, int num_q_heads,
                                   int num_kv_heads, int head_dim, int block_size,
                                   int max_seq_len, size_t* bytes_out) {
  using namespace pa;
  if (bytes_out == nullptr) return fail(PA_ERR_INVALID, "pa_decode_multi_workspace_size: NULL bytes_out");
  int rc = check_shape(batch, num_q_heads, num_kv_heads, head_dim, block_size, max_seq_len);
  if (rc != PA_OK) return rc;
  if (num_query_tokens < 1) return fail(PA_ERR_INVALID, "num_query_tokens %d below 1", num_query_tokens);
  if (num_q_heads / num_kv_heads * num_query_tokens > 4 * kMaxGroup)
    return fail(PA_ERR_UNSUPPORTED, "group x query tokens above %d columns", 4 * kMaxGroup);
  Plan plan;
  rc = make_plan(batch, num_q_heads, num_kv_heads, head_dim, block_size, max_seq_len, kForceBalanced,
                 &plan, num_query_tokens);
  if (rc != PA_OK) return rc;
  *bytes_out = plan.bytes;
  return PA_OK;
}

int pa_decode_multi(pa_bf16* out, const pa_bf16* q, const pa_bf16* kv_pool,
                    const int32_t* block_tables, const int32_t* seq_lens, int batch,
                    int num_query_tokens, int num_q_heads, int num_kv_heads, int head_dim,
                    int block_size, int num_blocks, int max_blocks_per_seq, int max_seq_len,
                    float scale, void* workspace, size_t workspace_bytes, void* stream) {
  return pa::decode_impl(out, q, kv_pool, block_tables, seq_lens, batch, num_q_heads, num_kv_heads,
                         head_dim, block_size, num_blocks, max_blocks_per_seq, max_seq_len, scale,
                         workspace, workspace_bytes, PA_DECODE_AUTO, pa::kForceBalanced, stream,
                         num_query_tokens);
}

int pa_decode_append(pa_bf16* out, const pa_bf16* q, pa_bf16* kv_pool, const pa_bf16* new_k,
                     const pa_bf16* new_v, const int64_t* slot_mapping, const int32_t* block_tables,
                     const int32_t* seq_lens, int batch, int num_q_heads, int num_kv_heads,
                     int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                     int max_seq_len, float scale, void* workspace, size_t workspace_bytes,
                     void* stream) {
  if (batch > 0 && (new_k == nullptr || new_v == nullptr || slot_mapping == nullptr))
    return pa::fail(PA_ERR_INVALID, "pa_decode_append: NULL new_k, new_v or slot_mapping");
  return pa::decode_impl(out, q, kv_pool, block_tables, seq_lens, batch, num_q_heads, num_kv_heads,
                         head_dim, block_size, num_blocks, max_blocks_per_seq, max_seq_len, scale,
                         workspace, workspace_bytes, PA_DECODE_AUTO, 0, stream, 1, new_k, new_v,
                         slot_mapping);
}

int pa_decode_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                             int block_size, int max_seq_len, size_t* bytes_out,
                             int* num_partitions_out) {
  return pa_decode_workspace_size_ex(batch, num_q_heads, num_kv_heads, head_dim, block_size,
                                     max_seq_len, 0, bytes_out, num_partitions_out, nullptr);
}

int pa_decode(pa_bf16* out, const pa_bf16* q, const pa_bf16* kv_pool, const int32_t* block_tables,
              const int32_t* seq_lens, int batch, int num_q_heads, int num_kv_heads, int head_dim,
              int block_size, int num_blocks, int max_blocks_per_seq, int max_seq_len, float scale,
              void* workspace, size_t workspace_bytes, void* stream) {
  return pa::decode_impl(out, q, kv_pool, block_tables, seq_lens, batch, num_q_heads,
                         num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq,
                         max_seq_len, scale, workspace, workspace_bytes, PA_DECODE_AUTO, 0, stream);
}

int pa_decode_ex(pa_bf16* out, const pa_bf16* q, const pa_bf16* kv_pool,
                 const int32_t* block_tables, const int32_t* seq_lens, int batch, int num_q_heads,
                 int num_kv_heads, int head_dim, int block_size, int num_blocks,
                 int max_blocks_per_seq, int max_seq_len, float scale, void* workspace,
                 size_t workspace_bytes, int variant, int partition_tokens, void* stream) {
  return pa::decode_impl(out, q, kv_pool, block_tables, seq_lens, batch, num_q_heads,
                         num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq,
                         max_seq_len, scale, workspace, workspace_bytes, variant, partition_tokens,
                         stream);
}

int pa_decode_contiguous_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                        int max_len, size_t* bytes_out) {
  using namespace pa;
  if (bytes_out == nullptr) return fail(PA_ERR_INVALID, "pa_decode_contiguous_workspace_size: NULL bytes_out");
  Plan plan;
  int rc = contiguous_plan(batch, num_q_heads, num_kv_heads, head_dim, max_len, &plan);
  if (rc != PA_OK) return rc;
  *bytes_out = plan.bytes;
  return PA_OK;
}

int pa_decode_contiguous(pa_bf16* out, const pa_bf16* q, const pa_bf16* kv_cache, const int32_t* seq_lens,
                         int batch, int num_q_heads, int num_kv_heads, int head_dim, int max_len,
                         float scale, void* workspace, size_t workspace_bytes, int variant, void* stream) {
  return pa::decode_contiguous_impl(out, q, kv_cache, seq_lens, batch, num_q_heads, num_kv_heads, head_dim,
                                    max_len, scale, workspace, workspace_bytes, variant, stream);
}

}  // extern "C"
