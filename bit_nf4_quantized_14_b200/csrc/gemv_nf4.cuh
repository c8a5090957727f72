// Small-token QLoRA forward (decode shapes, T <= 64): Y = X W_hat^T + sU B^T, and the adapter projection
// sU = s X A^T that feeds it.
//
// For a handful of tokens every weight element is used T times, so the layer is bound by streaming the
// NF4 codes from HBM (0.52 B per weight); the work per byte is far too small for a 128 x 256 tensor-core
// tile. The pages ask for the weight to be "dequantized to bfloat16 on the fly, block by block, and
// multiplied in 16-bit precision" (PEFT page, zerotofrontier.app/sft/peft, "Paged optimizers, and QLoRA
// end to end"; dequantization fused into the matrix multiply: same page, "The real way"). Here the
// dequantization never materialises a weight tile:
//   * TMA streams tiles of 112 weight rows x 256 contraction elements (128 code bytes per row, 128-byte
//     swizzle) and the matching 64-wide boxes of X through a ring of stages;
//   * each consumer warp owns 16 rows and builds the A fragments of mma.sync m16n8k16 (bf16, fp32
//     accumulate) directly from code bytes: one byte permute and one shared-memory lookup per byte in a
//     256-entry table of bf16 level pairs, replicated per lane so lookups never conflict; two CTAs share
//     an SM (for T <= 32) so that two stage pipelines run out of step;
//   * the block constant c1_hat = fma(decode(e4m3), s2, mu) multiplies the fp32 block accumulator once per
//     64-element block: y += c1_hat * sum_k bf16(level[code_k]) * x_k.
// The one difference from the fused GEMM's W_hat = bf16(level * c1_hat) is where the bf16 rounding falls
// (on the level instead of the product): both round each weight once, to a relative 2^-9.
//
// Work is split stream-K: the tiles x stages sequence is cut into gridDim.x contiguous ranges. A tile
// covered by one CTA is finished in registers; otherwise each warp writes its fp32 partial and, per 16
// rows, the last warp to arrive (atomic ticket) adds the partials in CTA order (deterministic), applies
// the LoRA term and writes Y. The adapter projection sU runs first in single-warp CTAs beside it.
// Every mbarrier wait is bounded; on expiry the status word records a timeout and the CTA unwinds.
#pragma once

#include <cuda.h>

#include "codec.cuh"
#include "common.cuh"

namespace qnf4 {

constexpr int kGvWarps = 7;                       // consumer warps, 16 rows each (8 warps per CTA)
constexpr int kGvRows = 16 * kGvWarps;            // rows per tile
constexpr int kGvThreads = 32 * (kGvWarps + 1);   // + one producer warp
constexpr int kGvRowBytes = 128;                  // code bytes per row per stage (256 elements)
constexpr int kGvStageK = 256;
constexpr int kGvTileBytes = kGvRows * kGvRowBytes;
constexpr int kGvLutBytes = 256 * 128;            // entry e: 32 lanes x 4 B at e * 128
constexpr int kGvMaxTokens = 64;

template <int NT>
struct GvCfg {
  static constexpr int TP = 8 * NT;                          // tokens padded to the MMA's n8 tiles
  static constexpr int X_BOX = TP * 128;                     // one 64-wide box of X
  static constexpr int STAGE_BYTES = kGvTileBytes + 4 * X_BOX;
  static constexpr int CTAS_PER_SM = NT <= 4 ? 2 : 1;          // two independent pipelines per SM
  static constexpr int AVAIL = (227 / CTAS_PER_SM) * 1024 - 1024 - 256 - kGvLutBytes;
  static constexpr int STAGES = (AVAIL / STAGE_BYTES) < 8 ? (AVAIL / STAGE_BYTES) : 8;
  static constexpr int SMEM_BYTES = 1024 + kGvLutBytes + STAGES * STAGE_BYTES + 256;
  static constexpr int SLOT = kGvWarps * 32 * NT * 4;          // floats of one CTA's partial tile
  static_assert(STAGES >= 2, "ring depth");
  static_assert(STAGE_BYTES % 1024 == 0 && X_BOX % 1024 == 0, "swizzle atoms stay 1 KB aligned");
};

struct GvParams {
  int T, rows, K;            // tokens, output rows (N), contraction
  int spt, tiles;            // stages per tile, tiles of kGvRows rows
  int64_t total;             // tiles * spt
  int maxseg;                // partial slots per CTA
  int kbw;                   // 64-element blocks per weight row (K / 64)
  const uint8_t* e4m3;
  const float* s2;
  const float* mu;
  const __nv_bfloat16* sU;   // LoRA epilogue operands: sU (T x r), B (rows x r)
  const __nv_bfloat16* Bw;
  int r;
  __nv_bfloat16* out;        // Y[t * ldo + row]
  int64_t ldo;
  float* part;               // [gridDim.x * maxseg][kGvWarps][32 lanes][NT * 4]
  unsigned* ticket;          // one per (tile, consumer warp), zero on entry; left at zero
};

__device__ __forceinline__ int64_t gv_start(int c, int64_t total, int G) {
  return static_cast<int64_t>(c) * total / G;
}
// The CTA whose stage range holds flat stage f.
__device__ __forceinline__ int gv_owner(int64_t f, int64_t total, int G) {
  int c = static_cast<int>((f * G) / total);
  while (c + 1 < G && gv_start(c + 1, total, G) <= f) ++c;
  while (c > 0 && gv_start(c, total, G) > f) --c;
  return c;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
// A fragment register of one code byte: the pair (level[hi nibble], level[lo nibble]) as bf16, from the
// lane's own copy of the table (entry byte at byte * 128 + lane * 4; lut_lane includes lane * 4).
template <int kByte>
__device__ __forceinline__ uint32_t lut_pair(uint32_t lut_lane, uint32_t w) {
  return lds32(lut_lane + (__byte_perm(w, 0u, 0x4440u | kByte) << 7));
}
__device__ __forceinline__ uint32_t ldg32_or0(const __nv_bfloat16* p, bool ok) {
  return ok ? __ldg(reinterpret_cast<const unsigned int*>(p)) : 0u;
}

// Block constants: lane L of a warp owns row (L & 15) of the warp's 16 rows and blocks 2 (L >> 4) and
// 2 (L >> 4) + 1 of the stage's 4; the raw bytes are fetched a stage ahead, decoded when the stage starts,
// and every thread takes its rows' values by shuffle.
struct GvConsts {
  uint32_t e[2];
  float s2[2];
  __device__ void load(const GvParams& p, int row, int st, int lane) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int kb = st * 4 + 2 * (lane >> 4) + q;
      const bool ok = row < p.rows && kb < p.kbw;
      const int64_t blk = ok ? static_cast<int64_t>(row) * p.kbw + kb : 0;
      e[q] = ok ? __ldg(p.e4m3 + blk) : 0u;
      s2[q] = ok ? __ldg(p.s2 + blk / kGroup) : 0.0f;
    }
  }
};

template <int NT>
__global__ void __launch_bounds__(kGvThreads, GvCfg<NT>::CTAS_PER_SM)
    nf4_gemv_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmX,
                    const GvParams p, const CodebookArg cb) {
  using C = GvCfg<NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint32_t* lut = reinterpret_cast<uint32_t*>(base);
  uint8_t* stages = base + kGvLutBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(stages + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int64_t f0 = gv_start(cta, p.total, G), f1 = gv_start(cta + 1, p.total, G);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGvWarps);
    }
    fence_barrier_init();
  }
  // lut[e * 32 + l] = bf16 pair (level[e >> 4], level[e & 15]), one copy per lane l
  for (int i = threadIdx.x; i < 256 * 32; i += kGvThreads) {
    const int e = i >> 5;
    lut[e * 32 + (i & 31)] = pack_bf16x2(cb.levels[e >> 4], cb.levels[e & 15]);
  }
  __syncthreads();

  if (warp == kGvWarps) {                              // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmX);
      int64_t i = 0;
      for (int64_t f = f0; f < f1; ++f, ++i) {
        const int slot = static_cast<int>(i % C::STAGES);
        if (i >= C::STAGES && !mbar_wait(&empty[slot], static_cast<uint32_t>(((i / C::STAGES) - 1) & 1))) break;
        const int tile = static_cast<int>(f / p.spt), st = static_cast<int>(f % p.spt);
        uint8_t* sA = stages + slot * C::STAGE_BYTES;
        uint8_t* sX = sA + kGvTileBytes;
        mbar_arrive_expect_tx(&full[slot], C::STAGE_BYTES);
        tma_load_2d(sA, &tmA, &full[slot], st * kGvRowBytes, tile * kGvRows);
#pragma unroll
        for (int b = 0; b < 4; ++b) tma_load_2d(sX + b * C::X_BOX, &tmX, &full[slot], st * kGvStageK + 64 * b, 0);
      }
      // drain: the last phase issued into each slot has landed before the CTA may exit
      const int64_t issued = i;
      for (int64_t k = (issued > C::STAGES ? issued - C::STAGES : 0); k < issued; ++k)
        mbar_wait_short(&full[k % C::STAGES], static_cast<uint32_t>((k / C::STAGES) & 1));
    }
    return;
  }

  // ---------------------------------------- consumers ----------------------------------------------
  // Contraction order inside a 64-element block: the MMA's k index is permuted so that lane j's four
  // k16 steps cover the contiguous elements 16j .. 16j+15 of the block (step s: 16j+4s .. 16j+4s+3), the
  // same permutation for A and for X, so the sum is unchanged. Lane j then needs bytes 8j .. 8j+7 of a
  // row's 32 code bytes (one 8-byte load) and elements 16j .. 16j+15 of a token's 64 (two 16-byte loads).
  const int g = lane >> 2, j = lane & 3;
  const uint32_t lut_lane = smem_u32(lut) + 4u * lane;
  const int rl0 = 16 * warp + g;                                   // tile-local rows of this thread
  const float mu = *p.mu;
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
  bool waited_primary = false;
  int64_t i = 0;
  bool aborted = false;
  GvConsts nx;
  if (f0 < f1) nx.load(p, static_cast<int>(f0 / p.spt) * kGvRows + 16 * warp + (lane & 15), static_cast<int>(f0 % p.spt), lane);
  for (int64_t f = f0; f < f1; ++f, ++i) {
    const int tile = static_cast<int>(f / p.spt), st = static_cast<int>(f % p.spt);
    const int row0 = tile * kGvRows + rl0, row1 = row0 + 8;
    // decode this stage's constants (lane-owned), prefetch the next stage's, then gather by shuffle
    const float own0 = __fmaf_rn(decode_e4m3(static_cast<uint8_t>(nx.e[0])), nx.s2[0], mu);
    const float own1 = __fmaf_rn(decode_e4m3(static_cast<uint8_t>(nx.e[1])), nx.s2[1], mu);
    if (f + 1 < f1)
      nx.load(p, static_cast<int>((f + 1) / p.spt) * kGvRows + 16 * warp + (lane & 15),
              static_cast<int>((f + 1) % p.spt), lane);
    float chat[2][4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const float v = (b & 1) ? own1 : own0;                       // same register for every lane
      chat[0][b] = __shfl_sync(0xffffffffu, v, g + 16 * (b >> 1));
      chat[1][b] = __shfl_sync(0xffffffffu, v, g + 8 + 16 * (b >> 1));
    }
    const int slot = static_cast<int>(i % C::STAGES);
    if (!mbar_wait(&full[slot], static_cast<uint32_t>((i / C::STAGES) & 1))) {
      aborted = true;
      break;
    }
    const uint32_t sA = smem_u32(stages + slot * C::STAGE_BYTES);
    const uint32_t sX = sA + kGvTileBytes;
    const uint32_t rowA0 = sA + rl0 * kGvRowBytes, rowA1 = rowA0 + 8 * kGvRowBytes;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      if (st * 4 + b >= p.kbw) break;                              // beyond K in the last stage
      // code bytes 8j .. 8j+7 of block b: chunk 2b + j/2 of the row, 8-byte half j & 1
      const uint32_t cc = (static_cast<uint32_t>((2 * b + (j >> 1)) ^ g) << 4) + 8u * (j & 1);
      const uint2 u0 = lds64(rowA0 + cc), u1 = lds64(rowA1 + cc);
      // A fragments per k16 step s: code byte 2s (elements 16j+4s, +1) and 2s+1 (+2, +3) of the 8
      uint32_t a[4][4];
      a[0][0] = lut_pair<0>(lut_lane, u0.x); a[0][2] = lut_pair<1>(lut_lane, u0.x);
      a[1][0] = lut_pair<2>(lut_lane, u0.x); a[1][2] = lut_pair<3>(lut_lane, u0.x);
      a[2][0] = lut_pair<0>(lut_lane, u0.y); a[2][2] = lut_pair<1>(lut_lane, u0.y);
      a[3][0] = lut_pair<2>(lut_lane, u0.y); a[3][2] = lut_pair<3>(lut_lane, u0.y);
      a[0][1] = lut_pair<0>(lut_lane, u1.x); a[0][3] = lut_pair<1>(lut_lane, u1.x);
      a[1][1] = lut_pair<2>(lut_lane, u1.x); a[1][3] = lut_pair<3>(lut_lane, u1.x);
      a[2][1] = lut_pair<0>(lut_lane, u1.y); a[2][3] = lut_pair<1>(lut_lane, u1.y);
      a[3][1] = lut_pair<2>(lut_lane, u1.y); a[3][3] = lut_pair<3>(lut_lane, u1.y);
      const uint32_t cX0 = static_cast<uint32_t>((2 * j) ^ g) << 4, cX1 = static_cast<uint32_t>((2 * j + 1) ^ g) << 4;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const uint32_t xr = sX + b * C::X_BOX + (8 * t + g) * 128;
        const uint4 xlo = lds128(xr + cX0), xhi = lds128(xr + cX1);
        const uint32_t wx[8] = {xlo.x, xlo.y, xlo.z, xlo.w, xhi.x, xhi.y, xhi.z, xhi.w};
        float blk[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int s2i = 0; s2i < 4; ++s2i)
          mma_bf16_16816(blk, a[s2i][0], a[s2i][1], a[s2i][2], a[s2i][3], wx[2 * s2i], wx[2 * s2i + 1]);
        acc[t][0] = __fmaf_rn(chat[0][b], blk[0], acc[t][0]);
        acc[t][1] = __fmaf_rn(chat[0][b], blk[1], acc[t][1]);
        acc[t][2] = __fmaf_rn(chat[1][b], blk[2], acc[t][2]);
        acc[t][3] = __fmaf_rn(chat[1][b], blk[3], acc[t][3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);

    // ------------------------------ end of this CTA's part of a tile ------------------------------
    if (st == p.spt - 1 || f == f1 - 1) {
      const int64_t tf0 = static_cast<int64_t>(tile) * p.spt, tf1 = tf0 + p.spt;
      const bool whole = f0 <= tf0 && f1 >= tf1;
      bool finish = whole;
      if (!whole) {
        const int c_first = gv_owner(tf0, p.total, G), c_last = gv_owner(tf1 - 1, p.total, G);
        const int first_tile = static_cast<int>(f0 / p.spt);
        float* mine = p.part + (static_cast<int64_t>(cta) * p.maxseg + (tile - first_tile)) * C::SLOT +
                      (warp * 32 + lane) * (NT * 4);
#pragma unroll
        for (int t = 0; t < NT; ++t) reinterpret_cast<float4*>(mine)[t] = make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
        __threadfence();
        unsigned last = 0;
        if (lane == 0)
          last = (atomicAdd(&p.ticket[tile * kGvWarps + warp], 1u) == static_cast<unsigned>(c_last - c_first)) ? 1u : 0u;
        finish = __shfl_sync(0xffffffffu, last, 0) != 0;
        if (finish) {               // this warp arrived last for its 16 rows: add every part in CTA order
          __threadfence();
#pragma unroll
          for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
          constexpr int PB = NT >= 4 ? 2 : 4;                     // partials in flight per round
          for (int c0 = c_first; c0 <= c_last; c0 += PB) {
            float4 v[PB][NT];
#pragma unroll
            for (int u = 0; u < PB; ++u) {
              const int c = c0 + u;
              const int ft = static_cast<int>(gv_start(c <= c_last ? c : c_last, p.total, G) / p.spt);
              const float* src = p.part + (static_cast<int64_t>(c <= c_last ? c : c_last) * p.maxseg + (tile - ft)) * C::SLOT +
                                 (warp * 32 + lane) * (NT * 4);
#pragma unroll
              for (int t = 0; t < NT; ++t)
                v[u][t] = (c <= c_last) ? __ldcg(reinterpret_cast<const float4*>(src) + t) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < PB; ++u)
#pragma unroll
              for (int t = 0; t < NT; ++t) {
                acc[t][0] += v[u][t].x; acc[t][1] += v[u][t].y; acc[t][2] += v[u][t].z; acc[t][3] += v[u][t].w;
              }
          }
          if (lane == 0) p.ticket[tile * kGvWarps + warp] = 0u;
        }
      }
      if (finish) {
        if (!waited_primary) {          // sU comes from the preceding launch in the stream
          asm volatile("griddepcontrol.wait;" ::: "memory");
          waited_primary = true;
        }
        // LoRA term: acc += sU[t][:] . B[row][:], one more contraction over r with scale 1; each round of
        // four k16 steps issues all of its loads before the first MMA
        for (int kk0 = 0; kk0 < p.r; kk0 += 64) {
          uint32_t la[4][4], lb[4][NT][2];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int ka = kk0 + 16 * q + 2 * j, kb2 = ka + 8;
            la[q][0] = ldg32_or0(p.Bw + static_cast<int64_t>(row0) * p.r + ka, row0 < p.rows && ka < p.r);
            la[q][1] = ldg32_or0(p.Bw + static_cast<int64_t>(row1) * p.r + ka, row1 < p.rows && ka < p.r);
            la[q][2] = ldg32_or0(p.Bw + static_cast<int64_t>(row0) * p.r + kb2, row0 < p.rows && kb2 < p.r);
            la[q][3] = ldg32_or0(p.Bw + static_cast<int64_t>(row1) * p.r + kb2, row1 < p.rows && kb2 < p.r);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
              const int n = 8 * t + g;
              lb[q][t][0] = ldg32_or0(p.sU + static_cast<int64_t>(n) * p.r + ka, n < p.T && ka < p.r);
              lb[q][t][1] = ldg32_or0(p.sU + static_cast<int64_t>(n) * p.r + kb2, n < p.T && kb2 < p.r);
            }
          }
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int t = 0; t < NT; ++t) mma_bf16_16816(acc[t], la[q][0], la[q][1], la[q][2], la[q][3], lb[q][t][0], lb[q][t][1]);
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const int tok = 8 * t + 2 * j;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int row = (q < 2) ? row0 : row1, tk = tok + (q & 1);
            if (row < p.rows && tk < p.T) p.out[static_cast<int64_t>(tk) * p.ldo + row] = __float2bfloat16_rn(acc[t][q]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
    }
  }
  if (aborted) raise_status(kStatusTimeout);
}

// ------------------------------------------------------------------------------------------------
// sU = s X A^T for T <= kGvMaxTokens: one warp per (16 rows of A, contraction slice). Fragments come
// straight from global memory (both operands bf16, the same in-block k permutation as above), the next
// 64-element block's loads in flight while the current one multiplies. Slices of the same 16 rows are
// added by the last warp to arrive, in slice order. The CTAs are single warps without shared memory, so
// they run beside the NF4 launch that follows (which waits for this grid only before its LoRA term).
// ------------------------------------------------------------------------------------------------
struct GuParams {
  int T, r, K, kslices, kb_per_slice;
  const __nv_bfloat16* X;
  const __nv_bfloat16* A;
  float s;
  __nv_bfloat16* sU;          // T x r
  float* part;                // [r/16 groups][kslices][32 lanes][NT * 4]
  unsigned* ticket;           // one per group of 16 rows, zero on entry; left at zero
};

template <int NT>
__global__ void __launch_bounds__(32) lora_u_kernel(const GuParams p) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x, g = lane >> 2, j = lane & 3;
  const int grp = blockIdx.x, slice = blockIdx.y;
  const int r0 = 16 * grp + g, r1 = r0 + 8;
  const int kb0 = slice * p.kb_per_slice;
  const int kb1 = min(p.K / 64, kb0 + p.kb_per_slice);
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
  auto ld16 = [&](const __nv_bfloat16* row, bool ok, int kb, uint4& lo, uint4& hi) {
    if (ok) {
      const uint4* q = reinterpret_cast<const uint4*>(row + kb * 64 + 16 * j);
      lo = __ldg(q);
      hi = __ldg(q + 1);
    } else {
      lo = make_uint4(0, 0, 0, 0);
      hi = lo;
    }
  };
  uint4 a0lo, a0hi, a1lo, a1hi, xlo[NT], xhi[NT];
  const __nv_bfloat16* A0 = p.A + static_cast<int64_t>(r0) * p.K;
  const __nv_bfloat16* A1 = p.A + static_cast<int64_t>(r1) * p.K;
  if (kb0 < kb1) {
    ld16(A0, r0 < p.r, kb0, a0lo, a0hi);
    ld16(A1, r1 < p.r, kb0, a1lo, a1hi);
#pragma unroll
    for (int t = 0; t < NT; ++t) ld16(p.X + static_cast<int64_t>(8 * t + g) * p.K, 8 * t + g < p.T, kb0, xlo[t], xhi[t]);
  }
  for (int kb = kb0; kb < kb1; ++kb) {
    const uint32_t wa0[8] = {a0lo.x, a0lo.y, a0lo.z, a0lo.w, a0hi.x, a0hi.y, a0hi.z, a0hi.w};
    const uint32_t wa1[8] = {a1lo.x, a1lo.y, a1lo.z, a1lo.w, a1hi.x, a1hi.y, a1hi.z, a1hi.w};
    uint32_t wx[NT][8];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      wx[t][0] = xlo[t].x; wx[t][1] = xlo[t].y; wx[t][2] = xlo[t].z; wx[t][3] = xlo[t].w;
      wx[t][4] = xhi[t].x; wx[t][5] = xhi[t].y; wx[t][6] = xhi[t].z; wx[t][7] = xhi[t].w;
    }
    if (kb + 1 < kb1) {                                          // next block's loads in flight
      ld16(A0, r0 < p.r, kb + 1, a0lo, a0hi);
      ld16(A1, r1 < p.r, kb + 1, a1lo, a1hi);
#pragma unroll
      for (int t = 0; t < NT; ++t)
        ld16(p.X + static_cast<int64_t>(8 * t + g) * p.K, 8 * t + g < p.T, kb + 1, xlo[t], xhi[t]);
    }
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int s = 0; s < 4; ++s)
        mma_bf16_16816(acc[t], wa0[2 * s], wa1[2 * s], wa0[2 * s + 1], wa1[2 * s + 1], wx[t][2 * s], wx[t][2 * s + 1]);
  }
  bool finish = true;
  if (p.kslices > 1) {
    float* mine = p.part + (static_cast<int64_t>(grp) * p.kslices + slice) * (32 * NT * 4) + lane * NT * 4;
#pragma unroll
    for (int t = 0; t < NT; ++t) reinterpret_cast<float4*>(mine)[t] = make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
    __threadfence();
    unsigned last = 0;
    if (lane == 0) last = (atomicAdd(&p.ticket[grp], 1u) == static_cast<unsigned>(p.kslices - 1)) ? 1u : 0u;
    finish = __shfl_sync(0xffffffffu, last, 0) != 0;
    if (finish) {
      __threadfence();
#pragma unroll
      for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
      constexpr int UNR = NT >= 8 ? 1 : 8 / NT;                 // partials in flight per round
      for (int sl0 = 0; sl0 < p.kslices; sl0 += UNR) {
        float4 v[UNR][NT];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
          const int sl = sl0 + u;
          const float* src = p.part + (static_cast<int64_t>(grp) * p.kslices + sl) * (32 * NT * 4) + lane * NT * 4;
#pragma unroll
          for (int t = 0; t < NT; ++t)
            v[u][t] = (sl < p.kslices) ? __ldcg(reinterpret_cast<const float4*>(src) + t) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u)                           // in slice order
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            acc[t][0] += v[u][t].x; acc[t][1] += v[u][t].y; acc[t][2] += v[u][t].z; acc[t][3] += v[u][t].w;
          }
      }
      if (lane == 0) p.ticket[grp] = 0u;
    }
  }
  if (finish) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int tok = 8 * t + 2 * j;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int row = (q < 2) ? r0 : r1, tk = tok + (q & 1);
        if (row < p.r && tk < p.T) p.sU[static_cast<int64_t>(tk) * p.r + row] = __float2bfloat16_rn(p.s * acc[t][q]);
      }
    }
  }
}

}  // namespace qnf4
