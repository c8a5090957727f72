// Small-token QLoRA forward (decode shapes, T <= 64): Y = X W_hat^T + sU B^T, and the adapter projection
// sU = s X A^T that feeds it.
//
// For a handful of tokens every weight element is used T times, so the layer is bound by streaming the
// NF4 codes from HBM (0.52 B per weight); the work per byte is far too small for a 128 x 256 tensor-core
// tile. The pages ask for the weight to be "dequantized to bfloat16 on the fly, block by block, and
// multiplied in 16-bit precision" (PEFT page, zerotofrontier.app/sft/peft, "Paged optimizers, and QLoRA
// end to end"; dequantization fused into the matrix multiply: same page, "The real way"). Here the
// dequantization never materialises a weight tile:
//   * TMA streams tiles of 240 weight rows x 256 contraction elements (128 code bytes per row, 128-byte
//     swizzle) and the matching 64-wide boxes of X through a ring of stages;
//   * each consumer warp owns 16 rows and builds the A fragments of mma.sync m16n8k16 (bf16, fp32
//     accumulate) directly from code bytes: one shared-memory lookup per byte in a 256-entry table of
//     bf16 level pairs, replicated per lane so lookups never conflict;
//   * the block constant c1_hat = fma(decode(e4m3), s2, mu) multiplies the fp32 block accumulator once per
//     64-element block: y += c1_hat * sum_k bf16(level[code_k]) * x_k.
// The one difference from the fused GEMM's W_hat = bf16(level * c1_hat) is where the bf16 rounding falls
// (on the level instead of the product): both round each weight once, to a relative 2^-9.
//
// Work is split stream-K: the tiles x stages sequence is cut into gridDim.x contiguous ranges. A tile
// covered by one CTA is finished in registers; otherwise each warp writes its fp32 partial and, per 16
// rows, the last warp to arrive (atomic ticket) adds the partials in CTA order (deterministic), applies
// the LoRA term and writes Y. The dense variant (kDense) runs the same pipeline on a bf16 matrix (the adapter A) to produce sU.
// Every mbarrier wait is bounded; on expiry the status word records a timeout and the CTA unwinds.
#pragma once

#include <cuda.h>

#include "codec.cuh"
#include "common.cuh"

namespace qnf4 {

constexpr int kGvWarps = 15;                      // consumer warps, 16 rows each (16 warps per CTA)
constexpr int kGvRows = 16 * kGvWarps;            // rows per tile
constexpr int kGvThreads = 32 * (kGvWarps + 1);   // + one producer warp
constexpr int kGvRowBytes = 128;                  // A-operand bytes per row per stage
constexpr int kGvTileBytes = kGvRows * kGvRowBytes;
constexpr int kGvLutBytes = 256 * 32 * 4;
constexpr int kGvMaxTokens = 64;

template <int NT, bool kDense>
struct GvCfg {
  static constexpr int TP = 8 * NT;                          // tokens padded to the MMA's n8 tiles
  static constexpr int KB = kDense ? 1 : 4;                  // 64-element blocks per stage
  static constexpr int STAGE_K = 64 * KB;
  static constexpr int X_BOX = TP * 128;                     // one 64-wide box of X
  static constexpr int STAGE_BYTES = kGvTileBytes + KB * X_BOX;
  static constexpr int LUT_BYTES = kDense ? 0 : kGvLutBytes;
  static constexpr int AVAIL = 227 * 1024 - 1024 - 256 - LUT_BYTES;
  static constexpr int STAGES = (AVAIL / STAGE_BYTES) < 8 ? (AVAIL / STAGE_BYTES) : 8;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + LUT_BYTES + 256;
  static constexpr int SLOT = kGvWarps * 32 * NT * 4;          // floats of one CTA's partial tile
  static_assert(STAGES >= 2, "ring depth");
  static_assert(STAGE_BYTES % 1024 == 0 && X_BOX % 1024 == 0, "swizzle atoms stay 1 KB aligned");
};

struct GvParams {
  int T, rows, K;            // tokens, output rows (N, or r for the dense variant), contraction
  int spt, tiles;            // stages per tile, tiles of kGvRows rows
  int64_t total;             // tiles * spt
  int maxseg;                // partial slots per CTA
  int kbw;                   // NF4: 64-element blocks per weight row (K / 64)
  const uint8_t* e4m3;
  const float* s2;
  const float* mu;
  const __nv_bfloat16* sU;   // NF4: LoRA epilogue operands (sU: T x r, B: rows x r); null for dense
  const __nv_bfloat16* Bw;
  int r;
  float out_scale;           // applied to the result before the bf16 store (s for the dense variant)
  __nv_bfloat16* out;        // out[t * ldo + row]
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
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
// The A fragment register for code byte j of word w: the pair (level[hi nibble], level[lo nibble]).
__device__ __forceinline__ uint32_t lut_pair(uint32_t lut_lane, uint32_t w, uint32_t sel) {
  return lds32(lut_lane + (__byte_perm(w, 0u, sel) << 7));
}
__device__ __forceinline__ uint32_t ldg32_or0(const __nv_bfloat16* p, bool ok) {
  return ok ? __ldg(reinterpret_cast<const unsigned int*>(p)) : 0u;
}

template <int NT, bool kDense>
__global__ void __launch_bounds__(kGvThreads, 1)
    nf4_gemv_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmX,
                    const GvParams p, const CodebookArg cb) {
  using C = GvCfg<NT, kDense>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint32_t* lut = reinterpret_cast<uint32_t*>(base + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + C::STAGES * C::STAGE_BYTES + C::LUT_BYTES);
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
  if constexpr (!kDense) {      // lut[e * 32 + l] = bf16 pair (level[e >> 4], level[e & 15]) for every lane l
    for (int i = threadIdx.x; i < 256 * 32; i += kGvThreads) {
      const int e = i >> 5;
      lut[i] = pack_bf16x2(cb.levels[e >> 4], cb.levels[e & 15]);
    }
  }
  __syncthreads();
  // the NF4 launch that consumes sU may start now (it waits for this grid before reading sU)
  if constexpr (kDense) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == kGvWarps) {                              // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmX);
      int64_t i = 0;
      bool ok = true;
      for (int64_t f = f0; f < f1 && ok; ++f, ++i) {
        const int slot = static_cast<int>(i % C::STAGES);
        if (i >= C::STAGES && !mbar_wait(&empty[slot], static_cast<uint32_t>(((i / C::STAGES) - 1) & 1))) {
          ok = false;
          break;
        }
        const int tile = static_cast<int>(f / p.spt), st = static_cast<int>(f % p.spt);
        uint8_t* sA = base + slot * C::STAGE_BYTES;
        uint8_t* sX = sA + kGvTileBytes;
        mbar_arrive_expect_tx(&full[slot], C::STAGE_BYTES);
        tma_load_2d(sA, &tmA, &full[slot], kDense ? st * 64 : st * 128, tile * kGvRows);
#pragma unroll
        for (int b = 0; b < C::KB; ++b) tma_load_2d(sX + b * C::X_BOX, &tmX, &full[slot], st * C::STAGE_K + 64 * b, 0);
      }
      // drain: the last phase issued into each slot has landed before the CTA may exit
      const int64_t issued = i;
      for (int64_t k = (issued > C::STAGES ? issued - C::STAGES : 0); k < issued; ++k)
        mbar_wait_short(&full[k % C::STAGES], static_cast<uint32_t>((k / C::STAGES) & 1));
    }
    return;
  }

  // ---------------------------------------- consumers ----------------------------------------------
  const int g = lane >> 2, j = lane & 3;
  const uint32_t sel = 0x4440u | static_cast<uint32_t>(j);        // byte j of a word into byte 0
  const uint32_t lut_lane = smem_u32(lut) + 4u * lane;
  const int rl0 = 16 * warp + g;                                   // tile-local rows of this thread
  const float mu = kDense ? 0.0f : *p.mu;
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
  bool waited_primary = false;
  int64_t i = 0;
  bool aborted = false;
  for (int64_t f = f0; f < f1; ++f, ++i) {
    const int tile = static_cast<int>(f / p.spt), st = static_cast<int>(f % p.spt);
    const int row0 = tile * kGvRows + rl0, row1 = row0 + 8;
    // block constants of this stage's blocks, fetched before waiting for the stage's data
    float chat[2][4];
    if constexpr (!kDense) {
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int kb = st * 4 + b;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = h ? row1 : row0;
          float c = 0.0f;
          if (row < p.rows && kb < p.kbw) {
            const int64_t blk = static_cast<int64_t>(row) * p.kbw + kb;
            c = __fmaf_rn(decode_e4m3(__ldg(p.e4m3 + blk)), __ldg(p.s2 + blk / kGroup), mu);
          }
          chat[h][b] = c;
        }
      }
    }
    const int slot = static_cast<int>(i % C::STAGES);
    if (!mbar_wait(&full[slot], static_cast<uint32_t>((i / C::STAGES) & 1))) {
      aborted = true;
      break;
    }
    const uint32_t sA = smem_u32(base + slot * C::STAGE_BYTES);
    const uint32_t sX = sA + kGvTileBytes;
    const uint32_t rowA0 = sA + rl0 * kGvRowBytes, rowA1 = rowA0 + 8 * kGvRowBytes;
    if constexpr (kDense) {
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const uint32_t c0 = static_cast<uint32_t>((2 * s) ^ g) << 4, c1 = static_cast<uint32_t>((2 * s + 1) ^ g) << 4;
        const uint32_t a0 = lds32(rowA0 + c0 + 4 * j), a1 = lds32(rowA1 + c0 + 4 * j);
        const uint32_t a2 = lds32(rowA0 + c1 + 4 * j), a3 = lds32(rowA1 + c1 + 4 * j);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const uint32_t xr = sX + (8 * t + g) * 128 + 4 * j;
          mma_bf16_16816(acc[t], a0, a1, a2, a3, lds32(xr + c0), lds32(xr + c1));
        }
      }
    } else {
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        if (st * 4 + b >= p.kbw) break;                            // beyond K in the last stage
        const uint32_t ch0 = static_cast<uint32_t>((2 * b) ^ g) << 4, ch1 = static_cast<uint32_t>((2 * b + 1) ^ g) << 4;
        const uint4 r0lo = lds128(rowA0 + ch0), r0hi = lds128(rowA0 + ch1);
        const uint4 r1lo = lds128(rowA1 + ch0), r1hi = lds128(rowA1 + ch1);
        const uint32_t w0[8] = {r0lo.x, r0lo.y, r0lo.z, r0lo.w, r0hi.x, r0hi.y, r0hi.z, r0hi.w};
        const uint32_t w1[8] = {r1lo.x, r1lo.y, r1lo.z, r1lo.w, r1hi.x, r1hi.y, r1hi.z, r1hi.w};
        float blk[NT][4];
#pragma unroll
        for (int t = 0; t < NT; ++t) blk[t][0] = blk[t][1] = blk[t][2] = blk[t][3] = 0.0f;
        const uint32_t xb = sX + b * C::X_BOX + 4 * j;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          // k16 step s: code bytes 8s + j (k = 16s + 2j, +1) and 8s + 4 + j (k + 8, +9) of each row
          const uint32_t a0 = lut_pair(lut_lane, w0[2 * s], sel), a2 = lut_pair(lut_lane, w0[2 * s + 1], sel);
          const uint32_t a1 = lut_pair(lut_lane, w1[2 * s], sel), a3 = lut_pair(lut_lane, w1[2 * s + 1], sel);
          const uint32_t c0 = static_cast<uint32_t>((2 * s) ^ g) << 4, c1 = static_cast<uint32_t>((2 * s + 1) ^ g) << 4;
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const uint32_t xr = xb + (8 * t + g) * 128;
            mma_bf16_16816(blk[t], a0, a1, a2, a3, lds32(xr + c0), lds32(xr + c1));
          }
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          acc[t][0] = __fmaf_rn(chat[0][b], blk[t][0], acc[t][0]);
          acc[t][1] = __fmaf_rn(chat[0][b], blk[t][1], acc[t][1]);
          acc[t][2] = __fmaf_rn(chat[1][b], blk[t][2], acc[t][2]);
          acc[t][3] = __fmaf_rn(chat[1][b], blk[t][3], acc[t][3]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);

    // ------------------------------ end of this CTA's part of a tile ------------------------------
    if (st == p.spt - 1 || f == f1 - 1) {
      const int64_t tf0 = static_cast<int64_t>(tile) * p.spt, tf1 = tf0 + p.spt;
      const bool whole = f0 <= tf0 && f1 >= tf1;
      bool finish = whole;
      int c_first = cta, c_last = cta;
      if (!whole) {
        c_first = gv_owner(tf0, p.total, G);
        c_last = gv_owner(tf1 - 1, p.total, G);
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
          for (int c = c_first; c <= c_last; ++c) {
            const int ft = static_cast<int>(gv_start(c, p.total, G) / p.spt);
            const float* src = p.part + (static_cast<int64_t>(c) * p.maxseg + (tile - ft)) * C::SLOT +
                               (warp * 32 + lane) * (NT * 4);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
              const float4 v = __ldcg(reinterpret_cast<const float4*>(src) + t);
              acc[t][0] += v.x; acc[t][1] += v.y; acc[t][2] += v.z; acc[t][3] += v.w;
            }
          }
          if (lane == 0) p.ticket[tile * kGvWarps + warp] = 0u;
        }
      }
      if (finish) {
        if constexpr (!kDense) {
          if (!waited_primary) {          // sU comes from the preceding launch in the stream
            asm volatile("griddepcontrol.wait;" ::: "memory");
            waited_primary = true;
          }
          // LoRA term: acc += sU[t][:] . B[row][:], one more contraction over r with scale 1
          for (int kk = 0; kk < p.r; kk += 16) {
            const int ka = kk + 2 * j, kb2 = ka + 8;
            const uint32_t a0 = ldg32_or0(p.Bw + static_cast<int64_t>(row0) * p.r + ka, row0 < p.rows && ka < p.r);
            const uint32_t a1 = ldg32_or0(p.Bw + static_cast<int64_t>(row1) * p.r + ka, row1 < p.rows && ka < p.r);
            const uint32_t a2 = ldg32_or0(p.Bw + static_cast<int64_t>(row0) * p.r + kb2, row0 < p.rows && kb2 < p.r);
            const uint32_t a3 = ldg32_or0(p.Bw + static_cast<int64_t>(row1) * p.r + kb2, row1 < p.rows && kb2 < p.r);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
              const int n = 8 * t + g;
              const uint32_t b0 = ldg32_or0(p.sU + static_cast<int64_t>(n) * p.r + ka, n < p.T && ka < p.r);
              const uint32_t b1 = ldg32_or0(p.sU + static_cast<int64_t>(n) * p.r + kb2, n < p.T && kb2 < p.r);
              mma_bf16_16816(acc[t], a0, a1, a2, a3, b0, b1);
            }
          }
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const int tok = 8 * t + 2 * j;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int row = (q < 2) ? row0 : row1, tk = tok + (q & 1);
            if (row < p.rows && tk < p.T)
              p.out[static_cast<int64_t>(tk) * p.ldo + row] = __float2bfloat16_rn(p.out_scale * acc[t][q]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
    }
  }
  if (aborted) raise_status(kStatusTimeout);
}

}  // namespace qnf4
