// Tensor-core GEMM engine for the adapter products of the QLoRA layer on sm_100a (tcgen05 + TMEM + TMA).
//
//   D[m][n] = sum_c A[m][c] * B[n][c]      (U = X A^T, V = dY B, dA = V^T X, dB = dY^T U: every product
//                                          has one side of r <= 256 columns and a long contraction)
//
// One CTA computes a 128 x BN tile of D in tensor memory (fp32), stepping its share of the contraction
// (grid.z splits it; the host picks the split) in blocks of 64 through a STAGES-deep shared-memory ring,
// and writes the fp32 tile to a partial buffer that split_reduce_kernel adds up in a fixed order. Roles:
//   warp 0      TMA producer (one thread): A and B tiles
//   warp 1      MMA issuer (one thread) and TMEM owner: tcgen05.mma kind::f16, bf16 in, fp32 accumulate
//   warps 2-5   epilogue: tcgen05.ld the accumulator and store the fp32 partial tile
//
// Operand layouts in shared memory are the canonical 128-byte-swizzled tcgen05 layouts:
//   K-major  : rows of 64 bf16 (128 B), 8-row atoms of 1 KB; 16-byte chunk c of row r sits at chunk
//              position c ^ (r & 7). Descriptor SBO = 1 KB; the k-th 16-wide step adds 32 B.
//   MN-major : 64-element (128 B) MN slices, one per contraction row; 64 such rows form an 8 KB column
//              block; column blocks follow each other along MN. Descriptor LBO = 8 KB (MN direction),
//              SBO = 1 KB (8 contraction rows); the k-th 16-deep step adds 2 KB.
// Every wait is bounded (common.cuh): a wait that gives up sets the status word and the CTA unwinds
// (draining its own in-flight copies and MMAs) instead of hanging.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace qnf4 {

struct GemmParams {
  int nkb_total;            // contraction blocks of 64
  int kb_split;             // contraction blocks per CTA along grid.z
  float* out;               // fp32 partials [z][Mpad][BN]
  int64_t part_stride;      // elements between the partial tiles of consecutive z
};

template <int BN_, bool A_MN_, bool B_MN_, int STAGES_>
struct GemmCfg {
  static constexpr int BN = BN_, BM = 128, BK = 64, STAGES = STAGES_;
  static constexpr bool A_MN = A_MN_, B_MN = B_MN_;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int NUM_THREADS = 6 * 32;
  static constexpr int TMEM_COLS = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static constexpr uint32_t IDESC = idesc_bf16(BM, BN, A_MN, B_MN);
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M = 128");
  static_assert(!B_MN || BN % 64 == 0, "MN-major B tiles are whole 64-wide column blocks");
  static_assert(STAGE_BYTES % 1024 == 0, "stage buffers keep 1 KB swizzle-atom alignment");
  static_assert(2 * STAGES + 1 <= BAR_BYTES / 8 - 2, "barrier area");
};

// --- operand tile loads (TMA) ------------------------------------------------------------------
template <bool MN, int ROWS>
__device__ __forceinline__ void load_bf16_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar,
                                               int row0, int kb) {
  if constexpr (!MN) {
    tma_load_2d(dst, map, bar, kb * 64, row0);                     // box {64 (contraction), ROWS}
  } else {
#pragma unroll
    for (int a = 0; a < ROWS / 64; ++a)                            // box {64 (MN), 64 (contraction)}
      tma_load_2d(dst + a * 8192, map, bar, row0 + 64 * a, kb * 64);
  }
}

template <bool MN>
__device__ __forceinline__ uint64_t operand_desc(uint32_t saddr, int k) {
  if constexpr (!MN) return sdesc_sw128(saddr + 32u * k, 16u, 1024u);
  else return sdesc_sw128(saddr + 2048u * k, 8192u, 1024u);
}

template <class C>
__global__ void __launch_bounds__(C::NUM_THREADS, 1)
    gemm_sm100_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = base;
  uint8_t* sB = base + C::STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * C::BM, n0 = blockIdx.x * C::BN;
  const int kb_begin = blockIdx.z * p.kb_split;
  const int kb_end = min(p.nkb_total, kb_begin + p.kb_split);
  const int total_it = kb_end - kb_begin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  int issued = 0;   // producer: iterations whose loads were issued

  if (warp == 0) {
    // ------------------------------- TMA producer -------------------------------
    if (lane == 0) {
      for (int it = 0; it < total_it; ++it) {
        const int s = it % C::STAGES, r = it / C::STAGES;
        if (it >= C::STAGES && !mbar_wait(&empty[s], (r - 1) & 1)) { *abort_flag = 1; break; }
        if (*abort_flag) break;
        const int kb = kb_begin + it;
        mbar_arrive_expect_tx(&full[s], C::A_BYTES + C::B_BYTES);
        load_bf16_tile<C::A_MN, C::BM>(sA + s * C::A_BYTES, &tmA, &full[s], m0, kb);
        load_bf16_tile<C::B_MN, C::BN>(sB + s * C::B_BYTES, &tmB, &full[s], n0, kb);
        issued = it + 1;
      }
    }
  } else if (warp == 1) {
    // ------------------------------- MMA issuer -------------------------------
    if (lane == 0) {
      for (int it = 0; it < total_it; ++it) {
        const int s = it % C::STAGES, r = it / C::STAGES;
        if (!mbar_wait(&full[s], r & 1)) { *abort_flag = 1; break; }
        if (*abort_flag) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(sA + s * C::A_BYTES);
        const uint32_t b_addr = smem_u32(sB + s * C::B_BYTES);
#pragma unroll
        for (int k = 0; k < C::BK / 16; ++k)
          umma_bf16_ss(tmem_d, operand_desc<C::A_MN>(a_addr, k), operand_desc<C::B_MN>(b_addr, k), C::IDESC,
                       (it > 0 || k > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      umma_commit(accf);   // also issued after a give-up, so teardown can wait for the MMAs
    }
  } else {
    // ------------------------------- epilogue -------------------------------
    const int q = warp & 3;
    const bool ok = mbar_wait(accf, 0);
    if (!ok) *abort_flag = 1;
    // tcgen05.ld is warp-collective: decide once per warp
    if (__all_sync(0xffffffffu, ok && !*abort_flag)) {
      tc_fence_after();
      const int m = m0 + 32 * q + lane;
      const uint32_t trow = tmem_d + (static_cast<uint32_t>(32 * q) << 16);
#pragma unroll 1
      for (int c = 0; c < C::BN / 16; ++c) {
        uint32_t v[16];
        tmem_ld16(trow + 16 * c, v);
        tmem_wait_ld();
        float* outp = p.out + blockIdx.z * p.part_stride + static_cast<int64_t>(m) * C::BN + 16 * c;
#pragma unroll
        for (int h = 0; h < 4; ++h)
          reinterpret_cast<uint4*>(outp)[h] = make_uint4(v[4 * h], v[4 * h + 1], v[4 * h + 2], v[4 * h + 3]);
      }
    }
  }

  // ------------------------------- teardown -------------------------------
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (warp == 0 && lane == 0) {
      // wait for this CTA's copies still in flight before its shared memory goes away
      for (int it = (issued > C::STAGES ? issued - C::STAGES : 0); it < issued; ++it)
        mbar_wait_short(&full[it % C::STAGES], (it / C::STAGES) & 1);
    }
    if (warp == 1 && lane == 0) mbar_wait_short(accf, 0);
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, C::TMEM_COLS);
  }
}

// Deterministic split reduction: out = scale * sum_z part[z] in fixed z order.
//   kRowsBf16 : out bf16 [M][R] (row-major, R = real columns)          -- U, V
//   kTransF32 : out fp32 [R][M] (transposed)                           -- dA
//   kRowsF32  : out fp32 [M][R]                                        -- dB
enum class Red { kRowsBf16, kTransF32, kRowsF32 };
template <Red MODE>
__global__ void __launch_bounds__(256) split_reduce_kernel(const float* __restrict__ part, int splits,
                                                           int64_t part_stride, int BN, int64_t M, int R,
                                                           float scale, void* __restrict__ out) {
  const int64_t total = M * R;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int64_t m, j;
    if constexpr (MODE == Red::kTransF32) { j = i / M; m = i % M; }   // writes coalesced along m
    else { m = i / R; j = i % R; }                                    // writes coalesced along j
    float acc = 0.0f;
    for (int z = 0; z < splits; ++z) acc += part[z * part_stride + m * BN + j];
    acc *= scale;
    if constexpr (MODE == Red::kRowsBf16) reinterpret_cast<__nv_bfloat16*>(out)[m * R + j] = __float2bfloat16_rn(acc);
    else if constexpr (MODE == Red::kTransF32) reinterpret_cast<float*>(out)[j * M + m] = acc;
    else reinterpret_cast<float*>(out)[m * R + j] = acc;
  }
}

}  // namespace qnf4
