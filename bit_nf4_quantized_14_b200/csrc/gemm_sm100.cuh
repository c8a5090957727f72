// Tensor-core GEMM engine for sm_100a (tcgen05 + TMEM + TMA), with an optional fused NF4 dequantizer.
//
//   D[m][n] = sum_c A[m][c] * B[n][c]   (+ sum_c A2[m][c] * B2[n][c], the LoRA segment)
//
// One CTA computes a 128 x BN tile of D in tensor memory (fp32), stepping the contraction in blocks of
// 64 through a STAGES-deep shared-memory ring. Warp roles:
//   warp 0      TMA producer (one thread): A tiles, and B tiles or packed NF4 code tiles
//   warp 1      MMA issuer (one thread) and TMEM owner: tcgen05.mma kind::f16, bf16 in, fp32 accumulate
//   warps 2-5   epilogue: tcgen05.ld the accumulator, convert, store
//   warps 6-13  (NF4 only) dequantizers: code tile -> bf16 tile in the tensor cores' swizzled layout
//
// The NF4 B operand realizes "dequantized to bfloat16 on the fly, block by block, and multiplied in
// 16-bit precision" (PEFT page, zerotofrontier.app/sft/peft, "Paged optimizers, and QLoRA end to end";
// fusing dequantization into the matrix multiply: same page, "The real way"). Each dequantizer thread
// expands one NF4 block (64 weights, one constant) per pipeline stage with exactly the rounding of the
// standalone dequantizer: w = bf16_rn(fp32(level[code] * fma(decode(e), s2, mu))).
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

#include "codec.cuh"
#include "common.cuh"

namespace qnf4 {

enum class BSrc { kTma, kNf4 };
enum class Epi { kBf16, kF32Partial };

struct GemmParams {
  int M, N;                 // output extent (rows, columns) for bounds in the bf16 epilogue
  int nkb_total;            // contraction blocks of 64 in the main segment
  int kb_split;             // contraction blocks per CTA along grid.z
  int nkb2;                 // contraction blocks of the LoRA segment (0: none)
  const uint8_t* e4m3;      // NF4 operand: E4M3 block constants, fp32 group scales, the mean
  const float* s2;
  const float* mu;
  int64_t w_rows, w_cols;   // NF4 operand: the stored weight is w_rows x w_cols (out x in)
  void* out;                // bf16 D[M][ldo]  or  fp32 partials [z][Mpad][BN]
  int64_t ldo;
  int64_t part_stride;
};

template <int BN_, bool A_MN_, bool B_MN_, BSrc BS_, bool LORA_, Epi EPI_, int STAGES_>
struct GemmCfg {
  static constexpr int BN = BN_, BM = 128, BK = 64, STAGES = STAGES_;
  static constexpr bool A_MN = A_MN_, B_MN = B_MN_, LORA = LORA_;
  static constexpr BSrc BS = BS_;
  static constexpr Epi EPI = EPI_;
  static constexpr bool NF4 = (BS == BSrc::kNf4);
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int C_BYTES = NF4 ? BN * BK / 2 : 0;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + C_BYTES;
  static constexpr int NUM_DEQ_WARPS = NF4 ? 8 : 0;
  static constexpr int NUM_THREADS = (6 + NUM_DEQ_WARPS) * 32;
  static constexpr int TMEM_COLS = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
  static constexpr uint32_t IDESC = idesc_bf16(BM, BN, A_MN, B_MN);
  static constexpr uint32_t IDESC2 = idesc_bf16(BM, BN, false, B_MN);   // LoRA: A2 is K-major
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M = 128");
  static_assert(!B_MN || BN % 64 == 0, "MN-major B tiles are whole 64-wide column blocks");
  static_assert(!NF4 || BN == 256, "the dequantizer maps one NF4 block per thread: 256 per stage");
  static_assert(STAGE_BYTES % 1024 == 0, "stage buffers keep 1 KB swizzle-atom alignment");
  static_assert(2 * STAGES + (NF4 ? STAGES : 0) + 1 <= BAR_BYTES / 8 - 2, "barrier area");
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
                      const __grid_constant__ CUtensorMap tmA2,
                      const __grid_constant__ CUtensorMap tmB2, const GemmParams p,
                      const CodebookArg cb) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = base;
  uint8_t* sB = base + C::STAGES * C::A_BYTES;
  uint8_t* sC = sB + C::STAGES * C::B_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* bfull = empty + C::STAGES;
  uint64_t* accf = bfull + C::STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * C::BM, n0 = blockIdx.x * C::BN;
  const int kb_begin = blockIdx.z * p.kb_split;
  const int kb_end = min(p.nkb_total, kb_begin + p.kb_split);
  const int nkb = kb_end - kb_begin;
  const int total_it = nkb + (C::LORA ? p.nkb2 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      if (C::NF4) mbar_init(&bfull[s], C::NUM_DEQ_WARPS);
    }
    mbar_init(accf, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (C::LORA) {
      tma_prefetch_desc(&tmA2);
      tma_prefetch_desc(&tmB2);
    }
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
        uint8_t* a_dst = sA + s * C::A_BYTES;
        uint8_t* b_dst = sB + s * C::B_BYTES;
        if (it < nkb) {
          const int kb = kb_begin + it;
          mbar_arrive_expect_tx(&full[s], C::A_BYTES + (C::NF4 ? C::C_BYTES : C::B_BYTES));
          load_bf16_tile<C::A_MN, C::BM>(a_dst, &tmA, &full[s], m0, kb);
          if constexpr (C::NF4) {
            uint8_t* c_dst = sC + s * C::C_BYTES;
            if constexpr (!C::B_MN) {
              tma_load_2d(c_dst, &tmB, &full[s], kb * 32, n0);           // {32 B, 256 rows}
            } else {
#pragma unroll
              for (int a = 0; a < 4; ++a)                                  // {32 B, 64 rows} x 4
                tma_load_2d(c_dst + a * 2048, &tmB, &full[s], n0 / 2 + 32 * a, kb * 64);
            }
          } else {
            load_bf16_tile<C::B_MN, C::BN>(b_dst, &tmB, &full[s], n0, kb);
          }
        } else {
          const int kb2 = it - nkb;
          mbar_arrive_expect_tx(&full[s], C::A_BYTES + C::B_BYTES);
          load_bf16_tile<false, C::BM>(a_dst, &tmA2, &full[s], m0, kb2);
          load_bf16_tile<C::B_MN, C::BN>(b_dst, &tmB2, &full[s], n0, kb2);
        }
        issued = it + 1;
      }
    }
  } else if (warp == 1) {
    // ------------------------------- MMA issuer -------------------------------
    if (lane == 0) {
      for (int it = 0; it < total_it; ++it) {
        const int s = it % C::STAGES, r = it / C::STAGES;
        const bool main_seg = it < nkb;
        if (!mbar_wait(&full[s], r & 1)) { *abort_flag = 1; break; }
        if (C::NF4 && main_seg && !mbar_wait(&bfull[s], r & 1)) { *abort_flag = 1; break; }
        if (*abort_flag) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(sA + s * C::A_BYTES);
        const uint32_t b_addr = smem_u32(sB + s * C::B_BYTES);
#pragma unroll
        for (int k = 0; k < C::BK / 16; ++k) {
          const uint64_t ad = main_seg ? operand_desc<C::A_MN>(a_addr, k) : operand_desc<false>(a_addr, k);
          const uint64_t bd = operand_desc<C::B_MN>(b_addr, k);
          umma_bf16_ss(tmem_d, ad, bd, main_seg ? C::IDESC : C::IDESC2, (it > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(accf);   // also issued after a give-up, so teardown can wait for the MMAs
    }
  } else if (warp < 6) {
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
        if constexpr (C::EPI == Epi::kBf16) {
          if (m < p.M) {
            __nv_bfloat16* outp = reinterpret_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(m) * p.ldo;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int n = n0 + 16 * c + 8 * h;
              if (n < p.N) {
                uint4 o;
                o.x = pack_bf16x2(__uint_as_float(v[8 * h + 0]), __uint_as_float(v[8 * h + 1]));
                o.y = pack_bf16x2(__uint_as_float(v[8 * h + 2]), __uint_as_float(v[8 * h + 3]));
                o.z = pack_bf16x2(__uint_as_float(v[8 * h + 4]), __uint_as_float(v[8 * h + 5]));
                o.w = pack_bf16x2(__uint_as_float(v[8 * h + 6]), __uint_as_float(v[8 * h + 7]));
                *reinterpret_cast<uint4*>(outp + n) = o;
              }
            }
          }
        } else {
          float* outp = reinterpret_cast<float*>(p.out) + blockIdx.z * p.part_stride +
                        static_cast<int64_t>(m) * C::BN + 16 * c;
#pragma unroll
          for (int h = 0; h < 4; ++h)
            reinterpret_cast<uint4*>(outp)[h] = make_uint4(v[4 * h], v[4 * h + 1], v[4 * h + 2], v[4 * h + 3]);
        }
      }
    }
  } else if constexpr (C::NF4) {
    // ------------------------------- NF4 dequantizers -------------------------------
    const int d = threadIdx.x - 6 * 32;             // 0..255: one NF4 block per stage
    int row, seg;                                   // row within the code tile, and its segment
    if constexpr (!C::B_MN) { row = d; seg = 0; }   // K-major: weight row n0 + d
    else { row = d & 63; seg = d >> 6; }            // MN-major: weight row kb*64 + row, cols n0 + 64 seg
    const int kb_w = static_cast<int>(p.w_cols / 64);
    const float qreg = cb.levels[lane & 15];
    const float mu = *p.mu;
    const int h = (row >> 2) & 1;                   // read order of the two 16-byte halves (no conflicts)
    const uint32_t c_off = seg * (C::B_MN ? 2048 : 0) + row * 32;
    const uint32_t b_off = (C::B_MN ? seg * 8192 : 0) + row * 128;
    const uint32_t rsw = row & 7;
    // Constants of the block this thread expands at contraction block kb. Rows or columns past the
    // weight's edge (zero-filled codes) get a zero scale, so they contribute exact zeros.
    auto scale_of = [&](int kb, uint8_t& e, float& s, bool& valid) {
      int64_t wr, wc;                               // weight row, and weight column block
      if constexpr (!C::B_MN) { wr = n0 + row; wc = kb; }
      else { wr = static_cast<int64_t>(kb) * 64 + row; wc = n0 / 64 + seg; }
      valid = wr < p.w_rows && wc < kb_w;
      const int64_t blk = wr * kb_w + wc;
      e = valid ? p.e4m3[blk] : 0;
      s = valid ? p.s2[blk / kGroup] : 0.0f;
    };
    uint8_t e_next = 0;
    float s_next = 0.0f;
    bool v_next = false;
    if (nkb > 0) scale_of(kb_begin, e_next, s_next, v_next);
    for (int it = 0; it < nkb; ++it) {
      const int s = it % C::STAGES, r = it / C::STAGES;
      const float chat = v_next ? __fmaf_rn(decode_e4m3(e_next), s_next, mu) : 0.0f;
      if (it + 1 < nkb) scale_of(kb_begin + it + 1, e_next, s_next, v_next);
      const bool ok = mbar_wait(&full[s], r & 1);
      // the lookups below are warp-wide shuffles: every lane takes the same branch
      if (!__all_sync(0xffffffffu, ok && !*abort_flag)) { *abort_flag = 1; break; }
      const uint32_t cbase = smem_u32(sC + s * C::C_BYTES) + c_off;
      const uint32_t bbase = smem_u32(sB + s * C::B_BYTES) + b_off;
      uint32_t cw[8];
      asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(cw[0]), "=r"(cw[1]), "=r"(cw[2]), "=r"(cw[3]) : "r"(cbase + 16 * h));
      asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(cw[4]), "=r"(cw[5]), "=r"(cw[6]), "=r"(cw[7]) : "r"(cbase + 16 * (h ^ 1)));
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t x = cw[j];
        const uint32_t word = static_cast<uint32_t>(j) ^ (4u * h);   // which 8 weights these are
        const float v0 = __fmul_rn(lut16(qreg, x >> 4), chat);
        const float v1 = __fmul_rn(lut16(qreg, x), chat);
        const float v2 = __fmul_rn(lut16(qreg, x >> 12), chat);
        const float v3 = __fmul_rn(lut16(qreg, x >> 8), chat);
        const float v4 = __fmul_rn(lut16(qreg, x >> 20), chat);
        const float v5 = __fmul_rn(lut16(qreg, x >> 16), chat);
        const float v6 = __fmul_rn(lut16(qreg, x >> 28), chat);
        const float v7 = __fmul_rn(lut16(qreg, x >> 24), chat);
        st_shared_v4(bbase + ((word ^ rsw) << 4), pack_bf16x2(v0, v1), pack_bf16x2(v2, v3),
                     pack_bf16x2(v4, v5), pack_bf16x2(v6, v7));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bfull[s]);
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
