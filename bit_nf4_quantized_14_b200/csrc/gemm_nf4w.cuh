// Fused NF4-dequantize + tensor-core GEMM for the QLoRA linear layer on sm_100a (persistent, 1 CTA/SM).
//
//   forward   Y^T[f][t]  = sum_k W~[f][k]  X[t][k]  + sum_j B[f][j]  U[t][j]      (f = out feature)
//   backward  dX^T[f][t] = sum_n W~[n][f]  dY[t][n] + sum_j A[j][f]  V[t][j]      (f = in feature)
//
// (PEFT page, zerotofrontier.app/sft/peft, "Paged optimizers, and QLoRA end to end": the frozen NF4
// weight is dequantized to bf16 on the fly, block by block, multiplied in 16-bit precision, and the bf16
// LoRA adapter is added to the output; "The real way": dequantization fused into the matrix multiply.
// U = s X A^T and V = s dY B come from the adapter kernels.)
//
// The dequantized weight is the MMA's A operand (128 features x 64 contraction per stage), expanded
// with exactly the standalone dequantizer's rounding, w = bf16_rn(fp32(level[code] * fma(decode(e), s2,
// mu))); the 256 tokens of a tile are the N operand. A 128 x 256 output tile needs 8192 dequantized
// weights per 64-deep stage of 2 M multiply-adds.
//
// Three shared-memory rings decouple the producers from the tensor cores:
//   token ring  (SX x 32 KB)  X / dY (or U / V) tiles by TMA, read by the MMA only
//   code ring   (SC x 5 KB)   packed NF4 code tiles and the stage's fp32 block constants (expanded once
//                             per call by nf4_expand_scales_kernel into a TMA-friendly layout), both by
//                             TMA on one mbarrier; it runs furthest ahead because the dequantizers need
//                             it before the tensor cores need anything
//   weight ring (SA x 16 KB)  bf16 weight tiles written by the dequantizers (for the LoRA segment: the
//                             adapter rows copied by the same threads), read by the MMA
// Warp roles: warp 0 token producer (TMA); warp 1 MMA issuer and TMEM owner (two 256-column fp32
// accumulators, so a tile's epilogue overlaps the next tile's main loop); warps 2-5 epilogue (tcgen05.ld,
// bf16, transpose through shared memory, TMA store); warp 6 code producer (TMA); warps 7..
// the dequantizers, in GROUPS groups of 8 warps that take alternate contraction slots, so that several
// slots are being expanded at once (one group's per-slot latency is longer than an MMA stage). Every wait
// is bounded (common.cuh); after a give-up the CTA drains its own copies and MMAs and exits.
#pragma once

#include <cuda.h>

#include "codec.cuh"
#include "common.cuh"

namespace qnf4 {

struct NF4GemmParams {
  int T;                   // tokens: the N extent of the MMA, rows of the bf16 output
  int F;                   // output features: the M extent, columns of the output
  int nkb;                 // contraction blocks of 64 in the weight segment
  int nkb2;                // contraction blocks of 64 in the LoRA segment
  int tiles_f, num_tiles;  // 128-feature tiles; tiles total (tiles_f x token tiles)
  int r;                   // adapter rank
  int64_t w_rows, w_cols;  // the stored weight is w_rows x w_cols (out x in)
  const __nv_bfloat16* lora_w;   // B (forward, N x r) or A (backward, r x K): the LoRA segment's A operand
};

template <bool BWD_, int GROUPS_>
struct NF4WCfg {
  static constexpr bool BWD = BWD_;     // weight enters transposed (MN-major A); LoRA A operand likewise
  static constexpr int GROUPS = GROUPS_;               // dequantizer groups, alternating slots
  static constexpr int GROUP_WARPS = 8;
  static constexpr int NUM_DEQ_WARPS = GROUPS * GROUP_WARPS;
  static constexpr int DEQ_THREADS = GROUP_WARPS * 32; // threads sharing one slot
  static constexpr int SX = 4, SC = 8, SA = 3;
  static constexpr int BM = 128, BN = 256, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;          // bf16 weight tile
  static constexpr int X_BYTES = BN * BK * 2;          // bf16 token tile
  static constexpr int C_BYTES = BM * BK / 2;          // packed codes
  static constexpr int K_BYTES = BWD ? 64 * 4 * 4 : BM * 4;   // fp32 constants: {4 block cols, 64 rows} / 128 rows
  static constexpr int CS_BYTES = C_BYTES + K_BYTES;   // one code-ring slot
  static constexpr int EPI_BUF = 16 * 32 * 2;          // 16 tokens x 32 features, bf16
  static constexpr int EPI_BYTES = 4 * 2 * EPI_BUF;    // 4 epilogue warps, double-buffered
  static constexpr int NUM_THREADS = (7 + NUM_DEQ_WARPS) * 32;
  static constexpr int EPW = BM * BK / DEQ_THREADS;    // weights per dequantizer thread per stage
  static constexpr int NCH = EPW / 8;                  // 16-byte chunks per dequantizer thread
  static constexpr int TMEM_COLS = 512;
  static constexpr int NUM_BARS = 2 * SX + 2 * SC + 2 * SA + 5;
  static constexpr int BAR_BYTES = (NUM_BARS * 8 + 8 + 127) / 128 * 128;
  static constexpr int SMEM_BYTES = SX * X_BYTES + SA * A_BYTES + SC * CS_BYTES + EPI_BYTES + BAR_BYTES + 1024;
  static constexpr uint32_t IDESC = idesc_bf16(BM, BN, BWD, false);
  static_assert(GROUPS == 1 || GROUPS == 2, "dequantizer groups");
  static_assert(X_BYTES % 1024 == 0 && A_BYTES % 1024 == 0 && CS_BYTES % 128 == 0, "alignment");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
};

__device__ __forceinline__ void tma_store_2d(const void* tmap, const void* smem_src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(tmap),
               "r"(smem_u32(smem_src)), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Eight NF4 codes (one 32-bit word: byte b holds weight 2b in its high nibble, 2b+1 in its low nibble)
// -> eight bf16, packed as the 16-byte chunk the operand layout stores.
__device__ __forceinline__ uint4 dequant8(uint32_t x, float qreg, float chat) {
  const float v0 = __fmul_rn(lut16(qreg, x >> 4), chat), v1 = __fmul_rn(lut16(qreg, x), chat);
  const float v2 = __fmul_rn(lut16(qreg, x >> 12), chat), v3 = __fmul_rn(lut16(qreg, x >> 8), chat);
  const float v4 = __fmul_rn(lut16(qreg, x >> 20), chat), v5 = __fmul_rn(lut16(qreg, x >> 16), chat);
  const float v6 = __fmul_rn(lut16(qreg, x >> 28), chat), v7 = __fmul_rn(lut16(qreg, x >> 24), chat);
  return make_uint4(pack_bf16x2(v0, v1), pack_bf16x2(v2, v3), pack_bf16x2(v4, v5), pack_bf16x2(v6, v7));
}

// A dequantizer thread's share of a stage: EPW consecutive weights of one operand row (NCH 16-byte
// chunks). Consecutive threads read consecutive code bytes, and the 8 lanes of every 16-byte store phase
// write 8 different bank groups of the swizzled tile (see the store loop).
template <class C>
struct DeqMap {
  int row;          // forward: weight row within the tile; backward: contraction row (a weight row)
  int part;         // which EPW-wide slice of the row (64 weights forward, 128 features backward)
  int atom;         // backward: 64-feature column block (0/1) of the slice; forward: 0
  uint32_t c_off;   // byte offset of this thread's codes in the code tile
  uint32_t a_off;   // byte offset of the row in the weight tile
  uint32_t chunk0;  // first 16-byte chunk (within the 128-byte row) this thread writes
  uint32_t k_idx;   // index of this thread's constant in the stage's constants tile (before the
                    // backward's column offset within the 4-wide box)
  __device__ explicit DeqMap(int d) {
    constexpr int PER_ROW = (C::BWD ? 128 : 64) / C::EPW;
    row = d / PER_ROW;
    part = d % PER_ROW;
    const int first = part * C::EPW;
    atom = C::BWD ? first / 64 : 0;
    c_off = static_cast<uint32_t>(row * (C::BWD ? 64 : 32) + first / 2);
    a_off = static_cast<uint32_t>(atom * 8192 + row * 128);
    chunk0 = static_cast<uint32_t>((first % 64) / 8);
    k_idx = static_cast<uint32_t>(C::BWD ? row * 4 + atom : row);
  }
};

template <class C>
__global__ void __launch_bounds__(C::NUM_THREADS, 1)
    nf4_linear_gemm_kernel(const __grid_constant__ CUtensorMap tmX,     // X or dY   [T][C], box {64, 256}
                           const __grid_constant__ CUtensorMap tmC,     // NF4 codes of the weight
                           const __grid_constant__ CUtensorMap tmK,     // expanded fp32 block constants
                           const __grid_constant__ CUtensorMap tmUV,    // U or V    [T][r], box {64, 256}
                           const __grid_constant__ CUtensorMap tmOut,   // Y or dX   [T][F], box {32, 16}
                           const NF4GemmParams p, const CodebookArg cb) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sX = base;
  uint8_t* sA = sX + C::SX * C::X_BYTES;
  uint8_t* sC = sA + C::SA * C::A_BYTES;
  uint8_t* sE = sC + C::SC * C::CS_BYTES;
  uint64_t* xfull = reinterpret_cast<uint64_t*>(sE + C::EPI_BYTES);
  uint64_t* xempty = xfull + C::SX;
  uint64_t* cfull = xempty + C::SX;
  uint64_t* cempty = cfull + C::SC;
  uint64_t* afull = cempty + C::SC;
  uint64_t* aempty = afull + C::SA;
  uint64_t* tfull = aempty + C::SA;      // [2]
  uint64_t* tempty = tfull + 2;          // [2]
  uint64_t* drain = tempty + 2;          // completes once every MMA this CTA issued has finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int iters = p.nkb + p.nkb2;     // contraction slots per tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SX; ++s) { mbar_init(&xfull[s], 1); mbar_init(&xempty[s], 1); }
    for (int s = 0; s < C::SC; ++s) { mbar_init(&cfull[s], 1); mbar_init(&cempty[s], C::GROUP_WARPS); }
    for (int s = 0; s < C::SA; ++s) { mbar_init(&afull[s], C::GROUP_WARPS); mbar_init(&aempty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], 4); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmC);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmUV);
    tma_prefetch_desc(&tmOut);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  int x_issued = 0;     // token producer: ring uses whose loads were issued
  int c_issued = 0;     // code producer: likewise

  if (warp == 0) {
    // ------------------------------- token producer -------------------------------
    if (lane == 0) {
      int it = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles && !*abort_flag; tile += gridDim.x) {
        const int t0 = (tile / p.tiles_f) * C::BN;
        for (int i = 0; i < iters; ++i, ++it) {
          const int s = it % C::SX, r = it / C::SX;
          if (it >= C::SX && !mbar_wait(&xempty[s], (r - 1) & 1)) { *abort_flag = 1; break; }
          if (*abort_flag) break;
          mbar_arrive_expect_tx(&xfull[s], C::X_BYTES);
          if (i < p.nkb) tma_load_2d(sX + s * C::X_BYTES, &tmX, &xfull[s], i * 64, t0);
          else tma_load_2d(sX + s * C::X_BYTES, &tmUV, &xfull[s], (i - p.nkb) * 64, t0);
          x_issued = it + 1;
        }
      }
    }
  } else if (warp == 6) {
    // ------------------------------- code producer -------------------------------
    if (lane == 0) {
      int it = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles && !*abort_flag; tile += gridDim.x) {
        const int f0 = (tile % p.tiles_f) * C::BM;
        for (int i = 0; i < p.nkb; ++i, ++it) {
          const int s = it % C::SC, r = it / C::SC;
          if (it >= C::SC && !mbar_wait(&cempty[s], (r - 1) & 1)) { *abort_flag = 1; break; }
          if (*abort_flag) break;
          uint8_t* slot = sC + s * C::CS_BYTES;
          mbar_arrive_expect_tx(&cfull[s], C::C_BYTES + C::K_BYTES);
          if constexpr (!C::BWD) {
            tma_load_2d(slot, &tmC, &cfull[s], i * 32, f0);                            // codes {32 B, 128}
            tma_load_2d(slot + C::C_BYTES, &tmK, &cfull[s], f0, i);                    // consts {128, 1}
          } else {
            tma_load_2d(slot, &tmC, &cfull[s], f0 / 2, i * 64);                        // codes {64 B, 64}
            tma_load_2d(slot + C::C_BYTES, &tmK, &cfull[s], (f0 / 64) & ~3, i * 64);   // consts {4, 64}
          }
          c_issued = it + 1;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------- MMA issuer -------------------------------
    if (lane == 0) {
      int it = 0, lt = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++lt) {
        const int b = lt & 1, u = lt >> 1;
        if (lt >= 2 && !mbar_wait(&tempty[b], (u - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * C::BN);
        for (int i = 0; i < iters; ++i, ++it) {
          const int sx = it % C::SX, sa = it % C::SA;
          if (!mbar_wait(&xfull[sx], (it / C::SX) & 1) || !mbar_wait(&afull[sa], (it / C::SA) & 1) ||
              *abort_flag) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + sa * C::A_BYTES);
          const uint32_t b_addr = smem_u32(sX + sx * C::X_BYTES);
#pragma unroll
          for (int k = 0; k < C::BK / 16; ++k) {
            const uint64_t ad = C::BWD ? sdesc_sw128(a_addr + 2048u * k, 8192u, 1024u)
                                       : sdesc_sw128(a_addr + 32u * k, 16u, 1024u);
            const uint64_t bd = sdesc_sw128(b_addr + 32u * k, 16u, 1024u);
            umma_bf16_ss(d_tmem, ad, bd, C::IDESC, (i > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&xempty[sx]);
          umma_commit(&aempty[sa]);
        }
        if (!ok) break;
        umma_commit(&tfull[b]);
      }
      if (!ok) *abort_flag = 1;
      umma_commit(drain);
    }
  } else if (warp < 6) {
    // ------------------------------- epilogue -------------------------------
    const int q = warp & 3;                    // TMEM lane quadrant this warp may access
    uint8_t* ebuf = sE + q * 2 * C::EPI_BUF;
    int lt = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++lt) {
      const int f0 = (tile % p.tiles_f) * C::BM, t0 = (tile / p.tiles_f) * C::BN;
      const int b = lt & 1, u = lt >> 1;
      const bool ok = mbar_wait(&tfull[b], u & 1);
      if (!__all_sync(0xffffffffu, ok && !*abort_flag)) { *abort_flag = 1; break; }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(b * C::BN);
#pragma unroll 1
      for (int c = 0; c < C::BN / 16; ++c) {
        uint32_t v[16];
        tmem_ld16(taddr + 16 * c, v);
        tmem_wait_ld();
        uint8_t* buf = ebuf + (c & 1) * C::EPI_BUF;
        if (lane == 0) bulk_wait_read_1();      // the store that last used this buffer has read it
        __syncwarp();
        uint16_t* col = reinterpret_cast<uint16_t*>(buf) + lane;   // [token][32 features]
#pragma unroll
        for (int t = 0; t < 16; ++t) col[t * 32] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[t])));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmOut, buf, f0 + 32 * q, t0 + 16 * c);
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[b]);
    }
    if (lane == 0) bulk_wait_all();
  } else {
    // ------------------------------- dequantizers -------------------------------
    const int group = (warp - 7) / C::GROUP_WARPS;   // this warp takes the slots with ia % GROUPS == group
    const DeqMap<C> m(threadIdx.x - 7 * 32 - group * C::DEQ_THREADS);
    const float qreg = cb.levels[lane & 15];
    const bool rev = C::BWD && m.atom;           // store order, see below
    const uint32_t rsw = static_cast<uint32_t>(m.row & 7);
    int ic = 0, ia = 0;      // code-ring and weight-ring uses
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
      const int f0 = (tile % p.tiles_f) * C::BM;
      for (int i = 0; i < iters; ++i, ++ia) {
        if (ia % C::GROUPS != group) {           // another group's slot: only keep the code-ring count
          if (i < p.nkb) ++ic;
          continue;
        }
        const int sa = ia % C::SA;
        uint32_t w[C::NCH * 4];                  // this thread's share of the stage, as 16-byte chunks
        if (i < p.nkb) {
          const int sc = ic % C::SC;
          ok = mbar_wait(&cfull[sc], (ic / C::SC) & 1);
          // the lookups below are warp-wide shuffles: every lane takes the same branch
          if (!__all_sync(0xffffffffu, ok && !*abort_flag)) { ok = false; break; }
          const uint8_t* slot = sC + sc * C::CS_BYTES;
          // the block's expanded constant; the backward box starts at the 4-aligned block column
          const uint32_t kq = C::BWD ? m.k_idx + static_cast<uint32_t>((f0 / 64) & 3) : m.k_idx;
          const float chat = reinterpret_cast<const float*>(slot + C::C_BYTES)[kq];
          uint32_t cw[C::NCH];
          if constexpr (C::NCH == 4) {
            const uint4 v = *reinterpret_cast<const uint4*>(slot + m.c_off);
            cw[0] = v.x; cw[1] = v.y; cw[2] = v.z; cw[3] = v.w;
          } else {
            const uint2 v = *reinterpret_cast<const uint2*>(slot + m.c_off);
            cw[0] = v.x; cw[1] = v.y;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&cempty[sc]);
          ++ic;
#pragma unroll
          for (int j = 0; j < C::NCH; ++j) {
            const uint4 o = dequant8(cw[j], qreg, chat);
            w[4 * j] = o.x; w[4 * j + 1] = o.y; w[4 * j + 2] = o.z; w[4 * j + 3] = o.w;
          }
        } else {
          // LoRA segment: copy this thread's share of the adapter (bf16) into the operand layout
          const int kb2 = i - p.nkb;
#pragma unroll
          for (int j = 0; j < C::NCH; ++j) {
            int64_t fr, jc;        // row and column of 8 adapter weights in the stored adapter
            bool valid;
            if constexpr (!C::BWD) {   // B: N x r, row = out feature, contiguous along j
              fr = f0 + m.row; jc = static_cast<int64_t>(kb2) * 64 + m.part * C::EPW + 8 * j;
              valid = fr < p.w_rows && jc < p.r;
            } else {                   // A: r x K, row = j, contiguous along the in feature
              fr = static_cast<int64_t>(kb2) * 64 + m.row; jc = f0 + m.part * C::EPW + 8 * j;
              valid = fr < p.r && jc < p.w_cols;
            }
            const int64_t ld = C::BWD ? p.w_cols : p.r;
            uint4 o = make_uint4(0, 0, 0, 0);
            if (valid) o = __ldg(reinterpret_cast<const uint4*>(p.lora_w + fr * ld + jc));
            w[4 * j] = o.x; w[4 * j + 1] = o.y; w[4 * j + 2] = o.z; w[4 * j + 3] = o.w;
          }
        }
        // the weight-ring slot must be free: its previous use has been read by the tensor cores
        if (ia >= C::SA) ok = mbar_wait(&aempty[sa], ((ia / C::SA) - 1) & 1);
        if (!__all_sync(0xffffffffu, ok && !*abort_flag)) { ok = false; break; }
        uint8_t* dst = sA + sa * C::A_BYTES + m.a_off;
#pragma unroll
        for (int j = 0; j < C::NCH; ++j) {
          // backward: a row's two 64-feature blocks store their chunks in opposite orders, so the
          // 8 lanes of one store phase (one row, both blocks) never hit the same bank group
          const int jr = C::NCH - 1 - j;
          const uint4 val = rev ? make_uint4(w[4 * jr], w[4 * jr + 1], w[4 * jr + 2], w[4 * jr + 3])
                                : make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          const uint32_t pos = (m.chunk0 + static_cast<uint32_t>(rev ? jr : j)) ^ rsw;
          *reinterpret_cast<uint4*>(dst + (pos << 4)) = val;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[sa]);
      }
    }
    if (!ok) *abort_flag = 1;
  }

  // ------------------------------- teardown -------------------------------
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // wait for this CTA's copies still in flight before its shared memory goes away
    if (warp == 0 && lane == 0)
      for (int it = (x_issued > C::SX ? x_issued - C::SX : 0); it < x_issued; ++it)
        mbar_wait_short(&xfull[it % C::SX], (it / C::SX) & 1);
    if (warp == 6 && lane == 0)
      for (int it = (c_issued > C::SC ? c_issued - C::SC : 0); it < c_issued; ++it)
        mbar_wait_short(&cfull[it % C::SC], (it / C::SC) & 1);
    if (warp == 1 && lane == 0) mbar_wait_short(drain, 0);
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace qnf4
