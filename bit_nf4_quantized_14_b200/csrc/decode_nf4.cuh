// Decode-sized QLoRA forward (T <= 16 tokens), one launch:
//     Y = X W_hat^T + sU B^T,   sU = s X A^T   (s = alpha / r),
// with W stored as NF4 codes plus double-quantized block constants. The weight is "dequantized to
// bfloat16 on the fly, block by block, and multiplied in 16-bit precision" (PEFT page,
// zerotofrontier.app/sft/peft, "Paged optimizers, and QLoRA end to end"), inside the matrix multiply
// (same page, "The real way"); the adapter term is the explainer's X L1 L2 (QLoRA explainer,
// prism.theerrors.in, "Putting it together").
//
// With a handful of tokens every weight is used T times, so the layer is bound by streaming 0.52 B per
// weight from HBM. The design keeps the per-weight work to two instructions (a byte permute and a
// shared-memory load per two weights) and moves everything else off that path:
//   * persistent grid, one CTA per SM (cooperative launch: every CTA resident). The rows of W (in units
//     of 8) and the rows of A (the adapter projection, also in units of 8, each weighted 4x for its 4x
//     bytes per element) are split into contiguous ranges, one per CTA; each CTA contracts its units over
//     the whole K, so no partial sum crosses CTAs;
//   * a TMA ring of stages, each 16 blocks (1024 contraction elements) of up to 8 NF4 units or 2 A units,
//     one three-dimensional box per stage (block, row, bytes of the block): codes land as
//     [block][row][32 B], which the fragment loads read without bank conflicts, and A rows as
//     [block][row][128 B] with the 128-byte swizzle; consumer warp w takes block w of every stage;
//   * mma.sync m16n8k16: the A operand is X (16 token rows, padded), the B operand is 8 rows of one
//     64-element block. For NF4 rows it is built from code bytes: prmt forms (byte << 8 | lane * 4) and one
//     shared-memory load fetches the bf16 pair (level[hi], level[lo]) from a 256-entry table replicated
//     per lane (entries 256 B apart, so the address needs no further arithmetic and never conflicts);
//   * the block constant c1_hat = fma(decode(e4m3), s2, mu) multiplies the fp32 result of each block's
//     four MMAs; a scale warp computes the stage's constants one stage ahead;
//   * at the end of each pass the 16 warps' partial sums meet in shared memory and are added in warp
//     order (deterministic). A units come first: their sums, times s and rounded to bf16, are sU, which
//     the CTA publishes with a per-call tag; a gather warp in every CTA waits for all of sU and copies it
//     into shared memory, and the adapter term sU B^T is one more contraction per unit at the end, against
//     B rows brought in by TMA.
// The one difference from the fused GEMM's W_hat = bf16(level * c1_hat) is where the bf16 rounding falls
// (on the level instead of the product): both round each weight once, to a relative 2^-9.
// sU's summation order depends only on K (not on the grid), and the backward recomputes it with this
// kernel in a projection-only mode, so the recomputed U is bit-identical to the forward's.
// Every wait is bounded (mbarriers and tags); on expiry the status word records a timeout and the CTA
// unwinds without further waits. Named barriers among the consumer warps are reached on every path.
#pragma once

#include <cuda.h>

#include "codec.cuh"
#include "common.cuh"

namespace qnf4 {

constexpr int kDcWarps = 16;                          // consumer warps: warp w takes block w of a stage
constexpr int kDcThreads = 32 * (kDcWarps + 2);       // + scale/TMA warp + gather warp
constexpr int kDcUnits = 8;                           // NF4 units per pass (8 rows each)
constexpr int kDcAUnits = 2;                          // A units per pass
constexpr int kDcALoad = 4;                           // an A unit weighs as much as 4 NF4 units
constexpr int kDcStages = 4;                          // ring slots
constexpr int kDcStageBlocks = 16;
constexpr int kDcSlotBytes = 32 * 1024;               // NF4: [col box 0..3][unit 0..7]; A: [unit][block]
constexpr int kDcLutBytes = 256 * 256;                // entry e at e * 256: lane copies in bytes 0..127
constexpr int kDcCbufBytes = kDcStageBlocks * 4 * kDcUnits * 2 * 4;   // [block][j][unit][2] fp32
constexpr int kDcMaxTokens = 16;
constexpr int kDcMaxRank = 256;
constexpr int kDcOffRing = kDcLutBytes;
constexpr int kDcOffCbuf = kDcOffRing + kDcStages * kDcSlotBytes;
constexpr int kDcOffSU = kDcOffCbuf + 2 * kDcCbufBytes;
constexpr int kDcSUBytes = kDcMaxTokens * kDcMaxRank * 2;
constexpr int kDcOffBase = kDcOffSU + kDcSUBytes;
constexpr int kDcSmemBytes = 227 * 1024;
constexpr int kDcOffBar = kDcSmemBytes - 256;
constexpr int kDcBaseBytes = kDcOffBar - kDcOffBase;  // per-CTA fp32 results awaiting the adapter term
static_assert(kDcBaseBytes >= 16 * 1024, "shared-memory budget");
static_assert(kDcAUnits * kDcStageBlocks * 1024 <= kDcSlotBytes, "an A stage fits a slot");

struct DecParams {
  int T, N, K, r, RP;        // RP: r rounded up to 64
  int nkb;                   // K / 64
  int units;                 // N / 8: NF4 units
  int aunits;                // r / 8: A units
  int u_only;                // 1: compute sU only (the backward's recompute)
  int base_in_smem;          // per-CTA fp32 results fit in shared memory
  float s;
  const __nv_bfloat16* X;    // T x K
  const uint8_t* e4m3;       // N * K / 64
  const float* s2;
  const float* mu;
  __nv_bfloat16* Y;          // T x N
  __nv_bfloat16* U;          // T x r: sU in bf16
  uint64_t* tags;            // one per A unit
  float* base_ws;            // [unit][T][8] fp32 when the shared copy does not fit
  uint64_t seq;              // this call's tag value
};

// Tensor maps of one call: codes as (32 bytes of a block, row, block) with a box height for every
// pass size of 1..8 units; A as (64 elements of a block, row, block) for passes of 1 or 2 units
// (128-byte swizzle); B as (r elements, row) for the adapter stages.
struct DcMaps {
  CUtensorMap c[kDcUnits];
  CUtensorMap a[kDcAUnits];
  CUtensorMap b;
};

__device__ __forceinline__ void dc_mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t dc_prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// Shared-memory loads as plain C++ loads from the __shared__ array (byte offsets from its start): the
// compiler knows their address space and schedules them freely among the lookups and MMAs, and keeps
// them after the mbarrier waits that publish the buffers (volatile asm with a memory clobber).
__device__ __forceinline__ uint32_t dc_ld32(const uint8_t* sm, uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(sm + off);
}
__device__ __forceinline__ uint2 dc_ld64(const uint8_t* sm, uint32_t off) {
  return *reinterpret_cast<const uint2*>(sm + off);
}
__device__ __forceinline__ uint4 dc_ld128(const uint8_t* sm, uint32_t off) {
  return *reinterpret_cast<const uint4*>(sm + off);
}
__device__ __forceinline__ void dc_bar_consumers() {   // the 16 consumer warps only
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kDcWarps) : "memory");
}
// Byte k of w looked up in this lane's table copy: offset (w.byte_k << 8) | lane * 4 in one permute.
template <int k>
__device__ __forceinline__ uint32_t dc_pair(const uint8_t* sm, uint32_t w, uint32_t lanebyte) {
  return dc_ld32(sm, dc_prmt(w, lanebyte, 0x5504u | (k << 4)));
}
// The fp32 partial-sum buffer of a pass lives in the free halves of the table's 256-byte entries.
__device__ __forceinline__ float* dc_red(uint8_t* sm, int idx) {
  return reinterpret_cast<float*>(sm + ((idx >> 5) << 8) + 128 + ((idx & 31) << 2));
}
// X operand fragments of one 64-element block for token rows g and g + 8 (clamped to T - 1; rows past
// T repeat the last token and their results are discarded): elements 16 j .. 16 j + 15 of the block.
template <int TT>
__device__ __forceinline__ void dc_load_x(const __nv_bfloat16* X, int K, int T, int blk, int g, int j, uint4 (&x)[TT / 4]) {
  const int t0 = min(g, T - 1);
  const uint4* p0 = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(t0) * K + blk * 64 + 16 * j);
  x[0] = __ldg(p0);
  x[1] = __ldg(p0 + 1);
  if constexpr (TT == 16) {
    const int t1 = min(g + 8, T - 1);
    const uint4* p1 = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(t1) * K + blk * 64 + 16 * j);
    x[2] = __ldg(p1);
    x[3] = __ldg(p1 + 1);
  }
}
__device__ __forceinline__ uint32_t dc_word(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}
// m16n8k16 step s (of the 4 in a 64-element block) against B fragments (b0, b1); the X operand holds
// elements 16 j + 4 s .. + 3 of token rows g (and g + 8): the same in-block order as the B fragments.
template <int TT>
__device__ __forceinline__ void dc_step(float (&d)[4], const uint4 (&x)[TT / 4], int s, uint32_t b0, uint32_t b1) {
  const uint32_t a0 = dc_word(x[s >> 1], 2 * (s & 1)), a2 = dc_word(x[s >> 1], 2 * (s & 1) + 1);
  uint32_t a1 = 0, a3 = 0;
  if constexpr (TT == 16) {
    a1 = dc_word(x[2 + (s >> 1)], 2 * (s & 1));
    a3 = dc_word(x[2 + (s >> 1)], 2 * (s & 1) + 1);
  }
  dc_mma(d, a0, a1, a2, a3, b0, b1);
}

// The CTA's share: on a load axis where A unit a spans [4a, 4a + 4) and NF4 unit k sits at 4 na + k,
// CTA c takes the units whose start lies in [c L / G, (c + 1) L / G), L = 4 na + nu.
struct DcShare { int a0, na, u0, nu; };
__device__ __forceinline__ DcShare dc_share(int cta, int G, int nu_all, int na_all) {
  const int64_t L = static_cast<int64_t>(kDcALoad) * na_all + nu_all;
  const int64_t lo = static_cast<int64_t>(cta) * L / G, hi = static_cast<int64_t>(cta + 1) * L / G;
  const int64_t abase = static_cast<int64_t>(kDcALoad) * na_all;
  auto clamp = [](int64_t v, int64_t hi_) { return static_cast<int>(v < 0 ? 0 : v > hi_ ? hi_ : v); };
  DcShare s;
  s.a0 = clamp((lo + kDcALoad - 1) / kDcALoad, na_all);
  s.na = clamp((hi + kDcALoad - 1) / kDcALoad, na_all) - s.a0;
  s.u0 = clamp(lo - abase, nu_all);
  s.nu = clamp(hi - abase, nu_all) - s.u0;
  return s;
}
// Pass q of the CTA: A passes (up to 2 A units) first, then NF4 passes of near-equal size (up to 8).
struct DcPass { bool isA; int cnt, first; };
__device__ __forceinline__ DcPass dc_pass(const DcShare& sh, int npa, int npn, int q) {
  DcPass r;
  if (q < npa) {
    r.isA = true;
    r.first = q * kDcAUnits;
    r.cnt = min(kDcAUnits, sh.na - r.first);
  } else {
    const int k = q - npa, b = sh.nu / npn, e = sh.nu % npn;
    r.isA = false;
    r.cnt = b + (k < e ? 1 : 0);
    r.first = k * b + min(k, e);
  }
  return r;
}

template <int TT>
__global__ void __launch_bounds__(kDcThreads, 1)
    nf4_decode_kernel(const __grid_constant__ DcMaps maps, const DecParams p, const CodebookArg cb) {
  extern __shared__ __align__(1024) uint8_t dc_smem[];
  uint8_t* dsm = dc_smem;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  uint64_t* full = reinterpret_cast<uint64_t*>(dsm + kDcOffBar);
  uint64_t* empty = full + kDcStages;
  uint64_t* sready = empty + kDcStages;
  uint64_t* suready = sready + 2;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(suready + 1);

  const DcShare sh = dc_share(cta, G, p.units, p.aunits);
  const int npa = (sh.na + kDcAUnits - 1) / kDcAUnits;
  const int npn = p.u_only ? 0 : (sh.nu + kDcUnits - 1) / kDcUnits;
  const int spp = (p.nkb + kDcStageBlocks - 1) / kDcStageBlocks;      // stages per pass
  const int nrb = p.RP / 64;                                           // 64-wide column boxes of B
  const int ulora = 32 / nrb;                                          // units per adapter stage
  const int nmain = (npa + npn) * spp;
  const int total = nmain + (p.u_only ? 0 : (sh.nu + ulora - 1) / ulora);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDcStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDcWarps);
    }
    mbar_init(&sready[0], 1);
    mbar_init(&sready[1], 1);
    mbar_init(suready, 1);
    *abort_flag = (smem_u32(dsm) & 1023u) != 0 ? 1 : 0;   // the swizzled boxes need 1 KB alignment
    fence_barrier_init();
  }
  __syncthreads();
  if (*abort_flag) {
    if (threadIdx.x == 0) raise_status(kStatusTimeout);
    return;
  }

  if (warp == kDcWarps) {
    // ================================ TMA + block constants ================================
    if (total == 0) return;
    if (lane == 0) tma_prefetch_desc(&maps.b);
    auto issue = [&](int i) {                       // lane 0
      const int slot = i % kDcStages;
      uint8_t* sb = dsm + kDcOffRing + slot * kDcSlotBytes;
      if (i < nmain) {
        const int st = i % spp;
        const DcPass ps = dc_pass(sh, npa, npn, i / spp);
        // one box per stage: 16 blocks x the pass's rows (blocks past K read as zeros and still count)
        if (ps.isA) {
          mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(ps.cnt * kDcStageBlocks * 1024));
          tma_load_3d(sb, &maps.a[ps.cnt - 1], &full[slot], 0, (sh.a0 + ps.first) * 8, st * kDcStageBlocks);
        } else {
          mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(ps.cnt * kDcStageBlocks * 256));
          tma_load_3d(sb, &maps.c[ps.cnt - 1], &full[slot], 0, (sh.u0 + ps.first) * 8, st * kDcStageBlocks);
        }
      } else {
        const int first = (i - nmain) * ulora, cntl = min(ulora, sh.nu - first);
        mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(cntl * nrb * min(p.r, 64) * 16));
        for (int u = 0; u < cntl; ++u)
          for (int c = 0; c < nrb; ++c)
            tma_load_2d(sb + (u * nrb + c) * 1024, &maps.b, &full[slot], c * 64, (sh.u0 + first + u) * 8);
      }
    };
    // Block constants of an NF4 stage, rows lane and lane + 32 of its pass. The raw E4M3 bytes and group
    // scales are loaded three stages ahead (a ring of three register sets), so decoding a stage never
    // waits for memory.
    const float mu = __ldg(p.mu);
    struct Raw { uint32_t ew[2][4]; float sa[2], sz[2]; };
    auto fetch = [&](int i, Raw& f) {
      if (i >= nmain) return;
      const DcPass ps = dc_pass(sh, npa, npn, i / spp);
      if (ps.isA) return;
      const int blk0 = (i % spp) * kDcStageBlocks, nbh = min(kDcStageBlocks, p.nkb - blk0);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int rho = lane + 32 * h;
        if (rho < ps.cnt * 8) {
          const int64_t e0 = static_cast<int64_t>((sh.u0 + ps.first) * 8 + rho) * p.nkb + blk0;
          const uint8_t* src = p.e4m3 + e0;
          if (nbh == 16 && (reinterpret_cast<uintptr_t>(src) & 15) == 0) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
            f.ew[h][0] = v.x; f.ew[h][1] = v.y; f.ew[h][2] = v.z; f.ew[h][3] = v.w;
          } else if (nbh == 16 && (reinterpret_cast<uintptr_t>(src) & 7) == 0) {
            const uint2 v0 = __ldg(reinterpret_cast<const uint2*>(src)), v1 = __ldg(reinterpret_cast<const uint2*>(src) + 1);
            f.ew[h][0] = v0.x; f.ew[h][1] = v0.y; f.ew[h][2] = v1.x; f.ew[h][3] = v1.y;
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t v = 0;
#pragma unroll
              for (int b = 0; b < 4; ++b)
                if (4 * q + b < nbh) v |= static_cast<uint32_t>(__ldg(src + 4 * q + b)) << (8 * b);
              f.ew[h][q] = v;
            }
          }
          f.sa[h] = __ldg(p.s2 + (e0 >> 8));
          f.sz[h] = __ldg(p.s2 + ((e0 + nbh - 1) >> 8));
        }
      }
    };
    Raw r0, r1, r2;
    auto scales = [&](int i) {                      // whole warp; decodes r0 (stage i), then shifts the ring
      const int cbi = i & 1;
      if (i < nmain) {
        const DcPass ps = dc_pass(sh, npa, npn, i / spp);
        if (!ps.isA) {
          const int blk0 = (i % spp) * kDcStageBlocks, nbh = min(kDcStageBlocks, p.nkb - blk0);
          float* cbuf = reinterpret_cast<float*>(dsm + kDcOffCbuf + cbi * kDcCbufBytes);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int rho = lane + 32 * h;
            if (rho < ps.cnt * 8) {
              // the group of block b: g0 for b below the first group boundary in the stage, else the next
              const int64_t e0 = static_cast<int64_t>((sh.u0 + ps.first) * 8 + rho) * p.nkb + blk0;
              const int bsplit = static_cast<int>(256 - (e0 & 255));   // >= 1; >= 16: one group
              float* dst = cbuf + ((rho & 7) >> 1) * (kDcUnits * 2) + (rho >> 3) * 2 + (rho & 1);
#pragma unroll
              for (int b = 0; b < 16; ++b) {
                const float s2v = b < bsplit ? r0.sa[h] : r0.sz[h];
                const uint8_t e = static_cast<uint8_t>(r0.ew[h][b >> 2] >> (8 * (b & 3)));
                dst[b * (4 * kDcUnits * 2)] = b < nbh ? __fmaf_rn(decode_e4m3(e), s2v, mu) : 0.0f;
              }
            }
          }
        }
      }
      r0 = r1;
      r1 = r2;
      fetch(i + 3, r2);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sready[cbi]);
    };
    if (lane == 0)
      for (int i = 0; i < min(kDcStages, total); ++i) issue(i);
    fetch(0, r0);
    fetch(1, r1);
    fetch(2, r2);
    scales(0);
    // Iteration i: the constants of stage i + 1 (their buffer last held stage i - 1's, released at
    // iteration i - 1), then wait until every consumer warp is done with stage i and refill its slot.
    int issued = min(kDcStages, total);
    for (int i = 0; i < total; ++i) {
      if (*abort_flag) break;
      if (i + 1 < total) scales(i + 1);
      if (lane == 0) {
        if (!mbar_wait(&empty[i % kDcStages], static_cast<uint32_t>((i / kDcStages) & 1))) {
          *abort_flag = 1;
        } else if (i + kDcStages < total) {
          issue(i + kDcStages);
          issued = i + kDcStages + 1;
        }
      }
      __syncwarp();
    }
    if (lane == 0)                                  // every issued copy has landed before the CTA exits
      for (int k = max(0, issued - kDcStages); k < issued; ++k)
        mbar_wait_short(&full[k % kDcStages], static_cast<uint32_t>((k / kDcStages) & 1));
    return;
  }

  if (warp == kDcWarps + 1) {
    // ==================== gather sU (every A unit's tag) into shared memory ====================
    if (p.u_only) return;
    bool ok = true;
    for (int a = 0; a < p.aunits && ok; ++a)
      if (!wait_word_eq(p.tags + a, p.seq)) ok = false;
    // [T][RP] bf16, columns past r zero; 16-byte pieces, four in flight per lane
    const int pieces = p.T * (p.RP / 8), per_row = p.RP / 8;
    for (int k0 = 0; k0 < pieces; k0 += 128) {
      uint4 v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int k = k0 + q * 32 + lane;
        const int t = k / per_row, c8 = k % per_row;
        v[q] = (ok && k < pieces && 8 * c8 < p.r)
                   ? __ldcg(reinterpret_cast<const uint4*>(p.U + static_cast<int64_t>(t) * p.r + 8 * c8))
                   : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int k = k0 + q * 32 + lane;
        if (k < pieces) reinterpret_cast<uint4*>(dsm + kDcOffSU)[k] = v[q];
      }
    }
    if (!ok) *abort_flag = 1;
    __syncwarp();
    if (lane == 0) mbar_arrive(suready);
    return;
  }

  // ======================================== consumers ========================================
  const int w = warp, g = lane >> 2, j = lane & 3;
  const uint32_t lanebyte = 4u * lane;
  const int T = p.T;
  if (nmain == 0) return;                           // u_only and no A unit here: nothing to do
  // the lookup table: entry e = (level[e >> 4], level[e & 15]) as a bf16 pair, one copy per lane
  for (int i = threadIdx.x; i < 256 * 32; i += 32 * kDcWarps) {
    const int e = i >> 5;
    reinterpret_cast<uint32_t*>(dsm)[e * 64 + (i & 31)] = pack_bf16x2(cb.levels[e >> 4], cb.levels[e & 15]);
  }
  dc_bar_consumers();

  float* base = p.base_in_smem ? reinterpret_cast<float*>(dsm + kDcOffBase)
                               : p.base_ws + static_cast<int64_t>(sh.u0) * T * 8;   // [unit][T][8]
  bool live = true;
  int i = 0;                                        // global stage index
  // X fragments for this warp's block column, PD stages ahead (a ring of register sets shifted each stage;
  // X stays in L2, so its latency is that of an L2 hit)
  constexpr int PD = TT == 16 ? 1 : 2;
  uint4 xr[PD + 1][TT / 4];
  auto xvalid = [&](int ii) { return ii < nmain && (ii % spp) * kDcStageBlocks + w < p.nkb; };
#pragma unroll
  for (int k = 0; k < PD; ++k)
    if (xvalid(k)) dc_load_x<TT>(p.X, p.K, T, (k % spp) * kDcStageBlocks + w, g, j, xr[k]);
  for (int q = 0; q < npa + npn; ++q) {
    const DcPass ps = dc_pass(sh, npa, npn, q);
    float acc[kDcUnits][TT == 16 ? 4 : 2];
#pragma unroll
    for (int u = 0; u < kDcUnits; ++u)
#pragma unroll
      for (int c = 0; c < (TT == 16 ? 4 : 2); ++c) acc[u][c] = 0.0f;
    for (int st = 0; st < spp; ++st, ++i) {
      const int slot = i % kDcStages;
      const int blk = st * kDcStageBlocks + w;
      const bool has = blk < p.nkb;
      if (xvalid(i + PD)) dc_load_x<TT>(p.X, p.K, T, ((i + PD) % spp) * kDcStageBlocks + w, g, j, xr[PD]);
      const uint4 (&xa)[TT / 4] = xr[0];
      if (live && *abort_flag) live = false;
      if (live && !mbar_wait(&sready[i & 1], static_cast<uint32_t>((i >> 1) & 1))) live = false;
      if (live && !mbar_wait(&full[slot], static_cast<uint32_t>((i / kDcStages) & 1))) live = false;
      if (!live) *abort_flag = 1;
      const uint32_t sbase = kDcOffRing + slot * kDcSlotBytes;
      if (live && has && ps.isA) {
        // bf16 rows of A: lane (g, j) reads elements 16 j .. 16 j + 15 of row g (chunks 2 j, 2 j + 1)
#pragma unroll
        for (int a = 0; a < kDcAUnits; ++a) {
          if (a >= ps.cnt) break;
          const uint32_t rb = sbase + (w * ps.cnt + a) * 1024 + g * 128;
          const uint4 v0 = dc_ld128(dsm, rb + (((2 * j) ^ g) << 4)), v1 = dc_ld128(dsm, rb + (((2 * j + 1) ^ g) << 4));
          float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
          dc_step<TT>(d, xa, 0, v0.x, v0.y);
          dc_step<TT>(d, xa, 1, v0.z, v0.w);
          dc_step<TT>(d, xa, 2, v1.x, v1.y);
          dc_step<TT>(d, xa, 3, v1.z, v1.w);
#pragma unroll
          for (int c = 0; c < (TT == 16 ? 4 : 2); ++c) acc[a][c] += d[c];
        }
      } else if (live && has) {
        const uint32_t sb = sbase + w * (ps.cnt * 256) + g * 32 + j * 8;
        const uint32_t cs_base = kDcOffCbuf + (i & 1) * kDcCbufBytes + ((w * 4 + j) * kDcUnits) * 8;
#pragma unroll
        for (int u = 0; u < kDcUnits; u += 2) {
          if (u >= ps.cnt) break;
          const uint4 cs = dc_ld128(dsm, cs_base + u * 8);      // (unit u: rows 2j, 2j+1), (unit u+1: ...)
#pragma unroll
          for (int uu = 0; uu < 2; ++uu) {
            if (u + uu >= ps.cnt) break;
            const uint2 cw = dc_ld64(dsm, sb + (u + uu) * 256);
            uint32_t b[8];
            b[0] = dc_pair<0>(dsm, cw.x, lanebyte); b[1] = dc_pair<1>(dsm, cw.x, lanebyte);
            b[2] = dc_pair<2>(dsm, cw.x, lanebyte); b[3] = dc_pair<3>(dsm, cw.x, lanebyte);
            b[4] = dc_pair<0>(dsm, cw.y, lanebyte); b[5] = dc_pair<1>(dsm, cw.y, lanebyte);
            b[6] = dc_pair<2>(dsm, cw.y, lanebyte); b[7] = dc_pair<3>(dsm, cw.y, lanebyte);
            float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int s = 0; s < 4; ++s) dc_step<TT>(d, xa, s, b[2 * s], b[2 * s + 1]);
            const float c0 = __uint_as_float(uu ? cs.z : cs.x), c1 = __uint_as_float(uu ? cs.w : cs.y);
            acc[u + uu][0] = __fmaf_rn(c0, d[0], acc[u + uu][0]);
            acc[u + uu][1] = __fmaf_rn(c1, d[1], acc[u + uu][1]);
            if constexpr (TT == 16) {
              acc[u + uu][2] = __fmaf_rn(c0, d[2], acc[u + uu][2]);
              acc[u + uu][3] = __fmaf_rn(c1, d[3], acc[u + uu][3]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
#pragma unroll
      for (int k = 0; k < PD; ++k)
#pragma unroll
        for (int m = 0; m < TT / 4; ++m) xr[k][m] = xr[k + 1][m];
    }
    // ---- end of pass: the 16 warps' partial sums, added in warp order; tokens in rounds of 8 ----
    const int rows = ps.cnt * 8;
#pragma unroll
    for (int half = 0; half < (TT == 16 ? 2 : 1); ++half) {
      const int tr0 = 8 * half, tn = min(8, T - tr0);
      if (tn <= 0) break;
      if (g < tn) {
#pragma unroll
        for (int u = 0; u < kDcUnits; ++u) {
          if (u >= ps.cnt) break;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int idx = ((w * rows) + u * 8 + 2 * j + hh) * tn + g;
            *dc_red(dsm, idx) = acc[u][2 * half + hh];
          }
        }
      }
      dc_bar_consumers();
      for (int o = threadIdx.x; o < rows * tn; o += 32 * kDcWarps) {
        const int ro = o / tn, t = o % tn;
        float sum = 0.0f;
#pragma unroll
        for (int ww = 0; ww < kDcWarps; ++ww) sum += *dc_red(dsm, (ww * rows + ro) * tn + t);
        if (ps.isA)                                 // sU = bf16(s * X A^T), column 8 (unit) + row
          p.U[static_cast<int64_t>(tr0 + t) * p.r + (sh.a0 + ps.first) * 8 + ro] = __float2bfloat16_rn(p.s * sum);
        else
          base[(static_cast<int64_t>(ps.first + ro / 8) * T + tr0 + t) * 8 + (ro & 7)] = sum;
      }
      dc_bar_consumers();
    }
    if (ps.isA && threadIdx.x == 0) {               // this pass's piece of sU is complete and visible
      __threadfence();
      for (int a = 0; a < ps.cnt; ++a) st_release_u64(p.tags + sh.a0 + ps.first + a, p.seq);
    }
  }
  if (p.u_only) return;
  // ---- adapter term and output: Y = bf16(base + sU B^T) per unit ----
  const int nl = total - nmain;
  const uint32_t su = kDcOffSU;
  const int bw = min(p.r, 64) * 2;                  // bytes per row of a B column box
  bool su_ok = live;
  if (su_ok && !mbar_wait(suready, 0)) su_ok = false;
  if (su_ok && *abort_flag) su_ok = false;
  for (int l = 0; l < nl; ++l, ++i) {
    const int slot = i % kDcStages;
    if (su_ok && *abort_flag) su_ok = false;
    bool ok = su_ok && mbar_wait(&sready[i & 1], static_cast<uint32_t>((i >> 1) & 1)) &&
              mbar_wait(&full[slot], static_cast<uint32_t>((i / kDcStages) & 1));
    if (!ok) {
      su_ok = false;
      *abort_flag = 1;
    }
    const int first = l * ulora, cntl = min(ulora, sh.nu - first);
    const uint32_t sb = kDcOffRing + slot * kDcSlotBytes;
    for (int uu = w; ok && uu < cntl; uu += kDcWarps) {
      const int ul = first + uu;
      float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      for (int rc = 0; rc < nrb; ++rc) {
        const uint32_t bb = sb + (uu * nrb + rc) * 1024 + g * bw;
        uint4 bv[2], av[TT / 4];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int off = 32 * j + 16 * hh;
          bv[hh] = off < bw ? dc_ld128(dsm, bb + off) : make_uint4(0, 0, 0, 0);
          av[hh] = dc_ld128(dsm, su + (min(g, T - 1) * p.RP + rc * 64 + 16 * j) * 2 + 16 * hh);
          if constexpr (TT == 16) av[2 + hh] = dc_ld128(dsm, su + (min(g + 8, T - 1) * p.RP + rc * 64 + 16 * j) * 2 + 16 * hh);
        }
#pragma unroll
        for (int s = 0; s < 4; ++s) dc_step<TT>(d, av, s, dc_word(bv[s >> 1], 2 * (s & 1)), dc_word(bv[s >> 1], 2 * (s & 1) + 1));
      }
      const int n = (sh.u0 + ul) * 8 + 2 * j;
#pragma unroll
      for (int half = 0; half < (TT == 16 ? 2 : 1); ++half) {
        const int t = g + 8 * half;
        if (t < T) {
          const float2 bs = *reinterpret_cast<const float2*>(base + (static_cast<int64_t>(ul) * T + t) * 8 + 2 * j);
          const __nv_bfloat162 y = __floats2bfloat162_rn(bs.x + d[2 * half], bs.y + d[2 * half + 1]);
          *reinterpret_cast<__nv_bfloat162*>(p.Y + static_cast<int64_t>(t) * p.N + n) = y;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
  if (!live || !su_ok) raise_status(kStatusTimeout);
}

}  // namespace qnf4
