// Decode-sized QLoRA forward (T <= 16 tokens), one launch:
//     Y = X W_hat^T + sU B^T,   sU = s X A^T   (s = alpha / r),
// with W stored as NF4 codes plus double-quantized block constants. The weight is expanded to bf16 block
// by block while the contraction consumes it and multiplied in 16-bit arithmetic (PEFT page,
// zerotofrontier.app/sft/peft, "Paged optimizers, and QLoRA end to end"; the fused form: same page, "The
// real way"); the adapter term is the explainer's X L1 L2 (QLoRA explainer, prism.theerrors.in, "Putting
// it together").
//
// With a handful of tokens every weight is used T times, so the layer is bound by streaming 0.52 B per
// weight from HBM. The design keeps the per-weight work to two instructions (a byte permute and a
// shared-memory load per two weights) and keeps the HBM stream out of shared memory:
//   * persistent grid, one CTA per SM (cooperative launch: every CTA resident). The rows of W and of A
//     (the adapter projection), in tiles of 16 rows, are split into contiguous ranges, one per CTA (an A
//     tile weighs 4 NF4 tiles: bf16 against 4-bit); each CTA contracts its tiles over the whole K, so no
//     partial sum crosses CTAs;
//   * passes of up to 4 tiles (2 above 8 tokens), each a sequence of stages of 16 blocks (1024 contraction
//     elements); each of the 8 consumer warps takes 2 blocks of every stage (fewer, fuller warps: less
//     per-stage bookkeeping per weight). A stage (64 rows x 512 B of codes, or 16 A rows x 2 KB) comes into a ring of 4
//     shared-memory slots by cp.async three stages ahead, ~96 KB per SM in flight without holding
//     registers: each warp copies 8 whole 512-byte row segments (contiguous runs, which HBM serves a quarter
//     faster than 32-byte pieces of 64 rows), one named barrier per stage publishes the slot, and 16-byte
//     pieces are XOR-swizzled by row so the fragment loads are free of bank conflicts. The A stages and the
//     NF4 stages run in two loops, each holding only its own code: the stage code is large, and keeping one
//     copy of it per loop keeps the instruction cache warm;
//   * mma.sync m16n8k16 with the weight as the 16-row A operand and X as the 8-token B operand. The A
//     fragments come from code bytes: one prmt forms the whole shared address (1 << 16 | byte << 8 |
//     lane * 4) and one shared-memory load fetches the bf16 pair (level[hi], level[lo]) from a 256-entry
//     table at shared address 64 KB, replicated per lane (entries 256 B apart: no bank conflicts). Inside each 64-element block the MMA's k index is
//     permuted (the same permutation on both operands) so lane j's 16 elements are 16 j .. 16 j + 15;
//   * the block constant c1_hat = fma(decode(e4m3), s2, mu) multiplies the fp32 result of each block's four
//     MMAs (run as two chains of two); two helper warps (alternate stages) decode each stage's constants into a ring of shared-memory
//     buffers ahead of the consumers;
//   * at the end of each pass the 16 warps' partial sums meet in shared memory and are added in warp
//     order (deterministic). A tiles come first: their sums, times s and rounded to bf16, are sU, which the
//     CTA publishes with a per-call tag; a gather warp in every CTA waits for all of sU and copies it into
//     shared memory, and the adapter term sU B^T is one more contraction per tile at the end, with B rows
//     loaded straight into the MMA's A operand.
// The one difference from the fused GEMM's W_hat = bf16(level * c1_hat) is where the bf16 rounding falls
// (on the level instead of the product): both round each weight once, to a relative 2^-9.
// sU's summation order depends only on K (not on the grid), and the backward recomputes it with this
// kernel in a projection-only mode, so the recomputed U is bit-identical to the forward's.
// Every wait is bounded (mbarriers and tags); on expiry the status word records a timeout and the CTA
// unwinds without further waits. Named barriers among the consumer warps are reached on every path.
#pragma once

#include <type_traits>

#include "codec.cuh"
#include "common.cuh"

namespace qnf4 {

constexpr int kDcWarps = 8;                           // consumer warps: warp w takes blocks 2 w, 2 w + 1 of a stage
constexpr int kDcScaleWarps = 2;                      // constants warps, alternate NF4 stages
constexpr int kDcThreads = 32 * (kDcWarps + kDcScaleWarps + 1);   // + constants warps + gather warp
constexpr int kDcMaxTiles = 4;                        // NF4 tiles per pass (2 when T > 8)
constexpr int kDcALoad = 4;                           // an A tile weighs as much as 4 NF4 tiles
constexpr int kDcStageBlocks = 16;
constexpr int kDcBpw = kDcStageBlocks / kDcWarps;     // blocks per consumer warp and stage
constexpr int kDcRowsPw = 64 / kDcWarps;              // NF4 rows each warp copies per stage
constexpr int kDcARowsPw = 16 / kDcWarps;             // A rows each warp copies per stage
constexpr int kDcRing = 4;                            // stage slots
constexpr int kDcSlotBytes = 32 * 1024;               // one stage: 64 rows x 512 B, or 16 A rows x 2 KB
constexpr int kDcCRing = 4;                           // constant buffers (stages) in flight
constexpr int kDcMaxTokens = 16;
constexpr int kDcMaxRank = 256;
// Shared memory. The lookup table (256 entries of 256 bytes, lane copies in bytes 0..127, the pass's partial
// sums in bytes 128..255) sits at shared address 64 KB, so a byte permute forms a lookup's whole address
// (0x1 << 16 | byte << 8 | lane * 4) with no add. Below it, from the dynamic base (a few KB at most): the
// constant buffers, sU, the barriers and ring slot 0; above it, at 128 KB, ring slots 1..3.
constexpr uint32_t kDcLutAddr = 1u << 16;
constexpr uint32_t kDcHighAddr = 2u << 16;
constexpr int kDcCbufBytes = kDcStageBlocks * kDcMaxTiles * 8 * 8;   // [block][tile][g] (row g, row g + 8)
constexpr int kDcOffCbuf = 0;
constexpr int kDcOffSU = kDcOffCbuf + kDcCRing * kDcCbufBytes;
constexpr int kDcSUBytes = kDcMaxTokens * kDcMaxRank * 2;
constexpr int kDcOffBar = kDcOffSU + kDcSUBytes;
constexpr int kDcOffSlot0 = kDcOffBar + 1024;
constexpr int kDcMaxBase = static_cast<int>(kDcLutAddr) - (kDcOffSlot0 + kDcSlotBytes);   // dynamic base limit
constexpr int kDcSmemBytes = static_cast<int>(kDcHighAddr) + (kDcRing - 1) * kDcSlotBytes;  // enough for base 0
static_assert(kDcMaxBase >= 4096 && kDcSmemBytes <= 227 * 1024, "shared-memory budget");
static_assert(kDcCRing % kDcScaleWarps == 0, "each constants buffer belongs to one constants warp");

struct DecParams {
  int T, N, K, r, RP;        // RP: r rounded up to 64
  int nkb;                   // K / 64
  int tiles;                 // ceil(N / 16): NF4 tiles
  int atiles;                // ceil(r / 16): A tiles
  int u_only;                // 1: compute sU only (the backward's recompute)
  float s;
  const __nv_bfloat16* X;    // T x K
  const uint8_t* codes;      // N x K / 2
  const uint8_t* e4m3;       // N * K / 64
  const float* s2;
  const float* mu;
  const __nv_bfloat16* A;    // r x K
  const __nv_bfloat16* B;    // N x r
  __nv_bfloat16* Y;          // T x N
  __nv_bfloat16* U;          // T x r: sU in bf16
  uint64_t* tags;            // one per A tile
  float* base_ws;            // [tile][16][T] fp32: NF4 results awaiting the adapter term
  uint64_t seq;              // this call's tag value
};

__device__ __forceinline__ void dc_mma(float& d0, float& d1, float& d2, float& d3, uint32_t a0, uint32_t a1,
                                       uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d0), "+f"(d1), "+f"(d2), "+f"(d3)
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t dc_prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// Shared-memory loads by 32-bit shared address. Table lookups are plain asm (their addresses depend on
// code bytes read after the barriers that publish the table and the stage, and the compiler may schedule
// them freely); loads of ring slots and constant buffers are volatile, so they stay after the waits and
// barriers that publish those buffers.
__device__ __forceinline__ uint32_t dc_lut(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 dc_ld64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ float2 dc_ldf2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 dc_ld128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
// 16 bytes global -> shared through L2 only (cp.async.cg); src_bytes 0 writes 16 zero bytes and reads
// nothing. Completion is tracked per thread in commit groups.
__device__ __forceinline__ void dc_cp16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void dc_cp16_full(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void dc_cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void dc_cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory");
}
__device__ __forceinline__ void dc_bar_consumers() {   // the 16 consumer warps only
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kDcWarps) : "memory");
}
// Byte k of w looked up in this lane's table copy: with lanebyte = 0x10000 | lane * 4, one permute gives
// the address kDcLutAddr | (w.byte_k << 8) | lane * 4.
template <int k>
__device__ __forceinline__ uint32_t dc_pair(uint32_t w, uint32_t lanebyte) {
  return dc_lut(dc_prmt(w, lanebyte, 0x7604u | (k << 4)));
}
// The fp32 partial-sum buffer of a pass lives in the free halves of the table's 256-byte entries.
__device__ __forceinline__ float* dc_red(uint8_t* sm, int idx) {
  return reinterpret_cast<float*>(sm + ((idx >> 5) << 8) + 128 + ((idx & 31) << 2));
}
__device__ __forceinline__ uint32_t dc_word(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// The CTA's share: on a load axis where A tile a spans [4a, 4a + 4) and NF4 tile k sits at 4 na + k,
// CTA c takes the tiles whose start lies in [c L / G, (c + 1) L / G), L = 4 na + nt.
struct DcShare { int a0, na, t0, nt; };
__device__ __forceinline__ DcShare dc_share(int cta, int G, int nt_all, int na_all) {
  const int64_t L = static_cast<int64_t>(kDcALoad) * na_all + nt_all;
  const int64_t lo = static_cast<int64_t>(cta) * L / G, hi = static_cast<int64_t>(cta + 1) * L / G;
  const int64_t abase = static_cast<int64_t>(kDcALoad) * na_all;
  auto clamp = [](int64_t v, int64_t hi_) { return static_cast<int>(v < 0 ? 0 : v > hi_ ? hi_ : v); };
  DcShare s;
  s.a0 = clamp((lo + kDcALoad - 1) / kDcALoad, na_all);
  s.na = clamp((hi + kDcALoad - 1) / kDcALoad, na_all) - s.a0;
  s.t0 = clamp(lo - abase, nt_all);
  s.nt = clamp(hi - abase, nt_all) - s.t0;
  return s;
}
// Pass q of the CTA: one A tile per pass first, then NF4 passes of near-equal size (up to PT tiles):
// nb = nt / npn tiles each, the first ne = nt % npn passes one more.
struct DcPass { bool isA; int cnt, first; };
__device__ __forceinline__ DcPass dc_pass(int npa, int nb, int ne, int q) {
  DcPass r;
  if (q < npa) {
    r.isA = true;
    r.first = q;
    r.cnt = 1;
  } else {
    const int k = q - npa;
    r.isA = false;
    r.cnt = nb + (k < ne ? 1 : 0);
    r.first = k * nb + min(k, ne);
  }
  return r;
}
// Position in the CTA's flat stage sequence, advanced one stage at a time (no divisions per stage).
struct DcCursor {
  int i, q, st;
  DcPass ps;
  __device__ __forceinline__ void init(int npa, int nb, int ne) {
    i = 0; q = 0; st = 0;
    ps = dc_pass(npa, nb, ne, 0);
  }
  __device__ __forceinline__ void next(int spp, int npa, int nb, int ne) {
    ++i;
    if (++st == spp) {
      st = 0;
      ++q;
      ps = dc_pass(npa, nb, ne, q);
    }
  }
};

// Registers of one stage for one lane: code words (NF4: tile q's rows g and g + 8 in c[q]; A: 32 bytes
// of row g in c[0], c[1] and of row g + 8 in c[2], c[3]) and X words (token g in x[0], x[1]; token
// g + 8 in x[2], x[3]).
template <int TT> struct DcRegs {
  uint4 c[4];
  uint4 x[kDcBpw][TT / 4];
};
// The A fragments of one 64-element block when the operand is bf16 already (A or B rows): MMA step s
// takes words 2 s and 2 s + 1 of the lane's 16 elements in rows g (c[0], c[1]) and g + 8 (c[2], c[3]).
__device__ __forceinline__ void dc_frag_bf16(const uint4 (&c)[4], uint32_t (&a)[16]) {
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    a[4 * s] = dc_word(c[s >> 1], 2 * (s & 1));
    a[4 * s + 1] = dc_word(c[2 + (s >> 1)], 2 * (s & 1));
    a[4 * s + 2] = dc_word(c[s >> 1], 2 * (s & 1) + 1);
    a[4 * s + 3] = dc_word(c[2 + (s >> 1)], 2 * (s & 1) + 1);
  }
}
// One 64-element block: d (rows g, g + 8 x tokens 2 j, 2 j + 1; + 8 for the second token half) +=
// A fragments x the lane's X words; MMA step s uses elements 16 j + 4 s .. + 3 of both operands.
template <int TT>
__device__ __forceinline__ void dc_block_mma(float (&d)[TT == 16 ? 8 : 4], const uint32_t (&a)[16],
                                             const uint4 (&x)[TT / 4]) {
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const uint4& xv = x[s >> 1];
    dc_mma(d[0], d[1], d[2], d[3], a[4 * s], a[4 * s + 1], a[4 * s + 2], a[4 * s + 3], dc_word(xv, 2 * (s & 1)),
           dc_word(xv, 2 * (s & 1) + 1));
    if constexpr (TT == 16) {
      const uint4& xw = x[2 + (s >> 1)];
      dc_mma(d[4], d[5], d[6], d[7], a[4 * s], a[4 * s + 1], a[4 * s + 2], a[4 * s + 3], dc_word(xw, 2 * (s & 1)),
             dc_word(xw, 2 * (s & 1) + 1));
    }
  }
}

// The same contraction as dc_block_mma with the four MMA steps in two chains (steps 0, 2 into d0 and 1, 3
// into d1), so two MMA latencies are in flight instead of one; the caller adds d0 + d1.
template <int TT>
__device__ __forceinline__ void dc_block_mma2(float (&d0)[TT == 16 ? 8 : 4], float (&d1)[TT == 16 ? 8 : 4],
                                              const uint32_t (&a)[16], const uint4 (&x)[TT / 4]) {
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    float (&d)[TT == 16 ? 8 : 4] = (s & 1) ? d1 : d0;
    const uint4& xv = x[s >> 1];
    dc_mma(d[0], d[1], d[2], d[3], a[4 * s], a[4 * s + 1], a[4 * s + 2], a[4 * s + 3], dc_word(xv, 2 * (s & 1)),
           dc_word(xv, 2 * (s & 1) + 1));
    if constexpr (TT == 16) {
      const uint4& xw = x[2 + (s >> 1)];
      dc_mma(d[4], d[5], d[6], d[7], a[4 * s], a[4 * s + 1], a[4 * s + 2], a[4 * s + 3], dc_word(xw, 2 * (s & 1)),
             dc_word(xw, 2 * (s & 1) + 1));
    }
  }
}

template <int TT>
__global__ void __launch_bounds__(kDcThreads, 1) nf4_decode_kernel(const DecParams p, const CodebookArg cb) {
  constexpr int PT = TT == 16 ? 2 : kDcMaxTiles;      // tiles per pass (4 spill at 16 tokens: slower)
  constexpr int NACC = TT == 16 ? 8 : 4;
  extern __shared__ __align__(1024) uint8_t dc_smem[];
  uint8_t* dsm = dc_smem;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  uint64_t* cready = reinterpret_cast<uint64_t*>(dsm + kDcOffBar);
  uint64_t* cfree = cready + kDcCRing;
  uint64_t* suready = cfree + kDcCRing;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(suready + 1);

  const DcShare sh = dc_share(cta, G, p.tiles, p.atiles);
  const int npa = sh.na;
  const int npn = p.u_only ? 0 : (sh.nt + PT - 1) / PT;
  const int spp = (p.nkb + kDcStageBlocks - 1) / kDcStageBlocks;      // stages per pass
  const int nmain = (npa + npn) * spp;
  const int pnb = npn ? sh.nt / npn : 0, pne = npn ? sh.nt % npn : 0;
  const int nfirst = npa * spp;                                        // stages before the first NF4 one

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDcCRing; ++s) {
      mbar_init(&cready[s], 1);
      mbar_init(&cfree[s], kDcWarps);
    }
    mbar_init(suready, 1);
    *abort_flag = smem_u32(dsm) > static_cast<uint32_t>(kDcMaxBase) ? 1 : 0;   // the layout needs a low base
    fence_barrier_init();
  }
  __syncthreads();
  if (*abort_flag) {
    if (threadIdx.x == 0) raise_status(kStatusTimeout);
    return;
  }
  // shared address of ring slot s
  auto slot_addr = [&](int s) -> uint32_t {
    return s == 0 ? smem_u32(dsm) + kDcOffSlot0 : kDcHighAddr + static_cast<uint32_t>(s - 1) * kDcSlotBytes;
  };

  if (warp >= kDcWarps && warp < kDcWarps + kDcScaleWarps) {
    // ============== block constants of NF4 stages k = sw, sw + 2, ... (sw: this constants warp) ==============
    const int sw = warp - kDcWarps;
    if (nmain == 0) return;
    const int nnf = nmain - nfirst;
    if (nnf == 0) return;
    const float mu = __ldg(p.mu);
    // Rows lane and lane + 32 of the pass: the raw E4M3 bytes and group scales of NF4 stage k.
    struct Raw { uint32_t ew[2][4]; float sa[2], sz[2]; };
    auto fetch = [&](int k, Raw& f) {
      if (k >= nnf) return;
      const int i = nfirst + k;
      const DcPass ps = dc_pass(npa, pnb, pne, i / spp);
      const int blk0 = (i % spp) * kDcStageBlocks, nbh = min(kDcStageBlocks, p.nkb - blk0);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int rho = lane + 32 * h;
        const int row = (sh.t0 + ps.first) * 16 + rho;
        if (rho < ps.cnt * 16 && row < p.N) {
          const int64_t e0 = static_cast<int64_t>(row) * p.nkb + blk0;
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
    // cbuf[block][tile][g] = (c1_hat of row g, of row g + 8) of the tile: what lane (g, j) of the consumer
    // warp that takes the block multiplies its MMA results by
    auto decode = [&](int k, const Raw& r) {
      const int i = nfirst + k;
      const DcPass ps = dc_pass(npa, pnb, pne, i / spp);
      const int blk0 = (i % spp) * kDcStageBlocks, nbh = min(kDcStageBlocks, p.nkb - blk0);
      float* cbuf = reinterpret_cast<float*>(dsm + kDcOffCbuf + (k % kDcCRing) * kDcCbufBytes);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int rho = lane + 32 * h;
        const int row = (sh.t0 + ps.first) * 16 + rho;
        if (rho < ps.cnt * 16) {
          const int64_t e0 = static_cast<int64_t>(row) * p.nkb + blk0;
          const int bsplit = static_cast<int>(256 - (e0 & 255));   // blocks below it take the first scale
          const bool valid = row < p.N;
          float* dst = cbuf + ((rho >> 4) * 8 + (rho & 7)) * 2 + ((rho >> 3) & 1);
#pragma unroll
          for (int b = 0; b < 16; b += 2) {               // two E4M3 values per conversion (exact in fp16)
            const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
                static_cast<__nv_fp8x2_storage_t>(r.ew[h][b >> 2] >> (8 * (b & 3))), __NV_E4M3);
            const float2 dv = __half22float2(__half2(hr));
            dst[b * (kDcMaxTiles * 16)] =
                valid && b < nbh ? __fmaf_rn(dv.x, b < bsplit ? r.sa[h] : r.sz[h], mu) : 0.0f;
            dst[(b + 1) * (kDcMaxTiles * 16)] =
                valid && b + 1 < nbh ? __fmaf_rn(dv.y, b + 1 < bsplit ? r.sa[h] : r.sz[h], mu) : 0.0f;
          }
        }
      }
    };
    // Fetch and decode in sequence (one copy of the code; the two warps between them stay ahead of the
    // consumers by up to kDcCRing stages, which covers the load latency).
    bool go = true;
    for (int k = sw; k < nnf && go; k += kDcScaleWarps) {
      Raw r;
      fetch(k, r);
      // its buffer last held NF4 stage k - R: wait until every consumer warp has read it
      if (k >= kDcCRing && lane == 0 &&
          !mbar_wait(&cfree[k % kDcCRing], static_cast<uint32_t>(((k / kDcCRing) - 1) & 1)))
        *abort_flag = 1;
      __syncwarp();
      if (*abort_flag) {
        go = false;
        break;
      }
      decode(k, r);
      __syncwarp();
      if (lane == 0) mbar_arrive(&cready[k % kDcCRing]);
    }
    return;
  }

  if (warp == kDcWarps + kDcScaleWarps) {
    // ==================== gather sU (every A tile's tag) into shared memory ====================
    if (p.u_only) return;
    bool ok = true;
    for (int a = 0; a < p.atiles && ok; ++a)
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
  const uint32_t lanebyte = 0x10000u | (4u * lane);
  const uint32_t sb = smem_u32(dsm);
  uint8_t* lut = dsm + (kDcLutAddr - sb);            // generic pointer to the table
  const int T = p.T;
  if (nmain == 0) return;                           // u_only and no A tile here: nothing to do
  // the lookup table: entry e = (level[e >> 4], level[e & 15]) as a bf16 pair, one copy per lane
  for (int i = threadIdx.x; i < 256 * 32; i += 32 * kDcWarps) {
    const int e = i >> 5;
    reinterpret_cast<uint32_t*>(lut)[e * 64 + (i & 31)] = pack_bf16x2(cb.levels[e >> 4], cb.levels[e & 15]);
  }
  dc_bar_consumers();

  float* base = p.base_ws + static_cast<int64_t>(sh.t0) * 16 * T;   // [tile][16][T]
  // Stage c's bytes into slot c.i % R, one commit group per stage (empty past the end); this warp's share:
  // NF4 rows 4 w .. 4 w + 3 of the pass (512 B each, piece pc of row rho at rho * 512 + (pc ^ (rho & 7)) * 16),
  // or A row w (2 KB, piece pc at w * 2048 + (pc ^ (w & 7)) * 16). Pieces outside the matrix are zero-filled
  // without a read.
  auto issue = [&](const DcCursor& c, auto nf4_only) {
    if (c.i < nmain) {
      const uint32_t slot = slot_addr(c.i % kDcRing);
      if (!decltype(nf4_only)::value && c.ps.isA) {
#pragma unroll
        for (int ra = 0; ra < kDcARowsPw; ++ra) {
          const int rho = kDcARowsPw * w + ra;
          const int row = (sh.a0 + c.ps.first) * 16 + rho;
          const int64_t e0 = static_cast<int64_t>(row) * p.K + c.st * 1024;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int pc = lane + 32 * m;
            const bool ok = row < p.r && c.st * 1024 + 8 * pc < p.K;
            dc_cp16(slot + rho * 2048 + ((pc ^ (rho & 7)) << 4), ok ? p.A + e0 + 8 * pc : p.A, ok ? 16u : 0u);
          }
        }
      } else {
        const int b0 = c.st * 512 + 16 * lane;
        const int rho0 = kDcRowsPw * w;
        const int row0 = (sh.t0 + c.ps.first) * 16 + rho0;
        if (rho0 + kDcRowsPw <= c.ps.cnt * 16 && row0 + kDcRowsPw <= p.N && c.st * 512 + 512 <= p.K / 2) {
          // the common case: whole row segments
          const uint8_t* src = p.codes + static_cast<int64_t>(row0) * (p.K / 2) + b0;
#pragma unroll
          for (int m = 0; m < kDcRowsPw; ++m)
            dc_cp16_full(slot + (rho0 + m) * 512 + ((lane ^ ((rho0 + m) & 7)) << 4), src + m * (p.K / 2));
        } else {
#pragma unroll
          for (int m = 0; m < kDcRowsPw; ++m) {
            const int rho = rho0 + m;
            const int row = row0 + m;
            const bool ok = rho < c.ps.cnt * 16 && row < p.N && b0 < p.K / 2;
            const uint8_t* src = ok ? p.codes + static_cast<int64_t>(row) * (p.K / 2) + b0 : p.codes;
            dc_cp16(slot + rho * 512 + ((lane ^ (rho & 7)) << 4), src, ok ? 16u : 0u);
          }
        }
      }
    }
    dc_cp_commit();
  };
  // stage c's X words of blocks kDcBpw w + b (zero where there are none)
  auto loadx = [&](const DcCursor& c, DcRegs<TT>& R) {
#pragma unroll
    for (int b = 0; b < kDcBpw; ++b) {
#pragma unroll
      for (int q = 0; q < TT / 4; ++q) R.x[b][q] = make_uint4(0, 0, 0, 0);
      const int blk = c.st * kDcStageBlocks + kDcBpw * w + b;
      if (c.i >= nmain || blk >= p.nkb) continue;
      const __nv_bfloat16* xp = p.X + blk * 64 + 16 * j;
      if (g < T) {
        R.x[b][0] = __ldg(reinterpret_cast<const uint4*>(xp + static_cast<int64_t>(g) * p.K));
        R.x[b][1] = __ldg(reinterpret_cast<const uint4*>(xp + static_cast<int64_t>(g) * p.K + 8));
      }
      if constexpr (TT == 16) {
        if (g + 8 < T) {
          R.x[b][2] = __ldg(reinterpret_cast<const uint4*>(xp + static_cast<int64_t>(g + 8) * p.K));
          R.x[b][3] = __ldg(reinterpret_cast<const uint4*>(xp + static_cast<int64_t>(g + 8) * p.K + 8));
        }
      }
    }
  };

  float acc[PT][NACC];
  bool live = true;
  int knf = 0;                                      // NF4 stages computed so far (the constants ring index)
  auto stage = [&](const DcCursor& c, DcRegs<TT>& R, auto is_a) {
    const DcPass& ps = c.ps;
    if (c.st == 0) {
#pragma unroll
      for (int q = 0; q < PT; ++q)
#pragma unroll
        for (int e = 0; e < NACC; ++e) acc[q][e] = 0.0f;
    }
    const uint32_t slot = slot_addr(c.i % kDcRing);
    if (live && *abort_flag) live = false;
    if constexpr (decltype(is_a)::value) {
#pragma unroll
      for (int b = 0; b < kDcBpw; ++b) {
        const int bw = kDcBpw * w + b;              // block of the stage
        if (!live || c.st * kDcStageBlocks + bw >= p.nkb) continue;
        // A rows are bf16 already: row g in c[0..1], g + 8 in c[2..3]
        const uint32_t r0 = slot + g * 2048, r1 = slot + (g + 8) * 2048;
        R.c[0] = dc_ld128(r0 + (((8 * bw + 2 * j) ^ g) << 4));
        R.c[1] = dc_ld128(r0 + (((8 * bw + 2 * j + 1) ^ g) << 4));
        R.c[2] = dc_ld128(r1 + (((8 * bw + 2 * j) ^ g) << 4));
        R.c[3] = dc_ld128(r1 + (((8 * bw + 2 * j + 1) ^ g) << 4));
        uint32_t a[16];
        dc_frag_bf16(R.c, a);
        dc_block_mma<TT>(acc[0], a, R.x[b]);
      }
    } else {
      const int k = knf++, cslot = k % kDcCRing;
      if (live && !mbar_wait(&cready[cslot], static_cast<uint32_t>((k / kDcCRing) & 1))) live = false;
      if (!live) *abort_flag = 1;
      float2 cs[kDcBpw][PT];
#pragma unroll
      for (int b = 0; b < kDcBpw; ++b) {
        const uint32_t cbase = kDcOffCbuf + cslot * kDcCbufBytes + ((kDcBpw * w + b) * kDcMaxTiles * 8 + g) * 8;
#pragma unroll
        for (int q = 0; q < PT; ++q) cs[b][q] = dc_ldf2(sb + cbase + q * 64);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&cfree[cslot]);
      // Tiles outer, blocks inner: the kDcBpw blocks of a tile are independent chains the scheduler can
      // interleave. Blocks past K need no test: their constants are 0 and their X words 0, and the stale codes
      // of their slot bytes only ever look up finite levels.
      if (live) {
#pragma unroll
        for (int q = 0; q < PT; ++q) {
          if (q >= ps.cnt) break;
#pragma unroll
          for (int b = 0; b < kDcBpw; ++b) {
            const int bw = kDcBpw * w + b;
            // this lane's 8 bytes of block bw in rows g and g + 8 of tile q: piece 2 bw + j / 2 (swizzled), half j & 1
            const uint32_t pof = ((((2 * bw + (j >> 1)) ^ g) & 31) << 4) + 8 * (j & 1);
            const uint2 c0 = dc_ld64(slot + (q * 16 + g) * 512 + pof);
            const uint2 c1 = dc_ld64(slot + (q * 16 + g + 8) * 512 + pof);
            // A fragments: a[4 s + 0..3] = (row g, elements 4 s, 4 s + 1), (row g + 8, same),
            // (row g, 4 s + 2, 4 s + 3), (row g + 8, same) of this lane's 16; byte 2 s and 2 s + 1 of 8
            uint32_t a[16];
            a[0] = dc_pair<0>(c0.x, lanebyte);  a[1] = dc_pair<0>(c1.x, lanebyte);
            a[2] = dc_pair<1>(c0.x, lanebyte);  a[3] = dc_pair<1>(c1.x, lanebyte);
            a[4] = dc_pair<2>(c0.x, lanebyte);  a[5] = dc_pair<2>(c1.x, lanebyte);
            a[6] = dc_pair<3>(c0.x, lanebyte);  a[7] = dc_pair<3>(c1.x, lanebyte);
            a[8] = dc_pair<0>(c0.y, lanebyte);  a[9] = dc_pair<0>(c1.y, lanebyte);
            a[10] = dc_pair<1>(c0.y, lanebyte); a[11] = dc_pair<1>(c1.y, lanebyte);
            a[12] = dc_pair<2>(c0.y, lanebyte); a[13] = dc_pair<2>(c1.y, lanebyte);
            a[14] = dc_pair<3>(c0.y, lanebyte); a[15] = dc_pair<3>(c1.y, lanebyte);
            float d0[NACC], d1[NACC];
#pragma unroll
            for (int e = 0; e < NACC; ++e) d0[e] = d1[e] = 0.0f;
            dc_block_mma2<TT>(d0, d1, a, R.x[b]);
#pragma unroll
            for (int e = 0; e < NACC; ++e)
              acc[q][e] = __fmaf_rn((e & 2) ? cs[b][q].y : cs[b][q].x, d0[e] + d1[e], acc[q][e]);
          }
        }
      }
    }
    if (c.st != spp - 1) return;
    // ---- end of pass: the 16 warps' partial sums, added in warp order ----
    const int rows = ps.cnt * 16, prow = 16 * PT;
#pragma unroll
    for (int q = 0; q < PT; ++q) {
      if (q >= ps.cnt) break;
#pragma unroll
      for (int e = 0; e < NACC; ++e) {
        // accumulator e = 4 th + 2 hh + u: row 16 q + g + 8 hh, token 2 j + u + 8 th
        const int row = 16 * q + g + 8 * ((e >> 1) & 1), tok = 2 * j + (e & 1) + 8 * (e >> 2);
        if (tok < T) *dc_red(lut, (w * prow + row) * T + tok) = acc[q][e];
      }
    }
    dc_bar_consumers();
    for (int o = threadIdx.x; o < rows * T; o += 32 * kDcWarps) {
      const int ro = o / T, t = o % T;
      float sum = 0.0f;
#pragma unroll
      for (int ww = 0; ww < kDcWarps; ++ww) sum += *dc_red(lut, (ww * prow + ro) * T + t);
      if constexpr (decltype(is_a)::value) {        // sU = bf16(s * X A^T): column = A row
        const int arow = (sh.a0 + ps.first) * 16 + ro;
        if (arow < p.r) p.U[static_cast<int64_t>(t) * p.r + arow] = __float2bfloat16_rn(p.s * sum);
      } else {
        base[(static_cast<int64_t>(ps.first) * 16 + ro) * T + t] = sum;
      }
    }
    dc_bar_consumers();
    if (decltype(is_a)::value && threadIdx.x == 0) {   // this A tile's piece of sU is complete and visible
      __threadfence();
      st_release_u64(p.tags + sh.a0 + ps.first, p.seq);
    }
  };

  // The flat stage sequence, A stages first, then NF4 stages (two loops, each with only its own code). At
  // stage i: load stage i's X words (their latency overlaps the waits), wait for this thread's copies of
  // stage i, then a barrier of the consumer warps (every warp's copies of stage i landed; every warp is done
  // with stage i - 1, whose slot the copies of stage i + R - 1 reuse), issue those copies, compute.
  using kA = std::integral_constant<bool, true>;      // stage(): an A stage
  using kNF4 = std::integral_constant<bool, false>;   // stage(): an NF4 stage
  using kAnyStage = std::integral_constant<bool, false>;   // issue(): A or NF4
  using kNF4Only = std::integral_constant<bool, true>;     // issue(): NF4 only
  DcCursor cc, ci;
  cc.init(npa, pnb, pne);
  ci.init(npa, pnb, pne);
#pragma unroll
  for (int i = 0; i < kDcRing - 1; ++i) {
    issue(ci, kAnyStage{});
    ci.next(spp, npa, pnb, pne);
  }
  DcRegs<TT> rg;
  while (cc.i < nfirst) {
    loadx(cc, rg);
    dc_cp_wait<kDcRing - 2>();
    dc_bar_consumers();
    issue(ci, kAnyStage{});
    ci.next(spp, npa, pnb, pne);
    stage(cc, rg, kA{});
    cc.next(spp, npa, pnb, pne);
  }
  while (cc.i < nmain) {                            // every stage issued from here on is an NF4 stage
    loadx(cc, rg);
    dc_cp_wait<kDcRing - 2>();
    dc_bar_consumers();
    issue(ci, kNF4Only{});
    ci.next(spp, npa, pnb, pne);
    stage(cc, rg, kNF4{});
    cc.next(spp, npa, pnb, pne);
  }
  dc_cp_wait<0>();
  if (p.u_only) {
    if (!live) raise_status(kStatusTimeout);
    return;
  }
  // ---- adapter term and output: Y = bf16(base + sU B^T), tile by tile across the warps ----
  bool su_ok = live && mbar_wait(suready, 0) && !*abort_flag;
  if (!su_ok) *abort_flag = 1;
  for (int tl = w; su_ok && tl < sh.nt; tl += kDcWarps) {
    float d[NACC];
#pragma unroll
    for (int c = 0; c < NACC; ++c) d[c] = 0.0f;
    for (int rc = 0; rc < p.RP / 64; ++rc) {
      DcRegs<TT> R;
      const int e0 = rc * 64 + 16 * j;              // this lane's 16 adapter columns of the chunk
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int n = (sh.t0 + tl) * 16 + g + 8 * h;
        const __nv_bfloat16* bp = p.B + static_cast<int64_t>(n) * p.r + e0;
        R.c[2 * h] = (n < p.N && e0 < p.r) ? __ldg(reinterpret_cast<const uint4*>(bp)) : make_uint4(0, 0, 0, 0);
        R.c[2 * h + 1] =
            (n < p.N && e0 + 8 < p.r) ? __ldg(reinterpret_cast<const uint4*>(bp + 8)) : make_uint4(0, 0, 0, 0);
      }
      const uint32_t su = kDcOffSU + (min(g, T - 1) * p.RP + e0) * 2;
      R.x[0][0] = dc_ld128(sb + su);
      R.x[0][1] = dc_ld128(sb + su + 16);
      if constexpr (TT == 16) {
        const uint32_t su1 = kDcOffSU + (min(g + 8, T - 1) * p.RP + e0) * 2;
        R.x[0][2] = dc_ld128(sb + su1);
        R.x[0][3] = dc_ld128(sb + su1 + 16);
      }
      uint32_t a[16];
      dc_frag_bf16(R.c, a);
      dc_block_mma<TT>(d, a, R.x[0]);
    }
#pragma unroll
    for (int c = 0; c < NACC; ++c) {
      const int rl = g + 8 * ((c >> 1) & 1), tok = 2 * j + (c & 1) + 8 * (c >> 2);
      const int n = (sh.t0 + tl) * 16 + rl;
      if (tok < T && n < p.N)
        p.Y[static_cast<int64_t>(tok) * p.N + n] =
            __float2bfloat16_rn(base[(static_cast<int64_t>(tl) * 16 + rl) * T + tok] + d[c]);
    }
  }
  if (!live || !su_ok) raise_status(kStatusTimeout);
}

}  // namespace qnf4
