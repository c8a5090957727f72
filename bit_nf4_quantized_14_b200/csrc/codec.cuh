// NF4 codec kernels: blockwise quantization with double-quantized constants, and dequantization.
//
// Method (PEFT page, zerotofrontier.app/sft/peft, "Block-wise quantization in one page",
// "NF4, derived from normal quantiles", "Double quantization", "The real way"; QLoRA explainer,
// prism.theerrors.in, "For the curious"):
//   pass 1  per block of 64 consecutive elements: absmax c1, 4-bit codes (two per byte), and per slab
//           of 64 blocks the fp64 balanced-tree sum of its c1 values;
//   pass 1b the mean mu of all c1: the fp64 balanced tree continued over the slab sums, / nb, -> fp32;
//   pass 2  per group of 256 blocks: d = c1 - mu, s2 = max|d| / 448, e = E4M3(d / s2) (round to nearest
//           even, satfinite).
//   dequant c1_hat = fma(decode(e), s2, mu); w_hat = fp32(level[code] * c1_hat) -> bf16 (RNE) or fp32.
//
// Codes: the pages ask for the index of the nearest level. The library's rule is
// code = #{j : w > T_j * a}, T_j the fp32-rounded level midpoints, a > 0 the block absmax, evaluated
// exactly; ties go to the lower index; a block with a = 0 codes as the level of least magnitude (7, the
// exact zero, for NF4). For fp32 w, T_j and a:
//   w > T_j * a  <=>  w > RD(T_j * a)
// where RD is the fp32 product rounded toward -inf (no fp32 value lies strictly between RD(P) and an
// inexact P, subnormals included), so one __fmul_rd and one compare decide a threshold exactly.
//
// Finding the one threshold to test. With t = w / a in [-1, 1], an fma with a magic constant puts the
// integer b = 16 + round(15 * t') (t' = t up to a relative 2^-20 from the approximate reciprocal) into
// the low five mantissa bits; bucket b spans 1/15 in t, less than the smallest gap between two
// thresholds (0.0805), so it holds at most one threshold. A 32-entry table (one entry per lane) gives
// lo(b), the number of thresholds certainly below t, and then code = lo + [w > RD(T_lo * a)] exactly.
// The table is built and checked on the host (every bucket, widened by 2^-18, holds at most one
// threshold); a block whose absmax is below 2^-120 is first scaled by 2^64 so the reciprocal stays finite.
#pragma once

#include <cuda_fp8.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace qnf4 {

struct CodebookArg {       // passed by value: lives in the kernel-parameter constant bank
  float levels[16];
  float thresholds[15];
};
struct BucketArg {         // bucket b -> lo(b), 4 bits each; the code of an all-zero block in every nibble
  uint32_t lo_nibbles[4];
  uint32_t zero_codes;
  uint32_t step_mask;      // bit b = lo(b) - lo(b - 1) (bit 0 = lo(0)): lo(b) = popc(bits 0..b)
};

constexpr int kBlock = 64;          // first-level block (weights per absmax constant)
constexpr int kGroup = 256;         // second-level block (constants per fp32 scale)
constexpr int kGroupElems = kBlock * kGroup;
constexpr int kSlabBlocks = 64;     // pass 1: one warp owns a slab of 64 blocks
constexpr int kSlabElems = kSlabBlocks * kBlock;
constexpr int kStepElems = 512;     // one warp step: 8 blocks, 16 elements per lane
constexpr float kBucketScale = 15.0f;
constexpr float kBucketBias = 12582928.0f;   // 1.5 * 2^23 + 16
constexpr double kBucketWiden = 0x1p-18;     // table margin in units of t

__device__ __forceinline__ float rcp_approx(float x) {   // within 1 ulp, subnormal results kept
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float fmax_nan(float a, float b) {   // NaN-propagating maximum
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

template <typename InT> struct Scalar;
template <> struct Scalar<float> {
  __device__ static float load(const float* p) { return *p; }
};
template <> struct Scalar<__nv_bfloat16> {
  __device__ static float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
};

// One lane's 16 consecutive elements, kept as raw bits so the next step's loads can be in flight
// while the current step computes.
template <typename InT> struct Raw16;
template <> struct Raw16<float> {
  uint4 v[4];
  __device__ void load(const float* p) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = __ldcs(q + k);
  }
  __device__ void widen(float (&x)[16]) const {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[4 * k] = __uint_as_float(v[k].x); x[4 * k + 1] = __uint_as_float(v[k].y);
      x[4 * k + 2] = __uint_as_float(v[k].z); x[4 * k + 3] = __uint_as_float(v[k].w);
    }
  }
};
template <> struct Raw16<__nv_bfloat16> {
  uint4 v[2];
  __device__ void load(const __nv_bfloat16* p) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
    v[0] = __ldcs(q);
    v[1] = __ldcs(q + 1);
  }
  __device__ void widen(float (&x)[16]) const {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t u[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        x[8 * k + 2 * i] = __uint_as_float(u[i] << 16);
        x[8 * k + 2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
      }
    }
  }
};

// Code of one element. tbtab: lane b holds T_lo(b), the one threshold that can lie in bucket b (+inf when
// lo(b) = 15 or the codebook has fewer thresholds); lo(b) = popc(bits 0..b of the step mask). The bucket's
// shuffle and the popcount do not depend on each other.
template <bool kScaled>
__device__ __forceinline__ uint32_t nf4_code(float x, float a, float sc, float r15, float tbtab, uint32_t step_mask) {
  const float xs = kScaled ? x * sc : x;
  const uint32_t zb = __float_as_uint(__fmaf_rn(xs, r15, kBucketBias));   // bucket in the low 5 bits
  const float tl = __shfl_sync(0xffffffffu, tbtab, static_cast<int>(zb));
  const uint32_t lo = __popc(step_mask << (~zb & 31u));
  return lo + ((x > __fmul_rd(tl, a)) ? 1u : 0u);
}
// Codes of 16 elements as 8 bytes, byte i = (code[2i] << 4) | code[2i+1] (even element high nibble).
template <bool kScaled>
__device__ __forceinline__ void nf4_codes16(const float (&x)[16], float a, float sc, float r15, float tbtab,
                                            uint32_t step_mask, uint32_t& w0, uint32_t& w1) {
  w0 = 0;
  w1 = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t hi = nf4_code<kScaled>(x[2 * i], a, sc, r15, tbtab, step_mask);
    const uint32_t lo = nf4_code<kScaled>(x[2 * i + 1], a, sc, r15, tbtab, step_mask);
    const uint32_t b = (hi << 4) | lo;
    if (i < 4) w0 |= b << (8 * i);
    else w1 |= b << (8 * (i - 4));
  }
}

// One step of a warp: lanes 4k..4k+3 hold block k's 64 elements (16 each). Returns the team's absmax
// (NaN if the block holds a NaN); flags a non-finite block in `bad`.
__device__ __forceinline__ float block_codes(const float (&x)[16], float tbtab, uint32_t step_mask, uint32_t zero_codes,
                                             uint32_t& bad, uint32_t& w0, uint32_t& w1) {
  float m = fmax_nan(fmax_nan(fmax_nan(fabsf(x[0]), fabsf(x[1])), fmax_nan(fabsf(x[2]), fabsf(x[3]))),
                     fmax_nan(fmax_nan(fabsf(x[4]), fabsf(x[5])), fmax_nan(fabsf(x[6]), fabsf(x[7]))));
  m = fmax_nan(m, fmax_nan(fmax_nan(fmax_nan(fabsf(x[8]), fabsf(x[9])), fmax_nan(fabsf(x[10]), fabsf(x[11]))),
                           fmax_nan(fmax_nan(fabsf(x[12]), fabsf(x[13])), fmax_nan(fabsf(x[14]), fabsf(x[15])))));
  m = fmax_nan(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = fmax_nan(m, __shfl_xor_sync(0xffffffffu, m, 2));
  const float a = m;
  bad |= (a <= 3.402823466e38f) ? 0u : 1u;        // false for NaN and +inf
  const bool tiny = a < 0x1p-120f;
  const float sc = tiny ? 0x1p64f : 1.0f;
  const float r15 = kBucketScale * rcp_approx(a * sc);
  if (__any_sync(0xffffffffu, tiny)) nf4_codes16<true>(x, a, sc, r15, tbtab, step_mask, w0, w1);
  else nf4_codes16<false>(x, a, sc, r15, tbtab, step_mask, w0, w1);
  if (!(a > 0.0f)) {                                // all-zero block (or NaN): the zero code
    w0 = zero_codes;
    w1 = zero_codes;
  }
  return a;
}

// Pass 1 for fp32 input. Persistent CTAs, two per SM; CTA c owns a contiguous range of whole slabs. One
// producer lane brings each slab into a ring of shared-memory slots with one bulk copy (a ring of 96 KB per CTA keeps
// ~190 KB per SM in flight, what HBM needs to stay busy); consumer warp w takes step w (blocks 8w..8w+7)
// of every slab, writes its codes straight to global memory and its 8 constants to the slot's constant
// buffer, and the last of the eight warps to finish a slab (a shared-memory counter) writes the slab's
// 64 constants and their fp64 balanced-tree sum. A ragged last slab is done by one warp of the last CTA
// with direct loads and bounds on every element. Without double quantization (ssum and ticket null) c1
// is the stored constant array and pass 1 is all.
template <typename InT> struct Q1 {
  static constexpr int kSlabBytes = kSlabElems * static_cast<int>(sizeof(InT));
  static constexpr int kCtasPerSm = 2;
  static constexpr int kSlots = (96 * 1024) / kSlabBytes;
  static constexpr int kOffCb = kSlots * kSlabBytes;                      // [slot][64] fp32 constants
  static constexpr int kOffCnt = kOffCb + kSlots * kSlabBlocks * 4;       // [slot] finished-warp counters
  static constexpr int kOffBar = kOffCnt + kSlots * 4 + 8 - (kSlots * 4) % 8;
  static constexpr int kOffRag = kOffBar + 2 * kSlots * 8;                // full[slot], empty[slot]
  static constexpr int kSmemBytes = kOffRag + kSlabBlocks * 4;            // the ragged slab's constants
};
constexpr int kQ1Consumers = 8;                       // = steps per slab
constexpr int kQ1Threads = 32 * (kQ1Consumers + 1);
static_assert(kQ1Consumers * kStepElems == kSlabElems, "one step per consumer warp");

// One lane's 16 elements of a slab slot: this lane's 64 contiguous bytes are read in
// 16-byte chunks starting at a lane-dependent chunk, so every 128-byte wavefront serves 8 distinct lanes
// (no bank conflicts); the chunks land rotated and the packed codes are rotated back.
template <typename InT> struct SlotRead;
template <> struct SlotRead<float> {
  static __device__ __forceinline__ int rot(int lane) { return (lane >> 1) & 3; }
  static __device__ __forceinline__ void load(const uint8_t* p, int r, float (&x)[16]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = *reinterpret_cast<const uint4*>(p + 16 * ((c + r) & 3));
      x[4 * c] = __uint_as_float(v.x); x[4 * c + 1] = __uint_as_float(v.y);
      x[4 * c + 2] = __uint_as_float(v.z); x[4 * c + 3] = __uint_as_float(v.w);
    }
  }
  static __device__ __forceinline__ uint2 unrotate(uint32_t w0, uint32_t w1, int r) {   // 16-bit pieces
    const uint64_t v = (static_cast<uint64_t>(w1) << 32) | w0;
    const uint64_t o = r ? ((v << (16 * r)) | (v >> (64 - 16 * r))) : v;
    return make_uint2(static_cast<uint32_t>(o), static_cast<uint32_t>(o >> 32));
  }
};
template <typename InT>
__global__ void __launch_bounds__(kQ1Threads, Q1<InT>::kCtasPerSm) nf4_quantize_pass1(
    const InT* __restrict__ w, int64_t n, uint8_t* __restrict__ codes, float* __restrict__ c1,
    double* __restrict__ ssum, int64_t nslabs, CodebookArg cb, BucketArg bk, unsigned* __restrict__ ticket) {
  using L = Q1<InT>;
  extern __shared__ __align__(1024) uint8_t q1_smem[];
  float* cbuf = reinterpret_cast<float*>(q1_smem + L::kOffCb);
  unsigned* cnt = reinterpret_cast<unsigned*>(q1_smem + L::kOffCnt);
  uint64_t* full = reinterpret_cast<uint64_t*>(q1_smem + L::kOffBar);
  uint64_t* empty = full + L::kSlots;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (ticket && blockIdx.x == 0 && threadIdx.x == 0) *ticket = 0u;    // arrival counter of the mean pass
  const int64_t nb = (n + kBlock - 1) / kBlock;
  const int64_t nfull = n / kSlabElems;
  const int64_t s0 = nfull * blockIdx.x / gridDim.x, s1 = nfull * (blockIdx.x + 1) / gridDim.x;
  const int nmine = static_cast<int>(s1 - s0);
  if (threadIdx.x == 0) {
    for (int k = 0; k < L::kSlots; ++k) {
      mbar_init(&full[k], 1);
      mbar_init(&empty[k], kQ1Consumers + 1);     // the eight readers and the slab's finisher
      cnt[k] = 0u;
    }
    fence_barrier_init();
  }
  __syncthreads();

  // constants out, and the slab's 64-leaf fp64 tree (leaf pairs per lane, then a butterfly of subtrees)
  auto finish_slab = [&](int64_t s, const float* cbs) {
    const float l0 = cbs[2 * lane], l1 = cbs[2 * lane + 1];
    const int64_t gb = s * kSlabBlocks + 2 * lane;
    if (gb + 1 < nb) *reinterpret_cast<float2*>(c1 + gb) = make_float2(l0, l1);
    else if (gb < nb) c1[gb] = l0;
    double t = static_cast<double>(l0) + static_cast<double>(l1);
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const double r = __shfl_down_sync(0xffffffffu, t, off);
      if ((lane & (2 * off - 1)) == 0) t = t + r;    // left subtree + right subtree
    }
    if (lane == 0 && ssum) ssum[s] = t;
  };

  if (warp == kQ1Consumers) {                     // producer
    if (lane == 0) {
      for (int i = 0; i < nmine; ++i) {
        const int k = i % L::kSlots;
        if (i >= L::kSlots && !mbar_wait(&empty[k], ((i / L::kSlots) - 1) & 1)) break;
        mbar_arrive_expect_tx(&full[k], L::kSlabBytes);
        bulk_load(q1_smem + k * L::kSlabBytes, w + (s0 + i) * kSlabElems, L::kSlabBytes, &full[k]);
      }
    }
  } else {
    const uint32_t lo_lane = (bk.lo_nibbles[lane >> 3] >> (4 * (lane & 7))) & 0xFu;
    const float tbtab = (lo_lane < 15) ? cb.thresholds[lo_lane] : __int_as_float(0x7F800000);
    const int rot = SlotRead<InT>::rot(lane);
    uint32_t bad = 0;
    for (int i = 0; i < nmine; ++i) {
      const int k = i % L::kSlots;
      if (!mbar_wait(&full[k], (i / L::kSlots) & 1)) break;
      float x[16];
      SlotRead<InT>::load(q1_smem + k * L::kSlabBytes + (warp * kStepElems + 16 * lane) * sizeof(InT), rot, x);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[k]);
      uint32_t w0, w1;
      const float a = block_codes(x, tbtab, bk.step_mask, bk.zero_codes, bad, w0, w1);
      const int64_t s = s0 + i;
      *reinterpret_cast<uint2*>(codes + ((s * kSlabElems + warp * kStepElems + 16 * lane) >> 1)) =
          SlotRead<InT>::unrotate(w0, w1, rot);
      float* cbs = cbuf + k * kSlabBlocks;
      if ((lane & 3) == 0) cbs[warp * 8 + (lane >> 2)] = a;
      __threadfence_block();
      __syncwarp();
      unsigned last = 0;
      if (lane == 0) last = (atomicAdd(&cnt[k], 1u) == kQ1Consumers - 1) ? 1u : 0u;
      if (__shfl_sync(0xffffffffu, last, 0)) {    // the last warp of this slab: publish it
        __threadfence_block();
        finish_slab(s, cbs);
        __syncwarp();
        if (lane == 0) {
          cnt[k] = 0u;
          mbar_arrive(&empty[k]);
        }
      }
    }
    if (nfull < nslabs && blockIdx.x == gridDim.x - 1 && warp == 0) {   // the ragged last slab
      const int64_t s = nfull;
      float* cbs = reinterpret_cast<float*>(q1_smem + L::kOffRag);
      for (int it = 0; it < kSlabElems / kStepElems; ++it) {
        const int64_t e0 = s * kSlabElems + it * kStepElems + 16 * lane;
        float x[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] = (e0 + e < n) ? Scalar<InT>::load(w + e0 + e) : 0.0f;
        uint32_t w0, w1;
        const float a = block_codes(x, tbtab, bk.step_mask, bk.zero_codes, bad, w0, w1);
        for (int b = 0; b < 8; ++b) {
          const int64_t idx = e0 + 2 * b;
          if (idx < n) {
            uint32_t byte = ((b < 4 ? w0 : w1) >> (8 * (b & 3))) & 0xFFu;
            if (idx + 1 >= n) byte &= 0xF0u;                     // odd n: the final low nibble is 0
            codes[idx >> 1] = static_cast<uint8_t>(byte);
          }
        }
        if ((lane & 3) == 0) cbs[it * 8 + (lane >> 2)] = a;
      }
      __syncwarp();
      finish_slab(s, cbs);
    }
    if (bad) raise_status(kStatusNonfinite);
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Pass 1 for bf16 input. Each warp owns slabs gw, gw + nw, ... and walks them as a flat sequence of
// 8-block steps straight from global memory, loading step i + 1 while step i computes (three CTAs of eight
// warps per SM: half the bytes per element of fp32 input leave the issue rate, not HBM, as the limit, and
// more warps per SM serve it better than a shared-memory ring). Per slab it writes the 64 block constants
// and their fp64 balanced-tree sum; a ragged last slab is done by one warp with bounds on every element.
constexpr int kQuantThreads = 256;
constexpr int kQuantMinBlocks = 3;
template <typename InT>
__global__ void __launch_bounds__(kQuantThreads, kQuantMinBlocks) nf4_quantize_pass1_direct(
    const InT* __restrict__ w, int64_t n, uint8_t* __restrict__ codes, float* __restrict__ c1,
    double* __restrict__ ssum, int64_t nslabs, CodebookArg cb, BucketArg bk, unsigned* __restrict__ ticket) {
  __shared__ float c1buf[kQuantThreads / 32][kSlabBlocks];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (ticket && blockIdx.x == 0 && threadIdx.x == 0) *ticket = 0u;    // arrival counter of the mean pass
  const uint32_t lo_lane = (bk.lo_nibbles[lane >> 3] >> (4 * (lane & 7))) & 0xFu;
  const float tbtab = (lo_lane < 15) ? cb.thresholds[lo_lane] : __int_as_float(0x7F800000);
  const int64_t nb = (n + kBlock - 1) / kBlock;
  const int64_t nfull = n / kSlabElems;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * (kQuantThreads / 32) + warp;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (kQuantThreads / 32);
  float* cb_w = c1buf[warp];
  uint32_t bad = 0;

  auto finish_slab = [&](int64_t s) {      // constants out, and the slab's 64-leaf fp64 tree
    __syncwarp();
    const float l0 = cb_w[2 * lane], l1 = cb_w[2 * lane + 1];
    const int64_t gb = s * kSlabBlocks + 2 * lane;
    if (gb + 1 < nb) *reinterpret_cast<float2*>(c1 + gb) = make_float2(l0, l1);
    else if (gb < nb) c1[gb] = l0;
    double t = static_cast<double>(l0) + static_cast<double>(l1);
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const double r = __shfl_down_sync(0xffffffffu, t, off);
      if ((lane & (2 * off - 1)) == 0) t = t + r;    // left subtree + right subtree
    }
    if (lane == 0 && ssum) ssum[s] = t;
    __syncwarp();
  };

  const int64_t my_slabs = (gw < nfull) ? (nfull - 1 - gw) / nw + 1 : 0;
  const int64_t steps = my_slabs * (kSlabElems / kStepElems);
  Raw16<InT> cur, nxt;
  if (steps > 0) nxt.load(w + gw * kSlabElems + 16 * lane);
  for (int64_t i = 0; i < steps; ++i) {
    const int64_t s = gw + (i >> 3) * nw;
    const int it = static_cast<int>(i & 7);
    cur = nxt;
    if (i + 1 < steps)
      nxt.load(w + (gw + ((i + 1) >> 3) * nw) * kSlabElems + ((i + 1) & 7) * kStepElems + 16 * lane);
    float x[16];
    cur.widen(x);
    const int64_t e0 = s * kSlabElems + it * kStepElems + 16 * lane;
    uint32_t w0, w1;
    const float a = block_codes(x, tbtab, bk.step_mask, bk.zero_codes, bad, w0, w1);
    *reinterpret_cast<uint2*>(codes + (e0 >> 1)) = make_uint2(w0, w1);
    if ((lane & 3) == 0) cb_w[it * 8 + (lane >> 2)] = a;
    if (it == 7) finish_slab(s);
  }
  if (nfull < nslabs && gw == nfull % nw) {          // the ragged last slab
    const int64_t s = nfull;
    for (int it = 0; it < kSlabElems / kStepElems; ++it) {
      const int64_t e0 = s * kSlabElems + it * kStepElems + 16 * lane;
      float x[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) x[e] = (e0 + e < n) ? Scalar<InT>::load(w + e0 + e) : 0.0f;
      uint32_t w0, w1;
      const float a = block_codes(x, tbtab, bk.step_mask, bk.zero_codes, bad, w0, w1);
      for (int b = 0; b < 8; ++b) {
        const int64_t idx = e0 + 2 * b;
        if (idx < n) {
          uint32_t byte = ((b < 4 ? w0 : w1) >> (8 * (b & 3))) & 0xFFu;
          if (idx + 1 >= n) byte &= 0xF0u;                     // odd n: the final low nibble is 0
          codes[idx >> 1] = static_cast<uint8_t>(byte);
        }
      }
      if ((lane & 3) == 0) cb_w[it * 8 + (lane >> 2)] = a;
    }
    finish_slab(s);
  }
  if (bad) raise_status(kStatusNonfinite);
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Pass 1b. The fp64 balanced tree over the slab sums zero-padded to P = 2^ceil(log2 ns) leaves (the
// same value as the tree over all block constants padded with zeros: zero subtrees add exactly 0).
// CTA q reduces the aligned subtree of P / gridDim.x <= 2048 leaves; the last CTA to arrive combines
// the gridDim.x subtree sums (a power of two) and writes mu = fp32(S / nb).
constexpr int kTreeThreads = 256;
constexpr int kTreeLeavesPerCta = 8 * kTreeThreads;
__device__ __forceinline__ double cta_tree(double v, int nvals, double* sh) {
  sh[threadIdx.x] = v;
  __syncthreads();
  for (int len = nvals / 2; len >= 1; len >>= 1) {
    double x = 0.0;
    if (static_cast<int>(threadIdx.x) < len) x = sh[2 * threadIdx.x] + sh[2 * threadIdx.x + 1];
    __syncthreads();
    if (static_cast<int>(threadIdx.x) < len) sh[threadIdx.x] = x;
    __syncthreads();
  }
  return sh[0];
}
__global__ void __launch_bounds__(kTreeThreads) nf4_mean(const double* __restrict__ ssum, int64_t ns,
                                                        int64_t nb, double* __restrict__ partial,
                                                        unsigned* __restrict__ ticket, float* __restrict__ mu_out) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ double sh[kTreeThreads];
  __shared__ int is_last;
  int64_t P = 1;
  while (P < ns) P <<= 1;
  const int64_t L = P / gridDim.x;
  const int per = static_cast<int>(L > kTreeThreads ? L / kTreeThreads : 1);   // 1, 2, 4 or 8
  const int nv = static_cast<int>(L > kTreeThreads ? kTreeThreads : L);
  double v = 0.0;
  if (static_cast<int>(threadIdx.x) < nv) {
    const int64_t first = static_cast<int64_t>(blockIdx.x) * L + static_cast<int64_t>(threadIdx.x) * per;
    double x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = (i < per && first + i < ns) ? ssum[first + i] : 0.0;
    if (per == 1) v = x[0];
    else if (per == 2) v = x[0] + x[1];
    else if (per == 4) v = (x[0] + x[1]) + (x[2] + x[3]);
    else v = ((x[0] + x[1]) + (x[2] + x[3])) + ((x[4] + x[5]) + (x[6] + x[7]));
  }
  const double cta = cta_tree(v, nv, sh);
  if (gridDim.x == 1) {
    if (threadIdx.x == 0) *mu_out = __double2float_rn(cta / static_cast<double>(nb));
    return;
  }
  if (threadIdx.x == 0) {
    partial[blockIdx.x] = cta;
    __threadfence();
    is_last = (atomicAdd(ticket, 1u) == gridDim.x - 1) ? 1 : 0;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  const int q = static_cast<int>(gridDim.x);
  const int nv2 = q > kTreeThreads ? kTreeThreads : q;
  const int per2 = q / nv2;                  // a power of two
  double u = 0.0;
  if (static_cast<int>(threadIdx.x) < nv2) {
    // balanced sum of per2 consecutive subtree sums: a binary counter of completed subtrees
    const volatile double* pp = partial + static_cast<int64_t>(threadIdx.x) * per2;
    double st[32];
    int top = 0;
    for (int i = 0; i < per2; ++i) {
      double x = pp[i];
      int k = i, lvl = 0;
      while (k & 1) {
        x = st[lvl] + x;
        k >>= 1;
        ++lvl;
      }
      st[lvl] = x;
      top = lvl;
    }
    u = st[top];
  }
  const double S = cta_tree(u, nv2, sh);
  if (threadIdx.x == 0) {
    *mu_out = __double2float_rn(S / static_cast<double>(nb));
    *ticket = 0u;
  }
}

// Pass 2. One warp per group of 256 constants; each lane handles 8 consecutive constants.
__global__ void __launch_bounds__(256) nf4_dq_pass2(const float* __restrict__ c1, int64_t nblocks,
                                                    const float* __restrict__ mu_ptr,
                                                    uint8_t* __restrict__ e_out,
                                                    float* __restrict__ s2_out, int64_t ngroups) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (g >= ngroups) return;
  const float mu = *mu_ptr;
  const int64_t b0 = g * kGroup + 8 * lane;
  float d[8];
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    d[i] = (b0 + i < nblocks) ? __fsub_rn(c1[b0 + i], mu) : 0.0f;
    m = fmaxf(m, fabsf(d[i]));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  const float s2 = __fdiv_rn(m, 448.0f);
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t e = 0;
    if (s2 > 0.0f) {
      const float t = __fdiv_rn(d[i], s2);
      e = static_cast<uint32_t>(__nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3));
    }
    if (i < 4) lo |= e << (8 * i); else hi |= e << (8 * (i - 4));
  }
  if (b0 + 8 <= nblocks) {
    *reinterpret_cast<uint2*>(e_out + b0) = make_uint2(lo, hi);
  } else {
    for (int i = 0; i < 8; ++i)
      if (b0 + i < nblocks) e_out[b0 + i] = static_cast<uint8_t>(((i < 4) ? lo : hi) >> (8 * (i & 3)));
  }
  if (lane == 0) s2_out[g] = s2;
}

// ------------------------------------------------------------------------------------------------
// Dequantize. A CTA owns groups (16384 elements) blockIdx.x, +gridDim.x, ...; a group's 8 KiB of codes
// and 256 E4M3 constants come into shared memory by bulk copies kDeqStages groups ahead. Each thread
// turns 4 code bytes (8 elements) into 16 bytes of bf16 (or 32 of fp32) per chunk; the 16 levels sit one
// per lane (16-lane shuffle segments). A ragged last group is read straight from global memory.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ float decode_e4m3(uint8_t e) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(e), __NV_E4M3);
  return __half2float(__half(h));
}

// The 8 values of one chunk (4 code bytes; byte b holds element 2b high, 2b+1 low). Whole warp.
__device__ __forceinline__ void dequant8(uint32_t x, float sc, float qreg, float (&v)[8]) {
  v[0] = __fmul_rn(lut16(qreg, x >> 4), sc);
  v[1] = __fmul_rn(lut16(qreg, x), sc);
  v[2] = __fmul_rn(lut16(qreg, x >> 12), sc);
  v[3] = __fmul_rn(lut16(qreg, x >> 8), sc);
  v[4] = __fmul_rn(lut16(qreg, x >> 20), sc);
  v[5] = __fmul_rn(lut16(qreg, x >> 16), sc);
  v[6] = __fmul_rn(lut16(qreg, x >> 28), sc);
  v[7] = __fmul_rn(lut16(qreg, x >> 24), sc);
}
template <bool kBf16Out>
__device__ __forceinline__ void store8(const float (&v)[8], void* __restrict__ out, int64_t chunk) {
  if constexpr (kBf16Out) {
    uint4 o;
    o.x = pack_bf16x2(v[0], v[1]); o.y = pack_bf16x2(v[2], v[3]);
    o.z = pack_bf16x2(v[4], v[5]); o.w = pack_bf16x2(v[6], v[7]);
    __stcs(reinterpret_cast<uint4*>(out) + chunk, o);
  } else {
    float4* o = reinterpret_cast<float4*>(out) + 2 * chunk;
    __stcs(o, make_float4(v[0], v[1], v[2], v[3]));
    __stcs(o + 1, make_float4(v[4], v[5], v[6], v[7]));
  }
}

constexpr int kDeqThreads = 256;
constexpr int kDeqStages = 8;
constexpr uint32_t kDeqCodeBytes = kGroupElems / 2;
constexpr uint32_t kDeqSmemBytes = kDeqStages * (kDeqCodeBytes + kGroup * 4);   // enough for either kind

// kSingle: the constants are stored as fp32 c1 per block (no second level); `c1` replaces e4m3/s2/mu.
template <bool kBf16Out, bool kSingle>
__global__ void __launch_bounds__(kDeqThreads) nf4_dequantize_kernel(
    const uint8_t* __restrict__ codes, const uint8_t* __restrict__ e4m3, const float* __restrict__ s2,
    const float* __restrict__ mu_ptr, const float* __restrict__ c1, int64_t n, void* __restrict__ out,
    CodebookArg cb) {
  constexpr uint32_t kConstBytes = kSingle ? kGroup * 4 : kGroup;
  constexpr uint32_t kStageBytes = kDeqCodeBytes + kConstBytes;
  extern __shared__ __align__(128) unsigned char dsm[];
  __shared__ uint64_t bars[kDeqStages];
  const int tid = threadIdx.x, lane = tid & 31;
  const float qreg = cb.levels[lane & 15];
  const float mu = kSingle ? 0.0f : *mu_ptr;
  const int64_t nfull = n / kGroupElems;
  const int64_t ngroups = (n + kGroupElems - 1) / kGroupElems;
  const int64_t my =
      (static_cast<int64_t>(blockIdx.x) < ngroups) ? (ngroups - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  if (tid == 0) {
    for (int s = 0; s < kDeqStages; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncthreads();
  int64_t issued = 0;   // thread 0: iterations whose copies are issued (a ragged group issues none)
  auto issue_upto = [&](int64_t lim) {
    for (; issued < lim && issued < my; ++issued) {
      const int64_t g = blockIdx.x + issued * gridDim.x;
      if (g >= nfull) continue;
      const int s = static_cast<int>(issued % kDeqStages);
      unsigned char* st = dsm + s * kStageBytes;
      mbar_arrive_expect_tx(&bars[s], kStageBytes);
      bulk_load(st, codes + g * kDeqCodeBytes, kDeqCodeBytes, &bars[s]);
      if constexpr (kSingle) bulk_load(st + kDeqCodeBytes, c1 + g * kGroup, kConstBytes, &bars[s]);
      else bulk_load(st + kDeqCodeBytes, e4m3 + g * kGroup, kConstBytes, &bars[s]);
    }
  };
  if (tid == 0) issue_upto(kDeqStages);
  int64_t i = 0;
  int timed_out = 0;
  for (; i < my; ++i) {
    const int64_t g = blockIdx.x + i * gridDim.x;
    const float sg = kSingle ? 0.0f : s2[g];
    if (g < nfull) {
      const int s = static_cast<int>(i % kDeqStages);
      if (!mbar_wait(&bars[s], static_cast<uint32_t>((i / kDeqStages) & 1))) timed_out = 1;
      const unsigned char* st = dsm + s * kStageBytes;
      const uint32_t* cw = reinterpret_cast<const uint32_t*>(st);
      const uint8_t* ev = st + kDeqCodeBytes;
      const float* cv = reinterpret_cast<const float*>(st + kDeqCodeBytes);
#pragma unroll 4
      for (int k = 0; k < kGroupElems / 8 / kDeqThreads; ++k) {
        const int j = tid + kDeqThreads * k;           // chunk within the group; its block is j / 8
        float v[8];
        const float sc = kSingle ? cv[j >> 3] : __fmaf_rn(decode_e4m3(ev[j >> 3]), sg, mu);
        dequant8(cw[j], sc, qreg, v);
        store8<kBf16Out>(v, out, g * (kGroupElems / 8) + j);
      }
    } else {
      // ragged last group: whole 8-element chunks from global memory, then the last n % 8 elements
      const int64_t c_end = n / 8;
      for (int64_t cw0 = g * (kGroupElems / 8) + (tid - lane); cw0 < c_end; cw0 += kDeqThreads) {
        const int64_t c = cw0 + lane;                  // cw0 is the warp's first chunk: warp-uniform loop
        const bool ok = c < c_end;
        const uint32_t x = ok ? reinterpret_cast<const uint32_t*>(codes)[c] : 0u;
        const int64_t blk = (c * 8) / kBlock;
        const float sc = !ok ? 0.0f : kSingle ? c1[blk] : __fmaf_rn(decode_e4m3(e4m3[blk]), sg, mu);
        float v[8];
        dequant8(x, sc, qreg, v);
        if (ok) store8<kBf16Out>(v, out, c);
      }
      if (tid == 0) {
        for (int64_t e = c_end * 8; e < n; ++e) {
          const uint8_t byte = codes[e / 2];
          const uint32_t code = (e & 1) ? (byte & 0xFu) : (byte >> 4);
          const float sc = kSingle ? c1[e / kBlock] : __fmaf_rn(decode_e4m3(e4m3[e / kBlock]), sg, mu);
          const float v = __fmul_rn(cb.levels[code], sc);
          if constexpr (kBf16Out) reinterpret_cast<__nv_bfloat16*>(out)[e] = __float2bfloat16_rn(v);
          else reinterpret_cast<float*>(out)[e] = v;
        }
      }
    }
    // every thread is done with the stage; the abort decision is uniform
    if (__syncthreads_or(timed_out)) break;
    if (tid == 0) {
      fence_proxy_async_smem();
      issue_upto(i + 1 + kDeqStages);
    }
  }
  if (tid == 0 && i < my) {          // after a timeout: wait briefly for copies still in flight
    for (int64_t j = i; j < issued; ++j) {
      if (blockIdx.x + j * gridDim.x < nfull)
        mbar_wait_short(&bars[j % kDeqStages], static_cast<uint32_t>((j / kDeqStages) & 1));
    }
  }
}

// Expand the double-quantized block constants of an NF4 weight (w_rows x w_cols, blocks of 64 along a
// row) to fp32, c1_hat = fma(decode(e), s2, mu) -- the same single rounding as the dequantizer -- in the
// layout the fused linear kernel loads one stage of at a time:
//   by_column  out[kb * ld + n]  (one row per block column: a stage's 128 rows are contiguous)
//   by_row     out[n * ld + kb]  (one row per weight row, ld a multiple of 4: a stage reads 4 columns)
template <bool kByColumn>
__global__ void __launch_bounds__(256) nf4_expand_scales_kernel(const uint8_t* __restrict__ e4m3,
                                                                const float* __restrict__ s2,
                                                                const float* __restrict__ mu_ptr,
                                                                int64_t w_rows, int64_t kb_w, int64_t ld,
                                                                float* __restrict__ out) {
  const float mu = *mu_ptr;
  const int64_t total = w_rows * kb_w;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int64_t n, kb;
    if constexpr (kByColumn) { kb = i / w_rows; n = i % w_rows; }   // writes coalesced along n
    else { n = i / kb_w; kb = i % kb_w; }                           // reads and writes along kb
    const int64_t blk = n * kb_w + kb;
    const float c = __fmaf_rn(decode_e4m3(e4m3[blk]), s2[blk / kGroup], mu);
    if constexpr (kByColumn) out[kb * ld + n] = c;
    else out[n * ld + kb] = c;
  }
}

}  // namespace qnf4
