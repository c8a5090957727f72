// NF4 codec kernels: blockwise quantization with double-quantized constants, and dequantization.
//
// Method (PEFT page, zerotofrontier.app/sft/peft, "Block-wise quantization in one page",
// "NF4, derived from normal quantiles", "Double quantization", "The real way"; QLoRA explainer,
// prism.theerrors.in, "For the curious"):
//   pass 1  per block of 64 consecutive elements: absmax c1, 4-bit codes (two per byte), and per group
//           of 256 blocks the fp64 balanced-tree sum of its c1 values;
//   pass 1b the mean mu of all c1: the fp64 balanced tree continued over the group sums, / nb, -> fp32;
//   pass 2  per group: d = c1 - mu, s2 = max|d| / 448, e = E4M3(d / s2) (round to nearest even, satfinite).
//   dequant c1_hat = fma(decode(e), s2, mu); w_hat = fp32(level[code] * c1_hat) -> bf16 (RNE) or fp32.
//
// Codes: the pages ask for the index of the nearest level. The library's rule is
// code = #{j : w > T_j * a}, T_j the fp32-rounded level midpoints, a > 0 the block absmax, evaluated
// exactly; ties go to the lower index; a block with a = 0 codes as 7. For fp32 w, T_j and a:
//   w > T_j * a  <=>  w > RD(T_j * a)
// where RD is the fp32 product rounded toward -inf (no fp32 value lies strictly between RD(P) and an
// inexact P, subnormals included), so one __fmul_rd and one compare decide each threshold exactly.
#pragma once

#include <cuda_fp8.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace qnf4 {

struct CodebookArg {       // passed by value: lives in the kernel-parameter constant bank
  float levels[16];
  float thresholds[15];
};

constexpr int kBlock = 64;          // first-level block (weights per absmax constant)
constexpr int kGroup = 256;         // second-level block (constants per fp32 scale)
constexpr int kGroupElems = kBlock * kGroup;
constexpr int kQuantThreads = 256;

// Code of w in a block with absmax a > 0. T points at the 15 thresholds in shared memory.
__device__ __forceinline__ uint32_t nf4_code(float w, float a, const float* T, float t7) {
  uint32_t c = (w > __fmul_rd(t7, a)) ? 8u : 0u;
  c += (w > __fmul_rd(T[c + 3], a)) ? 4u : 0u;
  c += (w > __fmul_rd(T[c + 1], a)) ? 2u : 0u;
  c += (w > __fmul_rd(T[c], a)) ? 1u : 0u;
  return c;
}

template <typename InT> struct QuantVec;
template <> struct QuantVec<float> {          // 4 fp32 per 16-byte load, 16 lanes per block
  static constexpr int kElems = 4;
  __device__ static void widen(const uint4& v, float (&x)[4]) {
    x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
  }
  __device__ static float load1(const float* p) { return *p; }
};
template <> struct QuantVec<__nv_bfloat16> {  // 8 bf16 per 16-byte load, 8 lanes per block
  static constexpr int kElems = 8;
  __device__ static void widen(const uint4& v, float (&x)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  __device__ static float load1(const __nv_bfloat16* p) { return __bfloat162float(*p); }
};

// fp64 balanced-tree sum of the 256 block constants of a group held in shared memory (one warp):
// lane l sums leaves 8l..8l+7 as a balanced tree, then the 32 lane sums are combined pairwise.
__device__ __forceinline__ double group_tree_sum(const float* c1s, int lane) {
  double v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = static_cast<double>(c1s[8 * lane + i]);
  double s = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const double r = __shfl_down_sync(0xffffffffu, s, off);
    if ((lane & (2 * off - 1)) == 0) s = s + r;   // left subtree + right subtree
  }
  return s;
}

// Pass 1. Grid-stride over groups of 256 blocks; 256 threads per CTA. Writes codes, c1 (fp32,
// workspace) and the group's fp64 tree sum (workspace).
template <typename InT>
__global__ void __launch_bounds__(kQuantThreads) nf4_quantize_pass1(
    const InT* __restrict__ w, int64_t n, uint8_t* __restrict__ codes, float* __restrict__ c1,
    double* __restrict__ gsum, int64_t ngroups, CodebookArg cb) {
  using V = QuantVec<InT>;
  constexpr int E = V::kElems;                 // elements per thread per load
  constexpr int LPB = kBlock / E;              // lanes per block
  constexpr int LOADS = kGroupElems / E / kQuantThreads;  // 16-byte loads per thread per group
  __shared__ float T[16];
  __shared__ float c1s[kGroup];
  const int tid = threadIdx.x, lane = tid & 31;
  if (tid < 15) T[tid] = cb.thresholds[tid];
  __syncthreads();
  const float t7 = T[7];

  for (int64_t g = blockIdx.x; g < ngroups; g += gridDim.x) {
    const int64_t gbase = g * kGroupElems;
    const bool full = gbase + kGroupElems <= n;
    if (full) {
      uint4 v[LOADS];
      const uint4* src = reinterpret_cast<const uint4*>(w + gbase);
#pragma unroll
      for (int i = 0; i < LOADS; ++i) v[i] = __ldcs(src + tid + kQuantThreads * i);
#pragma unroll
      for (int i = 0; i < LOADS; ++i) {
        float x[E];
        V::widen(v[i], x);
        uint32_t m = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) m = max(m, __float_as_uint(x[e]) & 0x7FFFFFFFu);
#pragma unroll
        for (int off = LPB / 2; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
        const int blk = (tid + kQuantThreads * i) / LPB;  // block index within the group
        if (m >= 0x7F800000u) {
          if ((lane % LPB) == 0) raise_status(kStatusNonfinite);
        }
        const float a = __uint_as_float(m);
        uint32_t packed = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const uint32_t c = (a > 0.0f) ? nf4_code(x[e], a, T, t7) : 7u;
          // byte e/2 of this thread's code bytes: even element high nibble, odd element low nibble
          packed |= c << (8 * (e >> 1) + ((e & 1) ? 0 : 4));
        }
        const int64_t ebase = gbase + static_cast<int64_t>(E) * (tid + kQuantThreads * i);
        if constexpr (E == 4) {
          *reinterpret_cast<uint16_t*>(codes + ebase / 2) = static_cast<uint16_t>(packed);
        } else {
          *reinterpret_cast<uint32_t*>(codes + ebase / 2) = packed;
        }
        if ((lane % LPB) == 0) c1s[blk] = a;
      }
    } else {
      // Ragged last group: scalar loads, one block per LPB-lane team, bounds on every element.
      for (int blk = tid / LPB; blk < kGroup; blk += kQuantThreads / LPB) {
        const int64_t b0 = gbase + static_cast<int64_t>(blk) * kBlock;
        float x[E];
        uint32_t m = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int64_t idx = b0 + (lane % LPB) * E + e;
          x[e] = (idx < n) ? V::load1(w + idx) : 0.0f;
          m = max(m, __float_as_uint(x[e]) & 0x7FFFFFFFu);
        }
#pragma unroll
        for (int off = LPB / 2; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (m >= 0x7F800000u && (lane % LPB) == 0) raise_status(kStatusNonfinite);
        const float a = __uint_as_float(m);
#pragma unroll
        for (int e = 0; e < E; e += 2) {
          const int64_t idx = b0 + (lane % LPB) * E + e;
          if (idx < n) {
            const uint32_t hi = (a > 0.0f) ? nf4_code(x[e], a, T, t7) : 7u;
            const uint32_t lo = (idx + 1 < n) ? ((a > 0.0f) ? nf4_code(x[e + 1], a, T, t7) : 7u) : 0u;
            codes[idx / 2] = static_cast<uint8_t>((hi << 4) | lo);
          }
        }
        if ((lane % LPB) == 0) c1s[blk] = (b0 < n) ? a : 0.0f;
      }
    }
    __syncthreads();
    const int64_t nb = (n + kBlock - 1) / kBlock;
    for (int b = tid; b < kGroup; b += kQuantThreads) {
      const int64_t gb = g * kGroup + b;
      if (gb < nb) c1[gb] = c1s[b];
    }
    if (tid < 32) {
      const double s = group_tree_sum(c1s, lane);
      if (lane == 0) gsum[g] = s;
    }
    __syncthreads();
  }
}

// Pass 1b. One CTA: the fp64 balanced tree over the group sums zero-padded to P = 2^ceil(log2 ng)
// leaves, continued to the root; mu = fp32(fp64(S / nb)).
constexpr int kMeanThreads = 1024;
__global__ void __launch_bounds__(kMeanThreads) nf4_mean(const double* __restrict__ gsum,
                                                        int64_t ngroups, int64_t nblocks,
                                                        float* __restrict__ mu_out) {
  __shared__ double s[kMeanThreads];
  int64_t P = 1;
  while (P < ngroups) P <<= 1;
  const int nthreads = static_cast<int>(P < kMeanThreads ? P : kMeanThreads);
  const int64_t chunk = P / nthreads;            // a power of two
  const int tid = threadIdx.x;
  double v = 0.0;
  if (tid < nthreads) {
    // serial balanced tree over leaves [tid*chunk, (tid+1)*chunk): a binary counter of subtrees
    double stack[48];
    int top_level = 0;
    for (int64_t i = 0; i < chunk; ++i) {
      const int64_t idx = static_cast<int64_t>(tid) * chunk + i;
      double x = (idx < ngroups) ? gsum[idx] : 0.0;
      int64_t k = i;
      int lvl = 0;
      while (k & 1) {
        x = stack[lvl] + x;   // left sibling + right
        k >>= 1;
        ++lvl;
      }
      stack[lvl] = x;
      top_level = lvl;
    }
    v = stack[top_level];
  }
  s[tid] = v;
  __syncthreads();
  for (int len = nthreads / 2; len >= 1; len >>= 1) {
    double x = 0.0;
    if (tid < len) x = s[2 * tid] + s[2 * tid + 1];
    __syncthreads();
    if (tid < len) s[tid] = x;
    __syncthreads();
  }
  if (tid == 0) *mu_out = __double2float_rn(s[0] / static_cast<double>(nblocks));
}

// Pass 2. One warp per group of 256 constants; each lane handles 8 consecutive constants.
__global__ void __launch_bounds__(256) nf4_dq_pass2(const float* __restrict__ c1, int64_t nblocks,
                                                    const float* __restrict__ mu_ptr,
                                                    uint8_t* __restrict__ e_out,
                                                    float* __restrict__ s2_out, int64_t ngroups) {
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

// Dequantize. Each thread turns 4 code bytes (8 elements) per step into 8 bf16 (16 B) or 8 fp32;
// a warp writes 512 contiguous bytes of bf16. The 16 levels sit one per lane (16-lane segments).
__device__ __forceinline__ float decode_e4m3(uint8_t e) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(e), __NV_E4M3);
  return __half2float(__half(h));
}
__device__ __forceinline__ float block_scale(const uint8_t* e4m3, const float* s2, float mu,
                                             int64_t blk) {
  return __fmaf_rn(decode_e4m3(e4m3[blk]), s2[blk / kGroup], mu);
}

template <bool kBf16Out>
__global__ void __launch_bounds__(256) nf4_dequantize_kernel(
    const uint8_t* __restrict__ codes, const uint8_t* __restrict__ e4m3,
    const float* __restrict__ s2, const float* __restrict__ mu_ptr, int64_t n,
    void* __restrict__ out, CodebookArg cb) {
  const int lane = threadIdx.x & 31;
  const float qreg = cb.levels[lane & 15];
  const float mu = *mu_ptr;
  const int64_t nchunks = n / 8;                       // full 8-element chunks
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  constexpr int U = 4;
  for (int64_t c0 = static_cast<int64_t>(blockIdx.x) * blockDim.x * U + threadIdx.x; ;
       c0 += stride * U) {
    // all lanes of a warp stay in the loop together (the lookups are warp-wide shuffles)
    const int64_t warp_first = c0 - lane;
    if (warp_first >= nchunks) break;
    uint32_t cw[U];
    float sc[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t c = c0 + static_cast<int64_t>(u) * blockDim.x;
      const bool ok = c < nchunks;
      cw[u] = ok ? __ldcs(reinterpret_cast<const uint32_t*>(codes) + c) : 0u;
      sc[u] = ok ? block_scale(e4m3, s2, mu, (c * 8) / kBlock) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t c = c0 + static_cast<int64_t>(u) * blockDim.x;
      const uint32_t x = cw[u];
      float v[8];
      // byte b of x holds element 2b (high nibble) and 2b+1 (low nibble)
      v[0] = __fmul_rn(lut16(qreg, x >> 4), sc[u]);
      v[1] = __fmul_rn(lut16(qreg, x), sc[u]);
      v[2] = __fmul_rn(lut16(qreg, x >> 12), sc[u]);
      v[3] = __fmul_rn(lut16(qreg, x >> 8), sc[u]);
      v[4] = __fmul_rn(lut16(qreg, x >> 20), sc[u]);
      v[5] = __fmul_rn(lut16(qreg, x >> 16), sc[u]);
      v[6] = __fmul_rn(lut16(qreg, x >> 28), sc[u]);
      v[7] = __fmul_rn(lut16(qreg, x >> 24), sc[u]);
      if (c < nchunks) {
        if constexpr (kBf16Out) {
          uint4 o;
          o.x = pack_bf16x2(v[0], v[1]); o.y = pack_bf16x2(v[2], v[3]);
          o.z = pack_bf16x2(v[4], v[5]); o.w = pack_bf16x2(v[6], v[7]);
          __stcs(reinterpret_cast<uint4*>(out) + c, o);
        } else {
          float4* o = reinterpret_cast<float4*>(out) + 2 * c;
          __stcs(o, make_float4(v[0], v[1], v[2], v[3]));
          __stcs(o + 1, make_float4(v[4], v[5], v[6], v[7]));
        }
      }
    }
  }
  // ragged tail (n % 8 elements): one thread, byte loads
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    for (int64_t i = nchunks * 8; i < n; ++i) {
      const uint8_t byte = codes[i / 2];
      const uint32_t code = (i & 1) ? (byte & 0xFu) : (byte >> 4);
      const float v = __fmul_rn(cb.levels[code], block_scale(e4m3, s2, mu, i / kBlock));
      if constexpr (kBf16Out) reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(v);
      else reinterpret_cast<float*>(out)[i] = v;
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
