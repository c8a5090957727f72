// Statistics of a codebook's codes, for the codebook comparison: per-level counts and sums of the
// normalised values, the squared error, code entropy, RMS error and one Lloyd update.
#pragma once

#include <cmath>

#include "codec.cuh"

namespace qnf4 {

// Codebook comparison (PEFT page, zerotofrontier.app/sft/peft, "NF4, derived from normal quantiles": a
// Gaussian matrix in blocks of 64 under several codebooks, with code entropy, RMS error and Lloyd's
// algorithm). The quantizer and the dequantizer of codec.cuh take any sorted codebook of 2..16 levels;
// these two kernels measure what a codebook did to a tensor:
//   per level j  count_j = #{elements with code j},  sum_j = sum of u = w / a over those elements (fp64;
//                u is formed as w * fp64(1/a), within one fp64 ulp of the quotient; 0 where a = 0);
//   overall      sse = sum of (w_hat - w)^2 in fp64, w_hat = RN32(q[code] * a) (what the dequantizer
//                writes in fp32), and from these the code entropy in bits, the RMS error and the Lloyd
//                update of the levels, q_j <- RN32(sum_j / count_j) (unchanged where count_j = 0).
// Every lane sums its own elements in order, a warp combines its lanes in lane order (the squared error by
// a fixed shuffle tree), a CTA its warps in order and the final kernel the CTAs in order, so a result
// depends only on the input and the grid.
constexpr int kStatThreads = 128;
constexpr int kStatWarps = kStatThreads / 32;
constexpr int kStatVals = 33;          // 16 counts, 16 sums of u, the squared-error sum
constexpr int kStatMaxCtas = 2048;
constexpr int kStatOut = 51;           // counts[16], sums[16], sse, entropy, rms, levels after one Lloyd step[16]

template <typename InT>
__global__ void __launch_bounds__(kStatThreads) codebook_stats_partial(const InT* __restrict__ w,
                                                                      const uint8_t* __restrict__ codes,
                                                                      const float* __restrict__ absmax, int64_t n,
                                                                      CodebookArg cb, double* __restrict__ partial) {
  // Lane-private accumulators indexed by code: [warp][level][lane], so one element costs one shared
  // load-add-store of its own level's slot instead of a pass over all 16 levels.
  __shared__ double acc_u[kStatWarps][16][32];
  __shared__ uint32_t acc_n[kStatWarps][16][32];
  __shared__ double red[kStatWarps][kStatVals];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float qreg = cb.levels[lane & 15];
#pragma unroll
  for (int j = 0; j < 16; ++j) { acc_u[warp][j][lane] = 0.0; acc_n[warp][j][lane] = 0u; }
  double* my_u = &acc_u[warp][0][lane];
  uint32_t* my_n = &acc_n[warp][0][lane];
  double sse = 0.0;
  const int64_t nsteps = (n + kStepElems - 1) / kStepElems;
  const int64_t nbytes = (n + 1) / 2;
  for (int64_t st = static_cast<int64_t>(blockIdx.x) * kStatWarps + warp; st < nsteps;
       st += static_cast<int64_t>(gridDim.x) * kStatWarps) {
    const int64_t e0 = st * kStepElems + 16 * lane;    // this lane: 16 elements of block e0 / 64
    const bool full = (st + 1) * kStepElems <= n;      // the same for the whole warp
    float x[16];
    uint32_t c0 = 0u, c1 = 0u;
    if (full) {
      Raw16<InT> r;
      r.load(w + e0);
      r.widen(x);
      const uint2 cc = *reinterpret_cast<const uint2*>(codes + (e0 >> 1));
      c0 = cc.x;
      c1 = cc.y;
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) x[e] = (e0 + e < n) ? Scalar<InT>::load(w + e0 + e) : 0.0f;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const int64_t ib = (e0 >> 1) + b;
        const uint32_t v = (ib < nbytes) ? codes[ib] : 0u;
        if (b < 4) c0 |= v << (8 * b);
        else c1 |= v << (8 * (b - 4));
      }
    }
    const float a = (e0 < n) ? absmax[e0 / kBlock] : 0.0f;
    const double ad = a;
    const double ra = (a > 0.0f) ? 1.0 / ad : 0.0;      // u = w * fp64(1/a): within one fp64 ulp of w / a
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint32_t byte = ((e < 8 ? c0 : c1) >> (8 * ((e >> 1) & 3))) & 0xFFu;
      const uint32_t code = (e & 1) ? (byte & 0xFu) : (byte >> 4);
      const float q = lut16(qreg, code);                                   // the whole warp takes part
      if (full || e0 + e < n) {
        const double xd = x[e];
        const double d = static_cast<double>(__fmul_rn(q, a)) - xd;
        sse = fma(d, d, sse);
        my_u[code * 32] += xd * ra;
        my_n[code * 32] += 1u;
      }
    }
  }
  __syncwarp();
  // warp totals in a fixed order: lane j sums level j's 32 slots of u, lane 16 + j its counts
  double v;
  {
    const int j = lane & 15;
    double t = 0.0;
    if (lane < 16) {
      for (int l = 0; l < 32; ++l) t += acc_u[warp][j][l];
    } else {
      uint32_t c = 0u;
      for (int l = 0; l < 32; ++l) c += acc_n[warp][j][l];
      t = static_cast<double>(c);
    }
    v = t;
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) sse += __shfl_xor_sync(0xffffffffu, sse, off);
  red[warp][lane < 16 ? 16 + lane : lane - 16] = v;     // [0..15] counts, [16..31] sums
  if (lane == 0) red[warp][32] = sse;
  __syncthreads();
  if (threadIdx.x < kStatVals) {
    double t = 0.0;
    for (int wi = 0; wi < kStatWarps; ++wi) t += red[wi][threadIdx.x];
    partial[static_cast<int64_t>(blockIdx.x) * kStatVals + threadIdx.x] = t;
  }
}

__global__ void __launch_bounds__(64) codebook_stats_final(const double* __restrict__ partial, int nctas, int64_t n,
                                                          CodebookArg cb, int nlevels, double* __restrict__ out) {
  __shared__ double tot[kStatVals];
  const int t = threadIdx.x;
  if (t < kStatVals) {
    double s = 0.0;
    for (int g = 0; g < nctas; ++g) s += partial[static_cast<int64_t>(g) * kStatVals + t];
    tot[t] = s;
  }
  __syncthreads();
  if (t < 16) {
    out[t] = tot[t];
    out[16 + t] = tot[16 + t];
    const bool used = t < nlevels && tot[t] > 0.0;
    out[35 + t] = used ? static_cast<double>(static_cast<float>(tot[16 + t] / tot[t]))
                       : static_cast<double>(cb.levels[t]);
  }
  if (t == 0) {
    const double nd = static_cast<double>(n);
    double h = 0.0;
    for (int j = 0; j < 16; ++j) {
      if (tot[j] > 0.0) {
        const double p = tot[j] / nd;
        h -= p * log2(p);
      }
    }
    out[32] = tot[32];
    out[33] = h;
    out[34] = sqrt(tot[32] / nd);
  }
}

}  // namespace qnf4
