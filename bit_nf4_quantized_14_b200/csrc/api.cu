// The library's C ABI (declared in include/qlora_nf4.h): argument checks, workspace layout, tensor-map
// construction and kernel launches for the NF4 codec and the QLoRA linear layer. This is the only
// translation unit with device code, so every kernel shares one status word per device.
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <limits>
#include <cstdio>
#include <cstdlib>
#include <atomic>
#include <cstring>
#include <mutex>
#include <random>
#include <string>
#include <vector>

#include "qlora_nf4.h"
#include "codec.cuh"
#include "codebook_study.cuh"
#include "adamw.cuh"
#include "gemm_nf4w.cuh"
#include "gemm_sm100.cuh"
#include "gemv_nf4.cuh"
#include "decode_nf4.cuh"
#include "selftest.cuh"

namespace qnf4 {
void build_nf4_codebook(float levels[16], float thresholds[15]);   // codebook.cpp

namespace {

constexpr int64_t kMaxNumel = int64_t(1) << 40;
constexpr int64_t kMaxTokens = int64_t(65535) * 128;   // grid.y limit of the 128-row tiles
constexpr int kTargetCtas = 2 * 148;                    // split heuristic: two waves of a B200
std::atomic<int64_t> g_launches{0};
// With QLORA_DEBUG set in the environment, a failed CUDA call is described on stderr (where and why).
inline bool debug_on() {
  static const bool on = std::getenv("QLORA_DEBUG") != nullptr;
  return on;
}
inline int cuda_fail(cudaError_t e, const char* what, int line) {
  if (debug_on()) std::fprintf(stderr, "qlora: %s failed at api.cu:%d: %s\n", what, line, cudaGetErrorString(e));
  return QLORA_ERR_CUDA;
}
inline int launched_at(int line) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? QLORA_OK : cuda_fail(e, "kernel launch", line);
}
#define launched() launched_at(__LINE__)

// Host-side fault injection for tests of callers' error handling: with QLORA_FAULT_INJECT set to
// "<entry point>" or "<entry point>:<k>", the k-th call (the first by default) of that entry point made
// since the variable took its current value fails with QLORA_ERR_CUDA, as a launch failure would: after
// its argument checks, before it enqueues anything. No GPU state is touched.
std::mutex g_inject_mu;
std::string g_inject_armed;          // the variable's value when last seen (empty: unset)
long g_inject_calls = 0;
std::atomic<bool> g_inject_seen{false};
bool injected_fault(const char* entry) {
  const char* v = std::getenv("QLORA_FAULT_INJECT");
  if (!v || !*v) {
    if (g_inject_seen.load(std::memory_order_relaxed)) {      // unset since: forget the count
      std::lock_guard<std::mutex> g(g_inject_mu);
      g_inject_armed.clear();
      g_inject_seen.store(false, std::memory_order_relaxed);
    }
    return false;
  }
  std::lock_guard<std::mutex> g(g_inject_mu);
  g_inject_seen.store(true, std::memory_order_relaxed);
  std::string& armed = g_inject_armed;
  long& calls = g_inject_calls;
  if (armed != v) { armed = v; calls = 0; }
  const std::string spec(v);
  const size_t colon = spec.find(':');
  const std::string name = spec.substr(0, colon);
  long k = 1;
  if (colon != std::string::npos) k = std::strtol(spec.c_str() + colon + 1, nullptr, 10);
  if (name != entry) return false;
  if (++calls != k) return false;
  if (debug_on()) std::fprintf(stderr, "qlora: injected launch failure in %s (call %ld)\n", entry, calls);
  return true;
}
#define INJECT(entry) \
  do { if (injected_fault(entry)) return QLORA_ERR_CUDA; } while (0)

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

const CodebookArg& codebook() {
  static CodebookArg cb;
  static std::once_flag once;
  std::call_once(once, [] { build_nf4_codebook(cb.levels, cb.thresholds); });
  return cb;
}

// The quantizer's bucket table for a codebook of nl levels: bucket b (1..31) covers t = w/a in
// [(b - 16.5)/15, (b - 15.5)/15], widened by kBucketWiden for the approximate reciprocal; lo(b) counts the
// thresholds below it. Valid only if every widened bucket holds at most one threshold (true for the NF4
// thresholds, whose closest pair is 0.0805 apart against a bucket width of 0.0667). Also sets the code of
// an all-zero block: the level of least magnitude, the lower index on a tie (NF4: 7, its exact zero).
bool build_buckets(const CodebookArg& cb, int nl, BucketArg* out) {
  *out = BucketArg{};
  bool ok = true;
  for (int b = 0; b < 32; ++b) {
    const double jl = (b - 16.5) / 15.0 - kBucketWiden, ju = (b - 15.5) / 15.0 + kBucketWiden;
    int lo = 0, inside = 0;
    for (int j = 0; j < nl - 1; ++j) {
      const double t = cb.thresholds[j];
      lo += (t < jl) ? 1 : 0;
      inside += (t >= jl && t <= ju) ? 1 : 0;
    }
    if (inside > 1) ok = false;
    out->lo_nibbles[b / 8] |= static_cast<uint32_t>(lo) << (4 * (b % 8));
  }
  int z = 0;
  for (int j = 1; j < nl; ++j)
    if (std::fabs(cb.levels[j]) < std::fabs(cb.levels[z])) z = j;
  out->zero_codes = 0x11111111u * static_cast<uint32_t>(z);
  // lo(b) as a popcount: lo never drops and rises by at most one from one bucket to the next (two
  // thresholds inside one bucket's span would share a widened bucket, rejected above)
  int prev = 0;
  for (int b = 0; b < 32; ++b) {
    const int lo = static_cast<int>((out->lo_nibbles[b / 8] >> (4 * (b % 8))) & 0xFu);
    const int step = lo - prev;
    if (step < 0 || step > 1) ok = false;
    else if (step == 1) out->step_mask |= 1u << b;
    prev = lo;
  }
  return ok;
}

struct Buckets { BucketArg arg; bool ok; };
const Buckets& buckets() {
  static Buckets bk;
  static std::once_flag once;
  std::call_once(once, [] { bk.ok = build_buckets(codebook(), 16, &bk.arg); });
  return bk;
}

// Kernel arguments for a caller's codebook (host array of nl levels): false unless 2 <= nl <= 16, the
// levels are finite, in [-1, 1] and strictly ascending, and the bucket table is valid. Thresholds are the
// fp32 roundings of the fp64 level midpoints; thresholds past nl - 1 are +inf (never crossed) and levels
// past nl are 0 (never looked up).
bool make_codebook(const float* lv, int nl, CodebookArg* cb, BucketArg* bk) {
  if (!lv || nl < 2 || nl > 16) return false;
  for (int j = 0; j < nl; ++j) {
    if (!(std::fabs(lv[j]) <= 1.0f)) return false;             // also rejects NaN
    if (j > 0 && !(lv[j] > lv[j - 1])) return false;
  }
  *cb = CodebookArg{};
  for (int j = 0; j < 16; ++j) cb->levels[j] = j < nl ? lv[j] : 0.0f;
  for (int j = 0; j < 15; ++j)
    cb->thresholds[j] = j < nl - 1 ? static_cast<float>((static_cast<double>(lv[j]) + lv[j + 1]) / 2.0)
                                   : std::numeric_limits<float>::infinity();
  return build_buckets(*cb, nl, bk);
}

// Launch with programmatic stream serialization: the kernel may start while its predecessor in the
// stream drains, and waits for it (griddepcontrol.wait) before touching its results.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), unsigned grid, unsigned block, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Workspace of the quantizer: per-block constants (fp32), per-slab tree sums (fp64), the mean pass's
// per-CTA subtree sums (fp64) and its arrival counter; each part 256-byte aligned.
struct QuantWs { size_t c1, ssum, partial, ticket, total; int64_t nslabs; unsigned mean_ctas; };
QuantWs quant_ws(int64_t n) {
  const int64_t nb = cdiv(n, kBlock), ns = cdiv(n, kSlabElems);
  int64_t P = 1;
  while (P < ns) P <<= 1;
  QuantWs w;
  w.nslabs = ns;
  w.mean_ctas = static_cast<unsigned>(std::max<int64_t>(1, P / kTreeLeavesPerCta));
  w.c1 = 0;
  w.ssum = align256(static_cast<size_t>(nb) * 4);
  w.partial = w.ssum + align256(static_cast<size_t>(ns) * 8);
  w.ticket = w.partial + align256(static_cast<size_t>(w.mean_ctas) * 8);
  w.total = w.ticket + 256;
  return w;
}

// ---- device checks ------------------------------------------------------------------------------
// Also clears this host thread's pending non-sticky runtime error (cudaGetLastError is per thread, and a
// caller's own earlier query -- an event or stream poll returning cudaErrorNotReady, for instance -- would
// otherwise be reported as a failure of the launches that follow). A sticky error from a device fault is
// returned again by every later call, so it is not hidden.
// It also makes the device's primary context current on the calling thread (cudaSetDevice does so since
// CUDA 12): the tensor maps are encoded through the driver API, which needs a current context, and a
// thread that has made no runtime call yet -- PyTorch's autograd worker, for one -- has none.
int check_device(int* num_sms) {
  (void)cudaGetLastError();
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "cudaGetDevice / cudaSetDevice", __LINE__);
  int major = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
  if (major != 10) return QLORA_ERR_UNSUPPORTED;
  if (num_sms) *num_sms = sms;
  return QLORA_OK;
}

// ---- profiling ----------------------------------------------------------------------------------
struct ProfRec { int cls; cudaEvent_t a, b; };
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof;

struct ProfScope {     // records an event pair around the launches in its lifetime
  int cls; cudaStream_t st; cudaEvent_t a = nullptr, b = nullptr; bool on;
  ProfScope(int c, cudaStream_t s) : cls(c), st(s) {
    { std::lock_guard<std::mutex> g(g_prof_mu); on = g_prof_on; }
    if (on && cudaEventCreate(&a) == cudaSuccess && cudaEventCreate(&b) == cudaSuccess) cudaEventRecord(a, st);
    else on = false;
  }
  ~ProfScope() {
    if (!on) return;
    cudaEventRecord(b, st);
    std::lock_guard<std::mutex> g(g_prof_mu);
    g_prof.push_back({cls, a, b});
  }
};

// ---- tensor maps --------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D row-major tensor: `inner` contiguous elements per row, `outer` rows, row pitch = `pitch` elements.
enum class TmType { kBf16, kU8, kF32 };
bool make_tmap_t(CUtensorMap* m, const void* ptr, TmType t, uint64_t inner, uint64_t outer, uint64_t pitch,
                 uint32_t box_inner, uint32_t box_outer, bool swizzle128) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint64_t esz = t == TmType::kBf16 ? 2 : t == TmType::kU8 ? 1 : 4;
  const CUtensorMapDataType dt = t == TmType::kBf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                 : t == TmType::kU8  ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                     : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch * esz};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && debug_on())
    std::fprintf(stderr, "qlora: tensor map (ptr %p, dims %llu x %llu, stride %llu B, box %u x %u, swizzle %d) -> %d\n",
                 ptr, (unsigned long long)inner, (unsigned long long)outer, (unsigned long long)(pitch * esz),
                 box_inner, box_outer, (int)swizzle128, (int)r);
  return r == CUDA_SUCCESS;
}
bool make_tmap(CUtensorMap* m, const void* ptr, bool bf16, uint64_t inner, uint64_t outer,
               uint32_t box_inner, uint32_t box_outer, bool swizzle128 = true) {
  return make_tmap_t(m, ptr, bf16 ? TmType::kBf16 : TmType::kU8, inner, outer, inner, box_inner, box_outer,
                     bf16 && swizzle128);
}
// bf16 operand tiles: K-major tiles are {64 contraction, rows}; MN-major tiles are {64 MN, 64 contraction}.
bool tmap_kmajor(CUtensorMap* m, const void* p, uint64_t contraction, uint64_t rows, uint32_t box_rows) {
  return make_tmap(m, p, true, contraction, rows, 64, box_rows);
}
bool tmap_mnmajor(CUtensorMap* m, const void* p, uint64_t mn, uint64_t contraction) {
  return make_tmap(m, p, true, mn, contraction, 64, 64);
}

// ---- GEMM launches ------------------------------------------------------------------------------
template <class C>
int launch_gemm(dim3 grid, const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p, cudaStream_t st) {
  auto kern = gemm_sm100_kernel<C>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
  kern<<<grid, C::NUM_THREADS, C::SMEM_BYTES, st>>>(a, b, p);
  return launched();
}

// Pitch (in blocks) of the expanded-constants buffer of a weight with K columns: a multiple of 4, so
// the rows of the by-row layout are 16-byte aligned for TMA.
inline int64_t scales_pitch(int64_t K) { return (K / 64 + 3) / 4 * 4; }

// Fused weight GEMM of the linear layer (gemm_nf4w.cuh). act = X (fwd) or dY (bwd), T x Cn row-major;
// lora_w = B (fwd, N x r) or A (bwd, r x K); uv = s U or s V (T x r); out = Y (T x N) or dX (T x K);
// scales = workspace for the expanded block constants (N x scales_pitch(K) fp32).
template <bool BWD>
int launch_nf4_linear(const void* act, int64_t T, const qlora_nf4_tensor* W, const void* lora_w, int r,
                      const void* uv, void* out, float* scales, cudaStream_t st) {
  using Cfg = NF4WCfg<BWD, 2>;
  const int64_t N = W->rows, K = W->cols, kb_w = K / 64;
  const int64_t Cn = BWD ? N : K, F = BWD ? K : N;
  int sms = 0;
  if (int e = check_device(&sms)) return e;
  // the stage-friendly fp32 constants: by column (kb_w rows of N) forward, by row (N rows) backward
  const int64_t ld = BWD ? scales_pitch(K) : N;
  const unsigned eg = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(cdiv(N * kb_w, 256), int64_t(sms) * 8)));
  if (BWD)
    nf4_expand_scales_kernel<false><<<eg, 256, 0, st>>>(W->absmax_e4m3, W->scale2, W->offset, N, kb_w, ld, scales);
  else
    nf4_expand_scales_kernel<true><<<eg, 256, 0, st>>>(W->absmax_e4m3, W->scale2, W->offset, N, kb_w, ld, scales);
  if (int e = launched()) return e;
  CUtensorMap tx, tc, tk, tuv, to;
  bool ok = tmap_kmajor(&tx, act, Cn, T, 256) && tmap_kmajor(&tuv, uv, r, T, 256) &&
            make_tmap(&to, out, true, F, T, 32, 16, false);
  if (!BWD)
    ok = ok && make_tmap(&tc, W->codes, false, K / 2, N, 32, 128) &&
         make_tmap_t(&tk, scales, TmType::kF32, N, kb_w, N, 128, 1, false);
  else
    ok = ok && make_tmap(&tc, W->codes, false, K / 2, N, 64, 64) &&
         make_tmap_t(&tk, scales, TmType::kF32, kb_w, N, ld, 4, 64, false);
  if (!ok) return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
  NF4GemmParams p{};
  p.T = static_cast<int>(T); p.F = static_cast<int>(F);
  p.nkb = static_cast<int>(cdiv(Cn, 64)); p.nkb2 = static_cast<int>(cdiv(r, 64));
  p.tiles_f = static_cast<int>(cdiv(F, 128));
  p.num_tiles = static_cast<int>(p.tiles_f * cdiv(T, 256));
  p.r = r;
  p.w_rows = N; p.w_cols = K;
  p.lora_w = static_cast<const __nv_bfloat16*>(lora_w);
  auto kern = nf4_linear_gemm_kernel<Cfg>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(p.num_tiles, sms));
  kern<<<grid, Cfg::NUM_THREADS, Cfg::SMEM_BYTES, st>>>(tx, tc, tk, tuv, to, p, codebook());
  return launched();
}

// The adapter GEMMs stream X or dY once: a ring of about 96 KB keeps two CTAs on every SM.
template <int BN> constexpr int skinny_stages() {
  constexpr int stage = 128 * 64 * 2 + BN * 64 * 2;
  return std::max(2, std::min(6, (96 * 1024) / stage));
}

// Split of the contraction: the number of slices s (each at least 4 blocks) that minimises
// waves(s) * (blocks per slice + 4), waves counted against kTargetCtas resident CTAs (two per SM of a
// B200), so that the grid fills whole waves instead of leaving a short last one; the +4 charges each
// slice its pipeline fill and its partial-sum write.
struct Split { int splits, kb_split; };
Split choose_split(int64_t tiles, int64_t nkb) {
  const int64_t max_s = std::max<int64_t>(1, nkb / 4);
  int64_t best_s = 1, best_cost = INT64_MAX;
  for (int64_t s = 1; s <= max_s; ++s) {
    const int64_t kb = cdiv(nkb, s), real_s = cdiv(nkb, kb);
    const int64_t cost = cdiv(tiles * real_s, kTargetCtas) * (kb + 4);   // + pipeline fill and partials
    if (cost < best_cost) { best_cost = cost; best_s = real_s; }
  }
  const int64_t kb_split = cdiv(nkb, best_s);
  return {static_cast<int>(cdiv(nkb, kb_split)), static_cast<int>(kb_split)};
}

enum class Skinny { kU, kV, kGrad };   // operand majors: (K,K), (K,MN), (MN,MN)

// D[M][BN] partials = A (M x C) * B (BN x C)^T over contraction C, split along C.
template <int BN, Skinny S>
int launch_skinny(const CUtensorMap& a, const CUtensorMap& b, int64_t M, int64_t C, float* part,
                  int64_t part_stride, cudaStream_t st) {
  constexpr bool AMN = (S == Skinny::kGrad), BMN = (S != Skinny::kU);
  using Cfg = GemmCfg<BN, AMN, BMN, skinny_stages<BN>()>;
  const int64_t tiles = cdiv(M, 128), nkb = cdiv(C, 64);
  const Split sp = choose_split(tiles, nkb);
  GemmParams p{};
  p.nkb_total = static_cast<int>(nkb);
  p.kb_split = sp.kb_split;
  p.out = part;
  p.part_stride = part_stride;
  return launch_gemm<Cfg>(dim3(1, static_cast<unsigned>(tiles), sp.splits), a, b, p, st);
}
template <Skinny S>
int launch_skinny_bn(int bn, const CUtensorMap& a, const CUtensorMap& b, int64_t M, int64_t C, float* part,
                     int64_t part_stride, cudaStream_t st) {
  switch (bn) {
    case 64: return launch_skinny<64, S>(a, b, M, C, part, part_stride, st);
    case 128: return launch_skinny<128, S>(a, b, M, C, part, part_stride, st);
    case 192: return launch_skinny<192, S>(a, b, M, C, part, part_stride, st);
    case 256: return launch_skinny<256, S>(a, b, M, C, part, part_stride, st);
  }
  return QLORA_ERR_INVALID_ARG;
}
int64_t skinny_part_elems(int64_t M, int64_t C, int bn) {
  const int64_t tiles = cdiv(M, 128);
  const Split sp = choose_split(tiles, cdiv(C, 64));
  return static_cast<int64_t>(sp.splits) * tiles * 128 * bn;
}

int reduce_after(const float* part, int64_t M, int64_t C, int R, int bn, float scale, void* out,
                 Red mode, cudaStream_t st) {
  const int64_t tiles = cdiv(M, 128);
  const Split sp = choose_split(tiles, cdiv(C, 64));
  const int64_t stride = tiles * 128 * bn;
  const int64_t total = M * R;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(cdiv(total, 256), 148 * 16));
  switch (mode) {
    case Red::kRowsBf16:
      split_reduce_kernel<Red::kRowsBf16><<<grid, 256, 0, st>>>(part, sp.splits, stride, bn, M, R, scale, out);
      break;
    case Red::kTransF32:
      split_reduce_kernel<Red::kTransF32><<<grid, 256, 0, st>>>(part, sp.splits, stride, bn, M, R, scale, out);
      break;
    case Red::kRowsF32:
      split_reduce_kernel<Red::kRowsF32><<<grid, 256, 0, st>>>(part, sp.splits, stride, bn, M, R, scale, out);
      break;
  }
  return launched();
}

// ---- argument checks ----------------------------------------------------------------------------
int check_nf4(const qlora_nf4_tensor* q) {
  if (!q || !q->codes || !q->absmax_e4m3 || !q->scale2 || !q->offset) return QLORA_ERR_INVALID_ARG;
  if (q->rows <= 0 || q->cols <= 0 || q->rows > kMaxNumel / q->cols) return QLORA_ERR_SHAPE;
  if (!aligned16(q->codes) || !aligned16(q->absmax_e4m3) || !aligned16(q->scale2) || !aligned16(q->offset))
    return QLORA_ERR_ALIGNMENT;
  return QLORA_OK;
}

struct LinearWs { size_t sU, sV, scales, part, total; };
// ---- small-token path (T <= kGvMaxTokens): the stream-K GEMV kernels ---------------------------
constexpr int kGvMaxCtas = 512;          // grid cap of the NF4 GEMV (>= two CTAs per SM of any B200)
constexpr int kGuMaxSlices = 32;         // contraction slices of the adapter projection
inline int gv_nt(int64_t T) { return T <= 8 ? 1 : T <= 16 ? 2 : T <= 32 ? 4 : 8; }
struct GvShape { int spt, tiles; int64_t total; };
inline GvShape gv_shape(int64_t rows, int64_t K) {
  GvShape g;
  g.spt = static_cast<int>(cdiv(K, kGvStageK));
  g.tiles = static_cast<int>(cdiv(rows, kGvRows));
  g.total = static_cast<int64_t>(g.spt) * g.tiles;
  return g;
}
inline int gv_maxseg(const GvShape& g, int G) {
  return static_cast<int>(cdiv(cdiv(g.total, G), g.spt)) + 1;
}
// Partial slots a launch of up to `cap` CTAs can need (the largest G * maxseg over G <= cap).
inline int64_t gv_slots(const GvShape& g, int cap) {
  int64_t best = 0;
  for (int G = 1; G <= std::min<int64_t>(cap, g.total); ++G) best = std::max<int64_t>(best, int64_t(G) * gv_maxseg(g, G));
  return best;
}
struct GuShape { int groups, kslices, kb_per_slice; };
inline GuShape gu_shape(int64_t K, int r) {
  const int nkb = static_cast<int>(K / 64);
  GuShape u;
  u.groups = static_cast<int>(cdiv(r, 16));
  u.kb_per_slice = static_cast<int>(cdiv(nkb, std::min(nkb, kGuMaxSlices)));
  u.kslices = static_cast<int>(cdiv(nkb, u.kb_per_slice));
  return u;
}
// Layout inside the linear workspace's fp32 region (offsets in bytes): NF4 partials, adapter partials,
// then the two ticket arrays (NF4: one per tile and consumer warp; adapter: one per 16 rows).
struct GemvWs { size_t part_w, part_u, ticket_w, ticket_u, ticket_bytes, total; };
GemvWs gemv_ws(int64_t T, int64_t N, int64_t K, int r) {
  const int nt = gv_nt(T);
  const int64_t slot = int64_t(kGvWarps) * 32 * nt * 4 * 4;      // bytes of one partial tile
  const GvShape gw = gv_shape(N, K);
  const GuShape gu = gu_shape(K, r);
  GemvWs w;
  w.part_w = 0;
  w.part_u = align256(static_cast<size_t>(gv_slots(gw, kGvMaxCtas) * slot));
  w.ticket_w = w.part_u + align256(static_cast<size_t>(gu.groups) * gu.kslices * 32 * nt * 4 * 4);
  w.ticket_u = w.ticket_w + align256(static_cast<size_t>(gw.tiles) * kGvWarps * 4);
  w.total = w.ticket_u + align256(static_cast<size_t>(gu.groups) * 4);
  w.ticket_bytes = w.total - w.ticket_w;
  return w;
}

// ---- decode path (T <= kDcMaxTokens): one cooperative launch of nf4_decode_kernel ---------------
// Workspace of the decode path (offsets in bytes): one tag per 16-row tile of A, and the per-CTA results
// awaiting the adapter term when they do not fit in shared memory ([tile][16][T] fp32).
struct DecWs { size_t tags, base, total; };
DecWs dec_ws(int64_t T, int64_t N, int r) {
  DecWs w;
  w.tags = 0;
  w.base = align256(static_cast<size_t>(cdiv(r, 16)) * 8);
  w.total = w.base + align256(static_cast<size_t>(cdiv(N, 16)) * 16 * T * 4);
  return w;
}
// A value no earlier call in this process used and that uninitialised memory is unlikely to hold: the
// tree's tags compare equal to it only once this call has written them.
uint64_t next_call_tag() {
  static std::atomic<uint64_t> ctr{[] {
    std::random_device rd;
    return (static_cast<uint64_t>(rd()) << 32) ^ rd() ^ 0x9E3779B97F4A7C15ull;
  }()};
  uint64_t v;
  do { v = ctr.fetch_add(1, std::memory_order_relaxed); } while (v == 0 || v == ~0ull);
  return v;
}

LinearWs linear_ws(int64_t T, int64_t N, int64_t K, int r) {
  const int bn = static_cast<int>(cdiv(r, 64) * 64);
  int64_t part = 0;
  if (T <= kGvMaxTokens) part = static_cast<int64_t>(gemv_ws(T, N, K, r).total / 4);
  if (T <= kDcMaxTokens) part = std::max<int64_t>(part, static_cast<int64_t>(dec_ws(T, N, r).total / 4));
  part = std::max(part, skinny_part_elems(T, K, bn));   // U
  part = std::max(part, skinny_part_elems(T, N, bn));   // V
  part = std::max(part, skinny_part_elems(K, T, bn));   // dA
  part = std::max(part, skinny_part_elems(N, T, bn));   // dB
  LinearWs w;
  w.sU = 0;
  w.sV = align256(static_cast<size_t>(T) * r * 2);
  w.scales = w.sV + align256(static_cast<size_t>(T) * r * 2);
  w.part = w.scales + align256(static_cast<size_t>(N) * scales_pitch(K) * 4);
  w.total = w.part + align256(static_cast<size_t>(part) * 4);
  return w;
}

int check_linear(const void* X, int64_t T, const qlora_nf4_tensor* W, const void* A, const void* B, int r,
                 float alpha, void* ws, size_t ws_bytes) {
  if (!X || !A || !B) return QLORA_ERR_INVALID_ARG;
  if (int e = check_nf4(W)) return e;
  if (r < 8 || r > 256 || r % 8 != 0 || !std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
  if (T < 1 || T > kMaxTokens || W->cols % 64 != 0 || W->rows % 8 != 0 || W->rows > (int64_t(1) << 30) ||
      W->cols > (int64_t(1) << 30))
    return QLORA_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(ws)) return QLORA_ERR_ALIGNMENT;
  if (!ws || ws_bytes < linear_ws(T, W->rows, W->cols, r).total) return QLORA_ERR_WORKSPACE;
  return QLORA_OK;
}

// sU = s * X A^T (T x r, bf16) via the split adapter GEMM and its reduction.
template <int NT>
int launch_gemv_nt(const CUtensorMap& ta, const CUtensorMap& tx, const GvParams& p, int grid, cudaStream_t st) {
  using C = GvCfg<NT>;
  auto kern = nf4_gemv_kernel<NT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGvThreads);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];               // may start while the adapter projection runs
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, ta, tx, p, codebook()) != cudaSuccess) return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
  return launched();
}

// sU = s * X A^T for T <= kGvMaxTokens; clears both ticket arrays of the small-token path first.
int gemv_sU(const void* X, int64_t T, int64_t K, const void* A, int r, float s, void* sU, char* gws,
            const GemvWs& L, cudaStream_t st) {
  if (cudaMemsetAsync(gws + L.ticket_w, 0, L.ticket_bytes, st) != cudaSuccess) return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
  const GuShape u = gu_shape(K, r);
  GuParams p = {};
  p.T = static_cast<int>(T);
  p.r = r;
  p.K = static_cast<int>(K);
  p.kslices = u.kslices;
  p.kb_per_slice = u.kb_per_slice;
  p.X = static_cast<const __nv_bfloat16*>(X);
  p.A = static_cast<const __nv_bfloat16*>(A);
  p.s = s;
  p.sU = static_cast<__nv_bfloat16*>(sU);
  p.part = reinterpret_cast<float*>(gws + L.part_u);
  p.ticket = reinterpret_cast<unsigned*>(gws + L.ticket_u);
  const dim3 grid(u.groups, u.kslices);
  switch (gv_nt(T)) {
    case 1: lora_u_kernel<1><<<grid, 32, 0, st>>>(p); break;
    case 2: lora_u_kernel<2><<<grid, 32, 0, st>>>(p); break;
    case 4: lora_u_kernel<4><<<grid, 32, 0, st>>>(p); break;
    default: lora_u_kernel<8><<<grid, 32, 0, st>>>(p); break;
  }
  return launched();
}

// Y = X W_hat^T + sU B^T for T <= kGvMaxTokens (right after gemv_sU on the same stream).
int gemv_fwd(const void* X, int64_t T, const qlora_nf4_tensor* W, const void* B, int r, const void* sU, void* Y,
             char* gws, const GemvWs& L, int sms, cudaStream_t st) {
  const int64_t N = W->rows, K = W->cols;
  const int nt = gv_nt(T);
  CUtensorMap ta, tx;
  if (!make_tmap_t(&ta, W->codes, TmType::kU8, K / 2, N, K / 2, kGvRowBytes, kGvRows, true) ||
      !make_tmap_t(&tx, X, TmType::kBf16, K, T, K, 64, 8 * nt, true))
    return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
  const GvShape g = gv_shape(N, K);
  const int per_sm = nt <= 4 ? GvCfg<1>::CTAS_PER_SM : GvCfg<8>::CTAS_PER_SM;
  const int G = static_cast<int>(std::min<int64_t>(std::min<int64_t>(g.total, int64_t(sms) * per_sm), kGvMaxCtas));
  GvParams p = {};
  p.T = static_cast<int>(T);
  p.rows = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.spt = g.spt;
  p.tiles = g.tiles;
  p.total = g.total;
  p.maxseg = gv_maxseg(g, G);
  p.kbw = static_cast<int>(K / 64);
  p.e4m3 = W->absmax_e4m3;
  p.s2 = W->scale2;
  p.mu = W->offset;
  p.sU = static_cast<const __nv_bfloat16*>(sU);
  p.Bw = static_cast<const __nv_bfloat16*>(B);
  p.r = r;
  p.out = static_cast<__nv_bfloat16*>(Y);
  p.ldo = N;
  p.part = reinterpret_cast<float*>(gws + L.part_w);
  p.ticket = reinterpret_cast<unsigned*>(gws + L.ticket_w);
  switch (nt) {
    case 1: return launch_gemv_nt<1>(ta, tx, p, G, st);
    case 2: return launch_gemv_nt<2>(ta, tx, p, G, st);
    case 4: return launch_gemv_nt<4>(ta, tx, p, G, st);
    default: return launch_gemv_nt<8>(ta, tx, p, G, st);
  }
}

// Decode-sized forward (or, with u_only, the adapter projection sU alone) in one cooperative launch:
// one CTA per SM, every CTA resident, which the waits for sU written by other CTAs require. sU's
// summation order does not depend on the grid, so the backward's recompute gives the forward's U.
int launch_decode(const void* X, int64_t T, const qlora_nf4_tensor* W, const void* A, const void* B, int r, float s,
                  void* Y, void* U, char* dws, bool u_only, cudaStream_t st) {
  int sms = 0;
  if (int e = check_device(&sms)) return e;
  const int64_t N = W->rows, K = W->cols;
  const DecWs L = dec_ws(T, N, r);
  const int64_t tiles = cdiv(N, 16), atiles = cdiv(r, 16);
  const int64_t load = u_only ? kDcALoad * atiles : tiles + kDcALoad * atiles;
  const int G = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(load, std::min(sms, kGvMaxCtas))));
  DecParams p{};
  p.T = static_cast<int>(T); p.N = static_cast<int>(N); p.K = static_cast<int>(K); p.r = r;
  p.RP = static_cast<int>(cdiv(r, 64) * 64);
  p.nkb = static_cast<int>(K / 64);
  p.tiles = static_cast<int>(tiles);
  p.atiles = static_cast<int>(atiles);
  p.u_only = u_only ? 1 : 0;
  p.s = s;
  p.X = static_cast<const __nv_bfloat16*>(X);
  p.codes = W->codes;
  p.e4m3 = W->absmax_e4m3;
  p.s2 = W->scale2;
  p.mu = W->offset;
  p.A = static_cast<const __nv_bfloat16*>(A);
  p.B = static_cast<const __nv_bfloat16*>(B);
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.U = static_cast<__nv_bfloat16*>(U);
  p.tags = reinterpret_cast<uint64_t*>(dws + L.tags);
  p.base_ws = reinterpret_cast<float*>(dws + L.base);
  p.seq = next_call_tag();
  auto kern = T <= 8 ? nf4_decode_kernel<8> : nf4_decode_kernel<16>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kDcSmemBytes) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "cudaFuncSetAttribute", __LINE__);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(G));
  cfg.blockDim = dim3(kDcThreads);
  cfg.dynamicSmemBytes = kDcSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, p, codebook()) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "cooperative launch", __LINE__);
  return launched();
}

int compute_sU(const void* X, int64_t T, int64_t K, const void* A, int r, float s, void* sU, float* part,
               cudaStream_t st) {
  const int bn = static_cast<int>(cdiv(r, 64) * 64);
  CUtensorMap ta, tb;
  if (!tmap_kmajor(&ta, X, K, T, 128) || !tmap_kmajor(&tb, A, K, r, bn)) return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
  const int64_t stride = cdiv(T, 128) * 128 * bn;
  if (int e = launch_skinny_bn<Skinny::kU>(bn, ta, tb, T, K, part, stride, st)) return e;
  return reduce_after(part, T, K, r, bn, s, sU, Red::kRowsBf16, st);
}

// ---- fixed scratch of qlora_nf4_quantize_noalloc ---------------------------------------------------
// The quantizer's workspace (quant_ws) for the largest accepted input, 2^26 elements: 2^20 fp32
// per-block constants, 2^14 fp64 slab sums, 8 fp64 subtree sums and the arrival counter. Smaller inputs
// use a prefix of each part. In host code `g_noalloc_scratch` names a host-side stand-in, never the
// device array: its device address is looked up once per device with cudaGetSymbolAddress and cached.
constexpr int64_t kNoallocBlocks = QLORA_NOALLOC_MAX_NUMEL / kBlock;
constexpr int64_t kNoallocSlabs = QLORA_NOALLOC_MAX_NUMEL / kSlabElems;
constexpr size_t kNoallocC1Bytes = static_cast<size_t>(kNoallocBlocks) * 4;
constexpr size_t kNoallocSsumBytes = static_cast<size_t>(kNoallocSlabs) * 8;
static_assert(kNoallocC1Bytes + kNoallocSsumBytes + 256 + 256 == QLORA_NOALLOC_SCRATCH_BYTES, "scratch layout");
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
struct NoallocSlot { unsigned long long ctx_id; void* ptr; };
NoallocSlot g_noalloc_slot[kMaxDevices] = {};

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[QLORA_NOALLOC_SCRATCH_BYTES];

namespace {
// Identity of the calling thread's current context: cuCtxGetId through the runtime's driver entry
// point (the library links no driver library); 0 if it is unavailable.
unsigned long long current_ctx_id() {
  using GetCur = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCur get_cur = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<GetCur>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (get_cur && get_cur(&c) == CUDA_SUCCESS && c && get_id && get_id(c, &id) == CUDA_SUCCESS) return id;
  return 0;
}

// Device address of this device's scratch array. The set-up -- cudaGetSymbolAddress with the device
// current -- runs on the first call on a device, and again if that device's context was replaced since
// (after a cudaDeviceReset the module, and with it the array, may be loaded at another address).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail(cudaGetLastError(), "cudaGetDevice", __LINE__);
  if (dev < 0 || dev >= kMaxDevices) return QLORA_ERR_UNSUPPORTED;
  const unsigned long long ctx = current_ctx_id();
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc_slot[dev];
  if (!slot.ptr || ctx == 0 || slot.ctx_id != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
      return cuda_fail(cudaGetLastError(), "cudaGetSymbolAddress", __LINE__);
    slot.ptr = p;
    slot.ctx_id = ctx;
  }
  *out = slot.ptr;
  return QLORA_OK;
}

// Pass 1 on stream st: persistent, Q1<InT>::kCtasPerSm CTAs per SM (fewer when there are fewer whole slabs).
// With ssum and ticket null it writes the fp32 constants as they are (the single-quantization format).
template <typename InT>
int launch_pass1_t(const InT* w, int64_t n, uint8_t* codes, float* c1, double* ssum, unsigned* ticket,
                   const CodebookArg& cb, const BucketArg& bk, int sms, cudaStream_t st) {
  if (cudaFuncSetAttribute(nf4_quantize_pass1<InT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Q1<InT>::kSmemBytes) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "cudaFuncSetAttribute", __LINE__);
  const int64_t nfull = n / kSlabElems;
  const unsigned grid =
      static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(nfull, int64_t(sms) * Q1<InT>::kCtasPerSm)));
  nf4_quantize_pass1<InT><<<grid, kQ1Threads, Q1<InT>::kSmemBytes, st>>>(w, n, codes, c1, ssum, cdiv(n, kSlabElems),
                                                                          cb, bk, ticket);
  return launched();
}
int launch_pass1(const void* w, int w_dtype, int64_t n, uint8_t* codes, float* c1, double* ssum, unsigned* ticket,
                 const CodebookArg& cb, const BucketArg& bk, int sms, cudaStream_t st) {
  if (w_dtype == QLORA_F32)
    return launch_pass1_t(static_cast<const float*>(w), n, codes, c1, ssum, ticket, cb, bk, sms, st);
  const unsigned grid = static_cast<unsigned>(
      std::max<int64_t>(1, std::min<int64_t>(cdiv(cdiv(n, kSlabElems), kQuantThreads / 32), int64_t(sms) * kQuantMinBlocks)));
  nf4_quantize_pass1_direct<__nv_bfloat16><<<grid, kQuantThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(w), n, codes, c1, ssum, cdiv(n, kSlabElems), cb, bk, ticket);
  return launched();
}

// Passes 1, 1b and 2 of the quantizer on stream st, workspace laid out by quant_ws(n).
int run_quantize(const void* w, int w_dtype, int64_t n, const qlora_nf4_tensor* out, void* ws, cudaStream_t st) {
  int sms = 0;
  if (int e = check_device(&sms)) return e;
  const Buckets& bk = buckets();
  if (!bk.ok) return QLORA_ERR_UNSUPPORTED;
  const QuantWs L = quant_ws(n);
  char* base = static_cast<char*>(ws);
  float* c1 = reinterpret_cast<float*>(base + L.c1);
  double* ssum = reinterpret_cast<double*>(base + L.ssum);
  double* partial = reinterpret_cast<double*>(base + L.partial);
  unsigned* ticket = reinterpret_cast<unsigned*>(base + L.ticket);
  const int64_t nb = cdiv(n, kBlock), ng = cdiv(nb, kGroup);
  if (int e = launch_pass1(w, w_dtype, n, out->codes, c1, ssum, ticket, codebook(), bk.arg, sms, st)) return e;
  if (launch_pdl(nf4_mean, L.mean_ctas, kTreeThreads, st, ssum, L.nslabs, nb, partial, ticket, out->offset) !=
      cudaSuccess)
    return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
  if (int e = launched()) return e;
  if (launch_pdl(nf4_dq_pass2, static_cast<unsigned>(cdiv(ng, 8)), 256u, st, c1, nb, out->offset,
                 out->absmax_e4m3, out->scale2, ng) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
  return launched();
}

// The bulk-copy dequantizer in either constant format (double-quantized, or fp32 per block).
int launch_dequant(bool bf16, bool single, const uint8_t* codes, const uint8_t* e4m3, const float* s2,
                   const float* mu, const float* c1, int64_t n, void* out, int sms, cudaStream_t st,
                   const CodebookArg& cb) {
  auto kern = bf16 ? (single ? nf4_dequantize_kernel<true, true> : nf4_dequantize_kernel<true, false>)
                   : (single ? nf4_dequantize_kernel<false, true> : nf4_dequantize_kernel<false, false>);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kDeqSmemBytes) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDeqThreads, kDeqSmemBytes) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
  const unsigned grid = static_cast<unsigned>(
      std::max<int64_t>(1, std::min<int64_t>(cdiv(n, kGroupElems), int64_t(sms) * std::max(per_sm, 1))));
  kern<<<grid, kDeqThreads, kDeqSmemBytes, st>>>(codes, e4m3, s2, mu, c1, n, out, cb);
  return launched();
}

// Pass 1 alone, with fp32 block constants kept as they are (no slab sums, no mean pass).
int launch_pass1_single(const void* w, int w_dtype, int64_t n, uint8_t* codes, float* absmax,
                        const CodebookArg& cb, const BucketArg& bk, int sms, cudaStream_t st) {
  return launch_pass1(w, w_dtype, n, codes, absmax, nullptr, nullptr, cb, bk, sms, st);
}

static_assert(kStatOut == QLORA_CODEBOOK_STATS_LEN, "codebook statistics layout");
int64_t stat_ctas(int64_t n) { return std::min<int64_t>(cdiv(cdiv(n, kStepElems), kStatThreads / 32), kStatMaxCtas); }
}  // namespace
}  // namespace qnf4

using namespace qnf4;

// ================================== C ABI ==========================================================
extern "C" {

int qlora_nf4_codebook(float* levels, float* thresholds) {
  if (!levels || !thresholds) return QLORA_ERR_INVALID_ARG;
  const CodebookArg& cb = codebook();
  std::memcpy(levels, cb.levels, sizeof(cb.levels));
  std::memcpy(thresholds, cb.thresholds, sizeof(cb.thresholds));
  return QLORA_OK;
}

int qlora_nf4_storage_bytes(int64_t n, size_t* codes, size_t* absmax, size_t* scale2, size_t* offset) {
  if (n <= 0 || n > kMaxNumel) return QLORA_ERR_SHAPE;
  const int64_t nb = cdiv(n, kBlock), ng = cdiv(nb, kGroup);
  if (codes) *codes = static_cast<size_t>(cdiv(n, 2));
  if (absmax) *absmax = static_cast<size_t>(nb);
  if (scale2) *scale2 = static_cast<size_t>(ng) * 4;
  if (offset) *offset = 4;
  return QLORA_OK;
}

int qlora_nf4_quantize_workspace(int64_t n, size_t* bytes) {
  if (!bytes) return QLORA_ERR_INVALID_ARG;
  if (n <= 0 || n > kMaxNumel) return QLORA_ERR_SHAPE;
  *bytes = quant_ws(n).total;
  return QLORA_OK;
}

int qlora_nf4_quantize(const void* w, int w_dtype, int64_t rows, int64_t cols, const qlora_nf4_tensor* out,
                       void* workspace, size_t workspace_bytes, qlora_stream_t stream) {
  if (!w) return QLORA_ERR_INVALID_ARG;
  if (w_dtype != QLORA_F32 && w_dtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || rows > kMaxNumel / cols) return QLORA_ERR_SHAPE;
  if (int e = check_nf4(out)) return e;
  if (out->rows != rows || out->cols != cols) return QLORA_ERR_SHAPE;
  if (!aligned16(w) || !aligned16(workspace)) return QLORA_ERR_ALIGNMENT;
  const int64_t n = rows * cols;
  if (!workspace || workspace_bytes < quant_ws(n).total) return QLORA_ERR_WORKSPACE;
  INJECT("qlora_nf4_quantize");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope prof(QLORA_PROF_QUANTIZE, st);
  return run_quantize(w, w_dtype, n, out, workspace, st);
}

int qlora_nf4_quantize_noalloc(const void* w, int w_dtype, int64_t rows, int64_t cols,
                               const qlora_nf4_tensor* out, qlora_stream_t stream) {
  if (!w) return QLORA_ERR_INVALID_ARG;
  if (w_dtype != QLORA_F32 && w_dtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || rows > kMaxNumel / cols) return QLORA_ERR_SHAPE;
  if (rows * cols > QLORA_NOALLOC_MAX_NUMEL) return QLORA_ERR_TOO_LARGE;
  if (int e = check_nf4(out)) return e;
  if (out->rows != rows || out->cols != cols) return QLORA_ERR_SHAPE;
  if (!aligned16(w)) return QLORA_ERR_ALIGNMENT;
  INJECT("qlora_nf4_quantize_noalloc");
  if (int e = check_device(nullptr)) return e;
  void* scratch = nullptr;
  if (int e = noalloc_scratch(&scratch)) return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope prof(QLORA_PROF_QUANTIZE, st);
  return run_quantize(w, w_dtype, rows * cols, out, scratch, st);
}

int qlora_nf4_dequantize(const qlora_nf4_tensor* q, void* out, int out_dtype, qlora_stream_t stream) {
  if (!out) return QLORA_ERR_INVALID_ARG;
  if (out_dtype != QLORA_F32 && out_dtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
  if (int e = check_nf4(q)) return e;
  if (!aligned16(out)) return QLORA_ERR_ALIGNMENT;
  INJECT("qlora_nf4_dequantize");
  int sms = 0;
  if (int e = check_device(&sms)) return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n = q->rows * q->cols;
  ProfScope prof(QLORA_PROF_DEQUANTIZE, st);
  return launch_dequant(out_dtype == QLORA_BF16, false, q->codes, q->absmax_e4m3, q->scale2, q->offset, nullptr, n,
                        out, sms, st, codebook());
}

int qlora_nf4_quantize_single(const void* w, int w_dtype, int64_t rows, int64_t cols, void* codes, float* absmax,
                              qlora_stream_t stream) {
  if (!w || !codes || !absmax) return QLORA_ERR_INVALID_ARG;
  if (w_dtype != QLORA_F32 && w_dtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || rows > kMaxNumel / cols) return QLORA_ERR_SHAPE;
  if (!aligned16(w) || !aligned16(codes) || !aligned16(absmax)) return QLORA_ERR_ALIGNMENT;
  INJECT("qlora_nf4_quantize_single");
  int sms = 0;
  if (int e = check_device(&sms)) return e;
  const Buckets& bk = buckets();
  if (!bk.ok) return QLORA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope prof(QLORA_PROF_QUANTIZE, st);
  return launch_pass1_single(w, w_dtype, rows * cols, static_cast<uint8_t*>(codes), absmax, codebook(), bk.arg, sms,
                             st);
}

int qlora_nf4_dequantize_single(const void* codes, const float* absmax, int64_t rows, int64_t cols, void* out,
                                int out_dtype, qlora_stream_t stream) {
  if (!codes || !absmax || !out) return QLORA_ERR_INVALID_ARG;
  if (out_dtype != QLORA_F32 && out_dtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || rows > kMaxNumel / cols) return QLORA_ERR_SHAPE;
  if (!aligned16(codes) || !aligned16(absmax) || !aligned16(out)) return QLORA_ERR_ALIGNMENT;
  INJECT("qlora_nf4_dequantize_single");
  int sms = 0;
  if (int e = check_device(&sms)) return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope prof(QLORA_PROF_DEQUANTIZE, st);
  return launch_dequant(out_dtype == QLORA_BF16, true, static_cast<const uint8_t*>(codes), nullptr, nullptr, nullptr,
                        absmax, rows * cols, out, sms, st, codebook());
}

int qlora_codebook_quantize(const void* w, int w_dtype, int64_t n, const float* levels, int nlevels, void* codes,
                            float* absmax, qlora_stream_t stream) {
  if (!w || !codes || !absmax) return QLORA_ERR_INVALID_ARG;
  if (w_dtype != QLORA_F32 && w_dtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
  if (n <= 0 || n > kMaxNumel) return QLORA_ERR_SHAPE;
  CodebookArg cb;
  BucketArg bk;
  if (!make_codebook(levels, nlevels, &cb, &bk)) return QLORA_ERR_CODEBOOK;
  if (!aligned16(w) || !aligned16(codes) || !aligned16(absmax)) return QLORA_ERR_ALIGNMENT;
  INJECT("qlora_codebook_quantize");
  int sms = 0;
  if (int e = check_device(&sms)) return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope prof(QLORA_PROF_QUANTIZE, st);
  return launch_pass1_single(w, w_dtype, n, static_cast<uint8_t*>(codes), absmax, cb, bk, sms, st);
}

int qlora_codebook_dequantize(const void* codes, const float* absmax, int64_t n, const float* levels, int nlevels,
                              void* out, int out_dtype, qlora_stream_t stream) {
  if (!codes || !absmax || !out) return QLORA_ERR_INVALID_ARG;
  if (out_dtype != QLORA_F32 && out_dtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
  if (n <= 0 || n > kMaxNumel) return QLORA_ERR_SHAPE;
  CodebookArg cb;
  BucketArg bk;
  if (!make_codebook(levels, nlevels, &cb, &bk)) return QLORA_ERR_CODEBOOK;
  if (!aligned16(codes) || !aligned16(absmax) || !aligned16(out)) return QLORA_ERR_ALIGNMENT;
  INJECT("qlora_codebook_dequantize");
  int sms = 0;
  if (int e = check_device(&sms)) return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope prof(QLORA_PROF_DEQUANTIZE, st);
  return launch_dequant(out_dtype == QLORA_BF16, true, static_cast<const uint8_t*>(codes), nullptr, nullptr, nullptr,
                        absmax, n, out, sms, st, cb);
}

int qlora_codebook_stats_workspace(int64_t n, size_t* bytes) {
  if (!bytes) return QLORA_ERR_INVALID_ARG;
  if (n <= 0 || n > kMaxNumel) return QLORA_ERR_SHAPE;
  *bytes = align256(static_cast<size_t>(stat_ctas(n)) * kStatVals * sizeof(double));
  return QLORA_OK;
}

int qlora_codebook_stats(const void* w, int w_dtype, const void* codes, const float* absmax, int64_t n,
                         const float* levels, int nlevels, double* stats, void* workspace, size_t workspace_bytes,
                         qlora_stream_t stream) {
  if (!w || !codes || !absmax || !stats) return QLORA_ERR_INVALID_ARG;
  if (w_dtype != QLORA_F32 && w_dtype != QLORA_BF16) return QLORA_ERR_INVALID_ARG;
  if (n <= 0 || n > kMaxNumel) return QLORA_ERR_SHAPE;
  CodebookArg cb;
  BucketArg bk;
  if (!make_codebook(levels, nlevels, &cb, &bk)) return QLORA_ERR_CODEBOOK;
  const int64_t G = stat_ctas(n);
  if (!workspace || workspace_bytes < static_cast<size_t>(G) * kStatVals * sizeof(double)) return QLORA_ERR_WORKSPACE;
  if (!aligned16(w) || !aligned16(codes) || !aligned16(absmax) || !aligned16(stats) || !aligned16(workspace))
    return QLORA_ERR_ALIGNMENT;
  INJECT("qlora_codebook_stats");
  if (int e = check_device(nullptr)) return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  double* part = static_cast<double*>(workspace);
  const uint8_t* c = static_cast<const uint8_t*>(codes);
  if (w_dtype == QLORA_F32)
    codebook_stats_partial<float><<<static_cast<unsigned>(G), kStatThreads, 0, st>>>(static_cast<const float*>(w), c,
                                                                                    absmax, n, cb, part);
  else
    codebook_stats_partial<__nv_bfloat16><<<static_cast<unsigned>(G), kStatThreads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(w), c, absmax, n, cb, part);
  if (int e = launched()) return e;
  codebook_stats_final<<<1, 64, 0, st>>>(part, static_cast<int>(G), n, cb, nlevels, stats);
  return launched();
}

int qlora_adamw_step(float* p, const float* g, float* m, float* v, void* p_bf16, int64_t n, int64_t step, float lr,
                     float beta1, float beta2, float eps, float weight_decay, qlora_stream_t stream) {
  if (!p || !g || !m || !v) return QLORA_ERR_INVALID_ARG;
  if (step < 1 || !(lr >= 0.0f) || !(lr < INFINITY) || !(beta1 >= 0.0f && beta1 < 1.0f) ||
      !(beta2 >= 0.0f && beta2 < 1.0f) || !(eps > 0.0f && eps < INFINITY) || !(weight_decay >= 0.0f) ||
      !(weight_decay < INFINITY))
    return QLORA_ERR_INVALID_ARG;
  if (n <= 0 || n > kMaxNumel) return QLORA_ERR_SHAPE;
  if (!aligned16(p) || !aligned16(g) || !aligned16(m) || !aligned16(v) || !aligned16(p_bf16)) return QLORA_ERR_ALIGNMENT;
  INJECT("qlora_adamw_step");
  int sms = 0;
  if (int e = check_device(&sms)) return e;
  AdamWArgs a;
  const double t = static_cast<double>(step);
  a.keep = static_cast<float>(1.0 - static_cast<double>(lr) * weight_decay);
  a.beta1 = beta1;
  a.one_minus_beta1 = static_cast<float>(1.0 - beta1);
  a.beta2 = beta2;
  a.one_minus_beta2 = static_cast<float>(1.0 - beta2);
  a.step_size = static_cast<float>(lr / (1.0 - std::pow(static_cast<double>(beta1), t)));
  a.inv_bc2_sqrt = static_cast<float>(1.0 / std::sqrt(1.0 - std::pow(static_cast<double>(beta2), t)));
  a.eps = eps;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const unsigned grid = static_cast<unsigned>(
      std::max<int64_t>(1, std::min<int64_t>(cdiv(n / 4, kAdamThreads), int64_t(sms) * 8)));
  if (p_bf16)
    adamw_kernel<true><<<grid, kAdamThreads, 0, st>>>(p, g, m, v, static_cast<__nv_bfloat16*>(p_bf16), n, a);
  else
    adamw_kernel<false><<<grid, kAdamThreads, 0, st>>>(p, g, m, v, nullptr, n, a);
  return launched();
}

int qlora_paged_alloc(size_t bytes, void** ptr) {
  if (!ptr || bytes == 0) return QLORA_ERR_INVALID_ARG;
  *ptr = nullptr;
  if (int e = check_device(nullptr)) return e;
  if (cudaMallocManaged(ptr, bytes, cudaMemAttachGlobal) != cudaSuccess) {
    *ptr = nullptr;
    return cuda_fail(cudaGetLastError(), "cudaMallocManaged", __LINE__);
  }
  return QLORA_OK;
}

int qlora_paged_free(void* ptr) {
  if (!ptr) return QLORA_OK;
  if (cudaFree(ptr) != cudaSuccess) return cuda_fail(cudaGetLastError(), "cudaFree", __LINE__);
  return QLORA_OK;
}

int qlora_paged_prefetch(const void* ptr, size_t bytes, int to_device, qlora_stream_t stream) {
  if (!ptr || bytes == 0) return QLORA_ERR_INVALID_ARG;
  if (int e = check_device(nullptr)) return e;
  int dev = 0, concurrent = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&concurrent, cudaDevAttrConcurrentManagedAccess, dev) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "cudaDeviceGetAttribute", __LINE__);
  if (!concurrent) return QLORA_ERR_UNSUPPORTED;
  if (cudaMemPrefetchAsync(ptr, bytes, to_device ? dev : cudaCpuDeviceId, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return cuda_fail(cudaGetLastError(), "cudaMemPrefetchAsync", __LINE__);
  return QLORA_OK;
}

int qlora_linear_workspace(int64_t T, int64_t N, int64_t K, int r, size_t* bytes) {
  if (!bytes) return QLORA_ERR_INVALID_ARG;
  if (r < 8 || r > 256 || r % 8 != 0) return QLORA_ERR_INVALID_ARG;
  if (T < 1 || T > kMaxTokens || N < 8 || K < 64 || N % 8 || K % 64) return QLORA_ERR_SHAPE;
  *bytes = linear_ws(T, N, K, r).total;
  return QLORA_OK;
}

int qlora_linear_fwd(const void* X, int64_t T, const qlora_nf4_tensor* W, const void* A, const void* B, int r,
                     float alpha, void* Y, void* U_out, void* workspace, size_t workspace_bytes,
                     qlora_stream_t stream) {
  if (!Y) return QLORA_ERR_INVALID_ARG;
  if (int e = check_linear(X, T, W, A, B, r, alpha, workspace, workspace_bytes)) return e;
  if (!aligned16(Y) || !aligned16(U_out)) return QLORA_ERR_ALIGNMENT;
  INJECT("qlora_linear_fwd");
  if (int e = check_device(nullptr)) return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t N = W->rows, K = W->cols;
  const float s = alpha / static_cast<float>(r);
  const LinearWs L = linear_ws(T, N, K, r);
  char* ws = static_cast<char*>(workspace);
  void* sU = U_out ? U_out : ws + L.sU;
  float* part = reinterpret_cast<float*>(ws + L.part);
  if (T <= kDcMaxTokens) {                      // decode-sized: one launch, projection included
    ProfScope prof(QLORA_PROF_FWD_GEMM, st);
    return launch_decode(X, T, W, A, B, r, s, Y, sU, ws + L.part, false, st);
  }
  if (T <= kGvMaxTokens) {                      // small token counts: the stream-K GEMV kernels
    int sms = 0;
    if (int e = check_device(&sms)) return e;
    const GemvWs G = gemv_ws(T, N, K, r);
    {
      ProfScope prof(QLORA_PROF_LORA, st);
      if (int e = gemv_sU(X, T, K, A, r, s, sU, ws + L.part, G, st)) return e;
    }
    ProfScope prof(QLORA_PROF_FWD_GEMM, st);
    return gemv_fwd(X, T, W, B, r, sU, Y, ws + L.part, G, sms, st);
  }
  {
    ProfScope prof(QLORA_PROF_LORA, st);
    if (int e = compute_sU(X, T, K, A, r, s, sU, part, st)) return e;
  }
  ProfScope prof(QLORA_PROF_FWD_GEMM, st);
  return launch_nf4_linear<false>(X, T, W, B, r, sU, Y, reinterpret_cast<float*>(ws + L.scales), st);
}

int qlora_linear_bwd(const void* dY, const void* X, int64_t T, const qlora_nf4_tensor* W, const void* A,
                     const void* B, int r, float alpha, const void* U, void* dX, float* dA, float* dB,
                     void* workspace, size_t workspace_bytes, qlora_stream_t stream) {
  if (!dY || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  if (int e = check_linear(X, T, W, A, B, r, alpha, workspace, workspace_bytes)) return e;
  if (!aligned16(dY) || !aligned16(U) || !aligned16(dX) || !aligned16(dA) || !aligned16(dB))
    return QLORA_ERR_ALIGNMENT;
  INJECT("qlora_linear_bwd");
  if (int e = check_device(nullptr)) return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t N = W->rows, K = W->cols;
  const float s = alpha / static_cast<float>(r);
  const int bn = static_cast<int>(cdiv(r, 64) * 64);
  const LinearWs L = linear_ws(T, N, K, r);
  char* ws = static_cast<char*>(workspace);
  float* part = reinterpret_cast<float*>(ws + L.part);
  void* sV = ws + L.sV;
  const void* sU = U;
  {
    ProfScope prof(QLORA_PROF_LORA, st);
    if (!sU) {                                  // the forward's own projection, so U is identical
      if (T <= kDcMaxTokens) {
        if (int e = launch_decode(X, T, W, A, B, r, s, nullptr, ws + L.sU, ws + L.part, true, st)) return e;
      } else if (T <= kGvMaxTokens) {
        if (int e = gemv_sU(X, T, K, A, r, s, ws + L.sU, ws + L.part, gemv_ws(T, N, K, r), st)) return e;
      } else if (int e = compute_sU(X, T, K, A, r, s, ws + L.sU, part, st)) {
        return e;
      }
      sU = ws + L.sU;
    }
    // sV = s * dY B  (T x r): contraction over the N output features; B is N x r, i.e. MN-major.
    CUtensorMap tdy, tbl;
    if (!tmap_kmajor(&tdy, dY, N, T, 128) || !tmap_mnmajor(&tbl, B, r, N)) return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
    if (int e = launch_skinny_bn<Skinny::kV>(bn, tdy, tbl, T, N, part, cdiv(T, 128) * 128 * bn, st)) return e;
    if (int e = reduce_after(part, T, N, r, bn, s, sV, Red::kRowsBf16, st)) return e;
  }
  if (dX) {
    ProfScope prof(QLORA_PROF_BWD_GEMM, st);
    if (int e = launch_nf4_linear<true>(dY, T, W, A, r, sV, dX, reinterpret_cast<float*>(ws + L.scales), st)) return e;
  }
  ProfScope prof(QLORA_PROF_LORA, st);
  {
    // dA^T[k][j] = sum_t X[t][k] sV[t][j]  -> dA (r x K), transposed in the reduction
    CUtensorMap tx, tv;
    if (!tmap_mnmajor(&tx, X, K, T) || !tmap_mnmajor(&tv, sV, r, T)) return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
    if (int e = launch_skinny_bn<Skinny::kGrad>(bn, tx, tv, K, T, part, cdiv(K, 128) * 128 * bn, st)) return e;
    if (int e = reduce_after(part, K, T, r, bn, 1.0f, dA, Red::kTransF32, st)) return e;
  }
  {
    // dB[n][j] = sum_t dY[t][n] sU[t][j]
    CUtensorMap tdy, tu;
    if (!tmap_mnmajor(&tdy, dY, N, T) || !tmap_mnmajor(&tu, sU, r, T)) return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
    if (int e = launch_skinny_bn<Skinny::kGrad>(bn, tdy, tu, N, T, part, cdiv(N, 128) * 128 * bn, st)) return e;
    if (int e = reduce_after(part, N, T, r, bn, 1.0f, dB, Red::kRowsF32, st)) return e;
  }
  return QLORA_OK;
}

int qlora_set_wait_limit(uint64_t ns) {
  if (ns != 0 && (ns < 1000 || ns > kWaitLimitNs)) return QLORA_ERR_INVALID_ARG;
  if (int e = check_device(nullptr)) return e;
  const unsigned long long v = ns ? ns : kWaitLimitNs;
  if (cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "cudaMemcpyToSymbol", __LINE__);
  return QLORA_OK;
}

int qlora_selftest_wait(int kind, qlora_stream_t stream) {
  if (kind != QLORA_SELFTEST_MBARRIER && kind != QLORA_SELFTEST_DEVICE_WORD) return QLORA_ERR_INVALID_ARG;
  if (int e = check_device(nullptr)) return e;
  bounded_wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(kind);
  return launched();
}

int qlora_get_status(int* device_status, qlora_stream_t stream) {
  if (!device_status) return QLORA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess)
    return cuda_fail(cudaGetLastError(), "CUDA call or tensor-map encode", __LINE__);
  *device_status = static_cast<int>(v);
  if (v & kStatusTimeout) return QLORA_ERR_TIMEOUT;
  if (v & kStatusNonfinite) return QLORA_ERR_NONFINITE;
  return QLORA_OK;
}

const char* qlora_error_string(int code) {
  switch (code) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument";
    case QLORA_ERR_SHAPE: return "unsupported or inconsistent shape";
    case QLORA_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case QLORA_ERR_CUDA: return "CUDA call or kernel launch failed";
    case QLORA_ERR_NONFINITE: return "non-finite value in a quantized input";
    case QLORA_ERR_TIMEOUT: return "a kernel gave up waiting (bounded wait expired)";
    case QLORA_ERR_UNSUPPORTED: return "device is not an sm_100 GPU";
    case QLORA_ERR_TOO_LARGE: return "input exceeds the fixed scratch of the no-allocation quantize (2^26 elements)";
    case QLORA_ERR_CODEBOOK: return "codebook not 2..16 ascending levels in [-1, 1], or two thresholds within one bucket";
  }
  return "unknown error code";
}

int qlora_profile_enable(int on) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  g_prof_on = (on != 0);
  return QLORA_OK;
}

int qlora_profile_read(int64_t* launches, double* total_ms) {
  if (!launches || !total_ms) return QLORA_ERR_INVALID_ARG;
  std::vector<ProfRec> recs;
  {
    std::lock_guard<std::mutex> g(g_prof_mu);
    recs.swap(g_prof);
  }
  for (int i = 0; i < QLORA_PROF_COUNT; ++i) { launches[i] = 0; total_ms[i] = 0.0; }
  int rc = QLORA_OK;
  for (auto& r : recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
      rc = QLORA_ERR_CUDA;
    launches[r.cls] += 1;
    total_ms[r.cls] += ms;
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  return rc;
}

int64_t qlora_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
