// C ABI of the routed MoE FFN forward pass: argument checks, workspace layout,
// TMA descriptors and kernel launches.  One translation unit so the device
// status word is shared by every kernel.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>

#include "backward.cuh"
#include "common.cuh"
#include "expert_fused.cuh"
#include "gemm_tc.cuh"
#include "int4_gemm.cuh"
#include "permute.cuh"
#include "quant.cuh"
#include "router.cuh"
#include "tree_router.cuh"
#include "wgrad.cuh"

namespace moe {

static std::atomic<unsigned long long> g_launches{0};
static std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};

static inline void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

#define MOE_CUDA_TRY(expr)                       \
  do {                                           \
    cudaError_t err_ = (expr);                   \
    if (err_ != cudaSuccess) return MOE_CUDA_ERROR; \
  } while (0)

#define MOE_LAUNCH_CHECK()                       \
  do {                                           \
    count_launch();                              \
    if (cudaGetLastError() != cudaSuccess) return MOE_CUDA_ERROR; \
  } while (0)

// Every kernel is launched with programmatic stream serialisation (programmatic dependent launch): its
// grid may be scheduled while the previous kernel on the stream drains, and it waits (griddepcontrol.wait,
// first statement of every kernel here) before touching memory.  This hides most of the launch gap between
// the short kernels of one forward, also inside CUDA graphs.
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
#ifndef MOE_NO_PDL
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
#endif
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

#define MOE_LAUNCH(kern, grid, block, smem, st, ...)                                                      \
  do {                                                                                                   \
    if (launch_pdl(kern, dim3(grid), dim3(block), (size_t)(smem), st, 1u, __VA_ARGS__) != cudaSuccess)   \
      return MOE_CUDA_ERROR;                                                                             \
  } while (0)

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
static inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

// ------------------------------------------------------------------ shape checks

static int check_shape(const moe_shape* s) {
  if (s == nullptr) return MOE_INVALID_ARGUMENT;
  if (s->T < 1 || s->T > (1ll << 24)) return MOE_UNSUPPORTED_SHAPE;
  if (s->E < 1 || s->E > kMaxE) return MOE_UNSUPPORTED_SHAPE;
  if (s->k < 1 || s->k > 16) return MOE_UNSUPPORTED_SHAPE;
  if (s->k > s->E) return MOE_INVALID_ARGUMENT;
  if (s->d < 16 || s->d % 16 != 0 || s->d > 65536) return MOE_UNSUPPORTED_SHAPE;
  if (s->H < 16 || s->H % 16 != 0 || s->H > 65536) return MOE_UNSUPPORTED_SHAPE;
  if (s->H_s < 0 || s->H_s % 16 != 0 || s->H_s > 65536) return MOE_UNSUPPORTED_SHAPE;
  if (s->capacity < 0) return MOE_INVALID_ARGUMENT;
  if (s->act != MOE_ACT_SWIGLU && s->act != MOE_ACT_GEGLU) return MOE_INVALID_ARGUMENT;
  if (s->wfmt != MOE_WFMT_BF16 && s->wfmt != MOE_WFMT_INT4_G128) return MOE_INVALID_ARGUMENT;
  if (s->renorm != 0 && s->renorm != 1) return MOE_INVALID_ARGUMENT;
  if (s->flags & ~MOE_FLAG_SINGLE_CTA_GEMM) return MOE_INVALID_ARGUMENT;
  if (s->wfmt == MOE_WFMT_INT4_G128 && (s->d % 128 != 0 || s->H % 128 != 0 || s->H_s % 128 != 0))
    return MOE_UNSUPPORTED_SHAPE;
  const long long R = s->capacity > 0 ? (long long)s->E * s->capacity : s->T * s->k;
  if (R >= (1ll << 31) - 256) return MOE_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

static inline long long grouped_rows(const moe_shape* s) {
  return s->capacity > 0 ? (long long)s->E * s->capacity : s->T * s->k;
}

static int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  return dev;
}

// SM count of the current device, queried once per device.
static int num_sms() {
  static std::atomic<int> cache[64];
  const int dev = current_device();
  if (dev < 0 || dev >= 64) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  n = 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Router split-K so that small-T, wide-d routers still fill the GPU.
static int router_splits(const moe_shape* s, int* k_per_split) {
  const long long ctas = cdiv(s->T, kLgBM) * cdiv(s->E, kLgBN);
  int ns = 1;
  const long long want = 2ll * num_sms();
  if (ctas < want) ns = (int)std::min<long long>(cdiv(want, ctas), std::max(1, s->d / 256));
  int kps = (int)cdiv(cdiv(s->d, ns), kLgBK) * kLgBK;
  ns = (int)cdiv(s->d, kps);
  *k_per_split = kps;
  return ns;
}

// ------------------------------------------------------------------ workspace layout

struct Workspace {
  size_t part, wsplit, wnorm, xcs, xrs, xq, i4part, cnt, psum, idx, w, counts, fP, slot, drop, kept, offs, xperm, h, yperm, hs, ys, shtab;
  size_t cidx, ncand, zmax, snc, zex, ecount, elist, xnorm2;   // certified selection over the screening logits
  size_t total;
};

// Split-reduction partials of the INT4 shared expert (decode batches: T <= 256): up to 8 ranges of
// T x max(2 H_s, d) fp32.
static size_t i4part_floats(const moe_shape* s) {
  if (s->wfmt != MOE_WFMT_INT4_G128 || s->H_s == 0 || s->T > 256) return 0;
  return (size_t)8 * s->T * std::max(2 * s->H_s, s->d);
}

static bool use_tc_router(const moe_shape* s);

static Workspace ws_layout(const moe_shape* s) {
  Workspace L{};
  int kps = 0;
  const int ns = router_splits(s, &kps);
  const long long nchunks = cdiv(s->T, kChunk);
  const long long R = grouped_rows(s);
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align256(o + bytes); return at; };
  L.part = take((size_t)ns * s->T * s->E * 4);
  L.wsplit = take((size_t)2 * s->E * s->d * 2);
  L.wnorm = take((size_t)s->E * 4);
  // routed rows, then the shared expert's token rows (its copy is written with the routed one)
  const long long xs_rows = grouped_rows(s) + s->T;   // rows of xs_cols elements
  const int xs_cols = std::max(s->d, std::max(s->H, s->H_s));
  L.xcs = take(s->wfmt == MOE_WFMT_INT4_G128 ? (size_t)xs_rows * (xs_cols / 128) * 4 : 16);
  L.xrs = take(s->wfmt == MOE_WFMT_INT4_G128 ? (size_t)xs_rows * 4 : 16);
  L.xq = take(s->wfmt == MOE_WFMT_INT4_G128 ? (size_t)xs_rows * xs_cols * 2 : 16);
  L.i4part = take(i4part_floats(s) * 4 + 16);
  L.cnt = take((size_t)nchunks * s->E * 4);
  L.psum = take((size_t)nchunks * s->E * 4);
  L.idx = take((size_t)s->T * s->k * 4);
  L.w = take((size_t)s->T * s->k * 4);
  L.counts = take((size_t)s->E * 4);
  L.fP = take((size_t)2 * s->E * 4 + 16);
  L.slot = take((size_t)s->T * s->k * 4);
  L.drop = take((size_t)s->T * s->k);
  L.kept = take((size_t)s->E * 4);
  L.offs = take((size_t)(s->E + 1) * 4);
  L.xperm = take((size_t)R * s->d * 2);
  L.h = take((size_t)R * s->H * 2);
  L.yperm = take((size_t)R * s->d * 2);
  L.hs = take((size_t)s->T * std::max(s->H_s, 16) * 2);
  L.ys = take((size_t)s->T * s->d * 2);
  L.shtab = take(64);
  L.cidx = take((size_t)s->T * kSelMaxCand);
  L.ncand = take((size_t)s->T * 4);
  L.zmax = take((size_t)s->T * 4);
  L.snc = take((size_t)s->T * 4);
  L.zex = take((size_t)s->T * kSelMaxCand * 4);
  L.ecount = take((size_t)s->E * 4);
  L.xnorm2 = take((size_t)s->T * 4);
  L.elist = use_tc_router(s) ? take((size_t)s->E * s->T * 4) : take(16);
  L.total = o;
  return L;
}

// ------------------------------------------------------------------ TMA descriptors

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tensor [outer..., rows, K] (K innermost), box = 64 x box_rows (x 1).
static int make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, int box_rows) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return MOE_CUDA_ERROR;
  cuuint64_t strides[2];
  strides[0] = dims[0] * 2;
  if (rank == 3) strides[1] = dims[0] * dims[1] * 2;
  cuuint32_t box[3] = {(cuuint32_t)kBK, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_CUDA_ERROR;
}

template <int MODE, int BN, int CG>
static int launch_gemm_t(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p, long long ub_mtiles,
                         cudaStream_t st) {
  using Cfg = GemmCfg<BN, CG, MODE == kModeScreen ? 2 : 1>;
  constexpr int OUTN = (MODE == kModeSwiGLU || MODE == kModeGeGLU) ? BN / 2 : BN;
  // the shared-memory opt-in is set once per device for each instantiation
  static std::atomic<unsigned long long> done_mask{0};
  const int dev = current_device();
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(done_mask.load(std::memory_order_relaxed) & bit)) {
    MOE_CUDA_TRY(cudaFuncSetAttribute(k_grouped_gemm<MODE, BN, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)Cfg::kSmemBytes));
    done_mask.fetch_or(bit);
  }
  const long long tiles = ub_mtiles * cdiv(p.N, OUTN);
  if (CG == 1) {
    const int grid = (int)std::max<long long>(1, std::min<long long>(num_sms(), tiles));
    MOE_LAUNCH((k_grouped_gemm<MODE, BN, 1>), grid, 256, Cfg::kSmemBytes, st, ta, tb, p);
  } else {
    // clusters of 2 CTAs, one pair per two SMs
    const int pairs = (int)std::max<long long>(1, std::min<long long>(num_sms() / 2, tiles));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cfg.stream = st;
    MOE_CUDA_TRY(launch_pdl(k_grouped_gemm<MODE, BN, CG>, cfg.gridDim, cfg.blockDim, cfg.dynamicSmemBytes, st, 2u,
                            ta, tb, p));
  }
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

// CTA pairs (M = 256 tiles) for the bf16 expert GEMMs when the groups are large enough
// to fill them: on average at least 192 rows per group.
static bool use_pair_gemm(int mode, int BN, long long R, int n_groups, bool allow_pair) {
  return allow_pair && mode != kModeScreen && BN == 256 && R >= 192ll * n_groups;
}

// out[R, N] = epilogue(A[R, K] . B_g^T) over groups.  B is [n_groups, b_rows, K].
// Column tile: 256, 128 or 64, the one with the least modelled time = waves x time per tile.  Per k-step a
// tile costs max(MMA, operand traffic): the MMA scales with BN, the L2 -> SM traffic with 128 + BN rows,
// which measured about 1.1 MMA-column units per row on B200 (a 128 x 256 tile runs at ~60% of the tensor
// peak).  Narrow tiles are therefore only chosen where they cut the number of waves substantially.
static int pick_bn(bool glu, int N, long long mtiles) {
  const int sms = num_sms();
  int best = 0;
  double best_cost = 0.0;
  for (int bn : {256, 128, 64}) {
    const int outn = glu ? bn / 2 : bn;
    if (bn > 64 && outn / 2 >= N) continue;  // mostly padding
    const long long tiles = mtiles * cdiv(N, outn);
    const double per_tile = std::max((double)bn, 1.1 * (128.0 + bn));
    const double cost = (double)cdiv(tiles, sms) * per_tile;
    if (best == 0 || cost < best_cost * 0.97) { best = bn; best_cost = cost; }
  }
  return best == 0 ? 64 : best;
}

// Mode-specific inputs of grouped_gemm beyond the operands.
struct GemmExtras {
  const float* bias = nullptr;       // router screen: per-expert logit bias
};

static int grouped_gemm(int mode, const void* A, long long R, int K, const void* B, int n_groups, int b_rows,
                        int up_row0, int N, const int32_t* gstart, const int32_t* grows, void* out,
                        cudaStream_t st, bool allow_pair, const GemmExtras& ex = GemmExtras{}) {
  if (R == 0) return MOE_OK;
  const bool glu = mode == kModeSwiGLU || mode == kModeGeGLU;
  const long long ub_m = grows ? (R / kBM + n_groups) : cdiv(R, kBM);
  // router screen: one column tile as wide as the expert count (fewer A re-reads); CTA pairs (256-row tiles,
  // half the B tiles per CTA) once the batch fills a wave of single-CTA tiles
  const bool router = mode == kModeScreen;
  const int BN = router ? (N <= 64 ? 64 : N <= 128 ? 128 : N <= 192 ? 192 : 256) : pick_bn(glu, N, ub_m);
  const bool pair = router ? (allow_pair && R >= (long long)kBM * num_sms())
                           : use_pair_gemm(mode, BN, R, n_groups, allow_pair);
  const int box_rows = (glu || pair) ? BN / 2 : BN;
  CUtensorMap ta, tb;
  cuuint64_t da[2] = {(cuuint64_t)K, (cuuint64_t)R};
  cuuint64_t db[3] = {(cuuint64_t)(router ? 2 * K : K), (cuuint64_t)b_rows, (cuuint64_t)n_groups};
  int rc = make_map(&ta, A, 2, da, kBM);
  if (rc) return rc;
  rc = make_map(&tb, B, 3, db, box_rows);
  if (rc) return rc;
  GemmParams p;
  p.group_start = gstart;
  p.group_rows = grows;
  p.n_groups = n_groups;
  p.R = R;
  p.K = K;
  p.N = N;
  p.up_row0 = up_row0;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.ldo = N;
  p.wait_limit_ns = g_wait_limit_ns.load();
  p.out_f32 = reinterpret_cast<float*>(out);
  p.bias = ex.bias;
  const long long ub = grows ? (R / kBM + n_groups) : cdiv(R, kBM);
  if (pair) {
    const long long ub2 = grows ? (R / (2 * kBM) + n_groups) : cdiv(R, 2 * kBM);
    if (mode == kModePlain) return launch_gemm_t<kModePlain, 256, 2>(ta, tb, p, ub2, st);
    if (mode == kModeSwiGLU) return launch_gemm_t<kModeSwiGLU, 256, 2>(ta, tb, p, ub2, st);
    if (mode == kModeGeGLU) return launch_gemm_t<kModeGeGLU, 256, 2>(ta, tb, p, ub2, st);
    if (mode == kModeScreen && BN == 256) return launch_gemm_t<kModeScreen, 256, 2>(ta, tb, p, ub2, st);
    if (mode == kModeScreen && BN == 192) return launch_gemm_t<kModeScreen, 192, 2>(ta, tb, p, ub2, st);
    if (mode == kModeScreen && BN == 128) return launch_gemm_t<kModeScreen, 128, 2>(ta, tb, p, ub2, st);
    if (mode == kModeScreen && BN == 64) return launch_gemm_t<kModeScreen, 64, 2>(ta, tb, p, ub2, st);
    return MOE_UNSUPPORTED_SHAPE;
  }
#define MOE_GEMM_CASE(M_, BN_) \
  if (mode == M_ && BN == BN_) return launch_gemm_t<M_, BN_, 1>(ta, tb, p, ub, st);
  MOE_GEMM_CASE(kModePlain, 256) MOE_GEMM_CASE(kModePlain, 128) MOE_GEMM_CASE(kModePlain, 64)
  MOE_GEMM_CASE(kModeSwiGLU, 256) MOE_GEMM_CASE(kModeSwiGLU, 128) MOE_GEMM_CASE(kModeSwiGLU, 64)
  MOE_GEMM_CASE(kModeGeGLU, 256) MOE_GEMM_CASE(kModeGeGLU, 128) MOE_GEMM_CASE(kModeGeGLU, 64)
  MOE_GEMM_CASE(kModeScreen, 256) MOE_GEMM_CASE(kModeScreen, 192) MOE_GEMM_CASE(kModeScreen, 128)
  MOE_GEMM_CASE(kModeScreen, 64)
#undef MOE_GEMM_CASE
  return MOE_UNSUPPORTED_SHAPE;
}

// ------------------------------------------------------------------ launch helpers

// Selection kernel.  Large batches: one CTA of 8 warps per 32-token chunk, chunk tables formed in the kernel.
// Small batches (T <= 2048): 4 tokens per CTA so the tokens spread over the SMs; the probabilities are written
// to p_scratch (which may be `part` itself: each warp writes its row after reading it) and k_chunk_stats forms
// the chunk tables.
static int launch_topk(const moe_shape* s, const float* part, int nsplit, const float* bias, float* logits,
                       int32_t* idx, float* w, int32_t* cnt, float* psum, float* p_scratch, cudaStream_t st,
                       RefineArgs refine = RefineArgs{nullptr, nullptr, nullptr, nullptr, 0, 0.f}) {
  const int nchunks = (int)cdiv(s->T, kChunk);
  const int epl = (int)cdiv(s->E, 32);
  const bool small = s->T <= 2048;
  // the certifying recompute holds the token's inputs in registers when d <= 1024
  const bool xreg = refine.x != nullptr && refine.d <= 1024;
  // warps per CTA: small batches 4 tokens per CTA, so that the tokens spread over the SMs (tables by
  // k_chunk_stats); large batches 8 warps per 32-token chunk with the chunk tables formed in the kernel
  const int nw = small ? 4 : 8;
#define MOE_TOPK_CASE(N_, NW_, XR_, ST_)                                                                          \
  if (epl <= N_ && nw == NW_ && xreg == XR_) {                                                                    \
    const size_t smem = ST_ ? (size_t)2 * NW_ * s->E * sizeof(float) : 0;                                         \
    if (smem > 48 * 1024) {                                                                                       \
      static std::atomic<unsigned long long> attr_done{0};                                                        \
      const unsigned long long bit = 1ull << (current_device() & 63);                                             \
      if (!(attr_done.load() & bit)) {                                                                            \
        MOE_CUDA_TRY(cudaFuncSetAttribute(k_router_topk<N_, NW_, XR_, ST_>,                                       \
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,                           \
                                          2 * NW_ * kMaxRouterE * (int)sizeof(float)));                           \
        attr_done.fetch_or(bit);                                                                                  \
      }                                                                                                           \
    }                                                                                                             \
    const unsigned grid = ST_ ? (unsigned)nchunks : (unsigned)cdiv(s->T, NW_);                                    \
    MOE_LAUNCH((k_router_topk<N_, NW_, XR_, ST_>), grid, NW_ * 32, smem, st, part, nsplit, bias, logits, idx, w, cnt, psum,  \
                                                                   psum ? p_scratch : nullptr, (int)s->T, s->E,  \
                                                                   s->k, s->renorm, refine);                      \
    MOE_LAUNCH_CHECK();                                                                                           \
    if (!ST_) {                                                                                                   \
      MOE_LAUNCH((k_chunk_stats), nchunks, 256, 0, st, idx, p_scratch, cnt, psum, (int)s->T, s->E, s->k);                   \
      MOE_LAUNCH_CHECK();                                                                                         \
    }                                                                                                             \
    return MOE_OK;                                                                                                \
  }
#define MOE_TOPK_EPL(NW_, XR_, ST_)                                                                               \
  MOE_TOPK_CASE(1, NW_, XR_, ST_) MOE_TOPK_CASE(2, NW_, XR_, ST_) MOE_TOPK_CASE(4, NW_, XR_, ST_)                 \
  MOE_TOPK_CASE(6, NW_, XR_, ST_) MOE_TOPK_CASE(8, NW_, XR_, ST_) MOE_TOPK_CASE(12, NW_, XR_, ST_)                \
  MOE_TOPK_CASE(16, NW_, XR_, ST_)
  MOE_TOPK_EPL(8, false, true) MOE_TOPK_EPL(8, true, true) MOE_TOPK_EPL(4, false, false) MOE_TOPK_EPL(4, true, false)
#undef MOE_TOPK_EPL
#undef MOE_TOPK_CASE
  return MOE_UNSUPPORTED_SHAPE;
}

static int launch_scan(const moe_shape* s, int32_t* cnt, const float* psum, int32_t* counts, float* f, float* P,
                       cudaStream_t st) {
  const int nchunks = (int)cdiv(s->T, kChunk);
  MOE_LAUNCH((k_chunk_scan), s->E, 256, 0, st, cnt, psum, counts, f, P, nchunks, s->E, (int)s->T);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

static int launch_scatter(const moe_shape* s, const void* x, const int32_t* idx, const int32_t* cbase,
                          const int32_t* counts, int32_t* slot, uint8_t* drop, int32_t* row_src, void* x_perm,
                          int32_t* kept, int32_t* offs, cudaStream_t st, bool move_rows = true,
                          const float* aux_f = nullptr, const float* aux_p = nullptr, float* aux = nullptr) {
  const int nchunks = (int)cdiv(s->T, kChunk);
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  __nv_bfloat16* xp = reinterpret_cast<__nv_bfloat16*>(x_perm);
  const unsigned mv_blocks = (unsigned)cdiv(s->T * (long long)(s->d / 8), 256);
#define MOE_SCATTER_CASE(N_)                                                                                  \
  if (s->k <= N_) {                                                                                           \
    MOE_LAUNCH((k_scatter<N_>), (unsigned)cdiv(nchunks, 4), 128, 0, st, xb, idx, cbase, counts, (int)s->T, s->d, s->E,   \
                                                              s->k, s->capacity,                              \
                                           slot, drop, row_src, xp, kept, offs, aux_f, aux_p, aux);           \
    MOE_LAUNCH_CHECK();                                                                                       \
    if (move_rows) {                                                                                          \
      MOE_LAUNCH((k_move_rows<N_>), mv_blocks, 256, 0, st, xb, slot, (int)s->T, s->d, s->k, xp);                       \
      MOE_LAUNCH_CHECK();                                                                                     \
    }                                                                                                         \
    return MOE_OK;                                                                                            \
  }
  MOE_SCATTER_CASE(2) MOE_SCATTER_CASE(4) MOE_SCATTER_CASE(8) MOE_SCATTER_CASE(16)
#undef MOE_SCATTER_CASE
  return MOE_UNSUPPORTED_SHAPE;
}

// Fused routed expert FFN (bf16, hidden 128 or 256): h stays in shared memory.  y [R, d] bf16.
template <int MODE, int H, int CG>
static int launch_fused_t(const void* A, long long R, int d, const void* w13, const void* w2, int n_groups,
                          const int32_t* gstart, const int32_t* grows, void* y, cudaStream_t st) {
  using Cfg = FusedCfg<H, CG>;
  static std::atomic<unsigned long long> done_mask{0};
  const unsigned long long bit = 1ull << (current_device() & 63);
  if (!(done_mask.load(std::memory_order_relaxed) & bit)) {
    MOE_CUDA_TRY(cudaFuncSetAttribute(k_expert_fused<MODE, H, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)Cfg::kSmemBytes));
    done_mask.fetch_or(bit);
  }
  CUtensorMap tx, t13, t2;
  const cuuint64_t dx[2] = {(cuuint64_t)d, (cuuint64_t)R};
  const cuuint64_t d13[3] = {(cuuint64_t)d, (cuuint64_t)(2 * H), (cuuint64_t)n_groups};
  const cuuint64_t d2[3] = {(cuuint64_t)H, (cuuint64_t)d, (cuuint64_t)n_groups};
  int rc = make_map(&tx, A, 2, dx, kBM);
  if (rc) return rc;
  rc = make_map(&t13, w13, 3, d13, 128);
  if (rc) return rc;
  rc = make_map(&t2, w2, 3, d2, CG == 2 ? 128 : 256);
  if (rc) return rc;
  GemmParams p{};
  p.group_start = gstart;
  p.group_rows = grows;
  p.n_groups = n_groups;
  p.R = R;
  p.K = d;
  p.N = d;
  p.up_row0 = H;
  p.out = reinterpret_cast<__nv_bfloat16*>(y);
  p.ldo = d;
  p.wait_limit_ns = g_wait_limit_ns.load();
  const long long TM = (long long)kBM * CG;
  const long long tiles = grows ? (R / TM + n_groups) : cdiv(R, TM);
  const int units = (int)std::max<long long>(1, std::min<long long>(num_sms() / CG, tiles));
  MOE_CUDA_TRY(launch_pdl(k_expert_fused<MODE, H, CG>, dim3((unsigned)(CG * units)), dim3(256), Cfg::kSmemBytes, st,
                          (unsigned)CG, tx, t13, t2, p));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

static bool fused_ffn_ok(const moe_shape* s, int hidden) {
  return s->wfmt == MOE_WFMT_BF16 && (hidden == 128 || hidden == 256);
}

static int launch_fused(const moe_shape* s, int hidden, long long R, const void* A, const int32_t* gstart,
                        const int32_t* grows, int n_groups, const void* w13, const void* w2, void* y,
                        cudaStream_t st) {
  if (R == 0) return MOE_OK;
  const bool pair = !(s->flags & MOE_FLAG_SINGLE_CTA_GEMM) && R >= 192ll * n_groups;
  const bool geglu = s->act == MOE_ACT_GEGLU;
#define MOE_FUSED_FFN(M_, H_, CG_) \
  if ((M_ == kModeGeGLU) == geglu && hidden == H_ && (CG_ == 2) == pair) \
    return launch_fused_t<M_, H_, CG_>(A, R, s->d, w13, w2, n_groups, gstart, grows, y, st);
  MOE_FUSED_FFN(kModeSwiGLU, 256, 2) MOE_FUSED_FFN(kModeSwiGLU, 256, 1) MOE_FUSED_FFN(kModeSwiGLU, 128, 2)
  MOE_FUSED_FFN(kModeSwiGLU, 128, 1) MOE_FUSED_FFN(kModeGeGLU, 256, 2) MOE_FUSED_FFN(kModeGeGLU, 256, 1)
  MOE_FUSED_FFN(kModeGeGLU, 128, 2) MOE_FUSED_FFN(kModeGeGLU, 128, 1)
#undef MOE_FUSED_FFN
  return MOE_UNSUPPORTED_SHAPE;
}

// Optional scratch for the offset-code kernel, written by k_int4_act_prep: xcs [R, K/128] (the offsets' share
// of each group), xrs [R] (row scales 2^e) and xq [R, K] f16 (the scaled, fragment-ordered copy of A).
// Without it the exact-code kernel runs.
struct Int4Scratch {
  float* xcs;
  float* xrs;
  void* xq;
  float* part = nullptr;        // split-reduction partials (dense groups with few tasks), or none
  size_t part_floats = 0;
  // grouping of a routed batch: the activation copy is formed from the token rows (src_x, src_T tokens) and
  // slot_pos directly, with no bf16 grouped copy in between (the first GEMM of the routed FFN only)
  const void* src_x = nullptr;
  long long src_T = 0;
  const int32_t* slot_pos = nullptr;
  int slot_k = 0;
  const Int4Scratch* also = nullptr;   // with slot_pos: also write token t's copy to row t of these buffers
  bool prepped = false;         // xcs, xrs, xq already hold this GEMM's activations: no preparation launch
};

static int int4_gemm(bool glu, int act, const void* A, long long R, int K, const void* wq, const void* wsc,
                     int n_groups, int b_rows, int up_row0, int N, const int32_t* gstart, const int32_t* grows,
                     void* out, cudaStream_t st, Int4Scratch scr = Int4Scratch{nullptr, nullptr, nullptr}) {
  float* xcs = scr.xq != nullptr ? scr.xcs : nullptr;
  float* xrs = scr.xrs;
  if (R == 0) return MOE_OK;
  Int4Params p;
  p.wq = reinterpret_cast<const uint8_t*>(wq);
  p.ws = reinterpret_cast<const __nv_bfloat16*>(wsc);
  p.act = reinterpret_cast<const __nv_bfloat16*>(A);
  p.group_start = gstart;
  p.group_rows = grows;
  p.n_groups = n_groups;
  p.R = R;
  p.K = K;
  p.N = N;
  p.b_rows = b_rows;
  p.up_row0 = up_row0;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.ldo = N;
  p.ksplit = 1;
  p.part = nullptr;
  // A single dense group with too few (16 or 32 rows x 8 tokens) tasks to occupy every warp of every SM
  // (the shared expert of a decode batch) splits each task's reduction into contiguous slab ranges; fp32
  // partials go to scratch and k_int4_splitk_reduce adds them in order.
  {
    const long long base = (long long)(N / (glu ? 16 : 32)) * cdiv(R, 8);
    const long long warps = (long long)num_sms() * kI4Warps;
    const int nslab = (int)cdiv(K, 256);
    if (grows == nullptr && scr.part != nullptr && scr.xq != nullptr && base < warps) {
      const int ks = (int)std::min<long long>(std::min(nslab / 2, 8), cdiv(2 * warps, base));
      if (ks > 1 && (size_t)ks * R * (glu ? 2 * N : N) <= scr.part_floats) {
        p.ksplit = ks;
        p.part = scr.part;
      }
    }
  }
  {
    // 2-D byte map over all experts' packed rows; box = 16 rows x 128 bytes (256 inputs)
    EncodeTiledFn enc = get_encoder();
    if (!enc) return MOE_CUDA_ERROR;
    CUtensorMap tm;
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)n_groups * (cuuint64_t)b_rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {128, 16};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(wq), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MOE_CUDA_ERROR;
    const int dev = current_device();
    const unsigned long long bit = 1ull << (dev & 63);
    static std::atomic<unsigned long long> done{0};
    if (!(done.load() & bit)) {
#define MOE_I4_ATTR(G_, A_, O_, S_)                                                                          \
      MOE_CUDA_TRY(cudaFuncSetAttribute(k_int4_stream<G_, A_, O_, S_>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                        kI4Smem));
      MOE_I4_ATTR(false, kModePlain, false, false) MOE_I4_ATTR(true, kModeSwiGLU, false, false)
      MOE_I4_ATTR(true, kModeGeGLU, false, false) MOE_I4_ATTR(false, kModePlain, true, false)
      MOE_I4_ATTR(true, kModeSwiGLU, true, false) MOE_I4_ATTR(true, kModeGeGLU, true, false)
      MOE_I4_ATTR(false, kModePlain, true, true) MOE_I4_ATTR(true, kModeSwiGLU, true, true)
      MOE_I4_ATTR(true, kModeGeGLU, true, true)
#undef MOE_I4_ATTR
      MOE_CUDA_TRY(cudaFuncSetAttribute(k_int4_dense<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kI4DSmem));
      MOE_CUDA_TRY(cudaFuncSetAttribute(k_int4_dense<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kI4DSmem));
      done.fetch_or(bit);
    }
    if (xcs != nullptr && !scr.prepped) {
      const int pt = (int)std::min<long long>(1024, std::max<long long>(64, cdiv(K / 8, 32) * 32));
      if (scr.slot_pos != nullptr)
        MOE_LAUNCH((k_int4_act_prep), (unsigned)scr.src_T, pt, 0, st, reinterpret_cast<const __nv_bfloat16*>(scr.src_x),
                   K, xcs, xrs, reinterpret_cast<__half*>(scr.xq), scr.slot_pos, scr.slot_k,
                   scr.also ? scr.also->xcs : nullptr, scr.also ? scr.also->xrs : nullptr,
                   scr.also ? reinterpret_cast<__half*>(scr.also->xq) : nullptr);
      else
        MOE_LAUNCH((k_int4_act_prep), (unsigned)R, pt, 0, st, reinterpret_cast<const __nv_bfloat16*>(A), K, xcs, xrs,
                   reinterpret_cast<__half*>(scr.xq), (const int32_t*)nullptr, 0, (float*)nullptr, (float*)nullptr,
                   (__half*)nullptr);
      MOE_LAUNCH_CHECK();
    }
    if (xcs != nullptr) p.act = reinterpret_cast<const __nv_bfloat16*>(scr.xq);   // f16 bytes: raw fragments
    if (grows == nullptr && xcs != nullptr && scr.part != nullptr && R <= 256) {
      // one dense group of a small batch (the shared expert of a decode batch): CTA tasks of kI4DWarps weight
      // blocks over 64 rows, each weight dequantised once per 64 rows; the reduction split so that the tasks
      // fill the SMs once (a second partial round would double the time)
      const long long base = cdiv(N / (glu ? 16 : 32), kI4DWarps) * cdiv(R, kI4DRows);
      int ks = (int)std::min<long long>(std::min<long long>(8, cdiv(K, 256)), std::max<long long>(1, num_sms() / base));
      while (ks > 1 && (size_t)ks * R * (glu ? 2 * N : N) > scr.part_floats) --ks;
      if ((size_t)ks * R * (glu ? 2 * N : N) <= scr.part_floats) {
        p.ksplit = ks;
        p.part = scr.part;
        const int grid = (int)std::max<long long>(1, std::min<long long>(num_sms(), base * ks));
        const unsigned long long lim = g_wait_limit_ns.load();
        if (glu) MOE_LAUNCH((k_int4_dense<true>), grid, kI4DWarps * 32, kI4DSmem, st, tm, p, lim, xcs, xrs);
        else MOE_LAUNCH((k_int4_dense<false>), grid, kI4DWarps * 32, kI4DSmem, st, tm, p, lim, xcs, xrs);
        MOE_LAUNCH_CHECK();
        const unsigned blocks = (unsigned)cdiv(R * N, 256);
        __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out);
        if (!glu) MOE_LAUNCH((k_int4_splitk_reduce<false, kModePlain>), blocks, 256, 0, st, p.part, p.ksplit, R, N, o);
        else if (act == MOE_ACT_SWIGLU)
          MOE_LAUNCH((k_int4_splitk_reduce<true, kModeSwiGLU>), blocks, 256, 0, st, p.part, p.ksplit, R, N, o);
        else MOE_LAUNCH((k_int4_splitk_reduce<true, kModeGeGLU>), blocks, 256, 0, st, p.part, p.ksplit, R, N, o);
        MOE_LAUNCH_CHECK();
        return MOE_OK;
      }
    }
    const long long rows_per_task = glu ? 16 : 32;
    const long long ub = (long long)(N / rows_per_task) * (grows ? cdiv(R, 8) + n_groups : cdiv(R, 8)) * p.ksplit;
    const int grid = (int)std::max<long long>(1, std::min<long long>(num_sms(), cdiv(ub, kI4Warps)));
    const unsigned long long lim = g_wait_limit_ns.load();
    const int nt = kI4Warps * 32;
#define MOE_I4_LAUNCH(G_, A_, O_, S_) \
  MOE_LAUNCH((k_int4_stream<G_, A_, O_, S_>), grid, nt, kI4Smem, st, tm, p, lim, xcs, xrs)
    if (xcs != nullptr && p.ksplit > 1) {
      if (!glu) MOE_I4_LAUNCH(false, kModePlain, true, true);
      else if (act == MOE_ACT_SWIGLU) MOE_I4_LAUNCH(true, kModeSwiGLU, true, true);
      else MOE_I4_LAUNCH(true, kModeGeGLU, true, true);
    } else if (xcs != nullptr) {
      if (!glu) MOE_I4_LAUNCH(false, kModePlain, true, false);
      else if (act == MOE_ACT_SWIGLU) MOE_I4_LAUNCH(true, kModeSwiGLU, true, false);
      else MOE_I4_LAUNCH(true, kModeGeGLU, true, false);
    } else {
      if (!glu) MOE_I4_LAUNCH(false, kModePlain, false, false);
      else if (act == MOE_ACT_SWIGLU) MOE_I4_LAUNCH(true, kModeSwiGLU, false, false);
      else MOE_I4_LAUNCH(true, kModeGeGLU, false, false);
    }
#undef MOE_I4_LAUNCH
    MOE_LAUNCH_CHECK();
    if (p.ksplit > 1) {
      const unsigned blocks = (unsigned)cdiv(R * N, 256);
      __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out);
      if (!glu) MOE_LAUNCH((k_int4_splitk_reduce<false, kModePlain>), blocks, 256, 0, st, p.part, p.ksplit, R, N, o);
      else if (act == MOE_ACT_SWIGLU)
        MOE_LAUNCH((k_int4_splitk_reduce<true, kModeSwiGLU>), blocks, 256, 0, st, p.part, p.ksplit, R, N, o);
      else MOE_LAUNCH((k_int4_splitk_reduce<true, kModeGeGLU>), blocks, 256, 0, st, p.part, p.ksplit, R, N, o);
      MOE_LAUNCH_CHECK();
    }
    return MOE_OK;
  }
}

// Gated expert FFN over groups of rows: h = act(A W1^T) * (A W3^T), y = h W2^T.
// scr (optional, INT4 only): scratch of at least R * max(d, hidden) / 128 floats (group sums) and
// R * max(d, hidden) bf16 (fragment-ordered activations).
static int expert_ffn_impl(const moe_shape* s, int hidden, long long R, const void* A, const int32_t* gstart,
                           const int32_t* grows, int n_groups, const void* w13, const void* s13, const void* w2,
                           const void* s2, void* h, void* y, cudaStream_t st,
                           Int4Scratch scr = Int4Scratch{nullptr, nullptr, nullptr}) {
  int rc;
  if (s->wfmt == MOE_WFMT_INT4_G128) {
    rc = int4_gemm(true, s->act, A, R, s->d, w13, s13, n_groups, 2 * hidden, hidden, hidden, gstart, grows, h, st,
                   scr);
    if (rc) return rc;
    Int4Scratch scr2 = scr;
    scr2.slot_pos = nullptr;   // h is already grouped
    scr2.prepped = false;
    return int4_gemm(false, s->act, h, R, hidden, w2, s2, n_groups, s->d, 0, s->d, gstart, grows, y, st, scr2);
  }
  if (h == nullptr) return launch_fused(s, hidden, R, A, gstart, grows, n_groups, w13, w2, y, st);
  const int mode = s->act == MOE_ACT_SWIGLU ? kModeSwiGLU : kModeGeGLU;
  const bool pair = !(s->flags & MOE_FLAG_SINGLE_CTA_GEMM);
  rc = grouped_gemm(mode, A, R, s->d, w13, n_groups, 2 * hidden, hidden, hidden, gstart, grows, h, st, pair);
  if (rc) return rc;
  return grouped_gemm(kModePlain, h, R, hidden, w2, n_groups, s->d, 0, s->d, gstart, grows, y, st, pair);
}

// Fused CUDA-core router when W_r^T fits in shared memory: returns its experts-per-lane template, else 0.
// Lane-per-token router for E <= 16 (W_r^T as [d][EC + 4] fp32 in shared memory, at most 160 KiB).  Wider
// expert counts use the expert-per-lane router: every lane busy, no shared-memory bank conflicts.
static int lanes_router_ec(const moe_shape* s) {
  const int ec = s->E <= 8 ? 8 : s->E <= 16 ? 16 : 0;
  if (ec == 0 || (size_t)s->d * (ec + 4) * 4 > 160 * 1024) return 0;
  return ec;
}

static int launch_lanes_router(const moe_shape* s, int ec, const void* x, const float* w_router, const float* bias,
                               float* logits, int32_t* idx, float* w, int32_t* cnt, float* psum, cudaStream_t st) {
  // 4 lanes per token when one lane per token would leave SMs idle or the chains long (E * d FMAs each)
  const int kp = (cdiv(s->T, 256) < 2 * num_sms() || (long long)ec * s->d > 4096) ? 4 : 1;
  const size_t smem = (size_t)s->d * (ec + 4) * 4;
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  const int dev = current_device();
  const unsigned long long bit = 1ull << (dev & 63);
#define MOE_LANES_CASE(N_, KP_)                                                                                    \
  if (ec == N_ && kp == KP_) {                                                                                    \
    static std::atomic<unsigned long long> done{0};                                                               \
    if (!(done.load() & bit)) {                                                                                   \
      MOE_CUDA_TRY(cudaFuncSetAttribute(k_router_lanes<N_, KP_>, cudaFuncAttributeMaxDynamicSharedMemorySize,      \
                                        160 * 1024));                                                             \
      done.fetch_or(bit);                                                                                         \
    }                                                                                                             \
    MOE_LAUNCH((k_router_lanes<N_, KP_>), (unsigned)cdiv(s->T, 256 / KP_), 256, smem, st, xb, w_router, bias,      \
               logits, idx, w, cnt, psum, (int)s->T, s->d, s->E, s->k, s->renorm);                                \
    MOE_LAUNCH_CHECK();                                                                                           \
    return MOE_OK;                                                                                                \
  }
  MOE_LANES_CASE(8, 1) MOE_LANES_CASE(16, 1) MOE_LANES_CASE(8, 4) MOE_LANES_CASE(16, 4)
#undef MOE_LANES_CASE
  return MOE_UNSUPPORTED_SHAPE;
}

static int fused_router_epl(const moe_shape* s) {
  if (s->E > 256) return 0;
  const int epl = s->E <= 32 ? 1 : s->E <= 64 ? 2 : s->E <= 128 ? 4 : 8;
  const size_t bytes = (size_t)s->d * (epl * 32 + 1) * 4;
  return bytes <= 160 * 1024 ? epl : 0;
}

static int launch_fused_router(const moe_shape* s, int epl, const void* x, const float* w_router, const float* bias,
                               float* logits, int32_t* idx, float* w, int32_t* cnt, float* psum, cudaStream_t st) {
  const int nchunks = (int)cdiv(s->T, kChunk);
  const size_t smem = (size_t)s->d * (epl * 32 + 1) * 4;
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  const int dev = current_device();
  const unsigned long long bit = 1ull << (dev & 63);
#define MOE_FUSED_CASE(N_)                                                                                        \
  if (epl == N_) {                                                                                                \
    static std::atomic<unsigned long long> done{0};                                                               \
    if (!(done.load() & bit)) {                                                                                   \
      MOE_CUDA_TRY(cudaFuncSetAttribute(k_router_fused<N_, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize,        \
                                        160 * 1024));                                                             \
      done.fetch_or(bit);                                                                                         \
    }                                                                                                             \
    MOE_LAUNCH((k_router_fused<N_, 8>), nchunks, 256, smem, st, xb, w_router, bias, logits, idx, w, cnt, psum, (int)s->T,    \
                                                      s->d, s->E, s->k, s->renorm);                               \
    MOE_LAUNCH_CHECK();                                                                                           \
    return MOE_OK;                                                                                                \
  }
  MOE_FUSED_CASE(1) MOE_FUSED_CASE(2) MOE_FUSED_CASE(4) MOE_FUSED_CASE(8)
#undef MOE_FUSED_CASE
  return MOE_UNSUPPORTED_SHAPE;
}

// Large routers go to the tensor cores as an exact three-way bf16 split of W_r
// (fp32 accumulation); small ones stay on the fp32 CUDA-core GEMM.
// Decode router: dynamic shared memory of the staged x slice (16 tokens x one input slice, fp32).
static constexpr size_t kSkinnyMaxSmem = 100 * 1024;
static std::atomic<unsigned long long> g_skinny_attr{0};   // per-device bit: shared-memory opt-in done
static size_t skinny_smem(int d) { return (size_t)kSkTok * skinny_slice(d) * sizeof(float); }

static bool use_tc_router(const moe_shape* s) {
  return s->E % 16 == 0 && s->d % 64 == 0 && (double)s->T * s->E * s->d >= (double)(1ll << 28);
}

// True when route_impl, asked for neither logits nor statistics, takes the tensor-core screen and selection
// path: the screen's fp32 logits (bias included) are then left in the workspace at L.part, [T, E].
static bool route_keeps_screen(const moe_shape* s) {
  return lanes_router_ec(s) == 0 && fused_router_epl(s) == 0 && use_tc_router(s) && s->E <= 256 &&
         s->d <= kSelMaxD;
}

static int route_impl(const moe_shape* s, const void* x, const float* w_router, const float* bias,
                      const float* logits_in, float* logits, int32_t* idx, float* w, int32_t* counts, float* aux_f,
                      float* aux_p, float* aux, uint8_t* ws, cudaStream_t st, bool defer_aux = false) {
  const Workspace L = ws_layout(s);
  float* part = reinterpret_cast<float*>(ws + L.part);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  float* psum = reinterpret_cast<float*>(ws + L.psum);
  float* f = aux_f ? aux_f : reinterpret_cast<float*>(ws + L.fP);
  float* P = aux_p ? aux_p : reinterpret_cast<float*>(ws + L.fP) + s->E;
  int rc;
  int nsplit = 1;
  // chunk probability sums only when the load-balance statistic (f, P or aux) is requested
  const bool want_fp = aux_f || aux_p || aux;
  float* psum_w = want_fp ? psum : nullptr;
  const int ec_lanes = lanes_router_ec(s);
  const int epl_fused = fused_router_epl(s);
  if (logits_in == nullptr && ec_lanes > 0) {
    rc = launch_lanes_router(s, ec_lanes, x, w_router, bias, logits, idx, w, cnt, psum_w, st);
  } else if (logits_in == nullptr && epl_fused > 0) {
    rc = launch_fused_router(s, epl_fused, x, w_router, bias, logits, idx, w, cnt, psum_w, st);
  } else if (logits_in == nullptr && use_tc_router(s)) {
    __nv_bfloat16* wsplit = reinterpret_cast<__nv_bfloat16*>(ws + L.wsplit);
    float* wnorm = reinterpret_cast<float*>(ws + L.wnorm);
    // screening bound, relative to ||x_t|| max_e ||w_e|| (>= sum |x_i w_i|): the split's representation error
    // 2^-16, fp32 accumulation of 2d products in any rounding direction plus the bias add, and the error of the
    // exact recompute's own d-term fp32 chain; all with a 2^-7 margin
    const float gamma = (float)((std::ldexp(1.0, -16) + (2.0 * s->d + 2.0) * std::ldexp(1.0, -23) +
                                 (s->d + 2.0) * std::ldexp(1.0, -24)) *
                                (1.0 + std::ldexp(1.0, -7)));
    const bool want_stats = aux_f || aux_p || aux;
    // without logits or statistics to return, the selection lists candidates and recomputes them by expert
    const bool select = logits == nullptr && !want_stats && s->E <= 256 && s->d <= kSelMaxD;
    int32_t* ecount = reinterpret_cast<int32_t*>(ws + L.ecount);
    float* xnorm2 = reinterpret_cast<float*>(ws + L.xnorm2);
    MOE_LAUNCH((k_router_prep), (unsigned)(cdiv(s->E, 8) + (select ? cdiv(s->T, 8) : 0)), 256, 0, st, w_router, wsplit,
               wnorm, s->E, s->d, select ? ecount : nullptr, s->E,
               select ? reinterpret_cast<const __nv_bfloat16*>(x) : nullptr, xnorm2, (int)s->T);
    MOE_LAUNCH_CHECK();
    GemmExtras ex;
    ex.bias = bias;
    rc = grouped_gemm(kModeScreen, x, s->T, s->d, wsplit, 1, s->E, 0, s->E, nullptr, nullptr, part, st,
                      !(s->flags & MOE_FLAG_SINGLE_CTA_GEMM), ex);
    if (rc) return rc;
    if (select) {
      SelectArgs sa{part, xnorm2, reinterpret_cast<const __nv_bfloat16*>(x), wnorm, gamma, (int)s->T, s->d, s->E, s->k,
                    reinterpret_cast<uint8_t*>(ws + L.cidx), reinterpret_cast<int32_t*>(ws + L.ncand),
                    reinterpret_cast<float*>(ws + L.zmax), reinterpret_cast<float*>(ws + L.snc), ecount,
                    reinterpret_cast<int32_t*>(ws + L.elist), cnt};
      const unsigned nch = (unsigned)cdiv(s->T, kChunk);
      const int epl = s->E <= 64 ? 2 : s->E <= 128 ? 4 : s->E <= 192 ? 6 : 8;
      if (epl == 2) MOE_LAUNCH((k_router_select<2>), nch, 256, 0, st, sa);
      else if (epl == 4) MOE_LAUNCH((k_router_select<4>), nch, 256, 0, st, sa);
      else if (epl == 6) MOE_LAUNCH((k_router_select<6>), nch, 256, 0, st, sa);
      else MOE_LAUNCH((k_router_select<8>), nch, 256, 0, st, sa);
      MOE_LAUNCH_CHECK();
      float* zex = reinterpret_cast<float*>(ws + L.zex);
      // 16-byte input slices per lane (d <= kSelMaxD: at most 8); entries per batch and resident CTAs chosen so
      // that the input loads of a batch and the W_r slices fit the registers
      const int vpl = (int)cdiv(s->d / 8, 32);
#define MOE_RECOMP(V_, N_, M_)                                                                                \
  MOE_LAUNCH((k_router_recompute<V_, N_, M_>), (unsigned)(M_ * num_sms()), 256, 0, st,                        \
             reinterpret_cast<const __nv_bfloat16*>(x), w_router, bias, ecount, sa.elist, zex, (int)s->T, s->d, s->E)
      switch (vpl) {
        case 1: MOE_RECOMP(1, 8, 3); break;
        case 2: MOE_RECOMP(2, 4, 3); break;
        case 3: MOE_RECOMP(3, 4, 2); break;
        case 4: MOE_RECOMP(4, 4, 2); break;
        case 5: MOE_RECOMP(5, 3, 2); break;
        case 6: MOE_RECOMP(6, 2, 2); break;
        case 7: MOE_RECOMP(7, 1, 2); break;
        default: MOE_RECOMP(8, 1, 2); break;
      }
#undef MOE_RECOMP
      MOE_LAUNCH_CHECK();
      const unsigned nfin = (unsigned)cdiv(s->T, 32);
#define MOE_FINISH(N_)                                                                                        \
  MOE_LAUNCH((k_router_finish<N_>), nfin, 256, 0, st, sa.ncand, sa.cidx, zex, sa.zmax, sa.snc, sa.x, w_router, bias, \
             idx, w, cnt, (int)s->T, s->d, s->E, s->k, s->renorm)
      if (epl == 2) MOE_FINISH(2);
      else if (epl == 4) MOE_FINISH(4);
      else if (epl == 6) MOE_FINISH(6);
      else MOE_FINISH(8);
#undef MOE_FINISH
      MOE_LAUNCH_CHECK();
      rc = MOE_OK;
    } else {
      RefineArgs ref{reinterpret_cast<const __nv_bfloat16*>(x), w_router, bias, wnorm, s->d, gamma};
      rc = launch_topk(s, part, 1, nullptr, logits, idx, w, cnt, psum_w, part, st, ref);
    }
  } else if (logits_in == nullptr && s->T <= 256 && skinny_smem(s->d) <= kSkinnyMaxSmem) {
    const unsigned long long bit = 1ull << (current_device() & 63);
    if (!(g_skinny_attr.load() & bit)) {
      MOE_CUDA_TRY(cudaFuncSetAttribute(k_router_skinny, cudaFuncAttributeMaxDynamicSharedMemorySize, kSkinnyMaxSmem));
      g_skinny_attr.fetch_or(bit);
    }
    dim3 grid((unsigned)cdiv(s->E, 8 * kSkExp), (unsigned)cdiv(s->T, kSkTok), kSkSplit);
    MOE_LAUNCH((k_router_skinny), grid, 256, skinny_smem(s->d), st, reinterpret_cast<const __nv_bfloat16*>(x), w_router, part,
                                                           (int)s->T, s->d, s->E);
    MOE_LAUNCH_CHECK();
    rc = launch_topk(s, part, 1, bias, logits, idx, w, cnt, psum_w, part, st);
  } else if (logits_in == nullptr) {
    int kps = 0;
    nsplit = router_splits(s, &kps);
    dim3 grid((unsigned)cdiv(s->T, kLgBM), (unsigned)cdiv(s->E, kLgBN), (unsigned)nsplit);
    MOE_LAUNCH((k_router_logits), grid, 128, 0, st, reinterpret_cast<const __nv_bfloat16*>(x), w_router, part, (int)s->T,
                                          s->d, s->E, kps);
    MOE_LAUNCH_CHECK();
    rc = launch_topk(s, part, nsplit, bias, logits, idx, w, cnt, psum_w, part, st);
  } else {
    rc = launch_topk(s, logits_in, 1, nullptr, nullptr, idx, w, cnt, psum_w, part, st);
  }
  if (rc) return rc;
  rc = launch_scan(s, cnt, want_fp ? psum : nullptr, counts, want_fp ? f : nullptr, want_fp ? P : nullptr, st);
  if (rc) return rc;
  if (aux && !defer_aux) {   // deferred: the caller's grouping kernel forms aux from f and P
    MOE_LAUNCH((k_aux_finalize), 1, 32, 0, st, f, P, aux, s->E);
    MOE_LAUNCH_CHECK();
  }
  return MOE_OK;
}


// ------------------------------------------------------------------ backward (input gradient)

// Row splits of a dense weight gradient (one group of `rows` rows).  The time goes as the waves of tiles times
// the rows per split, so n minimises ceil(n tiles / 148) / n over 1 <= n <= min(32, rows / 512), the fewest
// splits among equals (fewer partials to add).  148 is B200's SM count; the rule does not ask the device, so
// that the workspace size does not depend on it either.
struct WgradSplit {
  int n, chunk;
};
static int wgrad_bn(int N) { return N >= 256 ? 256 : (N > 64 ? 128 : 64); }
// rows per chunk of a hot expert's weight gradient (32 reduction steps of 64 rows)
constexpr int kWgradSplitRows = 2048;
static WgradSplit wgrad_split(long long rows, int M, int N) {
  const long long tiles = cdiv(M, kBM) * cdiv(N, wgrad_bn(N));
  const long long nmax = std::max<long long>(1, std::min<long long>(32, rows / 512));
  long long n = 1;
  for (long long c = 2; c <= nmax; ++c)   // waves(c) / c < waves(n) / n
    if (cdiv(c * tiles, 148) * n < cdiv(n * tiles, 148) * c) n = c;
  const long long chunk = cdiv(cdiv(rows, n), 64) * 64;
  return WgradSplit{(int)cdiv(rows, chunk), (int)chunk};
}

// Scratch of moe_backward_x past the forward's regions (which it reuses: routing, grouping, x_perm for dx of the
// grouped rows, h for dh').
struct BwdWorkspace {
  size_t gu, doutp, gus, dhs, dxs, logits, dw, dz, wrt, dxr, part, partsh, wpart, wlist, total;
  int ldE;   // columns of dz and W_r^T: E rounded up to whole 64-column reduction steps
};

static BwdWorkspace bwd_layout(const moe_shape* s) {
  const Workspace F = ws_layout(s);
  BwdWorkspace B{};
  const long long R = grouped_rows(s);
  size_t o = F.total;
  auto take = [&](size_t bytes) { size_t at = o; o = align256(o + bytes); return at; };
  B.ldE = (int)((s->E + 63) / 64 * 64);
  B.gu = take((size_t)R * 2 * s->H * 2);
  B.doutp = take((size_t)R * s->d * 2);
  B.gus = take((size_t)s->T * 2 * std::max(s->H_s, 16) * 2);
  B.dhs = take((size_t)s->T * std::max(s->H_s, 16) * 2);
  B.dxs = take((size_t)s->T * s->d * 2);
  B.logits = take((size_t)s->T * s->E * 4);
  B.dw = take((size_t)s->T * s->k * 4);
  B.dz = take((size_t)s->T * B.ldE * 2);
  B.wrt = take((size_t)s->d * B.ldE * 2);
  B.dxr = take((size_t)s->T * s->d * 2);
  // split partials of the dense weight gradients: the router's, and (apart, since the shared expert's chain may
  // run on a second stream) the shared expert's two
  auto need = [&](int M, int N) {
    const WgradSplit sp = wgrad_split(s->T, M, N);
    return sp.n > 1 ? (size_t)sp.n * M * N * 4 : (size_t)0;
  };
  B.part = take(need(s->E, s->d));
  B.partsh = take(s->H_s > 0 ? std::max(need(2 * s->H_s, s->d), need(s->d, s->H_s)) : 0);
  // chunk partials of hot experts' weight gradients: the chunks of groups above kWgradSplitRows rows number at
  // most 2 R / kWgradSplitRows (each such group adds at most one partial chunk beyond R / kWgradSplitRows)
  B.wpart = take((size_t)2 * cdiv(R, kWgradSplitRows) * std::max(2 * s->H, s->H) * s->d * 4);
  B.wlist = take((size_t)(1 + 3 * s->E) * 4);
  B.total = o;
  return B;
}

static int launch_glu_bwd(int act, void* gu, void* dh, long long rows, int H, bool write_h, cudaStream_t st) {
  const unsigned blocks = (unsigned)cdiv(rows * (H / 8), 256);
  if (act == MOE_ACT_SWIGLU)
    MOE_LAUNCH((k_glu_bwd<kModeSwiGLU>), blocks, 256, 0, st, reinterpret_cast<__nv_bfloat16*>(gu),
               reinterpret_cast<__nv_bfloat16*>(dh), rows, H, (int)write_h);
  else
    MOE_LAUNCH((k_glu_bwd<kModeGeGLU>), blocks, 256, 0, st, reinterpret_cast<__nv_bfloat16*>(gu),
               reinterpret_cast<__nv_bfloat16*>(dh), rows, H, (int)write_h);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

static int launch_glu_bwd_slots(int act, void* gu, void* dhp, const int32_t* slot, const float* w,
                                long long n_slots, int H, bool write_wh, float* dw, cudaStream_t st) {
  const unsigned blocks = (unsigned)cdiv(n_slots, 8);
  if (act == MOE_ACT_SWIGLU)
    MOE_LAUNCH((k_glu_bwd_slots<kModeSwiGLU>), blocks, 256, 0, st, reinterpret_cast<__nv_bfloat16*>(gu),
               reinterpret_cast<__nv_bfloat16*>(dhp), slot, w, n_slots, H, (int)write_wh, dw);
  else
    MOE_LAUNCH((k_glu_bwd_slots<kModeGeGLU>), blocks, 256, 0, st, reinterpret_cast<__nv_bfloat16*>(gu),
               reinterpret_cast<__nv_bfloat16*>(dhp), slot, w, n_slots, H, (int)write_wh, dw);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

// Copy row t of src to the grouped row of each of its kept slots (the row move of the dispatch, for any [T, d]
// bf16 tensor).
static int launch_move_rows(const moe_shape* s, const void* src, const int32_t* slot, void* dst, cudaStream_t st) {
  const unsigned blocks = (unsigned)cdiv(s->T * (long long)(s->d / 8), 256);
  const __nv_bfloat16* a = reinterpret_cast<const __nv_bfloat16*>(src);
  __nv_bfloat16* b = reinterpret_cast<__nv_bfloat16*>(dst);
  if (s->k <= 2) MOE_LAUNCH((k_move_rows<2>), blocks, 256, 0, st, a, slot, (int)s->T, s->d, s->k, b);
  else if (s->k <= 4) MOE_LAUNCH((k_move_rows<4>), blocks, 256, 0, st, a, slot, (int)s->T, s->d, s->k, b);
  else if (s->k <= 8) MOE_LAUNCH((k_move_rows<8>), blocks, 256, 0, st, a, slot, (int)s->T, s->d, s->k, b);
  else MOE_LAUNCH((k_move_rows<16>), blocks, 256, 0, st, a, slot, (int)s->T, s->d, s->k, b);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

// ------------------------------------------------------------------ weight gradients

template <int BN>
static int launch_wgrad_t(const CUtensorMap& ta, const CUtensorMap& tb, const WgradParams& p, cudaStream_t st) {
  using Cfg = WgradCfg<BN>;
  static std::atomic<unsigned long long> done_mask{0};
  const int dev = current_device();
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(done_mask.load(std::memory_order_relaxed) & bit)) {
    MOE_CUDA_TRY(cudaFuncSetAttribute(k_wgrad_gemm<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)Cfg::kSmemBytes));
    done_mask.fetch_or(bit);
  }
  const long long tiles = cdiv(p.M, kBM) * cdiv(p.N, BN) * p.G;
  const int grid = (int)std::max<long long>(1, std::min<long long>(num_sms(), tiles));
  MOE_LAUNCH((k_wgrad_gemm<BN>), grid, 256, Cfg::kSmemBytes, st, ta, tb, p);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

// out[g] [M, N] fp32 = A_g^T B_g over the rows of group g, A [R, lda] and B [R, N] bf16 row-major (columns
// M .. lda of A are not read into the output).  Groups: (gstart, grows) [G] on the device, or nullptr: one
// group of all R rows, split by wgrad_split into partials in `part` (>= n * M * N floats) summed into out.
static int wgrad_gemm(const void* A, int lda, int M, const void* B, int N, long long R, const int32_t* gstart,
                      const int32_t* grows, int G, float* out, float* part, cudaStream_t st, int split_rows = 0,
                      int32_t* split_list = nullptr) {
  if (N % 8 || lda % 8 || lda < M) return MOE_UNSUPPORTED_SHAPE;   // 16-byte row strides for TMA
  CUtensorMap ta, tb;
  cuuint64_t da[2] = {(cuuint64_t)lda, (cuuint64_t)std::max<long long>(R, 1)};
  cuuint64_t db[2] = {(cuuint64_t)N, (cuuint64_t)std::max<long long>(R, 1)};
  int rc = make_map(&ta, A, 2, da, 64);
  if (rc) return rc;
  rc = make_map(&tb, B, 2, db, 64);
  if (rc) return rc;
  WgradParams p;
  p.group_start = gstart;
  p.group_rows = grows;
  p.R = R;
  p.M = M;
  p.N = N;
  p.out_stride = (long long)M * N;
  p.wait_limit_ns = g_wait_limit_ns.load();
  p.split_rows = gstart != nullptr ? split_rows : 0;
  p.part = part;
  p.split_list = gstart != nullptr && split_rows > 0 ? split_list : nullptr;
  WgradSplit sp{1, (int)std::max<long long>(R, 1)};
  if (gstart == nullptr) {
    sp = wgrad_split(R, M, N);
    p.G = sp.n;
    p.chunk = sp.chunk;
    p.out = sp.n > 1 ? part : out;
  } else {
    p.G = G;
    p.chunk = 0;
    p.out = out;
  }
  const int BN = wgrad_bn(N);
  if (BN == 256) rc = launch_wgrad_t<256>(ta, tb, p, st);
  else if (BN == 128) rc = launch_wgrad_t<128>(ta, tb, p, st);
  else rc = launch_wgrad_t<64>(ta, tb, p, st);
  if (rc) return rc;
  if (gstart == nullptr && sp.n > 1) {
    const long long n = (long long)M * N;
    MOE_LAUNCH((k_sum_splits), (unsigned)cdiv(n / 4, 256), 256, 0, st, part, sp.n, n, out);
    MOE_LAUNCH_CHECK();
  }
  if (p.split_list != nullptr) {   // the hot groups' chunks (the list may be empty)
    MOE_LAUNCH((k_wgrad_reduce), (unsigned)(4 * num_sms()), 256, 0, st, part, split_list, (long long)M * N, out);
    MOE_LAUNCH_CHECK();
  }
  return MOE_OK;
}

// ------------------------------------------------------------------ hierarchical router

// E = branch^levels checked without overflow; the tree's own limits (the full layer's grouping keeps E <= 512).
static int check_tree(const moe_shape* s, int branch, int levels) {
  if (s == nullptr) return MOE_INVALID_ARGUMENT;
  if (s->T < 1 || s->T > (1ll << 24)) return MOE_UNSUPPORTED_SHAPE;
  if (s->d < 16 || s->d % 16 != 0 || s->d > 65536) return MOE_UNSUPPORTED_SHAPE;
  if (s->k < 1 || s->k > 16) return MOE_UNSUPPORTED_SHAPE;
  if (s->renorm != 0 && s->renorm != 1) return MOE_INVALID_ARGUMENT;
  if (branch < 2 || branch > kTreeMaxBranch || levels < 1) return MOE_UNSUPPORTED_SHAPE;
  const int n = branch * levels;
  if (n > kTreeMaxLogits || n % 4 != 0) return MOE_UNSUPPORTED_SHAPE;
  long long E = 1;
  for (int l = 0; l < levels; ++l) {
    E *= branch;
    if (E > kTreeMaxE) return MOE_UNSUPPORTED_SHAPE;
  }
  if (E != s->E) return MOE_INVALID_ARGUMENT;
  if (s->k > s->E) return MOE_INVALID_ARGUMENT;
  return MOE_OK;
}

struct TreeWorkspace {
  size_t wsplit, wnorm, z, total;
};

static TreeWorkspace tree_layout(const moe_shape* s, int n) {
  TreeWorkspace W{};
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align256(o + bytes); return at; };
  W.wsplit = take((size_t)2 * n * s->d * 2);
  W.wnorm = take((size_t)n * 4);
  W.z = take((size_t)s->T * n * 4);
  W.total = o;
  return W;
}

// Fork of independent work onto a caller's second stream: an event recorded on `main` that `side` waits for,
// and a join event (owned here, released however the call returns) that `main` waits for later.
struct SideFork {
  cudaEvent_t join = nullptr;
  ~SideFork() { if (join != nullptr) cudaEventDestroy(join); }
  int start(cudaStream_t main, cudaStream_t side) {
    cudaEvent_t fork = nullptr;
    if (cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess) return MOE_CUDA_ERROR;
    const bool ok = cudaEventCreateWithFlags(&join, cudaEventDisableTiming) == cudaSuccess &&
                    cudaEventRecord(fork, main) == cudaSuccess && cudaStreamWaitEvent(side, fork, 0) == cudaSuccess;
    cudaEventDestroy(fork);
    return ok ? MOE_OK : MOE_CUDA_ERROR;
  }
  int end(cudaStream_t side) { return cudaEventRecord(join, side) == cudaSuccess ? MOE_OK : MOE_CUDA_ERROR; }
  int wait(cudaStream_t main) { return cudaStreamWaitEvent(main, join, 0) == cudaSuccess ? MOE_OK : MOE_CUDA_ERROR; }
};

}  // namespace moe

using namespace moe;

// ====================================================================== C ABI

extern "C" {

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_INVALID_ARGUMENT: return "invalid argument";
    case MOE_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_CUDA_ERROR: return "CUDA error";
    case MOE_DEVICE_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

uint64_t moe_launch_count(void) { return g_launches.load(); }

int moe_set_wait_limit_ns(uint64_t ns) {
  if (ns == 0) return MOE_INVALID_ARGUMENT;
  g_wait_limit_ns.store(ns);
  return MOE_OK;
}

int64_t moe_grouped_rows(const moe_shape* s) { return s ? grouped_rows(s) : -1; }

int moe_capacity(int64_t T, int32_t k, int32_t E, double factor, int32_t* capacity) {
  if (!capacity || T < 1 || k < 1 || E < 1 || !std::isfinite(factor)) return MOE_INVALID_ARGUMENT;
  if (factor <= 0.0) { *capacity = 0; return MOE_OK; }
  // factor as an exact decimal num / 10^6, then C = ceil(num * T * k / (10^6 * E)) in integers
  const long long num = llround(factor * 1e6);
  const __int128 top = (__int128)num * T * k;
  const __int128 den = (__int128)1000000 * E;
  const __int128 c = (top + den - 1) / den;
  if (c > (1ll << 30)) return MOE_UNSUPPORTED_SHAPE;
  *capacity = (int32_t)c;
  return MOE_OK;
}

int moe_workspace_size(const moe_shape* s, size_t* bytes) {
  if (!bytes) return MOE_INVALID_ARGUMENT;
  int rc = check_shape(s);
  if (rc) return rc;
  *bytes = ws_layout(s).total;
  return MOE_OK;
}

int moe_route(const moe_shape* s, const void* x, const float* w_router, const float* bias, float* logits,
              int32_t* topk_idx, float* topk_w, int32_t* counts, float* aux_f, float* aux_p, float* aux,
              void* workspace, size_t ws_bytes, moe_stream_t stream) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (!x || !w_router || !topk_idx || !topk_w || !counts || !workspace) return MOE_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(workspace)) return MOE_INVALID_ARGUMENT;
  if (ws_bytes < ws_layout(s).total) return MOE_WORKSPACE_TOO_SMALL;
  return route_impl(s, x, w_router, bias, nullptr, logits, topk_idx, topk_w, counts, aux_f, aux_p, aux,
                    reinterpret_cast<uint8_t*>(workspace), stream);
}

int moe_route_from_logits(const moe_shape* s, const float* logits, int32_t* topk_idx, float* topk_w,
                          int32_t* counts, float* aux_f, float* aux_p, float* aux, void* workspace,
                          size_t ws_bytes, moe_stream_t stream) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (!logits || !topk_idx || !topk_w || !counts || !workspace) return MOE_INVALID_ARGUMENT;
  if (!aligned16(workspace)) return MOE_INVALID_ARGUMENT;
  if (ws_bytes < ws_layout(s).total) return MOE_WORKSPACE_TOO_SMALL;
  return route_impl(s, nullptr, nullptr, nullptr, logits, nullptr, topk_idx, topk_w, counts, aux_f, aux_p, aux,
                    reinterpret_cast<uint8_t*>(workspace), stream);
}

int moe_permute(const moe_shape* s, const void* x, const int32_t* topk_idx, int32_t* slot_pos,
                uint8_t* drop_mask, int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* row_src,
                void* x_perm, void* workspace, size_t ws_bytes, moe_stream_t stream) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (!x || !topk_idx || !slot_pos || !kept || !offsets || !x_perm || !workspace) return MOE_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(x_perm) || !aligned16(workspace)) return MOE_INVALID_ARGUMENT;
  const Workspace L = ws_layout(s);
  if (ws_bytes < L.total) return MOE_WORKSPACE_TOO_SMALL;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  int32_t* cts = counts ? counts : reinterpret_cast<int32_t*>(ws + L.counts);
  const int nchunks = (int)cdiv(s->T, kChunk);
  MOE_LAUNCH((k_chunk_hist), nchunks, 256, s->E * sizeof(int), stream, topk_idx, cnt, (int)s->T, s->E, s->k);
  MOE_LAUNCH_CHECK();
  rc = launch_scan(s, cnt, nullptr, cts, nullptr, nullptr, stream);
  if (rc) return rc;
  return launch_scatter(s, x, topk_idx, cnt, cts, slot_pos, drop_mask, row_src, x_perm, kept, offsets, stream);
}

int moe_expert_ffn(const moe_shape* s, int32_t n_groups, int32_t hidden, int64_t R, const void* x_grouped,
                   const int32_t* group_start, const int32_t* group_rows, const void* w13, const void* s13,
                   const void* w2, const void* s2, void* h, void* y, moe_stream_t stream) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (n_groups < 1 || n_groups > kMaxGroupsSmem || R < 0 || R >= (1ll << 31) - 256) return MOE_INVALID_ARGUMENT;
  if (hidden < 16 || hidden % 16 != 0) return MOE_UNSUPPORTED_SHAPE;
  if ((group_start == nullptr) != (group_rows == nullptr)) return MOE_INVALID_ARGUMENT;
  if (group_start == nullptr && n_groups != 1) return MOE_INVALID_ARGUMENT;
  if (R == 0) return MOE_OK;
  if (!x_grouped || !w13 || !w2 || !y) return MOE_INVALID_ARGUMENT;
  if (h == nullptr && !fused_ffn_ok(s, hidden)) return MOE_INVALID_ARGUMENT;
  if (!aligned16(x_grouped) || !aligned16(w13) || !aligned16(w2) || (h && !aligned16(h)) || !aligned16(y))
    return MOE_INVALID_ARGUMENT;
  if (s->wfmt == MOE_WFMT_INT4_G128) {
    if (hidden % 128 != 0) return MOE_UNSUPPORTED_SHAPE;
    if (!s13 || !s2 || !aligned16(s13) || !aligned16(s2)) return MOE_INVALID_ARGUMENT;
  }
  return expert_ffn_impl(s, hidden, R, x_grouped, group_start, group_rows, n_groups, w13, s13, w2, s2, h, y,
                         stream);
}

int moe_combine(const moe_shape* s, const void* y_perm, const int32_t* slot_pos, const float* topk_w,
                const void* y_shared, void* out, moe_stream_t stream) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (!y_perm || !slot_pos || !topk_w || !out) return MOE_INVALID_ARGUMENT;
  if (!aligned16(y_perm) || !aligned16(out) || (y_shared && !aligned16(y_shared))) return MOE_INVALID_ARGUMENT;
  const __nv_bfloat16* yp = reinterpret_cast<const __nv_bfloat16*>(y_perm);
  const __nv_bfloat16* ysh = reinterpret_cast<const __nv_bfloat16*>(y_shared);
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out);
  // 8 tokens per CTA; the columns split into ranges of whole 32-lane sweeps until there are about two CTAs
  // per SM (a decode batch of 64 tokens would otherwise occupy 8 SMs)
  const unsigned tok_blocks = (unsigned)cdiv(s->T, 8);
  const int sweeps = (int)cdiv(s->d / 8, 32);
  const int ranges = (int)std::max<long long>(1, std::min<long long>(sweeps, cdiv(2ll * num_sms(), tok_blocks)));
  const int vpr = (int)cdiv(sweeps, ranges) * 32;
  const dim3 grid(tok_blocks, (unsigned)cdiv(s->d / 8, vpr));
#define MOE_COMBINE_CASE(N_)                                                                                   \
  if (s->k <= N_) {                                                                                            \
    MOE_LAUNCH((k_combine<N_>), grid, 256, 0, stream, yp, slot_pos, topk_w, ysh, o, (int)s->T, s->d, s->k, vpr);   \
    MOE_LAUNCH_CHECK();                                                                                        \
    return MOE_OK;                                                                                             \
  }
  MOE_COMBINE_CASE(2) MOE_COMBINE_CASE(4) MOE_COMBINE_CASE(8) MOE_COMBINE_CASE(16)
#undef MOE_COMBINE_CASE
  return MOE_UNSUPPORTED_SHAPE;
}

int moe_forward(const moe_shape* s, const void* x, const float* w_router, const float* bias, const void* w13,
                const void* s13, const void* w2, const void* s2, const void* w13_sh, const void* s13_sh,
                const void* w2_sh, const void* s2_sh, void* out, int32_t* topk_idx, float* topk_w,
                int32_t* counts, uint8_t* drop_mask, float* aux_f, float* aux_p, float* aux, void* workspace,
                size_t ws_bytes, moe_stream_t stream, moe_stream_t side_stream) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (!x || !w_router || !w13 || !w2 || !out || !workspace) return MOE_INVALID_ARGUMENT;
  if (s->H_s > 0 && (!w13_sh || !w2_sh)) return MOE_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(w13) || !aligned16(w2) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return MOE_INVALID_ARGUMENT;
  if (s->wfmt == MOE_WFMT_INT4_G128 &&
      (!s13 || !s2 || !aligned16(s13) || !aligned16(s2) || (s->H_s > 0 && (!s13_sh || !s2_sh))))
    return MOE_INVALID_ARGUMENT;
  const Workspace L = ws_layout(s);
  if (ws_bytes < L.total) return MOE_WORKSPACE_TOO_SMALL;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  int32_t* idx = topk_idx ? topk_idx : reinterpret_cast<int32_t*>(ws + L.idx);
  float* w = topk_w ? topk_w : reinterpret_cast<float*>(ws + L.w);
  int32_t* cts = counts ? counts : reinterpret_cast<int32_t*>(ws + L.counts);
  int32_t* slot = reinterpret_cast<int32_t*>(ws + L.slot);
  int32_t* kept = reinterpret_cast<int32_t*>(ws + L.kept);
  int32_t* offs = reinterpret_cast<int32_t*>(ws + L.offs);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  void* xperm = ws + L.xperm;
  void* hbuf = ws + L.h;
  void* yperm = ws + L.yperm;
  const long long R = grouped_rows(s);
  const bool int4 = s->wfmt == MOE_WFMT_INT4_G128;

  // bf16 experts: the shared expert needs only x, so with a side stream it runs there from the start, beside the
  // routing, grouping and routed experts, and joins before the combine.  (INT4: its activation copy is formed
  // with the routed one, so it stays in order.)
  void* ys = nullptr;
  SideFork fork;
  const bool forked = s->H_s > 0 && !int4 && side_stream != nullptr && side_stream != stream;
  if (forked) {
    rc = fork.start(stream, side_stream);
    if (rc) return rc;
    ys = ws + L.ys;
    rc = expert_ffn_impl(s, s->H_s, s->T, x, nullptr, nullptr, 1, w13_sh, s13_sh, w2_sh, s2_sh, ws + L.hs, ys,
                         side_stream, Int4Scratch{nullptr, nullptr, nullptr});
    if (rc) return rc;
    rc = fork.end(side_stream);
    if (rc) return rc;
  }

  rc = route_impl(s, x, w_router, bias, nullptr, nullptr, idx, w, cts, aux_f, aux_p, aux, ws, stream, true);
  if (rc) return rc;
  const float* f_used = aux_f ? aux_f : reinterpret_cast<const float*>(ws + L.fP);
  const float* p_used = aux_p ? aux_p : reinterpret_cast<const float*>(ws + L.fP) + s->E;
  // INT4: the grouped activation copy is formed by k_int4_act_prep from x and the slots, so no bf16 rows move
  rc = launch_scatter(s, x, idx, cnt, cts, slot, drop_mask, nullptr, xperm, kept, offs, stream, !int4, f_used, p_used,
                      aux);
  if (rc) return rc;
  const Int4Scratch scr = int4 ? Int4Scratch{reinterpret_cast<float*>(ws + L.xcs), reinterpret_cast<float*>(ws + L.xrs),
                                             ws + L.xq, reinterpret_cast<float*>(ws + L.i4part), i4part_floats(s)}
                               : Int4Scratch{nullptr, nullptr, nullptr};
  Int4Scratch scr_routed = scr, scr_shared = scr;
  if (int4) {
    scr_routed.src_x = x;
    scr_routed.src_T = s->T;
    scr_routed.slot_pos = slot;
    scr_routed.slot_k = s->k;
    if (s->H_s > 0) {
      // the shared expert's input copy, written with the routed one: past the R routed rows of the widest
      // reduction, so that the routed down GEMM's own copy (R rows of H) leaves it intact
      const long long cols = std::max(s->d, std::max(s->H, s->H_s));
      scr_shared.xcs = scr.xcs + (size_t)R * (cols / 128);
      scr_shared.xrs = scr.xrs + R;
      scr_shared.xq = reinterpret_cast<__half*>(scr.xq) + (size_t)R * cols;
      scr_shared.prepped = true;
      scr_routed.also = &scr_shared;
    }
  }
  rc = expert_ffn_impl(s, s->H, R, xperm, offs, kept, s->E, w13, s13, w2, s2, hbuf, yperm, stream, scr_routed);
  if (rc) return rc;
  if (s->H_s > 0 && !forked) {
    ys = ws + L.ys;
    rc = expert_ffn_impl(s, s->H_s, s->T, x, nullptr, nullptr, 1, w13_sh, s13_sh, w2_sh, s2_sh, ws + L.hs, ys,
                         stream, scr_shared);
    if (rc) return rc;
  }
  if (forked && (rc = fork.wait(stream))) return rc;
  return moe_combine(s, yperm, slot, w, ys, out, stream);
}

int moe_transpose_experts(const void* w, int64_t n, int32_t rows, int32_t cols, void* wt, moe_stream_t stream) {
  if (!w || !wt || n < 1 || n > 65535 || rows < 1 || cols < 1) return MOE_INVALID_ARGUMENT;
  const dim3 grid((unsigned)cdiv(cols, 32), (unsigned)cdiv(rows, 32), (unsigned)n);
  MOE_LAUNCH((k_transpose_bf16), grid, dim3(32, 8), 0, stream, reinterpret_cast<const __nv_bfloat16*>(w),
             reinterpret_cast<__nv_bfloat16*>(wt), (int)rows, (int)cols);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

int moe_backward_workspace_size(const moe_shape* s, size_t* bytes) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (!bytes) return MOE_INVALID_ARGUMENT;
  *bytes = bwd_layout(s).total;
  return MOE_OK;
}

int moe_backward(const moe_shape* s, const void* x, const float* w_router, const float* bias, const void* w13,
                 const void* w13t, const void* w2t, const void* w13_sh, const void* w13t_sh, const void* w2t_sh,
                 const void* dout, float aux_coef, float* dx, float* dw13, float* dw2, float* dw13_sh,
                 float* dw2_sh, float* dw_router, void* workspace, size_t ws_bytes, moe_stream_t stream,
                 moe_stream_t side_stream) {
  int rc = check_shape(s);
  if (rc) return rc;
  if (s->wfmt != MOE_WFMT_BF16) return MOE_UNSUPPORTED_SHAPE;
  if (!x || !w_router || !w13 || !w13t || !w2t || !dout || !dx || !workspace) return MOE_INVALID_ARGUMENT;
  if (s->H_s > 0 && (!w13_sh || !w13t_sh || !w2t_sh)) return MOE_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(w13) || !aligned16(w13t) || !aligned16(w2t) ||
      !aligned16(dout) || !aligned16(dx) || !aligned16(dw13) || !aligned16(dw2) || !aligned16(dw13_sh) ||
      !aligned16(dw2_sh) || !aligned16(dw_router) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return MOE_INVALID_ARGUMENT;
  const Workspace L = ws_layout(s);
  const BwdWorkspace B = bwd_layout(s);
  if (ws_bytes < B.total) return MOE_WORKSPACE_TOO_SMALL;
  cudaStream_t st = stream;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + L.idx);
  float* w = reinterpret_cast<float*>(ws + L.w);
  int32_t* cts = reinterpret_cast<int32_t*>(ws + L.counts);
  int32_t* slot = reinterpret_cast<int32_t*>(ws + L.slot);
  uint8_t* drop = reinterpret_cast<uint8_t*>(ws + L.drop);
  int32_t* kept = reinterpret_cast<int32_t*>(ws + L.kept);
  int32_t* offs = reinterpret_cast<int32_t*>(ws + L.offs);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  void* xperm = ws + L.xperm;   // the grouped rows, then dx of the grouped rows
  void* hbuf = ws + L.h;        // dh' = dout W2 of the grouped rows, then w h
  void* gu = ws + B.gu;         // [g | u] of the grouped rows, then [dg | du]
  void* doutp = ws + B.doutp;   // dout of the grouped rows
  float* logits = reinterpret_cast<float*>(ws + B.logits);
  float* dwb = reinterpret_cast<float*>(ws + B.dw);
  __nv_bfloat16* dz = reinterpret_cast<__nv_bfloat16*>(ws + B.dz);
  __nv_bfloat16* wrt = reinterpret_cast<__nv_bfloat16*>(ws + B.wrt);
  void* dxr = ws + B.dxr;
  float* part = reinterpret_cast<float*>(ws + B.part);
  const long long R = grouped_rows(s);
  const bool pair = !(s->flags & MOE_FLAG_SINGLE_CTA_GEMM);

  // shared expert on the tokens: [g | u] recomputed, dh = dout W2, [dg | du] (and h), its weight gradients,
  // dx = [dg | du] W13.  It depends on the inputs only: with a side stream it runs there, beside the routed
  // chain, from a fork event on `stream`, and joins before the final sum.
  void* dxs = nullptr;
  SideFork fork;
  const bool forked = s->H_s > 0 && side_stream != nullptr && side_stream != stream;
  if (s->H_s > 0) {
    cudaStream_t sst = st;
    if (forked) {
      rc = fork.start(st, side_stream);
      if (rc) return rc;
      sst = side_stream;
    }
    float* partsh = reinterpret_cast<float*>(ws + B.partsh);
    void* gus = ws + B.gus;
    void* dhs = ws + B.dhs;
    dxs = ws + B.dxs;
    rc = grouped_gemm(kModePlain, x, s->T, s->d, w13_sh, 1, 2 * s->H_s, 0, 2 * s->H_s, nullptr, nullptr, gus, sst,
                      pair);
    if (rc) return rc;
    rc = grouped_gemm(kModePlain, dout, s->T, s->d, w2t_sh, 1, s->H_s, 0, s->H_s, nullptr, nullptr, dhs, sst, pair);
    if (rc) return rc;
    rc = launch_glu_bwd(s->act, gus, dhs, s->T, s->H_s, dw2_sh != nullptr, sst);
    if (rc) return rc;
    if (dw2_sh) {
      rc = wgrad_gemm(dout, s->d, s->d, dhs, s->H_s, s->T, nullptr, nullptr, 1, dw2_sh, partsh, sst);
      if (rc) return rc;
    }
    if (dw13_sh) {
      rc = wgrad_gemm(gus, 2 * s->H_s, 2 * s->H_s, x, s->d, s->T, nullptr, nullptr, 1, dw13_sh, partsh, sst);
      if (rc) return rc;
    }
    rc = grouped_gemm(kModePlain, gus, s->T, 2 * s->H_s, w13t_sh, 1, s->d, 0, s->d, nullptr, nullptr, dxs, sst,
                      pair);
    if (rc) return rc;
    if (forked && (rc = fork.end(sst))) return rc;
  }

  // forward recompute: routing, grouping, [g | u].  The softmax backward takes the logits of every expert: the
  // tensor-core screen's (two-term bf16 split of W_r, fp32 accumulation, within about 2^-16 |x| |w_e| of the
  // fp32 logits) where the routing runs through it, else the router's own fp32 logits.
  const bool screen = route_keeps_screen(s);
  rc = route_impl(s, x, w_router, bias, nullptr, screen ? nullptr : logits, idx, w, cts, nullptr, nullptr, nullptr,
                  ws, st);
  if (rc) return rc;
  const float* z_all = screen ? reinterpret_cast<const float*>(ws + L.part) : logits;
  rc = launch_scatter(s, x, idx, cnt, cts, slot, drop, nullptr, xperm, kept, offs, st, true);
  if (rc) return rc;
  rc = grouped_gemm(kModePlain, xperm, R, s->d, w13, s->E, 2 * s->H, 0, 2 * s->H, offs, kept, gu, st, pair);
  if (rc) return rc;

  // routed experts: dout of the grouped rows, dh' = dout W2, the gate gradients and [dg | du] (dh = w dh'),
  // the weight gradients (dW2 = dout^T (w h), dW13 = [dg | du]^T x), dx = [dg | du] W13
  rc = launch_move_rows(s, dout, slot, doutp, st);
  if (rc) return rc;
  rc = grouped_gemm(kModePlain, doutp, R, s->d, w2t, s->E, s->H, 0, s->H, offs, kept, hbuf, st, pair);
  if (rc) return rc;
  rc = launch_glu_bwd_slots(s->act, gu, hbuf, slot, w, s->T * (long long)s->k, s->H, dw2 != nullptr, dwb, st);
  if (rc) return rc;
  float* wpart = reinterpret_cast<float*>(ws + B.wpart);
  int32_t* wlist = reinterpret_cast<int32_t*>(ws + B.wlist);
  // an expert holds at most C rows (capacity) or T (one row per token): chunk only when that can exceed a chunk
  const int split = (s->capacity > 0 ? (long long)s->capacity : s->T) > kWgradSplitRows ? kWgradSplitRows : 0;
  if (dw2) {
    rc = wgrad_gemm(doutp, s->d, s->d, hbuf, s->H, R, offs, kept, s->E, dw2, wpart, st, split, wlist);
    if (rc) return rc;
  }
  if (dw13) {
    rc = wgrad_gemm(gu, 2 * s->H, 2 * s->H, xperm, s->d, R, offs, kept, s->E, dw13, wpart, st, split, wlist);
    if (rc) return rc;
  }
  rc = grouped_gemm(kModePlain, gu, R, 2 * s->H, w13t, s->E, s->d, 0, s->d, offs, kept, xperm, st, pair);
  if (rc) return rc;

  // router: dz through the gates, the statistic and the softmax, then dz W_r (bf16 operands, fp32 accumulation)
  // and dW_r = dz^T x
  const int epl = (int)cdiv(s->E, 32);
  const unsigned tb = (unsigned)cdiv(s->T, 8);
#define MOE_RBWD(N_)                                                                                          \
  MOE_LAUNCH((k_router_bwd<N_>), tb, 256, 0, st, z_all, idx, w, dwb, cts, aux_coef, (int)s->T, s->E, s->k,     \
             s->renorm, B.ldE, dz)
  if (epl <= 1) MOE_RBWD(1);
  else if (epl <= 2) MOE_RBWD(2);
  else if (epl <= 4) MOE_RBWD(4);
  else if (epl <= 8) MOE_RBWD(8);
  else MOE_RBWD(16);
#undef MOE_RBWD
  MOE_LAUNCH_CHECK();
  if (dw_router) {
    rc = wgrad_gemm(dz, B.ldE, s->E, x, s->d, s->T, nullptr, nullptr, 1, dw_router, part, st);
    if (rc) return rc;
  }
  {
    const dim3 grid((unsigned)cdiv(s->d, 32), (unsigned)cdiv(B.ldE, 32));
    MOE_LAUNCH((k_transpose_router), grid, dim3(32, 8), 0, st, w_router, wrt, s->E, s->d, B.ldE);
    MOE_LAUNCH_CHECK();
  }
  rc = grouped_gemm(kModePlain, dz, s->T, B.ldE, wrt, 1, s->d, 0, s->d, nullptr, nullptr, dxr, st, pair);
  if (rc) return rc;

  // dx = the token's grouped rows (slot order) + the shared expert's part + the router's part, fp32
  if (forked && (rc = fork.wait(st))) return rc;
  MOE_LAUNCH((k_bwd_final), (unsigned)cdiv(s->T * (long long)(s->d / 8), 256), 256, 0, st,
             reinterpret_cast<const __nv_bfloat16*>(xperm), slot, reinterpret_cast<const __nv_bfloat16*>(dxs),
             reinterpret_cast<const __nv_bfloat16*>(dxr), (int)s->T, s->d, s->k, dx);
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

int moe_backward_x(const moe_shape* s, const void* x, const float* w_router, const float* bias, const void* w13,
                   const void* w13t, const void* w2t, const void* w13_sh, const void* w13t_sh, const void* w2t_sh,
                   const void* dout, float aux_coef, float* dx, void* workspace, size_t ws_bytes,
                   moe_stream_t stream) {
  return moe_backward(s, x, w_router, bias, w13, w13t, w2t, w13_sh, w13t_sh, w2t_sh, dout, aux_coef, dx, nullptr,
                      nullptr, nullptr, nullptr, nullptr, workspace, ws_bytes, stream, nullptr);
}

int moe_route_tree_workspace_size(const moe_shape* s, int32_t branch, int32_t levels, size_t* bytes) {
  const int rc = check_tree(s, branch, levels);
  if (rc) return rc;
  if (!bytes) return MOE_INVALID_ARGUMENT;
  *bytes = tree_layout(s, branch * levels).total;
  return MOE_OK;
}

int moe_route_tree(const moe_shape* s, int32_t branch, int32_t levels, const void* x, const float* w_tree,
                   const float* bias_tree, int32_t* topk_idx, float* topk_w, int32_t* counts, float* level_logits,
                   void* workspace, size_t ws_bytes, moe_stream_t stream) {
  int rc = check_tree(s, branch, levels);
  if (rc) return rc;
  if (!x || !w_tree || !topk_idx || !topk_w || !workspace) return MOE_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(w_tree) || !aligned16(level_logits) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return MOE_INVALID_ARGUMENT;
  const int n = branch * levels;
  const TreeWorkspace W = tree_layout(s, n);
  if (ws_bytes < W.total) return MOE_WORKSPACE_TOO_SMALL;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  __nv_bfloat16* wsplit = reinterpret_cast<__nv_bfloat16*>(ws + W.wsplit);
  float* z = level_logits ? level_logits : reinterpret_cast<float*>(ws + W.z);
  // the levels' routers as one screening operand [n, 2d] (bf16 high and low terms), counts zeroed alongside
  MOE_LAUNCH((k_router_prep), (unsigned)cdiv(n, 8), 256, 0, stream, w_tree, wsplit,
             reinterpret_cast<float*>(ws + W.wnorm), n, s->d, counts, counts ? s->E : 0,
             static_cast<const __nv_bfloat16*>(nullptr), static_cast<float*>(nullptr), (int)s->T);
  MOE_LAUNCH_CHECK();
  GemmExtras ex;
  ex.bias = bias_tree;
  rc = grouped_gemm(kModeScreen, x, s->T, s->d, wsplit, 1, n, 0, n, nullptr, nullptr, z, stream,
                    !(s->flags & MOE_FLAG_SINGLE_CTA_GEMM), ex);
  if (rc) return rc;
  // lanes per token: enough for kTreeCPL children each
  const int G = branch <= 2 * kTreeCPL ? 2 : (branch <= 4 * kTreeCPL ? 4 : 8);
  const unsigned blocks = (unsigned)cdiv(s->T * G, kTreeThreads);
#define MOE_TREE(K_, G_)                                                                                      \
  MOE_LAUNCH((k_router_tree<K_, G_>), blocks, kTreeThreads, 0, stream, z, (int)s->T, (int)branch, (int)levels,  \
             s->k, s->renorm, topk_idx, topk_w, counts)
#define MOE_TREE_K(G_)                     \
  if (s->k <= 2) MOE_TREE(2, G_);          \
  else if (s->k <= 4) MOE_TREE(4, G_);     \
  else if (s->k <= 8) MOE_TREE(8, G_);     \
  else MOE_TREE(16, G_);
  if (G == 2) { MOE_TREE_K(2) }
  else if (G == 4) { MOE_TREE_K(4) }
  else { MOE_TREE_K(8) }
#undef MOE_TREE_K
#undef MOE_TREE
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

int moe_quantize_int4(const float* w, int64_t rows, int32_t K, uint8_t* q, void* scales, moe_stream_t stream) {
  if (!w || !q || !scales || rows < 0 || K <= 0 || K % 128 != 0) return MOE_INVALID_ARGUMENT;
  if (!aligned16(w) || (reinterpret_cast<uintptr_t>(q) & 1u) || (reinterpret_cast<uintptr_t>(scales) & 1u))
    return MOE_INVALID_ARGUMENT;
  if (rows == 0) return MOE_OK;
  const long long items = rows * (K / 128);
  MOE_LAUNCH((k_quantize_int4), (unsigned)cdiv(items, 8), 256, 0, stream, w, rows, K, q,
                                                                 reinterpret_cast<__nv_bfloat16*>(scales));
  MOE_LAUNCH_CHECK();
  return MOE_OK;
}

int moe_get_status(moe_stream_t stream, int32_t* device_status, uint32_t* site) {
  if (!device_status) return MOE_INVALID_ARGUMENT;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_CUDA_ERROR;
  unsigned int st = 0, where = 0, zero = 0;
  MOE_CUDA_TRY(cudaMemcpyFromSymbol(&st, g_status, sizeof(st)));
  MOE_CUDA_TRY(cudaMemcpyFromSymbol(&where, g_status_site, sizeof(where)));
  MOE_CUDA_TRY(cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)));
  MOE_CUDA_TRY(cudaMemcpyToSymbol(g_status_site, &zero, sizeof(zero)));
  *device_status = (int32_t)st;
  if (site) *site = where;
  return MOE_OK;
}

}  // extern "C"

namespace moe {
// One mbarrier that nothing arrives on; the bounded wait must give up.
__global__ void k_selftest_wait(unsigned long long limit_ns) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, limit_ns, &abort_flag, 0x7F01);
}
}  // namespace moe

extern "C" int moe_selftest_wait_timeout(moe_stream_t stream) {
  MOE_LAUNCH((moe::k_selftest_wait), 1, 32, 0, stream, moe::g_wait_limit_ns.load());
  count_launch();
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_CUDA_ERROR;
}

// ====================================================================== allocation-free grouping
//
// moe_permute_noalloc: the grouping of moe_permute for callers that cannot
// hand the library a workspace.  Its scratch (the per-chunk expert histogram
// and, when the caller passes no counts buffer, the per-expert counts) lives in
// the fixed array below, which every GPU that loads this library keeps for the
// life of the process.  Host code must not pass the array's name to a kernel:
// on the host it is only a stand-in symbol, so the device address is looked up
// once per device with cudaGetSymbolAddress and cached.

namespace moe {

constexpr long long kNoAllocHistInts = 262144;  // ceil(T / 32) * E must not exceed this
constexpr int kNoAllocCountInts = kMaxE;

static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocHistInts + kNoAllocCountInts];

static std::mutex g_noalloc_mu;
static int32_t* g_noalloc_ptr[64];

// Device address of the scratch array on the current device (set up on the first call per device).
static int noalloc_scratch(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_CUDA_ERROR;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MOE_CUDA_ERROR;
    g_noalloc_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return MOE_OK;
}

}  // namespace moe

extern "C" int moe_permute_noalloc(const moe_shape* s, const void* x, const int32_t* topk_idx, int32_t* slot_pos,
                                   uint8_t* drop_mask, int32_t* counts, int32_t* kept, int32_t* offsets,
                                   int32_t* row_src, void* x_perm, moe_stream_t stream) {
  using namespace moe;
  int rc = check_shape(s);
  if (rc) return rc;
  if (!x || !topk_idx || !slot_pos || !kept || !offsets || !x_perm) return MOE_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(x_perm)) return MOE_INVALID_ARGUMENT;
  const long long nchunks = cdiv(s->T, kChunk);
  if (nchunks * s->E > kNoAllocHistInts) return MOE_UNSUPPORTED_SHAPE;  // beyond the fixed scratch
  int32_t* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc) return rc;
  int32_t* cnt = scratch;                                   // fully rewritten by k_chunk_hist every call
  int32_t* cts = counts ? counts : scratch + kNoAllocHistInts;  // fully rewritten by k_chunk_scan
  MOE_LAUNCH((k_chunk_hist), (unsigned)nchunks, 256, s->E * sizeof(int), stream, topk_idx, cnt, (int)s->T, s->E, s->k);
  MOE_LAUNCH_CHECK();
  rc = launch_scan(s, cnt, nullptr, cts, nullptr, nullptr, stream);
  if (rc) return rc;
  return launch_scatter(s, x, topk_idx, cnt, cts, slot_pos, drop_mask, row_src, x_perm, kept, offsets, stream);
}
