// C ABI of the Muon update library: argument checking, shape grouping,
// workspace ownership and the launch sequence of one step.
//
// Launch sequence of muon_step (all on the caller's stream):
//   flat_kernel (momentum + partial norms) -> cast_kernel (normalise,
//   transpose to rows <= cols, fp32 master + bf16 operand) -> T x
//   [kGram, kPoly, kBx] tensor-core launches over every shape group ->
//   out_kernel (scale and apply).
// Sources: "NanoGPT Speedrun: The Ultimate Guide to Pushing LLM Training
// Efficiency to Its Limits", section "Optimizer and Training Strategy Tuning"
// (orthogonalise the Nesterov-momentum update of hidden matrices by
// Newton-Schulz), and "The NanoGPT speedrun", paragraph "Six records account
// for most of the speedup" (five Newton-Schulz steps, nearest semi-orthogonal
// matrix).
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include <cuda_bf16.h>

#include "internal.h"
#include "muon.h"

using namespace muon;
typedef __nv_bfloat16 bf16;

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr int kMaxDim = 32768;
constexpr int kMaxStepsArg = 100;
constexpr float kNormEps = 1e-7f;
constexpr float kCoefA = 3.4445f, kCoefB = -4.7750f, kCoefC = 2.0315f;
constexpr double kNeuronEps = 1e-10;  // guard inside the per-neuron 1 / sqrt(v + eps)

thread_local std::string t_err;

int set_err(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_err = buf;
  return code;
}

#define CUDA_TRY(call)                                                                     \
  do {                                                                                     \
    cudaError_t e_ = (call);                                                               \
    if (e_ != cudaSuccess)                                                                 \
      return set_err(MUON_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));       \
  } while (0)

#define MUON_TRY(expr)           \
  do {                           \
    int r_ = (expr);             \
    if (r_ != MUON_OK) return r_; \
  } while (0)

struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
  int* status = nullptr;
};

struct DevInfo {
  int sms = 0, major = 0, minor = 0;
};

std::mutex g_mu;
std::map<std::pair<int, uintptr_t>, Workspace> g_ws;
std::map<int, DevInfo> g_dev;
unsigned long long g_timeout_ns = 2000000000ull;
int g_inject = 0;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int get_encoder() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  static cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSuccess;
  std::call_once(once, [] {
    void* fn = nullptr;
    err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (!g_encode)
    return set_err(MUON_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s, query %d)",
                   cudaGetErrorString(err), static_cast<int>(q));
  return MUON_OK;
}

// ------------------------------------------------------------ kernel timing
struct ProfRec {
  int kind;
  cudaEvent_t a, b;
};
bool g_prof_on = false;
// While set on a thread, the timing hooks stay inert on that thread (they
// would otherwise create CUDA event objects); used by the allocation-free call.
thread_local bool t_hooks_off = false;
std::vector<ProfRec> g_prof;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Brackets one launch with events on its stream while timing is on.
struct ProfScope {
  int kind;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  ProfScope(int k, cudaStream_t st) : kind(k), s(st) {
    if (t_hooks_off) return;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_prof_on) return;
    a = take_event();
    if (a) cudaEventRecord(a, s);
  }
  ~ProfScope() {
    if (!a) return;
    std::lock_guard<std::mutex> lk(g_mu);
    cudaEvent_t b = take_event();
    if (!b) return;
    cudaEventRecord(b, s);
    g_prof.push_back({kind, a, b});
  }
};

int device_info(DevInfo* out) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_dev.find(dev);
    if (it != g_dev.end()) {
      *out = it->second;
      return MUON_OK;
    }
  }
  DevInfo d;
  CUDA_TRY(cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev));
  CUDA_TRY(cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev));
  CUDA_TRY(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
  if (d.major != 10 || d.minor != 0)
    return set_err(MUON_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
                   dev, d.major, d.minor);
  std::lock_guard<std::mutex> lk(g_mu);
  g_dev[dev] = d;
  *out = d;
  return MUON_OK;
}

// Workspace of (current device, stream), grown stream-ordered to >= need bytes.
int get_workspace(cudaStream_t s, size_t need, Workspace** out) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace& w = g_ws[{dev, reinterpret_cast<uintptr_t>(s)}];
  if (!w.status) {
    CUDA_TRY(cudaMalloc(&w.status, 256));
    CUDA_TRY(cudaMemset(w.status, 0, 256));
  }
  if (w.bytes < need) {
    if (w.ptr) {
      CUDA_TRY(cudaFreeAsync(w.ptr, s));
      w.ptr = nullptr;
      w.bytes = 0;
    }
    size_t nb = std::max(need, static_cast<size_t>(1) << 21);
    nb = (nb + (static_cast<size_t>(1) << 21) - 1) & ~((static_cast<size_t>(1) << 21) - 1);
    cudaError_t e = cudaMallocAsync(&w.ptr, nb, s);
    if (e != cudaSuccess) {
      cudaGetLastError();
      w.ptr = nullptr;
      return set_err(MUON_ERR_ALLOC, "workspace of %zu bytes: %s", nb, cudaGetErrorString(e));
    }
    w.bytes = nb;
  }
  *out = &w;
  return MUON_OK;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline long long round8(long long x) { return (x + 7) / 8 * 8; }
inline long long round16(long long x) { return (x + 15) / 16 * 16; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// 3-D tensor map {inner, rows, batch} over a contiguous batch with row stride
// `ld` and matrix stride `mat_stride` (elements); `esize` 1 = int8, 2 = bf16,
// 4 = fp32.
int make_map(CUtensorMap* map, const void* base, int esize, uint64_t inner, uint64_t rows,
             uint64_t batch, uint64_t ld, uint64_t mat_stride, uint32_t box_inner, uint32_t box_rows,
             CUtensorMapSwizzle swz) {
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {ld * esize, mat_stride * esize};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  const CUtensorMapDataType dt = esize == 1   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                              : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUresult r = g_encode(map, dt, 3, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_err(MUON_ERR_CUDA,
                   "cuTensorMapEncodeTiled failed (%d) for %llux%llux%llu ld %llu box %ux%u",
                   static_cast<int>(r), (unsigned long long)inner, (unsigned long long)rows,
                   (unsigned long long)batch, (unsigned long long)ld, box_inner, box_rows);
  return MUON_OK;
}

// Maps of the symmetric-output GEMMs: D (m x m) from an operand S (m x k, K-major),
// D = S S^T (kGram) or b S + c S S (kPoly, with S = A symmetric and e = A).
int sym_maps(tc::Maps& M, const void* S, int m, int k, long long lds, long long ss, void* D,
             long long ldd, long long sd, int batch, bool with_e) {
  MUON_TRY(make_map(&M.p, S, 2, k, m, batch, lds, ss, 64, tc::BM, CU_TENSOR_MAP_SWIZZLE_128B));
  MUON_TRY(make_map(&M.q, S, 2, k, m, batch, lds, ss, 64, tc::BNH, CU_TENSOR_MAP_SWIZZLE_128B));
  // epilogue chunks of kSymChunk columns: rows of 64 or 128 bytes
  const CUtensorMapSwizzle cswz =
      tc::kSymChunk == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (with_e)
    MUON_TRY(make_map(&M.e, S, 2, m, m, batch, lds, ss, tc::kSymChunk, tc::BM, cswz));
  else
    M.e = M.p;
  MUON_TRY(make_map(&M.d, D, 2, m, m, batch, ldd, sd, tc::kSymChunk, tc::BM, cswz));
  MUON_TRY(make_map(&M.mt, D, 2, m, m, batch, ldd, sd, tc::BM, tc::kSymChunk, CU_TENSOR_MAP_SWIZZLE_NONE));
  MUON_TRY(make_map(&M.s, D, 2, m, m, batch, ldd, sd, 64, tc::BM, CU_TENSOR_MAP_SWIZZLE_128B));
  return MUON_OK;
}

// Maps of X' = a X + B X with X carried as the pair bf16 hi + int8 lo: B
// (m x m), hi of X (m x n: MN-major operand and epilogue chunks), lo of X
// (read and written in place), hi of X' (written).  Epilogue chunks are
// `chunk` (64 or 32) columns wide: hi rows of 2 chunk bytes, lo rows of
// chunk bytes, each swizzled over its full width.
int bx_maps(tc::Maps& M, const void* B, long long ldb, long long sb, const void* Xhi,
            void* Xlo, void* Xhi_out, int m, int n, long long ldx, long long sx, int batch,
            int chunk = 64) {
  MUON_TRY(make_map(&M.p, B, 2, m, m, batch, ldb, sb, 64, tc::BM, CU_TENSOR_MAP_SWIZZLE_128B));
  MUON_TRY(make_map(&M.q, Xhi, 2, n, m, batch, ldx, sx, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B));
  const CUtensorMapSwizzle hs = chunk == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const CUtensorMapSwizzle ls = chunk == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  MUON_TRY(make_map(&M.e, Xhi, 2, n, m, batch, ldx, sx, chunk, tc::BM, hs));
  MUON_TRY(make_map(&M.mt, Xlo, 1, n, m, batch, ldx, sx, chunk, tc::BM, ls));
  MUON_TRY(make_map(&M.d, Xhi_out, 2, n, m, batch, ldx, sx, chunk, tc::BM, hs));
  M.s = M.d;  // unused
  return MUON_OK;
}

// One shape class of the iteration: `batch` matrices X (m x n, m <= n) laid
// out contiguously in the workspace with padded row strides.
struct NsGroup {
  int batch = 0, m = 0, n = 0;
  long long ldn = 0, ldm = 0;
  float* xf = nullptr;          // fp32 path: ping buffer of X
  float* xf1 = nullptr;         // fp32 path: pong buffer of X
  bf16* xb[2] = {nullptr, nullptr};  // bf16 path: hi of X (ping-pong; the GEMM operand)
  int8_t* xlo = nullptr;             // bf16 path: lo of X, X = hi + q 2^(E(hi) - 15)
  bf16* A = nullptr;
  bf16* B = nullptr;
  float* Af = nullptr;
  float* Bf = nullptr;
  int mat_base = 0;             // bf16 path: index of the group's first matrix in the scale array
};

// Bytes of workspace a group needs; assigns its offsets from `base` (or counts
// only, when base is null).
size_t layout_group(NsGroup& g, char* base, size_t off, bool fp32) {
  g.ldn = round16(g.n);  // 16-byte rows for the int8 lo as well
  g.ldm = round8(g.m);
  const size_t xe = static_cast<size_t>(g.batch) * g.m * g.ldn;
  const size_t ae = static_cast<size_t>(g.batch) * g.m * g.ldm;
  auto take = [&](size_t bytes) {
    off = align_up(off, 1024);
    char* p = base ? base + off : nullptr;
    off += bytes;
    return p;
  };
  if (!fp32) {
    g.xb[0] = reinterpret_cast<bf16*>(take(xe * 2));
    g.xb[1] = reinterpret_cast<bf16*>(take(xe * 2));
    g.xlo = reinterpret_cast<int8_t*>(take(xe));
    g.A = reinterpret_cast<bf16*>(take(ae * 2));
    g.B = reinterpret_cast<bf16*>(take(ae * 2));
  } else {
    g.xf = reinterpret_cast<float*>(take(xe * 4));
    g.xf1 = reinterpret_cast<float*>(take(xe * 4));
    g.Af = reinterpret_cast<float*>(take(ae * 4));
    g.Bf = reinterpret_cast<float*>(take(ae * 4));
  }
  return off;
}

tc::Group tc_group(int batch, int m, int n, int k, bool sym, int tile_begin) {
  tc::Group G{};
  G.batch = batch;
  G.m = m;
  G.n = n;
  G.k = k;
  G.tiles_m = (m + tc::PM - 1) / tc::PM;
  G.tiles_n = sym ? (m + tc::BN - 1) / tc::BN : (n + tc::BN - 1) / tc::BN;
  G.tiles_per_mat = sym ? tc::sym_tiles(m) : G.tiles_m * G.tiles_n;
  G.tile_begin = tile_begin;
  G.mat_base = 0;
  return G;
}

#ifdef MUON_TRACE
unsigned long long* g_trace = nullptr;  // device buffer for kernel timestamps
#endif

void init_tc_params(tc::Params& P, int* status, float a, float b, float c) {
  P.ngroups = 0;
  P.total_tiles = 0;
  P.a = a;
  P.b = b;
  P.c = c;
  P.xscale = nullptr;
  P.status = status;
  P.timeout_ns = g_timeout_ns;
  P.inject = 0;
  P.reverse = 0;
  P.trace = nullptr;
#ifdef MUON_TRACE
  P.trace = g_trace;
#endif
}

int launch_tc(int epi, tc::Params& P, int sms, cudaStream_t s, const tc::LaunchApply* apply = nullptr) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_inject) {
      P.inject = g_inject;
      g_inject = 0;
    }
  }
  ProfScope prof(epi == tc::kBxApply ? MUON_KERNEL_BX_APPLY : MUON_KERNEL_GRAM + epi, s);
  CUDA_TRY(tc::launch(epi, P, sms / 2, s, apply));  // one CTA pair per two SMs
  P.inject = 0;
  return MUON_OK;
}

// A caller's matrix: its layout (rows x cols), its iteration shape m x n
// (m <= n, transposed when rows > cols), and its place in a shape group.
struct MatInfo {
  int rows, cols, m, n, transposed, group, index;
};

// The caller's buffers that the last step's BX epilogue writes directly:
// kind 0, fp32 weights W updated by the apply (kBxApply); kind 1, bf16
// buffers receiving X_T itself (kBx, mode 3: matrices in X's layout only).
struct ApplySpec {
  const std::vector<MatInfo>* mats = nullptr;
  const std::vector<void*>* w = nullptr;  // W (kind 0) or the output (kind 1) of matrix i, caller's layout
  int kind = 0;
  float lr = 0.f, wd = 0.f;
  int cautious = 0;        // kind 0: decay only where W and O have the same sign
  std::vector<char> done;  // out: matrix i was finished by the GEMM epilogue
};

// fl(lr * scale) with scale = sqrt(max(1, rows / cols)), as the apply pass uses.
float apply_ls(const MatInfo& M, float lr) {
  const float ratio = static_cast<float>(M.rows) / static_cast<float>(M.cols);
  const float scale = ratio > 1.0f ? sqrtf(ratio) : 1.0f;
  return lr * scale;
}

// Table of the groups [g0, g1) of the last BX launch.  Kind 0: every matrix
// whose W rows are 16-byte strided (cols % 4 == 0) among the first kMaxApply
// gets a tensor map over W and mode 1 (W = X) or 2 (W = X^T).  Kind 1: every
// such matrix in X's layout (not transposed) with 16-byte bf16 rows (cols % 8
// == 0) gets a map over its output and mode 3.  The rest keep mode 0.
int build_apply_table(const std::vector<NsGroup>& gs, size_t g0, size_t g1, ApplySpec& A,
                      tc::LaunchApply& T) {
  T.nmat = 0;
  T.mat_base = gs[g0].mat_base;
  T.lw = A.lr * A.wd;
  T.cautious = A.cautious;
  int span = 0;
  for (size_t gi = g0; gi < g1; ++gi) span += gs[gi].batch;
  T.nmat = std::min(span, tc::kMaxApply);
  for (int j = 0; j < T.nmat; ++j) T.mat[j] = tc::ApplyMat{0, 0.f};
  const std::vector<MatInfo>& mats = *A.mats;
  for (size_t i = 0; i < mats.size(); ++i) {
    const MatInfo& M = mats[i];
    if (M.group < static_cast<int>(g0) || M.group >= static_cast<int>(g1)) continue;
    const int j = gs[M.group].mat_base + M.index - T.mat_base;
    if (j >= T.nmat) continue;
    const void* W = (*A.w)[i];
    if (A.kind == 1) {
      if (M.transposed || M.cols % 8 != 0) continue;
      MUON_TRY(make_map(&T.w[j], W, 2, M.cols, M.rows, 1, M.cols, static_cast<uint64_t>(M.rows) * M.cols, 64,
                        tc::BM, CU_TENSOR_MAP_SWIZZLE_128B));
      T.mat[j] = tc::ApplyMat{3, 0.f};
      A.done[i] = 1;
      continue;
    }
    if (M.cols % 4 != 0) continue;
    if (!M.transposed)
      MUON_TRY(make_map(&T.w[j], W, 4, M.cols, M.rows, 1, M.cols, static_cast<uint64_t>(M.rows) * M.cols, 32,
                        tc::BM, CU_TENSOR_MAP_SWIZZLE_128B));
    else
      MUON_TRY(make_map(&T.w[j], W, 4, M.cols, M.rows, 1, M.cols, static_cast<uint64_t>(M.rows) * M.cols, 32,
                        tc::bx_apply_chunk(), CU_TENSOR_MAP_SWIZZLE_128B));
    T.mat[j] = tc::ApplyMat{M.transposed ? 2 : 1, apply_ls(M, A.lr)};
    A.done[i] = 1;
  }
  return MUON_OK;
}

// T steps of X <- a_t X + (b_t A + c_t A^2) X on bf16 operands, X carried as
// the pair hi + lo; step t uses abc[3t .. 3t+2].  On entry each group's xb[0]
// / xlo hold X0 / s with s = xscale[mat_base + i] per matrix (s = 1 when
// xscale is null); on exit xb[T % 2] / xlo hold X_T (for T >= 1; X0 / s
// itself for T = 0) -- except for the matrices that `apply` (when given, and
// T >= 1) marks done: their last step updated the caller's weights instead.
int run_ns_bf16(std::vector<NsGroup>& gs, int steps, const float* abc, int* status, int sms,
                cudaStream_t s, const float* xscale, ApplySpec* apply = nullptr) {
  if (steps <= 0 || gs.empty()) return MUON_OK;
  MUON_TRY(get_encoder());
  const float a = abc[0], b = abc[1], c = abc[2];
  for (size_t g0 = 0; g0 < gs.size(); g0 += tc::kMaxGroups) {
    const size_t g1 = std::min(gs.size(), g0 + tc::kMaxGroups);
    tc::Params gram[2], poly, bx[2];
    for (int par = 0; par < 2; ++par) {
      init_tc_params(gram[par], status, a, b, c);
      init_tc_params(bx[par], status, a, b, c);
    }
    init_tc_params(poly, status, a, b, c);
    for (size_t gi = g0; gi < g1; ++gi) {
      NsGroup& G = gs[gi];
      const int k = static_cast<int>(gi - g0);
      const long long xs = static_cast<long long>(G.m) * G.ldn;
      const long long as = static_cast<long long>(G.m) * G.ldm;
      for (int par = 0; par < 2; ++par) {
        gram[par].grp[k] = tc_group(G.batch, G.m, G.m, G.n, true, gram[par].total_tiles);
        MUON_TRY(sym_maps(gram[par].map[k], G.xb[par], G.m, G.n, G.ldn, xs, G.A, G.ldm, as,
                          G.batch, false));
        gram[par].total_tiles += G.batch * gram[par].grp[k].tiles_per_mat;
        gram[par].ngroups = k + 1;

        bx[par].grp[k] = tc_group(G.batch, G.m, G.n, G.m, false, bx[par].total_tiles);
        MUON_TRY(bx_maps(bx[par].map[k], G.B, G.ldm, as, G.xb[par], G.xlo, G.xb[par ^ 1], G.m, G.n,
                         G.ldn, xs, G.batch));
        bx[par].total_tiles += G.batch * bx[par].grp[k].tiles_per_mat;
        bx[par].ngroups = k + 1;
      }
      poly.grp[k] = tc_group(G.batch, G.m, G.m, G.m, true, poly.total_tiles);
      MUON_TRY(sym_maps(poly.map[k], G.A, G.m, G.m, G.ldm, as, G.B, G.ldm, as, G.batch, true));
      poly.total_tiles += G.batch * poly.grp[k].tiles_per_mat;
      poly.ngroups = k + 1;
    }
    for (size_t gi = g0; gi < g1; ++gi) {
      const int k = static_cast<int>(gi - g0);
      for (int par = 0; par < 2; ++par) {
        gram[par].grp[k].mat_base = gs[gi].mat_base;
        bx[par].grp[k].mat_base = gs[gi].mat_base;
      }
    }
    // the first step folds the per-matrix scale into its Gram and BX epilogues
    tc::Params gram0 = gram[0], bx0 = bx[0];
    gram0.xscale = xscale;
    bx0.xscale = xscale;
    // Each launch reads what the one before it wrote (X -> A -> B -> X'), and
    // the tail of that output is what L2 still holds: consecutive launches
    // walk the tiles in opposite directions, the first Gram backwards (the
    // pass that wrote X_0 went forwards).
    int backwards = 1;
    int cur = 0;
    for (int t = 0; t < steps; ++t) {
      // the step's own (a, b, c): B = b A + c A^2 in kPoly, a X in kBx
      poly.b = abc[3 * t + 1];
      poly.c = abc[3 * t + 2];
      tc::Params& bxt = t == 0 ? bx0 : bx[cur];
      bxt.a = abc[3 * t];
      tc::Params& gramt = t == 0 ? gram0 : gram[cur];
      gramt.reverse = backwards;
      poly.reverse = backwards ^ 1;
      bxt.reverse = backwards;
      backwards ^= 1;
      MUON_TRY(launch_tc(tc::kGram, gramt, sms, s));
      MUON_TRY(launch_tc(tc::kPoly, poly, sms, s));
      if (apply && t == steps - 1) {
        tc::LaunchApply table;
        MUON_TRY(build_apply_table(gs, g0, g1, *apply, table));
        if (apply->kind == 0) {
          // kBxApply reads and writes X's pair in chunks of its own width
          tc::Params bxa = bxt;
          for (size_t gi = g0; gi < g1; ++gi) {
            NsGroup& G = gs[gi];
            const int k = static_cast<int>(gi - g0);
            const long long xs = static_cast<long long>(G.m) * G.ldn;
            const long long as = static_cast<long long>(G.m) * G.ldm;
            MUON_TRY(bx_maps(bxa.map[k], G.B, G.ldm, as, G.xb[cur], G.xlo, G.xb[cur ^ 1], G.m, G.n, G.ldn,
                             xs, G.batch, tc::bx_apply_chunk()));
          }
          MUON_TRY(launch_tc(tc::kBxApply, bxa, sms, s, &table));
        } else {
          MUON_TRY(launch_tc(tc::kBx, bxt, sms, s, &table));
        }
      } else {
        MUON_TRY(launch_tc(tc::kBx, bxt, sms, s));
      }
      cur ^= 1;
    }
  }
  return MUON_OK;
}

// Where a group's result X_T lives: fp32, or the pair bf16 hi + int8 residual.
struct Result {
  const float* f = nullptr;
  const bf16* hi = nullptr;
  const int8_t* lo = nullptr;
};

Result bf16_result(const NsGroup& g, int steps) {
  Result r;
  r.hi = g.xb[steps & 1];
  r.lo = g.xlo;
  return r;
}

// fp32 SIMT verification path (step t uses abc[3t .. 3t+2]); on exit
// *final_xf of each group holds X_T.
int run_ns_fp32(std::vector<NsGroup>& gs, int steps, const float* abc, cudaStream_t s,
                std::vector<float*>& final_xf) {
  final_xf.clear();
  for (NsGroup& G : gs) {
    float* x[2] = {G.xf, G.xf1};
    int cur = 0;
    const long long xs = static_cast<long long>(G.m) * G.ldn;
    const long long as = static_cast<long long>(G.m) * G.ldm;
    for (int t = 0; t < steps; ++t) {
      simt::Params p{};
      p.batch = G.batch;
      p.a = abc[3 * t];
      p.b = abc[3 * t + 1];
      p.c = abc[3 * t + 2];
      // A = X X^T
      p.m = G.m; p.n = G.m; p.k = G.n;
      p.P = x[cur]; p.ldp = G.ldn; p.sp = xs;
      p.Q = x[cur]; p.ldq = G.ldn; p.sq = xs;
      p.E = nullptr; p.lde = 0; p.se = 0;
      p.D = G.Af; p.ldd = G.ldm; p.sd = as;
      {
        ProfScope prof(MUON_KERNEL_SIMT, s);
        CUDA_TRY(simt::launch(simt::kGram, p, s));
      }
      // B = bA + c A A
      p.k = G.m;
      p.P = G.Af; p.ldp = G.ldm; p.sp = as;
      p.Q = G.Af; p.ldq = G.ldm; p.sq = as;
      p.E = G.Af; p.lde = G.ldm; p.se = as;
      p.D = G.Bf;
      {
        ProfScope prof(MUON_KERNEL_SIMT, s);
        CUDA_TRY(simt::launch(simt::kPoly, p, s));
      }
      // X' = aX + B X
      p.n = G.n; p.k = G.m;
      p.P = G.Bf; p.ldp = G.ldm; p.sp = as;
      p.Q = x[cur]; p.ldq = G.ldn; p.sq = xs;
      p.E = x[cur]; p.lde = G.ldn; p.se = xs;
      p.D = x[cur ^ 1]; p.ldd = G.ldn; p.sd = xs;
      {
        ProfScope prof(MUON_KERNEL_SIMT, s);
        CUDA_TRY(simt::launch(simt::kBx, p, s));
      }
      cur ^= 1;
    }
    final_xf.push_back(x[cur]);
  }
  return MUON_OK;
}

bool finite(float v) { return std::isfinite(v); }

// Group matrices by (m, n) = (min, max); larger n first (longer K in kGram).
void group_shapes(const std::vector<std::pair<int, int>>& shapes, std::vector<MatInfo>& mats,
                  std::vector<NsGroup>& groups) {
  std::map<std::pair<int, int>, int, std::greater<std::pair<int, int>>> key;
  mats.resize(shapes.size());
  for (size_t i = 0; i < shapes.size(); ++i) {
    MatInfo& M = mats[i];
    M.rows = shapes[i].first;
    M.cols = shapes[i].second;
    M.transposed = M.rows > M.cols;
    M.m = std::min(M.rows, M.cols);
    M.n = std::max(M.rows, M.cols);
    key.emplace(std::make_pair(M.n, M.m), 0);
  }
  groups.clear();
  for (auto& kv : key) {
    kv.second = static_cast<int>(groups.size());
    NsGroup g;
    g.n = kv.first.first;
    g.m = kv.first.second;
    groups.push_back(g);
  }
  for (size_t i = 0; i < shapes.size(); ++i) {
    MatInfo& M = mats[i];
    M.group = key[std::make_pair(M.n, M.m)];
    M.index = groups[M.group].batch++;
  }
}

// Flat momentum / sum-of-squares pass over matrices [i0, i1) of `srcs`.
int launch_flat_chunked(const std::vector<const void*>& srcs, const std::vector<float*>& bufs,
                        const std::vector<long long>& numels, int src_kind, float beta,
                        int nesterov, float* partials, std::vector<int>& part_begin,
                        std::vector<int>& part_count, cudaStream_t s) {
  const int count = static_cast<int>(srcs.size());
  part_begin.assign(count, 0);
  part_count.assign(count, 0);
  int global_blk = 0;
  for (int i0 = 0; i0 < count; i0 += ew::kMaxMats) {
    const int i1 = std::min(count, i0 + ew::kMaxMats);
    ew::FlatParams fp{};
    fp.src_kind = src_kind;
    fp.beta = beta;
    fp.omb = 1.0f - beta;
    fp.nesterov = nesterov;
    fp.partials = partials + global_blk;
    int blk = 0;
    for (int i = i0; i < i1; ++i) {
      ew::FlatMat& F = fp.mat[i - i0];
      F.src = srcs[i];
      F.buf = bufs.empty() ? nullptr : bufs[i];
      F.numel = numels[i];
      F.blk_begin = blk;
      const int nb = static_cast<int>((numels[i] + ew::kFlatChunk - 1) / ew::kFlatChunk);
      part_begin[i] = global_blk + blk;
      part_count[i] = nb;
      blk += nb;
    }
    fp.nmat = i1 - i0;
    fp.nblocks = blk;
    ProfScope prof(MUON_KERNEL_FLAT, s);
    CUDA_TRY(ew::launch_flat(fp, s));
    global_blk += blk;
  }
  return MUON_OK;
}

int count_flat_blocks(const std::vector<long long>& numels) {
  long long nb = 0;
  for (long long n : numels) nb += (n + ew::kFlatChunk - 1) / ew::kFlatChunk;
  return static_cast<int>(nb);
}

// Normalise (+ transpose) every matrix into its group's workspace buffers.
int launch_cast_chunked(const std::vector<MatInfo>& mats, std::vector<NsGroup>& groups,
                        const std::vector<const void*>& src0, const std::vector<const float*>& src1,
                        int src_kind, float beta, int nesterov, const float* partials,
                        const std::vector<int>& part_begin, const std::vector<int>& part_count,
                        cudaStream_t s) {
  const int count = static_cast<int>(mats.size());
  for (int i0 = 0; i0 < count; i0 += ew::kMaxMats) {
    const int i1 = std::min(count, i0 + ew::kMaxMats);
    ew::CastParams cp{};
    cp.src_kind = src_kind;
    cp.beta = beta;
    cp.omb = 1.0f - beta;
    cp.nesterov = nesterov;
    cp.eps = kNormEps;
    cp.partials = partials;
    int tiles = 0;
    for (int i = i0; i < i1; ++i) {
      const MatInfo& M = mats[i];
      const NsGroup& G = groups[M.group];
      ew::CastMat& C = cp.mat[i - i0];
      C.src0 = src0[i];
      C.src1 = src1.empty() ? nullptr : src1[i];
      C.rows = M.rows;
      C.cols = M.cols;
      C.transposed = M.transposed;
      C.tiles_n = (M.n + ew::kTile - 1) / ew::kTile;
      C.tile_begin = tiles;
      C.part_begin = part_begin[i];
      C.part_count = part_count[i];
      const long long off = static_cast<long long>(M.index) * G.m * G.ldn;
      C.xf = G.xf + off;
      C.ld = G.ldn;
      C.vec = (M.cols % 8 == 0) && aligned16(src0[i]) && (src1.empty() || aligned16(src1[i]));
      tiles += ((M.m + ew::kTile - 1) / ew::kTile) * C.tiles_n;
    }
    cp.nmat = i1 - i0;
    cp.ntiles = tiles;
    ProfScope prof(MUON_KERNEL_CAST, s);
    CUDA_TRY(ew::launch_cast(cp, s));
  }
  return MUON_OK;
}

// Blocks of the prep pass of one matrix.
int prep_tiles(const MatInfo& M) {
  return ((M.rows + ew::kPrepRows - 1) / ew::kPrepRows) * ((M.cols + ew::kPrepCols - 1) / ew::kPrepCols);
}

int count_prep_blocks(const std::vector<MatInfo>& mats) {
  long long nb = 0;
  for (const MatInfo& M : mats) nb += prep_tiles(M);
  return static_cast<int>(nb);
}

// Index of every group's first matrix in the per-matrix scale array.
void assign_mat_base(std::vector<NsGroup>& groups) {
  int base = 0;
  for (NsGroup& g : groups) {
    g.mat_base = base;
    base += g.batch;
  }
}

// Momentum (src_kind kFromMomentum) or a plain read of bf16 X (kFromBf16), u
// written as hi + lo into the group workspaces, partial sums of u^2 per block.
int launch_prep_chunked(const std::vector<MatInfo>& mats, std::vector<NsGroup>& groups,
                        const std::vector<const void*>& src, const std::vector<float*>& bufs,
                        int src_kind, float beta, int nesterov, double* partials,
                        std::vector<int>& part_begin, std::vector<int>& part_count,
                        cudaStream_t s) {
  const int count = static_cast<int>(mats.size());
  part_begin.assign(count, 0);
  part_count.assign(count, 0);
  int global_blk = 0;
  for (int i0 = 0; i0 < count; i0 += ew::kMaxMats) {
    const int i1 = std::min(count, i0 + ew::kMaxMats);
    ew::PrepParams pp{};
    pp.src_kind = src_kind;
    pp.beta = beta;
    pp.omb = 1.0f - beta;
    pp.nesterov = nesterov;
    pp.partials = partials + global_blk;
    int tiles = 0;
    for (int i = i0; i < i1; ++i) {
      const MatInfo& M = mats[i];
      const NsGroup& G = groups[M.group];
      ew::PrepMat& P = pp.mat[i - i0];
      P.src = src[i];
      P.buf = bufs.empty() ? nullptr : bufs[i];
      P.rows = M.rows;
      P.cols = M.cols;
      P.transposed = M.transposed;
      P.tiles_c = (M.cols + ew::kPrepCols - 1) / ew::kPrepCols;
      P.tile_begin = tiles;
      const long long off = static_cast<long long>(M.index) * G.m * G.ldn;
      P.xhi = G.xb[0] + off;
      P.xlo = G.xlo + off;
      P.ld = G.ldn;
      P.vec = (M.cols % 8 == 0);  // every pointer is 16-byte aligned (checked on entry)
      part_begin[i] = global_blk + tiles;
      part_count[i] = prep_tiles(M);
      tiles += part_count[i];
    }
    pp.nmat = i1 - i0;
    pp.ntiles = tiles;
    ProfScope prof(MUON_KERNEL_PREP, s);
    CUDA_TRY(ew::launch_prep(pp, s));
    global_blk += tiles;
  }
  return MUON_OK;
}

// s = 1 / (||u|| + eps) of every matrix into xscale[mat_base + index].
int launch_scale_chunked(const std::vector<MatInfo>& mats, const std::vector<NsGroup>& groups,
                         const double* partials, const std::vector<int>& part_begin,
                         const std::vector<int>& part_count, float* xscale, cudaStream_t s) {
  const int count = static_cast<int>(mats.size());
  for (int i0 = 0; i0 < count; i0 += ew::kMaxMats) {
    const int i1 = std::min(count, i0 + ew::kMaxMats);
    ew::ScaleParams sp{};
    sp.partials = partials;
    sp.eps = 1e-7;  // the same epsilon as kNormEps, in fp64
    for (int i = i0; i < i1; ++i) {
      const MatInfo& M = mats[i];
      const NsGroup& G = groups[M.group];
      ew::ScaleMat& S = sp.mat[i - i0];
      S.part_begin = part_begin[i];
      S.part_count = part_count[i];
      const long long off = static_cast<long long>(M.index) * G.m * G.ldn;
      S.xhi = G.xb[0] + off;
      S.xlo = G.xlo + off;
      S.m = G.m;
      S.n = G.n;
      S.ld = G.ldn;
      S.scale = xscale + G.mat_base + M.index;
    }
    sp.nmat = i1 - i0;
    ProfScope prof(MUON_KERNEL_SCALE, s);
    CUDA_TRY(ew::launch_scale(sp, s));
  }
  return MUON_OK;
}

// Workspace of the bf16 path: prep partials, per-matrix scales, then the
// groups' buffers.  With base null only the size is computed.
struct BfLayout {
  double* partials = nullptr;
  float* xscale = nullptr;
};

size_t bf16_layout(const std::vector<MatInfo>& mats, std::vector<NsGroup>& groups, char* base,
                   BfLayout& L) {
  const size_t nblk = static_cast<size_t>(count_prep_blocks(mats));
  size_t off = 0;
  L.partials = base ? reinterpret_cast<double*>(base + off) : nullptr;
  off = align_up(off + nblk * 8, 1024);
  L.xscale = base ? reinterpret_cast<float*>(base + off) : nullptr;
  off = align_up(off + mats.size() * 4, 1024);
  for (NsGroup& g : groups) off = layout_group(g, base, off, false);
  return off;
}

// prep (momentum or plain read) -> per-matrix scale -> T Newton-Schulz steps.
int run_bf16_path(const std::vector<MatInfo>& mats, std::vector<NsGroup>& groups,
                  const BfLayout& L, const std::vector<const void*>& src,
                  const std::vector<float*>& bufs, int src_kind, float beta, int nesterov,
                  const float* abc, int steps, int* status, int sms, cudaStream_t s,
                  ApplySpec* apply = nullptr) {
  std::vector<int> pb, pc;
  MUON_TRY(launch_prep_chunked(mats, groups, src, bufs, src_kind, beta, nesterov, L.partials, pb,
                               pc, s));
  MUON_TRY(launch_scale_chunked(mats, groups, L.partials, pb, pc, L.xscale, s));
  return run_ns_bf16(groups, steps, abc, status, sms, s, L.xscale, apply);
}

// mode 0: apply into W; 1: bf16 write-back; 2: fp32 write-back.  O of matrix i
// is read from its group's result (X layout, transposed back).  Matrices that
// `done` marks (already applied by the last GEMM) are left out.
int launch_out_chunked(const std::vector<MatInfo>& mats, const std::vector<NsGroup>& groups,
                       const std::vector<Result>& res, const std::vector<void*>& ys, int mode,
                       float lr, float wd, cudaStream_t s, const float* oscale = nullptr,
                       const std::vector<char>* done = nullptr, int cautious = 0,
                       const std::vector<const float*>* rowf = nullptr) {
  std::vector<int> todo;
  for (int i = 0; i < static_cast<int>(mats.size()); ++i)
    if (!done || !(*done)[i]) todo.push_back(i);
  const int count = static_cast<int>(todo.size());
  for (int i0 = 0; i0 < count; i0 += ew::kMaxMats) {
    const int i1 = std::min(count, i0 + ew::kMaxMats);
    ew::OutParams op{};
    op.mode = mode;
    op.lw = lr * wd;
    op.cautious = cautious;
    int tiles = 0;
    for (int t = i0; t < i1; ++t) {
      const int i = todo[t];
      const MatInfo& M = mats[i];
      const NsGroup& G = groups[M.group];
      ew::OutMat& O = op.mat[t - i0];
      O.y = ys[i];
      const long long roff = static_cast<long long>(M.index) * G.m * G.ldn;
      const Result& R = res[M.group];
      O.o = R.f ? R.f + roff : nullptr;
      O.o_hi = R.f ? nullptr : static_cast<const void*>(R.hi + roff);
      O.o_lo = R.f ? nullptr : static_cast<const void*>(R.lo + roff);
      O.rows = M.rows;
      O.cols = M.cols;
      O.o_transposed = M.transposed;
      O.ld = G.ldn;
      O.tiles_c = (M.cols + ew::kTile - 1) / ew::kTile;
      O.tile_begin = tiles;
      O.ls = apply_ls(M, lr);
      O.oscale = oscale ? oscale + G.mat_base + M.index : nullptr;
      O.rowf = rowf ? (*rowf)[i] : nullptr;
      O.vec = (M.cols % 8 == 0) && (G.ldn % 8 == 0) && aligned16(ys[i]);
      tiles += ((M.rows + ew::kTile - 1) / ew::kTile) * O.tiles_c;
    }
    op.nmat = i1 - i0;
    op.ntiles = tiles;
    ProfScope prof(MUON_KERNEL_OUT, s);
    CUDA_TRY(ew::launch_out(op, s));
  }
  return MUON_OK;
}

// Per-neuron rescale (NorMuon reading): row sums of O^2 of every caller W,
// then the state update and the row factors.  rsq / rowf hold one entry per
// W row, matrices in order; rowf_ptrs[i] is matrix i's first factor.
int launch_norm_chunked(const std::vector<MatInfo>& mats, const std::vector<NsGroup>& groups,
                        const std::vector<Result>& res, const float* oscale, float* const* state,
                        float beta2, double* rsq, float* rowf, std::vector<const float*>& rowf_ptrs,
                        cudaStream_t s) {
  const int count = static_cast<int>(mats.size());
  std::vector<long long> base(count);
  long long rows = 0;
  for (int i = 0; i < count; ++i) {
    base[i] = rows;
    rows += mats[i].rows;
  }
  rowf_ptrs.resize(count);
  for (int i = 0; i < count; ++i) rowf_ptrs[i] = rowf + base[i];
  for (int i0 = 0; i0 < count; i0 += ew::kMaxMats) {
    const int i1 = std::min(count, i0 + ew::kMaxMats);
    ew::NormStatParams sp{};
    sp.rsq = rsq;
    int blk = 0;
    for (int i = i0; i < i1; ++i) {
      const MatInfo& M = mats[i];
      const NsGroup& G = groups[M.group];
      const Result& R = res[M.group];
      const long long roff = static_cast<long long>(M.index) * G.m * G.ldn;
      ew::NormMat& N = sp.mat[i - i0];
      N.hi = R.hi + roff;
      N.lo = R.lo + roff;
      N.oscale = oscale ? oscale + G.mat_base + M.index : nullptr;
      N.m = G.m;
      N.n = G.n;
      N.ld = G.ldn;
      N.transposed = M.transposed;
      N.blk_begin = blk;
      N.row_base = base[i];
      blk += M.transposed ? (M.rows + ew::kNormRowsTall - 1) / ew::kNormRowsTall
                          : (M.rows + ew::kNormRowsWide - 1) / ew::kNormRowsWide;
    }
    sp.nmat = i1 - i0;
    sp.nblocks = blk;
    {
      ProfScope prof(MUON_KERNEL_NORM, s);
      CUDA_TRY(ew::launch_norm_stats(sp, s));
    }
    ew::NormFacParams fp{};
    fp.rsq = rsq;
    fp.rowf = rowf;
    fp.beta2 = beta2;
    fp.omb2 = 1.0f - beta2;
    fp.eps = kNeuronEps;
    for (int i = i0; i < i1; ++i) {
      ew::NormFacMat& F = fp.mat[i - i0];
      F.v = state[i];
      F.rows = mats[i].rows;
      F.cols = mats[i].cols;
      F.row_base = base[i];
    }
    fp.nmat = i1 - i0;
    ProfScope prof(MUON_KERNEL_NORM, s);
    CUDA_TRY(ew::launch_norm_factors(fp, s));
  }
  return MUON_OK;
}

int check_shape(long long r, long long c, int i) {
  if (r < 1 || c < 1 || r > kMaxDim || c > kMaxDim)
    return set_err(MUON_ERR_SHAPE, "matrix %d has shape %lldx%lld (each side must be in 1..%d)", i,
                   r, c, kMaxDim);
  return MUON_OK;
}

int check_ptr(const void* p, const char* what, int i) {
  if (!p) return set_err(MUON_ERR_ARG, "%s[%d] is NULL", what, i);
  if (!aligned16(p)) return set_err(MUON_ERR_ARG, "%s[%d] is not 16-byte aligned", what, i);
  return MUON_OK;
}

// ------------------------------------------------- allocation-free variant
// Device scratch of muon_ns_orthogonalize_static.  A file-scope __device__
// array: every GPU that loads this library holds it until the process exits.
// Host code must not pass `g_static_scratch` itself to a kernel (on the host it
// is only a stand-in symbol); its device address comes from
// cudaGetSymbolAddress, looked up once per device.
constexpr size_t kStaticScratchBytes = static_cast<size_t>(24) << 20;  // 24 MiB
constexpr size_t kStaticStatusBytes = 1024;  // status slot used when the caller passes none

struct HooksOff {
  HooksOff() { t_hooks_off = true; }
  ~HooksOff() { t_hooks_off = false; }
};

}  // namespace

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {

std::mutex g_static_mu;
std::map<int, char*> g_static_addr;  // device ordinal -> device address of g_static_scratch

int static_scratch_address(char** out) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_static_mu);
  auto it = g_static_addr.find(dev);
  if (it != g_static_addr.end()) {
    *out = it->second;
    return MUON_OK;
  }
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
  if (e != cudaSuccess || !p)
    return set_err(MUON_ERR_CUDA, "cudaGetSymbolAddress of the static scratch on device %d: %s", dev,
                   cudaGetErrorString(e));
  g_static_addr[dev] = static_cast<char*>(p);
  *out = static_cast<char*>(p);
  return MUON_OK;
}

}  // namespace

// =============================================================================
extern "C" {

int muon_version(void) { return kVersion; }

#ifdef MUON_TRACE
// Trace builds only: device buffer that tensor-core launches stamp into.
int muon_debug_trace(void* dev_buffer) {
  g_trace = static_cast<unsigned long long*>(dev_buffer);
  return MUON_OK;
}
#endif

const char* muon_last_error(void) { return t_err.c_str(); }

int muon_set_wait_timeout_ms(int ms) {
  if (ms < 1 || ms > 600000) return set_err(MUON_ERR_ARG, "timeout %d ms out of range 1..600000", ms);
  std::lock_guard<std::mutex> lk(g_mu);
  g_timeout_ns = static_cast<unsigned long long>(ms) * 1000000ull;
  return MUON_OK;
}

int muon_set_fault_injection(int mode) {
  if (mode < 0 || mode > 1) return set_err(MUON_ERR_ARG, "fault injection mode %d unknown", mode);
  std::lock_guard<std::mutex> lk(g_mu);
  g_inject = mode;
  return MUON_OK;
}

}  // extern "C"

namespace {

// muon_ns_orthogonalize with a table of (a, b, c) per step (host, 3 * steps).
int ns_orthogonalize(int batch, int m, int n, void* const* X_ptrs, const float* abc, int steps,
                     int dtype, void* stream) {
  if (batch < 0 || batch > 65535) return set_err(MUON_ERR_ARG, "batch %d out of range 0..65535", batch);
  if (steps < 0 || steps > kMaxStepsArg) return set_err(MUON_ERR_ARG, "steps %d out of range 0..%d", steps, kMaxStepsArg);
  if (dtype != MUON_BF16 && dtype != MUON_FP32) return set_err(MUON_ERR_ARG, "dtype %d unknown", dtype);
  if (steps > 0 && !abc) return set_err(MUON_ERR_ARG, "coefficient table is NULL");
  for (int i = 0; i < 3 * steps; ++i)
    if (!finite(abc[i])) return set_err(MUON_ERR_ARG, "coefficient %d of step %d is not finite", i % 3, i / 3);
  MUON_TRY(check_shape(m, n, 0));
  if (batch == 0) return MUON_OK;
  if (!X_ptrs) return set_err(MUON_ERR_ARG, "X_ptrs is NULL");
  for (int i = 0; i < batch; ++i) MUON_TRY(check_ptr(X_ptrs[i], "X_ptrs", i));
  DevInfo dev;
  MUON_TRY(device_info(&dev));
  cudaStream_t s = as_stream(stream);
  const bool fp32 = (dtype == MUON_FP32);

  std::vector<std::pair<int, int>> shapes(batch, std::make_pair(m, n));
  std::vector<MatInfo> mats;
  std::vector<NsGroup> groups;
  group_shapes(shapes, mats, groups);
  std::vector<const void*> src(X_ptrs, X_ptrs + batch);
  std::vector<void*> ys(X_ptrs, X_ptrs + batch);
  std::vector<Result> res;
  if (!fp32) {
    assign_mat_base(groups);
    BfLayout L;
    size_t off = bf16_layout(mats, groups, nullptr, L);
    Workspace* ws = nullptr;
    MUON_TRY(get_workspace(s, off, &ws));
    bf16_layout(mats, groups, static_cast<char*>(ws->ptr), L);
    // the last step writes X_T straight into the callers' buffers where it can
    // (only the prep pass reads them, so writing in place is safe)
    ApplySpec wb;
    wb.mats = &mats;
    wb.w = &ys;
    wb.kind = 1;
    wb.done.assign(batch, 0);
    MUON_TRY(run_bf16_path(mats, groups, L, src, {}, ew::kFromBf16, 0.f, 0, abc, steps,
                           ws->status, dev.sms, s, &wb));
    for (NsGroup& g : groups) res.push_back(bf16_result(g, steps));
    MUON_TRY(launch_out_chunked(mats, groups, res, ys, 1, 0.f, 0.f, s, steps == 0 ? L.xscale : nullptr,
                                &wb.done));
    return MUON_OK;
  }
  // fp32 verification path: normalised fp32 X, SIMT GEMMs
  std::vector<long long> numels(batch, static_cast<long long>(m) * n);
  const int nblk = count_flat_blocks(numels);
  size_t off = align_up(static_cast<size_t>(nblk) * 4, 1024);
  for (NsGroup& g : groups) off = layout_group(g, nullptr, off, true);
  Workspace* ws = nullptr;
  MUON_TRY(get_workspace(s, off, &ws));
  char* base = static_cast<char*>(ws->ptr);
  float* partials = reinterpret_cast<float*>(base);
  off = align_up(static_cast<size_t>(nblk) * 4, 1024);
  for (NsGroup& g : groups) off = layout_group(g, base, off, true);
  std::vector<int> pb, pc;
  MUON_TRY(launch_flat_chunked(src, {}, numels, ew::kFromF32, 0.f, 0, partials, pb, pc, s));
  MUON_TRY(launch_cast_chunked(mats, groups, src, {}, ew::kFromF32, 0.f, 0, partials, pb, pc, s));
  std::vector<float*> final_xf;
  MUON_TRY(run_ns_fp32(groups, steps, abc, s, final_xf));
  for (float* f : final_xf) {
    Result r;
    r.f = f;
    res.push_back(r);
  }
  MUON_TRY(launch_out_chunked(mats, groups, res, ys, 2, 0.f, 0.f, s));
  return MUON_OK;
}

std::vector<float> constant_schedule(float a, float b, float c, int steps);

// muon_step with its options: flags (MUON_CAUTIOUS_WD) and, when
// neuron_state is given, the per-neuron rescale of the update (NorMuon
// reading) with second-moment coefficient beta2.
int step_impl(int count, float* const* params, const void* const* grads, float* const* momentum_bufs,
              const int64_t* shapes, float beta, int nesterov, float lr, float wd, int steps,
              const float* schedule, int flags, float* const* neuron_state, float beta2, void* stream) {
  if (count < 0) return set_err(MUON_ERR_ARG, "count %d < 0", count);
  if (steps < 0 || steps > kMaxStepsArg) return set_err(MUON_ERR_ARG, "steps %d out of range 0..%d", steps, kMaxStepsArg);
  if (schedule)
    for (int i = 0; i < 3 * steps; ++i)
      if (!finite(schedule[i]))
        return set_err(MUON_ERR_ARG, "coefficient %d of step %d is not finite", i % 3, i / 3);
  if (!finite(beta) || beta < 0.f || beta > 1.f) return set_err(MUON_ERR_ARG, "beta must be in [0, 1]");
  if (!finite(lr) || !finite(wd)) return set_err(MUON_ERR_ARG, "lr and wd must be finite");
  if (flags & ~MUON_CAUTIOUS_WD) return set_err(MUON_ERR_ARG, "unknown flags 0x%x", flags);
  if (neuron_state && (!finite(beta2) || beta2 < 0.f || beta2 > 1.f))
    return set_err(MUON_ERR_ARG, "beta2 must be in [0, 1]");
  if (count == 0) return MUON_OK;
  if (!params || !grads || !momentum_bufs || !shapes)
    return set_err(MUON_ERR_ARG, "params, grads, momentum_bufs and shapes must be non-NULL");
  std::vector<std::pair<int, int>> shp(count);
  for (int i = 0; i < count; ++i) {
    MUON_TRY(check_shape(shapes[2 * i], shapes[2 * i + 1], i));
    shp[i] = std::make_pair(static_cast<int>(shapes[2 * i]), static_cast<int>(shapes[2 * i + 1]));
    MUON_TRY(check_ptr(params[i], "params", i));
    MUON_TRY(check_ptr(grads[i], "grads", i));
    MUON_TRY(check_ptr(momentum_bufs[i], "momentum_bufs", i));
    if (neuron_state) {
      if (!neuron_state[i]) return set_err(MUON_ERR_ARG, "neuron_state[%d] is NULL", i);
      if (reinterpret_cast<uintptr_t>(neuron_state[i]) & 3u)
        return set_err(MUON_ERR_ARG, "neuron_state[%d] is not 4-byte aligned", i);
    }
  }
  DevInfo dev;
  MUON_TRY(device_info(&dev));
  cudaStream_t s = as_stream(stream);

  std::vector<MatInfo> mats;
  std::vector<NsGroup> groups;
  group_shapes(shp, mats, groups);
  assign_mat_base(groups);
  BfLayout L;
  size_t off = bf16_layout(mats, groups, nullptr, L);
  long long wrows = 0;
  for (const MatInfo& M : mats) wrows += M.rows;
  const size_t norm_off = align_up(off, 1024);
  if (neuron_state) off = align_up(norm_off + static_cast<size_t>(wrows) * 8, 1024) + static_cast<size_t>(wrows) * 4;
  Workspace* ws = nullptr;
  MUON_TRY(get_workspace(s, off, &ws));
  char* base = static_cast<char*>(ws->ptr);
  bf16_layout(mats, groups, base, L);

  std::vector<const void*> gsrc(grads, grads + count);
  std::vector<float*> bufs(momentum_bufs, momentum_bufs + count);
  const std::vector<float> abc = schedule ? std::vector<float>(schedule, schedule + 3 * steps)
                                          : constant_schedule(kCoefA, kCoefB, kCoefC, steps);
  std::vector<void*> ys(params, params + count);
  const int cautious = (flags & MUON_CAUTIOUS_WD) ? 1 : 0;
  // the last step applies the update to W in its epilogue where it can; the
  // per-neuron rescale needs every row's norm first, so it takes the pass
  ApplySpec apply;
  apply.mats = &mats;
  apply.w = &ys;
  apply.lr = lr;
  apply.wd = wd;
  apply.cautious = cautious;
  apply.done.assign(count, 0);
  MUON_TRY(run_bf16_path(mats, groups, L, gsrc, bufs, ew::kFromMomentum, beta, nesterov,
                         abc.data(), steps, ws->status, dev.sms, s, neuron_state ? nullptr : &apply));
  std::vector<Result> res;
  for (NsGroup& g : groups) res.push_back(bf16_result(g, steps));
  const float* oscale = steps == 0 ? L.xscale : nullptr;
  if (!neuron_state)
    return launch_out_chunked(mats, groups, res, ys, 0, lr, wd, s, oscale, &apply.done, cautious);
  double* rsq = reinterpret_cast<double*>(base + norm_off);
  float* rowf = reinterpret_cast<float*>(base + align_up(norm_off + static_cast<size_t>(wrows) * 8, 1024));
  std::vector<const float*> rowf_ptrs;
  MUON_TRY(launch_norm_chunked(mats, groups, res, oscale, neuron_state, beta2, rsq, rowf, rowf_ptrs, s));
  return launch_out_chunked(mats, groups, res, ys, 0, lr, wd, s, oscale, nullptr, cautious, &rowf_ptrs);
}

// muon_apply with its options: flags (MUON_CAUTIOUS_WD) and optional per-row
// factors of O (row_scale[i][r] multiplies row r of matrix i's update first).
int apply_impl(int count, float* const* params, const float* const* updates, const int64_t* shapes,
               float lr, float wd, int flags, const float* const* row_scale, void* stream) {
  if (count < 0) return set_err(MUON_ERR_ARG, "count %d < 0", count);
  if (!finite(lr) || !finite(wd)) return set_err(MUON_ERR_ARG, "lr and wd must be finite");
  if (flags & ~MUON_CAUTIOUS_WD) return set_err(MUON_ERR_ARG, "unknown flags 0x%x", flags);
  if (count == 0) return MUON_OK;
  if (!params || !updates || !shapes) return set_err(MUON_ERR_ARG, "params, updates and shapes must be non-NULL");
  for (int i = 0; i < count; ++i) {
    MUON_TRY(check_shape(shapes[2 * i], shapes[2 * i + 1], i));
    MUON_TRY(check_ptr(params[i], "params", i));
    MUON_TRY(check_ptr(updates[i], "updates", i));
    if (row_scale && (!row_scale[i] || (reinterpret_cast<uintptr_t>(row_scale[i]) & 3u)))
      return set_err(MUON_ERR_ARG, "row_scale[%d] is NULL or not 4-byte aligned", i);
  }
  DevInfo dev;
  MUON_TRY(device_info(&dev));
  cudaStream_t s = as_stream(stream);
  for (int i0 = 0; i0 < count; i0 += ew::kMaxMats) {
    const int i1 = std::min(count, i0 + ew::kMaxMats);
    ew::OutParams op{};
    op.mode = 0;
    op.lw = lr * wd;
    op.cautious = (flags & MUON_CAUTIOUS_WD) ? 1 : 0;
    int tiles = 0;
    for (int i = i0; i < i1; ++i) {
      const int r = static_cast<int>(shapes[2 * i]), c = static_cast<int>(shapes[2 * i + 1]);
      ew::OutMat& O = op.mat[i - i0];
      O.y = params[i];
      O.o = updates[i];
      O.rows = r;
      O.cols = c;
      O.o_transposed = 0;
      O.ld = c;
      O.tiles_c = (c + ew::kTile - 1) / ew::kTile;
      O.tile_begin = tiles;
      const float ratio = static_cast<float>(r) / static_cast<float>(c);
      const float scale = ratio > 1.0f ? sqrtf(ratio) : 1.0f;
      O.ls = lr * scale;
      O.rowf = row_scale ? row_scale[i] : nullptr;
      O.vec = (c % 8 == 0) && aligned16(params[i]) && aligned16(updates[i]);
      tiles += ((r + ew::kTile - 1) / ew::kTile) * O.tiles_c;
    }
    op.nmat = i1 - i0;
    op.ntiles = tiles;
    ProfScope prof(MUON_KERNEL_OUT, s);
    CUDA_TRY(ew::launch_out(op, s));
  }
  return MUON_OK;
}

// The fixed triple as a table of `steps` rows.
std::vector<float> constant_schedule(float a, float b, float c, int steps) {
  std::vector<float> t;
  for (int i = 0; i < steps; ++i) {
    t.push_back(a);
    t.push_back(b);
    t.push_back(c);
  }
  return t;
}

}  // namespace

extern "C" {

int muon_ns_orthogonalize(int batch, int m, int n, void* const* X_ptrs, float a, float b, float c,
                          int steps, int dtype, void* stream) {
  t_err.clear();
  if (steps < 0 || steps > kMaxStepsArg) return set_err(MUON_ERR_ARG, "steps %d out of range 0..%d", steps, kMaxStepsArg);
  if (!finite(a) || !finite(b) || !finite(c)) return set_err(MUON_ERR_ARG, "coefficients must be finite");
  const std::vector<float> abc = constant_schedule(a, b, c, steps);
  return ns_orthogonalize(batch, m, n, X_ptrs, abc.data(), steps, dtype, stream);
}

int muon_ns_orthogonalize_schedule(int batch, int m, int n, void* const* X_ptrs, const float* coeffs,
                                   int steps, int dtype, void* stream) {
  t_err.clear();
  return ns_orthogonalize(batch, m, n, X_ptrs, coeffs, steps, dtype, stream);
}

int muon_ns_orthogonalize_static(int batch, int m, int n, void* const* X_ptrs, float a, float b,
                                 float c, int steps, int* status_dev, void* stream) {
  t_err.clear();
  if (batch < 0 || batch > 65535) return set_err(MUON_ERR_ARG, "batch %d out of range 0..65535", batch);
  if (steps < 0 || steps > kMaxStepsArg) return set_err(MUON_ERR_ARG, "steps %d out of range 0..%d", steps, kMaxStepsArg);
  if (!finite(a) || !finite(b) || !finite(c)) return set_err(MUON_ERR_ARG, "coefficients must be finite");
  MUON_TRY(check_shape(m, n, 0));
  if (status_dev && (reinterpret_cast<uintptr_t>(status_dev) & 3u))
    return set_err(MUON_ERR_ARG, "status_dev is not 4-byte aligned");
  if (batch == 0) return MUON_OK;
  if (!X_ptrs) return set_err(MUON_ERR_ARG, "X_ptrs is NULL");
  for (int i = 0; i < batch; ++i) MUON_TRY(check_ptr(X_ptrs[i], "X_ptrs", i));

  std::vector<std::pair<int, int>> shapes(batch, std::make_pair(m, n));
  std::vector<MatInfo> mats;
  std::vector<NsGroup> groups;
  group_shapes(shapes, mats, groups);
  assign_mat_base(groups);
  BfLayout L;
  const size_t need = bf16_layout(mats, groups, nullptr, L);
  if (need + kStaticStatusBytes > kStaticScratchBytes)
    return set_err(MUON_ERR_SHAPE,
                   "batch %d of %dx%d needs %zu bytes of scratch; the static scratch holds %zu "
                   "(use muon_ns_orthogonalize, which allocates its workspace)",
                   batch, m, n, need + kStaticStatusBytes, kStaticScratchBytes);
  DevInfo dev;
  MUON_TRY(device_info(&dev));
  char* scratch = nullptr;
  MUON_TRY(static_scratch_address(&scratch));
  cudaStream_t s = as_stream(stream);
  int* status = status_dev;
  if (!status) {
    status = reinterpret_cast<int*>(scratch);
    CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int), s));
  }
  HooksOff no_hooks;
  bf16_layout(mats, groups, scratch + kStaticStatusBytes, L);

  std::vector<const void*> src(X_ptrs, X_ptrs + batch);
  const std::vector<float> abc = constant_schedule(a, b, c, steps);
  std::vector<void*> ys(X_ptrs, X_ptrs + batch);
  ApplySpec wb;  // as in ns_orthogonalize: the last step writes X_T where it can
  wb.mats = &mats;
  wb.w = &ys;
  wb.kind = 1;
  wb.done.assign(batch, 0);
  MUON_TRY(run_bf16_path(mats, groups, L, src, {}, ew::kFromBf16, 0.f, 0, abc.data(), steps, status,
                         dev.sms, s, &wb));
  std::vector<Result> res;
  for (NsGroup& g : groups) res.push_back(bf16_result(g, steps));
  MUON_TRY(launch_out_chunked(mats, groups, res, ys, 1, 0.f, 0.f, s, steps == 0 ? L.xscale : nullptr,
                              &wb.done));
  return MUON_OK;
}

int muon_step(int count, float* const* params, const void* const* grads,
              float* const* momentum_bufs, const int64_t* shapes, float beta, int nesterov,
              float lr, float wd, int steps, void* stream) {
  t_err.clear();
  return step_impl(count, params, grads, momentum_bufs, shapes, beta, nesterov, lr, wd, steps, nullptr,
                   0, nullptr, 0.f, stream);
}

int muon_step_ex(int count, float* const* params, const void* const* grads,
                 float* const* momentum_bufs, const int64_t* shapes, float beta, int nesterov,
                 float lr, float wd, int steps, const float* schedule, int flags,
                 float* const* neuron_state, float beta2, void* stream) {
  t_err.clear();
  return step_impl(count, params, grads, momentum_bufs, shapes, beta, nesterov, lr, wd, steps, schedule,
                   flags, neuron_state, beta2, stream);
}

int muon_momentum(int count, const void* const* grads, float* const* momentum_bufs,
                  const int64_t* shapes, float beta, int nesterov, float* sumsq_out,
                  void* stream) {
  t_err.clear();
  if (count < 0) return set_err(MUON_ERR_ARG, "count %d < 0", count);
  if (!finite(beta) || beta < 0.f || beta > 1.f) return set_err(MUON_ERR_ARG, "beta must be in [0, 1]");
  if (count == 0) return MUON_OK;
  if (!grads || !momentum_bufs || !shapes) return set_err(MUON_ERR_ARG, "grads, momentum_bufs and shapes must be non-NULL");
  std::vector<long long> numels(count);
  for (int i = 0; i < count; ++i) {
    MUON_TRY(check_shape(shapes[2 * i], shapes[2 * i + 1], i));
    numels[i] = shapes[2 * i] * shapes[2 * i + 1];
    MUON_TRY(check_ptr(grads[i], "grads", i));
    MUON_TRY(check_ptr(momentum_bufs[i], "momentum_bufs", i));
  }
  DevInfo dev;
  MUON_TRY(device_info(&dev));
  cudaStream_t s = as_stream(stream);
  const int nblk = count_flat_blocks(numels);
  Workspace* ws = nullptr;
  MUON_TRY(get_workspace(s, static_cast<size_t>(nblk) * 4, &ws));
  float* partials = static_cast<float*>(ws->ptr);
  std::vector<const void*> gsrc(grads, grads + count);
  std::vector<float*> bufs(momentum_bufs, momentum_bufs + count);
  std::vector<int> pb, pc;
  MUON_TRY(launch_flat_chunked(gsrc, bufs, numels, ew::kFromMomentum, beta, nesterov, partials, pb,
                               pc, s));
  if (sumsq_out) {
    for (int i0 = 0; i0 < count; i0 += ew::kMaxMats) {
      const int i1 = std::min(count, i0 + ew::kMaxMats);
      ew::SumParams sp{};
      sp.partials = partials;
      sp.out = sumsq_out + i0;
      sp.nmat = i1 - i0;
      for (int i = i0; i < i1; ++i) {
        sp.part_begin[i - i0] = pb[i];
        sp.part_count[i - i0] = pc[i];
      }
      ProfScope prof(MUON_KERNEL_SUMS, s);
      CUDA_TRY(ew::launch_sums(sp, s));
    }
  }
  return MUON_OK;
}

int muon_apply(int count, float* const* params, const float* const* updates, const int64_t* shapes,
               float lr, float wd, void* stream) {
  t_err.clear();
  return apply_impl(count, params, updates, shapes, lr, wd, 0, nullptr, stream);
}

int muon_apply_ex(int count, float* const* params, const float* const* updates, const int64_t* shapes,
                  float lr, float wd, int flags, const float* const* row_scale, void* stream) {
  t_err.clear();
  return apply_impl(count, params, updates, shapes, lr, wd, flags, row_scale, stream);
}

static int stage_common(int batch, int m, int k, DevInfo* dev, Workspace** ws, cudaStream_t s) {
  if (batch < 0 || batch > 65535) return set_err(MUON_ERR_ARG, "batch %d out of range", batch);
  MUON_TRY(check_shape(m, k, 0));
  if (m % 8 || k % 8) return set_err(MUON_ERR_SHAPE, "m (%d) and k/n (%d) must be multiples of 8", m, k);
  MUON_TRY(device_info(dev));
  MUON_TRY(get_encoder());
  MUON_TRY(get_workspace(s, 0, ws));
  return MUON_OK;
}

int muon_gram_bf16(int batch, int m, int k, const void* X, void* A, void* stream) {
  t_err.clear();
  if (batch == 0) return MUON_OK;
  if (!X || !A || !aligned16(X) || !aligned16(A)) return set_err(MUON_ERR_ARG, "X and A must be non-NULL and 16-byte aligned");
  cudaStream_t s = as_stream(stream);
  DevInfo dev;
  Workspace* ws = nullptr;
  MUON_TRY(stage_common(batch, m, k, &dev, &ws, s));
  tc::Params P;
  init_tc_params(P, ws->status, 0.f, 0.f, 0.f);
  P.grp[0] = tc_group(batch, m, m, k, true, 0);
  MUON_TRY(sym_maps(P.map[0], X, m, k, k, static_cast<long long>(m) * k, A, m,
                    static_cast<long long>(m) * m, batch, false));
  P.ngroups = 1;
  P.total_tiles = batch * P.grp[0].tiles_per_mat;
  return launch_tc(tc::kGram, P, dev.sms, s);
}

int muon_poly_bf16(int batch, int m, const void* A, void* B, float b, float c, void* stream) {
  t_err.clear();
  if (batch == 0) return MUON_OK;
  if (!A || !B || !aligned16(A) || !aligned16(B)) return set_err(MUON_ERR_ARG, "A and B must be non-NULL and 16-byte aligned");
  if (A == B) return set_err(MUON_ERR_ARG, "B must not alias A");
  cudaStream_t s = as_stream(stream);
  DevInfo dev;
  Workspace* ws = nullptr;
  MUON_TRY(stage_common(batch, m, m, &dev, &ws, s));
  tc::Params P;
  init_tc_params(P, ws->status, 0.f, b, c);
  const long long as = static_cast<long long>(m) * m;
  P.grp[0] = tc_group(batch, m, m, m, true, 0);
  MUON_TRY(sym_maps(P.map[0], A, m, m, m, as, B, m, as, batch, true));
  P.ngroups = 1;
  P.total_tiles = batch * P.grp[0].tiles_per_mat;
  return launch_tc(tc::kPoly, P, dev.sms, s);
}

int muon_bx_bf16(int batch, int m, int n, const void* B, const void* Xhi, void* Xlo, void* Xhi_out,
                 float a, void* stream) {
  t_err.clear();
  if (batch == 0) return MUON_OK;
  if (!B || !Xhi || !Xlo || !Xhi_out || !aligned16(B) || !aligned16(Xhi) || !aligned16(Xlo) ||
      !aligned16(Xhi_out))
    return set_err(MUON_ERR_ARG, "B, Xhi, Xlo and Xhi_out must be non-NULL and 16-byte aligned");
  if (Xhi == Xhi_out) return set_err(MUON_ERR_ARG, "Xhi_out must not alias Xhi");
  if (m > n) return set_err(MUON_ERR_SHAPE, "muon_bx_bf16 expects m <= n (got %dx%d)", m, n);
  if (n % 16)
    return set_err(MUON_ERR_SHAPE, "muon_bx_bf16 needs n (%d) a multiple of 16 (16-byte rows of the int8 Xlo)", n);
  cudaStream_t s = as_stream(stream);
  DevInfo dev;
  Workspace* ws = nullptr;
  MUON_TRY(stage_common(batch, m, n, &dev, &ws, s));
  tc::Params P;
  init_tc_params(P, ws->status, a, 0.f, 0.f);
  const long long xs = static_cast<long long>(m) * n, as = static_cast<long long>(m) * m;
  P.grp[0] = tc_group(batch, m, n, m, false, 0);
  MUON_TRY(bx_maps(P.map[0], B, m, as, Xhi, Xlo, Xhi_out, m, n, n, xs, batch));
  P.ngroups = 1;
  P.total_tiles = batch * P.grp[0].tiles_per_mat;
  return launch_tc(tc::kBx, P, dev.sms, s);
}

int muon_bx_apply_bf16(int batch, int m, int n, int ldx, const void* B, int ldb, const void* Xhi,
                       void* Xlo, float* const* W_ptrs, int tall, float a, float lr, float wd, int flags,
                       void* stream) {
  t_err.clear();
  if (flags & ~MUON_CAUTIOUS_WD) return set_err(MUON_ERR_ARG, "unknown flags 0x%x", flags);
  if (batch < 0 || batch > 65535) return set_err(MUON_ERR_ARG, "batch %d out of range 0..65535", batch);
  if (!finite(a) || !finite(lr) || !finite(wd)) return set_err(MUON_ERR_ARG, "a, lr and wd must be finite");
  if (batch == 0) return MUON_OK;
  MUON_TRY(check_shape(m, n, 0));
  if (m > n) return set_err(MUON_ERR_SHAPE, "muon_bx_apply_bf16 expects m <= n (got %dx%d)", m, n);
  if (ldx < n || ldx % 16 || ldb < m || ldb % 8)
    return set_err(MUON_ERR_SHAPE,
                   "row strides: ldx (%d) must be >= n (%d) and a multiple of 16, ldb (%d) >= m (%d) "
                   "and a multiple of 8", ldx, n, ldb, m);
  if (!B || !Xhi || !Xlo || !aligned16(B) || !aligned16(Xhi) || !aligned16(Xlo))
    return set_err(MUON_ERR_ARG, "B, Xhi and Xlo must be non-NULL and 16-byte aligned");
  if (!W_ptrs) return set_err(MUON_ERR_ARG, "W_ptrs is NULL");
  for (int i = 0; i < batch; ++i) MUON_TRY(check_ptr(W_ptrs[i], "W_ptrs", i));
  DevInfo dev;
  MUON_TRY(device_info(&dev));
  MUON_TRY(get_encoder());
  cudaStream_t s = as_stream(stream);

  // One shape group over the caller's contiguous batch, laid out as the
  // iteration's workspace would be (matrix strides m * ldx and m * ldb).
  std::vector<NsGroup> gs(1);
  NsGroup& G = gs[0];
  G.batch = batch;
  G.m = m;
  G.n = n;
  G.ldn = ldx;
  G.ldm = ldb;
  G.mat_base = 0;
  G.B = static_cast<bf16*>(const_cast<void*>(B));
  G.xb[0] = static_cast<bf16*>(const_cast<void*>(Xhi));
  G.xlo = static_cast<int8_t*>(Xlo);
  std::vector<MatInfo> mats(batch);
  for (int i = 0; i < batch; ++i)
    mats[i] = MatInfo{tall ? n : m, tall ? m : n, m, n, tall ? 1 : 0, 0, i};
  std::vector<void*> ws_ptrs(W_ptrs, W_ptrs + batch);
  ApplySpec apply;
  apply.mats = &mats;
  apply.w = &ws_ptrs;
  apply.kind = 0;
  apply.lr = lr;
  apply.wd = wd;
  apply.cautious = (flags & MUON_CAUTIOUS_WD) ? 1 : 0;
  apply.done.assign(batch, 0);
  tc::LaunchApply table;
  MUON_TRY(build_apply_table(gs, 0, 1, apply, table));
  // Matrices the epilogue cannot update (past the table, or W rows not 16-byte
  // strided) get X' as the pair: hi into a workspace buffer, q into Xlo.
  bool any_pair = false;
  for (int i = 0; i < batch; ++i) any_pair |= !apply.done[i];
  Workspace* ws = nullptr;
  const size_t hi_bytes = static_cast<size_t>(batch) * m * ldx * 2;
  MUON_TRY(get_workspace(s, any_pair ? hi_bytes : 0, &ws));
  G.xb[1] = any_pair ? static_cast<bf16*>(ws->ptr) : G.xb[0];

  tc::Params P;
  init_tc_params(P, ws->status, a, 0.f, 0.f);
  P.grp[0] = tc_group(batch, m, n, m, false, 0);
  const long long xs = static_cast<long long>(m) * ldx, as = static_cast<long long>(m) * ldb;
  MUON_TRY(bx_maps(P.map[0], G.B, ldb, as, G.xb[0], G.xlo, G.xb[1], m, n, ldx, xs, batch,
                   tc::bx_apply_chunk()));
  P.ngroups = 1;
  P.total_tiles = batch * P.grp[0].tiles_per_mat;
  MUON_TRY(launch_tc(tc::kBxApply, P, dev.sms, s, &table));
  if (!any_pair) return MUON_OK;
  std::vector<Result> res(1);
  res[0].hi = G.xb[1];
  res[0].lo = G.xlo;
  return launch_out_chunked(mats, gs, res, ws_ptrs, 0, lr, wd, s, nullptr, &apply.done, apply.cautious);
}

int muon_get_status(void* stream) {
  t_err.clear();
  cudaStream_t s = as_stream(stream);
  CUDA_TRY(cudaStreamSynchronize(s));
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  int* st = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_ws.find({dev, reinterpret_cast<uintptr_t>(s)});
    if (it == g_ws.end() || !it->second.status) return MUON_OK;
    st = it->second.status;
  }
  int v = 0;
  CUDA_TRY(cudaMemcpy(&v, st, sizeof(int), cudaMemcpyDeviceToHost));
  if (v != 0) {
    CUDA_TRY(cudaMemset(st, 0, sizeof(int)));
    set_err(v, "device status %d (a bounded device-side wait ran out)", v);
  }
  return v;
}

int muon_profile_begin(void) {
  t_err.clear();
  std::lock_guard<std::mutex> lk(g_mu);
  for (ProfRec& r : g_prof) {
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_prof.clear();
  g_prof_on = true;
  return MUON_OK;
}

int muon_profile_end(int kinds, double* total_ms, int* launches) {
  t_err.clear();
  std::vector<ProfRec> recs;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    g_prof_on = false;
    recs.swap(g_prof);
  }
  for (int k = 0; k < kinds; ++k) {
    if (total_ms) total_ms[k] = 0.0;
    if (launches) launches[k] = 0;
  }
  int n = 0;
  int rc = MUON_OK;
  for (ProfRec& r : recs) {
    float ms = 0.f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess && rc == MUON_OK)
      rc = set_err(MUON_ERR_CUDA, "kernel timing: %s", cudaGetErrorString(e));
    if (r.kind >= 0 && r.kind < kinds) {
      if (total_ms) total_ms[r.kind] += ms;
      if (launches) launches[r.kind] += 1;
    }
    ++n;
  }
  {
    std::lock_guard<std::mutex> lk(g_mu);
    for (ProfRec& r : recs) {
      g_event_pool.push_back(r.a);
      g_event_pool.push_back(r.b);
    }
  }
  return rc == MUON_OK ? n : rc;
}

int muon_workspace_bytes(void* stream, long long* bytes) {
  t_err.clear();
  if (!bytes) return set_err(MUON_ERR_ARG, "bytes is NULL");
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_ws.find({dev, reinterpret_cast<uintptr_t>(stream)});
  *bytes = 0;
  if (it != g_ws.end()) *bytes = static_cast<long long>(it->second.bytes) + (it->second.status ? 256 : 0);
  return MUON_OK;
}

int muon_release(void) {
  t_err.clear();
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  CUDA_TRY(cudaDeviceSynchronize());
  {
    // a context re-created after a reset places the static scratch anew
    std::lock_guard<std::mutex> lk(g_static_mu);
    g_static_addr.erase(dev);
  }
  std::lock_guard<std::mutex> lk(g_mu);
  for (auto it = g_ws.begin(); it != g_ws.end();) {
    if (it->first.first == dev) {
      if (it->second.ptr) cudaFree(it->second.ptr);
      if (it->second.status) cudaFree(it->second.status);
      it = g_ws.erase(it);
    } else {
      ++it;
    }
  }
  return MUON_OK;
}

}  // extern "C"
