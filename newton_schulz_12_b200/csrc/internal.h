// Host-side interface between the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace muon {

// ----------------------------------------------------------------- tcgen05 GEMMs
namespace tc {

constexpr int kMaxGroups = 4;        // shape groups per launch
constexpr int BM = 128;              // tile rows per CTA (TMEM lanes)
constexpr int PM = 2 * BM;           // tile rows per CTA pair (one M = 256 pair MMA)
constexpr int BN = 256;              // tile columns (fp32 TMEM columns per accumulator)
constexpr int BNH = BN / 2;          // rows of the column operand each CTA of a pair stages
constexpr int BK = 64;               // K per stage: one 128-byte swizzle row of bf16
constexpr int kChunk = 32;           // base epilogue chunk width (columns)
#ifndef MUON_SYM_CHUNK
#define MUON_SYM_CHUNK 64
#endif
// Epilogue chunk width of the symmetric-output kernels (kGram / kPoly): 32 or 64.
constexpr int kSymChunk = MUON_SYM_CHUNK;
static_assert(kSymChunk == 32 || kSymChunk == 64, "symmetric chunk width");
// Warp roles: warp 0 copies operands, warp 1 issues the MMAs, warps
// 2 .. 1 + epilogue warps do the epilogue math (their count per kernel kind
// is in gemm_tc.cu), then the IO warp (stores) and, for kPoly / kBx /
// kBxApply, a loader warp (epilogue operand copies).

// kBxApply: the last step's kBx, whose epilogue also applies the result to
// the caller's weights (ApplyTable) instead of writing X_T.
enum Epi : int { kGram = 0, kPoly = 1, kBx = 2, kBxApply = 3 };

// Work unit: a PM x BN pair tile of D, rows split between the two CTAs of a
// cluster (CTA rank r owns rows [PM*tm2 + BM*r, +BM)).
struct Group {
  int batch;  // matrices in the group
  int m;      // rows of D
  int n;      // columns of D (= m for kGram / kPoly)
  int k;      // reduction length
  int tiles_m;        // pair-tile rows: ceil(m / PM)
  int tiles_n;        // tile columns: ceil(n / BN)
  int tiles_per_mat;  // pair tiles per matrix
  int tile_begin;     // first pair tile of the group in the launch
  int mat_base;       // index of the group's first matrix in Params::xscale
};

// Tensor maps of one group (3-D: {inner, rows, batch}).
// kBx uses e = hi chunk of X (read), mt = lo chunk of X (int8, read and
// written in place), d = hi chunk of X' (written); 64 x 128 boxes, hi with
// 128-byte swizzle, lo with 64-byte swizzle.
struct Maps {
  CUtensorMap p;   // rows of D: X (kGram), A (kPoly), B (kBx); K-major, box 64 x 128
  CUtensorMap q;   // columns of D: X / A K-major box 64 x 128; X MN-major box 64 x 64 (kBx)
  CUtensorMap e;   // epilogue input chunk, bf16 kSymChunk x 128: A (kPoly); hi of X (kBx)
  CUtensorMap d;   // direct output chunk, bf16 kSymChunk x 128: A (kGram), B (kPoly); hi of X' (kBx)
  CUtensorMap mt;  // mirrored output chunk, bf16 128 x kSymChunk (kGram / kPoly); lo of X (kBx)
  CUtensorMap s;   // symmetrised diagonal block half, bf16 64 x 128 (kGram / kPoly)
};

struct Params {
  Maps map[kMaxGroups];
  Group grp[kMaxGroups];
  int ngroups;
  int total_tiles;  // pair tiles
  float a, b, c;
  // Per-matrix factor s of X = s * (hi + lo), or null (s = 1): kGram scales
  // A by s^2, kBx scales X' by s.
  const float* xscale;
  int* status;
  unsigned long long timeout_ns;
  int inject;  // 1: withhold one operand copy in CTA 0 (timeout-path test)
  unsigned long long* trace;  // timestamps (only recorded in builds with MUON_TRACE)
  // 1: the pairs take the tiles in descending order, so a launch starts on
  // the matrices whose operands the previous launch touched last (still in L2)
  int reverse;
};

// Final-step apply (kBxApply): per matrix of the launch, either X_T is written
// as the pair (mode 0; the apply runs as its own pass later), or the caller's
// fp32 W is updated in place from O = X_T, W' = (W - lw W) - ls O, with W
// read and written through its own tensor map: mode 1, W has X's layout
// (boxes of 32 x 128, one per 32 columns of a chunk); mode 2, W = X^T (a tall
// matrix; box 32 x chunk width, four per chunk).
constexpr int kMaxApply = 160;  // matrices per launch with a table entry (the table is a
                                // __grid_constant__ parameter: about 22 KB at 160)

// A kBx launch may carry the same table with mode 3: the matrix's X_T goes to
// the caller's bf16 buffer in X's layout (its tensor map; box 64 x 128) as
// the hi of the pair, i.e. X_T rounded to nearest, and no residual is kept.
struct ApplyMat {
  int mode;  // 0, 1 or 2 as above (kBxApply), 0 or 3 (kBx)
  float ls;  // fl(lr * scale)
};

template <int N>
struct ApplyTable {
  CUtensorMap w[N];
  ApplyMat mat[N];
  int nmat;      // entries in use; matrices past them take mode 0
  int mat_base;  // Group::mat_base value of entry 0
  float lw;      // fl(lr * wd)
  int cautious;  // 1: decay only where W and O have the same sign
};
using LaunchApply = ApplyTable<kMaxApply>;

// Trace layout (MUON_TRACE builds): per CTA < kTraceCtas, per tile < kTraceTiles,
// kTraceSlots %globaltimer stamps: 0 copier first issue, 1 copier last issue,
// 2 MMA start, 3 MMA last commit, 4 epilogue start, 5..11 chunk starts, 12
// end; kGram / kPoly chunk kNCh-3, compute leader: 13 accumulator loaded, 14
// operand chunk landed, 15 staging pair free, 16 chunk handed to the IO
// thread; IO thread: 17 operand chunk consumed, 18 chunk ready, 19 stores
// issued and the oldest pair released.
constexpr int kTraceCtas = 16, kTraceTiles = 24, kTraceSlots = 20;

// Symmetric-output pair tiles per m x m matrix: the 256 x 256 tiles on or
// above the diagonal.
inline int sym_tiles(int m) {
  const int t = (m + PM - 1) / PM;
  return t * (t + 1) / 2;
}

size_t smem_bytes(int epi);
// Epilogue chunk width (columns) of kBxApply: its launch takes maps of X's
// pair with boxes this wide, and mode-2 W maps with boxes of 32 x this.
int bx_apply_chunk();
// `max_pairs` bounds the number of CTA pairs (clusters) of the persistent grid;
// `apply` is the table of a kBxApply launch (required) or of a kBx launch
// (optional; ignored by the other kinds).
cudaError_t launch(int epi, const Params& p, int max_pairs, cudaStream_t stream,
                   const LaunchApply* apply = nullptr);

}  // namespace tc

// ----------------------------------------------------------- fp32 SIMT GEMMs
namespace simt {

enum Mode : int { kGram = 0, kPoly = 1, kBx = 2 };

struct Params {
  int batch, m, n;  // D is m x n (n = m for kGram / kPoly); K = k
  int k;
  const float* P;   // rows of D: X (kGram), A (kPoly), B (kBx)
  const float* Q;   // X (kGram, k-contiguous rows), A (kPoly), X (kBx, n-contiguous rows)
  const float* E;   // epilogue operand: A (kPoly), X (kBx)
  float* D;
  long long ldp, ldq, lde, ldd;  // row strides (elements)
  long long sp, sq, se, sd;      // matrix strides (elements)
  float a, b, c;
};

cudaError_t launch(int mode, const Params& p, cudaStream_t stream);

}  // namespace simt

// ----------------------------------------------------------- elementwise steps
namespace ew {

constexpr int kMaxMats = 128;  // matrices per launch
constexpr int kFlatThreads = 256;
constexpr int kFlatChunk = 8192;  // elements per block of the flat kernels
constexpr int kTile = 64;         // tile edge of the transposing kernels

enum SrcKind : int { kFromMomentum = 0, kFromBf16 = 1, kFromF32 = 2 };

struct FlatMat {
  const void* src;  // grad (bf16) for momentum; X (bf16/f32) for sumsq
  float* buf;       // momentum buffer (in/out), momentum only
  long long numel;
  int blk_begin;    // first block of this matrix
};

struct FlatParams {
  FlatMat mat[kMaxMats];
  int nmat, nblocks;
  int src_kind;       // kFromMomentum, kFromBf16, kFromF32
  float beta, omb;
  int nesterov;
  float* partials;    // one per block
};

struct CastMat {
  const void* src0;   // grad (bf16) or X (bf16 / f32)
  const float* src1;  // updated momentum buffer (kFromMomentum) or null
  int rows, cols;     // source layout
  int transposed;     // rows > cols: X = U^T
  int tiles_n;        // 64-wide tiles along X's columns
  int tile_begin;
  int part_begin, part_count;
  float* xf;          // fp32 X (m x n, row stride ld)
  long long ld;
  int vec;            // source rows are 16-byte aligned (cols % 8 == 0): 128-bit loads
};

struct CastParams {
  CastMat mat[kMaxMats];
  int nmat, ntiles;
  int src_kind;
  float beta, omb;
  int nesterov;
  float eps;
  const float* partials;
};

// Apply (W' = (W - lw W) - ls O) or write-back (Y = cast(O)) over tiles of the
// caller's matrix; O is read from an m x n buffer, transposed when needed.
struct OutMat {
  void* y;            // W (fp32, in/out) or destination X (bf16 / f32)
  const float* o;     // fp32 update / result (X layout, or W layout if !o_transposed); or null
  const void* o_hi;   // else the result as the pair bf16 hi + int8 lo (X layout)
  const void* o_lo;
  int rows, cols;     // caller layout of y
  int o_transposed;   // O[r][s] = o[s * ld + r]
  long long ld;
  int tiles_c;        // 64-wide tiles along y's columns
  int tile_begin;
  float ls;           // fl(lr * scale)
  const float* oscale;  // O = oscale[0] * (hi + lo) when set (result of zero steps)
  const float* rowf;  // apply only: O's row r (caller layout) is multiplied by rowf[r] first, or null
  int vec;            // cols % 8 == 0 and ld % 8 == 0: 128-bit accesses
};

struct OutParams {
  OutMat mat[kMaxMats];
  int nmat, ntiles;
  int mode;           // 0: apply, 1: write bf16, 2: write f32
  float lw;           // fl(lr * wd)
  int cautious;       // apply only: decay only where W and O have the same sign
};

// Per-neuron rescale of the update (NorMuon reading).  For each row r of the
// caller's W (rows x cols) with O its update:
//   rsq_r  = sum over the row of bf16(O)^2              (fp64, fixed order)
//   v'_r   = fl(fl(beta2 v_r) + fl(omb2 fl32(rsq_r / cols)))     (fp32 state)
//   f_r    = 1 / sqrt(v'_r + eps)                        (fp64)
//   g      = sqrt(sum_r rsq_r / sum_r f_r^2 rsq_r)       (1 if the sum is 0)
//   rowf_r = fl32(f_r g)      -- O's row r is multiplied by rowf_r before the apply,
// so the update keeps its Frobenius norm and only its split over rows changes.
// The row sums read the bf16 part of the result pair (O rounded to nearest
// bf16) in X's layout (W = X, or W = X^T when transposed); the apply pass
// then multiplies the pair's value.
struct NormMat {
  const void* hi;     // bf16 part of O's pair (X layout, m x n, row stride ld)
  const void* lo;     // its int8 residual (not read by the row sums)
  const float* oscale;  // O = fl(oscale[0] * pair) when set, else the pair's value
  int m, n;
  long long ld;
  int transposed;     // W rows are X's columns
  int blk_begin;
  long long row_base; // index of the matrix's first W row in rsq / rowf
};

struct NormStatParams {
  NormMat mat[kMaxMats];
  int nmat, nblocks;
  double* rsq;
};

struct NormFacMat {
  float* v;           // the caller's second-moment state, one fp32 per W row (in/out)
  int rows, cols;     // W
  long long row_base;
};

struct NormFacParams {
  NormFacMat mat[kMaxMats];
  int nmat;
  const double* rsq;
  float* rowf;
  float beta2, omb2;
  double eps;
};

constexpr int kNormRowsWide = 32;   // W rows per stats block when W = X (rows of X)
constexpr int kNormRowsTall = 64;   // W rows per stats block when W = X^T (columns of X)

// One pass over the caller's matrices: momentum (or a plain read of X), the
// Nesterov blend u, and u written to the workspace as the pair bf16 hi + int8 lo
// (transposed when tall), plus a partial sum of u^2 per block.  Blocks cover
// kPrepRows x kPrepCols tiles of the caller's layout.
constexpr int kPrepRows = 64, kPrepCols = 128;

struct PrepMat {
  const void* src;    // grad (bf16) or X (bf16)
  float* buf;         // momentum buffer (in/out), or null
  int rows, cols;     // caller layout
  int transposed;     // rows > cols: X = U^T
  int tiles_c;        // tiles along the caller's columns
  int tile_begin;
  void* xhi;          // workspace X (m x n, row stride ld): hi (bf16) and lo (int8) of u
  void* xlo;
  long long ld;
  int vec;            // cols % 8 == 0: 128-bit accesses of the caller's rows
};

struct PrepParams {
  PrepMat mat[kMaxMats];
  int nmat, ntiles;
  int src_kind;       // kFromMomentum or kFromBf16
  float beta, omb;
  int nesterov;
  double* partials;   // sum of u^2 per block (fp64: no overflow for any bf16 / fp32 u)
};

// Per-matrix scale of the first Newton-Schulz step: s = 1 / (||u||_F + eps)
// from the partials; matrices with ||u|| outside [2^-40, 2^40] have their
// workspace pair rescaled by an exact power of two first.
struct ScaleMat {
  int part_begin, part_count;
  void* xhi;          // workspace pair of the matrix (m rows, row stride ld)
  void* xlo;
  int m, n;
  long long ld;
  float* scale;       // destination of s
};

struct ScaleParams {
  ScaleMat mat[kMaxMats];
  int nmat;
  const double* partials;
  double eps;
};

struct SumParams {
  const float* partials;
  int part_begin[kMaxMats];
  int part_count[kMaxMats];
  float* out;
  int nmat;
};

cudaError_t launch_flat(const FlatParams& p, cudaStream_t s);
cudaError_t launch_cast(const CastParams& p, cudaStream_t s);
cudaError_t launch_out(const OutParams& p, cudaStream_t s);
cudaError_t launch_sums(const SumParams& p, cudaStream_t s);
cudaError_t launch_prep(const PrepParams& p, cudaStream_t s);
cudaError_t launch_scale(const ScaleParams& p, cudaStream_t s);
cudaError_t launch_norm_stats(const NormStatParams& p, cudaStream_t s);
cudaError_t launch_norm_factors(const NormFacParams& p, cudaStream_t s);

}  // namespace ew

}  // namespace muon
