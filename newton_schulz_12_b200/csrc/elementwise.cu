// Memory-bound steps of the Muon update on sm_100a.
//
//   prep_kernel   the bf16 path's first pass: momentum lerp + Nesterov blend
//                 (buf written in place), u written to the iteration layout
//                 (transposed to rows <= cols when the matrix is tall) as the
//                 pair bf16 hi + int8 lo, and an fp64 partial of sum(u^2) per
//                 block.  The 1 / ||u|| factor is applied later, inside the
//                 first Newton-Schulz step.
//   scale_kernel  per-matrix s = 1 / (||u||_F + eps) from those partials.
//   flat_kernel   momentum on its own (muon_momentum) or the partial of
//                 sum(x^2) of the fp32 verification path; 128-bit accesses,
//                 fixed-order block reduction.
//   cast_kernel   fp32 verification path: X0 = x / (||x||_F + eps) in fp32,
//                 transposed when tall; 64x64 tiles through shared memory so
//                 both the read and the (possibly transposed) write coalesce.
//   out_kernel    W' = (W - lw W) - ls O (the apply), or the write-back of the
//                 result into the caller's bf16 / fp32 buffer, with O read
//                 (from fp32 or from the pair) through the same transposing tile.
//   sums_kernel   per-matrix sum of flat_kernel's partials.
//   norm_stats_kernel / norm_factor_kernel
//                 the per-neuron rescale (NorMuon reading): row sums of O^2 of
//                 the caller's W rows, the fp32 second-moment state and the
//                 factor each row of O is multiplied by before the apply.
//
// Operation order of momentum and apply is fixed with explicit round-to-nearest
// intrinsics (no contraction into FMA) so that they are bit-exact against an
// fp32 computation of the same order:
//   buf' = (beta*buf) + (omb*g),  u = (omb*g) + (beta*buf'),  omb = 1 - beta
//   W'   = (W - lw*W) - ls*O,     lw = lr*wd,  ls = lr*scale
//          (cautious decay: the lw*W term only where W and O have the same sign)
// ("NanoGPT Speedrun: The Ultimate Guide...", section "Optimizer and Training
// Strategy Tuning": orthogonalise after the Nesterov-momentum update.)
#include "common.cuh"
#include "internal.h"

namespace muon {
namespace ew {

constexpr int kVec = 8;                                    // elements per thread access
constexpr int kIters = kFlatChunk / (kFlatThreads * kVec);  // 4

template <typename Mats>
__device__ __forceinline__ int find_mat(const Mats& mats, int nmat, int key_of_block) {
  int lo = 0, hi = nmat - 1;
  while (lo < hi) {  // last index with begin <= key
    const int mid = (lo + hi + 1) >> 1;
    if (mats[mid].blk_begin <= key_of_block) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ float block_sum_fixed(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
  if (threadIdx.x == 0) {
    for (int w = 0; w < kFlatThreads / 32; ++w) s += red[w];
  }
  return s;
}

struct MomentumOp {
  float beta, omb;
  int nesterov;
  __device__ __forceinline__ float operator()(float g, float& buf) const {
    const float nb = __fadd_rn(__fmul_rn(beta, buf), __fmul_rn(omb, g));
    buf = nb;
    return nesterov ? __fadd_rn(__fmul_rn(omb, g), __fmul_rn(beta, nb)) : nb;
  }
};

__global__ void __launch_bounds__(kFlatThreads) flat_kernel(const __grid_constant__ FlatParams p) {
  __shared__ float red[kFlatThreads / 32];
  const int blk = blockIdx.x;
  const int mi = find_mat(p.mat, p.nmat, blk);
  const FlatMat& M = p.mat[mi];
  const long long start = static_cast<long long>(blk - M.blk_begin) * kFlatChunk;
  const long long end = min(start + kFlatChunk, M.numel);
  const MomentumOp op{p.beta, p.omb, p.nesterov};
  float acc = 0.f;

#pragma unroll
  for (int it = 0; it < kIters; ++it) {
    const long long e = start + static_cast<long long>(it * kFlatThreads + threadIdx.x) * kVec;
    if (e >= end) continue;
    if (e + kVec <= end) {
      float x[kVec];
      if (p.src_kind == kFromF32) {
        const float4* s4 = reinterpret_cast<const float4*>(static_cast<const float*>(M.src) + e);
        const float4 a = s4[0], b = s4[1];
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
      } else {
        const uint4 w = *reinterpret_cast<const uint4*>(static_cast<const bf16*>(M.src) + e);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          x[2 * h] = bf16_bits_to_f32(static_cast<uint16_t>(ws[h] & 0xFFFFu));
          x[2 * h + 1] = bf16_bits_to_f32(static_cast<uint16_t>(ws[h] >> 16));
        }
      }
      if (p.src_kind == kFromMomentum) {
        float4* b4 = reinterpret_cast<float4*>(M.buf + e);
        float4 m0 = b4[0], m1 = b4[1];
        float mb[kVec] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
        for (int q = 0; q < kVec; ++q) {
          const float u = op(x[q], mb[q]);
          acc = fmaf(u, u, acc);
        }
        b4[0] = make_float4(mb[0], mb[1], mb[2], mb[3]);
        b4[1] = make_float4(mb[4], mb[5], mb[6], mb[7]);
      } else {
#pragma unroll
        for (int q = 0; q < kVec; ++q) acc = fmaf(x[q], x[q], acc);
      }
    } else {
      for (long long q = e; q < end; ++q) {
        float x;
        if (p.src_kind == kFromF32) x = static_cast<const float*>(M.src)[q];
        else x = bf16_bits_to_f32(static_cast<const uint16_t*>(M.src)[q]);
        if (p.src_kind == kFromMomentum) {
          float mb = M.buf[q];
          const float u = op(x, mb);
          M.buf[q] = mb;
          acc = fmaf(u, u, acc);
        } else {
          acc = fmaf(x, x, acc);
        }
      }
    }
  }
  const float s = block_sum_fixed(acc, red);
  if (threadIdx.x == 0) p.partials[blk] = s;
}

// Sum of a matrix's partials in a fixed order: lane l adds partials l, l+32,
// ... then a fixed xor tree.  Called by one full warp.
__device__ __forceinline__ float warp_sum_partials(const float* partials, int begin, int count) {
  const int lane = threadIdx.x & 31;
  float s = 0.f;
  for (int q = lane; q < count; q += 32) s += partials[begin + q];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

__global__ void sums_kernel(const __grid_constant__ SumParams p) {
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (w >= p.nmat) return;
  const float s = warp_sum_partials(p.partials, p.part_begin[w], p.part_count[w]);
  if ((threadIdx.x & 31) == 0) p.out[w] = s;
}

constexpr int kTileThreads = 256;

template <typename Mats>
__device__ __forceinline__ int find_tile_mat(const Mats& mats, int nmat, int t) {
  int lo = 0, hi = nmat - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (mats[mid].tile_begin <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ---------------------------------------------------------------- tile kernels
// One 64x64 tile per block; thread t owns two runs of 8 consecutive elements
// (rows t/8 and t/8 + 32, columns 8*(t%8) .. +7) and moves them with 128-bit
// accesses when the rows are 16-byte aligned (`vec`), else element by element.
// A tall matrix's tile is transposed through shared memory so that both the
// read and the write run along rows.

__device__ __forceinline__ void unpack_bf16x8(const uint4 w, float (&x)[8]) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    x[2 * h] = bf16_bits_to_f32(static_cast<uint16_t>(ws[h] & 0xFFFFu));
    x[2 * h + 1] = bf16_bits_to_f32(static_cast<uint16_t>(ws[h] >> 16));
  }
}

// u[k] = U[r][c + k] for k < 8 (0 outside the matrix); U is the momentum
// update (recomputed from g and the updated buffer with flat_kernel's
// rounding) or the caller's X.
__device__ __forceinline__ void load_u8(const CastParams& p, const CastMat& M, int r, int c,
                                        float (&u)[8]) {
  const int cnt = r < M.rows ? min(8, M.cols - c) : 0;
  const long long idx = static_cast<long long>(r) * M.cols + c;
  if (cnt == 8 && M.vec) {
    if (p.src_kind == kFromF32) {
      const float4* s4 = reinterpret_cast<const float4*>(static_cast<const float*>(M.src0) + idx);
      const float4 a = s4[0], b = s4[1];
      u[0] = a.x; u[1] = a.y; u[2] = a.z; u[3] = a.w;
      u[4] = b.x; u[5] = b.y; u[6] = b.z; u[7] = b.w;
      return;
    }
    float g[8];
    unpack_bf16x8(*reinterpret_cast<const uint4*>(static_cast<const bf16*>(M.src0) + idx), g);
    if (p.src_kind == kFromMomentum) {
      const float4* b4 = reinterpret_cast<const float4*>(M.src1 + idx);
      const float4 a = b4[0], b = b4[1];
      const float nb[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int k = 0; k < 8; ++k)
        u[k] = p.nesterov ? __fadd_rn(__fmul_rn(p.omb, g[k]), __fmul_rn(p.beta, nb[k])) : nb[k];
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) u[k] = g[k];
    }
    return;
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float v = 0.f;
    if (k < cnt) {
      if (p.src_kind == kFromF32) {
        v = static_cast<const float*>(M.src0)[idx + k];
      } else {
        const float g = bf16_bits_to_f32(static_cast<const uint16_t*>(M.src0)[idx + k]);
        if (p.src_kind == kFromMomentum) {
          const float nb = M.src1[idx + k];
          v = p.nesterov ? __fadd_rn(__fmul_rn(p.omb, g), __fmul_rn(p.beta, nb)) : nb;
        } else {
          v = g;
        }
      }
    }
    u[k] = v;
  }
}

// X[i][j + k] = u[k] / den in fp32 (the verification path).
__device__ __forceinline__ void store_x8(const CastMat& M, int i, int j, int m, int n, float den,
                                         const float (&u)[8]) {
  if (i >= m || j >= n) return;
  const long long o = static_cast<long long>(i) * M.ld + j;
  float x[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) x[k] = __fdiv_rn(u[k], den);
  if (j + 8 <= n) {  // the workspace row stride is a multiple of 8: always aligned
    float4* f4 = reinterpret_cast<float4*>(M.xf + o);
    f4[0] = make_float4(x[0], x[1], x[2], x[3]);
    f4[1] = make_float4(x[4], x[5], x[6], x[7]);
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < n - j) M.xf[o + k] = x[k];
  }
}

__global__ void __launch_bounds__(kTileThreads) cast_kernel(const __grid_constant__ CastParams p) {
  __shared__ float tile[kTile][kTile + 1];
  __shared__ float s_den;
  const int mi = find_tile_mat(p.mat, p.nmat, blockIdx.x);
  const CastMat& M = p.mat[mi];
  const int local = blockIdx.x - M.tile_begin;
  const int ti = local / M.tiles_n, tj = local - ti * M.tiles_n;
  const int m = M.transposed ? M.cols : M.rows;  // X is m x n
  const int n = M.transposed ? M.rows : M.cols;
  const int i0 = ti * kTile, j0 = tj * kTile;
  if (threadIdx.x < 32) {
    const float ss = warp_sum_partials(p.partials, M.part_begin, M.part_count);
    if (threadIdx.x == 0) s_den = __fadd_rn(__fsqrt_rn(ss), p.eps);
  }
  const int y = threadIdx.x >> 3, xg = (threadIdx.x & 7) * 8;
  float u[2][8];
  if (!M.transposed) {
#pragma unroll
    for (int h = 0; h < 2; ++h) load_u8(p, M, i0 + y + 32 * h, j0 + xg, u[h]);
    __syncthreads();
    const float den = s_den;
#pragma unroll
    for (int h = 0; h < 2; ++h) store_x8(M, i0 + y + 32 * h, j0 + xg, m, n, den, u[h]);
  } else {
    // X[i0 + a][j0 + b] = U[j0 + b][i0 + a]: read U rows j0.., columns i0..
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      load_u8(p, M, j0 + y + 32 * h, i0 + xg, u[h]);
#pragma unroll
      for (int k = 0; k < 8; ++k) tile[y + 32 * h][xg + k] = u[h][k];
    }
    __syncthreads();
    const float den = s_den;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float t[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) t[k] = tile[xg + k][y + 32 * h];
      store_x8(M, i0 + y + 32 * h, j0 + xg, m, n, den, t);
    }
  }
}

// o[k] = O[r][c + k] read from the m x n result buffer (row stride ld) as laid
// out there: rows r of that buffer, columns c.. (0 outside it).  The buffer is
// fp32, or the pair bf16 hi + int8 residual.
__device__ __forceinline__ void load_o8(const OutMat& M, int r, int c, int orows, int ocols,
                                        float (&o)[8]) {
  const int cnt = r < orows ? min(8, ocols - c) : 0;
  const long long idx = static_cast<long long>(r) * M.ld + c;
  if (M.o_hi) {
    const float f = M.oscale ? *M.oscale : 1.0f;
    if (cnt == 8 && M.vec) {
      pair_decode8(*reinterpret_cast<const uint4*>(static_cast<const bf16*>(M.o_hi) + idx),
                   *reinterpret_cast<const uint2*>(static_cast<const int8_t*>(M.o_lo) + idx), o);
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] *= f;
      return;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float v = 0.f;
      if (k < cnt) {
        const uint32_t fb = static_cast<uint32_t>(static_cast<const uint16_t*>(M.o_hi)[idx + k]) << 16;
        const int q = static_cast<const int8_t*>(M.o_lo)[idx + k];
        v = fmaf(static_cast<float>(q), lo8_unit(fb), __uint_as_float(fb)) * f;
      }
      o[k] = v;
    }
    return;
  }
  if (cnt == 8 && M.vec) {
    const float4* s4 = reinterpret_cast<const float4*>(M.o + idx);
    const float4 a = s4[0], b = s4[1];
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
    return;
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) o[k] = k < cnt ? M.o[idx + k] : 0.f;
}

// One weight after the apply: W' = (W - d) - ls O with d = fl(lw W), or d = 0
// where cautious decay masks it (W and O not of the same sign), each
// operation rounded to nearest, no fused multiply-add.
__device__ __forceinline__ float apply_one(float w, float o, float lw, float ls, int cautious) {
  const bool decay = !cautious || (w > 0.f && o > 0.f) || (w < 0.f && o < 0.f);
  const float d = decay ? __fmul_rn(lw, w) : 0.0f;
  return __fsub_rn(__fsub_rn(w, d), __fmul_rn(ls, o));
}

// Y[r][c + k] op= o[k]: the apply W' = (W - lw W) - ls O, or a write-back.
// With a row factor (NorMuon), O's row r is fl(O * rowf[r]) first.
__device__ __forceinline__ void update_y8(const OutParams& p, const OutMat& M, int r, int c,
                                          float (&o)[8]) {
  if (r >= M.rows || c >= M.cols) return;
  const long long idx = static_cast<long long>(r) * M.cols + c;
  const int cnt = min(8, M.cols - c);
  if (p.mode == 0 && M.rowf) {
    const float f = M.rowf[r];
#pragma unroll
    for (int k = 0; k < 8; ++k) o[k] = __fmul_rn(o[k], f);
  }
  if (cnt == 8 && M.vec) {
    if (p.mode == 0) {
      float4* w4 = reinterpret_cast<float4*>(static_cast<float*>(M.y) + idx);
      const float4 a = w4[0], b = w4[1];
      float w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int k = 0; k < 8; ++k) w[k] = apply_one(w[k], o[k], p.lw, M.ls, p.cautious);
      w4[0] = make_float4(w[0], w[1], w[2], w[3]);
      w4[1] = make_float4(w[4], w[5], w[6], w[7]);
    } else if (p.mode == 1) {
      uint4 v;
      v.x = pack_bf16x2(o[0], o[1]);
      v.y = pack_bf16x2(o[2], o[3]);
      v.z = pack_bf16x2(o[4], o[5]);
      v.w = pack_bf16x2(o[6], o[7]);
      *reinterpret_cast<uint4*>(static_cast<bf16*>(M.y) + idx) = v;
    } else {
      float4* y4 = reinterpret_cast<float4*>(static_cast<float*>(M.y) + idx);
      y4[0] = make_float4(o[0], o[1], o[2], o[3]);
      y4[1] = make_float4(o[4], o[5], o[6], o[7]);
    }
    return;
  }
  for (int k = 0; k < cnt; ++k) {
    if (p.mode == 0) {
      float* W = static_cast<float*>(M.y);
      W[idx + k] = apply_one(W[idx + k], o[k], p.lw, M.ls, p.cautious);
    } else if (p.mode == 1) {
      static_cast<bf16*>(M.y)[idx + k] = __float2bfloat16_rn(o[k]);
    } else {
      static_cast<float*>(M.y)[idx + k] = o[k];
    }
  }
}

__global__ void __launch_bounds__(kTileThreads) out_kernel(const __grid_constant__ OutParams p) {
  __shared__ float tile[kTile][kTile + 1];
  const int mi = find_tile_mat(p.mat, p.nmat, blockIdx.x);
  const OutMat& M = p.mat[mi];
  const int local = blockIdx.x - M.tile_begin;
  const int tr = local / M.tiles_c, tcn = local - tr * M.tiles_c;
  const int r0 = tr * kTile, c0 = tcn * kTile;
  const int y = threadIdx.x >> 3, xg = (threadIdx.x & 7) * 8;
  if (!M.o_transposed) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float o[8];
      load_o8(M, r0 + y + 32 * h, c0 + xg, M.rows, M.cols, o);
      update_y8(p, M, r0 + y + 32 * h, c0 + xg, o);
    }
  } else {
    // O[r0 + a][c0 + b] = buffer[c0 + b][r0 + a]
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float o[8];
      load_o8(M, c0 + y + 32 * h, r0 + xg, M.cols, M.rows, o);
#pragma unroll
      for (int k = 0; k < 8; ++k) tile[y + 32 * h][xg + k] = o[k];
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float o[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] = tile[xg + k][y + 32 * h];
      update_y8(p, M, r0 + y + 32 * h, c0 + xg, o);
    }
  }
}

// ------------------------------------------------------------------ prep kernel
// One kPrepRows x kPrepCols tile of the caller's matrix per block (8192
// elements, as a flat_kernel block).  Thread t owns column group t % 16
// (eight consecutive columns) of rows t / 16 + 16 h, h = 0..3, and issues all
// of its loads before any arithmetic.  A wide matrix's hi / lo are written
// straight from registers (X = U); a tall one's go through a shared-memory
// transpose (X = U^T) so that the writes also run along X's rows.
constexpr int kPrepThreads = 256;
#ifndef MUON_PREP_MIN_BLOCKS
#define MUON_PREP_MIN_BLOCKS 3  // resident blocks per SM the register budget aims for
#endif
constexpr int kPrepUnits = kPrepRows * kPrepCols / (kPrepThreads * 8);  // 4 runs of 8 per thread

// Eight values of u as the pair: bf16 hi (16 bytes) and int8 lo (8 bytes).
__device__ __forceinline__ void store_pair8(void* hi_base, void* lo_base, long long off, int cnt,
                                            const float (&v)[8]) {
  uint4 hi;
  uint2 lo;
  pair_encode8(v, hi, lo);
  if (cnt == 8) {  // the workspace row stride is a multiple of 16: aligned
    *reinterpret_cast<uint4*>(static_cast<bf16*>(hi_base) + off) = hi;
    *reinterpret_cast<uint2*>(static_cast<int8_t*>(lo_base) + off) = lo;
    return;
  }
  const uint32_t h[4] = {hi.x, hi.y, hi.z, hi.w};
  const uint32_t l[2] = {lo.x, lo.y};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    if (k < cnt) {
      static_cast<uint16_t*>(hi_base)[off + k] = static_cast<uint16_t>(h[k >> 1] >> (16 * (k & 1)));
      static_cast<uint8_t*>(lo_base)[off + k] = static_cast<uint8_t>(l[k >> 2] >> (8 * (k & 3)));
    }
  }
}

// Fixed-order fp64 block sum (result in thread 0); contains a block barrier.
__device__ __forceinline__ double block_sum_f64(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double s = 0.0;
  if (threadIdx.x == 0) {
    for (int w = 0; w < kPrepThreads / 32; ++w) s += red[w];
  }
  return s;
}

__global__ void __launch_bounds__(kPrepThreads, MUON_PREP_MIN_BLOCKS) prep_kernel(const __grid_constant__ PrepParams p) {
  __shared__ float tile[kPrepRows][kPrepCols + 1];
  __shared__ double red[kPrepThreads / 32];
  const int mi = find_tile_mat(p.mat, p.nmat, blockIdx.x);
  const PrepMat& M = p.mat[mi];
  const int local = blockIdx.x - M.tile_begin;
  const int tr = local / M.tiles_c, tcn = local - tr * M.tiles_c;
  const int r0 = tr * kPrepRows, c0 = tcn * kPrepCols;
  const int cg = threadIdx.x & 15, ry = threadIdx.x >> 4;
  const int c = c0 + 8 * cg;
  const MomentumOp op{p.beta, p.omb, p.nesterov};
  const bool mom = (p.src_kind == kFromMomentum);
  float u[kPrepUnits][8];

  if (M.vec) {
    // cols % 8 == 0: a run is either wholly inside the row or wholly outside
    uint4 g4[kPrepUnits];
    float4 b4[kPrepUnits][2];
#pragma unroll
    for (int h = 0; h < kPrepUnits; ++h) {
      const int r = r0 + ry + 16 * h;
      if (r < M.rows && c < M.cols) {
        const long long idx = static_cast<long long>(r) * M.cols + c;
        g4[h] = *reinterpret_cast<const uint4*>(static_cast<const bf16*>(M.src) + idx);
        if (mom) {
          const float4* q = reinterpret_cast<const float4*>(M.buf + idx);
          b4[h][0] = q[0];
          b4[h][1] = q[1];
        }
      }
    }
#pragma unroll
    for (int h = 0; h < kPrepUnits; ++h) {
      const int r = r0 + ry + 16 * h;
      if (r < M.rows && c < M.cols) {
        float x[8];
        unpack_bf16x8(g4[h], x);
        if (mom) {
          float mb[8] = {b4[h][0].x, b4[h][0].y, b4[h][0].z, b4[h][0].w,
                         b4[h][1].x, b4[h][1].y, b4[h][1].z, b4[h][1].w};
#pragma unroll
          for (int k = 0; k < 8; ++k) u[h][k] = op(x[k], mb[k]);
          float4* q = reinterpret_cast<float4*>(M.buf + static_cast<long long>(r) * M.cols + c);
          q[0] = make_float4(mb[0], mb[1], mb[2], mb[3]);
          q[1] = make_float4(mb[4], mb[5], mb[6], mb[7]);
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) u[h][k] = x[k];
        }
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) u[h][k] = 0.f;
      }
    }
  } else {
#pragma unroll
    for (int h = 0; h < kPrepUnits; ++h) {
      const int r = r0 + ry + 16 * h;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float v = 0.f;
        if (r < M.rows && c + k < M.cols) {
          const long long idx = static_cast<long long>(r) * M.cols + c + k;
          const float x = bf16_bits_to_f32(static_cast<const uint16_t*>(M.src)[idx]);
          if (mom) {
            float mb = M.buf[idx];
            v = op(x, mb);
            M.buf[idx] = mb;
          } else {
            v = x;
          }
        }
        u[h][k] = v;
      }
    }
  }

  double acc = 0.0;
#pragma unroll
  for (int h = 0; h < kPrepUnits; ++h)
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const double w = u[h][k];
      acc = fma(w, w, acc);
    }

  if (!M.transposed) {
#pragma unroll
    for (int h = 0; h < kPrepUnits; ++h) {
      const int r = r0 + ry + 16 * h;
      if (r < M.rows && c < M.cols)
        store_pair8(M.xhi, M.xlo, static_cast<long long>(r) * M.ld + c, min(8, M.cols - c), u[h]);
    }
  } else {
#pragma unroll
    for (int h = 0; h < kPrepUnits; ++h)
#pragma unroll
      for (int k = 0; k < 8; ++k) tile[ry + 16 * h][8 * cg + k] = u[h][k];
  }
  const double s = block_sum_f64(acc, red);  // its barrier also publishes the tile
  if (threadIdx.x == 0) p.partials[blockIdx.x] = s;
  if (M.transposed) {
    // X rows c0 + xr (caller columns), X columns r0 + 8 xg .. +7 (caller rows)
    const int xg = threadIdx.x & 7;
#pragma unroll
    for (int q = 0; q < kPrepUnits; ++q) {
      const int xr = (threadIdx.x >> 3) + 32 * q;
      const int xrow = c0 + xr, xcol = r0 + 8 * xg;
      if (xrow < M.cols && xcol < M.rows) {
        float v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = tile[8 * xg + k][xr];
        store_pair8(M.xhi, M.xlo, static_cast<long long>(xrow) * M.ld + xcol, min(8, M.rows - xcol), v);
      }
    }
  }
}

// One block per matrix: s = 1 / (||u||_F + eps) from the matrix's partials in
// a fixed order.  Outside [2^-40, 2^40] the norm is first brought to [1, 2)
// by scaling the workspace pair with an exact power of two (both factors at
// least 2^-64), so that the first Gram product of the unnormalised pair
// neither overflows nor loses its leading terms to underflow.
constexpr int kScaleThreads = 256;

__global__ void __launch_bounds__(kScaleThreads) scale_kernel(const __grid_constant__ ScaleParams p) {
  __shared__ float s_f[2];
  __shared__ double s_red[kScaleThreads / 32];
  const ScaleMat& M = p.mat[blockIdx.x];
  {
    // thread t adds partials t, t+256, ...; then a fixed xor tree per warp
    // and the eight warp sums in order: a fixed summation order
    double ss = 0.0;
    for (int q = threadIdx.x; q < M.part_count; q += kScaleThreads) ss += p.partials[M.part_begin + q];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
      ss = 0.0;
      for (int w = 0; w < kScaleThreads / 32; ++w) ss += s_red[w];
      double den = sqrt(ss) + p.eps;
      float f1 = 1.0f, f2 = 1.0f;
      if (isfinite(den) && (den > 0x1p40 || den < 0x1p-40)) {
        const int e = ilogb(den);  // e <= 150 for any fp32 / bf16 u: both factors are normal fp32
        f1 = ldexpf(1.0f, -(e / 2));
        f2 = ldexpf(1.0f, -(e - e / 2));
        den = (den * f1) * f2;
      }
      s_f[0] = f1;
      s_f[1] = f2;
      *M.scale = static_cast<float>(1.0 / den);
    }
  }
  __syncthreads();
  const float f1 = s_f[0], f2 = s_f[1];
  if (f1 == 1.0f && f2 == 1.0f) return;
  // lo counts in units of hi's exponent, so only hi changes
  const long long units = static_cast<long long>(M.m) * M.ld / 8;
  for (long long i = threadIdx.x; i < units; i += kScaleThreads) {
    uint4* ph = reinterpret_cast<uint4*>(static_cast<bf16*>(M.xhi)) + i;
    float h[8];
    unpack_bf16x8(*ph, h);
    uint32_t oh[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) oh[k] = pack_bf16x2((h[2 * k] * f1) * f2, (h[2 * k + 1] * f1) * f2);
    *ph = make_uint4(oh[0], oh[1], oh[2], oh[3]);
  }
}

// ------------------------------------------------------- per-neuron rescale
// Row sums of O^2 over the caller's W rows (NorMuon reading), from the bf16
// part of O's pair: hi is O rounded to nearest bf16, |O - hi| <= 2^-8 |hi|
// (half a bf16 unit), so every square, and with it every row sum, is within
// a relative 2^-7 + 2^-14 of O's (the update itself carries a 3e-2
// tolerance).  Reading 2 B per
// element instead of 3, with no residual to decode, keeps the pass at the
// memory's rate.  O = oscale * pair when oscale is set (zero steps): the
// sums are then scaled by oscale^2.  W = X: a block takes kNormRowsWide rows
// of X, four per warp, the lanes running along the row with 16-byte loads;
// W = X^T: a block takes kNormRowsTall columns of X, eight threads per row
// segment, 32 row groups summed in shared memory in a fixed order.  Each
// thread sums its own squares in fp32 (at most max(m, n) / 32 of them:
// relative error below 1e-5), the threads' partials are combined in fp64;
// every order is fixed.
constexpr int kNormThreads = 256;
constexpr int kNormFactorThreads = 1024;  // one block per matrix: up to 4096 rows

// Squares of eight bf16 values (one 16-byte word of hi) added to acc[0..7].
__device__ __forceinline__ void add_squares8(const uint4 w, float (&acc)[8]) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const float a = __uint_as_float(ws[h] << 16), b = __uint_as_float(ws[h] & 0xFFFF0000u);
    acc[2 * h] = fmaf(a, a, acc[2 * h]);
    acc[2 * h + 1] = fmaf(b, b, acc[2 * h + 1]);
  }
}

// The 16-byte word of hi at (row i, columns c .. c+7), zeros past column n
// (rows are 16-byte strided, ld % 16 == 0, and c % 8 == 0).
__device__ __forceinline__ uint4 load_hi8(const NormMat& M, int i, int c) {
  const bf16* row = static_cast<const bf16*>(M.hi) + static_cast<long long>(i) * M.ld;
  if (c + 8 <= M.n) return *reinterpret_cast<const uint4*>(row + c);
  uint32_t h[4] = {0u, 0u, 0u, 0u};
  const uint16_t* r16 = reinterpret_cast<const uint16_t*>(row);
  for (int k = 0; k < 8 && c + k < M.n; ++k) h[k >> 1] |= static_cast<uint32_t>(r16[c + k]) << (16 * (k & 1));
  return make_uint4(h[0], h[1], h[2], h[3]);
}

constexpr int kNormBatch = 8;  // 16-byte loads a thread has in flight

// At most 64 registers, so that four blocks (32 warps) share an SM: the pass
// is bound by the loads each SM keeps in flight.
__global__ void __launch_bounds__(kNormThreads, 4) norm_stats_kernel(const __grid_constant__ NormStatParams p) {
  __shared__ double red[32][kNormRowsTall + 1];
  int lo = 0, hi = p.nmat - 1;  // last matrix whose first block is <= blockIdx.x
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.mat[mid].blk_begin <= static_cast<int>(blockIdx.x)) lo = mid; else hi = mid - 1;
  }
  const NormMat& M = p.mat[lo];
  const int local = blockIdx.x - M.blk_begin;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const double s2 = M.oscale ? static_cast<double>(*M.oscale) * static_cast<double>(*M.oscale) : 1.0;
  if (!M.transposed) {
    // two of the warp's rows at a time, the lanes along them, four words of
    // each row in flight per lane; each lane's squares of a row summed in
    // fp32 in a fixed order, the lanes in fp64
    constexpr int kB = kNormBatch / 2;
    for (int j = 0; j < kNormRowsWide / 8; j += 2) {
      const int ia = local * kNormRowsWide + warp * (kNormRowsWide / 8) + j, ib = ia + 1;
      if (ia >= M.m) break;  // warp-uniform
      const bool has_b = ib < M.m;
      float pa[8], pb[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) pa[k] = pb[k] = 0.f;
      for (int c0 = 8 * lane; c0 < M.n; c0 += 256 * kB) {
        uint4 wa[kB], wb[kB];
#pragma unroll
        for (int q = 0; q < kB; ++q) {
          const int c = c0 + 256 * q;
          wa[q] = c < M.n ? load_hi8(M, ia, c) : make_uint4(0u, 0u, 0u, 0u);
          wb[q] = (has_b && c < M.n) ? load_hi8(M, ib, c) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int q = 0; q < kB; ++q)
          if (c0 + 256 * q < M.n) {  // rows shorter than a batch: no idle squares
            add_squares8(wa[q], pa);
            add_squares8(wb[q], pb);
          }
      }
      double a = 0.0, b = 0.0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        a += static_cast<double>(pa[k]);
        b += static_cast<double>(pb[k]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
      }
      if (lane == 0) {
        p.rsq[M.row_base + ia] = a * s2;
        if (has_b) p.rsq[M.row_base + ib] = b * s2;
      }
    }
    return;
  }
  const int u = threadIdx.x & 7, g = threadIdx.x >> 3;
  const int c0 = local * kNormRowsTall;
  // each thread's squares of a column (at most m / 32 of them) summed in
  // fp32 in order, the 32 row groups in fp64
  float acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.f;
  if (c0 + 8 * u < M.n) {
    for (int i0 = g; i0 < M.m; i0 += 32 * kNormBatch) {
      uint4 w[kNormBatch];
#pragma unroll
      for (int q = 0; q < kNormBatch; ++q)
        w[q] = i0 + 32 * q < M.m ? load_hi8(M, i0 + 32 * q, c0 + 8 * u) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int q = 0; q < kNormBatch; ++q)
        if (i0 + 32 * q < M.m) add_squares8(w[q], acc);
    }
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) red[g][8 * u + k] = static_cast<double>(acc[k]);
  __syncthreads();
  if (threadIdx.x < kNormRowsTall && c0 + static_cast<int>(threadIdx.x) < M.n) {
    double s = 0.0;
    for (int q = 0; q < 32; ++q) s += red[q][threadIdx.x];
    p.rsq[M.row_base + c0 + threadIdx.x] = s * s2;
  }
}

// One block per matrix: the state update and the row factors (see NormFacParams).
__global__ void __launch_bounds__(kNormFactorThreads) norm_factor_kernel(const __grid_constant__ NormFacParams p) {
  __shared__ double red[2][kNormFactorThreads / 32];
  __shared__ double s_g;
  const NormFacMat& M = p.mat[blockIdx.x];
  const double* rsq = p.rsq + M.row_base;
  double s0 = 0.0, s1 = 0.0;
  for (int i = threadIdx.x; i < M.rows; i += kNormFactorThreads) {
    const double rs = rsq[i];
    const float r32 = __double2float_rn(rs / static_cast<double>(M.cols));
    const float v = __fadd_rn(__fmul_rn(p.beta2, M.v[i]), __fmul_rn(p.omb2, r32));
    M.v[i] = v;
    const double f = 1.0 / sqrt(static_cast<double>(v) + p.eps);
    s0 += rs;
    s1 += f * f * rs;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s0 += __shfl_xor_sync(0xffffffffu, s0, o);
    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
  }
  if ((threadIdx.x & 31) == 0) {
    red[0][threadIdx.x >> 5] = s0;
    red[1][threadIdx.x >> 5] = s1;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double t0 = 0.0, t1 = 0.0;
    for (int w = 0; w < kNormFactorThreads / 32; ++w) {
      t0 += red[0][w];
      t1 += red[1][w];
    }
    s_g = t1 > 0.0 ? sqrt(t0 / t1) : 1.0;
  }
  __syncthreads();
  const double gsc = s_g;
  for (int i = threadIdx.x; i < M.rows; i += kNormFactorThreads) {
    const double f = 1.0 / sqrt(static_cast<double>(M.v[i]) + p.eps);  // this thread wrote v[i]
    p.rowf[M.row_base + i] = __double2float_rn(f * gsc);
  }
}

cudaError_t launch_norm_stats(const NormStatParams& p, cudaStream_t s) {
  if (p.nblocks <= 0) return cudaSuccess;
  norm_stats_kernel<<<p.nblocks, kNormThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_norm_factors(const NormFacParams& p, cudaStream_t s) {
  if (p.nmat <= 0) return cudaSuccess;
  norm_factor_kernel<<<p.nmat, kNormFactorThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_prep(const PrepParams& p, cudaStream_t s) {
  if (p.ntiles <= 0) return cudaSuccess;
  prep_kernel<<<p.ntiles, kPrepThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_scale(const ScaleParams& p, cudaStream_t s) {
  if (p.nmat <= 0) return cudaSuccess;
  scale_kernel<<<p.nmat, kScaleThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_flat(const FlatParams& p, cudaStream_t s) {
  if (p.nblocks <= 0) return cudaSuccess;
  flat_kernel<<<p.nblocks, kFlatThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_cast(const CastParams& p, cudaStream_t s) {
  if (p.ntiles <= 0) return cudaSuccess;
  cast_kernel<<<p.ntiles, kTileThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_out(const OutParams& p, cudaStream_t s) {
  if (p.ntiles <= 0) return cudaSuccess;
  out_kernel<<<p.ntiles, kTileThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_sums(const SumParams& p, cudaStream_t s) {
  if (p.nmat <= 0) return cudaSuccess;
  const int warps_per_block = 4;
  sums_kernel<<<(p.nmat + warps_per_block - 1) / warps_per_block, 32 * warps_per_block, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace ew
}  // namespace muon
