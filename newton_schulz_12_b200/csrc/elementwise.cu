// Memory-bound steps of the Muon update on sm_100a.
//
//   flat_kernel   momentum lerp + Nesterov blend (buf written in place) and a
//                 per-block partial of sum(u^2); or, for the plain
//                 orthogonalisation entry, the partial of sum(x^2) only.
//                 128-bit loads/stores, fixed-order block reduction.
//   cast_kernel   X0 = u / (||u||_F + eps), transposed to rows <= cols when the
//                 matrix is tall, written as the fp32 master X and its bf16
//                 operand copy.  64x64 tiles staged through shared memory so
//                 both the read and the (possibly transposed) write coalesce.
//   out_kernel    W' = (W - lw W) - ls O (the apply), or the write-back of the
//                 result into the caller's bf16 / fp32 buffer, with O read
//                 through the same transposing tile.
//   sums_kernel   per-matrix sum of the partials (same order as cast_kernel).
//
// Operation order of momentum and apply is fixed with explicit round-to-nearest
// intrinsics (no contraction into FMA) so that they are bit-exact against an
// fp32 computation of the same order:
//   buf' = (beta*buf) + (omb*g),  u = (omb*g) + (beta*buf'),  omb = 1 - beta
//   W'   = (W - lw*W) - ls*O,     lw = lr*wd,  ls = lr*scale
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
  // source region: U rows [sr0, sr0+64), cols [sc0, sc0+64)
  const int sr0 = M.transposed ? j0 : i0;
  const int sc0 = M.transposed ? i0 : j0;
  const int tx = threadIdx.x & (kTile - 1), ty = threadIdx.x >> 6;
#pragma unroll 4
  for (int y = ty; y < kTile; y += kTileThreads / kTile) {
    const int r = sr0 + y, c = sc0 + tx;
    float u = 0.f;
    if (r < M.rows && c < M.cols) {
      const long long idx = static_cast<long long>(r) * M.cols + c;
      if (p.src_kind == kFromF32) {
        u = static_cast<const float*>(M.src0)[idx];
      } else {
        const float g = bf16_bits_to_f32(static_cast<const uint16_t*>(M.src0)[idx]);
        if (p.src_kind == kFromMomentum) {
          // recompute u from g and the already updated buffer (same rounding as flat_kernel)
          const float nb = M.src1[idx];
          u = p.nesterov ? __fadd_rn(__fmul_rn(p.omb, g), __fmul_rn(p.beta, nb)) : nb;
        } else {
          u = g;
        }
      }
    }
    tile[y][tx] = u;
  }
  __syncthreads();
  const float den = s_den;
#pragma unroll 4
  for (int y = ty; y < kTile; y += kTileThreads / kTile) {
    const int i = i0 + y, j = j0 + tx;
    if (i < m && j < n) {
      const float u = M.transposed ? tile[tx][y] : tile[y][tx];
      const float x = __fdiv_rn(u, den);
      const long long o = static_cast<long long>(i) * M.ld + j;
      M.xf[o] = x;
      if (M.xb) static_cast<bf16*>(M.xb)[o] = __float2bfloat16_rn(x);
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
  const int tx = threadIdx.x & (kTile - 1), ty = threadIdx.x >> 6;

  // stage O's tile: O[r][c] = o[c*ld + r] when transposed, else o[r*ld + c]
  const int orow0 = M.o_transposed ? c0 : r0;
  const int ocol0 = M.o_transposed ? r0 : c0;
  const int orows = M.o_transposed ? M.cols : M.rows;
  const int ocols = M.o_transposed ? M.rows : M.cols;
#pragma unroll 4
  for (int y = ty; y < kTile; y += kTileThreads / kTile) {
    const int r = orow0 + y, c = ocol0 + tx;
    tile[y][tx] = (r < orows && c < ocols) ? M.o[static_cast<long long>(r) * M.ld + c] : 0.f;
  }
  __syncthreads();
#pragma unroll 4
  for (int y = ty; y < kTile; y += kTileThreads / kTile) {
    const int r = r0 + y, c = c0 + tx;
    if (r < M.rows && c < M.cols) {
      const float o = M.o_transposed ? tile[tx][y] : tile[y][tx];
      const long long idx = static_cast<long long>(r) * M.cols + c;
      if (p.mode == 0) {
        float* W = static_cast<float*>(M.y);
        const float w = W[idx];
        W[idx] = __fsub_rn(__fsub_rn(w, __fmul_rn(p.lw, w)), __fmul_rn(M.ls, o));
      } else if (p.mode == 1) {
        static_cast<bf16*>(M.y)[idx] = __float2bfloat16_rn(o);
      } else {
        static_cast<float*>(M.y)[idx] = o;
      }
    }
  }
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
