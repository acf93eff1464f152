// fp32 SIMT GEMMs of the Newton-Schulz iteration (verification mode).
//
// True fp32 fused multiply-adds on the CUDA cores (no TF32): the fp32 mode of
// muon_ns_orthogonalize exists to check the iteration itself to ~1e-4, which
// a 10-bit-mantissa tensor-core path could not.  Throughput is not a goal.
//
//   kGram  D = P P^T              (P = X; full product, symmetric by construction)
//   kPoly  D = b E + c P P^T      (P = E = A symmetric, so P P^T = A A)
//   kBx    D = a E + P Q          (P = B, Q = E = X; D is the other ping-pong X)
//
// 64x64 output tile per 256-thread block, 4x4 outputs per thread, K in slices
// of 16 staged through shared memory; batch index in blockIdx.z.  Each output
// accumulates its K terms in increasing k, so reruns are bit-identical.
#include "common.cuh"
#include "internal.h"

namespace muon {
namespace simt {

constexpr int T = 64, KS = 16;

template <int MODE>
__global__ void __launch_bounds__(256) simt_kernel(const __grid_constant__ Params p) {
  __shared__ float Ps[KS][T + 4];
  __shared__ float Qs[KS][T + 4];
  const int b = blockIdx.z;
  const int i0 = blockIdx.y * T, j0 = blockIdx.x * T;
  const float* P = p.P + static_cast<long long>(b) * p.sp;
  const float* Q = p.Q + static_cast<long long>(b) * p.sq;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};

  for (int k0 = 0; k0 < p.k; k0 += KS) {
    // P tile: rows i0..i0+63, k0..k0+15  -> Ps[k][row]
    for (int e = threadIdx.x; e < T * KS; e += 256) {
      const int kk = e & (KS - 1), r = e >> 4;
      const int gi = i0 + r, gk = k0 + kk;
      Ps[kk][r] = (gi < p.m && gk < p.k) ? P[static_cast<long long>(gi) * p.ldp + gk] : 0.f;
    }
    // Q tile: Qs[k][col] = Q(k, j): row-contiguous in k for gram/poly, in j for bx
    for (int e = threadIdx.x; e < T * KS; e += 256) {
      int kk, c;
      if (MODE == kBx) { c = e & (T - 1); kk = e >> 6; }
      else { kk = e & (KS - 1); c = e >> 4; }
      const int gj = j0 + c, gk = k0 + kk;
      float v = 0.f;
      if (gj < p.n && gk < p.k)
        v = (MODE == kBx) ? Q[static_cast<long long>(gk) * p.ldq + gj]
                          : Q[static_cast<long long>(gj) * p.ldq + gk];
      Qs[kk][c] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      float a[4], bq[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = Ps[kk][ty * 4 + r];
#pragma unroll
      for (int c = 0; c < 4; ++c) bq[c] = Qs[kk][tx * 4 + c];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(a[r], bq[c], acc[r][c]);
    }
    __syncthreads();
  }

  float* D = p.D + static_cast<long long>(b) * p.sd;
  const float* E = p.E ? p.E + static_cast<long long>(b) * p.se : nullptr;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = i0 + ty * 4 + r;
    if (i >= p.m) continue;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = j0 + tx * 4 + c;
      if (j >= p.n) continue;
      float v = acc[r][c];
      if (MODE == kPoly) v = fmaf(p.c, v, p.b * E[static_cast<long long>(i) * p.lde + j]);
      if (MODE == kBx) v = fmaf(p.a, E[static_cast<long long>(i) * p.lde + j], v);
      D[static_cast<long long>(i) * p.ldd + j] = v;
    }
  }
}

cudaError_t launch(int mode, const Params& p, cudaStream_t stream) {
  if (p.batch <= 0) return cudaSuccess;
  dim3 grid((p.n + T - 1) / T, (p.m + T - 1) / T, p.batch);
  switch (mode) {
    case kGram: simt_kernel<kGram><<<grid, 256, 0, stream>>>(p); break;
    case kPoly: simt_kernel<kPoly><<<grid, 256, 0, stream>>>(p); break;
    case kBx: simt_kernel<kBx><<<grid, 256, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace simt
}  // namespace muon
