// Tensor-core GEMMs of the Newton-Schulz iteration on sm_100a.
//
// One Newton-Schulz step is X <- aX + (bA + cA^2)X with A = X X^T ("The
// NanoGPT speedrun", record #3: five such steps replace the momentum update by
// its nearest semi-orthogonal matrix).  It is three dense contractions, each a
// grouped, persistent launch over every matrix of every shape group:
//
//   kGram  A  = X X^T            upper 128x128 tiles only, mirrored on store
//   kPoly  B  = b A + c A A      A symmetric, so A A = A A^T: again upper tiles
//   kBx    X' = a X + B X        fp32 master X in the epilogue, bf16 copy out
//
// Structure of one CTA (one per SM, persistent over a static tile stride):
//   warp 0      one thread issues bulk tensor copies of 128x64 bf16 operand
//               tiles (128-byte swizzle) into a 6-stage shared-memory ring;
//   warp 1      allocates 256 tensor-memory columns (two 128x128 fp32
//               accumulators) and one thread issues tcgen05.mma (M=128, N=128,
//               K=16) per 16-wide K slice, committing each stage back to the
//               copier and each finished accumulator to the epilogue;
//   warps 2-5   read the accumulator with tcgen05.ld (one row per thread),
//               apply the step's epilogue and store to global memory, while
//               the MMA warp fills the other accumulator.
// Every wait is bounded (WaitCtl); on expiry the CTA drains and exits.
#include "common.cuh"
#include "internal.h"

namespace muon {
namespace tc {

constexpr uint32_t kTileBytesP = BM * BK * 2;  // 16 KiB
constexpr uint32_t kTileBytesQ = BN * BK * 2;  // 16 KiB
constexpr uint32_t kTmemCols = 2 * BN;         // two accumulators
constexpr int kNumBars = 2 * kStages + 5;      // full, empty, tfull x2, tempty x2, drain

size_t smem_bytes() {
  return 1024 /* alignment slack */ + kStages * (kTileBytesP + kTileBytesQ) + kNumBars * 8 + 16;
}

struct TileCoord {
  int g, b, tm, tn;
};

template <int EPI>
__device__ __forceinline__ TileCoord decode_tile(const Params& p, int t) {
  TileCoord c;
  int g = 0;
  while (g + 1 < p.ngroups && t >= p.grp[g + 1].tile_begin) ++g;
  const Group& G = p.grp[g];
  const int local = t - G.tile_begin;
  c.g = g;
  c.b = local / G.tiles_per_mat;
  int r = local - c.b * G.tiles_per_mat;
  if (EPI == kBx) {
    // column panel outer, row panel inner: neighbouring CTAs share X's panel
    c.tn = r / G.tiles_m;
    c.tm = r - c.tn * G.tiles_m;
  } else {
    // upper triangle, row by row: row tm holds tiles tm..tiles_m-1
    int tm = 0, len = G.tiles_m;
    while (r >= len) {
      r -= len;
      ++tm;
      --len;
    }
    c.tm = tm;
    c.tn = tm + r;
  }
  return c;
}

// ------------------------------------------------------------------ epilogues
// Symmetric output (kGram / kPoly): D[i][j] for the tile's upper part and the
// mirror D[j][i]; on a diagonal tile only j >= i is taken, so every element of
// D is written exactly once per side and D is bit-exactly symmetric.
template <int EPI>
__device__ __forceinline__ void store_symmetric(const Params& p, const Group& G, int b, int tm,
                                                int tn, int row, int col0, float (&v)[32]) {
  const int m = G.m;
  const int i = tm * BM + row;
  if (i >= m) return;
  const long long base = static_cast<long long>(b) * G.mat_stride;
  bf16* D = static_cast<bf16*>(G.d) + base;
  const bool diag = (tm == tn);
  const bool full = (col0 + 32 <= m);

  if (EPI == kPoly) {
    const bf16* A = static_cast<const bf16*>(G.e) + base + static_cast<long long>(i) * G.ld + col0;
    if (full) {
      const uint4* a4 = reinterpret_cast<const uint4*>(A);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 w = a4[q];
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float lo = bf16_bits_to_f32(static_cast<uint16_t>(ws[h] & 0xFFFFu));
          const float hi = bf16_bits_to_f32(static_cast<uint16_t>(ws[h] >> 16));
          v[q * 8 + 2 * h] = fmaf(p.c, v[q * 8 + 2 * h], p.b * lo);
          v[q * 8 + 2 * h + 1] = fmaf(p.c, v[q * 8 + 2 * h + 1], p.b * hi);
        }
      }
    } else {
      const uint16_t* a16 = reinterpret_cast<const uint16_t*>(A);
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const float av = (col0 + q < m) ? bf16_bits_to_f32(a16[q]) : 0.f;
        v[q] = fmaf(p.c, v[q], p.b * av);
      }
    }
  }

  // direct store of row i
  bf16* drow = D + static_cast<long long>(i) * G.ld + col0;
  if (full && !diag) {
    uint4* d4 = reinterpret_cast<uint4*>(drow);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 w;
      w.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
      w.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
      w.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
      w.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
      d4[q] = w;
    }
  } else {
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      const int j = col0 + q;
      if (j < m && (!diag || j >= i)) drow[q] = __float2bfloat16_rn(v[q]);
    }
  }
  // mirrored store: D[j][i]; consecutive lanes hold consecutive i (coalesced)
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const int j = col0 + q;
    if (j < m && (!diag || j > i))
      D[static_cast<long long>(j) * G.ld + i] = __float2bfloat16_rn(v[q]);
  }
}

// X' = a X + acc; fp32 master X updated in place, bf16 operand copy written to
// the other ping-pong buffer.
__device__ __forceinline__ void store_bx(const Params& p, const Group& G, int b, int tm, int row,
                                         int col0, float (&v)[32]) {
  const int i = tm * BM + row;
  if (i >= G.m) return;
  const long long off = static_cast<long long>(b) * G.mat_stride + static_cast<long long>(i) * G.ld + col0;
  float* xf = G.xf + off;
  bf16* xo = static_cast<bf16*>(G.d) + off;
  if (col0 + 32 <= G.n) {
    float4* x4 = reinterpret_cast<float4*>(xf);
    uint4* o4 = reinterpret_cast<uint4*>(xo);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float4 x = x4[q];
      x.x = fmaf(p.a, x.x, v[4 * q + 0]);
      x.y = fmaf(p.a, x.y, v[4 * q + 1]);
      x.z = fmaf(p.a, x.z, v[4 * q + 2]);
      x.w = fmaf(p.a, x.w, v[4 * q + 3]);
      x4[q] = x;
      v[4 * q + 0] = x.x;
      v[4 * q + 1] = x.y;
      v[4 * q + 2] = x.z;
      v[4 * q + 3] = x.w;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 w;
      w.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
      w.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
      w.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
      w.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
      o4[q] = w;
    }
  } else {
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      if (col0 + q < G.n) {
        const float x = fmaf(p.a, xf[q], v[q]);
        xf[q] = x;
        xo[q] = __float2bfloat16_rn(x);
      }
    }
  }
}

// ---------------------------------------------------------------------- kernel
template <int EPI>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sP = smem;
  uint8_t* sQ = smem + kStages * kTileBytesP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sQ + kStages * kTileBytesQ);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * kStages + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * kStages + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * kStages + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 4 * 32);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < p.ngroups; ++g) {
      tma_prefetch_map(&p.map_p[g]);
      tma_prefetch_map(&p.map_q[g]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  WaitCtl ctl;
  ctl.abort_flag = abort_flag;
  ctl.status = p.status;
  ctl.timeout_ns = p.timeout_ns;
  ctl.where = 0;
  const unsigned long long drain_ns =
      p.timeout_ns < 50000000ull ? p.timeout_ns : 50000000ull;

  if (warp == 0) {
    // ------------------------------------------------------------ copier
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool inject = (p.inject == 1 && blockIdx.x == 0);
      bool ok = true;
      for (int t = blockIdx.x; t < p.total_tiles && ok; t += gridDim.x) {
        const TileCoord tc = decode_tile<EPI>(p, t);
        const Group& G = p.grp[tc.g];
        const int kblocks = (G.k + BK - 1) / BK;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, ctl)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(stage), kTileBytesP + kTileBytesQ);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (inject) {
            inject = false;  // withhold this stage's copies: its consumer's wait runs out
          } else {
            const uint32_t dP = smem_u32(sP + stage * kTileBytesP);
            const uint32_t dQ = smem_u32(sQ + stage * kTileBytesQ);
            tma_load_3d(dP, &p.map_p[tc.g], full_bar(stage), kb * BK, tc.tm * BM, tc.b);
            if (EPI == kBx) {
              tma_load_3d(dQ, &p.map_q[tc.g], full_bar(stage), tc.tn * BN, kb * BK, tc.b);
              tma_load_3d(dQ + 8192, &p.map_q[tc.g], full_bar(stage), tc.tn * BN + 64, kb * BK,
                          tc.b);
            } else {
              tma_load_3d(dQ, &p.map_q[tc.g], full_bar(stage), kb * BK, tc.tn * BN, tc.b);
            }
          }
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // abort: let the copies already issued land before the CTA exits
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s)) mbar_wait_drain(full_bar(s), (issued_parity >> s) & 1u, drain_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(BN, EPI == kBx);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.total_tiles && ok; t += gridDim.x) {
        const TileCoord tc = decode_tile<EPI>(p, t);
        const int kblocks = (p.grp[tc.g].k + BK - 1) / BK;
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, ctl)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t aP = smem_u32(sP + stage * kTileBytesP);
          const uint32_t aQ = smem_u32(sQ + stage * kTileBytesQ);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t adesc = sdesc_sw128(aP + kk * 32, 16, 1024);
            const uint64_t bdesc = (EPI == kBx) ? sdesc_sw128(aQ + kk * 2048, 8192, 1024)
                                                : sdesc_sw128(aQ + kk * 32, 16, 1024);
            tc_mma_bf16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // every MMA issued by this thread has completed once drain_bar flips
      tc_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0, drain_ns > 1000000ull ? drain_ns : 1000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int lane_base = 32 * (warp & 3);
    const int row = lane_base + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x) {
      const TileCoord tc = decode_tile<EPI>(p, t);
      const Group& G = p.grp[tc.g];
      bool ok = mbar_wait(tfull_bar(acc), acc_phase, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld_32x32(tmem_base + (static_cast<uint32_t>(lane_base) << 16) +
                          static_cast<uint32_t>(acc * BN + ch * 32),
                      r);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = __uint_as_float(r[q]);
        const int col0 = tc.tn * BN + ch * 32;
        if (EPI == kBx)
          store_bx(p, G, tc.b, tc.tm, row, col0, v);
        else
          store_symmetric<EPI>(p, G, tc.b, tc.tm, tc.tn, row, col0, v);
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int EPI>
static cudaError_t launch_one(const Params& p, int grid, cudaStream_t stream) {
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = smem_bytes();
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  gemm_kernel<EPI><<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch(int epi, const Params& p, int grid, cudaStream_t stream) {
  if (p.total_tiles <= 0) return cudaSuccess;
  switch (epi) {
    case kGram: return launch_one<kGram>(p, grid, stream);
    case kPoly: return launch_one<kPoly>(p, grid, stream);
    case kBx: return launch_one<kBx>(p, grid, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tc
}  // namespace muon
