// Tensor-core GEMMs of the Newton-Schulz iteration on sm_100a.
//
// One Newton-Schulz step is X <- aX + (bA + cA^2)X with A = X X^T ("The
// NanoGPT speedrun", record #3: five such steps replace the momentum update by
// its nearest semi-orthogonal matrix).  It is three dense contractions, each a
// grouped, persistent launch over every matrix of every shape group:
//
//   kGram  A  = X X^T            tiles touching the upper triangle, mirrored
//   kPoly  B  = b A + c A A      A symmetric, so A A = A A^T: same tiling
//   kBx    X' = a X + B X        fp32 master X updated in place, bf16 copy out
//
// One CTA per SM, persistent over a static tile stride; 128 x 256 output tiles.
//   warp 0      one thread issues bulk tensor copies of the operand tiles
//               (128x64 and 256x64 bf16, 128-byte swizzle) into a ring of
//               STAGES shared-memory stages;
//   warp 1      allocates 512 tensor-memory columns (two 128x256 fp32
//               accumulators); one thread issues tcgen05.mma (M=128, N=256,
//               K=16), commits each stage back to the copier and each finished
//               accumulator to the epilogue;
//   warps 2-5   the epilogue: per 32-column chunk, tcgen05.ld (one row per
//               thread), combine with the chunk's epilogue operand (prefetched
//               by bulk copy into a 4-slot ring), write swizzled staging in
//               shared memory, and hand it to bulk tensor stores -- no
//               row-strided global accesses; the other accumulator fills
//               meanwhile.
// Symmetric outputs: a chunk strictly above the diagonal 128x128 block is
// stored twice (direct, and transposed through a second staging buffer); the
// diagonal block is assembled in shared memory, its lower half overwritten
// from its upper half, and stored once; chunks strictly below it are skipped.
// So A and B are bit-exactly symmetric.
// Every wait is bounded (WaitCtl); on expiry the CTA drains and exits.
#include "common.cuh"
#include "internal.h"

namespace muon {
namespace tc {

constexpr uint32_t kTileBytesP = BM * BK * 2;               // 16 KiB
constexpr uint32_t kTileBytesQ = BN * BK * 2;               // 32 KiB
constexpr uint32_t kStageBytes = kTileBytesP + kTileBytesQ;  // 48 KiB
constexpr uint32_t kTmemCols = 2 * BN;                      // two accumulators
constexpr uint32_t kChunkBf16 = BM * kChunk * 2;            // 8 KiB
constexpr uint32_t kChunkF32 = BM * kChunk * 4;             // 16 KiB

template <int EPI>
struct Cfg {
  static constexpr int kStages = (EPI == kGram) ? 4 : 3;
  // epilogue operand ring
  static constexpr uint32_t kSlotBytes = (EPI == kBx) ? kChunkF32 : (EPI == kPoly ? kChunkBf16 : 0);
  static constexpr uint32_t kSlotsBytes = kSlotBytes * kEpiSlots;
  // staging: kBx two bf16 output chunks; kGram / kPoly 2 direct + 2 mirror chunks,
  // aliased by the 128 x 128 diagonal block (2 x [128 rows][64 cols] bf16)
  static constexpr uint32_t kStagingBytes = (EPI == kBx) ? 2 * kChunkBf16 : 4 * kChunkBf16;
  static constexpr uint32_t kRingBytes = kStages * kStageBytes;
  static constexpr int kNumBars = 2 * kStages + 5 + kEpiSlots;
  static constexpr size_t kSmem =
      1024 + kRingBytes + kSlotsBytes + kStagingBytes + kNumBars * 8 + 16;
};

size_t smem_bytes(int epi) {
  switch (epi) {
    case kGram: return Cfg<kGram>::kSmem;
    case kPoly: return Cfg<kPoly>::kSmem;
    default: return Cfg<kBx>::kSmem;
  }
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
    // row tile tm holds column tiles (tm / 2) .. tiles_n - 1
    int tm = 0;
    while (true) {
      const int len = G.tiles_n - (tm >> 1);
      if (r < len) break;
      r -= len;
      ++tm;
    }
    c.tm = tm;
    c.tn = (tm >> 1) + r;
  }
  return c;
}

// Role of one 32-column epilogue chunk of a symmetric-output tile.
enum ChunkKind : int { kSkip = 0, kUpper = 1, kDiag = 2, kPlain = 3 };

template <int EPI>
__device__ __forceinline__ int chunk_kind(const Group& G, int tm, int col0) {
  if (EPI == kBx) return col0 < G.n ? kPlain : kSkip;
  if (col0 >= G.m) return kSkip;
  const int d0 = tm * BM;
  if (col0 + kChunk <= d0) return kSkip;  // strictly below the diagonal block
  if (col0 >= d0 + BM) return kUpper;     // strictly above it
  return kDiag;
}

// Byte offset of 16-byte unit `u` of row `r` in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128(int r, int u) {
  return static_cast<uint32_t>(r * 128 + ((u ^ (r & 7)) << 4));
}
// Same for a 64-byte-swizzled tile (rows of 64 bytes).
__device__ __forceinline__ uint32_t sw64(int r, int u) {
  return static_cast<uint32_t>(r * 64 + ((u ^ ((r >> 1) & 3)) << 4));
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c,
                                             uint32_t& d) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}
__device__ __forceinline__ uint16_t ld_shared_u16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint16_t bf16_bits(float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&h);
}

// AND of `v` over the 128 epilogue threads (hardware barrier 3).  Every
// possibly-failing wait of the epilogue is followed by this, so the four
// epilogue warps always take the same branch and never strand one another at
// a later barrier.
__device__ __forceinline__ bool epi_all(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 3, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return out != 0;
}

// ---------------------------------------------------------------------- kernel
template <int EPI>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ Params p) {
  using C = Cfg<EPI>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  uint8_t* slots = ring + C::kRingBytes;
  uint8_t* staging = slots + C::kSlotsBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + C::kStagingBytes);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * S + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * S + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * S + 4);
  auto efull_bar = [&](int s) { return bar0 + 8u * (2 * S + 5 + s); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 4 * 32);
    }
    mbar_init(drain_bar, 1);
    for (int s = 0; s < kEpiSlots; ++s) mbar_init(efull_bar(s), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < p.ngroups; ++g) {
      tma_prefetch_map(&p.map[g].p);
      tma_prefetch_map(&p.map[g].q);
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
  const unsigned long long drain_ns = p.timeout_ns < 50000000ull ? p.timeout_ns : 50000000ull;
  const int my_tiles =
      blockIdx.x < p.total_tiles ? (p.total_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ copier
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool inject = (p.inject == 1 && blockIdx.x == 0);
      bool ok = true;
      for (int k = 0; k < my_tiles && ok; ++k) {
        const TileCoord tc = decode_tile<EPI>(p, blockIdx.x + k * gridDim.x);
        const Group& G = p.grp[tc.g];
        const Maps& M = p.map[tc.g];
        const int kblocks = (G.k + BK - 1) / BK;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, ctl)) {
            ok = false;
            break;
          }
          // kBx: 64-column boxes wholly beyond n are not copied (their
          // accumulator columns are never stored)
          int qboxes = BN / 64;
          if (EPI == kBx) {
            const int left = G.n - tc.tn * BN;
            qboxes = left >= BN ? BN / 64 : (left + 63) / 64;
          }
          mbar_arrive_expect_tx(full_bar(stage), kTileBytesP + qboxes * 8192u);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (inject) {
            inject = false;  // withhold this stage's copies: its consumer's wait runs out
          } else {
            const uint32_t dP = smem_u32(ring + stage * kStageBytes);
            const uint32_t dQ = dP + kTileBytesP;
            tma_load_3d(dP, &M.p, full_bar(stage), kb * BK, tc.tm * BM, tc.b);
            if (EPI == kBx) {
              for (int c = 0; c < qboxes; ++c)
                tma_load_3d(dQ + c * 8192, &M.q, full_bar(stage), tc.tn * BN + c * 64, kb * BK, tc.b);
            } else {
              tma_load_3d(dQ, &M.q, full_bar(stage), kb * BK, tc.tn * BN, tc.b);
            }
          }
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        for (int s = 0; s < S; ++s)
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
      for (int k = 0; k < my_tiles && ok; ++k) {
        const TileCoord tc = decode_tile<EPI>(p, blockIdx.x + k * gridDim.x);
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
          const uint32_t aP = smem_u32(ring + stage * kStageBytes);
          const uint32_t aQ = aP + kTileBytesP;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t adesc = sdesc_sw128(aP + kk * 32, 16, 1024);
            const uint64_t bdesc = (EPI == kBx) ? sdesc_sw128(aQ + kk * 2048, 8192, 1024)
                                                : sdesc_sw128(aQ + kk * 32, 16, 1024);
            tc_mma_bf16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));
          if (++stage == S) {
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
      tc_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0, drain_ns > 1000000ull ? drain_ns : 1000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int lane_base = 32 * (warp & 3);
    const int r = lane_base + lane;  // tile row owned by this thread
    const bool leader = (warp == 2 && lane == 0);
    const int total_chunks = my_tiles * kChunks;
    const uint32_t slots_u32 = smem_u32(slots);
    const uint32_t stage_u32 = smem_u32(staging);

    // Epilogue operand prefetch of chunk s into slot s % kEpiSlots (leader only).
    int pend[kEpiSlots] = {-1, -1, -1, -1};  // last chunk issued per slot
    auto issue_eload = [&](int s) {
      if (EPI == kGram || s >= total_chunks) return;
      const int slot = s % kEpiSlots;
      pend[slot] = s;
      const TileCoord tc = decode_tile<EPI>(p, blockIdx.x + (s / kChunks) * gridDim.x);
      const Group& G = p.grp[tc.g];
      const int col0 = tc.tn * BN + (s % kChunks) * kChunk;
      const int kind = chunk_kind<EPI>(G, tc.tm, col0);
      if (kind == kSkip) {
        mbar_arrive(efull_bar(slot));
      } else {
        mbar_arrive_expect_tx(efull_bar(slot), C::kSlotBytes);
        tma_load_3d(slots_u32 + slot * C::kSlotBytes, &p.map[tc.g].e, efull_bar(slot), col0,
                    tc.tm * BM, tc.b);
      }
    };
    if (leader) {
      for (int g = 0; g < p.ngroups; ++g) {
        tma_prefetch_map(&p.map[g].e);
        tma_prefetch_map(&p.map[g].d);
        tma_prefetch_map(&p.map[g].mt);
        tma_prefetch_map(&p.map[g].s);
      }
      for (int s = 0; s < kEpiSlots; ++s) issue_eload(s);
    }

    int acc = 0;
    uint32_t acc_phase = 0;
    int prev_kind = kSkip;
    bool ok = true;
    for (int k = 0; k < my_tiles && ok; ++k) {
      const TileCoord tc = decode_tile<EPI>(p, blockIdx.x + k * gridDim.x);
      const Group& G = p.grp[tc.g];
      const Maps& M = p.map[tc.g];
      const int row0 = tc.tm * BM;
      const bool w = epi_all(mbar_wait(tfull_bar(acc), acc_phase, ctl));
      if (!w) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int c = 0; c < kChunks; ++c) {
        const int s = k * kChunks + c;
        const int col0 = tc.tn * BN + c * kChunk;
        const int kind = chunk_kind<EPI>(G, tc.tm, col0);
        float v[32];
        if (kind != kSkip) {
          uint32_t rr[32];
          __syncwarp();
          tmem_ld_32x32(tmem_base + (static_cast<uint32_t>(lane_base) << 16) +
                            static_cast<uint32_t>(acc * BN + c * kChunk),
                        rr);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 32; ++q) v[q] = __uint_as_float(rr[q]);
        }
        if (c == kChunks - 1) {
          // accumulator fully read: hand it back to the MMA warp
          tc_fence_before();
          mbar_arrive(tempty_bar(acc));
        }
        if (kind == kSkip) {
          // nothing loaded for this chunk; its slot goes to chunk s + kEpiSlots
          if (leader) issue_eload(s + kEpiSlots);
          continue;
        }
        const int slot = s % kEpiSlots;
        if (EPI != kGram) {
          const bool e = epi_all(mbar_wait(efull_bar(slot), (s / kEpiSlots) & 1, ctl));
          if (!e) {
            ok = false;
            break;
          }
        }
        if (EPI == kBx) {
          // X' = a X + acc, in place in the slot; bf16 copy to staging[s % 2]
          const uint32_t es = slots_u32 + slot * C::kSlotBytes;
          const uint32_t os = stage_u32 + (s & 1) * kChunkBf16;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            uint32_t x0, x1, x2, x3;
            const uint32_t addr = es + sw128(r, u);
            ld_shared_v4(addr, x0, x1, x2, x3);
            const float y0 = fmaf(p.a, __uint_as_float(x0), v[4 * u + 0]);
            const float y1 = fmaf(p.a, __uint_as_float(x1), v[4 * u + 1]);
            const float y2 = fmaf(p.a, __uint_as_float(x2), v[4 * u + 2]);
            const float y3 = fmaf(p.a, __uint_as_float(x3), v[4 * u + 3]);
            st_shared_v4(addr, __float_as_uint(y0), __float_as_uint(y1), __float_as_uint(y2),
                         __float_as_uint(y3));
            v[4 * u + 0] = y0;
            v[4 * u + 1] = y1;
            v[4 * u + 2] = y2;
            v[4 * u + 3] = y3;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u)
            st_shared_v4(os + sw64(r, u), pack_bf16x2(v[8 * u + 0], v[8 * u + 1]),
                         pack_bf16x2(v[8 * u + 2], v[8 * u + 3]), pack_bf16x2(v[8 * u + 4], v[8 * u + 5]),
                         pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
          fence_async_smem();
          named_bar(1, 128);
          if (leader) {
            tma_store_3d(&M.e, es, col0, row0, tc.b);
            tma_store_3d(&M.d, os, col0, row0, tc.b);
            bulk_commit();
            bulk_wait_read_all();
            issue_eload(s + kEpiSlots);
          }
          prev_kind = kind;
          continue;
        }

        if (EPI == kPoly) {
          // B = b A + c acc with A's chunk from the slot (bf16, 64-byte swizzle)
          const uint32_t es = slots_u32 + slot * C::kSlotBytes;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t a4[4];
            ld_shared_v4(es + sw64(r, u), a4[0], a4[1], a4[2], a4[3]);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float lo = bf16_bits_to_f32(static_cast<uint16_t>(a4[h] & 0xFFFFu));
              const float hi = bf16_bits_to_f32(static_cast<uint16_t>(a4[h] >> 16));
              v[8 * u + 2 * h] = fmaf(p.c, v[8 * u + 2 * h], p.b * lo);
              v[8 * u + 2 * h + 1] = fmaf(p.c, v[8 * u + 2 * h + 1], p.b * hi);
            }
          }
        }

        if (kind == kUpper) {
          if (prev_kind == kDiag) named_bar(2, 128);  // staging is aliased by the diagonal block
          const uint32_t ds = stage_u32 + (s & 1) * kChunkBf16;      // direct [128][32]
          const uint32_t ms = stage_u32 + (2 + (s & 1)) * kChunkBf16;  // mirror [32][128]
#pragma unroll
          for (int u = 0; u < 4; ++u)
            st_shared_v4(ds + sw64(r, u), pack_bf16x2(v[8 * u + 0], v[8 * u + 1]),
                         pack_bf16x2(v[8 * u + 2], v[8 * u + 3]), pack_bf16x2(v[8 * u + 4], v[8 * u + 5]),
                         pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
#pragma unroll
          for (int q = 0; q < 32; ++q) st_shared_u16(ms + q * 256 + r * 2, bf16_bits(v[q]));
          fence_async_smem();
          named_bar(1, 128);
          if (leader) {
            tma_store_3d(&M.d, ds, col0, row0, tc.b);
            tma_store_3d(&M.mt, ms, row0, col0, tc.b);
            bulk_commit();
            bulk_wait_read_all();
            if (EPI == kPoly) issue_eload(s + kEpiSlots);
          }
        } else {  // kDiag: chunk dq of the 128 x 128 diagonal block
          const int dq = (col0 - row0) / kChunk;
          if (dq == 0) named_bar(2, 128);  // previous stores done reading the staging
          const uint32_t sb = stage_u32 + (dq >> 1) * (2 * kChunkBf16);  // [128][64] half
#pragma unroll
          for (int u = 0; u < 4; ++u)
            st_shared_v4(sb + sw128(r, (dq & 1) * 4 + u), pack_bf16x2(v[8 * u + 0], v[8 * u + 1]),
                         pack_bf16x2(v[8 * u + 2], v[8 * u + 3]), pack_bf16x2(v[8 * u + 4], v[8 * u + 5]),
                         pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
          if (EPI == kPoly) {
            named_bar(1, 128);  // every thread has read its slot
            if (leader) issue_eload(s + kEpiSlots);
          }
          if (dq == 3 || col0 + kChunk >= G.m) {
            // block complete: lower half := transpose of the upper half
            named_bar(1, 128);
            for (int j = 0; j < r; ++j) {
              const uint32_t src = stage_u32 + (r >> 6) * (2 * kChunkBf16) +
                                   static_cast<uint32_t>(j * 128 + ((((r & 63) >> 3) ^ (j & 7)) << 4) + (r & 7) * 2);
              const uint32_t dst = stage_u32 + (j >> 6) * (2 * kChunkBf16) +
                                   static_cast<uint32_t>(r * 128 + ((((j & 63) >> 3) ^ (r & 7)) << 4) + (j & 7) * 2);
              st_shared_u16(dst, ld_shared_u16(src));
            }
            fence_async_smem();
            named_bar(1, 128);
            if (leader) {
              tma_store_3d(&M.s, stage_u32, row0, row0, tc.b);
              if (row0 + 64 < G.m)  // never start a store wholly outside the matrix
                tma_store_3d(&M.s, stage_u32 + 2 * kChunkBf16, row0 + 64, row0, tc.b);
              bulk_commit();
              bulk_wait_read_all();
            }
          }
        }
        prev_kind = kind;
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (leader) {
      bulk_wait_all();
      if (!ok) {
        // prefetched epilogue operands still in flight land before exit
        for (int s = 0; s < kEpiSlots; ++s)
          if (pend[s] >= 0) mbar_wait_drain(efull_bar(s), (pend[s] / kEpiSlots) & 1, drain_ns);
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
  const size_t smem = Cfg<EPI>::kSmem;
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
