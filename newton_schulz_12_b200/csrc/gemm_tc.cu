// Tensor-core GEMMs of the Newton-Schulz iteration on sm_100a.
//
// One Newton-Schulz step is X <- aX + (bA + cA^2)X with A = X X^T ("The
// NanoGPT speedrun", record #3: five such steps replace the momentum update by
// its nearest semi-orthogonal matrix).  It is three dense contractions, each a
// grouped, persistent launch over every matrix of every shape group:
//
//   kGram  A  = X X^T            tiles on or above the diagonal, mirrored
//   kPoly  B  = b A + c A A      A symmetric, so A A = A A^T: same tiling
//   kBx    X' = a X + B X        X carried as the pair bf16 hi + int8 residual
//   kBxApply  the last step's kBx: X_T goes straight into the caller's
//          weights, W' = (W - lw W) - ls X_T, W read and written by bulk
//          tensor copies next to X's epilogue chunk (the update is never
//          stored as X_T and read back by a separate pass)
//
// CTAs run in clusters of two on an SM pair, one cluster per pair tile of
// 256 x 256 outputs at a time, persistent over a static tile stride.  One
// tcgen05.mma (cta_group::2, M = 256, N = 256, K = 16), issued by the leader
// CTA, reads 128 rows of the row operand and 128 of the 256 column-operand
// rows from EACH CTA's shared memory and writes each CTA's 128 x 256 half of
// the tile into that CTA's tensor memory: per CTA a 64-deep K stage is 32 KiB
// (16 KiB of its own rows + its half of the shared columns) instead of 48 KiB,
// so more stages fit and fewer bytes cross from L2 per MMA.
// Roles, in both CTAs:
//   warp 0      one thread issues bulk tensor copies of this CTA's operand
//               tiles (128x64 bf16, 128-byte swizzle) into a ring of stages;
//               the bytes of both CTAs complete on the leader's barrier;
//   warp 1      allocates 512 tensor-memory columns (two 128x256 fp32
//               accumulators) for the pair; in the leader one thread issues
//               the pair MMAs and commits each stage back to both copiers and
//               each finished accumulator to both epilogues;
//   warps 2-9   the epilogue: per 64-column chunk, tcgen05.ld (one row per
//               thread, two warps per lane quarter), combine with the chunk's
//               epilogue operand (prefetched by bulk copy into a ring of
//               slots), write swizzled staging in shared memory -- no
//               row-strided global accesses; the other accumulator fills
//               meanwhile;
//   warp 10     one thread issues the epilogue's bulk stores;
//   warp 11     (kPoly, kBx) one thread issues the epilogue operand copies.
// Symmetric outputs: a chunk strictly above the diagonal 128x128 block is
// stored twice (direct, and transposed through a second staging buffer); the
// diagonal block is assembled in shared memory, its lower half overwritten
// from its upper half, and stored once; chunks strictly below it are skipped.
// So A and B are bit-exactly symmetric.
// Every wait is bounded (WaitCtl); on expiry both CTAs of the pair drain and exit.
#include "common.cuh"
#include "internal.h"

namespace muon {
namespace tc {

constexpr uint32_t kTileBytesP = BM * BK * 2;               // 16 KiB: this CTA's rows
constexpr uint32_t kTileBytesQ = BNH * BK * 2;              // 16 KiB: its half of the columns
constexpr uint32_t kStageBytes = kTileBytesP + kTileBytesQ;  // 32 KiB
constexpr uint32_t kTmemCols = 2 * BN;                      // two accumulators
constexpr uint32_t kChunkBf16 = BM * kChunk * 2;            // 8 KiB
constexpr size_t kMaxSmem = 232448;                         // 227 KiB per CTA on sm_100

// Shared memory per CTA is split between the operand ring (K stages) and the
// epilogue (operand slots, output staging); the split is a compile-time
// choice per kernel.
// Defaults for 64-column symmetric chunks (their staging pairs are 32 KiB);
// with 32-column chunks the staging halves and one more stage fits.
#ifndef MUON_GRAM_STAGES
#define MUON_GRAM_STAGES (MUON_SYM_CHUNK == 64 ? 5 : 6)
#endif
#ifndef MUON_POLY_STAGES
#define MUON_POLY_STAGES (MUON_SYM_CHUNK == 64 ? 4 : 5)
#endif
#ifndef MUON_POLY_SLOTS
#define MUON_POLY_SLOTS (MUON_SYM_CHUNK == 64 ? 2 : 4)
#endif
#ifndef MUON_GRAM_SBUF
#define MUON_GRAM_SBUF 2
#endif
#ifndef MUON_POLY_SBUF
#define MUON_POLY_SBUF 2
#endif
#ifndef MUON_BX_STAGES
#define MUON_BX_STAGES 4
#endif
#ifndef MUON_BX_SLOTS
#define MUON_BX_SLOTS 4
#endif
// kBxApply slots also hold the chunk's W (fp32): with 32-column chunks a slot
// is 28 KiB and 4 fit next to 3 stages, so 3 chunks can be in flight
#ifndef MUON_BXA_CHUNK
#define MUON_BXA_CHUNK 32
#endif
#ifndef MUON_BXA_STAGES
#define MUON_BXA_STAGES 3
#endif
#ifndef MUON_BXA_SLOTS
#define MUON_BXA_SLOTS (MUON_BXA_CHUNK == 32 ? 4 : 2)
#endif
static_assert(MUON_BXA_CHUNK == 32 || MUON_BXA_CHUNK == 64, "kBxApply chunk width");

// kBx and kBxApply share the operands, the tiling and X's epilogue chunks.
template <int EPI>
__host__ __device__ constexpr bool is_bx() {
  return EPI == kBx || EPI == kBxApply;
}

template <int EPI>
struct Cfg {
  static constexpr int kStages =
      (EPI == kGram) ? MUON_GRAM_STAGES
                     : (EPI == kPoly ? MUON_POLY_STAGES : (EPI == kBx ? MUON_BX_STAGES : MUON_BXA_STAGES));
  // epilogue operand ring of kSlots chunks (kGram: none, the count only sizes barriers)
  // kBx slot: the hi and lo bf16 chunks of X (8 KiB each); kPoly slot: A's chunk
  static constexpr int kSlots =
      (EPI == kBx) ? MUON_BX_SLOTS : (EPI == kBxApply ? MUON_BXA_SLOTS : MUON_POLY_SLOTS);
  // kBx works on 64-column chunks (128-byte rows in global memory), the
  // symmetric kernels on kSymChunk-column chunks
  static constexpr int kCW = (EPI == kBx) ? 2 * kChunk : (EPI == kBxApply ? MUON_BXA_CHUNK : kSymChunk);
  static constexpr int kNCh = BN / kCW;  // per tile
  // bytes of one bf16 chunk, 128 rows x kCW columns
  static constexpr uint32_t kChunkBytes = BM * kCW * 2;
  // kBx / kBxApply slot: hi (bf16, 128 rows x 2 kCW bytes) then lo (int8,
  // 128 rows x kCW bytes); kBxApply: then W's 128 x kCW fp32 chunk; kPoly
  // slot: A's chunk
  static constexpr uint32_t kXBytes = BM * kCW * 3;  // the pair of X's chunk
  static constexpr uint32_t kLoOff = BM * kCW * 2;
  static constexpr uint32_t kWOff = kXBytes;
  static constexpr uint32_t kWBytes = BM * kCW * 4;
  static constexpr uint32_t kSlotBytes = (EPI == kBx)        ? kXBytes
                                         : (EPI == kBxApply) ? kXBytes + kWBytes
                                         : (EPI == kPoly)    ? kChunkBytes
                                                             : 0;
  static constexpr uint32_t kSlotsBytes = kSlotBytes * kSlots;
  // kGram / kPoly output staging: kSBuf pairs of a direct [128][kCW] and a
  // mirrored [kCW][128] chunk, laid out as d0 .. d(kSBuf-1), m0 .. m(kSBuf-1).
  // A diagonal 128 x 128 block (two [128][64] halves, 128-byte swizzle)
  // aliases d0 d1 and m0 m1 (32-column chunks) or d0 and d1 (64-column).
  static constexpr int kSBuf = (EPI == kGram) ? MUON_GRAM_SBUF : (EPI == kPoly ? MUON_POLY_SBUF : 2);
  static_assert(kSBuf >= 2, "the diagonal block takes staging pairs 0 and 1");
  static constexpr uint32_t kStagingBytes = is_bx<EPI>() ? 0 : 2 * kSBuf * kChunkBytes;
  // ready barriers: kBx one per slot; kGram / kPoly one per staging pair + the block
  static constexpr int kReady = is_bx<EPI>() ? kSlots : kSBuf + 1;
  static constexpr uint32_t kRingBytes = kStages * kStageBytes;
  // full, empty, tfull x2, tempty x2, drain, efull, ready, sfree, econs
  static constexpr int kNumBars = 2 * kStages + 5 + 2 * kSlots + kReady + kSBuf;
  static constexpr size_t kSmem =
      1024 + kRingBytes + kSlotsBytes + kStagingBytes + kNumBars * 8 + 16;
};

static_assert(Cfg<kGram>::kSmem <= kMaxSmem, "kGram shared memory");
static_assert(Cfg<kPoly>::kSmem <= kMaxSmem, "kPoly shared memory");
static_assert(Cfg<kBx>::kSmem <= kMaxSmem, "kBx shared memory");
static_assert(Cfg<kBxApply>::kSmem <= kMaxSmem, "kBxApply shared memory");
static_assert(Cfg<kBxApply>::kWOff % 1024 == 0 && Cfg<kBxApply>::kSlotBytes % 1024 == 0,
              "W chunks start on the 1 KiB boundary of the 128-byte swizzle");

int bx_apply_chunk() { return Cfg<kBxApply>::kCW; }

size_t smem_bytes(int epi) {
  switch (epi) {
    case kGram: return Cfg<kGram>::kSmem;
    case kPoly: return Cfg<kPoly>::kSmem;
    case kBxApply: return Cfg<kBxApply>::kSmem;
    default: return Cfg<kBx>::kSmem;
  }
}

struct TileCoord {
  int g, b, tm, tn;
};

// Pair tile t of the launch, seen from CTA `rank` of the pair: tm is the
// CTA's own 128-row tile, tn the pair's 256-column tile.
template <int EPI>
__device__ __forceinline__ TileCoord decode_tile(const Params& p, int t, int rank) {
  TileCoord c;
  if (p.reverse) t = p.total_tiles - 1 - t;
  int g = 0;
  while (g + 1 < p.ngroups && t >= p.grp[g + 1].tile_begin) ++g;
  const Group& G = p.grp[g];
  const int local = t - G.tile_begin;
  c.g = g;
  c.b = local / G.tiles_per_mat;
  int r = local - c.b * G.tiles_per_mat;
  int tm2;
  if (is_bx<EPI>()) {
    // column panel outer, row panel inner: neighbouring pairs share X's panel
    c.tn = r / G.tiles_m;
    tm2 = r - c.tn * G.tiles_m;
  } else {
    // pair row tm2 holds column tiles tm2 .. tiles_n - 1
    tm2 = 0;
    while (r >= G.tiles_n - tm2) {
      r -= G.tiles_n - tm2;
      ++tm2;
    }
    c.tn = tm2 + r;
  }
  c.tm = 2 * tm2 + rank;
  return c;
}

// Role of one epilogue chunk (kCW columns) of an output tile.
enum ChunkKind : int { kSkip = 0, kUpper = 1, kDiag = 2, kPlain = 3 };

template <int EPI>
__device__ __forceinline__ int chunk_kind(const Group& G, int tm, int col0) {
  constexpr int W = is_bx<EPI>() ? 2 * kChunk : kSymChunk;
  // a CTA whose rows lie wholly below the matrix stores nothing
  if (is_bx<EPI>()) return (col0 < G.n && tm * BM < G.m) ? kPlain : kSkip;
  if (col0 >= G.m) return kSkip;
  const int d0 = tm * BM;
  if (col0 + W <= d0) return kSkip;  // strictly below the diagonal block
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

// Same for a 32-byte-swizzled tile (rows of 32 bytes).
__device__ __forceinline__ uint32_t sw32(int r, int u) {
  return static_cast<uint32_t>(r * 32 + ((u ^ ((r >> 2) & 1)) << 4));
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

// Bytes of one K stage over BOTH CTAs of the pair (armed on the leader's barrier).
template <int EPI>
__device__ __forceinline__ uint32_t pair_stage_bytes(const Group& G, int tn) {
  if (!is_bx<EPI>()) return 2 * kStageBytes;  // out-of-range rows are zero-filled, still counted
  // kBx: 64-column boxes of X wholly beyond n are not copied
  const int left = G.n - tn * BN;
  const int boxes = left >= BN ? BN / 64 : (left + 63) / 64;
  return 2 * kTileBytesP + static_cast<uint32_t>(boxes) * 8192u;
}

// Table entry of matrix b of group G in a kBxApply launch, or -1 (mode 0).
template <int N>
__device__ __forceinline__ int apply_entry(const ApplyTable<N>& t, const Group& G, int b) {
  const int j = G.mat_base + b - t.mat_base;
  return (j >= 0 && j < t.nmat && t.mat[j].mode != 0) ? j : -1;
}

// Bytes of W's chunk (CW columns of X) at (row0, col0) that the loader
// copies: mode 1, CW / 32 boxes of 32 x 128; mode 2, four boxes of 32 x CW.
// Boxes wholly outside W are neither copied nor stored.
template <int CW>
__device__ __forceinline__ uint32_t w_chunk_bytes(int mode, const Group& G, int row0, int col0) {
  uint32_t q = 0;
  if (mode == 1) {
    for (int h = 0; h < CW / 32; ++h) q += (col0 + 32 * h < G.n) ? 1u : 0u;
    return q * (BM * 32 * 4);
  }
  for (int i = 0; i < 4; ++i) q += (row0 + 32 * i < G.m) ? 1u : 0u;
  return q * (32 * CW * 4);
}

// W' = (W - d) - ls O with d = fl(lw W) -- or d = 0 under cautious decay where
// W and O do not have the same sign -- each operation rounded to nearest in fp32.
__device__ __forceinline__ float apply_w(float w, float o, float lw, float ls, int cautious) {
  const bool decay = !cautious || (w > 0.f && o > 0.f) || (w < 0.f && o < 0.f);
  const float d = decay ? __fmul_rn(lw, w) : 0.0f;
  return __fsub_rn(__fsub_rn(w, d), __fmul_rn(ls, o));
}

#ifdef MUON_TRACE
__device__ __forceinline__ void trace_stamp(const Params& p, int tile, int slot) {
  if (p.trace && blockIdx.x < kTraceCtas && tile < kTraceTiles)
    p.trace[(blockIdx.x * kTraceTiles + tile) * kTraceSlots + slot] = global_ns();
}
#define TRACE(tile, slot) trace_stamp(p, tile, slot)
#else
#define TRACE(tile, slot) \
  do {                    \
  } while (0)
#endif

// ---------------------------------------------------------------------- kernel
// Epilogue math warps per kernel kind: 8 (two per TMEM lane quarter), and 16
// for the fused apply, whose epilogue (W's stream) bounds it.  Measured on
// the GPT-2-small set: 16 warps slow kBx by 11 % (its epilogue is off the
// critical path, and more warps contend with the copy and MMA threads) and
// speed kBxApply up by 12 %.
#ifndef MUON_EPI_WARPS
#define MUON_EPI_WARPS 8
#endif
#ifndef MUON_BXA_EPI_WARPS
#define MUON_BXA_EPI_WARPS 16
#endif
template <int EPI>
__host__ __device__ constexpr int epi_warps() {
  return EPI == kBxApply ? MUON_BXA_EPI_WARPS : MUON_EPI_WARPS;
}
template <int EPI>
__host__ __device__ constexpr int epi_threads() {
  return 32 * epi_warps<EPI>();
}
// The IO warp follows the epilogue warps; kPoly and kBx add a loader warp after it.
template <int EPI>
__host__ __device__ constexpr int io_warp() {
  return 2 + epi_warps<EPI>();
}
template <int EPI>
__host__ __device__ constexpr int threads_of() {
  static_assert(epi_warps<EPI>() == 8 || epi_warps<EPI>() == 16, "epilogue warps: 8 or 16");
  return 32 * (io_warp<EPI>() + 1) + (EPI == kGram ? 0 : 32);
}

// NT: entries of the per-matrix table (1 where the launch has none).
template <int EPI, int NT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(threads_of<EPI>(), 1)
    gemm_kernel(const __grid_constant__ Params p, const __grid_constant__ ApplyTable<NT> tab) {
  using C = Cfg<EPI>;
  constexpr int kEpiThreads = epi_threads<EPI>();
  constexpr int kIoWarp = io_warp<EPI>();
  constexpr int S = C::kStages;
  constexpr int K = C::kSlots;
  extern __shared__ uint8_t smem_raw[];
  // identical layout in both CTAs: the pair MMA addresses the partner's
  // operands at this CTA's offsets
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
  const int rank = static_cast<int>(cluster_ctarank());  // 0 = leader
  const uint32_t peer = static_cast<uint32_t>(rank ^ 1);
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * S + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * S + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * S + 4);
  auto efull_bar = [&](int s) { return bar0 + 8u * (2 * S + 5 + s); };
  constexpr int NB = C::kSBuf;
  auto ready_bar = [&](int s) { return bar0 + 8u * (2 * S + 5 + K + s); };
  auto sfree_bar = [&](int b) { return bar0 + 8u * (2 * S + 5 + K + C::kReady + b); };
  // staging addresses (kGram / kPoly): direct and mirror chunk of pair b, and
  // the two [128][64] halves of a diagonal block
  auto econs_bar = [&](int s) { return bar0 + 8u * (2 * S + 5 + K + C::kReady + NB + s); };
  auto stg_direct = [&](uint32_t base, int b) { return base + static_cast<uint32_t>(b) * C::kChunkBytes; };
  auto stg_mirror = [&](uint32_t base, int b) {
    return base + static_cast<uint32_t>(NB + b) * C::kChunkBytes;
  };
  auto stg_half = [&](uint32_t base, int h) {
    return C::kCW == 64 ? stg_direct(base, h) : base + static_cast<uint32_t>(h ? NB : 0) * kChunkBf16;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);   // leader's: its arrive + both CTAs' bytes
      mbar_init(empty_bar(s), 1);  // one commit from the leader's MMA thread
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      // one arrival per epilogue warp; the leader's also takes the partner's relayed one
      mbar_init(tempty_bar(a), kEpiThreads / 32 + (rank == 0 ? 1 : 0));
    }
    mbar_init(drain_bar, 1);
    for (int s = 0; s < K; ++s) {
      mbar_init(efull_bar(s), 1);
      // kPoly: every compute thread has read the slot; kBx: the slot's stores
      // have read it (one arrival from the store thread)
      mbar_init(econs_bar(s), is_bx<EPI>() ? 1 : kEpiThreads);
    }
    for (int s = 0; s < C::kReady; ++s) mbar_init(ready_bar(s), kEpiThreads);
    for (int b = 0; b < NB; ++b) mbar_init(sfree_bar(b), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < p.ngroups; ++g) {
      tma_prefetch_map(&p.map[g].p);
      tma_prefetch_map(&p.map[g].q);
    }
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before either touches the other's
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  WaitCtl ctl;
  ctl.abort_flag = abort_flag;
  ctl.status = p.status;
  ctl.timeout_ns = p.timeout_ns;
  ctl.where = 0;
  ctl.peer_abort = cluster_addr(smem_u32(const_cast<int*>(abort_flag)), peer);
  const unsigned long long drain_ns = p.timeout_ns < 50000000ull ? p.timeout_ns : 50000000ull;
  const int my_tiles = pair < p.total_tiles ? (p.total_tiles - 1 - pair) / npairs + 1 : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ copier (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool inject = (p.inject == 1 && blockIdx.x == 0);
      bool ok = true;
      for (int k = 0; k < my_tiles && ok; ++k) {
        const TileCoord tc = decode_tile<EPI>(p, pair + k * npairs, rank);
        const Group& G = p.grp[tc.g];
        const Maps& M = p.map[tc.g];
        const int kblocks = (G.k + BK - 1) / BK;
        const uint32_t bytes = pair_stage_bytes<EPI>(G, tc.tn);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, ctl)) {
            ok = false;
            break;
          }
          if (kb == 0) TRACE(k, 0);
          if (kb == kblocks - 1) TRACE(k, 1);
          const uint32_t fbar = cluster_addr(full_bar(stage), 0);  // the leader's barrier
          if (rank == 0) {
            mbar_arrive_expect_tx(full_bar(stage), bytes);
            issued_mask |= 1u << stage;
            issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          }
          if (inject) {
            inject = false;  // withhold this stage's copies: its consumer's wait runs out
          } else {
            const uint32_t dP = smem_u32(ring + stage * kStageBytes);
            const uint32_t dQ = dP + kTileBytesP;
            const int qcol = tc.tn * BN + rank * BNH;  // this CTA's half of the columns
            tma_load_3d_pair(dP, &M.p, fbar, kb * BK, tc.tm * BM, tc.b);
            if (is_bx<EPI>()) {
              for (int c = 0; c < BNH / 64; ++c)
                if (qcol + c * 64 < G.n)
                  tma_load_3d_pair(dQ + c * 8192, &M.q, fbar, qcol + c * 64, kb * BK, tc.b);
            } else {
              tma_load_3d_pair(dQ, &M.q, fbar, kb * BK, qcol, tc.b);
            }
          }
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // the leader's barriers count both CTAs' copies: once they complete,
        // nothing is still landing in either CTA's ring
        for (int s = 0; s < S; ++s)
          if (issued_mask & (1u << s)) mbar_wait_drain(full_bar(s), (issued_parity >> s) & 1u, drain_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16(PM, BN, is_bx<EPI>());
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int k = 0; k < my_tiles && ok; ++k) {
        const TileCoord tc = decode_tile<EPI>(p, pair + k * npairs, rank);
        const int kblocks = (p.grp[tc.g].k + BK - 1) / BK;
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, ctl)) break;
        tc_fence_after();
        TRACE(k, 2);
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
            const uint64_t bdesc = is_bx<EPI>() ? sdesc_sw128(aQ + kk * 2048, 8192, 1024)
                                                : sdesc_sw128(aQ + kk * 32, 16, 1024);
            tc_mma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          // stage consumed in both CTAs
          tc_commit_pair(empty_bar(stage));
          tc_commit_pair(cluster_addr(empty_bar(stage), peer));
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        TRACE(k, 3);
        tc_commit_pair(tfull_bar(acc));
        tc_commit_pair(cluster_addr(tfull_bar(acc), peer));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      tc_commit_pair(drain_bar);
      mbar_wait_drain(drain_bar, 0, drain_ns > 1000000ull ? drain_ns : 1000000ull);
    } else if (lane == 0) {
      // partner CTA: relay "accumulator drained" to the leader's MMA thread,
      // one remote arrival per tile instead of one per epilogue warp
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int k = 0; k < my_tiles; ++k) {
        if (!mbar_wait(tempty_bar(acc), acc_phase, ctl)) break;
        mbar_arrive_remote(cluster_addr(tempty_bar(acc), 0));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue warps and IO (warp kIoWarp)
    constexpr int NCH = C::kNCh, CW = C::kCW;
    const int total_chunks = my_tiles * NCH;
    const uint32_t slots_u32 = smem_u32(slots);
    const uint32_t stage_u32 = smem_u32(staging);

    if (warp >= kIoWarp) {
      // ---------------------------------------------------------- IO threads
      // Warp kIoWarp issues the epilogue's bulk stores of what the compute warps
      // finished, draining each store before the buffer it read is handed
      // back.  The operand chunk copies into the slot ring come from the next warp,
      // so that a copy issue stalled on the tensor-copy unit never delays a
      // store: kPoly refills a slot once the compute warps have read it, kBx
      // (whose results are stored from the slot itself) once its stores have.
      constexpr bool kLoaderWarp = (EPI != kGram);
      const bool loads_here = (EPI != kGram) && (kLoaderWarp ? warp == kIoWarp + 1 : warp == kIoWarp);
      if (lane == 0) {
        for (int g = 0; g < p.ngroups; ++g) {
          tma_prefetch_map(&p.map[g].e);
          tma_prefetch_map(&p.map[g].d);
          tma_prefetch_map(&p.map[g].mt);
          tma_prefetch_map(&p.map[g].s);
        }
        int pend[K];
        for (int q = 0; q < K; ++q) pend[q] = -1;
        auto issue_eload = [&](int s) {
          if (EPI == kGram || s >= total_chunks) return;
          const int slot = s % K;
          pend[slot] = s;
          const TileCoord tc = decode_tile<EPI>(p, pair + (s / NCH) * npairs, rank);
          const int col0 = tc.tn * BN + (s % NCH) * CW;
          const int row0 = tc.tm * BM;
          const Group& G = p.grp[tc.g];
          const bool skip = is_bx<EPI>() ? !(col0 < G.n && row0 < G.m)
                                         : chunk_kind<EPI>(G, tc.tm, col0) == kSkip;
          if (skip) {
            mbar_arrive(efull_bar(slot));
          } else {
            const uint32_t dst = slots_u32 + slot * C::kSlotBytes;
            const int j = (EPI == kBxApply) ? apply_entry(tab, G, tc.b) : -1;
            const int mode = j >= 0 ? tab.mat[j].mode : 0;
            const uint32_t bytes = is_bx<EPI>() ? C::kXBytes : C::kSlotBytes;
            mbar_arrive_expect_tx(efull_bar(slot), bytes + (mode ? w_chunk_bytes<CW>(mode, G, row0, col0) : 0u));
            tma_load_3d(dst, &p.map[tc.g].e, efull_bar(slot), col0, row0, tc.b);
            if (is_bx<EPI>())  // lo half of X next to its hi half
              tma_load_3d(dst + C::kLoOff, &p.map[tc.g].mt, efull_bar(slot), col0, row0, tc.b);
            if (mode == 1) {  // W as X: CW / 32 boxes of 32 columns x 128 rows
              for (int h = 0; h < CW / 32; ++h)
                if (col0 + 32 * h < G.n)
                  tma_load_3d(dst + C::kWOff + h * (BM * 32 * 4), &tab.w[j], efull_bar(slot), col0 + 32 * h,
                              row0, 0);
            } else if (mode == 2) {  // W = X^T: four boxes of 32 columns x CW rows
              for (int q = 0; q < 4; ++q)
                if (row0 + 32 * q < G.m)
                  tma_load_3d(dst + C::kWOff + q * (32 * CW * 4), &tab.w[j], efull_bar(slot), row0 + 32 * q,
                              col0, 0);
            }
          }
        };
        if (loads_here)
          for (int s = 0; s < K; ++s) issue_eload(s);
        if (kLoaderWarp && warp == kIoWarp + 1) {
          if (EPI == kPoly) {
            // refill each slot as soon as every compute thread has read it
            for (int s = 0; s < total_chunks; ++s) {
              mbar_wait(econs_bar(s % K), (s / K) & 1, ctl);
              if (s % NCH == NCH - 3) TRACE(s / NCH, 17);
              issue_eload(s + K);
            }
          } else {
            // kBx: chunk s + K goes into chunk s's slot as soon as chunk s's own
            // stores have read it (the store thread waits for that right after
            // issuing them), so the loader runs K chunks ahead
            for (int s = 0; s + K < total_chunks; ++s) {
              mbar_wait(econs_bar(s % K), (s / K) & 1, ctl);
              issue_eload(s + K);
            }
          }
        }
        const int io_chunks = (kLoaderWarp && warp == kIoWarp + 1) ? 0 : total_chunks;
        int njob[NB + 1];  // kGram / kPoly: jobs seen per ready barrier (staging pairs, then the block)
        for (int q = 0; q <= NB; ++q) njob[q] = 0;
        int nup = 0;       // strictly-upper chunks so far (staging pair = nup % NB)
        int hq[NB];        // FIFO of staging pairs whose stores may still be reading them
        int hq_head = 0, hq_n = 0;
        for (int s = 0; s < io_chunks; ++s) {
          const int k = s / NCH, c = s % NCH;
          const TileCoord tc = decode_tile<EPI>(p, pair + k * npairs, rank);
          const Group& G = p.grp[tc.g];
          const Maps& M = p.map[tc.g];
          const int row0 = tc.tm * BM;
          const int col0 = tc.tn * BN + c * CW;
          const int kind = chunk_kind<EPI>(G, tc.tm, col0);
          if (is_bx<EPI>()) {
            const int slot = s % K;
            mbar_wait(ready_bar(slot), (s / K) & 1, ctl);
            if (kind != kSkip) {  // never start a store wholly outside the matrix
              const uint32_t hs = slots_u32 + slot * C::kSlotBytes;
              const int j = (NT > 1) ? apply_entry(tab, G, tc.b) : -1;
              const int mode = j >= 0 ? tab.mat[j].mode : 0;
              if (EPI == kBxApply && mode == 1) {
                for (int h = 0; h < CW / 32; ++h)
                  if (col0 + 32 * h < G.n) tma_store_3d(&tab.w[j], hs + C::kWOff + h * (BM * 32 * 4), col0 + 32 * h, row0, 0);
              } else if (EPI == kBxApply && mode == 2) {
                for (int q = 0; q < 4; ++q)
                  if (row0 + 32 * q < G.m) tma_store_3d(&tab.w[j], hs + C::kWOff + q * (32 * CW * 4), row0 + 32 * q, col0, 0);
              } else if (EPI == kBx && mode == 3) {
                tma_store_3d(&tab.w[j], hs, col0, row0, 0);  // hi' -> the caller's bf16 buffer; no residual
              } else {
                tma_store_3d(&M.d, hs, col0, row0, tc.b);               // hi' -> the other hi buffer
                tma_store_3d(&M.mt, hs + C::kLoOff, col0, row0, tc.b);  // lo' -> lo, in place
              }
              bulk_commit();
              asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");  // chunk s drained
            } else {
              bulk_wait_read_all();
            }
            mbar_arrive(econs_bar(s % K));  // the loader may refill chunk s's slot
            continue;
          }
          if (kind == kUpper) {
            const int b = nup % NB;
            ++nup;
            mbar_wait(ready_bar(b), njob[b] & 1, ctl);
            ++njob[b];
            if (c == NCH - 3) TRACE(k, 18);
            tma_store_3d(&M.d, stg_direct(stage_u32, b), col0, row0, tc.b);
            tma_store_3d(&M.mt, stg_mirror(stage_u32, b), row0, col0, tc.b);
            bulk_commit();
            hq[(hq_head + hq_n) % NB] = b;
            ++hq_n;
            // up to NB chunks' stores in flight: once all pairs are taken,
            // release the oldest as soon as its stores have read it (the
            // compute warps need it for the next chunk)
            if (hq_n == NB) {
              asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(NB - 1) : "memory");
              mbar_arrive(sfree_bar(hq[hq_head]));
              hq_head = (hq_head + 1) % NB;
              --hq_n;
            }
            if (c == NCH - 3) TRACE(k, 19);
            continue;
          }
          if (kind == kDiag && col0 == row0 && hq_n > 0) {
            // a diagonal block starts: it takes staging pairs 0 and 1
            bulk_wait_read_all();
            for (; hq_n > 0; --hq_n, hq_head = (hq_head + 1) % NB) mbar_arrive(sfree_bar(hq[hq_head]));
          }
          if (kind == kDiag && ((col0 - row0) / CW == BM / CW - 1 || col0 + CW >= G.m)) {
            mbar_wait(ready_bar(NB), njob[NB] & 1, ctl);
            ++njob[NB];
            tma_store_3d(&M.s, stg_half(stage_u32, 0), row0, row0, tc.b);
            if (row0 + 64 < G.m)  // never start a store wholly outside the matrix
              tma_store_3d(&M.s, stg_half(stage_u32, 1), row0 + 64, row0, tc.b);
            bulk_commit();
            bulk_wait_read_all();
            mbar_arrive(sfree_bar(0));  // the block used staging pairs 0 and 1
            mbar_arrive(sfree_bar(1));
          }
        }
        bulk_wait_all();
        for (; hq_n > 0; --hq_n, hq_head = (hq_head + 1) % NB) mbar_arrive(sfree_bar(hq[hq_head]));
        if (loads_here)
          for (int q = 0; q < K; ++q)  // operand copies still in flight land before exit
            if (pend[q] >= 0) mbar_wait_drain(efull_bar(q), (pend[q] / K) & 1, drain_ns);
      }
      __syncwarp();
    } else {
      // ---------------------------------------------------------- compute warps
      // NP = epi_warps / 4 warps per TMEM lane quarter: warp w reads lanes
      // 32*(w%4).. and the part `hf` (of NP) of each chunk's columns.  A failed
      // (timed-out) wait is recorded and the schedule continues -- every later
      // wait then returns at once -- so the compute warps always meet at the
      // same barriers.
      constexpr int NP = epi_warps<EPI>() / 4;
      const int lane_base = 32 * (warp & 3);
      const int hf = (warp - 2) >> 2;
      const int r = lane_base + lane;  // tile row owned by this thread
      const bool leader = (warp == 2 && lane == 0);
      int acc = 0;
      uint32_t acc_phase = 0;
      int nuse[NB];  // kGram / kPoly: jobs that used staging pair b so far
      for (int q = 0; q < NB; ++q) nuse[q] = 0;

      int nup = 0;
      for (int k = 0; k < my_tiles; ++k) {
        const TileCoord tc = decode_tile<EPI>(p, pair + k * npairs, rank);
        const Group& G = p.grp[tc.g];
        const int row0 = tc.tm * BM;
        // X = s (hi + lo) on the first step: A = s^2 acc, X' = s (a (hi + lo) + acc)
        float xs = 1.0f;
        if (EPI != kPoly && p.xscale) {
          xs = p.xscale[G.mat_base + tc.b];
          if (EPI == kGram) xs = xs * xs;
        }
        mbar_wait(tfull_bar(acc), acc_phase, ctl);
        tc_fence_after();
        if (leader) TRACE(k, 4);
        if (is_bx<EPI>()) {
          const int j = (EPI == kBxApply) ? apply_entry(tab, G, tc.b) : -1;
          const int mode = j >= 0 ? tab.mat[j].mode : 0;
          const float lsc = j >= 0 ? tab.mat[j].ls : 0.f;  // fl(lr * scale)
          // BCW-column chunks c (64 for kBx, MUON_BXA_CHUNK for kBxApply): thread
          // (r, hf) takes accumulator columns VB hf .. +VB-1 of the chunk
          constexpr int BCW = C::kCW, VB = BCW / NP;
          const int sr = r;
          for (int c = 0; c < C::kNCh; ++c) {
            if (leader && c > 0) TRACE(k, 4 + c);
            const int s = k * C::kNCh + c;
            const int col0 = tc.tn * BN + c * C::kCW;
            const bool live = chunk_kind<EPI>(G, tc.tm, col0) != kSkip;
            float v[VB];
            if (live) {
              uint32_t rr[VB];
              __syncwarp();
              const uint32_t ta = tmem_base + (static_cast<uint32_t>(lane_base) << 16) +
                                  static_cast<uint32_t>(acc * BN + c * C::kCW + hf * VB);
              if constexpr (VB == 32)
                tmem_ld_32x32(ta, rr);
              else if constexpr (VB == 16)
                tmem_ld_32x32_x16(ta, rr);
              else
                tmem_ld_32x32_x8(ta, rr);
              tmem_ld_wait();
#pragma unroll
              for (int q = 0; q < VB; ++q) v[q] = __uint_as_float(rr[q]);
            }
            if (c == C::kNCh - 1) {
              // accumulator fully read: one arrival per warp hands it back (in
              // the partner CTA through the relay thread of warp 1)
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(tempty_bar(acc));
            }
            const int slot = s % K;
            mbar_wait(efull_bar(slot), (s / K) & 1, ctl);
            // X = hi + lo from the slot; X' = a X + acc (times s on the first
            // step) written back in place as the pair (hi', lo') for the IO
            // thread to store.  Columns VB hf + 8 uu .. +7 are 16-byte unit
            // (VB / 8) hf + uu of the hi row (2 BCW bytes, swizzled over its
            // width) and the 8 bytes at offset VB hf + 8 uu of the lo row
            // (BCW bytes, likewise: unit (VB hf + 8 uu) / 16, half by bit 3).
            if (live) {
              const uint32_t hs = slots_u32 + slot * C::kSlotBytes;
              const uint32_t ls = hs + C::kLoOff;
#pragma unroll
              for (int uu = 0; uu < VB / 8; ++uu) {
                const int hu = (VB / 8) * hf + uu;  // 16-byte unit of the hi row
                const int lb = VB * hf + 8 * uu;    // byte offset in the lo row
                const uint32_t ha = hs + (BCW == 64 ? sw128(sr, hu) : sw64(sr, hu));
                const uint32_t la = ls + (BCW == 64 ? sw64(sr, lb >> 4) : sw32(sr, lb >> 4)) + (lb & 8);
                uint4 h4;
                uint2 l2;
                ld_shared_v4(ha, h4.x, h4.y, h4.z, h4.w);
                asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(l2.x), "=r"(l2.y) : "r"(la) : "memory");
                float x[8];
                pair_axpy8(h4, l2, v + 8 * uu, p.a, xs, x);  // two values per fp32 instruction
                if (EPI == kBxApply && mode == 1) {
                  // W's row sr, columns VB hf + 8 uu ..: box (VB hf) / 32 (32
                  // fp32 per 128-byte row, 128-byte swizzle), 16-byte units
                  // ((VB hf) % 32) / 4 + 2 uu and the next
                  const uint32_t wb = hs + C::kWOff + ((VB * hf) / 32) * (BM * 32 * 4);
                  const int u0 = ((VB * hf) % 32) / 4 + 2 * uu;
#pragma unroll
                  for (int h = 0; h < 2; ++h) {
                    const uint32_t wa = wb + sw128(sr, u0 + h);
                    uint32_t w[4];
                    ld_shared_v4(wa, w[0], w[1], w[2], w[3]);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                      w[e] = __float_as_uint(apply_w(__uint_as_float(w[e]), x[4 * h + e], tab.lw, lsc, tab.cautious));
                    st_shared_v4(wa, w[0], w[1], w[2], w[3]);
                  }
                } else if (EPI == kBxApply && mode == 2) {
                  // W = X^T: X's column VB hf + 8 uu + e is row VB hf + 8 uu + e
                  // of box (warp & 3) (BCW rows of 128 bytes), whose 32 columns
                  // are this lane quarter's rows
                  const uint32_t wb = hs + C::kWOff + (warp & 3) * (32 * BCW * 4);
#pragma unroll
                  for (int e = 0; e < 8; ++e) {
                    const int row = VB * hf + 8 * uu + e;
                    const uint32_t wa =
                        wb + static_cast<uint32_t>(row * 128 + ((((lane >> 2) ^ row) & 7) << 4) + (lane & 3) * 4);
                    float w;
                    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(w) : "r"(wa) : "memory");
                    w = apply_w(w, x[e], tab.lw, lsc, tab.cautious);
                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(wa), "f"(w) : "memory");
                  }
                } else {
                  pair_encode8_x2(x, h4, l2);
                  st_shared_v4(ha, h4.x, h4.y, h4.z, h4.w);
                  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(la), "r"(l2.x), "r"(l2.y) : "memory");
                }
              }
              fence_async_smem();
            }
            mbar_arrive(ready_bar(slot));
          }
        } else {
        // kCW-column chunks: thread (r, hf) takes accumulator columns
        // VPT hf .. VPT hf + VPT-1 of the chunk, i.e. 16-byte units
        // UPT hf .. UPT hf + UPT-1 of the chunk's swizzled row (64-byte
        // swizzle for 32-column chunks, 128-byte for 64-column ones)
        constexpr int SCW = C::kCW, VPT = SCW / NP, UPT = VPT / 8;
        auto swz = [](int row, int u) { return SCW == 64 ? sw128(row, u) : sw64(row, u); };
        for (int c = 0; c < C::kNCh; ++c) {
          if (leader && c > 0) TRACE(k, 4 + c);
          const int s = k * C::kNCh + c;
          const int col0 = tc.tn * BN + c * SCW;
          const int kind = chunk_kind<EPI>(G, tc.tm, col0);
          float v[VPT];
          if (kind != kSkip) {
            uint32_t rr[VPT];
            __syncwarp();
            const uint32_t ta = tmem_base + (static_cast<uint32_t>(lane_base) << 16) +
                                static_cast<uint32_t>(acc * BN + c * SCW + hf * VPT);
            if constexpr (VPT == 32)
              tmem_ld_32x32(ta, rr);
            else if constexpr (VPT == 16)
              tmem_ld_32x32_x16(ta, rr);
            else
              tmem_ld_32x32_x8(ta, rr);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < VPT; ++q) v[q] = __uint_as_float(rr[q]);
          }
          if (leader && c == C::kNCh - 3) TRACE(k, 13);
          if (c == C::kNCh - 1) {
            // accumulator fully read: one arrival per warp hands it back (in
            // the partner CTA through the relay thread of warp 1)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar(acc));
          }
          const int slot = s % K;
          if (EPI == kPoly) mbar_wait(efull_bar(slot), (s / K) & 1, ctl);
          if (leader && c == C::kNCh - 3) TRACE(k, 14);

          // ------------------------------------------------ kGram / kPoly
          if (EPI == kGram && kind != kSkip) {
#pragma unroll
            for (int q = 0; q < VPT; ++q) v[q] *= xs;
          }
          if (EPI == kPoly) {
            if (kind != kSkip) {
              // B = b A + c acc with A's chunk from the slot (bf16, swizzled like the staging)
              const uint32_t es = slots_u32 + slot * C::kSlotBytes;
#pragma unroll
              for (int uu = 0; uu < UPT; ++uu) {
                uint32_t a4[4];
                ld_shared_v4(es + swz(r, UPT * hf + uu), a4[0], a4[1], a4[2], a4[3]);
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                  const float lo = bf16_bits_to_f32(static_cast<uint16_t>(a4[h] & 0xFFFFu));
                  const float hi = bf16_bits_to_f32(static_cast<uint16_t>(a4[h] >> 16));
                  v[8 * uu + 2 * h] = fmaf(p.c, v[8 * uu + 2 * h], p.b * lo);
                  v[8 * uu + 2 * h + 1] = fmaf(p.c, v[8 * uu + 2 * h + 1], p.b * hi);
                }
              }
            }
            mbar_arrive(econs_bar(slot));  // slot read (or unused): the loader may refill it
          }
          if (kind == kUpper) {
            const int b = nup % NB;
            ++nup;
            if (nuse[b] > 0) mbar_wait(sfree_bar(b), (nuse[b] - 1) & 1, ctl);
            ++nuse[b];
            if (leader && c == C::kNCh - 3) TRACE(k, 15);
            const uint32_t ds = stg_direct(stage_u32, b);  // direct [128][SCW]
            const uint32_t ms = stg_mirror(stage_u32, b);  // mirror [SCW][128]
            uint32_t pk[VPT / 2];  // each value rounded to bf16 once, for both copies
#pragma unroll
            for (int q = 0; q < VPT / 2; ++q) pk[q] = pack_bf16x2(v[2 * q], v[2 * q + 1]);
#pragma unroll
            for (int uu = 0; uu < UPT; ++uu)
              st_shared_v4(ds + swz(r, UPT * hf + uu), pk[4 * uu], pk[4 * uu + 1], pk[4 * uu + 2], pk[4 * uu + 3]);
#pragma unroll
            for (int q = 0; q < VPT; ++q)
              st_shared_u16(ms + (VPT * hf + q) * 256 + r * 2, static_cast<uint16_t>(pk[q >> 1] >> (16 * (q & 1))));
            fence_async_smem();
            mbar_arrive(ready_bar(b));
            if (leader && c == C::kNCh - 3) TRACE(k, 16);
          } else if (kind == kDiag) {  // chunk dq of the 128 x 128 diagonal block
            const int dq = (col0 - row0) / SCW;
            if (dq == 0) {
              // the block occupies staging pairs 0 and 1: wait for their last stores
              for (int b = 0; b < 2; ++b) {
                if (nuse[b] > 0) mbar_wait(sfree_bar(b), (nuse[b] - 1) & 1, ctl);
                ++nuse[b];
              }
            }
            // columns dq SCW .. of the block: half (dq SCW) / 64, first unit ((dq SCW) % 64) / 8
            const uint32_t sb = stg_half(stage_u32, (dq * SCW) >> 6);  // [128][64] half
            const int u0 = ((dq * SCW) & 63) >> 3;
#pragma unroll
            for (int uu = 0; uu < UPT; ++uu)
              st_shared_v4(sb + sw128(r, u0 + UPT * hf + uu), pack_bf16x2(v[8 * uu + 0], v[8 * uu + 1]),
                           pack_bf16x2(v[8 * uu + 2], v[8 * uu + 3]), pack_bf16x2(v[8 * uu + 4], v[8 * uu + 5]),
                           pack_bf16x2(v[8 * uu + 6], v[8 * uu + 7]));
            if (dq == BM / SCW - 1 || col0 + SCW >= G.m) {
              // block complete: lower half := transpose of the upper half.
              // Row r takes S[r][j] = S[j][r] for j < r, eight columns per
              // 16-byte write; the NP warps of a lane quarter split the groups.
              named_bar(1, kEpiThreads);
              auto s_addr = [&](int row, int col) {
                return stg_half(stage_u32, col >> 6) +
                       static_cast<uint32_t>(row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2);
              };
              for (int j0 = 8 * hf; j0 < r; j0 += 8 * NP) {
                uint32_t t[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const uint32_t lo = (j0 + 2 * q < r) ? ld_shared_u16(s_addr(j0 + 2 * q, r)) : 0u;
                  const uint32_t hi = (j0 + 2 * q + 1 < r) ? ld_shared_u16(s_addr(j0 + 2 * q + 1, r)) : 0u;
                  t[q] = lo | (hi << 16);
                }
                if (j0 + 8 <= r) {
                  st_shared_v4(s_addr(r, j0), t[0], t[1], t[2], t[3]);
                } else {
#pragma unroll
                  for (int q = 0; q < 8; ++q)
                    if (j0 + q < r) st_shared_u16(s_addr(r, j0 + q), static_cast<uint16_t>(t[q >> 1] >> (16 * (q & 1))));
                }
              }
              fence_async_smem();
              mbar_arrive(ready_bar(NB));
            }
          }
        }
        }
        if (leader) TRACE(k, 12);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
    }
  }

  // Every role above ends after bounded waits; the pair meets here so that no
  // MMA, copy or remote arrival still targets a CTA that frees its memory.
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

template <int EPI, int NT>
static cudaError_t launch_one(const Params& p, const ApplyTable<NT>& tab, int max_pairs, cudaStream_t stream) {
  static thread_local int configured_device = -1;
  static thread_local int resident_pairs = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = Cfg<EPI>::kSmem;
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<EPI, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    // clusters of two that fit at once: the persistent grid never waits for a second wave
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * max_pairs, 1, 1);
    cfg.blockDim = dim3(threads_of<EPI>(), 1, 1);
    cfg.dynamicSmemBytes = smem;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, gemm_kernel<EPI, NT>, &cfg);
    if (e != cudaSuccess) return e;
    resident_pairs = n;
    configured_device = dev;
  }
  int pairs = p.total_tiles < max_pairs ? p.total_tiles : max_pairs;
  if (resident_pairs > 0 && pairs > resident_pairs) pairs = resident_pairs;
  gemm_kernel<EPI, NT><<<2 * pairs, threads_of<EPI>(), smem, stream>>>(p, tab);
  return cudaGetLastError();
}

cudaError_t launch(int epi, const Params& p, int max_pairs, cudaStream_t stream, const LaunchApply* apply) {
  if (p.total_tiles <= 0) return cudaSuccess;
  if (max_pairs < 1) max_pairs = 1;
  const ApplyTable<1> none{};
  switch (epi) {
    case kGram: return launch_one<kGram, 1>(p, none, max_pairs, stream);
    case kPoly: return launch_one<kPoly, 1>(p, none, max_pairs, stream);
    case kBx:  // with a table: the hi of its mode-3 matrices goes to the caller's buffers
      return apply ? launch_one<kBx, kMaxApply>(p, *apply, max_pairs, stream)
                   : launch_one<kBx, 1>(p, none, max_pairs, stream);
    case kBxApply:
      if (!apply) return cudaErrorInvalidValue;
      return launch_one<kBxApply, kMaxApply>(p, *apply, max_pairs, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tc
}  // namespace muon
