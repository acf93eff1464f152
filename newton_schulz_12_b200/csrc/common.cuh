// Shared device helpers of the sm_100a Muon kernels: status codes, bounded
// waits, mbarrier / bulk-tensor copy / tcgen05 wrappers written as inline PTX.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace muon {

// Device status word values (mirror muon_status in include/muon.h).
constexpr int kStatusOk = 0;
constexpr int kStatusTimeout = -5;

typedef __nv_bfloat16 bf16;

// ---------------------------------------------------------------------------
// Bounded waiting.  Every spin in these kernels ends after `timeout_ns` of
// %globaltimer; the waiter then records kStatusTimeout and raises the CTA's
// abort flag so the other roles leave their loops too.
// ---------------------------------------------------------------------------
struct WaitCtl {
  volatile int* abort_flag;  // shared memory, one per CTA
  int* status;               // global status word
  unsigned long long timeout_ns;
  int where;                 // tag recorded with the failure (which wait)
  uint32_t peer_abort;       // shared::cluster address of the partner CTA's flag, or 0
};

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with parity `parity` of `bar` has completed, for at
// most ctl.timeout_ns.  Returns false (and raises the abort flag, recording
// the status once) when the limit is reached or another role already aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const WaitCtl& ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*ctl.abort_flag) return false;
    if (global_ns() - t0 > ctl.timeout_ns) {
      *ctl.abort_flag = 1;
      if (ctl.peer_abort)  // the partner CTA of a pair leaves its loops too
        asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(ctl.peer_abort), "r"(1) : "memory");
      atomicCAS(ctl.status, kStatusOk, kStatusTimeout);
      return false;
    }
  }
}

// Short bounded wait used only while tearing down after an abort.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity,
                                                unsigned long long limit_ns) {
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// ---------------------------------------------------------------------------
// Clusters of two CTAs (an SM pair sharing one tcgen05 MMA)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %cluster_ctarank;" : "=r"(r));
  return r;
}
// Address in the shared::cluster window of the same offset in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
// All threads of both CTAs; orders prior shared-memory writes (barrier
// initialisation included) before the partner's later accesses.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// Arrive once on an mbarrier given by its shared::cluster address (any CTA of the cluster).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cbar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cbar) : "memory");
}

// ---------------------------------------------------------------------------
// Bulk tensor copies (global -> shared), completing on an mbarrier.
// The innermost coordinate is always a multiple of 64 bf16 elements here.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_map(const void* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* map, uint32_t bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Pair form: the box lands in this CTA's shared memory, and the byte count is
// credited to the mbarrier at shared::cluster address `cbar` (the pair
// leader's), so one barrier tracks the operands of both CTAs.
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const void* map, uint32_t cbar,
                                                 int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(cbar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Shared -> global bulk tensor store (tracked by bulk groups, not mbarriers).
__device__ __forceinline__ void tma_store_3d(const void* map, uint32_t src, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// All committed bulk stores of this thread have finished READING shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// All committed bulk stores of this thread are complete (writes performed).
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Order this thread's generic shared-memory writes before later async-proxy reads.
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Barrier among `count` threads (multiple of 32) on hardware barrier `id`.
__device__ __forceinline__ void named_bar(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory, MMA, commit, loads
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t holder_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   holder_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// Pair forms: one warp of EACH CTA of the pair executes them; the two CTAs
// receive the same tensor-memory address.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t holder_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   holder_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Pair MMA (M = 256 over two CTAs): each CTA supplies 128 rows of A and half
// of B's N rows from the same shared-memory offsets, and receives its 128
// rows of D, all N columns, in its own tensor memory.  Issued by the leader.
__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                 uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the mbarrier at shared::cluster address `cbar` (either CTA
// of the pair) when every pair MMA issued so far by this thread completes.
__device__ __forceinline__ void tc_commit_pair(uint32_t cbar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   cbar)
               : "memory");
}

// Arrive once on `bar` when every MMA issued so far by this thread completes.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// 32 lanes x 32 columns of 32-bit values: thread t of the warp receives lane
// (base lane + t), columns [col, col+32).
__device__ __forceinline__ void tmem_ld_32x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
// 32 lanes x 16 columns: thread t receives lane (base lane + t), columns [col, col+16).
__device__ __forceinline__ void tmem_ld_32x32_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
// 32 lanes x 8 columns: thread t receives lane (base lane + t), columns [col, col+8).
__device__ __forceinline__ void tmem_ld_32x32_x8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Shared-memory matrix descriptors (tcgen05 format, 128-byte swizzle).
//   bits  0-13 start address >> 4      bits 16-29 leading byte offset >> 4
//   bits 32-45 stride byte offset >> 4 bits 46-47 version (1 on sm_100)
//   bits 61-63 layout (2 = 128-byte swizzle)
// K-major: rows of 64 bf16 (128 B) along K, 8-row groups 1024 B apart (SBO);
//          the leading offset is unused for this layout and set to 16 B.
// MN-major: 64 bf16 along M/N per 128-B row, consecutive K rows 128 B apart,
//          8-row K groups `sbo` apart, 64-wide M/N chunks `lbo` apart.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 2ull << 61;
  return d;
}

// Instruction descriptor of kind::f16 with bf16 A/B, fp32 D, M x N
// (M = 128 for one CTA, 256 for a pair).
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n, bool b_mn_major) {
  return (1u << 4)                        // D format: f32
         | (1u << 7)                      // A format: bf16
         | (1u << 10)                     // B format: bf16
         | ((b_mn_major ? 1u : 0u) << 16) // B major-ness
         | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Small numeric helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------------------
// The pair X = hi + lo that carries X between Newton-Schulz steps: hi =
// bf16(X) (round to nearest even), lo an int8 q with X ~ hi + q * 2^(E - 15),
// E the exponent of hi.  |X - hi| <= 2^(E - 8), so (X - hi) / 2^(E-15) lies in
// [-128, 128]; q is its nearest-even rounding clamped to [-128, 127], and
// |X - (hi + q 2^(E-15))| <= 2^(E - 16) (2^(E - 15) in the one clamped case,
// X exactly halfway above hi): about 16 significant bits.  Where hi is 0,
// subnormal or below 2^-111, q is ignored (the value is hi).
// ---------------------------------------------------------------------------
// Branch-free: the exponent comes from hi's bits with masks, and E < -111 is
// handled by integer max on those bits (the decoder's unit is then 0, so q
// there carries nothing; the encoder writes 0 or any small value).
//
// fb: fp32 bits of a bf16 (the bf16 in the upper half).  2^(E - 15), or 0
// when E < -111.
__device__ __forceinline__ float lo8_unit(uint32_t fb) {
  const int eb = static_cast<int>(fb & 0x7F800000u) - (15 << 23);
  return __int_as_float(max(eb, 0));
}

// 2^(15 - E) with E clamped below at -111 (exact power of two).
__device__ __forceinline__ float lo8_inv_unit(uint32_t fb) {
  return __uint_as_float(0x86800000u - max(fb & 0x7F800000u, 16u << 23));
}

// fp32 bits of element k (0 = low half) of a bf16x2 word.
__device__ __forceinline__ uint32_t bf16_word_bits(uint32_t w, int k) {
  return k ? (w & 0xFFFF0000u) : (w << 16);
}

// Eight values -> eight bf16 (uint4) and eight int8 (uint2) of the pair.
// d = x - hi is exact in fp32 and scaling by 2^(15 - E) is exact, so q is
// the nearest-even rounding of t = d / 2^(E - 15), clamped to [-128, 127].
// t lies in [-128, 128] (|d| is at most half a bf16 unit of hi), so only 128
// needs the clamp; adding 1.5 * 2^23 then rounds t to the nearest integer
// (ties to even, the fp32 unit at that magnitude is 1) and leaves it, two's
// complement, in the low byte of the sum's bits.  No int/float conversion
// instruction is used (those run at an eighth of the fp32 rate).
__device__ __forceinline__ void pair_encode8(const float (&v)[8], uint4& hi, uint2& lo) {
  uint32_t h[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) h[k] = pack_bf16x2(v[2 * k], v[2 * k + 1]);
  uint32_t m[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t fb = bf16_word_bits(h[k >> 1], k & 1);
    const float t = fminf((v[k] - __uint_as_float(fb)) * lo8_inv_unit(fb), 127.0f);
    m[k] = __float_as_uint(t + 12582912.0f);
  }
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(w[k]) : "r"(m[2 * k]), "r"(m[2 * k + 1]));
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  uint32_t l0, l1;
  asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(l0) : "r"(w[0]), "r"(w[1]));
  asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(l1) : "r"(w[2]), "r"(w[3]));
  lo = make_uint2(l0, l1);
}

// Packed pairs of fp32 (f32x2 arithmetic, each lane rounded to nearest as
// its scalar form would be).
__device__ __forceinline__ unsigned long long f2(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_split(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b, unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long f2_mul(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long f2_sub(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// x' = fl(fl(a x + acc) * s) for eight values of the pair (hi, lo), decoded
// and updated two at a time with packed fp32 arithmetic: per value the same
// operations, in the same order, as pair_decode8 then fmaf and *.
__device__ __forceinline__ void pair_axpy8(const uint4 hi, const uint2 lo, const float* acc, float a, float s,
                                           float (&x)[8]) {
  const uint32_t h[4] = {hi.x, hi.y, hi.z, hi.w};
  const uint32_t l[2] = {lo.x, lo.y};
  const unsigned long long magic2 = f2(12582912.0f, 12582912.0f), a2 = f2(a, a), s2 = f2(s, s);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t fb0 = h[j] << 16, fb1 = h[j] & 0xFFFF0000u;
    const int k0 = 2 * j, k1 = 2 * j + 1;
    const uint32_t sel0 = (k0 & 3) | ((8 | (k0 & 3)) * 0x1110), sel1 = (k1 & 3) | ((8 | (k1 & 3)) * 0x1110);
    uint32_t q0, q1;
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(q0) : "r"(l[k0 >> 2]), "r"(sel0));
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(q1) : "r"(l[k1 >> 2]), "r"(sel1));
    const unsigned long long qf = f2_sub(f2(__int_as_float(static_cast<int>(q0) + 0x4B400000),
                                             __int_as_float(static_cast<int>(q1) + 0x4B400000)),
                                          magic2);
    const unsigned long long v =
        f2_fma(qf, f2(lo8_unit(fb0), lo8_unit(fb1)), f2(__uint_as_float(fb0), __uint_as_float(fb1)));
    f2_split(f2_mul(f2_fma(a2, v, f2(acc[k0], acc[k1])), s2), x[k0], x[k1]);
  }
}

// pair_encode8 with its fp32 arithmetic two values at a time (same result).
__device__ __forceinline__ void pair_encode8_x2(const float (&x)[8], uint4& hi, uint2& lo) {
  const unsigned long long magic2 = f2(12582912.0f, 12582912.0f);
  uint32_t hh[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) hh[k] = pack_bf16x2(x[2 * k], x[2 * k + 1]);
  uint32_t m[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t fb0 = hh[j] << 16, fb1 = hh[j] & 0xFFFF0000u;
    const unsigned long long d = f2_sub(f2(x[2 * j], x[2 * j + 1]), f2(__uint_as_float(fb0), __uint_as_float(fb1)));
    float t0, t1;
    f2_split(f2_mul(d, f2(lo8_inv_unit(fb0), lo8_inv_unit(fb1))), t0, t1);
    float m0, m1;
    f2_split(f2_add(f2(fminf(t0, 127.0f), fminf(t1, 127.0f)), magic2), m0, m1);
    m[2 * j] = __float_as_uint(m0);
    m[2 * j + 1] = __float_as_uint(m1);
  }
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(w[k]) : "r"(m[2 * k]), "r"(m[2 * k + 1]));
  uint32_t l0, l1;
  asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(l0) : "r"(w[0]), "r"(w[1]));
  asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(l1) : "r"(w[2]), "r"(w[3]));
  hi = make_uint4(hh[0], hh[1], hh[2], hh[3]);
  lo = make_uint2(l0, l1);
}

// Eight values of the pair back to fp32: hi + q * 2^(E - 15).  q is
// sign-extended from its byte with one byte permute, and turned into a float
// exactly as the bits of 1.5 * 2^23 + q minus 1.5 * 2^23.
__device__ __forceinline__ void pair_decode8(const uint4 hi, const uint2 lo, float (&v)[8]) {
  const uint32_t h[4] = {hi.x, hi.y, hi.z, hi.w};
  const uint32_t l[2] = {lo.x, lo.y};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t fb = bf16_word_bits(h[k >> 1], k & 1);
    uint32_t q;
    const uint32_t sel = (k & 3) | ((8 | (k & 3)) * 0x1110);  // byte k & 3, its sign in bytes 1..3
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(q) : "r"(l[k >> 2]), "r"(sel));
    const float qf = __int_as_float(static_cast<int>(q) + 0x4B400000) - 12582912.0f;
    v[k] = fmaf(qf, lo8_unit(fb), __uint_as_float(fb));
  }
}

}  // namespace muon
