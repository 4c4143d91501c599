// Device-side building blocks for the sm_100a kernels: the Philox4x32-10
// generator, the Box-Muller transform, and thin inline-PTX wrappers for
// mbarriers, TMA tile loads and the tcgen05 tensor-core / tensor-memory
// instructions.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lg {

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy
// as 1, 2, 3", SC'11): ten rounds of the two-multiplier S-P network with a
// Weyl key schedule.  Key = (seed mod 2^32, seed >> 32); block j uses the
// counter (j mod 2^32, j >> 32, 0, 0).
// ---------------------------------------------------------------------------
struct Words4 {
  uint32_t w0, w1, w2, w3;
};

__device__ __forceinline__ Words4 philox4x32_10(uint64_t block, uint32_t k0, uint32_t k1) {
  uint32_t c0 = (uint32_t)block, c1 = (uint32_t)(block >> 32), c2 = 0u, c3 = 0u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
    const uint32_t n1 = (uint32_t)p1;
    const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
    const uint32_t n3 = (uint32_t)p0;
    c0 = n0;
    c1 = n1;
    c2 = n2;
    c3 = n3;
  }
  return Words4{c0, c1, c2, c3};
}

// Box-Muller (Box and Muller, Ann. Math. Statist. 29, 1958) on one pair of
// words: u1 = ((a >> 8) + 1) 2^-24 in (0, 1], u2 = (b >> 8) 2^-24 in [0, 1);
// returns rho cos(2 pi u2) and rho sin(2 pi u2) with rho = sqrt(-2 ln u1), in
// double and within a few double ulps of the exact values, so that the FP32
// results (and any blend computed from them in double) round as the exact
// values would.  Both uniforms are 24-bit integers scaled by 2^-24, which lets
// every range reduction below be exact integer work; the three constant tables
// come from gen_bm_tables.py and are staged in shared memory by the caller.
// ---------------------------------------------------------------------------
struct alignas(16) BmLogEntry {
  double inv_c;  // 1 / c_i cut to 28 significant bits, c_i = 1 + i / 256
  double y;      // -2 times the log term: 2 ln(inv_c), or 2 ln(2 inv_c) for i > LG_BM_LOG_SWITCH
};
struct alignas(16) BmTrigEntry {
  double s, c;  // sin, cos of the entry's angle (exact 0 and +-1 at quarter turns)
};
struct BmTables {
  const BmLogEntry* log;      // 257 entries
  const BmTrigEntry* coarse;  // 4096 entries: 2 pi i / 4096
  const BmTrigEntry* fine;    // 2049 entries: 2 pi k 2^-24, k = 0..2048
};
constexpr int kBmLogSwitch = 106;
constexpr int kBmCoarseBits = 12;  // 4096 coarse angles; the remainder takes the other 12 of 24 bits

__device__ __forceinline__ double bits_to_double(uint64_t b) { return __longlong_as_double((long long)b); }
__device__ __forceinline__ double hilo_to_double(uint32_t hi, uint32_t lo) {
  return __hiloint2double((int)hi, (int)lo);
}

// y = -2 ln(n 2^-24) for an integer n in [1, 2^24] (Tang's table method).
// With n = m 2^kf, m in [1, 2), the nearest grid point c_i = 1 + i/256 gives
// r = m inv_c - 1 exactly (m has <= 24 significant bits, inv_c 28) and
// |r| <= 2^-9 + 2^-27, so -2 log1p(r) = r q(r), q the Horner form of
// -2 + r - 2r^2/3 + r^3/2 - 2r^4/5 + r^5/3 (the log1p series to r^6), is
// within 2^-56 |r|.  Past c = sqrt 2 the entry already holds the term of c/2
// and the exponent is one higher, so a nonzero multiple of ln 2 always
// dominates the table term (|ln u1| >= ln 2 - 0.35) and no step cancels by
// more than a factor of two.
__device__ __forceinline__ double neg2_ln_grid24(uint32_t n, const BmLogEntry* tab) {
  // n <= 2^24 converts to FP32 exactly: its exponent field is kf + 127 and its
  // 23 fraction bits are those of m = n 2^-kf.
  const uint32_t fb = __float_as_uint(__uint2float_rn(n));
  const uint32_t frac = fb & 0x7FFFFFu;
  const uint32_t i = ((frac >> 14) + 1u) >> 1;              // nearest c_i = 1 + i/256: 0..256
  const BmLogEntry e = tab[i];
  const uint32_t j = 151u - (fb >> 23) - (i > (uint32_t)kBmLogSwitch ? 1u : 0u);  // 24 - kf (- 1): 0..24
  // m in [1, 2) from the fraction bits (exact)
  const double m = hilo_to_double(0x3FF00000u | (frac >> 3), frac << 29);
  const double r = fma(m, e.inv_c, -1.0);
  double q = 1.0 / 3.0;
  q = fma(q, r, -2.0 / 5.0);
  q = fma(q, r, 1.0 / 2.0);
  q = fma(q, r, -2.0 / 3.0);
  q = fma(q, r, 1.0);
  q = fma(q, r, -2.0);
  const double jd = __uint2double_rn(j);  // exact
  const double base = fma(jd, 1.3862943611198906188, e.y);  // 2 j ln 2 + table term
  return fma(r, q, base);
}

// sqrt(y) for y = +-0 or y in [2^-24, 64): an FP32 reciprocal square root
// seed r (relative error e, |e| < 2^-22 with the truncation of y to FP32),
// then one third-order (Householder) step on sqrt(y) = t (1 - h)^(-1/2) with
// t = y r and h = 1 - y r^2 = -2e - e^2: t (1 + h/2 + 3h^2/8) leaves a
// truncation error of 5h^3/16 < 2^-64 relative, so the result is within
// ~1.5 double ulps.
__device__ __forceinline__ double sqrt_seeded(double y) {
  // max as signed: -0 (high word 0x80000000) takes the finite seed too
  const uint32_t hi = (uint32_t)max(__double2hiint(y), 0x3E700000);
  const float yf = __uint_as_float((hi - (896u << 20)) << 3);        // y truncated to FP32
  float rf;
  asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(rf) : "f"(yf));
  const uint32_t rb = __float_as_uint(rf);
  const double r = hilo_to_double((rb >> 3) + (896u << 20), rb << 29);
  const double t = y * r;
  const double h = fma(-t, r, 1.0);
  return fma(t * h, fma(h, 0.375, 0.5), t);
}

// sin and cos of 2 pi b 2^-24 for the integer b = w >> 8 of a 32-bit word w:
// b = iu 2^12 + rd with iu the nearest 1/4096 turn and rd in [-2048, 2048),
// both read off w by exact integer work, then the angle-addition formulas on
// the coarse entry of iu and the fine entry of |rd| (sin negated for rd < 0).
// Near a zero of sin or cos the coarse term is exactly zero, so the result
// keeps full relative accuracy; elsewhere the angle is at least half a coarse
// step from the zero, so each result is at least about half the larger of
// its two products and the sum loses at most one bit.
__device__ __forceinline__ void sincos_turn24(uint32_t w, const BmTables& tab, double& s, double& c) {
  // (w + 2^19) >> 20 = (b + 2^11) >> 12 = iu; past the top it wraps to 0, the
  // same angle.
  const uint32_t iu = (w + (1u << 19)) >> 20;
  // the low 12 bits of b, taken as a signed 12-bit integer, are rd
  const uint32_t lo = w << 12;
  const int rd = (int)lo >> 20;
  const BmTrigEntry a = tab.coarse[iu];
  const BmTrigEntry f = tab.fine[abs(rd)];
  // sin of the remainder with the sign of rd (lo's sign bit)
  const double sf = hilo_to_double((uint32_t)__double2hiint(f.s) ^ (lo & 0x80000000u), (uint32_t)__double2loint(f.s));
  s = fma(a.s, f.c, a.c * sf);
  c = fma(a.c, f.c, -(a.s * sf));
}

__device__ __forceinline__ void box_muller(uint32_t a, uint32_t b, const BmTables& tab, double& e_cos,
                                           double& e_sin) {
  const double rho = sqrt_seeded(neg2_ln_grid24((a >> 8) + 1u, tab.log));
  double s, c;
  sincos_turn24(b, tab, s, c);
  e_cos = rho * c;
  e_sin = rho * s;
}

// The radius and the angle of one pair of words (rho and cos, sin), for a
// caller that scales rho once before using both products.
__device__ __forceinline__ void box_muller_polar(uint32_t a, uint32_t b, const BmTables& tab, double& rho, double& c,
                                                 double& s) {
  rho = sqrt_seeded(neg2_ln_grid24((a >> 8) + 1u, tab.log));
  sincos_turn24(b, tab, s, c);
}

// ---------------------------------------------------------------------------
// Shared-memory addresses, mbarriers, timers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
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

// try_wait with a suspend-time hint: the thread sleeps until the phase
// completes or about `hint_ns` pass, instead of re-polling.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// ---------------------------------------------------------------------------
// Thread-block clusters: rank, distributed shared memory, cluster barriers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void ld_shared_cluster_v4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c,
                                                     uint32_t& d) {
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "r"(addr)
               : "memory");
}
// Arrive on an mbarrier in another CTA of the cluster (release at cluster scope).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Relaxed form, for a signal that publishes no data written by the arriving
// thread (for example "my tensor-memory loads have completed").
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// try_wait with acquire at cluster scope: makes other CTAs' writes that
// preceded their release-arrive visible to this thread.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_try_wait_cluster_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMA: 2-D tiled bulk tensor load global -> shared, completion counted in
// bytes on an mbarrier.  c0 is the innermost (contiguous) coordinate.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int32_t c0,
                                            int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

// Pair form (CTA pair of a 2-SM MMA): this CTA's tile lands in its own
// shared memory; the transaction bytes are counted on `bar`, a cluster
// address of the pair leader's mbarrier.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar, int32_t c0,
                                                 int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

// TMA tensor store shared -> global (bulk-group completion) with an L2
// cache policy; out-of-range rows and columns of the box are not written.
__device__ __forceinline__ void tma_store_2d_hint(const CUtensorMap* map, uint32_t src, int32_t c0, int32_t c1,
                                                  uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most 0 bulk groups of this thread are still reading their
// shared-memory source (the buffer may be rewritten) / still in flight.
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// L2 eviction-priority policies for loads that carry a cache hint.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// tma_load_2d / tma_load_2d_pair with an L2 cache policy.
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap* map, uint32_t bar, int32_t c0,
                                                 int32_t c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%3, "
      "%4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair_hint(uint32_t dst, const CUtensorMap* map, uint32_t bar, int32_t c0,
                                                      int32_t c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], "
      "[%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}

// 16-byte global store with an L2 cache policy, bypassing L1.
__device__ __forceinline__ void st_global_v4_hint(void* ptr, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                                  uint64_t policy) {
  asm volatile("st.global.L1::no_allocate.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(ptr), "r"(a),
               "r"(b), "r"(c), "r"(d), "l"(policy)
               : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory allocation, MMA issue, commit, TMEM <-> registers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major bf16 tile whose rows are
// 128 bytes (64 elements) and stored with the 128-byte swizzle: 8-row groups
// 1024 bytes apart (stride byte offset), leading byte offset unused, version
// 1 (sm_100), layout type 2 (SWIZZLE_128B).  The tile base must be 1024-byte
// aligned; stepping K by 16 elements adds 32 bytes to the start address.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;            // leading byte offset (16 B; ignored for this layout)
  d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset: 1024 B between 8-row groups
  d |= (uint64_t)1 << 46;            // descriptor version for sm_100
  d |= (uint64_t)2 << 61;            // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: bf16 A and B (both K-major), FP32 D.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int m, int n) {
  return (1u << 4)                       // D format: F32
         | (1u << 7)                     // A format: BF16
         | (1u << 10)                    // B format: BF16
         | ((uint32_t)(n >> 3) << 17)    // N / 8
         | ((uint32_t)(m >> 4) << 24);   // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]^T, one 128 x N x 16 step.
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, one 128 x N x 16 step; A is 128 lanes x
// 8 columns of packed bf16 pairs (element k of a row in column k/2, low half
// for even k).
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on an mbarrier when all previously issued tcgen05 operations of
// this thread have completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// 2-SM (CTA pair) variants.  Allocation and release are issued by the same
// warp in both CTAs of the pair; the MMA is issued by the pair leader only
// and reads A / writes D in each CTA's own memories, with B split between
// the two CTAs' shared memories.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void umma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Block-scaled MXFP8 MMA (E4M3 A and B in shared memory, E8M0 scale factors
// in tensor memory), SM pair: D[M=256, N] (+)= (A x sfa) (B x sfb)^T over
// K = 32.  The scale-factor IDs (which byte of each 32-bit scale word) are
// in the instruction descriptor.
__device__ __forceinline__ void umma_mx_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Instruction descriptor, kind::mxf8f6f4 with block scaling: E4M3 A and B
// (both K-major), E8M0 scale factors, dense K = 32; sf_a / sf_b select the
// byte of the 32-bit scale word each row's scale is taken from.
__host__ __device__ constexpr uint32_t idesc_mx_e4m3(int m, int n, uint32_t sf_a, uint32_t sf_b) {
  return (sf_b << 4)                      // B scale-factor ID
         | (0u << 7) | (0u << 10)        // A, B format: E4M3
         | ((uint32_t)(n >> 3) << 17)    // N / 8
         | (1u << 23)                    // scale format: E8M0
         | ((uint32_t)(m >> 4) << 24)    // M / 16
         | (sf_a << 29);                 // A scale-factor ID
}

// Shared-memory descriptor of 32 rows of 16 bytes stored contiguously, no
// swizzle (four 8-row core matrices 128 bytes apart): the source layout of a
// tcgen05.cp 32x128b copy.
__device__ __forceinline__ uint64_t plain_rows16_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(128 >> 4) << 16;  // leading byte offset (one core matrix along the row)
  d |= (uint64_t)(128 >> 4) << 32;  // stride byte offset: 128 B between 8-row core matrices
  d |= (uint64_t)1 << 46;           // descriptor version for sm_100
  return d;                          // layout type 0: no swizzle
}

// Shared -> tensor memory copy of 32 rows x 128 bits, replicated to all four
// lane quarters (lanes 32 q + i, columns taddr .. +3 get row i), in both CTAs
// of an SM pair.  Ordered with the issuing thread's later tcgen05.mma.
__device__ __forceinline__ void tmem_cp_32x128b_x4_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Arrive once on the mbarrier at offset `bar` in every CTA of `cta_mask` when
// all previously issued tcgen05 operations of this thread have completed.
__device__ __forceinline__ void umma_commit_pair_mc(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(cta_mask)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns -> 32 registers per thread.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}

// 32 lanes x 16 consecutive 32-bit columns -> 16 registers per thread.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}

// 32 lanes x 8 / 4 consecutive 32-bit columns <-> registers.
__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st_32x32b_x4(uint32_t taddr, const uint32_t (&v)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(v[0]), "r"(v[1]),
               "r"(v[2]), "r"(v[3])
               : "memory");
}
__device__ __forceinline__ void tmem_ld_32x32b_x4(uint32_t taddr, uint32_t (&v)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
               : "r"(taddr));
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "r"(addr) : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);  // .x (low half) = lo, .y = hi
  return *reinterpret_cast<uint32_t*>(&p);
}

}  // namespace lg
