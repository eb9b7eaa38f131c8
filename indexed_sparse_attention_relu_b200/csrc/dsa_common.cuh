// dsa_common.cuh -- sm_100a building blocks shared by the DSA kernels:
// inline-PTX wrappers for mbarriers (with time-bounded waits), tcgen05
// (TMEM allocation, MMA, commit, TMEM load/store), TMA tile loads, cp.async
// gathers, the UMMA shared-memory / instruction descriptors, and the sticky
// device status word.
//
// Every wait in this library is bounded: after g_wait_limit_ns of wall time a
// wait records DSA_ERR_DEVICE_TIMEOUT in the status word and returns false;
// the caller then stops its loop and reaches the kernel's teardown (TMEM is
// always released). Nothing here traps.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dsa.h"

namespace dsa {

// ---------------------------------------------------------------- status word
// First device-side error code since the last dsa_read_device_status().
// Defined here: every kernel of the library is compiled in one translation unit.
__device__ int g_device_status = 0;

__device__ __forceinline__ void set_device_status(int code) {
  atomicCAS(&g_device_status, 0, code);
}

// Wall-time limit of every bounded wait, in ns. 2 s is far above any legal
// wait; dsa_debug_set_wait_limit() lowers it so a test can make a wait run
// out in milliseconds.
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;
__device__ uint64_t g_wait_limit_ns = kDefaultWaitLimitNs;

// Test hook: non-zero makes the two-CTA attention's score CTA withhold its
// first "P ready" signal, so the value CTA's bounded wait for it runs out
// (set by dsa_debug_withhold_signal(); 0 in normal operation).
__device__ int g_debug_withhold = 0;

// ---------------------------------------------------------------- debug build
// With DSA_DEBUG the tensor-core kernels request kCanaryBytes more dynamic
// shared memory and thread 0 writes a fixed pattern right after the kernel's
// layout at entry and checks it at exit: a layout that wrote past its end
// shows up as DSA_ERR_DEVICE_LAYOUT. Without DSA_DEBUG both are no-ops.
#ifdef DSA_DEBUG
constexpr int kCanaryBytes = 16;
#else
constexpr int kCanaryBytes = 0;
#endif
constexpr int canary_offset(int layout_bytes) { return (layout_bytes + 15) / 16 * 16; }
__device__ __forceinline__ void canary_set(uint8_t* smem, int layout_bytes) {
#ifdef DSA_DEBUG
  if (threadIdx.x == 0)
    *reinterpret_cast<uint4*>(smem + canary_offset(layout_bytes)) = make_uint4(0xD5A0C0DEu, 0x5EA1ED00u, 0xC0FFEE11u, 0xB200B200u);
#else
  (void)smem;
  (void)layout_bytes;
#endif
}
__device__ __forceinline__ void canary_check(const uint8_t* smem, int layout_bytes) {
#ifdef DSA_DEBUG
  if (threadIdx.x == 0) {
    const uint4 c = *reinterpret_cast<const uint4*>(smem + canary_offset(layout_bytes));
    if (c.x != 0xD5A0C0DEu || c.y != 0x5EA1ED00u || c.z != 0xC0FFEE11u || c.w != 0xB200B200u)
      set_device_status(DSA_ERR_DEVICE_LAYOUT);
  }
#else
  (void)smem;
  (void)layout_bytes;
#endif
}

// ---------------------------------------------------------------- cache rows
// Where logical row s of sequence b lives in a cache (index keys, their FP8
// scales and the latent KV rows all share it). Contiguous caches: row
// b * L_max + s. Paged caches (block table; the paged key cache the fused
// indexer reads, section 3 of "Optimizing Inference for New Model
// Architectures ..."): a pool of num_pages pages of page_size rows, and row
// table[b * max_pages + s / page_size] * page_size + s % page_size. A page id
// outside [0, num_pages) is never dereferenced: row() reports it (ok = false)
// and returns row 0, which the caller masks.
struct CacheMap {
  const int32_t* table;  // [B, max_pages] or null (contiguous)
  int32_t L_max;
  int32_t page_size;     // multiple of 64 (paged)
  int32_t max_pages;     // ceil(L_max / page_size)
  int32_t num_pages;

  __device__ __forceinline__ bool paged() const { return table != nullptr; }
  __device__ __forceinline__ int32_t row(int b, int s, bool& ok) const {
    if (table == nullptr) {
      ok = true;
      return b * L_max + s;
    }
    const int32_t pg = __ldg(table + static_cast<int64_t>(b) * max_pages + s / page_size);
    ok = static_cast<uint32_t>(pg) < static_cast<uint32_t>(num_pages);
    return ok ? pg * page_size + s % page_size : 0;
  }
  // As row(), recording a bad page id in the status word.
  __device__ __forceinline__ int32_t row_checked(int b, int s) const {
    bool ok;
    const int32_t r = row(b, s, ok);
    if (!ok) set_device_status(DSA_ERR_DEVICE_INDEX);
    return r;
  }
};

__device__ __forceinline__ uint64_t wait_limit_ns() {
  return *reinterpret_cast<volatile uint64_t*>(&g_wait_limit_ns);
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking check that the phase with the given parity has completed (for
// a thread that polls several barriers: try_wait may suspend the thread on one
// of them while another becomes ready).
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete. Bounded: returns
// false (and records a timeout) after g_wait_limit_ns, or as soon as *abort is
// set by another role that already gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  const uint64_t limit = wait_limit_ns();
  while (true) {
    if (mbar_try(a, parity)) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > limit) {
      set_device_status(DSA_ERR_DEVICE_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

// Warp-uniform variant for roles that go on to warp-collective tcgen05 ops:
// every lane waits, and the warp proceeds only if all lanes succeeded.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------- programmatic dependent launch
// Lets the next kernel of the chain be scheduled once every CTA of this grid
// has started (it still waits for this grid's results, see below).
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Waits until the preceding grid has completed and its writes are visible
// (returns at once when the kernel was launched without a programmatic edge).
__device__ __forceinline__ void pdl_wait_prior() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Loads of data that the preceding kernel of a chain writes (indexer scores,
// Top-K indices). Under programmatic dependent launch that kernel may still
// be running when this one starts, so the data is not read-only for this
// kernel's lifetime: the read-only (non-coherent) path must not serve it, and
// the load must not be moved above pdl_wait_prior(). A volatile asm is kept in
// program order with the wait (also a volatile asm) and is an ordinary
// coherent global load.
__device__ __forceinline__ int32_t ld_dep(const int32_t* ptr) {
  int32_t v;
  asm volatile("ld.global.b32 %0, [%1];" : "=r"(v) : "l"(ptr));
  return v;
}
__device__ __forceinline__ float ld_dep(const float* ptr) {
  float v;
  asm volatile("ld.global.f32 %0, [%1];" : "=f"(v) : "l"(ptr));
  return v;
}
__device__ __forceinline__ float4 ld_dep4(const float* ptr) {
  float4 v;
  asm volatile("ld.global.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(ptr));
  return v;
}

// ---------------------------------------------------------------- clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t local_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
  return r;
}

// All threads of all CTAs of the cluster (used once, right after barrier
// initialisation: every CTA of a cluster is resident together and reaches it).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on a local barrier whose arrivals come from other CTAs.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_cluster(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  const uint64_t limit = wait_limit_ns();
  while (true) {
    if (mbar_try_cluster(a, parity)) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > limit) {
      set_device_status(DSA_ERR_DEVICE_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

// ---------------------------------------------------------------- proxies
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// ---------------------------------------------------------------- bulk copies
// `bytes` (a multiple of 16) from global `src` to shared `dst` (both 16-byte
// aligned) through the async proxy; completes as bytes on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------- cp.async
// 16-byte global->shared copy; src_bytes < 16 zero-fills the rest (0 = all zeros).
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Four rows (y0..y3) x one box of columns starting at x, written as four
// consecutive box rows at dst (the map's swizzle applies). A row coordinate
// outside the tensor reads zeros.
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y0, int32_t y1,
                                            int32_t y2, int32_t y3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3), "r"(smem_u32(bar))
      : "memory");
}

// Named barrier `id` (1..15) over `count` threads (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
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

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16. A (M x 16 per
// instruction, K-major) sits in TMEM with row m in lane m and the 16 bf16
// elements of the K step packed two per 32-bit column (8 columns, even
// element in the low half).
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on `bar` when every tcgen05 op issued so far by this thread completes.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bits, 16 consecutive columns: thread i gets lane (base + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}

// 16 lanes x 256 bits, 8 repetitions along the columns (64 columns): thread
// t holds rows (t/4) and (t/4 + 8) of the 16-lane window at the address, and
// in repetition j the columns 8j + 2(t%4) and 8j + 2(t%4) + 1; registers
// [4j .. 4j+3] = (row t/4: col, col+1), (row t/4+8: col, col+1).
__device__ __forceinline__ void tmem_ld16x256_x8(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Hardware base-2 exponential (MUFU.EX2 through the PTX ex2.approx.ftz
// instruction); ex2(-inf) = +0.
// Packed fp32 pair arithmetic of sm_100 (one instruction for two lanes of work).
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("mul.f32x2 %0, %1, %2;"
      : "=l"(reinterpret_cast<uint64_t&>(d))
      : "l"(reinterpret_cast<const uint64_t&>(a)), "l"(reinterpret_cast<const uint64_t&>(b)));
  return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("add.f32x2 %0, %1, %2;"
      : "=l"(reinterpret_cast<uint64_t&>(d))
      : "l"(reinterpret_cast<const uint64_t&>(a)), "l"(reinterpret_cast<const uint64_t&>(b)));
  return d;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Sequence of token t from cu_q[0..B]: one warp, 32 boundaries per round
// (coalesced) instead of a dependent binary search; every lane gets the answer.
__device__ __forceinline__ int seq_of_token_warp(const int32_t* __restrict__ cu_q, int B, int t) {
  const int lane = threadIdx.x & 31;
  // stride through the boundaries in rounds of 32 until the bracket is found
  int lo = 0, hi = B;          // answer in [lo, hi)
  while (hi - lo > 1) {
    const int span = hi - lo;
    const int step = (span + 31) / 32;
    const int pos = lo + lane * step;                    // candidate lower bound
    const bool le = pos < hi && __ldg(cu_q + pos) <= t;  // cu_q[pos] <= t
    const unsigned m = __ballot_sync(0xffffffffu, le);
    const int last = 31 - __clz(m);                      // last lane with cu_q[pos] <= t (lane 0 always)
    const int nlo = lo + last * step;
    hi = min(hi, nlo + step);
    lo = nlo;
  }
  return lo;
}

// Arrives on `bar` once every cp.async issued so far by this thread has landed
// (the barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor for tcgen05.mma (sm_100 format): start
// address, leading/stride byte offsets (16-byte units), version 1, base
// offset 0, swizzle mode 2 = 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;  // descriptor version for sm_100
  d |= 2ull << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                                   // D format: f32
         | (1u << 7)                                 // A format: bf16
         | (1u << 10)                                // B format: bf16
         | (static_cast<uint32_t>(a_mn_major) << 15)  // A major
         | (static_cast<uint32_t>(b_mn_major) << 16)  // B major
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a 128-byte
// swizzled atom column whose rows are 128 bytes apart (atoms 1024-B aligned).
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// Order-preserving map from fp32 to uint32 (-0 and +0 map to the same key).
__device__ __forceinline__ uint32_t float_order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }
__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

// Sequence of token t from cu_q[0..B] (binary search).
__device__ __forceinline__ int seq_of_token(const int32_t* __restrict__ cu_q, int B, int t) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu_q + mid) <= t)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

}  // namespace dsa
