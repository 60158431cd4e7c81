// Internal declarations shared by the libmoe.so translation units: launch
// helpers, device-side PTX wrappers (mbarrier, TMA, tcgen05) and the kernel
// entry points each .cu file provides to moe_api.cu.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace moe {

// --------------------------------------------------------------- constants
constexpr int kMaxE = MOE_MAX_EXPERTS;
constexpr int kMaxK = MOE_MAX_TOPK;
constexpr int kRowAlign = MOE_ROW_ALIGN;
// Tokens per block of the permutation's first (counting) pass.
constexpr int kPermBlock = 256;
// Bounded waits: a kernel that waits longer than this on an on-chip barrier
// gives up, reports through its error word and exits.
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s

// Device error codes ORed into the error word.
enum : int {
  kErrTimeoutProducer = 1 << 0,
  kErrTimeoutMma = 1 << 1,
  kErrTimeoutEpilogue = 1 << 2,
  kErrTimeoutDrain = 1 << 3,
  kErrRowOverflow = 1 << 4,
};

inline int64_t pad_rows(int64_t n) { return (n + kRowAlign - 1) / kRowAlign * kRowAlign; }

// ---------------------------------------------------------- device helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// mbarrier --------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Programmatic dependent launch.  A kernel launched with
// launch_kernel(..., pdl = true) may start while the previous kernel in the
// stream is still running; it must call pdl_wait() before touching anything
// that kernel (or any earlier stream work) writes.  pdl_trigger() lets the
// next such kernel launch once every CTA of this one has called it.  Both
// are no-ops for kernels launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase with the given parity to complete; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitTimeoutNs) return false;
  }
  return true;
}

// TMA (tiled tensor copies, global -> shared, completion on an mbarrier) ----
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
// TMA store of a 2-D box from this CTA's shared memory (bulk-group
// completion: commit, then wait for the reads of the shared-memory source).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, uint32_t src, int32_t c0,
                                             int32_t c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(src), "r"(c0), "r"(c1)
               : "memory");
}
// Same, with an L2 eviction-priority policy (from make_policy_evict_first).
__device__ __forceinline__ void tma_store_2d_hint(const CUtensorMap* m, uint32_t src, int32_t c0,
                                                  int32_t c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], "
      "%4;" ::"l"(reinterpret_cast<uint64_t>(m)),
      "r"(src), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}
// L2 policy: lines written with it are the first candidates for eviction.
__device__ __forceinline__ uint64_t make_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N committed bulk groups still read their source.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until at most N committed bulk groups are still incomplete.
template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// 16-byte asynchronous copy global -> shared (cp.async, L2 only); the
// bytes past src_bytes (0 or 16) are zero-filled.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// Wait until at most N committed cp.async groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Untiled bulk copy shared -> global of `bytes` contiguous bytes (both
// addresses 16-byte aligned, bytes a multiple of 16), completion tracked by
// the issuing thread's bulk groups (bulk_commit / bulk_wait_read).
__device__ __forceinline__ void bulk_store_1d(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(src), "r"(bytes)
               : "memory");
}
// Untiled bulk copy global -> shared of `bytes` contiguous bytes (both
// addresses 16-byte aligned, bytes a multiple of 16), completion on `bar`.
__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void* src, uint32_t bytes,
                                             uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                            int32_t c0, int32_t c1, int32_t c2, int32_t c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// tcgen05 (5th-generation tensor cores, accumulators in tensor memory) -----
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
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
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem] * B[smem], bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on an mbarrier once every tcgen05 op this thread issued so far is done.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tc_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tc_ld_32cols(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
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
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Clusters of two CTAs (a tcgen05 CTA pair) ---------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(addr), "r"(rank));
  return out;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// 32-bit load from a shared::cluster address (another CTA's shared memory).
__device__ __forceinline__ uint32_t ld_shared_cluster_u32(uint32_t cluster_addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}
// Arrive on an mbarrier that may live in another CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// TMA loads of one CTA of a pair; completion is counted on `bar`, a
// shared::cluster address that may be the leader CTA's barrier.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                                 int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                                 int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d_pair(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                                 int32_t c0, int32_t c1, int32_t c2, int32_t c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
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
// D[tmem of both CTAs] (+)= A[smem of both CTAs] * B[smem of both CTAs]:
// M is split across the pair (128 rows each), N across their B tiles.
__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                 uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on an mbarrier (either CTA of the pair) once every pair MMA this
// thread issued so far is done.
__device__ __forceinline__ void tc_commit_pair(uint32_t cluster_bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   cluster_bar)
               : "memory");
}

// Shared-memory matrix descriptor for tcgen05.mma, 128-byte swizzle.
// K-major operand (rows of 64 bf16 along K): sbo = 1024 (8-row group stride).
// MN-major operand (rows of 64 bf16 along M/N, one row per K index):
//   lbo = byte stride between 64-element M/N blocks, sbo = 1024.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2) << 61;  // 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16 with bf16 A/B, fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major,
                                                      bool b_mn_major) {
  return (1u << 4)                                 // D format: f32
         | (1u << 7)                               // A format: bf16
         | (1u << 10)                              // B format: bf16
         | ((a_mn_major ? 1u : 0u) << 15)          // A major
         | ((b_mn_major ? 1u : 0u) << 16)          // B major
         | (static_cast<uint32_t>(N >> 3) << 17)   // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);  // M / 16
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Eight consecutive elements of a row of the expert outputs o, as loaded
// (one 16-byte vector of bf16, or two of fp32), so a caller can issue every
// load of an iteration before any arithmetic.  Streaming loads: o is read
// once.
template <bool BF16>
struct Row8;
template <>
struct Row8<true> {
  uint4 v;
  __device__ __forceinline__ void load(const void* o, int64_t row, int d, int c8) {
    v = __ldcs(reinterpret_cast<const uint4*>(o) + row * (d / 8) + c8);
  }
  __device__ __forceinline__ void zero() { v = make_uint4(0u, 0u, 0u, 0u); }
  // acc[i] += g * element i (bf16 -> fp32 is exact: the high 16 bits).
  __device__ __forceinline__ void fma_into(float g, float (&acc)[8]) const {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] = fmaf(g, __uint_as_float(w[i] << 16), acc[2 * i]);
      acc[2 * i + 1] = fmaf(g, __uint_as_float(w[i] & 0xffff0000u), acc[2 * i + 1]);
    }
  }
};
template <>
struct Row8<false> {
  float4 a, b;
  __device__ __forceinline__ void load(const void* o, int64_t row, int d, int c8) {
    const float4* r = reinterpret_cast<const float4*>(o) + row * (d / 4) + c8 * 2;
    a = __ldcs(r);
    b = __ldcs(r + 1);
  }
  __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void fma_into(float g, float (&acc)[8]) const {
    acc[0] = fmaf(g, a.x, acc[0]);
    acc[1] = fmaf(g, a.y, acc[1]);
    acc[2] = fmaf(g, a.z, acc[2]);
    acc[3] = fmaf(g, a.w, acc[3]);
    acc[4] = fmaf(g, b.x, acc[4]);
    acc[5] = fmaf(g, b.y, acc[5]);
    acc[6] = fmaf(g, b.z, acc[6]);
    acc[7] = fmaf(g, b.w, acc[7]);
  }
};

// ------------------------------------------------- launchers (host side)
struct RouteArgs {
  const void* x;
  const void* Wg;
  const float* bias;
  int T, d, E, k;
  int32_t* idx;
  float* gate;
  float* margin;
  int gating;        // moe_gating
  float gate_scale;  // multiplies every gate
  float* scores = nullptr;  // non-null: write softmax over all E to [E, T] instead of TopK
  int32_t* err = nullptr;   // device error word for the routers' bounded waits
  // Counting half of the permutation, filled by the streaming router only
  // (launch_route reports whether it did): per (token, slot) the rank among
  // earlier assignments to the same expert in the token's range [T, k], and
  // per range the assignments per expert [G, E] (route_ranges).
  int32_t* lrank = nullptr;
  int32_t* hist = nullptr;
};
// `ranked` (nullable) is set to whether lrank/hist were written.
cudaError_t launch_route(const RouteArgs& a, moe_dtype dtype, cudaStream_t s, int num_sms,
                         bool* ranked = nullptr);

// Token ranges shared by the streaming router and the permutation: G ranges
// of whole 8-token groups, range c = [c*T8/G*8, min(T, (c+1)*T8/G*8)), so
// ranges differ by at most 8 tokens; MT = rows per router tile (<= 128).
constexpr int kMaxRouteRanges = 256;
struct RouteRanges {
  int G, T8, MT;
};
RouteRanges route_ranges(int T, int num_sms);
// Streaming router (route_stream.cu): bf16, E % 8 == 0.  MOE_ROUTE_STREAM=0
// turns it off, for measurements.
bool route_stream_supported(const RouteArgs& a);
cudaError_t launch_route_stream(const RouteArgs& a, int num_sms, cudaStream_t s);
// Tensor-core router (route_tc.cu): bf16, E % 8 == 0.  MOE_ROUTE_TC=0 turns
// it off, for measurements.
bool route_tc_supported(const RouteArgs& a);
cudaError_t launch_route_tc(const RouteArgs& a, cudaStream_t s);

// Whether kernels of the forward chain are launched with programmatic
// dependent launch (default on; MOE_PDL=0 turns it off, for measurements).
bool pdl_enabled();
// Whether the placement kernel carries rows out with bulk stores from
// shared memory (default on for rows up to 8 KB; MOE_PLACE_BULK=0 turns it
// off, for measurements).
bool place_bulk();

// cudaLaunchKernelEx with an optional cluster size and, when `pdl` and
// pdl_enabled(), programmatic stream serialization.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, int cluster, bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl && pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

struct PermuteArgs {
  const void* x;
  const int32_t* idx;
  int T, d, E, k;
  int capacity;  // INT32_MAX when dropless
  void* xp;
  int32_t* pos;
  int32_t* counts;
  int32_t* kept_counts;
  int32_t* offsets;
  int32_t* block_base;  // [nblk * E] scratch
  unsigned int* ticket; // scratch counter
  const int32_t* order = nullptr;  // queue order (token at position i), or null
  const int32_t* prior = nullptr;  // per-expert assignments of earlier shards, or null
  bool ticket_zeroed = false;      // the caller already zeroed *ticket on this stream
};
// Permutation in two kernels over the route_ranges of T: local ranks and
// per-range counts (skipped when the router already wrote them into pos and
// hist), then positions -- prefix over the ranges, capacity, 128-row aligned
// offsets -- and the row copy.  pos holds the local ranks in between.
struct RankedPermuteArgs {
  const void* x;
  const int32_t* idx;
  int T, d, E, k;
  int capacity;                    // INT32_MAX when dropless
  void* xp;
  int32_t* pos;
  int32_t* counts;
  int32_t* kept_counts;
  int32_t* offsets;
  int32_t* hist;                   // [kMaxRouteRanges * E] scratch
  const int32_t* order = nullptr;  // queue order (token at position i), or null
  const int32_t* prior = nullptr;  // per-expert assignments of earlier shards, or null
  bool ranked = false;             // pos / hist already hold the local ranks and counts
  int num_sms = 148;
};
size_t ranked_permute_scratch_bytes(int E);
cudaError_t launch_ranked_permute(const RankedPermuteArgs& a, moe_dtype dtype, cudaStream_t s);

cudaError_t launch_expert_counts(const int32_t* idx, int T, int E, int k, int32_t* counts,
                                 cudaStream_t s);
cudaError_t launch_rank_prefix(const int32_t* gathered, int n_ranks, int E, int rank,
                               int32_t* prior, cudaStream_t s);
size_t permute_scratch_bytes(int T, int E);
cudaError_t launch_permute(const PermuteArgs& a, moe_dtype dtype, cudaStream_t s);
// xp[pos[t, j]] = x[t] for every pos[t, j] >= 0 (pos is [T, npos], npos <= kMaxE).
cudaError_t launch_row_copy(const void* x, const int32_t* pos, int T, int npos, int d,
                            moe_dtype dtype, void* xp, cudaStream_t s);

size_t priority_scratch_bytes(int T);
// Stable argsort of the tokens by descending slot-0 gate into order[T].
cudaError_t launch_priority_order(const float* gate, int T, int k, int32_t* order, void* scratch,
                                  cudaStream_t s);

// Expert-choice routing (expert_choice.cu).  n = tokens each expert takes,
// npad = n rounded up to the 128-row block.
size_t ec_select_scratch_bytes(int T, int E);
cudaError_t launch_ec_select(const float* scores, int T, int E, int n, int npad, void* scratch,
                             int32_t* tok, int32_t* pos, int32_t* kept_counts, int32_t* offsets,
                             cudaStream_t s);
// o [rows, d] in the layer dtype (bf16 or fp32).
cudaError_t launch_ec_combine(const void* o, const int32_t* pos, const float* scores, int T,
                              int d, int E, moe_dtype dtype, void* y, cudaStream_t s);

struct FfnArgs {
  const void* xp;
  int64_t rows;
  const int32_t* offsets;
  const int32_t* kept_counts;
  const void* W1;
  const void* W3;
  const void* W2;
  int E, d, H;
  moe_act act;
  void* h;
  void* o;  // [rows, d] in the layer dtype
  int32_t* dev_error;
};
// `between` (may be null) is recorded on the stream after the up projection.
moe_status launch_ffn_tc(const FfnArgs& a, cudaStream_t s, int num_sms,
                         cudaEvent_t between);                                  // bf16, tcgen05
moe_status launch_ffn_simt(const FfnArgs& a, cudaStream_t s, cudaEvent_t between);  // fp32

struct CombineArgs {
  const void* o;  // [rows, d] in the layer dtype
  const int32_t* pos;
  const float* gate;
  int T, d, k;
  void* y;
};
cudaError_t launch_combine(const CombineArgs& a, moe_dtype dtype, cudaStream_t s);

// Measurement aid (probe.cu): read `bytes` (a multiple of 16) of `buf` once
// with streaming 16-byte loads; one XOR word per warp lands in *sink.
cudaError_t launch_stream_read(const void* buf, size_t bytes, uint32_t* sink, int num_sms,
                               cudaStream_t s);

}  // namespace moe
