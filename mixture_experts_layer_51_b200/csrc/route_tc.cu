// Router on the 5th-generation tensor cores: logits = x . W_g (+ bias) for a
// tile of 128 tokens, then TopK and the softmax (or, for expert choice, the
// softmax over all E) per token, in one kernel.
//
// Pages: "How do Mixture of Expert Models Work?", "The Math Behind MoEs"
// (G(x) = Softmax(TopK(x . W_g))); "[Paper Club] Upcycling Large Language
// Models into Mixture of Experts" (one learnable router matrix).
//
// The router reads every byte of x once and does ~E flop per byte, so it is
// bound by HBM; what matters is keeping enough bytes in flight.  Here one
// thread issues TMA loads of 128 x 64 tiles of x (128-byte swizzle) and of
// the matching 64 x 64 tile of W_g (its E columns, zero-filled to 64) into
// an 8-stage ring (192 KB in flight per SM), and one thread issues
// tcgen05.mma (M = 128 tokens, N = 64, K = 16, fp32 accumulate in tensor
// memory).  After the last K step each of the 128 threads reads its token's
// 64 accumulator columns (tcgen05.ld: TMEM lane = token) and selects in
// registers -- no shared-memory round trip for the logits.
//
// Used for bf16 when E % 8 == 0 (W_g's rows must be 16-byte multiples for
// TMA) and the batch is large (see route_tc_supported); route.cu's mma.sync
// kernel covers the rest.  Every wait is bounded;
// on time-out the kernel sets a bit in the error word (when one is given)
// and leaves.

#include <math.h>
#include <stdlib.h>

#include <cudaTypedefs.h>

#include <mutex>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kTM = 128;           // tokens per CTA (UMMA M)
constexpr int kTN = 64;            // accumulator columns (UMMA N; experts zero-padded)
constexpr int kTK = 64;            // K elements per stage (one 128-byte swizzle row)
constexpr int kStages = 8;
constexpr int kAStage = kTM * kTK * 2;   // 16 KB
constexpr int kBStage = kTK * kTN * 2;   // 8 KB
constexpr int kStageBytes = kAStage + kBStage;
constexpr int kThreads = 128;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*barriers*/ + 1024 /*alignment*/;
static_assert(kSmemBytes <= 232448, "shared memory");

struct RouteTcCtl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull;
  uint32_t tmem_base;
  int abort_flag;
};

template <int KM>
__device__ __forceinline__ void insert_sorted_tc(float (&tv)[KM], int (&ti)[KM], float v, int ei) {
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    // larger value, or equal value and lower expert (an entry pushed down
    // the list keeps its place in front of an equal logit of a higher one)
    const bool take = (ei >= 0) & ((ti[j] < 0) | (v > tv[j]) | ((v == tv[j]) & (ei < ti[j])));
    const float tvj = tv[j];
    const int tij = ti[j];
    tv[j] = take ? v : tvj;
    ti[j] = take ? ei : tij;
    v = take ? tvj : v;
    ei = take ? tij : ei;
  }
}

template <int KM>
__global__ void __launch_bounds__(kThreads, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    const float* __restrict__ bias, int T, int d, int E, int k,
                    int32_t* __restrict__ idx, float* __restrict__ gate,
                    float* __restrict__ margin, int gating, float gate_scale,
                    float* __restrict__ scores, int32_t* __restrict__ err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  RouteTcCtl& c = *reinterpret_cast<RouteTcCtl*>(smem + kStages * kStageBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * kTM;
  const int nk = (d + kTK - 1) / kTK;
  const uint32_t smem_base = smem_u32(smem);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&c.full[s]), 1);
      mbar_init(smem_u32(&c.empty[s]), 1);
    }
    mbar_init(smem_u32(&c.tfull), 1);
    c.abort_flag = 0;
    fence_mbar_init();
    fence_async_shared();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&c.tmem_base), kTN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  pdl_wait();  // x (and W_g) may come from the previous kernel in the stream

  bool timed_out = false;
  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    for (int kb = 0; kb < nk; ++kb) {
      if (!mbar_wait(smem_u32(&c.empty[stage]), phase ^ 1)) {
        timed_out = true;
        break;
      }
      const uint32_t full = smem_u32(&c.full[stage]);
      const uint32_t a_dst = smem_base + stage * kStageBytes;
      mbar_arrive_expect_tx(full, kStageBytes);
      tma_load_2d(a_dst, &tmX, full, kb * kTK, t0);
      tma_load_2d(a_dst + kAStage, &tmW, full, 0, kb * kTK);
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (timed_out) {
      c.abort_flag = 1;
      if (err) atomicOr(err, kErrTimeoutProducer);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(kTM, kTN, false, true);
    const uint64_t adesc0 = smem_desc_sw128(smem_base, 16, 1024);
    const uint64_t bdesc0 = smem_desc_sw128(smem_base + kAStage, kBStage, 1024);
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    for (int kb = 0; kb < nk; ++kb) {
      if (!mbar_wait(smem_u32(&c.full[stage]), phase)) {
        timed_out = true;
        break;
      }
      tc_fence_after();
      const uint64_t soff = static_cast<uint64_t>((stage * kStageBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < kTK / 16; ++kk) {
        // A: K-major, 16-element steps are 32 bytes inside the swizzled row;
        // B: N-major, 16 K-rows are 2 KB.
        const uint64_t adesc = adesc0 + soff + static_cast<uint64_t>((kk * 32) >> 4);
        const uint64_t bdesc = bdesc0 + soff + static_cast<uint64_t>((kk * 2048) >> 4);
        tc_mma_bf16(tmem, adesc, bdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
      }
      ++issued;
      tc_commit(smem_u32(&c.empty[stage]));
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1;
      }
    }
    // The accumulator is complete (or, after a time-out, every issued MMA
    // has landed) when this commit arrives.
    tc_commit(smem_u32(&c.tfull));
    if (timed_out) {
      c.abort_flag = 1;
      if (err) atomicOr(err, kErrTimeoutMma);
    }
    (void)issued;
  }

  // ---------------------------------------------------------- epilogue
  // Thread tid owns token t0 + tid = TMEM lane tid (warp w reads lanes
  // 32w .. 32w+31).
  const bool have = mbar_wait(smem_u32(&c.tfull), 0);
  tc_fence_after();
  float l[kTN];
  {
    float a[32], b[32];
    const uint32_t base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    tc_ld_32cols(base, a);
    tc_ld_32cols(base + 32, b);
    tc_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      l[i] = a[i];
      l[32 + i] = b[i];
    }
  }
  const int t = t0 + tid;
  const bool ok = have && !c.abort_flag;
  if (!have && err) atomicOr(err, kErrTimeoutEpilogue);
  if (ok && t < T) {
#pragma unroll
    for (int e = 0; e < kTN; ++e)
      if (e < E && bias) l[e] += bias[e];
    float m = -INFINITY;
#pragma unroll
    for (int e = 0; e < kTN; ++e)
      if (e < E) m = fmaxf(m, l[e]);
    if (scores) {
      // Expert-choice affinities, expert-major [E, T]: consecutive threads
      // write consecutive tokens.
      float sum = 0.f;
#pragma unroll
      for (int e = 0; e < kTN; ++e)
        if (e < E) sum += expf(l[e] - m);
      const float inv = 1.f / sum;
#pragma unroll
      for (int e = 0; e < kTN; ++e)
        if (e < E) scores[(int64_t)e * T + t] = expf(l[e] - m) * inv;
    } else {
      float tv[KM];
      int ti[KM];
#pragma unroll
      for (int j = 0; j < KM; ++j) {
        tv[j] = -INFINITY;
        ti[j] = -1;
      }
#pragma unroll
      for (int e = 0; e < kTN; ++e)
        if (e < E) insert_sorted_tc<KM>(tv, ti, l[e], e);
      float denom = 0.f;
      if (gating == MOE_GATE_SOFTMAX_TOPK) {
#pragma unroll
        for (int e = 0; e < kTN; ++e)
          if (e < E) denom += expf(l[e] - m);
      } else {
#pragma unroll
        for (int j = 0; j < KM; ++j)
          if (j < k) denom += expf(tv[j] - m);
      }
      const float inv = gate_scale / denom;
#pragma unroll
      for (int j = 0; j < KM; ++j) {
        if (j < k) {
          idx[(int64_t)t * k + j] = ti[j];
          gate[(int64_t)t * k + j] = expf(tv[j] - m) * inv;
        }
      }
      if (margin) {
        float mg = INFINITY;
#pragma unroll
        for (int j = 1; j < KM; ++j) {
          const float gap = tv[j - 1] - tv[j];
          mg = (j == k && k < E) ? gap : mg;
        }
        margin[t] = mg;
      }
    }
  }
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTN);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 route_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2-D bf16 matrix [rows, cols] (cols contiguous) with a box of box_cols x
// box_rows and 128-byte swizzle; boxes past the matrix read zeros.
bool route_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
               uint32_t box_rows) {
  auto fn = route_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KM>
cudaError_t launch_route_tc_km(const RouteArgs& a, const CUtensorMap& mx, const CUtensorMap& mw,
                               cudaStream_t s) {
  auto kern = route_tc_kernel<KM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, dim3((a.T + kTM - 1) / kTM), dim3(kThreads), kSmemBytes, s, 1, true,
                       mx, mw, a.bias, a.T, a.d, a.E, a.k, a.idx, a.gate, a.margin, a.gating,
                       a.gate_scale, a.scores, a.err);
}

}  // namespace

// Measured on the B200 against route.cu's mma.sync kernel: this kernel wins
// when the grid has at least ~128 tiles of 128 tokens and the per-token
// epilogue is light (the expert-choice affinities: 16384 x 2048, E = 64:
// 20 vs 31 us; top-2 of 32: 39 vs 41 us) and loses with fewer tiles (8192
// tokens: 55 vs 33 us) or a long TopK chain (top-8 of 64: 73 vs 59 us).
// MOE_ROUTE_TC=0 / 1 forces the choice (where the kernel applies).
bool route_tc_supported(const RouteArgs& a) {
  static const int forced = [] {
    const char* v = getenv("MOE_ROUTE_TC");
    return v ? (v[0] == '0' ? 0 : 1) : -1;
  }();
  if (!(a.E % 8 == 0 && a.E <= kTN && a.d % 8 == 0 && a.T > 0)) return false;
  if (forced >= 0) return forced == 1;
  const int tiles = (a.T + kTM - 1) / kTM;
  return tiles >= 128 && (a.scores != nullptr || a.k <= 2);
}

cudaError_t launch_route_tc(const RouteArgs& a, cudaStream_t s) {
  CUtensorMap mx, mw;
  // x [T, d]: 64 x 128 boxes; W_g [d, E]: 64 (experts, zero beyond E) x 64 boxes.
  if (!route_map(&mx, a.x, a.T, a.d, kTK, kTM) || !route_map(&mw, a.Wg, a.d, a.E, kTN, kTK))
    return cudaErrorInvalidValue;
  if (a.scores || a.k <= 2) return launch_route_tc_km<3>(a, mx, mw, s);
  if (a.k <= 4) return launch_route_tc_km<5>(a, mx, mw, s);
  return launch_route_tc_km<kMaxK + 1>(a, mx, mw, s);
}

}  // namespace moe
