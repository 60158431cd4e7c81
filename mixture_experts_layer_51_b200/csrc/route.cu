// Router: logits = x . W_g (+ bias), then TopK and the softmax over the k
// selected logits, fused into one kernel per dtype.
//
// Pages: "How do Mixture of Expert Models Work?", "The Math Behind MoEs"
// (G(x) = Softmax(TopK(x . W_g))); "[Paper Club] Upcycling Large Language
// Models into Mixture of Experts" (the router is one learnable matrix; the
// expert indices are the experts with the highest probability).  The OpenMoE
// issue "Some questions want to know" notes that routing built from many
// small kernels and one-hot vectors runs at low utilisation, which is why
// the GEMM, the selection and the softmax share one launch here and the
// logits never leave the chip.
//
// The router GEMM has N = E <= 64 columns: ~E flop per byte of x, far below
// the B200 ridge point, so the kernel is bound by reading x from HBM.  The bf16
// path uses warp-level mma.sync (m16n8k16, fp32 accumulate) only so the
// multiply-adds keep up with HBM at E = 32..64; x streams through a cp.async
// ring in shared memory.  The fp32 path uses plain fp32 FMA.

#include <float.h>
#include <math.h>
#include <stdlib.h>

#include "moe_internal.cuh"
#include "route_select.cuh"

namespace moe {
namespace {

constexpr int kRouteThreads = 128; // 4 warps: (BM/16) token tiles x (4 / (BM/16)) K groups

// Shared-memory row strides (bf16 elements), padded so ldmatrix rows fall
// in different banks.
__host__ __device__ constexpr int x_stride(int BK) { return BK + 8; }
__host__ __device__ constexpr int wg_stride(int NT) { return NT * 8 + 8; }
__host__ __device__ constexpr int stage_bytes(int NT, int BM, int BK) {
  return BM * x_stride(BK) * 2 + BK * wg_stride(NT) * 2;
}

// TopK over one token's E logits (descending; equal logits keep the lower
// expert first), then softmax over the k selected ones.  `get(e)` returns
// the logit of expert e.  The running top-(k+1) list lives in registers:
// each new logit bubbles down a fixed compare-and-swap chain; an entry moves
// in front of another when its logit is larger, or equal with a lower
// expert, so an entry pushed down keeps its place before an equal logit of
// a higher expert.
template <int KM, typename Get>
__device__ __forceinline__ void topk_softmax_store(Get get, int E, int k, int t, int32_t* idx,
                                                   float* gate, float* margin, int gating,
                                                   float gate_scale) {
  float tv[KM];
  int ti[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    tv[j] = -INFINITY;
    ti[j] = -1;
  }
  for (int e = 0; e < E; ++e) {
    float v = get(e);
    int ei = e;
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      // An unfilled slot (ti < 0) always takes the value, so -inf logits
      // are still ranked in expert order.
      if (ti[j] < 0 || v > tv[j] || (v == tv[j] && ei < ti[j])) {
        const float tvj = tv[j];
        const int tij = ti[j];
        tv[j] = v;
        ti[j] = ei;
        v = tvj;
        ei = tij;
        if (ei < 0) break;
      }
    }
  }
  const float m = tv[0];
  float w[KM];
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    w[j] = (j < k) ? expf(tv[j] - m) : 0.f;
    s += w[j];
  }
  if (gating == MOE_GATE_SOFTMAX_TOPK) {
    // Switch order: normalise by the softmax denominator over all E logits.
    s = 0.f;
    for (int e = 0; e < E; ++e) s += expf(get(e) - m);
  }
  const float inv = gate_scale / s;
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    if (j < k) {
      idx[(int64_t)t * k + j] = ti[j];
      gate[(int64_t)t * k + j] = w[j] * inv;
    }
  }
  if (margin) {
    float mg = INFINITY;
#pragma unroll
    for (int j = 1; j < KM; ++j)
      if (j == k && k < E) mg = tv[j - 1] - tv[j];
    margin[t] = mg;
  }
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16 router.  NT = ceil(E / 8) column tiles of 8 experts; a cluster of CL
// CTAs shares one tile of BM = 64 tokens and splits the hidden dimension d:
// CTA q multiplies its contiguous range of 128-wide K chunks.  Inside a CTA
// the 4 warps each own 16 tokens.  x and the matching W_g rows stream
// through a cp.async ring in shared memory.  After the K loop every CTA
// leaves its partial logits [BM][E] in shared memory, and CTA q sums, for
// its BM/CL tokens, the CL partials read through distributed shared memory
// in rank order (a fixed order: deterministic), adds the bias, and selects.
//
// Selection: the P = 128 / (BM/CL) threads of a token each keep the sorted
// top-(k+1) list of a contiguous range of experts (a compare-and-swap
// chain), then merge lists in a butterfly over the P threads: each round
// inserts the higher-index half's entries into the lower half's list, so
// equal logits keep the lower expert first and every thread ends with the
// same list -- the stable descending order.
template <int NT, int BM, int BK, int STAGES, int CL, int KM>
__global__ void __launch_bounds__(kRouteThreads)
    route_bf16_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ Wg,
                      const float* __restrict__ bias, int T, int d, int E, int k,
                      int32_t* __restrict__ idx, float* __restrict__ gate,
                      float* __restrict__ margin, int gating, float gate_scale,
                      float* __restrict__ scores) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int WS = wg_stride(NT);
  constexpr int XS = x_stride(BK);
  constexpr int SB = stage_bytes(NT, BM, BK);
  constexpr int CPR = BK / 8;        // 16-byte chunks per x row per stage
  static_assert(BM == 64, "four warps of 16 tokens");
  constexpr int TPC = BM / CL;       // tokens each CTA selects for
  constexpr int P = kRouteThreads / TPC;  // threads per token in the selection
  constexpr int LS = NT * 8 + 1;     // logit row stride (floats), conflict-free
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const uint32_t q = CL > 1 ? cluster_ctarank() : 0u;
  const int t0 = static_cast<int>(blockIdx.x / CL) * BM;
  const int nk_all = (d + BK - 1) / BK;
  const int kc_begin = static_cast<int>(q) * nk_all / CL;
  const int kc_end = (static_cast<int>(q) + 1) * nk_all / CL;
  const int nk = kc_end - kc_begin;
  const bool vec_wg = (E % 8) == 0;
  pdl_wait();
  pdl_trigger();

  auto x_tile = [&](int st) { return smem + st * SB; };
  auto w_tile = [&](int st) { return smem + st * SB + BM * XS * 2; };

  auto load_stage = [&](int st, int kc) {
    const int k0 = kc * BK;
    // x: BM rows x CPR chunks of 16 bytes (each row segment contiguous).
    for (int i = tid; i < BM * CPR; i += kRouteThreads) {
      const int r = i / CPR, c = i % CPR;
      const int t = t0 + r, col = k0 + c * 8;
      const bool ok = (t < T) && (col < d);
      const __nv_bfloat16* src = ok ? x + (int64_t)t * d + col : x;
      cp_async16(smem_u32(x_tile(st) + (r * XS + c * 8) * 2), src, ok ? 16 : 0);
    }
    // W_g rows k0 .. k0+BK-1, columns 0 .. NT*8-1 (zero beyond E and d).
    if (vec_wg) {
      const int cpr = E / 8;  // 16-byte chunks per W_g row
      for (int i = tid; i < BK * NT; i += kRouteThreads) {
        const int r = i / NT, c = i % NT;
        const int row = k0 + r;
        const bool ok = (row < d) && (c < cpr);
        const __nv_bfloat16* src = ok ? Wg + (int64_t)row * E + c * 8 : Wg;
        cp_async16(smem_u32(w_tile(st) + (r * WS + c * 8) * 2), src, ok ? 16 : 0);
      }
    } else {
      __nv_bfloat16* wt = reinterpret_cast<__nv_bfloat16*>(w_tile(st));
      for (int i = tid; i < BK * NT * 8; i += kRouteThreads) {
        const int r = i / (NT * 8), c = i % (NT * 8);
        const int row = k0 + r;
        wt[r * WS + c] = (row < d && c < E) ? Wg[(int64_t)row * E + c] : __float2bfloat16(0.f);
      }
    }
  };

  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[n][i] = 0.f;

#pragma unroll
  for (int st = 0; st < STAGES - 1; ++st) {
    if (st < nk) load_stage(st, kc_begin + st);
    cp_async_commit();
  }

  for (int kk_c = 0; kk_c < nk; ++kk_c) {
    cp_async_wait<STAGES - 2>();
    __syncthreads();
    const int st = kk_c % STAGES;
    const uint32_t xa = smem_u32(x_tile(st));
    const uint32_t wa = smem_u32(w_tile(st));
#pragma unroll
    for (int kk = 0; kk < BK / 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(xa + ((warp * 16 + (lane & 15)) * XS + kk * 16 + (lane >> 4) * 8) * 2, a0, a1, a2,
              a3);
#pragma unroll
      for (int n = 0; n + 1 < NT; n += 2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(wa + ((kk * 16 + (lane & 15)) * WS + n * 8 + (lane >> 4) * 8) * 2, b0, b1, b2,
                  b3);
        mma_bf16_16816(acc[n], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(acc[n + 1], a0, a1, a2, a3, b2, b3);
      }
      if (NT & 1) {
        uint32_t b0, b1;
        ldsm_x2_t(wa + ((kk * 16 + (lane & 15)) * WS + (NT - 1) * 8) * 2, b0, b1);
        mma_bf16_16816(acc[NT - 1], a0, a1, a2, a3, b0, b1);
      }
    }
    const int nxt = kk_c + STAGES - 1;
    if (nxt < nk) load_stage(nxt % STAGES, kc_begin + nxt);
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();

  // This CTA's partial logits [BM][LS] (reusing the ring).
  float* part = reinterpret_cast<float*>(smem);
  {
    const int r = warp * 16 + (lane >> 2);
    const int c = (lane & 3) * 2;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      part[r * LS + n * 8 + c] = acc[n][0];
      part[r * LS + n * 8 + c + 1] = acc[n][1];
      part[(r + 8) * LS + n * 8 + c] = acc[n][2];
      part[(r + 8) * LS + n * 8 + c + 1] = acc[n][3];
    }
  }
  if (CL > 1) cluster_sync(); else __syncthreads();

  // Logits of this CTA's TPC tokens: the CL partials summed in rank order.
  float* fin = part + BM * LS;              // [TPC][LS]
  for (int i = tid; i < TPC * E; i += kRouteThreads) {
    const int rr = i / E, e = i - rr * E;
    const int r = static_cast<int>(q) * TPC + rr;
    float v;
    if (CL > 1) {
      const uint32_t a = smem_u32(&part[r * LS + e]);
      v = 0.f;
#pragma unroll
      for (int c = 0; c < CL; ++c) v += __uint_as_float(ld_shared_cluster_u32(mapa_shared(a, c)));
    } else {
      v = part[r * LS + e];
    }
    fin[rr * LS + e] = bias ? v + bias[e] : v;
  }
  // Every CTA has read the partials it needs before any CTA moves on.
  if (CL > 1) cluster_sync(); else __syncthreads();

  const int rr = tid / P, p = tid % P;
  const int t = t0 + static_cast<int>(q) * TPC + rr;
  const float* lrow = fin + rr * LS;
  if (scores) {
    // Expert-choice affinities: softmax over all E logits.
    float m, inv;
    softmax_stats(lrow, E, P, p, m, inv);
    // Expert-major output scores[e, t]: the tile is written with consecutive
    // threads on consecutive tokens, each value recomputed from the same
    // logit, maximum and reciprocal as the sum used.
    float* rowstat = fin + TPC * LS;  // [TPC][2]: max, 1/sum
    if (p == 0) {
      rowstat[2 * rr] = m;
      rowstat[2 * rr + 1] = inv;
    }
    __syncthreads();
    const int t_base = t0 + static_cast<int>(q) * TPC;
    for (int i = tid; i < TPC * E; i += kRouteThreads) {
      const int e = i / TPC, r2 = i - e * TPC;
      if (t_base + r2 < T)
        scores[(int64_t)e * T + t_base + r2] =
            expf(fin[r2 * LS + e] - rowstat[2 * r2]) * rowstat[2 * r2 + 1];
    }
    return;
  }
  select_token<KM>(lrow, E, k, P, p, t, t < T, gating, gate_scale, idx, gate, margin, nullptr);
}

// fp32 router: one warp per token; 8 experts at a time, each lane strides d,
// then a butterfly reduction (same order in every lane, deterministic).
__global__ void __launch_bounds__(256)
    route_fp32_kernel(const float* __restrict__ x, const float* __restrict__ Wg,
                      const float* __restrict__ bias, int T, int d, int E, int k,
                      int32_t* __restrict__ idx, float* __restrict__ gate,
                      float* __restrict__ margin, int gating, float gate_scale,
                      float* __restrict__ scores, int32_t* __restrict__ lrank,
                      int32_t* __restrict__ hist) {
  __shared__ float lg[8][kMaxE];
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t < T) {
    const float* xr = x + (int64_t)t * d;
    for (int e0 = 0; e0 < E; e0 += 8) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      for (int c = lane; c < d; c += 32) {
        const float xv = xr[c];
        const float* w = Wg + (int64_t)c * E + e0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (e0 + i < E) acc[i] = fmaf(xv, w[i], acc[i]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
      }
      if (lane == 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (e0 + i < E) lg[warp][e0 + i] = acc[i];
      }
    }
    __syncwarp();
    auto get = [&](int e) { return bias ? lg[warp][e] + bias[e] : lg[warp][e]; };
    if (scores) {
      // Expert-choice affinities (softmax over all E), same order of
      // operations in every lane.
      float m = -INFINITY;
      for (int e = 0; e < E; ++e) m = fmaxf(m, get(e));
      float sum = 0.f;
      for (int e = 0; e < E; ++e) sum += expf(get(e) - m);
      const float inv = 1.f / sum;
      for (int e = lane; e < E; e += 32) scores[(int64_t)e * T + t] = expf(get(e) - m) * inv;
    } else if (lane == 0) {
      topk_softmax_store<kMaxK + 1>(get, E, k, t, idx, gate, margin, gating, gate_scale);
    }
  }
  if (!lrank) return;
  // The counting half of the permutation, when this block's 8 tokens are one
  // token range: each assignment's rank among the block's earlier ones to
  // the same expert (-1 for an expert outside [0, E)), and the block's
  // assignments per expert.  (idx, written above by other warps, is visible
  // to the block after the barrier.)
  __syncthreads();
  const int t0 = blockIdx.x * 8, n = min(8, T - t0);
  const int tid = threadIdx.x;
  if (tid < n) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(int64_t)(t0 + tid) * k + j];
      int r = -1;
      if (e >= 0 && e < E) {
        r = 0;
        for (int q = 0; q < tid * k; ++q) r += idx[(int64_t)t0 * k + q] == e;
      }
      lrank[(int64_t)(t0 + tid) * k + j] = r;
    }
  }
  if (tid < E) {
    int c = 0;
    for (int q = 0; q < n * k; ++q) c += idx[(int64_t)t0 * k + q] == tid;
    hist[(int64_t)blockIdx.x * E + tid] = c;
  }
}

template <int NT, int BM, int BK, int STAGES, int CL, int KM>
cudaError_t launch_route_cfg(const RouteArgs& a, cudaStream_t s) {
  constexpr int smem = STAGES * stage_bytes(NT, BM, BK);
  constexpr int TPC = BM / CL;
  static_assert((BM + TPC) * (NT * 8 + 1) * 4 + TPC * 8 <= smem, "epilogue buffers");
  auto kern = route_bf16_kernel<NT, BM, BK, STAGES, CL, KM>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  return launch_kernel(kern, dim3(((a.T + BM - 1) / BM) * CL), dim3(kRouteThreads), smem, s, CL,
                       true, static_cast<const __nv_bfloat16*>(a.x),
                       static_cast<const __nv_bfloat16*>(a.Wg), a.bias, a.T, a.d, a.E, a.k, a.idx,
                       a.gate, a.margin, a.gating, a.gate_scale, a.scores);
}

// CTAs per token tile: the largest of 1, 2, 4 that keeps the grid within
// about two CTAs per SM and gives every CTA at least four 128-wide K chunks
// (a sweep on the B200: the 8192 x 4096 router is fastest with pairs, the
// 16384 x 2048 one with single CTAs).  MOE_ROUTE_CL (1, 2 or 4) overrides
// the choice, for measurements.
int route_cluster_size(int T, int d) {
  static const int forced = [] {
    const char* v = getenv("MOE_ROUTE_CL");
    return v ? atoi(v) : 0;
  }();
  if (forced == 1 || forced == 2 || forced == 4) return forced;
  const int tiles = (T + 63) / 64;
  const int chunks = (d + 127) / 128;
  int cl = 1;
  while (cl < 4 && tiles * cl * 2 <= 2 * 148 && chunks >= 8 * cl) cl *= 2;
  return cl;
}

template <int NT, int KM>
cudaError_t launch_route_nt(const RouteArgs& a, cudaStream_t s) {
  constexpr int ST = NT <= 2 ? 4 : 3;
  switch (route_cluster_size(a.T, a.d)) {
    case 4: return launch_route_cfg<NT, 64, 128, ST, 4, KM>(a, s);
    case 2: return launch_route_cfg<NT, 64, 128, ST, 2, KM>(a, s);
    default: return launch_route_cfg<NT, 64, 128, ST, 1, KM>(a, s);
  }
}

template <int KM>
cudaError_t launch_route_km(const RouteArgs& a, cudaStream_t s) {
  switch ((a.E + 7) / 8) {
    case 1: return launch_route_nt<1, KM>(a, s);
    case 2: return launch_route_nt<2, KM>(a, s);
    case 3: return launch_route_nt<3, KM>(a, s);
    case 4: return launch_route_nt<4, KM>(a, s);
    case 5: return launch_route_nt<5, KM>(a, s);
    case 6: return launch_route_nt<6, KM>(a, s);
    case 7: return launch_route_nt<7, KM>(a, s);
    default: return launch_route_nt<8, KM>(a, s);
  }
}

// KM = length of the running top lists (k + 1, rounded up to 3, 5 or 9);
// the affinity output uses none.
cudaError_t launch_route_bf16(const RouteArgs& a, cudaStream_t s) {
  if (a.scores || a.k <= 2) return launch_route_km<3>(a, s);
  if (a.k <= 4) return launch_route_km<5>(a, s);
  return launch_route_km<kMaxK + 1>(a, s);
}

}  // namespace

cudaError_t launch_route(const RouteArgs& a, moe_dtype dtype, cudaStream_t s, int num_sms,
                         bool* ranked) {
  if (ranked) *ranked = false;
  if (a.T == 0) return cudaSuccess;
  if (dtype == MOE_FP32) {
    // The blocks of 8 tokens are the permutation's token ranges when there
    // are at most as many groups of 8 as ranges: then the router also counts.
    const RouteRanges rg = route_ranges(a.T, num_sms);
    const bool count = a.lrank && a.hist && !a.scores && rg.G == rg.T8;
    const cudaError_t err = launch_kernel(
        route_fp32_kernel, dim3((a.T + 7) / 8), dim3(256), 0, s, 1, true,
        static_cast<const float*>(a.x), static_cast<const float*>(a.Wg), a.bias, a.T, a.d, a.E,
        a.k, a.idx, a.gate, a.margin, a.gating, a.gate_scale, a.scores,
        count ? a.lrank : nullptr, count ? a.hist : nullptr);
    if (ranked) *ranked = err == cudaSuccess && count;
    return err;
  }
  if (route_stream_supported(a)) {
    const cudaError_t err = launch_route_stream(a, num_sms, s);
    if (err != cudaErrorInvalidValue) {
      if (ranked) *ranked = err == cudaSuccess && a.lrank && a.hist;
      return err;  // else: no tensor map, fall through
    }
  }
  if (route_tc_supported(a)) {
    const cudaError_t err = launch_route_tc(a, s);
    if (err != cudaErrorInvalidValue) return err;  // else: no tensor map, use mma.sync
  }
  return launch_route_bf16(a, s);
}

}  // namespace moe
