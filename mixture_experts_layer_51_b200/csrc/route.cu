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

#include "moe_internal.cuh"

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
// each new logit bubbles down a fixed compare-and-swap chain, and a strict
// comparison leaves an equal earlier (lower-index) entry in front.
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
      if (v > tv[j] || ti[j] < 0) {
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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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

// bf16 router.  NT = ceil(E / 8) column tiles of 8 experts; BM tokens per
// CTA.  The 4 warps split the work as (BM/16) token tiles x KG K-groups:
// inside each 64-wide K stage, K-group g takes the 16-wide steps g, g+KG, ...
// The KG partial sums of a token tile are added in a fixed order at the end.
template <int NT, int BM, int BK, int STAGES, int KM>
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
  constexpr int MT = BM / 16;        // token tiles per CTA
  constexpr int KG = 4 / MT;         // K groups
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int mt = warp % MT, kg = warp / MT;
  const int t0 = blockIdx.x * BM;
  const int nk = (d + BK - 1) / BK;
  const bool vec_wg = (E % 8) == 0;

  auto x_tile = [&](int s) { return smem + s * SB; };
  auto w_tile = [&](int s) { return smem + s * SB + BM * XS * 2; };

  auto load_stage = [&](int s, int kc) {
    const int k0 = kc * BK;
    // x: BM rows x CPR chunks of 16 bytes (each row segment contiguous).
    for (int i = tid; i < BM * CPR; i += kRouteThreads) {
      const int r = i / CPR, c = i % CPR;
      const int t = t0 + r, col = k0 + c * 8;
      const bool ok = (t < T) && (col < d);
      const __nv_bfloat16* src = ok ? x + (int64_t)t * d + col : x;
      cp_async16(smem_u32(x_tile(s) + (r * XS + c * 8) * 2), src, ok ? 16 : 0);
    }
    // W_g rows k0 .. k0+BK-1, columns 0 .. NT*8-1 (zero beyond E and d).
    if (vec_wg) {
      const int cpr = E / 8;  // 16-byte chunks per W_g row
      for (int i = tid; i < BK * NT; i += kRouteThreads) {
        const int r = i / NT, c = i % NT;
        const int row = k0 + r;
        const bool ok = (row < d) && (c < cpr);
        const __nv_bfloat16* src = ok ? Wg + (int64_t)row * E + c * 8 : Wg;
        cp_async16(smem_u32(w_tile(s) + (r * WS + c * 8) * 2), src, ok ? 16 : 0);
      }
    } else {
      __nv_bfloat16* wt = reinterpret_cast<__nv_bfloat16*>(w_tile(s));
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
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < nk) load_stage(s, s);
    cp_async_commit();
  }

  for (int kc = 0; kc < nk; ++kc) {
    cp_async_wait<STAGES - 2>();
    __syncthreads();
    const int s = kc % STAGES;
    const uint32_t xa = smem_u32(x_tile(s));
    const uint32_t wa = smem_u32(w_tile(s));
#pragma unroll
    for (int kk = kg; kk < BK / 16; kk += KG) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(xa + ((mt * 16 + (lane & 15)) * XS + kk * 16 + (lane >> 4) * 8) * 2, a0, a1, a2,
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
    const int nxt = kc + STAGES - 1;
    if (nxt < nk) load_stage(nxt % STAGES, nxt);
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();

  // Partial logits to shared memory: [KG][BM][NT*8 + 1] fp32 (reuses the ring),
  // then each token's KG partials are added in group order.
  float* lg = reinterpret_cast<float*>(smem);
  constexpr int LS = NT * 8 + 1;
  {
    float* part = lg + kg * BM * LS;
    const int r = mt * 16 + (lane >> 2);
    const int c = (lane & 3) * 2;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      part[r * LS + n * 8 + c] = acc[n][0];
      part[r * LS + n * 8 + c + 1] = acc[n][1];
      part[(r + 8) * LS + n * 8 + c] = acc[n][2];
      part[(r + 8) * LS + n * 8 + c + 1] = acc[n][3];
    }
  }
  __syncthreads();
  auto logit = [&](int r, int e) {
    float v = lg[r * LS + e];
#pragma unroll
    for (int g = 1; g < KG; ++g) v += lg[(g * BM + r) * LS + e];
    return bias ? v + bias[e] : v;
  };
  if (scores) {
    // Expert-choice affinities: the softmax over all E logits of every
    // token, written as rows of [T, E].  One thread per token finds the
    // maximum and the denominator; then the whole CTA writes the BM x E
    // tile in index order (coalesced), each value recomputed from the same
    // logit and maximum, so it equals the term that entered the sum.
    float* rowstat = lg + KG * BM * LS;  // [BM][2]: max, 1/sum
    if (tid < BM) {
      float m = -INFINITY;
      for (int e = 0; e < E; ++e) m = fmaxf(m, logit(tid, e));
      float sum = 0.f;
      for (int e = 0; e < E; ++e) sum += expf(logit(tid, e) - m);
      rowstat[2 * tid] = m;
      rowstat[2 * tid + 1] = 1.f / sum;
    }
    __syncthreads();
    const int nrow = min(BM, T - t0);
    for (int i = tid; i < nrow * E; i += kRouteThreads) {
      const int r = i / E, e = i - r * E;
      scores[(int64_t)t0 * E + i] = expf(logit(r, e) - rowstat[2 * r]) * rowstat[2 * r + 1];
    }
    return;
  }
  if (tid < BM) {
    const int t = t0 + tid;
    if (t < T) {
      auto get = [&](int e) { return logit(tid, e); };
      topk_softmax_store<KM>(get, E, k, t, idx, gate, margin, gating, gate_scale);
    }
  }
}

// fp32 router: one warp per token; 8 experts at a time, each lane strides d,
// then a butterfly reduction (same order in every lane, deterministic).
__global__ void __launch_bounds__(256)
    route_fp32_kernel(const float* __restrict__ x, const float* __restrict__ Wg,
                      const float* __restrict__ bias, int T, int d, int E, int k,
                      int32_t* __restrict__ idx, float* __restrict__ gate,
                      float* __restrict__ margin, int gating, float gate_scale,
                      float* __restrict__ scores) {
  __shared__ float lg[8][kMaxE];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
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
    for (int e = lane; e < E; e += 32) scores[(int64_t)t * E + e] = expf(get(e) - m) * inv;
    return;
  }
  if (lane == 0) topk_softmax_store<kMaxK + 1>(get, E, k, t, idx, gate, margin, gating, gate_scale);
}

template <int NT, int BM, int BK, int STAGES, int KM>
cudaError_t launch_route_cfg(const RouteArgs& a, cudaStream_t s) {
  constexpr int smem = STAGES * stage_bytes(NT, BM, BK);
  static_assert(BM * (NT * 8 + 1) * 4 * (4 / (BM / 16)) + BM * 8 <= smem, "epilogue buffer");
  cudaError_t err = cudaFuncSetAttribute(route_bf16_kernel<NT, BM, BK, STAGES, KM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  const int grid = (a.T + BM - 1) / BM;
  route_bf16_kernel<NT, BM, BK, STAGES, KM><<<grid, kRouteThreads, smem, s>>>(
      static_cast<const __nv_bfloat16*>(a.x), static_cast<const __nv_bfloat16*>(a.Wg), a.bias, a.T,
      a.d, a.E, a.k, a.idx, a.gate, a.margin, a.gating, a.gate_scale, a.scores);
  return cudaGetLastError();
}

// Configurations chosen by a sweep on B200 (8192 x 4096, E = 8 and
// 16384 x 2048, E = 64): 64-token tiles with 128-wide K stages were fastest,
// because each stage re-streams a W_g chunk from L2 and larger token tiles
// amortise it; fewer, longer-lived CTAs beat finer tiles here.
template <int NT, int KM>
cudaError_t launch_route_nt(const RouteArgs& a, cudaStream_t s) {
  if (NT <= 2) return launch_route_cfg<NT, 64, 128, 4, KM>(a, s);
  return launch_route_cfg<NT, 64, 128, 3, KM>(a, s);
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

}  // namespace

cudaError_t launch_route(const RouteArgs& a, moe_dtype dtype, cudaStream_t s, int /*num_sms*/) {
  if (a.T == 0) return cudaSuccess;
  if (dtype == MOE_FP32) {
    route_fp32_kernel<<<(a.T + 7) / 8, 256, 0, s>>>(static_cast<const float*>(a.x),
                                                    static_cast<const float*>(a.Wg), a.bias, a.T,
                                                    a.d, a.E, a.k, a.idx, a.gate, a.margin,
                                                    a.gating, a.gate_scale, a.scores);
    return cudaGetLastError();
  }
  // KM = slots of the running top list (k + 1, rounded up to 3, 5 or 9);
  // the affinity output uses no list.
  if (a.scores || a.k <= 2) return launch_route_km<3>(a, s);
  if (a.k <= 4) return launch_route_km<5>(a, s);
  return launch_route_km<kMaxK + 1>(a, s);
}

}  // namespace moe
