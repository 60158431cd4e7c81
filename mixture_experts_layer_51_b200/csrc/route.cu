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

constexpr int kRouteBM = 32;      // tokens per CTA
constexpr int kRouteBK = 64;      // K (= d) per pipeline stage
constexpr int kRouteStages = 6;
constexpr int kRouteThreads = 64; // 2 warps x 16 tokens
constexpr int kXStride = kRouteBK + 8;  // bf16 elements per smem row of x (pad: no bank conflicts)

__host__ __device__ constexpr int wg_stride(int NT) { return NT * 8 + 8; }
__host__ __device__ constexpr int stage_bytes(int NT) {
  return kRouteBM * kXStride * 2 + kRouteBK * wg_stride(NT) * 2;
}

// TopK over one token's E logits (descending; equal logits keep the lower
// expert first), then softmax over the k selected ones.  `get(e)` returns
// the logit of expert e.
template <typename Get>
__device__ __forceinline__ void topk_softmax_store(Get get, int E, int k, int t, int32_t* idx,
                                                   float* gate, float* margin) {
  float tv[kMaxK + 1];
  int ti[kMaxK + 1];
  const int keep = (k + 1 < E) ? k + 1 : E;  // also track the (k+1)-th for the margin
  int n = 0;
  for (int e = 0; e < E; ++e) {
    const float v = get(e);
    if (n < keep || v > tv[n - 1]) {
      int p = (n < keep) ? n : n - 1;
      while (p > 0 && tv[p - 1] < v) {
        tv[p] = tv[p - 1];
        ti[p] = ti[p - 1];
        --p;
      }
      tv[p] = v;
      ti[p] = e;
      if (n < keep) ++n;
    }
  }
  const float m = tv[0];
  float w[kMaxK];
  float s = 0.f;
  for (int j = 0; j < k; ++j) {
    w[j] = expf(tv[j] - m);
    s += w[j];
  }
  const float inv = 1.0f / s;
  for (int j = 0; j < k; ++j) {
    idx[(int64_t)t * k + j] = ti[j];
    gate[(int64_t)t * k + j] = w[j] * inv;
  }
  if (margin) margin[t] = (k < E) ? (tv[k - 1] - tv[k]) : INFINITY;
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

// bf16 router.  NT = ceil(E / 8) column tiles of 8 experts.
template <int NT>
__global__ void __launch_bounds__(kRouteThreads)
    route_bf16_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ Wg,
                      const float* __restrict__ bias, int T, int d, int E, int k,
                      int32_t* __restrict__ idx, float* __restrict__ gate,
                      float* __restrict__ margin) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int WS = wg_stride(NT);
  constexpr int SB = stage_bytes(NT);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * kRouteBM;
  const int nk = (d + kRouteBK - 1) / kRouteBK;
  const bool vec_wg = (E % 8) == 0;

  auto x_tile = [&](int s) { return smem + s * SB; };
  auto w_tile = [&](int s) { return smem + s * SB + kRouteBM * kXStride * 2; };

  auto load_stage = [&](int s, int kc) {
    const int k0 = kc * kRouteBK;
    // x: kRouteBM rows x 8 chunks of 16 bytes.
    for (int i = tid; i < kRouteBM * 8; i += kRouteThreads) {
      const int r = i >> 3, c = i & 7;
      const int t = t0 + r, col = k0 + c * 8;
      const bool ok = (t < T) && (col < d);
      const __nv_bfloat16* src = ok ? x + (int64_t)t * d + col : x;
      cp_async16(smem_u32(x_tile(s) + (r * kXStride + c * 8) * 2), src, ok ? 16 : 0);
    }
    // W_g rows k0 .. k0+63, columns 0 .. NT*8-1 (zero beyond E and d).
    if (vec_wg) {
      const int cpr = E / 8;  // 16-byte chunks per W_g row
      for (int i = tid; i < kRouteBK * NT; i += kRouteThreads) {
        const int r = i / NT, c = i % NT;
        const int row = k0 + r;
        const bool ok = (row < d) && (c < cpr);
        const __nv_bfloat16* src = ok ? Wg + (int64_t)row * E + c * 8 : Wg;
        cp_async16(smem_u32(w_tile(s) + (r * WS + c * 8) * 2), src, ok ? 16 : 0);
      }
    } else {
      __nv_bfloat16* wt = reinterpret_cast<__nv_bfloat16*>(w_tile(s));
      for (int i = tid; i < kRouteBK * NT * 8; i += kRouteThreads) {
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
  for (int s = 0; s < kRouteStages - 1; ++s) {
    if (s < nk) load_stage(s, s);
    cp_async_commit();
  }

  for (int kc = 0; kc < nk; ++kc) {
    cp_async_wait<kRouteStages - 2>();
    __syncthreads();
    const int s = kc % kRouteStages;
    const uint32_t xa = smem_u32(x_tile(s));
    const uint32_t wa = smem_u32(w_tile(s));
#pragma unroll
    for (int kk = 0; kk < kRouteBK / 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(xa + ((warp * 16 + (lane & 15)) * kXStride + kk * 16 + (lane >> 4) * 8) * 2, a0, a1,
              a2, a3);
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
    const int nxt = kc + kRouteStages - 1;
    if (nxt < nk) load_stage(nxt % kRouteStages, nxt);
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();

  // Logits to shared memory: [kRouteBM][NT*8 + 1] fp32 (reuses the ring).
  float* lg = reinterpret_cast<float*>(smem);
  constexpr int LS = NT * 8 + 1;
  {
    const int r = warp * 16 + (lane >> 2);
    const int c = (lane & 3) * 2;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      lg[r * LS + n * 8 + c] = acc[n][0];
      lg[r * LS + n * 8 + c + 1] = acc[n][1];
      lg[(r + 8) * LS + n * 8 + c] = acc[n][2];
      lg[(r + 8) * LS + n * 8 + c + 1] = acc[n][3];
    }
  }
  __syncthreads();
  if (tid < kRouteBM) {
    const int t = t0 + tid;
    if (t < T) {
      const float* row = lg + tid * LS;
      auto get = [&](int e) { return bias ? row[e] + bias[e] : row[e]; };
      topk_softmax_store(get, E, k, t, idx, gate, margin);
    }
  }
}

// fp32 router: one warp per token; 8 experts at a time, each lane strides d,
// then a butterfly reduction (same order in every lane, deterministic).
__global__ void __launch_bounds__(256)
    route_fp32_kernel(const float* __restrict__ x, const float* __restrict__ Wg,
                      const float* __restrict__ bias, int T, int d, int E, int k,
                      int32_t* __restrict__ idx, float* __restrict__ gate,
                      float* __restrict__ margin) {
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
  if (lane == 0) {
    auto get = [&](int e) { return bias ? lg[warp][e] + bias[e] : lg[warp][e]; };
    topk_softmax_store(get, E, k, t, idx, gate, margin);
  }
}

template <int NT>
cudaError_t launch_route_nt(const RouteArgs& a, cudaStream_t s) {
  const int smem = kRouteStages * stage_bytes(NT);
  cudaError_t err =
      cudaFuncSetAttribute(route_bf16_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  const int grid = (a.T + kRouteBM - 1) / kRouteBM;
  route_bf16_kernel<NT><<<grid, kRouteThreads, smem, s>>>(
      static_cast<const __nv_bfloat16*>(a.x), static_cast<const __nv_bfloat16*>(a.Wg), a.bias, a.T,
      a.d, a.E, a.k, a.idx, a.gate, a.margin);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const RouteArgs& a, moe_dtype dtype, cudaStream_t s, int /*num_sms*/) {
  if (a.T == 0) return cudaSuccess;
  if (dtype == MOE_FP32) {
    route_fp32_kernel<<<(a.T + 7) / 8, 256, 0, s>>>(static_cast<const float*>(a.x),
                                                    static_cast<const float*>(a.Wg), a.bias, a.T,
                                                    a.d, a.E, a.k, a.idx, a.gate, a.margin);
    return cudaGetLastError();
  }
  switch ((a.E + 7) / 8) {
    case 1: return launch_route_nt<1>(a, s);
    case 2: return launch_route_nt<2>(a, s);
    case 3: return launch_route_nt<3>(a, s);
    case 4: return launch_route_nt<4>(a, s);
    case 5: return launch_route_nt<5>(a, s);
    case 6: return launch_route_nt<6>(a, s);
    case 7: return launch_route_nt<7>(a, s);
    default: return launch_route_nt<8>(a, s);
  }
}

}  // namespace moe
