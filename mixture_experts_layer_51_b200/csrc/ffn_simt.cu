// Grouped expert FFN in fp32 on the CUDA cores (the fp32 layer: tf32 tensor
// cores would not hold a 1e-5 relative error).
//
// Pages: "[Paper Club] Upcycling Large Language Models into Mixture of
// Experts" (each expert is the original two-layer FFN; all experts run as one
// grouped operation over their token blocks) and "How do Mixture of Expert
// Models Work?", "The Math Behind MoEs" (SwiGLU experts).
//
// One 64x64 output tile per CTA, 256 threads with a 4x4 micro-tile each,
// 32-deep K slabs copied into a 4-stage shared-memory ring with cp.async, so
// up to three slabs are in flight while one is multiplied (these layers are
// small -- a few slabs per tile -- and the memory latency is most of the
// time: every slab of a K <= 96 tile is requested at once).  The expert of a
// tile is found from the offsets staged in shared memory by one parallel
// read.  Expert blocks start on multiples of 128 rows, so a 64-row tile
// never straddles two experts; tiles made only of padding rows exit at once.

#include <math.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int BM = 64, BN = 64, BK = 32;
constexpr int kThreads = 256;
constexpr int kStages = 4;
constexpr int kAStride = BK + 4;  // floats per A row in shared memory (padded)
constexpr int kAFloats = BM * kAStride;
constexpr int kBFloats = BK * BN;

template <int MODE>
__host__ __device__ constexpr int stage_floats() {
  return kAFloats + kBFloats * (MODE == 1 ? 2 : 1);
}
template <int MODE>
__host__ __device__ constexpr int smem_bytes() {
  return kStages * stage_floats<MODE>() * 4;
}

__device__ __forceinline__ float gelu_erf(float z) {
  return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
}
__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

// MODE 0: out = A W (plain);  MODE 1: out = SiLU(A W) * (A W3);  MODE 2: out = GELU(A W).
// K and N are multiples of 8 (so every 16-byte copy lies inside a row) and
// A, W, W3 are 16-byte aligned.
template <int MODE>
__global__ void __launch_bounds__(kThreads)
    ffn_simt_kernel(const float* __restrict__ A, const int32_t* __restrict__ offsets,
                    const int32_t* __restrict__ kept, int E, const float* __restrict__ W,
                    const float* __restrict__ W3, float* __restrict__ out, int K, int N) {
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  __shared__ int s_off[kMaxE + 1], s_kept[kMaxE];
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x;
  if (tid <= E) s_off[tid] = offsets[tid];
  if (tid < E) s_kept[tid] = kept[tid];
  __syncthreads();
  const int r0 = blockIdx.x * BM;
  const int n0 = blockIdx.y * BN;
  if (r0 >= s_off[E]) return;
  int e = 0;
  while (e + 1 < E && s_off[e + 1] <= r0) ++e;
  const int valid = s_kept[e] - (r0 - s_off[e]);  // rows of this tile that are real
  if (valid <= 0) return;
  const float* We = W + (int64_t)e * K * N;
  const float* W3e = MODE == 1 ? W3 + (int64_t)e * K * N : nullptr;
  const int tr = tid / 16, tc = tid % 16;  // 16 x 16 threads, 4 x 4 outputs each
  const int nk = (K + BK - 1) / BK;
  // Slab kb into stage kb % kStages: A rows past `valid` and columns past K,
  // and weight rows past K or columns past N, are zero-filled.
  auto issue = [&](int kb) {
    float* As = sm + (kb % kStages) * stage_floats<MODE>();
    float* Bs = As + kAFloats;
    const int k0 = kb * BK;
#pragma unroll
    for (int q = 0; q < BM * BK / 4 / kThreads; ++q) {
      const int i = tid + q * kThreads;
      const int r = i / (BK / 4), c = (i % (BK / 4)) * 4;
      const bool ok = r < valid && k0 + c < K;
      cp_async16(smem_u32(As + r * kAStride + c), ok ? A + (int64_t)(r0 + r) * K + k0 + c : A,
                 ok ? 16 : 0);
    }
#pragma unroll
    for (int q = 0; q < BK * BN / 4 / kThreads; ++q) {
      const int i = tid + q * kThreads;
      const int r = i / (BN / 4), c = (i % (BN / 4)) * 4;
      const bool ok = k0 + r < K && n0 + c < N;
      const int64_t off = (int64_t)(k0 + r) * N + n0 + c;
      cp_async16(smem_u32(Bs + r * BN + c), ok ? We + off : We, ok ? 16 : 0);
      if (MODE == 1) cp_async16(smem_u32(Bs + kBFloats + r * BN + c), ok ? W3e + off : W3e, ok ? 16 : 0);
    }
  };
#pragma unroll
  for (int st = 0; st < kStages - 1; ++st) {
    if (st < nk) issue(st);
    cp_async_commit();
  }
  float acc[4][4] = {};
  float acc3[4][4] = {};
  for (int kb = 0; kb < nk; ++kb) {
    cp_async_wait<kStages - 2>();  // slab kb has landed (this thread's copies)
    __syncthreads();               // ... and everyone's; stage (kb - 1) % kStages is free
    if (kb + kStages - 1 < nk) issue(kb + kStages - 1);
    cp_async_commit();
    const float* As = sm + (kb % kStages) * stage_floats<MODE>();
    const float* Bs = As + kAFloats;
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[(tr * 4 + i) * kAStride + kk];
      const float4 b = *reinterpret_cast<const float4*>(Bs + kk * BN + tc * 4);
      const float bv[4] = {b.x, b.y, b.z, b.w};
      float b3v[4] = {0.f, 0.f, 0.f, 0.f};
      if (MODE == 1) {
        const float4 b3 = *reinterpret_cast<const float4*>(Bs + kBFloats + kk * BN + tc * 4);
        b3v[0] = b3.x;
        b3v[1] = b3.y;
        b3v[2] = b3.z;
        b3v[3] = b3.w;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(a[i], bv[j], acc[i][j]);
          if (MODE == 1) acc3[i][j] = fmaf(a[i], b3v[j], acc3[i][j]);
        }
    }
  }
  cp_async_wait<0>();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = tr * 4 + i;
    if (r >= valid) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tc * 4 + j;
      if (c >= N) continue;
      float v = acc[i][j];
      if (MODE == 1) v = silu(v) * acc3[i][j];
      if (MODE == 2) v = gelu_erf(v);
      out[(int64_t)(r0 + r) * N + c] = v;
    }
  }
}

template <int MODE>
cudaError_t launch_simt(dim3 grid, cudaStream_t s, const float* A, const FfnArgs& a,
                        const float* W, const float* W3, float* out, int K, int N) {
  static const cudaError_t attr = cudaFuncSetAttribute(
      ffn_simt_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes<MODE>());
  if (attr != cudaSuccess) return attr;
  return launch_kernel(ffn_simt_kernel<MODE>, grid, dim3(kThreads), smem_bytes<MODE>(), s, 1, true,
                       A, a.offsets, a.kept_counts, a.E, W, W3, out, K, N);
}

}  // namespace

moe_status launch_ffn_simt(const FfnArgs& a, cudaStream_t s, cudaEvent_t between) {
  const int row_tiles = static_cast<int>((a.rows + BM - 1) / BM);
  if (row_tiles == 0) return MOE_OK;
  const float* xp = static_cast<const float*>(a.xp);
  float* h = static_cast<float*>(a.h);
  const float* W1 = static_cast<const float*>(a.W1);
  const float* W3 = static_cast<const float*>(a.W3);
  const float* W2 = static_cast<const float*>(a.W2);
  const float* no_w = nullptr;
  const dim3 g1(row_tiles, (a.H + BN - 1) / BN);
  cudaError_t err = a.act == MOE_SWIGLU
                        ? launch_simt<1>(g1, s, xp, a, W1, W3, h, a.d, a.H)
                        : launch_simt<2>(g1, s, xp, a, W1, no_w, h, a.d, a.H);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  if (between && cudaEventRecord(between, s) != cudaSuccess) return MOE_ERR_CUDA;
  const dim3 g2(row_tiles, (a.d + BN - 1) / BN);
  err = launch_simt<0>(g2, s, h, a, W2, no_w, static_cast<float*>(a.o), a.H, a.d);
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
