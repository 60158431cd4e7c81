// Grouped expert FFN in fp32 on the CUDA cores (the fp32 layer: tf32 tensor
// cores would not hold a 1e-5 relative error).
//
// Pages: "[Paper Club] Upcycling Large Language Models into Mixture of
// Experts" (each expert is the original two-layer FFN; all experts run as one
// grouped operation over their token blocks) and "How do Mixture of Expert
// Models Work?", "The Math Behind MoEs" (SwiGLU experts).
//
// One 64x64 output tile per CTA, 256 threads with a 4x4 micro-tile each,
// 32-deep K slabs staged in shared memory, the next one prefetched into
// registers.  Expert blocks start on multiples
// of 128 rows, so a 64-row tile never straddles two experts; tiles made only
// of padding rows exit at once.

#include <math.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int BM = 64, BN = 64, BK = 32;
constexpr int kThreads = 256;
constexpr int kALoads = BM * BK / kThreads;  // elements of A each thread stages per slab
constexpr int kBLoads = BK * BN / kThreads;  // elements of each weight matrix

__device__ __forceinline__ int expert_of_row(const int32_t* offsets, int E, int row) {
  // offsets is ascending; E <= 64.
  int e = 0;
  while (e + 1 < E && offsets[e + 1] <= row) ++e;
  return e;
}

__device__ __forceinline__ float gelu_erf(float z) {
  return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
}
__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

// MODE 0: out = A W (plain);  MODE 1: out = SiLU(A W) * (A W3);  MODE 2: out = GELU(A W)
// The next K slab is loaded into registers while the current one is
// multiplied out of shared memory, so the global-load latency of a slab
// overlaps the FMAs of the one before (these layers are small: a few slabs
// per tile, and the latency is most of the time).
template <int MODE>
__global__ void __launch_bounds__(kThreads)
    ffn_simt_kernel(const float* __restrict__ A, const int32_t* __restrict__ offsets,
                    const int32_t* __restrict__ kept, int E, const float* __restrict__ W,
                    const float* __restrict__ W3, float* __restrict__ out, int K, int N) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN];
  __shared__ float B3s[MODE == 1 ? BK : 1][MODE == 1 ? BN : 1];
  pdl_wait();
  pdl_trigger();
  const int r0 = blockIdx.x * BM;
  const int n0 = blockIdx.y * BN;
  if (r0 >= offsets[E]) return;
  const int e = expert_of_row(offsets, E, r0);
  const int valid = kept[e] - (r0 - offsets[e]);  // rows of this tile that are real
  if (valid <= 0) return;
  const float* We = W + (int64_t)e * K * N;
  const float* W3e = MODE == 1 ? W3 + (int64_t)e * K * N : nullptr;
  const int tid = threadIdx.x;
  const int tr = tid / 16, tc = tid % 16;  // 16 x 16 threads, 4 x 4 outputs each
  float ra[kALoads], rb[kBLoads], rb3[MODE == 1 ? kBLoads : 1];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int q = 0; q < kALoads; ++q) {
      const int i = tid + q * kThreads;
      const int r = i / BK, c = i % BK;
      ra[q] = (r < valid && k0 + c < K) ? A[(int64_t)(r0 + r) * K + k0 + c] : 0.f;
    }
#pragma unroll
    for (int q = 0; q < kBLoads; ++q) {
      const int i = tid + q * kThreads;
      const int r = i / BN, c = i % BN;
      const bool ok = (k0 + r < K) && (n0 + c < N);
      rb[q] = ok ? We[(int64_t)(k0 + r) * N + n0 + c] : 0.f;
      if (MODE == 1) rb3[q] = ok ? W3e[(int64_t)(k0 + r) * N + n0 + c] : 0.f;
    }
  };
  float acc[4][4] = {};
  float acc3[4][4] = {};
  fetch(0);
  for (int k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
    for (int q = 0; q < kALoads; ++q) {
      const int i = tid + q * kThreads;
      As[i % BK][i / BK] = ra[q];
    }
#pragma unroll
    for (int q = 0; q < kBLoads; ++q) {
      const int i = tid + q * kThreads;
      Bs[i / BN][i % BN] = rb[q];
      if (MODE == 1) B3s[i / BN][i % BN] = rb3[q];
    }
    __syncthreads();
    if (k0 + BK < K) fetch(k0 + BK);  // in flight during the FMAs below
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4], b3[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][tr * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        b[j] = Bs[kk][tc * 4 + j];
        if (MODE == 1) b3[j] = B3s[kk][tc * 4 + j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
          if (MODE == 1) acc3[i][j] = fmaf(a[i], b3[j], acc3[i][j]);
        }
    }
    __syncthreads();
  }
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
  const dim3 g1(row_tiles, (a.H + BN - 1) / BN), th(kThreads);
  cudaError_t err =
      a.act == MOE_SWIGLU
          ? launch_kernel(ffn_simt_kernel<1>, g1, th, 0, s, 1, true, xp, a.offsets, a.kept_counts,
                          a.E, W1, W3, h, a.d, a.H)
          : launch_kernel(ffn_simt_kernel<2>, g1, th, 0, s, 1, true, xp, a.offsets, a.kept_counts,
                          a.E, W1, no_w, h, a.d, a.H);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  if (between && cudaEventRecord(between, s) != cudaSuccess) return MOE_ERR_CUDA;
  const dim3 g2(row_tiles, (a.d + BN - 1) / BN);
  const float* hc = h;
  err = launch_kernel(ffn_simt_kernel<0>, g2, th, 0, s, 1, true, hc, a.offsets, a.kept_counts,
                      a.E, W2, no_w, static_cast<float*>(a.o), a.H, a.d);
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
