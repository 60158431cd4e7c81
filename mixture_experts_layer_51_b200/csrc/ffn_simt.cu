// Grouped expert FFN in fp32 on the CUDA cores (the fp32 layer: tf32 tensor
// cores would not hold a 1e-5 relative error).
//
// Pages: "[Paper Club] Upcycling Large Language Models into Mixture of
// Experts" (each expert is the original two-layer FFN; all experts run as one
// grouped operation over their token blocks) and "How do Mixture of Expert
// Models Work?", "The Math Behind MoEs" (SwiGLU experts).
//
// One 64x64 output tile per CTA, 256 threads with a 4x4 micro-tile each,
// 16-deep K slabs staged in shared memory.  Expert blocks start on multiples
// of 128 rows, so a 64-row tile never straddles two experts; tiles made only
// of padding rows exit at once.

#include <math.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int BM = 64, BN = 64, BK = 16;

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
template <int MODE>
__global__ void __launch_bounds__(256)
    ffn_simt_kernel(const float* __restrict__ A, const int32_t* __restrict__ offsets,
                    const int32_t* __restrict__ kept, int E, const float* __restrict__ W,
                    const float* __restrict__ W3, float* __restrict__ out, int K, int N) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN];
  __shared__ float B3s[MODE == 1 ? BK : 1][MODE == 1 ? BN : 1];
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
  float acc[4][4] = {};
  float acc3[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int i = tid; i < BM * BK; i += 256) {
      const int r = i / BK, c = i % BK;
      As[c][r] = (r < valid && k0 + c < K) ? A[(int64_t)(r0 + r) * K + k0 + c] : 0.f;
    }
    for (int i = tid; i < BK * BN; i += 256) {
      const int r = i / BN, c = i % BN;
      const bool ok = (k0 + r < K) && (n0 + c < N);
      Bs[r][c] = ok ? We[(int64_t)(k0 + r) * N + n0 + c] : 0.f;
      if (MODE == 1) B3s[r][c] = ok ? W3e[(int64_t)(k0 + r) * N + n0 + c] : 0.f;
    }
    __syncthreads();
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
  dim3 g1(row_tiles, (a.H + BN - 1) / BN);
  if (a.act == MOE_SWIGLU)
    ffn_simt_kernel<1><<<g1, 256, 0, s>>>(xp, a.offsets, a.kept_counts, a.E,
                                          static_cast<const float*>(a.W1),
                                          static_cast<const float*>(a.W3), h, a.d, a.H);
  else
    ffn_simt_kernel<2><<<g1, 256, 0, s>>>(xp, a.offsets, a.kept_counts, a.E,
                                          static_cast<const float*>(a.W1), nullptr, h, a.d, a.H);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  if (between && cudaEventRecord(between, s) != cudaSuccess) return MOE_ERR_CUDA;
  dim3 g2(row_tiles, (a.d + BN - 1) / BN);
  ffn_simt_kernel<0><<<g2, 256, 0, s>>>(h, a.offsets, a.kept_counts, a.E,
                                        static_cast<const float*>(a.W2), nullptr, static_cast<float*>(a.o), a.H, a.d);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
