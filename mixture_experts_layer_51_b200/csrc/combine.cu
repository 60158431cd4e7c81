// Un-permute and gate-weighted combine.
//
// Pages: "[Paper Club] Upcycling Large Language Models into Mixture of
// Experts" -- after the expert computation the tokens are put back in their
// original order and the router probability scales each expert's output;
// "How do Mixture of Expert Models Work?", "The Math Behind MoEs" --
// y = sum_i G(x)_i E_i(x).
//
// A gather, not a scatter: one warp owns one output token and reads its k
// expert rows (pos[t, j] >= 0), accumulating gate * o in fp32 in slot order
// j = 0..k-1, then rounds once to the output dtype.  No atomics, so the sum
// order is fixed and the result deterministic.  Bound by HBM: it reads the
// kept rows of o (in the layer dtype) and writes y once.

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kCombineWarps = 8;

// BF16: o and y are bf16 (else both fp32).  KJ = slots this instantiation
// handles (2 for k <= 2, else kMaxK); CH = 8-element chunks per lane per
// iteration, so that every lane has about 128 (k <= 2) or 256 bytes of loads
// in flight whatever the element size.
template <bool BF16, int KJ, int CH>
__global__ void __launch_bounds__(kCombineWarps * 32)
    combine_kernel(const void* __restrict__ o, const int32_t* __restrict__ pos,
                   const float* __restrict__ gate, int T, int d, int k, void* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kCombineWarps + warp;
  if (t >= T) return;
  int p[KJ];
  float g[KJ];
  {
    const int pl = lane < k ? pos[(int64_t)t * k + lane] : -1;
    const float gl = lane < k ? gate[(int64_t)t * k + lane] : 0.f;
#pragma unroll
    for (int j = 0; j < KJ; ++j) {
      p[j] = __shfl_sync(0xffffffffu, pl, j);
      g[j] = __shfl_sync(0xffffffffu, gl, j);
    }
  }
  const int n8 = d / 8;  // 8-element chunks per row
  for (int c0 = lane; c0 < n8; c0 += 32 * CH) {
    Row8<BF16> v[KJ][CH];
    // Issue every load of this iteration before any arithmetic.
#pragma unroll
    for (int j = 0; j < KJ; ++j) {
#pragma unroll
      for (int h = 0; h < CH; ++h) {
        const int c8 = c0 + h * 32;
        if (j < k && p[j] >= 0 && c8 < n8)
          v[j][h].load(o, p[j], d, c8);
        else
          v[j][h].zero();
      }
    }
#pragma unroll
    for (int h = 0; h < CH; ++h) {
      const int c8 = c0 + h * 32;
      if (c8 >= n8) break;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < KJ; ++j) {
        // Slot order j = 0..k-1; absent slots add nothing.
        if (j < k && p[j] >= 0) v[j][h].fma_into(g[j], acc);
      }
      if (BF16) {
        uint4 q;
        q.x = pack_bf16x2(acc[0], acc[1]);
        q.y = pack_bf16x2(acc[2], acc[3]);
        q.z = pack_bf16x2(acc[4], acc[5]);
        q.w = pack_bf16x2(acc[6], acc[7]);
        reinterpret_cast<uint4*>(y)[(int64_t)t * n8 + c8] = q;
      } else {
        float4* yr = reinterpret_cast<float4*>(y) + (int64_t)t * (d / 4) + c8 * 2;
        yr[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        yr[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      }
    }
  }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, moe_dtype dtype, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  const int grid = (a.T + kCombineWarps - 1) / kCombineWarps;
  const dim3 th(kCombineWarps * 32);
  auto go = [&](auto kern) {
    return launch_kernel(kern, dim3(grid), th, 0, s, 1, true, a.o, a.pos, a.gate, a.T, a.d, a.k,
                         a.y);
  };
  if (dtype == MOE_BF16)
    return a.k <= 2 ? go(combine_kernel<true, 2, 4>) : go(combine_kernel<true, kMaxK, 2>);
  return a.k <= 2 ? go(combine_kernel<false, 2, 2>) : go(combine_kernel<false, kMaxK, 1>);
}

}  // namespace moe
