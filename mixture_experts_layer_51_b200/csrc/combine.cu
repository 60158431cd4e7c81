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
// kept rows of o (fp32) and writes y once.

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kCombineWarps = 8;

// CH = 8-element chunks per lane per iteration: 2 for k <= 2 (more loads in
// flight per lane), 1 otherwise (k rows already give 2k loads per chunk).
template <bool OUT_BF16, int CH>
__global__ void __launch_bounds__(kCombineWarps * 32)
    combine_kernel(const float4* __restrict__ o, const int32_t* __restrict__ pos,
                   const float* __restrict__ gate, int T, int d, int k, void* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kCombineWarps + warp;
  if (t >= T) return;
  constexpr int KJ = CH == 2 ? 2 : kMaxK;  // slots this instantiation handles
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
  const int d4 = d / 4;   // float4 per row of o
  const int n8 = d / 8;   // 8-element chunks per row
  for (int c0 = lane; c0 < n8; c0 += 32 * CH) {
    float4 v[KJ][CH][2];
    // Issue every load of this iteration before any arithmetic.
#pragma unroll
    for (int j = 0; j < KJ; ++j) {
#pragma unroll
      for (int h = 0; h < CH; ++h) {
        const int c8 = c0 + h * 32;
        if (j < k && p[j] >= 0 && c8 < n8) {
          const float4* row = o + (int64_t)p[j] * d4 + c8 * 2;
          v[j][h][0] = __ldcs(row);
          v[j][h][1] = __ldcs(row + 1);
        } else {
          v[j][h][0] = make_float4(0.f, 0.f, 0.f, 0.f);
          v[j][h][1] = v[j][h][0];
        }
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
        // Slot order j = 0..k-1; absent slots hold zeros and add exactly 0.
        if (j < k && p[j] >= 0) {
          const float4 a = v[j][h][0], b = v[j][h][1];
          acc[0] = fmaf(g[j], a.x, acc[0]);
          acc[1] = fmaf(g[j], a.y, acc[1]);
          acc[2] = fmaf(g[j], a.z, acc[2]);
          acc[3] = fmaf(g[j], a.w, acc[3]);
          acc[4] = fmaf(g[j], b.x, acc[4]);
          acc[5] = fmaf(g[j], b.y, acc[5]);
          acc[6] = fmaf(g[j], b.z, acc[6]);
          acc[7] = fmaf(g[j], b.w, acc[7]);
        }
      }
      if (OUT_BF16) {
        uint4 q;
        q.x = pack_bf16x2(acc[0], acc[1]);
        q.y = pack_bf16x2(acc[2], acc[3]);
        q.z = pack_bf16x2(acc[4], acc[5]);
        q.w = pack_bf16x2(acc[6], acc[7]);
        reinterpret_cast<uint4*>(y)[(int64_t)t * n8 + c8] = q;
      } else {
        float4* yr = reinterpret_cast<float4*>(y) + (int64_t)t * d4 + c8 * 2;
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
  const float4* o = reinterpret_cast<const float4*>(a.o);
  const dim3 th(kCombineWarps * 32);
  auto go = [&](auto kern) {
    return launch_kernel(kern, dim3(grid), th, 0, s, 1, true, o, a.pos, a.gate, a.T, a.d, a.k, a.y);
  };
  if (dtype == MOE_BF16)
    return a.k <= 2 ? go(combine_kernel<true, 2>) : go(combine_kernel<true, 1>);
  return a.k <= 2 ? go(combine_kernel<false, 2>) : go(combine_kernel<false, 1>);
}

}  // namespace moe
