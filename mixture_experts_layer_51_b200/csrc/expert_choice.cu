// Expert-choice routing: every expert takes a fixed number of tokens.
//
// Page: "[Paper Club] Upcycling Large Language Models into Mixture of
// Experts", the Q&A on expert choice -- the selection is reversed: instead of
// each token picking k experts, each expert picks a fixed number of tokens,
// so a token may be processed by no expert, by several, or by all.  The
// affinity an expert ranks tokens by is the router probability
// Softmax(x . W_g) over all experts ("How do Mixture of Expert Models
// Work?", "The Math Behind MoEs"), computed by the router kernel
// (RouteArgs::scores).  Each expert takes n = min(C, T) tokens,
// C = ceil(cf * T * k / E); equal affinities go to the lower position.
//
// Kernels here:
//   ec_select_kernel   one CTA per expert: radix select of the n-th largest
//                      affinity in its column (4 passes of 8 bits over
//                      order-preserving 32-bit keys), then one ordered pass
//                      that marks the chosen tokens and ranks them in
//                      position order (block-wide ballot scans) -- writes
//                      the expert's token list and pos[t, e].
//   ec_gather_kernel   xp row (e, r) = x[token r of expert e] (16-byte copies).
//   ec_combine_kernel  one warp per token: y_t = sum over the experts that
//                      took t, ascending e, of affinity * o row, fp32, one
//                      rounding.  A gather (no atomics): deterministic.
// The expert FFNs in between are the grouped GEMMs of the token-choice path.

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;

// Ascending order of these keys is descending order of the float (the
// sign-aware flip turns float order into unsigned order; the complement
// reverses it).
__device__ __forceinline__ uint32_t desc_key(float v) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t asc = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return ~asc;
}

// Exclusive prefix of a per-thread flag over the CTA in thread order, and
// the CTA total.  `wsum` holds kSelWarps ints; the caller synchronises
// before `wsum` is reused.
__device__ __forceinline__ int cta_exclusive_scan(bool flag, int* wsum, int* total) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned b = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) wsum[warp] = __popc(b);
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll 4
  for (int w = 0; w < kSelWarps; ++w) {
    const int c = wsum[w];
    before += (w < warp) ? c : 0;
    all += c;
  }
  *total = all;
  return before + __popc(b & ((1u << lane) - 1u));
}

__global__ void __launch_bounds__(kSelThreads)
    ec_select_kernel(const float* __restrict__ scores, int T, int E, int n, int npad,
                     uint32_t* __restrict__ keys_t, int32_t* __restrict__ tok,
                     int32_t* __restrict__ pos, int32_t* __restrict__ kept_counts,
                     int32_t* __restrict__ offsets) {
  __shared__ uint32_t hist[256];
  __shared__ int wsum_a[kSelWarps], wsum_b[kSelWarps];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need;
  const int e = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t* keys = keys_t + (int64_t)e * T;

  for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
  __syncthreads();
  // The column of affinities as keys (a strided read of [T, E]; the
  // transposed copy makes the later passes contiguous) and the histogram of
  // the top byte.
  for (int t = tid; t < T; t += kSelThreads) {
    const uint32_t key = desc_key(scores[(int64_t)t * E + e]);
    keys[t] = key;
    atomicAdd(&hist[key >> 24], 1u);
  }
  __syncthreads();

  uint32_t prefix = 0;  // the n-th smallest key, one byte per pass
  int need = n;         // how many of the keys matching prefix are still wanted
  if (n > 0) {
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      if (pass > 0) {
        for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
        __syncthreads();
        for (int t = tid; t < T; t += kSelThreads) {
          const uint32_t key = keys[t];
          if ((key >> (shift + 8)) == (prefix >> (shift + 8))) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
      }
      if (warp == 0) {
        // Lane l owns buckets 8l .. 8l+7; find the bucket holding the
        // need-th key (1-based) in ascending order.
        int c[8], sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          c[j] = static_cast<int>(hist[lane * 8 + j]);
          sum += c[j];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += u;
        }
        int before = incl - sum;
        if (before < need && need <= incl) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (need <= before + c[j]) {
              s_prefix = prefix | (static_cast<uint32_t>(lane * 8 + j) << shift);
              s_need = need - before;
              break;
            }
            before += c[j];
          }
        }
      }
      __syncthreads();
      prefix = s_prefix;
      need = s_need;
      __syncthreads();
    }
  }

  // Chosen: key < prefix, or key == prefix among the first `need` such
  // tokens in position order.  Rows follow position order.
  const int32_t row0 = e * npad;
  int carry_eq = 0, carry_sel = 0;
  for (int base = 0; base < T; base += kSelThreads) {
    const int t = base + tid;
    const uint32_t key = t < T ? keys[t] : 0xffffffffu;
    const bool eq = n > 0 && t < T && key == prefix;
    const bool lt = n > 0 && t < T && key < prefix;
    int tot_eq, tot_sel;
    const int eq_rank = carry_eq + cta_exclusive_scan(eq, wsum_a, &tot_eq);
    const bool chosen = lt || (eq && eq_rank < need);
    const int row = carry_sel + cta_exclusive_scan(chosen, wsum_b, &tot_sel);
    if (t < T) {
      pos[(int64_t)t * E + e] = chosen ? row0 + row : -1;
      if (chosen) tok[(int64_t)e * n + row] = t;
    }
    carry_eq += tot_eq;
    carry_sel += tot_sel;
    __syncthreads();  // wsum_a / wsum_b are rewritten by the next chunk
  }
  if (tid == 0) kept_counts[e] = n;
  if (e == 0)
    for (int i = tid; i <= E; i += kSelThreads) offsets[i] = i * npad;
}

constexpr int kGatherWarps = 8;

// One warp per xp row; 16-byte vectors, four loads in flight per lane.
__global__ void __launch_bounds__(kGatherWarps * 32)
    ec_gather_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ tok, int n, int npad,
                     int dvec, uint4* __restrict__ xp) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * kGatherWarps + warp;
  const int e = blockIdx.y;
  if (r >= n) return;
  const int t = tok[(int64_t)e * n + r];
  const uint4* src = x + (int64_t)t * dvec;
  uint4* dst = xp + ((int64_t)e * npad + r) * dvec;
  for (int v0 = lane; v0 < dvec; v0 += 32 * 4) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (v0 + u * 32 < dvec) v[u] = __ldcs(src + v0 + u * 32);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (v0 + u * 32 < dvec) dst[v0 + u * 32] = v[u];
  }
}

constexpr int kEcCombineWarps = 8;

template <bool OUT_BF16>
__global__ void __launch_bounds__(kEcCombineWarps * 32)
    ec_combine_kernel(const float4* __restrict__ o, const int32_t* __restrict__ pos,
                      const float* __restrict__ scores, int T, int d, int E,
                      void* __restrict__ y) {
  __shared__ int sp[kEcCombineWarps][kMaxE];
  __shared__ float sg[kEcCombineWarps][kMaxE];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kEcCombineWarps + warp;
  if (t >= T) return;
  // The experts that took t, ascending e, compacted into this warp's list.
  int nsel = 0;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    const int p = e < E ? pos[(int64_t)t * E + e] : -1;
    const unsigned b = __ballot_sync(0xffffffffu, p >= 0);
    if (p >= 0) {
      const int i = nsel + __popc(b & ((1u << lane) - 1u));
      sp[warp][i] = p;
      sg[warp][i] = scores[(int64_t)t * E + e];
    }
    nsel += __popc(b);
  }
  __syncwarp();
  const int d4 = d / 4, n8 = d / 8;
  for (int c8 = lane; c8 < n8; c8 += 32) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int j0 = 0; j0 < nsel; j0 += 4) {
      float4 v[4][2];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (j0 + u < nsel) {
          const float4* row = o + (int64_t)sp[warp][j0 + u] * d4 + c8 * 2;
          v[u][0] = __ldcs(row);
          v[u][1] = __ldcs(row + 1);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (j0 + u < nsel) {
          const float g = sg[warp][j0 + u];
          acc[0] = fmaf(g, v[u][0].x, acc[0]);
          acc[1] = fmaf(g, v[u][0].y, acc[1]);
          acc[2] = fmaf(g, v[u][0].z, acc[2]);
          acc[3] = fmaf(g, v[u][0].w, acc[3]);
          acc[4] = fmaf(g, v[u][1].x, acc[4]);
          acc[5] = fmaf(g, v[u][1].y, acc[5]);
          acc[6] = fmaf(g, v[u][1].z, acc[6]);
          acc[7] = fmaf(g, v[u][1].w, acc[7]);
        }
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

}  // namespace

size_t ec_select_scratch_bytes(int T, int E) {
  return (static_cast<size_t>(T) * E * 4 + 255) / 256 * 256;
}

cudaError_t launch_ec_select(const float* scores, int T, int E, int n, int npad, void* scratch,
                             int32_t* tok, int32_t* pos, int32_t* kept_counts, int32_t* offsets,
                             cudaStream_t s) {
  ec_select_kernel<<<E, kSelThreads, 0, s>>>(scores, T, E, n, npad,
                                             static_cast<uint32_t*>(scratch), tok, pos,
                                             kept_counts, offsets);
  return cudaGetLastError();
}

cudaError_t launch_ec_gather(const void* x, const int32_t* tok, int E, int n, int npad, int d,
                             moe_dtype dtype, void* xp, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int dvec = d * (dtype == MOE_BF16 ? 2 : 4) / 16;
  const dim3 grid((n + kGatherWarps - 1) / kGatherWarps, E);
  ec_gather_kernel<<<grid, kGatherWarps * 32, 0, s>>>(static_cast<const uint4*>(x), tok, n, npad,
                                                      dvec, static_cast<uint4*>(xp));
  return cudaGetLastError();
}

cudaError_t launch_ec_combine(const float* o, const int32_t* pos, const float* scores, int T,
                              int d, int E, moe_dtype dtype, void* y, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int grid = (T + kEcCombineWarps - 1) / kEcCombineWarps;
  const float4* o4 = reinterpret_cast<const float4*>(o);
  if (dtype == MOE_BF16)
    ec_combine_kernel<true><<<grid, kEcCombineWarps * 32, 0, s>>>(o4, pos, scores, T, d, E, y);
  else
    ec_combine_kernel<false><<<grid, kEcCombineWarps * 32, 0, s>>>(o4, pos, scores, T, d, E, y);
  return cudaGetLastError();
}

}  // namespace moe
