// Batch Priority Routing: the order in which tokens reach the expert queues.
//
// Page: "Scaling Vision with Sparse Mixture of Experts", "Priority Routing"
// -- instead of dropping the tokens that arrive last once an expert is full,
// tokens are sorted by an importance score and the least important ones are
// skipped.  The score is the token's largest gate (its slot-0 gate); equal
// scores keep their position order.
//
// This file computes that order as a stable argsort of the T scores,
// descending: an LSD radix sort of 32-bit keys (4 passes of 8 bits), each pass
// a 256-bucket counting sort --
//   histogram: per 256-element block, digit counts (shared-memory atomics:
//              counts do not depend on the order the atomics land);
//   scan:      one CTA turns the [digit][block] counts into exclusive
//              offsets (digit-major, so equal digits keep block order);
//   scatter:   within a block, an element's rank among equal digits comes
//              from __match_any_sync and per-warp counts, in element order.
// Every placement follows from counts in element order, so the sort is
// stable and deterministic.  moe_permute then serves tokens in this order.

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kSortBlock = 256;  // elements per block = threads per CTA
constexpr int kSortWarps = kSortBlock / 32;

// Descending order of the score as an ascending order of unsigned keys:
// the usual sign-aware bit flip makes float order unsigned order, and the
// complement reverses it.
__device__ __forceinline__ uint32_t descending_key(float v) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t asc = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return ~asc;
}

__global__ void __launch_bounds__(kSortBlock)
    prio_keys_kernel(const float* __restrict__ gate, int T, int k, uint32_t* __restrict__ keys,
                     int32_t* __restrict__ vals) {
  const int t = blockIdx.x * kSortBlock + threadIdx.x;
  if (t >= T) return;
  keys[t] = descending_key(gate[(int64_t)t * k]);
  vals[t] = t;
}

__global__ void __launch_bounds__(kSortBlock)
    radix_hist_kernel(const uint32_t* __restrict__ keys, int T, int shift, int nblk,
                      uint32_t* __restrict__ hist) {
  __shared__ uint32_t h[256];
  const int tid = threadIdx.x;
  h[tid] = 0;
  __syncthreads();
  const int i = blockIdx.x * kSortBlock + tid;
  if (i < T) atomicAdd(&h[(keys[i] >> shift) & 255u], 1u);
  __syncthreads();
  hist[(int64_t)tid * nblk + blockIdx.x] = h[tid];
}

// Exclusive scan of n counts in place, one CTA of 1024 threads: each thread
// sums a contiguous segment, the segment sums are scanned, then each thread
// rewrites its segment.
__global__ void __launch_bounds__(1024) radix_scan_kernel(uint32_t* __restrict__ a, int n) {
  __shared__ uint32_t wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int seg = (n + 1023) / 1024;
  const int b = tid * seg, e = min(n, b + seg);
  uint32_t s = 0;
  for (int i = b; i < e; ++i) s += a[i];
  // block exclusive scan of s
  uint32_t v = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) wsum[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    wsum[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  uint32_t run = v - s + (warp > 0 ? wsum[warp - 1] : 0u);  // exclusive prefix of this segment
  for (int i = b; i < e; ++i) {
    const uint32_t c = a[i];
    a[i] = run;
    run += c;
  }
}

__global__ void __launch_bounds__(kSortBlock)
    radix_scatter_kernel(const uint32_t* __restrict__ keys_in, const int32_t* __restrict__ vals_in,
                         int T, int shift, int nblk, const uint32_t* __restrict__ offs,
                         uint32_t* __restrict__ keys_out, int32_t* __restrict__ vals_out) {
  __shared__ uint32_t wcnt[kSortWarps][256];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kSortWarps * 256; i += kSortBlock) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  const int i = blockIdx.x * kSortBlock + tid;
  const bool valid = i < T;
  const uint32_t key = valid ? keys_in[i] : 0u;
  const uint32_t digit = valid ? (key >> shift) & 255u : 256u;  // 256: no element
  const unsigned peers = __match_any_sync(0xffffffffu, digit);
  const unsigned lt = (1u << lane) - 1u;
  const uint32_t rank = __popc(peers & lt);
  if (valid && rank == 0) wcnt[warp][digit] = __popc(peers);
  __syncthreads();
  // exclusive prefix over warps, per digit (thread tid owns digit tid)
  {
    uint32_t run = 0;
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) {
      const uint32_t c = wcnt[w][tid];
      wcnt[w][tid] = run;
      run += c;
    }
  }
  __syncthreads();
  if (valid) {
    const uint32_t dst = offs[(int64_t)digit * nblk + blockIdx.x] + wcnt[warp][digit] + rank;
    keys_out[dst] = key;
    vals_out[dst] = vals_in[i];
  }
}

}  // namespace

size_t priority_scratch_bytes(int T) {
  const size_t nblk = (static_cast<size_t>(T) + kSortBlock - 1) / kSortBlock;
  const size_t a = (static_cast<size_t>(T) * 4 + 255) / 256 * 256;
  return 3 * a + (256 * nblk * 4 + 255) / 256 * 256;  // keys x2, vals (the other is `order`)
}

cudaError_t launch_priority_order(const float* gate, int T, int k, int32_t* order, void* scratch,
                                  cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int nblk = (T + kSortBlock - 1) / kSortBlock;
  const size_t a = (static_cast<size_t>(T) * 4 + 255) / 256 * 256;
  uint8_t* p = static_cast<uint8_t*>(scratch);
  uint32_t* keys[2] = {reinterpret_cast<uint32_t*>(p), reinterpret_cast<uint32_t*>(p + a)};
  // Four passes ping-pong between the two value buffers and end in `order`.
  int32_t* vals[2] = {order, reinterpret_cast<int32_t*>(p + 2 * a)};
  uint32_t* hist = reinterpret_cast<uint32_t*>(p + 3 * a);
  prio_keys_kernel<<<nblk, kSortBlock, 0, s>>>(gate, T, k, keys[0], vals[0]);
  cudaError_t err = cudaGetLastError();
  for (int pass = 0; pass < 4 && err == cudaSuccess; ++pass) {
    const int in = pass & 1, out = in ^ 1;
    radix_hist_kernel<<<nblk, kSortBlock, 0, s>>>(keys[in], T, pass * 8, nblk, hist);
    radix_scan_kernel<<<1, 1024, 0, s>>>(hist, 256 * nblk);
    radix_scatter_kernel<<<nblk, kSortBlock, 0, s>>>(keys[in], vals[in], T, pass * 8, nblk, hist,
                                                     keys[out], vals[out]);
    err = cudaGetLastError();
  }
  return err;
}

}  // namespace moe
