// Measurement aid: a plain streaming read of a device buffer.
//
// The router reads x once (T * d elements) and the permutation and combine
// are copies, so their speed is best judged against what a kernel that does
// nothing but read the same number of bytes reaches on the same GPU at the
// same size: at tens of megabytes the ramp-up and drain of a single launch
// are a visible part of its time.  This kernel is that yardstick.  Every CTA
// takes one contiguous slice of the buffer; each thread keeps eight 16-byte
// streaming loads in flight and folds them into an XOR so the loads cannot be
// dropped; one word per warp is XORed into *sink.

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kProbeThreads = 512;
constexpr int kProbeUnroll = 8;

__global__ void __launch_bounds__(kProbeThreads)
    stream_read_kernel(const uint4* __restrict__ p, int64_t n16, uint32_t* __restrict__ sink) {
  pdl_wait();
  pdl_trigger();
  const int64_t per = (n16 + gridDim.x - 1) / gridDim.x;
  const int64_t begin = static_cast<int64_t>(blockIdx.x) * per;
  const int64_t end = begin + per < n16 ? begin + per : n16;
  uint32_t acc = 0;
  for (int64_t i = begin + threadIdx.x; i < end; i += kProbeThreads * kProbeUnroll) {
    uint4 v[kProbeUnroll];
#pragma unroll
    for (int u = 0; u < kProbeUnroll; ++u) {
      const int64_t j = i + static_cast<int64_t>(u) * kProbeThreads;
      v[u] = j < end ? __ldcs(p + j) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kProbeUnroll; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) atomicXor(sink, acc);
}

}  // namespace

cudaError_t launch_stream_read(const void* buf, size_t bytes, uint32_t* sink, int num_sms,
                               cudaStream_t s) {
  const int64_t n16 = static_cast<int64_t>(bytes / 16);
  if (n16 == 0) return cudaSuccess;
  // Two 512-thread CTAs per SM: 1024 threads x 8 x 16 bytes = 128 KB of
  // loads in flight per SM.
  const int grid = 2 * num_sms;
  return launch_kernel(stream_read_kernel, dim3(grid), dim3(kProbeThreads), 0, s, 1, true,
                       static_cast<const uint4*>(buf), n16, sink);
}

}  // namespace moe
