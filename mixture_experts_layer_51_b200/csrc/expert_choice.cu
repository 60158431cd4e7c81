// Expert-choice routing: every expert takes a fixed number of tokens.
//
// Page: "[Paper Club] Upcycling Large Language Models into Mixture of
// Experts", the Q&A on expert choice -- the selection is reversed: instead of
// each token picking k experts, each expert picks a fixed number of tokens,
// so a token may be processed by no expert, by several, or by all.  The
// affinity an expert ranks tokens by is the router probability
// Softmax(x . W_g) over all experts ("How do Mixture of Expert Models
// Work?", "The Math Behind MoEs"), computed by the router kernel
// (RouteArgs::scores) as an expert-major [E, T] matrix.  Each expert takes n = min(C, T) tokens,
// C = ceil(cf * T * k / E); equal affinities go to the lower position.
//
// Kernels here:
//   ec_select_kernel   a cluster of CTAs per expert: radix select of the n-th
//                      largest affinity in its (contiguous, expert-major)
//                      column (4 passes of 8 bits over order-preserving
//                      32-bit keys, histograms merged through distributed
//                      shared memory), then one ordered pass that marks the
//                      chosen tokens and ranks them in position order
//                      (CTA-wide ballot scans, slice offsets from the
//                      cluster) -- writes the expert's token list and its
//                      row of positions, pos_t[e, t];
//   ec_transpose_kernel  pos [T, E] from pos_t, through shared memory.
// The chosen x rows are copied by the token-major row copy of the
// permutation (read once, written once per expert that took the token).
//   ec_combine_kernel  one warp per token: y_t = sum over the experts that
//                      took t, ascending e, of affinity * o row, fp32, one
//                      rounding.  A gather (no atomics): deterministic.
// The expert FFNs in between are the grouped GEMMs of the token-choice path.

#include "moe_internal.cuh"

namespace moe {
namespace {

// Selection: a cluster of kSelCta CTAs per expert, CTA r owning the r-th
// contiguous slice of token positions.  Every pass builds per-CTA digit
// histograms (warp-aggregated shared-memory atomics: integer counts, so the
// order they land in does not matter), then every CTA reads all kSelCta
// histograms of its cluster through distributed shared memory and sums them
// in rank order, so all CTAs find the same bucket.  The last pass exchanges
// per-slice counts the same way to give each slice its starting ranks.
// CTAs per expert (one cluster).  Four rather than eight: on the 64-expert,
// 16384-token layer the permutation stage (selection, transpose, copy) took
// 145.5 us with clusters of four and 159 us with clusters of eight, whose
// 512 CTAs need more than one round of the SMs; two measured the same as four.
constexpr int kSelCta = 4;
constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kKeyRegs = 16;     // key chunks a thread keeps in registers

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
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) {
    const int c = wsum[w];
    before += (w < warp) ? c : 0;
    all += c;
  }
  *total = all;
  return before + __popc(b & ((1u << lane) - 1u));
}

// Adds 1 to hist[bin] for every lane with bin < 256; lanes with the same
// bin are combined first, so a popular bin takes one atomic per warp.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin) {
  const unsigned peers = __match_any_sync(0xffffffffu, bin);
  const int lane = threadIdx.x & 31;
  if (bin < 256u && lane == __ffs(peers) - 1)
    atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
}

// scores: [E, T] (expert-major: each expert's column is contiguous).
// pos_t: [E, T] (expert-major) positions; ec_transpose_kernel turns them
// into the token-major pos [T, E] the copy and the combine read.
__global__ void __launch_bounds__(kSelThreads)
    ec_select_kernel(const float* __restrict__ scores, int T, int E, int n, int npad,
                     int32_t* __restrict__ pos_t, int32_t* __restrict__ tok,
                     int32_t* __restrict__ kept_counts, int32_t* __restrict__ offsets) {
  __shared__ uint32_t hist[2][256];  // alternate passes, so one cluster barrier per pass
  __shared__ uint32_t tot[256];      // cluster-wide histogram of the current pass
  __shared__ int slice_cnt[2];       // this slice's keys below the cut and equal to it
  __shared__ int wsum_a[kSelWarps], wsum_b[kSelWarps];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need;
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x / kSelCta;
  const uint32_t r = cluster_ctarank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (T + kSelCta - 1) / kSelCta;
  const int t_begin = min(T, static_cast<int>(r) * per), t_end = min(T, t_begin + per);
  const float* col = scores + (int64_t)e * T;  // this expert's affinities, contiguous
  auto key_at = [&](int t) { return desc_key(__ldg(col + t)); };
  // A slice of up to kKeyRegs chunks of kSelThreads keys is read once into
  // registers; the six passes below then read no memory for their keys.
  // (The condition is the same for every CTA: per is.)
  const bool cached = per <= kKeyRegs * kSelThreads;
  uint32_t kc[kKeyRegs];
#pragma unroll
  for (int j = 0; j < kKeyRegs; ++j) {
    const int t = t_begin + j * kSelThreads + tid;
    kc[j] = (cached && t < t_end) ? key_at(t) : 0u;
  }
  // Visits the slice's tokens in chunks of kSelThreads, in position order:
  // f(t, valid, key).  Every thread makes the same calls (the warp votes and
  // block barriers inside f need that).
  auto visit = [&](auto&& f) {
    if (cached) {
#pragma unroll
      for (int j = 0; j < kKeyRegs; ++j) {
        if (t_begin + j * kSelThreads < t_end) {
          const int t = t_begin + j * kSelThreads + tid;
          f(t, t < t_end, kc[j]);
        }
      }
    } else {
      for (int b0 = t_begin; b0 < t_end; b0 += kSelThreads) {
        const int t = b0 + tid;
        f(t, t < t_end, t < t_end ? key_at(t) : 0u);
      }
    }
  };

  for (int i = tid; i < 512; i += kSelThreads) (&hist[0][0])[i] = 0;
  __syncthreads();
  // The histogram of the keys' top byte over this slice.
  visit([&](int, bool valid, uint32_t key) { hist_add(hist[0], valid ? key >> 24 : 256u); });

  uint32_t prefix = 0;  // the n-th smallest key of the column, one byte per pass
  int need = n;         // how many keys equal to the final prefix are taken
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    uint32_t* h = hist[pass & 1];
    if (pass > 0) {
      for (int i = tid; i < 256; i += kSelThreads) h[i] = 0;
      __syncthreads();
      visit([&](int, bool valid, uint32_t key) {
        uint32_t bin = 256u;
        if (valid && (key >> (shift + 8)) == (prefix >> (shift + 8))) bin = (key >> shift) & 255u;
        hist_add(h, bin);
      });
    }
    // Every CTA's histogram of this pass is complete before any is read;
    // the other buffer is rewritten only after the next barrier.
    cluster_sync();
    if (tid < 256) {
      const uint32_t local = smem_u32(&h[tid]);
      uint32_t sum = 0;
      for (uint32_t q = 0; q < kSelCta; ++q) sum += ld_shared_cluster_u32(mapa_shared(local, q));
      tot[tid] = sum;
    }
    __syncthreads();
    if (warp == 0 && n > 0) {
      // Lane l owns buckets 8l .. 8l+7; find the bucket holding the
      // need-th key (1-based) in ascending order.
      int c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = static_cast<int>(tot[lane * 8 + j]);
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
    if (n > 0) {
      prefix = s_prefix;
      need = s_need;
    }
  }

  // Chosen: key < prefix, or key == prefix among the first `need` such
  // tokens in position order.  First every slice counts both kinds; the
  // counts of the lower slices give this slice's starting ranks.
  int lt_n = 0, eq_n = 0;
  visit([&](int, bool valid, uint32_t key) {
    lt_n += (valid && n > 0 && key < prefix);
    eq_n += (valid && n > 0 && key == prefix);
  });
  {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lt_n += __shfl_xor_sync(0xffffffffu, lt_n, o);
      eq_n += __shfl_xor_sync(0xffffffffu, eq_n, o);
    }
    if (lane == 0) {
      wsum_a[warp] = lt_n;
      wsum_b[warp] = eq_n;
    }
    __syncthreads();
    if (tid == 0) {
      int a = 0, b = 0;
      for (int w = 0; w < kSelWarps; ++w) {
        a += wsum_a[w];
        b += wsum_b[w];
      }
      slice_cnt[0] = a;
      slice_cnt[1] = b;
    }
  }
  cluster_sync();
  int eq_before = 0, row_before = 0;
  for (uint32_t q = 0; q < r; ++q) {
    const int lt_q =
        static_cast<int>(ld_shared_cluster_u32(mapa_shared(smem_u32(&slice_cnt[0]), q)));
    const int eq_q =
        static_cast<int>(ld_shared_cluster_u32(mapa_shared(smem_u32(&slice_cnt[1]), q)));
    const int take_q = max(0, min(eq_q, need - eq_before));
    row_before += lt_q + take_q;
    eq_before += eq_q;
  }
  // No CTA may leave (or reuse its shared memory) while others read it.
  cluster_sync();

  const int32_t row0 = e * npad;
  int carry_eq = eq_before, carry_sel = row_before;
  visit([&](int t, bool valid, uint32_t key) {
    const bool eq = n > 0 && valid && key == prefix;
    const bool lt = n > 0 && valid && key < prefix;
    int tot_eq, tot_sel;
    const int eq_rank = carry_eq + cta_exclusive_scan(eq, wsum_a, &tot_eq);
    const bool chosen = lt || (eq && eq_rank < need);
    const int row = carry_sel + cta_exclusive_scan(chosen, wsum_b, &tot_sel);
    if (valid) {
      pos_t[(int64_t)e * T + t] = chosen ? row0 + row : -1;
      if (chosen) tok[(int64_t)e * n + row] = t;
    }
    carry_eq += tot_eq;
    carry_sel += tot_sel;
    __syncthreads();  // wsum_a / wsum_b are rewritten by the next chunk
  });
  if (r == 0 && tid == 0) kept_counts[e] = n;
  if (blockIdx.x == 0)
    for (int i = tid; i <= E; i += kSelThreads) offsets[i] = i * npad;
}

// pos [T, E] from pos_t [E, T], through a 32 x 64 shared-memory tile:
// reads run along tokens, writes along experts.
constexpr int kTrE = 32, kTrT = 64;
__global__ void __launch_bounds__(256)
    ec_transpose_kernel(const int32_t* __restrict__ pos_t, int T, int E,
                        int32_t* __restrict__ pos) {
  __shared__ int32_t tile[kTrE][kTrT + 1];
  pdl_wait();
  pdl_trigger();
  const int t0 = blockIdx.x * kTrT, e0 = blockIdx.y * kTrE;
  for (int i = threadIdx.x; i < kTrE * kTrT; i += 256) {
    const int el = i / kTrT, tl = i - el * kTrT;
    if (e0 + el < E && t0 + tl < T) tile[el][tl] = pos_t[(int64_t)(e0 + el) * T + t0 + tl];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kTrE * kTrT; i += 256) {
    const int tl = i / kTrE, el = i - tl * kTrE;
    if (e0 + el < E && t0 + tl < T) pos[(int64_t)(t0 + tl) * E + e0 + el] = tile[el][tl];
  }
}

constexpr int kEcCombineWarps = 8;

// BF16: o and y are bf16 (else both fp32).
template <bool BF16>
__global__ void __launch_bounds__(kEcCombineWarps * 32)
    ec_combine_kernel(const void* __restrict__ o, const int32_t* __restrict__ pos,
                      const float* __restrict__ scores, int T, int d, int E,
                      void* __restrict__ y) {
  __shared__ int sp[kEcCombineWarps][kMaxE];
  __shared__ float sg[kEcCombineWarps][kMaxE];
  pdl_wait();
  pdl_trigger();
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
      sg[warp][i] = scores[(int64_t)e * T + t];
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
      Row8<BF16> v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (j0 + u < nsel) v[u].load(o, sp[warp][j0 + u], d, c8);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (j0 + u < nsel) v[u].fma_into(sg[warp][j0 + u], acc);
    }
    if (BF16) {
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
  int32_t* pos_t = static_cast<int32_t*>(scratch);
  cudaError_t err = launch_kernel(ec_select_kernel, dim3(E * kSelCta), dim3(kSelThreads), 0, s,
                                  kSelCta, true, scores, T, E, n, npad, pos_t, tok, kept_counts,
                                  offsets);
  if (err != cudaSuccess) return err;
  return launch_kernel(ec_transpose_kernel, dim3((T + kTrT - 1) / kTrT, (E + kTrE - 1) / kTrE),
                       dim3(256), 0, s, 1, true, static_cast<const int32_t*>(pos_t), T, E, pos);
}

cudaError_t launch_ec_combine(const void* o, const int32_t* pos, const float* scores, int T,
                              int d, int E, moe_dtype dtype, void* y, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int grid = (T + kEcCombineWarps - 1) / kEcCombineWarps;
  const dim3 th(kEcCombineWarps * 32);
  if (dtype == MOE_BF16)
    return launch_kernel(ec_combine_kernel<true>, dim3(grid), th, 0, s, 1, true, o, pos, scores, T,
                         d, E, y);
  return launch_kernel(ec_combine_kernel<false>, dim3(grid), th, 0, s, 1, true, o, pos, scores, T,
                       d, E, y);
}

}  // namespace moe
