// Permutation of tokens into one contiguous block per expert, with an
// optional capacity.
//
// Pages: "[Paper Club] Upcycling Large Language Models into Mixture of
// Experts" -- after routing, the tokens that chose expert e are gathered
// into one matrix for e, and depending on the capacity factor some tokens are
// dropped (Megatron-Core: dropless by default, or dropping with padding);
// "How do Mixture of Expert Models Work?", "Expert Capacity"; "Take a Closer
// Look at the MoE LLM Routing", "Drop-towards-the-End" -- the tokens that
// arrive later in the sequence are the ones dropped.
//
// The kept assignments of expert e are its first C in token position, so
// the permutation is a stable counting sort by expert:
//   pass 1 (count): per 256-token block, per-expert counts from warp ballots;
//     the last block to finish (atomic ticket) turns them into exclusive
//     per-expert bases, the counts, kept counts (min(count, C)) and the
//     128-row aligned block offsets.
//   pass 2 (rank): per 256-token block, rank = block base + counts of the
//     preceding warps in the block + ballot prefix inside the warp, giving
//     pos[t, j] (row in xp, or -1 when dropped);
//   pass 3 (copy): token-major, one warp per token reads its x row once and
//     writes it to each of its rows (16-byte vectors, eight in flight per
//     lane).  Splitting the ranks out of the copy keeps their dependent
//     ballots off the copy's critical path.
// Every rank is computed from counts in queue order: no atomics decide
// placement, so the output is deterministic.  The queue order is token
// position, or -- Batch Priority Routing -- a given permutation `order`
// (queue position i serves token order[i]); rows of an expert block then
// follow that order.

#include <stdlib.h>

#include <algorithm>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kWarpsPerBlock = kPermBlock / 32;  // 8 warps per block

// Bit e set when token t selected expert e.  Ids outside [0, E) (possible
// only when a caller passes its own idx) select nothing and are never kept.
__device__ __forceinline__ uint64_t expert_mask(const int32_t* __restrict__ idx, int t, int T,
                                                int k, int E) {
  uint64_t m = 0;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(int64_t)t * k + j];
      if (e >= 0 && e < E) m |= 1ull << e;
    }
  }
  return m;
}

// Token served at queue position i: order[i] (Batch Priority Routing) or i.
__device__ __forceinline__ int token_at(const int32_t* __restrict__ order, int i, int T) {
  return (order && i < T) ? order[i] : i;
}

// `prior` (nullable): per expert, assignments that earlier shards of the
// batch (lower positions, other ranks) already queued; this shard may keep
// cap[e] = max(0, C - prior[e]) more.
__global__ void __launch_bounds__(kPermBlock)
    permute_count_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ order, int T,
                         int E, int k, int C, const int32_t* __restrict__ prior, int nblk,
                         int32_t* __restrict__ block_base, unsigned int* __restrict__ ticket,
                         int32_t* __restrict__ cap, int32_t* __restrict__ counts,
                         int32_t* __restrict__ kept_counts, int32_t* __restrict__ offsets) {
  __shared__ int wcnt[kWarpsPerBlock][kMaxE];
  __shared__ int padded[kMaxE];
  __shared__ bool is_last;
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i = blockIdx.x * kPermBlock + tid;
  const uint64_t mask = i < T ? expert_mask(idx, token_at(order, i, T), T, k, E) : 0ull;
  for (int e = 0; e < E; ++e) {
    const unsigned b = __ballot_sync(0xffffffffu, (mask >> e) & 1ull);
    if (lane == 0) wcnt[warp][e] = __popc(b);
  }
  __syncthreads();
  if (tid < E) {
    int s = 0;
#pragma unroll
    for (int w = 0; w < kWarpsPerBlock; ++w) s += wcnt[w][tid];
    block_base[(int64_t)blockIdx.x * E + tid] = s;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = (atomicAdd(ticket, 1u) == static_cast<unsigned>(nblk - 1));
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // Last block: exclusive scan over blocks for every expert.
  if (tid < E) {
    int run = 0;
    int b = 0;
    for (; b + 8 <= nblk; b += 8) {
      int v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = __ldcg(block_base + (int64_t)(b + i) * E + tid);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        block_base[(int64_t)(b + i) * E + tid] = run;
        run += v[i];
      }
    }
    for (; b < nblk; ++b) {
      const int v = __ldcg(block_base + (int64_t)b * E + tid);
      block_base[(int64_t)b * E + tid] = run;
      run += v;
    }
    int ce = C;
    if (prior && C != INT32_MAX) ce = max(0, C - prior[tid]);
    cap[tid] = ce;
    const int kept = run < ce ? run : ce;
    counts[tid] = run;
    kept_counts[tid] = kept;
    padded[tid] = (kept + kRowAlign - 1) / kRowAlign * kRowAlign;
  }
  __syncthreads();
  if (tid == 0) {
    int off = 0;
    for (int e = 0; e < E; ++e) {
      offsets[e] = off;
      off += padded[e];
    }
    offsets[E] = off;
    *ticket = 0u;  // ready for the next call on this workspace
  }
}

// Ranks: one thread per queue position of a 256-token block.  Each warp
// counts, per expert, its lanes' assignments with one ballot per expert; the
// ranks inside the warp come from the same ballots (lanes below), the
// warps below come from the shared counts, and the blocks below from the
// scanned block_base.  Everything follows from counts in queue order, so
// positions are deterministic.
__global__ void __launch_bounds__(kPermBlock)
    permute_rank_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ order, int T,
                        int E, int k, const int32_t* __restrict__ cap,
                        const int32_t* __restrict__ block_base,
                        const int32_t* __restrict__ offsets, int32_t* __restrict__ pos) {
  __shared__ int wcnt[kWarpsPerBlock][kMaxE];
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int blk = blockIdx.x;
  const int i = blk * kPermBlock + tid;
  const int t = i < T ? token_at(order, i, T) : T;  // T: no token
  int ej[kMaxK];
  uint64_t mask = 0;
  for (int j = 0; j < k; ++j) {
    ej[j] = (t < T) ? idx[(int64_t)t * k + j] : -1;
    if (ej[j] >= 0 && ej[j] < E) mask |= 1ull << ej[j];
  }
  int rj[kMaxK];
  for (int j = 0; j < k; ++j) rj[j] = 0;
  const unsigned lt = (1u << lane) - 1u;
  for (int e = 0; e < E; ++e) {
    const unsigned b = __ballot_sync(0xffffffffu, (mask >> e) & 1ull);
    if (lane == 0) wcnt[warp][e] = __popc(b);
    if ((mask >> e) & 1ull) {
      const int r = __popc(b & lt);
      for (int j = 0; j < k; ++j)
        if (ej[j] == e) rj[j] = r;
    }
  }
  __syncthreads();
  if (t >= T) return;
  for (int j = 0; j < k; ++j) {
    const int e = ej[j];
    int p = -1;
    if (e >= 0 && e < E) {
      int r = block_base[(int64_t)blk * E + e] + rj[j];
      for (int w = 0; w < warp; ++w) r += wcnt[w][e];
      if (r < cap[e]) p = offsets[e] + r;
    }
    pos[(int64_t)t * k + j] = p;
  }
}

constexpr int kCopyWarps = 8;

// Token-major row copy: one warp per token reads its x row once (16-byte
// vectors, eight in flight per lane) and writes it to every destination row
// pos[t, 0..npos-1] that is >= 0.
__global__ void __launch_bounds__(kCopyWarps * 32)
    row_copy_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ pos, int T,
                    int npos, int dvec, uint4* __restrict__ xp) {
  __shared__ int dst[kCopyWarps][kMaxE];
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kCopyWarps + warp;
  if (t >= T) return;
  int nd = 0;
  for (int e0 = 0; e0 < npos; e0 += 32) {
    const int p = e0 + lane < npos ? pos[(int64_t)t * npos + e0 + lane] : -1;
    const unsigned b = __ballot_sync(0xffffffffu, p >= 0);
    if (p >= 0) dst[warp][nd + __popc(b & ((1u << lane) - 1u))] = p;
    nd += __popc(b);
  }
  __syncwarp();
  if (nd == 0) return;
  const uint4* src = x + (int64_t)t * dvec;
  for (int v0 = lane; v0 < dvec; v0 += 32 * 8) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (v0 + u * 32 < dvec) v[u] = __ldcs(src + v0 + u * 32);
    for (int j = 0; j < nd; ++j) {
      uint4* out = xp + (int64_t)dst[warp][j] * dvec;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (v0 + u * 32 < dvec) out[v0 + u * 32] = v[u];
    }
  }
}

}  // namespace

size_t permute_scratch_bytes(int T, int E) {
  const size_t nblk = (static_cast<size_t>(T) + kPermBlock - 1) / kPermBlock;
  size_t b = nblk * static_cast<size_t>(E) * sizeof(int32_t);
  b = (b + 255) / 256 * 256;
  return b + 512;  // + ticket counter (256 B) + per-expert capacities (256 B)
}

namespace {
__global__ void __launch_bounds__(kPermBlock)
    expert_count_kernel(const int32_t* __restrict__ idx, int T, int E, int k,
                        int32_t* __restrict__ counts) {
  __shared__ int wcnt[kMaxE];
  const int tid = threadIdx.x, lane = tid & 31;
  if (tid < kMaxE) wcnt[tid] = 0;
  __syncthreads();
  const int t = blockIdx.x * kPermBlock + tid;
  const uint64_t mask = t < T ? expert_mask(idx, t, T, k, E) : 0ull;
  for (int e = 0; e < E; ++e) {
    const unsigned b = __ballot_sync(0xffffffffu, (mask >> e) & 1ull);
    if (lane == 0 && b) atomicAdd(&wcnt[e], __popc(b));
  }
  __syncthreads();
  // Integer counts: the order the additions land in does not matter.
  if (tid < E && wcnt[tid]) atomicAdd(&counts[tid], wcnt[tid]);
}

__global__ void rank_prefix_kernel(const int32_t* __restrict__ gathered, int n_ranks, int E,
                                   int rank, int32_t* __restrict__ prior) {
  const int e = threadIdx.x;
  if (e >= E) return;
  int s = 0;
  for (int r = 0; r < rank && r < n_ranks; ++r) s += gathered[(int64_t)r * E + e];
  prior[e] = s;
}
}  // namespace

cudaError_t launch_expert_counts(const int32_t* idx, int T, int E, int k, int32_t* counts,
                                 cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s);
  if (err != cudaSuccess || T == 0) return err;
  expert_count_kernel<<<(T + kPermBlock - 1) / kPermBlock, kPermBlock, 0, s>>>(idx, T, E, k,
                                                                               counts);
  return cudaGetLastError();
}

cudaError_t launch_rank_prefix(const int32_t* gathered, int n_ranks, int E, int rank,
                               int32_t* prior, cudaStream_t s) {
  rank_prefix_kernel<<<1, kMaxE, 0, s>>>(gathered, n_ranks, E, rank, prior);
  return cudaGetLastError();
}

cudaError_t launch_permute(const PermuteArgs& a, moe_dtype dtype, cudaStream_t s) {
  if (a.T == 0) {
    // Still produce well-defined counts/offsets for an empty batch.
    cudaError_t err = cudaMemsetAsync(a.counts, 0, sizeof(int32_t) * a.E, s);
    if (err == cudaSuccess) err = cudaMemsetAsync(a.kept_counts, 0, sizeof(int32_t) * a.E, s);
    if (err == cudaSuccess) err = cudaMemsetAsync(a.offsets, 0, sizeof(int32_t) * (a.E + 1), s);
    return err;
  }
  const int nblk = (a.T + kPermBlock - 1) / kPermBlock;
  cudaError_t err = cudaSuccess;
  if (!a.ticket_zeroed) {
    err = cudaMemsetAsync(a.ticket, 0, sizeof(unsigned int), s);
    if (err != cudaSuccess) return err;
  }
  int32_t* cap = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(a.ticket) + 256);
  err = launch_kernel(permute_count_kernel, dim3(nblk), dim3(kPermBlock), 0, s, 1, true, a.idx,
                      a.order, a.T, a.E, a.k, a.capacity, a.prior, nblk, a.block_base, a.ticket,
                      cap, a.counts, a.kept_counts, a.offsets);
  if (err != cudaSuccess) return err;
  err = launch_kernel(permute_rank_kernel, dim3(nblk), dim3(kPermBlock), 0, s, 1, true, a.idx,
                      a.order, a.T, a.E, a.k, static_cast<const int32_t*>(cap),
                      static_cast<const int32_t*>(a.block_base),
                      static_cast<const int32_t*>(a.offsets), a.pos);
  if (err != cudaSuccess) return err;
  return launch_row_copy(a.x, a.pos, a.T, a.k, a.d, dtype, a.xp, s);
}

cudaError_t launch_row_copy(const void* x, const int32_t* pos, int T, int npos, int d,
                            moe_dtype dtype, void* xp, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int dvec = d * (dtype == MOE_BF16 ? 2 : 4) / 16;
  return launch_kernel(row_copy_kernel, dim3((T + kCopyWarps - 1) / kCopyWarps),
                       dim3(kCopyWarps * 32), 0, s, 1, true, static_cast<const uint4*>(x), pos, T,
                       npos, dvec, static_cast<uint4*>(xp));
}

// ------------------------------------------------------------------------
// The permutation over the router's token ranges (route_ranges).  Ranks are
// counted once per range -- by the streaming router as it selects, or by
// ranked_local_kernel -- and ranked_place_copy_kernel turns a (token, slot)
// with expert e and local rank lr into row offsets[e] + base_c[e] + lr, where
// base_c[e] sums the counts of the ranges before c; it is kept when that
// queue place is below the expert's capacity.  Every CTA of the second
// kernel recomputes the prefix it needs from the [G, E] count table (a few
// KB, read from L2), so no counter, ticket or second launch orders them, and
// nothing decided by atomics: the placement is deterministic.
namespace {

constexpr int kRankThreads = 256;
constexpr int kRankWarps = kRankThreads / 32;
constexpr int kPlaceWarps = 8;

__device__ __forceinline__ void range_of(int c, int G, int T8, int T, int& r0, int& r1) {
  r0 = static_cast<int>(static_cast<int64_t>(c) * T8 / G) * 8;
  r1 = min(T, static_cast<int>(static_cast<int64_t>(c + 1) * T8 / G) * 8);
}

// One CTA per range: queue positions [r0, r1) (position i serves token
// order[i], or i), 256 at a time, one thread each.  Writes lrank[t, j] (the
// rank among the range's earlier assignments to the same expert; -1 for an
// expert id outside [0, E)) and hist[c, e].
__global__ void __launch_bounds__(kRankThreads)
    ranked_local_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ order,
                        int T, int E, int k, int G, int T8, int32_t* __restrict__ lrank,
                        int32_t* __restrict__ hist) {
  __shared__ int cnt[kMaxE];
  __shared__ int wcnt[kRankWarps][kMaxE];
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  int r0, r1;
  range_of(c, G, T8, T, r0, r1);
  if (tid < E) cnt[tid] = 0;
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  for (int base = r0; base < r1; base += kRankThreads) {
    const int i = base + tid;
    const int t = i < r1 ? (order ? order[i] : i) : -1;
    // Slot arrays indexed only by unrolled loops up to kMaxK (registers).
    int ej[kMaxK], rj[kMaxK];
    uint64_t mask = 0;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      ej[j] = (t >= 0 && j < k) ? idx[(int64_t)t * k + j] : -1;
      rj[j] = -1;
      if (ej[j] >= 0 && ej[j] < E) mask |= 1ull << ej[j];
    }
    for (int e = 0; e < E; ++e) {
      const unsigned b = __ballot_sync(0xffffffffu, (mask >> e) & 1ull);
      if (lane == 0) wcnt[warp][e] = __popc(b);
      const int r = __popc(b & lt);
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) rj[j] = ((mask >> e) & 1ull) && ej[j] == e ? r : rj[j];
    }
    __syncthreads();
    if (t >= 0) {
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        if (j < k) {
          int r = -1;
          if (rj[j] >= 0) {
            const int e = ej[j];
            r = cnt[e] + rj[j];
            for (int w = 0; w < warp; ++w) r += wcnt[w][e];
          }
          lrank[(int64_t)t * k + j] = r;
        }
      }
    }
    __syncthreads();
    if (tid < E) {
      int sum = 0;
#pragma unroll
      for (int w = 0; w < kRankWarps; ++w) sum += wcnt[w][tid];
      cnt[tid] += sum;
    }
    __syncthreads();
  }
  if (tid < E) hist[(int64_t)c * E + tid] = cnt[tid];
}

// S CTAs per range.  Prologue: the prefix of the count table over the ranges
// before this one, the totals, the capacities (C, or C - prior[e] for a
// shard of a batch), kept counts and 128-row aligned offsets; CTA 0 writes
// counts, kept_counts and offsets.  Then one warp per queue position of
// this CTA's share of the range: pos[t, j] (in: local rank, out: row or -1)
// and the copy of x[t] to every kept row, reading the row once.  BULK: the
// warp copies the row into one of its two shared-memory row slots
// (cp.async), then one bulk store per kept row carries it out and is left
// in flight while the warp loads its next token into the other slot (the
// copy engine keeps far more bytes in flight than the threads' registers
// could).  Otherwise: 16-byte vectors, eight in flight per lane.
template <bool BULK>
__global__ void __launch_bounds__(kPlaceWarps * 32)
    ranked_place_copy_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ idx,
                             const int32_t* __restrict__ order, int T, int E, int k, int G, int T8,
                             int S, int C, const int32_t* __restrict__ prior,
                             const int32_t* __restrict__ hist, int32_t* __restrict__ pos,
                             int dvec, uint4* __restrict__ xp, int32_t* __restrict__ counts,
                             int32_t* __restrict__ kept_counts, int32_t* __restrict__ offsets) {
  __shared__ int red_b[kPlaceWarps * 32], red_t[kPlaceWarps * 32];
  __shared__ int s_base[kMaxE], s_cap[kMaxE], s_off[kMaxE + 1], s_kept[kMaxE];
  __shared__ int dst[kPlaceWarps][kMaxK];
  extern __shared__ __align__(128) uint8_t s_rows[];  // BULK: [warp][2][row bytes]
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x / S, sub = blockIdx.x - c * S;
  {
    // Thread (part, e) sums ranges part, part + parts, ... of column e.
    const int parts = (kPlaceWarps * 32) / E;
    const int e = tid % E, part = tid / E;
    int sb = 0, st = 0;
    if (part < parts) {
      for (int q = part; q < G; q += parts) {
        const int v = hist[(int64_t)q * E + e];
        st += v;
        sb += q < c ? v : 0;
      }
    }
    red_b[tid] = sb;
    red_t[tid] = st;
    __syncthreads();
    if (tid < E) {
      int b = 0, tot = 0;
      for (int q = 0; q < parts; ++q) {
        b += red_b[q * E + tid];
        tot += red_t[q * E + tid];
      }
      int cap = C;
      if (prior && C != INT32_MAX) cap = max(0, C - prior[tid]);
      s_base[tid] = b;
      s_cap[tid] = cap;
      s_kept[tid] = tot < cap ? tot : cap;
      if (blockIdx.x == 0) {
        counts[tid] = tot;
        kept_counts[tid] = s_kept[tid];
      }
    }
    __syncthreads();
    if (tid == 0) {
      int off = 0;
      for (int q = 0; q < E; ++q) {
        s_off[q] = off;
        off += (s_kept[q] + kRowAlign - 1) / kRowAlign * kRowAlign;
      }
      s_off[E] = off;
    }
    __syncthreads();
    if (blockIdx.x == 0 && tid <= E) offsets[tid] = s_off[tid];
  }
  int r0, r1;
  range_of(c, G, T8, T, r0, r1);
  const int len = r1 - r0;
  const int q0 = r0 + static_cast<int>(static_cast<int64_t>(sub) * len / S);
  const int q1 = r0 + static_cast<int>(static_cast<int64_t>(sub + 1) * len / S);
  const unsigned lt = (1u << lane) - 1u;
  const uint32_t row_bytes = static_cast<uint32_t>(dvec) * 16u;
  const uint32_t slot0 = smem_u32(s_rows) + static_cast<uint32_t>(warp) * 2u * row_bytes;
  int nrow = 0;  // BULK: rows this warp has loaded
  for (int i = q0 + warp; i < q1; i += kPlaceWarps) {
    const int t = order ? order[i] : i;
    int p = -1;
    if (lane < k) {
      const int e = idx[(int64_t)t * k + lane];
      const int lr = pos[(int64_t)t * k + lane];
      if (e >= 0 && e < E && lr >= 0) {
        // Kept when the queue place is below the capacity; comparing with
        // the kept count min(count, capacity) also bounds the row by
        // offsets[E] whatever the local ranks hold.
        const int r = s_base[e] + lr;
        if (r < s_kept[e]) p = s_off[e] + r;
      }
      pos[(int64_t)t * k + lane] = p;
    }
    const unsigned b = __ballot_sync(0xffffffffu, p >= 0);
    if (p >= 0) dst[warp][__popc(b & lt)] = p;
    const int nd = __popc(b);
    __syncwarp();
    if (BULK && nd > 0) {
      const uint32_t slot = slot0 + static_cast<uint32_t>(nrow & 1) * row_bytes;
      // The bulk stores from this slot (two rows ago) have read it.
      if (lane == 0 && nrow >= 2) bulk_wait_read<1>();
      __syncwarp();
      const uint4* src = x + (int64_t)t * dvec;
      for (int v = lane; v < dvec; v += 32) cp_async16(slot + v * 16, src + v, 16);
      cp_async_commit();
      cp_async_wait<0>();
      // The row is in shared memory (every lane's copies); make it visible
      // to the copy engine, then one bulk store per kept row.
      fence_async_shared();
      __syncwarp();
      if (lane == 0) {
        for (int j = 0; j < nd; ++j)
          bulk_store_1d(xp + (int64_t)dst[warp][j] * dvec, slot, row_bytes);
        bulk_commit();
      }
      ++nrow;
    } else if (nd > 0) {
      const uint4* src = x + (int64_t)t * dvec;
      for (int v0 = lane; v0 < dvec; v0 += 32 * 8) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (v0 + u * 32 < dvec) v[u] = __ldcs(src + v0 + u * 32);
        for (int j = 0; j < nd; ++j) {
          uint4* out = xp + (int64_t)dst[warp][j] * dvec;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (v0 + u * 32 < dvec) out[v0 + u * 32] = v[u];
        }
      }
    }
    __syncwarp();
  }
  // Every bulk store has finished with its slot before the CTA (and its
  // shared memory) goes away.
  if (BULK && lane == 0) bulk_wait<0>();
}

}  // namespace

size_t ranked_permute_scratch_bytes(int E) {
  return static_cast<size_t>(kMaxRouteRanges) * static_cast<size_t>(E) * sizeof(int32_t);
}

cudaError_t launch_ranked_permute(const RankedPermuteArgs& a, moe_dtype dtype, cudaStream_t s) {
  if (a.T == 0) {
    cudaError_t err = cudaMemsetAsync(a.counts, 0, sizeof(int32_t) * a.E, s);
    if (err == cudaSuccess) err = cudaMemsetAsync(a.kept_counts, 0, sizeof(int32_t) * a.E, s);
    if (err == cudaSuccess) err = cudaMemsetAsync(a.offsets, 0, sizeof(int32_t) * (a.E + 1), s);
    return err;
  }
  const RouteRanges rg = route_ranges(a.T, a.num_sms);
  cudaError_t err = cudaSuccess;
  if (!a.ranked) {
    err = launch_kernel(ranked_local_kernel, dim3(rg.G), dim3(kRankThreads), 0, s, 1, true, a.idx,
                        a.order, a.T, a.E, a.k, rg.G, rg.T8, a.pos, a.hist);
    if (err != cudaSuccess) return err;
  }
  // About four CTAs per SM over all ranges, each range's share at least a
  // few tokens.
  const int per_range = (rg.T8 * 8 + rg.G - 1) / rg.G;
  const int dvec = a.d * (dtype == MOE_BF16 ? 2 : 4) / 16;
  // Bulk copies when two row slots per warp fit beside three CTAs per SM
  // (rows up to 8 KB: d <= 4096 in bf16); as many CTAs per range as fill
  // the SMs once, so no CTA repeats the prologue in a second wave.
  const size_t slots = static_cast<size_t>(kPlaceWarps) * 2 * dvec * 16;
  const int per_sm = slots == 0 ? 4 : static_cast<int>(std::min<size_t>(4, (227u << 10) / slots));
  const bool bulk = place_bulk() && per_sm >= 1 && slots <= (128u << 10);
  const int fill = bulk ? per_sm : 4;
  const int S = std::max(1, std::min({8, (fill * a.num_sms) / rg.G, per_range / 4}));
  if (bulk) {
    static const cudaError_t attr = cudaFuncSetAttribute(
        ranked_place_copy_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, 128 << 10);
    if (attr != cudaSuccess) return attr;
    return launch_kernel(ranked_place_copy_kernel<true>, dim3(rg.G * S), dim3(kPlaceWarps * 32),
                         slots, s, 1, true, static_cast<const uint4*>(a.x), a.idx, a.order, a.T,
                         a.E, a.k, rg.G, rg.T8, S, a.capacity, a.prior,
                         static_cast<const int32_t*>(a.hist), a.pos, dvec,
                         static_cast<uint4*>(a.xp), a.counts, a.kept_counts, a.offsets);
  }
  return launch_kernel(ranked_place_copy_kernel<false>, dim3(rg.G * S), dim3(kPlaceWarps * 32), 0,
                       s, 1, true, static_cast<const uint4*>(a.x), a.idx, a.order, a.T, a.E, a.k,
                       rg.G, rg.T8, S, a.capacity, a.prior, static_cast<const int32_t*>(a.hist),
                       a.pos, dvec, static_cast<uint4*>(a.xp), a.counts, a.kept_counts, a.offsets);
}

bool place_bulk() {
  static const bool on = [] {
    const char* v = getenv("MOE_PLACE_BULK");
    return !(v && v[0] == '0');
  }();
  return on;
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("MOE_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

}  // namespace moe
