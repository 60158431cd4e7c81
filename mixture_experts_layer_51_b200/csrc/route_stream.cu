// Router for bf16 layers with E % 8 == 0: logits = x . W_g (+ bias), TopK
// and the gating softmax (or the expert-choice affinities) in one persistent
// kernel that streams x from HBM at the rate of a plain read.
//
// Pages: "How do Mixture of Expert Models Work?", "The Math Behind MoEs"
// (G(x) = Softmax(TopK(x . W_g))); "[Paper Club] Upcycling Large Language
// Models into Mixture of Experts" (one learnable router matrix; tokens of an
// expert are gathered into one block, Megatron-Core's fused permutation).
// The OpenMoE issue "Some questions want to know" notes that routing made
// of many small kernels and one-hot vectors runs at low utilisation: here
// the contraction, the selection and the first half of the permutation's
// bookkeeping share one launch, and the logits never leave the chip.
//
// The router reads every byte of x once and does ~E flop per byte, so HBM
// bounds it and the design question is bytes in flight.  One CTA per SM
// owns a contiguous range of tokens (whole 8-row groups, so ranges differ by
// at most 8 rows); a producer warp keeps a ring of TMA loads in flight --
// 64-column boxes of the range's rows (128-byte swizzle) and the matching
// rows of W_g -- about 190 KB per SM.  The contraction: for E <= 16 eight
// warps with mma.sync (m16n8k16, fp32 accumulate; each warp a 16-row tile
// and a share of every stage's K range, so no warp's dependent chain sets
// the pace); for larger E one thread issuing tcgen05.mma into tensor memory
// (N = 64), because eight warps re-reading a 64-expert W_g tile from shared
// memory would be bound by shared-memory bandwidth.  After the last stage of
// a tile of up to 128 rows the logits go to shared memory and the tile's
// tokens select (route_select.cuh).
//
// With `lrank`/`hist` the kernel also does the counting half of the
// permutation: for every selected (token, slot) its rank among the
// assignments to the same expert earlier in this CTA's range (lrank, in the
// shape of idx), and per CTA the number of assignments per expert (hist
// [G, E]).  The permutation kernel turns them into positions with a prefix
// over the CTAs -- no atomics, so placement is deterministic.
//
// Every mbarrier wait is bounded; on time-out the kernel sets a bit in the
// error word (when one is given), stops consuming, lets issued copies land
// and leaves.  No TMA multicast.

#include <math.h>
#include <stdlib.h>

#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "moe_internal.cuh"
#include "route_select.cuh"

namespace moe {
namespace {

constexpr int kRsConsumerWarps = 8;                        // epilogue / mma.sync warps
constexpr int kRsThreads = (kRsConsumerWarps + 1) * 32;     // + one producer warp
constexpr int kRsTcThreads = (kRsConsumerWarps + 2) * 32;   // + producer + MMA warp
constexpr int kRsMaxStages = 8;
constexpr int kRsMaxRows = 128;   // rows of one tile
constexpr int kRsSmemLimit = 232448;
constexpr int kRsTcN = 64;        // tcgen05 accumulator columns (experts, zero past E)

struct RsCtl {
  uint64_t full[kRsMaxStages];
  uint64_t empty[kRsMaxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
  float bias_s[kMaxE];               // the router bias (0 without one)
  int cnt[kMaxE];                    // assignments per expert so far in this range
  int wcnt[4][kMaxE];                // per-warp counts of the current tile
  int idx_s[kRsMaxRows][kMaxK];      // the tile's selected experts
  float rowstat[kRsMaxRows][2];      // expert choice: max and 1/sum per token
};

struct RsParams {
  int T, d, E, k;
  int G;            // CTAs = token ranges
  int T8;           // ceil(T / 8)
  int MT;           // rows per tile (multiple of 8, <= 128)
  int nch;          // 64-column chunks per stage
  int nk;           // stages per tile
  int stages;
  int a_chunk;      // bytes of one x chunk (MT rows x 128 bytes)
  int b_off;        // offset of the W_g rows in a stage
  int stage_bytes;  // bytes per stage (a multiple of 1024)
  int tx_bytes;     // bytes the x boxes of one stage deliver
  const uint8_t* wg;  // W_g [d, E] (for the bulk copies)
  int wg_bulk;      // 1: W_g rows by one untiled bulk copy per stage (dense [KC][E])
  int logit_off;    // offset of the logits buffer (mma.sync: the K-split partials)
  int ctl_off;      // offset of the control block
  int ls;           // logits row stride (floats)
  int nsplit;       // mma.sync: warps sharing a row tile's K range
  const float* bias;
  int32_t* idx;
  float* gate;
  float* margin;
  int gating;
  float gate_scale;
  float* scores;    // non-null: expert-choice affinities [E, T] instead of TopK
  int32_t* lrank;   // nullable: ranks within the range, [T, k]
  int32_t* hist;    // nullable: per-range counts, [G, E]
  int32_t* err;     // nullable: device error word
};

__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kRsConsumerWarps * 32) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void range_rows(const RsParams& p, int cta, int& r0, int& r1) {
  r0 = static_cast<int>(static_cast<int64_t>(cta) * p.T8 / p.G) * 8;
  r1 = min(p.T, static_cast<int>(static_cast<int64_t>(cta + 1) * p.T8 / p.G) * 8);
}

// The TMA producer (one thread): for every tile of the range and every K
// stage, wait for the stage to be free, then load the stage's x chunks
// (boxes of 64 columns x MT rows) and W_g rows onto its full barrier.
// Afterwards it waits until every issued copy has landed, so the shared
// memory outlives them even after an abort.
__device__ __forceinline__ void rs_produce(const CUtensorMap* tmX, const CUtensorMap* tmW,
                                           const RsParams& p, RsCtl& c, uint32_t smem_base,
                                           int r0, int ntiles) {
  const uint32_t full0 = smem_u32(&c.full[0]);
  const uint32_t empty0 = smem_u32(&c.empty[0]);
  int stage = 0, nissued = 0;
  uint32_t phase = 0;
  bool timed_out = false;
  for (int mt = 0; mt < ntiles; ++mt) {
    const int row = r0 + mt * p.MT;
    for (int kb = 0; kb < p.nk; ++kb) {
      if (c.abort_flag || !mbar_wait(empty0 + 8 * stage, phase ^ 1)) {
        timed_out = !c.abort_flag;
        c.abort_flag = 1;
        break;
      }
      const uint32_t full = full0 + 8 * stage;
      const uint32_t dst = smem_base + stage * p.stage_bytes;
      const int col0 = kb * p.nch * 64;
      // W_g rows col0 .. col0 + KC - 1 (those below d): contiguous when the
      // shared-memory rows are dense, so one untiled copy; a tensor box
      // (zero past d and E) otherwise.
      const int wrows = min(p.nch * 64, p.d - col0);
      const uint32_t wbytes = static_cast<uint32_t>(wrows) * p.E * 2;
      mbar_arrive_expect_tx(full, p.tx_bytes + (p.wg_bulk ? wbytes : 0u));
      for (int ch = 0; ch < p.nch; ++ch)
        tma_load_2d(dst + ch * p.a_chunk, tmX, full, col0 + ch * 64, row);
      if (p.wg_bulk)
        bulk_load_1d(dst + p.b_off, p.wg + static_cast<int64_t>(col0) * p.E * 2, wbytes, full);
      else
        tma_load_2d(dst + p.b_off, tmW, full, 0, col0);
      ++nissued;
      if (++stage == p.stages) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (c.abort_flag) break;
  }
  if (timed_out && p.err) atomicOr(p.err, kErrTimeoutProducer);
  // Stage s was filled (nissued - 1 - s) / stages + 1 times.
  for (int s = 0; s < p.stages && s < nissued; ++s) {
    const int fills = (nissued - 1 - s) / p.stages + 1;
    if (!mbar_wait(full0 + 8 * s, static_cast<uint32_t>(fills - 1) & 1u) && p.err)
      atomicOr(p.err, kErrTimeoutDrain);
  }
}

// Transposes the warp's 32 x 32 bit matrix whose row i is lane i's word:
// afterwards bit i of lane j's word is bit j of lane i's word before.  Five
// exchange steps; in step s, lanes i and i ^ s swap the s x s blocks off the
// diagonal.  All lanes of the warp must call it.
__device__ __forceinline__ uint32_t transpose_bits32(uint32_t x, int lane) {
  constexpr uint32_t kHigh[5] = {0xFFFF0000u, 0xFF00FF00u, 0xF0F0F0F0u, 0xCCCCCCCCu, 0xAAAAAAAAu};
#pragma unroll
  for (int q = 0; q < 5; ++q) {
    const int sh = 16 >> q;
    const uint32_t m = kHigh[q];
    const uint32_t y = __shfl_xor_sync(0xffffffffu, x, sh);
    x = (lane & sh) ? ((x & m) | ((y >> sh) & ~m)) : ((x & ~m) | ((y << sh) & m));
  }
  return x;
}

// After a tile's logits (bias added) are in shared memory: the tile's
// tokens select (or, for expert choice, write their affinities), and with
// lrank they are ranked among the range's assignments in token order.  All
// kRsConsumerWarps warps call it together (it synchronises them).
template <int KM>
__device__ __forceinline__ void rs_tile_epilogue(const RsParams& p, RsCtl& c,
                                                 const float* logits, int row0, int rows,
                                                 bool aborted) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Selection: P threads per token; every consumer thread takes part (the
  // shuffles need whole warps), threads past the tile only read.
  const int P = p.MT <= 32 ? 8 : (p.MT <= 64 ? 4 : 2);
  const int rr = tid / P, pp = tid % P;
  const bool valid = !aborted && rr < rows;
  const float* lrow = logits + min(rr, rows - 1) * p.ls;
  if (p.scores) {
    float m, inv;
    softmax_stats(lrow, p.E, P, pp, m, inv);
    if (valid && pp == 0) {
      c.rowstat[rr][0] = m;
      c.rowstat[rr][1] = inv;
    }
    consumer_sync();
    // Expert-major scores[e, t], consecutive threads on consecutive tokens,
    // each value recomputed from the same logit, maximum and reciprocal.
    if (!aborted) {
      for (int i = tid; i < rows * p.E; i += kRsConsumerWarps * 32) {
        const int e = i / rows, r2 = i - e * rows;
        p.scores[static_cast<int64_t>(e) * p.T + row0 + r2] =
            expf(logits[r2 * p.ls + e] - c.rowstat[r2][0]) * c.rowstat[r2][1];
      }
    }
    consumer_sync();
    return;
  }
  select_token<KM>(lrow, p.E, p.k, P, pp, row0 + rr, valid, p.gating, p.gate_scale, p.idx,
                   p.gate, p.margin, valid ? c.idx_s[rr] : nullptr);
  consumer_sync();  // idx_s complete; the logits buffer is free for the next tile
  if (!p.lrank) return;

  // Ranks among this range's assignments to the same expert, in token
  // order: one thread per token of the tile (warps 0-3).  Each lane holds
  // the set of its experts as a 64-bit mask; transposing the warp's 32 x 64
  // bit matrix leaves in lane j the set of lanes that chose expert j (low
  // word) and expert 32 + j (high word) -- what a ballot per expert would
  // give, for about a tenth of the instructions.  A lane's rank for expert e
  // is the number of earlier lanes in e's set; the warps below come from
  // shared counts, earlier tiles from the running per-expert count.
  // (The slot loops run to the compile-time bound KM - 1 >= k, so the slot
  // arrays stay in registers.)
  constexpr int KS = KM - 1;
  uint64_t mask = 0;
  int ej[KS], rj[KS];
  const bool have = !aborted && warp < 4 && tid < rows;
  if (warp < 4) {
#pragma unroll
    for (int j = 0; j < KS; ++j) {
      ej[j] = (have && j < p.k) ? c.idx_s[tid][j] : -1;
      rj[j] = 0;
      if (ej[j] >= 0) mask |= 1ull << ej[j];
    }
    uint32_t lo = static_cast<uint32_t>(mask), hi = static_cast<uint32_t>(mask >> 32);
    lo = transpose_bits32(lo, lane);
    if (p.E > 32) hi = transpose_bits32(hi, lane);  // zero otherwise
    if (lane < p.E) c.wcnt[warp][lane] = __popc(lo);
    if (lane + 32 < p.E) c.wcnt[warp][lane + 32] = __popc(hi);
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < KS; ++j) {
      const int e = ej[j];
      const unsigned blo = __shfl_sync(0xffffffffu, lo, e & 31);
      const unsigned bhi = __shfl_sync(0xffffffffu, hi, e & 31);
      rj[j] = __popc((e >= 32 ? bhi : blo) & lt);  // used only where e >= 0
    }
  }
  consumer_sync();
  if (have) {
#pragma unroll
    for (int j = 0; j < KS; ++j) {
      if (j < p.k) {
        const int e = ej[j];
        int r = c.cnt[e] + rj[j];
        for (int w = 0; w < warp; ++w) r += c.wcnt[w][e];
        p.lrank[static_cast<int64_t>(row0 + tid) * p.k + j] = r;
      }
    }
  }
  consumer_sync();
  if (tid < p.E) c.cnt[tid] += c.wcnt[0][tid] + c.wcnt[1][tid] + c.wcnt[2][tid] + c.wcnt[3][tid];
  consumer_sync();
}

__device__ __forceinline__ void rs_init(const RsParams& p, RsCtl& c, int empty_count) {
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(smem_u32(&c.full[s]), 1);
      mbar_init(smem_u32(&c.empty[s]), empty_count);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&c.tfull[a]), 1);
      mbar_init(smem_u32(&c.tempty[a]), 4);
    }
    mbar_init(smem_u32(&c.drain), 1);
    c.abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < kMaxE) c.cnt[threadIdx.x] = 0;
}

// mma.sync back end, for E <= 16 (NT = 1 or 2 column tiles of 8 experts;
// W_g rows dense in shared memory, NT * 16 bytes each, loaded by one
// untiled bulk copy per stage).  The warps split a tile as nrt row tiles of 16 x nsplit shares of
// each stage's 64-column chunks; each keeps two accumulator chains (even and
// odd 16-wide K steps) and loads a chunk's fragments before its MMAs.  The
// shares' partial logits are summed in a fixed order: deterministic.
template <int NT, int KM>
__global__ void __launch_bounds__(kRsThreads, 1)
    route_stream_kernel(const __grid_constant__ CUtensorMap tmX,
                        const __grid_constant__ CUtensorMap tmW, const RsParams p) {
  static_assert(NT == 1 || NT == 2, "mma.sync back end: E <= 16");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  RsCtl& c = *reinterpret_cast<RsCtl*>(smem + p.ctl_off);
  float* part = reinterpret_cast<float*>(smem + p.logit_off);  // [nsplit][MT][ls]
  constexpr int RB = NT * 16;             // bytes per (dense) W_g row in shared memory
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int r0, r1;
  range_rows(p, blockIdx.x, r0, r1);
  const int ntiles = (r1 - r0 + p.MT - 1) / p.MT;
  const int nrt = (p.MT + 15) / 16;
  const int nbusy = nrt * p.nsplit;
  const uint32_t smem_base = smem_u32(smem);

  rs_init(p, c, nbusy);
  // The last stage of a tile may carry fewer than KC rows of W_g; the rows
  // past d then keep whatever an earlier stage left there (finite weights,
  // multiplied by the zeros the x boxes hold past d) -- but never the
  // uninitialised contents of shared memory.
  for (int s = 0; s < p.stages; ++s) {
    uint4* wz = reinterpret_cast<uint4*>(smem + s * p.stage_bytes + p.b_off);
    for (int i = tid; i < p.nch * 64 * RB / 16; i += kRsThreads) wz[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  fence_async_shared();
  if (warp == kRsConsumerWarps && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  __syncthreads();
  // x and W_g may be written by the previous kernel in the stream.
  pdl_wait();
  pdl_trigger();

  if (warp == kRsConsumerWarps) {
    if (lane == 0) rs_produce(&tmX, &tmW, p, c, smem_base, r0, ntiles);
    return;
  }
  // The bias in shared memory (read after the first consumer barrier).
  if (tid < p.E) c.bias_s[tid] = p.bias ? p.bias[tid] : 0.f;

  const uint32_t full0 = smem_u32(&c.full[0]);
  const uint32_t empty0 = smem_u32(&c.empty[0]);
  const bool busy = warp < nbusy;
  const int rt = warp % nrt, ksh = warp / nrt;
  const int r = rt * 16 + (lane & 15);  // may pass MT: those rows are never kept
  const int plane = p.MT * p.ls;        // floats per partial
  int stage = 0;
  uint32_t phase = 0;
  for (int mt = 0; mt < ntiles; ++mt) {
    const int row0 = r0 + mt * p.MT;
    const int rows = min(p.MT, r1 - row0);
    float acc[2][NT][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[h][n][i] = 0.f;
    for (int kb = 0; kb < p.nk; ++kb) {
      if (busy) {
        bool ok = !c.abort_flag;
        if (ok && !mbar_wait(full0 + 8 * stage, phase)) {
          if (p.err) atomicOr(p.err, kErrTimeoutMma);
          c.abort_flag = 1;
          ok = false;
        }
        if (ok) {
          const uint32_t a_base = smem_base + stage * p.stage_bytes;
          const uint32_t b_base = a_base + p.b_off;
          for (int ch = ksh; ch < p.nch; ch += p.nsplit) {
            const uint32_t a_row = a_base + ch * p.a_chunk + r * 128;
            uint32_t a[4][4], b[4][NT][2];
#pragma unroll
            for (int q = 0; q < 4; ++q)
              ldsm_x4(a_row + ((((q * 2) + (lane >> 4)) ^ (r & 7)) << 4), a[q]);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int krow = ch * 64 + q * 16 + (lane & 15);
              const uint32_t b_row = b_base + krow * RB;
              if (NT == 2)
                ldsm_x4_t(b_row + ((lane >> 4) << 4), b[q][0][0], b[q][0][1], b[q][NT - 1][0],
                          b[q][NT - 1][1]);
              else
                ldsm_x2_t(b_row, b[q][0][0], b[q][0][1]);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int n = 0; n < NT; ++n) mma_16816(acc[q & 1][n], a[q], b[q][n][0], b[q][n][1]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * stage);
      }
      if (++stage == p.stages) {
        stage = 0;
        phase ^= 1;
      }
    }

    // Each share's partial logits, then their sum in share order plus the
    // bias, into share 0's plane.
    if (busy) {
      float* pl = part + ksh * plane;
      const int rr = rt * 16 + (lane >> 2);
      const int cc = (lane & 3) * 2;
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = rr + 8 * h;
          if (row < rows) {
            pl[row * p.ls + n * 8 + cc] = acc[0][n][2 * h] + acc[1][n][2 * h];
            pl[row * p.ls + n * 8 + cc + 1] = acc[0][n][2 * h + 1] + acc[1][n][2 * h + 1];
          }
        }
    }
    consumer_sync();
    for (int i = tid; i < rows * p.ls; i += kRsConsumerWarps * 32) {
      const int e = i % p.ls;
      if (e >= p.E) continue;
      float v = part[i];
      for (int q = 1; q < p.nsplit; ++q) v += part[q * plane + i];
      part[i] = p.bias ? v + c.bias_s[e] : v;
    }
    consumer_sync();
    rs_tile_epilogue<KM>(p, c, part, row0, rows, c.abort_flag != 0);
  }
  if (p.hist && tid < p.E) p.hist[static_cast<int64_t>(blockIdx.x) * p.E + tid] = c.cnt[tid];
}

// tcgen05 back end, for E > 16: one thread issues tcgen05.mma (M = 128 rows
// of the tile -- rows past MT read whatever follows in shared memory and are
// never kept -- N = 64 experts, zero past E; K = 16; fp32 accumulate in
// tensor memory, two accumulators so a tile's epilogue overlaps the next
// tile's MMAs).  Warps 0-3 read the accumulator (TMEM lane = tile row) into
// the logits buffer.
template <int KM>
__global__ void __launch_bounds__(kRsTcThreads, 1)
    route_stream_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                           const __grid_constant__ CUtensorMap tmW, const RsParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  RsCtl& c = *reinterpret_cast<RsCtl*>(smem + p.ctl_off);
  float* logits = reinterpret_cast<float*>(smem + p.logit_off);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int r0, r1;
  range_rows(p, blockIdx.x, r0, r1);
  const int ntiles = (r1 - r0 + p.MT - 1) / p.MT;
  const uint32_t smem_base = smem_u32(smem);
  constexpr int kMmaWarp = kRsConsumerWarps + 1;

  rs_init(p, c, 1);
  if (warp == kRsConsumerWarps && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&c.tmem_base), 2 * kRsTcN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  pdl_wait();
  pdl_trigger();

  if (warp == kRsConsumerWarps) {
    if (lane == 0) rs_produce(&tmX, &tmW, p, c, smem_base, r0, ntiles);
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kRsTcN, false, true);
      const uint32_t full0 = smem_u32(&c.full[0]);
      const uint32_t empty0 = smem_u32(&c.empty[0]);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool issued = false;
      for (int mt = 0; mt < ntiles && !c.abort_flag; ++mt) {
        if (!mbar_wait(smem_u32(&c.tempty[acc]), acc_phase ^ 1)) {
          if (p.err) atomicOr(p.err, kErrTimeoutMma);
          c.abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * kRsTcN);
        for (int kb = 0; kb < p.nk; ++kb) {
          if (c.abort_flag || !mbar_wait(full0 + 8 * stage, phase)) {
            if (!c.abort_flag && p.err) atomicOr(p.err, kErrTimeoutMma);
            c.abort_flag = 1;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_base + stage * p.stage_bytes;
          const uint32_t b_base = a_base + p.b_off;
          for (int ch = 0; ch < p.nch; ++ch) {
            // A: K-major rows of 128 bytes, 8-row groups 1 KB apart; B: W_g
            // rows of 64 experts (N-major), 16 K-rows = 2 KB.
            const uint64_t adesc = smem_desc_sw128(a_base + ch * p.a_chunk, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(b_base + ch * 8192, 8192, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc_mma_bf16(d_tmem, adesc + static_cast<uint64_t>((kk * 32) >> 4),
                          bdesc + static_cast<uint64_t>((kk * 2048) >> 4), idesc,
                          (kb > 0 || ch > 0 || kk > 0) ? 1u : 0u);
          }
          issued = true;
          tc_commit(empty0 + 8 * stage);
          if (++stage == p.stages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (c.abort_flag) break;
        tc_commit(smem_u32(&c.tfull[acc]));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      // Every issued MMA has completed before tensor memory is freed.
      if (issued) {
        tc_commit(smem_u32(&c.drain));
        if (!mbar_wait(smem_u32(&c.drain), 0) && p.err) atomicOr(p.err, kErrTimeoutDrain);
      }
    }
  } else {
    // The bias in shared memory (from global memory, each read would sit
    // between two logits stores it cannot pass).
    if (tid < p.E) c.bias_s[tid] = p.bias ? p.bias[tid] : 0.f;
    consumer_sync();
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int mt = 0; mt < ntiles; ++mt) {
      const int row0 = r0 + mt * p.MT;
      const int rows = min(p.MT, r1 - row0);
      if (warp < 4) {
        bool ok = !c.abort_flag;
        if (ok && !mbar_wait(smem_u32(&c.tfull[acc]), acc_phase)) {
          if (p.err) atomicOr(p.err, kErrTimeoutEpilogue);
          c.abort_flag = 1;
          ok = false;
        }
        tc_fence_after();
        float v[2][32];
        const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16) +
                               static_cast<uint32_t>(acc * kRsTcN);
        tc_ld_32cols(taddr, v[0]);
        tc_ld_32cols(taddr + 32, v[1]);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&c.tempty[acc]));
        const int row = warp * 32 + lane;
        if (ok && row < rows) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            // This half's 32 bias values read before its stores (a read
            // after a store through another float pointer would wait for
            // it); one half at a time keeps the registers to 96.
            float b[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) b[i] = p.bias ? c.bias_s[h * 32 + i] : 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int e = h * 32 + i;
              if (e < p.E) logits[row * p.ls + e] = p.bias ? v[h][i] + b[i] : v[h][i];
            }
          }
        }
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
      consumer_sync();
      rs_tile_epilogue<KM>(p, c, logits, row0, rows, c.abort_flag != 0);
    }
    if (p.hist && tid < p.E) p.hist[static_cast<int64_t>(blockIdx.x) * p.E + tid] = c.cnt[tid];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kRsTcN);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 rs_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2-D bf16 matrix [rows, cols] (cols contiguous), box box_cols x box_rows;
// parts of a box past the matrix read zeros.
bool rs_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
            uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = rs_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline int round1k(int v) { return (v + 1023) / 1024 * 1024; }

// Stage plan and launch.  EP = experts per W_g row in shared memory (8 or
// 16 for the mma.sync back end, 64 for tcgen05).  MOE_RS_NCH / MOE_RS_STAGES
// override the plan, for measurements.
cudaError_t launch_rs(const RouteArgs& a, int num_sms, cudaStream_t s) {
  const RouteRanges rg = route_ranges(a.T, num_sms);
  const bool tc = a.E > 16;
  const int EP = tc ? kRsTcN : (a.E <= 8 ? 8 : 16);
  // The fewest tiles per range.  (Two tiles on the tcgen05 path would let
  // the selection of the first overlap the streaming of the second, but each
  // tile streams all of W_g -- 64 experts wide, as large as half the range's
  // x at E = 64 -- through the same ring: measured slower, 39 vs 34 us on
  // the 16384 x 2048, E = 64, top-8 router.)  MOE_RS_TC_SPLIT=1 forces two
  // tiles, for measurements.
  static const int force_split = [] {
    const char* v = getenv("MOE_RS_TC_SPLIT");
    return v ? (v[0] == '0' ? 0 : 1) : -1;
  }();
  const int rmax = 8 * ((rg.T8 + rg.G - 1) / rg.G);
  const bool split = force_split == 1;
  const int mt_tc = split
                        ? std::min(kRsMaxRows, std::max(std::min(rmax, 32), 8 * ((rmax + 15) / 16)))
                        : rg.MT;
  RsParams p{};
  p.T = a.T;
  p.d = a.d;
  p.E = a.E;
  p.k = a.k;
  p.G = rg.G;
  p.T8 = rg.T8;
  p.MT = tc ? mt_tc : rg.MT;
  p.ls = EP + 1;
  p.a_chunk = p.MT * 128;
  const int nrt = (p.MT + 15) / 16;
  const int max_split = tc ? 1 : std::max(1, kRsConsumerWarps / nrt);
  // tcgen05 reads 128 rows from every chunk: keep what follows the last one
  // inside the allocation.
  const int slack = tc ? round1k((kRsMaxRows - p.MT) * 128) : 0;
  const int logit_bytes = round1k(max_split * p.MT * p.ls * 4);
  const int ctl_bytes = round1k(static_cast<int>(sizeof(RsCtl)));
  const int budget = kRsSmemLimit - 1024 - logit_bytes - ctl_bytes - slack;
  static const int force_nch = [] {
    const char* v = getenv("MOE_RS_NCH");
    return v ? atoi(v) : 0;
  }();
  static const int force_stages = [] {
    const char* v = getenv("MOE_RS_STAGES");
    return v ? atoi(v) : 0;
  }();
  const int chunks_d = (a.d + 63) / 64;
  auto stage_of = [&](int n) { return round1k(n * p.a_chunk) + round1k(n * 64 * EP * 2); };
  int nch = std::min(4, chunks_d);
  while (nch > 1 && budget / stage_of(nch) < 4) --nch;
  if (force_nch >= 1 && force_nch <= 4 && budget / stage_of(force_nch) >= 2) nch = force_nch;
  p.nch = nch;
  p.nk = (chunks_d + nch - 1) / nch;
  p.b_off = round1k(nch * p.a_chunk);
  p.stage_bytes = stage_of(nch);
  p.stages = std::min(kRsMaxStages, budget / p.stage_bytes);
  if (force_stages >= 2 && force_stages < p.stages) p.stages = force_stages;
  if (p.stages < 2) return cudaErrorInvalidValue;
  p.nsplit = std::min(max_split, nch);
  p.logit_off = p.stages * p.stage_bytes;
  p.ctl_off = p.logit_off + logit_bytes;
  const int smem = p.ctl_off + ctl_bytes + slack + 1024;
  p.bias = a.bias;
  p.idx = a.idx;
  p.gate = a.gate;
  p.margin = a.margin;
  p.gating = a.gating;
  p.gate_scale = a.gate_scale;
  p.scores = a.scores;
  p.lrank = a.lrank;
  p.hist = a.hist;
  p.err = a.err;
  p.wg = static_cast<const uint8_t*>(a.Wg);
  p.wg_bulk = tc ? 0 : 1;
  p.tx_bytes = nch * p.a_chunk + (tc ? nch * 64 * EP * 2 : 0);

  CUtensorMap mx, mw;
  if (!rs_map(&mx, a.x, a.T, a.d, 64, p.MT, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorInvalidValue;
  if (tc ? !rs_map(&mw, a.Wg, a.d, a.E, EP, nch * 64, CU_TENSOR_MAP_SWIZZLE_128B)
         : !rs_map(&mw, a.Wg, a.d, a.E, EP, 8, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  auto go = [&](auto kern, int threads) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(kern, dim3(p.G), dim3(threads), smem, s, 1, true, mx, mw, p);
  };
  const int km = (a.scores || a.k <= 2) ? 3 : (a.k <= 4 ? 5 : kMaxK + 1);
  if (tc) {
    if (km == 3) return go(route_stream_tc_kernel<3>, kRsTcThreads);
    if (km == 5) return go(route_stream_tc_kernel<5>, kRsTcThreads);
    return go(route_stream_tc_kernel<kMaxK + 1>, kRsTcThreads);
  }
  if (EP == 8) {
    if (km == 3) return go(route_stream_kernel<1, 3>, kRsThreads);
    if (km == 5) return go(route_stream_kernel<1, 5>, kRsThreads);
    return go(route_stream_kernel<1, kMaxK + 1>, kRsThreads);
  }
  if (km == 3) return go(route_stream_kernel<2, 3>, kRsThreads);
  if (km == 5) return go(route_stream_kernel<2, 5>, kRsThreads);
  return go(route_stream_kernel<2, kMaxK + 1>, kRsThreads);
}

}  // namespace

RouteRanges route_ranges(int T, int num_sms) {
  RouteRanges r{};
  r.T8 = (T + 7) / 8;
  r.G = std::max(1, std::min({num_sms, kMaxRouteRanges, r.T8}));
  // The longest range, in whole 8-row groups, split into tiles of <= 128 rows.
  const int rmax = 8 * ((r.T8 + r.G - 1) / r.G);
  const int ntiles = (rmax + kRsMaxRows - 1) / kRsMaxRows;
  r.MT = 8 * (((rmax / 8) + ntiles - 1) / ntiles);
  return r;
}

bool route_stream_supported(const RouteArgs& a) {
  static const int forced = [] {
    const char* v = getenv("MOE_ROUTE_STREAM");
    return v ? (v[0] == '0' ? 0 : 1) : -1;
  }();
  if (forced == 0) return false;
  return a.E % 8 == 0 && a.E <= kMaxE && a.d % 8 == 0 && a.T > 0;
}

cudaError_t launch_route_stream(const RouteArgs& a, int num_sms, cudaStream_t s) {
  return launch_rs(a, num_sms, s);
}

}  // namespace moe
