// Grouped expert FFN on the B200 5th-generation tensor cores (tcgen05).
//
// Pages: "[Paper Club] Upcycling Large Language Models into Mixture of
// Experts" -- the per-expert loop of GEMMs is replaced by one grouped GEMM
// that takes any number of experts and any number of tokens per expert;
// "How do Mixture of Expert Models Work?", "The Math Behind MoEs" -- Mixtral's
// experts are SwiGLU FFNs.  The pages name a CUTLASS grouped GEMM for this
// step but give no design; this kernel is written for sm_100a from scratch.
//
// Two launches of one persistent, warp-specialised kernel:
//   up:   h[rows, H] = SiLU(xp W1_e) * (xp W3_e)   (bf16 out; GELU variant)
//   down: o[rows, d] = h W2_e                      (bf16 out)
// Tiles are 256 rows x 256 accumulator columns, computed by a cluster of two
// CTAs (tcgen05 cta_group::2: each CTA holds 128 rows of A and half of the
// 256 B columns; the pair MMA writes each CTA's 128 rows into its own TMEM).
// For the up projection the 256 columns are 128 columns of W1 next to the
// same 128 columns of W3 (one CTA loads each), so one accumulator holds both
// halves of the SwiGLU and the epilogue writes SiLU(gate) * up directly: the
// two pre-activations never reach HBM.  MOE_TC_CTA_PAIR=0 selects one CTA
// per 128 x 256 tile instead.
//
// Roles per CTA (192 threads; 320 with MOE_EPI_WARPS=8):
//   warp 0      one thread issues TMA loads of A (K-major, 128B swizzle) and
//               B (weights [E, K, N] read N-major, 128B swizzle) into a ring
//               of three 64 KB stages of 128-wide K steps (six 32 KB stages
//               of 64-wide steps when K or N is not a multiple of 64), the
//               peer's bytes completing on the leader's barrier;
//   warp 1      the leader's thread issues tcgen05.mma (M=256, N=256, K=16,
//               bf16 in, fp32 accumulate in tensor memory) and commits stage
//               releases to both CTAs; the warp also owns the 512-column TMEM
//               allocation (two accumulators, so the epilogue of tile i
//               overlaps the MMAs of tile i+1);
//   warps 2-5   epilogue: tcgen05.ld of their 32 TMEM lanes, activation or
//               rounding to bf16, stores of the kept rows (h: 16-byte stores
//               per row; o: swizzled 32-row staging boxes and TMA stores).
//               (Eight epilogue warps, two per lane quadrant, measured no
//               faster once the SiLU division was the approximate one: the
//               IEEE division had made the SwiGLU epilogue, not the MMAs,
//               the limit of layers with K = 1024, by 1.6x.)
// The tile list (expert, m-block, n-block) is built on the device from the
// per-expert offsets, with the experts that have the most m-blocks first and
// m-blocks fastest, so concurrent CTAs share weight tiles in L2.  Every
// tile accumulates its K steps in ascending order, so a row's result does
// not depend on the other rows of the batch.  No host synchronisation is
// needed between the permutation and this kernel.
//
// Every wait on an mbarrier is bounded; on timeout a thread records an error
// bit, raises an abort flag, lets in-flight copies and MMAs land, frees TMEM
// and returns.  No TMA multicast is used anywhere.

#include <math.h>
#include <stdio.h>

#include <cudaTypedefs.h>

#include <stdlib.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int TM = 128;  // tile rows held by one CTA (UMMA M per CTA)
constexpr int TN = 256;  // accumulator columns (UMMA N)
#ifndef MOE_EPI_WARPS
#define MOE_EPI_WARPS 4
#endif
// Epilogue warps: 4 (one per TMEM lane quadrant) or 8 (two per quadrant,
// each taking half of the accumulator's columns).
constexpr int EPI_WARPS = MOE_EPI_WARPS;
static_assert(EPI_WARPS == 4 || EPI_WARPS == 8, "4 or 8 epilogue warps");
constexpr int EPI_SPLIT = EPI_WARPS / 4;  // epilogue warps per lane quadrant
constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;
constexpr uint32_t TMEM_COLS = 2 * TN;
constexpr int CONTROL_BYTES = 1536;
// Epilogue output staging: eight 4 KB boxes (32 rows x 128 bytes, 128-byte
// swizzled) that TMA stores drain to global memory; two per warp with four
// epilogue warps, one per warp with eight.
constexpr int OUT_BOX_BYTES = 32 * 128;
constexpr int OUT_BOXES_PER_WARP = 8 / EPI_WARPS;
constexpr int OUT_STAGE_BYTES = 8 * OUT_BOX_BYTES;
#ifndef MOE_PAIR_STAGES
#define MOE_PAIR_STAGES 6  // ring depth of the CTA-pair kernel with 64-wide K steps
#endif
// Shared-memory ring per K step of TKS elements (64 or 128):
//   A: 128 rows, stored as TKS/64 chunks of [128 rows][64] (16 KB each);
//   B: 4/CG chunks of 64 columns, each [TKS rows][64] (8 or 16 KB).
// One CTA per tile (CG = 1) holds all 256 B columns; a CTA pair (CG = 2)
// holds half of them per CTA.  The pair kernel with 128-wide steps has three
// 64 KB stages; with 64-wide steps six 32 KB stages; one CTA, four 48 KB.
template <int CG, int TKS>
struct Cfg {
  static constexpr int A_STAGE = TM * TKS * 2;
  static constexpr int A_CHUNK = TM * 64 * 2;
  static constexpr int B_CHUNK = 64 * TKS * 2;
  static constexpr int B_CHUNKS = 4 / CG;
  static constexpr int STAGE_BYTES = A_STAGE + B_CHUNKS * B_CHUNK;
  static constexpr int STAGES = CG == 1 ? 4 : (TKS == 64 ? MOE_PAIR_STAGES : 3);
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + OUT_STAGE_BYTES + CONTROL_BYTES + 1024;
  static_assert(SMEM_BYTES <= 232448, "more than 227 KB of shared memory");
};
constexpr int MAX_STAGES = 8;
constexpr int B_BOX_BYTES = 64 * 64 * 2;  // a 64 x 64 box (3-D fallback loads, TKS = 64)

enum Epi { EPI_SWIGLU = 0, EPI_GELU = 1, EPI_PLAIN = 2 };

struct TcParams {
  void* out;
  int64_t ld_out;  // elements per output row
  int n_out;       // valid output columns
  int K;           // reduction length
  int E;
  int n_tiles;     // column tiles per expert
  int64_t rows;    // rows of the A and output buffers
  int b_chunked;   // 1: B maps are 4-D {64, K, N/64, E}; one load covers a CTA's chunks
  const int32_t* offsets;
  const int32_t* kept;
  int32_t* err;
  int debug_stall;  // 1: the MMA issuer first waits on a barrier nobody arms (tests only)
  // 1: (CTA pairs, four epilogue warps) an expert's last block with at most
  // TM kept rows runs as an M = 128 pair tile -- 64 rows in each CTA -- so
  // its second half of padding rows is not computed.
  int half_tiles;
  // 1: the K steps of every other round of a unit run in reverse order.
  int k_serpentine;
};

struct Control {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint64_t never;  // armed by nobody: the failure-detection test waits on it
  uint32_t tmem_base;
  volatile int abort_flag;
  int total_tiles;
  int n_sched;
  int sched_e[kMaxE];
  int sched_mt[kMaxE];
  int sched_prefix[kMaxE + 1];
  int off[kMaxE];
  int kept[kMaxE];
};
static_assert(sizeof(Control) <= CONTROL_BYTES, "control block too large");

__device__ __forceinline__ void decode_tile(const Control& c, int t, int& e, int& m, int& n) {
  int s = 0;
  while (s + 1 < c.n_sched && c.sched_prefix[s + 1] <= t) ++s;
  e = c.sched_e[s];
  const int local = t - c.sched_prefix[s];
  const int mt = c.sched_mt[s];
  n = local / mt;
  m = local - n * mt;
}

// Whether the block of `m_row` (rows inside expert e's block) runs as an
// M = 128 pair tile: it is the expert's last and holds at most TM kept rows.
// Its accumulator then sits in TMEM lanes 0-63 (the CTA's 64 rows, tile
// columns 0..127) and lanes 64-127 (the same rows, columns 128..255), at
// TMEM columns 0..127.
template <int CG>
__device__ __forceinline__ bool is_half_tile(const TcParams& p, const Control& c, int e,
                                             int m_row) {
  return CG == 2 && EPI_WARPS == 4 && p.half_tiles && c.kept[e] - m_row <= TM;
}

#ifndef MOE_FAST_SILU
#define MOE_FAST_SILU 1
#endif
// SiLU(z) = z / (1 + e^-z).  The fast form divides with the approximate
// reciprocal (__fdividef): its error is a few fp32 ulps, far below the bf16
// rounding of h; for z < -88 the denominator overflows and the result is 0,
// SiLU's limit.
__device__ __forceinline__ float silu_f(float z) {
#if MOE_FAST_SILU
  return __fdividef(z, 1.0f + __expf(-z));
#else
  return z / (1.0f + __expf(-z));
#endif
}
__device__ __forceinline__ float gelu_f(float z) {
  return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
}

// CG = 1: one CTA computes a 128 x 256 tile.  CG = 2: a cluster of two CTAs
// computes a 256 x 256 tile with tcgen05 pair MMAs issued by the leader
// (rank 0): each CTA loads its own 128 rows of A and its half of the 256
// B columns; the pair MMA reads both CTAs' shared memory and writes each
// CTA's 128 accumulator rows into that CTA's tensor memory.  Stage-full and
// accumulator-empty barriers live in the leader; stage-empty and
// accumulator-full barriers in each CTA (the leader's commits reach both).
template <int EPI, int CG, int TKS>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    ffn_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                  const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmOut,
                  const TcParams p) {
  using C_ = Cfg<CG, TKS>;
  constexpr int STAGES = C_::STAGES;
  constexpr int STAGE_BYTES = C_::STAGE_BYTES;
  constexpr int A_STAGE = C_::A_STAGE;
  constexpr int B_CHUNK = C_::B_CHUNK;
  static_assert(TKS == 64 || CG == 2, "128-wide K steps only for CTA pairs");
  constexpr int TILE_M = TM * CG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Control& c = *reinterpret_cast<Control*>(smem + STAGES * STAGE_BYTES + OUT_STAGE_BYTES);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int group = blockIdx.x / CG;   // tile-processing unit (CTA or CTA pair)
  const int ngroups = gridDim.x / CG;

  // ------------------------------------------------------------ set-up
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&c.full[s]), 1);
      mbar_init(smem_u32(&c.empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&c.tfull[a]), 1);
      mbar_init(smem_u32(&c.tempty[a]), EPI_WARPS * CG);  // one arrive per epilogue warp of the group
    }
    mbar_init(smem_u32(&c.drain), 1);
    mbar_init(smem_u32(&c.never), 1);
    c.abort_flag = 0;
    fence_mbar_init();
    fence_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (EPI == EPI_SWIGLU) tma_prefetch_desc(&tmB1);
    tma_prefetch_desc(&tmOut);
  }
  if (warp == 1) {
    if (CG == 2) {
      tmem_alloc_pair(smem_u32(&c.tmem_base), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(&c.tmem_base), TMEM_COLS);
      tmem_relinquish();
    }
  }
  // Everything above overlaps the previous kernel's tail; the offsets and
  // every operand are read only after it has finished.
  pdl_wait();
  if (tid < p.E) {
    c.off[tid] = p.offsets[tid];
    c.kept[tid] = p.kept[tid];
  }
  __syncthreads();
  if (tid == 0) {
    // Schedule: experts with more m-blocks first (stable), empty ones skipped.
    int n = 0;
    for (int e = 0; e < p.E; ++e) {
      const int mt = (c.kept[e] + TILE_M - 1) / TILE_M;
      if (mt <= 0) continue;
      // An expert block must start on a 128-row boundary and its kept rows
      // must end inside the buffers; anything else is reported and skipped,
      // never written.  (Rows a pair tile reads past the block are padding
      // or the next block -- or past the buffer, where TMA reads zeros -- and
      // are never stored.)
      if (c.off[e] < 0 || (c.off[e] % TM) != 0 ||
          static_cast<int64_t>(c.off[e]) + ((c.kept[e] + TM - 1) / TM) * TM > p.rows) {
        if (leader) atomicOr(p.err, kErrRowOverflow);
        continue;
      }
      int q = n;
      while (q > 0 && c.sched_mt[q - 1] < mt) {
        c.sched_mt[q] = c.sched_mt[q - 1];
        c.sched_e[q] = c.sched_e[q - 1];
        --q;
      }
      c.sched_mt[q] = mt;
      c.sched_e[q] = e;
      ++n;
    }
    int acc = 0;
    for (int s = 0; s < n; ++s) {
      c.sched_prefix[s] = acc;
      acc += c.sched_mt[s] * p.n_tiles;
    }
    c.sched_prefix[n] = acc;
    c.n_sched = n;
    c.total_tiles = acc;
  }
  tc_fence_before();
  __syncthreads();
  if (CG == 2) cluster_sync();  // the peer's barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  const int total = c.total_tiles;
  const int nk = (p.K + TKS - 1) / TKS;
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t full0 = smem_u32(&c.full[0]);    // barriers of stage s are 8 bytes apart
  const uint32_t empty0 = smem_u32(&c.empty[0]);

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0, nissued = 0;
      uint32_t phase = 0;
      bool ok = true, timed_out = false;
      for (int t = group; t < total && ok; t += ngroups) {
        if (c.abort_flag) {
          ok = false;
          break;
        }
        int e, m, n;
        decode_tile(c, t, e, m, n);
        const bool half_m = is_half_tile<CG>(p, c, e, m * TILE_M);
        const int row0 =
            c.off[e] + m * TILE_M + static_cast<int>(rank) * (half_m ? TM / 2 : TM);
        // First 64-column chunk of this CTA's B columns (4-D weight maps).
        // SwiGLU pairs: each CTA holds one 64-column chunk of W1 next to the
        // same chunk of W3 (leader: the tile's first chunk, peer: its
        // second), so in either tile height every thread's accumulator row
        // holds the gate and the up value of the same h columns.
        const int c0 = CG == 2 ? (EPI == EPI_SWIGLU ? n * 2 + static_cast<int>(rank)
                                                    : n * 4 + 2 * static_cast<int>(rank))
                               : (EPI == EPI_SWIGLU ? n * 2 : n * 4);
        // (Opt-in) every other round of this unit runs its K steps from the
        // end: the tiles of a round then start where the previous round's
        // tiles, which read the same A row blocks, ended -- slices still in
        // L2.  The accumulation order then depends on where a tile falls in
        // the schedule, so a row's result (within fp32 rounding) depends on
        // the batch it came in; off by default.
        const bool k_down = p.k_serpentine && (((t - group) / ngroups) & 1);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1)) {
            ok = false;
            timed_out = true;
            break;
          }
          const int kq = k_down ? nk - 1 - kb : kb;  // the K step loaded
          const uint32_t full_local = full0 + 8 * stage;
          const uint32_t a_dst = smem_base + stage * STAGE_BYTES;
          const uint32_t b_dst = a_dst + A_STAGE;
          const int k0 = kq * TKS;
          if (CG == 1) {
            mbar_arrive_expect_tx(full_local, STAGE_BYTES);
            tma_load_2d(a_dst, &tmA, full_local, k0, row0);
            if (p.b_chunked) {
              tma_load_4d(b_dst, &tmB0, full_local, 0, k0, c0, e);
              if (EPI == EPI_SWIGLU)  // W1 chunks, then the same chunks of W3
                tma_load_4d(b_dst + 2 * B_CHUNK, &tmB1, full_local, 0, k0, c0, e);
            } else if (EPI == EPI_SWIGLU) {
              const int n0 = n * (TN / 2);
              tma_load_3d(b_dst + 0 * B_BOX_BYTES, &tmB0, full_local, n0, k0, e);
              tma_load_3d(b_dst + 1 * B_BOX_BYTES, &tmB0, full_local, n0 + 64, k0, e);
              tma_load_3d(b_dst + 2 * B_BOX_BYTES, &tmB1, full_local, n0, k0, e);
              tma_load_3d(b_dst + 3 * B_BOX_BYTES, &tmB1, full_local, n0 + 64, k0, e);
            } else {
              const int n0 = n * TN;
#pragma unroll
              for (int q = 0; q < 4; ++q)
                tma_load_3d(b_dst + q * B_BOX_BYTES, &tmB0, full_local, n0 + 64 * q, k0, e);
            }
          } else {
            // Both CTAs' bytes complete on the leader's full barrier, which
            // the leader arms for the whole pair.
            const uint32_t full_leader = mapa_shared(full_local, 0);
            if (leader) mbar_arrive_expect_tx(full_local, CG * STAGE_BYTES);
            if (TKS == 128)  // two 64-wide K chunks of A in one 3-D box
              tma_load_3d_pair(a_dst, &tmA, full_leader, 0, row0, kq * 2);
            else
              tma_load_2d_pair(a_dst, &tmA, full_leader, k0, row0);
            if (p.b_chunked) {
              tma_load_4d_pair(b_dst, &tmB0, full_leader, 0, k0, c0, e);
              if (EPI == EPI_SWIGLU) tma_load_4d_pair(b_dst + B_CHUNK, &tmB1, full_leader, 0, k0, c0, e);
            } else if (EPI == EPI_SWIGLU) {
              const int n0 = n * (TN / 2) + static_cast<int>(rank) * 64;
              tma_load_3d_pair(b_dst, &tmB0, full_leader, n0, k0, e);
              tma_load_3d_pair(b_dst + B_BOX_BYTES, &tmB1, full_leader, n0, k0, e);
            } else {
              const int n0 = n * TN + static_cast<int>(rank) * (TN / 2);
              tma_load_3d_pair(b_dst, &tmB0, full_leader, n0, k0, e);
              tma_load_3d_pair(b_dst + B_BOX_BYTES, &tmB0, full_leader, n0 + 64, k0, e);
            }
          }
          ++nissued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (ok) {
        // Tail: wait until the MMA has released every stage, so no
        // tcgen05.commit arrival is still in flight when the CTA exits.
        for (int i = 0; i < STAGES; ++i) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1)) {
            timed_out = true;
            break;
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok || timed_out) {
        if (timed_out) atomicOr(p.err, kErrTimeoutProducer);
        c.abort_flag = 1;
        // Let every issued copy land before the shared memory goes away:
        // stage s was filled (nissued - 1 - s) / STAGES + 1 times.
        if (CG == 1 || leader) {
          for (int s = 0; s < STAGES && s < nissued; ++s) {
            const int fills = (nissued - 1 - s) / STAGES + 1;
            if (!mbar_wait(full0 + 8 * s, static_cast<uint32_t>(fills - 1) & 1u))
              atomicOr(p.err, kErrTimeoutDrain);
          }
        }
        // The peer's copies complete on the leader's barriers, which the peer
        // cannot poll.  Nothing is needed here for them: a copy the leader
        // armed is covered by the leader's wait above, which ends before the
        // leader reaches the teardown cluster barrier, and the peer cannot
        // leave before that barrier.  A copy the leader never armed exists
        // only if the leader stopped issuing first; the MMA then stalls on
        // that stage and releases no more stages, so the peer issues nothing
        // more and leaves its loop only when one of its own bounded waits
        // (2 s) runs out -- its producer's on a stage that is never released,
        // or its epilogue's on an accumulator the stalled MMA never fills --
        // long after its last copy landed.
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0 && leader) {
      constexpr uint32_t idesc_full = idesc_bf16_f32(TILE_M, TN, false, true);
      constexpr uint32_t idesc_half = idesc_bf16_f32(TILE_M / 2, TN, false, true);
      // Descriptors of stage 0; a stage and a 16-wide K step only move the
      // 14-bit start-address field (addresses < 256 KB never carry out of it).
      const uint64_t adesc0 = smem_desc_sw128(smem_base, 16, 1024);
      const uint64_t bdesc0 = smem_desc_sw128(smem_base + A_STAGE, B_CHUNK, 1024);
      const uint32_t tfull0 = smem_u32(&c.tfull[0]);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true, timed_out = false, issued_any = false;
      // Failure-detection test: a wait that runs out, as if a load never
      // arrived; every role then gives up within its own bounded wait.
      if (p.debug_stall && !mbar_wait(smem_u32(&c.never), 0)) {
        ok = false;
        timed_out = true;
      }
      for (int t = group; t < total && ok; t += ngroups) {
        if (c.abort_flag) {
          ok = false;
          break;
        }
        if (!mbar_wait(smem_u32(&c.tempty[acc]), acc_phase ^ 1)) {
          ok = false;
          timed_out = true;
          break;
        }
        tc_fence_after();
        issued_any = true;
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * TN);
        int te, tm, tn;
        decode_tile(c, t, te, tm, tn);
        const uint32_t idesc = is_half_tile<CG>(p, c, te, tm * TILE_M) ? idesc_half : idesc_full;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase)) {
            ok = false;
            timed_out = true;
            break;
          }
          tc_fence_after();
          const uint64_t soff = static_cast<uint64_t>((stage * STAGE_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < TKS / 16; ++kk) {
            // A: K-major; 16-element steps are 32 bytes inside a 128-byte
            // swizzled row, then the next 64-wide chunk (16 KB on).
            const uint64_t adesc =
                adesc0 + soff + static_cast<uint64_t>(((kk >> 2) * C_::A_CHUNK + (kk & 3) * 32) >> 4);
            // B: N-major, 64-column chunks B_CHUNK apart; 16 K-rows = 2 KB.
            const uint64_t bdesc = bdesc0 + soff + static_cast<uint64_t>((kk * 2048) >> 4);
            const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
            if (CG == 2)
              tc_mma_bf16_pair(d_tmem, adesc, bdesc, idesc, accum);
            else
              tc_mma_bf16(d_tmem, adesc, bdesc, idesc, accum);
          }
          const uint32_t empty_local = empty0 + 8 * stage;
          if (CG == 2) {
            tc_commit_pair(empty_local);
            tc_commit_pair(mapa_shared(empty_local, 1));
          } else {
            tc_commit(empty_local);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        const uint32_t tfull_local = tfull0 + 8 * acc;
        if (CG == 2) {
          tc_commit_pair(tfull_local);
          tc_commit_pair(mapa_shared(tfull_local, 1));
        } else {
          tc_commit(tfull_local);
        }
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      if (!ok) {
        if (timed_out) atomicOr(p.err, kErrTimeoutMma);
        c.abort_flag = 1;
        if (issued_any) {
          // Wait for the MMAs already issued before TMEM is freed.
          if (CG == 2)
            tc_commit_pair(smem_u32(&c.drain));
          else
            tc_commit(smem_u32(&c.drain));
          if (!mbar_wait(smem_u32(&c.drain), 0)) atomicOr(p.err, kErrTimeoutDrain);
        }
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    // Each warp drains its 32 TMEM lanes (tile rows), applies the
    // activation and stores; the accumulator is released as soon as its last
    // columns are in registers.  Up projection (h): each lane writes its own
    // row.  Down projection (o): four 32-column loads per wait, rounded to
    // bf16; each 64-column row segment (128 bytes) goes into a swizzled
    // 32-row staging box in shared memory and one TMA store per box carries
    // it to global memory (whole lines, asynchronous; two boxes per warp
    // alternate) -- per-row 16-byte stores half-filled every sector and
    // throttled the down projection of short-K layers when o was fp32.  Rows of a box past the expert's kept rows are padding rows of
    // the same expert block (never read as results); a CTA whose 128-row
    // block starts past the kept rows stores nothing.
    const int quad = warp & 3;  // TMEM lanes this warp may read: 32*quad ..
    const int ew = warp - 2;    // epilogue warp index
    const int half = ew / 4;    // which share of the columns (0 with four warps)
    const uint32_t obuf0 = smem_base + STAGES * STAGE_BYTES + ew * OUT_BOXES_PER_WARP * OUT_BOX_BYTES;
    uint8_t* const obuf0_p = smem + STAGES * STAGE_BYTES + ew * OUT_BOXES_PER_WARP * OUT_BOX_BYTES;
    int nbox = 0;
    // o is far larger than L2 and not read again by this kernel: its lines
    // go first, so the weight and activation tiles other CTAs still read
    // stay resident.
    const uint64_t out_policy = make_policy_evict_first();
    // Stages this lane's 8 x 16 bytes as row `lane` of the next box and
    // issues its store at (col0, row0).
    auto store_box = [&](const uint4 (&v)[8], int col0, int row0) {
      const int b = nbox % OUT_BOXES_PER_WARP;
      // the store that last used this box has read it
      if (nbox >= OUT_BOXES_PER_WARP && lane == 0) bulk_wait_read<OUT_BOXES_PER_WARP - 1>();
      __syncwarp();
      uint8_t* rowp = obuf0_p + b * OUT_BOX_BYTES + lane * 128;
#pragma unroll
      for (int q = 0; q < 8; ++q) *reinterpret_cast<uint4*>(rowp + ((q ^ (lane & 7)) * 16)) = v[q];
      fence_async_shared();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d_hint(&tmOut, obuf0 + b * OUT_BOX_BYTES, col0, row0, out_policy);
        bulk_commit();
      }
      ++nbox;
    };
    auto release = [&](int a) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (CG == 2)
          mbar_arrive_cluster(mapa_shared(smem_u32(&c.tempty[a]), 0));
        else
          mbar_arrive(smem_u32(&c.tempty[a]));
      }
    };
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = group; t < total; t += ngroups) {
      int e, m, n;
      decode_tile(c, t, e, m, n);
      if (!mbar_wait(smem_u32(&c.tfull[acc]), acc_phase)) {
        atomicOr(p.err, kErrTimeoutEpilogue);
        c.abort_flag = 1;
        break;
      }
      if (c.abort_flag) break;
      tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quad * 32) << 16) +
                             static_cast<uint32_t>(acc * TN);
      // Full tiles: this warp's 32 rows of the CTA's 128.  Half tiles: 32 of
      // the CTA's 64 rows (quad & 1) and one half of the tile's columns
      // (quad >> 1), as the M = 128 pair accumulator lays them out.
      const bool half_m = is_half_tile<CG>(p, c, e, m * TILE_M);
      const int rsub = half_m ? (quad & 1) * 32 : quad * 32;
      const int chalf = half_m ? (quad >> 1) : 0;
      const int blk_row = m * TILE_M + static_cast<int>(rank) * (half_m ? TM / 2 : TM);
      const bool blk_ok = blk_row < c.kept[e];
      const int row0 = c.off[e] + blk_row + rsub;
      const int valid_rows = c.kept[e] - (blk_row + rsub);  // rows of this warp's box to keep
      if (EPI == EPI_SWIGLU || EPI == EPI_GELU) {
        // bf16 output (h): one 32-column chunk per TMEM wait, each lane
        // storing its own row's 64 bytes.  (Loading several chunks per wait
        // made this epilogue slower than the MMAs of a short tile: the
        // up projection of the 1024-wide layer lost 40%.)
        const int n0 = EPI == EPI_SWIGLU ? n * (TN / 2) + chalf * 64 : n * TN + chalf * (TN / 2);
        const int NCH = half_m ? (EPI == EPI_SWIGLU ? 2 : 4)
                               : (EPI == EPI_SWIGLU ? 4 : TN / 32) / EPI_SPLIT;  // chunks of this warp
        const bool row_ok = blk_ok && lane < valid_rows;
        __nv_bfloat16* dst_row =
            static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(row0 + lane) * p.ld_out;
#pragma unroll 1
        for (int ci = 0; ci < NCH; ++ci) {
          const int cc = half * NCH + ci;
          // TMEM columns of the gate (or GELU input) and up values of the h
          // columns n0 + 32 cc ..: a pair holds, per CTA, a W1 chunk next to
          // the same W3 chunk (64 columns each); one CTA, all of W1's
          // columns, then W3's.
          int gcol = cc * 32, ucol = TN / 2 + cc * 32;
          if (EPI == EPI_SWIGLU && CG == 2) {
            gcol = half_m ? cc * 32 : (cc >> 1) * 128 + (cc & 1) * 32;
            ucol = gcol + 64;
          }
          float g[32], u[32];
          tc_ld_32cols(tbase + gcol, g);
          if (EPI == EPI_SWIGLU) tc_ld_32cols(tbase + ucol, u);
          tc_wait_ld();
          if (ci == NCH - 1) release(acc);
          if (row_ok) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int col = n0 + cc * 32 + v * 8;
              if (col < p.n_out) {
                float r[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                  r[i] = EPI == EPI_SWIGLU ? silu_f(g[v * 8 + i]) * u[v * 8 + i]
                                           : gelu_f(g[v * 8 + i]);
                uint4 pk;
                pk.x = pack_bf16x2(r[0], r[1]);
                pk.y = pack_bf16x2(r[2], r[3]);
                pk.z = pack_bf16x2(r[4], r[5]);
                pk.w = pack_bf16x2(r[6], r[7]);
                *reinterpret_cast<uint4*>(dst_row + col) = pk;
              }
            }
          }
        }
      } else {
        const int n0 = n * TN + chalf * (TN / 2);
        const int NCH = half_m ? 4 : TN / 32 / EPI_SPLIT;  // 32-column chunks of this warp
#pragma unroll 1
        for (int c0 = half * NCH; c0 < (half + 1) * NCH; c0 += 4) {
          float g[4][32];
#pragma unroll
          for (int b = 0; b < 4; ++b) tc_ld_32cols(tbase + (c0 + b) * 32, g[b]);
          tc_wait_ld();
          if (c0 + 4 == (half + 1) * NCH) release(acc);
#pragma unroll
          for (int b = 0; b < 4; b += 2) {
            // Two 32-column chunks = one 64-column (128-byte) bf16 row
            // segment of the box.
            const int col0 = n0 + (c0 + b) * 32;
            if (blk_ok && col0 < p.n_out) {
              uint4 v[8];
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float* src = &g[b + (q >> 2)][(q & 3) * 8];
                v[q] = make_uint4(pack_bf16x2(src[0], src[1]), pack_bf16x2(src[2], src[3]),
                                  pack_bf16x2(src[4], src[5]), pack_bf16x2(src[6], src[7]));
              }
              store_box(v, col0, row0);
            }
          }
        }
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
    // Every store has completed (and read its staging box) before the CTA
    // can finish.
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }

  // ---------------------------------------------------------- teardown
  // The next kernel may launch now (not earlier: its CTAs would sit on the
  // SMs for the whole of this persistent kernel).
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  if (CG == 2) cluster_sync();  // no CTA leaves while its pair may still touch its memory
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if (CG == 2)
      tmem_dealloc_pair(tmem, TMEM_COLS);
    else
      tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 2-D bf16 matrix [rows, cols] (cols contiguous), box = 64 cols x box_rows.
bool make_map_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 weights [E, K, N] (N contiguous), box = 64 (N) x 64 (K) x 1.
bool make_map_3d(CUtensorMap* m, const void* base, uint64_t E, uint64_t K, uint64_t N) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {N, K, E};
  cuuint64_t strides[2] = {N * 2, K * N * 2};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D view {64, K, N/64, E} of bf16 weights [E, K, N] (N % 64 == 0): a box of
// {64, 64, chunks, 1} loads `chunks` adjacent 64-column chunks of 64 K-rows
// in one instruction, in the same shared-memory layout as separate 3-D boxes
// (chunk-major, 8 KB per chunk).
bool make_map_w4d(CUtensorMap* m, const void* base, uint64_t E, uint64_t K, uint64_t N,
                  uint32_t chunks, uint32_t krows) {
  auto fn = encode_fn();
  if (!fn || N % 64 != 0) return false;
  cuuint64_t dims[4] = {64, K, N / 64, E};
  cuuint64_t strides[3] = {N * 2, 128, K * N * 2};
  cuuint32_t box[4] = {64, krows, chunks, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D view {64, rows, K/64} of a bf16 activation matrix [rows, K] (K % 64 ==
// 0): a box {64, 128, 2} loads 128 rows x two 64-wide K chunks in one
// instruction, chunk-major.
bool make_map_a3d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K) {
  auto fn = encode_fn();
  if (!fn || K % 64 != 0) return false;
  cuuint64_t dims[3] = {64, rows, K / 64};
  cuuint64_t strides[2] = {K * 2, 128};
  cuuint32_t box[3] = {64, TM, 2};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D output matrix [rows, cols] (bf16 or fp32) for the epilogue's TMA
// stores: box = 128 bytes of a row x 32 rows, 128-byte swizzle.
bool make_map_out(CUtensorMap* m, void* base, uint64_t rows, uint64_t cols, bool f32) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * es};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / es), 32};
  cuuint32_t el[2] = {1, 1};
  return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base,
            dims, strides, box, el, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI, int CG, int TKS>
cudaError_t launch_one(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                       const CUtensorMap& out, const TcParams& p, int groups, cudaStream_t s) {
  constexpr int smem = Cfg<CG, TKS>::SMEM_BYTES;
  cudaError_t err = cudaFuncSetAttribute(ffn_tc_kernel<EPI, CG, TKS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  return launch_kernel(ffn_tc_kernel<EPI, CG, TKS>, dim3(groups * CG), dim3(NUM_THREADS), smem, s,
                       CG, true, a, b0, b1, out, p);
}

// Failure-detection tests: MOE_DEBUG_STALL_MMA=N makes the next N up
// projections stall their MMA issuer on a barrier nobody arms, so the
// bounded waits run out and the kernel reports through its error word.
int take_debug_stall() {
  static std::atomic<int> budget{[] {
    const char* v = getenv("MOE_DEBUG_STALL_MMA");
    return v ? atoi(v) : 0;
  }()};
  int cur = budget.load();
  while (cur > 0 && !budget.compare_exchange_weak(cur, cur - 1)) {
  }
  return cur > 0 ? 1 : 0;
}

// CTA pairs by default; MOE_TC_CTA_PAIR=0 selects one CTA per tile.
bool use_cta_pairs() {
  static const bool pairs = [] {
    const char* v = getenv("MOE_TC_CTA_PAIR");
    return !(v && v[0] == '0');
  }();
  return pairs;
}

// Half-height pair tiles for an expert's short last block (see
// is_half_tile); MOE_TC_HALF_TILES=0 computes it as a full pair tile, for
// measurements.
bool half_tiles() {
  static const bool on = [] {
    const char* v = getenv("MOE_TC_HALF_TILES");
    return !(v && v[0] == '0');
  }();
  return on;
}

// Reverse K order on alternate rounds of the down projection
// (TcParams::k_serpentine), MOE_TC_SERPENTINE=1: on the Mixtral shape the
// launch's DRAM reads fall from 2.62 to 2.07 GB (h and W2 are 1.41 GB) and
// its time by about 3 %, at the price of batch-invariant results.
bool serpentine() {
  static const bool on = [] {
    const char* v = getenv("MOE_TC_SERPENTINE");
    return v && v[0] == '1';
  }();
  return on;
}

template <int EPI>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const CUtensorMap& out, const TcParams& p, int num_sms, int64_t tiles_max,
                        bool wide_k, cudaStream_t s) {
  if (use_cta_pairs()) {
    const int groups = static_cast<int>(std::max<int64_t>(
        1, std::min<int64_t>(num_sms / 2, (tiles_max + 1) / 2)));
    return wide_k ? launch_one<EPI, 2, 128>(a, b0, b1, out, p, groups, s)
                  : launch_one<EPI, 2, 64>(a, b0, b1, out, p, groups, s);
  }
  const int groups = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(num_sms, tiles_max)));
  return launch_one<EPI, 1, 64>(a, b0, b1, out, p, groups, s);
}

}  // namespace

moe_status launch_ffn_tc(const FfnArgs& a, cudaStream_t s, int num_sms, cudaEvent_t between) {
  if (a.rows <= 0) return MOE_OK;
  CUtensorMap mx, mw1, mw3, mh, mw2, mh_out, mo_out;
  const bool swiglu = a.act == MOE_SWIGLU;
  const bool pairs = use_cta_pairs();
  // Weights: one 4-D load per K step and CTA when the columns come in whole
  // 64-wide chunks; per-chunk 3-D loads otherwise.  CTA pairs take 128-wide
  // K steps (one 3-D activation load + one 4-D weight load per 64 KB stage)
  // when K is also a multiple of 64.
  const bool up_chunked = a.H % 64 == 0, dn_chunked = a.d % 64 == 0;
  const bool up_wide = pairs && up_chunked && a.d % 64 == 0;
  const bool dn_wide = pairs && dn_chunked && a.H % 64 == 0;
  // Pairs: SwiGLU loads one chunk of W1 and the same chunk of W3 per CTA,
  // otherwise two adjacent chunks; one CTA: all chunks of its columns.
  const uint32_t up_chunks = pairs ? (swiglu ? 1 : 2) : (swiglu ? 2 : 4), dn_chunks = pairs ? 2 : 4;
  bool ok = (up_wide ? make_map_a3d(&mx, a.xp, a.rows, a.d) : make_map_2d(&mx, a.xp, a.rows, a.d, TM)) &&
            (dn_wide ? make_map_a3d(&mh, a.h, a.rows, a.H) : make_map_2d(&mh, a.h, a.rows, a.H, TM));
  const uint32_t up_kr = up_wide ? 128 : 64, dn_kr = dn_wide ? 128 : 64;
  ok = ok && (up_chunked ? make_map_w4d(&mw1, a.W1, a.E, a.d, a.H, up_chunks, up_kr) &&
                               (!swiglu || make_map_w4d(&mw3, a.W3, a.E, a.d, a.H, up_chunks, up_kr))
                         : make_map_3d(&mw1, a.W1, a.E, a.d, a.H) &&
                               (!swiglu || make_map_3d(&mw3, a.W3, a.E, a.d, a.H)));
  ok = ok && (dn_chunked ? make_map_w4d(&mw2, a.W2, a.E, a.H, a.d, dn_chunks, dn_kr)
                         : make_map_3d(&mw2, a.W2, a.E, a.H, a.d));
  ok = ok && make_map_out(&mh_out, a.h, a.rows, a.H, false) &&
       make_map_out(&mo_out, a.o, a.rows, a.d, false);
  if (!ok) return MOE_ERR_CUDA;
  const int64_t mtiles_max = (a.rows + TM - 1) / TM;

  TcParams up{};
  up.out = a.h;
  up.ld_out = a.H;
  up.n_out = a.H;
  up.K = a.d;
  up.E = a.E;
  up.n_tiles = swiglu ? (a.H + TN / 2 - 1) / (TN / 2) : (a.H + TN - 1) / TN;
  up.rows = a.rows;
  up.b_chunked = up_chunked ? 1 : 0;
  up.offsets = a.offsets;
  up.kept = a.kept_counts;
  up.err = a.dev_error;
  up.debug_stall = take_debug_stall();
  up.half_tiles = half_tiles() ? 1 : 0;
  up.k_serpentine = 0;  // A (xp) of an expert fits in L2 whatever the order
  cudaError_t err =
      swiglu ? launch_gemm<EPI_SWIGLU>(mx, mw1, mw3, mh_out, up, num_sms,
                                       mtiles_max * up.n_tiles, up_wide, s)
             : launch_gemm<EPI_GELU>(mx, mw1, mw1, mh_out, up, num_sms, mtiles_max * up.n_tiles,
                                     up_wide, s);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  if (between && cudaEventRecord(between, s) != cudaSuccess) return MOE_ERR_CUDA;

  TcParams dn{};
  dn.out = a.o;
  dn.ld_out = a.d;
  dn.n_out = a.d;
  dn.K = a.H;
  dn.E = a.E;
  dn.n_tiles = (a.d + TN - 1) / TN;
  dn.rows = a.rows;
  dn.b_chunked = dn_chunked ? 1 : 0;
  dn.offsets = a.offsets;
  dn.kept = a.kept_counts;
  dn.err = a.dev_error;
  dn.debug_stall = 0;
  dn.half_tiles = half_tiles() ? 1 : 0;
  dn.k_serpentine = serpentine() ? 1 : 0;
  err = launch_gemm<EPI_PLAIN>(mh, mw2, mw2, mo_out, dn, num_sms, mtiles_max * dn.n_tiles,
                                   dn_wide, s);
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
