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
// rows of W_g -- about 190 KB per SM, and eight consumer warps contract each
// stage with mma.sync (m16n8k16, fp32 accumulate): at E <= 64 that keeps
// pace with HBM.  After the last stage of a tile of up to 128 rows the
// logits go to shared memory and the tile's tokens select (route_select.cuh).
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

constexpr int kRsConsumerWarps = 8;
constexpr int kRsThreads = (kRsConsumerWarps + 1) * 32;  // + one producer warp
constexpr int kRsMaxStages = 8;
constexpr int kRsMaxRows = 128;   // rows of one tile (8 consumer warps x 16)
constexpr int kRsSmemLimit = 232448;

struct RsCtl {
  uint64_t full[kRsMaxStages];
  uint64_t empty[kRsMaxStages];
  volatile int abort_flag;
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
  int tx_bytes;     // bytes the TMA loads of one stage deliver
  int logit_off;    // offset of the logits buffer
  int ctl_off;      // offset of the control block
  int ls;           // logits row stride (floats)
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

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
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
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// NT = 8-expert column tiles (the W_g box is NT * 8 experts wide, zero past
// E; its rows are NT * 16 bytes, swizzled by the TMA in the mode of that
// width); KM = length of the running top lists.
template <int NT, int KM>
__global__ void __launch_bounds__(kRsThreads, 1)
    route_stream_kernel(const __grid_constant__ CUtensorMap tmX,
                        const __grid_constant__ CUtensorMap tmW, const RsParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  RsCtl& c = *reinterpret_cast<RsCtl*>(smem + p.ctl_off);
  float* logits = reinterpret_cast<float*>(smem + p.logit_off);
  constexpr int RB = NT * 16;             // bytes per W_g row in shared memory
  constexpr int SWZ_MASK = RB / 16 - 1;   // 16-byte units XORed by the TMA swizzle
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;
  const int r0 = static_cast<int>(static_cast<int64_t>(cta) * p.T8 / p.G) * 8;
  const int r1 = min(p.T, static_cast<int>(static_cast<int64_t>(cta + 1) * p.T8 / p.G) * 8);
  const int ntiles = (r1 - r0 + p.MT - 1) / p.MT;
  const int nbusy = min(kRsConsumerWarps, (p.MT + 15) / 16);
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t full0 = smem_u32(&c.full[0]);
  const uint32_t empty0 = smem_u32(&c.empty[0]);

  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, nbusy);
    }
    c.abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < kMaxE) c.cnt[tid] = 0;
  if (warp == kRsConsumerWarps && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  __syncthreads();
  // x and W_g may be written by the previous kernel in the stream.
  pdl_wait();
  pdl_trigger();

  if (warp == kRsConsumerWarps) {
    // ---------------------------------------------------------- producer
    if (lane != 0) return;
    int stage = 0, nissued = 0;
    uint32_t phase = 0;
    bool timed_out = false;
    for (int mt = 0; mt < ntiles && !timed_out; ++mt) {
      const int row = r0 + mt * p.MT;
      for (int kb = 0; kb < p.nk; ++kb) {
        if (c.abort_flag || !mbar_wait(empty0 + 8 * stage, phase ^ 1)) {
          timed_out = !c.abort_flag;
          c.abort_flag = 1;
          break;
        }
        const uint32_t full = full0 + 8 * stage;
        const uint32_t dst = smem_base + stage * p.stage_bytes;
        mbar_arrive_expect_tx(full, p.tx_bytes);
        const int col0 = kb * p.nch * 64;
        for (int ch = 0; ch < p.nch; ++ch)
          tma_load_2d(dst + ch * p.a_chunk, &tmX, full, col0 + ch * 64, row);
        tma_load_2d(dst + p.b_off, &tmW, full, 0, col0);
        ++nissued;
        if (++stage == p.stages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (c.abort_flag) break;
    }
    if (timed_out && p.err) atomicOr(p.err, kErrTimeoutProducer);
    // Every issued copy lands before the CTA can exit (consumed stages have
    // landed already; after an abort these waits are what keeps the shared
    // memory alive): stage s was filled (nissued - 1 - s) / stages + 1 times.
    for (int s = 0; s < p.stages && s < nissued; ++s) {
      const int fills = (nissued - 1 - s) / p.stages + 1;
      if (!mbar_wait(full0 + 8 * s, static_cast<uint32_t>(fills - 1) & 1u) && p.err)
        atomicOr(p.err, kErrTimeoutDrain);
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const bool busy = warp < nbusy;
  const int P = p.MT <= 32 ? 8 : (p.MT <= 64 ? 4 : 2);  // threads per token in the selection
  int stage = 0;
  uint32_t phase = 0;
  for (int mt = 0; mt < ntiles; ++mt) {
    const int row0 = r0 + mt * p.MT;
    const int rows = min(p.MT, r1 - row0);
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[n][i] = 0.f;
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
          const int r = warp * 16 + (lane & 15);  // may pass MT: those rows are never kept
          for (int ch = 0; ch < p.nch; ++ch) {
            const uint32_t a_row = a_base + ch * p.a_chunk + r * 128;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              uint32_t a0, a1, a2, a3;
              ldsm_x4(a_row + ((((ks * 2) + (lane >> 4)) ^ (r & 7)) << 4), a0, a1, a2, a3);
              const int krow = ch * 64 + ks * 16 + (lane & 15);
              const uint32_t b_row = b_base + krow * RB;
              const int sw = (krow * RB >> 7) & SWZ_MASK;
#pragma unroll
              for (int n = 0; n + 1 < NT; n += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(b_row + (((n + (lane >> 4)) ^ sw) << 4), b0, b1, b2, b3);
                mma_16816(acc[n], a0, a1, a2, a3, b0, b1);
                mma_16816(acc[n + 1], a0, a1, a2, a3, b2, b3);
              }
              if (NT & 1) {
                uint32_t b0, b1;
                ldsm_x2_t(b_row + (((NT - 1) ^ sw) << 4), b0, b1);
                mma_16816(acc[NT - 1], a0, a1, a2, a3, b0, b1);
              }
            }
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

    // Logits of the tile's rows (bias added) into shared memory.
    if (busy) {
      const int rr = warp * 16 + (lane >> 2);
      const int cc = (lane & 3) * 2;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = rr + 8 * h;
          if (row < rows) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int e = n * 8 + cc + q;
              if (e < p.E) logits[row * p.ls + e] = acc[n][2 * h + q] + (p.bias ? p.bias[e] : 0.f);
            }
          }
        }
      }
    }
    consumer_sync();
    const bool aborted = c.abort_flag != 0;

    // Selection: P threads per token; every consumer thread takes part (the
    // shuffles need whole warps), threads past the tile only read.
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
      continue;
    }
    select_token<KM>(lrow, p.E, p.k, P, pp, row0 + rr, valid, p.gating, p.gate_scale, p.idx,
                     p.gate, p.margin, valid ? c.idx_s[rr] : nullptr);
    if (!p.lrank) {
      consumer_sync();  // the logits buffer is rewritten by the next tile
      continue;
    }
    consumer_sync();

    // Ranks among this range's assignments to the same expert, in token
    // order: one thread per token of the tile (warps 0-3), a ballot per
    // expert; the warps below come from shared counts, earlier tiles from
    // the running per-expert count.
    uint64_t mask = 0;
    int rj[kMaxK];
    const bool have = !aborted && warp < 4 && tid < rows;
    if (warp < 4) {
      for (int j = 0; j < p.k; ++j) {
        rj[j] = 0;
        if (have) mask |= 1ull << c.idx_s[tid][j];
      }
      const unsigned lt = (1u << lane) - 1u;
      for (int e = 0; e < p.E; ++e) {
        const unsigned b = __ballot_sync(0xffffffffu, (mask >> e) & 1ull);
        if (lane == 0) c.wcnt[warp][e] = __popc(b);
        if ((mask >> e) & 1ull) {
          for (int j = 0; j < p.k; ++j)
            if (c.idx_s[tid][j] == e) rj[j] = __popc(b & lt);
        }
      }
    }
    consumer_sync();
    if (have) {
      for (int j = 0; j < p.k; ++j) {
        const int e = c.idx_s[tid][j];
        int r = c.cnt[e] + rj[j];
        for (int w = 0; w < warp; ++w) r += c.wcnt[w][e];
        p.lrank[static_cast<int64_t>(row0 + tid) * p.k + j] = r;
      }
    }
    consumer_sync();
    if (tid < p.E) {
      const int nw = min(4, (rows + 31) / 32);
      int s = 0;
      for (int w = 0; w < nw; ++w) s += c.wcnt[w][tid];
      c.cnt[tid] += s;
    }
    consumer_sync();
  }
  if (p.hist && tid < p.E) p.hist[static_cast<int64_t>(cta) * p.E + tid] = c.cnt[tid];
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

template <int NT>
cudaError_t launch_rs_nt(const RouteArgs& a, int num_sms, cudaStream_t s) {
  const RouteRanges rg = route_ranges(a.T, num_sms);
  constexpr int EP = NT * 8;
  RsParams p{};
  p.T = a.T;
  p.d = a.d;
  p.E = a.E;
  p.k = a.k;
  p.G = rg.G;
  p.T8 = rg.T8;
  p.MT = rg.MT;
  p.ls = EP + 1;
  p.a_chunk = p.MT * 128;
  p.logit_off = 0;  // placed after the ring below
  const int logit_bytes = round1k(p.MT * p.ls * 4);
  const int ctl_bytes = round1k(static_cast<int>(sizeof(RsCtl)));
  const int budget = kRsSmemLimit - 1024 - logit_bytes - ctl_bytes;
  const int chunks_d = (a.d + 63) / 64;
  int nch = std::min(4, chunks_d);
  auto stage_of = [&](int n) { return round1k(n * p.a_chunk) + round1k(n * 64 * EP * 2); };
  while (nch > 1 && budget / stage_of(nch) < 4) --nch;
  p.nch = nch;
  p.nk = (chunks_d + nch - 1) / nch;
  p.b_off = round1k(nch * p.a_chunk);
  p.stage_bytes = stage_of(nch);
  p.tx_bytes = nch * p.a_chunk + nch * 64 * EP * 2;
  p.stages = std::min(kRsMaxStages, budget / p.stage_bytes);
  if (p.stages < 2) return cudaErrorInvalidValue;
  p.logit_off = p.stages * p.stage_bytes;
  p.ctl_off = p.logit_off + logit_bytes;
  const int smem = p.ctl_off + ctl_bytes + 1024;
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

  CUtensorMap mx, mw;
  const CUtensorMapSwizzle wswz = EP == 8    ? CU_TENSOR_MAP_SWIZZLE_NONE
                                  : EP == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                  : EP == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                             : CU_TENSOR_MAP_SWIZZLE_128B;
  if (!rs_map(&mx, a.x, a.T, a.d, 64, p.MT, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !rs_map(&mw, a.Wg, a.d, a.E, EP, nch * 64, wswz))
    return cudaErrorInvalidValue;
  auto go = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(kern, dim3(p.G), dim3(kRsThreads), smem, s, 1, true, mx, mw, p);
  };
  if (a.scores || a.k <= 2) return go(route_stream_kernel<NT, 3>);
  if (a.k <= 4) return go(route_stream_kernel<NT, 5>);
  return go(route_stream_kernel<NT, kMaxK + 1>);
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
  switch ((a.E + 7) / 8) {
    case 1: return launch_rs_nt<1>(a, num_sms, s);
    case 2: return launch_rs_nt<2>(a, num_sms, s);
    case 3:
    case 4: return launch_rs_nt<4>(a, num_sms, s);
    default: return launch_rs_nt<8>(a, num_sms, s);
  }
}

}  // namespace moe
