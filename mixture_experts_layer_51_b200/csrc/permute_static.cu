// moe_permute_static: the permutation for callers that cannot allocate any
// device memory for it.
//
// moe_permute needs a small scratch buffer from its caller (per-block expert
// counts and a completion counter).  Some callers have no way to provide
// one at the point where they run the layer: a serving runtime that reserves
// all device memory up front for its own pool, or a plugin whose host
// framework forbids allocation inside its execute call.  This variant keeps
// that scratch in a fixed-size array owned by the library instead.  The
// caller still passes every input and output buffer; nothing here calls
// cudaMalloc, cudaFree or any allocating routine.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds it (MOE_PERMUTE_STATIC_MAX_INTS int32 plus a 512-byte
// slot for a counter and per-expert capacities) until the process exits.  In host code its name is only a
// host-side stand-in, so its device address is looked up with
// cudaGetSymbolAddress once per device (on the first call made with that
// device current) and that address is what the kernels receive.

#include <mutex>

#include "moe_internal.cuh"

namespace {

constexpr int kCounterInts = 128;  // 512 bytes: the completion counter and per-expert capacities

static __device__ __align__(256) int32_t g_permute_scratch[MOE_PERMUTE_STATIC_MAX_INTS + kCounterInts];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_permute_scratch on the current device.
moe_status scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

MOE_API moe_status moe_permute_static(const void* x, const int32_t* idx, int32_t T, int32_t d,
                                      int32_t E, int32_t k, double cf, moe_dtype dt, void* xp,
                                      int64_t xp_rows, int32_t* pos, int32_t* counts,
                                      int32_t* kept_counts, int32_t* offsets, void* stream) {
  if (T < 0 || d <= 0 || d % 8 != 0 || E < 1 || E > moe::kMaxE || k < 1 || k > moe::kMaxK ||
      k > E || (dt != MOE_BF16 && dt != MOE_FP32))
    return MOE_ERR_ARG;
  if (!counts || !kept_counts || !offsets) return MOE_ERR_ARG;
  const int64_t nblk = (static_cast<int64_t>(T) + moe::kPermBlock - 1) / moe::kPermBlock;
  // The fixed scratch holds one int32 per (256-token block, expert).
  if (nblk * E > MOE_PERMUTE_STATIC_MAX_INTS) return MOE_ERR_ARG;
  if (T > 0) {
    if (!x || !idx || !xp || !pos || !aligned16(x) || !aligned16(xp)) return MOE_ERR_ARG;
    if (xp_rows < moe_max_permuted_rows(T, E, k, cf)) return MOE_ERR_ARG;
  }
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (major != 10) return MOE_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  moe_status st = scratch_address(dev, &scratch);
  if (st != MOE_OK) return st;
  int32_t* block_base = static_cast<int32_t*>(scratch);
  // The counter sits after the largest count table and is zeroed on the
  // stream by launch_permute before the counting kernel runs.
  unsigned int* ticket = reinterpret_cast<unsigned int*>(block_base + MOE_PERMUTE_STATIC_MAX_INTS);
  const int32_t C = moe_capacity(T, E, k, cf);
  moe::PermuteArgs a{x,      idx,         T,       d,          E,     k,
                     C < 0 ? INT32_MAX : C, xp, pos, counts, kept_counts, offsets,
                     block_base, ticket};
  return moe::launch_permute(a, dt, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
