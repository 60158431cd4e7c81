// C ABI of libmoe.so: argument checks, workspace layout and the one-stream
// orchestration of route -> permute -> grouped FFN -> combine.  Every entry
// point is declared and documented in include/moe.h.

#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "moe_internal.cuh"

using namespace moe;

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t elt_size(moe_dtype dt) { return dt == MOE_BF16 ? 2 : 4; }

bool valid_dtype(moe_dtype dt) { return dt == MOE_BF16 || dt == MOE_FP32; }
bool valid_act(moe_act a) { return a == MOE_SWIGLU || a == MOE_GELU; }

bool valid_route_sizes(int32_t T, int32_t d, int32_t E, int32_t k) {
  return T >= 0 && d > 0 && d % 8 == 0 && E >= 1 && E <= kMaxE && k >= 1 && k <= kMaxK && k <= E;
}
bool valid_ffn_sizes(int32_t d, int32_t H) { return d > 0 && d % 8 == 0 && H > 0 && H % 8 == 0; }

// Stage events set by moe_set_stage_events for this host thread.
thread_local cudaEvent_t g_stage_events[MOE_NUM_STAGE_EVENTS] = {};
thread_local bool g_stage_events_on = false;

moe_status record_stage(int i, cudaStream_t s) {
  if (!g_stage_events_on) return MOE_OK;
  return cudaEventRecord(g_stage_events[i], s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Options with defaults filled in; false if they are invalid.
bool read_options(const moe_options* opt, int* gating, float* gate_scale, int* priority = nullptr) {
  *gating = MOE_GATE_TOPK_SOFTMAX;
  *gate_scale = 1.0f;
  if (priority) *priority = MOE_PRIORITY_POSITION;
  if (!opt) return true;
  if (opt->gating != MOE_GATE_TOPK_SOFTMAX && opt->gating != MOE_GATE_SOFTMAX_TOPK) return false;
  if (!(opt->gate_scale > 0.0f) || isinf(opt->gate_scale)) return false;
  if (opt->priority != MOE_PRIORITY_POSITION && opt->priority != MOE_PRIORITY_GATE) return false;
  for (int i = 0; i < 5; ++i)
    if (opt->reserved[i] != 0) return false;
  *gating = opt->gating;
  *gate_scale = opt->gate_scale;
  if (priority) *priority = opt->priority;
  return true;
}

struct DeviceInfo {
  int device = -1;
  int num_sms = 0;
  int major = 0;
};

moe_status device_info(DeviceInfo* out) {
  static std::atomic<int> sms_cache[64];
  static std::atomic<int> major_cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  out->device = dev;
  if (dev >= 0 && dev < 64 && sms_cache[dev].load() > 0) {
    out->num_sms = sms_cache[dev].load();
    out->major = major_cache[dev].load();
  } else {
    if (cudaDeviceGetAttribute(&out->num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&out->major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (dev >= 0 && dev < 64) {
      major_cache[dev].store(out->major);
      sms_cache[dev].store(out->num_sms);
    }
  }
  // The library carries sm_100a code only.
  return out->major == 10 ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

bool compute_layout(int32_t T, int32_t d, int32_t H, int32_t E, int32_t k, double cf,
                    moe_dtype dt, moe_act act, moe_ws_layout* L) {
  if (!valid_route_sizes(T, d, E, k) || !valid_ffn_sizes(d, H) || !valid_dtype(dt) ||
      !valid_act(act))
    return false;
  const int64_t rows = moe_max_permuted_rows(T, E, k, cf);
  // Row indices, offsets and positions are int32 on the device.
  if (rows < 0 || rows > INT32_MAX) return false;
  const size_t tk = static_cast<size_t>(T) * k;
  const size_t es = elt_size(dt);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  memset(L, 0, sizeof(*L));
  L->idx = take(tk * 4);
  L->gate = take(tk * 4);
  L->margin = take(static_cast<size_t>(T) * 4);
  L->pos = take(tk * 4);
  L->counts = take(kMaxE * 4);
  L->kept_counts = take(kMaxE * 4);
  L->offsets = take((kMaxE + 1) * 4);
  L->dev_error = take(4);
  L->scratch = take(ranked_permute_scratch_bytes(E));
  L->order = take(static_cast<size_t>(T) * 4);
  L->prio_scratch = take(priority_scratch_bytes(T));
  L->xp = take(static_cast<size_t>(rows) * d * es);
  L->h = take(static_cast<size_t>(rows) * H * es);
  L->o = take(static_cast<size_t>(rows) * d * es);
  L->total = off;
  L->rows = rows;
  return true;
}

}  // namespace

// ====================================================================== ABI
MOE_API const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_ARG: return "MOE_ERR_ARG: invalid argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: not supported on this device/config";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call failed";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE: a kernel reported an error";
  }
  return "MOE_UNKNOWN_STATUS";
}

MOE_API int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

MOE_API int32_t moe_capacity(int32_t T, int32_t E, int32_t k, double cf) {
  if (!(cf > 0.0) || isinf(cf) || E <= 0 || T < 0 || k <= 0) return -1;
  const double c = ceil(cf * static_cast<double>(T) * static_cast<double>(k) / static_cast<double>(E));
  if (c > static_cast<double>(INT32_MAX)) return INT32_MAX;
  return static_cast<int32_t>(c);
}

MOE_API int64_t moe_rows_for_capacity(int32_t T, int32_t E, int32_t k, int32_t C) {
  if (T < 0 || E < 1 || E > kMaxE || k < 1 || k > kMaxK || k > E) return -1;
  if (T == 0) return 0;
  int64_t rows = static_cast<int64_t>(T) * k + static_cast<int64_t>(E) * (kRowAlign - 1);
  if (C >= 0) rows = std::min<int64_t>(rows, static_cast<int64_t>(E) * pad_rows(C));
  return pad_rows(std::max<int64_t>(rows, kRowAlign));
}

MOE_API int64_t moe_max_permuted_rows(int32_t T, int32_t E, int32_t k, double cf) {
  return moe_rows_for_capacity(T, E, k, moe_capacity(T, E, k, cf));
}

MOE_API size_t moe_permute_workspace_bytes(int32_t T, int32_t E) {
  if (T < 0 || E < 1 || E > kMaxE) return 0;
  return ranked_permute_scratch_bytes(E);
}

MOE_API size_t moe_workspace_bytes(int32_t T, int32_t d, int32_t H, int32_t E, int32_t k,
                                   double cf, moe_dtype dt, moe_act act) {
  moe_ws_layout L;
  return compute_layout(T, d, H, E, k, cf, dt, act, &L) ? L.total : 0;
}

MOE_API moe_status moe_workspace_layout(int32_t T, int32_t d, int32_t H, int32_t E, int32_t k,
                                        double cf, moe_dtype dt, moe_act act, moe_ws_layout* out) {
  if (!out) return MOE_ERR_ARG;
  return compute_layout(T, d, H, E, k, cf, dt, act, out) ? MOE_OK : MOE_ERR_ARG;
}

namespace {
// Router; `err` (nullable) receives the routers' time-out bits.  With
// lrank/hist (nullable) the streaming router also writes the permutation's
// local ranks and per-range counts; *ranked says whether it did.
moe_status route_enqueue(const void* x, const void* Wg, const float* bias, int32_t T, int32_t d,
                         int32_t E, int32_t k, moe_dtype dt, const moe_options* opt,
                         int32_t* idx, float* gate, float* margin, void* stream, int32_t* err,
                         int32_t* lrank = nullptr, int32_t* hist = nullptr,
                         bool* ranked = nullptr) {
  if (ranked) *ranked = false;
  int gating;
  float gate_scale;
  if (!valid_route_sizes(T, d, E, k) || !valid_dtype(dt) || !read_options(opt, &gating, &gate_scale))
    return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !Wg || !idx || !gate || !aligned16(x) || !aligned16(Wg)) return MOE_ERR_ARG;
  DeviceInfo di;
  moe_status st = device_info(&di);
  if (st != MOE_OK) return st;
  RouteArgs a{x, Wg, bias, T, d, E, k, idx, gate, margin, gating, gate_scale};
  a.err = err;
  a.lrank = lrank;
  a.hist = hist;
  return launch_route(a, dt, static_cast<cudaStream_t>(stream), di.num_sms, ranked) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
}  // namespace

MOE_API moe_status moe_route_ex(const void* x, const void* Wg, const float* bias, int32_t T,
                                int32_t d, int32_t E, int32_t k, moe_dtype dt,
                                const moe_options* opt, int32_t* idx, float* gate, float* margin,
                                void* stream) {
  return route_enqueue(x, Wg, bias, T, d, E, k, dt, opt, idx, gate, margin, stream, nullptr);
}

MOE_API moe_status moe_route(const void* x, const void* Wg, const float* bias, int32_t T,
                             int32_t d, int32_t E, int32_t k, moe_dtype dt, int32_t* idx,
                             float* gate, float* margin, void* stream) {
  return moe_route_ex(x, Wg, bias, T, d, E, k, dt, nullptr, idx, gate, margin, stream);
}

namespace {
// `ranked`: pos and the scratch already hold the router's local ranks and
// per-range counts (the forward), so only the placement and copy run.
moe_status permute_enqueue(const void* x, const int32_t* idx, const int32_t* order,
                           const int32_t* prior, int32_t T, int32_t d, int32_t E, int32_t k,
                           int32_t capacity, moe_dtype dt, void* xp, int64_t xp_rows,
                           int32_t* pos, int32_t* counts, int32_t* kept_counts, int32_t* offsets,
                           void* ws, size_t ws_bytes, void* stream, bool ranked);
}  // namespace

MOE_API moe_status moe_permute_ex(const void* x, const int32_t* idx, const int32_t* order,
                                  const int32_t* prior, int32_t T, int32_t d, int32_t E,
                                  int32_t k, int32_t capacity, moe_dtype dt, void* xp,
                                  int64_t xp_rows, int32_t* pos, int32_t* counts,
                                  int32_t* kept_counts, int32_t* offsets, void* ws,
                                  size_t ws_bytes, void* stream) {
  return permute_enqueue(x, idx, order, prior, T, d, E, k, capacity, dt, xp, xp_rows, pos, counts,
                         kept_counts, offsets, ws, ws_bytes, stream, false);
}

namespace {
moe_status permute_enqueue(const void* x, const int32_t* idx, const int32_t* order,
                           const int32_t* prior, int32_t T, int32_t d, int32_t E, int32_t k,
                           int32_t capacity, moe_dtype dt, void* xp, int64_t xp_rows,
                           int32_t* pos, int32_t* counts, int32_t* kept_counts, int32_t* offsets,
                           void* ws, size_t ws_bytes, void* stream, bool ranked) {
  if (!valid_route_sizes(T, d, E, k) || !valid_dtype(dt)) return MOE_ERR_ARG;
  if (!counts || !kept_counts || !offsets) return MOE_ERR_ARG;
  if (T > 0) {
    if (!x || !idx || !xp || !pos || !ws || !aligned16(x) || !aligned16(xp) ||
        !aligned16(ws))
      return MOE_ERR_ARG;
    const int64_t need_rows = moe_rows_for_capacity(T, E, k, capacity);
    if (need_rows > INT32_MAX || xp_rows < need_rows) return MOE_ERR_ARG;
    if (ws_bytes < ranked_permute_scratch_bytes(E)) return MOE_ERR_ARG;
  }
  DeviceInfo di;
  moe_status st = device_info(&di);
  if (st != MOE_OK) return st;
  RankedPermuteArgs a{x, idx, T, d, E, k, capacity < 0 ? INT32_MAX : capacity, xp, pos, counts,
                      kept_counts, offsets, static_cast<int32_t*>(ws), order, prior, ranked,
                      di.num_sms};
  return launch_ranked_permute(a, dt, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
}  // namespace

MOE_API moe_status moe_permute(const void* x, const int32_t* idx, int32_t T, int32_t d, int32_t E,
                               int32_t k, double cf, moe_dtype dt, void* xp, int64_t xp_rows,
                               int32_t* pos, int32_t* counts, int32_t* kept_counts,
                               int32_t* offsets, void* ws, size_t ws_bytes, void* stream) {
  return moe_permute_ex(x, idx, nullptr, nullptr, T, d, E, k, moe_capacity(T, E, k, cf), dt, xp,
                        xp_rows, pos, counts, kept_counts, offsets, ws, ws_bytes, stream);
}

MOE_API moe_status moe_expert_counts(const int32_t* idx, int32_t T, int32_t E, int32_t k,
                                     int32_t* counts, void* stream) {
  if (T < 0 || E < 1 || E > kMaxE || k < 1 || k > kMaxK || k > E || !counts) return MOE_ERR_ARG;
  if (T > 0 && !idx) return MOE_ERR_ARG;
  DeviceInfo di;
  moe_status st = device_info(&di);
  if (st != MOE_OK) return st;
  return launch_expert_counts(idx, T, E, k, counts, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

MOE_API moe_status moe_rank_prefix(const int32_t* gathered, int32_t n_ranks, int32_t E,
                                   int32_t rank, int32_t* prior, void* stream) {
  if (n_ranks < 1 || rank < 0 || rank >= n_ranks || E < 1 || E > kMaxE || !gathered || !prior)
    return MOE_ERR_ARG;
  DeviceInfo di;
  moe_status st = device_info(&di);
  if (st != MOE_OK) return st;
  return launch_rank_prefix(gathered, n_ranks, E, rank, prior, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

MOE_API size_t moe_priority_workspace_bytes(int32_t T) {
  return T < 0 ? 0 : priority_scratch_bytes(T);
}

MOE_API moe_status moe_priority_order(const float* gate, int32_t T, int32_t k, int32_t* order,
                                      void* ws, size_t ws_bytes, void* stream) {
  if (T < 0 || k < 1 || k > kMaxK) return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!gate || !order || !ws || !aligned16(ws) || ws_bytes < priority_scratch_bytes(T))
    return MOE_ERR_ARG;
  DeviceInfo di;
  moe_status st = device_info(&di);
  if (st != MOE_OK) return st;
  return launch_priority_order(gate, T, k, order, ws, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

MOE_API moe_status moe_grouped_ffn(const void* xp, int64_t rows, const int32_t* offsets,
                                   const int32_t* kept_counts, const void* W1, const void* W3,
                                   const void* W2, int32_t E, int32_t d, int32_t H, moe_act act,
                                   moe_dtype dt, void* h, void* o, int32_t* dev_error,
                                   void* stream) {
  if (!valid_ffn_sizes(d, H) || E < 1 || E > kMaxE || !valid_act(act) || !valid_dtype(dt) ||
      rows < 0 || rows > INT32_MAX || rows % kRowAlign != 0)
    return MOE_ERR_ARG;
  if (rows == 0) return MOE_OK;
  if (!xp || !offsets || !kept_counts || !W1 || !W2 || !h || !o || !dev_error) return MOE_ERR_ARG;
  if (act == MOE_SWIGLU && !W3) return MOE_ERR_ARG;
  if (!aligned16(xp) || !aligned16(W1) || (W3 && !aligned16(W3)) || !aligned16(W2) ||
      !aligned16(h) || !aligned16(o))
    return MOE_ERR_ARG;
  DeviceInfo di;
  moe_status st = device_info(&di);
  if (st != MOE_OK) return st;
  FfnArgs a{xp, rows, offsets, kept_counts, W1, W3, W2, E, d, H, act, h, o, dev_error};
  cudaEvent_t between = g_stage_events_on ? g_stage_events[3] : nullptr;
  if (dt == MOE_BF16)
    return launch_ffn_tc(a, static_cast<cudaStream_t>(stream), di.num_sms, between);
  return launch_ffn_simt(a, static_cast<cudaStream_t>(stream), between);
}

MOE_API moe_status moe_set_stage_events(void* const* events) {
  if (!events) {
    g_stage_events_on = false;
    return MOE_OK;
  }
  for (int i = 0; i < MOE_NUM_STAGE_EVENTS; ++i)
    if (!events[i]) return MOE_ERR_ARG;
  for (int i = 0; i < MOE_NUM_STAGE_EVENTS; ++i)
    g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
  g_stage_events_on = true;
  return MOE_OK;
}

MOE_API moe_status moe_unpermute_combine(const void* o, const int32_t* pos, const float* gate,
                                         int32_t T, int32_t d, int32_t k, moe_dtype dt, void* y,
                                         void* stream) {
  if (T < 0 || d <= 0 || d % 8 != 0 || k < 1 || k > kMaxK || !valid_dtype(dt)) return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!o || !pos || !gate || !y || !aligned16(o) || !aligned16(y)) return MOE_ERR_ARG;
  DeviceInfo di;
  moe_status st = device_info(&di);
  if (st != MOE_OK) return st;
  CombineArgs a{o, pos, gate, T, d, k, y};
  return launch_combine(a, dt, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK
                                                                                 : MOE_ERR_CUDA;
}

namespace {

// The device pointers a whole forward reads and writes, checked before
// anything is enqueued: present, and 16-byte aligned where the kernels read
// or write them in 16-byte vectors or TMA boxes (the bias is read one float
// at a time).
bool forward_ptrs_ok(const void* x, const void* Wg, const void* W1, const void* W3,
                     const void* W2, moe_act act, const void* y) {
  if (!x || !Wg || !W1 || !W2 || !y || (act == MOE_SWIGLU && !W3)) return false;
  return aligned16(x) && aligned16(Wg) && aligned16(W1) &&
         (act != MOE_SWIGLU || aligned16(W3)) && aligned16(W2) && aligned16(y);
}

moe_status forward_enqueue(const void* x, const void* Wg, const float* bias, const void* W1,
                           const void* W3, const void* W2, int32_t T, int32_t d, int32_t H,
                           int32_t E, int32_t k, double cf, moe_act act, moe_dtype dt, void* y,
                           void* ws, size_t ws_bytes, const moe_ws_layout& L, cudaStream_t s,
                           bool clear_err = true, const moe_options* opt = nullptr) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  int32_t* idx = reinterpret_cast<int32_t*>(w + L.idx);
  float* gate = reinterpret_cast<float*>(w + L.gate);
  float* margin = reinterpret_cast<float*>(w + L.margin);
  int32_t* pos = reinterpret_cast<int32_t*>(w + L.pos);
  int32_t* counts = reinterpret_cast<int32_t*>(w + L.counts);
  int32_t* kept = reinterpret_cast<int32_t*>(w + L.kept_counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(w + L.offsets);
  int32_t* err = reinterpret_cast<int32_t*>(w + L.dev_error);
  if (clear_err && cudaMemsetAsync(err, 0, sizeof(int32_t), s) != cudaSuccess)
    return MOE_ERR_CUDA;
  int gating, priority;
  float gate_scale;
  read_options(opt, &gating, &gate_scale, &priority);
  const bool by_gate = priority == MOE_PRIORITY_GATE && moe_capacity(T, E, k, cf) >= 0;
  int32_t* hist = reinterpret_cast<int32_t*>(w + L.scratch);
  moe_status st = record_stage(0, s);
  if (st != MOE_OK) return st;
  // In position order the router also counts (local ranks into pos, the
  // per-range counts into the scratch), so the permutation is one kernel.
  bool ranked = false;
  st = route_enqueue(x, Wg, bias, T, d, E, k, dt, opt, idx, gate, margin, s, err,
                     by_gate ? nullptr : pos, by_gate ? nullptr : hist, &ranked);
  if (st == MOE_OK) st = record_stage(1, s);
  if (st != MOE_OK) return st;
  const int32_t* order = nullptr;
  if (by_gate) {
    st = moe_priority_order(gate, T, k, reinterpret_cast<int32_t*>(w + L.order),
                            w + L.prio_scratch, priority_scratch_bytes(T), s);
    if (st != MOE_OK) return st;
    order = reinterpret_cast<const int32_t*>(w + L.order);
  }
  st = permute_enqueue(x, idx, order, nullptr, T, d, E, k, moe_capacity(T, E, k, cf), dt, w + L.xp,
                       L.rows, pos, counts, kept, offsets, hist, ranked_permute_scratch_bytes(E),
                       s, ranked);
  if (st == MOE_OK) st = record_stage(2, s);
  if (st != MOE_OK) return st;
  st = moe_grouped_ffn(w + L.xp, L.rows, offsets, kept, W1, W3, W2, E, d, H, act, dt, w + L.h,
                       w + L.o, err, s);
  if (st == MOE_OK) st = record_stage(4, s);
  if (st != MOE_OK) return st;
  st = moe_unpermute_combine(w + L.o, pos, gate, T, d, k, dt, y, s);
  if (st == MOE_OK) st = record_stage(5, s);
  return st;
}

moe_status read_device_error(const moe_ws_layout& L, void* ws, cudaStream_t s, int32_t* out) {
  if (cudaMemcpyAsync(out, static_cast<uint8_t*>(ws) + L.dev_error, sizeof(int32_t),
                      cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace

MOE_API moe_status moe_forward_ex(const void* x, const void* Wg, const float* bias,
                                  const void* W1, const void* W3, const void* W2, int32_t T,
                                  int32_t d, int32_t H, int32_t E, int32_t k, double cf,
                                  moe_act act, moe_dtype dt, const moe_options* opt, void* y,
                                  void* ws, size_t ws_bytes, moe_stats* stats, void* stream) {
  moe_ws_layout L;
  int gating;
  float gate_scale;
  int priority;
  if (!compute_layout(T, d, H, E, k, cf, dt, act, &L)) return MOE_ERR_ARG;
  if (!read_options(opt, &gating, &gate_scale, &priority)) return MOE_ERR_ARG;
  if (T > 0 && (!forward_ptrs_ok(x, Wg, W1, W3, W2, act, y) || !ws || ws_bytes < L.total ||
                !aligned16(ws)))
    return MOE_ERR_ARG;
  if (T == 0) {
    if (stats) {
      memset(stats, 0, sizeof(*stats));
      stats->capacity = moe_capacity(T, E, k, cf);
    }
    return MOE_OK;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  moe_status st = forward_enqueue(x, Wg, bias, W1, W3, W2, T, d, H, E, k, cf, act, dt, y, ws,
                                  ws_bytes, L, s, true, opt);
  if (st != MOE_OK || !stats) return st;
  memset(stats, 0, sizeof(*stats));
  uint8_t* w = static_cast<uint8_t*>(ws);
  if (cudaMemcpyAsync(stats->counts, w + L.counts, sizeof(int32_t) * E, cudaMemcpyDeviceToHost,
                      s) != cudaSuccess ||
      cudaMemcpyAsync(stats->kept_counts, w + L.kept_counts, sizeof(int32_t) * E,
                      cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  st = read_device_error(L, ws, s, &stats->device_error);
  if (st != MOE_OK) return st;
  stats->assignments = static_cast<int64_t>(T) * k;
  for (int e = 0; e < E; ++e) stats->kept += stats->kept_counts[e];
  stats->capacity = moe_capacity(T, E, k, cf);
  return stats->device_error ? MOE_ERR_DEVICE : MOE_OK;
}

MOE_API moe_status moe_forward(const void* x, const void* Wg, const float* bias, const void* W1,
                               const void* W3, const void* W2, int32_t T, int32_t d, int32_t H,
                               int32_t E, int32_t k, double cf, moe_act act, moe_dtype dt, void* y,
                               void* ws, size_t ws_bytes, moe_stats* stats, void* stream) {
  return moe_forward_ex(x, Wg, bias, W1, W3, W2, T, d, H, E, k, cf, act, dt, nullptr, y, ws,
                        ws_bytes, stats, stream);
}

namespace {

// Copy streams and events for the chunked host forward, created once per
// device and kept for the life of the process (no device memory).
constexpr int kMaxHostChunks = 8;
struct HostPipe {
  bool ready = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t in[kMaxHostChunks] = {}, out[kMaxHostChunks] = {};
};
std::mutex g_pipe_mu;
HostPipe g_pipe[64];

moe_status host_pipe(int dev, HostPipe** out) {
  if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED;
  HostPipe& p = g_pipe[dev];
  if (!p.ready) {
    const unsigned f = cudaEventDisableTiming;
    if (cudaStreamCreateWithFlags(&p.h2d, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&p.d2h, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&p.start, f) != cudaSuccess ||
        cudaEventCreateWithFlags(&p.done, f) != cudaSuccess)
      return MOE_ERR_CUDA;
    for (int c = 0; c < kMaxHostChunks; ++c)
      if (cudaEventCreateWithFlags(&p.in[c], f) != cudaSuccess ||
          cudaEventCreateWithFlags(&p.out[c], f) != cudaSuccess)
        return MOE_ERR_CUDA;
    p.ready = true;
  }
  *out = &p;
  return MOE_OK;
}

// Dropless layers are split into up to 4 token chunks of >= 1024 tokens so
// the copy of chunk c+1 in and of chunk c-1 out overlap the forward of chunk
// c.  Tokens are independent without a capacity, so y is unchanged; with a
// capacity the batch stays whole (capacity is counted over the batch).
// MOE_HOST_CHUNKS (1 .. 8) overrides the upper bound, for measurements.
int host_chunks(int32_t T, double cf) {
  if (moe_capacity(T, 1, 1, cf) >= 0) return 1;
  static const int most = [] {
    const char* v = getenv("MOE_HOST_CHUNKS");
    const int n = v ? atoi(v) : 0;
    return (n >= 1 && n <= kMaxHostChunks) ? n : 4;
  }();
  int n = T / 1024;
  return n < 1 ? 1 : (n > most ? most : n);
}

}  // namespace

MOE_API moe_status moe_forward_host(const void* x_host, void* y_host, void* x_dev, void* y_dev,
                                    const void* Wg, const float* bias, const void* W1,
                                    const void* W3, const void* W2, int32_t T, int32_t d,
                                    int32_t H, int32_t E, int32_t k, double cf, moe_act act,
                                    moe_dtype dt, void* ws, size_t ws_bytes, void* stream) {
  moe_ws_layout L;
  if (!compute_layout(T, d, H, E, k, cf, dt, act, &L)) return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!x_host || !y_host || !forward_ptrs_ok(x_dev, Wg, W1, W3, W2, act, y_dev) || !ws ||
      ws_bytes < L.total || !aligned16(ws))
    return MOE_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t row_bytes = static_cast<size_t>(d) * elt_size(dt);
  const int nchunk = host_chunks(T, cf);
  if (nchunk == 1) {
    const size_t bytes = static_cast<size_t>(T) * row_bytes;
    if (cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    moe_status st = forward_enqueue(x_dev, Wg, bias, W1, W3, W2, T, d, H, E, k, cf, act, dt,
                                    y_dev, ws, ws_bytes, L, s);
    if (st != MOE_OK) return st;
    if (cudaMemcpyAsync(y_host, y_dev, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    int32_t derr = 0;
    st = read_device_error(L, ws, s, &derr);
    if (st != MOE_OK) return st;
    return derr ? MOE_ERR_DEVICE : MOE_OK;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe* p = nullptr;
  moe_status st = host_pipe(dev, &p);
  if (st != MOE_OK) return st;
  // Every chunk reuses the workspace on `s` in order; its layout for the
  // largest chunk fits inside the whole batch's.
  const int32_t base = T / nchunk, rem = T % nchunk;
  moe_ws_layout Lc;
  if (!compute_layout(base + (rem ? 1 : 0), d, H, E, k, cf, dt, act, &Lc)) return MOE_ERR_ARG;
  if (cudaMemsetAsync(static_cast<uint8_t*>(ws) + Lc.dev_error, 0, sizeof(int32_t), s) !=
          cudaSuccess ||
      cudaEventRecord(p->start, s) != cudaSuccess ||
      cudaStreamWaitEvent(p->h2d, p->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(p->d2h, p->start, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  int32_t t0 = 0;
  for (int c = 0; c < nchunk; ++c) {
    const int32_t tc = base + (c < rem ? 1 : 0);
    const size_t off = static_cast<size_t>(t0) * row_bytes, bytes = static_cast<size_t>(tc) * row_bytes;
    const uint8_t* xh = static_cast<const uint8_t*>(x_host) + off;
    uint8_t* xd = static_cast<uint8_t*>(x_dev) + off;
    uint8_t* yd = static_cast<uint8_t*>(y_dev) + off;
    uint8_t* yh = static_cast<uint8_t*>(y_host) + off;
    if (cudaMemcpyAsync(xd, xh, bytes, cudaMemcpyHostToDevice, p->h2d) != cudaSuccess ||
        cudaEventRecord(p->in[c], p->h2d) != cudaSuccess ||
        cudaStreamWaitEvent(s, p->in[c], 0) != cudaSuccess)
      return MOE_ERR_CUDA;
    // The largest chunk's layout serves every chunk (all regions are sized
    // for at least tc tokens), so the error word stays in one place.
    st = forward_enqueue(xd, Wg, bias, W1, W3, W2, tc, d, H, E, k, cf, act, dt, yd, ws, ws_bytes,
                         Lc, s, /*clear_err=*/false);
    if (st != MOE_OK) return st;
    if (cudaEventRecord(p->out[c], s) != cudaSuccess ||
        cudaStreamWaitEvent(p->d2h, p->out[c], 0) != cudaSuccess ||
        cudaMemcpyAsync(yh, yd, bytes, cudaMemcpyDeviceToHost, p->d2h) != cudaSuccess)
      return MOE_ERR_CUDA;
    t0 += tc;
  }
  if (cudaEventRecord(p->done, p->d2h) != cudaSuccess ||
      cudaStreamWaitEvent(s, p->done, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  int32_t derr = 0;
  st = read_device_error(Lc, ws, s, &derr);
  if (st != MOE_OK) return st;
  return derr ? MOE_ERR_DEVICE : MOE_OK;
}

// ======================================================= streaming pipeline
struct moe_pipeline {
  int depth = 0;
  int device = -1;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  struct Slot {
    cudaEvent_t in = nullptr;        // x copied in
    cudaEvent_t fwd_done = nullptr;  // forward finished (x_dev, ws free to rewrite)
    cudaEvent_t out_done = nullptr;  // y copied out (and the error word)
    bool used = false;
  } slot[MOE_PIPELINE_MAX_DEPTH];
  int32_t* err_host = nullptr;       // pinned, one word per slot
};

namespace {
void pipeline_release(moe_pipeline* p) {
  for (auto& sl : p->slot) {
    if (sl.in) cudaEventDestroy(sl.in);
    if (sl.fwd_done) cudaEventDestroy(sl.fwd_done);
    if (sl.out_done) cudaEventDestroy(sl.out_done);
  }
  if (p->h2d) cudaStreamDestroy(p->h2d);
  if (p->d2h) cudaStreamDestroy(p->d2h);
  if (p->err_host) cudaFreeHost(p->err_host);
  delete p;
}
}  // namespace

MOE_API moe_status moe_pipeline_create(int32_t depth, moe_pipeline** out) {
  if (!out || depth < 1 || depth > MOE_PIPELINE_MAX_DEPTH) return MOE_ERR_ARG;
  *out = nullptr;
  DeviceInfo di;
  moe_status st = device_info(&di);
  if (st != MOE_OK) return st;
  moe_pipeline* p = new moe_pipeline();
  p->depth = depth;
  p->device = di.device;
  const unsigned f = cudaEventDisableTiming;
  bool ok = cudaStreamCreateWithFlags(&p->h2d, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p->d2h, cudaStreamNonBlocking) == cudaSuccess &&
            cudaHostAlloc(reinterpret_cast<void**>(&p->err_host), sizeof(int32_t) * depth,
                          cudaHostAllocDefault) == cudaSuccess;
  for (int i = 0; ok && i < depth; ++i)
    ok = cudaEventCreateWithFlags(&p->slot[i].in, f) == cudaSuccess &&
         cudaEventCreateWithFlags(&p->slot[i].fwd_done, f) == cudaSuccess &&
         cudaEventCreateWithFlags(&p->slot[i].out_done, f) == cudaSuccess;
  if (!ok) {
    pipeline_release(p);
    return MOE_ERR_CUDA;
  }
  for (int i = 0; i < depth; ++i) p->err_host[i] = 0;
  *out = p;
  return MOE_OK;
}

MOE_API moe_status moe_pipeline_submit(moe_pipeline* p, int32_t slot, const void* x_host,
                                       void* y_host, void* x_dev, void* y_dev, const void* Wg,
                                       const float* bias, const void* W1, const void* W3,
                                       const void* W2, int32_t T, int32_t d, int32_t H,
                                       int32_t E, int32_t k, double cf, moe_act act,
                                       moe_dtype dt, const moe_options* opt, void* ws,
                                       size_t ws_bytes, void* stream) {
  if (!p || slot < 0 || slot >= p->depth) return MOE_ERR_ARG;
  moe_ws_layout L;
  int gating, priority;
  float gate_scale;
  if (!compute_layout(T, d, H, E, k, cf, dt, act, &L) ||
      !read_options(opt, &gating, &gate_scale, &priority))
    return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!x_host || !y_host || !forward_ptrs_ok(x_dev, Wg, W1, W3, W2, act, y_dev) || !ws ||
      ws_bytes < L.total || !aligned16(ws))
    return MOE_ERR_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev != p->device) return MOE_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto& sl = p->slot[slot];
  const size_t bytes = static_cast<size_t>(T) * d * elt_size(dt);
  // The slot's previous forward must be done with x_dev and ws, and its
  // previous copy-out done with y_dev, before they are rewritten.
  if (sl.used && (cudaStreamWaitEvent(p->h2d, sl.fwd_done, 0) != cudaSuccess ||
                  cudaStreamWaitEvent(s, sl.out_done, 0) != cudaSuccess))
    return MOE_ERR_CUDA;
  if (cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, p->h2d) != cudaSuccess ||
      cudaEventRecord(sl.in, p->h2d) != cudaSuccess ||
      cudaStreamWaitEvent(s, sl.in, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  moe_status st =
      forward_enqueue(x_dev, Wg, bias, W1, W3, W2, T, d, H, E, k, cf, act, dt, y_dev, ws, ws_bytes,
                      L, s, true, opt);
  if (st != MOE_OK) return st;
  if (cudaEventRecord(sl.fwd_done, s) != cudaSuccess ||
      cudaStreamWaitEvent(p->d2h, sl.fwd_done, 0) != cudaSuccess ||
      cudaMemcpyAsync(y_host, y_dev, bytes, cudaMemcpyDeviceToHost, p->d2h) != cudaSuccess ||
      cudaMemcpyAsync(p->err_host + slot, static_cast<uint8_t*>(ws) + L.dev_error,
                      sizeof(int32_t), cudaMemcpyDeviceToHost, p->d2h) != cudaSuccess ||
      cudaEventRecord(sl.out_done, p->d2h) != cudaSuccess)
    return MOE_ERR_CUDA;
  sl.used = true;
  return MOE_OK;
}

MOE_API moe_status moe_pipeline_wait(moe_pipeline* p, int32_t slot) {
  if (!p || slot < 0 || slot >= p->depth) return MOE_ERR_ARG;
  auto& sl = p->slot[slot];
  if (!sl.used) return MOE_OK;
  if (cudaEventSynchronize(sl.out_done) != cudaSuccess) return MOE_ERR_CUDA;
  return p->err_host[slot] ? MOE_ERR_DEVICE : MOE_OK;
}

MOE_API moe_status moe_pipeline_destroy(moe_pipeline* p) {
  if (!p) return MOE_OK;
  moe_status st = MOE_OK;
  for (int i = 0; i < p->depth; ++i)
    if (p->slot[i].used && cudaEventSynchronize(p->slot[i].out_done) != cudaSuccess)
      st = MOE_ERR_CUDA;
  pipeline_release(p);
  return st;
}

// ================================================================ graphs
struct moe_graph {
  cudaGraph_t graph;
  cudaGraphExec_t exec;
  int device;
};

MOE_API moe_status moe_forward_graph_create(const void* x, const void* Wg, const float* bias,
                                            const void* W1, const void* W3, const void* W2,
                                            int32_t T, int32_t d, int32_t H, int32_t E,
                                            int32_t k, double cf, moe_act act, moe_dtype dt,
                                            const moe_options* opt, void* y, void* ws,
                                            size_t ws_bytes, moe_graph** out) {
  if (!out) return MOE_ERR_ARG;
  *out = nullptr;
  moe_ws_layout L;
  int gating, priority;
  float gate_scale;
  if (!compute_layout(T, d, H, E, k, cf, dt, act, &L) ||
      !read_options(opt, &gating, &gate_scale, &priority))
    return MOE_ERR_ARG;
  if (T == 0 || !forward_ptrs_ok(x, Wg, W1, W3, W2, act, y) || !ws || ws_bytes < L.total ||
      !aligned16(ws))
    return MOE_ERR_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t cs = nullptr;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return MOE_ERR_CUDA;
  // Stage events are never recorded into a graph.
  const bool events_on = g_stage_events_on;
  g_stage_events_on = false;
  moe_status st = MOE_OK;
  cudaGraph_t graph = nullptr;
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    st = MOE_ERR_CUDA;
  } else {
    st = forward_enqueue(x, Wg, bias, W1, W3, W2, T, d, H, E, k, cf, act, dt, y, ws, ws_bytes, L,
                         cs, true, opt);
    // The capture always ends, whatever the enqueue returned.
    if (cudaStreamEndCapture(cs, &graph) != cudaSuccess && st == MOE_OK) st = MOE_ERR_CUDA;
  }
  g_stage_events_on = events_on;
  cudaGraphExec_t exec = nullptr;
  if (st == MOE_OK && (!graph || cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess))
    st = MOE_ERR_CUDA;
  cudaStreamDestroy(cs);
  moe_graph* g = nullptr;
  if (st == MOE_OK) {
    g = static_cast<moe_graph*>(malloc(sizeof(moe_graph)));
    if (!g) st = MOE_ERR_CUDA;
  }
  if (st != MOE_OK) {
    if (exec) cudaGraphExecDestroy(exec);
    if (graph) cudaGraphDestroy(graph);
    cudaGetLastError();  // a failed capture leaves no sticky error behind
    return st;
  }
  g->graph = graph;
  g->exec = exec;
  g->device = dev;
  *out = g;
  return MOE_OK;
}

MOE_API moe_status moe_forward_graph_launch(moe_graph* g, void* stream) {
  if (!g) return MOE_ERR_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev != g->device) return MOE_ERR_ARG;
  return cudaGraphLaunch(g->exec, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

MOE_API moe_status moe_forward_graph_nodes(const moe_graph* g, int32_t* kernels,
                                           int32_t* others) {
  if (!g || !kernels || !others) return MOE_ERR_ARG;
  size_t n = 0;
  if (cudaGraphGetNodes(g->graph, nullptr, &n) != cudaSuccess) return MOE_ERR_CUDA;
  cudaGraphNode_t nodes[64];
  if (n > 64) return MOE_ERR_CUDA;  // a forward holds a handful of nodes
  if (n > 0 && cudaGraphGetNodes(g->graph, nodes, &n) != cudaSuccess) return MOE_ERR_CUDA;
  int32_t nk = 0, no = 0;
  for (size_t i = 0; i < n; ++i) {
    cudaGraphNodeType t;
    if (cudaGraphNodeGetType(nodes[i], &t) != cudaSuccess) return MOE_ERR_CUDA;
    if (t == cudaGraphNodeTypeKernel) ++nk;
    else ++no;
  }
  *kernels = nk;
  *others = no;
  return MOE_OK;
}

MOE_API moe_status moe_forward_graph_destroy(moe_graph* g) {
  if (!g) return MOE_OK;
  moe_status st = MOE_OK;
  if (cudaGraphExecDestroy(g->exec) != cudaSuccess) st = MOE_ERR_CUDA;
  if (cudaGraphDestroy(g->graph) != cudaSuccess) st = MOE_ERR_CUDA;
  free(g);
  return st;
}

// ============================================================ expert choice
namespace {

bool ec_layout(int32_t T, int32_t d, int32_t H, int32_t E, int32_t k, double cf, moe_dtype dt,
               moe_act act, moe_ec_ws_layout* L) {
  if (T < 0 || d <= 0 || d % 8 != 0 || E < 1 || E > kMaxE || k < 1 || k > E ||
      !valid_ffn_sizes(d, H) || !valid_dtype(dt) || !valid_act(act))
    return false;
  const int32_t n = moe_expert_choice_tokens(T, E, k, cf);
  if (n < 0) return false;
  const int64_t npad = pad_rows(n);
  const int64_t rows = static_cast<int64_t>(E) * npad;
  if (rows > INT32_MAX || static_cast<int64_t>(T) * E > INT32_MAX) return false;
  const size_t es = elt_size(dt);
  const size_t te = static_cast<size_t>(T) * E;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  memset(L, 0, sizeof(*L));
  L->scores = take(te * 4);
  L->pos = take(te * 4);
  L->tok = take(static_cast<size_t>(E) * n * 4);
  L->kept_counts = take(kMaxE * 4);
  L->offsets = take((kMaxE + 1) * 4);
  L->dev_error = take(4);
  L->scratch = take(ec_select_scratch_bytes(T, E));
  L->xp = take(static_cast<size_t>(rows) * d * es);
  L->h = take(static_cast<size_t>(rows) * H * es);
  L->o = take(static_cast<size_t>(rows) * d * es);
  L->total = off;
  L->rows = rows;
  L->n = n;
  return true;
}

}  // namespace

MOE_API int32_t moe_expert_choice_tokens(int32_t T, int32_t E, int32_t k, double cf) {
  if (T < 0 || E < 1 || k < 1 || k > E) return -1;
  const int32_t C = moe_capacity(T, E, k, cf);
  return C < 0 ? -1 : std::min(C, T);
}

namespace {
moe_status ec_route_enqueue(const void* x, const void* Wg, const float* bias, int32_t T, int32_t d,
                            int32_t E, moe_dtype dt, float* scores, void* stream, int32_t* err) {
  if (T < 0 || d <= 0 || d % 8 != 0 || E < 1 || E > kMaxE || !valid_dtype(dt)) return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !Wg || !scores || !aligned16(x) || !aligned16(Wg)) return MOE_ERR_ARG;
  DeviceInfo di;
  moe_status st = device_info(&di);
  if (st != MOE_OK) return st;
  RouteArgs a{x, Wg, bias, T, d, E, 1, nullptr, nullptr, nullptr, MOE_GATE_TOPK_SOFTMAX, 1.0f,
              scores};
  a.err = err;
  return launch_route(a, dt, static_cast<cudaStream_t>(stream), di.num_sms) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
}  // namespace

MOE_API moe_status moe_expert_choice_route(const void* x, const void* Wg, const float* bias,
                                           int32_t T, int32_t d, int32_t E, moe_dtype dt,
                                           float* scores, void* stream) {
  return ec_route_enqueue(x, Wg, bias, T, d, E, dt, scores, stream, nullptr);
}

MOE_API size_t moe_expert_choice_select_workspace_bytes(int32_t T, int32_t E) {
  if (T < 0 || E < 1 || E > kMaxE) return 0;
  return ec_select_scratch_bytes(T, E);
}

MOE_API moe_status moe_expert_choice_select(const float* scores, int32_t T, int32_t E, int32_t n,
                                            int32_t* tok, int32_t* pos, int32_t* kept_counts,
                                            int32_t* offsets, void* ws, size_t ws_bytes,
                                            void* stream) {
  if (T < 0 || E < 1 || E > kMaxE || n < 0 || n > T) return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!scores || !pos || !kept_counts || !offsets || !ws || !aligned16(ws) ||
      ws_bytes < ec_select_scratch_bytes(T, E) || (n > 0 && !tok))
    return MOE_ERR_ARG;
  DeviceInfo di;
  moe_status st = device_info(&di);
  if (st != MOE_OK) return st;
  return launch_ec_select(scores, T, E, n, static_cast<int>(pad_rows(n)), ws, tok, pos,
                          kept_counts, offsets, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

MOE_API moe_status moe_expert_choice_permute(const void* x, const int32_t* pos, int32_t T,
                                             int32_t d, int32_t E, int32_t n, moe_dtype dt,
                                             void* xp, int64_t xp_rows, void* stream) {
  if (T < 0 || d <= 0 || d % 8 != 0 || E < 1 || E > kMaxE || n < 0 || n > T || !valid_dtype(dt))
    return MOE_ERR_ARG;
  if (n == 0) return MOE_OK;
  if (!x || !pos || !xp || !aligned16(x) || !aligned16(xp) ||
      xp_rows < static_cast<int64_t>(E) * pad_rows(n))
    return MOE_ERR_ARG;
  DeviceInfo di;
  moe_status st = device_info(&di);
  if (st != MOE_OK) return st;
  return launch_row_copy(x, pos, T, E, d, dt, xp, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

MOE_API moe_status moe_expert_choice_combine(const void* o, const int32_t* pos,
                                             const float* scores, int32_t T, int32_t d,
                                             int32_t E, moe_dtype dt, void* y, void* stream) {
  if (T < 0 || d <= 0 || d % 8 != 0 || E < 1 || E > kMaxE || !valid_dtype(dt)) return MOE_ERR_ARG;
  if (T == 0) return MOE_OK;
  if (!o || !pos || !scores || !y || !aligned16(o) || !aligned16(y)) return MOE_ERR_ARG;
  DeviceInfo di;
  moe_status st = device_info(&di);
  if (st != MOE_OK) return st;
  return launch_ec_combine(o, pos, scores, T, d, E, dt, y, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

MOE_API moe_status moe_expert_choice_layout(int32_t T, int32_t d, int32_t H, int32_t E, int32_t k,
                                            double cf, moe_dtype dt, moe_act act,
                                            moe_ec_ws_layout* layout) {
  if (!layout) return MOE_ERR_ARG;
  return ec_layout(T, d, H, E, k, cf, dt, act, layout) ? MOE_OK : MOE_ERR_ARG;
}

MOE_API size_t moe_expert_choice_workspace_bytes(int32_t T, int32_t d, int32_t H, int32_t E,
                                                 int32_t k, double cf, moe_dtype dt,
                                                 moe_act act) {
  moe_ec_ws_layout L;
  return ec_layout(T, d, H, E, k, cf, dt, act, &L) ? L.total : 0;
}

MOE_API moe_status moe_forward_expert_choice(const void* x, const void* Wg, const float* bias,
                                             const void* W1, const void* W3, const void* W2,
                                             int32_t T, int32_t d, int32_t H, int32_t E,
                                             int32_t k, double cf, moe_act act, moe_dtype dt,
                                             void* y, void* ws, size_t ws_bytes,
                                             moe_stats* stats, void* stream) {
  moe_ec_ws_layout L;
  if (!ec_layout(T, d, H, E, k, cf, dt, act, &L)) return MOE_ERR_ARG;
  if (T > 0 && (!forward_ptrs_ok(x, Wg, W1, W3, W2, act, y) || !ws || ws_bytes < L.total ||
                !aligned16(ws)))
    return MOE_ERR_ARG;
  if (stats) memset(stats, 0, sizeof(*stats));
  if (T == 0) {
    if (stats) stats->capacity = moe_capacity(T, E, k, cf);
    return MOE_OK;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* scores = reinterpret_cast<float*>(w + L.scores);
  int32_t* pos = reinterpret_cast<int32_t*>(w + L.pos);
  int32_t* tok = reinterpret_cast<int32_t*>(w + L.tok);
  int32_t* kept = reinterpret_cast<int32_t*>(w + L.kept_counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(w + L.offsets);
  int32_t* err = reinterpret_cast<int32_t*>(w + L.dev_error);
  if (cudaMemsetAsync(err, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  moe_status st = record_stage(0, s);
  if (st == MOE_OK) st = ec_route_enqueue(x, Wg, bias, T, d, E, dt, scores, s, err);
  if (st == MOE_OK) st = record_stage(1, s);
  if (st == MOE_OK)
    st = moe_expert_choice_select(scores, T, E, L.n, tok, pos, kept, offsets, w + L.scratch,
                                  ec_select_scratch_bytes(T, E), s);
  if (st == MOE_OK) st = moe_expert_choice_permute(x, pos, T, d, E, L.n, dt, w + L.xp, L.rows, s);
  if (st == MOE_OK) st = record_stage(2, s);
  if (st == MOE_OK && L.rows > 0)
    st = moe_grouped_ffn(w + L.xp, L.rows, offsets, kept, W1, W3, W2, E, d, H, act, dt, w + L.h,
                         w + L.o, err, s);
  else if (st == MOE_OK)
    st = record_stage(3, s);
  if (st == MOE_OK) st = record_stage(4, s);
  if (st == MOE_OK)
    st = moe_expert_choice_combine(w + L.o, pos, scores, T, d, E, dt, y,
                                   s);
  if (st == MOE_OK) st = record_stage(5, s);
  if (st != MOE_OK || !stats) return st;
  for (int e = 0; e < E; ++e) stats->counts[e] = stats->kept_counts[e] = L.n;
  stats->assignments = static_cast<int64_t>(E) * L.n;
  stats->kept = stats->assignments;
  stats->capacity = moe_capacity(T, E, k, cf);
  if (cudaMemcpyAsync(&stats->device_error, err, sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return stats->device_error ? MOE_ERR_DEVICE : MOE_OK;
}

MOE_API moe_status moe_probe_stream_read(const void* buf, size_t bytes, uint32_t* sink,
                                         void* stream) {
  if (bytes == 0) return MOE_OK;
  if (!buf || !sink || bytes % 16 != 0 || !aligned16(buf)) return MOE_ERR_ARG;
  DeviceInfo di;
  moe_status st = device_info(&di);
  if (st != MOE_OK) return st;
  return launch_stream_read(buf, bytes, sink, di.num_sms, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
