"""Thin Python binding of libmoe.so (include/moe.h), by the same names.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch provides device memory and the current stream.  Functions
accept torch tensors, allocate missing outputs with torch, pass raw pointers
through ctypes and raise ``MoeError`` on any non-OK status.  There is no
fallback: if libmoe.so is missing or was not built, the first call raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")

MOE_OK, MOE_ERR_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_DEVICE = range(5)
MOE_BF16, MOE_FP32 = 0, 1
MOE_SWIGLU, MOE_GELU = 0, 1
MOE_MAX_EXPERTS = 64
MOE_MAX_TOPK = 8
MOE_ROW_ALIGN = 128

EXPORTED = (
    "moe_status_string", "moe_abi_version", "moe_capacity", "moe_max_permuted_rows",
    "moe_permute_workspace_bytes", "moe_workspace_bytes", "moe_workspace_layout",
    "moe_route", "moe_permute", "moe_grouped_ffn", "moe_unpermute_combine",
    "moe_forward", "moe_forward_host", "moe_set_stage_events", "moe_permute_static",
    "moe_route_ex", "moe_forward_ex", "moe_permute_ex", "moe_priority_order",
    "moe_priority_workspace_bytes", "moe_rows_for_capacity", "moe_expert_counts",
    "moe_rank_prefix", "moe_expert_choice_tokens", "moe_expert_choice_route",
    "moe_expert_choice_select_workspace_bytes", "moe_expert_choice_select",
    "moe_expert_choice_permute", "moe_expert_choice_combine", "moe_expert_choice_layout",
    "moe_expert_choice_workspace_bytes", "moe_forward_expert_choice", "moe_pipeline_create",
    "moe_pipeline_submit", "moe_pipeline_wait", "moe_pipeline_destroy",
    "moe_forward_graph_create", "moe_forward_graph_launch", "moe_forward_graph_destroy",
    "moe_forward_graph_nodes",
    "moe_probe_stream_read",
)
MOE_PIPELINE_MAX_DEPTH = 4
MOE_ABI_VERSION = 2
MOE_GATE_TOPK_SOFTMAX, MOE_GATE_SOFTMAX_TOPK = 0, 1
MOE_PRIORITY_POSITION, MOE_PRIORITY_GATE = 0, 1
MOE_PERMUTE_STATIC_MAX_INTS = 1 << 18
MOE_NUM_STAGE_EVENTS = 6
STAGES = ("route", "permute", "ffn_up", "ffn_down", "combine")


class MoeError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class moe_stats(ctypes.Structure):
    _fields_ = [
        ("counts", ctypes.c_int32 * MOE_MAX_EXPERTS),
        ("kept_counts", ctypes.c_int32 * MOE_MAX_EXPERTS),
        ("assignments", ctypes.c_int64),
        ("kept", ctypes.c_int64),
        ("capacity", ctypes.c_int32),
        ("device_error", ctypes.c_int32),
    ]


class moe_options(ctypes.Structure):
    _fields_ = [("gating", ctypes.c_int32), ("gate_scale", ctypes.c_float),
                ("priority", ctypes.c_int32), ("reserved", ctypes.c_int32 * 5)]


def _options(gating="topk_softmax", gate_scale=1.0, priority="position"):
    if gating in ("topk_softmax", MOE_GATE_TOPK_SOFTMAX):
        g = MOE_GATE_TOPK_SOFTMAX
    elif gating in ("softmax_topk", MOE_GATE_SOFTMAX_TOPK):
        g = MOE_GATE_SOFTMAX_TOPK
    else:
        raise ValueError(gating)
    if priority in ("position", MOE_PRIORITY_POSITION):
        pr = MOE_PRIORITY_POSITION
    elif priority in ("gate", MOE_PRIORITY_GATE):
        pr = MOE_PRIORITY_GATE
    else:
        raise ValueError(priority)
    return moe_options(gating=g, gate_scale=float(gate_scale), priority=pr)


class moe_ws_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "idx", "gate", "margin", "pos", "counts", "kept_counts", "offsets", "dev_error",
        "scratch", "xp", "h", "o", "total")] + [("rows", ctypes.c_int64),
                                                 ("order", ctypes.c_size_t),
                                                 ("prio_scratch", ctypes.c_size_t)]


class moe_ec_ws_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "scores", "pos", "tok", "kept_counts", "offsets", "dev_error", "scratch", "xp", "h", "o",
        "total")] + [("rows", ctypes.c_int64), ("n", ctypes.c_int32)]


_lib_handle = None
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_D = ctypes.c_double
_SZ = ctypes.c_size_t


def lib():
    """The loaded libmoe.so (raises if it has not been built)."""
    global _lib_handle
    if _lib_handle is not None:
        return _lib_handle
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(
            f"{_LIB_PATH} is missing: build it with "
            "`python -m mixture_experts_layer_51_b200.build` (there is no CPU fallback)")
    L = ctypes.CDLL(_LIB_PATH)
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_status_string.argtypes = [ctypes.c_int]
    L.moe_abi_version.restype = _I32
    if L.moe_abi_version() != MOE_ABI_VERSION:
        raise RuntimeError(
            f"{_LIB_PATH} has ABI version {L.moe_abi_version()}, this binding expects "
            f"{MOE_ABI_VERSION}: rebuild it with `python -m mixture_experts_layer_51_b200.build`")
    L.moe_capacity.restype = _I32
    L.moe_capacity.argtypes = [_I32, _I32, _I32, _D]
    L.moe_max_permuted_rows.restype = _I64
    L.moe_max_permuted_rows.argtypes = [_I32, _I32, _I32, _D]
    L.moe_permute_workspace_bytes.restype = _SZ
    L.moe_permute_workspace_bytes.argtypes = [_I32, _I32]
    L.moe_workspace_bytes.restype = _SZ
    L.moe_workspace_bytes.argtypes = [_I32, _I32, _I32, _I32, _I32, _D, ctypes.c_int, ctypes.c_int]
    L.moe_workspace_layout.restype = ctypes.c_int
    L.moe_workspace_layout.argtypes = [_I32, _I32, _I32, _I32, _I32, _D, ctypes.c_int,
                                       ctypes.c_int, ctypes.POINTER(moe_ws_layout)]
    L.moe_route.restype = ctypes.c_int
    L.moe_route.argtypes = [_P, _P, _P, _I32, _I32, _I32, _I32, ctypes.c_int, _P, _P, _P, _P]
    L.moe_permute.restype = ctypes.c_int
    L.moe_permute.argtypes = [_P, _P, _I32, _I32, _I32, _I32, _D, ctypes.c_int, _P, _I64, _P,
                              _P, _P, _P, _P, _SZ, _P]
    L.moe_grouped_ffn.restype = ctypes.c_int
    L.moe_grouped_ffn.argtypes = [_P, _I64, _P, _P, _P, _P, _P, _I32, _I32, _I32, ctypes.c_int,
                                  ctypes.c_int, _P, _P, _P, _P]
    L.moe_unpermute_combine.restype = ctypes.c_int
    L.moe_unpermute_combine.argtypes = [_P, _P, _P, _I32, _I32, _I32, ctypes.c_int, _P, _P]
    L.moe_forward.restype = ctypes.c_int
    L.moe_forward.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _D,
                              ctypes.c_int, ctypes.c_int, _P, _P, _SZ,
                              ctypes.POINTER(moe_stats), _P]
    L.moe_forward_host.restype = ctypes.c_int
    L.moe_forward_host.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32,
                                   _I32, _D, ctypes.c_int, ctypes.c_int, _P, _SZ, _P]
    L.moe_permute_static.restype = ctypes.c_int
    L.moe_permute_static.argtypes = [_P, _P, _I32, _I32, _I32, _I32, _D, ctypes.c_int, _P, _I64,
                                     _P, _P, _P, _P, _P]
    L.moe_route_ex.restype = ctypes.c_int
    L.moe_route_ex.argtypes = [_P, _P, _P, _I32, _I32, _I32, _I32, ctypes.c_int,
                               ctypes.POINTER(moe_options), _P, _P, _P, _P]
    L.moe_forward_ex.restype = ctypes.c_int
    L.moe_forward_ex.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _D,
                                 ctypes.c_int, ctypes.c_int, ctypes.POINTER(moe_options), _P, _P,
                                 _SZ, ctypes.POINTER(moe_stats), _P]
    L.moe_permute_ex.restype = ctypes.c_int
    L.moe_permute_ex.argtypes = [_P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, ctypes.c_int, _P,
                                 _I64, _P, _P, _P, _P, _P, _SZ, _P]
    L.moe_rows_for_capacity.restype = _I64
    L.moe_rows_for_capacity.argtypes = [_I32, _I32, _I32, _I32]
    L.moe_expert_counts.restype = ctypes.c_int
    L.moe_expert_counts.argtypes = [_P, _I32, _I32, _I32, _P, _P]
    L.moe_rank_prefix.restype = ctypes.c_int
    L.moe_rank_prefix.argtypes = [_P, _I32, _I32, _I32, _P, _P]
    L.moe_expert_choice_tokens.restype = _I32
    L.moe_expert_choice_tokens.argtypes = [_I32, _I32, _I32, _D]
    L.moe_expert_choice_route.restype = ctypes.c_int
    L.moe_expert_choice_route.argtypes = [_P, _P, _P, _I32, _I32, _I32, ctypes.c_int, _P, _P]
    L.moe_expert_choice_select_workspace_bytes.restype = _SZ
    L.moe_expert_choice_select_workspace_bytes.argtypes = [_I32, _I32]
    L.moe_expert_choice_select.restype = ctypes.c_int
    L.moe_expert_choice_select.argtypes = [_P, _I32, _I32, _I32, _P, _P, _P, _P, _P, _SZ, _P]
    L.moe_expert_choice_permute.restype = ctypes.c_int
    L.moe_expert_choice_permute.argtypes = [_P, _P, _I32, _I32, _I32, _I32, ctypes.c_int, _P,
                                            _I64, _P]
    L.moe_expert_choice_combine.restype = ctypes.c_int
    L.moe_expert_choice_combine.argtypes = [_P, _P, _P, _I32, _I32, _I32, ctypes.c_int, _P, _P]
    L.moe_expert_choice_layout.restype = ctypes.c_int
    L.moe_expert_choice_layout.argtypes = [_I32, _I32, _I32, _I32, _I32, _D, ctypes.c_int,
                                           ctypes.c_int, ctypes.POINTER(moe_ec_ws_layout)]
    L.moe_expert_choice_workspace_bytes.restype = _SZ
    L.moe_expert_choice_workspace_bytes.argtypes = [_I32, _I32, _I32, _I32, _I32, _D,
                                                    ctypes.c_int, ctypes.c_int]
    L.moe_pipeline_create.restype = ctypes.c_int
    L.moe_pipeline_create.argtypes = [_I32, ctypes.POINTER(ctypes.c_void_p)]
    L.moe_pipeline_submit.restype = ctypes.c_int
    L.moe_pipeline_submit.argtypes = [_P, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _I32,
                                      _I32, _I32, _I32, _D, ctypes.c_int, ctypes.c_int,
                                      ctypes.POINTER(moe_options), _P, _SZ, _P]
    L.moe_pipeline_wait.restype = ctypes.c_int
    L.moe_pipeline_wait.argtypes = [_P, _I32]
    L.moe_pipeline_destroy.restype = ctypes.c_int
    L.moe_pipeline_destroy.argtypes = [_P]
    L.moe_forward_graph_create.restype = ctypes.c_int
    L.moe_forward_graph_create.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32,
                                           ctypes.c_double, ctypes.c_int, ctypes.c_int, _P, _P,
                                           _P, ctypes.c_size_t, ctypes.POINTER(ctypes.c_void_p)]
    L.moe_forward_graph_launch.restype = ctypes.c_int
    L.moe_forward_graph_launch.argtypes = [_P, _P]
    L.moe_forward_graph_destroy.restype = ctypes.c_int
    L.moe_forward_graph_destroy.argtypes = [_P]
    L.moe_forward_graph_nodes.restype = ctypes.c_int
    L.moe_forward_graph_nodes.argtypes = [_P, _P, _P]
    L.moe_forward_expert_choice.restype = ctypes.c_int
    L.moe_forward_expert_choice.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32,
                                            _D, ctypes.c_int, ctypes.c_int, _P, _P, _SZ,
                                            ctypes.POINTER(moe_stats), _P]
    L.moe_priority_workspace_bytes.restype = _SZ
    L.moe_priority_workspace_bytes.argtypes = [_I32]
    L.moe_priority_order.restype = ctypes.c_int
    L.moe_priority_order.argtypes = [_P, _I32, _I32, _P, _P, _SZ, _P]
    L.moe_set_stage_events.restype = ctypes.c_int
    L.moe_set_stage_events.argtypes = [ctypes.POINTER(ctypes.c_void_p)]
    L.moe_probe_stream_read.restype = ctypes.c_int
    L.moe_probe_stream_read.argtypes = [_P, _SZ, _P, _P]
    _lib_handle = L
    return L


# ------------------------------------------------------------------ helpers
def status_string(status):
    return lib().moe_status_string(int(status)).decode()


def _check(status, where):
    if status != MOE_OK:
        raise MoeError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    if t.dtype == torch.float32:
        return MOE_FP32
    raise TypeError(f"unsupported dtype {t.dtype}: use bfloat16 or float32")


def _act_code(act):
    if act in ("swiglu", MOE_SWIGLU):
        return MOE_SWIGLU
    if act in ("gelu", MOE_GELU):
        return MOE_GELU
    raise ValueError(act)


def _stream(device, stream=None):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _cf(capacity_factor):
    return 0.0 if capacity_factor is None else float(capacity_factor)


def moe_capacity(T, E, k, capacity_factor):
    return lib().moe_capacity(T, E, k, _cf(capacity_factor))


def moe_max_permuted_rows(T, E, k, capacity_factor):
    return lib().moe_max_permuted_rows(T, E, k, _cf(capacity_factor))


def moe_permute_workspace_bytes(T, E):
    return lib().moe_permute_workspace_bytes(T, E)


def moe_workspace_bytes(T, d, H, E, k, capacity_factor, dtype, act):
    code = MOE_BF16 if dtype in (torch.bfloat16, "bf16") else MOE_FP32
    return lib().moe_workspace_bytes(T, d, H, E, k, _cf(capacity_factor), code, _act_code(act))


def moe_workspace_layout(T, d, H, E, k, capacity_factor, dtype, act):
    code = MOE_BF16 if dtype in (torch.bfloat16, "bf16") else MOE_FP32
    L = moe_ws_layout()
    _check(lib().moe_workspace_layout(T, d, H, E, k, _cf(capacity_factor), code, _act_code(act),
                                      ctypes.byref(L)), "moe_workspace_layout")
    return L


def workspace_views(ws, layout, T, d, H, E, k, dtype):
    """Tensor views of the intermediates inside a moe_forward workspace."""
    def view(off, n, dt):
        nbytes = n * torch.empty((), dtype=dt).element_size()
        return ws[off:off + nbytes].view(dt)
    rows = layout.rows
    return dict(
        idx=view(layout.idx, T * k, torch.int32).view(T, k),
        gate=view(layout.gate, T * k, torch.float32).view(T, k),
        margin=view(layout.margin, T, torch.float32),
        pos=view(layout.pos, T * k, torch.int32).view(T, k),
        counts=view(layout.counts, E, torch.int32),
        kept_counts=view(layout.kept_counts, E, torch.int32),
        offsets=view(layout.offsets, E + 1, torch.int32),
        order=view(layout.order, T, torch.int32),
        dev_error=view(layout.dev_error, 1, torch.int32),
        xp=view(layout.xp, rows * d, dtype).view(rows, d),
        h=view(layout.h, rows * H, dtype).view(rows, H),
        o=view(layout.o, rows * d, dtype).view(rows, d),
    )


# ------------------------------------------------------------- entry points
def moe_route(x, Wg, bias, k, idx=None, gate=None, margin=None, stream=None,
              gating="topk_softmax", gate_scale=1.0):
    T, d = x.shape
    E = Wg.shape[1]
    dev = x.device
    idx = idx if idx is not None else torch.empty((T, k), dtype=torch.int32, device=dev)
    gate = gate if gate is not None else torch.empty((T, k), dtype=torch.float32, device=dev)
    margin = margin if margin is not None else torch.empty((T,), dtype=torch.float32, device=dev)
    opt = _options(gating, gate_scale)
    _check(lib().moe_route_ex(_ptr(x), _ptr(Wg), _ptr(bias), T, d, E, k, _dtype_code(x),
                              ctypes.byref(opt), _ptr(idx), _ptr(gate), _ptr(margin),
                              _stream(dev, stream)), "moe_route_ex")
    return idx, gate, margin


def moe_priority_order(gate, order=None, ws=None, stream=None):
    """Tokens by descending slot-0 gate, ties in position order (int32 [T])."""
    T, k = gate.shape
    dev = gate.device
    order = order if order is not None else torch.empty(T, dtype=torch.int32, device=dev)
    need = lib().moe_priority_workspace_bytes(T)
    ws = ws if ws is not None else torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(lib().moe_priority_order(_ptr(gate), T, k, _ptr(order), _ptr(ws), ws.numel(),
                                    _stream(dev, stream)), "moe_priority_order")
    return order


def moe_rows_for_capacity(T, E, k, capacity):
    return lib().moe_rows_for_capacity(T, E, k, -1 if capacity is None else int(capacity))


def moe_expert_counts(idx, E, counts=None, stream=None):
    """Per-expert assignment counts of idx [T, k] (int32 [E])."""
    T, k = idx.shape
    dev = idx.device
    counts = counts if counts is not None else torch.empty(E, dtype=torch.int32, device=dev)
    _check(lib().moe_expert_counts(_ptr(idx), T, E, k, _ptr(counts), _stream(dev, stream)),
           "moe_expert_counts")
    return counts


def moe_rank_prefix(gathered, rank, prior=None, stream=None):
    """prior[e] = sum of gathered[r, e] over r < rank (int32 [E])."""
    n, E = gathered.shape
    dev = gathered.device
    prior = prior if prior is not None else torch.empty(E, dtype=torch.int32, device=dev)
    _check(lib().moe_rank_prefix(_ptr(gathered), n, E, rank, _ptr(prior), _stream(dev, stream)),
           "moe_rank_prefix")
    return prior


def moe_permute(x, idx, E, capacity_factor, xp=None, pos=None, counts=None, kept_counts=None,
                offsets=None, ws=None, stream=None, order=None, prior=None, capacity=None):
    """Counting-sort permutation.  capacity (int, or None = from
    capacity_factor over this T) and prior (int32 [E] of earlier shards'
    assignments) serve a batch sharded over ranks."""
    T, d = x.shape
    k = idx.shape[1]
    dev = x.device
    C = moe_capacity(T, E, k, capacity_factor) if capacity is None else int(capacity)
    rows = moe_rows_for_capacity(T, E, k, C)
    xp = xp if xp is not None else torch.empty((max(rows, 0), d), dtype=x.dtype, device=dev)
    pos = pos if pos is not None else torch.empty((T, k), dtype=torch.int32, device=dev)
    counts = counts if counts is not None else torch.empty(E, dtype=torch.int32, device=dev)
    kept_counts = kept_counts if kept_counts is not None else torch.empty(E, dtype=torch.int32, device=dev)
    offsets = offsets if offsets is not None else torch.empty(E + 1, dtype=torch.int32, device=dev)
    wsb = moe_permute_workspace_bytes(T, E)
    ws = ws if ws is not None else torch.empty(wsb, dtype=torch.uint8, device=dev)
    _check(lib().moe_permute_ex(_ptr(x), _ptr(idx), _ptr(order), _ptr(prior), T, d, E, k,
                                C, _dtype_code(x), _ptr(xp), xp.shape[0],
                                _ptr(pos), _ptr(counts), _ptr(kept_counts), _ptr(offsets),
                                _ptr(ws), ws.numel(), _stream(dev, stream)), "moe_permute_ex")
    return dict(xp=xp, pos=pos, counts=counts, kept_counts=kept_counts, offsets=offsets)


def moe_permute_static(x, idx, E, capacity_factor, xp=None, pos=None, counts=None,
                       kept_counts=None, offsets=None, stream=None):
    """moe_permute using the library's own fixed scratch (no allocation by the
    library; outputs allocated here when not given)."""
    T, d = x.shape
    k = idx.shape[1]
    dev = x.device
    rows = moe_max_permuted_rows(T, E, k, capacity_factor)
    xp = xp if xp is not None else torch.empty((max(rows, 0), d), dtype=x.dtype, device=dev)
    pos = pos if pos is not None else torch.empty((T, k), dtype=torch.int32, device=dev)
    counts = counts if counts is not None else torch.empty(E, dtype=torch.int32, device=dev)
    kept_counts = kept_counts if kept_counts is not None else torch.empty(E, dtype=torch.int32, device=dev)
    offsets = offsets if offsets is not None else torch.empty(E + 1, dtype=torch.int32, device=dev)
    _check(lib().moe_permute_static(_ptr(x), _ptr(idx), T, d, E, k, _cf(capacity_factor),
                                    _dtype_code(x), _ptr(xp), xp.shape[0], _ptr(pos),
                                    _ptr(counts), _ptr(kept_counts), _ptr(offsets),
                                    _stream(dev, stream)), "moe_permute_static")
    return dict(xp=xp, pos=pos, counts=counts, kept_counts=kept_counts, offsets=offsets)


def moe_grouped_ffn(xp, offsets, kept_counts, W1, W3, W2, act, h=None, o=None, dev_error=None,
                    stream=None):
    rows, d = xp.shape
    E, _, H = W1.shape
    dev = xp.device
    h = h if h is not None else torch.empty((rows, H), dtype=xp.dtype, device=dev)
    o = o if o is not None else torch.empty((rows, d), dtype=xp.dtype, device=dev)
    dev_error = dev_error if dev_error is not None else torch.zeros(1, dtype=torch.int32, device=dev)
    _check(lib().moe_grouped_ffn(_ptr(xp), rows, _ptr(offsets), _ptr(kept_counts), _ptr(W1),
                                 _ptr(W3), _ptr(W2), E, d, H, _act_code(act), _dtype_code(xp),
                                 _ptr(h), _ptr(o), _ptr(dev_error), _stream(dev, stream)),
           "moe_grouped_ffn")
    return h, o, dev_error


def moe_unpermute_combine(o, pos, gate, dtype, y=None, stream=None):
    """y [T, d] (dtype) from the expert outputs o, which are in the layer
    dtype too."""
    if o.dtype != dtype:
        raise TypeError(f"o is {o.dtype}; the combine reads o in the layer dtype {dtype}")
    T, k = pos.shape
    d = o.shape[1]
    dev = o.device
    y = y if y is not None else torch.empty((T, d), dtype=dtype, device=dev)
    _check(lib().moe_unpermute_combine(_ptr(o), _ptr(pos), _ptr(gate), T, d, k,
                                       _dtype_code(y), _ptr(y), _stream(dev, stream)),
           "moe_unpermute_combine")
    return y


def moe_forward(x, Wg, bias, W1, W3, W2, k, capacity_factor, act, y=None, ws=None,
                stats=False, stream=None, gating="topk_softmax", gate_scale=1.0,
                priority="position"):
    """Whole layer.  Returns y, or (y, moe_stats) when stats=True."""
    T, d = x.shape
    E, _, H = W1.shape
    dev = x.device
    need = moe_workspace_bytes(T, d, H, E, k, capacity_factor, x.dtype, act)
    ws = ws if ws is not None else torch.empty(need, dtype=torch.uint8, device=dev)
    y = y if y is not None else torch.empty((T, d), dtype=x.dtype, device=dev)
    st = moe_stats() if stats else None
    opt = _options(gating, gate_scale, priority)
    status = lib().moe_forward_ex(_ptr(x), _ptr(Wg), _ptr(bias), _ptr(W1), _ptr(W3), _ptr(W2),
                                  T, d, H, E, k, _cf(capacity_factor), _act_code(act),
                                  _dtype_code(x), ctypes.byref(opt), _ptr(y), _ptr(ws),
                                  ws.numel(), ctypes.byref(st) if st is not None else None,
                                  _stream(dev, stream))
    _check(status, "moe_forward_ex")
    return (y, st) if stats else y


def moe_forward_host(x_host, Wg, bias, W1, W3, W2, k, capacity_factor, act, y_host=None,
                     x_dev=None, y_dev=None, ws=None, stream=None):
    """The layer on tokens in host memory (pinned for full bandwidth): copy in,
    forward, copy out, all inside the library call."""
    T, d = x_host.shape
    E, _, H = W1.shape
    dev = W1.device
    y_host = y_host if y_host is not None else torch.empty((T, d), dtype=x_host.dtype, pin_memory=True)
    x_dev = x_dev if x_dev is not None else torch.empty((T, d), dtype=x_host.dtype, device=dev)
    y_dev = y_dev if y_dev is not None else torch.empty((T, d), dtype=x_host.dtype, device=dev)
    need = moe_workspace_bytes(T, d, H, E, k, capacity_factor, x_host.dtype, act)
    ws = ws if ws is not None else torch.empty(need, dtype=torch.uint8, device=dev)
    _check(lib().moe_forward_host(_ptr(x_host), _ptr(y_host), _ptr(x_dev), _ptr(y_dev),
                                  _ptr(Wg), _ptr(bias), _ptr(W1), _ptr(W3), _ptr(W2), T, d, H,
                                  E, k, _cf(capacity_factor), _act_code(act),
                                  _dtype_code(x_host), _ptr(ws), ws.numel(),
                                  _stream(dev, stream)), "moe_forward_host")
    return y_host


class Pipeline:
    """Streaming forwards of host-resident batches (moe_pipeline_*): slot i
    owns a device input, output and workspace; submit() enqueues copy-in,
    forward and copy-out and returns at once, wait() blocks until the slot's
    host output is written.  Copies of one batch overlap the forward of
    another."""

    def __init__(self, layer, T, depth=2, stream=None):
        self.layer, self.T, self.depth = layer, T, depth
        dev, d = layer.device, layer.d
        self.stream = stream
        self.x_dev = [torch.empty((T, d), dtype=layer.dtype, device=dev) for _ in range(depth)]
        self.y_dev = [torch.empty((T, d), dtype=layer.dtype, device=dev) for _ in range(depth)]
        need = moe_workspace_bytes(T, d, layer.H, layer.E, layer.k, layer.cf, layer.dtype,
                                   layer.act)
        self.ws = [torch.empty(need, dtype=torch.uint8, device=dev) for _ in range(depth)]
        h = ctypes.c_void_p()
        _check(lib().moe_pipeline_create(depth, ctypes.byref(h)), "moe_pipeline_create")
        self._h = h

    def submit(self, slot, x_host, y_host):
        L = self.layer
        T, d = x_host.shape
        assert T == self.T and d == L.d
        _check(lib().moe_pipeline_submit(
            self._h, slot, _ptr(x_host), _ptr(y_host), _ptr(self.x_dev[slot]),
            _ptr(self.y_dev[slot]), _ptr(L.Wg), _ptr(L.bias), _ptr(L.W1), _ptr(L.W3),
            _ptr(L.W2), T, d, L.H, L.E, L.k, _cf(L.cf), _act_code(L.act), _dtype_code(x_host),
            ctypes.byref(_options(L.gating, L.gate_scale, L.priority)), _ptr(self.ws[slot]),
            self.ws[slot].numel(), _stream(L.device, self.stream)),
            "moe_pipeline_submit")

    def wait(self, slot):
        _check(lib().moe_pipeline_wait(self._h, slot), "moe_pipeline_wait")

    def close(self):
        if self._h:
            _check(lib().moe_pipeline_destroy(self._h), "moe_pipeline_destroy")
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_probe_stream_read(buf, sink, stream=None):
    """Measurement aid: read every byte of the device tensor ``buf`` once
    (a plain streaming read); ``sink`` is a 1-element int32 device tensor."""
    nbytes = buf.numel() * buf.element_size()
    _check(lib().moe_probe_stream_read(_ptr(buf), nbytes, _ptr(sink),
                                       _stream(buf.device, stream)), "moe_probe_stream_read")


def moe_set_stage_events(events):
    """Record ``events`` (six torch.cuda.Event, created with timing enabled)
    between the stages of the next forwards on this thread; None stops."""
    if events is None:
        _check(lib().moe_set_stage_events(None), "moe_set_stage_events")
        return
    arr = (ctypes.c_void_p * MOE_NUM_STAGE_EVENTS)()
    for i, ev in enumerate(events):
        arr[i] = ctypes.c_void_p(ev.cuda_event)
    _check(lib().moe_set_stage_events(arr), "moe_set_stage_events")


def stage_times_ms(events):
    """Per-stage durations (ms) from six recorded events."""
    return {name: events[i].elapsed_time(events[i + 1]) for i, name in enumerate(STAGES)}


class ForwardGraph:
    """One forward of ``layer`` on the tensors x -> y captured as a CUDA graph
    (moe_forward_graph_*): launch() replays it with one host call.  x, y and
    the workspace are held for the graph's lifetime; each launch reads what x
    holds when it runs."""

    def __init__(self, layer, x, y):
        T, d = x.shape
        assert d == layer.d and y.shape == x.shape and y.dtype == x.dtype
        self.x, self.y, self.ws = x, y, layer.workspace(T)
        self.layer = layer
        h = ctypes.c_void_p()
        _check(lib().moe_forward_graph_create(
            _ptr(x), _ptr(layer.Wg), _ptr(layer.bias), _ptr(layer.W1), _ptr(layer.W3),
            _ptr(layer.W2), T, d, layer.H, layer.E, layer.k, _cf(layer.cf), _act_code(layer.act),
            _dtype_code(x), ctypes.byref(_options(layer.gating, layer.gate_scale, layer.priority)),
            _ptr(y), _ptr(self.ws), self.ws.numel(), ctypes.byref(h)), "moe_forward_graph_create")
        self._h = h

    def launch(self, stream=None):
        _check(lib().moe_forward_graph_launch(self._h, _stream(self.x.device, stream)),
               "moe_forward_graph_launch")
        return self.y

    def nodes(self):
        """(kernel nodes, other nodes) of one launch (moe_forward_graph_nodes)."""
        nk, no = ctypes.c_int32(), ctypes.c_int32()
        _check(lib().moe_forward_graph_nodes(self._h, ctypes.byref(nk), ctypes.byref(no)),
               "moe_forward_graph_nodes")
        return nk.value, no.value

    def close(self):
        if self._h:
            _check(lib().moe_forward_graph_destroy(self._h), "moe_forward_graph_destroy")
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class MoELayer:
    """Weights plus a persistent workspace for repeated forwards on one
    device (no allocation per call)."""

    def __init__(self, Wg, bias, W1, W3, W2, k, capacity_factor=0.0, act="swiglu",
                 max_tokens=None, gating="topk_softmax", gate_scale=1.0, priority="position"):
        self.Wg, self.bias, self.W1, self.W3, self.W2 = Wg, bias, W1, W3, W2
        self.k, self.cf, self.act = k, capacity_factor, act
        self.gating, self.gate_scale, self.priority = gating, gate_scale, priority
        self.E, self.d, self.H = W1.shape
        self.dtype = W1.dtype
        self.device = W1.device
        self._ws = None
        self._ws_T = -1
        if max_tokens:
            self.workspace(max_tokens)

    def workspace(self, T):
        if self._ws is None or self._ws_T != T:
            need = moe_workspace_bytes(T, self.d, self.H, self.E, self.k, self.cf, self.dtype,
                                       self.act)
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
            self._ws_T = T
        return self._ws

    def layout(self, T):
        return moe_workspace_layout(T, self.d, self.H, self.E, self.k, self.cf, self.dtype,
                                    self.act)

    def intermediates(self, T):
        return workspace_views(self.workspace(T), self.layout(T), T, self.d, self.H, self.E,
                               self.k, self.dtype)

    def __call__(self, x, y=None, stats=False, stream=None):
        return moe_forward(x, self.Wg, self.bias, self.W1, self.W3, self.W2, self.k, self.cf,
                           self.act, y=y, ws=self.workspace(x.shape[0]), stats=stats,
                           stream=stream, gating=self.gating, gate_scale=self.gate_scale,
                           priority=self.priority)

    def graph(self, x, y=None):
        """A ForwardGraph of this layer on x (and y, allocated if None)."""
        y = y if y is not None else torch.empty_like(x)
        return ForwardGraph(self, x, y)


# ------------------------------------------------ expert-choice routing
def moe_expert_choice_tokens(T, E, k, capacity_factor):
    """Tokens each expert takes: min(T, C); -1 if the capacity factor is not
    a finite positive number."""
    return lib().moe_expert_choice_tokens(T, E, k, _cf(capacity_factor))


def moe_expert_choice_route(x, Wg, bias, scores=None, stream=None):
    """Affinities, expert-major [E, T] fp32: scores[e, t] = softmax over the
    E logits of token t, at expert e."""
    T, d = x.shape
    E = Wg.shape[1]
    dev = x.device
    scores = scores if scores is not None else torch.empty((E, T), dtype=torch.float32, device=dev)
    _check(lib().moe_expert_choice_route(_ptr(x), _ptr(Wg), _ptr(bias), T, d, E, _dtype_code(x),
                                         _ptr(scores), _stream(dev, stream)),
           "moe_expert_choice_route")
    return scores


def moe_expert_choice_select(scores, n, stream=None):
    """Each expert's n tokens from scores [E, T]: tok [E, n], pos [T, E],
    kept_counts, offsets."""
    E, T = scores.shape
    dev = scores.device
    tok = torch.empty((E, max(n, 0)), dtype=torch.int32, device=dev)
    pos = torch.empty((T, E), dtype=torch.int32, device=dev)
    kept_counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    wsb = lib().moe_expert_choice_select_workspace_bytes(T, E)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    _check(lib().moe_expert_choice_select(_ptr(scores), T, E, n, _ptr(tok), _ptr(pos),
                                          _ptr(kept_counts), _ptr(offsets), _ptr(ws), ws.numel(),
                                          _stream(dev, stream)), "moe_expert_choice_select")
    return dict(tok=tok, pos=pos, kept_counts=kept_counts, offsets=offsets)


def moe_expert_choice_permute(x, pos, n, xp=None, stream=None):
    """xp rows from pos [T, E] (moe_expert_choice_select): row pos[t, e] = x[t]."""
    T, d = x.shape
    E = pos.shape[1]
    npad = (n + MOE_ROW_ALIGN - 1) // MOE_ROW_ALIGN * MOE_ROW_ALIGN
    xp = xp if xp is not None else torch.empty((E * npad, d), dtype=x.dtype, device=x.device)
    _check(lib().moe_expert_choice_permute(_ptr(x), _ptr(pos), T, d, E, n, _dtype_code(x),
                                           _ptr(xp), xp.shape[0], _stream(x.device, stream)),
           "moe_expert_choice_permute")
    return xp


def moe_expert_choice_combine(o, pos, scores, dtype, y=None, stream=None):
    if o.dtype != dtype:
        raise TypeError(f"o is {o.dtype}; the combine reads o in the layer dtype {dtype}")
    T, E = pos.shape
    d = o.shape[1]
    y = y if y is not None else torch.empty((T, d), dtype=dtype, device=o.device)
    code = MOE_BF16 if dtype == torch.bfloat16 else MOE_FP32
    _check(lib().moe_expert_choice_combine(_ptr(o), _ptr(pos), _ptr(scores), T, d, E, code,
                                           _ptr(y), _stream(o.device, stream)),
           "moe_expert_choice_combine")
    return y


def moe_expert_choice_layout(T, d, H, E, k, capacity_factor, dtype, act):
    code = MOE_BF16 if dtype in (torch.bfloat16, "bf16") else MOE_FP32
    L = moe_ec_ws_layout()
    _check(lib().moe_expert_choice_layout(T, d, H, E, k, _cf(capacity_factor), code,
                                          _act_code(act), ctypes.byref(L)),
           "moe_expert_choice_layout")
    return L


class ExpertChoiceLayer:
    """An MoE layer with expert-choice routing: every expert takes the
    min(T, ceil(cf*T*k/E)) tokens with the highest softmax affinity to it.
    Holds its workspace; __call__ runs moe_forward_expert_choice."""

    def __init__(self, Wg, bias, W1, W3, W2, k, capacity_factor, act="swiglu"):
        self.Wg, self.bias, self.W1, self.W3, self.W2 = Wg, bias, W1, W3, W2
        self.k, self.cf, self.act = k, capacity_factor, act
        self.E, self.d, self.H = W1.shape
        self.dtype = W1.dtype
        self.device = W1.device
        self._ws = None
        self._ws_T = -1

    def layout(self, T):
        return moe_expert_choice_layout(T, self.d, self.H, self.E, self.k, self.cf, self.dtype,
                                        self.act)

    def workspace(self, T):
        if self._ws_T != T:
            need = self.layout(T).total
            self._ws = torch.empty(max(need, 256), dtype=torch.uint8, device=self.device)
            self._ws_T = T
        return self._ws

    def intermediates(self, T):
        """Views of scores, pos, tok, kept_counts, offsets, dev_error, xp."""
        L = self.layout(T)
        ws = self._ws

        def view(off, count, dt):
            nbytes = count * torch.empty((), dtype=dt).element_size()
            return ws[off:off + nbytes].view(dt)
        return dict(
            scores=view(L.scores, T * self.E, torch.float32).view(self.E, T),
            pos=view(L.pos, T * self.E, torch.int32).view(T, self.E),
            tok=view(L.tok, self.E * L.n, torch.int32).view(self.E, L.n),
            kept_counts=view(L.kept_counts, self.E, torch.int32),
            offsets=view(L.offsets, self.E + 1, torch.int32),
            dev_error=view(L.dev_error, 1, torch.int32),
            xp=view(L.xp, L.rows * self.d, self.dtype).view(L.rows, self.d),
            n=L.n, rows=L.rows)

    def __call__(self, x, y=None, stats=False, stream=None):
        T, d = x.shape
        ws = self.workspace(T)
        y = y if y is not None else torch.empty((T, d), dtype=x.dtype, device=x.device)
        st = moe_stats() if stats else None
        _check(lib().moe_forward_expert_choice(
            _ptr(x), _ptr(self.Wg), _ptr(self.bias), _ptr(self.W1), _ptr(self.W3), _ptr(self.W2),
            T, d, self.H, self.E, self.k, _cf(self.cf), _act_code(self.act), _dtype_code(x),
            _ptr(y), _ptr(ws), ws.numel(), ctypes.byref(st) if st is not None else None,
            _stream(x.device, stream)), "moe_forward_expert_choice")
        return (y, st) if stats else y
