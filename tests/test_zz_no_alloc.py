"""moe_permute_static: the permutation entry point that allocates nothing.

Some callers cannot allocate device memory where they run the layer (a
runtime that reserves all device memory for its own pool up front, a plugin
whose host framework forbids allocation inside its execute call).  For them
moe_permute_static keeps the permutation's scratch in a fixed array inside
the library instead of a caller-provided buffer.  These tests call it through
the C ABI and check that two calls in a row give exactly what moe_permute
(the entry point with caller-provided scratch) gives, and, directly, what the
fp64 oracle's capacity step gives on the same expert indices.  The file is
named to be collected last.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_51_b200 import moe as M
from mixture_experts_layer_51_b200.workloads import Workload, make_inputs

CASES = [
    Workload("dropless", T=1500, d=256, E=8, k=2, H=64, act="swiglu", dtype="bf16", cf=0.0, seed=21),
    Workload("capacity", T=2100, d=136, E=32, k=2, H=64, act="swiglu", dtype="bf16", cf=1.0,
             seed=22, tokens="zipf"),
    Workload("fp32", T=300, d=64, E=4, k=1, H=64, act="gelu", dtype="fp32", cf=1.25, seed=23),
]


def _static_call(x, idx, E, cf):
    """One moe_permute_static call through the C ABI into fresh outputs that
    start filled with garbage (so anything left unwritten shows up)."""
    T, d = x.shape
    k = idx.shape[1]
    dev = x.device
    rows = M.moe_max_permuted_rows(T, E, k, cf)
    out = dict(xp=torch.full((rows, d), 7, dtype=x.dtype, device=dev),
               pos=torch.full((T, k), -7, dtype=torch.int32, device=dev),
               counts=torch.full((E,), -7, dtype=torch.int32, device=dev),
               kept_counts=torch.full((E,), -7, dtype=torch.int32, device=dev),
               offsets=torch.full((E + 1,), -7, dtype=torch.int32, device=dev))
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = M.lib().moe_permute_static(
        p(x), p(idx), T, d, E, k, float(cf), M._dtype_code(x), p(out["xp"]), rows, p(out["pos"]),
        p(out["counts"]), p(out["kept_counts"]), p(out["offsets"]),
        ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    assert st == M.MOE_OK, M.status_string(st)
    return out


def _matches_oracle(got, idx, E, k, cf):
    """Counts, kept counts, 128-row aligned offsets and every position equal
    the oracle's first-C-by-position queue on the same indices."""
    T = idx.shape[0]
    idx_np = idx.cpu().numpy()
    C = oracle.capacity(T, E, k, cf)
    counts, kept_counts, rank, kept = oracle.assign_capacity(idx_np, E, C)
    assert np.array_equal(got["counts"].cpu().numpy(), counts)
    assert np.array_equal(got["kept_counts"].cpu().numpy(), kept_counts)
    align = M.MOE_ROW_ALIGN
    off = np.concatenate([[0], np.cumsum((kept_counts + align - 1) // align * align)])
    assert np.array_equal(got["offsets"].cpu().numpy(), off)
    want_pos = np.where(kept, off[idx_np] + rank, -1)
    assert np.array_equal(got["pos"].cpu().numpy(), want_pos)


def _same(ref, got):
    for key in ("counts", "kept_counts", "offsets", "pos"):
        assert torch.equal(ref[key], got[key]), key
    pos = ref["pos"].reshape(-1).long()
    kept = pos[pos >= 0]
    # The kept rows are exact copies; padding rows are unspecified.
    assert torch.equal(ref["xp"].index_select(0, kept), got["xp"].index_select(0, kept))


@pytest.mark.gpu
@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_static_permute_matches_permute_on_two_calls(w):
    dev = torch.device("cuda")
    inp = make_inputs(w, dev)
    idx, _, _ = M.moe_route(inp["x"], inp["Wg"], inp["bias"], w.k)
    ref = M.moe_permute(inp["x"], idx, w.E, w.cf)
    first = _static_call(inp["x"], idx, w.E, w.cf)
    second = _static_call(inp["x"], idx, w.E, w.cf)
    torch.cuda.synchronize()
    _same(ref, first)
    _same(ref, second)
    _matches_oracle(first, idx, w.E, w.k, w.cf)
    _matches_oracle(second, idx, w.E, w.k, w.cf)
    assert int(ref["kept_counts"].sum()) == int((ref["pos"] >= 0).sum())


@pytest.mark.gpu
def test_static_permute_after_a_larger_call():
    """The shared scratch keeps the previous call's contents; a smaller call
    after a larger one must not see them."""
    dev = torch.device("cuda")
    big, small = CASES[1], CASES[0].replace(T=77, E=32)
    for w in (big, small):
        inp = make_inputs(w, dev)
        idx, _, _ = M.moe_route(inp["x"], inp["Wg"], inp["bias"], w.k)
        ref = M.moe_permute(inp["x"], idx, w.E, w.cf)
        got = _static_call(inp["x"], idx, w.E, w.cf)
        torch.cuda.synchronize()
        _same(ref, got)
        _matches_oracle(got, idx, w.E, w.k, w.cf)


def test_static_permute_rejects_sizes_beyond_its_scratch():
    """ceil(T/256) * E above the fixed scratch is refused before any CUDA
    call (no GPU needed)."""
    E = 64
    T = (M.MOE_PERMUTE_STATIC_MAX_INTS // E) * 256 + 1
    fake = ctypes.c_void_p(0x10000)
    st = M.lib().moe_permute_static(fake, fake, T, 64, E, 2, 0.0, M.MOE_BF16, fake, 1 << 40,
                                    fake, fake, fake, fake, None)
    assert st == M.MOE_ERR_ARG
