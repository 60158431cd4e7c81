"""CPU checks of the C ABI: libmoe.so loads without a GPU, exports every
function include/moe.h declares, and its host-side logic (capacity, buffer
sizes, argument validation) behaves as documented.  No kernel is launched."""

import ctypes
import math
import os
import re

import numpy as np
import pytest
import torch

from mixture_experts_layer_51_b200 import moe as M
from mixture_experts_layer_51_b200.workloads import WORKLOADS
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(M._LIB_PATH):
        from mixture_experts_layer_51_b200 import build
        build.build()
    return M.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(M.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.moe_abi_version() == M.MOE_ABI_VERSION == 2


def test_status_strings(lib):
    for s in range(5):
        assert M.status_string(s).startswith("MOE_")


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_capacity_matches_oracle(lib, name):
    w = WORKLOADS[name]
    c = M.moe_capacity(w.T, w.E, w.k, w.cf)
    o = oracle.capacity(w.T, w.E, w.k, w.cf)
    assert c == (-1 if o is None else o)


def test_capacity_edge_values(lib):
    assert M.moe_capacity(100, 4, 2, 0.0) == -1
    assert M.moe_capacity(100, 4, 2, -2.0) == -1
    assert M.moe_capacity(100, 4, 2, math.inf) == -1
    assert M.moe_capacity(100, 4, 2, math.nan) == -1
    assert M.moe_capacity(10, 4, 1, 1.0) == 3
    assert M.moe_capacity(0, 4, 1, 1.0) == 0


@pytest.mark.parametrize("T,E,k,cf", [(256, 4, 1, 1.25), (4096, 8, 2, 0.0), (16384, 32, 2, 1.0),
                                       (16384, 64, 8, 0.0), (1, 1, 1, 0.0), (33, 7, 3, 0.5),
                                       (1000, 64, 1, 0.0)])
def test_max_permuted_rows_bounds_every_routing(lib, T, E, k, cf):
    """sum_e roundup(kept_e, 128) <= moe_max_permuted_rows for random,
    one-hot-skewed and spread-thin routings (kept counts from the oracle)."""
    import numpy as np
    rng = np.random.default_rng(T * 31 + E)
    rows = M.moe_max_permuted_rows(T, E, k, cf)
    assert rows % 128 == 0
    C = oracle.capacity(T, E, k, cf)
    routings = []
    for _ in range(5):
        routings.append(np.argsort(rng.standard_normal((T, E)), axis=1)[:, :k])
    skew = np.tile(np.arange(k), (T, 1))                 # everyone on experts 0..k-1
    routings.append(skew)
    thin = (np.arange(T)[:, None] * k + np.arange(k)[None, :]) % E   # round robin
    routings.append(thin)
    for idx in routings:
        _, kept_counts, _, _ = oracle.assign_capacity(idx, E, C)
        need = int(sum(-(-int(c) // 128) * 128 for c in kept_counts))
        assert need <= rows


def test_workspace_layout_is_consistent(lib):
    L = M.moe_workspace_layout(8192, 4096, 14336, 8, 2, 0.0, "bf16", "swiglu")
    offs = [L.idx, L.gate, L.margin, L.pos, L.counts, L.kept_counts, L.offsets, L.dev_error,
            L.scratch, L.order, L.prio_scratch, L.xp, L.h, L.o]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert L.rows == M.moe_max_permuted_rows(8192, 8, 2, 0.0)
    # xp, h and o in the layer dtype (bf16: 2 bytes)
    assert L.h - L.xp >= L.rows * 4096 * 2 and L.o - L.h >= L.rows * 14336 * 2
    assert L.total >= L.o + L.rows * 4096 * 2
    assert M.moe_workspace_bytes(8192, 4096, 14336, 8, 2, 0.0, "bf16", "swiglu") == L.total
    F = M.moe_workspace_layout(256, 64, 128, 4, 1, 1.25, "fp32", "gelu")
    assert F.total >= F.o + F.rows * 64 * 4


def test_invalid_arguments_are_rejected_before_any_cuda_call(lib):
    P = ctypes.c_void_p
    fake = P(0x10000)  # never dereferenced: validation fails first
    # k > E
    assert lib.moe_route(fake, fake, None, 16, 64, 2, 3, M.MOE_BF16, fake, fake, None, None) == M.MOE_ERR_ARG
    # E > 64
    assert lib.moe_route(fake, fake, None, 16, 64, 65, 2, M.MOE_BF16, fake, fake, None, None) == M.MOE_ERR_ARG
    # d % 8 != 0
    assert lib.moe_route(fake, fake, None, 16, 60, 8, 2, M.MOE_BF16, fake, fake, None, None) == M.MOE_ERR_ARG
    # null output
    assert lib.moe_route(fake, fake, None, 16, 64, 8, 2, M.MOE_BF16, None, fake, None, None) == M.MOE_ERR_ARG
    # misaligned x
    assert lib.moe_route(P(0x10004), fake, None, 16, 64, 8, 2, M.MOE_BF16, fake, fake, None, None) == M.MOE_ERR_ARG
    # bad dtype enum
    assert lib.moe_route(fake, fake, None, 16, 64, 8, 2, 7, fake, fake, None, None) == M.MOE_ERR_ARG
    # permute buffer too small
    assert lib.moe_permute(fake, fake, 64, 64, 8, 2, 0.0, M.MOE_BF16, fake, 128, fake, fake, fake,
                           fake, fake, 1 << 20, None) == M.MOE_ERR_ARG
    # grouped FFN: rows not a multiple of 128, missing W3 for SwiGLU
    assert lib.moe_grouped_ffn(fake, 100, fake, fake, fake, fake, fake, 8, 64, 64, M.MOE_SWIGLU,
                               M.MOE_BF16, fake, fake, fake, None) == M.MOE_ERR_ARG
    assert lib.moe_grouped_ffn(fake, 128, fake, fake, fake, None, fake, 8, 64, 64, M.MOE_SWIGLU,
                               M.MOE_BF16, fake, fake, fake, None) == M.MOE_ERR_ARG
    # forward: workspace too small
    st = lib.moe_forward(fake, fake, None, fake, fake, fake, 64, 64, 64, 8, 2, 0.0, M.MOE_SWIGLU,
                         M.MOE_BF16, fake, fake, 16, None, None)
    assert st == M.MOE_ERR_ARG
    # forward: a missing or misaligned weight or output is refused before
    # anything is enqueued (a workspace large enough, so only that differs)
    big = 1 << 40
    odd = P(0x10008)
    for args in [(fake, fake, None, odd, fake, fake),     # W1 misaligned
                 (fake, fake, None, fake, None, fake),    # SwiGLU without W3
                 (fake, fake, None, fake, fake, odd),     # W2 misaligned
                 (odd, fake, None, fake, fake, fake),     # x misaligned
                 (fake, None, None, fake, fake, fake)]:   # no router weights
        st = lib.moe_forward(*args, 64, 64, 64, 8, 2, 0.0, M.MOE_SWIGLU, M.MOE_BF16, fake, fake,
                             big, None, None)
        assert st == M.MOE_ERR_ARG, args
    st = lib.moe_forward(fake, fake, None, fake, fake, fake, 64, 64, 64, 8, 2, 0.0, M.MOE_SWIGLU,
                         M.MOE_BF16, odd, fake, big, None, None)  # y misaligned
    assert st == M.MOE_ERR_ARG
    # GELU ignores W3, aligned or not: the call gets past the checks (to the
    # first CUDA call, which fails here without a GPU)
    st = lib.moe_forward(fake, fake, None, fake, odd, fake, 64, 64, 64, 8, 2, 0.0, M.MOE_GELU,
                         M.MOE_BF16, fake, fake, big, None, None)
    assert st != M.MOE_ERR_ARG


def test_empty_batch_is_a_no_op(lib):
    # T == 0 does nothing and touches no device state.
    st = M.moe_stats()
    assert lib.moe_forward(None, None, None, None, None, None, 0, 64, 64, 8, 2, 1.0,
                           M.MOE_SWIGLU, M.MOE_BF16, None, None, 0, ctypes.byref(st), None) == M.MOE_OK
    assert st.capacity == 0 and st.kept == 0
    assert lib.moe_route(None, None, None, 0, 64, 8, 2, M.MOE_BF16, None, None, None, None) == M.MOE_OK


def test_invalid_options_are_rejected(lib):
    fake = ctypes.c_void_p(0x10000)
    for opt in (M.moe_options(gating=7, gate_scale=1.0), M.moe_options(gating=0, gate_scale=0.0),
                M.moe_options(gating=1, gate_scale=-2.0),
                M.moe_options(gating=0, gate_scale=float("inf"))):
        assert lib.moe_route_ex(fake, fake, None, 16, 64, 8, 2, M.MOE_BF16, ctypes.byref(opt),
                                fake, fake, None, None) == M.MOE_ERR_ARG
    pr = M.moe_options(gating=0, gate_scale=1.0, priority=5)
    assert lib.moe_route_ex(fake, fake, None, 16, 64, 8, 2, M.MOE_BF16, ctypes.byref(pr),
                            fake, fake, None, None) == M.MOE_ERR_ARG
    bad = M.moe_options(gating=0, gate_scale=1.0)
    bad.reserved[3] = 1
    assert lib.moe_route_ex(fake, fake, None, 16, 64, 8, 2, M.MOE_BF16, ctypes.byref(bad),
                            fake, fake, None, None) == M.MOE_ERR_ARG


@pytest.mark.parametrize("T,E,k,cf,bounds", [(1000, 8, 2, 1.0, (0, 400, 1000)),
                                              (600, 32, 2, 1.0, (0, 1, 300, 600)),
                                              (513, 64, 8, 0.5, (0, 100, 513))])
def test_rows_for_capacity_bounds_every_shard(lib, T, E, k, cf, bounds):
    """A shard under the whole batch's capacity never needs more rows than
    moe_rows_for_capacity(shard T, E, k, C) (kept counts from the oracle's
    shard rule, on a skewed routing)."""
    import numpy as np
    C = M.moe_capacity(T, E, k, cf)
    assert M.moe_rows_for_capacity(T, E, k, C) == M.moe_max_permuted_rows(T, E, k, cf)
    idx = np.tile(np.arange(k), (T, 1))
    idx[::3] = (idx[::3] + 1) % E
    prior = np.zeros(E, dtype=np.int64)
    for a, b in zip(bounds[:-1], bounds[1:]):
        _, kc, _, _ = oracle.assign_capacity_shard(idx[a:b], E, C, prior)
        need = int(sum(-(-int(c) // 128) * 128 for c in kc))
        assert need <= M.moe_rows_for_capacity(b - a, E, k, C)
        prior = prior + np.bincount(idx[a:b].reshape(-1), minlength=E)


def test_shard_entry_points_validate_arguments(lib):
    fake = ctypes.c_void_p(0x10000)
    assert lib.moe_expert_counts(fake, 16, 65, 2, fake, None) == M.MOE_ERR_ARG   # E > 64
    assert lib.moe_expert_counts(fake, 16, 8, 9, fake, None) == M.MOE_ERR_ARG    # k > E
    assert lib.moe_expert_counts(None, 16, 8, 2, fake, None) == M.MOE_ERR_ARG    # no idx
    assert lib.moe_rank_prefix(fake, 2, 8, 2, fake, None) == M.MOE_ERR_ARG       # rank >= n
    assert lib.moe_rank_prefix(fake, 0, 8, 0, fake, None) == M.MOE_ERR_ARG       # no ranks
    assert lib.moe_rank_prefix(None, 2, 8, 0, fake, None) == M.MOE_ERR_ARG
    # xp smaller than the shard's bound under the given capacity
    rows = M.moe_rows_for_capacity(64, 8, 2, 10)
    assert lib.moe_permute_ex(fake, fake, None, fake, 64, 64, 8, 2, 10, M.MOE_BF16, fake,
                              rows - 128, fake, fake, fake, fake, fake, 1 << 20,
                              None) == M.MOE_ERR_ARG


def test_expert_choice_sizes_and_validation(lib):
    import math
    assert M.moe_expert_choice_tokens(16384, 64, 8, 1.0) == 2048
    assert M.moe_expert_choice_tokens(100, 4, 2, 8.0) == 100        # capped at T
    assert M.moe_expert_choice_tokens(100, 4, 2, 0.0) == -1         # no dropless form
    assert M.moe_expert_choice_tokens(100, 4, 2, math.inf) == -1
    assert M.moe_expert_choice_tokens(100, 4, 5, 1.0) == -1         # k > E
    L = M.moe_expert_choice_layout(700, 256, 384, 64, 8, 1.0, "bf16", "swiglu")
    assert L.n == 88 and L.rows == 64 * 128
    offs = [L.scores, L.pos, L.tok, L.kept_counts, L.offsets, L.dev_error, L.scratch, L.xp, L.h,
            L.o]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert L.total >= L.o + L.rows * 256 * 2  # o in the layer dtype (bf16)
    assert lib.moe_expert_choice_workspace_bytes(700, 256, 384, 64, 8, 1.0, M.MOE_BF16,
                                                 M.MOE_SWIGLU) == L.total
    assert lib.moe_expert_choice_workspace_bytes(700, 256, 384, 64, 8, 0.0, M.MOE_BF16,
                                                 M.MOE_SWIGLU) == 0
    fake = ctypes.c_void_p(0x10000)
    # n > T, E > 64, misaligned x, xp too small, workspace too small
    assert lib.moe_expert_choice_select(fake, 10, 4, 11, fake, fake, fake, fake, fake, 1 << 20,
                                        None) == M.MOE_ERR_ARG
    assert lib.moe_expert_choice_route(fake, fake, None, 10, 64, 65, M.MOE_BF16, fake,
                                       None) == M.MOE_ERR_ARG
    assert lib.moe_expert_choice_permute(ctypes.c_void_p(0x10004), fake, 10, 64, 4, 3,
                                         M.MOE_BF16, fake, 512, None) == M.MOE_ERR_ARG
    assert lib.moe_expert_choice_permute(fake, fake, 10, 64, 4, 3, M.MOE_BF16, fake, 384,
                                         None) == M.MOE_ERR_ARG
    assert lib.moe_forward_expert_choice(fake, fake, None, fake, fake, fake, 64, 64, 64, 8, 2,
                                         1.0, M.MOE_SWIGLU, M.MOE_BF16, fake, fake, 16, None,
                                         None) == M.MOE_ERR_ARG


def test_pipeline_arguments_are_checked_before_any_cuda_call(lib):
    h = ctypes.c_void_p()
    assert lib.moe_pipeline_create(0, ctypes.byref(h)) == M.MOE_ERR_ARG
    assert lib.moe_pipeline_create(M.MOE_PIPELINE_MAX_DEPTH + 1, ctypes.byref(h)) == M.MOE_ERR_ARG
    assert lib.moe_pipeline_create(2, None) == M.MOE_ERR_ARG
    fake = ctypes.c_void_p(0x10000)
    assert lib.moe_pipeline_submit(None, 0, fake, fake, fake, fake, fake, None, fake, fake, fake,
                                   64, 64, 64, 8, 2, 0.0, M.MOE_SWIGLU, M.MOE_BF16, None, fake,
                                   1 << 20, None) == M.MOE_ERR_ARG
    assert lib.moe_pipeline_wait(None, 0) == M.MOE_ERR_ARG
    assert lib.moe_pipeline_destroy(None) == M.MOE_OK


def test_sizes_past_int32_rows_are_rejected(lib):
    """Rows, offsets and positions are int32 on the device: a layout whose
    permuted buffer would pass 2^31 rows is refused (workspace size 0)."""
    assert M.moe_workspace_bytes(300_000_000, 64, 64, 64, 8, 0.0, "bf16", "swiglu") == 0
    assert M.moe_workspace_bytes(1_000_000, 64, 64, 64, 8, 0.0, "bf16", "swiglu") > 0
    assert lib.moe_expert_choice_workspace_bytes(40_000_000, 64, 64, 64, 8, 1.0, M.MOE_BF16,
                                                 M.MOE_SWIGLU) == 0


def test_zipf_token_ids_are_reproducible_and_follow_the_law():
    """The skewed workload's token ids: the same seed gives the same ids, and
    the frequencies of the most common ids follow P(r) ~ r^-1.1 (within five
    standard errors of a 200000-draw sample)."""
    from mixture_experts_layer_51_b200.workloads import ZIPF_S, ZIPF_VOCAB, _zipf_ids
    n = 200000
    a = _zipf_ids(torch.Generator().manual_seed(3), n, "cpu").numpy()
    b = _zipf_ids(torch.Generator().manual_seed(3), n, "cpu").numpy()
    assert np.array_equal(a, b)
    assert a.min() >= 0 and a.max() < ZIPF_VOCAB
    r = np.arange(1, ZIPF_VOCAB + 1, dtype=np.float64)
    p = r ** -ZIPF_S
    p /= p.sum()
    freq = np.bincount(a, minlength=ZIPF_VOCAB) / n
    top = slice(0, 20)
    se = np.sqrt(p[top] * (1 - p[top]) / n)
    assert np.all(np.abs(freq[top] - p[top]) <= 5 * se)


def test_combines_require_o_in_the_layer_dtype():
    """o is stored in the layer dtype; handing the combines an fp32 o for a
    bf16 layer is refused before any library call."""
    o = torch.zeros(128, 64, dtype=torch.float32)
    pos = torch.zeros(4, 2, dtype=torch.int32)
    with pytest.raises(TypeError):
        M.moe_unpermute_combine(o, pos, torch.zeros(4, 2), torch.bfloat16)
    with pytest.raises(TypeError):
        M.moe_expert_choice_combine(o, pos, torch.zeros(2, 4), torch.bfloat16)


def test_graph_arguments_are_checked_before_any_cuda_call(lib):
    fake = ctypes.c_void_p(256)
    out = ctypes.c_void_p()
    args = [fake] * 6 + [64, 64, 128, 4, 2, 0.0, M.MOE_SWIGLU, M.MOE_BF16, None, fake, fake,
                         1 << 30]
    assert lib.moe_forward_graph_create(*args, None) == M.MOE_ERR_ARG          # no out
    bad_T = list(args)
    bad_T[6] = 0
    assert lib.moe_forward_graph_create(*bad_T, ctypes.byref(out)) == M.MOE_ERR_ARG
    small_ws = list(args)
    small_ws[-1] = 16
    assert lib.moe_forward_graph_create(*small_ws, ctypes.byref(out)) == M.MOE_ERR_ARG
    no_w3 = list(args)
    no_w3[4] = None
    assert lib.moe_forward_graph_create(*no_w3, ctypes.byref(out)) == M.MOE_ERR_ARG
    assert not out.value
    assert lib.moe_forward_graph_launch(None, None) == M.MOE_ERR_ARG
    assert lib.moe_forward_graph_destroy(None) == M.MOE_OK
    nk, no = ctypes.c_int32(-1), ctypes.c_int32(-1)
    assert lib.moe_forward_graph_nodes(None, ctypes.byref(nk), ctypes.byref(no)) == M.MOE_ERR_ARG
    assert nk.value == -1 and no.value == -1
