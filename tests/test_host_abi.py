"""Host-only checks of the C-ABI library: it loads, exports every entry point
that include/cce.h declares, and rejects bad arguments synchronously before
touching the GPU (no compute call is made here)."""

import ctypes
import os
import re

import pytest

from lm_head_cross_flash_b200 import build, cce

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return cce.lib()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names += re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", txt, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "defined")))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "cce_forward" in names and "cce_backward_dh" in names
    assert "orpo_loss_from_logps" in names and "orpo_grad_coeffs" in names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code, name in cce.STATUS_NAMES.items():
        assert lib.cce_status_string(code).decode() == name


def test_blockmax_cols(lib):
    assert lib.cce_blockmax_cols(1) == 1
    assert lib.cce_blockmax_cols(256) == 1
    assert lib.cce_blockmax_cols(257) == 2
    assert lib.cce_blockmax_cols(262144) == 1024
    assert lib.cce_blockmax_cols(73440) == 287
    assert lib.cce_blockmax_cols(0) == 0


def _head(V=1000, D=128, dtype=cce.CCE_BF16, w=4096, fmt=cce.CCE_W_DENSE):
    return cce._Head(fmt, dtype, V, D, w, None, None)


def test_workspace_sizes_monotonic(lib):
    h = _head()
    sz = [lib.cce_workspace_bytes(M, cce.CCE_BF16, ctypes.byref(h)) for M in (1, 100, 1000, 5000)]
    assert all(a <= b for a, b in zip(sz, sz[1:])) and sz[0] > 0
    lo = lib.cce_workspace_min_bytes(1000, cce.CCE_BF16, ctypes.byref(h))
    assert 0 < lo <= sz[2]
    big = _head(V=262144, D=2048)
    # default workspace at the long pair: a 1 GiB G'' chunk and the K-split buffer,
    # far below the 8.6 GB of fp32 logits it replaces
    assert lib.cce_workspace_bytes(8192, cce.CCE_BF16, ctypes.byref(big)) < 1280 << 20
    assert lib.cce_workspace_bytes(0, cce.CCE_BF16, ctypes.byref(h)) == 0
    bad = _head(D=96)
    assert lib.cce_workspace_bytes(10, cce.CCE_BF16, ctypes.byref(bad)) == 0


def test_forward_rejects_bad_arguments_before_launch(lib):
    h = _head()
    hp = ctypes.byref(h)
    P = ctypes.c_void_p
    a = P(4096)
    # null pointers
    assert lib.cce_forward(None, 1, 10, hp, a, a, a, None, None, a, 1 << 20, None) == 1
    assert lib.cce_forward(a, 1, 10, hp, None, a, a, None, None, a, 1 << 20, None) == 1
    # M <= 0, bad dtype, misaligned
    assert lib.cce_forward(a, 1, 0, hp, a, a, a, None, None, a, 1 << 20, None) == 1
    assert lib.cce_forward(a, 7, 10, hp, a, a, a, None, None, a, 1 << 20, None) == 1
    assert lib.cce_forward(P(4097), 1, 10, hp, a, a, a, None, None, a, 1 << 20, None) == 1
    # D not a multiple of 64, mixed dtypes, Q4 with f32 rows
    assert lib.cce_forward(a, 1, 10, ctypes.byref(_head(D=96)), a, a, a, None, None, a, 1 << 20, None) == 2
    assert lib.cce_forward(a, 0, 10, hp, a, a, a, None, None, a, 1 << 20, None) == 2
    # workspace too small
    assert lib.cce_forward(a, 1, 10, hp, a, a, a, None, None, a, 1024, None) == 4


def test_backward_rejects_bad_arguments_before_launch(lib):
    h = _head()
    hp = ctypes.byref(h)
    P = ctypes.c_void_p
    a = P(4096)
    f = ctypes.c_float
    assert lib.cce_backward_dh(a, 1, 10, hp, a, a, None, f(0), None, a, None, a, 1 << 24, None) == 1
    assert lib.cce_backward_dh(a, 1, 10, hp, a, a, a, f(-1.0), None, a, None, a, 1 << 24, None) == 1
    assert lib.cce_backward_dh(a, 1, 10, hp, a, a, a, f(float("nan")), None, a, None, a, 1 << 24, None) == 1
    assert lib.cce_backward_dh(a, 1, 10, hp, a, a, a, f(0), None, P(4100), None, a, 1 << 24, None) == 1
    assert lib.cce_backward_dh(a, 1, 10, hp, a, a, a, f(0), None, a, None, a, 4096, None) == 4


def test_orpo_rejects_bad_layouts(lib):
    P = ctypes.c_void_p
    a = P(4096)
    ws_ok = 1 << 12

    def L(*v):
        return ctypes.byref(cce._Layout(*v))

    bad = [
        (0, 10, 5, 15, 15, 20),    # overlap prompt / chosen
        (0, 5, 5, 5, 5, 20),       # empty chosen
        (0, 5, 5, 10, 10, 10),     # empty rejected
        (0, 5, 5, 10, 10, 21),     # beyond M
        (-1, 5, 5, 10, 10, 20),    # negative
        (0, 5, 10, 5, 10, 20),     # end < begin
    ]
    for lay in bad:
        assert lib.orpo_loss_from_logps(a, a, 20, L(*lay), 0.1, 0, a, a, ws_ok, None) == 1
        assert lib.orpo_grad_coeffs(a, a, 20, L(*lay), 0.1, 0, a, a, ws_ok, None) == 1
    good = L(0, 5, 5, 10, 10, 20)
    assert lib.orpo_loss_from_logps(a, a, 20, good, -0.1, 0, a, a, ws_ok, None) == 1
    assert lib.orpo_loss_from_logps(a, a, 20, good, float("nan"), 0, a, a, ws_ok, None) == 1
    assert lib.orpo_loss_from_logps(a, a, 20, good, 0.1, 2, a, a, ws_ok, None) == 1
    assert lib.orpo_loss_from_logps(a, a, 20, good, 0.1, 0, None, a, ws_ok, None) == 1
    assert lib.orpo_loss_from_logps(a, a, 20, good, 0.1, 0, a, a, 16, None) == 4


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(cce, "_lib", None)
    monkeypatch.setattr(cce, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        cce.lib()


def test_objective_rejects_bad_arguments(lib):
    P = ctypes.c_void_p
    a = P(4096)
    lay = ctypes.byref(cce._Layout(0, 5, 5, 10, 10, 20))
    for obj in [cce._Objective(3, 0.1, 1.0, 0.0, 0), cce._Objective(1, 0.1, -1.0, 0.0, 0),
                cce._Objective(1, 0.1, 1.0, float("inf"), 0), cce._Objective(2, -0.1, 1.0, 0.0, 0),
                cce._Objective(1, 0.1, 1.0, 0.0, 5)]:
        assert lib.pref_loss_from_logps(a, a, 20, lay, ctypes.byref(obj), a, a, 4096, None) == 1
        assert lib.pref_grad_coeffs(a, a, 20, lay, ctypes.byref(obj), a, a, 4096, None) == 1
    assert lib.pref_loss_from_logps(a, a, 20, lay, None, a, a, 4096, None) == 1


def test_query_plan_chunks_splits_and_staging(lib):
    """The host-side planner: forward/backward chunking, the dH K split,
    CTA pairs and staged dequantisation follow the workspace and M."""
    big = _head(V=262144, D=2048)
    ws = lib.cce_workspace_bytes(8192, cce.CCE_BF16, ctypes.byref(big))
    p = cce.cce_query_plan(8192, cce.CCE_BF16, big, ws)
    assert p["fwd_ok"] and p["bwd_ok"] and not p["fwd_staged"] and not p["bwd_staged"]
    assert p["fwd_chunk"] == 262144          # one forward launch over V
    assert 256 <= p["bwd_chunk"] < 262144 and p["bwd_chunk"] % 256 == 0
    assert 1 <= p["bwd_ksplit"] <= 4 and p["fwd_cta_pairs"] and p["bwd_cta_pairs"]
    # a wider workspace gives wider backward chunks
    p2 = cce.cce_query_plan(8192, cce.CCE_BF16, big, 4 * ws)
    assert p2["bwd_chunk"] > p["bwd_chunk"]
    # the minimum workspace (sized for a 256-wide chunk and no K split; the
    # forward's statistics may leave the backward room for a wider chunk)
    lo = lib.cce_workspace_min_bytes(8192, cce.CCE_BF16, ctypes.byref(big))
    p3 = cce.cce_query_plan(8192, cce.CCE_BF16, big, lo)
    assert p3["fwd_ok"] and p3["bwd_ok"] and p3["bwd_chunk"] >= 256 and p3["bwd_ksplit"] == 1
    p4 = cce.cce_query_plan(8192, cce.CCE_BF16, big, lo - 1)
    assert not p4["fwd_ok"] and not p4["bwd_ok"]
    # small M: few dH tiles, so the K split goes past 4 to fill the grid;
    # M <= 128 runs single-CTA tiles
    small = cce.cce_query_plan(64, cce.CCE_BF16, big,
                               lib.cce_workspace_bytes(64, cce.CCE_BF16, ctypes.byref(big)))
    assert small["bwd_ksplit"] > 4 and not small["bwd_cta_pairs"]


def test_query_plan_quant_staging(lib):
    q4 = cce._Head(cce.CCE_W_AFFINE_Q4_G64, cce.CCE_BF16, 128256, 4096, 4096, 4096, 4096)
    try:
        for mode, M, fwd, bwd in [(0, 32768, 1, 1), (0, 512, 1, 1), (0, 256, 0, 1),
                                  (0, 128, 0, 0), (1, 32768, 0, 0), (2, 128, 1, 1)]:
            cce.cce_set_quant_staging(mode)
            ws = lib.cce_workspace_bytes(M, cce.CCE_BF16, ctypes.byref(q4))
            p = cce.cce_query_plan(M, cce.CCE_BF16, q4, ws)
            assert p["fwd_staged"] == fwd and p["bwd_staged"] == bwd, (mode, M, p)
            # in-kernel dequantisation is single-CTA; so is M <= 128
            assert p["bwd_cta_pairs"] == (bwd and M > 128)
            # the minimum workspace always runs (staging falls back to in-kernel)
            lo = lib.cce_workspace_min_bytes(M, cce.CCE_BF16, ctypes.byref(q4))
            pl = cce.cce_query_plan(M, cce.CCE_BF16, q4, lo)
            assert pl["fwd_ok"] and pl["bwd_ok"] and not pl["bwd_staged"]
    finally:
        cce.cce_set_quant_staging(0)


def test_oversized_tile_counts_are_rejected(lib):
    """Shapes whose tile count would overflow the kernels' 32-bit tile ids
    are refused before anything is launched."""
    big = _head(V=1 << 30, D=2048)
    f = ctypes.c_void_p(4096)
    M = 1 << 30
    st = lib.cce_forward(f, cce.CCE_BF16, M, ctypes.byref(big), f, f, f, None, None, f,
                         1 << 40, None)
    assert cce.STATUS_NAMES[st] == "CCE_ERR_UNSUPPORTED"
    out = cce._Plan()
    assert lib.cce_query_plan(M, cce.CCE_BF16, ctypes.byref(big), 1 << 40,
                              ctypes.byref(out)) == 2
    # the same head at a modest M is accepted by the planner
    assert lib.cce_query_plan(8192, cce.CCE_BF16, ctypes.byref(big), 1 << 40,
                              ctypes.byref(out)) == 0


from hypothesis import given, settings, strategies as st


@settings(max_examples=200, deadline=None)
@given(M=st.integers(1, 70000), V=st.integers(1, 300000), D64=st.integers(1, 96),
       fmt=st.sampled_from([cce.CCE_W_DENSE, cce.CCE_W_AFFINE_Q4_G64, cce.CCE_W_AFFINE_Q8_G64]),
       frac=st.floats(0.0, 2.0))
def test_planner_invariants(lib, M, V, D64, fmt, frac):
    """For any shape and any workspace between the minimum and twice the
    default, the planner's choices are consistent: both calls fit, chunks are
    whole vocab tiles, K splits stay in range, staging and CTA pairs follow
    their documented thresholds."""
    D = 64 * D64
    h = cce._Head(fmt, cce.CCE_BF16, V, D, 4096, 4096 if fmt else None, 4096 if fmt else None)
    lo = lib.cce_workspace_min_bytes(M, cce.CCE_BF16, ctypes.byref(h))
    hi = lib.cce_workspace_bytes(M, cce.CCE_BF16, ctypes.byref(h))
    assert 0 < lo <= hi
    ws = int(lo + frac * (2 * hi - lo) / 2)
    p = cce.cce_query_plan(M, cce.CCE_BF16, h, ws)
    vmax = -(-V // 256) * 256
    n_rt = -(-M // 128)
    assert p["fwd_ok"] and p["bwd_ok"]
    assert p["bwd_chunk"] % 256 == 0 and 256 <= p["bwd_chunk"] <= vmax
    assert p["fwd_chunk"] % 256 == 0 and 256 <= p["fwd_chunk"] <= vmax
    assert 1 <= p["bwd_ksplit"] <= 32
    if fmt == cce.CCE_W_DENSE:
        assert not p["fwd_staged"] and not p["bwd_staged"]
        assert p["fwd_chunk"] == vmax  # one forward launch over the vocabulary
    else:
        assert not p["fwd_staged"] or n_rt >= 3
        assert not p["bwd_staged"] or n_rt >= 2
        if not p["fwd_staged"]:
            assert p["fwd_chunk"] == vmax
    if p["fwd_cta_pairs"] or p["bwd_cta_pairs"]:
        assert M > 128
    if fmt != cce.CCE_W_DENSE and not p["bwd_staged"]:
        assert not p["bwd_cta_pairs"]  # in-kernel dequantisation is single-CTA
    # the default workspace never needs a narrower chunk than the minimum one
    pd = cce.cce_query_plan(M, cce.CCE_BF16, h, hi)
    assert pd["bwd_chunk"] >= cce.cce_query_plan(M, cce.CCE_BF16, h, lo)["bwd_chunk"]
