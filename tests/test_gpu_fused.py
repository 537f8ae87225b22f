"""GPU parity of the fused backward (one kernel: recompute each vocab tile,
form the coefficient tile from the TMEM accumulator, contract it with W into
a dH accumulator held in TMEM) against the float64 oracle and against the
two-GEMM backward.

Shapes cover single CTAs (at most 128 rows) and CTA pairs; D from 64 to
2048, with a last 256-column slice that is partly past D (D = 320); groups
of 1 to 8 members; vocabularies from 1 to 20,000 with ragged tails; and row
counts that leave a remainder of row tiles shared between groups (several
partial dH buffers summed in a fixed order).  The filter and block skip,
the softcap, rows without a cotangent, and determinism (two calls give the
same bits) are checked as well."""

import numpy as np
import pytest
import torch

from lm_head_cross_flash_b200 import cce
from lm_head_cross_flash_b200 import synthetic as S
from oracle import flash_cce as O

from helpers import TOL_DH, oracle_W, rel_fro, upload

pytestmark = pytest.mark.gpu


def _fwd(wl, ws_bytes=None):
    """Forward, with a workspace sized for the fused backward at any M (the
    default setting takes the fused kernel from 1,024 rows only)."""
    H, head, labels = upload(wl)
    hd = cce.h_dtype(H)
    cce.cce_set_backward_mode(1)
    try:
        ws = cce.alloc_workspace(wl.M, hd, head, nbytes=ws_bytes)
    finally:
        cce.cce_set_backward_mode(0)
    f = dict(device="cuda", dtype=torch.float32)
    logp, lse = torch.empty(wl.M, **f), torch.empty(wl.M, **f)
    bm = torch.empty(cce.blockmax_cols(wl.V), wl.M, **f)
    cce.cce_forward(H, head, labels, logp, lse, None, bm, ws)
    torch.cuda.synchronize()
    assert cce.cce_device_status(ws) == 0
    return H, head, labels, ws, lse, bm


def _bwd(mode, H, head, labels, ws, lse, coeff, eps=0.0, bm=None, stats=None):
    dH = torch.full((H.shape[0], head.D), float("nan"), device="cuda")
    cce.cce_set_backward_mode(mode)
    try:
        cce.cce_backward_dh(H, head, labels, lse, coeff, eps, bm, dH, stats, ws)
        torch.cuda.synchronize()
    finally:
        cce.cce_set_backward_mode(0)
    assert cce.cce_device_status(ws) == 0
    return dH


CASES = [
    # (recipe, (P, Rc, Rr), D, V): single CTAs (M <= 128)
    (1, (1, 1, 1), 64, 31),
    (1, (3, 2, 2), 64, 1),
    (2, (8, 28, 28), 256, 5000),
    (2, (20, 50, 58), 2048, 20000),
    (1, (40, 44, 44), 320, 257),
    # CTA pairs
    (2, (100, 150, 131), 256, 4097),
    (1, (64, 200, 300), 320, 1000),
    (1, (300, 400, 500), 512, 3000),
    (2, (500, 1500, 2000), 1536, 7000),
    (2, (1000, 2000, 2000), 2048, 3000),
]


@pytest.mark.parametrize("cfg,split,D,V", CASES)
def test_fused_backward_matches_oracle_and_two_gemm(cfg, split, D, V):
    wl = S.make_custom(cfg, M_split=split, D=D, V=V)
    H, head, labels, ws, lse, _ = _fwd(wl)
    cce.cce_set_backward_mode(1)
    try:
        plan = cce.cce_query_plan(wl.M, cce.h_dtype(H), head, ws.numel())
    finally:
        cce.cce_set_backward_mode(0)
    assert plan["bwd_fused"], plan
    g = S.random_cotangent(wl)
    g[min(5, wl.M - 1):min(9, wl.M)] = 0.0
    coeff = torch.from_numpy(g).cuda()
    d_fused = _bwd(1, H, head, labels, ws, lse, coeff)
    d_again = _bwd(1, H, head, labels, ws, lse, coeff)
    assert torch.equal(d_fused, d_again)            # deterministic
    d_two = _bwd(2, H, head, labels, ws, lse, coeff)
    got = d_fused.cpu().numpy()
    W = oracle_W(wl)
    want = O.head_dh(wl.H, W, wl.labels, g, O.head_forward(wl.H, W, wl.labels)[1])
    err = rel_fro(got, want)
    print(f"M={wl.M} D={D} V={V}: groups {plan['bwd_fused_groups']} x "
          f"{plan['bwd_fused_members']}, buffers {plan['bwd_fused_buffers']}, "
          f"pairs {plan['bwd_cta_pairs']}: rel err {err:.2e}")
    assert err <= TOL_DH
    assert rel_fro(got, d_two.cpu().numpy()) <= 1e-5
    assert np.all(got[wl.labels < 0] == 0.0)
    assert np.all(got[min(5, wl.M - 1):min(9, wl.M)] == 0.0)


def test_fused_remainder_uses_several_buffers():
    """Twenty 256-row tiles over nine groups of eight pairs: two waves and a
    remainder of two row tiles (ten rounds each at V = 20,000) cut between
    all nine groups, so each of those row tiles gathers several partial dH
    slices."""
    wl = S.make_custom(2, M_split=(1000, 2000, 2000), D=2048, V=20000)
    H, head, labels = upload(wl)
    plan = cce.cce_query_plan(wl.M, cce.h_dtype(H), head,
                              cce.workspace_bytes(wl.M, cce.h_dtype(H), head))
    assert plan["bwd_fused"] and plan["bwd_fused_buffers"] >= 3, plan


@pytest.mark.parametrize("pairs", [True, False])
def test_fused_filter_block_skip_is_exact(pairs):
    """Strongly peaked rows (alpha = 22: the target holds all but about 7e-5
    of the mass, and a 256-wide vocab block rarely holds a probability above
    1e-6), so block skip removes about half of the tiles.  Skipping must give
    the same bits as the filter alone; both match the oracle with the same
    filter (at this peak nearly every non-target probability is below eps,
    so the filter itself changes dH by O(1): the unfiltered comparison
    belongs to the moderately peaked long-pair workload) and the two-GEMM
    backward with the same filter.  Rows of the response-scope prompt (zero
    cotangent) skip whole row tiles.  (Sharper peaks leave 1 - p_y below
    the fp32 resolution at 1, so the target coefficient p_y - 1 itself is
    known only to about 6e-8 absolute.)"""
    wl = S.make_custom(1, M_split=(260, 300, 340), D=256, V=60000, alpha=22.0)
    cce.cce_set_cta_pairs(pairs)
    try:
        H, head, labels, ws, lse, bm = _fwd(wl)
        W = oracle_W(wl)
        _, olse, _ = O.head_forward(wl.H, W, wl.labels)
        g = O.orpo_grad_coeffs(O.head_forward(wl.H, W, wl.labels)[0], wl.labels,
                               O.Layout(*wl.layout_tuple), wl.lam, wl.scope)
        coeff = torch.from_numpy(g.astype(np.float32)).cuda()
        stats = torch.zeros(2, dtype=torch.int64, device="cuda")
        d_skip = _bwd(1, H, head, labels, ws, lse, coeff, 1e-6, bm, stats)
        d_filt = _bwd(1, H, head, labels, ws, lse, coeff, 1e-6, None)
        d_two = _bwd(2, H, head, labels, ws, lse, coeff, 1e-6, None)
    finally:
        cce.cce_set_cta_pairs(True)
    skipped, total = stats.cpu().tolist()
    print(f"pairs={pairs}: skipped {skipped} of {total} tiles")
    assert skipped > total // 4
    diff = d_skip != d_filt
    if bool(diff.any()):
        rows = torch.nonzero(diff.any(dim=1)).flatten().tolist()
        err = (d_skip - d_filt).abs()[diff].max().item()
        raise AssertionError(f"skip and filter differ in {int(diff.sum())} elements of "
                             f"{len(rows)} rows (first {rows[:8]}), max |diff| {err:.3e}, "
                             f"NaN {int(torch.isnan(d_skip).sum())}/{int(torch.isnan(d_filt).sum())}")
    want = O.head_dh(wl.H, W, wl.labels, g, olse, filter_eps=1e-6)
    assert rel_fro(d_skip.cpu().numpy(), want) <= TOL_DH
    assert rel_fro(d_skip.cpu().numpy(), d_two.cpu().numpy()) <= 1e-5
    assert np.all(d_skip.cpu().numpy()[:wl.P] == 0.0)


@pytest.mark.parametrize("cap,split,D,V", [(30.0, (100, 150, 131), 256, 4097),
                                           (2.0, (20, 50, 58), 512, 3000)])
def test_fused_softcap(cap, split, D, V):
    wl = S.make_custom(2, M_split=split, D=D, V=V)
    H, head, labels = upload(wl)
    head = cce.Head(w=head.w, V=wl.V, D=wl.D, softcap=cap)
    hd = cce.h_dtype(H)
    cce.cce_set_backward_mode(1)
    try:
        ws = cce.alloc_workspace(wl.M, hd, head)
    finally:
        cce.cce_set_backward_mode(0)
    f = dict(device="cuda", dtype=torch.float32)
    logp, lse = torch.empty(wl.M, **f), torch.empty(wl.M, **f)
    cce.cce_forward(H, head, labels, logp, lse, None, None, ws)
    g = S.random_cotangent(wl)
    coeff = torch.from_numpy(g).cuda()
    d_fused = _bwd(1, H, head, labels, ws, lse, coeff)
    d_two = _bwd(2, H, head, labels, ws, lse, coeff)
    W = oracle_W(wl)
    _, olse, _ = O.head_forward(wl.H, W, wl.labels, softcap=cap)
    want = O.head_dh(wl.H, W, wl.labels, g, olse, softcap=cap)
    assert rel_fro(d_fused.cpu().numpy(), want) <= TOL_DH
    assert rel_fro(d_fused.cpu().numpy(), d_two.cpu().numpy()) <= 1e-5


def test_fused_workspace_too_small_is_reported():
    """Mode 1 (fused only) on a workspace below the fused layout is refused
    before anything is launched; mode 0 falls back to the two GEMMs."""
    wl = S.make_custom(2, M_split=(100, 150, 131), D=256, V=4097)
    H, head, labels, ws, lse, _ = _fwd(wl)
    hd = cce.h_dtype(H)
    lo = cce.workspace_min_bytes(wl.M, hd, head)
    if lo >= ws.numel():
        pytest.skip("the minimum workspace already holds the fused layout")
    small = cce.alloc_workspace(wl.M, hd, head, nbytes=lo)
    coeff = torch.from_numpy(S.random_cotangent(wl)).cuda()
    dH = torch.empty(wl.M, wl.D, device="cuda")
    cce.cce_set_backward_mode(1)
    try:
        with pytest.raises(cce.CCEError) as e:
            cce.cce_backward_dh(H, head, labels, lse, coeff, 0.0, None, dH, None, small)
        assert e.value.status == 4
    finally:
        cce.cce_set_backward_mode(0)
    cce.cce_backward_dh(H, head, labels, lse, coeff, 0.0, None, dH, None, small)
    torch.cuda.synchronize()
    assert cce.cce_device_status(small) == 0


@pytest.mark.parametrize("block_skip", [False, True])
def test_fused_pass_graph_replay(block_skip):
    """The whole head pass with the fused backward (the default from 1,024
    rows) captured in a CUDA graph and replayed gives the direct call's
    bits, also after new inputs are copied into the captured tensors; with
    the filter and block skip on, too (the skip plan, the mask table and the
    exchange counters are rebuilt inside the graph each replay)."""
    wl = S.make_custom(1, M_split=(100, 500, 500), D=256, V=30000, alpha=12.0)
    H, head, labels = upload(wl)
    hd = cce.h_dtype(H)
    direct = cce.HeadBuffers.alloc(wl.M, wl.D, wl.V, hd, head)
    graphed = cce.HeadBuffers.alloc(wl.M, wl.D, wl.V, hd, head)
    assert cce.cce_query_plan(wl.M, hd, head, direct.ws.numel())["bwd_fused"]
    eps = 1e-6 if block_skip else 0.0
    args = (wl.layout_tuple, wl.lam, wl.scope, eps, block_skip)
    g = cce.HeadPassGraph(H, head, labels, *args, graphed)
    for step in range(2):
        if step == 1:
            H.copy_(torch.roll(H, shifts=1, dims=0))
            labels.copy_(torch.roll(labels, shifts=3))
        g.replay()
        cce.orpo_head_pass(H, head, labels, *args, direct)
        torch.cuda.synchronize()
        assert cce.cce_device_status(graphed.ws) == 0
        assert cce.cce_device_status(direct.ws) == 0
        for name in ("logp", "lse", "out8", "coeff", "dH"):
            assert np.array_equal(getattr(graphed, name).cpu().numpy(),
                                  getattr(direct, name).cpu().numpy()), (step, name)
