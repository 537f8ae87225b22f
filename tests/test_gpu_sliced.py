"""GPU parity of the sliced backward (one kernel for at most 64 head rows:
clusters of up to 8 CTAs each own 256 columns of D, sum their partial
logits through distributed shared memory, form the coefficient tile and
contract it with W into a TMEM-resident dH) against the float64 oracle and
against the two-GEMM backward.

Shapes cover clusters of 1, 2, 4 and 8 CTAs (D from 64 to 2048, with a last
slice partly or wholly past D: D = 320, 1536), 1 to 64 rows, and
vocabularies from 1 to 20,000 with ragged tails.  The filter and block skip,
the softcap, rows without a cotangent, unlabelled rows and determinism (two
calls give the same bits) are checked as well."""

import numpy as np
import pytest
import torch

from lm_head_cross_flash_b200 import cce
from lm_head_cross_flash_b200 import synthetic as S
from oracle import flash_cce as O

from helpers import TOL_DH, oracle_W, rel_fro, upload

pytestmark = pytest.mark.gpu

# The sliced kernel sums the logits of its D slices in fp32 in another order
# than one accumulator over all of D, so a G'' value near a bf16 rounding
# boundary can round the other way: it agrees with the two-GEMM form to
# accumulation order, not bit for bit.
TOL_VS_TWO_GEMM = 1e-4


def _fwd(wl, head=None):
    """Forward, with a workspace sized for the sliced backward (mode 3)."""
    H, head0, labels = upload(wl)
    head = head0 if head is None else head
    hd = cce.h_dtype(H)
    cce.cce_set_backward_mode(3)
    try:
        ws = cce.alloc_workspace(wl.M, hd, head)
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
    # (recipe, (P, Rc, Rr), D, V)
    (1, (1, 1, 1), 64, 31),           # one CTA per cluster
    (1, (1, 1, 1), 64, 1),
    (2, (3, 2, 2), 256, 5000),
    (1, (8, 10, 12), 320, 257),       # two CTAs, the second slice mostly past D
    (2, (10, 10, 11), 512, 4097),     # two CTAs
    (1, (20, 20, 24), 1024, 3000),    # four CTAs, 64 rows
    (2, (16, 20, 24), 1536, 7000),    # eight CTAs, the last two slices past D
    (2, (20, 20, 24), 2048, 20000),   # eight CTAs, 64 rows
    (2, (2, 3, 4), 2048, 300),
]


@pytest.mark.parametrize("cfg,split,D,V", CASES)
def test_sliced_backward_matches_oracle_and_two_gemm(cfg, split, D, V):
    wl = S.make_custom(cfg, M_split=split, D=D, V=V)
    H, head, labels, ws, lse, _ = _fwd(wl)
    cce.cce_set_backward_mode(3)
    try:
        plan = cce.cce_query_plan(wl.M, cce.h_dtype(H), head, ws.numel())
    finally:
        cce.cce_set_backward_mode(0)
    assert plan["bwd_sliced"] and not plan["bwd_fused"], plan
    g = S.random_cotangent(wl)
    g[min(1, wl.M - 1):min(3, wl.M)] = 0.0
    coeff = torch.from_numpy(g).cuda()
    d_sl = _bwd(3, H, head, labels, ws, lse, coeff)
    d_again = _bwd(3, H, head, labels, ws, lse, coeff)
    assert torch.equal(d_sl, d_again)                    # deterministic
    d_two = _bwd(2, H, head, labels, ws, lse, coeff)
    got = d_sl.cpu().numpy()
    W = oracle_W(wl)
    want = O.head_dh(wl.H, W, wl.labels, g, O.head_forward(wl.H, W, wl.labels)[1])
    err = rel_fro(got, want)
    print(f"M={wl.M} D={D} V={V}: clusters {plan['bwd_sliced_clusters']} x "
          f"{plan['bwd_sliced_ctas']}: rel err {err:.2e}, vs two GEMMs "
          f"{rel_fro(got, d_two.cpu().numpy()):.2e}")
    assert err <= TOL_DH
    assert rel_fro(got, d_two.cpu().numpy()) <= TOL_VS_TWO_GEMM
    assert np.all(got[wl.labels < 0] == 0.0)
    assert np.all(got[min(1, wl.M - 1):min(3, wl.M)] == 0.0)


def test_sliced_filter_block_skip_is_exact():
    """Strongly peaked rows (alpha = 22), so block skip removes tiles; the
    skipped tiles are never loaded, and the result is the filter's to the
    bit; both match the oracle with the same filter and the two-GEMM
    backward with the same filter."""
    wl = S.make_custom(1, M_split=(20, 20, 24), D=256, V=60000, alpha=22.0)
    H, head, labels, ws, lse, bm = _fwd(wl)
    W = oracle_W(wl)
    _, olse, _ = O.head_forward(wl.H, W, wl.labels)
    g = O.orpo_grad_coeffs(O.head_forward(wl.H, W, wl.labels)[0], wl.labels,
                           O.Layout(*wl.layout_tuple), wl.lam, wl.scope)
    coeff = torch.from_numpy(g.astype(np.float32)).cuda()
    stats = torch.zeros(2, dtype=torch.int64, device="cuda")
    d_skip = _bwd(3, H, head, labels, ws, lse, coeff, 1e-6, bm, stats)
    d_filt = _bwd(3, H, head, labels, ws, lse, coeff, 1e-6, None)
    d_two = _bwd(2, H, head, labels, ws, lse, coeff, 1e-6, None)
    skipped, total = stats.cpu().tolist()
    print(f"skipped {skipped} of {total} tiles")
    assert skipped > 0
    assert torch.equal(d_skip, d_filt)
    want = O.head_dh(wl.H, W, wl.labels, g, olse, filter_eps=1e-6)
    assert rel_fro(d_skip.cpu().numpy(), want) <= TOL_DH
    assert rel_fro(d_skip.cpu().numpy(), d_two.cpu().numpy()) <= TOL_VS_TWO_GEMM


@pytest.mark.parametrize("cap,split,D,V", [(30.0, (10, 10, 11), 256, 4097),
                                           (2.0, (20, 20, 24), 2048, 3000)])
def test_sliced_softcap(cap, split, D, V):
    wl = S.make_custom(2, M_split=split, D=D, V=V)
    H, head0, labels = upload(wl)
    head = cce.Head(w=head0.w, V=wl.V, D=wl.D, softcap=cap)
    H, head, labels, ws, lse, _ = _fwd(wl, head)
    g = S.random_cotangent(wl)
    coeff = torch.from_numpy(g).cuda()
    d_sl = _bwd(3, H, head, labels, ws, lse, coeff)
    d_two = _bwd(2, H, head, labels, ws, lse, coeff)
    W = oracle_W(wl)
    _, olse, _ = O.head_forward(wl.H, W, wl.labels, softcap=cap)
    want = O.head_dh(wl.H, W, wl.labels, g, olse, softcap=cap)
    assert rel_fro(d_sl.cpu().numpy(), want) <= TOL_DH
    assert rel_fro(d_sl.cpu().numpy(), d_two.cpu().numpy()) <= TOL_VS_TWO_GEMM


def test_sliced_zero_cotangent_gives_zero():
    """Every row without a cotangent: the plan skips every tile, no cluster
    loads W, and dH is exactly zero."""
    wl = S.make_custom(2, M_split=(10, 10, 11), D=2048, V=5000)
    H, head, labels, ws, lse, _ = _fwd(wl)
    coeff = torch.zeros(wl.M, device="cuda")
    d = _bwd(3, H, head, labels, ws, lse, coeff)
    assert torch.count_nonzero(d).item() == 0


def test_sliced_outside_its_range_is_refused():
    """Mode 3 past 64 rows is CCE_ERR_UNSUPPORTED."""
    wl = S.make_custom(2, M_split=(30, 30, 40), D=256, V=3000)
    H, head, labels, ws, lse, _ = _fwd(wl)
    coeff = torch.from_numpy(S.random_cotangent(wl)).cuda()
    dH = torch.empty(wl.M, wl.D, device="cuda")
    cce.cce_set_backward_mode(3)
    try:
        with pytest.raises(cce.CCEError) as e:
            cce.cce_backward_dh(H, head, labels, lse, coeff, 0.0, None, dH, None, ws)
        assert e.value.status == 2
    finally:
        cce.cce_set_backward_mode(0)


@pytest.mark.parametrize("scope", ["full", "response"])
def test_sliced_through_the_real_pass(scope):
    """The whole head pass (forward, loss, cotangent, dH) with the sliced
    backward, against the oracle; the response scope zeroes the prompt rows'
    cotangent.  Then the same pass captured in a CUDA graph and replayed
    gives the direct call's bits."""
    wl = S.make_custom(2, M_split=(12, 24, 28), D=2048, V=9000)
    wl.scope = scope
    H, head, labels = upload(wl)
    hd = cce.h_dtype(H)
    cce.cce_set_backward_mode(3)
    try:
        direct = cce.HeadBuffers.alloc(wl.M, wl.D, wl.V, hd, head)
        graphed = cce.HeadBuffers.alloc(wl.M, wl.D, wl.V, hd, head)
        args = (wl.layout_tuple, wl.lam, wl.scope, wl.filter_eps, wl.block_skip)
        cce.orpo_head_pass(H, head, labels, *args, direct)
        g = cce.HeadPassGraph(H, head, labels, *args, graphed)
        g.replay()
        torch.cuda.synchronize()
    finally:
        cce.cce_set_backward_mode(0)
    assert cce.cce_device_status(direct.ws) == 0
    assert cce.cce_device_status(graphed.ws) == 0
    W = oracle_W(wl)
    L = O.Layout(*wl.layout_tuple)
    ologp, olse, _ = O.head_forward(wl.H, W, wl.labels)
    o = O.orpo_loss_from_logps(ologp, wl.labels, L, wl.lam, scope)
    gc = O.orpo_grad_coeffs(ologp, wl.labels, L, wl.lam, scope)
    odh = O.head_dh(wl.H, W, wl.labels, gc, olse)
    out8 = direct.out8.cpu().numpy()
    assert abs(out8[0] - o.loss) <= 1e-3 * abs(o.loss)
    assert rel_fro(direct.coeff.cpu().numpy(), gc) <= 1e-5
    assert rel_fro(direct.dH.cpu().numpy(), odh) <= TOL_DH
    for name in ("logp", "lse", "out8", "coeff", "dH"):
        assert np.array_equal(getattr(graphed, name).cpu().numpy(),
                              getattr(direct, name).cpu().numpy()), name
