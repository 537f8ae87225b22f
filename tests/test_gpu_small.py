"""GPU parity of the C-ABI library against the float64 oracle on small,
ragged shapes (several tiles plus tails), the integer-exact indexing design,
the ORPO epilogue, device-side error reporting and the timeout path."""

import dataclasses
import math

import numpy as np
import pytest
import torch

from lm_head_cross_flash_b200 import cce
from lm_head_cross_flash_b200 import synthetic as S
from oracle import flash_cce as O

from helpers import TOL_DH, TOL_LOGP, TOL_LOSS, oracle_W, rel_fro, run_pass, upload

pytestmark = pytest.mark.gpu


def _forward(wl):
    H, head, labels = upload(wl)
    hd = cce.h_dtype(H)
    ws = cce.alloc_workspace(wl.M, hd, head)
    f = dict(device="cuda", dtype=torch.float32)
    logp, lse, tgt = torch.empty(wl.M, **f), torch.empty(wl.M, **f), torch.zeros(wl.M, **f)
    bm = torch.empty(cce.blockmax_cols(wl.V), wl.M, **f)
    cce.cce_forward(H, head, labels, logp, lse, tgt, bm, ws)
    torch.cuda.synchronize()
    assert cce.cce_device_status(ws) == 0
    return (H, head, labels, ws), logp.cpu().numpy(), lse.cpu().numpy(), tgt.cpu().numpy(), bm.cpu().numpy()


SMALL = [
    # (cfg recipe, (P, Rc, Rr), D, V)
    (1, (1, 1, 1), 64, 31),
    (1, (3, 2, 2), 64, 1),
    (1, (40, 44, 44), 128, 256),
    (1, (40, 45, 44), 64, 257),
    (2, (100, 150, 131), 256, 4097),
    (1, (64, 200, 300), 192, 1000),
    (0, (8, 60, 60), 64, 300),
    (0, (32, 96, 128), 256, 4096),
    (4, (40, 45, 44), 128, 257),
    (4, (100, 150, 131), 256, 4097),
    (4, (64, 200, 300), 320, 1000),
]


@pytest.mark.parametrize("cfg,split,D,V", SMALL)
def test_forward_matches_oracle(cfg, split, D, V):
    wl = S.make_custom(cfg, M_split=split, D=D, V=V)
    _, logp, lse, tgt, bm = _forward(wl)
    ologp, olse, otgt = O.head_forward(wl.H, oracle_W(wl), wl.labels)
    assert np.max(np.abs(lse - olse)) <= TOL_LOGP
    assert np.max(np.abs(logp - ologp)) <= TOL_LOGP
    ok = wl.labels >= 0
    assert np.all(logp[~ok] == 0.0)
    assert np.max(np.abs(tgt[ok] - otgt[ok])) <= TOL_LOGP
    # blockmax: max logit per 256-wide vocab block
    Z = wl.H.astype(np.float64) @ oracle_W(wl).T
    nb = cce.blockmax_cols(V)
    want = np.stack([Z[:, b * 256:(b + 1) * 256].max(axis=1) for b in range(nb)])
    assert np.max(np.abs(bm - want)) <= TOL_LOGP


def test_integer_design_is_bit_exact():
    """Small-integer H and W are exact in bf16 and their dot products exact in
    fp32, so the gathered target logit must equal the integer exactly, for
    labels in every tile including the tail and the tile edges."""
    P, Rc, Rr, D, V = 50, 60, 70, 128, 1100
    M = P + Rc + Rr
    g = np.random.default_rng(5)
    H = g.integers(-3, 4, size=(M, D)).astype(np.float32)
    W = g.integers(-2, 3, size=(V, D)).astype(np.float32)
    labels = g.integers(0, V, size=M).astype(np.int32)
    edge = [0, 255, 256, 511, 512, 1023, 1024, 1099]
    labels[1:1 + len(edge)] = edge
    labels[0] = -1
    labels[17] = -5
    wl = S.make_custom(1, M_split=(P, Rc, Rr), D=D, V=V)
    wl.H, wl.W, wl.labels = H, W, labels
    wl.H_bits, wl.W_bits = S.f32_to_bf16_bits(H), S.f32_to_bf16_bits(W)
    _, logp, lse, tgt, _ = _forward(wl)
    exact = (H.astype(np.int64) @ W.astype(np.int64).T)
    ok = labels >= 0
    want = exact[np.nonzero(ok)[0], labels[ok]].astype(np.float32)
    assert np.array_equal(tgt[ok], want)
    assert np.all(logp[~ok] == 0.0)


@pytest.mark.parametrize("cfg,split,D,V", [(1, (40, 45, 44), 64, 257),
                                           (2, (100, 150, 131), 256, 4097),
                                           (0, (8, 60, 60), 64, 300),
                                           (4, (100, 150, 131), 256, 4097),
                                           (4, (64, 200, 300), 320, 1000)])
def test_backward_random_cotangent(cfg, split, D, V):
    """dH with a non-uniform cotangent (rows with zero cotangent stay 0)."""
    wl = S.make_custom(cfg, M_split=split, D=D, V=V)
    (H, head, labels, ws), logp, lse, _, bm = _forward(wl)
    g = S.random_cotangent(wl)
    g[5:9] = 0.0
    coeff = torch.from_numpy(g).cuda()
    dH = torch.full((wl.M, wl.D), float("nan"), device="cuda")
    lse_t = torch.from_numpy(lse).cuda()
    cce.cce_backward_dh(H, head, labels, lse_t, coeff, 0.0, None, dH, None, ws)
    torch.cuda.synchronize()
    assert cce.cce_device_status(ws) == 0
    dH = dH.cpu().numpy()
    want = O.head_dh(wl.H, oracle_W(wl), wl.labels, g, O.head_forward(wl.H, oracle_W(wl), wl.labels)[1])
    assert rel_fro(dH, want) <= TOL_DH, rel_fro(dH, want)
    assert np.all(dH[wl.labels < 0] == 0.0)
    assert np.all(dH[5:9] == 0.0)


def test_backward_narrow_workspace_chunks():
    """A workspace that only fits a 256-wide vocab chunk gives the same dH."""
    wl = S.make_custom(2, M_split=(60, 70, 80), D=128, V=1500)
    (H, head, labels, ws), logp, lse, _, _ = _forward(wl)
    g = torch.from_numpy(S.random_cotangent(wl)).cuda()
    lse_t = torch.from_numpy(lse).cuda()
    d1 = torch.empty(wl.M, wl.D, device="cuda")
    cce.cce_backward_dh(H, head, labels, lse_t, g, 0.0, None, d1, None, ws)
    small = cce.alloc_workspace(wl.M, cce.h_dtype(H), head,
                                nbytes=cce.workspace_min_bytes(wl.M, cce.h_dtype(H), head))
    d2 = torch.empty(wl.M, wl.D, device="cuda")
    cce.cce_backward_dh(H, head, labels, lse_t, g, 0.0, None, d2, None, small)
    torch.cuda.synchronize()
    assert rel_fro(d2.cpu().numpy(), d1.cpu().numpy()) < 1e-5


@pytest.mark.parametrize("cfg,scope", [(0, "full"), (0, "response"), (4, "full")])
def test_full_pass_small(cfg, scope):
    wl = S.make_custom(cfg, M_split=(32, 96, 128), D=256, V=4096)
    wl.scope = scope
    _, _, _, buf, st = run_pass(wl)
    assert st == 0
    W = oracle_W(wl)
    L = O.Layout(*wl.layout_tuple)
    ologp, olse, _ = O.head_forward(wl.H, W, wl.labels)
    o = O.orpo_loss_from_logps(ologp, wl.labels, L, wl.lam, scope)
    g = O.orpo_grad_coeffs(ologp, wl.labels, L, wl.lam, scope)
    odh = O.head_dh(wl.H, W, wl.labels, g, olse)
    assert np.max(np.abs(buf.logp.cpu().numpy() - ologp)) <= TOL_LOGP
    assert np.max(np.abs(buf.lse.cpu().numpy() - olse)) <= TOL_LOGP
    out8 = buf.out8.cpu().numpy()
    assert abs(out8[0] - o.loss) <= TOL_LOSS * abs(o.loss)
    assert rel_fro(buf.coeff.cpu().numpy(), g) <= 1e-5
    assert rel_fro(buf.dH.cpu().numpy(), odh) <= TOL_DH


def test_orpo_epilogue_matches_oracle_at_full_size():
    """The ORPO epilogue on seeded log-probs of the long-pair shape."""
    P, Rc, Rr = 1024, 3584, 3584
    M = P + Rc + Rr
    lp = S.random_logps(M, seed=3)
    y = np.random.default_rng(4).integers(-1, 1000, size=M).astype(np.int32)
    y[0] = -1
    L = O.Layout.contiguous(P, Rc, Rr)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    out8 = torch.empty(8, dtype=torch.float64, device="cuda")
    coeff = torch.empty(M, device="cuda")
    lpt, yt = torch.from_numpy(lp).cuda(), torch.from_numpy(y).cuda()
    for scope in ("full", "response"):
        for lam in (0.0, 0.1, 1.0):
            cce.orpo_loss_from_logps(lpt, yt, dataclasses.astuple(L), lam, scope, out8, ws)
            cce.orpo_grad_coeffs(lpt, yt, dataclasses.astuple(L), lam, scope, coeff, ws)
            torch.cuda.synchronize()
            assert cce.cce_device_status(ws) == 0
            o = O.orpo_loss_from_logps(lp, y, L, lam, scope)
            got = out8.cpu().numpy()
            want = np.array(o.as8())
            assert np.allclose(got, want, rtol=1e-12, atol=1e-14), (got, want)
            g = O.orpo_grad_coeffs(lp, y, L, lam, scope)
            assert np.allclose(coeff.cpu().numpy(), g, rtol=1e-6, atol=1e-12)


def test_device_errors_are_reported_not_trapped():
    wl = S.make_custom(1, M_split=(4, 4, 4), D=64, V=100)
    wl.labels[3] = 100  # == V
    H, head, labels = upload(wl)
    ws = cce.alloc_workspace(wl.M, cce.h_dtype(H), head)
    f = dict(device="cuda", dtype=torch.float32)
    logp, lse = torch.empty(wl.M, **f), torch.empty(wl.M, **f)
    cce.cce_forward(H, head, labels, logp, lse, None, None, ws)
    assert cce.cce_device_status(ws) == 5          # label out of range
    assert cce.cce_device_status(ws) == 0          # cleared
    # empty rejected segment: every rejected row ignored
    y = labels.clone()
    y[8:] = -1
    out8 = torch.empty(8, dtype=torch.float64, device="cuda")
    cce.orpo_loss_from_logps(logp, y, wl.layout_tuple, 0.1, "full", out8, ws)
    assert cce.cce_device_status(ws) == 7
    assert torch.isnan(out8).all()
    # the context is still usable
    cce.cce_forward(H, head, labels.clamp(max=99), logp, lse, None, None, ws)
    assert cce.cce_device_status(ws) == 0


def test_timeout_path_reports_and_recovers():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    cce.cce_set_wait_limit_ns(2_000_000)  # 2 ms
    try:
        cce.cce_selftest_wait_timeout(ws)
        assert cce.cce_device_status(ws) == 6
    finally:
        cce.cce_set_wait_limit_ns(0)
    assert cce.cce_device_status(ws) == 0


def test_synchronous_argument_errors():
    wl = S.make_custom(1, M_split=(4, 4, 4), D=64, V=100)
    H, head, labels = upload(wl)
    ws = cce.alloc_workspace(wl.M, cce.h_dtype(H), head)
    f = dict(device="cuda", dtype=torch.float32)
    logp, lse = torch.empty(wl.M, **f), torch.empty(wl.M, **f)
    with pytest.raises(cce.CCEError) as e:
        cce.cce_forward(H, head, labels, logp, lse, None, None, ws[:1024])
    assert e.value.status == 4
    bad = cce.Head(w=head.w, V=wl.V, D=96)
    with pytest.raises(cce.CCEError) as e:
        cce.cce_forward(H, bad, labels, logp, lse, None, None, ws)
    assert e.value.status == 2


@pytest.mark.parametrize("kind", ["orpo", "simpo", "orpo_margin"])
def test_objective_siblings_match_oracle(kind):
    """ORPO, SimPO and ORPO + SimPO margin on seeded log-probs (full size)."""
    P, Rc, Rr = 1024, 3584, 3584
    M = P + Rc + Rr
    lp = S.random_logps(M, seed=5, scale=3.0)
    y = np.random.default_rng(6).integers(-1, 1000, size=M).astype(np.int32)
    L = O.Layout.contiguous(P, Rc, Rr)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    out8 = torch.empty(8, dtype=torch.float64, device="cuda")
    coeff = torch.empty(M, device="cuda")
    lpt, yt = torch.from_numpy(lp).cuda(), torch.from_numpy(y).cuda()
    for scope in ("full", "response"):
        for lam, beta, gamma in ((0.1, 2.0, 0.5), (1.0, 0.5, 0.0)):
            cce.pref_loss_from_logps(lpt, yt, dataclasses.astuple(L), kind, lam, beta, gamma,
                                     scope, out8, ws)
            cce.pref_grad_coeffs(lpt, yt, dataclasses.astuple(L), kind, lam, beta, gamma,
                                 scope, coeff, ws)
            torch.cuda.synchronize()
            assert cce.cce_device_status(ws) == 0
            o = O.pref_loss_from_logps(lp, y, L, kind, lam, beta, gamma, scope)
            assert np.allclose(out8.cpu().numpy(), np.array(o.as8()), rtol=1e-12, atol=1e-14)
            g = O.pref_grad_coeffs(lp, y, L, kind, lam, beta, gamma, scope)
            assert np.allclose(coeff.cpu().numpy(), g, rtol=1e-6, atol=1e-12)


@pytest.mark.parametrize("cfg,cap,qmode", [(1, 30.0, 0), (2, 2.0, 0), (4, 30.0, 1),
                                           (4, 30.0, 2), (0, 5.0, 0)])
def test_softcap_forward_and_backward(cfg, cap, qmode):
    """Gemma-style logit capping: capped logits in the forward, the
    1 - tanh^2 factor in the backward (4-bit head: in-kernel and staged)."""
    cce.cce_set_quant_staging(qmode)
    try:
        _softcap_case(cfg, cap)
    finally:
        cce.cce_set_quant_staging(0)


def _softcap_case(cfg, cap):
    wl = S.make_custom(cfg, M_split=(60, 70, 80), D=128, V=1500)
    H, head, labels = upload(wl)
    head.softcap = cap
    hd = cce.h_dtype(H)
    ws = cce.alloc_workspace(wl.M, hd, head)
    f = dict(device="cuda", dtype=torch.float32)
    logp, lse = torch.empty(wl.M, **f), torch.empty(wl.M, **f)
    cce.cce_forward(H, head, labels, logp, lse, None, None, ws)
    g = S.random_cotangent(wl)
    dH = torch.empty(wl.M, wl.D, **f)
    cce.cce_backward_dh(H, head, labels, lse, torch.from_numpy(g).cuda(), 0.0, None, dH, None, ws)
    torch.cuda.synchronize()
    assert cce.cce_device_status(ws) == 0
    W = oracle_W(wl)
    ologp, olse, _ = O.head_forward(wl.H, W, wl.labels, softcap=cap)
    assert np.max(np.abs(logp.cpu().numpy() - ologp)) <= TOL_LOGP
    assert np.max(np.abs(lse.cpu().numpy() - olse)) <= TOL_LOGP
    want = O.head_dh(wl.H, W, wl.labels, g, olse, softcap=cap)
    assert rel_fro(dH.cpu().numpy(), want) <= TOL_DH


@pytest.mark.parametrize("qmode", [1, 2])
@pytest.mark.parametrize("split,D,V,cap", [((40, 45, 44), 128, 257, 0.0),
                                           ((100, 150, 131), 256, 4097, 0.0),
                                           ((64, 200, 300), 320, 1000, 30.0)])
def test_q8_head_forward_and_backward(split, D, V, cap, qmode):
    """8-bit affine head (group 64), dequantised in-kernel (1) or staged (2)."""
    wl = S.make_custom(4, M_split=split, D=D, V=V, wformat="q8g64")
    H, head, labels = upload(wl)
    head.softcap = cap
    cce.cce_set_quant_staging(qmode)
    try:
        _q8_pass_and_check(wl, H, head, labels, cap)
    finally:
        cce.cce_set_quant_staging(0)


def _q8_pass_and_check(wl, H, head, labels, cap):
    ws = cce.alloc_workspace(wl.M, cce.h_dtype(H), head)
    f = dict(device="cuda", dtype=torch.float32)
    logp, lse = torch.empty(wl.M, **f), torch.empty(wl.M, **f)
    cce.cce_forward(H, head, labels, logp, lse, None, None, ws)
    g = S.random_cotangent(wl)
    dH = torch.empty(wl.M, wl.D, **f)
    cce.cce_backward_dh(H, head, labels, lse, torch.from_numpy(g).cuda(), 0.0, None, dH, None, ws)
    torch.cuda.synchronize()
    assert cce.cce_device_status(ws) == 0
    W = oracle_W(wl)
    ologp, olse, _ = O.head_forward(wl.H, W, wl.labels, softcap=cap)
    assert np.max(np.abs(logp.cpu().numpy() - ologp)) <= TOL_LOGP
    assert np.max(np.abs(lse.cpu().numpy() - olse)) <= TOL_LOGP
    want = O.head_dh(wl.H, W, wl.labels, g, olse, softcap=cap)
    assert rel_fro(dH.cpu().numpy(), want) <= TOL_DH


def test_prefix_shared_pair_end_to_end():
    """Gather the head rows of a prefix-shared pair from one concatenated
    forward, run the head, scatter dH back; compare with the oracle."""
    P, Rc, Rr, D, V = 40, 70, 90, 128, 1500
    wl = S.make_custom(2, M_split=(P, Rc, Rr), D=D, V=V)
    Hcat, head, labels = upload(wl)           # treat the drawn rows as H_cat
    Hh = torch.empty_like(Hcat)
    cce.cce_prefix_gather(Hcat, P, Rc, Rr, Hh)
    torch.cuda.synchronize()
    idx = O.prefix_gather_index(P, Rc, Rr)
    assert torch.equal(Hh, Hcat[torch.from_numpy(idx).cuda()])
    buf = cce.HeadBuffers.alloc(wl.M, wl.D, wl.V, cce.h_dtype(Hh), head)
    cce.orpo_head_pass(Hh, head, labels, wl.layout_tuple, wl.lam, wl.scope, 0.0, False, buf)
    dcat = torch.empty_like(buf.dH)
    cce.cce_prefix_scatter(buf.dH, P, Rc, Rr, dcat)
    torch.cuda.synchronize()
    assert cce.cce_device_status(buf.ws) == 0
    W = oracle_W(wl)
    L = O.Layout(*wl.layout_tuple)
    Hh64 = O.prefix_gather(wl.H, P, Rc, Rr)
    want = O.prefix_scatter(O.orpo_head_grad(Hh64, W, wl.labels, L, wl.lam, wl.scope), P, Rc, Rr)
    assert rel_fro(dcat.cpu().numpy(), want) <= TOL_DH
    assert np.all(dcat.cpu().numpy()[P + Rc - 1] == 0)
    # the scatter is exact: sums of at most two fp32 values, in a fixed order
    G = np.random.default_rng(12).standard_normal((wl.M, D)).astype(np.float32)
    out = torch.empty(wl.M, D, device="cuda")
    cce.cce_prefix_scatter(torch.from_numpy(G).cuda(), P, Rc, Rr, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), O.prefix_scatter(G, P, Rc, Rr).astype(np.float32))


@pytest.mark.parametrize("cfg,split,D,V,cap,eps", [
    (1, (40, 45, 44), 128, 257, 0.0, 0.0),
    (2, (100, 150, 131), 256, 4097, 0.0, 0.0),
    (0, (8, 60, 60), 64, 300, 0.0, 0.0),
    (1, (64, 200, 300), 192, 1000, 30.0, 0.0),
    (3, (100, 150, 131), 256, 4097, 0.0, 1e-4),
])
def test_trainable_head_dw(cfg, split, D, V, cap, eps):
    """dW = sum_m coeff (onehot - p) H_m, and dH unchanged by asking for dW."""
    wl = S.make_custom(cfg, M_split=split, D=D, V=V)
    H, head, labels = upload(wl)
    head.softcap = cap
    hd = cce.h_dtype(H)
    ws = cce.alloc_workspace(wl.M, hd, head)
    f = dict(device="cuda", dtype=torch.float32)
    logp, lse = torch.empty(wl.M, **f), torch.empty(wl.M, **f)
    cce.cce_forward(H, head, labels, logp, lse, None, None, ws)
    g = S.random_cotangent(wl)
    g[: split[0] // 2] = 0.0            # a run of zero-cotangent rows
    coeff = torch.from_numpy(g).cuda()
    dH1 = torch.empty(wl.M, wl.D, **f)
    dH0 = torch.empty(wl.M, wl.D, **f)
    cce.cce_backward_dh(H, head, labels, lse, coeff, eps, None, dH0, None, ws)
    cce.cce_set_backward_mode(2)   # the two GEMMs per chunk, as the dW call runs them
    try:
        cce.cce_backward_dh(H, head, labels, lse, coeff, eps, None, dH1, None, ws)
    finally:
        cce.cce_set_backward_mode(0)
    dH2 = torch.empty(wl.M, wl.D, **f)
    dW = torch.full((wl.V, wl.D), float("nan"), **f)
    cce.cce_backward_dh_dw(H, head, labels, lse, coeff, eps, None, dH2, dW, None, ws)
    torch.cuda.synchronize()
    assert cce.cce_device_status(ws) == 0
    assert torch.equal(dH1, dH2)
    # the default backward (fused for dense bf16 heads) agrees to accumulation order
    assert rel_fro(dH0.cpu().numpy(), dH1.cpu().numpy()) <= 1e-5
    W = oracle_W(wl)
    olse = O.head_forward(wl.H, W, wl.labels, softcap=cap)[1]
    want = O.head_dw(wl.H, W, wl.labels, g, olse, filter_eps=eps, softcap=cap)
    if eps > 0:  # the filter is an approximation: compare with the unfiltered dW
        want = O.head_dw(wl.H, W, wl.labels, g, olse, softcap=cap)
    assert rel_fro(dW.cpu().numpy(), want) <= TOL_DH, rel_fro(dW.cpu().numpy(), want)


def test_trainable_head_rejects_quantised_heads():
    wl = S.make_custom(4, M_split=(8, 8, 8), D=128, V=300)
    H, head, labels = upload(wl)
    ws = cce.alloc_workspace(wl.M, cce.h_dtype(H), head)
    f = dict(device="cuda", dtype=torch.float32)
    z = torch.zeros(wl.M, **f)
    with pytest.raises(cce.CCEError) as e:
        cce.cce_backward_dh_dw(H, head, labels, z, z, 0.0, None, torch.empty(wl.M, wl.D, **f),
                               torch.empty(wl.V, wl.D, **f), None, ws)
    assert e.value.status == 2


@pytest.mark.parametrize("cfg,split,D,V,wformat", [(1, (40, 45, 44), 128, 257, None),
                                                   (2, (100, 150, 262), 256, 4097, None),
                                                   (1, (300, 400, 500), 512, 3000, None),
                                                   (1, (300, 400, 400), 448, 2000, None),
                                                   (0, (8, 60, 188), 64, 300, None),
                                                   (0, (40, 100, 116), 256, 1000, None),
                                                   (4, (40, 45, 44), 192, 3000, "q4g64"),
                                                   (4, (300, 400, 400), 512, 5000, "q4g64"),
                                                   (4, (40, 45, 44), 128, 3000, "q8g64"),
                                                   (4, (100, 150, 262), 320, 5000, "q8g64")])
def test_cta_pairs_match_single_cta(cfg, split, D, V, wformat):
    """The 2-CTA (cta_group::2) tiles and the single-CTA tiles agree, and both
    match the oracle.  Row counts are ones that take pairs (at least two
    128-row tiles, at most an eighth of padding): 129, 512, 1200, 1100 (nine
    row tiles, the last pair half empty) and 256 rows; K depths from 2 to 12
    steps of 64 wrap the 6-stage ring.  The 4- and 8-bit heads run with the
    in-kernel dequantisation, which stays on single-CTA tiles: both settings
    must give the same results."""
    wl = S.make_custom(cfg, M_split=split, D=D, V=V, wformat=wformat)
    outs = []
    for pairs in (True, False):
        cce.cce_set_cta_pairs(pairs)
        cce.cce_set_quant_staging(1)
        try:
            _, _, _, buf, st = run_pass(wl)
        finally:
            cce.cce_set_cta_pairs(True)
            cce.cce_set_quant_staging(0)
        assert st == 0
        outs.append((buf.logp.cpu().numpy(), buf.lse.cpu().numpy(), buf.dH.cpu().numpy()))
    (lp1, ls1, d1), (lp0, ls0, d0) = outs
    assert np.max(np.abs(lp1 - lp0)) <= 1e-5 and np.max(np.abs(ls1 - ls0)) <= 1e-5
    assert rel_fro(d1, d0) <= 1e-3
    W = oracle_W(wl)
    ologp, olse, _ = O.head_forward(wl.H, W, wl.labels)
    assert np.max(np.abs(lp1 - ologp)) <= TOL_LOGP


def _staged_two_chunk_ws(M, hd, head, V):
    """Smallest workspace (in steps of 64 vocab rows) on which both passes run
    staged fp16 chunks and neither fits the vocabulary in one chunk."""
    lo = cce.workspace_min_bytes(M, hd, head)
    step = 64 * (2 * M + 2 * head.D)
    for i in range(1, 20000):
        p = cce.cce_query_plan(M, hd, head, lo + i * step)
        if p["bwd_staged"] and p["fwd_staged"]:
            assert p["fwd_chunk"] < V and p["bwd_chunk"] < V, p
            return lo + i * step
    raise AssertionError("no workspace gives staged chunks")


@pytest.mark.parametrize("wformat", ["q4g64", "q8g64"])
@pytest.mark.parametrize("split,D,V,cap", [((40, 45, 44), 128, 20000, 0.0),
                                           ((100, 150, 262), 256, 30001, 0.0),
                                           ((300, 400, 400), 192, 18000, 30.0)])
def test_quant_staging_modes(wformat, split, D, V, cap):
    """4/8-bit heads dequantised in the GEMM (mode 1) and staged as fp16
    chunks (mode 2, on a workspace where both passes take two chunks or more)
    both match the oracle, and match each other to accumulation order (the
    fp16 weights are the same)."""
    wl = S.make_custom(4, M_split=split, D=D, V=V, wformat=wformat)
    H, head, labels = upload(wl)
    head.softcap = cap
    hd = cce.h_dtype(H)
    g = torch.from_numpy(S.random_cotangent(wl)).cuda()
    f = dict(device="cuda", dtype=torch.float32)
    outs = {}
    for mode in (1, 2):
        cce.cce_set_quant_staging(mode)
        try:
            ws_bytes = _staged_two_chunk_ws(wl.M, hd, head, V) if mode == 2 else None
            ws = cce.alloc_workspace(wl.M, hd, head, nbytes=ws_bytes)
            logp, lse = torch.empty(wl.M, **f), torch.empty(wl.M, **f)
            dH = torch.empty(wl.M, wl.D, **f)
            cce.cce_profile_enable(True)
            cce.cce_forward(H, head, labels, logp, lse, None, None, ws)
            cce.cce_backward_dh(H, head, labels, lse, g, 0.0, None, dH, None, ws)
            torch.cuda.synchronize()
            prof = cce.cce_profile_read()
        finally:
            cce.cce_profile_enable(False)
            cce.cce_set_quant_staging(0)
        assert cce.cce_device_status(ws) == 0
        n_deq = prof.get("dequant_chunk", (0.0, 0))[1]
        if mode == 1:
            assert n_deq == 0
        else:
            assert n_deq >= 4  # two or more chunks in each of the two passes
        outs[mode] = (logp.cpu().numpy(), lse.cpu().numpy(), dH.cpu().numpy())
    W = oracle_W(wl)
    ologp, olse, _ = O.head_forward(wl.H, W, wl.labels, softcap=cap)
    want = O.head_dh(wl.H, W, wl.labels, g.cpu().numpy(), olse, softcap=cap)
    for mode in (1, 2):
        lp, ls, dh = outs[mode]
        assert np.max(np.abs(lp - ologp)) <= TOL_LOGP
        assert np.max(np.abs(ls - olse)) <= TOL_LOGP
        assert rel_fro(dh, want) <= TOL_DH
    assert np.max(np.abs(outs[1][0] - outs[2][0])) <= 1e-4
    assert rel_fro(outs[2][2], outs[1][2]) <= 1e-3


@pytest.mark.parametrize("extra_kb", [0, 300, 600])
def test_small_m_many_k_splits(extra_kb):
    """M = 64 gives one dH tile per d-tile, so the dH GEMM splits K up to 32
    ways.  Workspaces between the minimum and a few chunks wide make vocab
    chunks whose last one is narrower than the split count (splits without K
    steps); dH must still match the oracle and the wide-workspace result."""
    wl = S.make_custom(2, M_split=(8, 28, 28), D=256, V=5000)
    (H, head, labels, ws), logp, lse, _, _ = _forward(wl)
    g = torch.from_numpy(S.random_cotangent(wl)).cuda()
    lse_t = torch.from_numpy(lse).cuda()
    d1 = torch.empty(wl.M, wl.D, device="cuda")
    cce.cce_backward_dh(H, head, labels, lse_t, g, 0.0, None, d1, None, ws)
    hd = cce.h_dtype(H)
    nbytes = cce.workspace_min_bytes(wl.M, hd, head) + 31 * wl.M * wl.D * 4 + extra_kb * 1024
    small = cce.alloc_workspace(wl.M, hd, head, nbytes=nbytes)
    d2 = torch.empty(wl.M, wl.D, device="cuda")
    cce.cce_backward_dh(H, head, labels, lse_t, g, 0.0, None, d2, None, small)
    torch.cuda.synchronize()
    assert cce.cce_device_status(ws) == 0 and cce.cce_device_status(small) == 0
    W = oracle_W(wl)
    want = O.head_dh(wl.H, W, wl.labels, g.cpu().numpy(), O.head_forward(wl.H, W, wl.labels)[1])
    assert rel_fro(d1.cpu().numpy(), want) <= TOL_DH
    assert rel_fro(d2.cpu().numpy(), want) <= TOL_DH
    assert rel_fro(d2.cpu().numpy(), d1.cpu().numpy()) < 1e-5


@pytest.mark.parametrize("cfg,split,D,V", [(0, (32, 96, 128), 256, 4096),
                                           (1, (100, 150, 262), 256, 3000),
                                           (4, (40, 45, 44), 128, 2000)])
def test_head_pass_graph_replay(cfg, split, D, V):
    """The whole head pass captured in a CUDA graph and replayed gives the
    same results, bit for bit, as direct calls, also after new inputs are
    copied into the captured tensors."""
    wl = S.make_custom(cfg, M_split=split, D=D, V=V)
    H, head, labels = upload(wl)
    hd = cce.h_dtype(H)
    direct = cce.HeadBuffers.alloc(wl.M, wl.D, wl.V, hd, head)
    graphed = cce.HeadBuffers.alloc(wl.M, wl.D, wl.V, hd, head)
    args = (wl.layout_tuple, wl.lam, wl.scope, wl.filter_eps, wl.block_skip)
    g = cce.HeadPassGraph(H, head, labels, *args, graphed)
    for step in range(2):
        if step == 1:  # new inputs into the captured tensors
            H.copy_(torch.roll(H, shifts=1, dims=0))
            labels.copy_(torch.roll(labels, shifts=3))
        g.replay()
        cce.orpo_head_pass(H, head, labels, *args, direct)
        torch.cuda.synchronize()
        assert cce.cce_device_status(graphed.ws) == 0
        assert cce.cce_device_status(direct.ws) == 0
        for name in ("logp", "lse", "out8", "coeff", "dH"):
            a = getattr(graphed, name).cpu().numpy()
            b = getattr(direct, name).cpu().numpy()
            assert np.array_equal(a, b), (step, name)


def test_domain_and_empty_segments_are_reported():
    """Device-side errors of the epilogue, reported through the status word:
    a mean log-prob >= 0 (outside the domain of log1mexp), an all-ignored
    batch, and empty segments reaching the sharded epilogue through zero
    counts.  Outputs are NaN losses and zero cotangents; nothing traps."""
    wl = S.make_custom(1, M_split=(4, 6, 6), D=64, V=300)
    H, head, labels = upload(wl)
    ws = cce.alloc_workspace(wl.M, cce.h_dtype(H), head)
    f = dict(device="cuda", dtype=torch.float32)
    out8 = torch.empty(8, dtype=torch.float64, device="cuda")
    coeff = torch.empty(wl.M, **f)
    # chosen rows with logp = 0: lw = 0, log1mexp undefined
    logp = torch.full((wl.M,), -3.0, **f)
    logp[4:10] = 0.0
    y = labels.clamp(min=0)
    cce.orpo_loss_from_logps(logp, y, wl.layout_tuple, 0.1, "full", out8, ws)
    assert cce.cce_device_status(ws) == 8
    assert torch.isnan(out8).all()
    cce.orpo_grad_coeffs(logp, y, wl.layout_tuple, 0.1, "full", coeff, ws)
    assert cce.cce_device_status(ws) == 8
    assert torch.count_nonzero(coeff).item() == 0
    # every label ignored: the forward is fine (logp = 0), the loss is not
    lp, lse = torch.empty(wl.M, **f), torch.empty(wl.M, **f)
    none = torch.full_like(labels, -1)
    cce.cce_forward(H, head, none, lp, lse, None, None, ws)
    assert cce.cce_device_status(ws) == 0
    assert torch.count_nonzero(lp).item() == 0 and torch.isfinite(lse).all()
    cce.orpo_loss_from_logps(lp, none, wl.layout_tuple, 0.1, "full", out8, ws)
    assert cce.cce_device_status(ws) == 7
    # sharded epilogue: all-reduced counts of zero for the chosen segment
    sums = torch.tensor([-3.0, 0.0, -12.0, 1.0, 0.0, 4.0], dtype=torch.float64,
                        device="cuda")
    cce.orpo_from_sums(sums, y, wl.layout_tuple, 0.1, "full", out8, coeff, ws)
    assert cce.cce_device_status(ws) == 7
    assert torch.isnan(out8).all()
    # and the partial sums of a valid shard equal the host sums
    logp = torch.linspace(-9.0, -1.0, wl.M, **f)
    cce.orpo_partial_sums(logp, y, wl.layout_tuple, sums, ws)
    torch.cuda.synchronize()
    assert cce.cce_device_status(ws) == 0
    lpn = logp.cpu().double().numpy()
    want = [lpn[0:4].sum(), lpn[4:10].sum(), lpn[10:16].sum(), 4, 6, 6]
    assert np.allclose(sums.cpu().numpy(), want, rtol=1e-12, atol=1e-12)
