"""Pins of the float64 oracle against facts fixed outside it.

Each test checks the oracle against something other than itself: closed forms
derived by hand (tests/golden/closed_forms.json), library routines (scipy's
logsumexp / log_softmax / log_expit, torch float64 autograd), finite
differences, invariances and hand-built bit patterns.  A dropped term, a wrong
sign, a wrong index or a transposed operand anywhere in the oracle fails at
least one of them.
"""

import math

import numpy as np
import pytest
import scipy.special as sps

from oracle import flash_cce as O

RNG = np.random.default_rng(2024)


def tiny_case(P=3, Rc=2, Rr=3, D=16, V=64, seed=0, ignore=(0,)):
    g = np.random.default_rng(seed)
    M = P + Rc + Rr
    H = g.standard_normal((M, D))
    W = g.standard_normal((V, D)) / math.sqrt(D)
    y = g.integers(0, V, size=M).astype(np.int32)
    for r in ignore:
        y[r] = -1
    return H, W, y, O.Layout.contiguous(P, Rc, Rr)


# --------------------------------------------------------------------------
# scalar pieces
# --------------------------------------------------------------------------

def test_log1mexp_closed_forms(golden):
    for x, want in golden["log1mexp"]["cases"]:
        assert O.log1mexp(x) == pytest.approx(want, rel=1e-14, abs=0.0)


def test_log1mexp_branches_agree_and_domain():
    x = -math.log(2.0)
    left = math.log1p(-math.exp(x))
    right = math.log(-math.expm1(x))
    assert O.log1mexp(x) == pytest.approx(left, rel=1e-15)
    assert O.log1mexp(x) == pytest.approx(right, rel=1e-15)
    for x in (-1e-300, -1e-5, -0.3, -0.7, -2.0, -30.0, -700.0):
        v = O.log1mexp(x)
        assert math.isfinite(v) and v < 0
    with pytest.raises(ValueError):
        O.log1mexp(0.0)
    with pytest.raises(ValueError):
        O.log1mexp(0.5)


def test_odds_ratio_definition(golden):
    # ORPO's odds are p / (1 - p) with p = exp(mean logp).
    for lw, lr, want in golden["odds_ratio"]["cases"]:
        assert O.orpo_log_odds(lw, lr) == pytest.approx(want, rel=1e-14)
    for lw, lr in [(-0.2, -0.9), (-3.0, -1.0), (-0.05, -0.051), (-8.0, -12.0)]:
        pw, pr = math.exp(lw), math.exp(lr)
        direct = math.log((pw / (1 - pw)) / (pr / (1 - pr)))
        assert O.orpo_log_odds(lw, lr) == pytest.approx(direct, rel=1e-12, abs=1e-12)


def test_softplus_sigmoid_against_scipy():
    for z in (-50.0, -3.0, -1e-8, 0.0, 0.7, 5.0, 40.0):
        assert O.softplus(-z) == pytest.approx(-sps.log_expit(z), rel=1e-14, abs=1e-300)
        assert O.sigmoid(z) == pytest.approx(sps.expit(z), rel=1e-14)


def test_equal_means_give_log2():
    H, W, y, L = tiny_case()
    logp = np.full(len(y), -2.5)
    o = O.orpo_loss_from_logps(logp, y, L, 0.3, "full")
    assert o.z == 0.0
    assert o.l_or == pytest.approx(math.log(2.0), rel=1e-15)


# --------------------------------------------------------------------------
# head forward
# --------------------------------------------------------------------------

def test_forward_against_scipy_log_softmax():
    H, W, y, L = tiny_case(P=5, Rc=7, Rr=6, D=24, V=97, seed=3)
    logp, lse, tgt = O.head_forward(H, W, y, block=4)
    Z = H @ W.T
    assert np.allclose(lse, sps.logsumexp(Z, axis=1), rtol=1e-14, atol=1e-13)
    ls = sps.log_softmax(Z, axis=1)
    for m in range(len(y)):
        if y[m] >= 0:
            assert logp[m] == pytest.approx(ls[m, y[m]], rel=1e-13, abs=1e-13)
            assert tgt[m] == pytest.approx(Z[m, y[m]], rel=1e-14, abs=1e-14)
        else:
            assert logp[m] == 0.0


def test_forward_rows_subset_matches_full():
    H, W, y, L = tiny_case(P=9, Rc=8, Rr=7, D=16, V=50, seed=5)
    full = O.head_forward(H, W, y)
    rows = np.array([0, 3, 11, 23])
    sub = O.head_forward(H, W, y, rows=rows, block=3)
    for a, b in zip(full, sub):
        assert np.allclose(a[rows], b, rtol=1e-14, atol=1e-14)


def test_h_zero_closed_form(golden):
    for case in golden["h_zero"]["cases"]:
        V, lam = case["V"], case["lambda"]
        P, Rc, Rr, D = 4, 5, 6, 8
        M = P + Rc + Rr
        H = np.zeros((M, D))
        g = np.random.default_rng(V)
        W = g.standard_normal((V, D))
        y = g.integers(0, V, size=M).astype(np.int32)
        y[0] = -1
        L = O.Layout.contiguous(P, Rc, Rr)
        logp, lse, _ = O.head_forward(H, W, y, block=8)
        assert np.allclose(lse, math.log(V), rtol=1e-14)
        assert np.allclose(logp[y >= 0], -math.log(V), rtol=1e-13)
        for scope in ("full", "response"):
            o = O.orpo_loss_from_logps(logp, y, L, lam, scope)
            assert o.loss == pytest.approx(case["loss"], rel=1e-12)
            assert o.nll == pytest.approx(case["nll"], rel=1e-12)
            assert o.l_or == pytest.approx(case["l_or"], rel=1e-12)
            # closed-form coefficients: sigma = 1/2, a = V / (V - 1)
            gco = O.orpo_grad_coeffs(logp, y, L, lam, scope)
            a = V / (V - 1.0)
            nP, nC, nR = P - 1, Rc, Rr
            sC = -1.0 / (nP + nC) if scope == "full" else -1.0 / nC
            sP = -1.0 / (nP + nC) if scope == "full" else 0.0
            assert gco[0] == 0.0
            assert np.allclose(gco[1:P], sP, rtol=1e-12)
            assert np.allclose(gco[P:P + Rc], lam * (-0.5) * a / nC + sC, rtol=1e-12)
            assert np.allclose(gco[P + Rc:], -lam * (-0.5) * a / nR, rtol=1e-12)
            # dH_m = g_m (W_y - mean_v W_v) at H = 0
            dH = O.head_dh(H, W, y, gco, lse, block=8)
            mean_w = W.mean(axis=0)
            for m in range(M):
                want = gco[m] * (W[y[m]] - mean_w) if y[m] >= 0 else np.zeros(D)
                assert np.allclose(dH[m], want, rtol=1e-10, atol=1e-14)


# --------------------------------------------------------------------------
# ORPO objective
# --------------------------------------------------------------------------

def test_combine_full_nll_identity():
    H, W, y, L = tiny_case(P=7, Rc=5, Rr=6, D=16, V=40, seed=9, ignore=(0, 8))
    logp, _, _ = O.head_forward(H, W, y)
    o = O.orpo_loss_from_logps(logp, y, L, 0.1, "full")
    # direct token-mean CE over the labelled prompt + chosen rows
    sel = np.zeros(len(y), bool)
    sel[L.prompt_begin:L.chosen_end] = True
    sel &= y >= 0
    Z = H @ W.T
    ce = -sps.log_softmax(Z, axis=1)[np.arange(len(y)), np.maximum(y, 0)]
    assert o.nll == pytest.approx(ce[sel].mean(), rel=1e-13)
    comb = O.combine_full_nll(o.n_prompt, o.pm, o.n_chosen, o.lw)
    assert comb == pytest.approx(o.nll, rel=1e-13)
    assert o.n_prompt == 6 and o.n_chosen == 4


def test_response_scope_is_masked_ce():
    H, W, y, L = tiny_case(P=6, Rc=5, Rr=4, D=12, V=33, seed=4)
    logp, _, _ = O.head_forward(H, W, y)
    o = O.orpo_loss_from_logps(logp, y, L, 0.7, "response")
    Z = H @ W.T
    ce = -sps.log_softmax(Z, axis=1)[np.arange(len(y)), np.maximum(y, 0)]
    mask = np.zeros(len(y), bool)
    mask[L.chosen_begin:L.chosen_end] = True
    assert o.nll == pytest.approx(ce[mask].mean(), rel=1e-13)
    assert o.nll == pytest.approx(-o.lw, rel=1e-15)
    assert o.loss == pytest.approx(o.nll + 0.7 * o.l_or, rel=1e-15)


@pytest.mark.parametrize("scope", ["full", "response"])
@pytest.mark.parametrize("lam", [0.0, 0.1, 1.0])
def test_coeffs_are_dL_dlogp(scope, lam):
    _, _, y, L = tiny_case(P=4, Rc=3, Rr=5, seed=1, ignore=(0, 5))
    g = np.random.default_rng(8)
    logp = -g.random(len(y)) * 4 - 0.05
    logp[y < 0] = 0.0
    coef = O.orpo_grad_coeffs(logp, y, L, lam, scope)
    h = 1e-6
    for m in range(len(y)):
        if y[m] < 0:
            assert coef[m] == 0.0
            continue
        lp, lm = logp.copy(), logp.copy()
        lp[m] += h
        lm[m] -= h
        fd = (O.orpo_loss_from_logps(lp, y, L, lam, scope).loss
              - O.orpo_loss_from_logps(lm, y, L, lam, scope).loss) / (2 * h)
        assert coef[m] == pytest.approx(fd, rel=1e-6, abs=1e-9)


@pytest.mark.parametrize("scope", ["full", "response"])
@pytest.mark.parametrize("lam", [0.0, 0.1, 1.0])
def test_finite_differences_dL_dH(scope, lam):
    """The pages' "real proof": central differences of the scalar loss."""
    H, W, y, L = tiny_case(seed=11)
    dH = O.orpo_head_grad(H, W, y, L, lam, scope)
    h = 1e-6
    fd = np.zeros_like(H)
    for m in range(H.shape[0]):
        for d in range(H.shape[1]):
            Hp, Hm = H.copy(), H.copy()
            Hp[m, d] += h
            Hm[m, d] -= h
            fd[m, d] = (O.orpo_head_loss(Hp, W, y, L, lam, scope)
                        - O.orpo_head_loss(Hm, W, y, L, lam, scope)) / (2 * h)
    assert np.allclose(dH, fd, rtol=1e-6, atol=1e-9)
    assert np.all(dH[0] == 0.0)          # ignored row
    if scope == "response":
        assert np.all(dH[:3] == 0.0)     # prompt rows carry no gradient


def test_against_torch_autograd():
    torch = pytest.importorskip("torch")
    H, W, y, L = tiny_case(P=5, Rc=6, Rr=4, D=20, V=70, seed=21, ignore=(0, 7))
    lam = 0.4
    for scope in ("full", "response"):
        Ht = torch.tensor(H, dtype=torch.float64, requires_grad=True)
        Wt = torch.tensor(W, dtype=torch.float64)
        yt = torch.tensor(np.maximum(y, 0), dtype=torch.long)
        ok = torch.tensor(y >= 0)
        lsm = torch.log_softmax(Ht @ Wt.T, dim=1)
        lp = torch.where(ok, lsm.gather(1, yt[:, None])[:, 0], torch.zeros(()))

        def seg(b, e):
            return lp[b:e][ok[b:e]].sum(), int(ok[b:e].sum())

        sP, nP = seg(L.prompt_begin, L.prompt_end)
        sC, nC = seg(L.chosen_begin, L.chosen_end)
        sR, nR = seg(L.rejected_begin, L.rejected_end)
        lw, lr = sC / nC, sR / nR
        nll = -(sP + sC) / (nP + nC) if scope == "full" else -lw
        z = (lw - lr) - (torch.log(-torch.expm1(lw)) - torch.log(-torch.expm1(lr)))
        loss = nll - lam * torch.nn.functional.logsigmoid(z)
        loss.backward()
        o = O.orpo_loss_from_logps(O.head_forward(H, W, y)[0], y, L, lam, scope)
        assert o.loss == pytest.approx(loss.item(), rel=1e-13)
        dH = O.orpo_head_grad(H, W, y, L, lam, scope)
        assert np.allclose(dH, Ht.grad.numpy(), rtol=1e-10, atol=1e-14)


# --------------------------------------------------------------------------
# invariances
# --------------------------------------------------------------------------

def test_shift_all_head_rows_invariance():
    H, W, y, L = tiny_case(P=4, Rc=4, Rr=4, D=8, V=30, seed=2)
    c = np.random.default_rng(1).standard_normal(8)
    a = O.orpo_head_grad(H, W, y, L, 0.2)
    b = O.orpo_head_grad(H, W + c, y, L, 0.2)
    assert np.allclose(a, b, rtol=1e-9, atol=1e-12)
    la, lb = O.head_forward(H, W, y)[0], O.head_forward(H, W + c, y)[0]
    assert np.allclose(la, lb, rtol=1e-12, atol=1e-12)


def test_vocab_permutation_invariance():
    H, W, y, L = tiny_case(P=4, Rc=4, Rr=4, D=8, V=30, seed=6)
    perm = np.random.default_rng(3).permutation(30)
    inv = np.argsort(perm)
    y2 = np.where(y >= 0, inv[np.maximum(y, 0)], -1).astype(np.int32)
    a = O.head_forward(H, W, y)
    b = O.head_forward(H, W[perm], y2)
    for u, v in zip(a, b):
        assert np.allclose(u, v, rtol=1e-12, atol=1e-12)
    assert np.allclose(O.orpo_head_grad(H, W, y, L, 0.5),
                       O.orpo_head_grad(H, W[perm], y2, L, 0.5), rtol=1e-10, atol=1e-13)


def test_row_permutation_within_segment():
    H, W, y, L = tiny_case(P=4, Rc=5, Rr=6, D=8, V=30, seed=7)
    perm = np.arange(len(y))
    perm[L.chosen_begin:L.chosen_end] = perm[L.chosen_begin:L.chosen_end][::-1]
    perm[L.rejected_begin:L.rejected_end] = np.roll(perm[L.rejected_begin:L.rejected_end], 2)
    la = O.orpo_head_loss(H, W, y, L, 0.1)
    lb = O.orpo_head_loss(H[perm], W, y[perm], L, 0.1)
    assert la == pytest.approx(lb, rel=1e-14)
    ga = O.orpo_head_grad(H, W, y, L, 0.1)
    gb = O.orpo_head_grad(H[perm], W, y[perm], L, 0.1)
    assert np.allclose(ga[perm], gb, rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------------------
# coefficient filter
# --------------------------------------------------------------------------

def test_filter_limits():
    H, W, y, L = tiny_case(P=4, Rc=4, Rr=4, D=8, V=30, seed=12)
    logp, lse, _ = O.head_forward(H, W, y)
    g = O.orpo_grad_coeffs(logp, y, L, 0.1)
    exact = O.head_dh(H, W, y, g, lse)
    assert np.array_equal(O.head_dh(H, W, y, g, lse, filter_eps=0.0), exact)
    # eps above every probability keeps only the target column: g (1 - p_y) W_y
    only_t = O.head_dh(H, W, y, g, lse, filter_eps=2.0)
    for m in range(len(y)):
        if y[m] < 0:
            assert np.all(only_t[m] == 0)
            continue
        p_y = math.exp(logp[m])
        assert np.allclose(only_t[m], g[m] * (1 - p_y) * W[y[m]], rtol=1e-12, atol=1e-15)
    # error grows with eps
    errs = [np.linalg.norm(O.head_dh(H, W, y, g, lse, filter_eps=e) - exact)
            for e in (1e-4, 1e-2, 1e-1)]
    assert errs[0] <= errs[1] <= errs[2]


def _filter_boundary_case():
    """One head row whose logits are (0, 0, -10, -10) through the first
    coordinate of W, with lse taken as 0, so the softmax values the filter
    sees are exactly (1, 1, e^-10, e^-10).  The second coordinate of W tags
    each vocabulary column, so dH shows which terms were kept."""
    W = np.array([[0.0, 1.0], [0.0, 2.0], [-10.0, 4.0], [-10.0, 8.0]])
    H = np.array([[1.0, 0.0]])
    y = np.array([2], dtype=np.int32)
    return H, W, y, np.array([0.0])


@pytest.mark.parametrize("eps", [1.0, 0.6])
def test_filter_boundary_by_hand(eps):
    """A term is dropped iff its softmax p < eps strictly, on p itself (not
    on g*p), and the target column is always kept.  eps = 1: the columns
    with p == eps stay.  eps = 0.6 with g = 0.5: |g*p| = 0.5 < eps <= p = 1,
    so those columns stay too.  Column 3 (p = e^-10 < eps, not the target)
    is dropped; column 2 is the target (p = e^-10, kept)."""
    H, W, y, lse = _filter_boundary_case()
    g = np.array([0.5])
    e10 = math.exp(-10.0)
    # kept terms: g * (onehot - p) = 0.5 * (-1, -1, 1 - e^-10, 0)
    G = 0.5 * np.array([-1.0, -1.0, 1.0 - e10, 0.0])
    want_dh = (G @ W)[None, :]
    assert want_dh[0, 1] == pytest.approx(0.5 * (-3.0 + 4.0 * (1.0 - e10)), rel=1e-15)
    got = O.head_dh(H, W, y, g, lse, filter_eps=eps)
    assert np.allclose(got, want_dh, rtol=1e-15, atol=0.0)
    # dW[v] = G_v * H: zero for the dropped column exactly
    want_dw = G[:, None] * H[0][None, :]
    got_w = O.head_dw(H, W, y, g, lse, filter_eps=eps)
    assert np.allclose(got_w, want_dw, rtol=1e-15, atol=0.0)
    assert np.all(got_w[3] == 0.0)
    # without the filter every column contributes
    G0 = 0.5 * np.array([-1.0, -1.0, 1.0 - e10, -e10])
    assert np.allclose(O.head_dh(H, W, y, g, lse), (G0 @ W)[None, :], rtol=1e-15, atol=0.0)
    assert np.allclose(O.head_dw(H, W, y, g, lse), G0[:, None] * H[0][None, :], rtol=1e-15,
                       atol=0.0)


def test_filter_just_above_p_drops_it():
    """eps one ulp above p = 1 drops the two non-target columns with p = 1 as
    well: only the target term g * (1 - e^-10) * W_y is left."""
    H, W, y, lse = _filter_boundary_case()
    g = np.array([0.5])
    e10 = math.exp(-10.0)
    eps = float(np.nextafter(1.0, 2.0))
    want = 0.5 * (1.0 - e10) * W[2]
    assert np.allclose(O.head_dh(H, W, y, g, lse, filter_eps=eps)[0], want, rtol=1e-15, atol=0)
    got_w = O.head_dw(H, W, y, g, lse, filter_eps=eps)
    assert np.all(got_w[[0, 1, 3]] == 0.0)
    assert got_w[2] == pytest.approx(0.5 * (1.0 - e10) * H[0], rel=1e-15)


# --------------------------------------------------------------------------
# 4-bit affine head format
# --------------------------------------------------------------------------

def test_bf16_bit_patterns():
    bits = np.array([0x3F80, 0x4000, 0xBF80, 0x3E00, 0x0000, 0x4049], dtype=np.uint16)
    want = [1.0, 2.0, -1.0, 0.125, 0.0, 3.140625]
    assert O.bf16_bits_to_f64(bits).tolist() == want


def test_dequant_nibble_order_and_affine():
    # one row, D = 64: word k holds elements 8k..8k+7, low nibble first
    words = np.zeros((1, 8), dtype=np.uint32)
    words[0, 0] = 0x76543210
    words[0, 1] = 0xFEDCBA98
    words[0, 7] = 0x0000000F
    one = np.array([[0x3F80]], dtype=np.uint16)     # scale 1.0
    zero = np.array([[0x0000]], dtype=np.uint16)    # bias 0.0
    w = O.dequant_affine_q4(words, one, zero)
    assert w.shape == (1, 64)
    assert w[0, :16].tolist() == list(range(16))
    assert w[0, 56] == 15.0 and w[0, 57:].tolist() == [0.0] * 7
    half = np.array([[0x3F00]], dtype=np.uint16)    # 0.5
    neg2 = np.array([[0xC000]], dtype=np.uint16)    # -2.0
    w2 = O.dequant_affine_q4(words, half, neg2)
    assert np.array_equal(w2, w * 0.5 - 2.0)


def test_dequant_groups_select_their_own_scale():
    V, D = 3, 128
    words = np.full((V, D // 8), 0x11111111, dtype=np.uint32)   # every q = 1
    sc = np.array([[0x3F80, 0x4000]] * V, dtype=np.uint16)      # 1.0 | 2.0
    bi = np.array([[0x0000, 0x3F80]] * V, dtype=np.uint16)      # 0.0 | 1.0
    w = O.dequant_affine_q4(words, sc, bi)
    assert np.all(w[:, :64] == 1.0) and np.all(w[:, 64:] == 3.0)


# --------------------------------------------------------------------------
# objective siblings (SimPO, ORPO + margin)
# --------------------------------------------------------------------------

def test_simpo_equal_means_closed_form():
    _, _, y, L = tiny_case(P=4, Rc=3, Rr=5, seed=2)
    logp = np.full(len(y), -1.7)
    for gamma in (0.0, 0.5, 2.0):
        o = O.pref_loss_from_logps(logp, y, L, "simpo", 0.1, beta=2.5, gamma=gamma)
        assert o.loss == pytest.approx(math.log1p(math.exp(gamma)), rel=1e-14)
        h = O.pref_loss_from_logps(logp, y, L, "orpo_margin", 0.3, beta=2.5, gamma=gamma)
        assert h.loss == pytest.approx(1.7 + 0.3 * math.log1p(math.exp(gamma)), rel=1e-14)


def test_simpo_against_published_form():
    _, _, y, L = tiny_case(P=4, Rc=3, Rr=5, seed=3)
    g = np.random.default_rng(4)
    logp = -g.random(len(y)) * 3 - 0.1
    logp[y < 0] = 0.0
    o = O.pref_loss_from_logps(logp, y, L, "simpo", 0.0, beta=2.0, gamma=0.7)
    lw = logp[L.chosen_begin:L.chosen_end][y[L.chosen_begin:L.chosen_end] >= 0].mean()
    lr = logp[L.rejected_begin:L.rejected_end][y[L.rejected_begin:L.rejected_end] >= 0].mean()
    assert o.loss == pytest.approx(-sps.log_expit(2.0 * (lw - lr) - 0.7), rel=1e-13)


@pytest.mark.parametrize("kind", ["simpo", "orpo_margin"])
@pytest.mark.parametrize("scope", ["full", "response"])
def test_sibling_coeffs_are_dL_dlogp(kind, scope):
    _, _, y, L = tiny_case(P=4, Rc=3, Rr=5, seed=1, ignore=(0, 5))
    g = np.random.default_rng(8)
    logp = -g.random(len(y)) * 4 - 0.05
    logp[y < 0] = 0.0
    args = dict(lam=0.4, beta=1.7, gamma=0.3, sft_scope=scope)
    coef = O.pref_grad_coeffs(logp, y, L, kind, **args)
    h = 1e-6
    for m in range(len(y)):
        if y[m] < 0:
            assert coef[m] == 0.0
            continue
        lp, lm = logp.copy(), logp.copy()
        lp[m] += h
        lm[m] -= h
        fd = (O.pref_loss_from_logps(lp, y, L, kind, **args).loss
              - O.pref_loss_from_logps(lm, y, L, kind, **args).loss) / (2 * h)
        assert coef[m] == pytest.approx(fd, rel=1e-6, abs=1e-9)


# --------------------------------------------------------------------------
# logit softcap
# --------------------------------------------------------------------------

@pytest.mark.parametrize("cap", [0.7, 3.0])
def test_softcap_finite_differences(cap):
    H, W, y, L = tiny_case(seed=13)
    H = H * 2.0
    dH = O.orpo_head_grad(H, W, y, L, 0.3, "full", softcap=cap)
    h = 1e-6
    fd = np.zeros_like(H)
    for m in range(H.shape[0]):
        for d in range(H.shape[1]):
            Hp, Hm = H.copy(), H.copy()
            Hp[m, d] += h
            Hm[m, d] -= h
            fd[m, d] = (O.orpo_head_loss(Hp, W, y, L, 0.3, "full", softcap=cap)
                        - O.orpo_head_loss(Hm, W, y, L, 0.3, "full", softcap=cap)) / (2 * h)
    assert np.allclose(dH, fd, rtol=1e-6, atol=1e-9)


def test_softcap_limits():
    H, W, y, L = tiny_case(P=5, Rc=7, Rr=6, D=24, V=97, seed=3)
    plain = O.head_forward(H, W, y)
    big = O.head_forward(H, W, y, softcap=1e7)
    for a, b in zip(plain, big):
        assert np.allclose(a, b, rtol=1e-9, atol=1e-9)
    cap = 0.5
    logp, lse, tgt = O.head_forward(H, W, y, softcap=cap)
    Z = cap * np.tanh((H @ W.T) / cap)
    assert np.all(np.abs(tgt) <= cap)
    assert np.allclose(lse, sps.logsumexp(Z, axis=1), rtol=1e-14, atol=1e-13)


def test_dequant_q8_byte_order_and_affine():
    words = np.zeros((1, 16), dtype=np.uint32)
    words[0, 0] = 0x03020100
    words[0, 1] = 0xFF807F10
    one = np.array([[0x3F80]], dtype=np.uint16)
    zero = np.array([[0x0000]], dtype=np.uint16)
    w = O.dequant_affine_q8(words, one, zero)
    assert w.shape == (1, 64)
    assert w[0, :8].tolist() == [0, 1, 2, 3, 16, 127, 128, 255]
    w2 = O.dequant_affine_q8(words, np.array([[0x3E80]], np.uint16), np.array([[0xBF80]], np.uint16))
    assert np.array_equal(w2, w * 0.25 - 1.0)


# --------------------------------------------------------------------------
# prefix-shared gather
# --------------------------------------------------------------------------

def test_prefix_gather_index_matches_the_stated_map():
    P, Rc, Rr = 5, 3, 4
    idx = O.prefix_gather_index(P, Rc, Rr)
    assert idx.tolist() == [0, 0, 1, 2, 3,     # prompt rows 1..4 <- 0..3
                            4, 5, 6,           # chosen[k] <- P-1+k
                            4,                 # rejected[0] <- P-1
                            8, 9, 10]          # rejected[k] <- P+Rc+k-1


def test_prefix_scatter_is_the_adjoint():
    g = np.random.default_rng(9)
    P, Rc, Rr, D = 6, 5, 7, 3
    M = P + Rc + Rr
    Hc = g.standard_normal((M, D))
    G = g.standard_normal((M, D))
    lhs = np.sum(O.prefix_gather(Hc, P, Rc, Rr) * G)
    rhs = np.sum(Hc * O.prefix_scatter(G, P, Rc, Rr))
    assert lhs == pytest.approx(rhs, rel=1e-13)
    d = O.prefix_scatter(G, P, Rc, Rr)
    assert np.allclose(d[P - 1], G[P] + G[P + Rc])   # both first response tokens
    assert np.all(d[P + Rc - 1] == 0) and np.all(d[M - 1] == 0)


def test_prefix_shared_loss_gradient_by_finite_differences():
    """The whole prefix-shared head: L(H_cat) and its gradient."""
    g = np.random.default_rng(10)
    P, Rc, Rr, D, V = 4, 3, 3, 8, 20
    M = P + Rc + Rr
    Hc = g.standard_normal((M, D))
    W = g.standard_normal((V, D)) / math.sqrt(D)
    y = g.integers(0, V, size=M).astype(np.int32)
    y[0] = -1
    L = O.Layout.contiguous(P, Rc, Rr)

    def loss(Hc_):
        return O.orpo_head_loss(O.prefix_gather(Hc_, P, Rc, Rr), W, y, L, 0.2)

    grad = O.prefix_scatter(O.orpo_head_grad(O.prefix_gather(Hc, P, Rc, Rr), W, y, L, 0.2),
                            P, Rc, Rr)
    h = 1e-6
    for r in range(M):
        for d in range(D):
            Hp, Hm = Hc.copy(), Hc.copy()
            Hp[r, d] += h
            Hm[r, d] -= h
            assert grad[r, d] == pytest.approx((loss(Hp) - loss(Hm)) / (2 * h), rel=1e-6, abs=1e-9)


# --------------------------------------------------------------------------
# trainable head: dL/dW
# --------------------------------------------------------------------------

@pytest.mark.parametrize("cap", [0.0, 2.0])
def test_head_dw_finite_differences(cap):
    H, W, y, L = tiny_case(P=3, Rc=2, Rr=3, D=6, V=10, seed=17)
    logp, lse, _ = O.head_forward(H, W, y, softcap=cap)
    g = O.orpo_grad_coeffs(logp, y, L, 0.4, "full")
    dW = O.head_dw(H, W, y, g, lse, softcap=cap)
    h = 1e-6
    for v in range(W.shape[0]):
        for d in range(W.shape[1]):
            Wp, Wm = W.copy(), W.copy()
            Wp[v, d] += h
            Wm[v, d] -= h
            fd = (O.orpo_head_loss(H, Wp, y, L, 0.4, "full", softcap=cap)
                  - O.orpo_head_loss(H, Wm, y, L, 0.4, "full", softcap=cap)) / (2 * h)
            assert dW[v, d] == pytest.approx(fd, rel=1e-6, abs=1e-9)


# --------------------------------------------------------------------------
# randomised: the whole oracle path against torch float64 autograd
# --------------------------------------------------------------------------

from hypothesis import given, settings, strategies as hst


def _autograd_reference(torch, H, W, y, L, lam, scope, cap):
    """Loss and dL/dH by autograd over materialised float64 logits (the
    objective of Training design §1 written with torch primitives)."""
    Ht = torch.tensor(H, dtype=torch.float64, requires_grad=True)
    Wt = torch.tensor(W, dtype=torch.float64)
    S = Ht @ Wt.T
    if cap > 0:
        S = cap * torch.tanh(S / cap)
    yt = torch.tensor(np.maximum(y, 0), dtype=torch.long)
    ok = torch.tensor(y >= 0)
    lp = torch.where(ok, torch.log_softmax(S, dim=1).gather(1, yt[:, None])[:, 0],
                     torch.zeros((), dtype=torch.float64))

    def seg(b, e):
        return lp[b:e][ok[b:e]].sum(), int(ok[b:e].sum())

    sP, nP = seg(L.prompt_begin, L.prompt_end)
    sC, nC = seg(L.chosen_begin, L.chosen_end)
    sR, nR = seg(L.rejected_begin, L.rejected_end)
    lw, lr = sC / nC, sR / nR
    nll = -(sP + sC) / (nP + nC) if scope == "full" else -lw
    z = (lw - lr) - (torch.log(-torch.expm1(lw)) - torch.log(-torch.expm1(lr)))
    loss = nll - lam * torch.nn.functional.logsigmoid(z)
    loss.backward()
    return loss.item(), Ht.grad.numpy()


@settings(max_examples=60, deadline=None)
@given(P=hst.integers(1, 6), Rc=hst.integers(1, 6), Rr=hst.integers(1, 6),
       D=hst.integers(1, 12), V=hst.integers(2, 40), lam=hst.floats(0.0, 2.0),
       scope=hst.sampled_from(["full", "response"]), cap=hst.sampled_from([0.0, 3.0]),
       order=hst.permutations([0, 1, 2]), seed=hst.integers(0, 2**31 - 1),
       n_ignore=hst.integers(0, 3))
def test_randomised_against_torch_autograd(P, Rc, Rr, D, V, lam, scope, cap, order, seed,
                                           n_ignore):
    """Random sizes, segment order, ignored rows, lambda, scope and softcap:
    the oracle's loss and dH equal torch autograd through materialised
    logits."""
    torch = pytest.importorskip("torch")
    g = np.random.default_rng(seed)
    sizes = [P, Rc, Rr]
    starts, b = [0, 0, 0], 0
    for k in order:                     # segments laid out in a random order
        starts[k] = b
        b += sizes[k]
    M = b
    L = O.Layout(starts[0], starts[0] + P, starts[1], starts[1] + Rc, starts[2], starts[2] + Rr)
    H = g.standard_normal((M, D))
    W = g.standard_normal((V, D)) / math.sqrt(D)
    y = g.integers(0, V, size=M).astype(np.int32)
    keep = {L.chosen_begin, L.rejected_begin}   # one labelled row in each response
    for r in g.choice(M, size=min(n_ignore, M), replace=False):
        if int(r) not in keep:
            y[r] = -1
    want_loss, want_dH = _autograd_reference(torch, H, W, y, L, lam, scope, cap)
    logp = O.head_forward(H, W, y, softcap=cap)[0]
    o = O.orpo_loss_from_logps(logp, y, L, lam, scope)
    assert o.loss == pytest.approx(want_loss, rel=1e-11, abs=1e-12)
    dH = O.orpo_head_grad(H, W, y, L, lam, scope, softcap=cap)
    assert np.allclose(dH, want_dH, rtol=1e-8, atol=1e-12)
