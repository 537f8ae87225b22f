"""GPU parity of the transposed small-M forwards of 4/8-bit heads (the
logits computed as S^T = W_t H^T with the dequantised head tile in tensor
memory as the MMA's A operand; the narrow form up to 128 head rows, the wide
form of 128-row units up to 256) against the float64 oracle and against the
tiled GEMM forward with in-kernel dequantisation (forward mode 1).

Shapes cover 3 to 128 head rows (N = 16, 48, 64, 80, 128: one or two
accumulator buffers, one to four 32-column chunks), D from 512 to 2048,
vocabularies from 31 rows (one partial block) to more 256-row blocks than
SMs (several blocks per CTA, both buffer parities) with ragged tails, the
softcap, and unlabelled rows."""

import numpy as np
import pytest
import torch

from lm_head_cross_flash_b200 import cce
from lm_head_cross_flash_b200 import synthetic as S
from oracle import flash_cce as O

from helpers import TOL_DH, TOL_LOGP, oracle_W, rel_fro, upload

pytestmark = pytest.mark.gpu

# Both forms take the same fp16 weights and H and accumulate in fp32 over K
# in the same order of 16-wide steps, then reduce the block's (max, sum)
# in another order: the block maxima agree to the last bits of the logits,
# lse and logp to the fp32 rounding of the exp-sums.
TOL_VS_GEMM = 2e-5


def _forward(mode, H, head, labels, M, V):
    """mode: 0 choose, 1 the tiled GEMM, 2 the wide transposed form."""
    f = dict(device="cuda", dtype=torch.float32)
    cce.cce_set_forward_mode(mode)
    try:
        ws = cce.alloc_workspace(M, cce.h_dtype(H), head)
        plan = cce.cce_query_plan(M, cce.h_dtype(H), head, ws.numel())
        logp, lse = torch.empty(M, **f), torch.empty(M, **f)
        tgt = torch.full((M,), float("nan"), **f)
        bm = torch.empty(cce.blockmax_cols(V), M, **f)
        cce.cce_profile_enable(True)
        cce.cce_forward(H, head, labels, logp, lse, tgt, bm, ws)
        torch.cuda.synchronize()
        prof = cce.cce_profile_read()
    finally:
        cce.cce_profile_enable(False)
        cce.cce_set_forward_mode(0)
    assert cce.cce_device_status(ws) == 0
    return plan, prof, logp.cpu().numpy(), lse.cpu().numpy(), tgt.cpu().numpy(), bm.cpu().numpy()


CASES = [
    # (wformat, (P, Rc, Rr), D, V, softcap)
    ("q4g64", (1, 1, 1), 512, 31, 0.0),            # M = 3: N = 16, one partial block
    ("q4g64", (5, 5, 6), 512, 257, 0.0),           # a last block of one row
    ("q4g64", (10, 10, 12), 1024, 4097, 0.0),
    ("q8g64", (10, 10, 13), 512, 3000, 0.0),       # N = 48: two chunks, the second half used
    ("q4g64", (20, 20, 24), 2048, 20000, 0.0),     # N = 64: two accumulator buffers
    ("q4g64", (20, 20, 25), 512, 5000, 0.0),       # N = 80: one buffer
    ("q8g64", (40, 40, 48), 1024, 9000, 0.0),      # N = 128
    ("q4g64", (30, 30, 40), 512, 3001, 30.0),      # softcap
    ("q4g64", (20, 20, 24), 512, 148 * 256 * 2 + 17, 0.0),   # 3 blocks per CTA
    ("q8g64", (30, 30, 36), 512, 148 * 256 * 3, 0.0),        # N = 96, one buffer, 3 per CTA
]


WIDE_CASES = [
    ("q4g64", (40, 45, 44), 512, 4097, 0.0),       # M = 129: N = 144, five chunks
    ("q8g64", (50, 70, 80), 1024, 3001, 0.0),      # M = 200: N = 208
    ("q4g64", (60, 90, 90), 2048, 20000, 0.0),     # M = 240: N = 240, eight chunks
    ("q4g64", (40, 80, 80), 512, 257, 30.0),       # softcap, a last block of one row
    ("q8g64", (50, 80, 80), 512, 148 * 256 * 2 + 17, 0.0),  # 3 blocks per CTA
]

SMALL_IN_WIDE = [
    ("q4g64", (1, 1, 1), 512, 31, 0.0),            # mode 2 from 3 rows: N = 16
    ("q4g64", (20, 20, 24), 1024, 5000, 0.0),      # N = 64
    ("q8g64", (40, 40, 48), 512, 9000, 0.0),       # N = 128
    ("q4g64", (60, 98, 98), 2048, 20000, 0.0),     # M = 256: N = 256, eight full chunks
]


@pytest.mark.parametrize("mode,form,case", [(0, 1, c) for c in CASES] +
                         [(0, 2, c) for c in WIDE_CASES] + [(2, 2, c) for c in SMALL_IN_WIDE])
def test_q_small_m_forward_matches_oracle_and_gemm(mode, form, case):
    wformat, split, D, V, cap = case
    wl = S.make_custom(4, M_split=split, D=D, V=V, wformat=wformat)
    H, head, labels = upload(wl)
    head.softcap = cap
    M = wl.M
    plan, prof, logp, lse, tgt, bm = _forward(mode, H, head, labels, M, V)
    assert plan["fwd_q_small_m"] == form and plan["fwd_staged"] == 0, plan
    assert prof.get("fwd_q_small_m", (0.0, 0))[1] == 1, prof
    assert prof.get("fwd_lse_gemm", (0.0, 0))[1] == 0, prof
    plan1, prof1, logp1, lse1, tgt1, bm1 = _forward(1, H, head, labels, M, V)
    assert plan1["fwd_q_small_m"] == 0
    assert prof1.get("fwd_q_small_m", (0.0, 0))[1] == 0

    W = oracle_W(wl)
    ologp, olse, otgt = O.head_forward(wl.H, W, wl.labels, softcap=cap)
    lab = wl.labels >= 0
    print(f"{wformat} M={M} D={D} V={V}: |dlse| {np.max(np.abs(lse - olse)):.2e}, "
          f"vs GEMM {np.max(np.abs(lse - lse1)):.2e}")
    assert np.max(np.abs(lse - olse)) <= TOL_LOGP
    assert np.max(np.abs(logp - ologp)) <= TOL_LOGP
    assert np.max(np.abs(tgt[lab] - otgt[lab])) <= TOL_LOGP
    assert np.all(logp[~lab] == 0.0)
    # against the GEMM form: the same logits, reduced in another order
    assert np.max(np.abs(lse - lse1)) <= TOL_VS_GEMM * max(1.0, np.max(np.abs(lse1)))
    assert np.max(np.abs(tgt[lab] - tgt1[lab])) <= TOL_VS_GEMM * max(1.0, np.max(np.abs(tgt1[lab])))
    assert np.max(np.abs(bm - bm1)) <= TOL_VS_GEMM * max(1.0, np.max(np.abs(bm1)))
    # every block maximum is the maximum of that block's logits
    Z = O.softcap_logits(np.asarray(wl.H, np.float64) @ W.T, cap)
    cols = bm.shape[0]
    want_bm = np.stack([Z[:, 256 * b:min(V, 256 * b + 256)].max(axis=1) for b in range(cols)])
    assert np.max(np.abs(bm - want_bm)) <= TOL_LOGP


def test_q_small_m_not_taken_outside_its_range():
    """257 rows, D not a multiple of 512, or forward mode 1: the GEMM form."""
    for split, D in (((40, 110, 107), 512), ((20, 20, 24), 256)):
        wl = S.make_custom(4, M_split=split, D=D, V=3000, wformat="q4g64")
        H, head, labels = upload(wl)
        plan = cce.cce_query_plan(wl.M, cce.h_dtype(H), head, 1 << 34)
        assert plan["fwd_q_small_m"] == 0, (split, D)
    wl = S.make_custom(4, M_split=(20, 20, 24), D=512, V=3000, wformat="q4g64")
    H, head, labels = upload(wl)
    assert cce.cce_query_plan(wl.M, cce.h_dtype(H), head, 1 << 34)["fwd_q_small_m"] == 1
    cce.cce_set_forward_mode(1)
    try:
        assert cce.cce_query_plan(wl.M, cce.h_dtype(H), head, 1 << 34)["fwd_q_small_m"] == 0
    finally:
        cce.cce_set_forward_mode(0)


@pytest.mark.parametrize("wformat", ["q4g64", "q8g64"])
def test_q_small_m_through_the_real_pass(wformat):
    """The whole head pass (forward with the transposed kernel, loss,
    cotangent, dH) against the oracle; the same pass captured in a CUDA
    graph and replayed gives the direct call's bits."""
    wl = S.make_custom(4, M_split=(12, 24, 28), D=1024, V=9000, wformat=wformat)
    H, head, labels = upload(wl)
    hd = cce.h_dtype(H)
    direct = cce.HeadBuffers.alloc(wl.M, wl.D, wl.V, hd, head)
    graphed = cce.HeadBuffers.alloc(wl.M, wl.D, wl.V, hd, head)
    args = (wl.layout_tuple, wl.lam, wl.scope, wl.filter_eps, wl.block_skip)
    cce.cce_profile_enable(True)
    try:
        cce.orpo_head_pass(H, head, labels, *args, direct)
        torch.cuda.synchronize()
        prof = cce.cce_profile_read()
    finally:
        cce.cce_profile_enable(False)
    assert prof.get("fwd_q_small_m", (0.0, 0))[1] == 1, prof
    g = cce.HeadPassGraph(H, head, labels, *args, graphed)
    g.replay()
    torch.cuda.synchronize()
    assert cce.cce_device_status(direct.ws) == 0
    assert cce.cce_device_status(graphed.ws) == 0
    W = oracle_W(wl)
    L = O.Layout(*wl.layout_tuple)
    ologp, olse, _ = O.head_forward(wl.H, W, wl.labels)
    o = O.orpo_loss_from_logps(ologp, wl.labels, L, wl.lam, wl.scope)
    gc = O.orpo_grad_coeffs(ologp, wl.labels, L, wl.lam, wl.scope)
    odh = O.head_dh(wl.H, W, wl.labels, gc, olse)
    out8 = direct.out8.cpu().numpy()
    assert abs(out8[0] - o.loss) <= 1e-3 * abs(o.loss)
    assert rel_fro(direct.dH.cpu().numpy(), odh) <= TOL_DH
    for name in ("logp", "lse", "out8", "coeff", "dH"):
        assert np.array_equal(getattr(graphed, name).cpu().numpy(),
                              getattr(direct, name).cpu().numpy()), name
