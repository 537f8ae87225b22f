"""The fp16 path of 4- and 8-bit heads: values fp16 cannot hold are
reported, not turned silently into inf / NaN or flushed; a flat softmax over
a 128k vocabulary (probabilities near 5e-6, subnormal in plain fp16) keeps
the oracle's tolerances through the 2^14-scaled coefficient tile."""

import numpy as np
import pytest
import torch

from lm_head_cross_flash_b200 import cce
from lm_head_cross_flash_b200 import synthetic as S
from oracle import flash_cce as O

from helpers import TOL_DH, TOL_LOGP, oracle_W, rel_fro, upload

pytestmark = pytest.mark.gpu

FP16_RANGE = 9


def _pass_status(H, head, labels, M, V, qmode):
    hd = cce.h_dtype(H)
    ws = cce.alloc_workspace(M, hd, head)
    f = dict(device="cuda", dtype=torch.float32)
    logp, lse = torch.empty(M, **f), torch.empty(M, **f)
    cce.cce_set_quant_staging(qmode)
    try:
        cce.cce_forward(H, head, labels, logp, lse, None, None, ws)
        torch.cuda.synchronize()
        st_f = cce.cce_device_status(ws)
        coeff = torch.full((M,), 1.0 / M, **f)
        dH = torch.empty(M, head.D, **f)
        cce.cce_backward_dh(H, head, labels, lse, coeff, 0.0, None, dH, None, ws)
        torch.cuda.synchronize()
        st_b = cce.cce_device_status(ws)
    finally:
        cce.cce_set_quant_staging(0)
    return st_f, st_b


@pytest.mark.parametrize("qmode", [1, 2])
@pytest.mark.parametrize("wformat", ["q4g64", "q8g64"])
def test_hidden_value_beyond_fp16_is_reported(qmode, wformat):
    wl = S.make_custom(4, M_split=(100, 150, 131), D=128, V=3000, wformat=wformat)
    H, head, labels = upload(wl)
    assert _pass_status(H, head, labels, wl.M, wl.V, qmode) == (0, 0)
    H2 = H.clone()
    H2[37, 5] = 1.0e5          # finite in bf16, beyond the largest fp16
    assert _pass_status(H2, head, labels, wl.M, wl.V, qmode) == (FP16_RANGE, FP16_RANGE)


@pytest.mark.parametrize("which", ["scales", "biases"])
def test_scale_or_bias_outside_fp16_normal_range_is_reported(which):
    wl = S.make_custom(4, M_split=(100, 150, 131), D=128, V=3000)
    H, head, labels = upload(wl)
    t = getattr(head, which).clone()
    t[17, 1] = 1.0e-6          # subnormal in fp16
    h2 = cce.Head(w=head.w, V=head.V, D=head.D, fmt=head.fmt,
                  scales=t if which == "scales" else head.scales,
                  biases=t if which == "biases" else head.biases)
    for qmode in (1, 2):
        assert _pass_status(H, h2, labels, wl.M, wl.V, qmode) == (FP16_RANGE, FP16_RANGE)
    t[17, 1] = 0.0             # zero is exact
    h3 = cce.Head(w=head.w, V=head.V, D=head.D, fmt=head.fmt,
                  scales=t if which == "scales" else head.scales,
                  biases=t if which == "biases" else head.biases)
    assert _pass_status(H, h3, labels, wl.M, wl.V, 1) == (0, 0)


@pytest.mark.parametrize("qmode,split", [(1, (20, 22, 22)), (2, (100, 150, 134))])
def test_flat_softmax_over_128k_vocabulary(qmode, split):
    """Flat rows (H ~ N(0, 1), no peak) over the long-context vocabulary:
    every probability is about 5e-6.  logp, lse and dH match the oracle."""
    wl = S.make_custom(4, M_split=split, D=128, V=128256, alpha=0.0)
    H, head, labels = upload(wl)
    hd = cce.h_dtype(H)
    ws = cce.alloc_workspace(wl.M, hd, head)
    f = dict(device="cuda", dtype=torch.float32)
    logp, lse = torch.empty(wl.M, **f), torch.empty(wl.M, **f)
    g = S.random_cotangent(wl)
    coeff = torch.from_numpy(g).cuda()
    dH = torch.empty(wl.M, wl.D, **f)
    cce.cce_set_quant_staging(qmode)
    try:
        cce.cce_forward(H, head, labels, logp, lse, None, None, ws)
        cce.cce_backward_dh(H, head, labels, lse, coeff, 0.0, None, dH, None, ws)
        torch.cuda.synchronize()
    finally:
        cce.cce_set_quant_staging(0)
    assert cce.cce_device_status(ws) == 0
    W = oracle_W(wl)
    ologp, olse, _ = O.head_forward(wl.H, W, wl.labels)
    assert np.max(np.exp(-olse)) < 1e-5          # the softmax is flat
    assert np.max(np.abs(logp.cpu().numpy() - ologp)) <= TOL_LOGP
    assert np.max(np.abs(lse.cpu().numpy() - olse)) <= TOL_LOGP
    want = O.head_dh(wl.H, W, wl.labels, g, olse)
    err = rel_fro(dH.cpu().numpy(), want)
    print(f"qmode {qmode}: flat 128k softmax, dH rel err {err:.2e}")
    assert err <= TOL_DH
