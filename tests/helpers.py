"""Shared helpers of the GPU tests: upload a workload, run the head, and
compute the oracle's answers on the same inputs."""

from __future__ import annotations

import numpy as np
import torch

from lm_head_cross_flash_b200 import cce
from lm_head_cross_flash_b200 import synthetic as S
from oracle import flash_cce as O

# Tolerances fixed by the benchmark spec of the head (per-token logp and lse
# absolute, scalar loss relative, dH relative Frobenius).
TOL_LOGP = 2e-3
TOL_LOSS = 1e-3
TOL_DH = 1e-2


def upload(wl: S.Workload, device="cuda"):
    """Device tensors (H, head, labels) of a workload."""
    return cce.upload_workload(wl, device)


def oracle_W(wl: S.Workload) -> np.ndarray:
    """The head's weights exactly as the method defines them (float64)."""
    if wl.wformat == "q4g64":
        return O.dequant_affine_q4(wl.q_packed, wl.q_scales, wl.q_biases)
    if wl.wformat == "q8g64":
        return O.dequant_affine_q8(wl.q_packed, wl.q_scales, wl.q_biases)
    return wl.W.astype(np.float64)


def oracle_layout(wl: S.Workload) -> O.Layout:
    return O.Layout(*wl.layout_tuple)


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def run_pass(wl: S.Workload, device="cuda", ws_bytes=None, block_skip=None):
    H, head, labels = upload(wl, device)
    hd = cce.h_dtype(H)
    buf = cce.HeadBuffers.alloc(wl.M, wl.D, wl.V, hd, head, device, ws_bytes)
    bs = wl.block_skip if block_skip is None else block_skip
    cce.orpo_head_pass(H, head, labels, wl.layout_tuple, wl.lam, wl.scope, wl.filter_eps,
                       bs, buf)
    torch.cuda.synchronize()
    st = cce.cce_device_status(buf.ws)
    return H, head, labels, buf, st
