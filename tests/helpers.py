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
    if wl.dtype == "bf16":
        H = torch.from_numpy(wl.H_bits.view(np.int16)).to(device).view(torch.bfloat16)
    else:
        H = torch.from_numpy(wl.H).to(device)
    if wl.wformat == "q4g64":
        head = cce.Head(
            w=torch.from_numpy(wl.q_packed.view(np.int32)).to(device), V=wl.V, D=wl.D,
            fmt=cce.CCE_W_AFFINE_Q4_G64,
            scales=torch.from_numpy(wl.q_scales.view(np.int16)).to(device).view(torch.bfloat16),
            biases=torch.from_numpy(wl.q_biases.view(np.int16)).to(device).view(torch.bfloat16))
    elif wl.dtype == "bf16":
        head = cce.Head(w=torch.from_numpy(wl.W_bits.view(np.int16)).to(device).view(torch.bfloat16),
                        V=wl.V, D=wl.D)
    else:
        head = cce.Head(w=torch.from_numpy(wl.W).to(device), V=wl.V, D=wl.D)
    labels = torch.from_numpy(wl.labels).to(device)
    return H, head, labels


def oracle_W(wl: S.Workload) -> np.ndarray:
    """The head's weights exactly as the method defines them (float64)."""
    if wl.wformat == "q4g64":
        return O.dequant_affine_q4(wl.q_packed, wl.q_scales, wl.q_biases)
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
