"""ctypes binding of ``libcce.so`` (declared in ``include/cce.h``).

Argument marshalling only: every step of the head runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (used for device memory and
streams); the functions keep the C names and raise ``CCEError`` for a
synchronous error status.  The library is loaded on first use; if it is
missing the call raises instead of falling back to anything else.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcce.so")

CCE_F32, CCE_BF16 = 0, 1
CCE_W_DENSE, CCE_W_AFFINE_Q4_G64, CCE_W_AFFINE_Q8_G64 = 0, 1, 2
SCOPE = {"full": 0, "response": 1}
VOCAB_BLOCK = 256

STATUS_NAMES = {
    0: "CCE_OK", 1: "CCE_ERR_INVALID_ARGUMENT", 2: "CCE_ERR_UNSUPPORTED",
    3: "CCE_ERR_CUDA", 4: "CCE_ERR_WORKSPACE_TOO_SMALL",
    5: "CCE_ERR_LABEL_OUT_OF_RANGE", 6: "CCE_ERR_DEVICE_TIMEOUT",
    7: "CCE_ERR_EMPTY_SEGMENT", 8: "CCE_ERR_DOMAIN", 9: "CCE_ERR_FP16_RANGE",
}


class CCEError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")
        self.status = status


class _Head(ctypes.Structure):
    _fields_ = [("format", ctypes.c_int), ("dtype", ctypes.c_int),
                ("V", ctypes.c_int64), ("D", ctypes.c_int64),
                ("w", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("biases", ctypes.c_void_p), ("softcap", ctypes.c_float)]


class _Objective(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("lam", ctypes.c_double), ("beta", ctypes.c_double),
                ("gamma", ctypes.c_double), ("sft_scope", ctypes.c_int)]


OBJECTIVES = {"orpo": 0, "simpo": 1, "orpo_margin": 2}


class _Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "prompt_begin", "prompt_end", "chosen_begin", "chosen_end",
        "rejected_begin", "rejected_end")]


class _Plan(ctypes.Structure):
    _fields_ = [("fwd_ok", ctypes.c_int), ("bwd_ok", ctypes.c_int),
                ("fwd_chunk", ctypes.c_int64), ("bwd_chunk", ctypes.c_int64),
                ("bwd_ksplit", ctypes.c_int),
                ("fwd_staged", ctypes.c_int), ("bwd_staged", ctypes.c_int),
                ("fwd_cta_pairs", ctypes.c_int), ("bwd_cta_pairs", ctypes.c_int),
                ("bwd_fused", ctypes.c_int), ("bwd_fused_groups", ctypes.c_int),
                ("bwd_fused_members", ctypes.c_int), ("bwd_fused_buffers", ctypes.c_int),
                ("bwd_sliced", ctypes.c_int), ("bwd_sliced_clusters", ctypes.c_int),
                ("bwd_sliced_ctas", ctypes.c_int), ("fwd_q_small_m", ctypes.c_int)]


_lib = None

_SIGS = {
    "cce_blockmax_cols": (ctypes.c_int64, [ctypes.c_int64]),
    "cce_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int, ctypes.POINTER(_Head)]),
    "cce_workspace_min_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int, ctypes.POINTER(_Head)]),
    "cce_forward": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.POINTER(_Head),
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "orpo_loss_from_logps": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                            ctypes.POINTER(_Layout), ctypes.c_double, ctypes.c_int,
                                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                            ctypes.c_void_p]),
    "orpo_grad_coeffs": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                        ctypes.POINTER(_Layout), ctypes.c_double, ctypes.c_int,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                        ctypes.c_void_p]),
    "orpo_partial_sums": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                         ctypes.POINTER(_Layout), ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_size_t, ctypes.c_void_p]),
    "orpo_from_sums": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                      ctypes.POINTER(_Layout), ctypes.c_double, ctypes.c_int,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_size_t, ctypes.c_void_p]),
    "cce_backward_dh": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.POINTER(_Head),
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_size_t, ctypes.c_void_p]),
    "cce_backward_dh_dw": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                          ctypes.POINTER(_Head), ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "cce_device_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "cce_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "cce_set_wait_limit_ns": (None, [ctypes.c_uint64]),
    "cce_set_cta_pairs": (None, [ctypes.c_int]),
    "cce_set_quant_staging": (None, [ctypes.c_int]),
    "cce_set_backward_mode": (None, [ctypes.c_int]),
    "cce_set_forward_mode": (None, [ctypes.c_int]),
    "cce_query_fused_schedule": (ctypes.c_int64, [ctypes.c_int64, ctypes.c_int,
                                                  ctypes.POINTER(_Head), ctypes.c_void_p,
                                                  ctypes.c_int64]),
    "cce_query_plan": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int, ctypes.POINTER(_Head),
                                      ctypes.c_size_t, ctypes.POINTER(_Plan)]),
    "cce_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "pref_loss_from_logps": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                            ctypes.POINTER(_Layout), ctypes.POINTER(_Objective),
                                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                            ctypes.c_void_p]),
    "pref_grad_coeffs": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                        ctypes.POINTER(_Layout), ctypes.POINTER(_Objective),
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                        ctypes.c_void_p]),
    "cce_prefix_gather": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                         ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_void_p, ctypes.c_void_p]),
    "cce_prefix_scatter": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                          ctypes.c_void_p]),
    "cce_profile_enable": (None, [ctypes.c_int]),
    "cce_profile_read": (ctypes.c_int, [ctypes.POINTER(ctypes.c_double),
                                        ctypes.POINTER(ctypes.c_longlong), ctypes.c_int]),
    "cce_profile_kind_name": (ctypes.c_char_p, [ctypes.c_int]),
    "cce_forward_noalloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(_Head),
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_void_p]),
}

NOALLOC_SCRATCH_BYTES = 32 << 20


def cce_forward_noalloc(H, head: "Head", labels, logp, lse, tgt_logit=None, blockmax=None,
                        status=None, stream=None):
    """Forward for callers that cannot allocate device memory: the library's
    fixed scratch array (NOALLOC_SCRATCH_BYTES) replaces the workspace.
    Calls share that array, so calls that overlap on the GPU race."""
    st = lib().cce_forward_noalloc(_p(H), H.shape[0], ctypes.byref(head.c()), _p(labels),
                                   _p(logp), _p(lse), _p(tgt_logit), _p(blockmax), _p(status),
                                   _stream(stream))
    _check(st, "cce_forward_noalloc")

PROFILE_KINDS = 32


def cce_profile_enable(on: bool):
    lib().cce_profile_enable(1 if on else 0)


def cce_profile_read() -> dict:
    """{kind name: (total ms, launches)} of the kernels recorded since
    ``cce_profile_enable(True)``; clears the records."""
    ms = (ctypes.c_double * PROFILE_KINDS)()
    n = (ctypes.c_longlong * PROFILE_KINDS)()
    k = lib().cce_profile_read(ms, n, PROFILE_KINDS)
    return {lib().cce_profile_kind_name(i).decode(): (ms[i], n[i])
            for i in range(min(k, PROFILE_KINDS))}


def lib():
    """Load ``libcce.so`` once; raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m lm_head_cross_flash_b200.build` (no fallback exists)")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(st: int, where: str):
    if st != 0:
        raise CCEError(st, where)


@dataclass
class Head:
    """The frozen head: dense ``w`` [V, D] (f32 or bf16), or a 4-bit affine
    head (``w`` uint32 [V, D/8] stored as int32, ``scales``/``biases`` bf16
    [V, D/64])."""

    w: torch.Tensor
    V: int
    D: int
    fmt: int = CCE_W_DENSE
    scales: torch.Tensor | None = None
    biases: torch.Tensor | None = None
    softcap: float = 0.0

    @property
    def dtype(self) -> int:
        if self.fmt in (CCE_W_AFFINE_Q4_G64, CCE_W_AFFINE_Q8_G64):
            return CCE_BF16
        return CCE_F32 if self.w.dtype == torch.float32 else CCE_BF16

    def c(self) -> _Head:
        return _Head(self.fmt, self.dtype, self.V, self.D, self.w.data_ptr(),
                     None if self.scales is None else self.scales.data_ptr(),
                     None if self.biases is None else self.biases.data_ptr(),
                     float(self.softcap))


def h_dtype(H: torch.Tensor) -> int:
    return CCE_F32 if H.dtype == torch.float32 else CCE_BF16


def blockmax_cols(V: int) -> int:
    return int(lib().cce_blockmax_cols(V))


def workspace_bytes(M: int, H_dtype: int, head: Head) -> int:
    return int(lib().cce_workspace_bytes(M, H_dtype, ctypes.byref(head.c())))


def workspace_min_bytes(M: int, H_dtype: int, head: Head) -> int:
    return int(lib().cce_workspace_min_bytes(M, H_dtype, ctypes.byref(head.c())))


def alloc_workspace(M: int, H_dtype: int, head: Head, device="cuda", nbytes=None):
    """Caller-side workspace (torch allocation) with a zeroed status word."""
    n = workspace_bytes(M, H_dtype, head) if nbytes is None else nbytes
    if n == 0:
        raise CCEError(1, "cce_workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def cce_forward(H, head: Head, labels, logp, lse, tgt_logit=None, blockmax=None,
                ws=None, stream=None):
    st = lib().cce_forward(_p(H), h_dtype(H), H.shape[0], ctypes.byref(head.c()),
                           _p(labels), _p(logp), _p(lse), _p(tgt_logit), _p(blockmax),
                           _p(ws), ws.numel(), _stream(stream))
    _check(st, "cce_forward")


def _layout(layout):
    return _Layout(*[int(x) for x in layout])


def orpo_loss_from_logps(logp, labels, layout, lam, sft_scope, out8, ws, stream=None):
    st = lib().orpo_loss_from_logps(_p(logp), _p(labels), logp.shape[0],
                                    ctypes.byref(_layout(layout)), float(lam),
                                    SCOPE.get(sft_scope, sft_scope), _p(out8), _p(ws),
                                    ws.numel(), _stream(stream))
    _check(st, "orpo_loss_from_logps")


def orpo_grad_coeffs(logp, labels, layout, lam, sft_scope, coeff, ws, stream=None):
    st = lib().orpo_grad_coeffs(_p(logp), _p(labels), logp.shape[0],
                                ctypes.byref(_layout(layout)), float(lam),
                                SCOPE.get(sft_scope, sft_scope), _p(coeff), _p(ws),
                                ws.numel(), _stream(stream))
    _check(st, "orpo_grad_coeffs")


def orpo_partial_sums(logp, labels, layout, sums6, ws, stream=None):
    """This shard's segment sums and counts (fp64 [6] on the device)."""
    st = lib().orpo_partial_sums(_p(logp), _p(labels), logp.shape[0],
                                 ctypes.byref(_layout(layout)), _p(sums6), _p(ws), ws.numel(),
                                 _stream(stream))
    _check(st, "orpo_partial_sums")


def orpo_from_sums(sums6, labels, layout, lam, sft_scope, out8, coeff, ws, stream=None):
    """Loss and this shard's dL/dlogp from the all-reduced segment sums."""
    st = lib().orpo_from_sums(_p(sums6), _p(labels), labels.shape[0],
                              ctypes.byref(_layout(layout)), float(lam),
                              SCOPE.get(sft_scope, sft_scope), _p(out8), _p(coeff), _p(ws),
                              ws.numel(), _stream(stream))
    _check(st, "orpo_from_sums")


def cce_backward_dh(H, head: Head, labels, lse, coeff, filter_eps, blockmax, dH,
                    skip_stats=None, ws=None, stream=None):
    st = lib().cce_backward_dh(_p(H), h_dtype(H), H.shape[0], ctypes.byref(head.c()),
                               _p(labels), _p(lse), _p(coeff), float(filter_eps),
                               _p(blockmax), _p(dH), _p(skip_stats), _p(ws), ws.numel(),
                               _stream(stream))
    _check(st, "cce_backward_dh")


def cce_device_status(ws, stream=None) -> int:
    return int(lib().cce_device_status(_p(ws), _stream(stream)))


def cce_set_wait_limit_ns(ns: int):
    lib().cce_set_wait_limit_ns(int(ns))


def cce_selftest_wait_timeout(ws, stream=None):
    _check(lib().cce_selftest_wait_timeout(_p(ws), ws.numel(), _stream(stream)),
           "cce_selftest_wait_timeout")


# ----------------------------------------------------------------------------
# one pass of the whole head
# ----------------------------------------------------------------------------

@dataclass
class HeadBuffers:
    """Device buffers of one head pass (outputs and the workspace)."""

    logp: torch.Tensor
    lse: torch.Tensor
    tgt: torch.Tensor
    blockmax: torch.Tensor
    out8: torch.Tensor
    coeff: torch.Tensor
    dH: torch.Tensor
    skip: torch.Tensor
    ws: torch.Tensor

    @staticmethod
    def alloc(M: int, D: int, V: int, H_dtype: int, head: Head, device="cuda",
              ws_bytes=None):
        f = dict(device=device, dtype=torch.float32)
        return HeadBuffers(
            logp=torch.empty(M, **f), lse=torch.empty(M, **f), tgt=torch.zeros(M, **f),
            blockmax=torch.empty(blockmax_cols(V), M, **f),
            out8=torch.empty(8, device=device, dtype=torch.float64),
            coeff=torch.empty(M, **f), dH=torch.empty(M, D, **f),
            skip=torch.zeros(2, device=device, dtype=torch.int64),
            ws=alloc_workspace(M, H_dtype, head, device, ws_bytes))


def orpo_head_pass(H, head: Head, labels, layout, lam, sft_scope, filter_eps,
                   block_skip: bool, buf: HeadBuffers, stream=None):
    """Forward, ORPO loss, cotangent and dH, all enqueued on one stream."""
    cce_forward(H, head, labels, buf.logp, buf.lse, buf.tgt, buf.blockmax, buf.ws, stream)
    orpo_loss_from_logps(buf.logp, labels, layout, lam, sft_scope, buf.out8, buf.ws, stream)
    orpo_grad_coeffs(buf.logp, labels, layout, lam, sft_scope, buf.coeff, buf.ws, stream)
    cce_backward_dh(H, head, labels, buf.lse, buf.coeff, filter_eps,
                    buf.blockmax if block_skip else None, buf.dH, buf.skip, buf.ws, stream)


def orpo_head_pass_sharded(H, head: Head, labels, layout, lam, sft_scope, filter_eps,
                           block_skip: bool, buf: HeadBuffers, group=None, stream=None):
    """One pair split by rows over the processes of ``group`` (one per GPU):
    this process holds some rows of each segment (``layout`` in its own row
    numbering).  Forward, then one all-reduce of the six segment sums, then
    the loss, this shard's cotangent and its dH rows.  The all-reduce runs on
    the device for NCCL and through host memory for gloo."""
    import torch.distributed as dist
    s = torch.cuda.current_stream() if stream is None else stream
    cce_forward(H, head, labels, buf.logp, buf.lse, buf.tgt, buf.blockmax, buf.ws, s)
    sums = torch.zeros(6, dtype=torch.float64, device=H.device)
    orpo_partial_sums(buf.logp, labels, layout, sums, buf.ws, s)
    if dist.get_backend(group) == "nccl":
        with torch.cuda.stream(s):
            dist.all_reduce(sums, group=group)
    else:
        s.synchronize()
        host = sums.cpu()
        dist.all_reduce(host, group=group)
        with torch.cuda.stream(s):
            sums.copy_(host)
    orpo_from_sums(sums, labels, layout, lam, sft_scope, buf.out8, buf.coeff, buf.ws, s)
    cce_backward_dh(H, head, labels, buf.lse, buf.coeff, filter_eps,
                    buf.blockmax if block_skip else None, buf.dH, buf.skip, buf.ws, s)


class HeadPassGraph:
    """``orpo_head_pass`` captured once into a CUDA graph and replayed.

    The library allocates nothing and never synchronises inside a call, and
    every launch goes to the stream it is given, so the whole pass (forward,
    merge, loss, cotangent, backward) is one graph.  The graph keeps the
    addresses of ``H``, ``labels`` and ``buf``: copy each step's inputs into
    those tensors, then ``replay()``.  The settings read at capture time
    (CTA pairs, quantised-head staging, the wait limit) are frozen into the
    graph.  Profiling must be off while capturing.
    """

    def __init__(self, H, head: Head, labels, layout, lam, sft_scope, filter_eps,
                 block_skip: bool, buf: HeadBuffers):
        self.args = (H, head, labels, layout, lam, sft_scope, filter_eps, block_skip, buf)
        side = torch.cuda.Stream(device=H.device)
        side.wait_stream(torch.cuda.current_stream(H.device))
        with torch.cuda.stream(side):  # first call outside the capture: one-time setup
            orpo_head_pass(*self.args, stream=side)
        torch.cuda.current_stream(H.device).wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            orpo_head_pass(*self.args, stream=torch.cuda.current_stream(H.device))

    def replay(self):
        self.graph.replay()


def upload_workload(wl, device="cuda"):
    """Device tensors (H, Head, labels) of a ``synthetic.Workload``."""
    import numpy as np
    if wl.dtype == "bf16":
        H = torch.from_numpy(wl.H_bits.view(np.int16)).to(device).view(torch.bfloat16)
    else:
        H = torch.from_numpy(wl.H).to(device)
    if wl.wformat in ("q4g64", "q8g64"):
        head = Head(w=torch.from_numpy(wl.q_packed.view(np.int32)).to(device), V=wl.V, D=wl.D,
                    fmt=CCE_W_AFFINE_Q4_G64 if wl.wformat == "q4g64" else CCE_W_AFFINE_Q8_G64,
                    scales=torch.from_numpy(wl.q_scales.view(np.int16)).to(device).view(torch.bfloat16),
                    biases=torch.from_numpy(wl.q_biases.view(np.int16)).to(device).view(torch.bfloat16))
    elif wl.dtype == "bf16":
        head = Head(w=torch.from_numpy(wl.W_bits.view(np.int16)).to(device).view(torch.bfloat16),
                    V=wl.V, D=wl.D)
    else:
        head = Head(w=torch.from_numpy(wl.W).to(device), V=wl.V, D=wl.D)
    labels = torch.from_numpy(wl.labels).to(device)
    return H, head, labels


def _objective(kind, lam, beta, gamma, sft_scope):
    return _Objective(OBJECTIVES.get(kind, kind), float(lam), float(beta), float(gamma),
                      SCOPE.get(sft_scope, sft_scope))


def pref_loss_from_logps(logp, labels, layout, kind, lam, beta, gamma, sft_scope, out8, ws,
                         stream=None):
    st = lib().pref_loss_from_logps(_p(logp), _p(labels), logp.shape[0],
                                    ctypes.byref(_layout(layout)),
                                    ctypes.byref(_objective(kind, lam, beta, gamma, sft_scope)),
                                    _p(out8), _p(ws), ws.numel(), _stream(stream))
    _check(st, "pref_loss_from_logps")


def pref_grad_coeffs(logp, labels, layout, kind, lam, beta, gamma, sft_scope, coeff, ws,
                     stream=None):
    st = lib().pref_grad_coeffs(_p(logp), _p(labels), logp.shape[0],
                                ctypes.byref(_layout(layout)),
                                ctypes.byref(_objective(kind, lam, beta, gamma, sft_scope)),
                                _p(coeff), _p(ws), ws.numel(), _stream(stream))
    _check(st, "pref_grad_coeffs")


def cce_prefix_gather(H_cat, P, Rc, Rr, H_head, stream=None):
    _check(lib().cce_prefix_gather(_p(H_cat), h_dtype(H_cat), P, Rc, Rr, H_cat.shape[1],
                                   _p(H_head), _stream(stream)), "cce_prefix_gather")


def cce_prefix_scatter(dH_head, P, Rc, Rr, dH_cat, stream=None):
    _check(lib().cce_prefix_scatter(_p(dH_head), P, Rc, Rr, dH_head.shape[1], _p(dH_cat),
                                    _stream(stream)), "cce_prefix_scatter")


def cce_backward_dh_dw(H, head: Head, labels, lse, coeff, filter_eps, blockmax, dH, dW,
                       skip_stats=None, ws=None, stream=None):
    st = lib().cce_backward_dh_dw(_p(H), h_dtype(H), H.shape[0], ctypes.byref(head.c()),
                                  _p(labels), _p(lse), _p(coeff), float(filter_eps),
                                  _p(blockmax), _p(dH), _p(dW), _p(skip_stats), _p(ws),
                                  ws.numel(), _stream(stream))
    _check(st, "cce_backward_dh_dw")


def cce_set_cta_pairs(on: bool):
    lib().cce_set_cta_pairs(1 if on else 0)


def cce_set_quant_staging(mode: int):
    """0: choose; 1: dequantise inside the GEMMs; 2: staged fp16 chunks."""
    lib().cce_set_quant_staging(int(mode))


def cce_set_backward_mode(mode: int):
    """Dense bf16 heads: 0 choose; 1 the grouped fused backward kernel; 2 two
    GEMMs per vocab chunk; 3 the sliced fused kernel (M <= 64, D <= 2048)."""
    lib().cce_set_backward_mode(int(mode))


def cce_set_forward_mode(mode: int):
    """4/8-bit heads: 0 choose (a transposed small-M kernel up to 240 head
    rows); 1 the tiled GEMM with in-kernel dequantisation at every M; 2 the
    transposed form of 129-240 rows for 1 to 256 rows."""
    lib().cce_set_forward_mode(int(mode))


def cce_query_fused_schedule(M: int, H_dtype: int, head: "Head | _Head"):
    """The fused backward's units as an int32 array [n, 6] (group, row tile,
    round, first, last, dH buffer), or None when the fused kernel does not
    take the problem (host-only)."""
    import numpy as np
    h = head.c() if isinstance(head, Head) else head
    n = lib().cce_query_fused_schedule(M, H_dtype, ctypes.byref(h), None, 0)
    if n < 0:
        return None
    out = np.zeros((max(n, 1), 6), dtype=np.int32)
    lib().cce_query_fused_schedule(M, H_dtype, ctypes.byref(h),
                                   out.ctypes.data_as(ctypes.c_void_p), n)
    return out[:n]


def cce_query_plan(M: int, H_dtype: int, head: "Head | _Head", ws_bytes: int) -> dict:
    """The chunking, K split, staging and CTA-pair plan the forward and
    backward would take with a workspace of ``ws_bytes`` (host-only)."""
    out = _Plan()
    h = head.c() if isinstance(head, Head) else head
    _check(lib().cce_query_plan(M, H_dtype, ctypes.byref(h), ws_bytes, ctypes.byref(out)),
           "cce_query_plan")
    return {n: getattr(out, n) for n, _ in _Plan._fields_}
