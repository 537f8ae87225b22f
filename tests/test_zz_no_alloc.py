"""The workspace-free forward (cce_forward_noalloc) against cce_forward.

This entry point exists for callers that cannot allocate device memory
(plugins handed only input/output pointers by a framework that owns every
device allocation, runtimes with a device-memory budget fixed at start-up).
It must give the same per-row logp, lse, target logits and block maxima as
the workspace entry point, on two calls in a row that reuse the library's
one scratch array, allocate no device memory, report a label >= V through
its status output, and refuse problems larger than that array.

The file is named so that pytest collects it last.
"""

import numpy as np
import pytest
import torch

from lm_head_cross_flash_b200 import cce
from lm_head_cross_flash_b200 import synthetic as S

from helpers import TOL_LOGP, upload

pytestmark = pytest.mark.gpu


def _reference(H, head, labels, M, V):
    ws = cce.alloc_workspace(M, cce.h_dtype(H), head)
    f = dict(device="cuda", dtype=torch.float32)
    out = dict(logp=torch.empty(M, **f), lse=torch.empty(M, **f), tgt=torch.zeros(M, **f),
               bm=torch.empty(cce.blockmax_cols(V), M, **f))
    cce.cce_forward(H, head, labels, out["logp"], out["lse"], out["tgt"], out["bm"], ws)
    torch.cuda.synchronize()
    assert cce.cce_device_status(ws) == 0
    return out


def _noalloc(H, head, labels, M, V, with_outputs):
    f = dict(device="cuda", dtype=torch.float32)
    st = torch.full((1,), 0xFF, dtype=torch.int32, device="cuda")
    out = dict(logp=torch.empty(M, **f), lse=torch.empty(M, **f), tgt=torch.zeros(M, **f),
               bm=torch.empty(cce.blockmax_cols(V), M, **f))
    cce.cce_forward_noalloc(H, head, labels, out["logp"], out["lse"],
                            out["tgt"] if with_outputs else None,
                            out["bm"] if with_outputs else None, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return out


def test_noalloc_forward_matches_workspace_forward_twice():
    cases = [S.make_custom(1, M_split=(100, 150, 131), D=256, V=4097),
             S.make_custom(2, M_split=(300, 400, 500), D=512, V=12000)]
    for i, wl in enumerate(cases):
        H, head, labels = upload(wl)
        ref = _reference(H, head, labels, wl.M, wl.V)
        got = _noalloc(H, head, labels, wl.M, wl.V, with_outputs=(i == 1))
        ok = torch.from_numpy(wl.labels >= 0).cuda()
        for k in ("logp", "lse"):
            assert (got[k] - ref[k]).abs().max().item() <= TOL_LOGP, k
        if i == 1:  # second call also returns the target logits and block maxima
            assert (got["tgt"][ok] - ref["tgt"][ok]).abs().max().item() <= TOL_LOGP
            assert (got["bm"] - ref["bm"]).abs().max().item() <= TOL_LOGP
        assert torch.all(got["logp"][~ok] == 0)


def test_noalloc_rejects_problems_beyond_the_array():
    wl = S.make_custom(1, M_split=(8, 8, 8), D=64, V=300)
    H, head, labels = upload(wl)
    big_M = 8192
    Hb = torch.zeros(big_M, wl.D, dtype=torch.bfloat16, device="cuda")
    yb = torch.zeros(big_M, dtype=torch.int32, device="cuda")
    big = cce.Head(w=torch.zeros(262144, wl.D, dtype=torch.bfloat16, device="cuda"),
                   V=262144, D=wl.D)
    f = dict(device="cuda", dtype=torch.float32)
    with pytest.raises(cce.CCEError) as e:
        cce.cce_forward_noalloc(Hb, big, yb, torch.empty(big_M, **f), torch.empty(big_M, **f))
    assert e.value.status == 4
    # f32 rows are not supported by this entry point
    with pytest.raises(cce.CCEError) as e:
        cce.cce_forward_noalloc(H.float(), cce.Head(w=head.w.float(), V=wl.V, D=wl.D), labels,
                                torch.empty(wl.M, **f), torch.empty(wl.M, **f))
    assert e.value.status == 2


def test_noalloc_allocates_nothing_and_reports_bad_labels():
    wl = S.make_custom(3, M_split=(64, 96, 97), D=128, V=3000)
    H, head, labels = upload(wl)
    f = dict(device="cuda", dtype=torch.float32)
    logp, lse = torch.empty(wl.M, **f), torch.empty(wl.M, **f)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    cce.cce_forward_noalloc(H, head, labels, logp, lse, None, None, st)  # warm-up call
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    torch.cuda.reset_peak_memory_stats()
    before = torch.cuda.memory_allocated()
    cce.cce_forward_noalloc(H, head, labels, logp, lse, None, None, st)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.max_memory_allocated() == before
    assert int(st.item()) == 0
    # one label equal to V: status bit 0, reported by this call only
    bad = labels.clone()
    bad[5] = wl.V
    cce.cce_forward_noalloc(H, head, bad, logp, lse, None, None, st)
    torch.cuda.synchronize()
    assert int(st.item()) & 1
    cce.cce_forward_noalloc(H, head, labels, logp, lse, None, None, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def test_noalloc_limit_counts_only_the_scratch_it_uses():
    """Block maxima and target logits passed by the caller take no room in
    the array: a problem that needs both in the array is refused, and fits
    once the caller supplies them."""
    V, D = 262144, 64
    cols = cce.blockmax_cols(V)
    per_row = 8 * cols                      # partial sums and maxima
    M = (cce.NOALLOC_SCRATCH_BYTES - 4096) // (per_row // 2 + 4) - 64
    assert M * (per_row + 4) > cce.NOALLOC_SCRATCH_BYTES
    wl = S.make_custom(2, M_split=(M // 4, M // 4, M - 2 * (M // 4)), D=D, V=V)
    H, head, labels = upload(wl)
    f = dict(device="cuda", dtype=torch.float32)
    with pytest.raises(cce.CCEError) as e:
        cce.cce_forward_noalloc(H, head, labels, torch.empty(M, **f), torch.empty(M, **f))
    assert e.value.status == 4
    ref = _reference(H, head, labels, M, V)
    got = _noalloc(H, head, labels, M, V, with_outputs=True)
    ok = torch.from_numpy(wl.labels >= 0).cuda()
    for k in ("logp", "lse"):
        assert (got[k] - ref[k]).abs().max().item() <= TOL_LOGP, k
    assert (got["tgt"][ok] - ref["tgt"][ok]).abs().max().item() <= TOL_LOGP
