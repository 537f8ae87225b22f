"""One pair split by rows over two processes (the one exchange step of the
path: an all-reduce of six segment sums between forward and backward)
against the same pair in one process.  Both processes share one GPU; their
kernels never wait on each other (the all-reduce is gloo, through host
memory)."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from lm_head_cross_flash_b200 import cce
from lm_head_cross_flash_b200 import synthetic as S

pytestmark = pytest.mark.gpu

SPLIT, D, V = (40, 70, 90), 256, 3000


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _shard_rows(rank, P, Rc, Rr):
    """Rank 0 takes the first half of every segment, rank 1 the rest."""
    rows, sizes = [], []
    for b, n in ((0, P), (P, Rc), (P + Rc, Rr)):
        h = n // 2
        lo, hi = (b, b + h) if rank == 0 else (b + h, b + n)
        rows.append(np.arange(lo, hi))
        sizes.append(hi - lo)
    p, c, r = sizes
    return np.concatenate(rows), (0, p, p, p + c, p + c, p + c + r)


def _upload_rows(wl, rows, device):
    H, head, labels = cce.upload_workload(wl, device)
    idx = torch.from_numpy(rows).to(device)
    return H.index_select(0, idx).contiguous(), head, labels.index_select(0, idx).contiguous()


def _worker(rank, port, q):
    import torch.distributed as dist
    try:
        torch.cuda.set_device(0)
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=2)
        wl = S.make_custom(2, M_split=SPLIT, D=D, V=V)
        rows, layout = _shard_rows(rank, *SPLIT)
        H, head, labels = _upload_rows(wl, rows, "cuda")
        buf = cce.HeadBuffers.alloc(H.shape[0], wl.D, wl.V, cce.h_dtype(H), head)
        cce.orpo_head_pass_sharded(H, head, labels, layout, wl.lam, wl.scope, 0.0, False, buf)
        torch.cuda.synchronize()
        q.put((rank, cce.cce_device_status(buf.ws), rows, buf.out8.cpu().numpy(),
               buf.coeff.cpu().numpy(), buf.logp.cpu().numpy(), buf.dH.cpu().numpy()))
        dist.destroy_process_group()
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((rank, repr(e)))


def test_row_sharded_pair_matches_one_process():
    wl = S.make_custom(2, M_split=SPLIT, D=D, V=V)
    H, head, labels = cce.upload_workload(wl, "cuda")
    ref = cce.HeadBuffers.alloc(wl.M, wl.D, wl.V, cce.h_dtype(H), head)
    cce.orpo_head_pass(H, head, labels, wl.layout_tuple, wl.lam, wl.scope, 0.0, False, ref)
    torch.cuda.synchronize()
    assert cce.cce_device_status(ref.ws) == 0
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=300) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
    for g in got:
        assert len(g) == 7, g
    out8_ref = ref.out8.cpu().numpy()
    coeff_ref = ref.coeff.cpu().numpy()
    logp_ref = ref.logp.cpu().numpy()
    dH_ref = ref.dH.cpu().numpy()
    for rank, st, rows, out8, coeff, logp, dH in got:
        assert st == 0
        assert np.allclose(out8, out8_ref, rtol=1e-12, atol=0), (rank, out8, out8_ref)
        assert np.allclose(logp, logp_ref[rows], rtol=0, atol=1e-6)
        assert np.allclose(coeff, coeff_ref[rows], rtol=1e-6, atol=1e-12)
        err = np.linalg.norm(dH - dH_ref[rows]) / np.linalg.norm(dH_ref[rows])
        assert err < 1e-5, (rank, err)
    # every row of the pair is covered once
    assert sorted(np.concatenate([g[2] for g in got]).tolist()) == list(range(wl.M))


def _nccl_worker(port, q):
    """One rank of an NCCL process group on GPU 0: the device all-reduce of
    the sharded pass runs on the caller's (non-default) stream."""
    import datetime

    import torch.distributed as dist
    try:
        torch.cuda.set_device(0)
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                world_size=1, timeout=datetime.timedelta(seconds=60),
                                device_id=torch.device("cuda", 0))
        assert dist.get_backend() == "nccl"
        wl = S.make_custom(2, M_split=SPLIT, D=D, V=V)
        H, head, labels = cce.upload_workload(wl, "cuda")
        ref = cce.HeadBuffers.alloc(wl.M, wl.D, wl.V, cce.h_dtype(H), head)
        cce.orpo_head_pass(H, head, labels, wl.layout_tuple, wl.lam, wl.scope, 0.0, False, ref)
        torch.cuda.synchronize()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        buf = cce.HeadBuffers.alloc(wl.M, wl.D, wl.V, cce.h_dtype(H), head)
        with torch.cuda.stream(side):
            cce.orpo_head_pass_sharded(H, head, labels, wl.layout_tuple, wl.lam, wl.scope, 0.0,
                                       False, buf, stream=side)
        side.synchronize()
        same = [torch.equal(getattr(buf, k), getattr(ref, k))
                for k in ("logp", "lse", "out8", "coeff", "dH")]
        q.put((cce.cce_device_status(buf.ws), same))
        dist.destroy_process_group()
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((repr(e), None))


def test_row_sharded_pair_nccl_branch_one_rank():
    """The NCCL branch of the sharded pass (device all-reduce of the six
    segment sums, ordered on the caller's stream) with a one-rank group on
    one GPU: the same bits as the unsharded pass."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_nccl_worker, args=(_free_port(), q))
    p.start()
    st, same = q.get(timeout=300)
    p.join(timeout=60)
    assert st == 0, st
    assert all(same), same
