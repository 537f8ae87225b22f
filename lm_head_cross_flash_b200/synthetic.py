"""Seeded synthetic workloads for the flash-CCE ORPO head.

This module only draws and formats inputs: random numbers, bfloat16 rounding
of the drawn values, the 4-bit affine storage format of the head, and the
head-row layout.  It holds none of the head's arithmetic (no logits, softmax,
loss or gradient) and imports neither the CUDA binding nor the oracle, so
both sides can consume the same inputs.

Workloads (the head shapes of one ORPO pair; rows are
``[prompt | chosen response | rejected response]``, row 0 unlabelled):

====  ===========================  ======  =====  ========  ========  =====================
id    name                         M       D      V         head      H
====  ===========================  ======  =====  ========  ========  =====================
0     tiny pair, fp32              256     256    4,096     fp32      N(0,1)
1     small pair, bf16, peaked     2,048   1,536  73,440    bf16      N(0,1)+4 W[y]/|W[y]|
2     long pair, bf16, flat        8,192   2,048  262,144   bf16      N(0,1)
3     long pair, bf16, peaked      8,192   2,048  262,144   bf16      N(0,1)+6 W[y]/|W[y]|
4     long context, 4-bit head     32,768  4,096  128,256   Q4 g64    N(0,1)+6 W[y]/|W[y]|
====  ===========================  ======  =====  ========  ========  =====================

Recipe (workload k): ``SeedSequence(1234 + k)`` spawns three streams — W,
labels, H noise.  W ~ N(0, 1/D) in float32, drawn in row blocks of 4,096 rows
(one child stream per block, so generation runs on several threads and stays
deterministic); labels uniform in [0, V); H noise N(0, 1) in row blocks of
1,024 rows.  Peaked workloads add alpha * W[y] / ||W[y]|| (the rounded bf16 W,
or the unquantised float32 W for the 4-bit head).  H and W are then rounded
to bfloat16 with round-to-nearest-even (workloads 1-4); workload 0 stays
float32.  Row 0's label is set to -1 (the unlabelled first prompt position).
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

LAMBDA = 0.1
VOCAB_TILE = 256  # tail rows of the vocab are sampled at this granularity
ROW_TILE = 128    # per-tile sampling: one row in every block of this many rows

CONFIGS = {
    0: dict(name="tiny_pair_fp32_M256_D256_V4096", P=32, Rc=96, Rr=128, D=256,
            V=4096, dtype="f32", wformat="dense", alpha=0.0, scope="full",
            filter_eps=0.0, block_skip=False),
    1: dict(name="small_pair_bf16_peaked_M2048_D1536_V73440", P=512, Rc=768,
            Rr=768, D=1536, V=73440, dtype="bf16", wformat="dense", alpha=4.0,
            scope="response", filter_eps=0.0, block_skip=False),
    2: dict(name="long_pair_bf16_flat_M8192_D2048_V262144", P=1024, Rc=3584,
            Rr=3584, D=2048, V=262144, dtype="bf16", wformat="dense",
            alpha=0.0, scope="full", filter_eps=0.0, block_skip=False),
    3: dict(name="long_pair_bf16_peaked_filtered_M8192_D2048_V262144", P=1024,
            Rc=3584, Rr=3584, D=2048, V=262144, dtype="bf16", wformat="dense",
            alpha=6.0, scope="full", filter_eps=1e-6, block_skip=True),
    4: dict(name="long_context_q4g64_M32768_D4096_V128256", P=4096, Rc=14336,
            Rr=14336, D=4096, V=128256, dtype="bf16", wformat="q4g64",
            alpha=6.0, scope="full", filter_eps=1e-6, block_skip=False),
}


def _threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------
# formats
# ----------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns of float32 values, round-to-nearest-even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def quantize_affine_q4(w: np.ndarray, group: int = 64):
    """Store float32 rows [V, D] as 4-bit affine groups of ``group`` along D.

    Per group: bias = min, scale = (max - min) / 15 (1 if the group is
    constant), both rounded to bfloat16; q = clip(rint((w - bias) / scale),
    0, 15) with round-half-even, using the rounded scale and bias.  Packing:
    element ``8k + j`` of a row goes to bits ``4j .. 4j+3`` of uint32 word
    ``k``.  Returns (packed uint32 [V, D/8], scales bf16 bits [V, D/group],
    biases bf16 bits [V, D/group]).
    """
    V, D = w.shape
    assert D % group == 0 and D % 8 == 0
    wg = w.reshape(V, D // group, group)
    mn = wg.min(axis=2)
    mx = wg.max(axis=2)
    scale = (mx - mn) / np.float32(15.0)
    scale = np.where(scale == 0, np.float32(1.0), scale).astype(np.float32)
    sb = f32_to_bf16_bits(scale)
    bb = f32_to_bf16_bits(mn)
    s = bf16_bits_to_f32(sb)[:, :, None]
    b = bf16_bits_to_f32(bb)[:, :, None]
    q = np.clip(np.rint((wg - b) / s), 0, 15).astype(np.uint32).reshape(V, D)
    packed = np.zeros((V, D // 8), dtype=np.uint32)
    for j in range(8):
        packed |= q[:, j::8] << np.uint32(4 * j)
    return packed, sb, bb


def quantize_affine_q8(w: np.ndarray, group: int = 64):
    """Store float32 rows [V, D] as 8-bit affine groups of ``group`` along D.

    As ``quantize_affine_q4`` with 255 levels: bias = min, scale =
    (max - min) / 255 (1 if constant), both bf16; q = clip(rint((w - bias) /
    scale), 0, 255).  Packing: element ``4k + j`` of a row is byte ``j`` of
    uint32 word ``k`` (low byte first).  Returns (packed uint32 [V, D/4],
    scales bf16 bits [V, D/group], biases bf16 bits [V, D/group]).
    """
    V, D = w.shape
    assert D % group == 0 and D % 4 == 0
    wg = w.reshape(V, D // group, group)
    mn = wg.min(axis=2)
    mx = wg.max(axis=2)
    scale = (mx - mn) / np.float32(255.0)
    scale = np.where(scale == 0, np.float32(1.0), scale).astype(np.float32)
    sb = f32_to_bf16_bits(scale)
    bb = f32_to_bf16_bits(mn)
    s = bf16_bits_to_f32(sb)[:, :, None]
    b = bf16_bits_to_f32(bb)[:, :, None]
    q = np.clip(np.rint((wg - b) / s), 0, 255).astype(np.uint32).reshape(V, D)
    packed = np.zeros((V, D // 4), dtype=np.uint32)
    for j in range(4):
        packed |= q[:, j::4] << np.uint32(8 * j)
    return packed, sb, bb


# ----------------------------------------------------------------------------
# workload
# ----------------------------------------------------------------------------

@dataclass
class Workload:
    """One seeded input set.  Arrays are host numpy arrays.

    * ``H``: float32 [M, D] (bf16-representable values for bf16 workloads);
      ``H_bits`` the bf16 bit patterns (uint16) or None for fp32.
    * dense head: ``W`` float32 [V, D] (bf16-representable for bf16) and
      ``W_bits``; 4-bit (8-bit) head: ``q_packed`` uint32 [V, D/8] ([V, D/4]),
      ``q_scales`` / ``q_biases`` bf16 bits [V, D/64], and ``W`` None.
    """

    cfg_id: int
    name: str
    M: int
    D: int
    V: int
    P: int
    Rc: int
    Rr: int
    dtype: str
    wformat: str
    scope: str
    lam: float
    filter_eps: float
    block_skip: bool
    labels: np.ndarray
    H: np.ndarray
    H_bits: np.ndarray | None
    W: np.ndarray | None = None
    W_bits: np.ndarray | None = None
    q_packed: np.ndarray | None = None
    q_scales: np.ndarray | None = None
    q_biases: np.ndarray | None = None
    extra: dict = field(default_factory=dict)

    @property
    def layout_tuple(self):
        P, Rc, Rr = self.P, self.Rc, self.Rr
        return (0, P, P, P + Rc, P + Rc, P + Rc + Rr)


def _draw_blocks(ss: np.random.SeedSequence, rows: int, cols: int, block: int,
                 scale: float, threads: int) -> np.ndarray:
    out = np.empty((rows, cols), dtype=np.float32)
    nb = (rows + block - 1) // block
    kids = ss.spawn(nb)

    def work(i):
        r0 = i * block
        r1 = min(rows, r0 + block)
        g = np.random.Generator(np.random.PCG64(kids[i]))
        blk = g.standard_normal((r1 - r0, cols), dtype=np.float32)
        if scale != 1.0:
            blk *= np.float32(scale)
        out[r0:r1] = blk

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, range(nb)))
    return out


def make_custom(cfg_id: int, *, M_split=None, D=None, V=None, dtype=None,
                wformat=None, alpha=None, seed=None, threads=None) -> Workload:
    """A workload with the recipe of ``cfg_id`` and optionally other sizes.

    ``M_split`` = (P, Rc, Rr).  Used for the small parity cases (ragged
    tails, several tiles) with the same draw recipe.
    """
    base = dict(CONFIGS[cfg_id])
    if M_split is not None:
        base["P"], base["Rc"], base["Rr"] = M_split
    for k, v in (("D", D), ("V", V), ("dtype", dtype), ("wformat", wformat),
                 ("alpha", alpha)):
        if v is not None:
            base[k] = v
    if M_split is not None or D is not None or V is not None:
        base["name"] = f"custom_from{cfg_id}_M{sum((base['P'], base['Rc'], base['Rr']))}_D{base['D']}_V{base['V']}"
    return _make(cfg_id, base, 1234 + cfg_id if seed is None else seed,
                 threads or _threads())


def make_workload(cfg_id: int, threads=None) -> Workload:
    return _make(cfg_id, dict(CONFIGS[cfg_id]), 1234 + cfg_id, threads or _threads())


def _make(cfg_id, c, seed, threads) -> Workload:
    P, Rc, Rr, D, V = c["P"], c["Rc"], c["Rr"], c["D"], c["V"]
    M = P + Rc + Rr
    ss = np.random.SeedSequence(seed)
    ss_w, ss_y, ss_h = ss.spawn(3)
    Wf = _draw_blocks(ss_w, V, D, 4096, 1.0 / math.sqrt(D), threads)
    labels = np.random.Generator(np.random.PCG64(ss_y)).integers(
        0, V, size=M).astype(np.int32)
    H = _draw_blocks(ss_h, M, D, 1024, 1.0, threads)

    wl = Workload(cfg_id=cfg_id, name=c["name"], M=M, D=D, V=V, P=P, Rc=Rc,
                  Rr=Rr, dtype=c["dtype"], wformat=c["wformat"],
                  scope=c["scope"], lam=LAMBDA, filter_eps=c["filter_eps"],
                  block_skip=c["block_skip"], labels=labels, H=H, H_bits=None)

    if c["wformat"] in ("q4g64", "q8g64"):
        per_word = 8 if c["wformat"] == "q4g64" else 4
        quant = quantize_affine_q4 if per_word == 8 else quantize_affine_q8
        packed = np.empty((V, D // per_word), dtype=np.uint32)
        sc = np.empty((V, D // 64), dtype=np.uint16)
        bi = np.empty((V, D // 64), dtype=np.uint16)
        blk = 4096

        def qwork(i):
            r0, r1 = i * blk, min(V, (i + 1) * blk)
            p_, s_, b_ = quant(Wf[r0:r1])
            packed[r0:r1], sc[r0:r1], bi[r0:r1] = p_, s_, b_

        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(qwork, range((V + blk - 1) // blk)))
        wl.q_packed, wl.q_scales, wl.q_biases = packed, sc, bi
        dirW = Wf                      # peaking direction: unquantised W
    elif c["dtype"] == "bf16":
        wl.W_bits = f32_to_bf16_bits(Wf)
        wl.W = bf16_bits_to_f32(wl.W_bits)
        dirW = wl.W
        del Wf
    else:
        wl.W = Wf
        dirW = Wf

    if c["alpha"]:
        rowsW = dirW[labels].astype(np.float64)
        nrm = np.linalg.norm(rowsW, axis=1, keepdims=True)
        H += (c["alpha"] * rowsW / nrm).astype(np.float32)
    if c["dtype"] == "bf16":
        wl.H_bits = f32_to_bf16_bits(H)
        wl.H = bf16_bits_to_f32(wl.H_bits)
    labels[0] = -1
    return wl


# ----------------------------------------------------------------------------
# sampling and synthetic cotangents
# ----------------------------------------------------------------------------

def sample_rows(wl: Workload, n_uniform: int = 48, seed: int = 7, per_tile: bool = False,
                edge: int = 4) -> np.ndarray:
    """Stratified rows for sampled parity at full size.

    Row 0; the first and last ``edge`` rows of each segment; up to 8 rows
    whose label falls in the last (possibly partial) vocab tile; with
    ``per_tile`` one seeded row inside every 128-row tile; ``n_uniform``
    uniform rows.  Sorted and unique.
    """
    M = wl.M
    rows = {0}
    for b, e in ((0, wl.P), (wl.P, wl.P + wl.Rc), (wl.P + wl.Rc, M)):
        rows.update(range(b, min(e, b + edge)))
        rows.update(range(max(b, e - edge), e))
    tail0 = ((wl.V - 1) // VOCAB_TILE) * VOCAB_TILE
    tail_rows = np.nonzero(wl.labels >= tail0)[0][:8]
    rows.update(int(r) for r in tail_rows)
    g = np.random.Generator(np.random.PCG64(seed))
    if per_tile:
        for t0 in range(0, M, ROW_TILE):
            rows.add(int(t0 + g.integers(0, min(ROW_TILE, M - t0))))
    rows.update(int(r) for r in g.integers(0, M, size=n_uniform))
    return np.array(sorted(rows), dtype=np.int64)


def random_cotangent(wl: Workload, seed: int = 11) -> np.ndarray:
    """A non-uniform per-row cotangent g ~ N(0,1)/M (0 on unlabelled rows)."""
    g = np.random.Generator(np.random.PCG64(seed)).standard_normal(wl.M)
    g = (g / wl.M).astype(np.float32)
    g[wl.labels < 0] = 0.0
    return g


def random_logps(M: int, seed: int = 13, scale: float = 8.0) -> np.ndarray:
    """Seeded negative per-token log-probs, for testing the ORPO epilogue."""
    g = np.random.Generator(np.random.PCG64(seed))
    return (-scale * g.random(M) - 1e-3).astype(np.float32)
