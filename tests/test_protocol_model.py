"""CPU models of the two fused backward kernels' synchronisation protocols.

Each model replays, step by step, the waits and signals that every role of
every CTA issues (the order the kernel code issues them in), over the
library's own schedule where one exists, with random skip patterns, and
checks that every role runs to the end: no deadlock.  The GPU waits are
bounded, so a protocol error shows as a device timeout, not a hang; these
models find such errors on the CPU first.  Planted mistakes (a wait one fill
too far, a missing signal, a missing arm) must make the models stall, which
shows that they can.

* The grouped fused kernel (fused_bwd.cuh): per member, a producer, an MMA
  issuer and the four epilogue warps; a FIFO ring of operand stages shared
  by the S-phase and dH-phase loads; the G'' exchange ring of DEPTH fills
  per (group, member) with its ready and consumed counters (each warp adds
  1 per fill, the consumer waits for 4 per fill); the S and dH accumulator
  barriers.  Besides running to the end, the model checks safety: when a
  consumer's wait for a fill passes, every warp's rows of that fill have
  landed.  One epilogue warp can be made slow (it moves only when nothing
  else can), which opens the windows a lagging warp leaves.  The lead cap is
  a bounded hint, not a dependency, and is left out.  A CTA pair runs as one
  member.
* The transposed small-M forwards (qsmall_fwd.cuh, qwide_fwd.cuh): the
  producer, the MMA issuer(s), the eight dequantisation warps and the four
  epilogue warps of one CTA, with the stage ring, the TMEM A ring, the
  accumulators and the epilogue's merge barrier as phase objects; safety
  (no stage, A slot, accumulator or merge buffer reused before its readers
  are done) is tracked apart from the barriers, and every role is held back
  in turn.
* The sliced kernel (slice_bwd.cuh): per CTA of a cluster, the S and dH
  loaders and MMA issuers, the drain warps and the reducer warps, with the
  double-buffered partial (pfull, pempty), G'' (gfull, gempty) and S
  accumulator (afull, aempty) barriers.  Barriers are phase objects: an
  arrival or byte count lands in whatever phase is current, and the model
  asserts it belongs to that phase's tile (so a sender that runs a phase
  ahead is an error, as it would be on the GPU).
"""

import ctypes
import random

import pytest

from lm_head_cross_flash_b200 import cce


# --------------------------------------------------------------- machinery --
def _run(procs, step, slow=()):
    """procs: list of (state, [op lists]).  Runs every op list as far as its
    next op allows, until nothing moves; the roles in `slow` ((process,
    role) pairs) take one op at a time, and only when no other role can
    move.  Returns the list of stuck (process, role, position, length)."""
    pos = [[0] * len(lists) for _, lists in procs]
    slow = set(slow)
    while True:
        moved = False
        for i, (st, lists) in enumerate(procs):
            for r, ops in enumerate(lists):
                if (i, r) in slow:
                    continue
                while pos[i][r] < len(ops) and step(st, *ops[pos[i][r]]):
                    pos[i][r] += 1
                    moved = True
        if moved:
            continue
        for i, r in sorted(slow):
            ops = procs[i][1][r]
            if pos[i][r] < len(ops) and step(procs[i][0], *ops[pos[i][r]]):
                pos[i][r] += 1
                moved = True
                break
        if not moved:
            break
    return [(i, r, pos[i][r], len(ops)) for i, (_, lists) in enumerate(procs)
            for r, ops in enumerate(lists) if pos[i][r] < len(ops)]


# ------------------------------------------------------ grouped fused kernel --
FB_DEPTH = 2


EPI_WARPS = 4


def _fused_model(M, V, D, skip_prob, seed, pairs=True, bug=None, slow=()):
    """Stuck roles plus safety violations (empty: the protocol is sound on
    this schedule and skip pattern).  bug: "consumed_off_by_one" (a
    publisher waits one fill too far), "no_consumed_on_skip" (the MMA warp
    does not release a skipped tile's slot), "skip_without_wait" (a warp
    counts a skipped tile without waiting for the slot's previous fill to
    be consumed).  slow: (process, role) pairs held back; a process is a
    (group, member) in order, its roles the producer, the MMA issuer and
    epilogue warps 0-3."""
    lib = cce.lib()
    h = cce._Head(cce.CCE_W_DENSE, cce.CCE_BF16, V, D, D, None, None)
    cce.cce_set_backward_mode(1)
    cce.cce_set_cta_pairs(pairs)
    try:
        plan = cce.cce_query_plan(M, cce.CCE_BF16, h,
                                  lib.cce_workspace_bytes(M, cce.CCE_BF16, ctypes.byref(h)))
        sched = cce.cce_query_fused_schedule(M, cce.CCE_BF16, h)
    finally:
        cce.cce_set_backward_mode(0)
        cce.cce_set_cta_pairs(True)
    assert plan["bwd_fused"]
    C, G = plan["bwd_fused_members"], plan["bwd_fused_groups"]
    c2 = bool(plan["bwd_cta_pairs"])
    nk = -(-D // 64)                  # K steps of an S tile
    kv = (256 if c2 else 128) // 64   # K steps of a dH tile
    nst = 6 if c2 else 4              # operand stages
    sbufs = 1 if c2 else 2            # S accumulators
    rng = random.Random(seed)
    skips = {}

    def skip(r, v):
        if (r, v) not in skips:
            skips[(r, v)] = rng.random() < skip_prob
        return skips[(r, v)]

    units = {g: [tuple(int(x) for x in row[1:]) for row in sched[sched[:, 0] == g]]
             for g in range(G)}
    shared = {"ready": {}, "consumed": {}, "landed": {}, "violations": []}
    procs = []
    for g in range(G):
        U = units[g]
        for p in range(C):
            P, X, E = [], [], []
            # producer: S loads of unit u, then the dH loads of unit u - 1
            for u in range(len(U) + 1):
                if u < len(U):
                    r, j = U[u][0], U[u][1]
                    if not skip(r, j * C + p):
                        P += [("load",)] * nk
                if u >= 1:
                    r, j = U[u - 1][0], U[u - 1][1]
                    fill = (u - 1) // FB_DEPTH
                    for q in range(C):
                        if skip(r, j * C + q):
                            continue
                        P.append(("wait_ready", (g, (u - 1) % FB_DEPTH, q), fill + 1))
                        P += [("load",)] * kv
            # MMA: S(u), then dH(u - 1)
            ns = nseg = 0
            dh_any = False
            for u in range(len(U) + 1):
                if u < len(U):
                    r, j = U[u][0], U[u][1]
                    if not skip(r, j * C + p):
                        X.append(("wait_s_empty", ns))
                        X += [("consume",)] * nk
                        X.append(("s_full",))
                        ns += 1
                if u >= 1:
                    r, j, first, last = U[u - 1][0], U[u - 1][1], U[u - 1][2], U[u - 1][3]
                    fill = (u - 1) // FB_DEPTH
                    if first:
                        dh_any = False
                    for q in range(C):
                        key = (g, (u - 1) % FB_DEPTH, q, p)
                        if skip(r, j * C + q):
                            if bug != "no_consumed_on_skip":
                                X.append(("set_consumed", key, fill + 1))
                            continue
                        if not dh_any:
                            X.append(("wait_dh_empty", nseg))
                        X += [("consume",)] * kv
                        X.append(("set_consumed", key, fill + 1))
                        dh_any = True
                    if last and dh_any:
                        X.append(("dh_full",))
                        nseg += 1
            # epilogue warps: publish their rows of G''(u) once every member
            # consumed the slot's previous fill; flush a finished segment's dH
            E = []
            for w in range(EPI_WARPS):
                Ew = []
                ns = nseg = 0
                prev, seg_any, prev_any = None, False, False
                for u in range(len(U)):
                    r, j, first = U[u][0], U[u][1], U[u][2]
                    if first:
                        seg_any = False
                    seg_any = seg_any or any(not skip(r, j * C + q) for q in range(C))
                    fill = u // FB_DEPTH
                    slot = (g, u % FB_DEPTH, p)
                    if not skip(r, j * C + p):
                        Ew.append(("wait_s_full", ns))
                        need = fill + 1 if bug == "consumed_off_by_one" else fill
                        if fill >= 1:
                            for c in range(C):
                                Ew.append(("wait_consumed", (g, u % FB_DEPTH, p, c), need))
                        Ew.append(("s_empty",))
                        ns += 1
                        Ew.append(("landed", slot, w, fill + 1))
                    elif fill >= 1 and bug != "skip_without_wait":
                        for c in range(C):
                            Ew.append(("wait_consumed", (g, u % FB_DEPTH, p, c), fill))
                    Ew.append(("ready_add", slot))
                    if u >= 1 and prev[3] and prev_any:
                        Ew += [("wait_dh_full", nseg), ("dh_empty",)]
                        nseg += 1
                    prev, prev_any = U[u], seg_any
                if prev is not None and prev_any:
                    Ew += [("wait_dh_full", nseg), ("dh_empty",)]
                E.append(Ew)
            st = dict(ring=0, s_full=0, s_empty=0, dh_full=0, dh_empty=0)
            procs.append((st, [P, X] + E))

    def step(st, op, *arg):
        if op == "load":
            if st["ring"] >= nst:
                return False
            st["ring"] += 1
            return True
        if op == "consume":
            if st["ring"] <= 0:
                return False
            st["ring"] -= 1
            return True
        if op == "wait_ready":
            if shared["ready"].get(arg[0], 0) < EPI_WARPS * arg[1]:
                return False
            late = [w for w in range(EPI_WARPS)
                    if shared["landed"].get((arg[0], w), 0) < arg[1]]
            if late:
                shared["violations"].append(("read before landed", arg[0], arg[1], late))
            return True
        if op == "landed":
            shared["landed"][(arg[0], arg[1])] = arg[2]
            return True
        if op == "set_consumed":
            shared["consumed"][arg[0]] = arg[1]
            return True
        if op == "wait_consumed":
            return shared["consumed"].get(arg[0], 0) >= arg[1]
        if op == "ready_add":
            shared["ready"][arg[0]] = shared["ready"].get(arg[0], 0) + 1
            return True
        if op == "wait_s_empty":
            return st["s_empty"] >= EPI_WARPS * (arg[0] - sbufs + 1)
        if op == "wait_s_full":
            return st["s_full"] > arg[0]
        if op == "wait_dh_empty":
            return st["dh_empty"] >= EPI_WARPS * arg[0]
        if op == "wait_dh_full":
            return st["dh_full"] > arg[0]
        if op in ("s_full", "s_empty", "dh_full", "dh_empty"):
            st[op] += 1
            return True
        raise ValueError(op)

    stuck = _run(procs, step, slow=slow)
    return stuck + shared["violations"]


FUSED_SHAPES = [(8192, 16384, 2048, True), (300, 1000, 320, True), (64, 20000, 2048, False),
                (5000, 3000, 2048, True), (2048, 7000, 1536, True), (1, 31, 64, False),
                (129, 4097, 256, True), (900, 6000, 256, False)]


@pytest.mark.parametrize("M,V,D,pairs", FUSED_SHAPES)
@pytest.mark.parametrize("skip_prob", [0.0, 0.3, 0.9])
def test_fused_protocol_runs_to_the_end(M, V, D, pairs, skip_prob):
    assert _fused_model(M, V, D, skip_prob, seed=M + V, pairs=pairs) == []


@pytest.mark.parametrize("bug,skip_prob", [("consumed_off_by_one", 0.0),
                                           ("no_consumed_on_skip", 0.3)])
def test_fused_protocol_model_catches_planted_mistakes(bug, skip_prob):
    assert _fused_model(2048, 7000, 1536, skip_prob, seed=5, bug=bug) != []


@pytest.mark.parametrize("M,V,D,pairs", [(900, 60000, 256, False), (900, 20000, 256, False),
                                         (300, 1000, 320, True), (2048, 7000, 1536, True),
                                         (8192, 16384, 2048, True)])
@pytest.mark.parametrize("skip_prob", [0.0, 0.3, 0.9])
def test_fused_protocol_is_safe_with_a_slow_warp(M, V, D, pairs, skip_prob):
    """One epilogue warp of group 0 moves only when nothing else can: no
    consumer may load a fill before that warp's rows of it have landed."""
    assert _fused_model(M, V, D, skip_prob, seed=M + V, pairs=pairs, slow=[(0, 2)]) == []


@pytest.mark.parametrize("role", range(6))
def test_fused_protocol_with_each_role_held_back(role):
    """The producer, the MMA issuer or one epilogue warp of group 0 held
    back in turn, with block skip: still no deadlock and no early load."""
    assert _fused_model(900, 60000, 256, 0.3, seed=11, pairs=False, slow=[(0, role)]) == []
    assert _fused_model(2048, 7000, 1536, 0.3, seed=12, pairs=True, slow=[(0, role)]) == []


def test_fused_protocol_model_catches_the_skipped_tile_race():
    """A warp that counts a skipped tile without first waiting for the
    slot's previous fill to be consumed lets its count stand in for a slow
    warp's count of that fill: the consumer then loads the fill before the
    slow warp's rows have landed (the model must report it)."""
    found = _fused_model(900, 60000, 256, 0.5, seed=7, pairs=False, bug="skip_without_wait",
                         slow=[(0, 2)])
    assert any(v[0] == "read before landed" for v in found), found[:3]


# ------------------------------------------------------------ sliced kernel --
class _Phase:
    """An mbarrier: a phase completes when `count` arrivals and the armed
    bytes have all landed; arrivals and bytes tagged with the tile they
    belong to, which must be the current phase's tile."""

    def __init__(self, count, tiles):
        self.count, self.tiles = count, tiles  # tiles: the tile of each phase, in order
        self.phase, self.arrived, self.tx = 0, 0, 0

    def cur(self):
        return self.tiles[self.phase] if self.phase < len(self.tiles) else None

    def _maybe_complete(self):
        if self.arrived == self.count and self.tx == 0:
            self.phase += 1
            self.arrived = 0

    def arrive(self, tile, expect=0):
        assert tile == self.cur(), f"arrival for tile {tile} in the phase of tile {self.cur()}"
        self.arrived += 1
        self.tx += expect
        self._maybe_complete()

    def bytes(self, tile, n):
        assert tile == self.cur(), f"bytes for tile {tile} in the phase of tile {self.cur()}"
        self.tx -= n
        self._maybe_complete()

    def done(self, tile):
        """Has the phase of `tile` completed?"""
        return tile in self.tiles[:self.phase]


class ProtocolError(AssertionError):
    """A signal that would land in another tile's barrier phase."""


def _sliced_model(n, ccl, ns=4, nd=2, nbuf=2, bug=None, slow=()):
    epi = 4
    tiles_of = lambda b: list(range(b, n, nbuf))
    ctas = []
    for c in range(ccl):
        st = dict(
            sring=0, dring=0,
            afull=[_Phase(1, tiles_of(b)) for b in range(nbuf)],
            aempty=[_Phase(epi, tiles_of(b)) for b in range(nbuf)],
            pfull=[_Phase(1, tiles_of(b)) for b in range(nbuf)],
            pempty=[_Phase(ccl * epi, [k for k in tiles_of(b) if k + nbuf < n])
                    for b in range(nbuf)],
            gfull=[_Phase(1 + epi, tiles_of(b)) for b in range(nbuf)],
            gempty=[_Phase(ccl, [k for k in tiles_of(b) if k + nbuf < n]) for b in range(nbuf)],
            dhfull=_Phase(1, [0]))
        ctas.append(st)
    part = 1      # bytes one drain warp sends to one reducer per tile
    grows = 1     # bytes one reducer warp copies to one peer per tile
    for st in ctas:   # the first tiles' arms
        for b in range(min(nbuf, n)):
            st["pfull"][b].arrive(b, expect=ccl * epi * part)
            st["gfull"][b].arrive(b, expect=(ccl - 1) * epi * grows)

    procs = []
    for c, st in enumerate(ctas):
        sprod = [("sload",)] * (4 * n)
        dprod = [("dload",)] * (4 * n)
        smma, dmma = [], []
        for k in range(n):
            b = k % nbuf
            if k >= nbuf:
                smma.append(("wait", c, "aempty", b, k - nbuf))
            smma += [("sconsume",)] * 4
            smma.append(("arrive", c, "afull", b, k, 0))
        for k in range(n):
            b = k % nbuf
            dmma.append(("wait", c, "gfull", b, k))
            dmma += [("dconsume",)] * 4
            if k + nbuf < n:
                dmma += [("arrive", q, "gempty", b, k, 0) for q in range(ccl)]
                if bug != "no_gfull_arm":
                    dmma.append(("arrive", c, "gfull", b, k + nbuf, (ccl - 1) * epi * grows))
        dmma.append(("arrive", c, "dhfull", 0, 0, 0))
        roles = [sprod, dprod, smma, dmma]
        for w in range(epi):   # drain warps
            d = []
            for j in range(n):
                b = j % nbuf
                d.append(("wait", c, "afull", b, j))
                d.append(("arrive", c, "aempty", b, j, 0))
                if j >= nbuf:
                    d.append(("wait", c, "pempty", b, j - nbuf))
                d += [("bytes", q, "pfull", b, j, part) for q in range(ccl)]
            d.append(("wait", c, "dhfull", 0, 0))
            roles.append(d)
        for w in range(epi):   # reducer warps
            r = []
            for k in range(n):
                b = k % nbuf
                r.append(("wait", c, "pfull", b, k))
                if k >= nbuf:
                    r.append(("wait", c, "gempty", b, k - nbuf))
                if k + nbuf < n:
                    if w == 0:
                        r.append(("arrive", c, "pfull", b, k + nbuf, ccl * epi * part))
                    if bug != "no_pempty":
                        r += [("arrive", q, "pempty", b, k, 0) for q in range(ccl)]
                r += [("bytes", q, "gfull", b, k, grows) for q in range(ccl) if q != c]
                r.append(("arrive", c, "gfull", b, k, 0))
            roles.append(r)
        procs.append((st, roles))

    def step(st, op, *a):
        if op == "sload":
            if st["sring"] >= ns:
                return False
            st["sring"] += 1
            return True
        if op == "sconsume":
            if st["sring"] <= 0:
                return False
            st["sring"] -= 1
            return True
        if op == "dload":
            if st["dring"] >= nd:
                return False
            st["dring"] += 1
            return True
        if op == "dconsume":
            if st["dring"] <= 0:
                return False
            st["dring"] -= 1
            return True
        cta, name, b, tile = a[0], a[1], a[2], a[3]
        bar = ctas[cta][name] if name == "dhfull" else ctas[cta][name][b]
        if op == "wait":
            return bar.done(tile)
        if bar.cur() != tile:
            # the protocol must never signal ahead of the barrier's phase
            raise ProtocolError(f"{op} for tile {tile} on {name}[{b}] of CTA {cta}, "
                                f"whose current phase is tile {bar.cur()}")
        if op == "arrive":
            bar.arrive(tile, expect=a[4])
        else:
            bar.bytes(tile, a[4])
        return True
        raise ValueError(op)

    return _run(procs, step, slow=slow)


@pytest.mark.parametrize("n", [0, 1, 2, 3, 4, 7, 30])
@pytest.mark.parametrize("ccl", [1, 2, 4, 8])
def test_sliced_protocol_runs_to_the_end(n, ccl):
    assert _sliced_model(n, ccl) == []


@pytest.mark.parametrize("ns,nd,nbuf", [(2, 1, 2), (4, 4, 2), (1, 1, 2), (4, 2, 1), (4, 2, 3)])
def test_sliced_protocol_other_depths(ns, nd, nbuf):
    """Ring depths and buffer counts other than the kernel's (4, 2, 2) also
    run to the end: nothing in the protocol relies on a particular depth."""
    assert _sliced_model(9, 8, ns=ns, nd=nd, nbuf=nbuf) == []


@pytest.mark.parametrize("bug", ["no_pempty", "no_gfull_arm"])
def test_sliced_protocol_model_catches_planted_mistakes(bug):
    assert _sliced_model(6, 4, bug=bug) != []


SLICED_ROLES = 4 + 4 + 4   # loaders and MMA issuers, drain warps, reducer warps


@pytest.mark.parametrize("n,ccl", [(5, 2), (9, 4), (7, 8), (6, 1)])
def test_sliced_protocol_with_a_slow_role(n, ccl):
    """Each role of the first and the last CTA in turn moves only when no
    other role can: the protocol still runs to the end, and no arrival or
    byte count lands in a phase that belongs to another tile."""
    for c in sorted({0, ccl - 1}):
        for r in range(SLICED_ROLES):
            assert _sliced_model(n, ccl, slow=[(c, r)]) == [], (c, r)


# ------------------------------------------------ transposed small-M forward --
def _qsmall_model(nblk, nk, nst, na, nacc, bug=None, slow=()):
    """One CTA of qsmall_fwd_kernel: the producer, the two MMA issuers
    (halves 0 and 1), eight dequantisation warps and four epilogue warps
    over nblk blocks of nk K steps; stage ring (full, empty), TMEM A ring
    (afull, aempty), accumulators (accfull, accempty; nacc buffers) and the
    epilogue's merge barrier (epibar, two by block parity), each a phase
    object tagged with its step or block.  Safety, tracked apart from the
    barriers: a stage is reloaded only after its previous step's ten reads,
    an A slot rewritten only after both issuers' MMAs of its previous step,
    an accumulator overwritten only after the four warps drained its
    previous block and drained only after both halves' MMAs, and a merge
    buffer rewritten only after every warp read it.  bug: "aempty_one_back"
    (a dequantisation warp waits for the slot's use two steps back instead
    of one), "accempty_parity" (the issuers wait for the wrong buffer use)."""
    steps = nblk * nk
    st_tiles = lambda s: [n for n in range(steps) if n % nst == s]
    a_tiles = lambda a: [n for n in range(steps) if n % na == a]
    b_tiles = lambda b, m: [u for u in range(nblk) if u % m == b]
    bars = {
        "full": [_Phase(1, st_tiles(s)) for s in range(nst)],
        "empty": [_Phase(10, st_tiles(s)) for s in range(nst)],
        "afull": [_Phase(8, a_tiles(a)) for a in range(na)],
        "aempty": [_Phase(2, a_tiles(a)) for a in range(na)],
        "accfull": [_Phase(2, b_tiles(b, nacc)) for b in range(nacc)],
        "accempty": [_Phase(4, b_tiles(b, nacc)) for b in range(nacc)],
        "epibar": [_Phase(4, b_tiles(p, 2)) for p in range(2)],
    }
    seen = {"stage_reads": {}, "mma_done": {}, "drained": {}, "mma_block": {},
            "red_written": {}, "red_read": {}, "violations": []}

    def bump(key, k):
        seen[key][k] = seen[key].get(k, 0) + 1

    P = []
    for n in range(steps):
        s = n % nst
        if n >= nst:
            P.append(("wait", "empty", s, n - nst))
        P += [("check_stage_free", n), ("arrive", "full", s, n)]
    I = []
    for h in range(2):
        ops = []
        for u in range(nblk):
            b = u % nacc
            prev = u - nacc if bug != "accempty_parity" else u - 2 * nacc
            if prev >= 0:
                ops.append(("wait", "accempty", b, prev))
            ops.append(("check_acc_free", u))
            for i in range(nk):
                n = u * nk + i
                ops += [("wait", "full", n % nst, n), ("wait", "afull", n % na, n),
                        ("mma", n, u), ("arrive", "empty", n % nst, n),
                        ("arrive", "aempty", n % na, n)]
            ops.append(("arrive", "accfull", b, u))
        I.append(ops)
    Dq = []
    for w in range(8):
        ops = []
        for n in range(steps):
            back = na if bug != "aempty_one_back" else 2 * na
            ops += [("wait", "full", n % nst, n), ("read_stage", n),
                    ("arrive", "empty", n % nst, n)]
            if n >= back:
                ops.append(("wait", "aempty", n % na, n - back))
            ops += [("check_slot_free", n), ("arrive", "afull", n % na, n)]
        Dq.append(ops)
    E = []
    for w in range(4):
        ops = []
        for u in range(nblk):
            b, par = u % nacc, u % 2
            ops += [("wait", "accfull", b, u), ("check_acc_ready", u), ("drain", u),
                    ("arrive", "accempty", b, u), ("check_red_free", w, u), ("write_red", w, u),
                    ("arrive", "epibar", par, u), ("wait", "epibar", par, u), ("read_red", w, u)]
        E.append(ops)
    procs = [({}, [P] + I + Dq + E)]

    def step(_, op, *a):
        v = seen["violations"]
        if op == "wait":
            return bars[a[0]][a[1]].done(a[2])
        if op == "arrive":
            bars[a[0]][a[1]].arrive(a[2])
            if a[0] == "full":  # the TMA bytes land with the arming
                pass
            return True
        if op == "check_stage_free":
            n = a[0]
            if n >= nst and seen["stage_reads"].get(n - nst, 0) < 10:
                v.append(("stage reloaded early", n))
            return True
        if op == "read_stage":
            bump("stage_reads", a[0])
            return True
        if op == "mma":
            bump("stage_reads", a[0])
            bump("mma_done", a[0])
            bump("mma_block", a[1])
            return True
        if op == "check_slot_free":
            n = a[0]
            if n >= na and seen["mma_done"].get(n - na, 0) < 2:
                v.append(("A slot rewritten early", n))
            return True
        if op == "check_acc_free":
            u = a[0]
            if u >= nacc and seen["drained"].get(u - nacc, 0) < 4:
                v.append(("accumulator overwritten early", u))
            return True
        if op == "check_acc_ready":
            if seen["mma_block"].get(a[0], 0) < 2 * nk:
                v.append(("accumulator drained early", a[0]))
            return True
        if op == "drain":
            bump("drained", a[0])
            return True
        if op == "check_red_free":
            w, u = a
            if u >= 2 and seen["red_read"].get(u - 2, 0) < 4:
                v.append(("merge buffer rewritten early", u))
            return True
        if op == "write_red":
            bump("red_written", a[1])
            return True
        if op == "read_red":
            if seen["red_written"].get(a[1], 0) < 4:
                v.append(("merge buffer read early", a[1]))
            bump("red_read", a[1])
            return True
        raise ValueError(op)

    try:
        stuck = _run(procs, step, slow=slow)
    except AssertionError as e:
        return [("phase", str(e))]
    return stuck + seen["violations"]


QSMALL_SHAPES = [(3, 5, 4, 2, 2), (3, 5, 6, 4, 2), (4, 7, 4, 2, 1), (5, 3, 6, 4, 1), (1, 1, 4, 2, 2)]
QSMALL_ROLES = 1 + 2 + 8 + 4


@pytest.mark.parametrize("nblk,nk,nst,na,nacc", QSMALL_SHAPES)
def test_qsmall_protocol_runs_to_the_end(nblk, nk, nst, na, nacc):
    """The transposed small-M forward's protocol (4-bit: 4 stages, 2 A
    slots; 8-bit: 6 stages, 4 slots; one or two accumulators) runs to the
    end, also with each role held back in turn, with no early reuse."""
    assert _qsmall_model(nblk, nk, nst, na, nacc) == []
    for r in range(QSMALL_ROLES):
        assert _qsmall_model(nblk, nk, nst, na, nacc, slow=[(0, r)]) == [], r


@pytest.mark.parametrize("bug", ["aempty_one_back", "accempty_parity"])
def test_qsmall_protocol_model_catches_planted_mistakes(bug):
    found = []
    for r in range(QSMALL_ROLES):
        found += _qsmall_model(4, 7, 4, 2, 2, bug=bug, slow=[(0, r)])
    assert found, bug


def _qwide_model(nblk, nk, nst=5, na=8, bug=None, slow=()):
    """One CTA of qwide_fwd_kernel: the producer, one MMA issuer, eight
    dequantisation warps and four epilogue warps; each block is two 128-row
    units of nk K steps run one after the other into one accumulator.  The
    same safety checks as _qsmall_model, per unit.  bug: "accempty_skip"
    (the issuer does not wait for the drain of the previous unit)."""
    units = 2 * nblk
    steps = units * nk
    st_tiles = lambda s: [n for n in range(steps) if n % nst == s]
    a_tiles = lambda a: [n for n in range(steps) if n % na == a]
    bars = {
        "full": [_Phase(1, st_tiles(s)) for s in range(nst)],
        "empty": [_Phase(9, st_tiles(s)) for s in range(nst)],
        "afull": [_Phase(8, a_tiles(a)) for a in range(na)],
        "aempty": [_Phase(1, a_tiles(a)) for a in range(na)],
        "accfull": [_Phase(1, list(range(units)))],
        "accempty": [_Phase(4, list(range(units)))],
        "epibar": [_Phase(4, [u for u in range(nblk) if u % 2 == p]) for p in range(2)],
    }
    seen = {"stage_reads": {}, "mma_done": {}, "drained": {}, "mma_unit": {},
            "red_written": {}, "red_read": {}, "violations": []}

    def bump(key, k):
        seen[key][k] = seen[key].get(k, 0) + 1

    P = []
    for n in range(steps):
        if n >= nst:
            P.append(("wait", "empty", n % nst, n - nst))
        P += [("check_stage_free", n), ("arrive", "full", n % nst, n)]
    X = []
    for t in range(units):
        if t >= 1 and bug != "accempty_skip":
            X.append(("wait", "accempty", 0, t - 1))
        X.append(("check_acc_free", t))
        for i in range(nk):
            n = t * nk + i
            X += [("wait", "full", n % nst, n), ("wait", "afull", n % na, n), ("mma", n, t),
                  ("arrive", "empty", n % nst, n), ("arrive", "aempty", n % na, n)]
        X.append(("arrive", "accfull", 0, t))
    Dq = []
    for w in range(8):
        ops = []
        for n in range(steps):
            ops += [("wait", "full", n % nst, n), ("read_stage", n),
                    ("arrive", "empty", n % nst, n)]
            if n >= na:
                ops.append(("wait", "aempty", n % na, n - na))
            ops += [("check_slot_free", n), ("arrive", "afull", n % na, n)]
        Dq.append(ops)
    E = []
    for w in range(4):
        ops = []
        for u in range(nblk):
            for h in range(2):
                t = 2 * u + h
                ops += [("wait", "accfull", 0, t), ("check_acc_ready", t), ("drain", t),
                        ("arrive", "accempty", 0, t)]
            ops += [("check_red_free", w, u), ("write_red", w, u), ("arrive", "epibar", u % 2, u),
                    ("wait", "epibar", u % 2, u), ("read_red", w, u)]
        E.append(ops)
    procs = [({}, [P, X] + Dq + E)]

    def step(_, op, *a):
        v = seen["violations"]
        if op == "wait":
            return bars[a[0]][a[1]].done(a[2])
        if op == "arrive":
            bars[a[0]][a[1]].arrive(a[2])
            return True
        if op == "check_stage_free":
            if a[0] >= nst and seen["stage_reads"].get(a[0] - nst, 0) < 9:
                v.append(("stage reloaded early", a[0]))
            return True
        if op == "read_stage":
            bump("stage_reads", a[0])
            return True
        if op == "mma":
            bump("stage_reads", a[0])
            bump("mma_done", a[0])
            bump("mma_unit", a[1])
            return True
        if op == "check_slot_free":
            if a[0] >= na and seen["mma_done"].get(a[0] - na, 0) < 1:
                v.append(("A slot rewritten early", a[0]))
            return True
        if op == "check_acc_free":
            if a[0] >= 1 and seen["drained"].get(a[0] - 1, 0) < 4:
                v.append(("accumulator overwritten early", a[0]))
            return True
        if op == "check_acc_ready":
            if seen["mma_unit"].get(a[0], 0) < nk:
                v.append(("accumulator drained early", a[0]))
            return True
        if op == "drain":
            bump("drained", a[0])
            return True
        if op == "check_red_free":
            if a[1] >= 2 and seen["red_read"].get(a[1] - 2, 0) < 4:
                v.append(("merge buffer rewritten early", a[1]))
            return True
        if op == "write_red":
            bump("red_written", a[1])
            return True
        if op == "read_red":
            if seen["red_written"].get(a[1], 0) < 4:
                v.append(("merge buffer read early", a[1]))
            bump("red_read", a[1])
            return True
        raise ValueError(op)

    try:
        stuck = _run(procs, step, slow=slow)
    except AssertionError as e:
        return [("phase", str(e))]
    return stuck + seen["violations"]


QWIDE_ROLES = 1 + 1 + 8 + 4


@pytest.mark.parametrize("nblk,nk", [(3, 5), (4, 9), (1, 1), (2, 16)])
def test_qwide_protocol_runs_to_the_end(nblk, nk):
    """The wide transposed forward's protocol (5 stages, 8 A slots, one
    accumulator for two units per block) runs to the end, also with each
    role held back in turn, with no early reuse."""
    assert _qwide_model(nblk, nk) == []
    for r in range(QWIDE_ROLES):
        assert _qwide_model(nblk, nk, slow=[(0, r)]) == [], r


def test_qwide_protocol_model_catches_a_planted_mistake():
    found = []
    for r in range(QWIDE_ROLES):
        found += _qwide_model(3, 5, bug="accempty_skip", slow=[(0, r)])
    assert any(f[0] == "accumulator overwritten early" for f in found), found[:3]
