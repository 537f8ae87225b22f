"""Float64 CPU oracle for the flash-CCE ORPO language-model head.

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow, obviously-correct
definition that the CUDA library is checked against.  Only the test suite,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import or call it.  It shares no code, constant table
or helper with the CUDA path (``lm_head_cross_flash_b200``), and it imports
nothing from that package.

Sources (three pages of the mlx-bun design documents):

* "Training — design (ORPO, flash-CCE head, prefix sharing, segmented
  backward)", mlx-bun 1.0.0 ``docs/design/orpo-training.md`` — cited below as
  *Training design*, with its section number.
* "ORPO training — design", mlx-bun 0.0.6 ``docs/design/orpo-training.md`` —
  cited as *ORPO design (0.0.6)*, with its section title.
* "flash-CCE host-buffer pin leak — post-mortem + L3 verification approach",
  mlx-bun 0.0.6 — cited as *Pin-leak post-mortem*.

The flash-CCE head is exact: it reaches the same numbers as the full-logits
head, only with the logits never stored (Training design §5.1, tier list;
Pin-leak post-mortem, "L3 verification approach").  So every function here is
the plain definition, with the ``[rows, V]`` logits materialised one row block
at a time in float64:

* ``head_forward``   logp_t = h_t . W_{y_t} - logsumexp_v(h_t . W_v)
  (Training design §5.1, first paragraph; ORPO design (0.0.6), "Ranked levers",
  lever 1).
* ``orpo_loss_from_logps``  L = NLL(chosen) + lambda * L_OR with
  L_OR = -log sigmoid(log_odds),
  log_odds = (lw - lr) - (log1mexp(lw) - log1mexp(lr)), lw/lr length-normalised
  response means, NLL in ``full`` or ``response`` scope (Training design §1;
  ORPO design (0.0.6), "The objective").
* ``orpo_grad_coeffs``  dL/dlogp_t, the cotangent that autograd hands the head
  (ORPO design (0.0.6), fused-head implementation spec, "ORPO-grad folding").
* ``head_dh``  dh_t = sum_v g_t (onehot_v - softmax_v) W_v, optionally with the
  coefficient filter (Training design §5.1, tier 4; ORPO design (0.0.6),
  "Backward (recompute vocab tiles from the saved LSE)").
* ``dequant_affine_q4``  4-bit affine group dequantisation w = q*scale + bias
  (Training design §5.6; ORPO design (0.0.6), "Mixed-precision quantized
  base").

Readings where the pages are silent:

* Head-row layout: rows ``[prompt_begin, prompt_end)`` are prompt positions,
  ``[chosen_begin, chosen_end)`` the chosen response, ``[rejected_begin,
  rejected_end)`` the rejected response.  A row whose label is negative is
  ignored (no loss term, zero gradient); its lse is still defined.
* ``log1mexp`` uses the two-branch form of Maechler (2012), "Accurately
  computing log(1 - exp(-|a|))": ``log(-expm1(x))`` for x > -ln 2, else
  ``log1p(-exp(x))``.  The pages' clipped form agrees wherever the clip does
  not bind; x >= 0 is outside the domain and raises.
* Coefficient filter: a softmax term with p < eps on a non-target column is
  dropped; the target column is always kept.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

LN2 = math.log(2.0)


# ----------------------------------------------------------------------------
# scalar helpers
# ----------------------------------------------------------------------------

def log1mexp(x: float) -> float:
    """log(1 - e^x) for x < 0 (Training design §1, "Implementation").

    Two-branch form of Maechler (2012): near 0 use log(-expm1(x)), far from 0
    use log1p(-exp(x)); both are exact to rounding on their branch.
    """
    x = float(x)
    if not x < 0.0:
        raise ValueError(f"log1mexp domain is x < 0, got {x!r}")
    if x > -LN2:
        return math.log(-math.expm1(x))
    return math.log1p(-math.exp(x))


def softplus(x: float) -> float:
    """log(1 + e^x), written so it neither overflows nor loses small values."""
    x = float(x)
    return max(x, 0.0) + math.log1p(math.exp(-abs(x)))


def sigmoid(x: float) -> float:
    x = float(x)
    if x >= 0:
        return 1.0 / (1.0 + math.exp(-x))
    e = math.exp(x)
    return e / (1.0 + e)


def orpo_log_odds(lw: float, lr: float) -> float:
    """log_odds = (lw - lr) - (log1mexp(lw) - log1mexp(lr)) (Training design §1)."""
    return (lw - lr) - (log1mexp(lw) - log1mexp(lr))


def combine_full_nll(n_prompt: int, pm: float, n_chosen: int, lw: float) -> float:
    """``combineFullNll``: NLL_full = -((P-1)*pm + M*lw) / ((P-1) + M).

    Training design §1, ``full`` scope.  On that page ``P-1`` is the number of
    labelled prompt positions and ``M`` the number of chosen-response tokens;
    here they are ``n_prompt`` and ``n_chosen``.
    """
    return -((n_prompt * pm + n_chosen * lw) / (n_prompt + n_chosen))


# ----------------------------------------------------------------------------
# layout
# ----------------------------------------------------------------------------

@dataclass(frozen=True)
class Layout:
    """Disjoint head-row ranges of one ORPO pair, each ``[begin, end)``."""

    prompt_begin: int
    prompt_end: int
    chosen_begin: int
    chosen_end: int
    rejected_begin: int
    rejected_end: int

    @staticmethod
    def contiguous(P: int, Rc: int, Rr: int) -> "Layout":
        return Layout(0, P, P, P + Rc, P + Rc, P + Rc + Rr)


def _segment_stats(logp: np.ndarray, labels: np.ndarray, b: int, e: int):
    sel = labels[b:e] >= 0
    n = int(sel.sum())
    s = float(np.sum(logp[b:e][sel], dtype=np.float64))
    return n, s


# ----------------------------------------------------------------------------
# head forward / backward (materialised logits, float64)
# ----------------------------------------------------------------------------

def _as64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def softcap_logits(Z, softcap: float):
    """Gemma-style logit soft-capping, cap * tanh(z / cap) (ORPO design
    (0.0.6), fused-head spec: "Gemma applies final_logit_softcapping"); a cap
    of 0 means none."""
    return Z if not softcap else softcap * np.tanh(Z / softcap)


def head_forward(H, W, labels, rows=None, block: int = 64, softcap: float = 0.0):
    """Per-row lse, target logit and logp of the LM head (Training design §5.1).

    ``H`` [M, D] and ``W`` [V, D] hold exactly the values the GPU consumes
    (bf16-rounded, or dequantised), converted to float64.  ``rows`` optionally
    restricts the computation to a subset of rows (sampled parity).  Returns
    ``(logp, lse, tgt)`` for the selected rows; ``logp`` and ``tgt`` are 0 for
    ignored rows (label < 0).  With ``softcap`` the logits are capped first
    and everything (lse, target, logp) uses the capped values.
    """
    H = _as64(H)
    W = _as64(W)
    labels = np.asarray(labels)
    idx = np.arange(H.shape[0]) if rows is None else np.asarray(rows)
    V = W.shape[0]
    n = idx.shape[0]
    lse = np.empty(n)
    tgt = np.zeros(n)
    for r0 in range(0, n, block):
        sel = idx[r0:r0 + block]
        Z = softcap_logits(H[sel] @ W.T, softcap)           # [rows, V] logits
        mx = Z.max(axis=1)
        lse[r0:r0 + len(sel)] = mx + np.log(np.exp(Z - mx[:, None]).sum(axis=1))
        y = labels[sel]
        ok = y >= 0
        if np.any(y >= V):
            raise ValueError("label >= V")
        tgt[r0:r0 + len(sel)][ok] = Z[np.nonzero(ok)[0], y[ok]]
    y = labels[idx]
    logp = np.where(y >= 0, tgt - lse, 0.0)
    return logp, lse, tgt


def head_dh(H, W, labels, coeff, lse, rows=None, filter_eps: float = 0.0,
            block: int = 64, softcap: float = 0.0):
    """dh_t = sum_v g_t (onehot(y_t)_v - p_tv) W_v, p = exp(z - lse).

    ORPO design (0.0.6), fused-head spec "Backward (recompute vocab tiles from
    the saved LSE)": the per-logit cotangent is g * (onehot - softmax), and
    dh = that . W.  ``coeff`` is g = dL/dlogp per row (0 for ignored rows).
    ``lse`` is the per-row lse of the selected rows.  With ``filter_eps`` > 0 a
    term whose softmax is below eps on a non-target column is dropped
    (Training design §5.1, "coeff filter").  With ``softcap`` the softmax is
    over the capped logits and each term carries d(capped)/d(raw) =
    1 - tanh^2(raw / cap) (the fused-head spec's "x sech^2").
    """
    H = _as64(H)
    W = _as64(W)
    labels = np.asarray(labels)
    coeff = _as64(coeff)
    idx = np.arange(H.shape[0]) if rows is None else np.asarray(rows)
    lse = _as64(lse)
    V, D = W.shape
    out = np.zeros((idx.shape[0], D))
    for r0 in range(0, idx.shape[0], block):
        sel = idx[r0:r0 + block]
        k = len(sel)
        Zr = H[sel] @ W.T
        Z = softcap_logits(Zr, softcap)
        P = np.exp(Z - lse[r0:r0 + k, None])
        y = labels[sel]
        onehot = np.zeros_like(P)
        ok = y >= 0
        onehot[np.nonzero(ok)[0], y[ok]] = 1.0
        if filter_eps > 0.0:
            drop = (P < filter_eps) & (onehot == 0.0)
            P = np.where(drop, 0.0, P)
        c = np.where(ok, coeff[sel], 0.0)
        G = c[:, None] * (onehot - P)
        if softcap:
            G = G * (1.0 - np.tanh(Zr / softcap) ** 2)
        out[r0:r0 + k] = G @ W
    return out


# ----------------------------------------------------------------------------
# ORPO objective
# ----------------------------------------------------------------------------

@dataclass
class OrpoOut:
    loss: float
    nll: float
    l_or: float
    lw: float
    lr: float
    pm: float
    z: float
    sig: float
    n_prompt: int
    n_chosen: int
    n_rejected: int

    def as8(self):
        """The eight fp64 scalars of the C-ABI output block, in its order."""
        return [self.loss, self.nll, self.l_or, self.lw, self.lr, self.pm,
                self.z, self.sig]


def orpo_loss_from_logps(logp, labels, layout: Layout, lam: float,
                         sft_scope: str = "full") -> OrpoOut:
    """``orpoLossFromLogps`` over head rows (Training design §1).

    lw, lr are length-normalised means of logp over the labelled rows of the
    chosen / rejected response; pm the mean over the labelled prompt rows.
    ``full``: NLL = -(sum_prompt + sum_chosen) / (n_prompt + n_chosen), which is
    ``combine_full_nll``; ``response``: NLL = -lw.  L = NLL + lam * L_OR.
    """
    logp = _as64(logp)
    labels = np.asarray(labels)
    L = layout
    nP, sP = _segment_stats(logp, labels, L.prompt_begin, L.prompt_end)
    nC, sC = _segment_stats(logp, labels, L.chosen_begin, L.chosen_end)
    nR, sR = _segment_stats(logp, labels, L.rejected_begin, L.rejected_end)
    if nC == 0 or nR == 0:
        raise ValueError("chosen and rejected need at least one labelled row")
    lw = sC / nC
    lr = sR / nR
    pm = sP / nP if nP > 0 else 0.0
    if sft_scope == "full":
        nll = -(sP + sC) / (nP + nC)
    elif sft_scope == "response":
        nll = -lw
    else:
        raise ValueError(sft_scope)
    z = orpo_log_odds(lw, lr)
    l_or = softplus(-z)                       # -log sigmoid(z)
    return OrpoOut(loss=nll + lam * l_or, nll=nll, l_or=l_or, lw=lw, lr=lr,
                   pm=pm, z=z, sig=sigmoid(z), n_prompt=nP, n_chosen=nC,
                   n_rejected=nR)


def orpo_grad_coeffs(logp, labels, layout: Layout, lam: float,
                     sft_scope: str = "full") -> np.ndarray:
    """g_t = dL/dlogp_t, the cotangent the head's backward receives.

    Derivation from the objective of Training design §1 (chain rule only):
    dL_OR/dz = sigmoid(z) - 1; dz/dlw = 1/(1 - e^lw) (the "1/(1-P)" factor the
    ORPO design (0.0.6) notes for the OR gradient); dz/dlr = -1/(1 - e^lr);
    dlw/dlogp_t = 1/n_chosen on chosen rows, dlr/dlogp_t = 1/n_rejected on
    rejected rows; the NLL term adds -1/(n_prompt + n_chosen) on prompt and
    chosen rows (``full``) or -1/n_chosen on chosen rows (``response``).
    Ignored rows get 0.
    """
    labels = np.asarray(labels)
    o = orpo_loss_from_logps(logp, labels, layout, lam, sft_scope)
    L = layout
    M = labels.shape[0]
    g = np.zeros(M)
    dz = o.sig - 1.0
    a_w = 1.0 / (-math.expm1(o.lw))
    a_r = 1.0 / (-math.expm1(o.lr))
    if sft_scope == "full":
        s_nll_c = s_nll_p = -1.0 / (o.n_prompt + o.n_chosen)
    else:
        s_nll_c, s_nll_p = -1.0 / o.n_chosen, 0.0
    g[L.prompt_begin:L.prompt_end] = s_nll_p
    g[L.chosen_begin:L.chosen_end] = lam * dz * a_w / o.n_chosen + s_nll_c
    g[L.rejected_begin:L.rejected_end] = -lam * dz * a_r / o.n_rejected
    g[labels < 0] = 0.0
    return g


def orpo_head_loss(H, W, labels, layout: Layout, lam: float,
                   sft_scope: str = "full", softcap: float = 0.0) -> float:
    """Scalar ORPO loss of the head as a function of H (for finite differences)."""
    logp, _, _ = head_forward(H, W, labels, softcap=softcap)
    return orpo_loss_from_logps(logp, labels, layout, lam, sft_scope).loss


def orpo_head_grad(H, W, labels, layout: Layout, lam: float,
                   sft_scope: str = "full", filter_eps: float = 0.0,
                   softcap: float = 0.0):
    """dL/dH through the head: coefficients, then ``head_dh``."""
    logp, lse, _ = head_forward(H, W, labels, softcap=softcap)
    g = orpo_grad_coeffs(logp, labels, layout, lam, sft_scope)
    return head_dh(H, W, labels, g, lse, filter_eps=filter_eps, softcap=softcap)


# ----------------------------------------------------------------------------
# 4-bit affine group quantisation (the stored head format)
# ----------------------------------------------------------------------------

def bf16_bits_to_f64(bits) -> np.ndarray:
    """Value of bfloat16 bit patterns (uint16) as float64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def dequant_affine_q4(packed, scales, biases, group: int = 64) -> np.ndarray:
    """w[v, d] = q[v, d] * scale[v, d // group] + bias[v, d // group].

    Affine 4-bit group quantisation as the head stores it (Training design
    §5.6: a vocab chunk is a row slice of ``w``/``scales``/``biases``, one
    quantisation spec per head).  ``packed`` is uint32 [V, D/8]: element
    ``8*k + j`` of a row is bits ``4j .. 4j+3`` of word ``k`` (low nibble
    first).  ``scales``/``biases`` are bfloat16 bit patterns [V, D/group].
    """
    packed = np.asarray(packed, dtype=np.uint32)
    V, W8 = packed.shape
    D = W8 * 8
    q = np.empty((V, D), dtype=np.float64)
    for j in range(8):
        q[:, j::8] = ((packed >> np.uint32(4 * j)) & np.uint32(0xF)).astype(np.float64)
    s = np.repeat(bf16_bits_to_f64(scales), group, axis=1)
    b = np.repeat(bf16_bits_to_f64(biases), group, axis=1)
    return q * s + b


# ----------------------------------------------------------------------------
# objective siblings on the same log-prob engine
# ----------------------------------------------------------------------------
#
# Training design §8.3 ("Objective variants and data") lists SimPO as a cheap
# sibling once the shared logp engine exists, and the UltraFeedback research
# notes (§6.1-6.3) define:
#   SimPO:            L = -log sigmoid(beta * (lw - lr) - gamma)   (no NLL term)
#   ORPO + margin:    L = NLL(chosen) + lambda * [-log sigmoid(beta*(lw-lr) - gamma)]
# (§6.2, the "gamma-hybrid", equal to the "SFT + SimPO single-stage" of §6.3).
# The design record writes the SimPO term as softplus(-beta((lw-lr) - gamma)),
# with gamma inside the beta product; the notes and the published SimPO loss
# (Meng et al. 2024) subtract gamma after scaling.  The latter is used here.

OBJECTIVES = ("orpo", "simpo", "orpo_margin")


def simpo_margin(lw: float, lr: float, beta: float, gamma: float) -> float:
    """u = beta * (lw - lr) - gamma; the SimPO term is softplus(-u)."""
    return beta * (lw - lr) - gamma


def pref_loss_from_logps(logp, labels, layout: Layout, kind: str, lam: float,
                         beta: float = 1.0, gamma: float = 0.0,
                         sft_scope: str = "full") -> OrpoOut:
    """Loss of one objective from per-row log-probs.

    ``orpo`` is ``orpo_loss_from_logps``.  For ``simpo`` and ``orpo_margin``
    the returned fields are: loss, nll (reported, added only by
    ``orpo_margin``), l_or = the SimPO term softplus(-u), lw, lr, pm, z = u,
    sig = sigmoid(u).
    """
    if kind == "orpo":
        return orpo_loss_from_logps(logp, labels, layout, lam, sft_scope)
    if kind not in OBJECTIVES:
        raise ValueError(kind)
    logp = _as64(logp)
    labels = np.asarray(labels)
    L = layout
    nP, sP = _segment_stats(logp, labels, L.prompt_begin, L.prompt_end)
    nC, sC = _segment_stats(logp, labels, L.chosen_begin, L.chosen_end)
    nR, sR = _segment_stats(logp, labels, L.rejected_begin, L.rejected_end)
    if nC == 0 or nR == 0:
        raise ValueError("chosen and rejected need at least one labelled row")
    lw, lr = sC / nC, sR / nR
    pm = sP / nP if nP > 0 else 0.0
    nll = -(sP + sC) / (nP + nC) if sft_scope == "full" else -lw
    u = simpo_margin(lw, lr, beta, gamma)
    term = softplus(-u)
    loss = term if kind == "simpo" else nll + lam * term
    return OrpoOut(loss=loss, nll=nll, l_or=term, lw=lw, lr=lr, pm=pm, z=u,
                   sig=sigmoid(u), n_prompt=nP, n_chosen=nC, n_rejected=nR)


def pref_grad_coeffs(logp, labels, layout: Layout, kind: str, lam: float,
                     beta: float = 1.0, gamma: float = 0.0,
                     sft_scope: str = "full") -> np.ndarray:
    """dL/dlogp of one objective (chain rule: d softplus(-u)/du = sigmoid(u) - 1,
    du/dlw = beta, du/dlr = -beta, dlw/dlogp = 1/n_chosen on chosen rows)."""
    if kind == "orpo":
        return orpo_grad_coeffs(logp, labels, layout, lam, sft_scope)
    labels = np.asarray(labels)
    o = pref_loss_from_logps(logp, labels, layout, kind, lam, beta, gamma, sft_scope)
    L = layout
    g = np.zeros(labels.shape[0])
    w = 1.0 if kind == "simpo" else lam
    d = w * (o.sig - 1.0) * beta
    if kind == "simpo":
        s_c = s_p = 0.0
    elif sft_scope == "full":
        s_c = s_p = -1.0 / (o.n_prompt + o.n_chosen)
    else:
        s_c, s_p = -1.0 / o.n_chosen, 0.0
    g[L.prompt_begin:L.prompt_end] = s_p
    g[L.chosen_begin:L.chosen_end] = d / o.n_chosen + s_c
    g[L.rejected_begin:L.rejected_end] = -d / o.n_rejected
    g[labels < 0] = 0.0
    return g


def dequant_affine_q8(packed, scales, biases, group: int = 64) -> np.ndarray:
    """8-bit affine groups: w[v, d] = q[v, d] * scale + bias, element
    ``4*k + j`` of a row in byte ``j`` of word ``k`` (low byte first);
    the 8-bit variant of the quantised head (Training design §5.1, "in-Metal
    4/8-bit affine dequant").  ``scales``/``biases``: bf16 bits [V, D/group]."""
    packed = np.asarray(packed, dtype=np.uint32)
    V, W4 = packed.shape
    D = W4 * 4
    q = np.empty((V, D), dtype=np.float64)
    for j in range(4):
        q[:, j::4] = ((packed >> np.uint32(8 * j)) & np.uint32(0xFF)).astype(np.float64)
    s = np.repeat(bf16_bits_to_f64(scales), group, axis=1)
    b = np.repeat(bf16_bits_to_f64(biases), group, axis=1)
    return q * s + b


# ----------------------------------------------------------------------------
# prefix-shared pair: head rows gathered from one concatenated forward
# ----------------------------------------------------------------------------

def prefix_gather_index(P: int, Rc: int, Rr: int) -> np.ndarray:
    """Source row of every head row for a prefix-shared pair.

    Training design §5.4: one forward over [prompt(P); chosen(Rc);
    rejected(Rr)] yields H_cat; the head gathers chosen[k] <- H_cat[P-1+k],
    rejected[0] <- H_cat[P-1], rejected[k>=1] <- H_cat[P+Rc+k-1].  The prompt
    rows of the ``full`` scope are the positions that predict the next prompt
    token, prompt row m <- H_cat[m-1].  Head row 0 (unlabelled: nothing
    predicts the first prompt token) reads H_cat[0].
    """
    M = P + Rc + Rr
    idx = np.empty(M, dtype=np.int64)
    idx[0] = 0
    idx[1:P] = np.arange(0, P - 1)                   # prompt
    idx[P:P + Rc] = P - 1 + np.arange(Rc)            # chosen[k] <- P-1+k
    idx[P + Rc] = P - 1                              # rejected[0] <- P-1
    idx[P + Rc + 1:] = P + Rc + np.arange(1, Rr) - 1  # rejected[k] <- P+Rc+k-1
    return idx


def prefix_gather(H_cat, P: int, Rc: int, Rr: int) -> np.ndarray:
    return np.asarray(H_cat)[prefix_gather_index(P, Rc, Rr)]


def prefix_scatter(dH_head, P: int, Rc: int, Rr: int) -> np.ndarray:
    """Adjoint of ``prefix_gather``: dH_cat[r] = sum of dH_head[m] over the
    head rows m that read row r (reverse mode sums the two branches'
    cotangents into the shared prefix)."""
    dH_head = _as64(dH_head)
    out = np.zeros_like(dH_head)
    np.add.at(out, prefix_gather_index(P, Rc, Rr), dH_head)
    return out


# ----------------------------------------------------------------------------
# trainable head: gradient with respect to W
# ----------------------------------------------------------------------------

def head_dw(H, W, labels, coeff, lse, filter_eps: float = 0.0, softcap: float = 0.0,
            block: int = 64) -> np.ndarray:
    """dW[v] = sum_m g_m (onehot(y_m)_v - p_mv) * cap'(s_mv) * H[m].

    The head's weight gradient for when the head stops being frozen (ORPO
    design (0.0.6), fused-head spec: explicit VJP inputs (h, baseW, ...), and
    the follow-on "head-LoRA / dC"): the same per-logit cotangent as
    ``head_dh``, contracted with H over the rows instead of with W over the
    vocabulary.  ``lse`` covers every row.
    """
    H = _as64(H)
    W = _as64(W)
    labels = np.asarray(labels)
    coeff = _as64(coeff)
    lse = _as64(lse)
    out = np.zeros_like(W)
    for r0 in range(0, H.shape[0], block):
        sel = slice(r0, r0 + block)
        Zr = H[sel] @ W.T
        Z = softcap_logits(Zr, softcap)
        P = np.exp(Z - lse[sel, None])
        y = labels[sel]
        onehot = np.zeros_like(P)
        ok = y >= 0
        onehot[np.nonzero(ok)[0], y[ok]] = 1.0
        if filter_eps > 0.0:
            P = np.where((P < filter_eps) & (onehot == 0.0), 0.0, P)
        c = np.where(ok, coeff[sel], 0.0)
        G = c[:, None] * (onehot - P)
        if softcap:
            G = G * (1.0 - np.tanh(Zr / softcap) ** 2)
        out += G.T @ H[sel]
    return out
