"""CPU double-precision oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
this package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code, header, table or helper with
the CUDA library; the only thing both sides share is the seeded input module
``workloads``, which holds no attention arithmetic.

Everything here is the plain definition written out in float64 with the score
matrix S and the probability matrix P materialised, as the standard
("Algorithm 0") formulation does.  The pages this follows, cited by title and
section:

* [MEM] "Flash Attention: Why Memory Traffic, Not Compute, Is the Bottleneck"
  (kgptalkie, day 24) -- §"The Problem Is Moving Intermediate Data" (QK^T, then
  softmax, then multiply by V), §"Softmax Looks Like an Obstacle" (running m, l,
  u and the e^{m-m'} rescale), §"Carry the Actual Values Through Both Tiles"
  (two-tile worked example), §"Causal Masks Still Apply".
* [EFF] "Efficient attention: memory-bound" (zerotofrontier) -- §"Standard
  attention, kernel by kernel" (S, then P, then O), §"Real code moves even
  more" (scale by 1/sqrt(d_k) before the softmax; the backward products dV,
  dP, dS, dQ, dK), §"The obstacle, a normalizer that needs the whole row"
  (P_ij from the row maximum and the normaliser).
* [FA] "FlashAttention" (aimlrounds interview track) -- §"Softmax without
  seeing the whole row" (online softmax, one log-sum-exp per row kept for the
  backward pass, the 8-key example), §"In practice" (GQA, causal masks,
  FlashDecoding's split of the KV cache).

Readings where the pages are silent (each is also listed in the design notes):

* scale multiplies QK^T before the softmax; LSE is the natural log of
  sum_j exp(S_ij) of the *scaled* scores;
* causal rule: key j is visible to query i iff j <= i + (Tk - Tq)
  (bottom-right alignment; for Tq == Tk this is the pages' j <= i);
* a row that sees no key (causal with Tq > Tk, or Tk == 0) has O = 0,
  LSE = -inf and zero gradients;
* GQA maps query head h to KV head h // (Hq // Hkv) (contiguous groups);
* D_i of the backward pass is sum_j P_ij dP_ij (the softmax Jacobian), not the
  rowsum(dO*O) shortcut the kernels use;
* sliding window ([FA §"In practice"] names "sliding windows" next to GQA and
  causal masks, without a definition): a causal local window of W >= 1 keys,
  query i sees key j iff i + (Tk - Tq) - W < j <= i + (Tk - Tq), i.e. its own
  diagonal key and the W - 1 keys before it.  W >= Tk is the causal mask.

The FP8 forward (FlashAttention-3's low-precision path, named in [FA §"In
practice"]) is checked against ``attention_forward_e4m3``: exact attention on
the dequantised E4M3 inputs.  E4M3 is decoded here from the format's
published definition (the OCP 8-bit floating-point specification, "FP8
Formats for Deep Learning", Micikevicius et al. 2022), not by a library.

Layouts follow the library: q, o, dq are [B, Tq, Hq, d]; k, v, dk, dv are
[B, Tk, Hkv, d]; lse is [B, Hq, Tq].  All arrays are float64.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "causal_visible",
    "window_visible",
    "head_forward",
    "head_backward",
    "attention_forward",
    "attention_backward",
    "decode_forward",
    "online_softmax_row",
    "combine_partials",
    "merge_partials",
    "e4m3_value",
    "e4m3_decode",
    "attention_forward_e4m3",
    "brute_force_row",
]

# Rows of Q processed at once.  Each row's softmax always sees the whole key
# row, so the panel size changes memory use only, never the arithmetic.
_PANEL_ROWS = 2048


def causal_visible(i: int, j, Tq: int, Tk: int):
    """Causal rule [MEM §"Causal Masks Still Apply"]: query i sees key j iff
    j <= i + (Tk - Tq).  For Tq == Tk this is "position 3 uses columns 0..3"."""
    return j <= i + (Tk - Tq)


def window_visible(i, j, Tq: int, Tk: int, window: int):
    """Sliding-window rule (reading of [FA §"In practice"]): the causal rule
    plus j > i + (Tk - Tq) - window, so each query sees its `window` most
    recent keys, its diagonal key included."""
    off = Tk - Tq
    return (j <= i + off) & (j > i + off - window)


def _visible(i, j, Tq: int, Tk: int, causal: bool, window):
    if window is not None:
        return window_visible(i, j, Tq, Tk, window)
    return causal_visible(i, j, Tq, Tk)


def _kv_head(h: int, Hq: int, Hkv: int) -> int:
    """GQA head map (reading of [FA §"In practice"]): contiguous groups."""
    return h // (Hq // Hkv)


def _visible_keys(r1: int, Tq: int, Tk: int, causal: bool) -> int:
    """Number of leading keys that any row < r1 can see.  Keys beyond it are
    masked for every row of the panel, so their probabilities are exactly 0."""
    if not causal:
        return Tk
    return max(0, min(Tk, (r1 - 1) + (Tk - Tq) + 1))


def _masked_scores(qp, kh, r0, Tq, Tk, scale, causal, window=None):
    """S = scale * Q K^T for query rows r0.. of the panel [EFF §"Standard
    attention, kernel by kernel", step 1], with masked entries set to -inf."""
    S = scale * (qp @ kh.T)
    if causal or window is not None:
        rows = np.arange(r0, r0 + qp.shape[0])[:, None]
        cols = np.arange(kh.shape[0])[None, :]
        S = np.where(_visible(rows, cols, Tq, Tk, causal, window), S, -np.inf)
    return S


def _softmax_stats(S):
    """Row maximum m, log-sum-exp and P = exp(S - LSE)
    [EFF §"The obstacle, a normalizer that needs the whole row"]."""
    m = S.max(axis=1) if S.shape[1] else np.full(S.shape[0], -np.inf)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    with np.errstate(invalid="ignore"):
        e = np.exp(S - m_safe[:, None])
    e[~finite] = 0.0
    l = e.sum(axis=1)
    with np.errstate(divide="ignore"):
        lse = np.where(finite, m_safe + np.log(np.where(finite, l, 1.0)), -np.inf)
    P = np.where(finite[:, None], e / np.where(finite, l, 1.0)[:, None], 0.0)
    return lse, P


def head_forward(qh, kh, vh, scale: float, causal: bool, rows=None, window=None):
    """One head: O = softmax(scale * Q K^T [+ mask]) V and LSE per row.

    qh [Tq, d], kh/vh [Tk, d].  ``rows`` optionally restricts the output to a
    subset of query rows (each row is independent, so this is the same
    definition evaluated only where asked).  ``window`` (an int >= 1, or
    None) applies the sliding-window rule, which includes the causal one.
    Returns (O [n, d], LSE [n]).
    """
    if window is not None:
        causal = True
    Tq, Tk = qh.shape[0], kh.shape[0]
    if rows is None:
        rows = np.arange(Tq)
    rows = np.asarray(rows, dtype=np.int64)
    O = np.zeros((len(rows), vh.shape[1]))
    LSE = np.full(len(rows), -np.inf)
    for p0 in range(0, len(rows), _PANEL_ROWS):
        sel = rows[p0:p0 + _PANEL_ROWS]
        nk = _visible_keys(int(sel.max()) + 1, Tq, Tk, causal) if len(sel) else 0
        S = scale * (qh[sel] @ kh[:nk].T)
        if causal:
            S = np.where(_visible(sel[:, None], np.arange(nk)[None, :], Tq, Tk, causal, window), S, -np.inf)
        lse, P = _softmax_stats(S)
        O[p0:p0 + len(sel)] = P @ vh[:nk]          # step 3: O = P V
        LSE[p0:p0 + len(sel)] = lse
    return O, LSE


def head_backward(qh, kh, vh, doh, scale: float, causal: bool, window=None):
    """One head's gradients of L = sum(dO * O) [EFF §"Real code moves even
    more", the backward products]: dV = P^T dO, dP = dO V^T,
    dS = P * (dP - D) with D_i = sum_j P_ij dP_ij, dQ = scale dS K,
    dK = scale dS^T Q.  ``window`` as in head_forward.
    Returns (dQ [Tq,d], dK [Tk,d], dV [Tk,d])."""
    if window is not None:
        causal = True
    Tq, Tk = qh.shape[0], kh.shape[0]
    dQ = np.zeros_like(qh)
    dK = np.zeros_like(kh)
    dV = np.zeros_like(vh)
    for r0 in range(0, Tq, _PANEL_ROWS):
        r1 = min(Tq, r0 + _PANEL_ROWS)
        nk = _visible_keys(r1, Tq, Tk, causal)
        if nk == 0:
            continue
        S = _masked_scores(qh[r0:r1], kh[:nk], r0, Tq, Tk, scale, causal, window)
        _, P = _softmax_stats(S)
        dO = doh[r0:r1]
        dV[:nk] += P.T @ dO
        dP = dO @ vh[:nk].T
        D = (P * dP).sum(axis=1, keepdims=True)
        dS = P * (dP - D)
        dQ[r0:r1] = scale * (dS @ kh[:nk])
        dK[:nk] += scale * (dS.T @ qh[r0:r1])
    return dQ, dK, dV


def attention_forward(q, k, v, scale: float, causal: bool, window=None):
    """Batched, multi-head (GQA) forward over BTHD arrays (``window`` as in
    head_forward).  Returns O [B,Tq,Hq,d] and LSE [B,Hq,Tq]."""
    B, Tq, Hq, d = q.shape
    Hkv = k.shape[2]
    O = np.zeros((B, Tq, Hq, v.shape[3]))
    LSE = np.zeros((B, Hq, Tq))
    for b in range(B):
        for h in range(Hq):
            g = _kv_head(h, Hq, Hkv)
            O[b, :, h], LSE[b, h] = head_forward(q[b, :, h], k[b, :, g], v[b, :, g], scale, causal,
                                                 window=window)
    return O, LSE


def attention_backward(q, k, v, do, scale: float, causal: bool, window=None):
    """Batched gradients; dK and dV of a KV head sum over its query heads."""
    B, Tq, Hq, d = q.shape
    Hkv = k.shape[2]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            g = _kv_head(h, Hq, Hkv)
            a, bk, bv = head_backward(q[b, :, h], k[b, :, g], v[b, :, g], do[b, :, h], scale, causal, window)
            dq[b, :, h] = a
            dk[b, :, g] += bk
            dv[b, :, g] += bv
    return dq, dk, dv


def e4m3_value(code: int) -> float:
    """Value of one E4M3 byte: bit 7 the sign, bits 3-6 the exponent field E
    (bias 7), bits 0-2 the mantissa field M.  E > 0: (1 + M/8) * 2^(E - 7);
    E = 0: subnormal (M/8) * 2^-6; E = 15 with M = 7 is NaN (the format has
    no infinities, so E = 15 with M < 7 are ordinary values up to 448)."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_E4M3_TABLE = None


def e4m3_decode(codes):
    """Element-wise ``e4m3_value`` of an array of E4M3 bytes (uint8)."""
    global _E4M3_TABLE
    if _E4M3_TABLE is None:
        _E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
    return _E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def attention_forward_e4m3(q8, k8, v8, q_descale, k_descale, v_descale, scale: float, causal: bool):
    """Exact attention on E4M3 inputs: each tensor's values are its decoded
    codes times its descale factor; then ``attention_forward``.  q8, k8, v8
    are uint8 code arrays in the library's layouts."""
    q = e4m3_decode(q8) * float(q_descale)
    k = e4m3_decode(k8) * float(k_descale)
    v = e4m3_decode(v8) * float(v_descale)
    return attention_forward(q, k, v, scale, causal)


def decode_forward(q, k_cache, v_cache, seqlens, scale: float, pairs=None, window=None):
    """One query token per sequence over the first seqlens[b] cached keys
    [FA §"In practice", FlashDecoding]: the unmasked forward with Tq = 1 (the
    query is the sequence's last position, so with a ``window`` it sees the
    last ``window`` keys).

    q [B,Hq,d]; caches [B,Tk_max,Hkv,d].  ``pairs`` optionally restricts the
    evaluation to a list of (b, h).  Returns O [B,Hq,d], LSE [B,Hq] (entries
    not in ``pairs`` are left at 0 / -inf)."""
    B, Hq, d = q.shape
    Hkv = k_cache.shape[2]
    O = np.zeros((B, Hq, v_cache.shape[3]))
    LSE = np.full((B, Hq), -np.inf)
    todo = pairs if pairs is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in todo:
        n = int(seqlens[b])
        g = _kv_head(h, Hq, Hkv)
        o, lse = head_forward(q[b, h][None, :], k_cache[b, :n, g], v_cache[b, :n, g], scale, False,
                              window=window)
        O[b, h], LSE[b, h] = o[0], lse[0]
    return O, LSE


def online_softmax_row(scores, values, tile: int):
    """The online softmax over one row, tile by tile, in the pages' notation
    [MEM §"Softmax Looks Like an Obstacle"; FA §"Softmax without seeing the
    whole row"]: keep m (largest score so far), l (sum of exponentials
    relative to m) and u (value-weighted sum); when a tile raises the maximum
    to m', multiply both l and u by e^{m - m'} before adding the tile's
    terms.  The output is u / l.

    ``values`` is [n] or [n, dv].  Returns (u/l, m + ln l, history) where
    history lists (m, l, u, u/l) after each tile."""
    s = [float(x) for x in scores]
    vals = np.asarray(values, dtype=np.float64)
    m = -math.inf
    l = 0.0
    u = np.zeros(vals.shape[1:]) if vals.ndim > 1 else 0.0
    history = []
    for t0 in range(0, len(s), tile):
        ts = s[t0:t0 + tile]
        m_new = max([m] + ts)
        corr = math.exp(m - m_new) if m != -math.inf else 0.0
        l = corr * l + sum(math.exp(x - m_new) for x in ts)
        u = corr * u + sum(math.exp(x - m_new) * vals[t0 + i] for i, x in enumerate(ts))
        m = m_new
        history.append((m, l, u, u / l))
    return u / l, m + math.log(l), history


def combine_partials(o_parts, lse_parts):
    """Split-KV combine [FA §"In practice", FlashDecoding]: chunk c holds its
    normalised output O_c and its log-sum-exp LSE_c.  Then
    LSE = log sum_c exp(LSE_c) and O = sum_c exp(LSE_c - LSE) O_c -- the same
    e^{m - m'} algebra as the online softmax, applied to whole chunks."""
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    o_parts = np.asarray(o_parts, dtype=np.float64)
    m = lse_parts.max()
    if not np.isfinite(m):
        return np.zeros(o_parts.shape[1:]), -np.inf
    w = np.exp(lse_parts - m)
    lse = m + math.log(w.sum())
    return (np.exp(lse_parts - lse)[:, None] * o_parts).sum(axis=0), lse


def merge_partials(o_parts, lse_parts):
    """Row-wise combine of R partial results of the same rows, e.g. decodes
    of R disjoint shares of every sequence's keys on R devices (FlashDecoding's
    split [FA §"In practice"] across devices).  o_parts [R, ..., d],
    lse_parts [R, ...]; each row is merged by ``combine_partials``.  Returns
    O [..., d], LSE [...]."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    R = lse_parts.shape[0]
    rows = lse_parts.reshape(R, -1)
    orows = o_parts.reshape(R, rows.shape[1], o_parts.shape[-1])
    O = np.zeros(orows.shape[1:])
    LSE = np.empty(rows.shape[1])
    for i in range(rows.shape[1]):
        O[i], LSE[i] = combine_partials(orows[:, i], rows[:, i])
    return O.reshape(o_parts.shape[1:]), LSE.reshape(lse_parts.shape[1:])


def brute_force_row(scores, values):
    """Softmax-weighted average of one row, term by term in pure Python:
    exp(s_j - max) / sum exp(s_k - max).  For tiny cases only."""
    mx = max(scores)
    w = [math.exp(x - mx) for x in scores]
    tot = sum(w)
    out = sum(wi * vi for wi, vi in zip(w, values)) / tot
    return out, mx + math.log(tot)
