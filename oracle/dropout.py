"""CPU double-precision oracle for attention with dropout on P.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle``: nothing on the product
path imports it.

What it computes.  "Efficient attention: memory-bound", section "Real code
moves even more", lists dropout among the elementwise steps a training forward
pass applies to the probabilities before the final product (scale, mask,
softmax, dropout, then P V), each a separate pass over the T x T matrix unless
fused.  Dropout with rate p keeps each probability with probability 1 - p and
scales the kept ones by 1 / (1 - p):

    O = (P * Z) V / (1 - p),      Z_ij in {0, 1},

with LSE that of the undropped row (the softmax itself is unchanged).  The
backward pass follows by the chain rule: dV = (P * Z)^T dO / (1 - p);
dP = (dO V^T) * Z / (1 - p); dS = P * (dP - D) with D_i = sum_j P_ij dP_ij
(= sum_c dO_ic O_ic, as without dropout); dQ = scale dS K; dK = scale dS^T Q.

Readings (the pages fix neither the generator nor the mask's layout):

* Z comes from a counter-based generator so that the backward pass can
  regenerate it instead of storing it: Philox-4x32-10 (Salmon, Moraes, Dror
  and Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011).  Each
  Philox block decides a 4 x 4 block of (query, key) pairs: the block of rows
  4a..4a+3 and keys 4c..4c+3 of head h of batch b uses the counter
  (a, c, b * Hq + h, offset) and the key (seed mod 2^32, seed div 2^32); its
  output word w (0..3) belongs to row 4a + w and byte j (0..3, little-endian)
  of that word to key 4c + j.  The square block lets a thread that owns a
  query row (forward) and one that owns a key row (backward) share blocks
  with three neighbours alike.
* The keep decision is 8-bit: keep iff the byte < t, t = round(256 (1 - p)),
  1 <= t <= 256, so the keep probability is exactly t / 256 and the kept
  values are scaled by 256 / t.  p is therefore used to the nearest 1/256.
* Masked (causal, window) entries have P = 0 whatever Z is.

The Philox rounds and key schedule are restated here from the paper; the same
code with the paper's 64-bit constants reproduces numpy's Philox (4x64-10)
bit generator, which pins the structure (``tests/test_oracle_dropout.py``).
"""

from __future__ import annotations

import numpy as np

from . import _kv_head, _masked_scores, _softmax_stats, _visible_keys, _PANEL_ROWS

__all__ = ["PHILOX", "philox4", "philox4x32", "keep_threshold", "dropout_keep",
           "head_forward_dropout", "head_backward_dropout",
           "attention_forward_dropout", "attention_backward_dropout"]

# (multipliers M0, M1), (Weyl key increments W0, W1) for word widths 32 and 64
PHILOX = {
    32: ((0xD2511F53, 0xCD9E8D57), (0x9E3779B9, 0xBB67AE85)),
    64: ((0xD2E7470EE14C6C93, 0xCA5A826395121157), (0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B)),
}


def philox4(counter, key, width=32, rounds=10):
    """One Philox-4xW block in pure Python integers.  Each round multiplies
    x0 and x2 by M0 and M1 into double-width products (hi, lo) and sets
    x = (hi1 ^ x1 ^ k0, lo1, hi0 ^ x3 ^ k1, lo0); the key (k0, k1) is bumped
    by (W0, W1) before every round after the first."""
    (m0, m1), (w0, w1) = PHILOX[width]
    mask = (1 << width) - 1
    x = [int(c) & mask for c in counter]
    k0, k1 = int(key[0]) & mask, int(key[1]) & mask
    for r in range(rounds):
        if r:
            k0, k1 = (k0 + w0) & mask, (k1 + w1) & mask
        p0, p1 = m0 * x[0], m1 * x[2]
        x = [(p1 >> width) ^ x[1] ^ k0, p1 & mask, (p0 >> width) ^ x[3] ^ k1, p0 & mask]
    return x


def philox4x32(c0, c1, c2, c3, k0, k1, rounds=10):
    """Philox-4x32 over arrays of counters (numpy broadcasting; the 32-bit
    products are exact in uint64).  Returns the four output words as uint64
    arrays holding 32-bit values."""
    (m0, m1), (w0, w1) = PHILOX[32]
    lo32 = np.uint64(0xFFFFFFFF)
    x0, x1, x2, x3 = (np.asarray(c, dtype=np.uint64) & lo32 for c in (c0, c1, c2, c3))
    k0, k1 = int(k0) & 0xFFFFFFFF, int(k1) & 0xFFFFFFFF
    for r in range(rounds):
        if r:
            k0, k1 = (k0 + w0) & 0xFFFFFFFF, (k1 + w1) & 0xFFFFFFFF
        p0 = x0 * np.uint64(m0)
        p1 = x2 * np.uint64(m1)
        x0, x1, x2, x3 = ((p1 >> np.uint64(32)) ^ x1 ^ np.uint64(k0), p1 & lo32,
                          (p0 >> np.uint64(32)) ^ x3 ^ np.uint64(k1), p0 & lo32)
    return x0, x1, x2, x3


def keep_threshold(p_drop: float) -> int:
    """t = round(256 (1 - p)); keep iff the random byte < t."""
    if not (0.0 <= p_drop < 1.0):
        raise ValueError("dropout rate must be in [0, 1)")
    return max(1, min(256, int(round(256.0 * (1.0 - p_drop)))))


def dropout_keep(seed: int, offset: int, bh: int, rows, cols, p_drop: float):
    """Z [len(rows), len(cols)] (bool) for the (batch, head) index
    bh = b * Hq + h, by the 4 x 4 block layout of the module header."""
    t = keep_threshold(p_drop)
    rows = np.asarray(rows, dtype=np.int64)[:, None]
    cols = np.asarray(cols, dtype=np.int64)[None, :]
    words = philox4x32(rows >> 2, cols >> 2, bh, offset, seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    w = rows & 3
    word = np.where(w == 0, words[0], np.where(w == 1, words[1], np.where(w == 2, words[2], words[3])))
    byte = (word >> (np.uint64(8) * (cols & 3).astype(np.uint64))) & np.uint64(0xFF)
    return byte < np.uint64(t)


def head_forward_dropout(qh, kh, vh, scale, causal, p_drop, seed, offset, bh, window=None):
    """One head's O with dropout on P and the undropped LSE.  Returns (O, LSE)."""
    if window is not None:
        causal = True
    Tq, Tk = qh.shape[0], kh.shape[0]
    inv_keep = 256.0 / keep_threshold(p_drop)
    O = np.zeros((Tq, vh.shape[1]))
    LSE = np.full(Tq, -np.inf)
    for r0 in range(0, Tq, _PANEL_ROWS):
        r1 = min(Tq, r0 + _PANEL_ROWS)
        nk = _visible_keys(r1, Tq, Tk, causal)
        if nk == 0:
            continue
        S = _masked_scores(qh[r0:r1], kh[:nk], r0, Tq, Tk, scale, causal, window)
        lse, P = _softmax_stats(S)
        Z = dropout_keep(seed, offset, bh, np.arange(r0, r1), np.arange(nk), p_drop)
        O[r0:r1] = ((P * Z) @ vh[:nk]) * inv_keep
        LSE[r0:r1] = lse
    return O, LSE


def head_backward_dropout(qh, kh, vh, doh, scale, causal, p_drop, seed, offset, bh, window=None):
    """One head's gradients of L = sum(dO * O) for head_forward_dropout.
    Returns (dQ, dK, dV)."""
    if window is not None:
        causal = True
    Tq, Tk = qh.shape[0], kh.shape[0]
    inv_keep = 256.0 / keep_threshold(p_drop)
    dQ, dK, dV = np.zeros_like(qh), np.zeros_like(kh), np.zeros_like(vh)
    for r0 in range(0, Tq, _PANEL_ROWS):
        r1 = min(Tq, r0 + _PANEL_ROWS)
        nk = _visible_keys(r1, Tq, Tk, causal)
        if nk == 0:
            continue
        S = _masked_scores(qh[r0:r1], kh[:nk], r0, Tq, Tk, scale, causal, window)
        _, P = _softmax_stats(S)
        Z = dropout_keep(seed, offset, bh, np.arange(r0, r1), np.arange(nk), p_drop)
        dO = doh[r0:r1]
        dV[:nk] += ((P * Z).T @ dO) * inv_keep
        dP = (dO @ vh[:nk].T) * Z * inv_keep
        D = (P * dP).sum(axis=1, keepdims=True)
        dS = P * (dP - D)
        dQ[r0:r1] = scale * (dS @ kh[:nk])
        dK[:nk] += scale * (dS.T @ qh[r0:r1])
    return dQ, dK, dV


def attention_forward_dropout(q, k, v, scale, causal, p_drop, seed, offset, window=None):
    """BTHD arrays; (batch b, query head h) uses bh = b * Hq + h."""
    B, Tq, Hq, _ = q.shape
    Hkv = k.shape[2]
    O = np.zeros(q.shape[:3] + (v.shape[3],))
    LSE = np.full((B, Hq, Tq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            g = _kv_head(h, Hq, Hkv)
            O[b, :, h], LSE[b, h] = head_forward_dropout(q[b, :, h], k[b, :, g], v[b, :, g], scale, causal,
                                                         p_drop, seed, offset, b * Hq + h, window)
    return O, LSE


def attention_backward_dropout(q, k, v, do, scale, causal, p_drop, seed, offset, window=None):
    """Gradients for attention_forward_dropout; dK, dV sum over a GQA group."""
    B, Tq, Hq, _ = q.shape
    Hkv = k.shape[2]
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            g = _kv_head(h, Hq, Hkv)
            a, bk, bv = head_backward_dropout(q[b, :, h], k[b, :, g], v[b, :, g], do[b, :, h], scale, causal,
                                              p_drop, seed, offset, b * Hq + h, window)
            dq[b, :, h] = a
            dk[b, :, g] += bk
            dv[b, :, g] += bv
    return dq, dk, dv
