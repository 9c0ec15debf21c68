"""Float64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` call it.  It shares no code with the CUDA library.

What it computes (the plain definition, materialised, in float64):

* Forward -- "FlashAttention" blog (ruizhehou.github.io), section 1 (standard
  attention): S = Q K^T / sqrt(d), P = softmax(S), O = P V, with the
  max-subtracted ("safe") softmax of section 2.2.  The CSDN FlashAttention-1
  tutorial, section 1, gives the same formula softmax(Q K^T / sqrt(d_k)) V.
  The scale is a parameter (1/sqrt(d) in every workload); the causal mask is
  the ``is_causal=True`` option of ``F.scaled_dot_product_attention`` quoted
  in the blog's section 5 (top-left aligned: key j is masked for query i when
  j > i).
* Saved statistic -- the blog's section 2.3 keeps m and l per row; this oracle
  returns the single per-row log-sum-exp L = m + ln(l) of the scaled scores,
  natural log.
* Backward -- the FlashAttention blog (section 2.3) only says that P is
  recomputed from Q, K and the saved statistics.  The gradients below are the
  calculus of the forward definition for the scalar f = sum(O * dO):
      dV = P^T dO,  dP = dO V^T,  D_i = sum_j P_ij dP_ij (= sum_d dO_id O_id),
      dS = P * (dP - D),  dQ = scale * dS K,  dK = scale * dS^T Q.
  Pinned by central finite differences and a library cross-check in tests.
* Grouped-query attention (GQA, named in the wiki's FlashAttention-2 history):
  query head h reads key/value head floor(h / g), g = Hq / Hkv; dK and dV of a
  key/value head sum over the g query heads of its group.
* Causal alignment when Nq < Nk (inference: the Nq queries are the last Nq
  positions of a sequence whose Nk keys are all cached) -- the blog and the
  CSDN tutorial only use Nq = Nk.  Reading adopted: bottom-right alignment,
  key j is masked for query i when j > i + (Nk - Nq); it equals the top-left
  mask when Nq = Nk.
  Selected with ``causal_offset = Nk - Nq``; the default 0 is top-left.
* Split-KV forward and the merge of partial results -- the key range of a
  row is cut into pieces, each piece gives (O_s, L_s) over its own keys, and
  the pieces are combined with the same rescaling identity that the online
  softmax of blog section 2.2 uses to combine two blocks' statistics:
      L = log sum_s exp(L_s),   O = sum_s exp(L_s - L) O_s.
  A piece that sees no key of a row has L_s = -inf and contributes nothing.
* Dropout on P (the blog's section 5 call passes dropout_p to
  F.scaled_dot_product_attention with 0).  Reading adopted: inverted
  dropout of the normalised probabilities, O = (P * Z) V / (1 - p) with
  Z_ij in {0, 1}, while L stays the log-sum-exp of the undropped scores.  The
  mask is a pure function of (seed, offset, batch*Hq + head, i, j): the
  counter-based generator Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
  "Parallel random numbers: as easy as 1, 2, 3", SC 2011) with key
  (seed mod 2^32, seed >> 32) and counter (j >> 2, i, b*Hq + h, offset mod
  2^32); output word j mod 4 is compared with floor(p * 2^32) and the element
  is kept when the word is not smaller.  Backward of f = sum(O * dO):
      dV = (P*Z)^T dO / (1-p),  dP = (dO V^T) * Z / (1-p),
      D_i = sum_j P_ij dP_ij (= sum_d dO_id O_id),  dS = P * (dP - D).
* Block-wise forms -- the online-softmax step of blog section 2.2 (normalise at
  every block, "v1") and the deferred-normalisation loop of blog section 4.1
  and the CSDN tutorial section 3 ("v2": keep O unnormalised, rescale by
  exp(m_old - m_new), divide by l once).  They exist so tests can show the
  recurrences equal the one-shot softmax; they are never the reference values.

Parity: every function here is pinned by tests/test_oracle.py (closed forms,
invariants, finite differences, torch float64 SDPA cross-check, a hand-worked
golden fixture).  No function is "parity unpinned".

Layout: dense [B, H, N, d] arrays (d fastest), any float dtype on input; all
arithmetic in float64.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "scores",
    "probs",
    "forward",
    "backward",
    "forward_rows",
    "lse_rows",
    "backward_rows",
    "backward_kv_rows",
    "blockwise_forward_v1",
    "blockwise_forward_v2",
    "merge_partials",
    "splitkv_forward",
    "philox4x32_10",
    "dropout_keep",
    "dropout_forward",
    "dropout_backward",
    "dropout_forward_rows",
    "dropout_backward_rows",
    "dropout_backward_kv_rows",
]


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def _kv_head(h: int, hq: int, hkv: int) -> int:
    """GQA mapping: query head h reads key/value head floor(h / g)."""
    if hq % hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return h // (hq // hkv)


def _causal_mask(nq: int, nk: int, offset: int = 0) -> np.ndarray:
    """True where key j is hidden from query i: j > i + offset (offset 0:
    top-left alignment; offset Nk - Nq: bottom-right)."""
    i = np.arange(nq)[:, None]
    j = np.arange(nk)[None, :]
    return j > i + offset


def scores(q2, k2, scale, causal, causal_offset=0):
    """Masked scaled scores S = scale * q k^T for one head; masked entries -inf.

    Standard attention, blog section 1; causal mask per blog section 5."""
    s = scale * (_f64(q2) @ _f64(k2).T)
    if causal:
        s = np.where(_causal_mask(s.shape[0], s.shape[1], causal_offset), -np.inf, s)
    return s


def probs(q2, k2, scale, causal, causal_offset=0):
    """P = softmax(S) row-wise, max-subtracted (blog section 2.2)."""
    s = scores(q2, k2, scale, causal, causal_offset)
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=1, keepdims=True)


def _head_forward(q2, k2, v2, scale, causal, causal_offset=0):
    s = scores(q2, k2, scale, causal, causal_offset)
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    p = e / l
    o = p @ _f64(v2)
    lse = (m + np.log(l))[:, 0]
    return o, lse, p


def forward(q, k, v, scale, causal, causal_offset=0):
    """O = softmax(scale * Q K^T [+ causal mask]) V and L = logsumexp per row.

    q: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d].  Returns (o [B,Hq,Nq,d],
    lse [B,Hq,Nq]) in float64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Nq, d = q.shape
    Hkv = k.shape[1]
    o = np.empty((B, Hq, Nq, v.shape[3]))
    lse = np.empty((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            kh = _kv_head(h, Hq, Hkv)
            o[b, h], lse[b, h], _ = _head_forward(q[b, h], k[b, kh], v[b, kh], scale, causal,
                                                  causal_offset)
    return o, lse


def backward(q, k, v, do, scale, causal):
    """Gradients of f = sum(O * dO) with respect to Q, K, V.

    P is rebuilt from the definition (not taken from the caller).  Returns
    (dq, dk, dv, D) with D = rowsum(P * dP) [B, Hq, Nq]."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Hq, Nq, d = q.shape
    Hkv = k.shape[1]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dsum = np.empty((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            kh = _kv_head(h, Hq, Hkv)
            _, _, p = _head_forward(q[b, h], k[b, kh], v[b, kh], scale, causal)
            dp = do[b, h] @ v[b, kh].T
            D = np.sum(p * dp, axis=1)
            ds = p * (dp - D[:, None])
            dq[b, h] = scale * (ds @ k[b, kh])
            dk[b, kh] += scale * (ds.T @ q[b, h])
            dv[b, kh] += p.T @ do[b, h]
            dsum[b, h] = D
    return dq, dk, dv, dsum


# ---------------------------------------------------------------------------
# Row-subset forms for full-size workloads.  Attention rows are independent
# (row i of O and L depends on q_i and all of K, V only), so these are the
# same definition restricted to chosen rows / columns, evaluated in row chunks
# so an N x N matrix never has to exist at once.
# ---------------------------------------------------------------------------

def _row_chunk_scores(q2, k2, scale, causal, rows, causal_offset=0):
    s = scale * (_f64(q2)[rows] @ _f64(k2).T)
    if causal:
        s = np.where(np.arange(k2.shape[0])[None, :] > np.asarray(rows)[:, None] + causal_offset,
                     -np.inf, s)
    return s


def forward_rows(q2, k2, v2, scale, causal, rows, causal_offset=0):
    """O and L for the given query rows of one head (q2 [Nq,d], k2/v2 [Nk,d])."""
    rows = np.asarray(rows)
    s = _row_chunk_scores(q2, k2, scale, causal, rows, causal_offset)
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    return (e / l) @ _f64(v2), (m + np.log(l))[:, 0]


def lse_rows(q2, k2, scale, causal, rows, chunk=2048):
    """L for the given rows, evaluated chunk by chunk."""
    rows = np.asarray(rows)
    out = np.empty(len(rows))
    for c in range(0, len(rows), chunk):
        r = rows[c:c + chunk]
        s = _row_chunk_scores(q2, k2, scale, causal, r)
        m = np.max(s, axis=1, keepdims=True)
        out[c:c + chunk] = (m + np.log(np.sum(np.exp(s - m), axis=1, keepdims=True)))[:, 0]
    return out


def backward_rows(q2, k2, v2, do2, scale, causal, rows):
    """dQ for the given query rows of one head.

    Row i of dS = P_i * (dP_i - D_i) needs only row i of P and dP, so dQ_i is
    local to the row.  Returns (dq_rows, D_rows)."""
    rows = np.asarray(rows)
    s = _row_chunk_scores(q2, k2, scale, causal, rows)
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    p = e / np.sum(e, axis=1, keepdims=True)
    dp = _f64(do2)[rows] @ _f64(v2).T
    D = np.sum(p * dp, axis=1)
    ds = p * (dp - D[:, None])
    return scale * (ds @ _f64(k2)), D


def backward_kv_rows(q_heads, k2, v2, do_heads, scale, causal, kv_rows, chunk=2048):
    """dK and dV for chosen key/value rows of one key/value head.

    q_heads, do_heads: lists of the [Nq, d] query / output-gradient matrices of
    the g query heads that read this key/value head.  Column j of P needs L_i
    and D_i of every query row; both are per-row quantities computed here from
    full rows, chunk by chunk.  Returns (dk_rows, dv_rows) summed over the
    group."""
    kv_rows = np.asarray(kv_rows)
    k2, v2 = _f64(k2), _f64(v2)
    dk = np.zeros((len(kv_rows), k2.shape[1]))
    dv = np.zeros((len(kv_rows), v2.shape[1]))
    for q2, do2 in zip(q_heads, do_heads):
        q2, do2 = _f64(q2), _f64(do2)
        nq = q2.shape[0]
        for c in range(0, nq, chunk):
            r = np.arange(c, min(c + chunk, nq))
            s = _row_chunk_scores(q2, k2, scale, causal, r)
            m = np.max(s, axis=1, keepdims=True)
            e = np.exp(s - m)
            p = e / np.sum(e, axis=1, keepdims=True)
            dp = do2[r] @ v2.T
            D = np.sum(p * dp, axis=1)
            pj = p[:, kv_rows]                      # [rows, J]
            dsj = pj * (dp[:, kv_rows] - D[:, None])
            dv += pj.T @ do2[r]
            dk += scale * (dsj.T @ q2[r])
    return dk, dv


# ---------------------------------------------------------------------------
# Block-wise recurrences (self-checks only).
# ---------------------------------------------------------------------------

def blockwise_forward_v1(q2, k2, v2, scale, causal, block):
    """Online softmax that renormalises O at every key block (blog section 2.2:
    O_new = (e^{m_prev - m_new} l_prev O_prev + e^{S - m_new} V) / l_new)."""
    q2, k2, v2 = _f64(q2), _f64(k2), _f64(v2)
    nq, nk = q2.shape[0], k2.shape[0]
    o = np.zeros((nq, v2.shape[1]))
    l = np.zeros((nq, 1))
    m = np.full((nq, 1), -np.inf)
    for j0 in range(0, nk, block):
        j1 = min(j0 + block, nk)
        s = scale * (q2 @ k2[j0:j1].T)
        if causal:
            s = np.where(np.arange(j0, j1)[None, :] > np.arange(nq)[:, None], -np.inf, s)
        m_new = np.maximum(m, np.max(s, axis=1, keepdims=True))
        # rows whose every key so far is masked keep m = -inf; guard the
        # factor e^{(-inf) - (-inf)} to 0 (nothing accumulated yet)
        alpha = np.where(np.isneginf(m_new), 0.0, np.exp(m - np.where(np.isneginf(m_new), 0.0, m_new)))
        e = np.where(np.isneginf(s), 0.0, np.exp(s - np.where(np.isneginf(m_new), 0.0, m_new)))
        l_new = alpha * l + np.sum(e, axis=1, keepdims=True)
        with np.errstate(invalid="ignore", divide="ignore"):
            o = np.where(l_new > 0, (alpha * l * o + e @ v2[j0:j1]) / np.where(l_new > 0, l_new, 1.0), 0.0)
        m, l = m_new, l_new
    return o, (m + np.log(l))[:, 0]


def blockwise_forward_v2(q2, k2, v2, scale, causal, block):
    """Deferred normalisation (blog section 4.1 "v2"; CSDN tutorial section 3):
    O~ <- e^{m - m_new} O~ + e^{S - m_new} V,  l <- e^{m - m_new} l + rowsum,
    and one final O = O~ / l."""
    q2, k2, v2 = _f64(q2), _f64(k2), _f64(v2)
    nq, nk = q2.shape[0], k2.shape[0]
    o_t = np.zeros((nq, v2.shape[1]))
    l = np.zeros((nq, 1))
    m = np.full((nq, 1), -np.inf)
    for j0 in range(0, nk, block):
        j1 = min(j0 + block, nk)
        s = scale * (q2 @ k2[j0:j1].T)
        if causal:
            s = np.where(np.arange(j0, j1)[None, :] > np.arange(nq)[:, None], -np.inf, s)
        m_new = np.maximum(m, np.max(s, axis=1, keepdims=True))
        safe = np.where(np.isneginf(m_new), 0.0, m_new)
        alpha = np.where(np.isneginf(m_new), 0.0, np.exp(m - safe))
        e = np.where(np.isneginf(s), 0.0, np.exp(s - safe))
        o_t = alpha * o_t + e @ v2[j0:j1]
        l = alpha * l + np.sum(e, axis=1, keepdims=True)
        m = m_new
    return o_t / l, (m + np.log(l))[:, 0]


# ---------------------------------------------------------------------------
# Split-KV forward: partial results over key ranges, merged by their LSE.
# ---------------------------------------------------------------------------

def merge_partials(o_parts, lse_parts):
    """Combine per-piece results of the same rows.

    o_parts [S, ..., d] holds each piece's normalised output over its own keys,
    lse_parts [S, ...] its log-sum-exp (-inf where the piece sees no key of the
    row).  Returns (o, lse) with lse = log sum_s exp(lse_s) and
    o = sum_s exp(lse_s - lse) o_s (the block-combination identity of blog
    section 2.2, applied to normalised pieces)."""
    o_parts, lse_parts = _f64(o_parts), _f64(lse_parts)
    m = np.max(lse_parts, axis=0)
    safe = np.where(np.isneginf(m), 0.0, m)
    w = np.where(np.isneginf(lse_parts), 0.0, np.exp(lse_parts - safe))
    tot = np.sum(w, axis=0)
    lse = safe + np.log(tot)
    o = np.sum(w[..., None] * o_parts, axis=0) / tot[..., None]
    return o, lse


def splitkv_forward(q, k, v, scale, causal, bounds, causal_offset=0):
    """Forward by pieces of the key range, then merge_partials.

    bounds: increasing key indices [0 = b_0, b_1, ..., b_S = Nk]; piece s covers
    keys [b_s, b_{s+1}).  Returns (o, lse, o_parts, lse_parts).  Each piece is
    the plain definition restricted to its keys (rows with no visible key in a
    piece get lse = -inf and o = 0)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    S = len(bounds) - 1
    o_parts = np.zeros((S, B, Hq, Nq, v.shape[3]))
    lse_parts = np.full((S, B, Hq, Nq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            kh = _kv_head(h, Hq, Hkv)
            s_full = scores(q[b, h], k[b, kh], scale, causal, causal_offset)
            for p_ in range(S):
                j0, j1 = bounds[p_], bounds[p_ + 1]
                sp = s_full[:, j0:j1]
                if sp.shape[1] == 0:
                    continue
                m = np.max(sp, axis=1, keepdims=True)
                live = ~np.isneginf(m[:, 0])
                safe = np.where(np.isneginf(m), 0.0, m)
                e = np.where(np.isneginf(sp), 0.0, np.exp(sp - safe))
                l = np.sum(e, axis=1, keepdims=True)
                with np.errstate(invalid="ignore", divide="ignore"):
                    op = np.where(live[:, None], (e @ v[b, kh, j0:j1]) / np.where(l > 0, l, 1.0), 0.0)
                    lp = np.where(live, (safe + np.log(np.where(l > 0, l, 1.0)))[:, 0], -np.inf)
                o_parts[p_, b, h] = op
                lse_parts[p_, b, h] = lp
    o, lse = merge_partials(o_parts, lse_parts)
    return o, lse, o_parts, lse_parts


# ---------------------------------------------------------------------------
# Dropout: Philox4x32-10 mask, forward and backward with the mask applied.
# ---------------------------------------------------------------------------

_PHILOX_M = (0xD2511F53, 0xCD9E8D57)      # round multipliers
_PHILOX_W = (0x9E3779B9, 0xBB67AE85)      # key increments (golden ratio, sqrt(3) - 1)
_U32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32 with 10 rounds, elementwise over arrays of 32-bit counters.

    One round maps (c0, c1, c2, c3) to
        (hi(M1*c2) ^ c1 ^ k0, lo(M1*c2), hi(M0*c0) ^ c3 ^ k1, lo(M0*c0))
    and the key is then advanced by (W0, W1) modulo 2^32.  Returns the four
    output words as uint64 arrays holding 32-bit values."""
    c = [np.asarray(x, dtype=np.uint64) & _U32 for x in (c0, c1, c2, c3)]
    k0 = np.uint64(int(k0) & 0xFFFFFFFF)
    k1 = np.uint64(int(k1) & 0xFFFFFFFF)
    m0, m1 = np.uint64(_PHILOX_M[0]), np.uint64(_PHILOX_M[1])
    for _ in range(10):
        p0 = m0 * c[0]
        p1 = m1 * c[2]
        c = [((p1 >> np.uint64(32)) ^ c[1] ^ k0) & _U32, p1 & _U32,
             ((p0 >> np.uint64(32)) ^ c[3] ^ k1) & _U32, p0 & _U32]
        k0 = (k0 + np.uint64(_PHILOX_W[0])) & _U32
        k1 = (k1 + np.uint64(_PHILOX_W[1])) & _U32
    return c


def dropout_keep(bh, rows, cols, p, seed, offset):
    """Keep mask Z [len(rows), len(cols)] of head index bh = b*Hq + h."""
    rows = np.asarray(rows, dtype=np.uint64)[:, None]
    cols = np.asarray(cols, dtype=np.uint64)[None, :]
    words = philox4x32_10(cols >> np.uint64(2), rows, np.uint64(bh), np.uint64(int(offset) & 0xFFFFFFFF),
                          int(seed) & 0xFFFFFFFF, int(seed) >> 32)
    pick = (cols & np.uint64(3)) + np.zeros_like(rows)
    w = np.choose(pick.astype(np.int64), words)
    thr = np.uint64(int(np.floor(np.float64(p) * 4294967296.0)))
    return w >= thr


def _head_probs(q2, k2, scale, causal, rows=None, causal_offset=0):
    if rows is None:
        s = scores(q2, k2, scale, causal, causal_offset)
    else:
        s = _row_chunk_scores(q2, k2, scale, causal, rows, causal_offset)
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    return e / l, (m + np.log(l))[:, 0]


def dropout_forward(q, k, v, scale, causal, p, seed, offset):
    """O = (P * Z) V / (1 - p), L = logsumexp of the undropped scores."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    o = np.empty((B, Hq, Nq, v.shape[3]))
    lse = np.empty((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            kh = _kv_head(h, Hq, Hkv)
            pr, lse[b, h] = _head_probs(q[b, h], k[b, kh], scale, causal)
            z = dropout_keep(b * Hq + h, np.arange(Nq), np.arange(Nk), p, seed, offset)
            o[b, h] = (pr * z) @ v[b, kh] / (1.0 - p)
    return o, lse


def dropout_backward(q, k, v, do, scale, causal, p, seed, offset):
    """Gradients of f = sum(O * dO) for dropout_forward; returns (dq, dk, dv, D)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dsum = np.empty((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            kh = _kv_head(h, Hq, Hkv)
            pr, _ = _head_probs(q[b, h], k[b, kh], scale, causal)
            z = dropout_keep(b * Hq + h, np.arange(Nq), np.arange(Nk), p, seed, offset)
            dv[b, kh] += (pr * z).T @ do[b, h] / (1.0 - p)
            dp = (do[b, h] @ v[b, kh].T) * z / (1.0 - p)
            D = np.sum(pr * dp, axis=1)
            ds = pr * (dp - D[:, None])
            dq[b, h] = scale * (ds @ k[b, kh])
            dk[b, kh] += scale * (ds.T @ q[b, h])
            dsum[b, h] = D
    return dq, dk, dv, dsum


def dropout_forward_rows(q2, k2, v2, scale, causal, rows, bh, p, seed, offset):
    """dropout_forward for chosen query rows of one head (bh = b*Hq + h)."""
    rows = np.asarray(rows)
    pr, lse = _head_probs(_f64(q2), _f64(k2), scale, causal, rows)
    z = dropout_keep(bh, rows, np.arange(k2.shape[0]), p, seed, offset)
    return (pr * z) @ _f64(v2) / (1.0 - p), lse


def dropout_backward_rows(q2, k2, v2, do2, scale, causal, rows, bh, p, seed, offset):
    """dQ and D for chosen query rows of one head (dropout)."""
    rows = np.asarray(rows)
    pr, _ = _head_probs(_f64(q2), _f64(k2), scale, causal, rows)
    z = dropout_keep(bh, rows, np.arange(k2.shape[0]), p, seed, offset)
    dp = (_f64(do2)[rows] @ _f64(v2).T) * z / (1.0 - p)
    D = np.sum(pr * dp, axis=1)
    ds = pr * (dp - D[:, None])
    return scale * (ds @ _f64(k2)), D


def dropout_backward_kv_rows(q_heads, k2, v2, do_heads, bhs, scale, causal, kv_rows, p, seed,
                             offset, chunk=2048):
    """dK and dV for chosen key rows of one key/value head (dropout); bhs are
    the b*Hq + h indices of the query heads in q_heads."""
    kv_rows = np.asarray(kv_rows)
    k2, v2 = _f64(k2), _f64(v2)
    dk = np.zeros((len(kv_rows), k2.shape[1]))
    dv = np.zeros((len(kv_rows), v2.shape[1]))
    for q2, do2, bh in zip(q_heads, do_heads, bhs):
        q2, do2 = _f64(q2), _f64(do2)
        nq = q2.shape[0]
        for c in range(0, nq, chunk):
            r = np.arange(c, min(c + chunk, nq))
            pr, _ = _head_probs(q2, k2, scale, causal, r)
            z = dropout_keep(bh, r, np.arange(k2.shape[0]), p, seed, offset)
            dp = (do2[r] @ v2.T) * z / (1.0 - p)
            D = np.sum(pr * dp, axis=1)
            pj, zj = pr[:, kv_rows], z[:, kv_rows]
            dsj = pj * (dp[:, kv_rows] - D[:, None])
            dv += (pj * zj).T @ do2[r] / (1.0 - p)
            dk += scale * (dsj.T @ q2[r])
    return dk, dv
