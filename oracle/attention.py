"""Float64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  This module is imported by ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` and by nothing else.  The product path (the C-ABI library and its
Python binding) never imports, links or calls it, and it shares no code with
the CUDA kernels.

Every function is the plain mathematical definition, evaluated in float64
numpy with no tiling, fusion or online rescaling.  Sources (page title, then
section):

* "Transformer、注意力机制与优化" (CMU 15-442/642 notes), section 数学公式:
  A(Q,K,V) = softmax(QK^T/sqrt(d)) V with Q, K, V in R^{N x d}; section
  标准注意力计算: the naive workflow S = QK^T -> mask (causal) -> softmax -> P V.
* same page, section 安全 Softmax 与在线 Softmax: the safe softmax
  m(x) = max_i x_i, f(x) = exp(x - m(x)), l(x) = sum f(x), softmax = f / l, and
  the two-block identity for m, f, l of a concatenated vector.
* "优化的注意力实现 (FlashAttention)" (apxml.com), section 优势与集成: the causal
  mask is the lower triangle ``tril(diagonal=0)`` filled with -inf above it,
  and the layout is (batch, heads, seq, head_dim).
* "FlashAttention 的基本原理", section 2.4 反向传播: gradients through O = PV
  (dV = P^T dO, dP = dO V^T), through the row-wise softmax, and through
  S = QK^T (dQ = dS K, dK = dS^T Q).  The row-wise softmax Jacobian gives
  dS = P * (dP - D) with D_i = sum_k dO_ik O_ik (the FlashAttention-2 form).
* "Transformer、注意力机制与优化", section Flash-Decoding: a single query
  attends to every cached key/value of its sequence.

Readings where the pages are silent:

* ``scale`` is an explicit argument; the pages use 1/sqrt(d).
* Causal alignment when Nq != Nk is bottom-right: key j is visible to query i
  iff j <= i + (Nk - Nq).  For Nq == Nk this is ``tril(diagonal=0)``.
* A query row that sees no key (causal with Nq > Nk, or Nk == 0) has output 0
  and log-sum-exp -inf.
* LSE is the natural log of sum_j exp(scale * q_i . k_j) over visible keys.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "causal_visible",
    "scaled_scores",
    "safe_softmax_stats",
    "merge_two_blocks",
    "softmax_rows",
    "attention_forward_head",
    "attention_forward",
    "attention_forward_rows",
    "attention_backward_head",
    "attention_backward",
    "attention_backward_q_rows",
    "attention_backward_kv_rows",
    "attention_row_block",
    "attention_backward_full_head",
    "decode_forward",
]


def causal_visible(nq: int, nk: int, rows=None, cols=None) -> np.ndarray:
    """Boolean visibility mask, bottom-right aligned (True = key visible).

    ``rows``/``cols`` optionally restrict the mask to given query/key indices.
    """
    i = np.arange(nq) if rows is None else np.asarray(rows)
    j = np.arange(nk) if cols is None else np.asarray(cols)
    return j[None, :] <= i[:, None] + (nk - nq)


def scaled_scores(q: np.ndarray, k: np.ndarray, scale: float, causal: bool,
                  nq_total: int | None = None, rows=None) -> np.ndarray:
    """S = scale * q k^T with -inf on masked entries (naive workflow steps 1-2).

    ``q`` holds the query rows ``rows`` (default: all) of a head whose total
    query length is ``nq_total`` (default: ``len(q)``).
    """
    s = scale * (q @ k.T)
    if causal:
        nq = q.shape[0] if nq_total is None else nq_total
        vis = causal_visible(nq, k.shape[0], rows=rows)
        s = np.where(vis, s, -np.inf)
    return s


def safe_softmax_stats(x: np.ndarray):
    """Row-wise m(x), f(x), l(x) of the safe softmax.

    Rows that are entirely -inf get m = -inf, f = 0, l = 0.
    """
    m = np.max(x, axis=-1) if x.shape[-1] > 0 else np.full(x.shape[:-1], -np.inf)
    shift = np.where(np.isfinite(m), m, 0.0)
    f = np.exp(x - shift[..., None])
    l = np.sum(f, axis=-1)
    return m, f, l


def merge_two_blocks(m1, f1, l1, m2, f2, l2):
    """m, f, l of the concatenation [x1 x2] from the two blocks' own m, f, l.

    m = max(m1, m2); f = [e^{m1-m} f1, e^{m2-m} f2]; l = e^{m1-m} l1 + e^{m2-m} l2.
    Blocks with m = -inf (empty or fully masked) contribute zero.
    """
    m = np.maximum(m1, m2)
    base = np.where(np.isfinite(m), m, 0.0)
    a1 = np.where(np.isfinite(m1), np.exp(np.where(np.isfinite(m1), m1, 0.0) - base), 0.0)
    a2 = np.where(np.isfinite(m2), np.exp(np.where(np.isfinite(m2), m2, 0.0) - base), 0.0)
    f = np.concatenate([a1[..., None] * f1, a2[..., None] * f2], axis=-1)
    l = a1 * l1 + a2 * l2
    return m, f, l


def softmax_rows(s: np.ndarray):
    """softmax(s) = f / l row-wise, with all-masked rows mapped to 0; returns (P, LSE)."""
    m, f, l = safe_softmax_stats(s)
    pos = l > 0
    p = np.where(pos[..., None], f / np.where(pos, l, 1.0)[..., None], 0.0)
    lse = np.where(pos, np.where(np.isfinite(m), m, 0.0) + np.log(np.where(pos, l, 1.0)), -np.inf)
    return p, lse


def attention_forward_head(q, k, v, scale: float, causal: bool):
    """O = softmax(scale q k^T [+ mask]) v and LSE for one (batch, head).

    q: [Nq, d], k, v: [Nk, d] float64.  Returns O [Nq, d], LSE [Nq].
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    if k.shape[0] == 0:
        return np.zeros((q.shape[0], v.shape[1])), np.full(q.shape[0], -np.inf)
    s = scaled_scores(q, k, scale, causal)
    p, lse = softmax_rows(s)
    return p @ v, lse


def attention_forward(q, k, v, scale: float, causal: bool):
    """Batched forward over [B, H, N, d] arrays (any float dtype, evaluated in float64)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, H, Nq, d = q.shape
    o = np.zeros((B, H, Nq, v.shape[-1]))
    lse = np.zeros((B, H, Nq))
    for b in range(B):
        for h in range(H):
            o[b, h], lse[b, h] = attention_forward_head(q[b, h], k[b, h], v[b, h], scale, causal)
    return o, lse


def attention_forward_rows(q_head, k_head, v_head, rows, scale: float, causal: bool,
                           block: int = 2048):
    """Forward for selected query rows of one head (each row uses its full score row).

    This is the same definition restricted to some outputs, for sizes where the
    whole N x N score matrix does not fit in host memory.
    """
    rows = np.asarray(rows)
    q = np.asarray(q_head[rows], np.float64)
    k = np.asarray(k_head, np.float64)
    v = np.asarray(v_head, np.float64)
    nq_total = q_head.shape[0]
    o = np.zeros((len(rows), v.shape[1]))
    lse = np.zeros(len(rows))
    for a in range(0, len(rows), block):
        sl = slice(a, a + block)
        s = scaled_scores(q[sl], k, scale, causal, nq_total=nq_total, rows=rows[sl])
        p, lse[sl] = softmax_rows(s)
        o[sl] = p @ v
    return o, lse


def attention_backward_head(q, k, v, do, scale: float, causal: bool):
    """dQ, dK, dV of <dO, O> for one head, from the plain definition.

    P is recomputed from the full scores; then dV = P^T dO, dP = dO v^T,
    D_i = sum_k dO_ik O_ik, dS = P * (dP - D), dQ = scale dS k, dK = scale dS^T q.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    if k.shape[0] == 0:
        return np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    s = scaled_scores(q, k, scale, causal)
    p, _ = softmax_rows(s)
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    drow = np.sum(do * o, axis=-1)
    ds = p * (dp - drow[:, None])
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv


def attention_backward(q, k, v, do, scale: float, causal: bool):
    """Batched backward over [B, H, N, d] arrays."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    B, H = q.shape[:2]
    for b in range(B):
        for h in range(H):
            dq[b, h], dk[b, h], dv[b, h] = attention_backward_head(
                q[b, h], k[b, h], v[b, h], do[b, h], scale, causal)
    return dq, dk, dv


def attention_backward_q_rows(q_head, k_head, v_head, do_head, rows, scale: float,
                              causal: bool, block: int = 1024):
    """dQ for selected query rows of one head.

    dQ_i depends only on row i: its scores, P_i, O_i, dP_i and D_i.
    """
    rows = np.asarray(rows)
    q = np.asarray(q_head[rows], np.float64)
    k = np.asarray(k_head, np.float64)
    v = np.asarray(v_head, np.float64)
    do = np.asarray(do_head[rows], np.float64)
    nq_total = q_head.shape[0]
    dq = np.zeros_like(q)
    for a in range(0, len(rows), block):
        sl = slice(a, a + block)
        s = scaled_scores(q[sl], k, scale, causal, nq_total=nq_total, rows=rows[sl])
        p, _ = softmax_rows(s)
        o = p @ v
        dp = do[sl] @ v.T
        drow = np.sum(do[sl] * o, axis=-1)
        ds = p * (dp - drow[:, None])
        dq[sl] = scale * (ds @ k)
    return dq


def attention_backward_kv_rows(q_head, k_head, v_head, do_head, keys, scale: float,
                               causal: bool, block: int = 1024):
    """dK, dV for selected key rows of one head.

    dK_j and dV_j sum over every query row that sees key j; each such row needs
    its full score row (for its softmax normaliser and O_i).  Under the causal
    mask the keys near the end are seen by few rows, which keeps this cheap.
    """
    keys = np.asarray(keys)
    qh = np.asarray(q_head, np.float64)
    k = np.asarray(k_head, np.float64)
    v = np.asarray(v_head, np.float64)
    doh = np.asarray(do_head, np.float64)
    nq, nk = qh.shape[0], k.shape[0]
    if causal:
        first = max(0, int(keys.min()) - (nk - nq))
    else:
        first = 0
    rows = np.arange(first, nq)
    dk = np.zeros((len(keys), k.shape[1]))
    dv = np.zeros((len(keys), v.shape[1]))
    for a in range(0, len(rows), block):
        r = rows[a:a + block]
        s = scaled_scores(qh[r], k, scale, causal, nq_total=nq, rows=r)
        p, _ = softmax_rows(s)
        o = p @ v
        dp_sel = doh[r] @ v[keys].T
        drow = np.sum(doh[r] * o, axis=-1)
        p_sel = p[:, keys]
        ds_sel = p_sel * (dp_sel - drow[:, None])
        dv += p_sel.T @ doh[r]
        dk += scale * (ds_sel.T @ qh[r])
    return dk, dv


def attention_row_block(q_head, k_head, v_head, do_head, r0: int, r1: int, scale: float, causal: bool):
    """Forward and backward of the query rows [r0, r1) of one head, each row with its whole score row.

    Returns (O, LSE, dQ) of those rows and their terms of dK and dV: dK = scale * sum_i dS_i^T q_i and
    dV = sum_i P_i^T dO_i are sums over query rows, so the terms of all row blocks add up to the full
    dK and dV (the plain definition, split along the sum).  Under the causal mask the keys past the
    block's last visible key have P = 0 and contribute nothing, so they are left out of the products
    and the dK, dV terms are returned for keys [0, kend) only (kend = the number of keys the block
    can see; Nk without the mask).
    """
    nq, nk = q_head.shape[0], k_head.shape[0]
    kend = nk if not causal else max(0, min(nk, (r1 - 1) + (nk - nq) + 1))
    q = np.asarray(q_head[r0:r1], np.float64)
    k = np.asarray(k_head[:kend], np.float64)
    v = np.asarray(v_head[:kend], np.float64)
    do = np.asarray(do_head[r0:r1], np.float64)
    if kend == 0:
        return (np.zeros((r1 - r0, v_head.shape[1])), np.full(r1 - r0, -np.inf), np.zeros_like(q),
                np.zeros((0, k_head.shape[1])), np.zeros((0, v_head.shape[1])))
    s = scale * (q @ k.T)
    if causal:
        s = np.where(causal_visible(nq, nk, rows=np.arange(r0, r1), cols=np.arange(kend)), s, -np.inf)
    p, lse = softmax_rows(s)
    o = p @ v
    dp = do @ v.T
    drow = np.sum(do * o, axis=-1)
    ds = p * (dp - drow[:, None])
    dq = scale * (ds @ k)
    return o, lse, dq, scale * (ds.T @ q), p.T @ do


def attention_backward_full_head(q_head, k_head, v_head, do_head, scale: float, causal: bool,
                                 block: int = 256, workers: int = 1):
    """dQ, dK, dV (and O, LSE) of one whole head, for sizes whose N x N matrices do not fit in host
    memory: the row blocks of ``attention_row_block`` summed.  ``workers`` > 1 evaluates the blocks
    on that many threads (numpy releases the interpreter lock in its kernels); the sums are the same
    up to the order of float64 additions."""
    import threading
    nq, nk = q_head.shape[0], k_head.shape[0]
    o = np.zeros((nq, v_head.shape[1]))
    lse = np.zeros(nq)
    dq = np.zeros((nq, q_head.shape[1]))
    dk = np.zeros((nk, k_head.shape[1]))
    dv = np.zeros((nk, v_head.shape[1]))
    lock = threading.Lock()

    def one(r0):
        r1 = min(nq, r0 + block)
        o[r0:r1], lse[r0:r1], dq[r0:r1], dk_t, dv_t = attention_row_block(q_head, k_head, v_head, do_head, r0, r1,
                                                                          scale, causal)
        with lock:
            dk[:len(dk_t)] += dk_t
            dv[:len(dv_t)] += dv_t

    starts = range(0, nq, block)
    if workers > 1:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(one, starts))
    else:
        for r0 in starts:
            one(r0)
    return o, lse, dq, dk, dv


def decode_forward(q, k_cache, v_cache, seqlens, scale: float):
    """Single-query attention against each sequence's first L_b cached keys.

    q: [B, H, d] (or [B, H, 1, d]); caches: [B, H, Lmax, d]; seqlens: [B].
    Returns O [B, H, d] and LSE [B, H].  Cache entries at or beyond L_b are
    never read.
    """
    q = np.asarray(q, np.float64)
    if q.ndim == 4:
        q = q[:, :, 0, :]
    B, H, d = q.shape
    o = np.zeros((B, H, v_cache.shape[-1]))
    lse = np.zeros((B, H))
    for b in range(B):
        L = int(seqlens[b])
        for h in range(H):
            kk = np.asarray(k_cache[b, h, :L], np.float64)
            vv = np.asarray(v_cache[b, h, :L], np.float64)
            ob, lb = attention_forward_head(q[b, h][None, :], kk, vv, scale, False)
            o[b, h] = ob[0]
            lse[b, h] = lb[0]
    return o, lse

