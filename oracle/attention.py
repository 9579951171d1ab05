"""CPU fp64 oracle for exact scaled-dot-product attention, forward and backward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
link this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it.  It shares no code with the CUDA
library and imports nothing from it.

What it computes
----------------
The pages on FlashAttention state that the tiled, IO-aware kernel reaches the
*same* result as standard attention, up to numerical precision
("FlashAttention-2" post on t.iss.one/s/quant_prune_distill/56, section
"Введение"; QbitAI FA1 article on 52ps.vip, section "FlashAttention", "IO
perceptual precision attention").  Standard attention materialises the full
score matrix (QbitAI FA2 article on baiyundou.net, section "实验评估", which
compares against PyTorch standard attention).  So this oracle is that plain
definition, written out in fp64 with no tiling, no online softmax and no
deferred rescaling:

    S   = scale * Q_h K_{kv(h)}^T                    [Nq x Nk]
    S_ij = -inf where causal and j > i               (top-left alignment)
    LSE_i = m_i + ln sum_j exp(S_ij - m_i),  m_i = max_j S_ij
    P   = exp(S - LSE)
    O   = P V_{kv(h)}

and the gradients of L = <O, dO> (the pages only say that the backward pass
recomputes the attention matrix block by block, same FA2 post, section
"Введение"; the formulas below are ordinary calculus):

    dV_kv += P^T dO
    dP     = dO V^T
    D_i    = sum_j P_ij dP_ij          (equals rowsum(dO * O))
    dS     = P * (dP - D)
    dQ     = scale * dS K
    dK_kv += scale * dS^T Q

Readings where the pages are silent (all listed in the design notes):
  * GQA/MQA (named on the baiyundou.net FA2 article, section "具体实现",
    "two small changes") maps query head h to kv head h // (Hq // Hkv).
  * Causal masking is top-left aligned: key j is visible to query i iff j <= i.
  * LSE is the natural-log logsumexp of the *scaled* scores.
  * Variable-length batches (not named on the pages; the FA2 article's
    section on parallelism over the sequence for small batches is the
    nearest passage): B sequences of different lengths are packed back to
    back, q as [total_q, Hq, d] and k, v as [total_k, Hkv, d], with
    cumulative offsets cu_q, cu_k of length B + 1.  Sequence b attends only
    within itself, causal top-left within the sequence; a sequence with
    queries but no keys gives O = 0, LSE = -inf.  LSE is [Hq, total_q].
  * Block-sparse attention (QbitAI FA1 article, results section, names
    block-sparse FlashAttention without defining it) takes a block mask of
    128 x 128 (query, key) blocks, shared by all batches and heads; a zero
    entry sets the block's scores to -inf, on top of the causal mask.  A row
    that sees no key at all gets O = 0, LSE = -inf and no gradient (the
    limits of an empty softmax).

Rows of the score matrix are independent (FA2 post, section "Параллелизм":
forward rows are independent), so processing query rows in chunks is exact;
it only bounds memory.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "BLOCK",
    "attention_forward_varlen",
    "attention_backward_varlen",
    "kv_head",
    "scores",
    "attention_forward",
    "attention_forward_rows",
    "attention_backward",
    "attention_backward_dq_rows",
    "attention_backward_kv_rows",
]

# Rows of S per chunk are chosen so one chunk of S holds at most this many
# fp64 elements (256 MiB).
_MAX_CHUNK_ELEMS = 1 << 25


def kv_head(h: int, hq: int, hkv: int) -> int:
    """KV head read by query head ``h``: contiguous groups of Hq/Hkv heads."""
    if hq % hkv != 0:
        raise ValueError(f"Hq={hq} is not a multiple of Hkv={hkv}")
    return h // (hq // hkv)


def _as64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# Block-sparse attention (QbitAI FA1 article, results section: block-sparse
# FlashAttention): a query row sees key j only where the (query block, key
# block) entry of a block mask is non-zero; blocks are BLOCK x BLOCK.
BLOCK = 128


def scores(q_rows: np.ndarray, k: np.ndarray, scale: float, causal: bool,
           row_index: np.ndarray, block_mask=None, col_index=None) -> np.ndarray:
    """Scaled, masked score rows S[r, j] for the query rows ``row_index``.

    q_rows: [R, d] (the rows themselves), k: [C, d] (the key rows), row_index:
    [R] absolute query positions, col_index: [C] absolute key positions of the
    rows of ``k`` (default 0..C-1; both are needed for the causal and block
    masks)."""
    s = scale * (q_rows @ k.T)
    j = (np.arange(k.shape[0]) if col_index is None else np.asarray(col_index))[None, :]
    if causal:
        s = np.where(j > row_index[:, None], -np.inf, s)
    if block_mask is not None:
        bm = np.asarray(block_mask) != 0
        visible = bm[(row_index // BLOCK)[:, None], j // BLOCK]
        s = np.where(visible, s, -np.inf)
    return s


def _softmax_stats(s: np.ndarray):
    """Row max-shifted logsumexp and the normalised probabilities.  A row with
    no visible key has LSE = -inf and P = 0 (so O = 0 and no gradient)."""
    m = s.max(axis=1)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    with np.errstate(divide="ignore"):
        lse = m_safe + np.log(np.exp(s - m_safe[:, None]).sum(axis=1))
    lse = np.where(empty, -np.inf, lse)
    p = np.where(empty[:, None], 0.0, np.exp(s - np.where(empty, 0.0, lse)[:, None]))
    return lse, p


def _chunk_rows(nq: int, nk: int) -> int:
    return max(1, min(nq, _MAX_CHUNK_ELEMS // max(1, nk)))


def attention_forward(q, k, v, causal: bool, scale: float, block_mask=None):
    """Exact attention forward.

    q: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d] (any float dtype; upcast to fp64).
    block_mask: optional [ceil(Nq/BLOCK), ceil(Nk/BLOCK)], shared by all
    batches and heads.  Returns (O [B, Hq, Nq, d] fp64, LSE [B, Hq, Nq] fp64)."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    b_, hq, nq, d = q.shape
    hkv, nk = k.shape[1], k.shape[2]
    o = np.empty((b_, hq, nq, d))
    lse = np.empty((b_, hq, nq))
    step = _chunk_rows(nq, nk)
    for b in range(b_):
        for h in range(hq):
            kvh = kv_head(h, hq, hkv)
            for r0 in range(0, nq, step):
                rows = np.arange(r0, min(nq, r0 + step))
                s = scores(q[b, h, rows], k[b, kvh], scale, causal, rows, block_mask)
                l_, p = _softmax_stats(s)
                lse[b, h, rows] = l_
                o[b, h, rows] = p @ v[b, kvh]
    return o, lse


def attention_forward_rows(q, k, v, causal: bool, scale: float, b: int, h: int,
                           rows, block_mask=None):
    """O and LSE of selected query rows of one (batch, head).

    Exact for any subset because forward rows are independent.
    Returns (O [R, d], LSE [R])."""
    hq, hkv = q.shape[1], k.shape[1]
    kvh = kv_head(h, hq, hkv)
    rows = np.asarray(rows, dtype=np.int64)
    qr = _as64(q[b, h, rows])
    kk = _as64(k[b, kvh])
    vv = _as64(v[b, kvh])
    s = scores(qr, kk, scale, causal, rows, block_mask)
    l_, p = _softmax_stats(s)
    return p @ vv, l_


def attention_backward(q, k, v, do, causal: bool, scale: float,
                       heads=None, return_aux: bool = False, block_mask=None):
    """Exact attention backward by the chain rule on the materialised P.

    q, do: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d].
    ``heads`` optionally restricts the work to a list of (b, kv_head) groups;
    gradients of the other groups are left as NaN.
    Returns (dQ, dK, dV) in fp64, plus (O, LSE, D) when ``return_aux``."""
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    b_, hq, nq, d = q.shape
    hkv, nk = k.shape[1], k.shape[2]
    g = hq // hkv
    if hq % hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    dq = np.full(q.shape, np.nan)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    o = np.full(q.shape, np.nan)
    lse = np.full((b_, hq, nq), np.nan)
    dd = np.full((b_, hq, nq), np.nan)
    groups = heads if heads is not None else [(b, j) for b in range(b_)
                                              for j in range(hkv)]
    step = _chunk_rows(nq, nk)
    for (b, kvh) in groups:
        kk, vv = k[b, kvh], v[b, kvh]
        dk_acc = np.zeros((nk, d))
        dv_acc = np.zeros((nk, d))
        for h in range(kvh * g, (kvh + 1) * g):
            for r0 in range(0, nq, step):
                rows = np.arange(r0, min(nq, r0 + step))
                qh, doh = q[b, h, rows], do[b, h, rows]
                s = scores(qh, kk, scale, causal, rows, block_mask)
                l_, p = _softmax_stats(s)
                dv_acc += p.T @ doh
                dp = doh @ vv.T
                d_row = (p * dp).sum(axis=1)
                ds = p * (dp - d_row[:, None])
                dq[b, h, rows] = scale * (ds @ kk)
                dk_acc += scale * (ds.T @ qh)
                o[b, h, rows] = p @ vv
                lse[b, h, rows] = l_
                dd[b, h, rows] = d_row
        dk[b, kvh] = dk_acc
        dv[b, kvh] = dv_acc
    if return_aux:
        return dq, dk, dv, (o, lse, dd)
    return dq, dk, dv


def attention_backward_dq_rows(q, k, v, do, causal: bool, scale: float, b: int, h: int,
                               rows, block_mask=None):
    """dQ of selected query rows of one (batch, head).

    Row i of dQ needs only row i of P and dP (D_i is a sum over that row), so
    any subset of rows is exact on its own.  Returns dQ [R, d] in fp64."""
    hq, hkv = q.shape[1], k.shape[1]
    kvh = kv_head(h, hq, hkv)
    rows = np.asarray(rows, dtype=np.int64)
    qr, dor = _as64(q[b, h, rows]), _as64(do[b, h, rows])
    kk, vv = _as64(k[b, kvh]), _as64(v[b, kvh])
    s = scores(qr, kk, scale, causal, rows, block_mask)
    _, p = _softmax_stats(s)
    dp = dor @ vv.T
    d_row = (p * dp).sum(axis=1)
    ds = p * (dp - d_row[:, None])
    return scale * (ds @ kk)


def attention_backward_kv_rows(q, k, v, do, causal: bool, scale: float, b: int, kvh: int,
                               keys, heads=None, block_mask=None):
    """dK and dV of selected key rows of one (batch, kv head).

    Key row j of dK and dV sums over every query row i of every query head
    of the kv group (the GQA/MQA sum of the FA2 article, section "具体实现"):

        dV_j = sum_h sum_i P_ij dO_i
        dK_j = scale * sum_h sum_i P_ij (dP_ij - D_i) q_i,  dP_ij = dO_i . v_j

    Each term needs row i's LSE_i (for P_ij = exp(S_ij - LSE_i)) and
    D_i = sum_j' P_ij' dP_ij', which are sums over the whole row.  So the
    function first takes every row of each query head in chunks (exact:
    rows are independent) to get LSE and D, exactly as attention_backward
    does, and then forms the columns of P, dP and dS of the selected keys
    only.  Under the causal mask a row chunk's scores are formed only for
    the keys up to its last row; the keys beyond are masked for every row of
    the chunk and add exp(-inf) = 0 to its sums.

    heads: the query heads of the group to sum over (default: all of them;
    a subset gives that subset's share of the sum).
    Returns (dK [K, d], dV [K, d]) in fp64."""
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    hq, nq = q.shape[1], q.shape[2]
    hkv, nk = k.shape[1], k.shape[2]
    g = hq // hkv
    keys = np.asarray(keys, dtype=np.int64)
    kk, vv = k[b, kvh], v[b, kvh]
    heads = range(kvh * g, (kvh + 1) * g) if heads is None else heads
    dk = np.zeros((len(keys), q.shape[3]))
    dv = np.zeros((len(keys), q.shape[3]))
    step = _chunk_rows(nq, nk)
    for h in heads:
        if kv_head(h, hq, hkv) != kvh:
            raise ValueError(f"query head {h} does not read kv head {kvh}")
        lse = np.empty(nq)
        dd = np.empty(nq)
        for r0 in range(0, nq, step):
            rows = np.arange(r0, min(nq, r0 + step))
            kmax = min(nk, int(rows[-1]) + 1) if causal else nk
            s = scores(q[b, h, rows], kk[:kmax], scale, causal, rows, block_mask)
            l_, p = _softmax_stats(s)
            dp = do[b, h, rows] @ vv[:kmax].T
            lse[rows] = l_
            dd[rows] = (p * dp).sum(axis=1)
        rows = np.arange(nq)
        s = scores(q[b, h], kk[keys], scale, causal, rows, block_mask, col_index=keys)
        empty = np.isneginf(lse)
        p = np.where(empty[:, None], 0.0, np.exp(s - np.where(empty, 0.0, lse)[:, None]))
        dp = do[b, h] @ vv[keys].T
        ds = p * (dp - dd[:, None])
        dv += p.T @ do[b, h]
        dk += scale * (ds.T @ q[b, h])
    return dk, dv


# ------------------------------------------------------------------ variable-length batches
def _seq_views(x, cu, b):
    """Rows cu[b]:cu[b+1] of a packed [total, H, d] tensor as [1, H, n, d]."""
    return np.ascontiguousarray(_as64(x[cu[b]:cu[b + 1]]).transpose(1, 0, 2)[None])


def attention_forward_varlen(q, k, v, cu_q, cu_k, causal: bool, scale: float):
    """Exact attention of B packed sequences, each on its own.

    q: [total_q, Hq, d]; k, v: [total_k, Hkv, d]; cu_q, cu_k: [B + 1]
    cumulative offsets (non-decreasing, starting at 0).  Returns
    (O [total_q, Hq, d], LSE [Hq, total_q]) in fp64."""
    cu_q, cu_k = [int(x) for x in cu_q], [int(x) for x in cu_k]
    hq, d = q.shape[1], q.shape[2]
    o = np.zeros((q.shape[0], hq, d))
    lse = np.full((hq, q.shape[0]), -np.inf)
    for b in range(len(cu_q) - 1):
        nq, nk = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        if nq == 0 or nk == 0:
            continue                      # no rows, or rows that see no key (O = 0)
        ob, lb = attention_forward(_seq_views(q, cu_q, b), _seq_views(k, cu_k, b),
                                   _seq_views(v, cu_k, b), causal, scale)
        o[cu_q[b]:cu_q[b + 1]] = ob[0].transpose(1, 0, 2)
        lse[:, cu_q[b]:cu_q[b + 1]] = lb[0]
    return o, lse


def attention_backward_varlen(q, k, v, do, cu_q, cu_k, causal: bool, scale: float):
    """Gradients of sum(O * dO) for attention_forward_varlen; returns
    (dQ [total_q, Hq, d], dK, dV [total_k, Hkv, d]) in fp64."""
    cu_q, cu_k = [int(x) for x in cu_q], [int(x) for x in cu_k]
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for b in range(len(cu_q) - 1):
        nq, nk = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        if nq == 0 or nk == 0:
            continue
        g = attention_backward(_seq_views(q, cu_q, b), _seq_views(k, cu_k, b),
                               _seq_views(v, cu_k, b), _seq_views(do, cu_q, b), causal, scale)
        dq[cu_q[b]:cu_q[b + 1]] = g[0][0].transpose(1, 0, 2)
        dk[cu_k[b]:cu_k[b + 1]] = g[1][0].transpose(1, 0, 2)
        dv[cu_k[b]:cu_k[b + 1]] = g[2][0].transpose(1, 0, 2)
    return dq, dk, dv
