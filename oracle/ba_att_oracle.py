"""Plain NumPy oracle for the BA-Att hot path (test infrastructure only).

All arithmetic runs in ``dtype`` (float64 by default; the CPU-baseline timing
passes float32). Inputs are arrays shaped [B, H, N_alloc, d]; only the first
``N`` rows of each head are tokens, the rest is padding and is never read.

Notation (used in every docstring below):
  b      block size; queries and keys share it unless a key block size b_k
         is given (asymmetric blocks), then query blocks have b rows and key
         blocks b_k rows
  nq, nk number of query / key blocks, ceil(N / b) and ceil(N / b_k); block i
         covers rows [i*b, min(N, (i+1)*b)) (b_k for key blocks)
  n_i    valid rows of query block i,  m_j  valid rows of key block j
  s      softmax scale (default d**-0.5)
  g(h)   KV head of query head h: h // (Hq // Hkv)  (grouped-query attention)

Citations: [BA-Att] is the page "Efficient Long-Context Modeling in Diffusion
Language Models via Block Approximate Sparse Attention"; [FlashBlock] is the
page "FlashBlock: Attention Caching for Efficient Long-Context Block Diffusion".
"""

from __future__ import annotations

import math

import numpy as np

NEG_INF = -np.inf


# ---------------------------------------------------------------------------
# Block geometry
# ---------------------------------------------------------------------------

def num_blocks(N: int, b: int) -> int:
    """Number of blocks covering N tokens with block size b (the last may be ragged)."""
    return -(-N // b)


def block_counts(N: int, b: int) -> np.ndarray:
    """Valid rows per block: b for every block but a ragged last one."""
    nb = num_blocks(N, b)
    return np.array([min(N, (i + 1) * b) - i * b for i in range(nb)], dtype=np.int64)


def keep_count(keep: float, nk: int) -> int:
    """How many key blocks a query block keeps.

    [BA-Att, "Core claim"/abstract]: the selector keeps a top fraction of the
    key blocks (50% sparsity in the experiments). Reading: k = ceil(keep*nk),
    at least one block; the 1e-9 guard keeps exact fractions exact.
    """
    if not (0.0 < keep <= 1.0):
        raise ValueError("keep must lie in (0, 1]")
    return max(1, int(math.ceil(keep * nk - 1e-9)))


# ---------------------------------------------------------------------------
# Stage one: block-wise pre-downsample statistics
# ---------------------------------------------------------------------------

def block_stats(X, N: int, b: int, dtype=np.float64):
    """Per-block mean and per-dimension population variance.

    [BA-Att, abstract; "What carries the argument"]: the attention space is
    downsampled block-wise before scoring, and the correction uses the
    diagonal (per-dimension) variances of Q and K inside each block.
    Reading: mean over the block's valid rows, variance with 1/n (so a block
    of identical rows has variance exactly zero).

    X: [B, H, N_alloc, d]. Returns mean, var: [B, H, nb, d] and counts: [nb].
    """
    X = np.asarray(X)
    B, H, _, d = X.shape
    counts = block_counts(N, b)
    nb = len(counts)
    mean = np.empty((B, H, nb, d), dtype=dtype)
    var = np.empty((B, H, nb, d), dtype=dtype)
    for i in range(nb):
        rows = X[:, :, i * b: i * b + counts[i], :].astype(dtype)
        mu = rows.sum(axis=2) / dtype(counts[i])
        dev = rows - mu[:, :, None, :]
        mean[:, :, i, :] = mu
        var[:, :, i, :] = (dev * dev).sum(axis=2) / dtype(counts[i])
    return mean, var, counts


def _kv_head(h: int, Hq: int, Hkv: int) -> int:
    return h // (Hq // Hkv)


def corrected_scores(q_mean, q_var, k_mean, k_var, k_counts, sm_scale: float,
                     dtype=np.float64, var_product: bool = True):
    """Covariance-compensated downsampled block scores S~[B, Hq, nq, nk].

    [BA-Att, abstract; "Core claim"]: blocks are scored in the compact
    downsampled space, and the plain pooled score is corrected with a term
    built from diagonal Q/K variances in place of the full covariance
    (off-diagonal terms are dropped, as the referee report notes).

    Reading: for q in query block i and k in key block j, model the logit
    x = s*q.k with q ~ N(qbar_i, diag(var_q,i)), k ~ N(kbar_j, diag(var_k,j))
    independent. Then
        E[x]   = s * qbar_i . kbar_j
        Var[x] = s^2 * V_ij,
        V_ij   = sum_m ( var_q,i,m * kbar_j,m^2 + qbar_i,m^2 * var_k,j,m
                         + var_q,i,m * var_k,j,m )
    (the exact variance of a sum of products of independent Gaussians), and
    the Gaussian moment generating function gives ln E[e^x] = E[x] + Var[x]/2.
    A key block of m_j tokens contributes m_j such terms, hence + ln m_j:
        S~_ij = s * qbar_i.kbar_j + (s^2 / 2) * V_ij + ln m_j.
    Query head h reads the statistics of KV head g(h).

    var_product=False drops the var_q * var_k term of V_ij (a selection
    variant: the correction from the means' cross terms only).
    """
    q_mean = np.asarray(q_mean, dtype=dtype)
    q_var = np.asarray(q_var, dtype=dtype)
    k_mean = np.asarray(k_mean, dtype=dtype)
    k_var = np.asarray(k_var, dtype=dtype)
    B, Hq, nq, _ = q_mean.shape
    Hkv, nk = k_mean.shape[1], k_mean.shape[2]
    s = dtype(sm_scale)
    log_m = np.log(np.asarray(k_counts, dtype=dtype))
    S = np.empty((B, Hq, nq, nk), dtype=dtype)
    for h in range(Hq):
        g = _kv_head(h, Hq, Hkv)
        qm, qv = q_mean[:, h], q_var[:, h]          # [B, nq, d]
        km, kv = k_mean[:, g], k_var[:, g]          # [B, nk, d]
        mean_term = s * (qm @ km.transpose(0, 2, 1))
        V = (qv @ (km * km).transpose(0, 2, 1)
             + (qm * qm) @ kv.transpose(0, 2, 1))
        if var_product:
            V = V + qv @ kv.transpose(0, 2, 1)
        S[:, h] = mean_term + dtype(0.5) * s * s * V + log_m[None, None, :]
    return S


def pooled_scores(q_mean, k_mean, k_counts, sm_scale: float, dtype=np.float64):
    """Uncorrected pooled block score s * qbar_i.kbar_j + ln m_j.

    The baseline that the correction compensates [BA-Att, abstract]; it is
    what S~ reduces to when every diagonal variance is zero.
    """
    q_mean = np.asarray(q_mean, dtype=dtype)
    k_mean = np.asarray(k_mean, dtype=dtype)
    B, Hq, nq, _ = q_mean.shape
    Hkv, nk = k_mean.shape[1], k_mean.shape[2]
    log_m = np.log(np.asarray(k_counts, dtype=dtype))
    S = np.empty((B, Hq, nq, nk), dtype=dtype)
    for h in range(Hq):
        g = _kv_head(h, Hq, Hkv)
        S[:, h] = dtype(sm_scale) * (q_mean[:, h] @ k_mean[:, g].transpose(0, 2, 1)) + log_m
    return S


def pre_downsample_map(S):
    """Pre-downsample block attention map A^_ij = softmax_j S~_ij (rows sum to 1)."""
    S = np.asarray(S)
    mx = S.max(axis=-1, keepdims=True)
    E = np.exp(S - mx)
    return E / E.sum(axis=-1, keepdims=True)


# ---------------------------------------------------------------------------
# Norm sorting: keep the top fraction of key blocks per query block
# ---------------------------------------------------------------------------

def select_topk(S, k: int, kmax: int | None = None):
    """Rank key blocks per query block and keep the first k.

    [BA-Att, "The pith"; abstract; Figure 2 caption]: a norm-sorting module
    ranks the downsampled blocks and the top fraction is attended.
    Reading: rank by S~ descending (the same order as the softmax-normalised
    block probability A^), equal scores resolved toward the lower key-block
    index; emit the kept indices in ascending order.

    Returns idx [..., kmax] int32 (entries past the count are -1) and
    cnt [...] int32.
    """
    S = np.asarray(S)
    nk = S.shape[-1]
    if kmax is None:
        kmax = k
    k = min(k, nk)
    # A stable sort of -S keeps lower indices first among equal scores.
    order = np.argsort(-S, axis=-1, kind="stable")[..., :k]
    kept = np.sort(order, axis=-1).astype(np.int32)
    idx = np.full(S.shape[:-1] + (kmax,), -1, dtype=np.int32)
    idx[..., :k] = kept
    cnt = np.full(S.shape[:-1], k, dtype=np.int32)
    return idx, cnt


def selection_scores(S, Hkv: int, force_diagonal: bool = False, shared_gqa: bool = False):
    """The scores a selection variant ranks, from the per-head S~ [B, Hq, nq, nk].

    Variants of the norm sorting (the pages fix none of them; each is a plain
    option around the ranking of "The pith"/"Core claim"):
      shared_gqa      the query heads of one KV group share one selection,
                      ranked by the mean of their S~ over the group;
      force_diagonal  query block i always keeps key block i (ranked first).
    ``select_topk`` of the result gives the lists.
    """
    R = np.array(S, dtype=np.float64, copy=True)
    B, Hq, nq, nk = R.shape
    if shared_gqa:
        G = Hq // Hkv
        R = np.repeat(R.reshape(B, Hkv, G, nq, nk).mean(axis=2), G, axis=1)
    if force_diagonal:
        n = min(nq, nk)
        R[..., np.arange(n), np.arange(n)] = np.inf
    return R


def select_by_mass(R, tau: float, kmax: int | None = None):
    """Keep, per row, the fewest top-ranked key blocks whose share of the
    softmax-normalised block probability reaches tau.

    A selection variant (the pages keep a fixed top fraction; this keeps a
    fixed share of the pre-downsample map A^ = softmax_j S~ instead): rank
    as ``select_topk`` does (R descending, ties to the lower index), take
    the shortest prefix whose A^ sum is >= tau (at least one block), emit it
    ascending. Returns (idx [..., kmax] -1 padded, cnt).
    """
    R = np.asarray(R, dtype=np.float64)
    nk = R.shape[-1]
    kmax = nk if kmax is None else kmax
    idx = np.full(R.shape[:-1] + (kmax,), -1, dtype=np.int32)
    cnt = np.zeros(R.shape[:-1], dtype=np.int32)
    for pos in np.ndindex(R.shape[:-1]):
        row = R[pos]
        order = np.argsort(-row, kind="stable")
        e = np.exp(row - row.max())
        share = np.cumsum(e[order]) / e.sum()
        m = int(np.searchsorted(share, tau, side="left")) + 1
        m = min(max(m, 1), nk)
        kept = np.sort(order[:m])
        idx[pos][:m] = kept
        cnt[pos] = m
    return idx, cnt


def mass_share_before(R, idx, cnt):
    """For each row, the A^ share of its kept blocks without the lowest-ranked
    one, and with it (the two sides of the tau cut); used to tell cuts that
    rounding may move (the share sits within a relative band of tau)."""
    R = np.asarray(R, dtype=np.float64)
    lo = np.zeros(cnt.shape)
    hi = np.zeros(cnt.shape)
    for pos in np.ndindex(cnt.shape):
        row = R[pos]
        e = np.exp(row - row.max())
        kept = idx[pos][: cnt[pos]]
        vals = np.sort(e[kept])                       # ascending: vals[0] is the lowest-ranked kept block
        hi[pos] = vals.sum() / e.sum()
        lo[pos] = (vals.sum() - vals[0]) / e.sum()
    return lo, hi


def near_tie_mask(S, k: int, rel: float = 1e-3):
    """Blocks whose score lies within ``rel`` of the selection threshold.

    The threshold is the k-th ranked block of the row. "Within rel of the
    threshold" is read two ways, and a block counts as a near-tie only when
    it is close in both (the narrower band):
      - on the corrected score itself: |S~_ij - S~_thr| <= rel * |S~_thr|;
      - on the normalised map A^ (a relative band on probabilities):
        |A^_ij - A^_thr| <= rel * A^_thr, i.e. |exp(S~_ij - S~_thr) - 1| <= rel,
        because A^ is proportional to exp(S~) within a row.
    Blocks in this band may legitimately fall either side of the cut under
    different rounding; outside it the kept set is fixed.
    """
    S = np.asarray(S, dtype=np.float64)
    srt = -np.sort(-S, axis=-1)
    thr = srt[..., min(k, S.shape[-1]) - 1][..., None]
    in_map_band = np.abs(np.expm1(S - thr)) <= rel
    in_score_band = np.abs(S - thr) <= rel * np.abs(thr)
    return in_map_band & in_score_band


# ---------------------------------------------------------------------------
# Stage two: attention over the kept blocks
# ---------------------------------------------------------------------------

def _block_rows(N: int, b: int, i: int) -> np.ndarray:
    return np.arange(i * b, min(N, (i + 1) * b))


def _attend(q, keys, vals, s, dtype):
    """Softmax attention of rows q over (keys, vals); returns O, natural-log LSE."""
    if keys.shape[0] == 0:
        return np.zeros((q.shape[0], vals.shape[1]), dtype=dtype), np.full(q.shape[0], NEG_INF, dtype=dtype)
    logits = dtype(s) * (q @ keys.T)
    mx = logits.max(axis=1, keepdims=True)
    E = np.exp(logits - mx)
    Z = E.sum(axis=1, keepdims=True)
    O = (E @ vals) / Z
    L = mx[:, 0] + np.log(Z[:, 0])
    return O, L


def masked_attention(Q, K, V, idx, cnt, N: int, b: int, sm_scale: float,
                     query_blocks=None, dtype=np.float64, b_k: int | None = None):
    """Block-sparse bidirectional attention over the kept key blocks.

    [BA-Att, abstract; Figure 4]: attention is computed only over the selected
    blocks, with no causal mask. For every valid row r of query block i:
        L_r = ln sum_{c in C_i} exp(s q_r . k_c),
        O_r = sum_{c in C_i} exp(s q_r . k_c - L_r) v_c,
    with C_i the valid keys of blocks idx[i, :cnt[i]]. An empty list gives
    O_r = 0 and L_r = -inf. Here the softmax is taken with an explicit
    probability matrix per query block; no online rescaling.

    query_blocks: optional iterable of (batch, head, i) to evaluate; rows of
    other blocks are left as NaN. b_k: key block size when it differs from the
    query block size b (the lists then index blocks of b_k keys).
    Returns O [B, Hq, N_alloc, d], LSE [B, Hq, N_alloc].
    """
    Q = np.asarray(Q)
    K = np.asarray(K)
    V = np.asarray(V)
    B, Hq, Na, d = Q.shape
    Hkv = K.shape[1]
    nq = num_blocks(N, b)
    O = np.full((B, Hq, Na, d), np.nan, dtype=dtype)
    LSE = np.full((B, Hq, Na), np.nan, dtype=dtype)
    if query_blocks is None:
        query_blocks = [(bb, h, i) for bb in range(B) for h in range(Hq) for i in range(nq)]
    for bb, h, i in query_blocks:
        g = _kv_head(h, Hq, Hkv)
        rows = _block_rows(N, b, i)
        blocks = [int(j) for j in idx[bb, h, i, : int(cnt[bb, h, i])]]
        bk = b if b_k is None else b_k
        keys = np.concatenate([_block_rows(N, bk, j) for j in blocks]) if blocks else np.zeros(0, dtype=np.int64)
        q = Q[bb, h, rows].astype(dtype)
        kk = K[bb, g, keys].astype(dtype)
        vv = V[bb, g, keys].astype(dtype)
        O[bb, h, rows], LSE[bb, h, rows] = _attend(q, kk, vv, sm_scale, dtype)
    return O, LSE


def block_rows_attention(Qr, K, V, idx, cnt, q_rows: int, N: int, b: int, sm_scale: float,
                         O_prev=None, L_prev=None, dtype=np.float64, b_k: int | None = None):
    """Attention of one range of query rows over listed key blocks, merged
    with a cached partial of those rows when one is given.

    [FlashBlock, "Core claim" and "What carries the argument"]: in block
    diffusion the current block's attention to the tokens outside it is
    cached as (A_out, L_out); each step recomputes only the attention inside
    the current block and combines the two in log space (Eq. 9, with the
    split of Eq. 5). Here: Qr [B, Hq, q_stride, d] holds the range's q_rows
    query rows, cut into query blocks of b rows (the last may be ragged);
    idx [B, Hq, nqr, kmax] / cnt [B, Hq, nqr] list, per query block of the
    range, the key blocks (of b_k keys, default b) it attends; keys >= N are
    not tokens. For every row r < q_rows of block i:
        L_r = ln sum_{c in C_i} exp(s q_r . k_c),
        O_r = sum_{c in C_i} exp(s q_r . k_c - L_r) v_c,
    then, with (O_prev, L_prev) [B, Hq, q_stride, d] / [B, Hq, q_stride],
    (O_r, L_r) = merge_lse(O_prev_r, L_prev_r, O_r, L_r).
    Rows >= q_rows are NaN. Returns O [B, Hq, q_stride, d], LSE [B, Hq, q_stride].
    """
    Qr = np.asarray(Qr)
    K = np.asarray(K)
    V = np.asarray(V)
    B, Hq, q_stride, d = Qr.shape
    Hkv = K.shape[1]
    bk = b if b_k is None else b_k
    O = np.full((B, Hq, q_stride, d), np.nan, dtype=dtype)
    LSE = np.full((B, Hq, q_stride), np.nan, dtype=dtype)
    for bb in range(B):
        for h in range(Hq):
            g = _kv_head(h, Hq, Hkv)
            for i in range(num_blocks(q_rows, b)):
                rows = _block_rows(q_rows, b, i)
                blocks = [int(j) for j in idx[bb, h, i, : int(cnt[bb, h, i])]]
                keys = (np.concatenate([_block_rows(N, bk, j) for j in blocks]) if blocks
                        else np.zeros(0, dtype=np.int64))
                o, l = _attend(Qr[bb, h, rows].astype(dtype), K[bb, g, keys].astype(dtype),
                               V[bb, g, keys].astype(dtype), sm_scale, dtype)
                if O_prev is not None:
                    o, l = merge_lse(np.asarray(O_prev)[bb, h, rows], np.asarray(L_prev)[bb, h, rows], o, l, dtype)
                O[bb, h, rows], LSE[bb, h, rows] = o, l
    return O, LSE


def dense_attention(Q, K, V, N: int, sm_scale: float, rows=None, dtype=np.float64):
    """Textbook dense softmax attention over all N valid keys (no mask).

    Written independently of ``masked_attention``: one full logit matrix per
    head, a row-wise softmax, then P @ V. ``rows`` optionally restricts the
    query rows (same for every head). Returns O [B, Hq, len(rows), d] and
    LSE [B, Hq, len(rows)].
    """
    Q = np.asarray(Q)
    K = np.asarray(K)
    V = np.asarray(V)
    B, Hq, _, d = Q.shape
    Hkv = K.shape[1]
    if rows is None:
        rows = np.arange(N)
    rows = np.asarray(rows)
    O = np.empty((B, Hq, len(rows), d), dtype=dtype)
    LSE = np.empty((B, Hq, len(rows)), dtype=dtype)
    for bb in range(B):
        for h in range(Hq):
            g = _kv_head(h, Hq, Hkv)
            q = Q[bb, h, rows].astype(dtype)
            k = K[bb, g, :N].astype(dtype)
            v = V[bb, g, :N].astype(dtype)
            logits = dtype(sm_scale) * (q @ k.T)
            mx = logits.max(axis=1, keepdims=True)
            P = np.exp(logits - mx)
            Z = P.sum(axis=1, keepdims=True)
            P = P / Z
            O[bb, h] = P @ v
            LSE[bb, h] = mx[:, 0] + np.log(Z[:, 0])
    return O, LSE


# ---------------------------------------------------------------------------
# Log-space merge of two partial attentions
# ---------------------------------------------------------------------------

def merge_lse(O1, L1, O2, L2, dtype=np.float64):
    """Combine two partial attentions over disjoint key sets.

    [FlashBlock, Eq. 5 and Eq. 9]: attention over the union of two key sets
    equals the weighted combination of the two partial outputs, each weighted
    by its partition function, evaluated stably after subtracting the larger
    log-normaliser:
        m = max(L1, L2), w_k = exp(L_k - m),
        O = (w1 O1 + w2 O2) / (w1 + w2),   L = m + ln(w1 + w2).
    Both partials empty (L1 = L2 = -inf) gives O = 0, L = -inf.
    O*: [..., d]; L*: [...].
    """
    O1 = np.asarray(O1, dtype=dtype)
    O2 = np.asarray(O2, dtype=dtype)
    L1 = np.asarray(L1, dtype=dtype)
    L2 = np.asarray(L2, dtype=dtype)
    m = np.maximum(L1, L2)
    empty = np.isneginf(m)
    m_safe = np.where(empty, 0.0, m)
    w1 = np.exp(L1 - m_safe)
    w2 = np.exp(L2 - m_safe)
    den = w1 + w2
    den_safe = np.where(empty, 1.0, den)
    O = (w1[..., None] * O1 + w2[..., None] * O2) / den_safe[..., None]
    O = np.where(empty[..., None], 0.0, O)
    L = np.where(empty, NEG_INF, m_safe + np.log(den_safe))
    return O.astype(dtype), L.astype(dtype)


def complement_lists(idx, cnt, nk: int, ckmax: int | None = None):
    """The key blocks each kept-block list leaves out, ascending, -1 padded.

    [FlashBlock, review page: the "sparse + cached residual" form of Fig. 6]:
    attention over the kept blocks and over the blocks the selector dropped
    are two disjoint partial attentions whose log-space merge (``merge_lse``,
    Eq. 9) is attention over every block. Entries outside [0, nk) in the
    input are ignored. ckmax (default nk) is the row stride of the result.
    """
    idx = np.asarray(idx)
    cnt = np.asarray(cnt)
    ckmax = nk if ckmax is None else ckmax
    cidx = np.full(cnt.shape + (ckmax,), -1, dtype=np.int32)
    ccnt = np.zeros(cnt.shape, dtype=np.int32)
    for pos in np.ndindex(cnt.shape):
        kept = {int(j) for j in idx[pos][: int(cnt[pos])] if 0 <= int(j) < nk}
        rest = [j for j in range(nk) if j not in kept]
        cidx[pos][: len(rest)] = rest
        ccnt[pos] = len(rest)
    return cidx, ccnt


def split_lists(idx, cnt, split_block: int):
    """Partition each kept-block list at a key-block boundary.

    [FlashBlock, Eq. 5]: the key set is split into a block-external span
    (blocks < split_block) and a block-internal span (blocks >= split_block);
    each span's partial attention is computed separately and merged with
    ``merge_lse``. Lists stay ascending; unused entries are -1.
    """
    idx = np.asarray(idx)
    cnt = np.asarray(cnt)
    kmax = idx.shape[-1]
    lo_idx = np.full_like(idx, -1)
    hi_idx = np.full_like(idx, -1)
    lo_cnt = np.zeros_like(cnt)
    hi_cnt = np.zeros_like(cnt)
    for pos in np.ndindex(cnt.shape):
        row = [int(j) for j in idx[pos][: int(cnt[pos])]]
        lo = [j for j in row if j < split_block]
        hi = [j for j in row if j >= split_block]
        lo_idx[pos][: len(lo)] = lo
        hi_idx[pos][: len(hi)] = hi
        lo_cnt[pos] = len(lo)
        hi_cnt[pos] = len(hi)
    assert lo_idx.shape[-1] == kmax
    return lo_idx, lo_cnt, hi_idx, hi_cnt


# ---------------------------------------------------------------------------
# The oracle post-downsample map and diagnostics
# ---------------------------------------------------------------------------

def post_downsample_map(Q, K, N: int, b: int, sm_scale: float, dtype=np.float64, b_k: int | None = None):
    """Exact post-downsample block map A[B, Hq, nq, nk] (key blocks of b_k rows if given).

    [BA-Att, "Core claim"; abstract]: the reference the selector approximates
    is the full softmax attention map aggregated to blocks after the softmax:
        A_ij = (1/n_i) sum_{r in I_i} sum_{c in J_j} P_rc,
    P the full row-softmax of s Q K^T over the valid keys. Rows sum to 1.
    Brute force; tiny inputs only.
    """
    Q = np.asarray(Q)
    K = np.asarray(K)
    B, Hq, _, _ = Q.shape
    Hkv = K.shape[1]
    counts = block_counts(N, b)
    bk = b if b_k is None else b_k
    kcounts = block_counts(N, bk)
    nb, nk = len(counts), len(kcounts)
    A = np.zeros((B, Hq, nb, nk), dtype=dtype)
    for bb in range(B):
        for h in range(Hq):
            g = _kv_head(h, Hq, Hkv)
            logits = dtype(sm_scale) * (Q[bb, h, :N].astype(dtype) @ K[bb, g, :N].astype(dtype).T)
            P = np.exp(logits - logits.max(axis=1, keepdims=True))
            P /= P.sum(axis=1, keepdims=True)
            for i in range(nb):
                ri = slice(i * b, i * b + counts[i])
                for j in range(nk):
                    cj = slice(j * bk, j * bk + kcounts[j])
                    A[bb, h, i, j] = P[ri, cj].sum() / counts[i]
    return A


def block_mass_via_lse(lse_single, lse_full, counts_q):
    """Post-downsample map from per-block log-normalisers (second route to A).

    With l_r^(j) the LSE of row r over key block j alone and l_r the LSE over
    all keys, the row's probability mass on block j is exp(l_r^(j) - l_r);
    averaging over the rows of query block i gives A_ij. lse_single has shape
    [nk, N] (one attention pass per single-block list), lse_full [N].
    """
    lse_single = np.asarray(lse_single, dtype=np.float64)
    lse_full = np.asarray(lse_full, dtype=np.float64)
    nk = lse_single.shape[0]
    nb = len(counts_q)
    b = int(counts_q[0])
    A = np.zeros((nb, nk))
    for i in range(nb):
        rows = slice(i * b, i * b + int(counts_q[i]))
        A[i] = np.exp(lse_single[:, rows] - lse_full[None, rows]).mean(axis=1)
    return A


def _rank(x):
    order = np.argsort(x, kind="stable")
    r = np.empty(len(x))
    r[order] = np.arange(len(x))
    return r


def spearman_vs_post(S, A):
    """Mean per-row Spearman rank correlation between a block score and A.

    Diagnostic for the correlation the Figure 2 caption of [BA-Att] refers to;
    the pages print no value for it. Pinned to scipy's Spearman rho and the
    closed form on tie-free rows, and to +1 / -1 for equal / reversed order.
    """
    S = np.asarray(S).reshape(-1, S.shape[-1])
    A = np.asarray(A).reshape(-1, A.shape[-1])
    vals = []
    for s_row, a_row in zip(S, A):
        rs, ra = _rank(s_row), _rank(a_row)
        rs -= rs.mean()
        ra -= ra.mean()
        den = math.sqrt((rs * rs).sum() * (ra * ra).sum())
        vals.append((rs * ra).sum() / den if den > 0 else 1.0)
    return float(np.mean(vals))


def topk_recall_vs_post(S, A, k: int):
    """Fraction of the exact-A top-k blocks that the S~ top-k also keeps.

    Diagnostic of selection quality; no value on the pages. Pinned by a
    hand-worked row, brute-force set intersection, and the 1 / 0 limits.
    """
    idx_s, _ = select_topk(S, k)
    idx_a, _ = select_topk(A, k)
    hits = 0
    total = 0
    for a_row, s_row in zip(idx_a.reshape(-1, k), idx_s.reshape(-1, k)):
        hits += len(set(a_row.tolist()) & set(s_row.tolist()))
        total += k
    return hits / total
