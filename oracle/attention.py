"""Plain fp64 CPU oracle for exact attention: forward, backward, softmax merge.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
it is called by ``tests/``, by ``__graft_entry__.smoke()`` and by the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``, and by nothing
else.  It shares no code with the CUDA path (no kernels, headers, helpers or
constants); both sides only share the seeded input generator, which holds none
of the method's arithmetic.

Sources (the pages this follows; cited by title and section):

[P1] "Flash Attention: Rivoluzionando l'Efficienza dei Modelli Transformer"
     (unite.ai): the ``standard_attention`` listing (definition of the result),
     section "La Matematica dietro Flash Attention" (softmax decomposition and
     the softmax merge), section "Dettagli di Implementazione" (the blockwise
     algorithm with running statistics M, L).
[P5] "Flash Attention: بهینه‌سازی مکانیزم توجه در ترنسفورمرها" (deepfa.ir):
     section "ساختار مکانیزم توجه" (Attention(Q,K,V) = softmax(QK^T/sqrt d) V),
     section "تکنیک 2: محاسبه مجدد" (the backward recomputes the attention
     matrix instead of storing it).
[P3] nearauto.com FlashAttention-2 digest, section on reducing non-matmul
     FLOPs (normalise once, outputs unchanged), and section
     "新機能: 最大256のヘッドディメンション、マルチクエリアテンション" (multi-query and
     grouped-query attention: one key/value head shared by a set of query
     heads); the unite.ai page lists the same variants under "FlashAttention-2".

Every function here is the plain definition written out in float64 with numpy:
the score matrix S and the probabilities P are materialised for whole rows,
the softmax is two-pass (max, then exp / sum).  The only exception is
``attention_fwd_blockwise``, which deliberately takes the pages' tiled steps so
that the merge identity can be pinned against the two-pass definition.

Readings where the pages are silent or garbled:
  * layout [B, H, N, d]: the pages' (batch, seq, d) with a head axis added;
  * lse is the natural log of sum_j exp(scale * q_i . k_j) over unmasked j;
  * causal masks j > i (top-left aligned, N_q == N_k);
  * the printed blockwise listing divides the output by the new running sum
    while rescaling the old (already divided) output by exp(m_old - m_new)
    alone; we keep the output unnormalised and divide once at the end;
  * the garbled merge formula is read as l = e^(m_x-m) l_x + e^(m_y-m) l_y and
    softmax(x u y) = [e^(m_x-m) l_x softmax(x), e^(m_y-m) l_y softmax(y)] / l;
  * the backward is the exact gradient of the forward (the pages only say
    "recompute"), with D_i = sum_j P_ij dP_ij;
  * fewer queries than keys (decode, N_q < N_k): the queries are the last
    N_q positions of the sequence, so causal query i sees keys j <= N_k - N_q + i
    (bottom-right alignment; with N_q == N_k it is the usual mask);
  * grouped-query attention: the pages say each set of query heads shares one
    key/value head but not which; the sets are contiguous, query head h using
    key/value head h // (H / H_kv), and a shared head's gradient is the sum of
    the gradients of its uses.
  * any number of queries against any number of keys (the library interface
    users of the integrations in [P5] "پیاده‌سازی و استفاده از Flash Attention"
    expect; the pages define no variant): causal alignment stays bottom-right,
    query i sees keys j <= N_k - N_q + i, so with N_q > N_k the first
    N_q - N_k queries see no key at all.  A query that sees no key (also
    N_k = 0) has O = 0 (the empty weighted sum) and lse = -inf (ln of an empty
    sum); its gradient is zero;
  * variable-length batches: sequence b is the packed rows cu_q[b]:cu_q[b+1]
    of q [T_q, H, d] and cu_k[b]:cu_k[b+1] of k, v [T_k, H_kv, d]; each
    sequence is its own attention problem; lse is stored [H, T_q].

Parity pins for every function live in tests/test_oracle.py; none of the
functions below is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "as_f64",
    "attention_fwd",
    "attention_fwd_rows",
    "attention_bwd",
    "attention_fwd_gqa",
    "attention_bwd_gqa",
    "attention_fwd_decode",
    "attention_fwd_general",
    "attention_bwd_general",
    "attention_fwd_varlen",
    "attention_bwd_varlen",
    "softmax_merge",
    "attention_fwd_blockwise",
    "bwd_operand_rounding_bound",
    "attention_bwd_sampled",
]


def as_f64(x) -> np.ndarray:
    """Return ``x`` as a C-contiguous float64 numpy array (exact for bf16/fp32)."""
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _scores(q_rows: np.ndarray, k: np.ndarray, scale: float, row_idx: np.ndarray,
            causal: bool) -> np.ndarray:
    """S = scale * Q K^T for the given query rows of one head, masked if causal.

    [P1] ``standard_attention`` listing: scores = Q K^T / sqrt(d_k);
    [P5] "ساختار مکانیزم توجه".  Causal: s_ij = -inf for j > i.
    """
    s = scale * (q_rows @ k.T)
    if causal:
        cols = np.arange(k.shape[0])
        s = np.where(cols[None, :] > row_idx[:, None], -np.inf, s)
    return s


def _softmax_rows(s: np.ndarray):
    """Two-pass safe softmax of complete rows; returns (P, lse).

    [P1] "La Matematica dietro Flash Attention", softmax decomposition:
    softmax(x) = exp(x - m) / sum exp(x - m) with m = max x.  The log-sum-exp
    is m + ln(sum exp(x - m)).
    """
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    denom = e.sum(axis=1, keepdims=True)
    p = e / denom
    lse = (m + np.log(denom))[:, 0]
    return p, lse


def attention_fwd(q, k, v, scale: float, causal: bool, panel_rows: int = 2048):
    """O = softmax(scale Q K^T) V and lse per row, for [B, H, N, d] inputs.

    [P1] ``standard_attention``; [P5] "ساختار مکانیزم توجه".  Materialises S
    and P one head at a time, in panels of complete rows (each row is formed in
    full before it is normalised), so memory stays bounded for long N.
    The value width may differ from d (O takes V's last dimension).
    Returns (O [B,H,N,d_v] float64, lse [B,H,N] float64).
    """
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    B, H, N, d = q.shape
    o = np.empty((B, H, N, v.shape[-1]), dtype=np.float64)
    lse = np.empty((B, H, N), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for r0 in range(0, N, panel_rows):
                rows = np.arange(r0, min(N, r0 + panel_rows))
                s = _scores(q[b, h, rows], k[b, h], scale, rows, causal)
                p, l_ = _softmax_rows(s)
                o[b, h, rows] = p @ v[b, h]
                lse[b, h, rows] = l_
    return o, lse


def attention_fwd_rows(q_rows, k, v, row_idx, scale: float, causal: bool):
    """Forward for selected query rows of ONE head, against all N keys.

    ``q_rows`` [R, d] are the query vectors of rows ``row_idx`` (their position
    in the sequence, used by the causal mask); ``k``, ``v`` are [N, d].  Same
    definition as ``attention_fwd``; used to check long sequences on sampled
    rows.  Returns (O [R, d], lse [R]).
    """
    q_rows, k, v = as_f64(q_rows), as_f64(k), as_f64(v)
    row_idx = np.asarray(row_idx, dtype=np.int64)
    s = _scores(q_rows, k, scale, row_idx, causal)
    p, lse = _softmax_rows(s)
    return p @ v, lse


def attention_bwd(q, k, v, do, scale: float, causal: bool):
    """Exact gradients (dQ, dK, dV) of sum(dO * O) for O = attention_fwd(...).

    [P5] "تکنیک 2: محاسبه مجدد": the backward recomputes P from Q, K (and the
    saved statistics) instead of reading a stored N x N matrix.  The pages give
    no formulas; the reading is the exact derivative of the forward:
        dV = P^T dO,   dP = dO V^T,   D_i = sum_j P_ij dP_ij,
        dS = P * (dP - D 1^T),   dQ = scale dS K,   dK = scale dS^T Q.
    P is this oracle's own fp64 probability matrix (not a device result).
    Returns float64 arrays shaped like q, k, v.
    """
    q, k, v, do = as_f64(q), as_f64(k), as_f64(v), as_f64(do)
    B, H, N, d = q.shape
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    rows = np.arange(N)
    for b in range(B):
        for h in range(H):
            s = _scores(q[b, h], k[b, h], scale, rows, causal)
            p, _ = _softmax_rows(s)
            dv[b, h] = p.T @ do[b, h]
            dp = do[b, h] @ v[b, h].T
            dd = (p * dp).sum(axis=1, keepdims=True)
            ds = p * (dp - dd)
            dq[b, h] = scale * (ds @ k[b, h])
            dk[b, h] = scale * (ds.T @ q[b, h])
    return dq, dk, dv


def attention_bwd_sampled(q, k, v, do, rows, keys, scale: float, causal: bool, panel_rows: int = 2048):
    """Selected entries of the exact gradients of ONE head, for sequences too long to
    hold S: dQ at query rows ``rows`` and dK, dV at key rows ``keys``.

    Same definition as ``attention_bwd`` ([P5] "تکنیک 2: محاسبه مجدد", read as the
    exact derivative): with P_ij = exp(scale q_i.k_j - lse_i) (masked entries 0),
    dP_ij = dO_i.v_j and D_i = sum_c dO_ic O_ic,
        dQ_i = scale sum_j P_ij (dP_ij - D_i) k_j,
        dV_j = sum_i P_ij dO_i,      dK_j = scale sum_i P_ij (dP_ij - D_i) q_i.
    lse and O of every row come from ``attention_fwd`` (complete rows, in panels);
    each requested dQ row then takes its complete row of P, and each requested key
    its complete column.  q, k, v, do are [N, d]; returns (dq [len(rows), d],
    dk [len(keys), d], dv [len(keys), d]) in float64.
    """
    q, k, v, do = as_f64(q), as_f64(k), as_f64(v), as_f64(do)
    N = q.shape[0]
    o, lse = attention_fwd(q[None, None], k[None, None], v[None, None], scale, causal, panel_rows)
    o, lse = o[0, 0], lse[0, 0]
    dd = (do * o).sum(axis=1)
    rows = np.asarray(rows, dtype=np.int64)
    keys = np.asarray(keys, dtype=np.int64)
    s = _scores(q[rows], k, scale, rows, causal)                      # complete rows
    p = np.exp(s - lse[rows, None])
    dq = scale * ((p * (do[rows] @ v.T - dd[rows, None])) @ k)
    st = scale * (q @ k[keys].T)                                      # complete columns
    if causal:
        st = np.where(keys[None, :] > np.arange(N)[:, None], -np.inf, st)
    pt = np.exp(st - lse[:, None])
    dst = pt * (do @ v[keys].T - dd[:, None])
    return dq, scale * (dst.T @ q), pt.T @ do


def _kv_head(h: int, H: int, H_kv: int) -> int:
    """Key/value head read by query head h: contiguous sets of H / H_kv query heads."""
    if H_kv < 1 or H % H_kv != 0:
        raise ValueError("the query head count must be a multiple of the key/value head count")
    return h // (H // H_kv)


def attention_fwd_gqa(q, k, v, scale: float, causal: bool):
    """Grouped-query (and multi-query, H_kv = 1) forward.

    [P3] "新機能: 最大256のヘッドディメンション、マルチクエリアテンション": a set of
    query heads shares one key/value head.  q is [B, H, N, d]; k, v are
    [B, H_kv, N, d] with H a multiple of H_kv.  Each query head is exactly the
    ``attention_fwd`` of its own queries against its set's keys and values.
    Returns (O [B,H,N,d_v], lse [B,H,N]) in float64.
    """
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    B, H, N, _ = q.shape
    H_kv = k.shape[1]
    o = np.empty((B, H, N, v.shape[-1]), dtype=np.float64)
    lse = np.empty((B, H, N), dtype=np.float64)
    for h in range(H):
        g = _kv_head(h, H, H_kv)
        o_h, lse_h = attention_fwd(q[:, h:h + 1], k[:, g:g + 1], v[:, g:g + 1], scale, causal)
        o[:, h], lse[:, h] = o_h[:, 0], lse_h[:, 0]
    return o, lse


def attention_bwd_gqa(q, k, v, do, scale: float, causal: bool):
    """Exact gradients of sum(dO * O) for O = attention_fwd_gqa(...).

    dQ of a query head is that head's ``attention_bwd`` dQ; a key/value head is
    an input of every query head in its set, so its dK and dV are the sums of
    those heads' dK and dV.  Returns float64 arrays shaped like q, k, v.
    """
    q, k, v, do = as_f64(q), as_f64(k), as_f64(v), as_f64(do)
    B, H, N, _ = q.shape
    H_kv = k.shape[1]
    dq = np.empty_like(q)
    dk, dv = np.zeros_like(k), np.zeros_like(v)
    for h in range(H):
        g = _kv_head(h, H, H_kv)
        dq_h, dk_h, dv_h = attention_bwd(q[:, h:h + 1], k[:, g:g + 1], v[:, g:g + 1], do[:, h:h + 1], scale, causal)
        dq[:, h] = dq_h[:, 0]
        dk[:, g] += dk_h[:, 0]
        dv[:, g] += dv_h[:, 0]
    return dq, dk, dv


def attention_fwd_decode(q, k, v, scale: float, causal: bool):
    """Attention of N_q queries against N_k >= N_q keys (decoding against a key/value cache).

    q is [B, H, N_q, d]; k, v are [B, H_kv, N_k, d] (H a multiple of H_kv, as in
    ``attention_fwd_gqa``).  The queries are the last N_q positions of the
    sequence: causal query i sees keys j <= N_k - N_q + i.  Same definition as
    ``attention_fwd`` otherwise ([P1] ``standard_attention``).  The decode
    workload itself is the one the gist.science FlashAttention-V page times
    ("decode"); splitting the keys and merging the partial results is [P1]'s
    softmax merge.  Returns (O [B,H,N_q,d_v], lse [B,H,N_q]) in float64.
    """
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    B, H, Nq, _ = q.shape
    H_kv, Nk = k.shape[1], k.shape[2]
    if Nq > Nk:
        raise ValueError("more queries than keys")
    rows = np.arange(Nk - Nq, Nk)
    o = np.empty((B, H, Nq, v.shape[-1]), dtype=np.float64)
    lse = np.empty((B, H, Nq), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            g = _kv_head(h, H, H_kv)
            s = _scores(q[b, h], k[b, g], scale, rows, causal)
            p, l_ = _softmax_rows(s)
            o[b, h] = p @ v[b, g]
            lse[b, h] = l_
    return o, lse


def _attend(q, k, v, scale: float, causal: bool):
    """One head of one sequence: N_q queries against N_k keys (either may be 0).

    [P1] ``standard_attention`` with the bottom-right causal reading of the
    module doc: S = scale Q K^T, s_ij = -inf for j > N_k - N_q + i; rows that
    keep at least one key get the two-pass softmax; rows that keep none get
    P = 0, O = 0, lse = -inf.  Returns (O [N_q, d_v], lse [N_q], P [N_q, N_k]).
    """
    nq, nk = q.shape[0], k.shape[0]
    s = scale * (q @ k.T)
    if causal:
        last_key = np.arange(nq)[:, None] + (nk - nq)
        s = np.where(np.arange(nk)[None, :] > last_key, -np.inf, s)
    p = np.zeros((nq, nk))
    lse = np.full(nq, -np.inf)
    seen = np.isfinite(s).any(axis=1) if nk > 0 else np.zeros(nq, dtype=bool)
    if seen.any():
        p[seen], lse[seen] = _softmax_rows(s[seen])
    return p @ v, lse, p


def _attend_grad(q, k, v, do, p, scale: float):
    """Exact gradients of one head of one sequence from its probabilities P
    (same formulas as ``attention_bwd``; rows with P = 0 contribute nothing)."""
    dv = p.T @ do
    dp = do @ v.T
    ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
    return scale * (ds @ k), scale * (ds.T @ q), dv


def attention_fwd_general(q, k, v, scale: float, causal: bool):
    """Forward for q [B, H, N_q, d] against k, v [B, H_kv, N_k, d], any N_q, N_k.

    Grouped heads as in ``attention_fwd_gqa``; each (b, h) is ``_attend``.
    Returns (O [B, H, N_q, d_v], lse [B, H, N_q]) in float64.
    """
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    B, H, Nq, _ = q.shape
    H_kv = k.shape[1]
    o = np.empty((B, H, Nq, v.shape[-1]))
    lse = np.empty((B, H, Nq))
    for b in range(B):
        for h in range(H):
            g = _kv_head(h, H, H_kv)
            o[b, h], lse[b, h], _ = _attend(q[b, h], k[b, g], v[b, g], scale, causal)
    return o, lse


def attention_bwd_general(q, k, v, do, scale: float, causal: bool):
    """Exact gradients of sum(dO * O) for O = attention_fwd_general(...); a
    shared key/value head sums the gradients of its uses."""
    q, k, v, do = as_f64(q), as_f64(k), as_f64(v), as_f64(do)
    B, H = q.shape[:2]
    H_kv = k.shape[1]
    dq = np.empty_like(q)
    dk, dv = np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            g = _kv_head(h, H, H_kv)
            _, _, p = _attend(q[b, h], k[b, g], v[b, g], scale, causal)
            dq[b, h], dk_h, dv_h = _attend_grad(q[b, h], k[b, g], v[b, g], do[b, h], p, scale)
            dk[b, g] += dk_h
            dv[b, g] += dv_h
    return dq, dk, dv


def _check_offsets(cu, total: int) -> np.ndarray:
    cu = np.asarray(cu, dtype=np.int64)
    if cu.ndim != 1 or cu.size < 1 or cu[0] != 0 or cu[-1] != total or np.any(np.diff(cu) < 0):
        raise ValueError("sequence offsets must start at 0, never decrease and end at the row count")
    return cu


def attention_fwd_varlen(q, k, v, cu_q, cu_k, scale: float, causal: bool):
    """Variable-length batch: q [T_q, H, d], k, v [T_k, H_kv, d] packed by sequence.

    Sequence b is rows cu_q[b]:cu_q[b+1] of q against rows cu_k[b]:cu_k[b+1]
    of k and v, each head by ``_attend``.  Returns (O [T_q, H, d_v],
    lse [H, T_q]) in float64.
    """
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    cu_q, cu_k = _check_offsets(cu_q, q.shape[0]), _check_offsets(cu_k, k.shape[0])
    if cu_q.size != cu_k.size:
        raise ValueError("query and key offsets describe different batch sizes")
    H, H_kv = q.shape[1], k.shape[1]
    o = np.zeros((q.shape[0], H, v.shape[-1]))
    lse = np.full((H, q.shape[0]), -np.inf)
    for b in range(cu_q.size - 1):
        qs, ks = slice(cu_q[b], cu_q[b + 1]), slice(cu_k[b], cu_k[b + 1])
        for h in range(H):
            g = _kv_head(h, H, H_kv)
            o[qs, h], lse[h, qs], _ = _attend(q[qs, h], k[ks, g], v[ks, g], scale, causal)
    return o, lse


def attention_bwd_varlen(q, k, v, do, cu_q, cu_k, scale: float, causal: bool):
    """Exact gradients of sum(dO * O) for O = attention_fwd_varlen(...)."""
    q, k, v, do = as_f64(q), as_f64(k), as_f64(v), as_f64(do)
    cu_q, cu_k = _check_offsets(cu_q, q.shape[0]), _check_offsets(cu_k, k.shape[0])
    if cu_q.size != cu_k.size:
        raise ValueError("query and key offsets describe different batch sizes")
    H, H_kv = q.shape[1], k.shape[1]
    dq = np.zeros_like(q)
    dk, dv = np.zeros_like(k), np.zeros_like(v)
    for b in range(cu_q.size - 1):
        qs, ks = slice(cu_q[b], cu_q[b + 1]), slice(cu_k[b], cu_k[b + 1])
        for h in range(H):
            g = _kv_head(h, H, H_kv)
            _, _, p = _attend(q[qs, h], k[ks, g], v[ks, g], scale, causal)
            dq[qs, h], dk_h, dv_h = _attend_grad(q[qs, h], k[ks, g], v[ks, g], do[qs, h], p, scale)
            dk[ks, g] += dk_h
            dv[ks, g] += dv_h
    return dq, dk, dv


def softmax_merge(m_x, l_x, o_x, m_y, l_y, o_y):
    """Merge two partial softmax-weighted results over disjoint key sets.

    [P1] "La Matematica dietro Flash Attention", softmax merge, read as: with
    m = max(m_x, m_y),  l = e^(m_x - m) l_x + e^(m_y - m) l_y, and the
    normalised partial outputs o_x = sum_{j in x} softmax(x)_j v_j (likewise
    o_y) combine into
        o = (e^(m_x - m) l_x o_x + e^(m_y - m) l_y o_y) / l.
    Arguments are per-row: m_*, l_* shaped [R], o_* shaped [R, d].  A row with
    m = -inf on one side (no unmasked key there) takes the other side alone.
    Returns (m, l, o).
    """
    m_x, l_x, o_x = as_f64(m_x), as_f64(l_x), as_f64(o_x)
    m_y, l_y, o_y = as_f64(m_y), as_f64(l_y), as_f64(o_y)
    m = np.maximum(m_x, m_y)
    with np.errstate(invalid="ignore"):
        a_x = np.where(np.isneginf(m_x), 0.0, np.exp(m_x - m))
        a_y = np.where(np.isneginf(m_y), 0.0, np.exp(m_y - m))
    w_x = a_x * l_x
    w_y = a_y * l_y
    l = w_x + w_y
    o = (w_x[:, None] * o_x + w_y[:, None] * o_y) / l[:, None]
    return m, l, o


def attention_fwd_blockwise(q, k, v, scale: float, causal: bool,
                            block_q: int = 64, block_k: int = 64):
    """The pages' tiled forward with running row max M and row sum L.

    [P1] "L'Algoritmo di Flash Attention" and "Dettagli di Implementazione":
    queries in blocks, and for each query block a loop over key/value blocks
    that updates M_new = max(M, rowmax S_block), L_new = e^(M - M_new) L +
    rowsum e^(S_block - M_new), and the output.  Reading (see module doc): the
    output is kept unnormalised, O <- e^(M - M_new) O + e^(S_block - M_new) V,
    and divided by L once after the last key block ([P3], fewer non-matmul
    FLOPs, same result).  Key blocks that are entirely masked are skipped.
    Returns (O, lse) like ``attention_fwd``; equal to it up to rounding.
    """
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    B, H, N, d = q.shape
    o_out = np.empty_like(q)
    lse_out = np.empty((B, H, N), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for i0 in range(0, N, block_q):
                rows = np.arange(i0, min(N, i0 + block_q))
                M = np.full(rows.size, -np.inf)
                L = np.zeros(rows.size)
                O = np.zeros((rows.size, d))
                for j0 in range(0, N, block_k):
                    if causal and j0 > rows[-1]:
                        break
                    cols = slice(j0, min(N, j0 + block_k))
                    s = _scores(q[b, h, rows], k[b, h, cols], scale,
                                rows - j0, causal)
                    m_new = np.maximum(M, s.max(axis=1))
                    p = np.exp(s - m_new[:, None])
                    with np.errstate(invalid="ignore"):
                        alpha = np.where(np.isneginf(M), 0.0, np.exp(M - m_new))
                    L = alpha * L + p.sum(axis=1)
                    O = alpha[:, None] * O + p @ v[b, h, cols]
                    M = m_new
                o_out[b, h, rows] = O / L[:, None]
                lse_out[b, h, rows] = M + np.log(L)
    return o_out, lse_out


def bwd_operand_rounding_bound(q, k, v, do, scale: float, causal: bool, unit_roundoff: float = 2.0 ** -8):
    """Elementwise first-order bound on how far rounding the backward's matrix-product
    operands moves the gradients (a tolerance term for the parity tests, not part
    of the attention definition).

    A backward on matrix units rounds P and dS to a narrower format with unit
    roundoff u (2^-8 for bfloat16) before the products dV = P^T dO, dQ = scale dS K
    and dK = scale dS^T Q.  If each operand entry moves by at most u times its
    size, the triangle inequality bounds each output entry's move by
        dV: u (|P|^T |dO|),   dQ: u scale (|dS| |K|),   dK: u scale (|dS|^T |Q|),
    with P and dS this oracle's own (the ``attention_bwd`` quantities).  Grouped
    heads (k, v with H_kv heads, as in ``attention_bwd_gqa``): a shared head's
    bound is the sum over its uses.  Returns (bq, bk, bv) shaped like q, k, v.
    """
    q, k, v, do = as_f64(q), as_f64(k), as_f64(v), as_f64(do)
    B, H, N, _ = q.shape
    H_kv = k.shape[1]
    bq = np.empty_like(q)
    bk, bv = np.zeros_like(k), np.zeros_like(v)
    rows = np.arange(N)
    for b in range(B):
        for h in range(H):
            g = _kv_head(h, H, H_kv)
            s = _scores(q[b, h], k[b, g], scale, rows, causal)
            p, _ = _softmax_rows(s)
            dp = do[b, h] @ v[b, g].T
            ds = np.abs(p * (dp - (p * dp).sum(axis=1, keepdims=True)))
            bq[b, h] = unit_roundoff * scale * (ds @ np.abs(k[b, g]))
            bk[b, g] += unit_roundoff * scale * (ds.T @ np.abs(q[b, h]))
            bv[b, g] += unit_roundoff * (p.T @ np.abs(do[b, h]))
    return bq, bk, bv
