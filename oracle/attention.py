"""Plain fp64 CPU oracle for exact softmax attention and its analytic backward.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or link
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it. It shares no code with the CUDA library and imports
nothing from the ``exact_io_aware_61_b200`` package.

What it computes (and where the pages define it):

* Scores ``S = Q K^T / sqrt(d)`` -- mentria.ai "Exact attention, sped up by
  never writing the giant grid down", section "So don't load it all. Work one
  block at a time." (block score equation). The scale is an explicit argument.
* The optional mask, applied to the scores before the softmax --
  fanfani.net "FlashAttention", section "The bottleneck was never the
  arithmetic". The pages do not define the mask; the reading taken here is the
  causal one: key ``j`` is visible to query ``i`` iff ``j <= i`` (square,
  top-left aligned).
* The max-subtracted softmax of each full score row -- mentria.ai, section
  "But softmax needs the whole row at once." (safe-softmax equation).
* ``O = P V`` and the per-row log-sum-exp ``LSE = m + ln(l)`` of the scaled
  scores, the statistics the forward keeps for the backward -- fanfani.net,
  section "The backward pass, and where the memory saving comes from";
  synthetic.wiki "FlashAttention: attention's bottleneck is the wire, not the
  maths", section "The backward pass buys memory with recompute".
* The blockwise online-softmax pass (running max ``m``, running normaliser
  ``l``, running output ``o``, each rescaled by ``exp(m_old - m_new)``) --
  fanfani.net, section "A pinch of math: making the softmax work in pieces";
  mentria.ai, section "The trick: keep a running max, and rebase as you go.".
  It exists here only to pin the full-row oracle against the pages' claim that
  the blockwise result is the same answer.
* The backward pass. The pages only say that the score blocks are recomputed
  from Q, K and the saved statistics; the gradient itself is the textbook
  derivative of the softmax definition above:
  ``dV = P^T dO``, ``dP = dO V^T``, ``D = rowsum(dO * O)``,
  ``dS = P * (dP - D)``, ``dQ = scale dS K``, ``dK = scale dS^T Q``.

Grouped-query attention (synthetic.wiki, section "Versions, and what the
numbers say", names MQA/GQA without a head mapping): query head ``h`` reads
KV head ``h // (Hq // Hkv)``; dK and dV sum over the query heads of a group.

A row with no visible key (impossible for the square causal mask, kept for
completeness) gets ``O = 0`` and ``LSE = -inf``.

Queries against a longer key sequence (a KV cache: ``Nq`` new queries, ``Nk``
cached keys that include them). The pages name the KV cache as what now
limits serving (fanfani.net, section "The backward pass, and where the memory
saving comes from"; synthetic.wiki, section "Where to be careful") without a
formula; the reading taken here is the usual one: the queries are the last ``Nq`` positions, so query ``i`` sits at
position ``Nk - Nq + i`` and, under the causal mask, sees keys ``j <= Nk - Nq
+ i``. ``merge_partial_states`` combines softmax states of disjoint key sets
with the rescale rule of fanfani.net, section "A pinch of math: making the
softmax work in pieces" (the same rule that carries the running state from one
key block to the next).

Variable-length batches (sequences of different lengths packed one after
another, ``[tokens, heads, d]``, located by cumulative offsets) are attention
within each sequence and nothing across sequences; the pages say nothing on
layouts ("the softmax attention you asked for", synthetic.wiki, section "Where
to be careful"), and the reading taken is the plain one.

Queries and keys at arbitrary sequence positions (``attention_forward_positions``)
and the merge of normalised outputs of disjoint key sets (``merge_outputs``) are
what attention sharded over the sequence dimension computes on each device and
combines across devices. The pages name parallelism over the sequence dimension
(synthetic.wiki, section "Versions, and what the numbers say") and give the
rescale rule that makes the merge exact (fanfani.net, section "A pinch of math:
making the softmax work in pieces"), but no formula for the sharded form; the
reading taken is the plain one: under the causal mask a key is visible to a query
iff its position is not after the query's, and a normalised output ``O_s`` with
its ``LSE_s`` is the softmax state ``(m = LSE_s, l = 1, o = O_s)`` of its key set.

Layouts: Q, O, dO, dQ are ``[B, Hq, N, d]``; K, V, dK, dV are
``[B, Hkv, N, d]``; LSE and D are ``[B, Hq, N]``. All arithmetic is float64.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "kv_head_of",
    "masked_scores",
    "softmax_rows",
    "attention_probs",
    "attention_forward",
    "attention_forward_rows",
    "online_softmax_forward",
    "attention_backward",
    "attention_backward_rows",
    "score_matrix_bytes",
    "attention_forward_kvcache",
    "attention_forward_varlen",
    "attention_backward_varlen",
    "partial_state",
    "merge_partial_states",
    "attention_forward_positions",
    "merge_outputs",
    "attention_backward_block",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def kv_head_of(hq: int, Hq: int, Hkv: int) -> int:
    """KV head read by query head ``hq``: contiguous groups of ``Hq // Hkv``."""
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return hq // (Hq // Hkv)


def masked_scores(q_bh, k_bh, scale: float, causal: bool, rows=None, keys=None) -> np.ndarray:
    """Scaled scores ``scale * Q K^T`` of one head, masked entries set to -inf.

    ``q_bh`` is ``[N, d]`` (or ``[len(rows), d]`` when ``rows`` lists the query
    positions it holds), ``k_bh`` is ``[N, d]`` (at positions ``keys`` when
    given, else ``0 .. N-1``). Returns ``[n_rows, N]``.
    """
    q_bh = _f64(q_bh)
    k_bh = _f64(k_bh)
    n_keys = k_bh.shape[0]
    s = scale * (q_bh @ k_bh.T)
    if causal:
        qpos = np.arange(q_bh.shape[0]) if rows is None else np.asarray(rows)
        kpos = np.arange(n_keys) if keys is None else np.asarray(keys)
        s = np.where(kpos[None, :] <= qpos[:, None], s, -np.inf)
    return s


def softmax_rows(s: np.ndarray):
    """Max-subtracted softmax of every row of ``s``.

    Returns ``(P, m, l)`` with ``m`` the row maximum and ``l`` the sum of
    ``exp(s - m)``, so that ``P = exp(s - m) / l``. Rows that are entirely
    -inf give ``P = 0``, ``m = -inf``, ``l = 0``.
    """
    m = np.max(s, axis=-1)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    e = np.exp(s - m_safe[..., None])  # exp(-inf) = 0 for masked entries
    l = np.sum(e, axis=-1)
    with np.errstate(invalid="ignore", divide="ignore"):
        p = np.where(finite[..., None], e / np.where(finite, l, 1.0)[..., None], 0.0)
    l = np.where(finite, l, 0.0)
    return p, m, l


def _lse(m, l):
    with np.errstate(divide="ignore"):
        return np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), -np.inf)


def attention_probs(q, k, scale: float, causal: bool) -> np.ndarray:
    """Full attention-weight tensor ``P`` of shape ``[B, Hq, N, N]``."""
    q = _f64(q)
    k = _f64(k)
    B, Hq, N, _ = q.shape
    Hkv = k.shape[1]
    p = np.empty((B, Hq, N, N))
    for b in range(B):
        for h in range(Hq):
            s = masked_scores(q[b, h], k[b, kv_head_of(h, Hq, Hkv)], scale, causal)
            p[b, h] = softmax_rows(s)[0]
    return p


def attention_forward(q, k, v, scale: float, causal: bool):
    """Exact attention, materialising each head's N x N score matrix.

    Returns ``(O [B,Hq,N,d], LSE [B,Hq,N])`` in float64.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    o = np.empty((B, Hq, N, v.shape[-1]))
    lse = np.empty((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            hk = kv_head_of(h, Hq, Hkv)
            s = masked_scores(q[b, h], k[b, hk], scale, causal)
            p, m, l = softmax_rows(s)
            o[b, h] = p @ v[b, hk]
            lse[b, h] = _lse(m, l)
    return o, lse


def attention_forward_rows(q, k, v, scale: float, causal: bool, b: int, h: int, rows):
    """Exact attention for the listed query positions of one (batch, head).

    Same definition as :func:`attention_forward`, restricted to the query
    positions ``rows`` of batch ``b``, query head ``h``; used to check sampled
    rows of workloads too large to materialise whole. Returns
    ``(O_rows [len(rows), d], LSE_rows [len(rows)])``.
    """
    rows = np.asarray(rows, dtype=np.int64)
    Hq = np.shape(q)[1]
    Hkv = np.shape(k)[1]
    hk = kv_head_of(h, Hq, Hkv)
    q_rows = _f64(np.asarray(q)[b, h][rows])
    k_bh = _f64(np.asarray(k)[b, hk])
    v_bh = _f64(np.asarray(v)[b, hk])
    s = masked_scores(q_rows, k_bh, scale, causal, rows=rows)
    p, m, l = softmax_rows(s)
    return p @ v_bh, _lse(m, l)


def online_softmax_forward(q, k, v, scale: float, causal: bool, block: int):
    """Blockwise online-softmax attention in float64, keys taken ``block`` at a time.

    Per query row it carries the running maximum ``m``, the running normaliser
    ``l`` and the running weighted sum ``o``. For each key block with block
    maximum ``m_blk``: ``m_new = max(m, m_blk)``, ``alpha = exp(m - m_new)``
    (0 while ``m`` is still -inf), ``l = alpha l + sum exp(s - m_new)``,
    ``o = alpha o + sum exp(s - m_new) v``. After the last block ``O = o / l``
    once, and ``LSE = m + ln l``. The last block may be shorter than ``block``.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    dv = v.shape[-1]
    o_out = np.empty((B, Hq, N, dv))
    lse_out = np.empty((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            hk = kv_head_of(h, Hq, Hkv)
            m = np.full(N, -np.inf)
            l = np.zeros(N)
            o = np.zeros((N, dv))
            for j0 in range(0, N, block):
                j1 = min(j0 + block, N)
                s = scale * (q[b, h] @ k[b, hk, j0:j1].T)
                if causal:
                    qpos = np.arange(N)[:, None]
                    kpos = np.arange(j0, j1)[None, :]
                    s = np.where(kpos <= qpos, s, -np.inf)
                m_blk = np.max(s, axis=1)
                m_new = np.maximum(m, m_blk)
                seen = np.isfinite(m_new)
                m_ref = np.where(seen, m_new, 0.0)
                with np.errstate(invalid="ignore"):
                    alpha = np.where(np.isfinite(m), np.exp(m - m_ref), 0.0)
                e = np.exp(s - m_ref[:, None])
                l = alpha * l + e.sum(axis=1)
                o = alpha[:, None] * o + e @ v[b, hk, j0:j1]
                m = m_new
            with np.errstate(invalid="ignore", divide="ignore"):
                o_out[b, h] = np.where(l[:, None] > 0, o / np.where(l > 0, l, 1.0)[:, None], 0.0)
            lse_out[b, h] = _lse(m, l)
    return o_out, lse_out


def attention_backward(q, k, v, do, scale: float, causal: bool):
    """Analytic gradients of ``O = softmax(scale Q K^T [+mask]) V``.

    Given the upstream gradient ``dO`` returns ``(dQ, dK, dV, D)`` where
    ``D = rowsum(dO * O)`` is the per-row term of the softmax Jacobian.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    do = _f64(do)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    D = np.empty((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            hk = kv_head_of(h, Hq, Hkv)
            s = masked_scores(q[b, h], k[b, hk], scale, causal)
            p = softmax_rows(s)[0]
            o = p @ v[b, hk]
            dv[b, hk] += p.T @ do[b, h]
            dp = do[b, h] @ v[b, hk].T
            D[b, h] = np.sum(do[b, h] * o, axis=1)
            ds = score_gradient(p, dp, D[b, h])
            dq[b, h] = scale * (ds @ k[b, hk])
            dk[b, hk] += scale * (ds.T @ q[b, h])
    return dq, dk, dv, D


def attention_backward_rows(q, k, v, do, scale: float, causal: bool, b: int, h: int, rows):
    """The backward restricted to the query positions ``rows`` of one (batch, head).

    Same formulas as :func:`attention_backward`. Returns ``(dQ_rows, dK_part,
    dV_part)``: the dQ rows of those queries and the share of dK and dV (of
    the KV head ``h`` reads) that those queries contribute. Summing the shares
    over a partition of all rows and heads of a group gives dK and dV.
    """
    rows = np.asarray(rows, dtype=np.int64)
    Hq = np.shape(q)[1]
    Hkv = np.shape(k)[1]
    hk = kv_head_of(h, Hq, Hkv)
    q_rows = _f64(np.asarray(q)[b, h][rows])
    do_rows = _f64(np.asarray(do)[b, h][rows])
    k_bh = _f64(np.asarray(k)[b, hk])
    v_bh = _f64(np.asarray(v)[b, hk])
    s = masked_scores(q_rows, k_bh, scale, causal, rows=rows)
    p = softmax_rows(s)[0]
    o_rows = p @ v_bh
    dv_part = p.T @ do_rows
    dp = do_rows @ v_bh.T
    D = np.sum(do_rows * o_rows, axis=1)
    ds = score_gradient(p, dp, D)
    return scale * (ds @ k_bh), scale * (ds.T @ q_rows), dv_part


def score_gradient(p, dp, D):
    """Gradient with respect to the (pre-softmax) scores: ``P * (dP - D)``."""
    return p * (dp - D[:, None])


def score_matrix_bytes(N: int, heads: int, bytes_per_element: int) -> int:
    """Bytes the unfused path would need to hold the N x N scores of ``heads`` heads."""
    return N * N * heads * bytes_per_element


def attention_forward_kvcache(q, k, v, scale: float, causal: bool):
    """Exact attention of ``Nq`` queries against ``Nk >= Nq`` keys.

    ``q`` is ``[B, Hq, Nq, d]``, ``k`` and ``v`` are ``[B, Hkv, Nk, d]``. Query
    ``i`` is at position ``Nk - Nq + i``; with ``causal`` it sees the keys at
    positions up to its own. Returns ``(O [B,Hq,Nq,d], LSE [B,Hq,Nq])``.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, Hq, Nq, _ = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if Nq > Nk:
        raise ValueError("a KV cache holds at least the queries' own positions")
    pos = Nk - Nq + np.arange(Nq)
    o = np.empty((B, Hq, Nq, v.shape[-1]))
    lse = np.empty((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            hk = kv_head_of(h, Hq, Hkv)
            p, m, l = softmax_rows(masked_scores(q[b, h], k[b, hk], scale, causal, rows=pos))
            o[b, h] = p @ v[b, hk]
            lse[b, h] = _lse(m, l)
    return o, lse


def partial_state(s, v):
    """Softmax state of one set of keys: ``(m, l, o)`` per query row.

    ``s`` holds the (masked) scaled scores ``[rows, keys]`` of the set and ``v``
    its values ``[keys, d]``: ``m`` is the row maximum, ``l = sum exp(s - m)``
    and ``o = sum exp(s - m) v`` (not divided by ``l``). A row with every key
    masked has ``m = -inf``, ``l = 0``, ``o = 0``.
    """
    p, m, l = softmax_rows(_f64(s))
    return m, l, (p * l[:, None]) @ _f64(v)


def merge_partial_states(ms, ls, os):
    """Combine softmax states of disjoint key sets into ``(O, LSE)``.

    ``ms``, ``ls`` are ``[sets, rows]`` and ``os`` is ``[sets, rows, d]``, each
    set's state as :func:`partial_state` gives it. With ``M = max_s m_s``, the
    states are rescaled by ``exp(m_s - M)`` and added: ``L = sum_s l_s
    exp(m_s - M)``, ``o = sum_s o_s exp(m_s - M)``; then ``O = o / L`` and
    ``LSE = M + ln L``.
    """
    ms, ls, os = _f64(ms), _f64(ls), _f64(os)
    M = np.max(ms, axis=0)
    M_safe = np.where(np.isfinite(M), M, 0.0)
    w = np.where(np.isfinite(ms), np.exp(ms - M_safe[None, :]), 0.0)
    L = np.sum(w * ls, axis=0)
    o = np.sum(w[:, :, None] * os, axis=0)
    with np.errstate(invalid="ignore", divide="ignore"):
        out = np.where(L[:, None] > 0, o / np.where(L > 0, L, 1.0)[:, None], 0.0)
    return out, _lse(M, L)


def attention_forward_varlen(q, k, v, cu_q, cu_k, scale: float, causal: bool):
    """Attention within each sequence of a packed variable-length batch.

    ``q`` is ``[total_q, Hq, d]`` and ``k``, ``v`` are ``[total_k, Hkv, d]``:
    sequence ``s`` owns query rows ``cu_q[s] .. cu_q[s+1]-1`` and key rows
    ``cu_k[s] .. cu_k[s+1]-1`` (``cu_q``, ``cu_k`` non-decreasing, starting at
    0, one entry more than sequences). A sequence may have fewer queries than
    keys; its queries are then its last positions, as in
    :func:`attention_forward_kvcache`. Returns ``(O [total_q, Hq, d], LSE
    [total_q, Hq])``.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    cu_q = np.asarray(cu_q, dtype=np.int64)
    cu_k = np.asarray(cu_k, dtype=np.int64)
    if cu_q.shape != cu_k.shape or cu_q[0] != 0 or cu_k[0] != 0:
        raise ValueError("cu_q and cu_k must start at 0 and have one entry per sequence boundary")
    Hq, Hkv = q.shape[1], k.shape[1]
    o = np.empty((q.shape[0], Hq, v.shape[-1]))
    lse = np.empty((q.shape[0], Hq))
    for s in range(len(cu_q) - 1):
        q0, q1, k0, k1 = cu_q[s], cu_q[s + 1], cu_k[s], cu_k[s + 1]
        if q1 - q0 > k1 - k0:
            raise ValueError("a sequence has more queries than keys")
        pos = (k1 - k0) - (q1 - q0) + np.arange(q1 - q0)
        for h in range(Hq):
            hk = kv_head_of(h, Hq, Hkv)
            p, m, l = softmax_rows(masked_scores(q[q0:q1, h], k[k0:k1, hk], scale, causal, rows=pos))
            o[q0:q1, h] = p @ v[k0:k1, hk]
            lse[q0:q1, h] = _lse(m, l)
    return o, lse


def attention_forward_positions(q, k, v, q_pos, k_pos, scale: float, causal: bool):
    """Exact attention of queries at sequence positions ``q_pos`` against keys at ``k_pos``.

    ``q`` is ``[B, Hq, Nq, d]``, ``k`` and ``v`` are ``[B, Hkv, Nk, d]``,
    ``q_pos`` has ``Nq`` and ``k_pos`` ``Nk`` integer entries (any order). With
    ``causal``, key ``j`` is visible to query ``i`` iff ``k_pos[j] <= q_pos[i]``.
    A row that sees no key gets ``O = 0`` and ``LSE = -inf``. Returns
    ``(O [B,Hq,Nq,d], LSE [B,Hq,Nq])``.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, Hq, Nq, _ = q.shape
    Hkv = k.shape[1]
    q_pos = np.asarray(q_pos, dtype=np.int64)
    k_pos = np.asarray(k_pos, dtype=np.int64)
    if q_pos.shape != (Nq,) or k_pos.shape != (k.shape[2],):
        raise ValueError("one position per query row and per key row")
    o = np.empty((B, Hq, Nq, v.shape[-1]))
    lse = np.empty((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            hk = kv_head_of(h, Hq, Hkv)
            s = masked_scores(q[b, h], k[b, hk], scale, causal, rows=q_pos, keys=k_pos)
            p, m, l = softmax_rows(s)
            o[b, h] = p @ v[b, hk]
            lse[b, h] = _lse(m, l)
    return o, lse


def merge_outputs(os, lses):
    """Combine the normalised outputs of disjoint key sets into ``(O, LSE)``.

    ``os`` is ``[sets, rows, d]`` and ``lses`` is ``[sets, rows]``: set ``s``
    gave ``O_s`` and ``LSE_s`` for its keys alone. ``(O_s, LSE_s)`` is the
    softmax state ``m = LSE_s``, ``l = 1``, ``o = O_s`` of its keys (both give
    ``l e^m = e^LSE_s`` and ``o / l = O_s``), so :func:`merge_partial_states`
    combines them; a set with ``LSE_s = -inf`` (no visible key) has ``l = 0``
    and contributes nothing.
    """
    os, lses = _f64(os), _f64(lses)
    finite = np.isfinite(lses)
    return merge_partial_states(lses, finite.astype(np.float64), np.where(finite[..., None], os, 0.0))


def attention_backward_varlen(q, k, v, do, cu_q, cu_k, scale: float, causal: bool):
    """Gradients of :func:`attention_forward_varlen` for the upstream gradient ``do``.

    Layouts as in the forward: ``q``, ``do`` are ``[total_q, Hq, d]``, ``k``,
    ``v`` are ``[total_k, Hkv, d]``. Each sequence is its own problem, with its
    queries at its last positions; the formulas are those of
    :func:`attention_backward`, per sequence and head, and dK, dV sum over the
    query heads of a KV head's group. A key no query sees gets zero gradient.
    Returns ``(dQ [total_q, Hq, d], dK [total_k, Hkv, d], dV [total_k, Hkv, d])``.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    do = _f64(do)
    cu_q = np.asarray(cu_q, dtype=np.int64)
    cu_k = np.asarray(cu_k, dtype=np.int64)
    if cu_q.shape != cu_k.shape or cu_q[0] != 0 or cu_k[0] != 0:
        raise ValueError("cu_q and cu_k must start at 0 and have one entry per sequence boundary")
    Hq, Hkv = q.shape[1], k.shape[1]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for sq in range(len(cu_q) - 1):
        q0, q1, k0, k1 = cu_q[sq], cu_q[sq + 1], cu_k[sq], cu_k[sq + 1]
        if q1 - q0 > k1 - k0:
            raise ValueError("a sequence has more queries than keys")
        pos = (k1 - k0) - (q1 - q0) + np.arange(q1 - q0)
        for h in range(Hq):
            hk = kv_head_of(h, Hq, Hkv)
            qs, ks, vs, dos = q[q0:q1, h], k[k0:k1, hk], v[k0:k1, hk], do[q0:q1, h]
            p = softmax_rows(masked_scores(qs, ks, scale, causal, rows=pos))[0]
            dv[k0:k1, hk] += p.T @ dos
            dp = dos @ vs.T
            D = np.sum(dos * (p @ vs), axis=1)
            ds = score_gradient(p, dp, D)
            dq[q0:q1, h] = scale * (ds @ ks)
            dk[k0:k1, hk] += scale * (ds.T @ qs)
    return dq, dk, dv


def attention_backward_block(q, k, v, do, lse, D, q_pos, k_pos, scale: float, causal: bool):
    """The share of one key block in the gradients, given the full rows' statistics.

    ``q``, ``do`` are ``[B, Hq, Nq, d]`` at positions ``q_pos``; ``k``, ``v``
    are ``[B, Hkv, Nk, d]`` at positions ``k_pos`` (one block of a longer key
    sequence); ``lse`` and ``D = rowsum(dO * O)`` are ``[B, Hq, Nq]`` for the
    queries' whole rows (every key block). With those, the weights of the
    block's keys are ``P = exp(scale S - LSE)`` (masked entries 0), and the
    block adds ``dQ += scale dS K``, ``dK = scale dS^T Q``, ``dV = P^T dO``
    with ``dS = P * (dP - D)``, ``dP = dO V^T`` (the formulas of
    :func:`attention_backward`, restricted to the block's keys). Summed over
    a partition of the keys they give :func:`attention_backward`. Returns
    ``(dQ [B,Hq,Nq,d], dK [B,Hkv,Nk,d], dV [B,Hkv,Nk,d])``.
    """
    q, k, v, do, lse, D = (_f64(x) for x in (q, k, v, do, lse, D))
    B, Hq = q.shape[:2]
    Hkv = k.shape[1]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            hk = kv_head_of(h, Hq, Hkv)
            s = masked_scores(q[b, h], k[b, hk], scale, causal, rows=q_pos, keys=k_pos)
            with np.errstate(invalid="ignore"):
                p = np.where(np.isfinite(s), np.exp(s - lse[b, h][:, None]), 0.0)
            dv[b, hk] += p.T @ do[b, h]
            ds = score_gradient(p, do[b, h] @ v[b, hk].T, D[b, h])
            dq[b, h] = scale * (ds @ k[b, hk])
            dk[b, hk] += scale * (ds.T @ q[b, h])
    return dq, dk, dv
