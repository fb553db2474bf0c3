"""Pins for the fp64 CPU oracle, each against something other than the oracle itself.

Every ``check_*`` function below takes the oracle module and raises
``AssertionError`` when a pin fails. The tests run every check on the real
oracle (all must pass) and, at the end of the file, on copies of the oracle
with a planted mistake (a dropped term, a wrong sign, an off-by-one mask, a
transposed operand) to show that each such mistake trips at least one pin.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.attention as ORACLE

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _qkv(B=1, Hq=2, Hkv=1, N=13, d=5, seed=0):
    return (_rand((B, Hq, N, d), seed), _rand((B, Hkv, N, d), seed + 1),
            _rand((B, Hkv, N, d), seed + 2))


# ---------------------------------------------------------------- forward pins

def check_rows_sum_to_one(o):
    # Softmax definition (mentria.ai, "But softmax needs the whole row at once."):
    # each row of weights sums to one.
    for causal in (False, True):
        q, k, _ = _qkv(Hq=4, Hkv=2, N=17, seed=3)
        p = o.attention_probs(q, k, 0.7, causal)
        assert np.all(p >= 0)
        assert np.max(np.abs(p.sum(-1) - 1.0)) < 1e-14
        if causal:
            upper = np.triu(np.ones((17, 17), bool), 1)
            assert np.all(p[..., upper] == 0)


def check_single_key_returns_value(o):
    # N = 1: the only weight is 1, so O = V and LSE is the single scaled score.
    q, k, v = _qkv(B=2, Hq=3, Hkv=3, N=1, d=6, seed=5)
    for causal in (False, True):
        out, lse = o.attention_forward(q, k, v, 0.4, causal)
        assert np.max(np.abs(out - v)) < 1e-15
        ref = 0.4 * np.einsum("bhnd,bhnd->bhn", q, k)
        assert np.max(np.abs(lse - ref)) < 1e-14


def check_zero_query_uniform(o):
    # Q = 0: every visible score is 0, so the weights are uniform over the
    # visible keys: the mean of V (no mask) or the prefix mean (causal), and
    # LSE = ln(number of visible keys).
    N = 11
    _, k, v = _qkv(Hq=2, Hkv=2, N=N, d=4, seed=7)
    q = np.zeros((1, 2, N, 4))
    out, lse = o.attention_forward(q, k, v, 1.3, False)
    assert np.max(np.abs(out - v.mean(axis=2, keepdims=True))) < 1e-14
    assert np.max(np.abs(lse - math.log(N))) < 1e-14
    out, lse = o.attention_forward(q, k, v, 1.3, True)
    prefix = np.cumsum(v, axis=2) / np.arange(1, N + 1)[None, None, :, None]
    assert np.max(np.abs(out - prefix)) < 1e-14
    assert np.max(np.abs(lse - np.log(np.arange(1, N + 1))[None, None, :])) < 1e-14


def check_online_matches_full(o):
    # The pages' claim: the blockwise recurrence gives the same answer as the
    # full-row softmax (fanfani.net, "A pinch of math"; mentria.ai, "Same
    # answer."). fp64, several block sizes including a ragged last block.
    q, k, v = _qkv(B=2, Hq=4, Hkv=2, N=37, d=8, seed=11)
    q = 3.0 * q  # spread the scores so the running max moves
    for causal in (False, True):
        ref_o, ref_l = o.attention_forward(q, k, v, 0.5, causal)
        for block in (1, 4, 16, 36, 37, 64):
            bo, bl = o.online_softmax_forward(q, k, v, 0.5, causal, block)
            assert np.max(np.abs(bo - ref_o)) < 1e-12
            assert np.max(np.abs(bl - ref_l)) < 1e-12


def check_kv_permutation_invariance(o):
    # Without a mask attention is a weighted sum over keys: permuting the
    # (key, value) pairs together leaves O and LSE unchanged.
    q, k, v = _qkv(Hq=2, Hkv=2, N=19, d=6, seed=13)
    perm = np.random.default_rng(0).permutation(19)
    o1, l1 = o.attention_forward(q, k, v, 0.6, False)
    o2, l2 = o.attention_forward(q, k[:, :, perm], v[:, :, perm], 0.6, False)
    assert np.max(np.abs(o1 - o2)) < 1e-13
    assert np.max(np.abs(l1 - l2)) < 1e-13


def check_large_scores_stable_one_hot(o):
    # Max subtraction keeps huge scores finite (fanfani.net, "A pinch of math",
    # the rescale factor is e to a non-positive power); with one key far ahead
    # the weights become one-hot and O picks that key's value.
    d, N = 4, 6
    k = np.zeros((1, 1, N, d))
    for j in range(N):
        k[0, 0, j, j % d] = 1.0 + 0.1 * j
    v = _rand((1, 1, N, d), 17)
    q = np.zeros((1, 1, 1, d))
    q[0, 0, 0, 1] = 5000.0  # favours key 5 (1.5 * 5000) over key 1 (1.1 * 5000)
    qN = np.repeat(q, N, axis=2)
    out, lse = o.attention_forward(qN, k, v, 1.0, False)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    assert np.max(np.abs(out[0, 0] - v[0, 0, 5][None, :])) < 1e-12
    assert np.max(np.abs(lse - 7500.0)) < 1e-9
    q2, k2, v2 = _qkv(Hq=2, Hkv=2, N=9, d=4, seed=19)
    out2, lse2 = o.attention_forward(50.0 * q2, k2, v2, 1.0, True)
    assert np.all(np.isfinite(out2)) and np.all(np.isfinite(lse2))


def check_gqa_equals_repeated_mha(o):
    # Grouped-query attention with group g is multi-head attention with each
    # KV head repeated g times along the head axis (contiguous groups).
    q, k, v = _qkv(B=2, Hq=6, Hkv=2, N=9, d=4, seed=23)
    kr, vr = np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1)
    do = _rand(q.shape, 29)
    for causal in (False, True):
        a = o.attention_forward(q, k, v, 0.8, causal)
        b = o.attention_forward(q, kr, vr, 0.8, causal)
        assert np.max(np.abs(a[0] - b[0])) < 1e-14 and np.max(np.abs(a[1] - b[1])) < 1e-14
        ga = o.attention_backward(q, k, v, do, 0.8, causal)
        gb = o.attention_backward(q, kr, vr, do, 0.8, causal)
        assert np.max(np.abs(ga[0] - gb[0])) < 1e-13
        dk_sum = gb[1].reshape(2, 2, 3, 9, 4).sum(axis=2)
        dv_sum = gb[2].reshape(2, 2, 3, 9, 4).sum(axis=2)
        assert np.max(np.abs(ga[1] - dk_sum)) < 1e-13
        assert np.max(np.abs(ga[2] - dv_sum)) < 1e-13


def check_worked_example(o):
    # Hand-derived closed form (tests/golden/worked_example_ln_scores.json).
    g = json.load(open(os.path.join(GOLDEN, "worked_example_ln_scores.json")))
    keys = np.log(np.array(g["k_log"], float))
    k = keys.reshape(1, 1, 3, 1)
    v = np.array(g["v"]).reshape(1, 1, 3, 1)
    q = np.array(g["q"]).reshape(1, 1, 3, 1)
    e = g["expected"]
    out, lse = o.attention_forward(q, k, v, 1.0, False)
    assert abs(out[0, 0, 0, 0] - e["non_causal_row_O"]) < 1e-12
    assert abs(math.exp(lse[0, 0, 0]) - e["non_causal_row_LSE_exp"]) < 1e-12
    out, lse = o.attention_forward(q, k, v, 1.0, True)
    assert np.max(np.abs(out[0, 0, :, 0] - np.array(e["causal_O"]))) < 1e-12
    assert np.max(np.abs(np.exp(lse[0, 0]) - np.array(e["causal_LSE_exp"]))) < 1e-12
    # One query row (q = 1) against the three keys, dO = 1 on that row only;
    # rows 1 and 2 (q = 0) carry no upstream gradient.
    q1 = q[:, :, :1]
    k1, v1 = k, v
    do = np.zeros((1, 1, 3, 1))
    do[0, 0, 0, 0] = 1.0
    qq = np.concatenate([q1, np.zeros((1, 1, 2, 1))], axis=2)
    dq, dk, dv, D = o.attention_backward(qq, k1, v1, do, 1.0, False)
    assert np.max(np.abs(dv[0, 0, :, 0] - np.array(e["bwd_single_row_dV"]))) < 1e-12
    assert np.max(np.abs(dk[0, 0, :, 0] - np.array(e["bwd_single_row_dS"]) * 1.0)) < 1e-12
    dq_expected = sum(s * kk for s, kk in zip(e["bwd_single_row_dS"], keys))
    assert abs(dq[0, 0, 0, 0] - dq_expected) < 1e-12
    assert abs(D[0, 0, 0] - 14.0) < 1e-12


def check_score_matrix_size(o):
    # The pages' only printed size: 8k tokens x 32 heads in half precision is
    # over four gigabytes per layer (tests/golden/score_matrix_size.json).
    g = json.load(open(os.path.join(GOLDEN, "score_matrix_size.json")))
    n = o.score_matrix_bytes(g["N"], g["heads"], g["bytes_per_element"])
    assert n > g["more_than_bytes"]
    assert n == 2 ** 32


# --------------------------------------------------------------- backward pins

def _loss(o, q, k, v, g, scale, causal):
    out, _ = o.attention_forward(q, k, v, scale, causal)
    return float(np.sum(out * g))


def check_backward_finite_differences(o):
    # Central differences of L = sum(O * G) against the analytic gradients.
    for causal, (Hq, Hkv) in ((False, (2, 2)), (True, (2, 1)), (True, (3, 3))):
        q, k, v = _qkv(B=1, Hq=Hq, Hkv=Hkv, N=6, d=3, seed=31 + Hq + Hkv)
        g = _rand(q.shape, 37)
        scale = 0.9
        dq, dk, dv, _ = o.attention_backward(q, k, v, g, scale, causal)
        h = 1e-6
        for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = np.zeros_like(x)
            it = np.nditer(x, flags=["multi_index"])
            for _ in it:
                idx = it.multi_index
                xp, xm = x.copy(), x.copy()
                xp[idx] += h
                xm[idx] -= h
                args_p = {"q": q, "k": k, "v": v}
                args_m = {"q": q, "k": k, "v": v}
                args_p[name], args_m[name] = xp, xm
                num[idx] = (_loss(o, args_p["q"], args_p["k"], args_p["v"], g, scale, causal)
                            - _loss(o, args_m["q"], args_m["k"], args_m["v"], g, scale, causal)) / (2 * h)
            rel = np.linalg.norm(num - grad) / max(np.linalg.norm(num), 1e-30)
            assert rel < 1e-6, (name, causal, rel)


def check_backward_invariants(o):
    # sum_j dV_j = sum_i dO_i (each row of P sums to one); D_i = sum_j P_ij dP_ij;
    # each row of dS sums to zero (softmax is shift invariant).
    q, k, v = _qkv(B=1, Hq=2, Hkv=2, N=15, d=4, seed=41)
    do = _rand(q.shape, 43)
    for causal in (False, True):
        dq, dk, dv, D = o.attention_backward(q, k, v, do, 0.5, causal)
        assert np.max(np.abs(dv.sum(axis=2) - do.sum(axis=2))) < 1e-12
        p = o.attention_probs(q, k, 0.5, causal)
        dp = np.einsum("bhid,bhjd->bhij", do, v)
        assert np.max(np.abs(D - np.sum(p * dp, axis=-1))) < 1e-12
        ds = p * (dp - D[..., None])
        assert np.max(np.abs(ds.sum(-1))) < 1e-12


def check_torch_sdpa_cross_check(o):
    # Independent library routine: torch's CPU fp64 scaled_dot_product_attention
    # and autograd on tiny shapes (GQA by repeating K/V heads).
    q, k, v = _qkv(B=2, Hq=4, Hkv=2, N=10, d=8, seed=47)
    do = _rand(q.shape, 53)
    for causal in (False, True):
        tq = torch.tensor(q, requires_grad=True)
        tk = torch.tensor(k, requires_grad=True)
        tv = torch.tensor(v, requires_grad=True)
        kr, vr = tk.repeat_interleave(2, dim=1), tv.repeat_interleave(2, dim=1)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, kr, vr, is_causal=causal, scale=0.3)
        ref.backward(torch.tensor(do))
        s = 0.3 * tq.detach() @ kr.detach().transpose(-1, -2)
        if causal:
            s = s.masked_fill(torch.ones(10, 10, dtype=torch.bool).triu(1), float("-inf"))
        ref_lse = torch.logsumexp(s, dim=-1)
        out, lse = o.attention_forward(q, k, v, 0.3, causal)
        assert np.max(np.abs(out - ref.detach().numpy())) < 1e-12
        assert np.max(np.abs(lse - ref_lse.numpy())) < 1e-12
        dq, dk, dv, _ = o.attention_backward(q, k, v, do, 0.3, causal)
        assert np.max(np.abs(dq - tq.grad.numpy())) < 1e-12
        assert np.max(np.abs(dk - tk.grad.numpy())) < 1e-12
        assert np.max(np.abs(dv - tv.grad.numpy())) < 1e-12


def check_rows_helper_matches_full(o):
    # The sampled-row entry point computes the same rows as the full oracle.
    q, k, v = _qkv(B=2, Hq=4, Hkv=2, N=23, d=4, seed=59)
    rows = [0, 1, 7, 22]
    for causal in (False, True):
        full_o, full_l = o.attention_forward(q, k, v, 0.45, causal)
        ro, rl = o.attention_forward_rows(q, k, v, 0.45, causal, 1, 3, rows)
        assert np.max(np.abs(ro - full_o[1, 3, rows])) < 1e-14
        assert np.max(np.abs(rl - full_l[1, 3, rows])) < 1e-14


def check_backward_rows_partition(o):
    # The row-restricted backward: its dQ rows are the full dQ rows, and its
    # dK/dV shares summed over a partition of all query rows (and the heads of
    # each group) give the full dK/dV.
    q, k, v = _qkv(B=1, Hq=4, Hkv=2, N=21, d=3, seed=61)
    do = _rand(q.shape, 67)
    parts = [np.arange(0, 21, 3), np.arange(1, 21, 3), np.arange(2, 21, 3)]
    for causal in (False, True):
        dq, dk, dv, _ = o.attention_backward(q, k, v, do, 0.7, causal)
        dk_sum, dv_sum = np.zeros_like(dk), np.zeros_like(dv)
        for h in range(4):
            for rows in parts:
                rq, rk, rv = o.attention_backward_rows(q, k, v, do, 0.7, causal, 0, h, rows)
                assert np.max(np.abs(rq - dq[0, h, rows])) < 1e-13
                dk_sum[0, h // 2] += rk
                dv_sum[0, h // 2] += rv
        assert np.max(np.abs(dk_sum - dk)) < 1e-12
        assert np.max(np.abs(dv_sum - dv)) < 1e-12


def check_kvcache_is_the_last_rows_of_the_square_problem(o):
    # Nq queries against Nk cached keys are the last Nq rows of the square
    # problem whose queries fill all Nk positions (causal: query i at position
    # Nk - Nq + i sees keys up to it), GQA included.
    qf, k, v = _qkv(B=2, Hq=4, Hkv=2, N=17, d=5, seed=71)
    for causal in (False, True):
        fo, fl = o.attention_forward(qf, k, v, 0.6, causal)
        for nq in (1, 3, 17):
            ko, kl = o.attention_forward_kvcache(qf[:, :, 17 - nq:], k, v, 0.6, causal)
            assert np.max(np.abs(ko - fo[:, :, 17 - nq:])) < 1e-13
            assert np.max(np.abs(kl - fl[:, :, 17 - nq:])) < 1e-13


def check_kvcache_single_query_sees_every_key(o):
    # One new query is the last position: the causal mask hides nothing, and
    # with a single cached key the output is that key's value (closed form).
    q, k, v = _qkv(B=1, Hq=2, Hkv=1, N=9, d=4, seed=73)
    q1 = q[:, :, -1:]
    co, cl = o.attention_forward_kvcache(q1, k, v, 0.8, True)
    no, nl = o.attention_forward_kvcache(q1, k, v, 0.8, False)
    assert np.max(np.abs(co - no)) < 1e-15 and np.max(np.abs(cl - nl)) < 1e-15
    so, sl = o.attention_forward_kvcache(q1, k[:, :, :1], v[:, :, :1], 0.8, True)
    assert np.max(np.abs(so[0, :, 0] - v[0, 0, 0])) < 1e-15
    assert np.max(np.abs(sl[0, :, 0] - 0.8 * q1[0, :, 0] @ k[0, 0, 0])) < 1e-14


def check_merge_partial_states_matches_full(o):
    # Softmax states of disjoint key chunks, merged with the rescale rule,
    # give the softmax over all keys -- including chunks that are entirely
    # masked for some rows under the causal mask.
    q, k, v = _qkv(B=1, Hq=1, Hkv=1, N=29, d=6, seed=79)
    for causal in (False, True):
        fo, fl = o.attention_forward(q, k, v, 0.5, causal)
        s = o.masked_scores(q[0, 0], k[0, 0], 0.5, causal)
        cuts = [0, 4, 5, 17, 29]
        states = [o.partial_state(s[:, a:b], v[0, 0, a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
        mo, ml = o.merge_partial_states(*(np.stack(x) for x in zip(*states)))
        assert np.max(np.abs(mo - fo[0, 0])) < 1e-13
        assert np.max(np.abs(ml - fl[0, 0])) < 1e-13


def _varlen_pack(seed=83):
    # three sequences: 5 queries / 9 keys, 7 / 7, 1 / 4; GQA 4 query heads on 2 KV heads
    nq, nk = [5, 7, 1], [9, 7, 4]
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((sum(nq), 4, 3))
    k = rng.standard_normal((sum(nk), 2, 3))
    v = rng.standard_normal((sum(nk), 2, 3))
    return q, k, v, np.cumsum([0] + nq), np.cumsum([0] + nk)


def check_varlen_is_each_sequence_alone(o):
    # A packed batch is each sequence's own (pinned) KV-cache problem: no key of
    # another sequence reaches a query.
    q, k, v, cq, ck = _varlen_pack()
    for causal in (False, True):
        po, pl = o.attention_forward_varlen(q, k, v, cq, ck, 0.7, causal)
        for s in range(3):
            qs = q[cq[s]:cq[s + 1]].transpose(1, 0, 2)[None]
            ks = k[ck[s]:ck[s + 1]].transpose(1, 0, 2)[None]
            vs = v[ck[s]:ck[s + 1]].transpose(1, 0, 2)[None]
            so, sl = o.attention_forward_kvcache(qs, ks, vs, 0.7, causal)
            assert np.max(np.abs(po[cq[s]:cq[s + 1]] - so[0].transpose(1, 0, 2))) < 1e-13
            assert np.max(np.abs(pl[cq[s]:cq[s + 1]] - sl[0].T)) < 1e-13


def check_varlen_sequence_order_invariance(o):
    # Packing the same sequences in another order moves their rows and nothing else.
    q, k, v, cq, ck = _varlen_pack(89)
    order = [2, 0, 1]
    qp = np.concatenate([q[cq[s]:cq[s + 1]] for s in order])
    kp = np.concatenate([k[ck[s]:ck[s + 1]] for s in order])
    vp = np.concatenate([v[ck[s]:ck[s + 1]] for s in order])
    cqp = np.cumsum([0] + [cq[s + 1] - cq[s] for s in order])
    ckp = np.cumsum([0] + [ck[s + 1] - ck[s] for s in order])
    for causal in (False, True):
        ao, al = o.attention_forward_varlen(q, k, v, cq, ck, 0.4, causal)
        bo, bl = o.attention_forward_varlen(qp, kp, vp, cqp, ckp, 0.4, causal)
        for i, s in enumerate(order):
            assert np.max(np.abs(bo[cqp[i]:cqp[i + 1]] - ao[cq[s]:cq[s + 1]])) < 1e-14
            assert np.max(np.abs(bl[cqp[i]:cqp[i + 1]] - al[cq[s]:cq[s + 1]])) < 1e-14



def check_positions_reduce_to_square_and_kvcache(o):
    # Queries and keys at positions 0..N-1 are the square problem; queries at
    # the last Nq of Nk positions are the (pinned) KV-cache problem.
    q, k, v = _qkv(B=2, Hq=4, Hkv=2, N=11, d=4, seed=97)
    for causal in (False, True):
        ao, al = o.attention_forward(q, k, v, 0.6, causal)
        po, pl = o.attention_forward_positions(q, k, v, np.arange(11), np.arange(11), 0.6, causal)
        assert np.max(np.abs(po - ao)) < 1e-14 and np.max(np.abs(pl - al)) < 1e-14
        ko, kl = o.attention_forward_kvcache(q[:, :, 7:], k, v, 0.6, causal)
        po, pl = o.attention_forward_positions(q[:, :, 7:], k, v, np.arange(7, 11), np.arange(11), 0.6, causal)
        assert np.max(np.abs(po - ko)) < 1e-14 and np.max(np.abs(pl - kl)) < 1e-14


def check_positions_brute_force(o):
    # Scalar loops over a tiny head with positions out of order, one query
    # that sees every key and one that sees none (O = 0, LSE = -inf).
    rng = np.random.default_rng(101)
    q = rng.standard_normal((1, 1, 4, 3))
    k = rng.standard_normal((1, 1, 5, 3))
    v = rng.standard_normal((1, 1, 5, 2))
    q_pos, k_pos = [5, -1, 2, 9], [3, 1, 4, 0, 2]
    out, lse = o.attention_forward_positions(q, k, v, q_pos, k_pos, 0.9, True)
    for i in range(4):
        vis = [j for j in range(5) if k_pos[j] <= q_pos[i]]
        if not vis:
            assert np.all(out[0, 0, i] == 0.0) and lse[0, 0, i] == -np.inf
            continue
        sc = {j: 0.9 * sum(q[0, 0, i, t] * k[0, 0, j, t] for t in range(3)) for j in vis}
        z = sum(math.exp(x) for x in sc.values())
        assert abs(lse[0, 0, i] - math.log(z)) < 1e-13
        for c in range(2):
            ref = sum(math.exp(sc[j]) * v[0, 0, j, c] for j in vis) / z
            assert abs(out[0, 0, i, c] - ref) < 1e-13
    assert len([j for j in range(5) if k_pos[j] <= 9]) == 5


def check_striped_shards_merge_to_full(o):
    # Token t on shard t % W: each shard's queries against each shard's keys,
    # merged over the key shards, give the full attention of those queries --
    # causal blocks with a row that sees nothing included (W = 3, N = 12, GQA).
    q, k, v = _qkv(B=1, Hq=4, Hkv=2, N=12, d=5, seed=103)
    W = 3
    for causal in (False, True):
        fo, fl = o.attention_forward(q, k, v, 0.45, causal)
        for r in range(W):
            qp = r + W * np.arange(12 // W)
            parts = [o.attention_forward_positions(q[:, :, r::W], k[:, :, c::W], v[:, :, c::W], qp,
                                                   c + W * np.arange(12 // W), 0.45, causal) for c in range(W)]
            if causal and r < W - 1:
                assert parts[W - 1][1][0, 0, 0] == -np.inf  # query r sees no key of shard W-1 > r
            os = np.stack([pp[0].reshape(-1, 5) for pp in parts])
            ls = np.stack([pp[1].reshape(-1) for pp in parts])
            mo, ml = o.merge_outputs(os, ls)
            assert np.max(np.abs(mo - fo[:, :, r::W].reshape(-1, 5))) < 1e-13
            assert np.max(np.abs(ml - fl[:, :, r::W].reshape(-1))) < 1e-13



def check_varlen_backward_square_sequences_are_the_square_backward(o):
    # Sequences with as many queries as keys are each the (pinned) square
    # backward of that sequence alone.
    rng = np.random.default_rng(107)
    lens = [6, 1, 9]
    cu = np.cumsum([0] + lens)
    q, k, v, do = (rng.standard_normal((cu[-1], h, 4)) for h in (4, 2, 2, 4))
    for causal in (False, True):
        dq, dk, dv = o.attention_backward_varlen(q, k, v, do, cu, cu, 0.6, causal)
        for s in range(3):
            sl = slice(cu[s], cu[s + 1])
            per = [x[sl].transpose(1, 0, 2)[None] for x in (q, k, v, do)]
            rq, rk, rv, _ = o.attention_backward(*per, 0.6, causal)
            assert np.max(np.abs(dq[sl] - rq[0].transpose(1, 0, 2))) < 1e-13
            assert np.max(np.abs(dk[sl] - rk[0].transpose(1, 0, 2))) < 1e-13
            assert np.max(np.abs(dv[sl] - rv[0].transpose(1, 0, 2))) < 1e-13


def check_varlen_backward_finite_differences(o):
    # Central differences of L = sum(O * G) through the (pinned) varlen
    # forward, on a pack whose sequences have fewer queries than keys (the
    # queries sit at the last positions) and GQA.
    rng = np.random.default_rng(109)
    cq, ck = np.array([0, 2, 5]), np.array([0, 4, 7])
    q, k, v = rng.standard_normal((5, 2, 3)), rng.standard_normal((7, 1, 3)), rng.standard_normal((7, 1, 3))
    g = rng.standard_normal((5, 2, 3))
    for causal in (False, True):
        dq, dk, dv = o.attention_backward_varlen(q, k, v, g, cq, ck, 0.8, causal)
        for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = np.zeros_like(x)
            for idx in np.ndindex(*x.shape):
                xp, xm = x.copy(), x.copy()
                xp[idx] += 1e-6
                xm[idx] -= 1e-6
                args = {"q": q, "k": k, "v": v}
                args[name] = xp
                fp = np.sum(o.attention_forward_varlen(args["q"], args["k"], args["v"], cq, ck, 0.8, causal)[0] * g)
                args[name] = xm
                fm = np.sum(o.attention_forward_varlen(args["q"], args["k"], args["v"], cq, ck, 0.8, causal)[0] * g)
                num[idx] = (fp - fm) / 2e-6
            assert np.max(np.abs(num - grad)) < 1e-7, name



def check_backward_blocks_sum_to_the_full_backward(o):
    # Striped key blocks (W = 3) of every query shard, each with the full rows'
    # LSE and D, add up to the (pinned) backward of the unsharded problem.
    q, k, v = _qkv(B=1, Hq=4, Hkv=2, N=12, d=5, seed=113)
    do = _rand((1, 4, 12, 5), 114)
    W = 3
    for causal in (False, True):
        fo, fl = o.attention_forward(q, k, v, 0.45, causal)
        rq, rk, rv, D = o.attention_backward(q, k, v, do, 0.45, causal)
        dq = np.zeros_like(q)
        dk = np.zeros_like(k)
        dv = np.zeros_like(v)
        for r in range(W):
            qp = r + W * np.arange(12 // W)
            for c in range(W):
                kp = c + W * np.arange(12 // W)
                bq, bk, bv = o.attention_backward_block(q[:, :, r::W], k[:, :, c::W], v[:, :, c::W], do[:, :, r::W],
                                                        fl[:, :, r::W], D[:, :, r::W], qp, kp, 0.45, causal)
                dq[:, :, r::W] += bq
                dk[:, :, c::W] += bk
                dv[:, :, c::W] += bv
        assert np.max(np.abs(dq - rq)) < 1e-12
        assert np.max(np.abs(dk - rk)) < 1e-12
        assert np.max(np.abs(dv - rv)) < 1e-12


ALL_CHECKS = [
    check_backward_blocks_sum_to_the_full_backward,
    check_varlen_backward_square_sequences_are_the_square_backward,
    check_varlen_backward_finite_differences,
    check_positions_reduce_to_square_and_kvcache,
    check_positions_brute_force,
    check_striped_shards_merge_to_full,
    check_varlen_is_each_sequence_alone,
    check_varlen_sequence_order_invariance,
    check_kvcache_is_the_last_rows_of_the_square_problem,
    check_kvcache_single_query_sees_every_key,
    check_merge_partial_states_matches_full,
    check_backward_rows_partition,
    check_rows_sum_to_one,
    check_single_key_returns_value,
    check_zero_query_uniform,
    check_online_matches_full,
    check_kv_permutation_invariance,
    check_large_scores_stable_one_hot,
    check_gqa_equals_repeated_mha,
    check_worked_example,
    check_score_matrix_size,
    check_backward_finite_differences,
    check_backward_invariants,
    check_torch_sdpa_cross_check,
    check_rows_helper_matches_full,
]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check(ORACLE)


# ------------------------------------------------------- planted mistakes
# Each mutation replaces one oracle helper with a plausible wrong version; at
# least one pin must fail on it.

def _mut_drop_D(p, dp, D):  # dropped term in the softmax Jacobian
    return p * dp


def _mut_sign_D(p, dp, D):  # wrong sign
    return p * (dp + D[:, None])


def _mut_mask_strict(q_bh, k_bh, scale, causal, rows=None, keys=None):  # off-by-one: j < i
    s = scale * (np.asarray(q_bh, float) @ np.asarray(k_bh, float).T)
    if causal:
        qpos = np.arange(s.shape[0]) if rows is None else np.asarray(rows)
        kpos = np.arange(s.shape[1]) if keys is None else np.asarray(keys)
        s = np.where(kpos[None, :] < qpos[:, None], s, -np.inf)
    return s


def _mut_no_scale(q_bh, k_bh, scale, causal, rows=None, keys=None):  # scale dropped
    return ORIG["masked_scores"](q_bh, k_bh, 1.0, causal, rows, keys)


def _mut_transposed_keys(q_bh, k_bh, scale, causal, rows=None, keys=None):  # K^T Q instead of Q K^T
    s = ORIG["masked_scores"](q_bh, k_bh, scale, False, rows)
    s = s.T if s.shape[0] == s.shape[1] else s
    if causal:
        qpos = np.arange(s.shape[0]) if rows is None else np.asarray(rows)
        kpos = np.arange(s.shape[1]) if keys is None else np.asarray(keys)
        s = np.where(kpos[None, :] <= qpos[:, None], s, -np.inf)
    return s


def _mut_varlen_backward_top_left(q, k, v, do, cu_q, cu_k, scale, causal):  # queries placed at positions 0..
    q, k, v, do = (np.asarray(x, float) for x in (q, k, v, do))
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for s in range(len(cu_q) - 1):
        sq, sk = slice(cu_q[s], cu_q[s + 1]), slice(cu_k[s], cu_k[s + 1])
        for h in range(q.shape[1]):
            hk = ORACLE.kv_head_of(h, q.shape[1], k.shape[1])
            p = ORACLE.softmax_rows(ORACLE.masked_scores(q[sq, h], k[sk, hk], scale, causal))[0]
            dv[sk, hk] += p.T @ do[sq, h]
            ds = ORACLE.score_gradient(p, do[sq, h] @ v[sk, hk].T, np.sum(do[sq, h] * (p @ v[sk, hk]), axis=1))
            dq[sq, h] = scale * (ds @ k[sk, hk])
            dk[sk, hk] += scale * (ds.T @ q[sq, h])
    return dq, dk, dv


def _mut_block_backward_local_lse(q, k, v, do, lse, D, q_pos, k_pos, scale, causal):  # block's own LSE
    _, local = ORACLE.attention_forward_positions(q, k, v, q_pos, k_pos, scale, causal)
    return ORIG["attention_backward_block"](q, k, v, do, np.where(np.isfinite(local), local, 0.0), D, q_pos, k_pos,
                                            scale, causal)


def _mut_positions_ignore_keys(q, k, v, q_pos, k_pos, scale, causal):  # key positions taken as 0..Nk-1
    return ORIG["attention_forward_positions"](q, k, v, q_pos, np.arange(np.shape(k)[2]), scale, causal)


def _mut_merge_outputs_plain_mean(os, lses):  # outputs averaged, LSE weights dropped
    os, lses = np.asarray(os, float), np.asarray(lses, float)
    return os.mean(axis=0), np.log(np.sum(np.exp(lses), axis=0))


def _mut_softmax_no_max(s):  # max subtraction dropped
    e = np.exp(s)
    l = e.sum(-1)
    return e / l[..., None], np.zeros(s.shape[:-1]), l


def _mut_softmax_wrong_norm(s):  # normalised by the max instead of the sum
    p, m, l = ORIG["softmax_rows"](s)
    return p * l[..., None] / np.max(p * l[..., None], axis=-1, keepdims=True), m, l


def _mut_kv_head(hq, Hq, Hkv):  # interleaved instead of contiguous groups
    return hq % Hkv


def _mut_kvcache_top_left(q, k, v, scale, causal):  # queries placed at positions 0..Nq-1
    q = np.asarray(q, float)
    k = np.asarray(k, float)
    v = np.asarray(v, float)
    B, Hq, Nq, _ = q.shape
    o = np.empty((B, Hq, Nq, v.shape[-1]))
    lse = np.empty((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            hk = ORACLE.kv_head_of(h, Hq, k.shape[1])
            p, m, l = ORACLE.softmax_rows(ORACLE.masked_scores(q[b, h], k[b, hk], scale, causal))
            o[b, h] = p @ v[b, hk]
            lse[b, h] = m + np.log(l)
    return o, lse


def _mut_varlen_leak(q, k, v, cu_q, cu_k, scale, causal):  # every query sees the whole pack
    kk = np.asarray(k, float)[None].transpose(0, 2, 1, 3)
    vv = np.asarray(v, float)[None].transpose(0, 2, 1, 3)
    qq = np.asarray(q, float)[None].transpose(0, 2, 1, 3)
    o, lse = ORACLE.attention_forward_kvcache(qq, kk, vv, scale, False)
    return o[0].transpose(1, 0, 2), lse[0].T


def _mut_merge_no_rescale(ms, ls, os):  # sums added without the exp(m_s - M) factors
    L = np.sum(ls, axis=0)
    return np.sum(os, axis=0) / L[:, None], np.max(ms, axis=0) + np.log(L)


ORIG = {name: getattr(ORACLE, name) for name in ("masked_scores", "softmax_rows", "score_gradient", "kv_head_of",
                                                 "attention_forward_positions", "attention_backward_block")}

MUTATIONS = [
    ("score_gradient", _mut_drop_D),
    ("score_gradient", _mut_sign_D),
    ("masked_scores", _mut_mask_strict),
    ("masked_scores", _mut_no_scale),
    ("masked_scores", _mut_transposed_keys),
    ("softmax_rows", _mut_softmax_no_max),
    ("softmax_rows", _mut_softmax_wrong_norm),
    ("kv_head_of", _mut_kv_head),
    ("attention_forward_kvcache", _mut_kvcache_top_left),
    ("merge_partial_states", _mut_merge_no_rescale),
    ("attention_forward_varlen", _mut_varlen_leak),
    ("attention_forward_positions", _mut_positions_ignore_keys),
    ("merge_outputs", _mut_merge_outputs_plain_mean),
    ("attention_backward_varlen", _mut_varlen_backward_top_left),
    ("attention_backward_block", _mut_block_backward_local_lse),
]


@pytest.mark.parametrize("target,mutant", MUTATIONS, ids=lambda x: getattr(x, "__name__", str(x)))
def test_planted_mistake_is_caught(monkeypatch, target, mutant):
    monkeypatch.setattr(ORACLE, target, mutant)
    failed = []
    for check in ALL_CHECKS:
        try:
            with np.errstate(all="ignore"):
                check(ORACLE)
        except (AssertionError, FloatingPointError, ValueError, IndexError):
            failed.append(check.__name__)
    assert failed, f"no pin caught the planted mistake {mutant.__name__}"
