"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Tolerances: float32 inputs, O and LSE max-abs <= 1e-5; bf16 inputs with fp32
accumulation, O max-abs <= 2e-2 and LSE max-abs <= 1e-3; gradients dQ, dK, dV
relative Frobenius error <= 2e-2. Inputs are the seeded synthetic tensors of
``exact_io_aware_61_b200.inputs``; the oracle gets the same values in fp64.
Full-size workloads are checked against the oracle head by head (every row
of the benchmark forward, every head of the training backward) or on sampled
rows and whole KV-head groups where a full check would take too long, plus
properties that hold at any size. Every output is written into a view of a
larger, canary-filled buffer, and the canaries are checked after each call
(``tests/guarded.py``).
"""

import numpy as np
import pytest
import torch

import oracle.attention as ORACLE
from exact_io_aware_61_b200 import inputs as INP
from tests.guarded import Guarded, check_all

pytestmark = pytest.mark.gpu

O_TOL_F32, LSE_TOL_F32 = 1e-5, 1e-5
O_TOL_BF16, LSE_TOL_BF16 = 2e-2, 1e-3
GRAD_TOL = 2e-2


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import exact_io_aware_61_b200 as fa_mod
    fa_mod.load()  # raises if the library is missing: no fallback
    return fa_mod


def _to_dev(t):
    return t.to("cuda").contiguous()


def _run_fwd(fa, inp, causal, scale):
    """fa_fwd into canary-guarded O and LSE (pre-filled with NaN, so a row the
    kernel never writes fails the comparison and a store outside them fails
    the guard check)."""
    q, k, v = (_to_dev(inp[n]) for n in ("q", "k", "v"))
    B, Hq, N, d = q.shape
    go = Guarded(q.shape, q.dtype, fill=float("nan"))
    gl = Guarded((B, Hq, N), torch.float32, fill=float("nan"))
    fa.fa_fwd(q, k, v, go.t, gl.t, causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    check_all(("O", go), ("LSE", gl))
    return go.t, gl.t


def _rel_fro(a, b):
    # relative Frobenius error with an RMS floor of 1e-3 under the reference:
    # with one key, dQ = scale P (dP - D) K = 0 exactly (P = 1, D = dP), and
    # the kernel's value is the rounding of dP - D
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-3 * np.sqrt(np.size(b)), 1e-30))


# ------------------------------------------------------------------ forward

@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_f32_b1_h2_n256_d64(fa, seed, causal):
    inp = INP.make_inputs(1, 2, 2, 256, 64, "f32", seed=seed)
    o, lse = _run_fwd(fa, inp, causal, 1 / 8)
    ro, rl = ORACLE.attention_forward(*(INP.as_f64(inp[n]) for n in "qkv"), 1 / 8, causal)
    assert np.max(np.abs(INP.as_f64(o) - ro)) <= O_TOL_F32
    assert np.max(np.abs(INP.as_f64(lse) - rl)) <= LSE_TOL_F32


@pytest.mark.parametrize("shape", [
    (1, 2, 2, 1, 64), (1, 1, 1, 5, 128), (2, 3, 3, 127, 64), (1, 2, 1, 129, 128),
    (1, 4, 2, 300, 64), (1, 2, 2, 300, 256), (2, 4, 1, 200, 128), (1, 1, 1, 1, 256),
])
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_f32_edge_shapes(fa, shape, causal):
    B, Hq, Hkv, N, d = shape
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "f32", seed=11)
    o, lse = _run_fwd(fa, inp, causal, d ** -0.5)
    ro, rl = ORACLE.attention_forward(*(INP.as_f64(inp[n]) for n in "qkv"), d ** -0.5, causal)
    assert np.max(np.abs(INP.as_f64(o) - ro)) <= O_TOL_F32
    assert np.max(np.abs(INP.as_f64(lse) - rl)) <= LSE_TOL_F32


BF16_EDGE = [
    (1, 1, 1, 1, 64), (1, 2, 2, 1, 128), (1, 1, 1, 1, 256),
    (1, 2, 2, 127, 64), (1, 2, 2, 128, 128), (1, 2, 2, 129, 128), (2, 3, 3, 300, 64),
    (1, 4, 1, 257, 128), (1, 4, 2, 384, 256), (1, 2, 2, 640, 128), (1, 8, 2, 1000, 64),
    (3, 2, 1, 513, 256),
]


@pytest.mark.parametrize("shape", BF16_EDGE, ids=lambda s: "b%d_h%d_kv%d_n%d_d%d" % s)
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_bf16_edge_shapes(fa, shape, causal):
    B, Hq, Hkv, N, d = shape
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "bf16", seed=N + d)
    o, lse = _run_fwd(fa, inp, causal, d ** -0.5)
    ro, rl = ORACLE.attention_forward(*(INP.as_f64(inp[n]) for n in "qkv"), d ** -0.5, causal)
    assert np.max(np.abs(INP.as_f64(o) - ro)) <= O_TOL_BF16
    assert np.max(np.abs(INP.as_f64(lse) - rl)) <= LSE_TOL_BF16


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_bf16_b4_h16_n2048_d64(fa, causal):
    w = INP.WORKLOADS["fwd_bf16_b4_h16_n2048_d64"]
    inp = INP.workload_inputs(w, seed=1001)
    o, lse = _run_fwd(fa, inp, causal, w.scale)
    ro, rl = ORACLE.attention_forward(*(INP.as_f64(inp[n]) for n in "qkv"), w.scale, causal)
    assert np.max(np.abs(INP.as_f64(o) - ro)) <= O_TOL_BF16
    assert np.max(np.abs(INP.as_f64(lse) - rl)) <= LSE_TOL_BF16


def _sample_rows(N, rng, n_random=24):
    fixed = [0, 1, 2, 127, 128, 129, N // 2, N - 129, N - 128, N - 2, N - 1]
    rows = set(r for r in fixed if 0 <= r < N)
    rows.update(int(x) for x in rng.integers(0, N, n_random))
    return sorted(rows)


def test_fwd_causal_bf16_b2_h32_n8192_d128_all_rows(fa):
    """The benchmark forward (B=2, H=32, N=8192, d=128, causal): every row of
    every head against the full oracle, one head at a time."""
    w = INP.WORKLOADS["fwd_causal_bf16_b2_h32_n8192_d128"]
    inp = INP.workload_inputs(w, seed=1003)
    o, lse = _run_fwd(fa, inp, True, w.scale)
    o_h, lse_h = o.float().cpu().numpy(), lse.cpu().numpy()
    q, k, v = (inp[n].float().numpy() for n in "qkv")
    worst_o = worst_l = 0.0
    for b in range(w.B):
        for h in range(w.Hq):
            sl = (slice(b, b + 1), slice(h, h + 1))
            ro, rl = ORACLE.attention_forward(q[sl], k[sl], v[sl], w.scale, True)
            worst_o = max(worst_o, float(np.max(np.abs(o_h[sl] - ro))))
            worst_l = max(worst_l, float(np.max(np.abs(lse_h[sl] - rl))))
    assert worst_o <= O_TOL_BF16, worst_o
    assert worst_l <= LSE_TOL_BF16, worst_l


@pytest.mark.parametrize("name", [
    "gqa_causal_bf16_b1_h32_kv8_n16384_d128",
    "gqa_causal_bf16_b1_h16_kv4_n8192_d256",
])
def test_fwd_bf16_gqa_all_rows(fa, name):
    """The grouped-query workloads (16k tokens at d = 128, 8k at d = 256):
    every row of every query head against the exact oracle, in blocks of 2048
    queries (each block a full softmax over all keys of its KV head)."""
    w = INP.WORKLOADS[name]
    inp = INP.workload_inputs(w, seed=1000 + len(name))
    o, lse = _run_fwd(fa, inp, True, w.scale)
    o_h, lse_h = o.float().cpu().numpy(), lse.cpu().numpy()
    q, k, v = (inp[n].float().numpy() for n in "qkv")
    worst_o = worst_l = 0.0
    for b in range(w.B):
        for h in range(w.Hq):
            for r0 in range(0, w.N, 2048):
                rows = list(range(r0, min(r0 + 2048, w.N)))
                ro, rl = ORACLE.attention_forward_rows(q, k, v, w.scale, True, b, h, rows)
                worst_o = max(worst_o, float(np.max(np.abs(o_h[b, h, rows] - ro))))
                worst_l = max(worst_l, float(np.max(np.abs(lse_h[b, h, rows] - rl))))
    assert worst_o <= O_TOL_BF16, worst_o
    assert worst_l <= LSE_TOL_BF16, worst_l
    assert np.all(np.isfinite(o_h)) and np.all(np.isfinite(lse_h))


def test_fwd_bf16_deterministic(fa):
    inp = INP.make_inputs(2, 4, 2, 1000, 128, "bf16", seed=5)
    o1, l1 = _run_fwd(fa, inp, True, 0.09)
    o2, l2 = _run_fwd(fa, inp, True, 0.09)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ----------------------------------------------------------------- backward

def _run_bwd(fa, inp, causal, scale, return_fwd=False):
    """fa_fwd, then fa_bwd into canary-guarded dQ, dK, dV and workspace."""
    q, k, v, do = (_to_dev(inp[n]) for n in ("q", "k", "v", "do"))
    o, lse = _run_fwd(fa, inp, causal, scale)
    B, Hq, N, d = q.shape
    gq = Guarded(q.shape, q.dtype, fill=float("nan"))
    gk = Guarded(k.shape, k.dtype, fill=float("nan"))
    gv = Guarded(v.shape, v.dtype, fill=float("nan"))
    gw = Guarded((max(fa.fa_bwd_workspace_size(B, Hq, k.shape[1], N, d), 16),), torch.uint8)
    fa.fa_bwd(q, k, v, o, lse, do, gq.t, gk.t, gv.t, gw.t, causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    check_all(("dQ", gq), ("dK", gk), ("dV", gv), ("workspace", gw))
    if return_fwd:
        return gq.t, gk.t, gv.t, o, lse
    return gq.t, gk.t, gv.t


BWD_SHAPES = [
    (1, 1, 1, 1, 64), (1, 2, 2, 100, 64), (1, 2, 2, 128, 128), (2, 2, 2, 257, 128),
    (1, 4, 2, 300, 64), (1, 4, 1, 384, 128), (1, 2, 2, 1000, 128), (2, 6, 3, 513, 64),
    (1, 8, 1, 2048, 128), (2, 4, 1, 1500, 64),  # MQA: the group's heads split over CTAs
    # d = 256 (64-key tiles, transposed dK/dV accumulators)
    (1, 1, 1, 1, 256), (2, 2, 1, 64, 256), (1, 2, 2, 200, 256), (1, 4, 2, 513, 256),
    (1, 8, 1, 1100, 256),  # MQA at d = 256: split over CTAs
]


@pytest.mark.parametrize("shape", BWD_SHAPES, ids=lambda s: "b%d_h%d_kv%d_n%d_d%d" % s)
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_bf16_shapes(fa, shape, causal):
    B, Hq, Hkv, N, d = shape
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "bf16", seed=3 * N + d, grad=True)
    dq, dk, dv = _run_bwd(fa, inp, causal, d ** -0.5)
    rq, rk, rv, _ = ORACLE.attention_backward(*(INP.as_f64(inp[n]) for n in ("q", "k", "v", "do")),
                                             d ** -0.5, causal)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        err = _rel_fro(INP.as_f64(got), ref)
        assert err <= GRAD_TOL, (name, err)


def test_bwd_train_causal_b2_h16_n4096_d128(fa):
    """The training workload (B=2, H=16, N=4096, d=128, causal): dQ, dK and dV
    of all 32 (batch, head) pairs against the full fp64 analytic backward."""
    w = INP.WORKLOADS["train_causal_bf16_b2_h16_n4096_d128"]
    inp = INP.workload_inputs(w, seed=1005)
    dq, dk, dv = _run_bwd(fa, inp, True, w.scale)
    dq_h, dk_h, dv_h = (INP.as_f64(t) for t in (dq, dk, dv))
    q, k, v, do = (inp[n].float().numpy() for n in ("q", "k", "v", "do"))
    for b in range(w.B):
        for h in range(w.Hq):
            sl = (slice(b, b + 1), slice(h, h + 1))
            rq, rk, rv, _ = ORACLE.attention_backward(q[sl], k[sl], v[sl], do[sl], w.scale, True)
            for name, got, ref in (("dq", dq_h[sl], rq), ("dk", dk_h[sl], rk), ("dv", dv_h[sl], rv)):
                err = _rel_fro(got, ref)
                assert err <= GRAD_TOL, (name, b, h, err)


def _group_identities(dk_h, dv_h, do_h, Hq, Hkv):
    """Checks that hold at any size, for every (batch, KV head):
    sum_j dV_j = sum over the group's query heads of sum_i dO_i (every row of P
    sums to one), and sum_j dK_j = 0 (every row of dS = P * (dP - D) sums to
    zero, since D_i = sum_j P_ij dP_ij). The second is measured against the
    size of the rows it sums: rounding alone leaves about 2^-9 of it."""
    g = Hq // Hkv
    for b in range(dk_h.shape[0]):
        for hk in range(Hkv):
            lhs = dv_h[b, hk].sum(axis=0)
            rhs = do_h[b, hk * g:(hk + 1) * g].sum(axis=(0, 1))
            assert _rel_fro(lhs, rhs) <= GRAD_TOL, ("sum dV", b, hk)
            zero = np.linalg.norm(dk_h[b, hk].sum(axis=0))
            scale = np.sqrt(np.sum(dk_h[b, hk] ** 2))
            assert zero <= GRAD_TOL * scale, ("sum dK", b, hk, zero / scale)


def test_bwd_causal_b1_h8_kv2_n4096_d256_all_heads(fa):
    """d = 256 backward at 4k tokens with GQA: every head of dQ, every KV head
    of dK and dV against the oracle in full."""
    B, Hq, Hkv, N, d = 1, 8, 2, 4096, 256
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "bf16", seed=4096 + d, grad=True)
    dq, dk, dv = _run_bwd(fa, inp, True, d ** -0.5)
    q, k, v, do = (INP.as_f64(inp[n]) for n in ("q", "k", "v", "do"))
    got_q, got_k, got_v = INP.as_f64(dq), INP.as_f64(dk), INP.as_f64(dv)
    g = Hq // Hkv
    for hk in range(Hkv):
        hs = slice(hk * g, (hk + 1) * g)
        rq, rk, rv, _ = ORACLE.attention_backward(q[:, hs], k[:, hk:hk + 1], v[:, hk:hk + 1], do[:, hs], d ** -0.5,
                                                  True)
        assert _rel_fro(got_q[:, hs], rq) <= GRAD_TOL
        assert _rel_fro(got_k[:, hk:hk + 1], rk) <= GRAD_TOL
        assert _rel_fro(got_v[:, hk:hk + 1], rv) <= GRAD_TOL


def test_bwd_causal_b1_h16_kv4_n8192_d256_one_group_full(fa):
    """The d = 256 GQA configuration at 8k tokens: dK and dV of one KV head
    (the last, so its CTAs run after every other group's) and the dQ of its
    four query heads against the oracle in full; sampled dQ rows on every
    other head."""
    B, Hq, Hkv, N, d = 1, 16, 4, 8192, 256
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "bf16", seed=8192 + d, grad=True)
    dq, dk, dv = _run_bwd(fa, inp, True, d ** -0.5)
    g = Hq // Hkv
    hk = Hkv - 1
    hs = slice(hk * g, (hk + 1) * g)
    q, k, v, do = (INP.as_f64(inp[n][:, sl]) for n, sl in (("q", hs), ("k", slice(hk, hk + 1)),
                                                            ("v", slice(hk, hk + 1)), ("do", hs)))
    rq, rk, rv, _ = ORACLE.attention_backward(q, k, v, do, d ** -0.5, True)
    assert _rel_fro(INP.as_f64(dq[:, hs]), rq) <= GRAD_TOL
    assert _rel_fro(INP.as_f64(dk[:, hk:hk + 1]), rk) <= GRAD_TOL
    assert _rel_fro(INP.as_f64(dv[:, hk:hk + 1]), rv) <= GRAD_TOL
    rng = np.random.default_rng(11)
    for h in range(0, hk * g):
        rows = sorted(set([0, 63, 64, N - 1] + [int(x) for x in rng.integers(0, N, 6)]))
        hkv = h // g
        qh, kh, vh, doh = (INP.as_f64(inp[n][:, sl]) for n, sl in (("q", slice(h, h + 1)), ("k", slice(hkv, hkv + 1)),
                                                                   ("v", slice(hkv, hkv + 1)), ("do", slice(h, h + 1))))
        rqr, _, _ = ORACLE.attention_backward_rows(qh, kh, vh, doh, d ** -0.5, True, 0, 0, rows)
        assert _rel_fro(INP.as_f64(dq[0, h, rows]), rqr) <= GRAD_TOL, h


def test_bwd_causal_b2_h32_n8192_d128(fa):
    """The benchmark backward (B=2, H=32, N=8192, d=128, causal), the shape
    bench.py times. Full fp64 dQ, dK, dV on one head from every group of 8
    consecutive (batch, head) pairs (8 heads, the first and last included);
    the dV and dK identities on every head; exact dQ on sampled rows of every
    head."""
    B, H, N, d = 2, 32, 8192, 128
    scale = d ** -0.5
    inp = INP.make_inputs(B, H, H, N, d, "bf16", seed=1003, grad=True)
    dq, dk, dv = _run_bwd(fa, inp, True, scale)
    dq_h, dk_h, dv_h = (INP.as_f64(t) for t in (dq, dk, dv))
    q, k, v, do = (inp[n].float().numpy() for n in ("q", "k", "v", "do"))
    for grp in range(B * H // 8):
        bh = 8 * grp + (grp * 3) % 8 if grp < B * H // 8 - 1 else B * H - 1
        b, h = divmod(bh, H)
        sl = (slice(b, b + 1), slice(h, h + 1))
        rq, rk, rv, _ = ORACLE.attention_backward(q[sl], k[sl], v[sl], do[sl], scale, True)
        for name, got, ref in (("dq", dq_h[sl], rq), ("dk", dk_h[sl], rk), ("dv", dv_h[sl], rv)):
            err = _rel_fro(got, ref)
            assert err <= GRAD_TOL, (name, b, h, err)
    _group_identities(dk_h, dv_h, do.astype(np.float64), H, H)
    rng = np.random.default_rng(13)
    worst = 0.0
    for b in range(B):
        for h in range(H):
            rows = _sample_rows(N, rng, n_random=6)
            rq, _, _ = ORACLE.attention_backward_rows(q, k, v, do, scale, True, b, h, rows)
            worst = max(worst, _rel_fro(dq_h[b, h, rows], rq))
    assert worst <= GRAD_TOL, worst


def test_bwd_gqa_causal_b1_h8_kv2_n4096_d128_full_group(fa):
    """GQA backward against the full oracle on one KV head and its whole group
    (dK and dV of a KV head sum over the group's four query heads)."""
    B, Hq, Hkv, N, d = 1, 8, 2, 4096, 128
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "bf16", seed=4096 + 8, grad=True)
    dq, dk, dv = _run_bwd(fa, inp, True, d ** -0.5)
    g = Hq // Hkv
    for hk in range(Hkv):
        qs, kvs = slice(hk * g, (hk + 1) * g), slice(hk, hk + 1)
        rq, rk, rv, _ = ORACLE.attention_backward(INP.as_f64(inp["q"][:, qs]), INP.as_f64(inp["k"][:, kvs]),
                                                 INP.as_f64(inp["v"][:, kvs]), INP.as_f64(inp["do"][:, qs]),
                                                 d ** -0.5, True)
        for name, got, ref in (("dq", dq[:, qs], rq), ("dk", dk[:, kvs], rk), ("dv", dv[:, kvs], rv)):
            err = _rel_fro(INP.as_f64(got), ref)
            assert err <= GRAD_TOL, (name, hk, err)


def test_bwd_gqa_causal_b1_h32_kv8_n16384_d128(fa):
    """GQA backward at the 16k-token GQA workload: dQ, dK and dV of the last KV
    head's group in full (dK and dV as the sum of the oracle's per-row-block
    shares over all 16384 queries of its four query heads), the dV and dK
    identities on every KV head, and exact dQ on sampled rows of every query
    head."""
    w = INP.WORKLOADS["gqa_causal_bf16_b1_h32_kv8_n16384_d128"]
    inp = INP.make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, "bf16", seed=16384 + 32, grad=True)
    dq, dk, dv = _run_bwd(fa, inp, True, w.scale)
    dq_h, dk_h, dv_h = (INP.as_f64(t) for t in (dq, dk, dv))
    q, k, v, do = (inp[n].float().numpy() for n in ("q", "k", "v", "do"))
    g = w.Hq // w.Hkv
    hk = w.Hkv - 1
    rk = np.zeros((w.N, w.d))
    rv = np.zeros((w.N, w.d))
    for h in range(hk * g, (hk + 1) * g):
        rq = np.zeros((w.N, w.d))
        for r0 in range(0, w.N, 2048):
            rows = list(range(r0, min(r0 + 2048, w.N)))
            dq_rows, dk_part, dv_part = ORACLE.attention_backward_rows(q, k, v, do, w.scale, True, 0, h, rows)
            rq[rows] = dq_rows
            rk += dk_part
            rv += dv_part
        assert _rel_fro(dq_h[0, h], rq) <= GRAD_TOL, ("dq", h)
    assert _rel_fro(dk_h[0, hk], rk) <= GRAD_TOL, "dk"
    assert _rel_fro(dv_h[0, hk], rv) <= GRAD_TOL, "dv"
    _group_identities(dk_h, dv_h, do.astype(np.float64), w.Hq, w.Hkv)
    rng = np.random.default_rng(11)
    worst = 0.0
    for h in range(w.Hq):
        rows = _sample_rows(w.N, rng, n_random=6)
        rq, _, _ = ORACLE.attention_backward_rows(q, k, v, do, w.scale, True, 0, h, rows)
        worst = max(worst, _rel_fro(dq_h[0, h, rows], rq))
    assert worst <= GRAD_TOL, worst


def test_pair_shards_on_one_gpu_match_the_single_call(fa):
    """The (batch, KV head) partition used across GPUs, run on one GPU: three
    emulated ranks each call fa_fwd and fa_bwd on views of their slice of the
    inputs and outputs. O and LSE equal the single call's bit for bit; dQ, dK
    and dV (f32 shares added in the order CTAs finish) agree to one bf16
    rounding step."""
    from exact_io_aware_61_b200.shard import kv_view, pair_range, q_view

    B, Hq, Hkv, N, d = 2, 8, 4, 1000, 128
    scale = d ** -0.5
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "bf16", seed=404, grad=True)
    q, k, v, do = (_to_dev(inp[n]) for n in ("q", "k", "v", "do"))
    o_full, lse_full = fa.forward(q, k, v, causal=True, scale=scale)
    ref = fa.backward(q, k, v, o_full, lse_full, do, causal=True, scale=scale)
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, Hq, N), float("nan"), device="cuda")
    grads = [torch.full_like(t, float("nan")) for t in ref]
    world = 3
    for rank in range(world):
        s = pair_range(B, Hq, Hkv, rank, world)
        qv, dov, ov, lv, dqv = (q_view(t, s) for t in (q, do, o, lse, grads[0]))
        kvv, vvv, dkv, dvv = (kv_view(t, s) for t in (k, v, grads[1], grads[2]))
        fa.fa_fwd(qv, kvv, vvv, ov, lv, True, scale)
        ws = torch.empty(max(fa.fa_bwd_workspace_size(*s.local_shape(), N, d), 16), dtype=torch.uint8,
                         device="cuda")
        fa.fa_bwd(qv, kvv, vvv, ov, lv, dov, dqv, dkv, dvv, ws, True, scale)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    assert torch.equal(o, o_full) and torch.equal(lse, lse_full)
    for got, want in zip(grads, ref):
        diff = (got.float() - want.float()).abs()
        assert bool(torch.all(diff <= 2.0 ** -7 * want.float().abs() + 1e-30))


# ------------------------------------------------------- KV-cache forward

KVCACHE_SHAPES = [  # (B, Hq, Hkv, Nq, Nk, d)
    (2, 8, 2, 1, 1000, 128),   # GQA decode, ragged Nk, several key splits
    (1, 4, 4, 4, 777, 64),     # MHA, four new queries
    (1, 32, 1, 2, 4096, 128),  # MQA, 64 query rows per KV head
    (3, 8, 8, 1, 64, 256),     # one key tile
    (1, 2, 1, 16, 16, 128),    # Nq = Nk: the square problem
    (1, 16, 2, 8, 5000, 256),  # 64 rows per KV head at d = 256
    (2, 4, 1, 1, 1, 64),       # a single cached key
    (1, 32, 1, 4, 3000, 128),  # 128 query rows per KV head (the tensor-core tile)
    (1, 64, 2, 4, 2000, 64),   # 128 rows at d = 64
    (1, 8, 1, 16, 1029, 128),  # one-tile splits: the last holds 5 keys, which 11 of the queries do not see
    (1, 32, 2, 8, 3000, 256),  # 128 rows at d = 256
]


def _run_kvcache(fa, q, k, v, causal, scale):
    """fa_fwd_kvcache into canary-guarded O, LSE and workspace."""
    q, k, v = (_to_dev(t) for t in (q, k, v))
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    go = Guarded(q.shape, q.dtype, fill=float("nan"))
    gl = Guarded((B, Hq, Nq), torch.float32, fill=float("nan"))
    gw = Guarded((max(fa.fa_fwd_kvcache_workspace_size(B, Hq, Hkv, Nq, Nk, d), 16),), torch.uint8)
    fa.fa_fwd_kvcache(q, k, v, go.t, gl.t, gw.t, causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    check_all(("O", go), ("LSE", gl), ("workspace", gw))
    return go.t, gl.t


def _kvcache_inputs(B, Hq, Hkv, Nq, Nk, d, seed):
    # the new queries are the last Nq rows of a seeded square problem
    inp = INP.make_inputs(B, Hq, Hkv, Nk, d, "bf16", seed=seed)
    return inp["q"][:, :, Nk - Nq:].contiguous(), inp["k"], inp["v"]


@pytest.mark.parametrize("shape", KVCACHE_SHAPES, ids=lambda s: "b%d_h%d_kv%d_nq%d_nk%d_d%d" % s)
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_kvcache_bf16(fa, shape, causal):
    B, Hq, Hkv, Nq, Nk, d = shape
    q, k, v = _kvcache_inputs(B, Hq, Hkv, Nq, Nk, d, seed=Nk + 7 * Nq + d)
    o, lse = _run_kvcache(fa, q, k, v, causal, d ** -0.5)
    ro, rl = ORACLE.attention_forward_kvcache(INP.as_f64(q), INP.as_f64(k), INP.as_f64(v), d ** -0.5, causal)
    assert np.max(np.abs(INP.as_f64(o) - ro)) <= O_TOL_BF16
    assert np.max(np.abs(INP.as_f64(lse) - rl)) <= LSE_TOL_BF16


def test_fwd_kvcache_decode_b8_h32_kv8_nk32768_d128(fa):
    """One new token per sequence against a 32k-token cache, the whole batch
    against the full oracle (one score row per head)."""
    B, Hq, Hkv, Nq, Nk, d = 8, 32, 8, 1, 32768, 128
    g = torch.Generator(device="cpu").manual_seed(32768)
    q = torch.randn((B, Hq, Nq, d), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hkv, Nk, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, Nk, d), generator=g).to(torch.bfloat16)
    o, lse = _run_kvcache(fa, q, k, v, True, d ** -0.5)
    ro, rl = ORACLE.attention_forward_kvcache(INP.as_f64(q), INP.as_f64(k), INP.as_f64(v), d ** -0.5, True)
    assert np.max(np.abs(INP.as_f64(o) - ro)) <= O_TOL_BF16
    assert np.max(np.abs(INP.as_f64(lse) - rl)) <= LSE_TOL_BF16


def test_fwd_kvcache_square_case_matches_fwd(fa):
    """With Nq = Nk the KV-cache path computes the square causal problem."""
    inp = INP.make_inputs(1, 8, 2, 8, 128, "bf16", seed=88)
    q, k, v = (_to_dev(inp[n]) for n in "qkv")
    o1, l1 = fa.forward_kvcache(q, k, v, causal=True)
    o2, l2 = fa.forward(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert float((o1.float() - o2.float()).abs().max()) <= O_TOL_BF16
    assert float((l1 - l2).abs().max()) <= LSE_TOL_BF16


# ---------------------------------------------------------- ABI behaviour

def test_abi_rejects_bad_arguments_without_writing(fa):
    q = torch.randn(1, 2, 64, 64, device="cuda").to(torch.bfloat16)
    k, v = q.clone(), q.clone()
    o = torch.full_like(q, 7.0)
    lse = torch.full((1, 2, 64), 7.0, device="cuda")

    import ctypes

    def ptr(t):
        return None if t is None else ctypes.c_void_p(t.data_ptr())

    def call(**kw):
        args = dict(q=q, k=k, v=v, o=o, lse=lse, B=1, Hq=2, Hkv=2, N=64, d=64, scale=0.125, causal=0, dtype=0)
        args.update(kw)
        lib = fa.load()
        return lib.fa_fwd(ptr(args["q"]), ptr(args["k"]), ptr(args["v"]), ptr(args["o"]), ptr(args["lse"]),
                          args["B"], args["Hq"], args["Hkv"], args["N"], args["d"], args["scale"], args["causal"],
                          args["dtype"], ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))

    assert call(N=-1) == fa.FA_ERR_INVALID
    assert call(d=96) == fa.FA_ERR_UNSUPPORTED
    assert call(Hq=3, Hkv=2) == fa.FA_ERR_INVALID
    assert call(q=None) == fa.FA_ERR_INVALID
    assert call(causal=2) == fa.FA_ERR_INVALID
    assert call(dtype=7) == fa.FA_ERR_INVALID
    assert call(scale=float("nan")) == fa.FA_ERR_INVALID
    qm = torch.empty(q.numel() + 8, dtype=torch.bfloat16, device="cuda")[1:1 + q.numel()].view(q.shape)
    assert call(q=qm) == fa.FA_ERR_INVALID  # 2-byte aligned pointer
    assert call(B=0) == fa.FA_OK and call(N=0) == fa.FA_OK  # empty problems: nothing to do
    torch.cuda.synchronize()
    assert torch.all(o == 7.0) and torch.all(lse == 7.0)
    # backward: unsupported dtype/d and a short workspace
    do = torch.randn_like(q)
    dq, dk, dv = (torch.full_like(q, 3.0) for _ in range(3))
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd(q, k, v, o, lse, do, dq, dk, dv, small, False, 0.125)
    assert e.value.status == fa.FA_ERR_WORKSPACE
    q32 = torch.zeros(1, 1, 8, 64, dtype=torch.float32, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.backward(q32, q32, q32, q32, torch.zeros(1, 1, 8, device="cuda"), q32)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.all(dq == 3.0) and torch.all(dk == 3.0) and torch.all(dv == 3.0)


def test_bounded_wait_timeout_reports_status(fa):
    assert fa.fa_last_device_status() == fa.FA_OK
    assert fa.fa_selftest_wait_timeout(50_000_000) == fa.FA_OK  # 50 ms
    assert fa.fa_last_device_status() == fa.FA_ERR_TIMEOUT
    assert fa.fa_last_device_status() == fa.FA_OK  # cleared by the read
    # the context is still usable afterwards
    inp = INP.make_inputs(1, 1, 1, 130, 64, "bf16", seed=2)
    o, lse = _run_fwd(fa, inp, True, 0.125)
    ro, rl = ORACLE.attention_forward(*(INP.as_f64(inp[n]) for n in "qkv"), 0.125, True)
    assert np.max(np.abs(INP.as_f64(o) - ro)) <= O_TOL_BF16
