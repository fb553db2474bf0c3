"""Packed variable-length and strided (BNHD) forward, fa_fwd_varlen, against
the fp64 oracle's attention_forward_varlen (attention within each sequence;
a sequence with fewer queries than keys places them at its last positions).

Tolerances as for the dense bf16 forward: O max-abs <= 2e-2, LSE max-abs <=
1e-3. Outputs are canary-guarded.
"""

import numpy as np
import pytest
import torch

import oracle.attention as ORACLE
from exact_io_aware_61_b200 import inputs as INP
from tests.guarded import Guarded, check_all

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 2e-2, 1e-3


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import exact_io_aware_61_b200 as fa_mod
    fa_mod.load()
    return fa_mod


def _run(fa, inp, causal, scale):
    q, k, v = (inp[n].cuda() for n in "qkv")
    cu_q, cu_k = inp["cu_q"].cuda(), inp["cu_k"].cuda()
    lens_q = (inp["cu_q"][1:] - inp["cu_q"][:-1]).tolist()
    go = Guarded(q.shape, q.dtype, fill=float("nan"))
    gl = Guarded(q.shape[:-1], torch.float32, fill=float("nan"))
    fa.fa_fwd_varlen(q, k, v, go.t, gl.t, cu_q, cu_k, max(lens_q), causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    check_all(("O", go), ("LSE", gl))
    return go.t, gl.t


PACKS = [  # (query lengths, key lengths, Hq, Hkv, d)
    ([1, 127, 129, 3000], [1, 127, 129, 3000], 8, 2, 128),
    ([1, 127, 129, 3000], [1, 127, 129, 3000], 4, 4, 64),
    ([300, 5, 1, 130], [300, 300, 17, 1000], 4, 1, 128),   # fewer queries than keys
    ([256, 255, 257, 512, 64], [256, 255, 257, 512, 64], 6, 3, 64),
]


@pytest.mark.parametrize("pack", PACKS, ids=lambda p: "q%s_k%s_h%d_kv%d_d%d" % (
    "-".join(map(str, p[0])), "-".join(map(str, p[1])), p[2], p[3], p[4]))
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_varlen_matches_oracle(fa, pack, causal):
    lens_q, lens_k, Hq, Hkv, d = pack
    inp = INP.make_varlen_inputs(lens_q, lens_k, Hq, Hkv, d, "bf16", seed=sum(lens_q) + d)
    scale = d ** -0.5
    o, lse = _run(fa, inp, causal, scale)
    ro, rl = ORACLE.attention_forward_varlen(*(INP.as_f64(inp[n]) for n in "qkv"), inp["cu_q"].numpy(),
                                            inp["cu_k"].numpy(), scale, causal)
    assert np.max(np.abs(INP.as_f64(o) - ro)) <= O_TOL
    assert np.max(np.abs(INP.as_f64(lse) - rl)) <= LSE_TOL


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_bnhd_equals_dense_bhnd(fa, causal):
    """Strided [B, N, H, d] inputs (the packed layout with equal lengths) give
    exactly what fa_fwd gives on the same values in [B, H, N, d]."""
    B, Hq, Hkv, N, d = 2, 8, 4, 1000, 128
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "bf16", seed=77)
    q, k, v = (inp[n].cuda() for n in "qkv")
    o_ref, lse_ref = fa.forward(q, k, v, causal=causal)
    qs, ks, vs = (t.transpose(1, 2).contiguous() for t in (q, k, v))
    o, lse = fa.forward_bnhd(qs, ks, vs, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    assert torch.equal(o.transpose(1, 2), o_ref)
    assert torch.equal(lse.transpose(1, 2), lse_ref)


def test_fwd_varlen_rejects_inconsistent_offsets(fa):
    """A sequence with more queries than keys (offsets are read on the device)
    is skipped and reported through the device status word; nothing is
    written for it."""
    inp = INP.make_varlen_inputs([8, 4], [8, 8], 2, 2, 64, "bf16", seed=3)
    inp["cu_k"] = torch.tensor([0, 8, 10], dtype=torch.int32)  # second sequence: 4 queries, 2 keys
    q, k, v = (inp[n].cuda() for n in "qkv")
    go = Guarded(q.shape, q.dtype, fill=5.0)
    gl = Guarded(q.shape[:-1], torch.float32, fill=5.0)
    fa.fa_fwd_varlen(q, k[:10], v[:10], go.t, gl.t, inp["cu_q"].cuda(), inp["cu_k"].cuda(), 8, True, 0.125)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_ERR_INVALID
    assert fa.fa_last_device_status() == fa.FA_OK
    assert torch.all(go.t[8:] == 5.0) and torch.all(gl.t[8:] == 5.0)
    check_all(("O", go), ("LSE", gl))


# ------------------------------------------------------------------ backward
# Gradients against attention_backward_varlen: relative Frobenius error <= 2e-2
# per tensor and per sequence (as for the dense backward), outputs guarded.

GRAD_TOL = 2e-2


def _rel(a, b):
    # relative Frobenius error, with an RMS floor of 1e-3 under the reference
    # (a one-key sequence has dQ = 0 exactly: dS = P (dP - D) with P = 1, D = dP)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-3 * np.sqrt(b.size), 1e-30))


def _run_bwd(fa, inp, o, lse, causal, scale):
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    cu_q, cu_k = inp["cu_q"].cuda(), inp["cu_k"].cuda()
    lq = (inp["cu_q"][1:] - inp["cu_q"][:-1]).tolist()
    lk = (inp["cu_k"][1:] - inp["cu_k"][:-1]).tolist()
    gq = Guarded(q.shape, q.dtype, fill=float("nan"))
    gk = Guarded(k.shape, k.dtype, fill=float("nan"))
    gv = Guarded(v.shape, v.dtype, fill=float("nan"))
    nbytes = fa.fa_bwd_varlen_workspace_size(len(lq), q.shape[0], k.shape[0], q.shape[1], k.shape[1], q.shape[2])
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    fa.fa_bwd_varlen(q, k, v, o, lse, do, gq.t, gk.t, gv.t, cu_q, cu_k, max(lq), max(lk), ws, causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    check_all(("dQ", gq), ("dK", gk), ("dV", gv))
    return gq.t, gk.t, gv.t


BWD_PACKS = PACKS + [
    ([0, 200, 3], [64, 200, 130], 4, 2, 128),   # a sequence without queries: its keys get zero gradients
    ([513, 2], [1100, 2], 16, 1, 64),            # MQA: the group is split over several CTAs per key tile
]


@pytest.mark.parametrize("pack", BWD_PACKS, ids=lambda p: "q%s_k%s_h%d_kv%d_d%d" % (
    "-".join(map(str, p[0])), "-".join(map(str, p[1])), p[2], p[3], p[4]))
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_varlen_matches_oracle(fa, pack, causal):
    lens_q, lens_k, Hq, Hkv, d = pack
    inp = INP.make_varlen_inputs(lens_q, lens_k, Hq, Hkv, d, "bf16", seed=sum(lens_k) + 7 * d, grad=True)
    scale = d ** -0.5
    o, lse = _run(fa, inp, causal, scale)
    dq, dk, dv = _run_bwd(fa, inp, o, lse, causal, scale)
    cq, ck = inp["cu_q"].numpy(), inp["cu_k"].numpy()
    rq, rk, rv = ORACLE.attention_backward_varlen(*(INP.as_f64(inp[n]) for n in ("q", "k", "v", "do")), cq, ck,
                                                 scale, causal)
    got = {"dq": INP.as_f64(dq), "dk": INP.as_f64(dk), "dv": INP.as_f64(dv)}
    want = {"dq": rq, "dk": rk, "dv": rv}
    for name in want:
        assert _rel(got[name], want[name]) <= GRAD_TOL, name
    for s in range(len(lens_q)):
        sq, sk = slice(cq[s], cq[s + 1]), slice(ck[s], ck[s + 1])
        if lens_q[s] == 0:
            assert np.all(got["dk"][sk] == 0.0) and np.all(got["dv"][sk] == 0.0)
            continue
        assert _rel(got["dq"][sq], rq[sq]) <= GRAD_TOL, ("dq", s)
        assert _rel(got["dk"][sk], rk[sk]) <= GRAD_TOL, ("dk", s)
        assert _rel(got["dv"][sk], rv[sk]) <= GRAD_TOL, ("dv", s)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_bnhd_matches_dense_bhnd(fa, causal):
    """Strided [B, N, H, d] backward against fa_bwd on the same values in
    [B, H, N, d]: dK and dV are summed in the same order (equal bits); dQ is
    accumulated with atomics, so it agrees to the rounding of the order."""
    B, Hq, Hkv, N, d = 2, 8, 4, 1000, 128
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "bf16", seed=79, grad=True)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, causal=causal)
    dq_ref, dk_ref, dv_ref = fa.backward(q, k, v, o, lse, do, causal=causal)
    t = lambda x: x.transpose(1, 2).contiguous()
    dq, dk, dv = fa.backward_bnhd(t(q), t(k), t(v), t(o), lse.transpose(1, 2).contiguous(), t(do), causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    assert torch.equal(dk.transpose(1, 2), dk_ref) and torch.equal(dv.transpose(1, 2), dv_ref)
    diff = (dq.transpose(1, 2).float() - dq_ref.float()).abs()
    assert torch.all(diff <= 2.0 ** -7 * dq_ref.float().abs() + 1e-6)


def test_bwd_varlen_no_queries_at_all_zeroes_dk_dv(fa):
    inp = INP.make_varlen_inputs([0, 0], [5, 300], 2, 2, 64, "bf16", seed=5, grad=True)
    k, v = inp["k"].cuda(), inp["v"].cuda()
    q = torch.zeros((16, 2, 64), dtype=torch.bfloat16, device="cuda")  # total_q = 0: pointers unused
    dk, dv = Guarded(k.shape, k.dtype, fill=3.0), Guarded(v.shape, v.dtype, fill=3.0)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    fa.fa_bwd_varlen(q[:0], k, v, q[:0], torch.zeros((0, 2), device="cuda"), q[:0], q[:0], dk.t, dv.t,
                     inp["cu_q"].cuda(), inp["cu_k"].cuda(), 0, 300, ws, True, 0.125)
    torch.cuda.synchronize()
    assert torch.all(dk.t == 0) and torch.all(dv.t == 0)
    check_all(("dK", dk), ("dV", dv))


def test_bwd_varlen_rejects_inconsistent_offsets_and_small_workspace(fa):
    inp = INP.make_varlen_inputs([8, 4], [8, 8], 2, 2, 64, "bf16", seed=3, grad=True)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = _run(fa, inp, True, 0.125)
    nbytes = fa.fa_bwd_varlen_workspace_size(2, 12, 16, 2, 2, 64)
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd_varlen(q, k, v, o, lse, do, torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                         inp["cu_q"].cuda(), inp["cu_k"].cuda(), 8, 8,
                         torch.empty(nbytes - 16, dtype=torch.uint8, device="cuda"), True, 0.125)
    assert e.value.status == fa.FA_ERR_WORKSPACE
    bad_k = torch.tensor([0, 8, 10], dtype=torch.int32, device="cuda")  # second sequence: 4 queries, 2 keys
    dk = Guarded(k[:10].shape, k.dtype, fill=5.0)
    fa.fa_bwd_varlen(q, k[:10].contiguous(), v[:10].contiguous(), o, lse, do, torch.empty_like(q), dk.t,
                     torch.empty_like(dk.t), inp["cu_q"].cuda(), bad_k, 8, 8,
                     torch.empty(nbytes, dtype=torch.uint8, device="cuda"), True, 0.125)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_ERR_INVALID
    assert fa.fa_last_device_status() == fa.FA_OK
    assert torch.all(dk.t[8:] == 5.0)
    check_all(("dK", dk))
