"""Parity of the sequence-sharding calls (fa_fwd_partial, fa_merge_partials, fa_bwd_partial) with the fp64 oracle.

``fa_fwd_partial`` is checked against ``attention_forward_positions`` with
query i at position i + diag_offset and key j at position j, over offsets that
cut tiles at every boundary (whole tiles with no visible key, rows of a tile
with none, offsets past +-N), for d = 64, 128 and 256. ``fa_merge_partials``
is checked against ``merge_outputs`` on the same bf16 values, including parts
and whole rows with LSE = -inf. The striped ring is then emulated on one GPU:
each rank's blocks run one after another through the library (no kernel waits
on another), are merged, and must equal the oracle's unsharded attention.
Tolerances are the forward's: O max-abs <= 2e-2, LSE max-abs <= 1e-3, with
rows that see no key required to be exactly O = 0, LSE = -inf.
"""

import numpy as np
import pytest
import torch

import oracle.attention as ORACLE
from exact_io_aware_61_b200 import inputs as INP
from exact_io_aware_61_b200 import seqpar
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


def _compare(o, lse, ro, rl):
    o = np.asarray(o, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    empty = np.isneginf(rl)
    assert np.array_equal(np.isneginf(lse), empty), "rows with no visible key differ"
    assert np.all(o[empty] == 0.0)
    assert np.max(np.abs(o[~empty] - ro[~empty]), initial=0.0) <= O_TOL
    assert np.max(np.abs(lse[~empty] - rl[~empty]), initial=0.0) <= LSE_TOL


def _partial(fa, q, k, v, causal, scale, diag):
    B, Hq, N, d = q.shape
    go = Guarded(q.shape, q.dtype, fill=float("nan"))
    gl = Guarded((B, Hq, N), torch.float32, fill=float("nan"))
    fa.fa_fwd_partial(q, k, v, go.t, gl.t, causal, scale, diag)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    check_all(("O", go), ("LSE", gl))
    return go.t, gl.t


PARTIAL_SHAPES = [(1, 2, 2, 300, 64), (1, 4, 2, 700, 128), (2, 2, 1, 385, 256), (1, 2, 2, 1, 128)]


@pytest.mark.parametrize("shape", PARTIAL_SHAPES, ids=lambda s: "b%d_h%d_kv%d_n%d_d%d" % s)
def test_fwd_partial_diagonal_offsets(fa, shape):
    B, Hq, Hkv, N, d = shape
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "bf16", seed=N + 3 * d)
    q, k, v = (inp[n].cuda().contiguous() for n in "qkv")
    qq, kk, vv = (INP.as_f64(inp[n]) for n in "qkv")
    offsets = sorted({-N - 5, -N, -N + 1, -300, -257, -256, -255, -129, -128, -127, -1, 0, 1, 127, 128, 255,
                      N - 1, N, N + 7})
    for diag in offsets:
        o, lse = _partial(fa, q, k, v, True, d ** -0.5, diag)
        ro, rl = ORACLE.attention_forward_positions(qq, kk, vv, np.arange(N) + diag, np.arange(N), d ** -0.5, True)
        _compare(INP.as_f64(o), INP.as_f64(lse), ro, rl)
    # without the mask the offset is ignored: the result is fa_fwd's, bit for bit
    o, lse = _partial(fa, q, k, v, False, d ** -0.5, -77)
    fo, fl = fa.forward(q, k, v, False, d ** -0.5)
    assert torch.equal(o, fo) and torch.equal(lse, fl)


def test_fwd_partial_offset_zero_is_fa_fwd(fa):
    inp = INP.make_inputs(2, 4, 2, 1000, 128, "bf16", seed=7)
    q, k, v = (inp[n].cuda().contiguous() for n in "qkv")
    o, lse = _partial(fa, q, k, v, True, 0.1, 0)
    fo, fl = fa.forward(q, k, v, True, 0.1)
    assert torch.equal(o, fo) and torch.equal(lse, fl)


def test_fwd_partial_rejects_f32(fa):
    q = torch.zeros(1, 1, 8, 64, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd_partial(q, q, q, torch.empty_like(q), torch.empty(1, 1, 8, device="cuda"), True, 0.1, -1)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("parts", [1, 3, 8, 37])
def test_merge_partials_matches_oracle(fa, d, parts):
    rng = np.random.default_rng(1000 * parts + d)
    rows = 1531
    o_parts = torch.from_numpy(rng.standard_normal((parts, rows, d))).to(torch.bfloat16)
    lse_np = rng.normal(3.0, 4.0, (parts, rows)).astype(np.float32)
    lse_np[rng.random((parts, rows)) < 0.2] = -np.inf   # parts that saw no key of a row
    lse_np[:, 5] = -np.inf                               # a row no part saw
    if parts > 1:
        lse_np[:, 6] = 80.0                              # equal, large LSEs
    lse_parts = torch.from_numpy(lse_np)
    go = Guarded((rows, d), torch.bfloat16, fill=float("nan"))
    gl = Guarded((rows,), torch.float32, fill=float("nan"))
    fa.fa_merge_partials(o_parts.cuda(), lse_parts.cuda(), go.t, gl.t)
    torch.cuda.synchronize()
    check_all(("O", go), ("LSE", gl))
    ro, rl = ORACLE.merge_outputs(o_parts.double().numpy(), lse_np.astype(np.float64))
    o = go.t.double().cpu().numpy()
    lse = gl.t.double().cpu().numpy()
    empty = np.isneginf(rl)
    assert empty[5] and np.array_equal(np.isneginf(lse), empty)
    assert np.all(o[empty] == 0.0)
    # float32 weights, one bf16 rounding of the result
    assert np.max(np.abs(o[~empty] - ro[~empty])) <= 2.0 ** -8 * np.max(np.abs(ro)) + 1e-6
    assert np.max(np.abs(lse[~empty] - rl[~empty])) <= 2e-5 * np.max(np.abs(rl[~empty])) + 1e-6


def test_merge_partials_rejects_overlap_and_bad_sizes(fa):
    parts = torch.zeros(2, 16, 64, dtype=torch.bfloat16, device="cuda")
    lse_parts = torch.zeros(2, 16, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.fa_merge_partials(parts, lse_parts, parts[0], torch.empty(16, device="cuda"))
    assert e.value.status == fa.FA_ERR_INVALID
    with pytest.raises(fa.FAError) as e:
        fa.fa_merge_partials(parts, lse_parts, torch.empty(16, 64, dtype=torch.bfloat16, device="cuda"),
                             lse_parts[1])
    assert e.value.status == fa.FA_ERR_INVALID
    bad = torch.zeros(2, 16, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.fa_merge_partials(bad, lse_parts, torch.empty(16, 96, dtype=torch.bfloat16, device="cuda"),
                             torch.empty(16, device="cuda"))
    assert e.value.status == fa.FA_ERR_INVALID


def _emulate_ring(fa, q, k, v, world, causal, scale):
    """Every rank's ring steps, one after another on one GPU: per rank, its
    blocks against every rank's K/V shard in ring order, then the merge."""
    shards = [[seqpar.shard_striped(t, r, world) for t in (q, k, v)] for r in range(world)]
    outs = []
    for r in range(world):
        qr = shards[r][0]
        o_parts = torch.empty((world,) + tuple(qr.shape), dtype=qr.dtype, device=qr.device)
        l_parts = torch.empty((world,) + tuple(qr.shape[:-1]), dtype=torch.float32, device=qr.device)
        for t, (src, diag) in enumerate(seqpar.ring_schedule(r, world, causal)):
            fa.fa_fwd_partial(qr, shards[src][1], shards[src][2], o_parts[t], l_parts[t], causal, scale, diag)
        go = Guarded(qr.shape, qr.dtype, fill=float("nan"))
        gl = Guarded(qr.shape[:-1], torch.float32, fill=float("nan"))
        fa.fa_merge_partials(o_parts, l_parts, go.t, gl.t)
        torch.cuda.synchronize()
        assert fa.fa_last_device_status() == fa.FA_OK
        check_all(("O", go), ("LSE", gl))
        outs.append((go.t.clone(), gl.t.clone()))
    o = seqpar.unshard_striped([x[0] for x in outs])
    lse = seqpar.unshard_striped([x[1][..., None] for x in outs])[..., 0]
    return o, lse


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_striped_ring_emulated_equals_unsharded(fa, world, causal):
    B, Hq, Hkv, d = 1, 4, 2, 128
    N = {2: 770, 3: 771, 4: 772}[world]  # shards of 385, 257 and 193 rows: ragged tiles
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "bf16", seed=17 + world)
    q, k, v = (inp[n].cuda().contiguous() for n in "qkv")
    o, lse = _emulate_ring(fa, q, k, v, world, causal, d ** -0.5)
    ro, rl = ORACLE.attention_forward(*(INP.as_f64(inp[n]) for n in "qkv"), d ** -0.5, causal)
    _compare(INP.as_f64(o), INP.as_f64(lse), ro, rl)


def test_striped_ring_emulated_w8_b2_h32_n8192_d128_sampled(fa):
    """Eight striped ranks on the benchmark shape (causal): sampled rows of
    every head against the oracle, plus LSE >= the local block's LSE on every
    row (adding keys never lowers the log-sum-exp)."""
    B, Hq, Hkv, N, d, W = 2, 32, 32, 8192, 128, 8
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "bf16", seed=2024)
    q, k, v = (inp[n].cuda().contiguous() for n in "qkv")
    o, lse = _emulate_ring(fa, q, k, v, W, True, d ** -0.5)
    fo, fl = fa.forward(q, k, v, True, d ** -0.5)
    # the same rows computed in one pass agree to the bf16 rounding of two paths
    assert torch.max(torch.abs(o.float() - fo.float())).item() <= O_TOL
    assert torch.max(torch.abs(lse - fl)).item() <= LSE_TOL
    rng = np.random.default_rng(5)
    for b, h in [(0, 0), (1, 31), (0, 17)]:
        qq, kk, vv = (INP.as_f64(inp[n][b:b + 1, h:h + 1]) for n in "qkv")
        rows = sorted(set([0, 1, 7, 8, 9, N - 1] + [int(x) for x in rng.integers(0, N, 12)]))
        ro, rl = ORACLE.attention_forward_rows(qq, kk, vv, d ** -0.5, True, 0, 0, rows)
        _compare(INP.as_f64(o[b, h, rows]), INP.as_f64(lse[b, h, rows]), ro, rl)



# --------------------------------------------------------------- backward

GRAD_TOL = 2e-2


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-3 * np.sqrt(b.size), 1e-30))


def test_bwd_partial_one_block_is_fa_bwd(fa):
    """One block with offset 0 against zeroed accumulators is fa_bwd: dK, dV
    bit for bit (head split 1), dQ to the rounding of its atomic order."""
    B, Hq, Hkv, N, d = 2, 8, 4, 1000, 128
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "bf16", seed=91, grad=True)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, True)
    dq_ref, dk_ref, dv_ref = fa.backward(q, k, v, o, lse, do, True)
    ws = torch.empty(fa.fa_bwd_workspace_size(B, Hq, Hkv, N, d), dtype=torch.uint8, device="cuda")
    gk = Guarded(k.shape, torch.float32, fill=0.0)
    gv = Guarded(v.shape, torch.float32, fill=0.0)
    fa.fa_bwd_prep(o, lse, do, ws, Hkv)
    fa.fa_bwd_partial(q, k, v, do, gk.t, gv.t, ws, True, d ** -0.5, 0)
    dq = torch.empty_like(q)
    fa.fa_bwd_dq(dq, ws, Hkv)
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    fa.fa_f32_to_bf16(gk.t, dk)
    fa.fa_f32_to_bf16(gv.t, dv)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    check_all(("dK acc", gk), ("dV acc", gv))
    assert torch.equal(dk, dk_ref) and torch.equal(dv, dv_ref)
    diff = (dq.float() - dq_ref.float()).abs()
    assert torch.all(diff <= 2.0 ** -7 * dq_ref.float().abs() + 1e-6)


def _emulate_ring_backward(fa, q, k, v, do, world, causal, scale):
    """Every rank's ring backward on one GPU: the forward shards from the
    emulated ring forward, then per rank its prep, one fa_bwd_partial per key
    block (the accumulators of each key shard are shared, as if they had
    travelled), its dQ; finally the accumulators to bf16."""
    o, lse = _emulate_ring(fa, q, k, v, world, causal, scale)
    shard = lambda t, r: seqpar.shard_striped(t, r, world)
    ks = [shard(k, c) for c in range(world)]
    vs = [shard(v, c) for c in range(world)]
    acc_k = [torch.zeros(t.shape, dtype=torch.float32, device="cuda") for t in ks]
    acc_v = [torch.zeros(t.shape, dtype=torch.float32, device="cuda") for t in vs]
    dqs = []
    for r in range(world):
        qr, dor = shard(q, r), shard(do, r)
        ops = seqpar.LibraryBackwardOps(qr, ks[r], causal, scale)
        ops.prep(shard(o, r), seqpar.shard_striped(lse[..., None], r, world)[..., 0].contiguous(), dor)
        for src, diag in seqpar.ring_schedule(r, world, causal):
            ops.block(qr, ks[src], vs[src], dor, acc_k[src], acc_v[src], diag)
        dq = torch.empty_like(qr)
        ops.finish(dq)
        dqs.append(dq)
    dks = [torch.empty_like(t) for t in ks]
    dvs = [torch.empty_like(t) for t in vs]
    for c in range(world):
        fa.fa_f32_to_bf16(acc_k[c], dks[c])
        fa.fa_f32_to_bf16(acc_v[c], dvs[c])
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == fa.FA_OK
    return tuple(seqpar.unshard_striped(x) for x in (dqs, dks, dvs))


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_striped_ring_backward_emulated_equals_unsharded(fa, world, causal):
    B, Hq, Hkv, d = 1, 4, 2, 128
    N = {2: 770, 3: 771, 4: 772}[world]
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "bf16", seed=29 + world, grad=True)
    q, k, v, do = (inp[n].cuda().contiguous() for n in ("q", "k", "v", "do"))
    dq, dk, dv = _emulate_ring_backward(fa, q, k, v, do, world, causal, d ** -0.5)
    rq, rk, rv, _ = ORACLE.attention_backward(*(INP.as_f64(inp[n]) for n in ("q", "k", "v", "do")), d ** -0.5, causal)
    assert _rel(INP.as_f64(dq), rq) <= GRAD_TOL
    assert _rel(INP.as_f64(dk), rk) <= GRAD_TOL
    assert _rel(INP.as_f64(dv), rv) <= GRAD_TOL


def test_striped_ring_backward_emulated_w4_d64_gqa(fa):
    B, Hq, Hkv, N, d, world = 2, 8, 2, 2048, 64, 4
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "bf16", seed=4242, grad=True)
    q, k, v, do = (inp[n].cuda().contiguous() for n in ("q", "k", "v", "do"))
    dq, dk, dv = _emulate_ring_backward(fa, q, k, v, do, world, True, d ** -0.5)
    rq, rk, rv, _ = ORACLE.attention_backward(*(INP.as_f64(inp[n]) for n in ("q", "k", "v", "do")), d ** -0.5, True)
    assert _rel(INP.as_f64(dq), rq) <= GRAD_TOL
    assert _rel(INP.as_f64(dk), rk) <= GRAD_TOL
    assert _rel(INP.as_f64(dv), rv) <= GRAD_TOL
