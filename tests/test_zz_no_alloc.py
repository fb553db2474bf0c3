"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers cannot give fa_bwd a workspace, because they run where the
device allocator must not be touched or have no allocator at all. For them
fa_bwd_noalloc keeps its scratch in a fixed array inside the library. This
test calls it through the C ABI twice in a row (the second call finds the
first call's leftovers in the shared array) and checks each result against
fa_bwd with a caller-allocated workspace: bit for bit where the backward is
deterministic (dK and dV when a KV head's query heads are not split over
CTAs), within one bf16 rounding step where f32 shares are added in whatever
order CTAs finish (dQ always; dK and dV with split heads), and against the
fp64 oracle at the gradient tolerance the other tests use. Outputs are canary-guarded. It lives
in its own file, collected last, and passes both alone in a fresh process and
after the rest of the suite.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle.attention as ORACLE
from exact_io_aware_61_b200 import inputs as INP
from tests.guarded import Guarded, check_all

pytestmark = pytest.mark.gpu

GRAD_TOL = 2e-2


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import exact_io_aware_61_b200 as fa_mod
    fa_mod.load()
    return fa_mod


def _rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _call_noalloc_abi(lib, q, k, v, o, lse, do, dq, dk, dv, causal, scale):
    B, Hq, N, d = q.shape
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.fa_bwd_noalloc(p(q), p(k), p(v), p(o), p(lse), p(do), p(dq), p(dk), p(dv), B, Hq, k.shape[1], N, d,
                              float(scale), int(causal), 0,
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _head_split(B, Hq, Hkv, N):
    ctas = B * Hkv * ((N + 127) // 128)
    g = Hq // Hkv
    return next((s for s in range(1, g + 1) if g % s == 0 and ctas * s >= 592), g)


@pytest.mark.parametrize("shape,causal", [((2, 2, 2, 300, 64), False), ((1, 4, 2, 1000, 128), True),
                                          ((4, 8, 8, 640, 128), True)])
def test_noalloc_matches_fa_bwd_twice(fa, shape, causal):
    lib = fa.load()
    B, Hq, Hkv, N, d = shape
    scale = d ** -0.5
    assert fa.fa_bwd_workspace_size(B, Hq, Hkv, N, d) <= fa._lib.NOALLOC_SCRATCH_BYTES
    split = _head_split(B, Hq, Hkv, N)
    for seed in (21, 22):  # two calls in a row on the shared scratch
        inp = INP.make_inputs(B, Hq, Hkv, N, d, "bf16", seed=seed, grad=True)
        q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
        o, lse = fa.forward(q, k, v, causal=causal, scale=scale)
        ref = fa.backward(q, k, v, o, lse, do, causal=causal, scale=scale)
        guards = [Guarded(t.shape, t.dtype, fill=float("nan")) for t in ref]
        rc = _call_noalloc_abi(lib, q, k, v, o, lse, do, *(g.t for g in guards), causal, scale)
        assert rc == fa.FA_OK, fa.status_string(rc)
        torch.cuda.synchronize()
        assert fa.fa_last_device_status() == fa.FA_OK
        check_all(*zip(("dq", "dk", "dv"), guards))
        oq, ok_, ov, _ = ORACLE.attention_backward(*(INP.as_f64(inp[n]) for n in ("q", "k", "v", "do")), scale,
                                                  causal)
        for name, g, r, o64 in zip(("dq", "dk", "dv"), guards, ref, (oq, ok_, ov)):
            got = g.t
            assert torch.isfinite(got).all(), name
            if name != "dq" and split == 1:
                assert torch.equal(got, r), (name, seed, "differs from fa_bwd")
            else:
                diff = (got.float() - r.float()).abs()
                assert bool(torch.all(diff <= 2.0 ** -7 * r.float().abs() + 1e-30)), (name, seed)
            err = _rel(got, torch.from_numpy(o64))
            assert err <= GRAD_TOL, (name, seed, err)


def test_noalloc_rejects_problems_beyond_its_scratch(fa):
    lib = fa.load()
    B, Hq, Hkv, N, d = 4, 32, 32, 32768, 128  # needs about 34 MB of scratch
    assert fa.fa_bwd_workspace_size(B, Hq, Hkv, N, d) > fa._lib.NOALLOC_SCRATCH_BYTES
    t = torch.zeros(16, dtype=torch.uint8, device="cuda")
    p = ctypes.c_void_p(t.data_ptr())
    rc = lib.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, B, Hq, Hkv, N, d, 0.1, 1, 0,
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == fa.FA_ERR_WORKSPACE
    assert torch.all(t == 0)
