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
