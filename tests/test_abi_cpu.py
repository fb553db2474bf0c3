"""Host-only checks of the C ABI: the library loads without a GPU, exports
every function ``include/fa.h`` declares, and rejects bad arguments before it
touches the device. No kernel is launched here."""

import ctypes
import os
import re

import pytest

import exact_io_aware_61_b200 as fa
from exact_io_aware_61_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.load()


def _declared():
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    return sorted(set(re.findall(r"FA_API\s+[\w\s\*]*?\b(fa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_status_string", "fa_last_device_status"):
        assert must in names
    assert sorted(fa.EXPORTED) == names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {fa.LIB_PATH}").read()
    exported = set(re.findall(r" T (fa_\w+)", out))
    assert set(_declared()) <= exported


def test_status_strings(lib):
    for code in range(6):
        s = fa.status_string(code)
        assert s.startswith("FA_")
    assert "unknown" in fa.status_string(99)


def _head_split(B, Hq, Hkv, N, d=128):
    """CTAs per (KV head, key tile) in the backward: 1 when B*Hkv*tiles >= 592,
    else the smallest divisor of the group size that reaches 592, else the
    group size. Key tiles of 128 keys, 64 at d = 256."""
    tile = 64 if d == 256 else 128
    ctas = B * Hkv * ((N + tile - 1) // tile)
    g = Hq // Hkv
    return next((s for s in range(1, g + 1) if g % s == 0 and ctas * s >= 592), g)


def test_workspace_formula(lib):
    # D and log2-scaled LSE padded to 128 rows per head, plus an f32 dQ accumulator
    B, Hq, Hkv, N, d = 2, 16, 16, 4096, 128
    assert _head_split(B, Hq, Hkv, N) == 1
    assert fa.fa_bwd_workspace_size(B, Hq, Hkv, N, d) == 4 * (2 * B * Hq * 4096 + B * Hq * N * d)
    # few CTAs (1 x 2 KV heads x 2 key tiles): the group of 2 is split, and f32
    # dK/dV accumulators are added
    assert _head_split(1, 4, 2, 129) == 2
    assert fa.fa_bwd_workspace_size(1, 4, 2, 129, 64) == 4 * (2 * 4 * 256 + 4 * 129 * 64 + 2 * 2 * 129 * 64)
    # the split rule on a few shapes: MQA at 16k tokens, GQA at 16k (no split)
    assert _head_split(1, 32, 1, 16384) == 8
    assert _head_split(1, 32, 8, 16384) == 1
    # d = 256 counts 64-key tiles: 1 x 4 KV heads x 74 tiles x 2 >= 592 (37 tiles x 4 at d = 128)
    assert _head_split(1, 16, 4, 4736, 256) == 2 and _head_split(1, 16, 4, 4736, 128) == 4
    assert fa.fa_bwd_workspace_size(1, 16, 4, 4736, 256) == 4 * (2 * 16 * 4736 + 16 * 4736 * 256 +
                                                               2 * 4 * 4736 * 256)
    assert fa.fa_bwd_workspace_size(2, 32, 32, 8192, 256) == 4 * (2 * 64 * 8192 + 64 * 8192 * 256)
    for shape in ((1, 32, 1, 16384, 128), (1, 32, 8, 16384, 128), (1, 8, 2, 4096, 128), (3, 6, 3, 700, 64)):
        B, Hq, Hkv, N, d = shape
        kv = 2 * B * Hkv * N * d if _head_split(B, Hq, Hkv, N) > 1 else 0
        want = 4 * (2 * B * Hq * ((N + 127) // 128 * 128) + B * Hq * N * d + kv)
        assert fa.fa_bwd_workspace_size(*shape) == want, shape
    assert fa.fa_bwd_workspace_size(1, 3, 2, 64, 64) == 0  # Hq not a multiple of Hkv
    # linear in N: nothing N x N
    a = fa.fa_bwd_workspace_size(1, 1, 1, 8192, 128)
    b = fa.fa_bwd_workspace_size(1, 1, 1, 16384, 128)
    assert b == 2 * a


def _fwd(lib, **kw):
    args = dict(B=1, Hq=2, Hkv=2, N=64, d=64, scale=0.125, causal=0, dtype=0)
    args.update(kw)
    p = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    return lib.fa_fwd(p, p, p, p, p, args["B"], args["Hq"], args["Hkv"], args["N"], args["d"],
                      args["scale"], args["causal"], args["dtype"], None)


def test_validation_before_any_device_work(lib):
    assert _fwd(lib, N=-1) == fa.FA_ERR_INVALID
    assert _fwd(lib, B=-2) == fa.FA_ERR_INVALID
    assert _fwd(lib, Hq=0) == fa.FA_ERR_INVALID
    assert _fwd(lib, Hq=3, Hkv=2) == fa.FA_ERR_INVALID
    assert _fwd(lib, d=96) == fa.FA_ERR_UNSUPPORTED
    assert _fwd(lib, causal=3) == fa.FA_ERR_INVALID
    assert _fwd(lib, dtype=5) == fa.FA_ERR_INVALID
    assert _fwd(lib, scale=float("inf")) == fa.FA_ERR_INVALID
    assert _fwd(lib, B=0) == fa.FA_OK  # empty problem
    assert _fwd(lib, N=0) == fa.FA_OK
    # null pointers
    assert lib.fa_fwd(None, None, None, None, None, 1, 1, 1, 8, 64, 0.1, 0, 0, None) == fa.FA_ERR_INVALID
    # misaligned pointer
    p, m = ctypes.c_void_p(64), ctypes.c_void_p(66)
    assert lib.fa_fwd(p, p, m, p, p, 1, 1, 1, 8, 64, 0.1, 0, 0, None) == fa.FA_ERR_INVALID
    # backward: f32 is not implemented; short workspace (d = 256 included)
    p = ctypes.c_void_p(64)
    args = [p] * 9
    assert lib.fa_bwd(*args, p, 1 << 30, 1, 1, 1, 8, 64, 0.1, 0, 1, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_bwd(*args, p, 16, 1, 1, 1, 8, 256, 0.1, 0, 0, None) == fa.FA_ERR_WORKSPACE
    assert lib.fa_bwd(*args, p, 16, 1, 1, 1, 8, 64, 0.1, 0, 0, None) == fa.FA_ERR_WORKSPACE
    assert lib.fa_bwd(*args, None, 1 << 30, 1, 1, 1, 8, 64, 0.1, 0, 0, None) == fa.FA_ERR_WORKSPACE
    assert lib.fa_selftest_wait_timeout(0, None) == fa.FA_ERR_INVALID


def _decode_tc_plan(B, Hkv, Nk):
    """Key splits and 128-key tiles per split of the tensor-core KV-cache
    forward (d = 64, 128): the smallest ceil(B*Hkv*S / 148) * (T + 2)."""
    tiles = -(-Nk // 128)
    best = None
    for s in range(1, min(tiles, 128) + 1):
        per = -(-tiles // s)
        used = -(-tiles // per)
        cost = -(-(B * Hkv * used) // 148) * (per + 2)
        if best is None or cost < best[0]:
            best = (cost, used, per)
    return best[1], best[2]


def test_kvcache_workspace_formula(lib):
    for shape in ((1, 32, 8, 1, 32768, 128), (8, 32, 8, 1, 32768, 128), (2, 8, 2, 4, 1000, 64),
                  (64, 16, 16, 1, 4096, 128), (4, 32, 8, 4, 16384, 128), (1, 1, 1, 1, 100, 64),
                  (1, 2, 1, 16, 16, 256), (2, 8, 4, 2, 5000, 256)):
        B, Hq, Hkv, Nq, Nk, d = shape
        S, T = _decode_tc_plan(B, Hkv, Nk)
        assert (S - 1) * T * 128 < Nk <= S * T * 128
        want = 0 if S == 1 else S * B * Hq * Nq * (2 * d + 4)
        assert fa.fa_fwd_kvcache_workspace_size(*shape) == want, shape
    # MQA at 4k keys and batch 64: 2 splits of 16 tiles (128 CTAs, one wave)
    assert _decode_tc_plan(64, 1, 4096) == (2, 16)
    assert fa.fa_fwd_kvcache_workspace_size(1, 2, 1, 9, 8, 64) == 0  # Nq > Nk
    assert fa.fa_fwd_kvcache_workspace_size(1, 3, 2, 1, 64, 64) == 0  # Hq not a multiple of Hkv


def test_kvcache_validation_before_any_device_work(lib):
    def call(B=1, Hq=4, Hkv=2, Nq=1, Nk=100, d=128, scale=0.1, causal=1, dtype=0, ws_bytes=1 << 30):
        p = ctypes.c_void_p(64)
        return lib.fa_fwd_kvcache(p, p, p, p, p, p, ws_bytes, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, None)
    assert call(Nq=101) == fa.FA_ERR_INVALID   # more queries than cached keys
    assert call(Nq=0) == fa.FA_ERR_INVALID
    assert call(Hq=3) == fa.FA_ERR_INVALID
    assert call(causal=2) == fa.FA_ERR_INVALID
    assert call(scale=float("nan")) == fa.FA_ERR_INVALID
    assert call(dtype=1) == fa.FA_ERR_UNSUPPORTED  # fp32
    assert call(d=96) == fa.FA_ERR_UNSUPPORTED
    assert call(Hq=32, Hkv=1, Nq=5) == fa.FA_ERR_UNSUPPORTED  # 160 query rows per KV head > 128
    assert call(Nk=100000, ws_bytes=16) == fa.FA_ERR_WORKSPACE  # several key splits: parts to merge
    assert call(B=0) == fa.FA_OK  # empty problem
    m = ctypes.c_void_p(66)
    p = ctypes.c_void_p(64)
    assert lib.fa_fwd_kvcache(p, m, p, p, p, p, 1 << 30, 1, 4, 2, 1, 100, 128, 0.1, 1, 0, None) == fa.FA_ERR_INVALID


def test_binding_fails_loudly_without_library(tmp_path):
    from exact_io_aware_61_b200 import _lib
    saved = _lib._handle
    _lib._handle = None
    try:
        with pytest.raises(RuntimeError, match="missing"):
            _lib.load(str(tmp_path / "nope.so"))
    finally:
        _lib._handle = saved


def test_varlen_validation_before_any_device_work(lib):
    def call(batch=2, max_q=8, tq=16, tk=16, Hq=4, Hkv=2, d=128, scale=0.1, causal=1, dtype=0, cu=64):
        p = ctypes.c_void_p(64)
        c = ctypes.c_void_p(cu)
        return lib.fa_fwd_varlen(p, p, p, p, p, c, c, batch, max_q, tq, tk, Hq, Hkv, d, scale, causal, dtype, None)
    assert call(batch=-1) == fa.FA_ERR_INVALID
    assert call(max_q=-1) == fa.FA_ERR_INVALID
    assert call(Hq=3) == fa.FA_ERR_INVALID
    assert call(causal=2) == fa.FA_ERR_INVALID
    assert call(scale=float("nan")) == fa.FA_ERR_INVALID
    assert call(d=256) == fa.FA_ERR_UNSUPPORTED
    assert call(dtype=1) == fa.FA_ERR_UNSUPPORTED
    assert call(tk=0) == fa.FA_ERR_INVALID            # queries but no keys
    assert call(max_q=17) == fa.FA_ERR_INVALID        # longer than all the queries
    assert call(cu=66) == fa.FA_ERR_INVALID           # misaligned offsets
    assert call(cu=0) == fa.FA_ERR_INVALID            # no offsets
    assert call(batch=0) == fa.FA_OK and call(tq=0, max_q=0) == fa.FA_OK  # empty


def test_sequence_sharding_calls_validate_before_any_device_work(lib):
    p, m = ctypes.c_void_p(64), ctypes.c_void_p(66)
    # fa_fwd_partial: fp32 and bad sizes
    assert lib.fa_fwd_partial(p, p, p, p, p, 1, 2, 2, 8, 64, 0.1, 1, -1, 1, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_fwd_partial(p, p, p, p, p, 1, 3, 2, 8, 64, 0.1, 1, -1, 0, None) == fa.FA_ERR_INVALID
    assert lib.fa_fwd_partial(p, p, p, p, p, 0, 2, 2, 8, 64, 0.1, 1, -1, 0, None) == fa.FA_OK  # empty
    # fa_merge_partials: sizes, head dimension, overlap of output and input, alignment
    assert lib.fa_merge_partials(p, p, 0, 16, ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 21), 64, 0, None) \
        == fa.FA_ERR_INVALID
    assert lib.fa_merge_partials(p, p, 2, 16, ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 21), 96, 0, None) \
        == fa.FA_ERR_INVALID
    assert lib.fa_merge_partials(ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 22), 2, 16, ctypes.c_void_p(1 << 20),
                                 ctypes.c_void_p(1 << 23), 64, 0, None) == fa.FA_ERR_INVALID   # o is part 0
    assert lib.fa_merge_partials(m, p, 2, 16, ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 21), 64, 0, None) \
        == fa.FA_ERR_INVALID
    assert lib.fa_merge_partials(p, p, 2, 0, p, p, 64, 0, None) == fa.FA_OK  # no rows
    # fa_bwd_partial: d = 256 and fp32 are not implemented; short workspace
    args = [p] * 6
    assert lib.fa_bwd_partial(*args, p, 1 << 30, 1, 2, 2, 8, 256, 0.1, 1, -1, 0, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_bwd_partial(*args, p, 1 << 30, 1, 2, 2, 8, 64, 0.1, 1, -1, 1, None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_bwd_partial(*args, p, 16, 1, 2, 2, 8, 64, 0.1, 1, -1, 0, None) == fa.FA_ERR_WORKSPACE
    # fa_f32_to_bf16: a count that is not a multiple of 4, misaligned pointers
    assert lib.fa_f32_to_bf16(p, p, 6, None) == fa.FA_ERR_INVALID
    assert lib.fa_f32_to_bf16(m, p, 8, None) == fa.FA_ERR_INVALID
    assert lib.fa_f32_to_bf16(p, p, 0, None) == fa.FA_OK
