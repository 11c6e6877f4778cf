"""Host-side checks of the C ABI (no GPU): the library builds and loads, exports
every entry point include/*.h declares, and rejects bad arguments before it
makes any CUDA call.  Every call here carries at least one invalid argument,
so nothing is ever launched."""

import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from exact_io_aware_49_b200 import build, binding
    build.build()
    return binding.load_library()


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        with open(h) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        for m in re.finditer(r"\b(fa_[a-z0-9_]+)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_entry_points():
    names = _declared_functions()
    for want in ("fa_fwd", "fa_fwd_ex", "fa_bwd", "fa_bwd_ex", "fa_bwd_workspace_size", "fa_bwd_prepare", "fa_bwd_tiles", "fa_bwd_finish",
                 "fa_dropout_mask", "fa_last_device_error", "fa_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, prefix in [(0, b"FA_OK"), (1, b"FA_ERR_INVALID_ARG"), (2, b"FA_ERR_UNSUPPORTED"),
                         (3, b"FA_ERR_CUDA"), (4, b"FA_ERR_TIMEOUT")]:
        assert lib.fa_status_string(code).startswith(prefix)
    assert lib.fa_status_string(99) == b"unknown fa_status"


A = 0x10000  # a 16-byte-aligned fake address; calls below never get past validation


def _fwd(lib, Q=A, K=A, V=A, O=A, L=A, B=1, H=1, N=128, d=64, causal=0, scale=0.125, p=0.0):
    return lib.fa_fwd(Q, K, V, O, L, B, H, N, d, causal, scale, p, 0, None)


@pytest.mark.parametrize("kw,want", [
    (dict(Q=0), 1), (dict(K=0), 1), (dict(V=0), 1), (dict(O=0), 1), (dict(L=0), 1),
    (dict(Q=A + 8), 1), (dict(O=A + 4), 1), (dict(L=A + 4), 1),
    (dict(B=0), 1), (dict(H=-1), 1), (dict(N=0), 1), (dict(d=0), 1),
    (dict(p=1.0), 1), (dict(p=-0.1), 1), (dict(p=float("nan")), 1),
    (dict(scale=0.0), 1), (dict(scale=-1.0), 1), (dict(scale=float("inf")), 1),
    (dict(d=48), 2), (dict(d=80), 2), (dict(d=160), 2), (dict(d=512), 2),
    (dict(B=1 << 16, H=1 << 8, N=1 << 7), 2),
])
def test_fwd_rejects_bad_arguments(lib, kw, want):
    assert _fwd(lib, **kw) == want


@pytest.mark.parametrize("d", [192, 256])
def test_wide_heads_validation(lib, d):
    """d = 192 / 256 pass the forward's and backward's validation (a null
    pointer still stops the call first); the staged backward entry points and
    the paged decode, which have no wide-head kernels, reject them."""
    assert _fwd(lib, d=d, O=0) == 1
    ws = lib.fa_bwd_workspace_size(1, 1, 128, d)
    assert lib.fa_bwd(A, A, A, A, A, A, 0, A, A, 1, 1, 128, d, 1, 0.125, 0.0, 0, A, ws, None) == 1
    assert lib.fa_bwd_tiles(A, A, A, A, A, A, 1, 1, 128, d, 1, 0.125, 0.0, 0, A, ws, None) == 2
    assert lib.fa_bwd_finish(A, 1, 1, 128, d, 0.125, A, ws, None) == 2
    assert lib.fa_decode_paged(A, A, A, A, A, A, A, 1, 8, 2, 1, d, 4, 64, 2, 128, 1, 0.125, 1, 0, A, 1 << 30,
                               None) == 2


def _bwd(lib, ws=A, ws_bytes=None, B=1, H=1, N=128, d=64, p=0.0, **ptrs):
    names = ["Q", "K", "V", "O", "dO", "L", "dQ", "dK", "dV"]
    vals = [ptrs.get(n, A) for n in names]
    if ws_bytes is None:
        ws_bytes = lib.fa_bwd_workspace_size(B, H, N, d)
    return lib.fa_bwd(*vals, B, H, N, d, 1, 0.125, p, 0, ws, ws_bytes, None)


def test_workspace_size_is_linear_in_n(lib):
    s1 = lib.fa_bwd_workspace_size(2, 3, 1024, 128)
    s2 = lib.fa_bwd_workspace_size(2, 3, 2048, 128)
    assert s1 == 2 * 3 * 1024 * 128 * 4 + 2 * (2 * 3 * 1024 * 4)
    assert s2 == 2 * s1
    assert lib.fa_bwd_workspace_size(0, 1, 128, 64) == 0
    # a partial last tile pads the per-row vectors to a multiple of 128 rows
    ragged = lib.fa_bwd_workspace_size(1, 2, 200, 64)
    assert ragged == (2 * 200 * 64 * 4 + 255) // 256 * 256 + 2 * ((2 * 256 * 4 + 255) // 256 * 256)


@pytest.mark.parametrize("kw,want", [
    (dict(ws=0), 1), (dict(ws=A + 16), 1), (dict(dQ=0), 1), (dict(dO=A + 2), 1), (dict(L=0), 1),
    (dict(ws_bytes=1000), 1), (dict(p=1.5), 1), (dict(d=320), 2), (dict(N=64, ws_bytes=100), 1),
])
def test_bwd_rejects_bad_arguments(lib, kw, want):
    assert _bwd(lib, **kw) == want


@pytest.mark.parametrize("dtype", [-1, 2, 7])
def test_ex_entry_points_reject_unknown_dtype(lib, dtype):
    # every other argument is valid: only the element type stops the call
    assert lib.fa_fwd_ex(A, A, A, A, A, 1, 1, 128, 64, 0, 0.125, 0.0, 0, dtype, None) == 1
    ws_ok = lib.fa_bwd_workspace_size(1, 1, 128, 64)
    assert lib.fa_bwd_ex(A, A, A, A, A, A, A, A, A, 1, 1, 128, 64, 1, 0.125, 0.0, 0, dtype, A, ws_ok, None) == 1


@pytest.mark.parametrize("dtype", [0, 1])
def test_ex_entry_points_validate_like_the_plain_ones(lib, dtype):
    ws_ok = lib.fa_bwd_workspace_size(1, 1, 128, 64)
    assert lib.fa_fwd_ex(0, A, A, A, A, 1, 1, 128, 64, 0, 0.125, 0.0, 0, dtype, None) == 1
    assert lib.fa_fwd_ex(A, A, A, A, A, 1, 1, 128, 80, 0, 0.125, 0.0, 0, dtype, None) == 2
    assert lib.fa_fwd_ex(A, A, A, A + 8, A, 1, 1, 128, 64, 0, 0.125, 0.0, 0, dtype, None) == 1
    assert lib.fa_bwd_ex(A, A, A, A, A, A, A, A, A, 1, 1, 128, 64, 1, 0.125, 1.0, 0, dtype, A, ws_ok, None) == 1
    assert lib.fa_bwd_ex(A, A, A, A, A, A, A, A, A, 1, 1, 128, 64, 1, 0.125, 0.0, 0, dtype, A, ws_ok - 4,
                         None) == 1
    assert lib.fa_bwd_ex(A, A, A, A, A, A, A, A, A, 1, 1, 128, 48, 1, 0.125, 0.0, 0, dtype, A, ws_ok, None) == 2


def _varlen_fwd(lib, cu_q=A, cu_k=A, B=1, H=1, tq=64, tk=64, mq=64, mk=64, d=64, scale=0.125, p=0.0, dtype=0):
    return lib.fa_fwd_varlen(A, A, A, A, A, cu_q, cu_k, B, H, tq, tk, mq, mk, d, 1, scale, p, 0, dtype, None)


@pytest.mark.parametrize("kw,want", [
    (dict(cu_q=0), 1), (dict(cu_k=0), 1), (dict(cu_q=A + 2), 1), (dict(B=0), 1), (dict(tq=0), 1),
    (dict(mq=65), 1), (dict(mk=0), 1), (dict(p=1.0), 1), (dict(dtype=3), 1), (dict(d=80), 2),
    (dict(H=1 << 12, tq=1 << 19, tk=1 << 19, mq=1 << 10, mk=1 << 10), 2),
])
def test_varlen_rejects_bad_arguments(lib, kw, want):
    assert _varlen_fwd(lib, **kw) == want


def test_varlen_workspace_size(lib):
    # accumulator H * total_q * d fp32, then two [B, H, pad128(max_q)] fp32 vectors
    assert lib.fa_bwd_varlen_workspace_size(3, 2, 500, 300, 64, 0) == 2 * 500 * 64 * 4 + 2 * (3 * 2 * 384 * 4)
    # deterministic: plus one uint32 counter per (b, h, query tile), rounded to 256 bytes
    assert lib.fa_bwd_varlen_workspace_size(3, 2, 500, 300, 64, 1) == \
        2 * 500 * 64 * 4 + 2 * (3 * 2 * 384 * 4) + 256
    assert lib.fa_bwd_varlen_workspace_size(0, 2, 500, 300, 64, 0) == 0
    ws = lib.fa_bwd_varlen_workspace_size(1, 1, 64, 64, 64, 0)
    assert lib.fa_bwd_varlen(A, A, A, A, A, A, A, A, A, A, A, 1, 1, 64, 64, 64, 64, 64, 1, 0.125, 0.0, 0, 0, 0, A,
                             ws - 4, None) == 1
    # a deterministic call needs the larger workspace
    assert lib.fa_bwd_varlen(A, A, A, A, A, A, A, A, A, A, A, 1, 1, 64, 64, 64, 64, 64, 1, 0.125, 0.0, 0, 0, 1, A,
                             ws, None) == 1


def test_qk_entry_points_validate(lib):
    assert lib.fa_fwd_qk(A, A, A, A, A, 1, 1, 128, 0, 64, 1, 0.125, 0.0, 0, 0, None) == 1
    assert lib.fa_fwd_qk(A, A, A, A, A, 1, 1, 128, 256, 80, 1, 0.125, 0.0, 0, 0, None) == 2
    ws = lib.fa_bwd_qk_workspace_size(1, 1, 128, 64, 0)
    assert ws == lib.fa_bwd_workspace_size(1, 1, 128, 64)
    assert lib.fa_bwd_qk_workspace_size(2, 3, 1000, 64, 1) == lib.fa_bwd_workspace_size(2, 3, 1000, 64) + 256
    assert lib.fa_bwd_qk(A, A, A, A, A, A, A, A, A, 1, 1, 128, 300, 64, 1, 0.125, 0.0, 0, 0, 0, A, ws - 4, None) == 1
    assert lib.fa_bwd_qk(A, A, A, A, A, A, 0, A, A, 1, 1, 128, 300, 64, 1, 0.125, 0.0, 0, 0, 0, A, ws, None) == 1
    assert lib.fa_bwd_qk(A, A, A, A, A, A, A, A, A, 1, 1, 128, 300, 64, 1, 0.125, 0.0, 0, 0, 1, A, ws, None) == 1


def test_stage_entry_points_reject_bad_arguments(lib):
    ws_ok = lib.fa_bwd_workspace_size(1, 1, 128, 64)
    assert lib.fa_bwd_prepare(0, A, A, 1, 1, 128, 64, A, ws_ok, None) == 1
    assert lib.fa_bwd_prepare(A, A, A, 1, 1, 128, 64, A, ws_ok - 4, None) == 1
    assert lib.fa_bwd_prepare(A, A, A, 1, 1, 128, 48, A, ws_ok, None) == 2
    assert lib.fa_bwd_tiles(A, A, A, A, A, 0, 1, 1, 128, 64, 1, 0.125, 0.0, 0, A, ws_ok, None) == 1
    assert lib.fa_bwd_tiles(A, A, A, A, A, A, 1, 1, 128, 64, 1, 0.125, 1.0, 0, A, ws_ok, None) == 1
    assert lib.fa_bwd_tiles(A, A, A, A, A, A, 1, 1, 128, 80, 1, 0.125, 0.0, 0, A, ws_ok, None) == 2
    assert lib.fa_bwd_finish(A + 8, 1, 1, 128, 64, 0.125, A, ws_ok, None) == 1
    assert lib.fa_bwd_finish(A, 1, 1, 128, 64, 0.125, A + 64, ws_ok, None) == 1
    assert lib.fa_bwd_finish(A, 1, 1, 128, 64, -1.0, A, ws_ok, None) == 1


def test_selftest_rejects_bad_limits_before_any_cuda_call(lib):
    assert lib.fa_selftest_wait_timeout(0, None) == 1
    assert lib.fa_selftest_wait_timeout(1000001, None) == 1


def test_mask_rejects_bad_arguments(lib):
    assert lib.fa_dropout_mask(None, 1, 1, 8, 0.1, 0, None) == 1
    assert lib.fa_dropout_mask(A, 0, 1, 8, 0.1, 0, None) == 1
    assert lib.fa_dropout_mask(A, 1, 1, 8, 1.0, 0, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from exact_io_aware_49_b200 import binding
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(ImportError):
        binding.load_library(str(tmp_path / "missing.so"))


def _decode(lib, Q=A, BT=A, SL=A, B=2, H=8, H_kv=2, Nq=1, d=128, pages=64, page=16, maxp=8, maxk=100, scale=0.1,
            splits=1, dtype=0, ws=0, ws_bytes=0):
    return lib.fa_decode_paged(Q, A, A, BT, SL, A, A, B, H, H_kv, Nq, d, pages, page, maxp, maxk, 1, scale, splits,
                               dtype, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,want", [
    (dict(Q=0), 1), (dict(BT=0), 1), (dict(SL=A + 2), 1), (dict(H=6, H_kv=4), 1), (dict(maxk=129), 1),
    (dict(scale=0.0), 1), (dict(dtype=5), 1), (dict(splits=-1), 1), (dict(splits=3), 1),  # no workspace
    (dict(page=8, maxp=16), 2), (dict(page=48), 2), (dict(d=80), 2), (dict(Nq=0), 1),
])
def test_decode_rejects_bad_arguments(lib, kw, want):
    assert _decode(lib, **kw) == want


def test_decode_split_choice_and_workspace(lib):
    # one split when there are already enough (sequence, head) blocks; more for few long sequences
    assert lib.fa_decode_num_splits(64, 8, 32, 1, 4096) == 1
    s = lib.fa_decode_num_splits(1, 8, 32, 1, 32768)
    assert 2 <= s <= 128
    assert lib.fa_decode_num_splits(1, 1, 1, 1, 100) == 1  # a single 128-key tile cannot be split
    assert lib.fa_decode_num_splits(1, 3, 4, 1, 100) == 0  # H not a multiple of H_kv
    assert lib.fa_decode_workspace_size(2, 8, 1, 128, 1) == 0
    # every split holds at least one 128-position tile, whatever the shape
    for B, H_kv, H, Nq, L in [(16, 8, 32, 1, 32768), (1, 8, 32, 1, 131072), (4, 8, 32, 4, 32768),
                              (3, 2, 8, 1, 1000), (1, 1, 1, 1, 129), (2, 1, 64, 16, 70000), (500, 8, 8, 1, 300)]:
        tiles = (L + 127) // 128
        s = lib.fa_decode_num_splits(B, H_kv, H, Nq, L)
        assert 1 <= s <= min(tiles, 128)
        per = (tiles + s - 1) // s
        assert (tiles + per - 1) // per == s, (B, H_kv, H, Nq, L, s)
    assert lib.fa_decode_workspace_size(2, 8, 1, 128, 4) == 2 * 8 * 4 * 128 * 4 + 256


@pytest.mark.parametrize("d", [32, 80, 128, 192, 256, 320])
def test_noalloc_takes_the_head_dims_fa_bwd_takes(lib, d):
    """With null pointers both backward entry points return the same status
    for every head dim: FA_ERR_INVALID_ARG where d is supported (the wide
    heads included), FA_ERR_UNSUPPORTED where it is not; both before any
    CUDA call."""
    vp, i, fl, u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_uint64
    f = lib.fa_bwd_noalloc
    f.argtypes = [vp] * 9 + [i, i, i, i, i, fl, fl, u64, vp]
    f.restype = i
    got = f(*([None] * 9), 1, 1, 256, d, 1, 0.1, 0.0, 0, None)
    want = lib.fa_bwd(*([None] * 9), 1, 1, 256, d, 1, 0.1, 0.0, 0, None, 0, None)
    assert got == want == (1 if d in (32, 128, 192, 256) else 2)
