"""Host-side checks of the Python binding (no GPU): every wrapper is driven with
stand-in CUDA tensors (the attributes the binding reads, no storage) against a
recording copy of the library, which launches nothing.  Checked: the routing to
the C entry points, the argument count and C types of every call against the
prototypes the loaded library declares, the size arguments, and that tensors on
another device, outputs of the wrong shape or type and workspace sizes in bytes
are handled before any call reaches the library."""

import contextlib
import ctypes
import math

import pytest
import torch

bf16, f16, f32, i32, u8 = torch.bfloat16, torch.float16, torch.float32, torch.int32, torch.uint8

# calls that compute sizes on the host; the recorder forwards them to the real library
_HOST_CALLS = {"fa_bwd_workspace_size", "fa_bwd_qk_workspace_size", "fa_bwd_varlen_workspace_size",
               "fa_decode_num_splits", "fa_decode_workspace_size", "fa_fwd_bwd_host_workspace_size"}


class FakeCuda:
    """The parts of a CUDA tensor the binding reads; data_ptr() is a distinct
    4 KB-aligned fake address and is never dereferenced."""
    _addr = 1 << 32

    def __init__(self, shape, dtype, index=0, contiguous=True):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device("cuda", index)
        self.is_cuda = True
        self._contiguous = contiguous
        FakeCuda._addr += 1 << 24
        self._ptr = FakeCuda._addr

    def dim(self):
        return len(self.shape)

    def is_contiguous(self):
        return self._contiguous

    def numel(self):
        return math.prod(self.shape)

    def element_size(self):
        return torch.empty((), dtype=self.dtype).element_size()

    def data_ptr(self):
        return self._ptr


class Recorder:
    def __init__(self, real):
        self.real = real
        self.calls = []

    def __getattr__(self, name):
        fn = getattr(self.real, name)
        if name in _HOST_CALLS:
            return fn

        def call(*args):
            assert len(args) == len(fn.argtypes), (name, len(args), len(fn.argtypes))
            for a, t in zip(args, fn.argtypes):
                if t is ctypes.c_void_p:
                    assert a is None or isinstance(a, (int, ctypes.c_void_p)), (name, a)
                elif isinstance(t, type) and issubclass(t, ctypes._Pointer):
                    assert isinstance(a, ctypes.Array) and a._type_ is t._type_, (name, a)
                else:
                    assert not isinstance(a, ctypes.c_void_p), (name, a)
                    t(a)  # raises TypeError for a value the C type cannot take
            self.calls.append((name, args))
            return 0
        return call


@pytest.fixture
def rec(monkeypatch):
    from exact_io_aware_49_b200 import binding, build
    build.build()
    real = binding.load_library()
    r = Recorder(real)
    monkeypatch.setattr(binding, "load_library", lambda path=None: r)
    monkeypatch.setattr(binding, "_stream", lambda t: ctypes.c_void_p(0))
    monkeypatch.setattr(binding, "_guard", lambda t: contextlib.nullcontext())
    monkeypatch.setattr(binding, "_on_device", lambda d: contextlib.nullcontext())
    return r


def _bhnd(B, H, N, d, dtype=bf16, index=0):
    return FakeCuda((B, H, N, d), dtype, index)


def _fwd_args(B=2, H=3, Nq=300, Nk=300, d=128, dtype=bf16):
    q = _bhnd(B, H, Nq, d, dtype)
    k, v = _bhnd(B, H, Nk, d, dtype), _bhnd(B, H, Nk, d, dtype)
    return q, k, v, _bhnd(B, H, Nq, d, dtype), FakeCuda((B, H, Nq), f32)


@pytest.mark.parametrize("Nq,Nk,dtype,entry", [(300, 300, bf16, "fa_fwd"), (300, 300, f16, "fa_fwd_ex"),
                                               (100, 300, bf16, "fa_fwd_qk"), (300, 100, f16, "fa_fwd_qk")])
def test_fwd_routing_and_arguments(rec, Nq, Nk, dtype, entry):
    from exact_io_aware_49_b200 import binding
    q, k, v, o, lse = _fwd_args(Nq=Nq, Nk=Nk, dtype=dtype)
    binding.fa_fwd(q, k, v, True, 0.125, 0.1, 7, out=o, lse=lse)
    (name, args), = rec.calls
    assert name == entry
    assert args[:5] == (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr())
    sizes = (2, 3, Nq, Nk, 128) if entry == "fa_fwd_qk" else (2, 3, Nq, 128)
    assert args[5:5 + len(sizes)] == sizes


@pytest.mark.parametrize("Nq,Nk,dtype,det,entry", [(256, 256, bf16, False, "fa_bwd"),
                                                   (256, 256, f16, False, "fa_bwd_ex"),
                                                   (256, 256, bf16, True, "fa_bwd_qk"),
                                                   (64, 256, bf16, False, "fa_bwd_qk")])
def test_bwd_routing_and_workspace_bytes(rec, Nq, Nk, dtype, det, entry):
    from exact_io_aware_49_b200 import binding
    q, k, v, o, lse = _fwd_args(Nq=Nq, Nk=Nk, dtype=dtype)
    do, dq = _bhnd(2, 3, Nq, 128, dtype), _bhnd(2, 3, Nq, 128, dtype)
    dk, dv = _bhnd(2, 3, Nk, 128, dtype), _bhnd(2, 3, Nk, 128, dtype)
    need = binding.fa_bwd_workspace_size(2, 3, Nq, 128) if entry == "fa_bwd" else 0
    ws = FakeCuda((1 << 20,), f32)  # 4 MB given as fp32: its size is passed in bytes
    binding.fa_bwd(q, k, v, o, do, lse, True, 0.125, 0.0, 1, workspace=ws, dq=dq, dk=dk, dv=dv, deterministic=det)
    (name, args), = rec.calls
    assert name == entry
    assert args[-3:-1] == (ws.data_ptr(), 4 << 20)
    assert need <= 4 << 20
    assert args[6:9] == (dq.data_ptr(), dk.data_ptr(), dv.data_ptr())
    if entry == "fa_bwd_qk":
        assert args[-4] == int(det)


def test_bwd_stages_calls_the_three_stages(rec):
    from exact_io_aware_49_b200 import binding
    q, k, v, o, lse = _fwd_args(Nq=512, Nk=512)
    do, dq, dk, dv = (_bhnd(2, 3, 512, 128) for _ in range(4))
    ws = FakeCuda((binding.fa_bwd_workspace_size(2, 3, 512, 128),), u8)
    seen = []
    binding.fa_bwd_stages(q, k, v, o, do, lse, True, workspace=ws, dq=dq, dk=dk, dv=dv, between=seen.append)
    assert [c[0] for c in rec.calls] == ["fa_bwd_prepare", "fa_bwd_tiles", "fa_bwd_finish"]
    assert seen == [0, 1, 2, 3]


def test_tensor_on_another_device_is_rejected(rec):
    from exact_io_aware_49_b200 import binding
    base = dict(zip(("q", "k", "v", "o", "lse"), _fwd_args()))
    base["do"], base["dq"], base["dk"], base["dv"] = (_bhnd(2, 3, 300, 128) for _ in range(4))
    for name in ("k", "v", "o", "lse"):
        a = dict(base)
        a[name] = FakeCuda(a[name].shape, a[name].dtype, index=1)
        with pytest.raises(ValueError, match="cuda:1"):
            binding.fa_fwd(a["q"], a["k"], a["v"], True, out=a["o"], lse=a["lse"])
    for name in ("k", "v", "o", "do", "lse", "dq", "dk", "dv"):
        a = dict(base)
        a[name] = FakeCuda(a[name].shape, a[name].dtype, index=1)
        with pytest.raises(ValueError, match="cuda:1"):
            binding.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], True,
                           workspace=FakeCuda((1 << 24,), u8), dq=a["dq"], dk=a["dk"], dv=a["dv"])
    with pytest.raises(ValueError, match="cuda:1"):
        binding.fa_bwd(base["q"], base["k"], base["v"], base["o"], base["do"], base["lse"], True,
                       workspace=FakeCuda((1 << 24,), u8, index=1), dq=base["dq"], dk=base["dk"], dv=base["dv"])
    assert rec.calls == []


@pytest.mark.parametrize("bad", [FakeCuda((2, 3, 299), f32), FakeCuda((2, 3, 300), bf16),
                                 FakeCuda((2, 3, 300), f32, contiguous=False)])
def test_bad_lse_is_rejected(rec, bad):
    from exact_io_aware_49_b200 import binding
    q, k, v, o, _ = _fwd_args()
    with pytest.raises(ValueError, match="lse"):
        binding.fa_fwd(q, k, v, True, out=o, lse=bad)
    with pytest.raises(ValueError, match="lse"):
        binding.fa_bwd(q, k, v, o, _bhnd(2, 3, 300, 128), bad, True, workspace=FakeCuda((1 << 24,), u8),
                       dq=_bhnd(2, 3, 300, 128), dk=_bhnd(2, 3, 300, 128), dv=_bhnd(2, 3, 300, 128))
    assert rec.calls == []


def _packed(lq, lk, H=2, d=64, dtype=bf16):
    tq, tk = sum(lq), sum(lk)
    q, o, do, dq = (FakeCuda((tq, H, d), dtype) for _ in range(4))
    k, v, dk, dv = (FakeCuda((tk, H, d), dtype) for _ in range(4))
    cq, ck = FakeCuda((len(lq) + 1,), i32), FakeCuda((len(lk) + 1,), i32)
    return dict(q=q, k=k, v=v, o=o, do=do, dq=dq, dk=dk, dv=dv, cq=cq, ck=ck, lse=FakeCuda((H, tq), f32))


def test_varlen_calls_and_output_checks(rec):
    from exact_io_aware_49_b200 import binding
    p = _packed([100, 1, 300], [250, 40, 300])
    binding.fa_fwd_varlen(p["q"], p["k"], p["v"], p["cq"], p["ck"], 300, 300, True, out=p["o"], lse=p["lse"])
    ws = FakeCuda((1 << 24,), u8)
    binding.fa_bwd_varlen(p["q"], p["k"], p["v"], p["o"], p["do"], p["lse"], p["cq"], p["ck"], 300, 300, True,
                          workspace=ws, dq=p["dq"], dk=p["dk"], dv=p["dv"], deterministic=True)
    assert [c[0] for c in rec.calls] == ["fa_fwd_varlen", "fa_bwd_varlen"]
    bwd = rec.calls[1][1]
    assert bwd[11:19] == (3, 2, 401, 590, 300, 300, 64, 1)  # B, H, total_q, total_k, max_q, max_k, d, causal
    # outputs of the wrong extent, type or device never reach the library
    for name, bad in (("dq", FakeCuda((400, 2, 64), bf16)), ("dk", FakeCuda((590, 2, 64), f16)),
                      ("dv", FakeCuda((590, 2, 64), bf16, index=1))):
        a = dict(p)
        a[name] = bad
        with pytest.raises(ValueError):
            binding.fa_bwd_varlen(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["cq"], a["ck"], 300, 300,
                                  True, workspace=ws, dq=a["dq"], dk=a["dk"], dv=a["dv"])
    with pytest.raises(ValueError, match="cuda:1"):
        binding.fa_fwd_varlen(p["q"], p["k"], p["v"], FakeCuda((4,), i32, index=1), p["ck"], 300, 300, True,
                              out=p["o"], lse=p["lse"])
    assert len(rec.calls) == 2


def test_decode_calls_and_output_checks(rec):
    from exact_io_aware_49_b200 import binding
    B, H, H_kv, Nq, d, page = 3, 8, 2, 2, 128, 16
    q = _bhnd(B, H, Nq, d)
    kc, vc = FakeCuda((40, page, H_kv, d), bf16), FakeCuda((40, page, H_kv, d), bf16)
    table, lens = FakeCuda((B, 13), i32), FakeCuda((B,), i32)
    o, lse = _bhnd(B, H, Nq, d), FakeCuda((B, H, Nq), f32)
    ws = FakeCuda((1 << 22,), u8)
    binding.fa_decode_paged(q, kc, vc, table, lens, 200, True, num_splits=2, out=o, lse=lse, workspace=ws)
    (name, args), = rec.calls
    assert name == "fa_decode_paged"
    assert args[7:17] == (B, H, H_kv, Nq, d, 40, page, 13, 200, 1)
    assert args[-4:-1] == (0, ws.data_ptr(), 1 << 22)  # dtype bf16, workspace pointer, bytes
    for kw in (dict(out=_bhnd(B, H, Nq, d, f16), lse=lse), dict(out=o, lse=FakeCuda((B, H), f32)),
               dict(out=o, lse=FakeCuda((B, H, Nq), f32, index=1))):
        with pytest.raises(ValueError):
            binding.fa_decode_paged(q, kc, vc, table, lens, 200, True, num_splits=2, workspace=ws, **kw)
    with pytest.raises(ValueError, match="cuda:1"):
        binding.fa_decode_paged(q, FakeCuda((40, page, H_kv, d), bf16, index=1), vc, table, lens, 200, True,
                                num_splits=2, out=o, lse=lse, workspace=ws)
    assert len(rec.calls) == 1


class FakeStream:
    def __init__(self, handle):
        self.cuda_stream = handle


def test_host_step_calls_and_checks(rec):
    from exact_io_aware_49_b200 import binding
    B, H, N, d = 1, 4, 300, 128
    q, k, v, do = (torch.zeros(B, H, N, d, dtype=bf16) for _ in range(4))
    need = binding.fa_fwd_bwd_host_workspace_size(B, H, N, d, 3)
    ws = FakeCuda((need,), u8)
    streams = [FakeStream(s) for s in (11, 22, 33)]
    o, lse, dq, dk, dv = binding.fa_fwd_bwd_host(q, k, v, do, True, None, 0.1, 5, groups=3, device="cuda:0",
                                                 workspace=ws, streams=streams)
    (name, args), = rec.calls
    assert name == "fa_fwd_bwd_host"
    assert args[9:13] == (B, H, N, d) and args[18] == 3 and args[20] == need
    assert [args[21][i] for i in range(3)] == [11, 22, 33]
    assert tuple(o.shape) == (B, H, N, d) and tuple(lse.shape) == (B, H, N) and not o.is_cuda
    with pytest.raises(ValueError):  # device tensors are not host buffers
        binding.fa_fwd_bwd_host(FakeCuda((B, H, N, d), bf16), k, v, do, True, workspace=ws, streams=streams,
                                device="cuda:0")
    with pytest.raises(ValueError):  # too small a workspace is caught before the call
        binding.fa_fwd_bwd_host(q, k, v, do, True, groups=3, device="cuda:0", workspace=FakeCuda((need - 1,), u8),
                                streams=streams)
    with pytest.raises(ValueError):
        binding.fa_fwd_bwd_host(q, k, v, do, True, groups=3, device="cuda:0", workspace=ws, streams=streams[:2])
    assert len(rec.calls) == 1
