"""Guard bands around every output and workspace (GPU).

compute-sanitizer is not available, so out-of-bounds writes are caught the
plain way: each output tensor and each workspace is carved out of a larger
device buffer whose first and last 4 KB hold a byte pattern, and after the
call the pattern must be intact.  The cases cover the layouts whose stores
are clipped by hand: head dimensions 32 and 96 (the kernels compute 64 / 128
columns and store only d), ragged lengths (partial last tiles), Nq != Nk,
packed sequences (rows of a neighbouring sequence) and the paged decode's
split partials.  The inputs are ordinary tensors; only what the library
writes is guarded."""

import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side; keeps the 256-byte alignment of a workspace
PATTERN = 0xA5


def _guarded(shape, dtype):
    nbytes = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
    buf = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
    return buf, buf[GUARD:GUARD + nbytes].view(dtype).view(shape)


def _intact(buf):
    return bool((buf[:GUARD] == PATTERN).all()) and bool((buf[-GUARD:] == PATTERN).all())


def _draw(shape, gen, dtype):
    return torch.randn(shape, generator=gen).to(dtype).cuda()


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal,p,dtype,det", [
    (1, 2, 300, 300, 64, True, 0.1, torch.bfloat16, False),
    (2, 1, 129, 129, 128, False, 0.0, torch.float16, False),
    (1, 2, 200, 333, 128, True, 0.1, torch.bfloat16, True),
    (1, 2, 257, 257, 96, True, 0.1, torch.bfloat16, False),
    (1, 1, 130, 130, 32, True, 0.0, torch.float16, False),
])
def test_fixed_layout_writes_stay_inside(B, H, Nq, Nk, d, causal, p, dtype, det):
    from exact_io_aware_49_b200 import binding
    lib = binding.load_library()
    gen = torch.Generator().manual_seed(Nq + d)
    q, do = _draw((B, H, Nq, d), gen, dtype), _draw((B, H, Nq, d), gen, dtype)
    k, v = _draw((B, H, Nk, d), gen, dtype), _draw((B, H, Nk, d), gen, dtype)
    ws_bytes = int(lib.fa_bwd_qk_workspace_size(B, H, Nq, d, int(det)))
    if Nq == Nk:
        ws_bytes = max(ws_bytes, binding.fa_bwd_workspace_size(B, H, Nq, d))
    bufs = {}
    bufs["o"], o = _guarded((B, H, Nq, d), dtype)
    bufs["lse"], lse = _guarded((B, H, Nq), torch.float32)
    bufs["dq"], dq = _guarded((B, H, Nq, d), dtype)
    bufs["dk"], dk = _guarded((B, H, Nk, d), dtype)
    bufs["dv"], dv = _guarded((B, H, Nk, d), dtype)
    bufs["ws"], ws = _guarded((ws_bytes,), torch.uint8)
    scale = d ** -0.5
    binding.fa_fwd(q, k, v, causal, scale, p, 3, out=o, lse=lse)
    binding.fa_bwd(q, k, v, o, do, lse, causal, scale, p, 3, workspace=ws, dq=dq, dk=dk, dv=dv, deterministic=det)
    torch.cuda.synchronize()
    assert binding.fa_last_device_error() == 0
    for name, buf in bufs.items():
        assert _intact(buf), f"a write left the {name} buffer"
    for t in (o, dq, dk, dv):
        assert bool(torch.isfinite(t.float()).all())


def test_packed_layout_writes_stay_inside():
    from exact_io_aware_49_b200 import binding
    lib = binding.load_library()
    d, H, dtype = 96, 2, torch.bfloat16
    lq, lk = [100, 1, 300], [250, 40, 300]
    gen = torch.Generator().manual_seed(7)
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32).cuda()
    cu_k = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32).cuda()
    tq, tk = sum(lq), sum(lk)
    q, do = _draw((tq, H, d), gen, dtype), _draw((tq, H, d), gen, dtype)
    k, v = _draw((tk, H, d), gen, dtype), _draw((tk, H, d), gen, dtype)
    ws_bytes = int(lib.fa_bwd_varlen_workspace_size(len(lq), H, tq, max(lq), d, 0))
    bufs = {}
    bufs["o"], o = _guarded((tq, H, d), dtype)
    bufs["lse"], lse = _guarded((H, tq), torch.float32)
    bufs["dq"], dq = _guarded((tq, H, d), dtype)
    bufs["dk"], dk = _guarded((tk, H, d), dtype)
    bufs["dv"], dv = _guarded((tk, H, d), dtype)
    bufs["ws"], ws = _guarded((ws_bytes,), torch.uint8)
    binding.fa_fwd_varlen(q, k, v, cu_q, cu_k, max(lq), max(lk), True, d ** -0.5, 0.1, 5, out=o, lse=lse)
    binding.fa_bwd_varlen(q, k, v, o, do, lse, cu_q, cu_k, max(lq), max(lk), True, d ** -0.5, 0.1, 5,
                          workspace=ws, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert binding.fa_last_device_error() == 0
    for name, buf in bufs.items():
        assert _intact(buf), f"a write left the {name} buffer"


def test_decode_writes_stay_inside():
    from exact_io_aware_49_b200 import binding
    lib = binding.load_library()
    d, H, H_kv, Nq, page, splits, dtype = 96, 8, 2, 2, 64, 3, torch.bfloat16
    lens = [700, 33, 2000]
    gen = torch.Generator().manual_seed(11)
    n_pages = [(L + page - 1) // page for L in lens]
    total = sum(n_pages) + 2
    kc, vc = _draw((total, page, H_kv, d), gen, dtype), _draw((total, page, H_kv, d), gen, dtype)
    perm = torch.randperm(total, generator=gen)
    table = torch.zeros(len(lens), max(n_pages), dtype=torch.int32)
    nxt = 0
    for b, n in enumerate(n_pages):
        table[b, :n] = perm[nxt:nxt + n].to(torch.int32)
        nxt += n
    q = _draw((len(lens), H, Nq, d), gen, dtype)
    lens_t = torch.tensor(lens, dtype=torch.int32).cuda()
    ws_bytes = int(lib.fa_decode_workspace_size(len(lens), H, Nq, d, splits))
    bufs = {}
    bufs["o"], o = _guarded((len(lens), H, Nq, d), dtype)
    bufs["lse"], lse = _guarded((len(lens), H, Nq), torch.float32)
    bufs["ws"], ws = _guarded((ws_bytes,), torch.uint8)
    binding.fa_decode_paged(q, kc, vc, table.cuda(), lens_t, max(lens), True, d ** -0.5, num_splits=splits, out=o,
                            lse=lse, workspace=ws)
    torch.cuda.synchronize()
    assert binding.fa_last_device_error() == 0
    for name, buf in bufs.items():
        assert _intact(buf), f"a write left the {name} buffer"
    assert bool(torch.isfinite(o.float()).all())
