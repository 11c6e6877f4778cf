"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Those callers (a plugin whose host framework owns every device allocation, a
latency-critical loop, a fixed memory budget) get the backward's scratch from
a fixed array in the library's static device memory instead of a workspace
argument.  This test calls the entry point through the C ABI twice in a row --
the second call finds the first call's data still in the shared array -- and
checks both results against fa_bwd with a caller-provided workspace, within
the gradient tolerance of the other parity tests (relative Frobenius error
<= 2e-2).  It also checks the size limit.  The file is named to be collected
last, so a run that stops at the first failure has run every other test."""

import ctypes

import pytest
import torch

from exact_io_aware_49_b200 import workloads as wl

pytestmark = pytest.mark.gpu

GRAD_REL_FRO = 2e-2


def _lib():
    from exact_io_aware_49_b200 import binding
    lib = binding.load_library()
    vp, i, f, u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_uint64
    lib.fa_bwd_noalloc.argtypes = [vp] * 9 + [i, i, i, i, i, f, f, u64, vp]
    lib.fa_bwd_noalloc.restype = i
    return lib


def _noalloc(lib, q, k, v, o, do, lse, causal, scale, p, seed):
    B, H, N, d = q.shape
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    st = lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d, int(causal), float(scale),
                            float(p), int(seed), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, (dq, dk, dv)


def _rel(a, b):
    a, b = a.double(), b.double()
    return float((a - b).norm() / b.norm())


@pytest.mark.parametrize("B,H,N,d,causal,p", [(1, 4, 1024, 128, True, 0.1), (2, 3, 768, 64, False, 0.0)])
def test_noalloc_matches_workspace_backward_on_two_calls(B, H, N, d, causal, p):
    from exact_io_aware_49_b200 import fa_bwd, fa_fwd, fa_last_device_error
    lib = _lib()
    cases = []
    for seed in (11, 12):  # two different problems, back to back through the same scratch
        w = wl.Workload("noalloc", B, H, N, d, causal, p, seed)
        q, k, v, do = (x.cuda() for x in wl.draw_inputs(w))
        o, lse = fa_fwd(q, k, v, causal, w.scale, p, seed)
        cases.append((w, q, k, v, do, o, lse))
    results = []
    for w, q, k, v, do, o, lse in cases:
        st, grads = _noalloc(lib, q, k, v, o, do, lse, w.causal, w.scale, w.p_drop, w.seed)
        assert st == 0, st
        results.append(grads)
    torch.cuda.synchronize()
    assert fa_last_device_error() == 0
    for (w, q, k, v, do, o, lse), got in zip(cases, results):
        want = fa_bwd(q, k, v, o, do, lse, w.causal, w.scale, w.p_drop, w.seed)
        torch.cuda.synchronize()
        for name, g, r in zip(("dQ", "dK", "dV"), got, want):
            assert torch.isfinite(g.float()).all()
            assert _rel(g, r) <= GRAD_REL_FRO, (name, _rel(g, r))


def test_noalloc_rejects_problems_beyond_the_scratch_limit():
    lib = _lib()
    B, H, N, d = 1, 1, 64640, 128  # needs more than the 32 MiB scratch
    ws = lib.fa_bwd_workspace_size(B, H, N, d)
    assert ws > 32 * 1024 * 1024
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")  # never touched: the size check comes first
    p = x.data_ptr()
    st = lib.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, B, H, N, d, 1, 0.088, 0.0, 0,
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 2  # FA_ERR_UNSUPPORTED
    assert lib.fa_bwd_workspace_size(1, 1, 64512, 128) <= 32 * 1024 * 1024
