"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Those callers (a plugin whose host framework owns every device allocation, a
latency-critical loop, a fixed memory budget) get the backward's scratch from
a fixed array in the library's static device memory instead of a workspace
argument.  This test calls the entry point through the C ABI three times in a
row on problems of different size and head dimension (d = 128, 64, and 192 on
the wide-head kernels) -- each call finds the previous call's data, laid out
for another shape, still in the shared array -- and checks every result:

* against fa_bwd with a caller-provided workspace: dK and dV bit for bit (the
  same kernels accumulate them in a fixed order), dQ within one bf16 rounding
  step per element (its fp32 partial sums are added in scheduling order);
* against the fp64 oracle on every head, within the gradient tolerance of the
  other parity tests (relative Frobenius error <= 2e-2).

It also checks the size limit and the order of the argument checks.  The file
is named to be collected last, so a run that stops at the first failure has
run every other test."""

import ctypes

import numpy as np
import pytest
import torch

from exact_io_aware_49_b200 import workloads as wl
from oracle import attention

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


def _one_rounding_step(got, want):
    """|got - want| <= one bf16 step at |want| elementwise, plus 2^-20 of the
    largest |want| for elements that cancel almost to zero (where a different
    order of the fp32 additions moves the result by more than its own step)."""
    g, w = got.double(), want.double()
    step = torch.where(w != 0, torch.exp2(torch.floor(torch.log2(w.abs())) - 7), torch.zeros_like(w))
    return bool(((g - w).abs() <= step + 2.0 ** -20 * w.abs().max()).all())


def test_noalloc_calls_in_a_row_match_fa_bwd_and_the_oracle():
    from exact_io_aware_49_b200 import fa_bwd, fa_fwd, fa_last_device_error
    lib = _lib()
    problems = [wl.Workload("noalloc_a", 1, 4, 1024, 128, True, 0.1, 11),
                wl.Workload("noalloc_b", 2, 3, 768, 64, False, 0.0, 12),
                wl.Workload("noalloc_c", 1, 2, 640, 192, True, 0.1, 13)]
    cases = []
    for w in problems:
        host = wl.draw_inputs(w)
        q, k, v, do = (x.cuda() for x in host)
        o, lse = fa_fwd(q, k, v, w.causal, w.scale, w.p_drop, w.seed)
        cases.append((w, host, q, k, v, do, o, lse))
    results = []
    for w, _, q, k, v, do, o, lse in cases:  # back to back through the same scratch
        st, grads = _noalloc(lib, q, k, v, o, do, lse, w.causal, w.scale, w.p_drop, w.seed)
        assert st == 0, st
        results.append(grads)
    torch.cuda.synchronize()
    assert fa_last_device_error() == 0
    for (w, host, q, k, v, do, o, lse), got in zip(cases, results):
        want = fa_bwd(q, k, v, o, do, lse, w.causal, w.scale, w.p_drop, w.seed)
        torch.cuda.synchronize()
        for g in got:
            assert torch.isfinite(g.float()).all()
        assert _one_rounding_step(got[0], want[0]), f"{w.name}: dQ differs from fa_bwd by more than rounding"
        assert torch.equal(got[1], want[1]), f"{w.name}: dK differs from fa_bwd"
        assert torch.equal(got[2], want[2]), f"{w.name}: dV differs from fa_bwd"
        got_cpu = [g.cpu() for g in got]
        for b in range(w.B):
            for h in range(w.H):
                args = [x[b, h].to(torch.float64).numpy() for x in host]
                ref = attention.backward(*args, causal=w.causal, scale=w.scale, p_drop=w.p_drop, seed=w.seed,
                                         b=b, h=h)
                for name, g, r in zip(("dQ", "dK", "dV"), got_cpu, ref[:3]):
                    rel = float(np.linalg.norm(g[b, h].double().numpy() - r) / np.linalg.norm(r))
                    assert rel <= GRAD_REL_FRO, (w.name, name, (b, h), rel)


def test_noalloc_checks_arguments_before_the_scratch_limit():
    """The same bad arguments get the same status as from fa_bwd, whatever the size."""
    lib = _lib()
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")  # never touched: the checks come first
    p = x.data_ptr()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    big = 1 << 20  # far beyond the scratch limit
    assert lib.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, 1, 1, big, 80, 1, 0.1, 0.0, 0, st) == 2  # unsupported d
    assert lib.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, 1, 1, big, 128, 1, 0.1, 1.0, 0, st) == 1  # p = 1
    assert lib.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, 1, 1, big, 128, 1, -1.0, 0.0, 0, st) == 1  # scale < 0
    assert lib.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, 0, 1, 128, 128, 1, 0.1, 0.0, 0, st) == 1  # B = 0


def _documented_limit_rows_d128():
    """The B*H*N limit at d = 128 that include/fa.h states for fa_bwd_noalloc."""
    import os
    import re
    hdr = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fa.h")
    with open(hdr) as f:
        m = re.search(r"B\*H\*N <= (\d+) rows at d = 128", f.read())
    assert m, "fa.h states the noalloc limit"
    return int(m.group(1))


def test_noalloc_rejects_problems_beyond_the_scratch_limit():
    lib = _lib()
    limit = _documented_limit_rows_d128()
    # the documented limit is the library's: the last row count that fits, then one tile more does not
    assert lib.fa_bwd_workspace_size(1, 1, limit, 128) <= 32 * 1024 * 1024
    B, H, N, d = 1, 1, limit + 128, 128
    assert lib.fa_bwd_workspace_size(B, H, N, d) > 32 * 1024 * 1024
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")  # never touched: the size check comes first
    p = x.data_ptr()
    st = lib.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, B, H, N, d, 1, 0.088, 0.0, 0,
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 2  # FA_ERR_UNSUPPORTED
