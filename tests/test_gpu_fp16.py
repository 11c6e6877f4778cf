"""GPU parity of the fp16 path (fa_fwd_ex / fa_bwd_ex with FA_DTYPE_F16) against
the fp64 oracle, on the same seeded recipe rounded to fp16 instead of bf16.

The oracle does not depend on the input type: it takes the fp16 values,
widened exactly to fp64.  The bounds are the bf16 ones (O max-abs 1e-2 beyond
the output rounding, O rel-Frobenius 5e-3, LSE 1e-3, gradients rel-Frobenius
2e-2); fp16 keeps 11 significant bits against bf16's 8, so the rounding
allowance on O is the fp16 half-ulp.  The bf16 path of the ``_ex`` entry
points must be bit-identical to the plain entry points."""

import ctypes

import pytest
import torch

from exact_io_aware_49_b200 import workloads as wl
from oracle import attention
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

F16_BITS = 11


def _run(q, k, v, do, causal, scale, p, seed):
    from exact_io_aware_49_b200 import fa_bwd, fa_fwd
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = fa_fwd(qd, kd, vd, causal, scale, p, seed)
    dq, dk, dv = fa_bwd(qd, kd, vd, o, dod, lse, causal, scale, p, seed)
    torch.cuda.synchronize()
    assert o.dtype == dq.dtype == dk.dtype == dv.dtype == torch.float16
    return o.cpu(), lse.cpu(), dq.cpu(), dk.cpu(), dv.cpu()


def _check_heads(q, k, v, do, res, heads, causal, scale, p, seed, grads=True):
    o, lse, dq, dk, dv = res
    for b, h in heads:
        args = [x[b, h].to(torch.float64).numpy() for x in (q, k, v, do)]
        kw = dict(causal=causal, scale=scale, p_drop=p, seed=seed, b=b, h=h)
        want_o, want_l = attention.forward(*args[:3], **kw)
        pu.check_o(pu.f64(o[b, h]), want_o, f"O {(b, h)}", bits=F16_BITS)
        pu.check_lse(pu.f64(lse[b, h]), want_l, f"LSE {(b, h)}")
        if grads:
            want_dq, want_dk, want_dv, _ = attention.backward(*args, **kw)
            pu.check_grad(pu.f64(dq[b, h]), want_dq, f"dQ {(b, h)}")
            pu.check_grad(pu.f64(dk[b, h]), want_dk, f"dK {(b, h)}")
            pu.check_grad(pu.f64(dv[b, h]), want_dv, f"dV {(b, h)}")


def test_causal_n1024_all_heads_fp16():
    w = wl.WORKLOADS[1]
    q, k, v, do = wl.draw_inputs(w, dtype=torch.float16)
    res = _run(q, k, v, do, w.causal, w.scale, w.p_drop, w.seed)
    _check_heads(q, k, v, do, res, [(b, h) for b in range(w.B) for h in range(w.H)], w.causal, w.scale,
                 w.p_drop, w.seed)


def test_causal_dropout_n4096_fp16():
    w = wl.WORKLOADS[2]
    q, k, v, do = wl.draw_inputs(w, dtype=torch.float16)
    res = _run(q, k, v, do, w.causal, w.scale, w.p_drop, w.seed)
    for t in res:
        assert torch.isfinite(t.float()).all()
    _check_heads(q, k, v, do, res, [(0, 0), (3, 15)], w.causal, w.scale, w.p_drop, w.seed)


def test_wide_logits_fp16_reduced():
    """The qk_std = 4 recipe (near one-hot rows) at a reduced size, fp16."""
    w = wl.WORKLOADS[3]
    q, k, v, do = wl.draw_inputs(w, B=1, H=2, N=2048, dtype=torch.float16)
    res = _run(q, k, v, do, w.causal, w.scale, w.p_drop, w.seed)
    _check_heads(q, k, v, do, res, [(0, 0), (0, 1)], w.causal, w.scale, w.p_drop, w.seed)


@pytest.mark.parametrize("B,H,N,d,causal,p", [
    (1, 1, 128, 128, True, 0.0),
    (1, 2, 384, 64, False, 0.1),
    (1, 1, 512, 64, True, 0.7),
    (1, 2, 77, 128, True, 0.1),
    (2, 1, 1000, 64, False, 0.0),
    (1, 1, 1, 128, False, 0.0),
])
def test_edge_shapes_fp16(B, H, N, d, causal, p):
    w = wl.Workload("edge", B, H, N, d, causal, p, 91)
    q, k, v, do = wl.draw_inputs(w, dtype=torch.float16)
    res = _run(q, k, v, do, causal, w.scale, p, 4321)
    _check_heads(q, k, v, do, res, [(b, h) for b in range(B) for h in range(H)], causal, w.scale, p, 4321)


def test_ex_entry_points_bf16_match_plain_bitwise():
    from exact_io_aware_49_b200 import binding
    lib = binding.load_library()
    w = wl.Workload("ex", 1, 2, 640, 128, True, 0.1, 17)
    q, k, v, do = (x.cuda() for x in wl.draw_inputs(w))
    B, H, N, d = q.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    o1, l1 = torch.empty_like(q), torch.empty(B, H, N, device="cuda")
    o2, l2 = torch.empty_like(q), torch.empty(B, H, N, device="cuda")
    common = (B, H, N, d, 1, w.scale, w.p_drop, 99)
    assert lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o1.data_ptr(), l1.data_ptr(), *common, stream) == 0
    assert lib.fa_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o2.data_ptr(), l2.data_ptr(), *common, 0,
                         stream) == 0
    ws_bytes = lib.fa_bwd_workspace_size(B, H, N, d)
    ws = torch.empty(ws_bytes, device="cuda", dtype=torch.uint8)
    g1 = [torch.empty_like(q) for _ in range(3)]
    g2 = [torch.empty_like(q) for _ in range(3)]
    ins = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o1.data_ptr(), do.data_ptr(), l1.data_ptr())
    assert lib.fa_bwd(*ins, *(g.data_ptr() for g in g1), *common, ws.data_ptr(), ws_bytes, stream) == 0
    assert lib.fa_bwd_ex(*ins, *(g.data_ptr() for g in g2), *common, 0, ws.data_ptr(), ws_bytes, stream) == 0
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1.view(torch.int32), l2.view(torch.int32))
    for a, b in zip(g1, g2):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_mixed_types_are_rejected_by_the_binding():
    from exact_io_aware_49_b200 import fa_fwd
    q = torch.zeros(1, 1, 128, 64, device="cuda", dtype=torch.float16)
    with pytest.raises(ValueError):
        fa_fwd(q, q.to(torch.bfloat16), q, True)


def test_no_device_wait_timed_out():
    from exact_io_aware_49_b200 import fa_last_device_error
    assert fa_last_device_error() == 0
