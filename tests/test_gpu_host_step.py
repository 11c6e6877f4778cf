"""GPU parity of fa_fwd_bwd_host: the training step on host buffers, cut into
groups of (b, h) units whose copies overlap the kernels on three streams.

The groups run the same kernels as fa_fwd / fa_bwd with the whole problem's
(b, h) in the dropout counters, so O, LSE, dK and dV must equal a device
fa_fwd + fa_bwd of the same inputs bit for bit, and dQ within one bf16
rounding step (its fp32 partial sums are added in scheduling order).  Every
head is also checked against the fp64 oracle."""

import numpy as np
import pytest
import torch

from exact_io_aware_49_b200 import workloads as wl
from oracle import attention
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


def _one_step(x, y):
    xd, yd = x.double(), y.double()
    step = torch.where(yd != 0, torch.exp2(torch.floor(torch.log2(yd.abs())) - 7), torch.zeros_like(yd))
    return bool(((xd - yd).abs() <= step + 2.0 ** -20 * yd.abs().max()).all())


@pytest.mark.parametrize("B,H,N,d,causal,p,groups", [
    (1, 5, 384, 128, True, 0.1, 2),    # groups of 3 and 2 units
    (2, 3, 200, 64, False, 0.3, 4),    # ragged N; 6 units in groups of 2 (4 asked, 3 formed)
    (2, 2, 256, 128, True, 0.0, 1),    # one group: no overlap, same result
    (1, 4, 130, 128, True, 0.1, 4),    # one unit per group
    (1, 9, 256, 128, True, 0.1, 9),    # staging slots reused twice, groups alternating compute streams
])
def test_host_step_matches_device_calls_and_oracle(B, H, N, d, causal, p, groups):
    from exact_io_aware_49_b200 import fa_bwd, fa_fwd, fa_fwd_bwd_host, fa_last_device_error
    w = wl.Workload("host_step", B, H, N, d, causal, p, 21)
    q, k, v, do = (x.pin_memory() for x in wl.draw_inputs(w))
    streams = [torch.cuda.Stream() for _ in range(3)]
    o, lse, dq, dk, dv = fa_fwd_bwd_host(q, k, v, do, causal, w.scale, p, w.seed, groups=groups,
                                          streams=streams)
    streams[2].synchronize()
    torch.cuda.synchronize()
    assert fa_last_device_error() == 0
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    od, lsed = fa_fwd(qd, kd, vd, causal, w.scale, p, w.seed)
    dqd, dkd, dvd = fa_bwd(qd, kd, vd, od, dod, lsed, causal, w.scale, p, w.seed)
    torch.cuda.synchronize()
    assert torch.equal(o, od.cpu()) and torch.equal(lse, lsed.cpu())
    assert torch.equal(dk, dkd.cpu()) and torch.equal(dv, dvd.cpu())
    assert _one_step(dq, dqd.cpu())

    def one(bh):
        b, h = bh
        args = [x[b, h].to(torch.float64).numpy() for x in (q, k, v, do)]
        kw = dict(causal=causal, scale=w.scale, p_drop=p, seed=w.seed, b=b, h=h)
        want_o, want_l = attention.forward(*args[:3], **kw)
        want_dq, want_dk, want_dv, _ = attention.backward(*args, **kw)
        pu.check_o(pu.f64(o[b, h]), want_o, f"O {(b, h)}")
        pu.check_lse(pu.f64(lse[b, h]), want_l, f"LSE {(b, h)}")
        for name, got, want in (("dQ", dq, want_dq), ("dK", dk, want_dk), ("dV", dv, want_dv)):
            pu.check_grad(pu.f64(got[b, h]), want, f"{name} {(b, h)}")

    pu.map_heads(one, [(b, h) for b in range(B) for h in range(H)])


def test_host_step_one_stream_and_calls_in_a_row():
    """The same stream given three times runs the step without overlap (and
    without the call's second compute stream); two calls in a row on the same
    streams and workspace reuse the staging slots: each result still equals
    the device calls bit for bit (dQ within one rounding step)."""
    from exact_io_aware_49_b200 import binding, fa_bwd, fa_fwd, fa_fwd_bwd_host, fa_last_device_error
    w1 = wl.Workload("host_step_a", 1, 6, 256, 128, True, 0.1, 31)
    w2 = wl.Workload("host_step_b", 1, 6, 256, 128, True, 0.1, 32)
    one = torch.cuda.Stream()
    three = [torch.cuda.Stream() for _ in range(3)]
    for streams in ([one, one, one], three):
        ws = torch.empty(binding.fa_fwd_bwd_host_workspace_size(1, 6, 256, 128, 3), dtype=torch.uint8,
                         device="cuda")
        got = []
        for w in (w1, w2):  # back to back, same workspace
            q, k, v, do = (x.pin_memory() for x in wl.draw_inputs(w))
            res = fa_fwd_bwd_host(q, k, v, do, True, w.scale, w.p_drop, w.seed, groups=3, workspace=ws,
                                  streams=streams)
            got.append(((q, k, v, do), res))
        streams[2].synchronize()
        torch.cuda.synchronize()
        assert fa_last_device_error() == 0
        for w, ((q, k, v, do), (o, lse, dq, dk, dv)) in zip((w1, w2), got):
            qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
            od, lsed = fa_fwd(qd, kd, vd, True, w.scale, w.p_drop, w.seed)
            dqd, dkd, dvd = fa_bwd(qd, kd, vd, od, dod, lsed, True, w.scale, w.p_drop, w.seed)
            torch.cuda.synchronize()
            assert torch.equal(o, od.cpu()) and torch.equal(lse, lsed.cpu())
            assert torch.equal(dk, dkd.cpu()) and torch.equal(dv, dvd.cpu())
            assert _one_step(dq, dqd.cpu())
