"""GPU parity for queries and keys of different lengths (Nq != Nk, causal
alignment bottom-right) and for packed variable-length batches, against the
fp64 oracle, through the C ABI (fa_fwd_qk / fa_bwd_qk, fa_fwd_varlen /
fa_bwd_varlen).

Every sequence of a packed batch is an independent problem: the oracle runs
it on its own, with b = its index in the batch for the dropout draws.  Rows
that see no key must come back as O = 0, LSE = -inf and zero dQ.  A fixed
batch repacked into the variable-length layout must give bit-identical O,
LSE, dK and dV to the fixed-length path (dQ equal up to the order of its
atomic sums)."""

import numpy as np
import pytest
import torch

from oracle import attention
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


def _draw(shape, g, dtype=torch.bfloat16):
    return torch.randn(shape, generator=g, dtype=torch.float32).to(dtype)


def _check_problem(q, k, v, do, o, lse, dq, dk, dv, causal, scale, p, seed, b, h, what):
    """q, do, o, dq: [Nq, d]; k, v, dk, dv: [Nk, d]; lse: [Nq]; all CPU."""
    args = [x.to(torch.float64).numpy() for x in (q, k, v, do)]
    kw = dict(causal=causal, scale=scale, p_drop=p, seed=seed, b=b, h=h)
    want_o, want_l = attention.forward(*args[:3], **kw)
    pu.check_o(pu.f64(o), want_o, f"O {what}")
    pu.check_lse(pu.f64(lse), want_l, f"LSE {what}")
    if dq is not None:
        want_dq, want_dk, want_dv, _ = attention.backward(*args, **kw)
        pu.check_grad(pu.f64(dv), want_dv, f"dV {what}")
        if k.shape[0] == 1:
            _check_single_key_grads(args, pu.f64(o), pu.f64(dq), pu.f64(dk), scale, what)
        else:
            pu.check_grad(pu.f64(dq), want_dq, f"dQ {what}")
            pu.check_grad(pu.f64(dk), want_dk, f"dK {what}")
        empty = np.isneginf(want_l)
        assert np.all(pu.f64(dq)[empty] == 0.0), f"dQ of rows that see no key {what}"


def _check_single_key_grads(args, o, dq, dk, scale, what):
    """One key: P = 1, so dP_i0 = D_i and dS = 0 exactly; dQ = dK = 0.  The
    kernel forms D_i = dO_i . O_i from the stored 16-bit O (the method's
    preprocessing), whose rounding (at most 2^-8 of each |O_ic|) leaves
    |dS_i0| <= 2^-8 sum_c |dO_ic O_ic|.  Checked against that bound, doubled
    for the fp32 sums: |dQ_i| <= scale |dS_i0| |K_0| and |dK_0| <= scale sum_i |dS_i0| |Q_i|."""
    q, k, v, do = args
    ds_bound = 2.0 ** -7 * np.abs(do * o).sum(axis=1)  # per query row
    k_norm = np.linalg.norm(k[0])
    assert np.all(np.linalg.norm(dq, axis=1) <= scale * ds_bound * k_norm + 1e-6), f"dQ (one key) {what}"
    assert np.linalg.norm(dk[0]) <= scale * float((ds_bound * np.linalg.norm(q, axis=1)).sum()) + 1e-6, \
        f"dK (one key) {what}"


# ---------------------------------------------------------------- Nq != Nk, fixed layout

@pytest.mark.parametrize("B,H,Nq,Nk,d,causal,p", [
    (1, 2, 128, 384, 64, True, 0.0),     # more keys: every query sees a prefix longer than itself
    (1, 2, 384, 128, 128, True, 0.1),    # fewer keys: the first 256 query rows see nothing
    (2, 1, 200, 77, 64, True, 0.1),      # ragged both ways, offset not a tile multiple
    (1, 1, 77, 1000, 128, False, 0.0),
    (1, 2, 1000, 2049, 64, True, 0.1),
    (1, 1, 640, 130, 128, True, 0.0),    # whole query tiles with no visible key
    (1, 1, 1, 300, 64, True, 0.0),       # one query: the decode shape
])
def test_rectangular(B, H, Nq, Nk, d, causal, p):
    from exact_io_aware_49_b200 import fa_bwd, fa_fwd
    g = torch.Generator().manual_seed(Nq * 7 + Nk)
    q, do = _draw((B, H, Nq, d), g), _draw((B, H, Nq, d), g)
    k, v = _draw((B, H, Nk, d), g), _draw((B, H, Nk, d), g)
    scale, seed = d ** -0.5, 321
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = fa_fwd(qd, kd, vd, causal, scale, p, seed)
    dq, dk, dv = fa_bwd(qd, kd, vd, o, dod, lse, causal, scale, p, seed)
    torch.cuda.synchronize()
    assert dk.shape == k.shape and dq.shape == q.shape
    o, lse, dq, dk, dv = (x.cpu() for x in (o, lse, dq, dk, dv))
    for b in range(B):
        for h in range(H):
            _check_problem(q[b, h], k[b, h], v[b, h], do[b, h], o[b, h], lse[b, h], dq[b, h], dk[b, h], dv[b, h],
                           causal, scale, p, seed, b, h, f"{(b, h)}")


# ---------------------------------------------------------------- packed variable length

def _pack(lengths, H, d, g, dtype=torch.bfloat16):
    total = int(sum(lengths))
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    return _draw((total, H, d), g, dtype), cu


def _run_varlen(lq, lk, H, d, causal, p, seed, dtype=torch.bfloat16):
    from exact_io_aware_49_b200 import fa_bwd_varlen, fa_fwd_varlen
    g = torch.Generator().manual_seed(sum(lq) * 3 + sum(lk))
    q, cu_q = _pack(lq, H, d, g, dtype)
    do, _ = _pack(lq, H, d, g, dtype)
    k, cu_k = _pack(lk, H, d, g, dtype)
    v, _ = _pack(lk, H, d, g, dtype)
    scale = d ** -0.5
    qd, kd, vd, dod, cqd, ckd = (x.cuda() for x in (q, k, v, do, cu_q, cu_k))
    o, lse = fa_fwd_varlen(qd, kd, vd, cqd, ckd, max(lq), max(lk), causal, scale, p, seed)
    dq, dk, dv = fa_bwd_varlen(qd, kd, vd, o, dod, lse, cqd, ckd, max(lq), max(lk), causal, scale, p, seed)
    torch.cuda.synchronize()
    return (q, k, v, do, cu_q, cu_k), tuple(x.cpu() for x in (o, lse, dq, dk, dv))


def _check_varlen(ins, outs, H, causal, scale, p, seed):
    q, k, v, do, cu_q, cu_k = ins
    o, lse, dq, dk, dv = outs
    for b in range(cu_q.numel() - 1):
        qs, qe = int(cu_q[b]), int(cu_q[b + 1])
        ks, ke = int(cu_k[b]), int(cu_k[b + 1])
        for h in range(H):
            _check_problem(q[qs:qe, h], k[ks:ke, h], v[ks:ke, h], do[qs:qe, h], o[qs:qe, h], lse[h, qs:qe],
                           dq[qs:qe, h], dk[ks:ke, h], dv[ks:ke, h], causal, scale, p, seed, b, h,
                           f"seq {b} head {h}")


@pytest.mark.parametrize("lq,lk,d,causal,p", [
    ([128, 1, 300, 77, 1024], None, 64, True, 0.1),
    ([256, 129, 513], None, 128, True, 0.0),
    ([100, 1, 257, 40], [300, 50, 257, 1], 64, True, 0.1),   # Nq != Nk per sequence, both directions
    ([200, 70], [90, 400], 128, False, 0.1),
])
def test_varlen(lq, lk, d, causal, p):
    lk = lq if lk is None else lk
    H, seed = 2, 77
    ins, outs = _run_varlen(lq, lk, H, d, causal, p, seed)
    _check_varlen(ins, outs, H, causal, d ** -0.5, p, seed)


def test_varlen_fp16():
    lq, lk, H, d = [150, 1, 384], [150, 1, 384], 2, 128
    ins, outs = _run_varlen(lq, lk, H, d, True, 0.1, 5, torch.float16)
    assert outs[0].dtype == torch.float16
    q, k, v, do, cu_q, cu_k = ins
    o, lse = outs[0], outs[1]
    for b in range(3):
        qs, qe = int(cu_q[b]), int(cu_q[b + 1])
        for h in range(H):
            args = [x[qs:qe, h].to(torch.float64).numpy() for x in (q, k, v)]
            want_o, want_l = attention.forward(*args, causal=True, scale=d ** -0.5, p_drop=0.1, seed=5, b=b, h=h)
            pu.check_o(pu.f64(o[qs:qe, h]), want_o, f"O {b} {h}", bits=11)
            pu.check_lse(pu.f64(lse[h, qs:qe]), want_l, f"LSE {b} {h}")


def test_varlen_equals_fixed_bitwise():
    """A fixed [B, H, N, d] batch packed as [B*N, H, d] with equal offsets gives
    the same bits through the variable-length path."""
    from exact_io_aware_49_b200 import fa_bwd, fa_bwd_varlen, fa_fwd, fa_fwd_varlen
    B, H, N, d, p, seed = 3, 2, 333, 128, 0.1, 9
    g = torch.Generator().manual_seed(1)
    q, k, v, do = (_draw((B, H, N, d), g).cuda() for _ in range(4))
    o, lse = fa_fwd(q, k, v, True, d ** -0.5, p, seed)
    dq, dk, dv = fa_bwd(q, k, v, o, do, lse, True, d ** -0.5, p, seed)

    def pack(x):
        return x.permute(0, 2, 1, 3).reshape(B * N, H, d).contiguous()

    cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int32, device="cuda")
    qp, kp, vp, dop = (pack(x) for x in (q, k, v, do))
    o2, lse2 = fa_fwd_varlen(qp, kp, vp, cu, cu, N, N, True, d ** -0.5, p, seed)
    dq2, dk2, dv2 = fa_bwd_varlen(qp, kp, vp, o2, dop, lse2, cu, cu, N, N, True, d ** -0.5, p, seed)
    torch.cuda.synchronize()
    assert torch.equal(pack(o).view(torch.int16), o2.view(torch.int16))
    assert torch.equal(lse.permute(1, 0, 2).reshape(H, B * N).view(torch.int32), lse2.view(torch.int32))
    for a, b2 in ((dk, dk2), (dv, dv2)):
        assert torch.equal(pack(a).view(torch.int16), b2.view(torch.int16))
    # dQ is summed over key tiles by fp32 atomic adds whose order is not fixed:
    # equal up to that summation order
    assert pu.rel_fro(pu.f64(pack(dq)), pu.f64(dq2)) < 1e-3


def test_varlen_binding_rejects_bad_offsets_tensor():
    from exact_io_aware_49_b200 import binding
    x = torch.zeros(64, 1, 64, device="cuda", dtype=torch.bfloat16)
    cu = torch.tensor([0, 64], dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        binding.fa_fwd_varlen(x, x, x, cu.to(torch.int64), cu, 64, 64, True)
    with pytest.raises(ValueError):
        binding.fa_fwd_varlen(x, x, x, cu.cpu(), cu, 64, 64, True)


def test_no_device_wait_timed_out():
    from exact_io_aware_49_b200 import fa_last_device_error
    assert fa_last_device_error() == 0
