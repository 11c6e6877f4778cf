"""GPU parity for head dimensions 32 and 96, which run on the 64- and
128-column kernels with the tensor maps reading the columns past d as zeros
and only d columns stored: forward, backward (default and deterministic),
packed variable length and paged decode, against the fp64 oracle."""

import numpy as np
import pytest
import torch

from oracle import attention, paged
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


def _draw(shape, gen, dtype=torch.bfloat16):
    return torch.randn(shape, generator=gen).to(dtype)


@pytest.mark.parametrize("d", [32, 96])
@pytest.mark.parametrize("B,H,N,causal,p,det,dtype", [
    (1, 2, 1000, True, 0.1, False, torch.bfloat16),
    (2, 1, 256, False, 0.0, False, torch.bfloat16),
    (1, 2, 333, True, 0.0, True, torch.bfloat16),
    (1, 1, 700, True, 0.1, False, torch.float16),
])
def test_fixed_layout(d, B, H, N, causal, p, det, dtype):
    from exact_io_aware_49_b200 import fa_bwd, fa_fwd
    gen = torch.Generator().manual_seed(d * 100 + N)
    q, k, v, do = (_draw((B, H, N, d), gen, dtype) for _ in range(4))
    scale, seed = d ** -0.5, 11
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = fa_fwd(qd, kd, vd, causal, scale, p, seed)
    dq, dk, dv = fa_bwd(qd, kd, vd, o, dod, lse, causal, scale, p, seed, deterministic=det)
    torch.cuda.synchronize()
    bits = 11 if dtype == torch.float16 else 8
    for b in range(B):
        for h in range(H):
            args = [x[b, h].to(torch.float64).numpy() for x in (q, k, v, do)]
            kw = dict(causal=causal, scale=scale, p_drop=p, seed=seed, b=b, h=h)
            want_o, want_l = attention.forward(*args[:3], **kw)
            want = attention.backward(*args, **kw)[:3]
            pu.check_o(pu.f64(o[b, h].cpu()), want_o, f"O {(b, h)}", bits=bits)
            pu.check_lse(pu.f64(lse[b, h].cpu()), want_l, f"LSE {(b, h)}")
            for got, w, name in zip((dq, dk, dv), want, ("dQ", "dK", "dV")):
                pu.check_grad(pu.f64(got[b, h].cpu()), w, f"{name} {(b, h)}")


@pytest.mark.parametrize("d", [32, 96])
def test_varlen(d):
    from exact_io_aware_49_b200 import fa_bwd_varlen, fa_fwd_varlen
    gen = torch.Generator().manual_seed(d)
    lq, lk, H = [100, 1, 300], [250, 40, 300], 2
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32)
    cu_k = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32)
    q, do = (_draw((sum(lq), H, d), gen) for _ in range(2))
    k, v = (_draw((sum(lk), H, d), gen) for _ in range(2))
    qd, kd, vd, dod, cq, ck = (x.cuda() for x in (q, k, v, do, cu_q, cu_k))
    o, lse = fa_fwd_varlen(qd, kd, vd, cq, ck, max(lq), max(lk), True, d ** -0.5, 0.1, 5)
    dq, dk, dv = fa_bwd_varlen(qd, kd, vd, o, dod, lse, cq, ck, max(lq), max(lk), True, d ** -0.5, 0.1, 5)
    torch.cuda.synchronize()
    o, lse, dq, dk, dv = (x.cpu() for x in (o, lse, dq, dk, dv))
    for b in (0, 2):  # sequence 1 has one query row
        qs, qe, ks, ke = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        for h in range(H):
            args = [x.to(torch.float64).numpy() for x in (q[qs:qe, h], k[ks:ke, h], v[ks:ke, h], do[qs:qe, h])]
            kw = dict(causal=True, scale=d ** -0.5, p_drop=0.1, seed=5, b=b, h=h)
            want_o, want_l = attention.forward(*args[:3], **kw)
            pu.check_o(pu.f64(o[qs:qe, h]), want_o, f"O seq {b}")
            pu.check_lse(pu.f64(lse[h, qs:qe]), want_l, f"LSE seq {b}")
            want = attention.backward(*args, **kw)[:3]
            for got, w, name in zip((dq[qs:qe, h], dk[ks:ke, h], dv[ks:ke, h]), want, ("dQ", "dK", "dV")):
                pu.check_grad(pu.f64(got), w, f"{name} seq {b}")


@pytest.mark.parametrize("d,page", [(32, 16), (96, 64)])
def test_decode(d, page):
    from exact_io_aware_49_b200 import fa_decode_paged
    gen = torch.Generator().manual_seed(d + page)
    lens, H, H_kv, Nq = [700, 33, 2000], 8, 2, 2
    n_pages = [(L + page - 1) // page for L in lens]
    total = sum(n_pages) + 3
    kc, vc = (_draw((total, page, H_kv, d), gen) for _ in range(2))
    perm = torch.randperm(total, generator=gen)
    table = torch.zeros(len(lens), max(n_pages), dtype=torch.int32)
    nxt = 0
    for b, n in enumerate(n_pages):
        table[b, :n] = perm[nxt:nxt + n].to(torch.int32)
        nxt += n
    q = _draw((len(lens), H, Nq, d), gen)
    lens_t = torch.tensor(lens, dtype=torch.int32)
    o, lse = fa_decode_paged(q.cuda(), kc.cuda(), vc.cuda(), table.cuda(), lens_t.cuda(), max(lens), True,
                             d ** -0.5)
    torch.cuda.synchronize()
    want_o, want_l = paged.decode_forward(q.to(torch.float64).numpy(), kc.to(torch.float64).numpy(),
                                          vc.to(torch.float64).numpy(), table.numpy(), lens_t.numpy(), causal=True,
                                          scale=d ** -0.5)
    for b in range(len(lens)):
        for h in range(H):
            pu.check_o(pu.f64(o[b, h].cpu()), want_o[b, h], f"O {(b, h)}")
            pu.check_lse(pu.f64(lse[b, h].cpu()), want_l[b, h], f"LSE {(b, h)}")


def test_no_device_wait_timed_out():
    from exact_io_aware_49_b200 import fa_last_device_error
    assert fa_last_device_error() == 0
