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


# ---------------------------------------------------------------- head dimensions 192 and 256

@pytest.mark.parametrize("d", [192, 256])
@pytest.mark.parametrize("B,H,Nq,Nk,causal,p,dtype", [
    (1, 2, 1000, 1000, True, 0.1, torch.bfloat16),    # ragged N, several 64-key tiles, dropout
    (2, 1, 256, 256, False, 0.0, torch.bfloat16),
    (1, 2, 333, 333, True, 0.0, torch.float16),
    (1, 1, 130, 130, False, 0.7, torch.bfloat16),     # threshold above 0x8000
    (1, 1, 1, 1, True, 0.0, torch.bfloat16),          # a single row and key
    (1, 2, 300, 1000, True, 0.1, torch.bfloat16),     # Nq < Nk: bottom-right causal alignment
    (1, 1, 1000, 300, True, 0.0, torch.bfloat16),     # Nq > Nk: leading rows see no key
])
def test_wide_forward(d, B, H, Nq, Nk, causal, p, dtype):
    """The wide-head forward kernel (one 128-row query tile per CTA, 64-key
    tiles, S double-buffered in tensor memory) against the oracle."""
    from exact_io_aware_49_b200 import fa_fwd, fa_last_device_error
    gen = torch.Generator().manual_seed(d * 10 + Nq + Nk)
    q = _draw((B, H, Nq, d), gen, dtype)
    k, v = (_draw((B, H, Nk, d), gen, dtype) for _ in range(2))
    scale, seed = d ** -0.5, 13
    o, lse = fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal, scale, p, seed)
    torch.cuda.synchronize()
    assert fa_last_device_error() == 0
    bits = 11 if dtype == torch.float16 else 8
    for b in range(B):
        for h in range(H):
            args = [x[b, h].to(torch.float64).numpy() for x in (q, k, v)]
            want_o, want_l = attention.forward(*args, causal=causal, scale=scale, p_drop=p, seed=seed, b=b, h=h)
            pu.check_o(pu.f64(o[b, h].cpu()), want_o, f"O {(b, h)}", bits=bits)
            pu.check_lse(pu.f64(lse[b, h].cpu()), want_l, f"LSE {(b, h)}")


@pytest.mark.parametrize("d", [192, 256])
def test_wide_forward_mask_and_guard_bands(d):
    """Q = 0 and V[j] = e_(j - w0) on a window of keys: O[i, c] != 0 exactly
    where key w0 + c is kept for row i (bit-exact dropout mask through the wide
    kernel), and the canary bands around O and LSE stay untouched."""
    from exact_io_aware_49_b200 import binding
    from oracle import philox
    B, H, N, p, seed = 1, 2, 700, 0.1, 3
    gen = torch.Generator().manual_seed(d)
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
    k = _draw((B, H, N, d), gen)
    v = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
    w0 = 0 if d == 192 else 500
    n_c = min(d, N - w0)
    v[:, :, w0:w0 + n_c, :n_c] = torch.eye(n_c, dtype=torch.bfloat16)
    band = 4096
    o_buf = torch.full((2 * band + B * H * N * d,), 12345, dtype=torch.int16, device="cuda")
    l_buf = torch.full((2 * band + B * H * N,), -7.0, dtype=torch.float32, device="cuda")
    o = o_buf[band:band + B * H * N * d].view(torch.bfloat16).view(B, H, N, d)
    lse = l_buf[band:band + B * H * N].view(B, H, N)
    binding.fa_fwd(q.cuda(), k.cuda(), v.cuda(), True, d ** -0.5, p, seed, out=o, lse=lse)
    torch.cuda.synchronize()
    assert bool((o_buf[:band] == 12345).all()) and bool((o_buf[-band:] == 12345).all())
    assert bool((l_buf[:band] == -7.0).all()) and bool((l_buf[-band:] == -7.0).all())
    got = (o[..., :n_c] != 0).cpu().numpy()
    rows, cols = np.arange(N), np.arange(w0, w0 + n_c)
    for h in range(H):
        want = philox.keep_mask(seed, 0, h, rows, cols, p)
        valid = cols[None, :] <= rows[:, None]
        np.testing.assert_array_equal(got[0, h][valid], want[valid])
        assert not got[0, h][~valid].any()


@pytest.mark.parametrize("d", [192, 256])
@pytest.mark.parametrize("B,H,Nq,Nk,causal,p,det,dtype", [
    (1, 2, 1000, 1000, True, 0.1, False, torch.bfloat16),  # ragged N, dropout
    (2, 1, 256, 256, False, 0.0, False, torch.bfloat16),
    (1, 1, 333, 333, True, 0.7, False, torch.float16),     # threshold above 0x8000
    (1, 2, 200, 700, True, 0.1, True, torch.bfloat16),     # Nq < Nk (deterministic is the only dQ order here)
    (1, 1, 700, 200, True, 0.0, False, torch.bfloat16),    # Nq > Nk: leading rows see no key
    (1, 2, 384, 384, False, 0.1, False, torch.bfloat16),   # non-causal with dropout
])
def test_wide_backward(d, B, H, Nq, Nk, causal, p, det, dtype):
    """The wide-head backward (a dK / dV kernel over 64-query tiles and a dQ
    kernel over 64-key tiles) against the oracle; dQ is written by one CTA per
    row, so two calls agree bit for bit."""
    from exact_io_aware_49_b200 import fa_bwd, fa_fwd, fa_last_device_error
    gen = torch.Generator().manual_seed(d + 7 * Nq + Nk)
    q, do = (_draw((B, H, Nq, d), gen, dtype) for _ in range(2))
    k, v = (_draw((B, H, Nk, d), gen, dtype) for _ in range(2))
    scale, seed = d ** -0.5, 17
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = fa_fwd(qd, kd, vd, causal, scale, p, seed)
    dq, dk, dv = fa_bwd(qd, kd, vd, o, dod, lse, causal, scale, p, seed, deterministic=det)
    dq2, dk2, dv2 = fa_bwd(qd, kd, vd, o, dod, lse, causal, scale, p, seed, deterministic=det)
    torch.cuda.synchronize()
    assert fa_last_device_error() == 0
    assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2)
    bits = 11 if dtype == torch.float16 else 8

    def one(bh):
        b, h = bh
        args = [x[b, h].to(torch.float64).numpy() for x in (q, k, v, do)]
        kw = dict(causal=causal, scale=scale, p_drop=p, seed=seed, b=b, h=h)
        want_o, want_l = attention.forward(*args[:3], **kw)
        pu.check_o(pu.f64(o[b, h].cpu()), want_o, f"O {(b, h)}", bits=bits)
        pu.check_lse(pu.f64(lse[b, h].cpu()), want_l, f"LSE {(b, h)}")
        want = attention.backward(*args, **kw)[:3]
        for got, w, name in zip((dq, dk, dv), want, ("dQ", "dK", "dV")):
            pu.check_grad(pu.f64(got[b, h].cpu()), w, f"{name} {(b, h)}")

    pu.map_heads(one, [(b, h) for b in range(B) for h in range(H)])


@pytest.mark.parametrize("d", [192, 256])
def test_wide_backward_mask_probe(d):
    """Bit-exact dropout mask through the wide dK / dV kernel: Q = 0 and dO
    rows one-hot over a window of d queries make dV[j, c] non-zero exactly
    where key j is kept for query w0 + c."""
    from exact_io_aware_49_b200 import fa_bwd, fa_fwd
    from oracle import philox
    B, H, N, p, seed = 1, 2, 500, 0.1, 23
    gen = torch.Generator().manual_seed(d + 1)
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    k, v = (_draw((B, H, N, d), gen).cuda() for _ in range(2))
    o, lse = fa_fwd(q, k, v, True, d ** -0.5, p, seed)
    cols = np.arange(N)
    for w0 in (0, N - min(d, N)):
        n_c = min(d, N - w0)
        do = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device="cuda")
        idx = torch.arange(n_c, device="cuda")
        do[:, :, w0 + idx, idx] = 1.0
        _, _, dv = fa_bwd(q, k, v, o, do, lse, True, d ** -0.5, p, seed)
        got = (dv[0, :, :, :n_c] != 0).cpu().numpy()
        rows = np.arange(w0, w0 + n_c)
        for h in range(H):
            want = philox.keep_mask(seed, 0, h, rows, cols, p).T
            valid = cols[:, None] <= rows[None, :]
            np.testing.assert_array_equal(got[h][valid], want[valid])
            assert not got[h][~valid].any()
