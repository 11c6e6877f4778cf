"""GPU parity of fa_decode_paged (attention over a paged key/value cache)
against the fp64 oracle (``oracle.paged.decode_forward``), through the C ABI.

Pages are scattered in shuffled order over a cache that also holds unused
pages; the positions of a sequence's last page past its length hold NaN, which
must not reach the output.  Tolerances are the forward ones: O max-abs <= 1e-2
beyond the 16-bit output rounding and rel-Frobenius <= 5e-3, LSE within 1e-3
(and -inf exactly for rows that see no position)."""

import numpy as np
import pytest
import torch

from oracle import attention, paged
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


def _make_cache(lens, page, H_kv, d, gen, dtype, extra_pages=5):
    """(k_cache, v_cache, block_table) with every sequence's pages scattered."""
    B = len(lens)
    max_pages = max(1, max((L + page - 1) // page for L in lens))
    total = sum((L + page - 1) // page for L in lens) + extra_pages
    perm = torch.randperm(total, generator=gen)
    k = torch.randn(total, page, H_kv, d, generator=gen).to(dtype)
    v = torch.randn(total, page, H_kv, d, generator=gen).to(dtype)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)  # unused entries are never read
    nxt = 0
    for b, L in enumerate(lens):
        n = (L + page - 1) // page
        for j in range(n):
            table[b, j] = int(perm[nxt])
            nxt += 1
        if L % page:
            last = int(table[b, n - 1])
            k[last, L % page:] = float("nan")
            v[last, L % page:] = float("nan")
    return k, v, table


def _run(B_lens, H, H_kv, Nq, d, page, causal, splits, dtype=torch.bfloat16, seed=0):
    from exact_io_aware_49_b200 import fa_decode_paged
    gen = torch.Generator().manual_seed(seed + 7 * len(B_lens) + page)
    B = len(B_lens)
    q = torch.randn(B, H, Nq, d, generator=gen).to(dtype)
    kc, vc, table = _make_cache(B_lens, page, H_kv, d, gen, dtype)
    lens = torch.tensor(B_lens, dtype=torch.int32)
    o, lse = fa_decode_paged(q.cuda(), kc.cuda(), vc.cuda(), table.cuda(), lens.cuda(), max(B_lens), causal,
                             d ** -0.5, num_splits=splits)
    torch.cuda.synchronize()
    return q, kc, vc, table, lens, o.cpu(), lse.cpu()


def _check(q, kc, vc, table, lens, o, lse, causal, bits=8):
    d = q.shape[-1]
    want_o, want_l = paged.decode_forward(q.to(torch.float64).numpy(), kc.to(torch.float64).numpy(),
                                          vc.to(torch.float64).numpy(), table.numpy(), lens.numpy(),
                                          causal=causal, scale=d ** -0.5)
    got_o = pu.f64(o)
    assert np.isfinite(got_o).all()
    B, H = q.shape[:2]
    for b in range(B):
        for h in range(H):
            pu.check_o(got_o[b, h], want_o[b, h], f"O {(b, h)}", bits=bits)
            pu.check_lse(pu.f64(lse[b, h]), want_l[b, h], f"LSE {(b, h)}")


@pytest.mark.parametrize("lens,H,H_kv,Nq,d,page,causal,splits", [
    ([1, 100, 1000], 8, 2, 1, 128, 16, True, 0),      # GQA group 4, one decode query
    ([3, 257, 700], 4, 4, 4, 64, 64, True, 0),        # multi-token decode; first sequence: rows that see nothing
    ([5000], 32, 1, 1, 128, 128, True, 0),            # group 32: two 16-row blocks per key/value head
    ([777, 2048], 8, 8, 2, 128, 32, False, 3),        # explicit split count
    ([4096] * 4, 16, 4, 1, 128, 64, True, 1),         # one split: final output written directly
    ([130, 129, 128, 127], 6, 3, 3, 64, 16, True, 0),  # lengths around the 128-key tile
])
def test_decode_matches_oracle(lens, H, H_kv, Nq, d, page, causal, splits):
    _check(*_run(lens, H, H_kv, Nq, d, page, causal, splits), causal)


def test_split_counts_agree():
    """Every split count is the same exact result up to rounding: P is rounded
    to 16 bits against each split's own running maximum, so the outputs may
    differ by the O bound (rel-Frobenius 5e-3); the fp32 LSE much less."""
    outs = []
    for splits in (1, 2, 5, 0):
        q, kc, vc, table, lens, o, lse = _run([3000, 1500], 8, 2, 1, 128, 16, True, splits, seed=3)
        _check(q, kc, vc, table, lens, o, lse, True)
        outs.append((o, lse))
    for o, lse in outs[1:]:
        assert pu.rel_fro(pu.f64(o), pu.f64(outs[0][0])) < pu.O_REL_FRO
        assert np.abs(pu.f64(lse) - pu.f64(outs[0][1])).max() < 1e-4


def test_decode_fp16():
    _check(*_run([600, 33], 8, 2, 2, 128, 16, True, 0, dtype=torch.float16), True, bits=11)


def test_no_device_wait_timed_out():
    from exact_io_aware_49_b200 import fa_last_device_error
    assert fa_last_device_error() == 0


def test_bench_shape_sampled_sequences():
    """The decode benchmark's launch: 16 sequences x 32768 cached positions,
    32 query / 8 key-value heads, one query, d = 128, pages of 64 in shuffled
    order, the split count fa_decode_num_splits picks (8 here).  The cache is
    drawn on the device; every query head of three sequences (first, middle,
    last) is checked against the oracle on those sequences' gathered pages."""
    from exact_io_aware_49_b200 import binding, fa_decode_paged
    B, H, H_kv, Nq, d, L, page = 16, 32, 8, 1, 128, 32768, 64
    lib = binding.load_library()
    splits = int(lib.fa_decode_num_splits(B, H_kv, H, Nq, L))
    assert splits > 1
    gen = torch.Generator(device="cuda").manual_seed(7)
    n_pages = B * (L // page)
    kc = torch.randn(n_pages, page, H_kv, d, generator=gen, device="cuda").to(torch.bfloat16)
    vc = torch.randn(n_pages, page, H_kv, d, generator=gen, device="cuda").to(torch.bfloat16)
    table = torch.randperm(n_pages, generator=gen, device="cuda").to(torch.int32).view(B, -1)
    q = torch.randn(B, H, Nq, d, generator=gen, device="cuda").to(torch.bfloat16)
    lens = torch.full((B,), L, dtype=torch.int32, device="cuda")
    o, lse = fa_decode_paged(q, kc, vc, table, lens, L, True, d ** -0.5, num_splits=splits)
    torch.cuda.synchronize()
    for b in (0, B // 2, B - 1):
        pages = table[b].long()
        k_b = kc[pages].reshape(L, H_kv, d).to(torch.float64).cpu().numpy()
        v_b = vc[pages].reshape(L, H_kv, d).to(torch.float64).cpu().numpy()
        q_b = q[b].to(torch.float64).cpu().numpy()

        def one(h):
            g = h // (H // H_kv)
            want_o, want_l = attention.forward(q_b[h], k_b[:, g], v_b[:, g], causal=True, scale=d ** -0.5)
            pu.check_o(pu.f64(o[b, h]), want_o, f"O seq {b} head {h}")
            pu.check_lse(pu.f64(lse[b, h]), want_l, f"LSE seq {b} head {h}")

        pu.map_heads(one, range(H))
