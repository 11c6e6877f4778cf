"""Shared helpers for the GPU parity tests: run the oracle on the same seeded
inputs and compare with the tolerances the method fixes (bf16 I/O, fp32
accumulation): O max-abs <= 1e-2 and relative Frobenius <= 5e-3; LSE
absolute <= 1e-3; dQ/dK/dV relative Frobenius <= 2e-2; masks bit-exact."""

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

from oracle import attention

O_MAX_ABS = 1e-2
O_REL_FRO = 5e-3
LSE_ABS = 1e-3
GRAD_REL_FRO = 2e-2


def f64(x):
    return x.detach().to("cpu", torch.float64).numpy()


def rel_fro(got, want):
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def bf16_half_ulp(x, bits=8):
    """Half a unit in the last place at |x| of a format with ``bits`` significant
    bits (8 for bf16, 11 for fp16): the largest error that rounding the exact
    value to the 16-bit output can introduce (normal range)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - bits), 0.0)


def check_o(got, want, what="", bits=8):
    """O max-abs <= 1e-2 on top of the bf16 output rounding, rel-Frobenius <= 5e-3.

    O is returned in bf16, so even the exact result rounded to bf16 differs from
    the fp64 oracle by up to half a bf16 ulp -- more than 1e-2 once |O| >= 2.56
    (near one-hot rows of wide-logit inputs, or 1/(1-p) at large p).  The
    max-abs bound therefore applies to the error beyond that rounding:
    |got - want| <= 1e-2 + half_ulp_bf16(want)."""
    excess = float((np.abs(got - want) - bf16_half_ulp(want, bits)).max())
    err = float(np.abs(got - want).max())
    rel = rel_fro(got, want)
    assert excess <= O_MAX_ABS and rel <= O_REL_FRO, \
        f"{what}: O max-abs {err:.3e} (beyond bf16 rounding {excess:.3e}) rel-fro {rel:.3e}"
    return err, rel


def check_lse(got, want, what=""):
    """|got - want| <= 1e-3; a row that sees no key must be -inf on both sides."""
    empty = np.isneginf(want)
    assert np.array_equal(np.isneginf(got), empty), f"{what}: LSE -inf rows differ"
    if empty.all():
        return 0.0
    err = float(np.abs(got[~empty] - want[~empty]).max())
    assert err <= LSE_ABS, f"{what}: LSE max-abs {err:.3e}"
    return err


def check_grad(got, want, what=""):
    """Relative Frobenius error <= 2e-2, with the reference norm floored at 1e-3
    for gradients that are identically zero (N = 1: a single key gets P = 1,
    so dS = 0 and dQ = dK = 0 exactly)."""
    rel = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-3))
    assert rel <= GRAD_REL_FRO, f"{what}: rel-fro {rel:.3e}"
    return rel


def oracle_fwd_head(q, k, v, b, h, causal, scale, p_drop, seed, rows=None):
    """Oracle O, LSE for head (b, h) of bf16 CPU tensors [B, H, N, d] (rows: optional sample)."""
    qh, kh, vh = (x[b, h].to(torch.float64).numpy() for x in (q, k, v))
    if rows is None:
        return attention.forward(qh, kh, vh, causal=causal, scale=scale, p_drop=p_drop, seed=seed, b=b, h=h)
    lse, o, _ = attention.row_stats(qh, kh, vh, np.zeros_like(vh), causal=causal, scale=scale, p_drop=p_drop,
                                    seed=seed, b=b, h=h, rows=rows)
    return o, lse


def map_heads(fn, items):
    """fn over ``items`` on a pool of host threads (NumPy releases the GIL in
    its array kernels, so per-head oracle work runs in parallel); returns the
    results in order and re-raises the first failure."""
    items = list(items)
    workers = max(1, min(len(items), len(os.sched_getaffinity(0))))
    with ThreadPoolExecutor(workers) as ex:
        return list(ex.map(fn, items))
