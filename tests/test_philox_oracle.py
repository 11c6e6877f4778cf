"""Pins for the oracle's Philox4x32-10 and dropout keep mask (CPU only).

* the published known-answer vectors of Philox4x32-10
  (``tests/golden/philox4x32_10_kat.txt``, cited there);
* bit-exact agreement with an independent implementation: ATen's header-only
  ``philox_engine`` compiled with g++ from the installed torch headers;
* the (i, j) -> output word / half mapping restated here against that engine;
* keep rate 1 - t/65536 within 5 sigma over 10^7 draws, and lag-1
  correlation along j, i, h and b within 5 sigma of zero.
"""

import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch

from oracle import philox

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def aten_philox():
    inc = os.path.join(os.path.dirname(torch.__file__), "include")
    src = os.path.join(HERE, "philox_aten_xcheck.cpp")
    tmp = tempfile.mkdtemp(prefix="philox_xcheck_")
    exe = os.path.join(tmp, "xcheck")
    subprocess.run(["g++", "-O1", "-std=c++17", "-I", inc, src, "-o", exe], check=True)

    def run(triples):
        text = "".join(f"{s} {ss} {o}\n" for s, ss, o in triples)
        out = subprocess.run([exe], input=text, capture_output=True, text=True, check=True).stdout
        return [tuple(int(x) for x in line.split()) for line in out.strip().splitlines()]

    return run


def _counters(rng, n):
    return [(int(rng.integers(0, 2**64, dtype=np.uint64)),) + tuple(int(x) for x in rng.integers(0, 2**32, size=4))
            for _ in range(n)]


def _kat():
    rows = []
    with open(os.path.join(HERE, "golden", "philox4x32_10_kat.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            lhs, rhs = line.split("->")
            rows.append(([int(x, 16) for x in lhs.split()], [int(x, 16) for x in rhs.split()]))
    return rows


def test_philox_known_answer_vectors():
    rows = _kat()
    assert len(rows) == 3
    for (c0, c1, c2, c3, k0, k1), want in rows:
        out = philox.philox4x32(*(np.array([x], dtype=np.uint64) for x in (c0, c1, c2, c3)), k0, k1)
        assert [int(np.asarray(r).ravel()[0]) for r in out] == want


def test_philox_matches_aten_engine(aten_philox):
    rng = np.random.default_rng(1234)
    cases = _counters(rng, 200) + [(0, 0, 0, 0, 0), (2**64 - 1, 2**32 - 1, 2**32 - 1, 2**32 - 1, 2**32 - 1)]
    triples = [(seed, (c3 << 32) | c2, (c1 << 32) | c0) for seed, c0, c1, c2, c3 in cases]
    ref = aten_philox(triples)
    for (seed, c0, c1, c2, c3), want in zip(cases, ref):
        got = philox.philox4x32(c0, c1, c2, c3, seed & 0xFFFFFFFF, seed >> 32)
        assert tuple(int(x) for x in got) == want


def test_uniform16_word_and_half_mapping(aten_philox):
    seed, b, h = 0x0123456789ABCDEF, 3, 5
    rows = np.array([0, 1, 77, 4095])
    cols = np.arange(0, 40)
    u = philox.uniform16(seed, b, h, rows, cols)
    triples = [(seed, (b << 32) | h, (int(i) << 32) | (int(j) >> 3)) for i in rows for j in cols]
    ref = aten_philox(triples)
    for n, (i_idx, j) in enumerate([(a, j) for a in range(len(rows)) for j in cols]):
        word = ref[n][(int(j) >> 1) & 3]
        want = (word >> 16) if (j & 1) else (word & 0xFFFF)
        assert u[i_idx, j] == want


def test_threshold_rounding():
    assert philox.keep_threshold(0.0) == 0
    assert philox.keep_threshold(0.1) == 6554  # 6553.6 -> 6554
    assert philox.keep_threshold(0.5) == 32768
    assert philox.keep_threshold(1.0 / 65536 * 2.5) == 2  # half -> even
    assert philox.keep_threshold(1.0 / 65536 * 3.5) == 4
    with pytest.raises(ValueError):
        philox.keep_threshold(1.0)
    with pytest.raises(ValueError):
        philox.keep_threshold(-0.1)


def test_p_zero_keeps_everything():
    z = philox.keep_mask(7, 0, 0, np.arange(16), np.arange(64), 0.0)
    assert z.all()


def test_keep_rate_within_5_sigma():
    t = philox.keep_threshold(0.1)
    rows = np.arange(2500)
    cols = np.arange(4000)
    u = philox.uniform16(2, 1, 3, rows, cols)
    n = u.size
    keep = (u >= t).mean()
    p_keep = 1.0 - t / 65536.0
    sigma = np.sqrt(p_keep * (1 - p_keep) / n)
    assert n >= 10**7
    assert abs(keep - p_keep) < 5 * sigma


def _lag1(a, b):
    a = a.astype(np.float64).ravel()
    b = b.astype(np.float64).ravel()
    r = np.corrcoef(a, b)[0, 1]
    return r, 1.0 / np.sqrt(a.size)


def test_lag1_correlations_within_5_sigma():
    seed = 99
    rows = np.arange(512)
    cols = np.arange(1024)
    u = philox.uniform16(seed, 0, 0, rows, cols)
    r, s = _lag1(u[:, :-1], u[:, 1:])  # along j
    assert abs(r) < 5 * s
    r, s = _lag1(u[:-1, :], u[1:, :])  # along i
    assert abs(r) < 5 * s
    u_h1 = philox.uniform16(seed, 0, 1, rows, cols)
    r, s = _lag1(u, u_h1)  # along h
    assert abs(r) < 5 * s
    u_b1 = philox.uniform16(seed, 1, 0, rows, cols)
    r, s = _lag1(u, u_b1)  # along b
    assert abs(r) < 5 * s
