"""The conservative Gumbel-key test of the build epilogues (gumbel_may_beat in
csrc/epi_util.cuh), checked on the host with its constants read from the
source.

The device test passes a token when w_lo < e_hi, with
  w_lo = 1 - U                        if 1 - U < 2^-7
       = c_w * (-__logf(U))           otherwise,
  e_hi = 2^((s - thr) log2 e + c_e),
and the exact key s + (-log(-log U)) is computed only for tokens that pass.
This emulates both approximations with errors at the ends of their stated
bounds (__logf: 2^-21 absolute near 1, 2^-21 relative elsewhere; ex2.approx:
2^-22 relative) and checks that no token whose fp32 key beats thr is
rejected, over random and adversarial (near-threshold) cases.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "draft_tree_construction_markov_b200", "csrc", "epi_util.cuh")


def _constants():
    txt = open(SRC).read()
    body = txt[txt.index("gumbel_may_beat"):]
    body = body[: body.index("\n}\n")]
    thr_v = float(re.search(r"v < ([0-9.e+-]+)f", body).group(1))
    c_w = float(re.search(r"-([0-9.]+)f \* __logf", body).group(1))
    c_e = float(re.search(r"kLog2e \+ ([0-9.e+-]+)f", body).group(1))
    return thr_v, c_w, c_e


def test_constants_are_the_documented_ones():
    thr_v, c_w, c_e = _constants()
    assert thr_v == 2.0 ** -7
    assert c_w == 0.999
    assert abs(c_e - np.log2(1.001)) < 1e-9


def test_filter_never_rejects_a_key_that_beats_the_bar():
    thr_v, c_w, c_e = _constants()
    f = np.float32
    rng = np.random.default_rng(0)
    n = 4_000_000
    word = rng.integers(0, 2 ** 32, n, dtype=np.uint64)
    m = (word >> np.uint64(9)).astype(np.float64)
    u = ((m + 0.5) * 2.0 ** -23).astype(f)
    v = ((f(0x7FFFFF) - m.astype(f)) + f(0.5)) * f(2.0 ** -23)
    assert np.array_equal(v.astype(np.float64), 1.0 - u.astype(np.float64))
    s = rng.normal(0, 4, n).astype(f)
    # thresholds spread over the range where keys are decided, plus
    # adversarial ones placed right at (or a rounding step below) each key
    thr = (rng.normal(0, 4, n) + rng.choice([0, 3, 8, 14, 16], n)).astype(f)
    key = (s.astype(np.float64) + (-np.log(-np.log(u.astype(np.float64))))).astype(f)
    adv = rng.random(n) < 0.5
    thr[adv] = np.nextafter(key[adv], f(-np.inf))
    beats = key > thr
    # __logf at the pessimistic end of its error bound (w_lo as large as it
    # can come out), ex2.approx at the small end (e_hi as small as it can)
    lu = np.log(u.astype(np.float64))
    lu_approx = np.where(u >= 0.5, lu - 2.0 ** -21, lu * (1 + 2.0 ** -21))
    w_lo = np.where(v < f(thr_v), v.astype(np.float64), c_w * (-lu_approx))
    x = (s.astype(np.float64) - thr.astype(np.float64)) * np.log2(np.e) + c_e
    e_hi = np.exp2(x) * (1 - 2.0 ** -22)
    passed = w_lo < e_hi
    missed = beats & ~passed
    assert beats.sum() > n // 4
    assert missed.sum() == 0, int(missed.sum())
    # and the test is tight: it lets through few tokens that cannot win
    assert (passed & ~beats).sum() < 0.01 * n
