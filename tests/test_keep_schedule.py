"""Chunk-aware growth schedule (host only, CPU): the library's hf_keep_schedule against
the oracle, and its argument checks."""
import ctypes
import math

import numpy as np
import pytest

import hybrid_sparse_linear_hf_b200 as hf
import oracle
from hybrid_sparse_linear_hf_b200 import _binding as B


def _cases(seed, count):
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < count:
        n = int(rng.integers(1, 40))
        full = int(rng.integers(1, 400))
        fill = int(rng.integers(1, 10))
        nKB = [max(1, (full * min(i + 1, fill)) // fill) for i in range(n)]
        t = float(rng.uniform(0.0, 0.95))
        s_base = float(rng.uniform(0.0, 0.999))
        out.append((nKB, s_base, t))
    return out


def test_schedule_matches_oracle():
    accepted = rejected = 0
    for nKB, s_base, t in _cases(5, 3000):
        try:
            r_o, s_o, beta_o = oracle.keep_schedule(nKB, s_base, t)
        except ValueError:
            with pytest.raises(hf.HfError) as e:
                hf.hf_keep_schedule(nKB, s_base, t)
            assert e.value.status == B.HF_ERR_INVALID_ARG
            rejected += 1
            continue
        r, s, beta = hf.hf_keep_schedule(nKB, s_base, t)
        accepted += 1
        assert abs(beta - beta_o) <= 1e-12 * max(1.0, abs(beta_o)), (nKB, s_base, t)
        assert np.allclose(s, s_o, rtol=0, atol=1e-12)
        for i, k in enumerate(nKB):
            if r[i] != r_o[i]:
                # a different rounding of s may only move an exact integer boundary
                x = (1.0 - s_o[i]) * k
                assert abs(x - round(x)) < 1e-9 and abs(r[i] - r_o[i]) == 1, (i, x, r[i], r_o[i])
    assert accepted > 500 and rejected > 100, (accepted, rejected)


def test_schedule_examples():
    r, s, beta = hf.hf_keep_schedule([10, 20], 0.9, 0.5)
    assert r == [10, 5] and s[0] == 0.0 and abs(s[1] - 0.75) < 1e-15 and abs(beta - 0.15) < 1e-15
    # 832x480: windows of 1, 2, ... 7 chunks of 4680 tokens (blocks of 128), then full
    nKB = [math.ceil(min(i + 1, 7) * 4680 / 128) for i in range(12)]
    r, s, _ = hf.hf_keep_schedule(nKB, 0.85, 0.75)
    assert r[0] == nKB[0] == 37 and nKB[6:] == [256] * 6
    assert all(s[i] < s[i + 1] for i in range(1, 11)) and s[-1] < 0.85
    assert abs(sum((1 - s[i]) * nKB[i] for i in range(12)) - 0.25 * sum(nKB)) < 1e-9


def test_schedule_argument_checks():
    L = hf.lib()
    r = (ctypes.c_int * 4)(-7, -7, -7, -7)
    s = (ctypes.c_double * 4)()
    kb = (ctypes.c_int * 4)(8, 8, 8, 8)
    bad = (ctypes.c_int * 4)(8, 0, 8, 8)
    for args in ((0, kb, 0.5, 0.5), (4, None, 0.5, 0.5), (4, bad, 0.5, 0.5), (4, kb, 1.0, 0.5),
                 (4, kb, 0.5, -0.01), (4, kb, float("nan"), 0.5), (4, kb, 0.2, 0.5)):
        assert L.hf_keep_schedule(*args, r, s, None) == B.HF_ERR_INVALID_ARG, args
        assert list(r) == [-7] * 4, "nothing is written on an error"
    assert L.hf_keep_schedule(4, kb, 0.8, 0.5, None, s, None) == B.HF_ERR_INVALID_ARG
    assert L.hf_keep_schedule(1, kb, 0.0, 0.9, r, None, None) == B.HF_OK and r[0] == 8
