"""Pins for the fp64 CPU oracle (no GPU).

The oracle is checked against things other than itself: hand-derived closed
forms (tests/golden), brute force in pure Python on inputs whose scores are
exact, a library routine (torch's CPU scaled_dot_product_attention in float64),
and invariants that the definition of exact softmax attention fixes.  A final
test plants mistakes in copies of the oracle's C source and checks that the
pins catch every one of them.
"""
import json
import math
import os
import re
import tempfile

import numpy as np
import pytest

import oracle
import synth

HERE = os.path.dirname(os.path.abspath(__file__))


def _rng(seed):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------
# Pin functions: each takes an oracle library handle and asserts.
# --------------------------------------------------------------------------

def pin_golden(lib):
    g = json.load(open(os.path.join(HERE, "golden", "closed_form.json")))
    for case in g["cases"]:
        r = oracle.attention(np.array(case["Q"]), np.array(case["K"]), np.array(case["V"]),
                             case["scale"], lib=lib)
        np.testing.assert_allclose(r["O"], np.array(case["O"]), rtol=0, atol=1e-12,
                                   err_msg=case["name"])
        np.testing.assert_allclose(r["L"], np.array(case["L"]), rtol=0, atol=1e-12,
                                   err_msg=case["name"])
        np.testing.assert_allclose(r["S"], np.array(case["S"]), rtol=1e-13, atol=0,
                                   err_msg=case["name"])


def _brute(q, k, v, scale):
    """Pure-Python exact attention with math.fsum (correctly rounded sums)."""
    B, H, N, d = q.shape
    M = k.shape[2]
    O = np.zeros((B, H, N, d))
    L = np.zeros((B, H, N))
    S = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            for i in range(N):
                a = [scale * math.fsum(float(q[b, h, i, t]) * float(k[b, h, j, t]) for t in range(d))
                     for j in range(M)]
                mx = max(a)
                e = [math.exp(x - mx) for x in a]
                s = math.fsum(e)
                L[b, h, i] = mx
                S[b, h, i] = s
                for c in range(d):
                    O[b, h, i, c] = math.fsum(e[j] * float(v[b, h, j, c]) for j in range(M)) / s
    return O, L, S


def pin_bruteforce(lib):
    rng = _rng(7)
    for (N, M, d, scale) in [(1, 1, 1, 1.0), (2, 3, 2, 0.5), (3, 5, 3, 1.0), (5, 8, 2, 0.5),
                             (8, 2, 3, 1.0), (4, 4, 1, 0.5)]:
        B, H = 2, 2
        q = rng.integers(-3, 4, size=(B, H, N, d)).astype(np.float64)
        k = rng.integers(-3, 4, size=(B, H, M, d)).astype(np.float64)
        v = rng.integers(-3, 4, size=(B, H, M, d)).astype(np.float64)
        Ob, Lb, Sb = _brute(q, k, v, scale)
        r = oracle.attention(q, k, v, scale, lib=lib)
        # integer products times 1 or 1/2 are exact in fp64, so L is exact
        assert np.array_equal(r["L"], Lb), (N, M, d)
        np.testing.assert_allclose(r["S"], Sb, rtol=1e-15, atol=0)
        np.testing.assert_allclose(r["O"], Ob, rtol=0, atol=1e-13)


def pin_sdpa(lib):
    torch = pytest.importorskip("torch")
    import torch.nn.functional as F
    for (B, H, N, M, d, cid) in [(1, 1, 256, 256, 40, 1), (2, 3, 37, 77, 8, 11), (1, 2, 65, 9, 16, 12)]:
        q, k, v = synth.make_qkv(synth.Shape("t", B, H, N, M, d), cid, dtype=np.float64)
        scale = float(np.float32(1.0 / math.sqrt(d)))
        r = oracle.attention(q, k, v, scale, lib=lib)
        ref = F.scaled_dot_product_attention(torch.from_numpy(q), torch.from_numpy(k),
                                             torch.from_numpy(v), scale=scale).numpy()
        np.testing.assert_allclose(r["O"], ref, rtol=0, atol=1e-12)


def pin_rows_sum_to_one(lib):
    q, k, v = synth.make_qkv(synth.Shape("t", 2, 2, 33, 70, 40), 21, dtype=np.float64)
    scale = 1.0 / math.sqrt(40)
    r = oracle.attention(q, k, v, scale, want_a=True, lib=lib)
    p = np.exp(r["A"] - r["L"][..., None]) / r["S"][..., None]
    assert np.max(np.abs(p.sum(-1) - 1.0)) <= 1e-13
    # L is attained: some score equals the row max, none exceeds it
    assert np.all(r["A"].max(-1) == r["L"])


def pin_identical_keys(lib):
    B, H, N, M, d = 2, 2, 9, 50, 40
    q, _, v = synth.make_qkv(synth.Shape("t", B, H, N, M, d), 22, dtype=np.float64)
    krow = synth.normal(99, (B, H, 1, d), np.float64)
    k = np.repeat(krow, M, axis=2)
    scale = 0.25
    r = oracle.attention(q, k, v, scale, lib=lib)
    np.testing.assert_allclose(r["O"], np.broadcast_to(v.mean(axis=2, keepdims=True), r["O"].shape),
                               rtol=0, atol=1e-13)
    assert np.all(r["S"] == M)
    np.testing.assert_allclose(r["L"], scale * np.einsum("bhnd,bhd->bhn", q, krow[:, :, 0]),
                               rtol=0, atol=1e-14)


def pin_one_hot(lib):
    B, H, N, M, d = 1, 2, 40, 64, 40
    scale = 1.0 / math.sqrt(d)
    beta = 30.0 / scale
    k = np.zeros((B, H, M, d))
    for j in range(d):
        k[:, :, j, j] = beta
    perm = _rng(3).permutation(N)
    q = np.zeros((B, H, N, d))
    for i in range(N):
        q[:, :, i, perm[i] % d] = 1.0
    v = synth.normal(5, (B, H, M, d), np.float64)
    r = oracle.attention(q, k, v, scale, lib=lib)
    tol = M * math.exp(-30.0) * np.abs(v).max() * 2
    for i in range(N):
        np.testing.assert_allclose(r["O"][:, :, i], v[:, :, perm[i] % d], rtol=0, atol=tol)
    np.testing.assert_allclose(r["L"], 30.0, rtol=1e-15)


def pin_permutation(lib):
    q, k, v = synth.make_qkv(synth.Shape("t", 2, 2, 17, 77, 40), 23, dtype=np.float64)
    scale = 1.0 / math.sqrt(40)
    r0 = oracle.attention(q, k, v, scale, lib=lib)
    perm = _rng(11).permutation(77)
    r1 = oracle.attention(q, k[:, :, perm], v[:, :, perm], scale, lib=lib)
    np.testing.assert_allclose(r1["O"], r0["O"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(r1["S"], r0["S"], rtol=1e-13)
    assert np.array_equal(r1["L"], r0["L"])


def pin_shift(lib):
    q, k, v = synth.make_qkv(synth.Shape("t", 1, 2, 13, 31, 16), 24, dtype=np.float64)
    scale = 0.3
    u = synth.normal(77, (1, 2, 1, 16), np.float64)
    r0 = oracle.attention(q, k, v, scale, lib=lib)
    r1 = oracle.attention(q, k + u, v, scale, lib=lib)
    np.testing.assert_allclose(r1["O"], r0["O"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(r1["S"], r0["S"], rtol=1e-11)
    shift = scale * np.einsum("bhnd,bhd->bhn", q, u[:, :, 0])
    np.testing.assert_allclose(r1["L"], r0["L"] + shift, rtol=0, atol=1e-12)


def pin_single_key(lib):
    q, k, v = synth.make_qkv(synth.Shape("t", 2, 3, 11, 1, 40), 25, dtype=np.float64)
    scale = 1.0 / math.sqrt(40)
    r = oracle.attention(q, k, v, scale, lib=lib)
    np.testing.assert_array_equal(r["O"], np.broadcast_to(v, r["O"].shape))
    assert np.all(r["S"] == 1.0)
    np.testing.assert_allclose(r["L"], scale * np.einsum("bhnd,bhd->bhn", q, k[:, :, 0]),
                               rtol=0, atol=1e-14)


PINS = [pin_golden, pin_bruteforce, pin_sdpa, pin_rows_sum_to_one, pin_identical_keys,
        pin_one_hot, pin_permutation, pin_shift, pin_single_key]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_empty_query_rows(oracle_lib):
    q = np.zeros((1, 1, 0, 8))
    k = np.ones((1, 1, 4, 8))
    r = oracle.attention(q, k, k, 1.0)
    assert r["O"].shape == (1, 1, 0, 8)


# --------------------------------------------------------------------------
# Planted mistakes: each mutant of oracle.c must fail at least one pin.
# --------------------------------------------------------------------------
MUTANTS = {
    "dropped scale": ("a[j] = scale * dot;", "a[j] = dot;"),
    "dropped max shift": ("e[j] = exp(a[j] - L);", "e[j] = exp(a[j]);"),
    "min instead of max": ("if (a[j] > L) L = a[j];", "if (a[j] < L) L = a[j];"),
    "no normalisation": ("o[c] = acc / S;", "o[c] = acc;"),
    "wrong sign": ("e[j] = exp(a[j] - L);", "e[j] = exp(L - a[j]);"),
    "wrong head for K": ("const double *Kh = K + bh * M * d;", "const double *Kh = K;"),
    "wrong V column": ("acc += e[j] * Vh[j * d + c];", "acc += e[j] * Vh[j * d];"),
    "first key skipped": ("S += e[j];", "if (j) S += e[j];"),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation anchor not found: {old}"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    so = str(tmp_path / "mutant.so")
    oracle.build(force=True, src=str(mutated), out=so)
    lib = oracle.load(so)
    caught = []
    for pin in PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant '{name}' passed every pin"
