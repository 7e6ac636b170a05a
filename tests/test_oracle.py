"""Pins for the fp64 oracle (CPU only).

Each check ties the oracle to something other than itself: a hand-worked
example, closed forms, invariants, special cases that reduce to a library
routine, or a separately written pure-Python brute force.  The last group
plants plausible mistakes in a copy of the oracle and checks that the pins
catch each one.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention as A
from io_aware_attention_02_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed=0, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# --------------------------------------------------------------------------
# hand-worked example
# --------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_two_token_hand_example(causal):
    g = json.load(open(os.path.join(GOLDEN, "two_token.json")))
    q, k, v = (np.array(g[n]) for n in ("q", "k", "v"))
    o, lse = A.attention_head(q, k, v, g["scale"], causal)
    want = g["causal" if causal else "non_causal"]
    np.testing.assert_allclose(o, np.array(want["O"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, np.array(want["LSE"]), rtol=0, atol=1e-15)


# --------------------------------------------------------------------------
# closed forms and invariants
# --------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_gives_that_row(causal):
    q, k = _rand((37, 8), 1), _rand((37, 8), 2)
    c = _rand((8,), 3)
    v = np.tile(c, (37, 1))
    o, _ = A.attention_head(q, k, v, 0.7, causal)
    np.testing.assert_allclose(o, np.tile(c, (37, 1)), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one_and_mask(causal):
    q, k = _rand((29, 16), 4), _rand((29, 16), 5)
    p = A.probabilities(q, k, 0.25, causal)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    assert (p >= 0).all()
    if causal:
        assert np.all(p[np.triu_indices(29, 1)] == 0.0)
        assert np.all(p[np.tril_indices(29)] > 0.0)


def test_causal_row0_identity():
    q, k, v = _rand((21, 8), 6), _rand((21, 8), 7), _rand((21, 8), 8)
    scale = 0.35
    o, lse = A.attention_head(q, k, v, scale, causal=True)
    np.testing.assert_allclose(o[0], v[0], rtol=0, atol=0)
    assert lse[0] == pytest.approx(scale * float(q[0] @ k[0]), abs=1e-14)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("zero", ["q", "k"])
def test_zero_q_or_k_is_uniform_attention(causal, zero):
    n, d = 19, 4
    q, k, v = _rand((n, d), 9), _rand((n, d), 10), _rand((n, d), 11)
    if zero == "q":
        q[:] = 0.0
    else:
        k[:] = 0.0
    o, lse = A.attention_head(q, k, v, 1.3, causal)
    for i in range(n):
        J = range(i + 1) if causal else range(n)
        np.testing.assert_allclose(o[i], v[list(J)].mean(axis=0), rtol=0, atol=1e-14)
        assert lse[i] == pytest.approx(math.log(len(J)), abs=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_lse_bounds(causal):
    q, k = _rand((64, 16), 12, 3.0), _rand((64, 16), 13)
    s = A.scores(q, k, 0.25, causal)
    _, lse = A.attention_head(q, k, _rand((64, 16), 14), 0.25, causal)
    smax = s.max(axis=1)
    count = np.isfinite(s).sum(axis=1)
    assert np.all(lse >= smax - 1e-12)
    assert np.all(lse <= smax + np.log(count) + 1e-12)


def test_key_shift_moves_lse_not_output():
    """k_j -> k_j + u adds scale <q_i, u> to every score of row i."""
    n, d, scale = 33, 8, 0.5
    q, k, v = _rand((n, d), 15), _rand((n, d), 16), _rand((n, d), 17)
    u = _rand((d,), 18)
    o1, l1 = A.attention_head(q, k, v, scale)
    o2, l2 = A.attention_head(q, k + u, v, scale)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2 - l1, scale * (q @ u), rtol=0, atol=1e-12)


def test_key_permutation_equivariance_non_causal():
    n, d = 40, 8
    q, k, v = _rand((n, d), 19), _rand((n, d), 20), _rand((n, d), 21)
    perm = np.random.default_rng(22).permutation(n)
    o1, l1 = A.attention_head(q, k, v, 0.3)
    o2, l2 = A.attention_head(q, k[perm], v[perm], 0.3)
    np.testing.assert_allclose(o2, o1, atol=1e-13)
    np.testing.assert_allclose(l2, l1, atol=1e-13)


def test_row_sampling_matches_full():
    n, d = 50, 8
    q, k, v = _rand((n, d), 23), _rand((n, d), 24), _rand((n, d), 25)
    rows = np.array([0, 3, 17, 49])
    for causal in (False, True):
        of, lf = A.attention_head(q, k, v, 0.4, causal)
        os_, ls = A.attention_head(q, k, v, 0.4, causal, rows=rows)
        np.testing.assert_array_equal(os_, of[rows])
        np.testing.assert_array_equal(ls, lf[rows])


# --------------------------------------------------------------------------
# independent implementations
# --------------------------------------------------------------------------

def _brute_force(q, k, v, scale, causal):
    """Two-pass pure-Python attention with math.fsum (written separately)."""
    n = len(q)
    out, lses = [], []
    for i in range(n):
        keys = range(i + 1) if causal else range(n)
        s = [scale * math.fsum(q[i][c] * k[j][c] for c in range(len(q[i]))) for j in keys]
        mx = max(s)
        w = [math.exp(x - mx) for x in s]
        tot = math.fsum(w)
        out.append([math.fsum(w[t] * v[j][c] for t, j in enumerate(keys)) / tot
                    for c in range(len(v[0]))])
        lses.append(mx + math.log(tot))
    return np.array(out), np.array(lses)


@pytest.mark.parametrize("n,d", [(1, 1), (2, 3), (5, 4), (8, 2), (7, 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_tiny(n, d, causal):
    q, k, v = _rand((n, d), 26 + n), _rand((n, d), 27 + d), _rand((n, d), 28)
    o, lse = A.attention_head(q, k, v, 0.8, causal)
    ob, lb = _brute_force(q.tolist(), k.tolist(), v.tolist(), 0.8, causal)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_float64(causal):
    """torch's scaled_dot_product_attention (float64, CPU) is an independent
    implementation of the same definition."""
    B, H, N, d = 2, 3, 70, 16
    q, k, v = (_rand((B, H, N, d), s) for s in (30, 31, 32))
    o, _ = A.attention(q, k, v, 1 / math.sqrt(d), causal)
    ot = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=causal)
    np.testing.assert_allclose(o, ot.numpy(), rtol=0, atol=1e-13)


def _online_softmax_model(q, k, v, scale, causal, br=16, bc=16, lazy=8.0):
    """fp64 restatement of the tiled online-softmax recurrence (dibro.site,
    'Arquitectura y metodo'; droidorbit.com, 'Mathematical Formulation'):
    blocks of Br query rows and Bc keys, fully-masked blocks skipped, running
    max m and sum l, output rescaled by exp(m_old - m_new) -- in the base-2
    form with a lazy threshold (the max is only raised when it grows by more
    than ``lazy`` in log2 units)."""
    n, d = q.shape
    c = scale / math.log(2.0)
    O = np.zeros((n, v.shape[1]))
    L = np.zeros(n)
    for r0 in range(0, n, br):
        r1 = min(n, r0 + br)
        m = np.full(r1 - r0, -np.inf)
        l = np.zeros(r1 - r0)
        acc = np.zeros((r1 - r0, v.shape[1]))
        last = (r1 - 1) if causal else n - 1
        for c0 in range(0, last + 1, bc):
            c1 = min(n, c0 + bc)
            s = (q[r0:r1] @ k[c0:c1].T) * c
            if causal:
                s = np.where(np.arange(c0, c1)[None, :] <= np.arange(r0, r1)[:, None], s, -np.inf)
            mb = s.max(axis=1)
            grow = mb > m + lazy
            m_new = np.where(grow | ~np.isfinite(m), np.maximum(m, mb), m)
            alpha = np.where(np.isfinite(m), np.exp2(m - m_new), 0.0)
            p = np.exp2(s - m_new[:, None])
            l = l * alpha + p.sum(axis=1)
            acc = acc * alpha[:, None] + p @ v[c0:c1]
            m = m_new
        O[r0:r1] = acc / l[:, None]
        L[r0:r1] = (m + np.log2(l)) * math.log(2.0)
    return O, L


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n", [16, 45, 64])
def test_online_softmax_recurrence_equals_definition(causal, n):
    q, k, v = _rand((n, 8), 40, 2.0), _rand((n, 8), 41, 2.0), _rand((n, 8), 42)
    o, lse = A.attention_head(q, k, v, 0.9, causal)
    om, lm = _online_softmax_model(q, k, v, 0.9, causal)
    np.testing.assert_allclose(om, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lm, lse, rtol=0, atol=1e-12)


def test_flop_convention():
    assert A.flops(4, 16, 8192, 128, False) == 4 * 4 * 16 * 8192 * 8192 * 128
    assert A.flops(4, 16, 8192, 128, True) == 2 * 4 * 16 * 8192 * 8192 * 128


# --------------------------------------------------------------------------
# planted mistakes: each mutant of the oracle must fail at least one pin
# --------------------------------------------------------------------------

def _mutant(kind):
    def f(q, k, v, scale, causal=False, rows=None):
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        n = q.shape[0]
        sc = 1.0 if kind == "no_scale" else scale
        s = sc * ((k @ q.T) if kind == "transposed" else (q @ k.T))
        if causal:
            j, i = np.arange(n)[None, :], np.arange(n)[:, None]
            keep = (j < i) | (i == 0) & (j == 0) if kind == "strict_mask" else (j <= i)
            s = np.where(keep, s, -np.inf)
        m = s.max(axis=0 if kind == "wrong_axis" else 1)
        m = m[None, :] if kind == "wrong_axis" else m[:, None]
        e = np.exp(s - m)
        l = e.sum(axis=1)
        o = (e / l[:, None]) @ v
        lse = (m[:, 0] if kind != "wrong_axis" else m[0]) + (0 if kind == "lse_no_log" else np.log(l))
        return o, lse
    return f


@pytest.mark.parametrize("kind", ["no_scale", "transposed", "strict_mask", "wrong_axis", "lse_no_log"])
def test_pins_catch_planted_mistakes(kind):
    f = _mutant(kind)
    failures = 0
    g = json.load(open(os.path.join(GOLDEN, "two_token.json")))
    q, k, v = (np.array(g[n]) for n in ("q", "k", "v"))
    for causal in (False, True):
        o, lse = f(q, k, v, 0.5 if kind == "no_scale" else g["scale"], causal)
        want = g["causal" if causal else "non_causal"]
        if kind == "no_scale":
            o_ref, l_ref = A.attention_head(q, k, v, 0.5, causal)
            want = {"O": o_ref, "LSE": l_ref}
        if not (np.allclose(o, want["O"], atol=1e-12) and np.allclose(lse, want["LSE"], atol=1e-12)):
            failures += 1
    # brute force on an asymmetric random case
    qq, kk, vv = _rand((6, 3), 50), _rand((6, 3), 51), _rand((6, 3), 52)
    for causal in (False, True):
        o, lse = f(qq, kk, vv, 0.7, causal)
        ob, lb = _brute_force(qq.tolist(), kk.tolist(), vv.tolist(), 0.7, causal)
        if not (np.allclose(o, ob, atol=1e-12) and np.allclose(lse, lb, atol=1e-12)):
            failures += 1
    assert failures > 0, f"mutant {kind} passed every pin"


# --------------------------------------------------------------------------
# generator sanity (shared input module; holds no attention arithmetic)
# --------------------------------------------------------------------------

def test_generator_is_keyed_per_head_and_bf16_rounded():
    q, k, v = inputs.qkv(2, 2, 64, 16, seed=0)
    assert q.dtype == torch.bfloat16 and q.shape == (2, 2, 64, 16)
    h = inputs.head_bf16(0, "k", 1, 0, 64, 16)
    assert torch.equal(h, k[1, 0])
    q2, _, _ = inputs.qkv(2, 2, 64, 16, seed=1)
    assert not torch.equal(q, q2)
    x = inputs.head_f32(0, "q", 0, 0, 256, 64)
    assert abs(float(x.mean())) < 0.05 and abs(float(x.std()) - 1) < 0.05


def test_generator_outliers():
    x = inputs.head_f32(0, "q", 0, 0, 8192, 128, outliers=True)
    big = np.abs(x) > 6
    frac = big.mean()
    assert 2e-4 < frac < 1.2e-3
    rows = inputs.sample_rows(8192, 64)
    assert len(rows) == 64 and rows[0] == 0 and rows[-1] == 8191 and 4096 in rows
    st = inputs.stratified_rows(65536, 256)
    assert len(st) == 256 and st[0] == 0 and st[-1] == 65535
