"""GPU parity of the backward kernels (attn_bwd) against the fp64 oracle's
gradients, called through the C ABI on seeded synthetic inputs.

Tolerance, from the kernel's rounding: P and dS are rounded to the input
dtype before the products that use them and every output is rounded to it
once, so each gradient carries about two bf16 roundings (unit roundoff
2^-9, i.e. ~1.1e-3 RMS relative each).  A CPU model of exactly those
roundings (tests/test_backward_tolerance.py) gives an RMSE of 2.2e-3 to
3.0e-3 of the gradient's RMS and a maximum error of 1.8e-3 to 6.5e-3 of its
largest entry (N 300 to 1000, d 64 and 128, causal and not, both modes).
The bounds below are about three times that.
"""

import math

import numpy as np
import pytest
import torch

from io_aware_attention_02_b200 import inputs
from oracle import backward as BK

pytestmark = pytest.mark.gpu

REL_RMSE = 1e-2        # RMSE / RMS(oracle)
REL_MAX = 2e-2         # max |error| / max |oracle|
# Gradients that vanish exactly (N = 1: dQ = dK = 0) are compared against
# these floors instead: the natural size of a gradient entry here is 0.05-1.
RMS_FLOOR = 1e-3
MAX_FLOOR = 1e-2


def _grad_errors(got, ref):
    g = got.detach().to("cpu", torch.float64).numpy()
    dif = g - ref
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return {"rel_rmse": float(np.sqrt(np.mean(dif ** 2))) / max(rms, RMS_FLOOR),
            "rel_max": float(np.abs(dif).max()) / max(float(np.abs(ref).max()), MAX_FLOOR),
            "finite": bool(np.isfinite(g).all())}


def _assert_ok(err, what):
    assert err["finite"], (what, err)
    assert err["rel_rmse"] <= REL_RMSE, (what, err)
    assert err["rel_max"] <= REL_MAX, (what, err)


def _run(lib, B, H, N, d, causal, dtype=torch.bfloat16, seed=0, scale=None, heads=None, deterministic=False):
    q, k, v = inputs.qkv(B, H, N, d, seed=seed, dtype=dtype)
    do = inputs.grad_out(B, H, N, d, seed=seed, dtype=dtype)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = lib.fwd(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = lib.bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=scale, deterministic=deterministic)
    torch.cuda.synchronize()
    code, where = lib.last_status()
    assert code == 0, where
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    out = []
    for b, h in heads:
        ref = BK.attention_backward_head(q[b, h], k[b, h], v[b, h], do[b, h], scale, causal)
        for name, got, r in zip(("dq", "dk", "dv"), (dq[b, h], dk[b, h], dv[b, h]), ref):
            out.append(((b, h, name), _grad_errors(got, r)))
    return out, (dq, dk, dv)


MODES = [pytest.param(False, id="fused"), pytest.param(True, id="deterministic")]


@pytest.mark.parametrize("det", MODES)
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 7, 100, 128, 129, 256, 257, 500])
def test_ragged_and_multi_tile(lib, d, causal, N, det):
    errs, _ = _run(lib, 1, 2, N, d, causal, seed=N, deterministic=det)
    for what, e in errs:
        _assert_ok(e, (N, d, causal, det, what))


@pytest.mark.parametrize("det", MODES)
@pytest.mark.parametrize("causal", [False, True])
def test_single_token_closed_form(lib, causal, det):
    """N = 1: P = 1, so dV = dO and dS = dO.v - dO.O = 0, hence dQ = dK = 0.

    dV is exact (P = 1 is exact in 16 bits).  dQ and dK vanish up to the
    difference of two fp32 sums of the same 128 products, dO.v by the tensor
    cores and dO.O by the row threads (|dO.v| reaches ~40 here, and the
    tensor-core sum is not correctly rounded), times scale * K: 2e-3 bounds
    that with room, against gradient entries of size 0.1 to 1 otherwise."""
    q, k, v = (t.cuda() for t in inputs.qkv(2, 3, 1, 128, seed=8))
    do = inputs.grad_out(2, 3, 1, 128, seed=8).cuda()
    o, lse = lib.fwd(q, k, v, causal=causal)
    dq, dk, dv = lib.bwd(q, k, v, o, do, lse, causal=causal, deterministic=det)
    torch.cuda.synchronize()
    assert torch.equal(dv, do)
    assert dq.abs().max().item() <= 2e-3 and dk.abs().max().item() <= 2e-3


@pytest.mark.parametrize("det", MODES)
@pytest.mark.parametrize("d", [8, 40, 96, 120])
@pytest.mark.parametrize("causal", [False, True])
def test_head_dims_padded(lib, d, causal, det):
    """Head dims below 128 that are not 64 or 128 run zero-padded."""
    errs, _ = _run(lib, 1, 2, 333, d, causal, seed=d, deterministic=det)
    for what, e in errs:
        _assert_ok(e, ("d", d, causal, what))


@pytest.mark.parametrize("det", MODES)
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_fp16(lib, d, causal, det):
    errs, _ = _run(lib, 2, 2, 300, d, causal, dtype=torch.float16, seed=9, deterministic=det)
    for what, e in errs:
        _assert_ok(e, ("fp16", d, causal, what))


@pytest.mark.parametrize("det", MODES)
@pytest.mark.parametrize("d", [64, 128])
def test_many_heads_wrap_the_persistent_grid(lib, d, det):
    """More work units than SMs: every CTA runs several units."""
    errs, _ = _run(lib, 3, 40, 256, d, True, seed=3, heads=[(0, 0), (1, 17), (2, 39)], deterministic=det)
    for what, e in errs:
        _assert_ok(e, what)


@pytest.mark.parametrize("det", MODES)
def test_scale_other_than_inverse_sqrt_d(lib, det):
    errs, _ = _run(lib, 1, 2, 200, 128, False, seed=4, scale=0.3, deterministic=det)
    for what, e in errs:
        _assert_ok(e, ("scale 0.3", what))


@pytest.mark.parametrize("det", MODES)
@pytest.mark.parametrize("causal", [False, True])
def test_long_sequence_heads(lib, causal, det):
    """N = 4096, d = 128: two heads of a four-head call, every entry."""
    errs, _ = _run(lib, 1, 4, 4096, 128, causal, seed=11, heads=[(0, 0), (0, 3)], deterministic=det)
    for what, e in errs:
        _assert_ok(e, ("4096", causal, what))


@pytest.mark.parametrize("det", MODES)
def test_repeatable_and_workspace_contents_irrelevant(lib, det):
    """Deterministic mode: bit-identical outputs.  Fused mode: dK and dV
    bit-identical (no atomics there), dQ within fp32 summation-order noise.
    A workspace filled with NaN bit patterns changes nothing."""
    B, H, N, d = 2, 3, 700, 128
    q, k, v = (t.cuda() for t in inputs.qkv(B, H, N, d, seed=21))
    do = inputs.grad_out(B, H, N, d, seed=21).cuda()
    o, lse = lib.fwd(q, k, v, causal=True)
    ws = torch.full((lib.bwd_workspace_bytes(B, H, N, d, det),), 0xFF, dtype=torch.uint8, device="cuda")
    a = lib.bwd(q, k, v, o, do, lse, causal=True, workspace=ws, deterministic=det)
    b = lib.bwd(q, k, v, o, do, lse, causal=True, deterministic=det)
    torch.cuda.synchronize()
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    if det:
        assert torch.equal(a[0], b[0])
    else:
        assert torch.isfinite(a[0].float()).all()
        assert (a[0].float() - b[0].float()).abs().max().item() <= 1e-2 * b[0].float().abs().max().item()


def test_fused_and_deterministic_paths_agree(lib):
    """The two paths agree to their rounding differences: the fused path
    computes dS from the 16-bit P it hands to dV (one more rounding of P,
    unit roundoff 2^-9) and sums dQ in another order; both are separately
    within the oracle bar above.  Bound: 1e-2 of the norm (measured 3.6e-3)."""
    B, H, N, d = 1, 4, 1000, 64
    q, k, v = (t.cuda() for t in inputs.qkv(B, H, N, d, seed=31))
    do = inputs.grad_out(B, H, N, d, seed=31).cuda()
    o, lse = lib.fwd(q, k, v, causal=False)
    a = lib.bwd(q, k, v, o, do, lse, deterministic=False)
    b = lib.bwd(q, k, v, o, do, lse, deterministic=True)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        rel = ((x.float() - y.float()).norm() / y.float().norm()).item()
        assert rel <= 1e-2, rel


def test_outputs_past_the_last_row_untouched(lib):
    """dQ, dK, dV are written for rows < N only: guard rows after the tensor
    (inside one allocation) keep their contents."""
    B, H, N, d = 1, 1, 130, 64
    q, k, v = (t.cuda() for t in inputs.qkv(B, H, N, d, seed=2))
    do = inputs.grad_out(B, H, N, d, seed=2).cuda()
    o, lse = lib.fwd(q, k, v)
    outs = []
    for _ in range(3):
        buf = torch.full((B * H * N * d + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
        outs.append(buf)
    views = [buf[:B * H * N * d].view(B, H, N, d) for buf in outs]
    for det in (False, True):
        lib.bwd(q, k, v, o, do, lse, dq=views[0], dk=views[1], dv=views[2], deterministic=det)
        torch.cuda.synchronize()
        for buf in outs:
            assert torch.all(buf[B * H * N * d:] == 7.0)


def test_bad_arguments_raise(lib):
    x = torch.zeros(1, 1, 128, 256, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 1, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(lib.AttnError):
        lib.bwd(x, x, x, x, x, lse)
    y = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        lib.bwd(y, y, y, y, y, lse[..., :64])
