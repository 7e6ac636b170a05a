"""Canary checks of the outputs: every output buffer is filled with NaN (or
the e4m3 NaN code) before the call, so an element a kernel forgets to write
shows up, and an output view inside a larger NaN-filled buffer shows any
write outside the view.  These stand in for an uninitialised-memory checker."""

import math

import pytest
import torch

from io_aware_attention_02_b200 import inputs

pytestmark = pytest.mark.gpu

NAN = float("nan")


def _nan_like(t, dtype=None):
    return torch.full(t.shape, NAN, dtype=dtype or t.dtype, device=t.device)


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 1, 1, 64, False), (2, 3, 129, 128, True), (1, 2, 1000, 96, False),
                                            (2, 2, 300, 256, True), (1, 3, 257, 40, True)])
def test_forward_writes_every_output(lib, B, H, N, d, causal):
    q, k, v = (t.cuda() for t in inputs.qkv(B, H, N, d, seed=N + d))
    o = _nan_like(q)
    lse = torch.full((B, H, N), NAN, dtype=torch.float32, device="cuda")
    lib.fwd(q, k, v, causal=causal, out=o, lse=lse)
    o_ref, l_ref = lib.fwd(q, k, v, causal=causal)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    assert lib.last_status()[0] == 0


@pytest.mark.parametrize("d,N", [(64, 300), (96, 130), (128, 77)])
def test_strided_forward_writes_only_its_view(lib, d, N):
    """O written as a [B, N, H, d] view of a [B, N, H, d + 8] buffer: the
    view is filled in, the 8 padding columns of every row stay NaN."""
    B, H = 2, 3
    q, k, v = (t.cuda() for t in inputs.qkv(B, H, N, d, seed=d))
    buf = torch.full((B, N, H, d + 8), NAN, dtype=q.dtype, device="cuda")
    view = buf[..., :d].transpose(1, 2)
    lib.fwd(q, k, v, out=view)
    o_ref, _ = lib.fwd(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(view, o_ref)
    assert torch.isnan(buf[..., d:].float()).all()


@pytest.mark.parametrize("Nq,Nk,d,causal", [(1, 1000, 128, True), (7, 300, 64, False), (130, 600, 128, True)])
def test_splitkv_writes_every_output(lib, Nq, Nk, d, causal):
    B, H = 2, 2
    q = torch.stack([torch.stack([inputs.head_bf16(1, "q", b, h, Nq, d) for h in range(H)]) for b in range(B)]).cuda()
    k = torch.stack([torch.stack([inputs.head_bf16(1, "k", b, h, Nk, d) for h in range(H)]) for b in range(B)]).cuda()
    v = torch.stack([torch.stack([inputs.head_bf16(1, "v", b, h, Nk, d) for h in range(H)]) for b in range(B)]).cuda()
    o = _nan_like(q)
    lse = torch.full((B, H, Nq), NAN, dtype=torch.float32, device="cuda")
    ws_bytes = int(lib.lib().attn_fwd_splitkv_workspace_bytes(B, H, Nq, d, 3))
    ws = torch.full((max(ws_bytes, 16),), 0xFF, dtype=torch.uint8, device="cuda")   # NaN bit patterns
    lib.fwd_splitkv(q, k, v, causal=causal, n_splits=3, out=o, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    assert lib.last_status()[0] == 0


@pytest.mark.parametrize("det", [False, True])
@pytest.mark.parametrize("N,d,causal", [(1, 64, False), (300, 128, True), (129, 64, True)])
def test_backward_writes_every_gradient(lib, det, N, d, causal):
    B, H = 2, 2
    q, k, v = (t.cuda() for t in inputs.qkv(B, H, N, d, seed=N))
    do = inputs.grad_out(B, H, N, d, seed=N).cuda()
    o, lse = lib.fwd(q, k, v, causal=causal)
    dq, dk, dv = _nan_like(q), _nan_like(q), _nan_like(q)
    lib.bwd(q, k, v, o, do, lse, causal=causal, dq=dq, dk=dk, dv=dv, deterministic=det)
    torch.cuda.synchronize()
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    assert lib.last_status()[0] == 0


def test_fp8_path_writes_every_output(lib):
    B, H, N, d = 2, 2, 300, 128
    q, k, v = (t.cuda() for t in inputs.qkv(B, H, N, d, seed=3, outliers=True))
    nb = (N + 127) // 128
    outs = []
    for x, rot in ((q, True), (k, True), (v, False)):
        codes = torch.full(x.shape, 0xFF, dtype=torch.uint8, device="cuda")      # the e4m3 NaN code
        desc = torch.full((B, H, nb), NAN, dtype=torch.float32, device="cuda")
        signs = torch.from_numpy(inputs.hadamard_signs(d, seed=1)) if rot else None
        lib.quant_fp8(x, hadamard=rot, signs=signs, out=codes, descale=desc)
        outs.append((codes, desc))
    o = torch.full((B, H, N, d), NAN, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H, N), NAN, dtype=torch.float32, device="cuda")
    (q8, qd), (k8, kd), (v8, vd) = outs
    lib.fwd_fp8(q8, k8, v8, qd, kd, vd, out=o, lse=lse)
    torch.cuda.synchronize()
    for codes, desc in outs:
        # finite inputs give no NaN code (0x7F / 0xFF) under saturating rounding
        assert not ((codes & 0x7F) == 0x7F).any()
        assert torch.isfinite(desc).all()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    assert lib.last_status()[0] == 0


def test_host_forward_writes_every_output(lib):
    B, H, N, d = 2, 5, 333, 64
    q, k, v = (t.pin_memory() for t in inputs.qkv(B, H, N, d, seed=9))
    o = torch.full(q.shape, NAN, dtype=q.dtype).pin_memory()
    lse = torch.full((B, H, N), NAN, dtype=torch.float32).pin_memory()
    lib.fwd_host(q, k, v, causal=True, scale=1 / math.sqrt(d), out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
