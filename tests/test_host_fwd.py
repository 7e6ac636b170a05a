"""GPU tests of attn_fwd_host (host buffers, transfers overlapped with the
computation in head chunks): its outputs must be bit-identical to attn_fwd
on the same inputs (same kernel, same per-head work), and it is checked
against the fp64 oracle once."""

import math

import numpy as np
import pytest
import torch

from io_aware_attention_02_b200 import inputs
from parity_util import assert_bf16_ok, errors, oracle_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 1, 1, 64, False), (1, 3, 300, 128, True), (2, 5, 1000, 64, False),
                                            (4, 16, 512, 128, True), (1, 7, 257, 256, False), (3, 2, 640, 96, True)])
@pytest.mark.parametrize("pinned", [True, False])
def test_matches_device_forward_bitwise(lib, B, H, N, d, causal, pinned):
    q, k, v = inputs.qkv(B, H, N, d, seed=N + d)
    if pinned:
        q, k, v = (t.pin_memory() for t in (q, k, v))
    o_h, l_h = lib.fwd_host(q, k, v, causal=causal)
    torch.cuda.synchronize()
    o_d, l_d = lib.fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o_h, o_d.cpu())
    assert torch.equal(l_h, l_d.cpu())
    code, where = lib.last_status()
    assert code == 0, where


def test_against_the_oracle(lib):
    q, k, v = (t.pin_memory() for t in inputs.qkv(2, 6, 700, 128, seed=3))
    o, l = lib.fwd_host(q, k, v, causal=True, scale=1 / math.sqrt(128))
    torch.cuda.synchronize()
    o_ref, l_ref = oracle_rows(q, k, v, 1 / math.sqrt(128), True)
    err = errors(o.reshape(12, 700, 128), l.reshape(12, 700), o_ref, l_ref)
    assert_bf16_ok(err, "host forward")


def test_fp16_no_lse_and_repeated_calls_share_the_workspace(lib):
    q, k, v = (t.pin_memory() for t in inputs.qkv(2, 4, 384, 64, seed=5, dtype=torch.float16))
    ws = torch.empty(int(lib.lib().attn_fwd_host_workspace_bytes(2, 4, 384, 64)), dtype=torch.uint8, device="cuda")
    outs = []
    for causal in (False, True, False):
        o, l = lib.fwd_host(q, k, v, causal=causal, workspace=ws, return_lse=False)
        outs.append(o)
        assert l is None
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[2])
    o_d, _ = lib.fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(outs[1], o_d.cpu())


def test_device_tensors_are_refused(lib):
    x = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        lib.fwd_host(x, x, x)
