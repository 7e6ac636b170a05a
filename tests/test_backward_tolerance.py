"""Where the backward's GPU tolerance comes from (CPU only).

The backward kernels round P and dS to bf16 before the products that use
them, compute D = rowsum(dO * O) from the 16-bit O the forward returned, and
round every gradient to bf16 once; the fused mode also forms dS from the
rounded P.  This file replays exactly those roundings in fp64 (a model of
the kernels' arithmetic, not a copy of it) on the inputs the GPU tests use
and checks that the resulting error against the fp64 oracle stays well
inside the bars tests/test_backward.py applies to the GPU (1e-2 of the RMS,
2e-2 of the largest entry).  The model gives 2.2e-3 to 3.0e-3 of the RMS and
1.8e-3 to 6.5e-3 of the largest entry; the bars leave a factor of about
three on top for the order in which the kernels' fp32 sums are taken, which
this model does not capture."""

import math

import numpy as np
import pytest
import torch

from io_aware_attention_02_b200 import inputs
from oracle import backward as BK

REL_RMSE = 1e-2
REL_MAX = 2e-2


def _bf16(x):
    return x.to(torch.bfloat16).to(torch.float64)


def _model(q, k, v, do, scale, causal, fused):
    """The gradients with the kernels' roundings, fp64 elsewhere."""
    n = q.shape[0]
    s = scale * q @ k.T
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), -math.inf)
    p = torch.exp(s - torch.logsumexp(s, 1, keepdim=True))
    o = _bf16(_bf16(p) @ v)                      # the forward's 16-bit output
    dvec = (do * o).sum(1, keepdim=True)
    dp = do @ v.T
    ds = (_bf16(p) if fused else p) * (dp - dvec)
    dv = _bf16(_bf16(p).T @ do)
    dq = _bf16(scale * _bf16(ds) @ k)
    dk = _bf16(scale * _bf16(ds).T @ q)
    return dq, dk, dv


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("N,d,causal", [(300, 64, False), (300, 128, True), (1000, 128, False), (700, 128, True)])
def test_modelled_rounding_sits_well_inside_the_gpu_bar(fused, N, d, causal):
    q, k, v = (t[0, 0].double() for t in inputs.qkv(1, 1, N, d, seed=N))
    do = inputs.grad_out(1, 1, N, d, seed=N)[0, 0].double()
    scale = 1 / math.sqrt(d)
    ref = BK.attention_backward_head(q.numpy(), k.numpy(), v.numpy(), do.numpy(), scale, causal)
    got = _model(q, k, v, do, scale, causal, fused)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        dif = g.numpy() - r
        rel_rmse = np.sqrt(np.mean(dif ** 2)) / np.sqrt(np.mean(r ** 2))
        rel_max = np.abs(dif).max() / np.abs(r).max()
        assert rel_rmse <= REL_RMSE / 2.5, (name, rel_rmse)
        assert rel_max <= REL_MAX / 2.5, (name, rel_max)
        # and the model is not trivially exact: the roundings do show
        assert rel_rmse >= 1e-4, (name, rel_rmse)
