"""Shared helpers for the GPU parity tests: run the CUDA path through the
binding, run the oracle on the same seeded inputs, compare with the stated
tolerances."""

import math

import numpy as np
import torch

from io_aware_attention_02_b200 import inputs
from oracle import attention as A

# Acceptance tolerances against the fp64 oracle.
BF16_MAX_ABS = 2e-2
BF16_RMSE = 3e-3
LSE_MAX_ABS = 1e-3
FP8_RMSE = 2.5e-2


def errors(o_gpu, lse_gpu, o_ref, lse_ref):
    o = o_gpu.detach().to("cpu", torch.float64).numpy() if torch.is_tensor(o_gpu) else np.asarray(o_gpu)
    dif = o - o_ref
    out = {"max_abs": float(np.abs(dif).max()), "rmse": float(np.sqrt(np.mean(dif ** 2)))}
    if lse_gpu is not None and lse_ref is not None:
        l = lse_gpu.detach().to("cpu", torch.float64).numpy() if torch.is_tensor(lse_gpu) else np.asarray(lse_gpu)
        out["lse_max_abs"] = float(np.abs(l - lse_ref).max())
    return out


def assert_bf16_ok(err, what=""):
    assert err["max_abs"] <= BF16_MAX_ABS, (what, err)
    assert err["rmse"] <= BF16_RMSE, (what, err)
    if "lse_max_abs" in err:
        assert err["lse_max_abs"] <= LSE_MAX_ABS, (what, err)


def oracle_rows(q, k, v, scale, causal, rows=None, heads=None):
    """Oracle over all (b, h) (or the listed (b, h) pairs) for the given rows.

    Returns (O [len(heads), R, d], LSE [len(heads), R]).
    """
    B, H = q.shape[0], q.shape[1]
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    os_, ls = [], []
    for b, h in heads:
        o, l = A.attention_head(q[b, h], k[b, h], v[b, h], scale, causal, rows)
        os_.append(o)
        ls.append(l)
    return np.stack(os_), np.stack(ls)


def run_and_compare(lib, B, H, N, d, causal, dtype=torch.bfloat16, seed=0, rows=None, heads=None,
                    scale=None):
    q, k, v = inputs.qkv(B, H, N, d, seed=seed, dtype=dtype)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o, lse = lib.fwd(qd, kd, vd, causal=causal, scale=scale)
    torch.cuda.synchronize()
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    o_ref, l_ref = oracle_rows(q, k, v, scale, causal, rows, heads)
    r = slice(None) if rows is None else rows
    o_g = torch.stack([o[b, h][r] for b, h in heads]).cpu()
    l_g = torch.stack([lse[b, h][r] for b, h in heads]).cpu()
    return errors(o_g, l_g, o_ref, l_ref), (o, lse)
