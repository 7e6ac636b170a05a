"""GPU runs of the debug build (every TMEM column range and shared-memory
byte range of the forward kernels checked before use; a failed check reports
ATTN_ERR_BOUNDS and skips the access) on small cases of each variant of the
two-tile kernel (head dims 64, 128) and the one-tile kernel (200 padded to
256, 256), bf16 and e4m3: no check fails, and the outputs are bit-identical
to the release build's on the same inputs."""

import math

import pytest
import torch

from io_aware_attention_02_b200 import binding, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dlib():
    from io_aware_attention_02_b200 import build
    build.build(debug=True)
    return binding.load_debug()


def _status(dl):
    where = (ctypes_int2())
    code = dl.attn_last_status(torch.cuda.current_stream().cuda_stream, where)
    return code, list(where)


def ctypes_int2():
    import ctypes
    return (ctypes.c_int * 2)()


def _fwd(l, q, k, v, causal):
    B, H, N, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    dt = binding.ATTN_BF16 if q.dtype == torch.bfloat16 else binding.ATTN_FP16
    code = l.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d,
                      1 / math.sqrt(d), int(causal), dt, torch.cuda.current_stream().cuda_stream)
    assert code == 0, code
    torch.cuda.synchronize()
    return o, lse


@pytest.mark.parametrize("d", [64, 128, 200, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 200, 700])
def test_bf16_debug_build_matches_release(lib, dlib, d, causal, N):
    q, k, v = (t.cuda() for t in inputs.qkv(2, 3, N, d, seed=N + d))
    o, lse = _fwd(binding.load(), q, k, v, causal)
    od, lsed = _fwd(dlib, q, k, v, causal)
    assert _status(dlib) == (0, [0, 0])
    assert torch.equal(o, od) and torch.equal(lse, lsed)


@pytest.mark.parametrize("d,vt", [(64, 0), (128, 0), (128, 1), (256, 0)])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_debug_build_matches_release(lib, dlib, d, vt, causal):
    N = 600
    q, k, v = (t.cuda() for t in inputs.qkv(1, 4, N, d, seed=d + vt, outliers=True))
    signs = torch.from_numpy(inputs.hadamard_signs(d, seed=1)).cuda()
    q8, qs = binding.quant_fp8(q, hadamard=True, signs=signs)
    k8, ks = binding.quant_fp8(k, hadamard=True, signs=signs)
    v8, vs = binding.quant_fp8(v)
    outs = []
    for l in (binding.load(), dlib):
        o = torch.empty_like(q)
        lse = torch.empty((1, 4, N), dtype=torch.float32, device=q.device)
        code = l.attn_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), qs.data_ptr(), ks.data_ptr(),
                              vs.data_ptr(), o.data_ptr(), lse.data_ptr(), 1, 4, N, d, 1 / math.sqrt(d),
                              int(causal), vt, torch.cuda.current_stream().cuda_stream)
        assert code == 0, code
        torch.cuda.synchronize()
        outs.append((o, lse))
    assert _status(dlib) == (0, [0, 0])
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_planted_range_failure_is_reported(lib, dlib):
    """Fault mode 2 makes CTA 0's first S-load range check fail (the load
    itself stays in range and is skipped): the debug build reports
    ATTN_ERR_BOUNDS with that check's id, and the next launch is clean."""
    q, k, v = (t.cuda() for t in inputs.qkv(1, 2, 300, 128, seed=3))
    assert dlib.attn_debug_set_fault(2, 0) == 0
    _fwd(dlib, q, k, v, False)
    code, where = _status(dlib)
    assert code == binding.ATTN_ERR_BOUNDS and where == [29, 0], (code, where)
    o, lse = _fwd(binding.load(), q, k, v, False)
    od, lsed = _fwd(dlib, q, k, v, False)
    assert _status(dlib) == (0, [0, 0])
    assert torch.equal(o, od) and torch.equal(lse, lsed)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(1, 1000), (200, 700)])
def test_splitkv_debug_build_matches_release(lib, dlib, d, causal, Nq, Nk):
    """The split-KV kernel's range checks (its Q tile, K/V ring, S buffers,
    O and P columns) on decode and prefill-against-cache shapes."""
    B, H = 2, 3
    g = torch.Generator().manual_seed(Nq + d)
    q = torch.randn(B, H, Nq, d, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(B, H, Nk, d, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, H, Nk, d, generator=g).to(torch.bfloat16).cuda()
    ns = 3
    ws_bytes = int(binding.load().attn_fwd_splitkv_workspace_bytes(B, H, Nq, d, ns))
    outs = []
    for l in (binding.load(), dlib):
        o = torch.empty_like(q)
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
        code = l.attn_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, Nq,
                                  Nk, d, 1 / math.sqrt(d), int(causal), ns, binding.ATTN_BF16, ws.data_ptr(),
                                  ws_bytes, torch.cuda.current_stream().cuda_stream)
        assert code == 0, code
        torch.cuda.synchronize()
        outs.append((o, lse))
    assert _status(dlib) == (0, [0, 0])
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
