"""attn_fwd_noalloc: the entry point for callers that cannot allocate device
memory (a pool-owned device, or a point where cudaMalloc is forbidden).  Its
kernel scratch is a static device array inside the library.  Checked through
the C ABI against attn_fwd on two calls in a row, with the tolerances the
other parity tests use.  Kept in a file that pytest collects last."""

import pytest
import torch

from io_aware_attention_02_b200 import inputs
from parity_util import BF16_MAX_ABS, LSE_MAX_ABS

pytestmark = pytest.mark.gpu


def test_noalloc_matches_attn_fwd_on_two_calls_in_a_row(lib):
    cases = [(2, 3, 700, 128, False, torch.bfloat16, 1), (1, 4, 333, 64, True, torch.float16, 2)]
    for B, H, N, d, causal, dt, seed in cases:
        q, k, v = (t.cuda() for t in inputs.qkv(B, H, N, d, seed=seed, dtype=dt))
        o_na, l_na = lib.fwd_noalloc(q, k, v, causal=causal)
        o_ref, l_ref = lib.fwd(q, k, v, causal=causal)
        torch.cuda.synchronize()
        assert float((o_na.float() - o_ref.float()).abs().max()) <= BF16_MAX_ABS
        assert float((l_na - l_ref).abs().max()) <= LSE_MAX_ABS
        assert torch.isfinite(o_na).all()
    assert lib.last_status()[0] == 0


def test_noalloc_rejects_bad_arguments(lib):
    x = torch.zeros(1, 1, 64, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.AttnError) as e:
        lib.fwd_noalloc(x, x, x)
    assert e.value.code == lib.ATTN_ERR_UNSUPPORTED
