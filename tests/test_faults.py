"""Bounded waits: a launch whose producer skips one load must end with
ATTN_ERR_TIMEOUT in the status word -- no hang, no trap -- and the context
must stay usable.  The failure is made on the host side of the kernel's
protocol (a test hook tells the producer not to issue one copy); nothing
faults the GPU."""

import pytest
import torch

from io_aware_attention_02_b200 import inputs
from parity_util import assert_bf16_ok, run_and_compare

pytestmark = pytest.mark.gpu


def test_timeout_is_reported_and_context_survives(lib):
    q, k, v = (t.cuda() for t in inputs.qkv(1, 2, 512, 64, seed=20))
    assert lib.last_status()[0] == 0
    lib.debug_set_fault(1, wait_limit_ms=50)
    o, lse = lib.fwd(q, k, v)
    code, where = lib.last_status()
    assert code == lib.ATTN_ERR_TIMEOUT, (code, where)
    assert where[1] == 0            # CTA 0 was the one told to skip
    # hook is one-shot: the next call is clean and correct
    err, _ = run_and_compare(lib, 1, 2, 512, 64, False, seed=20)
    assert_bf16_ok(err, "after timeout")
    assert lib.last_status()[0] == 0


def test_timeout_on_fp8_path(lib):
    x = inputs.qkv(1, 1, 256, 128, seed=21)[0].cuda()
    q8, qd = lib.quant_fp8(x)
    lib.debug_set_fault(1, wait_limit_ms=50)
    lib.fwd_fp8(q8, q8, q8, qd, qd, qd)
    assert lib.last_status()[0] == lib.ATTN_ERR_TIMEOUT
    lib.fwd_fp8(q8, q8, q8, qd, qd, qd)
    assert lib.last_status()[0] == 0
