"""attn_fwd_noalloc: the forward for callers that cannot let the library
allocate device memory -- a process whose device memory belongs to a pool
allocator or another runtime, or code running where cudaMalloc is not allowed.
Its only scratch (the record its bounded waits write on a timeout) is a static
device array inside the library, read back with attn_noalloc_last_status.

Checked through the C ABI: outputs bit-identical to attn_fwd (same kernel,
same schedule) on two calls in a row; a timeout made on the host side (the
producer told to skip one copy, 50 ms wait limit) reaches the shared record
and not attn_fwd's status word; and, in a fresh process, noalloc calls leave
attn_fwd's status word unallocated.  Kept in a file that pytest collects
last."""

import os
import subprocess
import sys
import textwrap

import pytest
import torch

from io_aware_attention_02_b200 import inputs

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_noalloc_matches_attn_fwd_on_two_calls_in_a_row(lib):
    cases = [(2, 3, 700, 128, False, torch.bfloat16, 1), (1, 4, 333, 64, True, torch.float16, 2)]
    for B, H, N, d, causal, dt, seed in cases:
        q, k, v = (t.cuda() for t in inputs.qkv(B, H, N, d, seed=seed, dtype=dt))
        o_ref, l_ref = lib.fwd(q, k, v, causal=causal)
        for _ in range(2):
            o_na, l_na = lib.fwd_noalloc(q, k, v, causal=causal)
            torch.cuda.synchronize()
            assert torch.equal(o_na, o_ref)
            assert torch.equal(l_na, l_ref)
        assert lib.noalloc_last_status()[0] == lib.ATTN_OK
    assert lib.last_status()[0] == lib.ATTN_OK


def test_noalloc_timeout_is_reported_in_its_own_record(lib):
    q, k, v = (t.cuda() for t in inputs.qkv(1, 2, 512, 64, seed=22))
    assert lib.noalloc_last_status()[0] == lib.ATTN_OK
    lib.debug_set_fault(1, wait_limit_ms=50)
    lib.fwd_noalloc(q, k, v)
    code, where = lib.noalloc_last_status()
    assert code == lib.ATTN_ERR_TIMEOUT, (code, where)
    assert where[1] == 0                         # CTA 0 was the one told to skip
    assert lib.last_status()[0] == lib.ATTN_OK   # attn_fwd's word never saw it
    # the reader cleared the record, and the next call is clean and exact
    assert lib.noalloc_last_status()[0] == lib.ATTN_OK
    o_na, l_na = lib.fwd_noalloc(q, k, v)
    o_ref, l_ref = lib.fwd(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(o_na, o_ref) and torch.equal(l_na, l_ref)
    assert lib.noalloc_last_status()[0] == lib.ATTN_OK


def test_noalloc_rejects_bad_arguments(lib):
    x = torch.zeros(1, 1, 64, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.AttnError) as e:
        lib.fwd_noalloc(x, x, x)
    assert e.value.code == lib.ATTN_ERR_UNSUPPORTED


def test_noalloc_allocates_nothing_in_a_fresh_process(lib):
    """A process whose first library calls are noalloc ones: attn_fwd's
    status word (the library's only allocation) must still not exist."""
    code = textwrap.dedent("""
        import sys, torch
        sys.path.insert(0, %r)
        from io_aware_attention_02_b200 import binding, inputs
        torch.cuda.set_device(0)
        q, k, v = (t.cuda() for t in inputs.qkv(1, 2, 300, 128, seed=3))
        torch.cuda.synchronize()
        o1, l1 = binding.fwd_noalloc(q, k, v)
        o2, l2 = binding.fwd_noalloc(q, k, v)
        assert binding.noalloc_last_status()[0] == binding.ATTN_OK
        assert binding.debug_status_allocated() == 0, "noalloc path allocated"
        o3, l3 = binding.fwd(q, k, v)
        torch.cuda.synchronize()
        assert binding.debug_status_allocated() == 1
        assert torch.equal(o1, o3) and torch.equal(o2, o3) and torch.equal(l1, l3)
        print("fresh-process noalloc ok")
    """) % ROOT
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "fresh-process noalloc ok" in r.stdout
