"""Failure detection without a GPU fault: a bounded wait that runs out.

The attention kernels never spin forever: every mbarrier wait gives up after a
time limit, records a code in the device error word and returns.  The library's
diagnostic entry point runs that same wait on a barrier nothing completes (with
a short limit); the host must then read code 1, the word must clear on read, and
the context must stay usable for a normal call."""
import ctypes
import math

import pytest
import torch

import oracle
from exact_attention_gqa_b200 import _capi, build, gqa_attn, gqa_attn_get_device_error
from parity import compare

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives():
    build.build()
    lib = _capi.load()
    assert gqa_attn_get_device_error() == 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.gqa_attn_selftest_timeout(20, stream) == 0
    torch.cuda.synchronize()
    assert gqa_attn_get_device_error() == 1       # kDevWaitTimeout
    assert gqa_attn_get_device_error() == 0       # read clears it
    assert lib.gqa_attn_selftest_timeout(0, stream) != 0   # limit out of range
    # the context is intact: a normal call still matches the oracle
    g = torch.Generator().manual_seed(3)
    q = torch.randn(1, 130, 8, 64, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 130, 2, 64, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 130, 2, 64, generator=g).to(torch.bfloat16)
    out, lse = gqa_attn(q.cuda(), k.cuda(), v.cuda(), causal=True)
    torch.cuda.synchronize()
    compare(out, lse, *oracle.attention(q, k, v, scale=1 / math.sqrt(64), causal=True))
    assert gqa_attn_get_device_error() == 0
