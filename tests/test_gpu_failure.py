"""GPU: failure detection without a fault.  A bounded wait that nothing completes
gives up after its limit, the status word reports ATTN_DEV_TIMEOUT, and the context
still computes correct results afterwards."""

import math
import time

import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

kv = pytest.importorskip("kv_cache_decode_attn_b200")
from tests.gpu_util import check_lse, check_o, f64  # noqa: E402


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kv.attn_get_device_status(clear=True)
    yield
    kv.attn_get_device_status(clear=True)


def test_bounded_wait_gives_up_and_reports_timeout():
    t0 = time.monotonic()
    kv.attn_selftest_wait_timeout()
    status = kv.attn_get_device_status(clear=True)          # synchronises
    elapsed = time.monotonic() - t0
    assert status == kv.ATTN_DEV_TIMEOUT
    assert 1.0 < elapsed < 30.0                               # the 2 s limit, not an endless wait
    # the context is still usable: a small prefill matches the oracle, with a clean status
    B, Hq, Hkv, N, d = 1, 4, 2, 200, 64
    q, k, v = synth.prefill_inputs(B, Hq, Hkv, N, d, seed=3, device="cuda")
    o = torch.empty(B, N, Hq, d, device="cuda")
    lse = torch.empty(B, Hq, N, device="cuda")
    kv.attn_prefill(q, k, v, o, lse, scale=1 / math.sqrt(d), causal=True)
    o_ref, lse_ref = oracle.prefill(f64(q), f64(k), f64(v), 1 / math.sqrt(d), True)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)
    assert kv.attn_get_device_status(clear=True) == 0
