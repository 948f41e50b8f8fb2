"""The bounded-wait failure path, exercised without faulting the GPU: a kernel
waits on an mbarrier nothing arrives on, gives up after a short limit, records
its site in the device status word and returns; the context stays usable."""

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_tiled_attention_29_b200 as fa2
    assert fa2.fa2_debug_status(None) == 0
    st = fa2.fa2_selftest_timeout(None, 20_000_000)  # 20 ms
    assert st == 0
    code = fa2.fa2_debug_status(None)
    assert code >> 16 == fa2.FA2_SITE_SELFTEST, hex(code)
    assert fa2.fa2_debug_status(None) == 0  # reading resets it
    # the context still runs real work afterwards
    q = torch.randn(1, 130, 2, 64, device="cuda").bfloat16()
    k = torch.randn(1, 130, 2, 64, device="cuda").bfloat16()
    o, lse = fa2.attention(q, k, k, causal=True)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    assert fa2.fa2_debug_status(None) == 0


def test_selftest_rejects_out_of_range_limits():
    import exact_tiled_attention_29_b200 as fa2
    assert fa2.fa2_selftest_timeout(None, 10) == 8
    assert fa2.fa2_selftest_timeout(None, 10**12) == 8
