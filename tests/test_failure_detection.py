"""Failure detection without a GPU fault: every wait in the kernels is
bounded, records an error code and raises the CTA's abort flag when it gives
up, and the other waits of the CTA then leave promptly.  The self-test entry
point waits on mbarriers that nothing completes (a flag nothing sets), so the
limit runs out on purpose; the context stays usable afterwards."""
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    import torch
    from sink_sliding_window_b200 import build, ops as _ops
    assert torch.cuda.is_available()
    build.build()
    return _ops

SELFTEST_TIMEOUT = 0x107        # the wait meant to give up
SELFTEST_TIMEOUT_ABORT = 0x108  # the wait meant to leave through the abort flag


def test_bounded_wait_gives_up_and_aborts_the_block(ops):
    import torch
    limit_ns = 2_000_000  # 2 ms
    vals, code = ops.selftest_wait(limit_ns)
    first_ok, first_us, second_ok, second_us = vals
    assert first_ok == 0 and second_ok == 0
    assert code == SELFTEST_TIMEOUT  # recorded once, by the wait that ran out
    assert 2000 <= first_us < 200_000
    # The second wait had 20 ms; it left through the abort flag soon after.
    assert second_us < 10 * limit_ns // 1000
    assert ops.device_error() == 0  # read and cleared
    # The context is still usable: a small forward runs and reports no error.
    q = torch.randn(128, 4, 64, device="cuda").to(torch.bfloat16)
    k = torch.randn(128, 1, 64, device="cuda").to(torch.bfloat16)
    v = torch.randn(128, 1, 64, device="cuda").to(torch.bfloat16)
    s = torch.zeros(4, device="cuda")
    out, lse = ops.fwd(q, k, v, s, None, 0, 0.125, batch=1, max_seqlen=128)
    torch.cuda.synchronize()
    assert ops.device_error() == 0
    assert torch.isfinite(out.float()).all()


def test_selftest_rejects_bad_arguments(ops):
    import torch
    out = torch.zeros(4, dtype=torch.int32, device="cuda")
    with pytest.raises(ops.SinkAttnError):
        ops.selftest_wait(0, out)
    with pytest.raises(ops.SinkAttnError):
        ops.selftest_wait(2_000_000_000, out)
