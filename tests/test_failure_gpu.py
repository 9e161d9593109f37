"""Device-side failure detection without a GPU fault: a bounded wait on a
barrier that nothing completes gives up, records EVO_ERR_TIMEOUT, and the
context stays usable for the next forward call."""
import pytest
import torch

import oracle
import triangle_biased_attention_b200 as evo
from triangle_biased_attention_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_only():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    evo.load_library()


def test_bounded_wait_reports_timeout_and_context_survives():
    assert evo.evo_attn_sync_status() == evo.EVO_OK
    result = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    assert evo.evo_attn_selftest_timeout(20_000_000, result.data_ptr()) == evo.EVO_OK  # 20 ms
    assert evo.evo_attn_sync_status() == evo.EVO_ERR_TIMEOUT
    assert result.item() == 0
    assert evo.evo_attn_sync_status() == evo.EVO_OK  # cleared by the previous read
    # the context is still good: a forward pass after the timeout is correct
    case = W.random_case(1, 2, 136, 2, 32, torch.bfloat16, seed=5, mask="tail", pair=True)
    dev = torch.device("cuda", 0)
    o, lse = evo.evo_attn(case.q.to(dev), case.k.to(dev), case.v.to(dev), case.mask.to(dev), case.pair.to(dev))
    assert evo.evo_attn_sync_status() == evo.EVO_OK
    o_ref, lse_ref = oracle.attention(case.q, case.k, case.v, case.mask, case.pair)
    parity.check(o.cpu(), lse.cpu(), o_ref, lse_ref, torch.bfloat16, "after timeout")


def test_status_follows_the_stream_device():
    """evo_attn_sync_status reads the status word of the stream's device.  On
    a box with one GPU this covers a side stream and the legacy default stream
    of the current device; with two or more it also launches on device 1
    while device 0 is current and reads the timeout back through device 1's
    stream."""
    side = torch.cuda.Stream()
    result = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    assert evo.evo_attn_selftest_timeout(5_000_000, result.data_ptr(), side.cuda_stream) == evo.EVO_OK
    assert evo.evo_attn_sync_status(side.cuda_stream) == evo.EVO_ERR_TIMEOUT
    assert evo.evo_attn_sync_status(None) == evo.EVO_OK
    if torch.cuda.device_count() < 2:
        return
    torch.cuda.set_device(0)
    other = torch.cuda.Stream(device=1)
    result1 = torch.full((1,), 7, dtype=torch.int32, device="cuda:1")
    assert evo.evo_attn_selftest_timeout(5_000_000, result1.data_ptr(), other.cuda_stream) == evo.EVO_OK
    assert torch.cuda.current_device() == 0
    assert evo.evo_attn_sync_status(other.cuda_stream) == evo.EVO_ERR_TIMEOUT
    assert torch.cuda.current_device() == 0
    assert evo.evo_attn_sync_status(other.cuda_stream) == evo.EVO_OK
