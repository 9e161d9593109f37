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
    parity.check(o.cpu(), lse.cpu(), o_ref, lse_ref, torch.bfloat16, "after timeout", strict=False)
