"""Failure detection on the GPU without a fault: a bounded wait that nothing
satisfies must give up, report MOBA_ERR_TIMEOUT through the status word and
leave the context usable for the next forward."""
import pytest
import torch

import long_context_prefill_block_b200 as moba
from moba_inputs import small_case
from parity import check_forward

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    moba.moba_device_status()  # clear
    assert moba.moba_selftest_bounded_wait() == 2
    assert moba.moba_device_status(clear=True) == moba.MOBA_ERR_TIMEOUT
    assert moba.moba_device_status() == 0
    q, k, v, cu = small_case((512, 300), 2, 1, 128, 128, 3, dtype=torch.bfloat16, seed=77)
    out = moba.moba_forward(q.cuda(), k.cuda(), v.cuda(), cu, 128, 3)
    assert moba.moba_device_status() == 0
    check_forward(q, k, v, cu, 128, 3, out)
