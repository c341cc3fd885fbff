"""Failure detection on the GPU without a fault: with the device-side wait
limit set to 0, the attention kernel's first unsatisfied wait gives up; the
kernel drains its in-flight copies and MMAs, frees TMEM, exits and records
SEER_ERR_TIMEOUT, which seer_check_status reports.  The context stays usable:
the next call with the normal limit returns the exact result."""
import numpy as np
import pytest
import torch

import long_context_prefill_attngate_b200 as seer
from long_context_prefill_attngate_b200 import build as seer_build
from long_context_prefill_attngate_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", ["sparse", "map"])
def test_wait_timeout_is_reported_and_recoverable(mode):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    seer_build.build()
    seer.lib()
    w = syn.custom("timeout", 1, 8, 2, 4096, 128, number=71)
    x = syn.make_inputs(w)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    mask = syn.random_mask(1, 8, 64, 0.3, seed=3).cuda()

    def run():
        if mode == "sparse":
            return seer.seer_block_sparse_prefill(q, k, v, mask)
        return seer.seer_attn_pooled_map(q, k, v)[1]

    good = run()
    seer.seer_check_status()
    try:
        seer.seer_set_wait_timeout_ns(0)
        run()
        with pytest.raises(seer.SeerError) as e:
            seer.seer_check_status()
        assert e.value.status == seer.SEER_ERR_TIMEOUT
    finally:
        seer.seer_set_wait_timeout_ns(2_000_000_000)
    again = run()
    seer.seer_check_status()
    assert torch.equal(again, good)
