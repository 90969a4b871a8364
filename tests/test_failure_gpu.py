"""Failure detection without a fault: a wait that nothing satisfies gives up after its
limit, the host reads FA_ERR_TIMEOUT, the error word is cleared by the report, and the
same context keeps computing correct results."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_64_b200 import binding, inputs
from parity import assert_bf16_close, to64

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_stays_usable():
    binding.check_device_error()  # start from a clear error word
    stream = torch.cuda.current_stream().cuda_stream
    assert binding.lib().fa_selftest_timeout(20_000_000, stream) == binding.FA_OK
    with pytest.raises(binding.FAError) as e:
        binding.check_device_error()
    assert e.value.status == binding.FA_ERR_TIMEOUT
    binding.check_device_error()  # the report cleared it
    ins = inputs.make_inputs(1, 2, 200, 64, seed=3)
    q, k, v = (ins[n].cuda() for n in ("Q", "K", "V"))
    O, _ = binding.fwd(q, k, v, causal=True)
    binding.check_device_error()
    for h in range(2):
        rO, _, _ = oracle.attention_head(to64(ins["Q"][0, h]), to64(ins["K"][0, h]),
                                         to64(ins["V"][0, h]), 0.125, True)
        assert_bf16_close(to64(O[0, h]), rO, f"after the timeout, head {h}")
