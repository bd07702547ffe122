"""Failure detection without a GPU fault.

Every internal wait of the tensor-core kernels is bounded; when one expires
the kernel records a code in the library's device error word and returns.
The self-test kernel waits on a barrier that nothing completes, so its wait
must run out; the host then reads LVX_ERR_DEVICE_TIMEOUT, and the CUDA
context must still run a normal attention call correctly afterwards.
"""

import pytest
import torch

from blockwise_long_context_b200 import binding as lvx
from blockwise_long_context_b200 import inputs


@pytest.mark.gpu
def test_expired_wait_is_reported_and_context_survives():
    lvx.lvx_last_device_error()                      # start from a clean error word
    lvx.lvx_selftest_wait_timeout()
    with pytest.raises(lvx.LvxError) as e:
        lvx.lvx_last_device_error()
    assert e.value.status == 5                        # LVX_ERR_DEVICE_TIMEOUT
    lvx.lvx_last_device_error()                      # reading cleared it
    # the context is still usable: a normal forward runs and matches a second run
    w = inputs.WORKLOADS["C1"].scaled(S_Q=256, S_KV=1024, H=2, H_kv=1, n_blocks=2)
    dev = {k: t.cuda() for k, t in inputs.make(w).items()}
    out1, lse1 = lvx.attention_forward(dev["q"], dev["k"], dev["v"], w.n_blocks)
    out2, lse2 = lvx.attention_forward(dev["q"], dev["k"], dev["v"], w.n_blocks)
    lvx.lvx_last_device_error()
    torch.cuda.synchronize()
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)
    assert torch.isfinite(out1.float()).all()
