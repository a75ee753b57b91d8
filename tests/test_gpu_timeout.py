"""The bounded-wait error path of the attention kernel, on the GPU, without a fault.

ress_debug_attn_forced_timeout makes every CTA's softmax warps wait on a barrier that
nothing completes, with a short limit; each CTA must then report RESS_ERR_DEVICE_TIMEOUT
in the error word, release its TMA and MMA warps, drain what they issued, free tensor
memory and exit.  Afterwards the same context must compute normally."""
import pytest
import torch

from block_sparse_global_b200 import ress as R
from block_sparse_global_b200 import workload as W
from parity import run_gpu

pytestmark = pytest.mark.gpu
TIMEOUT = 5  # RESS_ERR_DEVICE_TIMEOUT


@pytest.mark.parametrize("key_block", [128, 64])
def test_forced_wait_timeout_reports_and_context_recovers(key_block):
    wl = W.make_workload(1, key_block=key_block)
    layer = run_gpu(wl)                      # a normal layer: kept lists and the output
    dev = layer.out.device
    q, k, v = wl.q.to(dev), wl.k.to(dev), wl.v.to(dev)
    good = layer.out.clone()

    def attend_normally():
        layer.dev_err.zero_()
        layer.out.fill_(0)
        R.ress_block_sparse_attn(layer.shape, q, k, v, layer.kv_idx, layer.kv_cnt, None,
                                 layer.scale, layer.out, layer.lse, layer.dev_err)
        torch.cuda.synchronize()

    attend_normally()
    assert layer.device_error() == 0
    assert torch.equal(layer.out, good)

    for rep in range(2):
        layer.dev_err.zero_()
        sentinel = torch.full_like(layer.out, 7.0)
        R.ress_debug_attn_forced_timeout(layer.shape, q, k, v, layer.kv_idx, layer.kv_cnt,
                                         layer.scale, sentinel, layer.dev_err, 200_000)
        torch.cuda.synchronize()             # the kernel returned: nothing hung
        assert layer.device_error() == TIMEOUT, f"pass {rep}: error word {layer.device_error()}"
        assert torch.all(sentinel == 7.0), "a timed-out CTA must not write its output rows"

        # the context is intact: the next normal call computes the same output again
        attend_normally()
        assert layer.device_error() == 0
        assert torch.equal(layer.out, good)
