"""ress_drift_scores_static: the drift score for callers that cannot allocate device
memory (a plugin host that passes only inputs and outputs, or a runtime that reserves
all device memory up front and forbids cudaMalloc/cudaFree later).  It keeps its scratch
in a fixed static buffer inside libress.so instead of taking a workspace.

Checked through the C ABI against ress_drift_scores (the workspace entry point) on two
calls in a row with different shapes, so the second call also shows that leftovers of
the first in the shared buffer do not leak into its result.  This file is collected last
so that a run stopping at its first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_global_b200 import build as B
from block_sparse_global_b200 import ress as R
from block_sparse_global_b200 import workload as W
from block_sparse_global_b200.pipeline import SparseGlobalAttention

pytestmark = pytest.mark.gpu


def _layer_inputs(wl):
    dev = torch.device("cuda")
    b, h, n, _ = wl.q.shape
    layer = SparseGlobalAttention(b, h, n, device=dev)
    layer.load_output_projection(wl.w_o.to(dev))
    layer.scores(wl.q.to(dev), wl.k.to(dev), wl.v.to(dev))
    layer.drift()                                   # workspace entry point
    torch.cuda.synchronize()
    return layer


def test_static_scratch_drift_matches_workspace_drift_twice():
    B.build()
    R.load()
    cases = [W.make_workload(3, heads=8, views=12, method="drift"),   # 16488 tokens, 129 blocks
             W.make_workload(1, method="drift")]                       # 1024 tokens, 8 blocks
    for wl in cases:
        layer = _layer_inputs(wl)
        want = layer.s.clone()
        got = torch.full_like(layer.s, float("nan"))
        R.ress_drift_scores_static(layer.shape, layer.P, layer.v_pool, layer.v_bar, layer.gram, got)
        torch.cuda.synchronize()
        g, w = got.cpu().numpy(), want.cpu().numpy()
        assert np.isfinite(g).all()
        np.testing.assert_allclose(g, w, rtol=1e-4, atol=1e-7)


def test_static_scratch_rejects_shapes_beyond_its_limit():
    B.build()
    lib = R.load()
    fake = 0x7F0000000000   # aligned and never dereferenced: the call is rejected first
    too_big = R.make_shape(2, 16, 4096 * 128)          # 131072 pooled rows, about 34.6 MB
    assert R.ress_drift_workspace_bytes(too_big) > 8 << 20
    st = lib.ress_drift_scores_static(ctypes.byref(too_big), fake, fake, fake, fake, fake, None)
    assert st == 2   # RESS_ERR_UNSUPPORTED
    fits = R.make_shape(1, 16, 1074 * 128)             # the 100-view layer
    assert R.ress_drift_workspace_bytes(fits) <= 8 << 20
