"""llsa_index_transpose_noalloc: the index transpose for callers that cannot give the
library device memory (a plugin host that passes only inputs and outputs, or a runtime whose
device memory is fixed at start-up).  It must give exactly the CSR that the workspace
version gives, on consecutive calls that reuse its one internal scratch array.

This file sorts last so that a run stopping at the first failure has already run every
other test; it also passes when run alone in a fresh process.
"""
import ctypes

import pytest
import torch

from log_linear_hierarchical_b200 import _lib, api
from synthetic import WORKLOADS, make_config_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _selection(cfg):
    """idx of one workload, computed by the CUDA path."""
    dtype = torch.bfloat16
    inputs = {k: v.cuda() for k, v in make_config_inputs(cfg, with_do=False).items()}
    shape = api.make_shape(cfg.B, cfg.H, cfg.N, cfg.D, cfg.topk, cfg.levels, dtype)
    buf = api.LLSABuffers.allocate(shape, "cuda", dtype)
    api.llsa_build_pyramid(shape, inputs["q"], inputs["k"], inputs["v"], buf.q_pyr, buf.k_pyr, buf.v_pyr)
    api.llsa_select(shape, buf.q_pyr, buf.k_pyr, buf.idx)
    return shape, buf


def test_noalloc_transpose_equals_workspace_transpose_on_consecutive_calls():
    # two calls in a row on different workloads: the second reuses the scratch array that
    # the first left behind
    for cfg in (WORKLOADS["headline-65536"], WORKLOADS["two-level-16384"]):
        shape, buf = _selection(cfg)
        assert api.llsa_transpose_workspace_bytes(shape) <= _lib.NOALLOC_SCRATCH_BYTES
        api.llsa_index_transpose(shape, buf.idx, buf.row_ptr, buf.col, buf.ws_transpose)
        rp_ref, col_ref = buf.row_ptr.clone(), buf.col.clone()
        buf.row_ptr.fill_(-7)
        buf.col.fill_(-7)
        api.llsa_index_transpose_noalloc(shape, buf.idx, buf.row_ptr, buf.col)
        torch.cuda.synchronize()
        assert api.llsa_device_status() == 0
        assert torch.equal(buf.row_ptr, rp_ref)
        assert torch.equal(buf.col, col_ref)


def test_noalloc_transpose_rejects_shapes_beyond_its_scratch():
    # 8 x 16 heads of 4096 level-1 tokens with K = 16: ~33 MB of scratch > 8 MiB
    shape = api.make_shape(8, 16, 65536, 64, 16, 1, torch.bfloat16)
    assert api.llsa_validate_shape(shape) == 0
    assert api.llsa_transpose_workspace_bytes(shape) > _lib.NOALLOC_SCRATCH_BYTES
    # the C entry point itself rejects the shape before any launch (the binding would refuse
    # these 16-entry buffers earlier, by their size)
    t = torch.empty(16, dtype=torch.int32, device="cuda")
    status = _lib.load().llsa_index_transpose_noalloc(ctypes.byref(shape), t.data_ptr(), t.data_ptr(),
                                                      t.data_ptr(), None)
    assert status == 3  # LLSA_ERR_WORKSPACE
    with pytest.raises(ValueError):
        api.llsa_index_transpose_noalloc(shape, t, t, t)
