"""The autograd op (README usage section: a drop-in for scaled_dot_product_attention) holds
no memory past each step: forward and backward in a loop keep torch's allocated device
memory flat once the first iteration has warmed the caching allocator."""
import gc

import pytest
import torch

from llsa_testlib import inputs_for

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("levels,topk", [(1, 8), (2, 4)])
def test_forward_backward_loop_keeps_memory_flat(levels, topk):
    from log_linear_hierarchical_b200 import llsa_attention
    inputs = inputs_for(1, 2, 4096, 64, "bf16", "smooth", 13)
    q, k, v, do = (inputs[n].cuda() for n in ("q", "k", "v", "do"))
    for t in (q, k, v):
        t.requires_grad_(True)

    def step():
        o = llsa_attention(q, k, v, topk=topk, levels=levels)
        o.backward(do)
        q.grad = k.grad = v.grad = None

    step()
    torch.cuda.synchronize()
    gc.disable()            # a leak through a reference cycle must not be hidden by the collector
    try:
        base = torch.cuda.memory_allocated()
        for _ in range(20):
            step()
        torch.cuda.synchronize()
        after = torch.cuda.memory_allocated()
    finally:
        gc.enable()
    assert after == base, (base, after)


def test_output_does_not_keep_the_call_buffers_alive():
    """Once the output and the graph are dropped, the op's buffers are freed at once (no
    reference cycle left for the garbage collector)."""
    from log_linear_hierarchical_b200 import llsa_attention
    inputs = inputs_for(1, 2, 4096, 64, "bf16", "smooth", 14)
    q, k, v = (inputs[n].cuda().requires_grad_(True) for n in ("q", "k", "v"))
    torch.cuda.synchronize()
    gc.disable()
    try:
        base = torch.cuda.memory_allocated()
        o = llsa_attention(q, k, v, topk=4, levels=2)
        held = torch.cuda.memory_allocated()
        del o
        freed = torch.cuda.memory_allocated()
    finally:
        gc.enable()
    assert held > base
    assert freed == base, (base, held, freed)
