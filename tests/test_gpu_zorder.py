"""llsa_token_permute (quadtree token order) on the GPU: bit-exact against the oracle's
to_z_order / from_z_order, both directions, bf16 and fp32, and the round trip."""
import numpy as np
import pytest
import torch

from log_linear_hierarchical_b200 import api
from oracle.llsa_oracle import from_z_order, to_z_order
from synthetic import morton_order

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,N,dtype", [(1, 1, 256, torch.bfloat16), (2, 3, 4096, torch.bfloat16),
                                         (1, 2, 65536, torch.bfloat16), (1, 2, 4096, torch.float32),
                                         (1, 1, 1 << 20, torch.bfloat16)])
def test_token_permute_matches_oracle(B, H, N, dtype):
    g = torch.Generator().manual_seed(N + B + H)
    x = torch.randn(B, H, N, 64, generator=g).to(dtype)
    shape = api.make_shape(B, H, N, 64, 1, 1 if N // 16 <= 16384 else 2, dtype)
    src = x.cuda()
    z = torch.empty_like(src)
    back = torch.empty_like(src)
    api.llsa_token_permute(shape, src, z, to_z_order=True)
    api.llsa_token_permute(shape, z, back, to_z_order=False)
    torch.cuda.synchronize()
    xn = x.float().numpy()
    assert np.array_equal(z.float().cpu().numpy(), to_z_order(xn))
    assert np.array_equal(back.float().cpu().numpy(), xn)
    assert np.array_equal(from_z_order(z.float().cpu().numpy()), xn)
    assert api.llsa_device_status() == 0


def test_token_permute_agrees_with_the_input_generator_grid():
    # the synthetic smooth fields are laid out in Z order by the generator's own routine
    side = 64
    raster = torch.arange(side * side, dtype=torch.float32).repeat_interleave(64).reshape(1, 1, side * side, 64)
    shape = api.make_shape(1, 1, side * side, 64, 1, 1, torch.float32)
    src = raster.cuda()
    dst = torch.empty_like(src)
    api.llsa_token_permute(shape, src, dst, to_z_order=True)
    torch.cuda.synchronize()
    assert np.array_equal(dst[0, 0, :, 0].cpu().numpy().astype(np.int64), morton_order(side))
