"""The index transpose alone (skill page "Log Linear Sparse Attention", Core Technique 3), on
selections written directly, at sizes that take both of its paths: problems of at most 16
tiles of 4096 entries (the scatter and bucket kernels sum the histogram entries they need)
and larger ones (the histogram is scanned once by its own kernel).  Bit-exact against the
oracle's counting-sort transpose."""
import numpy as np
import pytest
import torch

from log_linear_hierarchical_b200 import api
from oracle import llsa_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def skewed_selection(rng, B, H, n, K, hot):
    """[B, H, n, K] ascending distinct keys; half of every list comes from `hot` popular keys."""
    out = np.empty((B, H, n, K), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            base = rng.integers(0, n, size=(n, 1))
            step = n // K
            spread = (base + np.arange(K)[None, :] * step) % n            # K distinct keys per row
            hot_keys = rng.choice(hot, size=(n, K // 2)) if K >= 2 else None
            if hot_keys is not None:
                # replace the first K/2 entries by popular keys where that keeps the row distinct
                for j in range(K // 2):
                    cand = hot_keys[:, j]
                    clash = (spread == cand[:, None]).any(axis=1)
                    spread[~clash, j] = cand[~clash]
            out[b, h] = np.sort(spread, axis=1)
    assert np.all(np.diff(out, axis=-1) > 0)
    return out


@pytest.mark.parametrize("B,H,N,K,levels", [
    (1, 1, 1 << 18, 64, 1),     # 16384 keys, 1M entries: 256 tiles, 64 buckets (scanned)
    (2, 3, 65536, 32, 1),       # 32 tiles per problem (scanned)
    (1, 2, 65536, 16, 1),       # 16 tiles (summed in place)
    (1, 1, 1 << 20, 4, 2),      # two levels: 64 tiles at level 1, 1 at level 2
])
def test_transpose_bitexact(B, H, N, K, levels):
    rng = np.random.default_rng(N + K)
    shape = api.make_shape(B, H, N, 64, K, levels, torch.bfloat16)
    idx_levels = []
    for lev in range(1, levels + 1):
        n = N // 16 ** lev
        idx_levels.append(skewed_selection(rng, B, H, n, min(K, n), hot=max(1, n // 64)))
    flat = torch.from_numpy(np.concatenate([x.ravel() for x in idx_levels])).cuda()
    row_ptr = torch.empty(api.llsa_row_ptr_elems(shape), dtype=torch.int32, device="cuda")
    col = torch.empty(api.llsa_index_elems(shape), dtype=torch.int32, device="cuda")
    ws = torch.empty((api.llsa_transpose_workspace_bytes(shape) + 3) // 4, dtype=torch.float32, device="cuda")
    assert api.llsa_device_status() == 0
    api.llsa_index_transpose(shape, flat, row_ptr, col, ws)
    torch.cuda.synchronize()
    assert api.llsa_device_status() == 0
    rps, cols = orc.index_transpose_all(idx_levels)
    got_rp, got_col = row_ptr.cpu().numpy(), col.cpu().numpy()
    ro = co = 0
    for rp, cl in zip(rps, cols):
        assert np.array_equal(got_rp[ro:ro + rp.size], rp.ravel())
        assert np.array_equal(got_col[co:co + cl.size], cl.ravel())
        ro += rp.size
        co += cl.size
    print("longest row", max(int(np.diff(r, axis=-1).max()) for r in rps))
