// L2 -> SM gather probe: a measurement aid for the attention kernels' roofline (no
// counterpart on the pages).  The attention kernels gather 16-token x 64-channel bf16 tiles
// by index with 2-D TMA copies; when the gathered tensors fit in the 126 MB L2 those copies
// are served from L2, so HBM bandwidth is not what bounds them.  This kernel does only that
// gather, with the same tensor-map box and swizzle, from a buffer the caller keeps resident
// in L2: every warp streams its share of a list of tile rows through a ring of mbarrier
// stages and does nothing else with them.  Its bytes per second is the gather ceiling the
// attention kernels are measured against.
#pragma once

#include "llsa_common.cuh"

namespace llsa {

constexpr int kProbeWarps = 4;

template <int STAGES>
__global__ void __launch_bounds__(kProbeWarps * 32) gather_probe_kernel(const __grid_constant__ CUtensorMap tm,
                                                                        const int* __restrict__ tile_rows,
                                                                        int ntiles, int rows) {
  extern __shared__ uint8_t probe_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(probe_smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  const uint32_t ring = smem_u32(base) + warp * STAGES * kSubTileBytes;
  __shared__ __align__(8) unsigned long long bars[kProbeWarps][STAGES];
  const uint32_t bar0 = smem_u32(&bars[warp][0]);
  const int gw = blockIdx.x * kProbeWarps + warp;
  const int tw = gridDim.x * kProbeWarps;
  const int mine = gw < ntiles ? (ntiles - 1 - gw) / tw + 1 : 0;
  if (lane == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(bar0 + 8 * s, 1);
    mbar_fence_init();
  }
  __syncwarp();
  auto issue = [&](int i) {
    const int row = checked_index(__ldg(tile_rows + gw + i * tw), rows);
    const uint32_t bar = bar0 + 8 * (i % STAGES);
    mbar_expect_tx(bar, kSubTileBytes);
    tma_load_2d(ring + (i % STAGES) * kSubTileBytes, &tm, 0, row, bar);
  };
  if (lane == 0)
    for (int i = 0; i < min(STAGES, mine); ++i) issue(i);
  int next = 0;
  bool ok = true;
  for (int i = 0; i < mine; ++i) {
    ok = __all_sync(0xffffffffu, mbar_wait(bar0 + 8 * (i % STAGES), (i / STAGES) & 1));
    if (!ok) break;
    next = i + 1;
    if (lane == 0 && i + STAGES < mine) issue(i + STAGES);
  }
  if (!ok)  // a copy did not land in time: one more bounded wait for each copy in flight
    for (int i = next; i < min(mine, next + STAGES); ++i) mbar_wait(bar0 + 8 * (i % STAGES), (i / STAGES) & 1);
}

template <int STAGES>
constexpr int gather_probe_smem() {
  return 1024 + kProbeWarps * STAGES * kSubTileBytes;
}

}  // namespace llsa
