// hbm_probe.cuh -- a read-only stream over a device buffer: the ceiling for
// kernels that only read HBM (decode reads K/V and writes almost nothing),
// beside the copy bandwidth that reads and writes.
#pragma once
#include <stdint.h>

#include "pkv_common.cuh"

namespace pkv {

// Chunks move the way decode moves pages: 1-D bulk copies into a ring of
// shared-memory stages, completion counted on an mbarrier per stage, so
// almost no instructions are spent per byte.  Chunk c (of `chunk` bytes; the
// last may be shorter) belongs to CTA c % gridDim.x; a CTA keeps
// kProbeRing / chunk of them in flight.  It folds the first 16 bytes of
// every chunk it received with XOR into sink[blockIdx.x], which shows that
// each copy landed.
constexpr int kProbeRing = 98304;  // bytes in flight per CTA (two CTAs per SM)
constexpr int kProbeMaxStages = kProbeRing / 4096;
constexpr int kProbeSmem = kProbeRing + kProbeMaxStages * 8;

__global__ void __launch_bounds__(32) hbm_read_probe_kernel(const unsigned char* __restrict__ buf, int64_t bytes,
                                                            int chunk, uint32_t* __restrict__ sink) {
  extern __shared__ __align__(128) unsigned char probe_ring[];
  if (threadIdx.x != 0) return;
  const int stages = kProbeRing / chunk;
  const uint32_t base = smem_addr(probe_ring);
  const uint32_t bars = base + kProbeRing;
  for (int s = 0; s < stages; ++s) mbar_init(bars + 8 * s, 1);
  fence_barrier_init();
  const int64_t nchunks = (bytes + chunk - 1) / chunk;
  const int64_t mine = nchunks > blockIdx.x ? (nchunks - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  const uint64_t pol = policy_evict_first();
  auto issue = [&](int64_t k) {  // this CTA's k-th chunk into stage k % stages
    const int64_t c = blockIdx.x + k * gridDim.x;
    const int64_t left = bytes - c * chunk;
    const uint32_t n = (uint32_t)(left < chunk ? left : chunk);
    const uint32_t bar = bars + 8 * (int)(k % stages);
    mbar_arrive_expect_tx(bar, n);
    bulk_g2s_hint(base + (int)(k % stages) * chunk, buf + c * chunk, n, bar, pol);
  };
  int64_t issued = 0;
  for (; issued < stages && issued < mine; ++issued) issue(issued);
  uint32_t acc = 0;
  int64_t k = 0;
  for (; k < mine; ++k) {
    const int s = (int)(k % stages);
    if (!mbar_wait(bars + 8 * s, (int)((k / stages) & 1))) break;
    const uint4 v = *reinterpret_cast<const uint4*>(probe_ring + s * chunk);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
    if (issued < mine) {
      fence_proxy_async_smem();
      issue(issued++);
    }
  }
  // after a timeout: let the copies in flight land before the CTA exits
  for (int64_t j = k; j < issued; ++j) mbar_wait(bars + 8 * (int)(j % stages), (int)((j / stages) & 1));
  sink[blockIdx.x] = acc;
}

}  // namespace pkv
