// fa_mask.cu -- writes the dropout keep mask Z[b, h, i, j] (uint8 0/1) with the
// same device Philox the attention kernels use.  Inspection/test export: the
// attention kernels themselves never materialise the mask ("Flash Attention"
// glossary, Key Components: the pattern is regenerated, not stored).
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa_internal.h"
#include "philox.cuh"

namespace fa {
namespace {

// One thread per (b*h, i, group of 8 keys).
__global__ void fa_dropout_mask_kernel(uint8_t* mask, int H, int N, uint32_t t, uint32_t seed_lo, uint32_t seed_hi,
                                       long long total_groups) {
  const int groups_per_row = (N + 7) / 8;
  const DropConst k = make_drop_const(t);
  for (long long gidx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; gidx < total_groups;
       gidx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int g = static_cast<int>(gidx % groups_per_row);
    const long long row = gidx / groups_per_row;  // (b*H + h) * N + i
    const int i = static_cast<int>(row % N);
    const int bh = static_cast<int>(row / N);
    const int h = bh % H, b = bh / H;
    uint32_t w[4];
    philox4x32_10(static_cast<uint32_t>(g), static_cast<uint32_t>(i), static_cast<uint32_t>(h),
                  static_cast<uint32_t>(b), seed_lo, seed_hi, w);
    uint8_t* dst = mask + row * N + g * 8;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t km = (t == 0) ? 0xFFFFFFFFu : keep_mask_2x16(w[e], k);
      const int j0 = g * 8 + 2 * e;
      if (j0 < N) dst[2 * e] = (km & 0xFFFFu) ? 1 : 0;
      if (j0 + 1 < N) dst[2 * e + 1] = (km >> 16) ? 1 : 0;
    }
  }
}

// Failure-detection self-test: one warp waits on an mbarrier that nothing will
// ever arrive on, with a wait limit of ``limit_ns``; the bounded wait gives up,
// records the timeout bit in the device error word and returns.
__global__ void fa_wait_timeout_probe_kernel(unsigned* err, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, err, limit_ns);
  __syncthreads();
}

}  // namespace

cudaError_t launch_wait_timeout_probe(unsigned* err, unsigned long long limit_ns, cudaStream_t stream) {
  fa_wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
  return cudaGetLastError();
}

cudaError_t launch_dropout_mask(uint8_t* mask, int B, int H, int N, uint32_t drop_t, uint32_t seed_lo,
                                uint32_t seed_hi, cudaStream_t stream) {
  const long long total = static_cast<long long>(B) * H * N * ((N + 7) / 8);
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 64) blocks = 148 * 64;
  if (blocks < 1) blocks = 1;
  fa_dropout_mask_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(mask, H, N, drop_t, seed_lo,
                                                                               seed_hi, total);
  return cudaGetLastError();
}

}  // namespace fa
