// fa_noalloc.cu -- fa_bwd_noalloc: the backward pass without a caller-provided
// workspace, for callers that cannot allocate device memory.
//
// Who needs it: code that runs where nobody may call cudaMalloc -- a plugin
// inside a host framework whose memory pool owns every device allocation,
// latency-critical loops that cannot afford the implicit synchronisation an
// allocation can cause, or deployments with a fixed, audited memory budget.
// Such callers still own and pass their inputs and outputs; only the
// backward's scratch (fp32 dQ accumulator, D, LSE in log2 units) moves into a
// fixed array that lives in this library's static device memory.
//
// The scratch array is a file-scope __device__ object: every GPU that loads
// the library holds FA_NOALLOC_SCRATCH_BYTES of device memory until the
// process exits.  In host code its name is only a host-side stand-in, so the
// device address is looked up with cudaGetSymbolAddress once per device, with
// that device current, on the first call made on it.
#include <cuda_runtime.h>
#include <math.h>

#include <atomic>

#include "../../include/fa.h"

namespace {

// 256-byte alignment matches what the workspace carve-up requires.
static __device__ __align__(256) unsigned char g_fa_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of the scratch array on the current device (nullptr on failure).
void* scratch_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p) return p;
  if (cudaGetSymbolAddress(&p, g_fa_noalloc_scratch) != cudaSuccess || !p) return nullptr;
  g_scratch_addr[dev].store(p, std::memory_order_release);
  return p;
}

}  // namespace

extern "C" fa_status fa_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                                    const float* LSE, void* dQ, void* dK, void* dV, int B, int H, int N, int d,
                                    int causal, float scale, float p_drop, uint64_t seed, void* stream) {
  // Validate the arguments first, with fa_bwd's rules and in its order (sizes,
  // scalars, supported head dimension), so that the same bad arguments get the
  // same status from both entry points; only then the scratch limit.  A
  // rejected call never touches the device.
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return FA_ERR_INVALID_ARG;
  if (!(p_drop >= 0.0f && p_drop < 1.0f)) return FA_ERR_INVALID_ARG;  // also rejects NaN
  if (!isfinite(scale) || !(scale > 0.0f)) return FA_ERR_INVALID_ARG;
  if (d != 32 && d != 64 && d != 96 && d != 128 && d != 192 && d != 256) return FA_ERR_UNSUPPORTED;
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (need == 0) return FA_ERR_INVALID_ARG;
  if (need > static_cast<size_t>(FA_NOALLOC_SCRATCH_BYTES)) return FA_ERR_UNSUPPORTED;
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV) return FA_ERR_INVALID_ARG;
  void* scratch = scratch_address();
  if (!scratch) return FA_ERR_CUDA;
  // The prepare stage rewrites every scratch word this call reads (it zeroes the
  // dQ accumulator and writes D and LSE2 for all B*H*N rows; the d = 192 / 256
  // kernels read only D and LSE2), so whatever an earlier call left in the
  // array does not matter.
  return fa_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, causal, scale, p_drop, seed, scratch, need, stream);
}
