// fa_internal.h -- launch interfaces between the C-ABI shim and the kernel
// translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

struct FwdArgs {
  CUtensorMap tmQ, tmK, tmV;  // 3-D maps over [B*H, N, d] 16-bit, 64 x 128 x 1 boxes, 128B swizzle
  void* O;                    // [B, H, N, d], same type as Q
  int f16;                    // element type of Q, K, V, O: 0 bf16, 1 fp16
  float* LSE;                 // fp32 [B, H, N]
  unsigned* err;              // device error word
  int B, H, N, d;
  int causal;
  float scale_log2;   // scale * log2(e)
  uint32_t drop_t;    // keep <=> u16 >= drop_t (0: no dropout)
  float drop_scale;   // 1 / (1 - p)
  uint32_t seed_lo, seed_hi;
  uint32_t philox_rk[20];  // Philox round keys of the seed (rounds 0..9, k0 / k1 interleaved)
};

struct BwdArgs {
  CUtensorMap tmQ, tmK, tmV, tmDO;  // same layout as the forward maps
  CUtensorMap tmDQacc;               // fp32 [B*H, N, d], 32-column x 128-row boxes, 128B swizzle
  int f16;  // element type of Q, K, V, O, dO, dQ, dK, dV: 0 bf16, 1 fp16
  const void* O;
  const void* dO;
  const float* LSE;
  void* dQ;
  void* dK;
  void* dV;
  float* dQacc;  // fp32 [B, H, N, d] workspace
  float* Dvec;   // fp32 [B, H, Npad] workspace: rowsum(dO * O); 0 past N
  float* lse2;   // fp32 [B, H, Npad] workspace: LSE * log2(e); +inf past N
  unsigned* err;
  int B, H, N, d;
  int causal;
  float scale;
  float scale_log2;
  uint32_t drop_t;
  float drop_scale;
  uint32_t seed_lo, seed_hi;
  uint32_t philox_rk[20];  // Philox round keys of the seed (rounds 0..9, k0 / k1 interleaved)
};

cudaError_t launch_fwd(const FwdArgs& a, cudaStream_t stream);
// The three backward stages; fa_bwd runs them in this order.  Only the fields
// each stage reads need to be set.
cudaError_t launch_bwd_prepare(const BwdArgs& a, cudaStream_t stream);  // O, dO, LSE -> Dvec, lse2, dQacc = 0
cudaError_t launch_bwd_tiles(const BwdArgs& a, cudaStream_t stream);    // maps, lse2, Dvec -> dK, dV, dQacc
cudaError_t launch_bwd_finish(const BwdArgs& a, cudaStream_t stream);   // dQacc -> dQ
cudaError_t launch_wait_timeout_probe(unsigned* err, unsigned long long limit_ns, cudaStream_t stream);
cudaError_t launch_dropout_mask(uint8_t* mask, int B, int H, int N, uint32_t drop_t, uint32_t seed_lo,
                                uint32_t seed_hi, cudaStream_t stream);

}  // namespace fa
