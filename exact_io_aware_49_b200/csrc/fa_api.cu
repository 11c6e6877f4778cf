// fa_api.cu -- the C ABI (include/fa.h): argument validation, TMA descriptor
// encoding, and launches on the caller's stream.  Validation happens before any
// CUDA call, so a rejected call enqueues nothing and touches no output.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "../../include/fa.h"
#include "fa_internal.h"
#include "philox.cuh"

namespace {

// Device word that bounded device waits set when they give up (one per device,
// in this module's static device memory).
__device__ unsigned g_fa_error_word;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [BH, N, d] row-major 3-D map with 128-byte boxes per row (64 bf16 / fp16
// or 32 fp32 columns) x 128 rows x 1 head and 128-byte swizzle.  Rows past N
// of a head are outside the tensor: loads zero-fill them, reductions skip them.
bool encode_head_map(CUtensorMap* tm, const void* base, long long BH, int N, int d, CUtensorMapDataType dt) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t esize = (dt == CU_TENSOR_MAP_DATA_TYPE_FLOAT32) ? 4 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * esize, static_cast<cuuint64_t>(N) * d * esize};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / esize), 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(tm, dt, 3,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

unsigned* error_word_ptr() {
  static unsigned* cache[128] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return nullptr;
  if (dev < 128 && cache[dev]) return cache[dev];
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_fa_error_word) != cudaSuccess) return nullptr;
  if (dev < 128) cache[dev] = static_cast<unsigned*>(p);
  return static_cast<unsigned*>(p);
}

CUtensorMapDataType elem_type(bool f16) {
  return f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
}

bool misaligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Shared validation of sizes / scalars.  Returns FA_OK or the error.
fa_status check_common(int B, int H, int N, int d, float scale, float p_drop) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return FA_ERR_INVALID_ARG;
  if (!(p_drop >= 0.0f && p_drop < 1.0f)) return FA_ERR_INVALID_ARG;  // also rejects NaN
  if (!isfinite(scale) || !(scale > 0.0f)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(B) * H * N;
  if (rows >= (1ll << 31)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

uint32_t drop_threshold(float p_drop) {
  // round-half-even(p * 65536) in double precision (default rounding mode)
  return static_cast<uint32_t>(nearbyint(static_cast<double>(p_drop) * 65536.0));
}

}  // namespace

extern "C" {

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: invalid argument";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: valid but unsupported configuration";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: CUDA call failed";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a bounded device wait gave up";
  }
  return "unknown fa_status";
}

}  // extern "C"

namespace {

fa_status fwd_impl(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int N, int d,
                   int causal, float scale, float p_drop, uint64_t seed, bool f16, void* stream) {
  if (!Q || !K || !V || !O || !LSE) return FA_ERR_INVALID_ARG;
  if (misaligned(Q, 16) || misaligned(K, 16) || misaligned(V, 16) || misaligned(O, 16) || misaligned(LSE, 16))
    return FA_ERR_INVALID_ARG;
  fa_status st = check_common(B, H, N, d, scale, p_drop);
  if (st != FA_OK) return st;

  fa::FwdArgs a;
  memset(&a, 0, sizeof(a));
  const long long BH = static_cast<long long>(B) * H;
  const CUtensorMapDataType dt = elem_type(f16);
  if (!encode_head_map(&a.tmQ, Q, BH, N, d, dt) || !encode_head_map(&a.tmK, K, BH, N, d, dt) ||
      !encode_head_map(&a.tmV, V, BH, N, d, dt))
    return FA_ERR_CUDA;
  a.f16 = f16 ? 1 : 0;
  a.O = O;
  a.LSE = LSE;
  a.err = error_word_ptr();
  if (!a.err) return FA_ERR_CUDA;
  a.B = B;
  a.H = H;
  a.N = N;
  a.d = d;
  a.causal = causal ? 1 : 0;
  a.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  a.drop_t = drop_threshold(p_drop);
  a.drop_scale = a.drop_t ? static_cast<float>(1.0 / (1.0 - static_cast<double>(p_drop))) : 1.0f;
  a.seed_lo = static_cast<uint32_t>(seed);
  a.seed_hi = static_cast<uint32_t>(seed >> 32);
  fa::philox_round_keys(seed, a.philox_rk);
  return fa::launch_fwd(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

bool dtype_ok(fa_dtype dtype) { return dtype == FA_DTYPE_BF16 || dtype == FA_DTYPE_F16; }

}  // namespace

extern "C" {

fa_status fa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int N, int d,
                 int causal, float scale, float p_drop, uint64_t seed, void* stream) {
  return fwd_impl(Q, K, V, O, LSE, B, H, N, d, causal, scale, p_drop, seed, false, stream);
}

fa_status fa_fwd_ex(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int N, int d,
                    int causal, float scale, float p_drop, uint64_t seed, fa_dtype dtype, void* stream) {
  if (!dtype_ok(dtype)) return FA_ERR_INVALID_ARG;
  return fwd_impl(Q, K, V, O, LSE, B, H, N, d, causal, scale, p_drop, seed, dtype == FA_DTYPE_F16, stream);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return 0;
  const size_t rows = static_cast<size_t>(B) * H * N;
  const size_t rows_pad = static_cast<size_t>(B) * H * ((static_cast<size_t>(N) + 127) / 128 * 128);
  return round_up(rows * d * sizeof(float), 256) + 2 * round_up(rows_pad * sizeof(float), 256);
}

}  // extern "C"

namespace {

// Workspace carve-up shared by the backward entry points.
void carve_workspace(fa::BwdArgs* a, void* workspace) {
  char* ws = static_cast<char*>(workspace);
  const size_t rows = static_cast<size_t>(a->B) * a->H * a->N;
  const size_t rows_pad = static_cast<size_t>(a->B) * a->H * ((static_cast<size_t>(a->N) + 127) / 128 * 128);
  const size_t acc_bytes = round_up(rows * a->d * sizeof(float), 256);
  const size_t vec_bytes = round_up(rows_pad * sizeof(float), 256);
  a->dQacc = reinterpret_cast<float*>(ws);
  a->Dvec = reinterpret_cast<float*>(ws + acc_bytes);
  a->lse2 = reinterpret_cast<float*>(ws + acc_bytes + vec_bytes);
}

fa_status check_workspace(const void* workspace, size_t workspace_bytes, int B, int H, int N, int d) {
  if (!workspace || misaligned(workspace, 256)) return FA_ERR_INVALID_ARG;
  if (workspace_bytes < fa_bwd_workspace_size(B, H, N, d)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

void fill_scalars(fa::BwdArgs* a, int B, int H, int N, int d, int causal, float scale, float p_drop,
                  uint64_t seed) {
  a->B = B;
  a->H = H;
  a->N = N;
  a->d = d;
  a->causal = causal ? 1 : 0;
  a->scale = scale;
  a->scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  a->drop_t = drop_threshold(p_drop);
  a->drop_scale = a->drop_t ? static_cast<float>(1.0 / (1.0 - static_cast<double>(p_drop))) : 1.0f;
  a->seed_lo = static_cast<uint32_t>(seed);
  a->seed_hi = static_cast<uint32_t>(seed >> 32);
  fa::philox_round_keys(seed, a->philox_rk);
}

fa_status prepare_impl(const void* O, const void* dO, const float* LSE, int B, int H, int N, int d,
                       void* workspace, size_t workspace_bytes, bool f16, void* stream) {
  if (!O || !dO || !LSE) return FA_ERR_INVALID_ARG;
  if (misaligned(O, 16) || misaligned(dO, 16) || misaligned(LSE, 16)) return FA_ERR_INVALID_ARG;
  fa_status st = check_common(B, H, N, d, 1.0f, 0.0f);
  if (st != FA_OK) return st;
  if ((st = check_workspace(workspace, workspace_bytes, B, H, N, d)) != FA_OK) return st;
  fa::BwdArgs a;
  memset(&a, 0, sizeof(a));
  fill_scalars(&a, B, H, N, d, 0, 1.0f, 0.0f, 0);
  carve_workspace(&a, workspace);
  a.f16 = f16 ? 1 : 0;
  a.O = O;
  a.dO = dO;
  a.LSE = LSE;
  return fa::launch_bwd_prepare(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status tiles_impl(const void* Q, const void* K, const void* V, const void* dO, void* dK, void* dV, int B,
                     int H, int N, int d, int causal, float scale, float p_drop, uint64_t seed, void* workspace,
                     size_t workspace_bytes, bool f16, void* stream) {
  if (!Q || !K || !V || !dO || !dK || !dV) return FA_ERR_INVALID_ARG;
  if (misaligned(Q, 16) || misaligned(K, 16) || misaligned(V, 16) || misaligned(dO, 16) || misaligned(dK, 16) ||
      misaligned(dV, 16))
    return FA_ERR_INVALID_ARG;
  fa_status st = check_common(B, H, N, d, scale, p_drop);
  if (st != FA_OK) return st;
  if ((st = check_workspace(workspace, workspace_bytes, B, H, N, d)) != FA_OK) return st;
  fa::BwdArgs a;
  memset(&a, 0, sizeof(a));
  const long long BH = static_cast<long long>(B) * H;
  const CUtensorMapDataType dt = elem_type(f16);
  if (!encode_head_map(&a.tmQ, Q, BH, N, d, dt) || !encode_head_map(&a.tmK, K, BH, N, d, dt) ||
      !encode_head_map(&a.tmV, V, BH, N, d, dt) || !encode_head_map(&a.tmDO, dO, BH, N, d, dt))
    return FA_ERR_CUDA;
  fill_scalars(&a, B, H, N, d, causal, scale, p_drop, seed);
  carve_workspace(&a, workspace);
  if (!encode_head_map(&a.tmDQacc, a.dQacc, BH, N, d, CU_TENSOR_MAP_DATA_TYPE_FLOAT32)) return FA_ERR_CUDA;
  a.f16 = f16 ? 1 : 0;
  a.dO = dO;
  a.dK = dK;
  a.dV = dV;
  a.err = error_word_ptr();
  if (!a.err) return FA_ERR_CUDA;
  return fa::launch_bwd_tiles(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status finish_impl(void* dQ, int B, int H, int N, int d, float scale, const void* workspace,
                      size_t workspace_bytes, bool f16, void* stream) {
  if (!dQ || misaligned(dQ, 16)) return FA_ERR_INVALID_ARG;
  fa_status st = check_common(B, H, N, d, scale, 0.0f);
  if (st != FA_OK) return st;
  if ((st = check_workspace(workspace, workspace_bytes, B, H, N, d)) != FA_OK) return st;
  fa::BwdArgs a;
  memset(&a, 0, sizeof(a));
  fill_scalars(&a, B, H, N, d, 0, scale, 0.0f, 0);
  carve_workspace(&a, const_cast<void*>(workspace));
  a.f16 = f16 ? 1 : 0;
  a.dQ = dQ;
  return fa::launch_bwd_finish(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status bwd_impl(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                   void* dQ, void* dK, void* dV, int B, int H, int N, int d, int causal, float scale, float p_drop,
                   uint64_t seed, void* workspace, size_t workspace_bytes, bool f16, void* stream) {
  // Validate everything up front so a rejected call launches none of the stages.
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV) return FA_ERR_INVALID_ARG;
  if (misaligned(Q, 16) || misaligned(K, 16) || misaligned(V, 16) || misaligned(O, 16) || misaligned(dO, 16) ||
      misaligned(LSE, 16) || misaligned(dQ, 16) || misaligned(dK, 16) || misaligned(dV, 16))
    return FA_ERR_INVALID_ARG;
  fa_status st = check_common(B, H, N, d, scale, p_drop);
  if (st != FA_OK) return st;
  if ((st = check_workspace(workspace, workspace_bytes, B, H, N, d)) != FA_OK) return st;
  if ((st = prepare_impl(O, dO, LSE, B, H, N, d, workspace, workspace_bytes, f16, stream)) != FA_OK) return st;
  if ((st = tiles_impl(Q, K, V, dO, dK, dV, B, H, N, d, causal, scale, p_drop, seed, workspace, workspace_bytes, f16,
                       stream)) != FA_OK)
    return st;
  return finish_impl(dQ, B, H, N, d, scale, workspace, workspace_bytes, f16, stream);
}

}  // namespace

extern "C" {

fa_status fa_bwd_prepare(const void* O, const void* dO, const float* LSE, int B, int H, int N, int d,
                         void* workspace, size_t workspace_bytes, void* stream) {
  return prepare_impl(O, dO, LSE, B, H, N, d, workspace, workspace_bytes, false, stream);
}

fa_status fa_bwd_tiles(const void* Q, const void* K, const void* V, const void* dO, void* dK, void* dV, int B,
                       int H, int N, int d, int causal, float scale, float p_drop, uint64_t seed, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return tiles_impl(Q, K, V, dO, dK, dV, B, H, N, d, causal, scale, p_drop, seed, workspace, workspace_bytes, false,
                    stream);
}

fa_status fa_bwd_finish(void* dQ, int B, int H, int N, int d, float scale, const void* workspace,
                        size_t workspace_bytes, void* stream) {
  return finish_impl(dQ, B, H, N, d, scale, workspace, workspace_bytes, false, stream);
}

fa_status fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                 void* dQ, void* dK, void* dV, int B, int H, int N, int d, int causal, float scale, float p_drop,
                 uint64_t seed, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, causal, scale, p_drop, seed, workspace,
                  workspace_bytes, false, stream);
}

fa_status fa_bwd_ex(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                    void* dQ, void* dK, void* dV, int B, int H, int N, int d, int causal, float scale, float p_drop,
                    uint64_t seed, fa_dtype dtype, void* workspace, size_t workspace_bytes, void* stream) {
  if (!dtype_ok(dtype)) return FA_ERR_INVALID_ARG;
  return bwd_impl(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, causal, scale, p_drop, seed, workspace,
                  workspace_bytes, dtype == FA_DTYPE_F16, stream);
}

fa_status fa_dropout_mask(uint8_t* mask, int B, int H, int N, float p_drop, uint64_t seed, void* stream) {
  if (!mask) return FA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || N <= 0) return FA_ERR_INVALID_ARG;
  if (!(p_drop >= 0.0f && p_drop < 1.0f)) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H * N >= (1ll << 31)) return FA_ERR_UNSUPPORTED;
  return fa::launch_dropout_mask(mask, B, H, N, drop_threshold(p_drop), static_cast<uint32_t>(seed),
                                 static_cast<uint32_t>(seed >> 32), static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? FA_OK
             : FA_ERR_CUDA;
}

fa_status fa_selftest_wait_timeout(uint32_t limit_us, void* stream) {
  if (limit_us == 0 || limit_us > 1000000u) return FA_ERR_INVALID_ARG;
  unsigned* err = error_word_ptr();
  if (!err) return FA_ERR_CUDA;
  return fa::launch_wait_timeout_probe(err, 1000ull * limit_us, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? FA_OK
             : FA_ERR_CUDA;
}

fa_status fa_last_device_error(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_fa_error_word, sizeof(v)) != cudaSuccess) return FA_ERR_CUDA;
  if (v) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_fa_error_word, &zero, sizeof(zero)) != cudaSuccess) return FA_ERR_CUDA;
    // bit 0: a bounded wait gave up; bit 1: the shared-memory layout did not fit (kernel did nothing)
    return (v & 1u) ? FA_ERR_TIMEOUT : FA_ERR_CUDA;
  }
  return FA_OK;
}

}  // extern "C"
