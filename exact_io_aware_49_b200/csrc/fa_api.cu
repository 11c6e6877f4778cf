// fa_api.cu -- the C ABI (include/fa.h): argument validation, TMA descriptor
// encoding, and launches on the caller's stream.  Validation happens before any
// CUDA call, so a rejected call enqueues nothing and touches no output.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>

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

// The driver's tensor-map encoder, looked up once.  The function-local static
// is initialised exactly once even when several host threads make their first
// call at the same time; a failed lookup is remembered as nullptr.
EncodeTiledFn get_encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 3-D map (d, T, G) over a 16-bit or fp32 tensor: column, token row, head
// coordinate, with token stride ``tok`` and head stride ``grp`` (elements).
// Boxes are 128 bytes of a row (64 16-bit or 32 fp32 columns) x 128 rows x 1
// head with 128-byte swizzle.  Rows past T are outside the tensor: loads
// zero-fill them, reductions skip them.
bool encode_map(CUtensorMap* tm, const void* base, int d, long long T, long long G, long long tok, long long grp,
                CUtensorMapDataType dt, int box_rows = 128) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t esize = (dt == CU_TENSOR_MAP_DATA_TYPE_FLOAT32) ? 4 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(G)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(tok) * esize, static_cast<cuuint64_t>(grp) * esize};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / esize), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(tm, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Device address of g_fa_error_word on the current device, cached per device.
// Concurrent first calls from several host threads may each look it up; they
// store the same address, and the atomics make those stores race-free.
unsigned* error_word_ptr() {
  static std::atomic<unsigned*> cache[128];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return nullptr;
  if (dev < 128) {
    unsigned* c = cache[dev].load(std::memory_order_acquire);
    if (c) return c;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_fa_error_word) != cudaSuccess) return nullptr;
  if (dev < 128) cache[dev].store(static_cast<unsigned*>(p), std::memory_order_release);
  return static_cast<unsigned*>(p);
}

CUtensorMapDataType elem_type(bool f16) {
  return f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
}

bool misaligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

long long pad128(long long n) { return (n + 127) / 128 * 128; }

fa_status check_scalars(int d, float scale, float p_drop) {
  if (!(p_drop >= 0.0f && p_drop < 1.0f)) return FA_ERR_INVALID_ARG;  // also rejects NaN
  if (!isfinite(scale) || !(scale > 0.0f)) return FA_ERR_INVALID_ARG;
  // 32 and 96 run on the 64- and 128-column kernels: the tensor maps read the
  // columns past d as zeros and only d columns are stored; 192 and 256 run on
  // the wide kernels (fa_fwd_wide.cu, fa_bwd_wide.cu; not the paged decode)
  if (d != 32 && d != 64 && d != 96 && d != 128 && d != 192 && d != 256) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Head dimensions of the 64- / 128-column kernels (the rest run on the wide ones).
bool narrow_head(int d) { return d <= 128; }

uint32_t drop_threshold(float p_drop) {
  // round-half-even(p * 65536) in double precision (default rounding mode)
  return static_cast<uint32_t>(nearbyint(static_cast<double>(p_drop) * 65536.0));
}

// One validated problem: the sequence layout plus the scalars every stage needs.
struct Problem {
  fa::SeqLayout seq;
  int d;
  int causal;
  float scale;
  float p_drop;
  uint64_t seed;
  bool f16;
  bool deterministic;  // backward: fixed order of the dQ additions
  long long groups() const { return seq.cu_q ? seq.H : static_cast<long long>(seq.units); }
};

// Fixed lengths: [B, H, Nq, d] queries, [B, H, Nk, d] keys.
fa_status fixed_problem(Problem* pb, int B, int H, int Nq, int Nk, int d, int causal, float scale, float p_drop,
                        uint64_t seed, bool f16) {
  if (B <= 0 || H <= 0 || Nq <= 0 || Nk <= 0 || d <= 0) return FA_ERR_INVALID_ARG;
  fa_status st = check_scalars(d, scale, p_drop);
  if (st != FA_OK) return st;
  const long long bh = static_cast<long long>(B) * H;
  if (bh * (Nq > Nk ? Nq : Nk) >= (1ll << 31) || bh * pad128(Nq) >= (1ll << 31)) return FA_ERR_UNSUPPORTED;
  memset(pb, 0, sizeof(*pb));
  pb->seq.B = B;
  pb->seq.H = H;
  pb->seq.units = B * H;  // < 2^31, checked above
  pb->seq.unit0 = 0;
  pb->seq.Nq = Nq;
  pb->seq.Nk = Nk;
  pb->seq.total_q = Nq;
  pb->seq.total_k = Nk;
  pb->seq.tok_stride = d;
  pb->seq.q_head_stride = static_cast<long long>(Nq) * d;
  pb->seq.k_head_stride = static_cast<long long>(Nk) * d;
  pb->d = d;
  pb->causal = causal ? 1 : 0;
  pb->scale = scale;
  pb->p_drop = p_drop;
  pb->seed = seed;
  pb->f16 = f16;
  return FA_OK;
}

// Packed variable lengths: [total_q, H, d] queries, [total_k, H, d] keys,
// device offsets cu_q / cu_k [B + 1].
fa_status packed_problem(Problem* pb, const int* cu_q, const int* cu_k, int B, int H, int total_q, int total_k,
                         int max_q, int max_k, int d, int causal, float scale, float p_drop, uint64_t seed,
                         bool f16) {
  if (!cu_q || !cu_k || misaligned(cu_q, 4) || misaligned(cu_k, 4)) return FA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || total_q <= 0 || total_k <= 0 || max_q <= 0 || max_k <= 0 || d <= 0)
    return FA_ERR_INVALID_ARG;
  if (max_q > total_q || max_k > total_k) return FA_ERR_INVALID_ARG;
  fa_status st = check_scalars(d, scale, p_drop);
  if (st != FA_OK) return st;
  const long long bh = static_cast<long long>(B) * H;
  if (static_cast<long long>(H) * (total_q > total_k ? total_q : total_k) >= (1ll << 31) ||
      bh * pad128(max_q) >= (1ll << 31) || bh * ((max_k + 127) / 128) >= (1ll << 31))
    return FA_ERR_UNSUPPORTED;
  memset(pb, 0, sizeof(*pb));
  pb->seq.cu_q = cu_q;
  pb->seq.cu_k = cu_k;
  pb->seq.B = B;
  pb->seq.H = H;
  pb->seq.units = B * H;  // < 2^31, checked above
  pb->seq.unit0 = 0;
  pb->seq.Nq = max_q;
  pb->seq.Nk = max_k;
  pb->seq.total_q = total_q;
  pb->seq.total_k = total_k;
  pb->seq.tok_stride = static_cast<long long>(H) * d;
  pb->seq.q_head_stride = d;
  pb->seq.k_head_stride = d;
  pb->d = d;
  pb->causal = causal ? 1 : 0;
  pb->scale = scale;
  pb->p_drop = p_drop;
  pb->seed = seed;
  pb->f16 = f16;
  return FA_OK;
}

// Workspace: fp32 dQ accumulator [G, total_q, d], then the fp32 D and
// LSE * log2(e) vectors [B * H, pad128(Nq)], then (deterministic mode only)
// one uint32 counter per (unit, query tile), each part rounded to 256 bytes.
size_t order_bytes(const Problem& pb) {
  return pb.deterministic ? static_cast<size_t>(pb.seq.units) * (pad128(pb.seq.Nq) / 128) * 4 : 0;
}

size_t workspace_bytes(const Problem& pb) {
  const size_t acc = static_cast<size_t>(pb.groups()) * pb.seq.total_q * pb.d * sizeof(float);
  const size_t vec = static_cast<size_t>(pb.seq.units) * pad128(pb.seq.Nq) * sizeof(float);
  return round_up(acc, 256) + 2 * round_up(vec, 256) + round_up(order_bytes(pb), 256);
}

bool encode_q_like(const Problem& pb, CUtensorMap* tm, const void* base, int box_rows = 128) {
  return encode_map(tm, base, pb.d, pb.seq.total_q, pb.groups(), pb.seq.tok_stride, pb.seq.q_head_stride,
                    elem_type(pb.f16), box_rows);
}

bool encode_k_like(const Problem& pb, CUtensorMap* tm, const void* base, int box_rows = 128) {
  return encode_map(tm, base, pb.d, pb.seq.total_k, pb.groups(), pb.seq.tok_stride, pb.seq.k_head_stride,
                    elem_type(pb.f16), box_rows);
}

void fill_common(const Problem& pb, fa::SeqLayout* seq, int* d, int* causal, float* scale_log2, uint32_t* drop_t,
                 float* drop_scale, uint32_t* seed_lo, uint32_t* seed_hi, uint32_t (&rk)[20]) {
  *seq = pb.seq;
  *d = pb.d;
  *causal = pb.causal;
  *scale_log2 = static_cast<float>(static_cast<double>(pb.scale) * 1.4426950408889634);
  *drop_t = drop_threshold(pb.p_drop);
  *drop_scale = *drop_t ? static_cast<float>(1.0 / (1.0 - static_cast<double>(pb.p_drop))) : 1.0f;
  *seed_lo = static_cast<uint32_t>(pb.seed);
  *seed_hi = static_cast<uint32_t>(pb.seed >> 32);
  fa::philox_round_keys(pb.seed, rk);
}

fa_status fwd_run(const Problem& pb, const void* Q, const void* K, const void* V, void* O, float* LSE,
                  void* stream) {
  if (!Q || !K || !V || !O || !LSE) return FA_ERR_INVALID_ARG;
  if (misaligned(Q, 16) || misaligned(K, 16) || misaligned(V, 16) || misaligned(O, 16) || misaligned(LSE, 16))
    return FA_ERR_INVALID_ARG;
  fa::FwdArgs a;
  memset(&a, 0, sizeof(a));
  // the wide-head kernel streams 64-key tiles
  const int kv_rows = narrow_head(pb.d) ? 128 : 64;
  if (!encode_q_like(pb, &a.tmQ, Q) || !encode_k_like(pb, &a.tmK, K, kv_rows) || !encode_k_like(pb, &a.tmV, V, kv_rows))
    return FA_ERR_CUDA;
  a.f16 = pb.f16 ? 1 : 0;
  a.O = O;
  a.LSE = LSE;
  a.err = error_word_ptr();
  if (!a.err) return FA_ERR_CUDA;
  fill_common(pb, &a.seq, &a.d, &a.causal, &a.scale_log2, &a.drop_t, &a.drop_scale, &a.seed_lo, &a.seed_hi,
              a.philox_rk);
  return fa::launch_fwd(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status check_workspace(const Problem& pb, const void* workspace, size_t bytes) {
  if (!workspace || misaligned(workspace, 256)) return FA_ERR_INVALID_ARG;
  if (bytes < workspace_bytes(pb)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

void bwd_args(const Problem& pb, fa::BwdArgs* a, void* workspace) {
  memset(a, 0, sizeof(*a));
  float scale_log2;
  fill_common(pb, &a->seq, &a->d, &a->causal, &scale_log2, &a->drop_t, &a->drop_scale, &a->seed_lo, &a->seed_hi,
              a->philox_rk);
  a->scale = pb.scale;
  a->scale_log2 = scale_log2;
  a->f16 = pb.f16 ? 1 : 0;
  char* ws = static_cast<char*>(workspace);
  const size_t acc = round_up(static_cast<size_t>(pb.groups()) * pb.seq.total_q * pb.d * sizeof(float), 256);
  const size_t vec = round_up(static_cast<size_t>(pb.seq.units) * pad128(pb.seq.Nq) * sizeof(float), 256);
  a->dQacc = reinterpret_cast<float*>(ws);
  a->Dvec = reinterpret_cast<float*>(ws + acc);
  a->lse2 = reinterpret_cast<float*>(ws + acc + vec);
  a->dq_order = pb.deterministic ? reinterpret_cast<unsigned*>(ws + acc + 2 * vec) : nullptr;
}

fa_status prepare_run(const Problem& pb, const void* O, const void* dO, const float* LSE, void* workspace,
                      size_t bytes, void* stream) {
  if (!O || !dO || !LSE) return FA_ERR_INVALID_ARG;
  if (misaligned(O, 16) || misaligned(dO, 16) || misaligned(LSE, 16)) return FA_ERR_INVALID_ARG;
  fa_status st = check_workspace(pb, workspace, bytes);
  if (st != FA_OK) return st;
  fa::BwdArgs a;
  bwd_args(pb, &a, workspace);
  a.O = O;
  a.dO = dO;
  a.LSE = LSE;
  return fa::launch_bwd_prepare(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status tiles_run(const Problem& pb, const void* Q, const void* K, const void* V, const void* dO, void* dK,
                    void* dV, void* workspace, size_t bytes, void* stream) {
  if (!narrow_head(pb.d)) return FA_ERR_UNSUPPORTED;  // wide heads: bwd_run's two-kernel path only
  if (!Q || !K || !V || !dO || !dK || !dV) return FA_ERR_INVALID_ARG;
  if (misaligned(Q, 16) || misaligned(K, 16) || misaligned(V, 16) || misaligned(dO, 16) || misaligned(dK, 16) ||
      misaligned(dV, 16))
    return FA_ERR_INVALID_ARG;
  fa_status st = check_workspace(pb, workspace, bytes);
  if (st != FA_OK) return st;
  fa::BwdArgs a;
  bwd_args(pb, &a, workspace);
  if (!encode_q_like(pb, &a.tmQ, Q) || !encode_k_like(pb, &a.tmK, K) || !encode_k_like(pb, &a.tmV, V) ||
      !encode_q_like(pb, &a.tmDO, dO))
    return FA_ERR_CUDA;
  // the accumulator is [G, total_q, d] fp32, contiguous
  if (!encode_map(&a.tmDQacc, a.dQacc, pb.d, pb.seq.total_q, pb.groups(), pb.d,
                  static_cast<long long>(pb.seq.total_q) * pb.d, CU_TENSOR_MAP_DATA_TYPE_FLOAT32))
    return FA_ERR_CUDA;
  a.dO = dO;
  a.dK = dK;
  a.dV = dV;
  a.err = error_word_ptr();
  if (!a.err) return FA_ERR_CUDA;
  return fa::launch_bwd_tiles(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status finish_run(const Problem& pb, void* dQ, const void* workspace, size_t bytes, void* stream) {
  if (!narrow_head(pb.d)) return FA_ERR_UNSUPPORTED;
  if (!dQ || misaligned(dQ, 16)) return FA_ERR_INVALID_ARG;
  fa_status st = check_workspace(pb, workspace, bytes);
  if (st != FA_OK) return st;
  fa::BwdArgs a;
  bwd_args(pb, &a, const_cast<void*>(workspace));
  a.dQ = dQ;
  return fa::launch_bwd_finish(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Head dimensions 192 / 256: the dK, dV kernel (64-query tiles against a
// 128-key tile) and the dQ kernel (64-key tiles against a 128-query tile),
// after the preprocess; dQ is written directly (no accumulator, no convert).
fa_status wide_tiles_run(const Problem& pb, const void* Q, const void* K, const void* V, const void* dO, void* dQ,
                         void* dK, void* dV, void* workspace, void* stream) {
  fa::BwdArgs a;
  bwd_args(pb, &a, workspace);
  CUtensorMap kv[4], qm[4];  // Q, K, V, dO
  const int kv_rows = fa::wide_kv_query_rows(pb.d);
  if (!encode_q_like(pb, &kv[0], Q, kv_rows) || !encode_k_like(pb, &kv[1], K, 128) ||
      !encode_k_like(pb, &kv[2], V, 128) || !encode_q_like(pb, &kv[3], dO, kv_rows) || !encode_q_like(pb, &qm[0], Q, 128) || !encode_k_like(pb, &qm[1], K, 64) ||
      !encode_k_like(pb, &qm[2], V, 64) || !encode_q_like(pb, &qm[3], dO, 128))
    return FA_ERR_CUDA;
  a.dQ = dQ;
  a.dK = dK;
  a.dV = dV;
  a.err = error_word_ptr();
  if (!a.err) return FA_ERR_CUDA;
  return fa::launch_bwd_wide(a, kv, qm, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status bwd_run(const Problem& pb, const void* Q, const void* K, const void* V, const void* O, const void* dO,
                  const float* LSE, void* dQ, void* dK, void* dV, void* workspace, size_t bytes, void* stream) {
  // Validate everything up front so a rejected call launches none of the stages.
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV) return FA_ERR_INVALID_ARG;
  if (misaligned(Q, 16) || misaligned(K, 16) || misaligned(V, 16) || misaligned(O, 16) || misaligned(dO, 16) ||
      misaligned(LSE, 16) || misaligned(dQ, 16) || misaligned(dK, 16) || misaligned(dV, 16))
    return FA_ERR_INVALID_ARG;
  fa_status st = check_workspace(pb, workspace, bytes);
  if (st != FA_OK) return st;
  if ((st = prepare_run(pb, O, dO, LSE, workspace, bytes, stream)) != FA_OK) return st;
  if (!narrow_head(pb.d)) return wide_tiles_run(pb, Q, K, V, dO, dQ, dK, dV, workspace, stream);
  if ((st = tiles_run(pb, Q, K, V, dO, dK, dV, workspace, bytes, stream)) != FA_OK) return st;
  return finish_run(pb, dQ, workspace, bytes, stream);
}

bool dtype_ok(fa_dtype dtype) { return dtype == FA_DTYPE_BF16 || dtype == FA_DTYPE_F16; }

// ------------------------------------------------------------ host-buffer step

// Device layout of fa_fwd_bwd_host's workspace: kHostSlots staging slots of
// the per-group tensors (Q, K, V, dO in; O, dQ, dK, dV out: [units, N, d]
// 16-bit each; LSE [units, N] fp32), then two backward workspaces of one
// group (even groups compute on the caller's compute stream, odd groups on a
// second one; the groups of one stream run in order and share its workspace).
constexpr int kHostSlots = 4;

struct HostPlan {
  int units_total;   // B * H
  int per_group;     // units in each group but possibly the last
  int groups;        // number of groups
  size_t tensor;     // bytes of one staged [per_group, N, d] 16-bit tensor, rounded to 256
  size_t lse;        // bytes of the staged [per_group, N] LSE, rounded to 256
  size_t slot;       // bytes of one staging slot
  size_t bwd;        // bytes of the shared backward workspace
};

bool host_plan(int B, int H, int N, int d, int groups, HostPlan* hp) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || groups <= 0) return false;
  const long long bh = static_cast<long long>(B) * H;
  if (bh >= (1ll << 31) || bh * N >= (1ll << 31)) return false;
  hp->units_total = static_cast<int>(bh);
  if (groups > hp->units_total) groups = hp->units_total;
  hp->per_group = (hp->units_total + groups - 1) / groups;
  hp->groups = (hp->units_total + hp->per_group - 1) / hp->per_group;
  hp->tensor = round_up(static_cast<size_t>(hp->per_group) * N * d * 2, 256);
  hp->lse = round_up(static_cast<size_t>(hp->per_group) * N * sizeof(float), 256);
  hp->slot = 8 * hp->tensor + hp->lse;
  Problem pb;
  memset(&pb, 0, sizeof(pb));
  pb.seq.B = B;
  pb.seq.H = H;
  pb.seq.units = hp->per_group;
  pb.seq.Nq = N;
  pb.seq.total_q = N;
  pb.d = d;
  hp->bwd = round_up(workspace_bytes(pb), 256);
  return true;
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

// ------------------------------------------------------------ forward

fa_status fa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int N, int d,
                 int causal, float scale, float p_drop, uint64_t seed, void* stream) {
  Problem pb;
  fa_status st = fixed_problem(&pb, B, H, N, N, d, causal, scale, p_drop, seed, false);
  return st != FA_OK ? st : fwd_run(pb, Q, K, V, O, LSE, stream);
}

fa_status fa_fwd_ex(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int N, int d,
                    int causal, float scale, float p_drop, uint64_t seed, fa_dtype dtype, void* stream) {
  if (!dtype_ok(dtype)) return FA_ERR_INVALID_ARG;
  Problem pb;
  fa_status st = fixed_problem(&pb, B, H, N, N, d, causal, scale, p_drop, seed, dtype == FA_DTYPE_F16);
  return st != FA_OK ? st : fwd_run(pb, Q, K, V, O, LSE, stream);
}

fa_status fa_fwd_qk(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int Nq, int Nk,
                    int d, int causal, float scale, float p_drop, uint64_t seed, fa_dtype dtype, void* stream) {
  if (!dtype_ok(dtype)) return FA_ERR_INVALID_ARG;
  Problem pb;
  fa_status st = fixed_problem(&pb, B, H, Nq, Nk, d, causal, scale, p_drop, seed, dtype == FA_DTYPE_F16);
  return st != FA_OK ? st : fwd_run(pb, Q, K, V, O, LSE, stream);
}

fa_status fa_fwd_varlen(const void* Q, const void* K, const void* V, void* O, float* LSE, const int32_t* cu_seqlens_q,
                        const int32_t* cu_seqlens_k, int B, int H, int total_q, int total_k, int max_seqlen_q,
                        int max_seqlen_k, int d, int causal, float scale, float p_drop, uint64_t seed,
                        fa_dtype dtype, void* stream) {
  if (!dtype_ok(dtype)) return FA_ERR_INVALID_ARG;
  Problem pb;
  fa_status st = packed_problem(&pb, cu_seqlens_q, cu_seqlens_k, B, H, total_q, total_k, max_seqlen_q, max_seqlen_k,
                                d, causal, scale, p_drop, seed, dtype == FA_DTYPE_F16);
  return st != FA_OK ? st : fwd_run(pb, Q, K, V, O, LSE, stream);
}

// ------------------------------------------------------------ backward

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  Problem pb;
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || static_cast<long long>(B) * H >= (1ll << 31)) return 0;
  memset(&pb, 0, sizeof(pb));
  pb.seq.B = B;
  pb.seq.H = H;
  pb.seq.units = B * H;
  pb.seq.Nq = N;
  pb.seq.total_q = N;
  pb.d = d;
  return workspace_bytes(pb);
}

size_t fa_bwd_qk_workspace_size(int B, int H, int Nq, int d, int deterministic) {
  Problem pb;
  if (B <= 0 || H <= 0 || Nq <= 0 || d <= 0 || static_cast<long long>(B) * H >= (1ll << 31)) return 0;
  memset(&pb, 0, sizeof(pb));
  pb.seq.B = B;
  pb.seq.H = H;
  pb.seq.units = B * H;
  pb.seq.Nq = Nq;
  pb.seq.total_q = Nq;
  pb.d = d;
  pb.deterministic = deterministic != 0;
  return workspace_bytes(pb);
}

size_t fa_bwd_varlen_workspace_size(int B, int H, int total_q, int max_seqlen_q, int d, int deterministic) {
  Problem pb;
  if (B <= 0 || H <= 0 || total_q <= 0 || max_seqlen_q <= 0 || d <= 0 || static_cast<long long>(B) * H >= (1ll << 31))
    return 0;
  memset(&pb, 0, sizeof(pb));
  pb.seq.cu_q = reinterpret_cast<const int*>(1);  // packed layout: G = H
  pb.seq.B = B;
  pb.seq.H = H;
  pb.seq.units = B * H;
  pb.seq.Nq = max_seqlen_q;
  pb.seq.total_q = total_q;
  pb.d = d;
  pb.deterministic = deterministic != 0;
  return workspace_bytes(pb);
}

fa_status fa_bwd_prepare(const void* O, const void* dO, const float* LSE, int B, int H, int N, int d,
                         void* workspace, size_t workspace_bytes, void* stream) {
  Problem pb;
  fa_status st = fixed_problem(&pb, B, H, N, N, d, 0, 1.0f, 0.0f, 0, false);
  return st != FA_OK ? st : prepare_run(pb, O, dO, LSE, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_tiles(const void* Q, const void* K, const void* V, const void* dO, void* dK, void* dV, int B,
                       int H, int N, int d, int causal, float scale, float p_drop, uint64_t seed, void* workspace,
                       size_t workspace_bytes, void* stream) {
  Problem pb;
  fa_status st = fixed_problem(&pb, B, H, N, N, d, causal, scale, p_drop, seed, false);
  return st != FA_OK ? st : tiles_run(pb, Q, K, V, dO, dK, dV, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_finish(void* dQ, int B, int H, int N, int d, float scale, const void* workspace,
                        size_t workspace_bytes, void* stream) {
  Problem pb;
  fa_status st = fixed_problem(&pb, B, H, N, N, d, 0, scale, 0.0f, 0, false);
  return st != FA_OK ? st : finish_run(pb, dQ, workspace, workspace_bytes, stream);
}

fa_status fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                 void* dQ, void* dK, void* dV, int B, int H, int N, int d, int causal, float scale, float p_drop,
                 uint64_t seed, void* workspace, size_t workspace_bytes, void* stream) {
  Problem pb;
  fa_status st = fixed_problem(&pb, B, H, N, N, d, causal, scale, p_drop, seed, false);
  return st != FA_OK ? st : bwd_run(pb, Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_ex(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                    void* dQ, void* dK, void* dV, int B, int H, int N, int d, int causal, float scale, float p_drop,
                    uint64_t seed, fa_dtype dtype, void* workspace, size_t workspace_bytes, void* stream) {
  if (!dtype_ok(dtype)) return FA_ERR_INVALID_ARG;
  Problem pb;
  fa_status st = fixed_problem(&pb, B, H, N, N, d, causal, scale, p_drop, seed, dtype == FA_DTYPE_F16);
  return st != FA_OK ? st : bwd_run(pb, Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_qk(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                    void* dQ, void* dK, void* dV, int B, int H, int Nq, int Nk, int d, int causal, float scale,
                    float p_drop, uint64_t seed, fa_dtype dtype, int deterministic, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (!dtype_ok(dtype)) return FA_ERR_INVALID_ARG;
  Problem pb;
  fa_status st = fixed_problem(&pb, B, H, Nq, Nk, d, causal, scale, p_drop, seed, dtype == FA_DTYPE_F16);
  if (st != FA_OK) return st;
  pb.deterministic = deterministic != 0;
  return bwd_run(pb, Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, workspace_bytes, stream);
}

fa_status fa_bwd_varlen(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                        void* dQ, void* dK, void* dV, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                        int B, int H, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int d,
                        int causal, float scale, float p_drop, uint64_t seed, fa_dtype dtype, int deterministic,
                        void* workspace, size_t workspace_bytes, void* stream) {
  if (!dtype_ok(dtype)) return FA_ERR_INVALID_ARG;
  Problem pb;
  fa_status st = packed_problem(&pb, cu_seqlens_q, cu_seqlens_k, B, H, total_q, total_k, max_seqlen_q, max_seqlen_k,
                                d, causal, scale, p_drop, seed, dtype == FA_DTYPE_F16);
  if (st != FA_OK) return st;
  pb.deterministic = deterministic != 0;
  return bwd_run(pb, Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, workspace_bytes, stream);
}

// ------------------------------------------------------------ host-buffer step

size_t fa_fwd_bwd_host_workspace_size(int B, int H, int N, int d, int groups) {
  HostPlan hp;
  if (!host_plan(B, H, N, d, groups, &hp)) return 0;
  return kHostSlots * hp.slot + 2 * hp.bwd;
}

fa_status fa_fwd_bwd_host(const void* Q, const void* K, const void* V, const void* dO, void* O, float* LSE,
                          void* dQ, void* dK, void* dV, int B, int H, int N, int d, int causal, float scale,
                          float p_drop, uint64_t seed, fa_dtype dtype, int groups, void* workspace,
                          size_t workspace_bytes_, void* const* streams) {
  if (!dtype_ok(dtype)) return FA_ERR_INVALID_ARG;
  Problem whole;
  fa_status st = fixed_problem(&whole, B, H, N, N, d, causal, scale, p_drop, seed, dtype == FA_DTYPE_F16);
  if (st != FA_OK) return st;
  HostPlan hp;
  if (!host_plan(B, H, N, d, groups, &hp)) return FA_ERR_INVALID_ARG;
  if (!Q || !K || !V || !dO || !O || !LSE || !dQ || !dK || !dV || !streams) return FA_ERR_INVALID_ARG;
  if (!workspace || misaligned(workspace, 256) || workspace_bytes_ < kHostSlots * hp.slot + 2 * hp.bwd)
    return FA_ERR_INVALID_ARG;
  cudaStream_t s_in = static_cast<cudaStream_t>(streams[0]);
  cudaStream_t s_cmp0 = static_cast<cudaStream_t>(streams[1]);
  cudaStream_t s_out = static_cast<cudaStream_t>(streams[2]);
  // odd groups compute on a second stream of the call's own, so that one
  // group's kernels start while the last wave of the previous group's runs
  // (only when the caller asked for overlap with three distinct streams)
  cudaStream_t s_cmp1 = s_cmp0;
  bool own_stream = false;
  if (s_cmp0 != s_in && s_cmp0 != s_out && hp.groups > 1) {
    if (cudaStreamCreateWithFlags(&s_cmp1, cudaStreamNonBlocking) != cudaSuccess) return FA_ERR_CUDA;
    own_stream = true;
  }
  char* ws = static_cast<char*>(workspace);
  char* bwd_ws0 = ws + kHostSlots * hp.slot;  // one backward workspace per compute stream
  char* bwd_ws1 = bwd_ws0 + hp.bwd;
  const size_t row = static_cast<size_t>(N) * d * 2;  // bytes of one unit of a 16-bit tensor
  // events: copy-in done, compute done, copy-out done, per group
  const int ng = hp.groups;
  cudaEvent_t* ev = new cudaEvent_t[3 * ng + 1];
  int made = 0;
  for (; made < 3 * ng + 1; ++made)
    if (cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming) != cudaSuccess) break;
  st = (made == 3 * ng + 1) ? FA_OK : FA_ERR_CUDA;
  // the call starts after the work already on the copy-out stream (an earlier
  // call's last copies still reading the staging slots this call refills)
  if (st == FA_OK && (cudaEventRecord(ev[3 * ng], s_out) != cudaSuccess ||
                      cudaStreamWaitEvent(s_in, ev[3 * ng], 0) != cudaSuccess ||
                      cudaStreamWaitEvent(s_cmp0, ev[3 * ng], 0) != cudaSuccess ||
                      cudaStreamWaitEvent(s_cmp1, ev[3 * ng], 0) != cudaSuccess))
    st = FA_ERR_CUDA;
  const char* src_in[4] = {static_cast<const char*>(Q), static_cast<const char*>(K), static_cast<const char*>(V),
                           static_cast<const char*>(dO)};
  char* dst_out[4] = {static_cast<char*>(O), static_cast<char*>(dQ), static_cast<char*>(dK), static_cast<char*>(dV)};
  for (int g = 0; st == FA_OK && g < ng; ++g) {
    const int u0 = g * hp.per_group;
    const int gu = (u0 + hp.per_group <= hp.units_total) ? hp.per_group : hp.units_total - u0;
    char* slot = ws + (g % kHostSlots) * hp.slot;
    char* in[4] = {slot, slot + hp.tensor, slot + 2 * hp.tensor, slot + 3 * hp.tensor};  // Q, K, V, dO
    char* out[4] = {slot + 4 * hp.tensor, slot + 5 * hp.tensor, slot + 6 * hp.tensor,
                    slot + 7 * hp.tensor};  // O, dQ, dK, dV
    float* lse = reinterpret_cast<float*>(slot + 8 * hp.tensor);
    cudaEvent_t ev_in = ev[3 * g], ev_cmp = ev[3 * g + 1], ev_out = ev[3 * g + 2];
    cudaStream_t s_cmp = (g & 1) ? s_cmp1 : s_cmp0;
    char* bwd_ws = (g & 1) ? bwd_ws1 : bwd_ws0;
    // copy-in: the slot's inputs are free once the group that used it last has computed
    if (g >= kHostSlots && cudaStreamWaitEvent(s_in, ev[3 * (g - kHostSlots) + 1], 0) != cudaSuccess) {
      st = FA_ERR_CUDA;
      break;
    }
    for (int k = 0; k < 4 && st == FA_OK; ++k)
      if (cudaMemcpyAsync(in[k], src_in[k] + static_cast<size_t>(u0) * row, static_cast<size_t>(gu) * row,
                          cudaMemcpyHostToDevice, s_in) != cudaSuccess)
        st = FA_ERR_CUDA;
    if (st != FA_OK || cudaEventRecord(ev_in, s_in) != cudaSuccess) {
      st = FA_ERR_CUDA;
      break;
    }
    // compute: after this group's inputs, and after the slot's outputs of the
    // group before have been copied out
    if (cudaStreamWaitEvent(s_cmp, ev_in, 0) != cudaSuccess ||
        (g >= kHostSlots && cudaStreamWaitEvent(s_cmp, ev[3 * (g - kHostSlots) + 2], 0) != cudaSuccess)) {
      st = FA_ERR_CUDA;
      break;
    }
    Problem pg = whole;  // the group as a problem of gu units starting at unit u0
    pg.seq.units = gu;
    pg.seq.unit0 = u0;
    if ((st = fwd_run(pg, in[0], in[1], in[2], out[0], lse, s_cmp)) != FA_OK) break;
    if ((st = bwd_run(pg, in[0], in[1], in[2], out[0], in[3], lse, out[1], out[2], out[3], bwd_ws, hp.bwd,
                      s_cmp)) != FA_OK)
      break;
    if (cudaEventRecord(ev_cmp, s_cmp) != cudaSuccess) {
      st = FA_ERR_CUDA;
      break;
    }
    // copy-out
    if (cudaStreamWaitEvent(s_out, ev_cmp, 0) != cudaSuccess) {
      st = FA_ERR_CUDA;
      break;
    }
    for (int k = 0; k < 4 && st == FA_OK; ++k)
      if (cudaMemcpyAsync(dst_out[k] + static_cast<size_t>(u0) * row, out[k], static_cast<size_t>(gu) * row,
                          cudaMemcpyDeviceToHost, s_out) != cudaSuccess)
        st = FA_ERR_CUDA;
    if (st == FA_OK && cudaMemcpyAsync(LSE + static_cast<size_t>(u0) * N, lse, static_cast<size_t>(gu) * N * 4,
                                       cudaMemcpyDeviceToHost, s_out) != cudaSuccess)
      st = FA_ERR_CUDA;
    if (st == FA_OK && cudaEventRecord(ev_out, s_out) != cudaSuccess) st = FA_ERR_CUDA;
  }
  // events and the stream may be destroyed while work on them is still queued
  for (int k = 0; k < made; ++k) cudaEventDestroy(ev[k]);
  if (own_stream) cudaStreamDestroy(s_cmp1);
  delete[] ev;
  return st;
}

// ------------------------------------------------------------ decoding over a paged cache

int fa_decode_num_splits(int B, int H_kv, int H, int Nq, int max_seqlen_k) {
  if (B <= 0 || H_kv <= 0 || H <= 0 || Nq <= 0 || max_seqlen_k <= 0 || H % H_kv != 0) return 0;
  const long long rows = static_cast<long long>(H / H_kv) * Nq;
  const long long chunks = (rows + fa::decode_rows_per_cta() - 1) / fa::decode_rows_per_cta();
  const long long ctas = static_cast<long long>(B) * H_kv * chunks;
  const int tiles = (max_seqlen_k + fa::decode_keys_per_tile() - 1) / fa::decode_keys_per_tile();
  // SMs of the device current at the first call (148 on B200; also the answer
  // without a device); a function-local static is initialised once, thread-safely
  static const int sms = [] {
    int dev = 0, n = 0;
    return (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
               ? n
               : 148;
  }();
  // One CTA per SM, each streaming its tiles at about the same rate, plus a
  // fixed cost per CTA (start-up, pipeline fill) worth about 4 tiles, and as
  // much again for the merge launch when split: estimated time = waves x
  // (tiles per CTA + 4) (+ 4).  Take the cheapest count, the fewest splits
  // among equals.
  int best = 1;
  long long best_cost = -1;
  for (int s = 1; s <= 128 && s <= tiles; ++s) {
    const int per = (tiles + s - 1) / s;
    if ((tiles + per - 1) / per != s) continue;  // no split without a tile
    const long long waves = (ctas * s + sms - 1) / sms;
    const long long cost = waves * (per + 4) + (s > 1 ? 4 : 0);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

size_t fa_decode_workspace_size(int B, int H, int Nq, int d, int num_splits) {
  if (B <= 0 || H <= 0 || Nq <= 0 || d <= 0 || num_splits <= 0) return 0;
  if (num_splits == 1) return 0;
  const size_t rows = static_cast<size_t>(B) * H * Nq * num_splits;
  return round_up(rows * d * sizeof(float), 256) + round_up(rows * sizeof(float), 256);
}

fa_status fa_decode_paged(const void* Q, const void* K_cache, const void* V_cache, const int32_t* block_table,
                          const int32_t* seqlens_k, void* O, float* LSE, int B, int H, int H_kv, int Nq, int d,
                          int num_pages, int page_size, int max_pages_per_seq, int max_seqlen_k, int causal,
                          float scale, int num_splits, fa_dtype dtype, void* workspace, size_t workspace_bytes,
                          void* stream) {
  if (!dtype_ok(dtype)) return FA_ERR_INVALID_ARG;
  if (!Q || !K_cache || !V_cache || !block_table || !seqlens_k || !O || !LSE) return FA_ERR_INVALID_ARG;
  if (misaligned(Q, 16) || misaligned(K_cache, 16) || misaligned(V_cache, 16) || misaligned(O, 16) ||
      misaligned(LSE, 4) || misaligned(block_table, 4) || misaligned(seqlens_k, 4))
    return FA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || H_kv <= 0 || Nq <= 0 || d <= 0 || num_pages <= 0 || page_size <= 0 ||
      max_pages_per_seq <= 0 || max_seqlen_k <= 0 || num_splits < 0)
    return FA_ERR_INVALID_ARG;
  if (H % H_kv != 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(max_seqlen_k) > static_cast<long long>(max_pages_per_seq) * page_size)
    return FA_ERR_INVALID_ARG;
  fa_status st = check_scalars(d, scale, 0.0f);
  if (st == FA_OK && !narrow_head(d)) st = FA_ERR_UNSUPPORTED;
  if (st != FA_OK) return st;
  if (page_size != 16 && page_size != 32 && page_size != 64 && page_size != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(num_pages) * page_size >= (1ll << 31) ||
      static_cast<long long>(B) * max_pages_per_seq >= (1ll << 31) ||
      static_cast<long long>(B) * H * Nq >= (1ll << 31) || B > 65535)
    return FA_ERR_UNSUPPORTED;
  const int splits = num_splits ? num_splits : fa_decode_num_splits(B, H_kv, H, Nq, max_seqlen_k);
  if (splits < 1 || splits > 1024) return FA_ERR_INVALID_ARG;
  if (splits > 1) {
    if (!workspace || misaligned(workspace, 256)) return FA_ERR_INVALID_ARG;
    if (workspace_bytes < fa_decode_workspace_size(B, H, Nq, d, splits)) return FA_ERR_INVALID_ARG;
  }
  const int group = H / H_kv;
  const int rows = group * Nq;
  const int chunks = (rows + fa::decode_rows_per_cta() - 1) / fa::decode_rows_per_cta();
  if (static_cast<long long>(H_kv) * chunks > 65535) return FA_ERR_UNSUPPORTED;

  fa::DecodeArgs a;
  memset(&a, 0, sizeof(a));
  const CUtensorMapDataType dt = elem_type(dtype == FA_DTYPE_F16);
  // (d, H_kv, num_pages * page_size) over [num_pages, page_size, H_kv, d]; one box = one page of one head
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return FA_ERR_CUDA;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H_kv),
                        static_cast<cuuint64_t>(num_pages) * page_size};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H_kv) * d * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(page_size)};
  cuuint32_t estr[3] = {1, 1, 1};
  if (enc(&a.tmK, dt, 3, const_cast<void*>(K_cache), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
          CUDA_SUCCESS ||
      enc(&a.tmV, dt, 3, const_cast<void*>(V_cache), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
          CUDA_SUCCESS)
    return FA_ERR_CUDA;
  fa::DecodeParams& p = a.p;
  p.Q = static_cast<const uint16_t*>(Q);
  p.O = static_cast<uint16_t*>(O);
  p.LSE = LSE;
  if (splits > 1) {
    const size_t prow = static_cast<size_t>(B) * H * Nq * splits;
    p.O_part = static_cast<float*>(workspace);
    p.LSE_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + round_up(prow * d * sizeof(float), 256));
  }
  p.block_table = block_table;
  p.seqlens = seqlens_k;
  p.err = error_word_ptr();
  if (!p.err) return FA_ERR_CUDA;
  p.H = H;
  p.Nq = Nq;
  p.group = group;
  p.rows = rows;
  p.row_chunks = chunks;
  p.max_pages = max_pages_per_seq;
  p.page = page_size;
  p.dh = d;
  const int tiles = (max_seqlen_k + fa::decode_keys_per_tile() - 1) / fa::decode_keys_per_tile();
  p.splits = splits;
  p.tiles_per_split = (tiles + splits - 1) / splits;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  a.B = B;
  a.H_kv = H_kv;
  a.d = d;
  a.f16 = dtype == FA_DTYPE_F16 ? 1 : 0;
  return fa::launch_decode(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// ------------------------------------------------------------ utilities

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
