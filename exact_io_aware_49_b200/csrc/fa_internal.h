// fa_internal.h -- launch interfaces between the C-ABI shim and the kernel
// translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

// Largest dynamic shared memory one CTA can opt into on sm_100 (227 KB); the
// wide-head kernels' layouts are checked against it at compile time (for the
// d <= 128 kernels, setting a size above the device's opt-in limit makes the
// launch return an error).
constexpr int kMaxSmemPerCta = 227 * 1024;

// Where the rows of one (sequence, head) unit live.  Units are numbered
// b * H + h; a launch processes ``units`` of them starting at ``unit0`` (a
// fixed-length problem split into groups of heads: the tensors then hold only
// the group, and unit0 keeps (b, h) -- and with them the dropout counters --
// those of the whole problem).
//  * Fixed length (cu_q == nullptr): every unit has Nq queries and Nk keys;
//    tensors are [B, H, N, d], so a unit's tokens are contiguous rows and the
//    head coordinate of unit u is u itself.
//  * Packed variable length: cu_q / cu_k are device int32 offsets [B + 1]
//    (sequence b owns query rows cu_q[b] .. cu_q[b+1] - 1); tensors are
//    [total, H, d] and the head coordinate is h.  Nq / Nk are then the
//    largest lengths (they size the grid and the padded per-row vectors).
// Row t of head coordinate g of an LSE-like [G, total] array is g * total + t.
struct SeqLayout {
  const int* cu_q;
  const int* cu_k;
  int B, H;
  int units;  // units this launch processes (B * H unless split into groups)
  int unit0;  // global number of the first of them (0 for packed layouts)
  int Nq, Nk;
  int total_q, total_k;         // rows per head coordinate (fixed: Nq, Nk)
  long long tok_stride;         // elements between consecutive tokens of one head
  long long q_head_stride;      // elements between head coordinates of Q, O, dO, dQ
  long long k_head_stride;      // elements between head coordinates of K, V, dK, dV
};

struct SeqUnit {
  int b, h;
  int q0, nq;  // first query row (within the head coordinate) and query count
  int k0, nk;
  int g;       // head coordinate
};

#ifdef __CUDACC__
// Offsets and lengths of one unit.  Packed offsets are clamped into the
// tensors and to the maximum lengths, so inconsistent offsets give wrong
// rows but never an access outside the tensors or the workspace.
__device__ __forceinline__ SeqUnit resolve_unit(const SeqLayout& L, int unit) {
  SeqUnit u;
  const int gu = unit + L.unit0;
  u.b = gu / L.H;
  u.h = gu - u.b * L.H;
  if (L.cu_q) {
    const int qa = min(max(L.cu_q[u.b], 0), L.total_q);
    const int qb = min(max(L.cu_q[u.b + 1], qa), L.total_q);
    const int ka = min(max(L.cu_k[u.b], 0), L.total_k);
    const int kb = min(max(L.cu_k[u.b + 1], ka), L.total_k);
    u.q0 = qa;
    u.nq = min(qb - qa, L.Nq);
    u.k0 = ka;
    u.nk = min(kb - ka, L.Nk);
    u.g = u.h;
  } else {
    u.q0 = 0;
    u.nq = L.Nq;
    u.k0 = 0;
    u.nk = L.Nk;
    u.g = unit;
  }
  return u;
}

// floor(a / b) for b > 0 and any sign of a
__device__ __forceinline__ int floor_div(int a, int b) { return (a >= 0) ? a / b : -((-a + b - 1) / b); }
#endif

struct FwdArgs {
  CUtensorMap tmQ, tmK, tmV;  // 3-D maps (d, token, head coordinate), 64 x 128 x 1 boxes, 128B swizzle
  void* O;                    // same layout and type as Q
  int f16;                    // element type of Q, K, V, O: 0 bf16, 1 fp16
  float* LSE;                 // fp32 [G, total_q]
  unsigned* err;              // device error word
  SeqLayout seq;
  int d;
  int causal;
  float scale_log2;   // scale * log2(e)
  uint32_t drop_t;    // keep <=> u16 >= drop_t (0: no dropout)
  float drop_scale;   // 1 / (1 - p)
  uint32_t seed_lo, seed_hi;
  uint32_t philox_rk[20];  // Philox round keys of the seed (rounds 0..9, k0 / k1 interleaved)
};

struct BwdArgs {
  CUtensorMap tmQ, tmK, tmV, tmDO;  // same layout as the forward maps
  CUtensorMap tmDQacc;               // fp32 [G, total_q, d], 32-column x 128-row boxes, 128B swizzle
  int f16;  // element type of Q, K, V, O, dO, dQ, dK, dV: 0 bf16, 1 fp16
  const void* O;
  const void* dO;
  const float* LSE;
  void* dQ;
  void* dK;
  void* dV;
  float* dQacc;  // fp32 [G, total_q, d] workspace
  float* Dvec;   // fp32 [B*H, Npad] workspace: rowsum(dO * O); 0 past a unit's queries
  float* lse2;   // fp32 [B*H, Npad] workspace: LSE * log2(e); +inf past a unit's queries and for rows that see no key
  unsigned* dq_order;  // deterministic mode: uint32 [B*H, Npad/128] workspace counters, else nullptr
  unsigned* err;
  SeqLayout seq;
  int d;
  int causal;
  float scale;
  float scale_log2;
  uint32_t drop_t;
  float drop_scale;
  uint32_t seed_lo, seed_hi;
  uint32_t philox_rk[20];  // Philox round keys of the seed (rounds 0..9, k0 / k1 interleaved)
};

// Decoding over a paged key/value cache (fa_decode.cu).
struct DecodeParams {
  const uint16_t* Q;   // [B, H, Nq, d]
  uint16_t* O;         // [B, H, Nq, d]
  float* LSE;          // [B, H, Nq]
  float* O_part;       // fp32 [B, H, Nq, splits, d] workspace (splits > 1)
  float* LSE_part;     // fp32 [B, H, Nq, splits] workspace (splits > 1)
  const int* block_table;  // [B, max_pages]
  const int* seqlens;      // [B]
  unsigned* err;
  int H, Nq, group;    // group = H / H_kv query heads per key/value head
  int rows;            // group * Nq query rows per key/value head
  int row_chunks;      // blocks of up to 16 rows
  int max_pages, page;
  int dh;  // head dimension of the tensors (D, or 32 / 96 padded to D = 64 / 128)
  int splits, tiles_per_split;
  int causal;
  float scale_log2;
};

struct DecodeArgs {
  CUtensorMap tmK, tmV;  // (d, H_kv, num_pages * page) maps, 64 x 1 x page boxes, 128B swizzle
  DecodeParams p;
  int B, H_kv, d, f16;
};

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);
int decode_rows_per_cta();
int decode_keys_per_tile();

cudaError_t launch_fwd(const FwdArgs& a, cudaStream_t stream);
// Head dimensions 192 and 256: one 128-row query tile per CTA, 64-key K/V tiles
// (the K and V tensor maps then have 64-row boxes).
cudaError_t launch_fwd_wide(const FwdArgs& a, cudaStream_t stream);
// The three backward stages; fa_bwd runs them in this order.  Only the fields
// each stage reads need to be set.
cudaError_t launch_bwd_prepare(const BwdArgs& a, cudaStream_t stream);  // O, dO, LSE -> Dvec, lse2, dQacc = 0
cudaError_t launch_bwd_tiles(const BwdArgs& a, cudaStream_t stream);    // maps, lse2, Dvec -> dK, dV, dQacc
cudaError_t launch_bwd_finish(const BwdArgs& a, cudaStream_t stream);   // dQacc -> dQ
// Head dimensions 192 and 256 (fa_bwd_wide.cu): maps_kv = Q, K, V, dO tensor
// maps with wide_kv_query_rows(d)-, 128-, 128-, wide_kv_query_rows(d)-row
// boxes; maps_q = the same with 128-, 64-, 64-, 128-row boxes.  Reads Dvec and
// lse2 (launch_bwd_prepare), writes dQ, dK, dV.
int wide_kv_query_rows(int d);
cudaError_t launch_bwd_wide(const BwdArgs& a, const CUtensorMap* maps_kv, const CUtensorMap* maps_q,
                            cudaStream_t stream);
cudaError_t launch_wait_timeout_probe(unsigned* err, unsigned long long limit_ns, cudaStream_t stream);
cudaError_t launch_dropout_mask(uint8_t* mask, int B, int H, int N, uint32_t drop_t, uint32_t seed_lo,
                                uint32_t seed_hi, cudaStream_t stream);

}  // namespace fa
