// fa_bwd.cu -- attention backward by recomputation for sm_100a.
//
// The backward pass stores no N x N intermediate: it recomputes the scores
// and probabilities tile by tile from the stored per-row statistic LSE and
// regenerates the dropout pattern from (seed, b, h, i, j) instead of reading
// a stored mask ("FlashAttention" glossary, Recomputation; "Flash Attention"
// glossary, How Flash Attention Works step 6 and Key Components).
//
// Gradients of L = sum(dO * O) with O = (P * Z / (1-p)) V, P = softmax(scale S):
//   dV = (P*Z/(1-p))^T dO            dP = (dO V^T) * Z / (1-p)
//   D_i = sum_c dO_ic O_ic            dS = P * (dP - D)
//   dQ = scale * dS K                 dK = scale * dS^T Q
//
// Three kernels:
//   1. preprocess: D_i = rowsum(dO * O) (fp32, from the stored 16-bit O),
//      LSE2_i = LSE_i * log2(e), and zeroing of the fp32 dQ accumulator;
//   2. main: one CTA per (sequence-or-batch entry, head, 128-key tile j)
//      keeps K_j, V_j in shared memory and dK_j, dV_j in tensor memory while
//      it streams the query tiles i that see a key of tile j (causal: query
//      position i + Nk - Nq >= j) through a two-stage TMA ring.  Per tile:
//        S^T = K_j Q_i^T and dP^T = V_j dO_i^T  (tcgen05, M = 128 keys)
//        P^T = exp2(S^T scale log2e - LSE2_i), masked, dropout-masked
//              -> written in the input type into TMEM over S^T
//        dV += P^T dO_i                          (A operand read from TMEM)
//        dS^T = P^T (dP^T Z/(1-p) - D_i)  -> 16-bit, 128B-swizzled in smem
//        dK += dS^T Q_i ;  dQ_i = dS K_j  (the same smem tile read K-major
//              for dK and MN-major for dQ)
//        dQ_i is read out of TMEM by a dedicated warpgroup, staged through the
//        tile's dO buffer (idle by then) and added to the fp32 accumulator
//        with TMA reduce-add.
//      Deterministic mode fixes the order of those fp32 additions: the key
//      tiles that contribute to a query tile are always 0 .. K, and key tile
//      kj adds only after a per-(unit, query tile) counter in the workspace
//      reaches kj, then increments it.  Query tiles are then visited in
//      descending order, so every key tile meets a given query tile at the
//      same iteration and each waits only for the previous one's add.
//      Warp roles: warpgroups 0/1 do the elementwise work for query columns
//      0-63 / 64-127 (one thread per key row, the TMEM lane); warp 8 issues
//      MMAs; warp 9 issues TMA; warpgroup 3 drains dQ.
//   3. convert: dQ = scale * dQacc, rounded to the input type.
// Inputs and outputs are all bf16 or all fp16 (the F16 template flag); every
// accumulation is fp32.  Each unit's rows come from a SeqLayout (fixed
// [B, H, N, d] or packed variable-length [total, H, d], Nq and Nk may differ);
// head dimensions 32 / 96 run on D = 64 / 128 with zero-filled columns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "fa_internal.h"
#include "philox.cuh"
#include "sm100.cuh"

namespace fa {
namespace {

// ============================================================ preprocess

// One warp per padded row (unit b*H + h, i < Npad): for the unit's queries
// i < nq, D = sum(dO * O) and LSE2 = LSE * log2(e) (+inf for a row that sees
// no key, LSE = -inf); for the padding rows, D = 0 and LSE2 = +inf (so
// exp2(x - LSE2) = 0).  Then the whole fp32 dQ accumulator is zeroed.
template <int D, bool F16>
__global__ void __launch_bounds__(256) fa_bwd_preprocess_kernel(const uint16_t* __restrict__ O,
                                                                const uint16_t* __restrict__ dO,
                                                                const float* __restrict__ LSE,
                                                                float* __restrict__ Dvec,
                                                                float* __restrict__ lse2,
                                                                float* __restrict__ dQacc, const SeqLayout seq,
                                                                int dh, int Npad, long long acc_vec4,
                                                                unsigned* __restrict__ dq_order, int n_order) {
  const int lane = threadIdx.x & 31;
  const int rows_pad = seq.units * Npad;  // < 2^31, checked on the host
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int prow = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); prow < rows_pad; prow += warps) {
    const int unit = prow / Npad;
    const int i = prow - unit * Npad;
    const SeqUnit su = resolve_unit(seq, unit);
    if (i >= su.nq) {
      if (lane == 0) {
        Dvec[prow] = 0.f;
        lse2[prow] = CUDART_INF_F;
      }
      continue;
    }
    const size_t row = static_cast<size_t>(su.q0 + i) * seq.tok_stride + static_cast<size_t>(su.g) * seq.q_head_stride;
    // lane covers elements [8*lane, 8*lane+8) when 8*lane < D
    float acc = 0.f;
    if (lane * 8 < dh) {
      const uint4 a = *reinterpret_cast<const uint4*>(O + row + lane * 8);
      const uint4 b = *reinterpret_cast<const uint4*>(dO + row + lane * 8);
      const uint32_t av[4] = {a.x, a.y, a.z, a.w};
      const uint32_t bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa2 = unpack2<F16>(av[e]);
        const float2 fb2 = unpack2<F16>(bv[e]);
        acc = fmaf(fa2.x, fb2.x, acc);
        acc = fmaf(fa2.y, fb2.y, acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const float l = LSE[static_cast<size_t>(su.g) * seq.total_q + su.q0 + i];
      Dvec[prow] = acc;
      lse2[prow] = (l == -CUDART_INF_F) ? CUDART_INF_F : l * 1.4426950408889634f;
    }
  }
  float4* zq = reinterpret_cast<float4*>(dQacc);
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < acc_vec4;
       idx += static_cast<long long>(gridDim.x) * blockDim.x)
    zq[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (dq_order)
    for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < n_order; idx += gridDim.x * blockDim.x)
      dq_order[idx] = 0u;
}

// ============================================================ dQ convert

// dQ row (g, t) = scale * accumulator row (g, t), rounded to the input type;
// 8 elements per thread.
template <bool F16>
__global__ void __launch_bounds__(256) fa_bwd_dq_convert_kernel(const float* __restrict__ dQacc,
                                                                uint16_t* __restrict__ dQ, float scale,
                                                                const SeqLayout seq, int d, long long n8) {
  const int per_row = d / 8;
  const int shift = (per_row == 16) ? 4 : (per_row == 8) ? 3 : (per_row == 4) ? 2 : -1;  // log2(d / 8), if any
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < n8;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    // fixed length: dQ has the accumulator's layout; packed: row g * total_q + t
    // of the accumulator is token t of head g in [total_q, H, d]
    long long dst = idx * 8;
    if (seq.cu_q) {
      const long long rowl = (shift >= 0) ? (idx >> shift) : idx / per_row;
      const int row = static_cast<int>(rowl);  // < 2^31 rows
      const int part = static_cast<int>(idx - rowl * per_row);
      const int g = row / seq.total_q;
      const int t = row - g * seq.total_q;
      dst = t * seq.tok_stride + g * seq.q_head_stride + part * 8;
    }
    const float4 a = reinterpret_cast<const float4*>(dQacc)[2 * idx];
    const float4 b = reinterpret_cast<const float4*>(dQacc)[2 * idx + 1];
    uint4 o;
    o.x = pack2<F16>(a.x * scale, a.y * scale);
    o.y = pack2<F16>(a.z * scale, a.w * scale);
    o.z = pack2<F16>(b.x * scale, b.y * scale);
    o.w = pack2<F16>(b.z * scale, b.w * scale);
    *reinterpret_cast<uint4*>(dQ + dst) = o;
  }
}

// ============================================================ main kernel

constexpr int kBwdThreads = 512;
constexpr int kBwdMmaWarp = 8;
constexpr int kBwdLoadWarp = 9;
// setmaxnreg split over the launch pool of 512 threads x 128 registers:
// two elementwise warpgroups, the dQ-drain warpgroup, the control warpgroup.
constexpr int kBwdLaunchRegs = 128;
constexpr int kEwRegs = 168;
constexpr int kDqRegs = 120;
constexpr int kCtlRegs = 56;
static_assert(2 * 128 * kEwRegs + 128 * kDqRegs + 128 * kCtlRegs <= kBwdThreads * kBwdLaunchRegs, "register split");

template <int D>
struct BwdSmem {
  static constexpr int kTile = 128 * D * 2;  // 128 rows x D 16-bit elements
  static constexpr int kBox = 128 * 128;     // 128 rows x 64 16-bit (one 128-byte swizzle span)
  static constexpr int kK = 0;
  static constexpr int kV = kTile;
  static constexpr int kQ = 2 * kTile;      // 2 stages
  static constexpr int kDO = 4 * kTile;     // 2 stages
  static constexpr int kDS = 6 * kTile;     // dS^T: 128 keys x 128 queries 16-bit = 2 boxes
  static constexpr int kVec = kDS + 2 * kBox;  // 2 stages x (LSE2[128], D[128]) fp32
  static constexpr int kBar = kVec + 2 * 1024;
  static constexpr int kNumBars = 18;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kUsed = kMisc + 16;
};

enum BwdBar {
  kKVFull = 0,
  kQFull0 = 1,   // +stage
  kDOFull0 = 3,  // +stage
  kEmpty0 = 5,   // +stage
  kSReady = 7,
  kDPReady = 8,
  kPReady = 9,
  kDSReady = 10,
  kDSFree = 11,
  kDQReady = 12,
  kDQFree = 13,
  kDKDVReady = 14,
  kDrain = 15,
  kDOStage0 = 16,  // +stage: the dQ drain has finished staging through that dO buffer
};

struct BwdParams {
  uint16_t* dK;  // bf16 or fp16 bits
  uint16_t* dV;
  float* dQacc;
  const float* lse2;
  const float* Dvec;
  unsigned* dq_order;  // deterministic mode: per (unit, query tile) count of dQ adds done; else nullptr
  unsigned* err;
  SeqLayout seq;
  int dh;  // head dimension of the tensors (D, or 32 / 96 padded to D = 64 / 128)
  float scale;
  float scale_log2;
  uint32_t drop_t;
  float drop_scale;
  uint32_t philox_rk[20];  // Philox round keys (read from the constant bank)
  int group, BH;
};

// MMA helpers.  The MMA warp runs its loop with all 32 lanes, so addresses
// and descriptors are warp-uniform values; ``leader`` (one elected lane)
// issues.  The descriptors are rebuilt from the tile base addresses at each
// use instead of being kept live across the loop (the warpgroup runs with few
// registers): an opaque copy of each base stops the compiler from hoisting
// them out of the loop.
__device__ __forceinline__ uint32_t opaque_u32(uint32_t x) {
  asm volatile("mov.b32 %0, %0;" : "+r"(x));
  return x;
}

// D[tmem] (+)= A[K-major tile] * B[K-major tile]^T, M = N = 128, K = D.
template <int D, bool F16>
__device__ __forceinline__ void mma_tile_kk(bool leader, uint32_t tmem_d, uint32_t a_smem, uint32_t b_smem) {
  a_smem = opaque_u32(a_smem);
  b_smem = opaque_u32(b_smem);
  constexpr uint32_t idesc = idesc_f32acc(128, 128, false, false, F16);
  if (leader) {
    const uint64_t da = sdesc_sw128(a_smem, 16, 1024), db = sdesc_sw128(b_smem, 16, 1024);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = ((kk / 4) * BwdSmem<D>::kBox + (kk % 4) * 32) >> 4;
      mma_ss(tmem_d, da + off, db + off, idesc, kk > 0);
    }
  }
}

// dV (+)= P^T dO : A = P^T (TMEM, 16-bit pairs), B = dO tile (MN-major),
// K = 128 queries, N = D.  P^T of query columns [64 g, 64 g + 64) lies over
// that group's own S^T columns: 32 TMEM columns from tmem_p + 64 g.
template <int D, bool F16>
__device__ __forceinline__ void mma_dv(bool leader, uint32_t tmem_d, uint32_t tmem_p, uint32_t do_smem,
                                       bool accumulate) {
  do_smem = opaque_u32(do_smem);
  constexpr uint32_t idesc = idesc_f32acc(128, D, false, true, F16);
  if (leader) {
    const uint64_t db = sdesc_sw128(do_smem, BwdSmem<D>::kBox, 1024);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_ts(tmem_d, tmem_p + (kk / 4) * 64 + (kk % 4) * 8, db + static_cast<uint32_t>((kk * 2048) >> 4), idesc,
             (accumulate || kk > 0) ? 1u : 0u);
  }
}

// dK (+)= dS^T Q : A = dS^T (smem, K-major over queries), B = Q tile (MN-major), N = D.
template <int D, bool F16>
__device__ __forceinline__ void mma_dk(bool leader, uint32_t tmem_d, uint32_t ds_smem, uint32_t q_smem,
                                       bool accumulate) {
  ds_smem = opaque_u32(ds_smem);
  q_smem = opaque_u32(q_smem);
  constexpr uint32_t idesc = idesc_f32acc(128, D, false, true, F16);
  if (leader) {
    const uint64_t da = sdesc_sw128(ds_smem, 16, 1024), db = sdesc_sw128(q_smem, BwdSmem<D>::kBox, 1024);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t a_off = ((kk / 4) * BwdSmem<D>::kBox + (kk % 4) * 32) >> 4;
      mma_ss(tmem_d, da + a_off, db + static_cast<uint32_t>((kk * 2048) >> 4), idesc, (accumulate || kk > 0) ? 1u : 0u);
    }
  }
}

// dQ_i = dS K : A = dS (the dS^T tile read MN-major, M = queries), B = K tile (MN-major), N = D.
template <int D, bool F16>
__device__ __forceinline__ void mma_dq(bool leader, uint32_t tmem_d, uint32_t ds_smem, uint32_t k_smem) {
  ds_smem = opaque_u32(ds_smem);
  k_smem = opaque_u32(k_smem);
  constexpr uint32_t idesc = idesc_f32acc(128, D, true, true, F16);
  if (leader) {
    const uint64_t da = sdesc_sw128(ds_smem, BwdSmem<D>::kBox, 1024), db = sdesc_sw128(k_smem, BwdSmem<D>::kBox, 1024);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t off = (kk * 2048) >> 4;
      mma_ss(tmem_d, da + off, db + off, idesc, kk > 0 ? 1u : 0u);
    }
  }
}

__device__ __forceinline__ void bwd_teardown(uint32_t tmem, bool dealloc) {
  tc_fence_before();
  asm volatile("bar.sync 1, %0;" ::"n"(kBwdThreads) : "memory");
  tc_fence_after();
  if (dealloc) tmem_dealloc(tmem, 512);
}

template <int D, bool CAUSAL, bool DROPOUT, bool F16, bool DET>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ BwdParams p) {
  using L = BwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (!smem_layout_fits(smem_raw, smem, L::kUsed, p.err)) return;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // 1-D grid over (unit group, key tile, unit), heaviest key tiles first
  // within each group of p.group units.
  const int n_kt_grid = (p.seq.Nk + 127) / 128;
  const int Npad = (p.seq.Nq + 127) / 128 * 128;  // padded rows per unit in the LSE2 / D vectors
  const int per_group = p.group * n_kt_grid;
  const int grp = blockIdx.x / per_group;
  const int rr = blockIdx.x - grp * per_group;
  const int gsz = min(p.group, p.BH - grp * p.group);
  const int kj = rr / gsz;                   // key tile (lowest first: the heaviest causal work)
  const int unit = grp * p.group + (rr - kj * gsz);
  const SeqUnit su = resolve_unit(p.seq, unit);
  if (kj * 128 >= su.nk) return;             // past this unit's keys: no work
  const int n_qt = (su.nq + 127) / 128;
  const int delta = su.nk - su.nq;           // query i sits at key position i + delta
  // first query tile with a row that sees a key of this tile: i + delta >= kj * 128
  const int q_first = CAUSAL ? max(0, floor_div(kj * 128 - delta, 128)) : 0;
  const int nq = n_qt - q_first;             // query tiles visited
  const bool key_valid = kj * 128 + static_cast<int>(threadIdx.x & 127) < su.nk;
  if (nq <= 0) {
    // no query sees these keys: dK = dV = 0 (threads 0-127 take dK, 128-255 dV)
    if (threadIdx.x < 256 && key_valid) {
      uint16_t* dst = ((threadIdx.x < 128) ? p.dK : p.dV) +
                      static_cast<size_t>(su.k0 + kj * 128 + (threadIdx.x & 127)) * p.seq.tok_stride +
                      static_cast<size_t>(su.g) * p.seq.k_head_stride;
      uint4* d4 = reinterpret_cast<uint4*>(dst);
      for (int e = 0; e < D / 8; ++e)
        if (e * 8 < p.dh) d4[e] = make_uint4(0u, 0u, 0u, 0u);
    }
    return;
  }
  const size_t vrow0 = static_cast<size_t>(unit) * Npad;  // this unit's rows in the padded LSE2 / D vectors
  // query tile of iteration it: ascending from q_first, or descending from the
  // last tile in deterministic mode
  constexpr bool det = DET;
  auto qi_of = [&](int it) { return det ? n_qt - 1 - it : q_first + it; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::kNumBars; ++i)
      mbar_init(&bars[i], (i == kPReady || i == kDSReady) ? 8u : (i == kDQFree ? 4u : 1u));
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S^T [0,128) (P^T of query columns 64g.. over [64g, 64g+32)), dP^T / dQ [128,256), dK, dV after.
  constexpr uint32_t kColS = 0, kColDP = 128, kColDK = 256, kColDV = 256 + D;
  const uint32_t sm_k = smem_u32(smem + L::kK), sm_v = smem_u32(smem + L::kV);
  const uint32_t sm_q = smem_u32(smem + L::kQ), sm_do = smem_u32(smem + L::kDO);
  const uint32_t sm_ds = smem_u32(smem + L::kDS);

  if (warp >= 8 && warp < 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtlRegs));
    if (warp == kBwdLoadWarp && lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_expect_tx(&bars[kKVFull], 2 * L::kTile);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(smem + L::kK + c * L::kBox, &tmK, c * 64, su.k0 + kj * 128, su.g, &bars[kKVFull]);
        tma_load_3d(smem + L::kV + c * L::kBox, &tmV, c * 64, su.k0 + kj * 128, su.g, &bars[kKVFull]);
      }
      int issued = 0;
      for (int it = 0; it < nq; ++it) {
        const int s = it & 1;
        const int qrow = qi_of(it) * 128;  // first query row of the tile within the unit
        if (it >= 2 && !mbar_wait(&bars[kEmpty0 + s], ((it >> 1) - 1) & 1, abort_flag, p.err)) break;
        mbar_expect_tx(&bars[kQFull0 + s], L::kTile + 1024);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::kQ + s * L::kTile + c * L::kBox, &tmQ, c * 64, su.q0 + qrow, su.g,
                      &bars[kQFull0 + s]);
        bulk_load_1d(smem + L::kVec + s * 1024, p.lse2 + vrow0 + qrow, 512, &bars[kQFull0 + s]);
        bulk_load_1d(smem + L::kVec + s * 1024 + 512, p.Dvec + vrow0 + qrow, 512, &bars[kQFull0 + s]);
        issued = it + 1;
        // the dO buffer doubles as the dQ drain's staging area two tiles back
        if (it >= 2 && !mbar_wait(&bars[kDOStage0 + s], ((it >> 1) - 1) & 1, abort_flag, p.err)) break;
        mbar_expect_tx(&bars[kDOFull0 + s], L::kTile);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::kDO + s * L::kTile + c * L::kBox, &tmDO, c * 64, su.q0 + qrow, su.g,
                      &bars[kDOFull0 + s]);
      }
      if (*abort_flag) {
        mbar_wait_drain(&bars[kKVFull], 0);
        for (int it = max(0, issued - 2); it < issued; ++it) {
          mbar_wait_drain(&bars[kQFull0 + (it & 1)], (it >> 1) & 1);
          mbar_wait_drain(&bars[kDOFull0 + (it & 1)], (it >> 1) & 1);
        }
      }
    } else if (warp == kBwdMmaWarp) {
      // ---------------------------------------------------------------- MMA issuer
      // the whole warp runs the loop; one elected lane issues and commits
      const bool leader = elect_one();
#define FA_WAIT(b, parity) __all_sync(0xffffffffu, mbar_wait((b), (parity), abort_flag, p.err))
      bool ok = FA_WAIT(&bars[kKVFull], 0) && FA_WAIT(&bars[kQFull0], 0);
      if (ok) {
        tc_fence_after();
        mma_tile_kk<D, F16>(leader, tmem + kColS, sm_k, sm_q);
        if (leader) mma_commit(&bars[kSReady]);
        ok = FA_WAIT(&bars[kDOFull0], 0);
        if (ok) {
          tc_fence_after();
          mma_tile_kk<D, F16>(leader, tmem + kColDP, sm_v, sm_do);
          if (leader) mma_commit(&bars[kDPReady]);
        }
      }
      for (int it = 0; ok && it < nq; ++it) {
        const int s = it & 1, s1 = (it + 1) & 1;
        const bool more = it + 1 < nq;
        if (!FA_WAIT(&bars[kPReady], it & 1)) { ok = false; break; }
        tc_fence_after();
        mma_dv<D, F16>(leader, tmem + kColDV, tmem + kColS, sm_do + s * L::kTile, it > 0);
        if (more) {
          if (!FA_WAIT(&bars[kQFull0 + s1], ((it + 1) >> 1) & 1)) { ok = false; break; }
          tc_fence_after();
          mma_tile_kk<D, F16>(leader, tmem + kColS, sm_k, sm_q + s1 * L::kTile);
          if (leader) mma_commit(&bars[kSReady]);
        }
        if (!FA_WAIT(&bars[kDSReady], it & 1)) { ok = false; break; }
        tc_fence_after();
        // dQ first: the dK MMA runs while the drain lifts dQ out of TMEM
        mma_dq<D, F16>(leader, tmem + kColDP, sm_ds, sm_k);
        if (leader) mma_commit(&bars[kDQReady]);
        mma_dk<D, F16>(leader, tmem + kColDK, sm_ds, sm_q + s * L::kTile, it > 0);
        if (leader) {
          mma_commit(&bars[kEmpty0 + s]);
          mma_commit(&bars[kDSFree]);
        }
        if (more) {
          if (!FA_WAIT(&bars[kDQFree], it & 1) || !FA_WAIT(&bars[kDOFull0 + s1], ((it + 1) >> 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_tile_kk<D, F16>(leader, tmem + kColDP, sm_v, sm_do + s1 * L::kTile);
          if (leader) mma_commit(&bars[kDPReady]);
        }
      }
#undef FA_WAIT
      if (ok) {
        if (leader) mma_commit(&bars[kDKDVReady]);
      } else {
        if (leader) mma_commit(&bars[kDrain]);
        mbar_wait_drain(&bars[kDrain], 0);
      }
    }
    __syncwarp();
    bwd_teardown(tmem, warp == kBwdMmaWarp);
  } else if (warp >= 12) {
    // ------------------------------------------------------------------ dQ drain
    // dQ_i leaves TMEM in two rounds of D/2 columns.  Each round is staged as
    // 32-column fp32 boxes (128-byte swizzled rows) in the dO buffer of this
    // tile -- idle since dV_i and dP^T_i read it, and not refilled until the
    // drain releases it -- and added into the fp32 accumulator by TMA
    // reduce-add.  TMEM is released right after the second load.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kDqRegs));
    constexpr int kCols = D / 2;       // columns per round
    constexpr int kBoxes = kCols / 32;  // 32-column fp32 boxes per round
    const int wq = warp & 3;
    const int c = wq * 32 + lane;  // query row within the tile == TMEM lane (keep bits: key row)
    const uint32_t t_row = tmem + (static_cast<uint32_t>(wq * 32) << 16) + kColDP;
    const bool leader = threadIdx.x == 12 * 32;
    volatile int* go = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);
    for (int it = 0; it < nq; ++it) {
      // one thread waits (bounded); the named barrier hands its verdict to all 128
      if (leader) *go = mbar_wait(&bars[kDQReady], it & 1, abort_flag, p.err) ? 1 : 0;
      asm volatile("bar.sync 2, 128;" ::: "memory");
      if (!*go) break;
      tc_fence_after();
      const int s = it & 1;
      const int qrow = qi_of(it) * 128;
      uint8_t* stage = smem + L::kDO + s * L::kTile;
      const uint32_t st_row = smem_u32(stage) + c * 128;
      uint32_t v[kCols];
#pragma unroll
      for (int k = 0; k < kCols / 32; ++k) tmem_ld32(t_row + 32 * k, v + 32 * k);
      tmem_ld_wait();
#pragma unroll
      for (int k = 0; k < kCols / 32; ++k) reg_fence32(v + 32 * k);
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        if (r > 0) asm volatile("bar.sync 2, 128;" ::: "memory");  // the first pass's reduce has read the buffer
#pragma unroll
        for (int bx = 0; bx < kBoxes; ++bx)
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            st_shared_v4(st_row + bx * L::kBox + ((q4 ^ (c & 7)) << 4), v[32 * bx + 4 * q4],
                         v[32 * bx + 4 * q4 + 1], v[32 * bx + 4 * q4 + 2], v[32 * bx + 4 * q4 + 3]);
        fence_proxy_async_smem();
        if (r == 0) {
#pragma unroll
          for (int k = 0; k < kCols / 32; ++k) tmem_ld32(t_row + kCols + 32 * k, v + 32 * k);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < kCols / 32; ++k) reg_fence32(v + 32 * k);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[kDQFree]);  // all of dQ is out of TMEM
        }
        asm volatile("bar.sync 2, 128;" ::: "memory");
        if (leader) {
          // deterministic: the key tiles before this one have added their part
          unsigned* order = det ? p.dq_order + static_cast<size_t>(unit) * (Npad / 128) + qrow / 128 : nullptr;
          if (det && r == 0) {
            counter_wait_eq(order, static_cast<unsigned>(kj), abort_flag, p.err);
            fence_proxy_async_global();
          }
#pragma unroll
          for (int bx = 0; bx < kBoxes; ++bx)
            // rows past the tensor are skipped; rows of the next packed
            // sequence receive exact zeros (their P is 0 here); boxes of
            // padded columns (head dimension 32 / 96) are not issued
            if (r * kCols + 32 * bx < p.dh)
              tma_reduce_add_3d(&tmDQ, stage + bx * L::kBox, r * kCols + 32 * bx, su.q0 + qrow, su.g);
          bulk_commit_group();
          if (det && r == 1) {
            // both halves are in the accumulator before the next key tile may add
            bulk_wait_group0();
            fence_proxy_async_global();
            counter_release_add(order, 1u);
          } else {
            bulk_wait_group_read0();
          }
        }
      }
      if (leader) mbar_arrive(&bars[kDOStage0 + s]);  // the dO buffer may be refilled
    }
    if (leader) bulk_wait_group0();
    bwd_teardown(tmem, false);
  } else {
    // ------------------------------------------------------------------ elementwise
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kEwRegs));
    const int g = warp >> 2;  // query columns [64 g, 64 g + 64)
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // key row within the tile == TMEM lane
    const uint32_t t_row = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float sl2 = p.scale_log2;
    const uint32_t ds_row = sm_ds + g * L::kBox + r * 128;
    const DropConst dk = make_drop_const(p.drop_t);
    const bool hi_t = p.drop_t > 0x8000u;
    const PhiloxFixed023 phx = philox_fix023(static_cast<uint32_t>((kj * 128 + r) >> 3), static_cast<uint32_t>(su.h),
                                             static_cast<uint32_t>(su.b), p.philox_rk);
    uint32_t zbn[2] = {0u, 0u};
    // both 32-query words of the group's 64 columns (8 Philox calls in lockstep)
    auto keep_tile = [&](int qi_next) {
      const uint32_t q0 = static_cast<uint32_t>(qi_next * 128 + 64 * g);
      if (hi_t)
        keep_bits<true, 2>(phx, q0, p.philox_rk, dk.c2, lane, zbn);
      else
        keep_bits<false, 2>(phx, q0, p.philox_rk, dk.c2, lane, zbn);
    };
    // keep bits of this thread's 64 query columns, computed one tile ahead
    // (at the end of the previous tile, while the warp would wait for S^T)
    if (DROPOUT) {
      keep_tile(qi_of(0));
    }
    // masking: query i = qi * 128 + c sees this thread's key j = kj * 128 + r
    // iff i + Nk - Nq >= j, i.e. c >= lo0 - qi * 128; query tiles up to qi_mask
    // hold such pairs for some key of the tile; a tile past the unit's last
    // key masks whole rows
    const int lo0 = CAUSAL ? kj * 128 + r - delta : -(1 << 30);
    const int qi_mask = CAUSAL ? floor_div(kj * 128 + 126 - delta, 128) : -1;
    const bool tile_past_keys = kj * 128 + 128 > su.nk;
    bool ok = true;
    for (int it = 0; it < nq; ++it) {
      const int s = it & 1;
      const int qi = qi_of(it);
      if (!mbar_wait(&bars[kQFull0 + s], (it >> 1) & 1, abort_flag, p.err) ||
          !mbar_wait(&bars[kSReady], it & 1, abort_flag, p.err)) { ok = false; break; }
      const uint32_t zb[2] = {zbn[0], zbn[1]};
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(t_row + kColS + 64 * g, sr);
      tmem_ld32(t_row + kColS + 64 * g + 32, sr + 32);
      tmem_ld_wait();
      reg_fence32(sr);
      reg_fence32(sr + 32);
      const float* lse2 = reinterpret_cast<const float*>(smem + L::kVec + s * 1024) + 64 * g;
      const float* dvec = lse2 + 128;
      float P[64];
#pragma unroll
      for (int c4 = 0; c4 < 16; ++c4) {
        const float4 l4 = *reinterpret_cast<const float4*>(lse2 + 4 * c4);
        P[4 * c4 + 0] = ex2_approx(fmaf(__uint_as_float(sr[4 * c4 + 0]), sl2, -l4.x));
        P[4 * c4 + 1] = ex2_approx(fmaf(__uint_as_float(sr[4 * c4 + 1]), sl2, -l4.y));
        P[4 * c4 + 2] = ex2_approx(fmaf(__uint_as_float(sr[4 * c4 + 2]), sl2, -l4.z));
        P[4 * c4 + 3] = ex2_approx(fmaf(__uint_as_float(sr[4 * c4 + 3]), sl2, -l4.w));
      }
      // masked: (causal) query columns whose position i + Nk - Nq lies before
      // this key, and the whole row for a key past the unit's keys; queries
      // past the unit's rows already get LSE2 = +inf
      if (qi <= qi_mask || tile_past_keys) {  // the same for the whole warp
        const int lo = key_valid ? lo0 - qi * 128 : 128;  // query columns c < lo are masked
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (64 * g + c < lo) P[c] = 0.f;
      }
      if (DROPOUT) {
        // dropped entries get the sign bit set; dS and the 16-bit pack read it
#pragma unroll
        for (int half = 0; half < 2; ++half)
#pragma unroll
          for (int k4 = 0; k4 < 8; ++k4) mark_dropped4(P + 32 * half + 4 * k4, zb[half] >> (4 * k4));
      }
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c)
        pk[c] = DROPOUT ? pack2_relu<F16>(P[2 * c], P[2 * c + 1]) : pack2<F16>(P[2 * c], P[2 * c + 1]);
      // over this group's own S^T columns: the other group may still be
      // reading its half of S^T from the same TMEM lanes
      tmem_st32(t_row + kColS + 64 * g, pk);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kPReady]);

      if (!mbar_wait(&bars[kDPReady], it & 1, abort_flag, p.err)) { ok = false; break; }
      tc_fence_after();
      uint32_t dr[64];
      tmem_ld32(t_row + kColDP + 64 * g, dr);
      tmem_ld32(t_row + kColDP + 64 * g + 32, dr + 32);
      tmem_ld_wait();
      reg_fence32(dr);
      reg_fence32(dr + 32);
      uint32_t dsk[32];
#pragma unroll
      for (int c4 = 0; c4 < 16; ++c4) {
        const float4 d4 = *reinterpret_cast<const float4*>(dvec + 4 * c4);
        const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 4 * c4 + e;
          const float dp = __uint_as_float(dr[c]);
          // kept: P (dP / (1-p) - D); dropped (sign set): -|P| D
          v[e] = DROPOUT ? fmaxf(P[c], 0.f) * (dp * p.drop_scale) - fabsf(P[c]) * dd[e] : P[c] * (dp - dd[e]);
        }
        dsk[2 * c4] = pack2<F16>(v[0], v[1]);
        dsk[2 * c4 + 1] = pack2<F16>(v[2], v[3]);
      }
      // the dS^T buffer is free once the previous tile's dK / dQ MMAs have read it
      if (it > 0 && !mbar_wait(&bars[kDSFree], (it - 1) & 1, abort_flag, p.err)) { ok = false; break; }
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        st_shared_v4(ds_row + ((ch ^ (r & 7)) << 4), dsk[4 * ch], dsk[4 * ch + 1], dsk[4 * ch + 2],
                     dsk[4 * ch + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kDSReady]);
      if (DROPOUT && it + 1 < nq) {
        keep_tile(qi_of(it + 1));
      }
    }
    if (ok && mbar_wait(&bars[kDKDVReady], 0, abort_flag, p.err)) {
      // -------------------------------------------------------------- dK / dV epilogue
      tc_fence_after();
      const uint32_t col = (g == 0) ? kColDK : kColDV;
      const float mul = (g == 0) ? p.scale : p.drop_scale;
      uint16_t* dst = ((g == 0) ? p.dK : p.dV) + static_cast<size_t>(su.k0 + kj * 128 + r) * p.seq.tok_stride +
                      static_cast<size_t>(su.g) * p.seq.k_head_stride;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(t_row + col + 32 * c, v);
        tmem_ld_wait();
        reg_fence32(v);
        uint32_t o[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          o[e] = pack2<F16>(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
        if (key_valid && 32 * c < p.dh) {  // padded columns are not stored
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) d4[e] = make_uint4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
        }
      }
    }
    bwd_teardown(tmem, false);
  }
}

template <int D, bool CAUSAL, bool DROPOUT, bool F16, bool DET>
cudaError_t launch_bwd_main(const BwdArgs& a, cudaStream_t stream) {
  auto kern = fa_bwd_kernel<D, CAUSAL, DROPOUT, F16, DET>;
  const int used = BwdSmem<D>::kUsed;
  int max_optin = 0, dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  // 1 KB of slack realigns the dynamic shared-memory base to 1024 bytes when
  // it is not already aligned; where the budget is tighter the base must be.
  const int smem = (used + 1024 <= max_optin) ? used + 1024 : used;
  if (smem > max_optin) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes attr;
  e = cudaFuncGetAttributes(&attr, kern);
  if (e != cudaSuccess) return e;
  if (attr.numRegs < kBwdLaunchRegs) return cudaErrorInvalidConfiguration;
  BwdParams p;
  p.dK = static_cast<uint16_t*>(a.dK);
  p.dV = static_cast<uint16_t*>(a.dV);
  p.dQacc = a.dQacc;
  p.dq_order = a.dq_order;
  p.lse2 = a.lse2;
  p.Dvec = a.Dvec;
  p.err = a.err;
  p.seq = a.seq;
  p.dh = a.d;
  p.scale = a.scale;
  p.scale_log2 = a.scale_log2;
  p.drop_t = a.drop_t;
  p.drop_scale = a.drop_scale;
  for (int r = 0; r < 20; ++r) p.philox_rk[r] = a.philox_rk[r];
  p.BH = a.seq.units;
  const int n_kt = (a.seq.Nk + 127) / 128;
  {
    // units per group: about 512 key-tile work units per group; the CTAs
    // running together then stream the same Q / dO tiles and add into the
    // same dQ rows through L2, heaviest (lowest) key tiles first
    p.group = (512 + n_kt / 2) / n_kt;
    if (p.group < 1) p.group = 1;
    if (p.group > p.BH) p.group = p.BH;
  }
  dim3 grid(static_cast<unsigned>(p.BH) * n_kt);
  kern<<<grid, kBwdThreads, smem, stream>>>(a.tmQ, a.tmK, a.tmV, a.tmDO, a.tmDQacc, p);
  return cudaGetLastError();
}

template <bool F16>
void launch_preprocess_typed(const BwdArgs& a, long long blocks, int Npad, long long acc_vec4, cudaStream_t stream) {
  const int n_order = a.dq_order ? a.seq.units * (Npad / 128) : 0;
  const uint16_t* O = static_cast<const uint16_t*>(a.O);
  const uint16_t* dO = static_cast<const uint16_t*>(a.dO);
  if (a.d <= 64)
    fa_bwd_preprocess_kernel<64, F16><<<static_cast<int>(blocks), 256, 0, stream>>>(
        O, dO, a.LSE, a.Dvec, a.lse2, a.dQacc, a.seq, a.d, Npad, acc_vec4, a.dq_order, n_order);
  else
    fa_bwd_preprocess_kernel<128, F16><<<static_cast<int>(blocks), 256, 0, stream>>>(
        O, dO, a.LSE, a.Dvec, a.lse2, a.dQacc, a.seq, a.d, Npad, acc_vec4, a.dq_order, n_order);
}

template <bool F16, bool DET>
cudaError_t launch_bwd_tiles_typed(const BwdArgs& a, cudaStream_t stream) {
  const bool drop = a.drop_t != 0;
  if (a.d <= 64) {
    if (a.causal)
      return drop ? launch_bwd_main<64, true, true, F16, DET>(a, stream)
                  : launch_bwd_main<64, true, false, F16, DET>(a, stream);
    return drop ? launch_bwd_main<64, false, true, F16, DET>(a, stream)
                : launch_bwd_main<64, false, false, F16, DET>(a, stream);
  }
  if (a.causal)
    return drop ? launch_bwd_main<128, true, true, F16, DET>(a, stream)
                : launch_bwd_main<128, true, false, F16, DET>(a, stream);
  return drop ? launch_bwd_main<128, false, true, F16, DET>(a, stream)
              : launch_bwd_main<128, false, false, F16, DET>(a, stream);
}

}  // namespace

cudaError_t launch_bwd_prepare(const BwdArgs& a, cudaStream_t stream) {
  const int Npad = (a.seq.Nq + 127) / 128 * 128;
  const long long rows_pad = static_cast<long long>(a.seq.units) * Npad;
  const long long groups = a.seq.cu_q ? a.seq.H : static_cast<long long>(a.seq.units);
  const long long acc_vec4 = groups * a.seq.total_q * a.d / 4;
  long long blocks = (rows_pad + 7) / 8;  // one warp per row, 8 warps per block
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  if (a.f16)
    launch_preprocess_typed<true>(a, blocks, Npad, acc_vec4, stream);
  else
    launch_preprocess_typed<false>(a, blocks, Npad, acc_vec4, stream);
  return cudaGetLastError();
}

cudaError_t launch_bwd_tiles(const BwdArgs& a, cudaStream_t stream) {
  // deterministic mode is a separate instantiation, so the default kernel
  // carries none of its code
  if (a.dq_order)
    return a.f16 ? launch_bwd_tiles_typed<true, true>(a, stream) : launch_bwd_tiles_typed<false, true>(a, stream);
  return a.f16 ? launch_bwd_tiles_typed<true, false>(a, stream) : launch_bwd_tiles_typed<false, false>(a, stream);
}

cudaError_t launch_bwd_finish(const BwdArgs& a, cudaStream_t stream) {
  const long long groups = a.seq.cu_q ? a.seq.H : static_cast<long long>(a.seq.units);
  const long long n8 = groups * a.seq.total_q * a.d / 8;
  long long blocks = (n8 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  uint16_t* dQ = static_cast<uint16_t*>(a.dQ);
  if (a.f16)
    fa_bwd_dq_convert_kernel<true><<<static_cast<int>(blocks), 256, 0, stream>>>(a.dQacc, dQ, a.scale, a.seq, a.d, n8);
  else
    fa_bwd_dq_convert_kernel<false><<<static_cast<int>(blocks), 256, 0, stream>>>(a.dQacc, dQ, a.scale, a.seq, a.d,
                                                                                 n8);
  return cudaGetLastError();
}

}  // namespace fa
