// fa_bwd_wide.cu -- attention backward for head dimensions 192 and 256
// (sm_100a).
//
// Same gradients as fa_bwd.cu (recomputation of P from the stored LSE, the
// dropout pattern regenerated from (seed, b, h, i, j); "FlashAttention"
// glossary, Recomputation; "Flash Attention" glossary, step 6 and Key
// Components):
//   dV = (P*Z/(1-p))^T dO    dP = (dO V^T) * Z/(1-p)    D_i = sum_c dO_ic O_ic
//   dS = P * (dP - D)        dQ = scale dS K            dK = scale dS^T Q
// At d = 192 / 256 the d <= 128 kernel's tensor memory (S^T, dP^T, dK, dV of
// a 128-key tile plus the dQ drain) does not fit, so the work is split in two
// kernels that each keep one kind of output on chip:
//  1. dK, dV: one CTA per (unit, 128-key tile[, half of the d columns at
//     d = 256]) keeps K and V in shared memory and dK, dV in tensor memory
//     while it streams query tiles of Q and dO through two stages (64
//     queries at d = 192, 32 at d = 256, where the resident K and V leave
//     room for only 64 KB of stages): S^T = K Q^T and
//     dP^T = V dO^T over the full d, P^T (masked, dropout-marked) back into
//     TMEM, dS^T into shared memory, dV += P^T dO and dK += dS^T Q for its
//     output columns (the two halves at d = 256 recompute S^T and dP^T);
//  2. dQ: one CTA per (unit, 128-query tile) keeps Q and dO in shared memory
//     and dQ in tensor memory while it streams 64-key tiles of K and V:
//     S = Q K^T, dP = dO V^T, dS into TMEM over S, dQ += dS K; dQ is written
//     once by its CTA, so it needs no accumulator and no ordering.
// D and LSE * log2(e) come from fa_bwd.cu's preprocess kernel.  Warps: 0-3
// elementwise (one thread per key row in kernel 1, per query row in kernel
// 2), 4 MMA issue, 5 TMA loads.
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

constexpr int kWThreads = 192;
constexpr int kWMma = 4;
constexpr int kWLoad = 5;
constexpr int kBox128 = 128 * 128;  // 128 rows x 64 columns of 16-bit (128-byte rows)
constexpr int kBox64 = 64 * 128;    // 64 rows x 64 columns

struct WideBwdParams {
  uint16_t* dQ;  // kernel 2
  uint16_t* dK;  // kernel 1
  uint16_t* dV;
  const float* lse2;
  const float* Dvec;
  unsigned* err;
  SeqLayout seq;
  float scale, scale_log2;
  uint32_t drop_t;
  float drop_scale;
  uint32_t philox_rk[20];
  int group, BH;
};

__device__ __forceinline__ void wide_bwd_teardown(uint32_t tmem, bool dealloc) {
  tc_fence_before();
  asm volatile("bar.sync 1, %0;" ::"n"(kWThreads) : "memory");
  tc_fence_after();
  if (dealloc) tmem_dealloc(tmem, 512);
}

// MMA helpers.  The MMA warps run their loops with all 32 lanes, so
// descriptors are warp-uniform values; ``leader`` (one elected lane) issues.
// Operands are descriptors of the tile's first box; each K-step adds its box
// / swizzle-atom offset (bytes / 16) to the start-address field.

// D[tmem] (+)= A * B^T over K = D (both K-major): A has 128 rows in 128-row
// boxes, B has 64 rows in 64-row boxes; N = 64.  a0 / b0: sdesc_sw128(x, 16, 1024).
template <int D, bool F16, int NB = 64>
__device__ __forceinline__ void mma_rows128_x_rows64(bool leader, uint32_t tmem_d, uint64_t a0, uint64_t b0) {
  // B has NB rows (64 or 32) in NB-row boxes; N = NB
  constexpr uint32_t idesc = idesc_f32acc(128, NB, false, false, F16);
  if (leader) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
      mma_ss(tmem_d, a0 + static_cast<uint32_t>(((kk / 4) * kBox128 + (kk % 4) * 32) >> 4),
             b0 + static_cast<uint32_t>(((kk / 4) * (NB * 128) + (kk % 4) * 32) >> 4), idesc, kk > 0);
  }
}

// D[tmem] (+)= A[tmem, 16-bit pairs] * B over K = 64 rows of B, N = NC columns
// of B (B MN-major in 64-row boxes 8 KB apart); b0: sdesc_sw128(first box, kBox64, 1024).
template <int NC, bool F16, int NB = 64>
__device__ __forceinline__ void mma_tmemA_x_rows64(bool leader, uint32_t tmem_d, uint32_t tmem_a, uint64_t b0,
                                                   bool accumulate) {
  // K = NB rows of B (64 or 32)
  constexpr uint32_t idesc = idesc_f32acc(128, NC, false, true, F16);
  if (leader) {
#pragma unroll
    for (int kk = 0; kk < NB / 16; ++kk)
      mma_ts(tmem_d, tmem_a + kk * 8, b0 + static_cast<uint32_t>((kk * 2048) >> 4), idesc,
             (accumulate || kk > 0) ? 1u : 0u);
  }
}

__device__ __forceinline__ uint64_t desc_off(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

// ============================================================ kernel 1: dK, dV

template <int D>
struct KvSmem {
  static constexpr int kCols = (D == 256) ? 128 : D;     // output columns per CTA
  static constexpr int kSplit = D / kCols;                // CTAs per key tile
  static constexpr int kQT = (D == 256) ? 32 : 64;        // queries per stage
  static constexpr int kStages = 2;
  static constexpr int kBoxQ = kQT * 128;                 // one 64-column box of a Q or dO stage
  static constexpr int kKV = (D / 64) * kBox128;          // K or V: 128 keys x D
  static constexpr int kQS = (D / 64) * kBoxQ;            // one Q or dO stage: kQT queries x D
  static constexpr int kK = 0;
  static constexpr int kV = kKV;
  static constexpr int kQ = 2 * kKV;
  static constexpr int kDO = kQ + kStages * kQS;
  static constexpr int kDS = kDO + kStages * kQS;         // dS^T: 128 keys x kQT queries in one 128-row box
  static constexpr int kVec = kDS + kBox128;              // stages x (LSE2[kQT], D[kQT]) fp32
  static constexpr int kVecStage = 2 * kQT * 4;
  static constexpr int kBar = kVec + kStages * kVecStage;
  // barriers: kv, full[S], empty[S], s, dp, p, ds, ds_free, dkdv, drain
  static constexpr int kNumBars = 1 + 2 * kStages + 7;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16 + 1024;
};
static_assert(KvSmem<192>::kBytes <= kMaxSmemPerCta && KvSmem<256>::kBytes <= kMaxSmemPerCta,
              "dK / dV kernel shared memory");

template <int D, bool CAUSAL, bool DROPOUT, bool F16>
__global__ void __launch_bounds__(kWThreads, 1)
    fa_bwd_wide_kv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                          const __grid_constant__ WideBwdParams p) {
  using L = KvSmem<D>;
  constexpr int S = L::kStages;
  constexpr int NC = L::kCols;
  constexpr int QT = L::kQT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (!smem_layout_fits(smem_raw, smem, L::kMisc + 16, p.err)) return;
  uint64_t* b = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* b_kv = b;
  uint64_t* b_full = b + 1;
  uint64_t* b_empty = b + 1 + S;
  uint64_t* b_s = b + 1 + 2 * S;
  uint64_t* b_dp = b_s + 1;
  uint64_t* b_p = b_s + 2;
  uint64_t* b_ds = b_s + 3;
  uint64_t* b_dsfree = b_s + 4;
  uint64_t* b_dkdv = b_s + 5;
  uint64_t* b_drain = b_s + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // 1-D grid over (unit group, key tile, column half, unit), heaviest key tiles first
  const int n_kt_grid = (p.seq.Nk + 127) / 128;
  const int per_group = p.group * n_kt_grid * L::kSplit;
  const int grp = blockIdx.x / per_group;
  const int rr = blockIdx.x - grp * per_group;
  const int gsz = min(p.group, p.BH - grp * p.group);
  const int kjh = rr / gsz;
  const int kj = kjh / L::kSplit;
  const int hc = kjh - kj * L::kSplit;  // which output columns: [hc * NC, hc * NC + NC)
  const int unit = grp * p.group + (rr - kjh * gsz);
  const SeqUnit su = resolve_unit(p.seq, unit);
  if (kj * 128 >= su.nk) return;
  const int Npad = (p.seq.Nq + 127) / 128 * 128;  // padded rows per unit in LSE2 / D
  const int n_qt = (su.nq + QT - 1) / QT;        // QT-query tiles
  const int delta = su.nk - su.nq;
  const int q_first = CAUSAL ? max(0, floor_div(kj * 128 - delta, QT)) : 0;
  const int nq = n_qt - q_first;
  const bool key_valid = kj * 128 + static_cast<int>(threadIdx.x & 127) < su.nk;
  if (nq <= 0) {
    // no query sees these keys: dK = dV = 0 on this CTA's columns
    if (threadIdx.x < 128 && key_valid) {
      const size_t row = static_cast<size_t>(su.k0 + kj * 128 + threadIdx.x) * p.seq.tok_stride +
                         static_cast<size_t>(su.g) * p.seq.k_head_stride + hc * NC;
      for (int e = 0; e < NC / 8; ++e) {
        reinterpret_cast<uint4*>(p.dK + row)[e] = make_uint4(0u, 0u, 0u, 0u);
        reinterpret_cast<uint4*>(p.dV + row)[e] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    return;
  }
  const size_t vrow0 = static_cast<size_t>(unit) * Npad;

  if (threadIdx.x == 0) {
    mbar_init(b_kv, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    mbar_init(b_s, 1);
    mbar_init(b_dp, 1);
    mbar_init(b_p, 4);
    mbar_init(b_ds, 4);
    mbar_init(b_dsfree, 1);
    mbar_init(b_dkdv, 1);
    mbar_init(b_drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kWMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM: S^T [0, QT) (P^T over [0, QT / 2)), dP^T [64, 64 + QT), dK [128, 128 + NC), dV after it
  constexpr uint32_t kColS = 0, kColDP = 64, kColDK = 128, kColDV = 128 + NC;
  const uint32_t sm_k = smem_u32(smem + L::kK), sm_v = smem_u32(smem + L::kV);
  const uint32_t sm_q = smem_u32(smem + L::kQ), sm_do = smem_u32(smem + L::kDO);
  const uint32_t sm_ds = smem_u32(smem + L::kDS);

  if (warp == kWLoad) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_expect_tx(b_kv, 2 * L::kKV);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(smem + L::kK + c * kBox128, &tmK, c * 64, su.k0 + kj * 128, su.g, b_kv);
        tma_load_3d(smem + L::kV + c * kBox128, &tmV, c * 64, su.k0 + kj * 128, su.g, b_kv);
      }
      int issued = 0;
      for (int it = 0; it < nq; ++it) {
        const int s = it % S;
        const int qrow = (q_first + it) * QT;
        if (it >= S && !mbar_wait(&b_empty[s], ((it / S) - 1) & 1, abort_flag, p.err)) break;
        mbar_expect_tx(&b_full[s], 2 * L::kQS + L::kVecStage);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(smem + L::kQ + s * L::kQS + c * L::kBoxQ, &tmQ, c * 64, su.q0 + qrow, su.g, &b_full[s]);
          tma_load_3d(smem + L::kDO + s * L::kQS + c * L::kBoxQ, &tmDO, c * 64, su.q0 + qrow, su.g, &b_full[s]);
        }
        bulk_load_1d(smem + L::kVec + s * L::kVecStage, p.lse2 + vrow0 + qrow, QT * 4, &b_full[s]);
        bulk_load_1d(smem + L::kVec + s * L::kVecStage + QT * 4, p.Dvec + vrow0 + qrow, QT * 4, &b_full[s]);
        issued = it + 1;
      }
      if (*abort_flag) {
        mbar_wait_drain(b_kv, 0);
        for (int it = max(0, issued - S); it < issued; ++it) mbar_wait_drain(&b_full[it % S], (it / S) & 1);
      }
    }
    __syncwarp();
    wide_bwd_teardown(tmem, false);
    return;
  }
  if (warp == kWMma) {
    {
      const bool leader = elect_one();
      const uint64_t dk_k = sdesc_sw128(sm_k, 16, 1024), dk_v = sdesc_sw128(sm_v, 16, 1024);
      const uint64_t dk_q = sdesc_sw128(sm_q, 16, 1024), dk_do = sdesc_sw128(sm_do, 16, 1024);
      const uint64_t dk_ds = sdesc_sw128(sm_ds, 16, 1024);
      const uint64_t dmn_q = sdesc_sw128(sm_q, L::kBoxQ, 1024), dmn_do = sdesc_sw128(sm_do, L::kBoxQ, 1024);
      const uint32_t col_off = hc * (NC / 64) * L::kBoxQ;  // this CTA's output columns
      // every lane waits; the vote keeps the warp's decision uniform
#define FA_WAIT(b, parity) __all_sync(0xffffffffu, mbar_wait((b), (parity), abort_flag, p.err))
      bool ok = FA_WAIT(b_kv, 0) && FA_WAIT(&b_full[0], 0);
      if (ok) {
        tc_fence_after();
        mma_rows128_x_rows64<D, F16, QT>(leader, tmem + kColS, dk_k, dk_q);
        if (leader) mma_commit(b_s);
        mma_rows128_x_rows64<D, F16, QT>(leader, tmem + kColDP, dk_v, dk_do);
        if (leader) mma_commit(b_dp);
      }
      for (int it = 0; ok && it < nq; ++it) {
        const int s = it % S;
        if (!FA_WAIT(b_p, it & 1)) { ok = false; break; }
        tc_fence_after();
        // dV += P^T dO (this CTA's columns)
        mma_tmemA_x_rows64<NC, F16, QT>(leader, tmem + kColDV, tmem + kColS,
                                        desc_off(dmn_do, s * L::kQS + col_off), it > 0);
        if (!FA_WAIT(b_ds, it & 1)) { ok = false; break; }
        tc_fence_after();
        // dK += dS^T Q : A = dS^T (128 keys x 64 queries, K-major), B = Q columns (MN-major)
        {
          constexpr uint32_t idesc = idesc_f32acc(128, NC, false, true, F16);
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < QT / 16; ++kk)
              mma_ss(tmem + kColDK, desc_off(dk_ds, kk * 32), desc_off(dmn_q, s * L::kQS + col_off + kk * 2048),
                     idesc, (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        if (leader) {
          mma_commit(b_dsfree);
          mma_commit(&b_empty[s]);
        }
        if (it + 1 < nq) {
          const int s1 = (it + 1) % S;
          if (!FA_WAIT(&b_full[s1], ((it + 1) / S) & 1)) { ok = false; break; }
          tc_fence_after();
          mma_rows128_x_rows64<D, F16, QT>(leader, tmem + kColS, dk_k, desc_off(dk_q, s1 * L::kQS));
          if (leader) mma_commit(b_s);
          mma_rows128_x_rows64<D, F16, QT>(leader, tmem + kColDP, dk_v, desc_off(dk_do, s1 * L::kQS));
          if (leader) mma_commit(b_dp);
        }
      }
#undef FA_WAIT
      if (ok) {
        if (leader) mma_commit(b_dkdv);
      } else {
        if (leader) mma_commit(b_drain);
        mbar_wait_drain(b_drain, 0);
      }
    }
    __syncwarp();
    wide_bwd_teardown(tmem, true);
    return;
  }

  // ------------------------------------------------------------ elementwise (thread = key row)
  const int r = warp * 32 + lane;
  const uint32_t t_row = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  const float sl2 = p.scale_log2;
  const DropConst dk = make_drop_const(p.drop_t);
  const bool hi_t = p.drop_t > 0x8000u;
  const PhiloxFixed023 phx = philox_fix023(static_cast<uint32_t>((kj * 128 + r) >> 3), static_cast<uint32_t>(su.h),
                                           static_cast<uint32_t>(su.b), p.philox_rk);
  const uint32_t ds_row = sm_ds + r * 128;
  // query i = qt * QT + c sees key j = kj * 128 + r iff i + delta >= j
  const int lo0 = CAUSAL ? kj * 128 + r - delta : -(1 << 30);
  const bool tile_past_keys = kj * 128 + 128 > su.nk;
  bool ok = true;
  for (int it = 0; it < nq; ++it) {
    const int s = it % S;
    const int qt = q_first + it;
    uint32_t zb[QT / 32];
#pragma unroll
    for (int w = 0; w < QT / 32; ++w) zb[w] = 0u;
    if (DROPOUT) {
      const uint32_t q0 = static_cast<uint32_t>(qt * QT);
      if (hi_t)
        keep_bits<true, QT / 32>(phx, q0, p.philox_rk, dk.c2, lane, zb);
      else
        keep_bits<false, QT / 32>(phx, q0, p.philox_rk, dk.c2, lane, zb);
    }
    if (!mbar_wait(&b_full[s], (it / S) & 1, abort_flag, p.err) || !mbar_wait(b_s, it & 1, abort_flag, p.err)) {
      ok = false;
      break;
    }
    tc_fence_after();
    uint32_t sr[QT];
#pragma unroll
    for (int c = 0; c < QT / 32; ++c) tmem_ld32(t_row + kColS + 32 * c, sr + 32 * c);
    tmem_ld_wait();
#pragma unroll
    for (int c = 0; c < QT / 32; ++c) reg_fence32(sr + 32 * c);
    const float* lse2 = reinterpret_cast<const float*>(smem + L::kVec + s * L::kVecStage);
    const float* dvec = lse2 + QT;
    float P[QT];
#pragma unroll
    for (int c4 = 0; c4 < QT / 4; ++c4) {
      const float4 l4 = *reinterpret_cast<const float4*>(lse2 + 4 * c4);
      P[4 * c4 + 0] = ex2_approx(fmaf(__uint_as_float(sr[4 * c4 + 0]), sl2, -l4.x));
      P[4 * c4 + 1] = ex2_approx(fmaf(__uint_as_float(sr[4 * c4 + 1]), sl2, -l4.y));
      P[4 * c4 + 2] = ex2_approx(fmaf(__uint_as_float(sr[4 * c4 + 2]), sl2, -l4.z));
      P[4 * c4 + 3] = ex2_approx(fmaf(__uint_as_float(sr[4 * c4 + 3]), sl2, -l4.w));
    }
    {
      // masked: query columns before this key's position (causal), every column
      // for a key past the unit's keys; queries past the unit have LSE2 = +inf
      const int lo = key_valid ? lo0 - qt * QT : QT;
      if ((CAUSAL && lo > 0) || tile_past_keys) {
#pragma unroll
        for (int c = 0; c < QT; ++c)
          if (c < lo) P[c] = 0.f;
      }
    }
    if (DROPOUT) {
#pragma unroll
      for (int half = 0; half < QT / 32; ++half)
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) mark_dropped4(P + 32 * half + 4 * k4, zb[half] >> (4 * k4));
    }
    uint32_t pk[QT / 2];
#pragma unroll
    for (int c = 0; c < QT / 2; ++c)
      pk[c] = DROPOUT ? pack2_relu<F16>(P[2 * c], P[2 * c + 1]) : pack2<F16>(P[2 * c], P[2 * c + 1]);
    if constexpr (QT == 64)
      tmem_st32(t_row + kColS, pk);
    else
      tmem_st16(t_row + kColS, pk);
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(b_p);
    if (!mbar_wait(b_dp, it & 1, abort_flag, p.err)) { ok = false; break; }
    tc_fence_after();
    uint32_t dr[QT];
#pragma unroll
    for (int c = 0; c < QT / 32; ++c) tmem_ld32(t_row + kColDP + 32 * c, dr + 32 * c);
    tmem_ld_wait();
#pragma unroll
    for (int c = 0; c < QT / 32; ++c) reg_fence32(dr + 32 * c);
    uint32_t dsk[QT / 2];
#pragma unroll
    for (int c4 = 0; c4 < QT / 4; ++c4) {
      const float4 d4 = *reinterpret_cast<const float4*>(dvec + 4 * c4);
      const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = 4 * c4 + e;
        const float dp = __uint_as_float(dr[c]);
        v[e] = DROPOUT ? fmaxf(P[c], 0.f) * (dp * p.drop_scale) - fabsf(P[c]) * dd[e] : P[c] * (dp - dd[e]);
      }
      dsk[2 * c4] = pack2<F16>(v[0], v[1]);
      dsk[2 * c4 + 1] = pack2<F16>(v[2], v[3]);
    }
    if (it > 0 && !mbar_wait(b_dsfree, (it - 1) & 1, abort_flag, p.err)) { ok = false; break; }
    // dS^T rows of QT queries (QT * 2 bytes of each 128-byte swizzled row)
#pragma unroll
    for (int ch = 0; ch < QT / 8; ++ch)
      st_shared_v4(ds_row + ((ch ^ (r & 7)) << 4), dsk[4 * ch], dsk[4 * ch + 1], dsk[4 * ch + 2], dsk[4 * ch + 3]);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(b_ds);
  }
  if (ok && mbar_wait(b_dkdv, 0, abort_flag, p.err)) {
    tc_fence_after();
    const size_t row = static_cast<size_t>(su.k0 + kj * 128 + r) * p.seq.tok_stride +
                       static_cast<size_t>(su.g) * p.seq.k_head_stride + hc * NC;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const uint32_t col = which ? kColDV : kColDK;
      const float mul = which ? p.drop_scale : p.scale;
      uint16_t* dst = (which ? p.dV : p.dK) + row;
#pragma unroll
      for (int c = 0; c < NC / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(t_row + col + 32 * c, v);
        tmem_ld_wait();
        reg_fence32(v);
        uint32_t o[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          o[e] = pack2<F16>(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
        if (key_valid) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) d4[e] = make_uint4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
        }
      }
    }
  }
  wide_bwd_teardown(tmem, false);
}

// ============================================================ kernel 2: dQ

template <int D>
struct QSmem {
  static constexpr int kStages = (D == 256) ? 1 : 2;
  static constexpr int kQD = (D / 64) * kBox128;  // Q or dO: 128 queries x D
  static constexpr int kKS = (D / 64) * kBox64;   // one K or V stage: 64 keys x D
  static constexpr int kQ = 0;
  static constexpr int kDO = kQD;
  static constexpr int kK = 2 * kQD;
  static constexpr int kV = kK + kStages * kKS;
  static constexpr int kBar = kV + kStages * kKS;
  // barriers: qdo, kfull[S], vfull[S], empty[S], s, dp, ds, dq, drain
  static constexpr int kNumBars = 1 + 3 * kStages + 5;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16 + 1024;
};
static_assert(QSmem<192>::kBytes <= kMaxSmemPerCta && QSmem<256>::kBytes <= kMaxSmemPerCta,
              "dQ kernel shared memory");

template <int D, bool CAUSAL, bool DROPOUT, bool F16>
__global__ void __launch_bounds__(kWThreads, 1)
    fa_bwd_wide_q_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                         const __grid_constant__ WideBwdParams p) {
  using L = QSmem<D>;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (!smem_layout_fits(smem_raw, smem, L::kMisc + 16, p.err)) return;
  uint64_t* b = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* b_qdo = b;
  uint64_t* b_kfull = b + 1;
  uint64_t* b_vfull = b + 1 + S;
  uint64_t* b_empty = b + 1 + 2 * S;
  uint64_t* b_s = b + 1 + 3 * S;
  uint64_t* b_dp = b_s + 1;
  uint64_t* b_ds = b_s + 2;
  uint64_t* b_dq = b_s + 3;
  uint64_t* b_drain = b_s + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_qt_grid = (p.seq.Nq + 127) / 128;
  const int per_group = p.group * n_qt_grid;
  const int grp = blockIdx.x / per_group;
  const int rr = blockIdx.x - grp * per_group;
  const int gsz = min(p.group, p.BH - grp * p.group);
  const int qt_lin = rr / gsz;
  const int unit = grp * p.group + (rr - qt_lin * gsz);
  const SeqUnit su = resolve_unit(p.seq, unit);
  const int qt = CAUSAL ? (n_qt_grid - 1 - qt_lin) : qt_lin;
  if (qt * 128 >= su.nq) return;
  const int Npad = (p.seq.Nq + 127) / 128 * 128;
  const int n_kt = (su.nk + 63) / 64;
  const int delta = su.nk - su.nq;
  const int last_row = min(su.nq - 1, qt * 128 + 127);
  const int nt = CAUSAL ? min(n_kt, max(0, floor_div(last_row + delta, 64) + 1)) : n_kt;
  const int r = threadIdx.x & 127;
  const int i = qt * 128 + r;
  const bool row_ok = i < su.nq;
  uint16_t* dq_row = p.dQ + static_cast<size_t>(su.q0 + i) * p.seq.tok_stride +
                     static_cast<size_t>(su.g) * p.seq.q_head_stride;
  if (nt == 0) {
    // no key is visible to these queries: dQ = 0
    if (threadIdx.x < 128 && row_ok)
      for (int e = 0; e < D / 8; ++e) reinterpret_cast<uint4*>(dq_row)[e] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(b_qdo, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&b_kfull[s], 1);
      mbar_init(&b_vfull[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    mbar_init(b_s, 1);
    mbar_init(b_dp, 1);
    mbar_init(b_ds, 4);
    mbar_init(b_dq, 1);
    mbar_init(b_drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kWMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM: S [0, 64) (dS over [0, 32)), dP [64, 128), dQ [128, 128 + D)
  constexpr uint32_t kColS = 0, kColDP = 64, kColDQ = 128;
  const uint32_t sm_q = smem_u32(smem + L::kQ), sm_do = smem_u32(smem + L::kDO);
  const uint32_t sm_k = smem_u32(smem + L::kK), sm_v = smem_u32(smem + L::kV);

  if (warp == kWLoad) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_expect_tx(b_qdo, 2 * L::kQD);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(smem + L::kQ + c * kBox128, &tmQ, c * 64, su.q0 + qt * 128, su.g, b_qdo);
        tma_load_3d(smem + L::kDO + c * kBox128, &tmDO, c * 64, su.q0 + qt * 128, su.g, b_qdo);
      }
      int issued = 0;
      for (int t = 0; t < nt; ++t) {
        const int s = t % S;
        if (t >= S && !mbar_wait(&b_empty[s], ((t / S) - 1) & 1, abort_flag, p.err)) break;
        mbar_expect_tx(&b_kfull[s], L::kKS);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::kK + s * L::kKS + c * kBox64, &tmK, c * 64, su.k0 + t * 64, su.g, &b_kfull[s]);
        mbar_expect_tx(&b_vfull[s], L::kKS);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::kV + s * L::kKS + c * kBox64, &tmV, c * 64, su.k0 + t * 64, su.g, &b_vfull[s]);
        issued = t + 1;
      }
      if (*abort_flag) {
        mbar_wait_drain(b_qdo, 0);
        for (int t = max(0, issued - S); t < issued; ++t) {
          mbar_wait_drain(&b_kfull[t % S], (t / S) & 1);
          mbar_wait_drain(&b_vfull[t % S], (t / S) & 1);
        }
      }
    }
    __syncwarp();
    wide_bwd_teardown(tmem, false);
    return;
  }
  if (warp == kWMma) {
    {
      const bool leader = elect_one();
      const uint64_t dk_q = sdesc_sw128(sm_q, 16, 1024), dk_do = sdesc_sw128(sm_do, 16, 1024);
      const uint64_t dk_k = sdesc_sw128(sm_k, 16, 1024), dk_v = sdesc_sw128(sm_v, 16, 1024);
      const uint64_t dmn_k = sdesc_sw128(sm_k, kBox64, 1024);
      // every lane waits; the vote keeps the warp's decision uniform
#define FA_WAIT(b, parity) __all_sync(0xffffffffu, mbar_wait((b), (parity), abort_flag, p.err))
      bool ok = FA_WAIT(b_qdo, 0);
      for (int t = 0; ok && t < nt; ++t) {
        const int s = t % S;
        if (!FA_WAIT(&b_kfull[s], (t / S) & 1) || !FA_WAIT(&b_vfull[s], (t / S) & 1)) { ok = false; break; }
        tc_fence_after();
        // S = Q K^T and dP = dO V^T (the previous tile's dS was read by its dQ product, issued before)
        mma_rows128_x_rows64<D, F16>(leader, tmem + kColS, dk_q, desc_off(dk_k, s * L::kKS));
        if (leader) mma_commit(b_s);
        mma_rows128_x_rows64<D, F16>(leader, tmem + kColDP, dk_do, desc_off(dk_v, s * L::kKS));
        if (leader) mma_commit(b_dp);
        if (!FA_WAIT(b_ds, t & 1)) { ok = false; break; }
        tc_fence_after();
        // dQ += dS K : A = dS in TMEM, B = K tile (MN-major, D columns)
        mma_tmemA_x_rows64<D, F16>(leader, tmem + kColDQ, tmem + kColS, desc_off(dmn_k, s * L::kKS), t > 0);
        if (leader) mma_commit(&b_empty[s]);
      }
#undef FA_WAIT
      if (ok) {
        if (leader) mma_commit(b_dq);
      } else {
        if (leader) mma_commit(b_drain);
        mbar_wait_drain(b_drain, 0);
      }
    }
    __syncwarp();
    wide_bwd_teardown(tmem, true);
    return;
  }

  // ------------------------------------------------------------ elementwise (thread = query row)
  const uint32_t t_row = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  const float sl2 = p.scale_log2;
  const float lse2_i = p.lse2[static_cast<size_t>(unit) * Npad + i];  // +inf past the unit's rows
  const float d_i = p.Dvec[static_cast<size_t>(unit) * Npad + i];
  const PhiloxFixed123 phx = philox_fix123(static_cast<uint32_t>(i), static_cast<uint32_t>(su.h),
                                           static_cast<uint32_t>(su.b), p.philox_rk);
  const uint32_t drop_c2 = make_drop_const(p.drop_t).c2;
  const bool hi_t = p.drop_t > 0x8000u;
  const int lim0 = CAUSAL ? min(su.nk - 1, i + delta) : su.nk - 1;  // key j visible iff j <= lim0
  bool ok = true;
  for (int t = 0; t < nt; ++t) {
    uint32_t W[2] = {0u, 0u};
    if (DROPOUT) {
      if (hi_t)
        draw_keep_words<true, 8>(static_cast<uint32_t>(t * 8), phx, p.philox_rk, drop_c2, W);
      else
        draw_keep_words<false, 8>(static_cast<uint32_t>(t * 8), phx, p.philox_rk, drop_c2, W);
    }
    if (!mbar_wait(b_s, t & 1, abort_flag, p.err) || !mbar_wait(b_dp, t & 1, abort_flag, p.err)) {
      ok = false;
      break;
    }
    tc_fence_after();
    uint32_t sr[64], dr[64];
    tmem_ld32(t_row + kColS, sr);
    tmem_ld32(t_row + kColS + 32, sr + 32);
    tmem_ld32(t_row + kColDP, dr);
    tmem_ld32(t_row + kColDP + 32, dr + 32);
    tmem_ld_wait();
    reg_fence32(sr);
    reg_fence32(sr + 32);
    reg_fence32(dr);
    reg_fence32(dr + 32);
    const int lim = lim0 - t * 64;  // key columns c > lim are masked
    uint32_t dsk[32];
#pragma unroll
    for (int c2 = 0; c2 < 32; ++c2) {
      float v[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = 2 * c2 + e;
        const float pv = (c > lim) ? 0.f : ex2_approx(fmaf(__uint_as_float(sr[c]), sl2, -lse2_i));
        const float dp = __uint_as_float(dr[c]);
        v[e] = pv * (dp * p.drop_scale - d_i);      // kept: P (dP / (1-p) - D)
        if (DROPOUT) {
          const uint32_t keep = keep_mask_pair(W, c2) & (e ? 0xFFFF0000u : 0x0000FFFFu);
          if (keep == 0u) v[e] = -pv * d_i;          // dropped: P (0 - D)
        }
      }
      dsk[c2] = pack2<F16>(v[0], v[1]);
    }
    // dS in the element type over S (S is consumed; this tile's dQ product reads it)
    tmem_st32(t_row + kColS, dsk);
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(b_ds);
  }
  if (ok && mbar_wait(b_dq, 0, abort_flag, p.err)) {
    tc_fence_after();
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t v[32];
      tmem_ld32(t_row + kColDQ + 32 * c, v);
      tmem_ld_wait();
      reg_fence32(v);
      uint32_t o[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        o[e] = pack2<F16>(__uint_as_float(v[2 * e]) * p.scale, __uint_as_float(v[2 * e + 1]) * p.scale);
      if (row_ok) {
        uint4* d4 = reinterpret_cast<uint4*>(dq_row + 32 * c);
#pragma unroll
        for (int e = 0; e < 4; ++e) d4[e] = make_uint4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
      }
    }
  }
  wide_bwd_teardown(tmem, false);
}

// ============================================================ launches

WideBwdParams wide_params(const BwdArgs& a, int n_tiles_per_unit, int units_per_group_target) {
  WideBwdParams p;
  p.dQ = static_cast<uint16_t*>(a.dQ);
  p.dK = static_cast<uint16_t*>(a.dK);
  p.dV = static_cast<uint16_t*>(a.dV);
  p.lse2 = a.lse2;
  p.Dvec = a.Dvec;
  p.err = a.err;
  p.seq = a.seq;
  p.scale = a.scale;
  p.scale_log2 = a.scale_log2;
  p.drop_t = a.drop_t;
  p.drop_scale = a.drop_scale;
  for (int r = 0; r < 20; ++r) p.philox_rk[r] = a.philox_rk[r];
  p.BH = a.seq.units;
  p.group = (units_per_group_target + n_tiles_per_unit / 2) / n_tiles_per_unit;
  if (p.group < 1) p.group = 1;
  if (p.group > p.BH) p.group = p.BH;
  return p;
}

template <int D, bool CAUSAL, bool DROPOUT, bool F16>
cudaError_t launch_wide_bwd_t(const BwdArgs& a, const CUtensorMap* maps_kv, const CUtensorMap* maps_q,
                              cudaStream_t stream) {
  {
    auto kern = fa_bwd_wide_kv_kernel<D, CAUSAL, DROPOUT, F16>;
    const int smem = KvSmem<D>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int n_kt = (a.seq.Nk + 127) / 128;
    WideBwdParams p = wide_params(a, n_kt * KvSmem<D>::kSplit, 256);
    dim3 grid(static_cast<unsigned>(p.BH) * n_kt * KvSmem<D>::kSplit);
    kern<<<grid, kWThreads, smem, stream>>>(maps_kv[0], maps_kv[1], maps_kv[2], maps_kv[3], p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    auto kern = fa_bwd_wide_q_kernel<D, CAUSAL, DROPOUT, F16>;
    const int smem = QSmem<D>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int n_qt = (a.seq.Nq + 127) / 128;
    WideBwdParams p = wide_params(a, n_qt, 256);
    dim3 grid(static_cast<unsigned>(p.BH) * n_qt);
    kern<<<grid, kWThreads, smem, stream>>>(maps_q[0], maps_q[1], maps_q[2], maps_q[3], p);
    return cudaGetLastError();
  }
}

template <int D, bool F16>
cudaError_t launch_wide_bwd_d(const BwdArgs& a, const CUtensorMap* mkv, const CUtensorMap* mq, cudaStream_t st) {
  const bool drop = a.drop_t != 0;
  if (a.causal)
    return drop ? launch_wide_bwd_t<D, true, true, F16>(a, mkv, mq, st)
                : launch_wide_bwd_t<D, true, false, F16>(a, mkv, mq, st);
  return drop ? launch_wide_bwd_t<D, false, true, F16>(a, mkv, mq, st)
              : launch_wide_bwd_t<D, false, false, F16>(a, mkv, mq, st);
}

}  // namespace

// maps_kv: Q, K, V, dO with 64-, 128-, 128-, 64-row boxes (kernel 1);
// maps_q: Q, K, V, dO with 128-, 64-, 64-, 128-row boxes (kernel 2).
int wide_kv_query_rows(int d) { return d > 192 ? KvSmem<256>::kQT : KvSmem<192>::kQT; }

cudaError_t launch_bwd_wide(const BwdArgs& a, const CUtensorMap* maps_kv, const CUtensorMap* maps_q,
                            cudaStream_t stream) {
  if (a.d == 192)
    return a.f16 ? launch_wide_bwd_d<192, true>(a, maps_kv, maps_q, stream)
                 : launch_wide_bwd_d<192, false>(a, maps_kv, maps_q, stream);
  if (a.d == 256)
    return a.f16 ? launch_wide_bwd_d<256, true>(a, maps_kv, maps_q, stream)
                 : launch_wide_bwd_d<256, false>(a, maps_kv, maps_q, stream);
  return cudaErrorInvalidValue;
}

}  // namespace fa
