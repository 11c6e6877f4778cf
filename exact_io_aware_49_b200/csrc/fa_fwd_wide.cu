// fa_fwd_wide.cu -- fused attention forward for head dimensions 192 and 256
// (sm_100a).
//
// Same computation as fa_fwd.cu (scores, causal mask, online softmax with a
// running maximum and denominator, Philox dropout, O += P V, O and LSE;
// "FlashAttention" glossary, Tiling; "DL0056 FlashAttention", Mathematical
// Formulation; "Flash Attention" glossary, steps 1-5), for the head sizes the
// pages say often fall back to other kernels ("Flash Attention" glossary,
// Practical Limits and Common Pitfalls).  The d <= 128 kernel keeps two
// 128-row query tiles per CTA; at d = 192 / 256 their output accumulators no
// longer fit the 512 tensor-memory columns, so this kernel
//  * owns one 128-row query tile per CTA and streams 64-key K/V tiles
//    (3 stages at d = 192, 2 at d = 256; K and V stages are released
//    separately: K after S = Q K^T, V after O += P V);
//  * double-buffers S in tensor memory (2 x 64 columns, then O in d
//    columns): S_{t+2} = Q K_{t+2}^T is issued right after O += P_t V_t, so the
//    tensor core computes the next scores while the softmax warps work;
//  * runs one softmax warpgroup (thread = query row) with the lazy rescale
//    of fa_fwd.cu; since S_{t+1} was issued before O += P_{t-1} V_{t-1}, a
//    rescale of O first waits for that product (a barrier committed after
//    every P V product);
//  * with dropout, a fourth group of warps draws the keep bits (one thread
//    per query row, 8 Philox calls per 64-key tile in lockstep) up to two
//    tiles ahead into a two-buffer shared-memory ring that the softmax warps
//    read; with one softmax warp per sub-partition the draw then overlaps
//    the softmax instead of preceding it.
// Warps: 0-3 softmax, 4 MMA issue, 5 TMA loads, 6-9 keep words (dropout only).
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

constexpr int kWBM = 128;        // query rows per CTA
constexpr int kWBN = 64;         // keys per tile
constexpr int kWThreads = 192;   // 4 softmax warps, MMA warp, TMA warp
constexpr int kWThreadsDrop = 320;  // + 4 keep-word warps (dropout)
constexpr int kWMmaWarp = 4;
constexpr int kWLoadWarp = 5;
constexpr int kWKeepWarp0 = 6;
constexpr float kWRescaleTau = 8.0f;  // lazy-rescale threshold, log2 units

template <int D>
struct WideSmem {
  static constexpr int kStages = (D == 192) ? 3 : 2;
  static constexpr int kQBox = 128 * 128;  // 128 rows x 64 columns of 16-bit (128-byte rows)
  static constexpr int kKVBox = 64 * 128;  // 64 rows x 64 columns
  static constexpr int kKVTile = (D / 64) * kKVBox;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + (D / 64) * kQBox;
  static constexpr int kV = kK + kStages * kKVTile;
  // dropout keep words drawn by the keep-word warps: [buffer][word 0..1][row]
  static constexpr int kKeep = kV + kStages * kKVTile;
  static constexpr int kBar = kKeep + 2 * 2 * 128 * 4;
  // barriers: q, kfull[S], kempty[S], vfull[S], vempty[S], s_full[2], p_ready[2], pv_done, o_ready, drain,
  // keep_full[2], keep_empty[2]
  static constexpr int kNumBars = 1 + 4 * kStages + 7 + 4;
  // tmem slot, abort flag, the unit's first query row and head coordinate
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16 + 1024;  // + slack for 1024-byte alignment
};
static_assert(WideSmem<192>::kBytes <= kMaxSmemPerCta && WideSmem<256>::kBytes <= kMaxSmemPerCta,
              "wide forward shared memory");

struct WideBars {
  uint64_t *q, *kfull, *kempty, *vfull, *vempty, *s_full, *p_ready, *pv_done, *o_ready, *drain, *keep_full,
      *keep_empty;
};

template <int D>
__device__ __forceinline__ WideBars wide_bars(uint8_t* smem) {
  using L = WideSmem<D>;
  constexpr int S = L::kStages;
  uint64_t* b = reinterpret_cast<uint64_t*>(smem + L::kBar);
  WideBars r;
  r.q = b;
  r.kfull = b + 1;
  r.kempty = b + 1 + S;
  r.vfull = b + 1 + 2 * S;
  r.vempty = b + 1 + 3 * S;
  r.s_full = b + 1 + 4 * S;
  r.p_ready = r.s_full + 2;
  r.pv_done = r.s_full + 4;
  r.o_ready = r.s_full + 5;
  r.drain = r.s_full + 6;
  r.keep_full = r.s_full + 7;
  r.keep_empty = r.s_full + 9;
  return r;
}

struct WideParams {
  uint16_t* O;  // bf16 or fp16 bits
  float* LSE;
  unsigned* err;
  SeqLayout seq;
  float scale_log2;
  uint32_t drop_t;
  float drop_scale;
  uint32_t philox_rk[20];
  int group, BH;
};

// S = Q K^T : M = 128 query rows, N = 64 keys, K = D (both K-major).  a0 /
// b0 are the descriptors of the Q tile and the K stage; each K-step adds its
// box / swizzle-atom offset (bytes / 16) to the start-address field.  The
// whole MMA warp calls this; ``leader`` (one elected lane) issues.
template <int D, bool F16>
__device__ __forceinline__ void wide_qk(bool leader, uint32_t tmem_s, uint64_t a0, uint64_t b0) {
  using L = WideSmem<D>;
  constexpr uint32_t idesc = idesc_f32acc(128, kWBN, false, false, F16);
  if (leader) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
      mma_ss(tmem_s, a0 + static_cast<uint32_t>(((kk / 4) * L::kQBox + (kk % 4) * 32) >> 4),
             b0 + static_cast<uint32_t>(((kk / 4) * L::kKVBox + (kk % 4) * 32) >> 4), idesc, kk > 0);
  }
}

// O (+)= P V : M = 128, N = D, K = 64 keys; P (16-bit pairs) in TMEM over S,
// V MN-major in shared memory (64-column boxes 8 KB apart), b0 the descriptor
// of its stage.
template <int D, bool F16>
__device__ __forceinline__ void wide_pv(bool leader, uint32_t tmem_o, uint32_t tmem_p, uint64_t b0,
                                        bool accumulate) {
  constexpr uint32_t idesc = idesc_f32acc(128, D, false, true, F16);
  if (leader) {
#pragma unroll
    for (int kk = 0; kk < kWBN / 16; ++kk)
      mma_ts(tmem_o, tmem_p + kk * 8, b0 + static_cast<uint32_t>((kk * 2048) >> 4), idesc,
             (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <bool DROPOUT>
__device__ __forceinline__ void wide_teardown(uint32_t tmem, bool dealloc) {
  tc_fence_before();
  asm volatile("bar.sync 1, %0;" ::"n"(DROPOUT ? kWThreadsDrop : kWThreads) : "memory");
  tc_fence_after();
  if (dealloc) tmem_dealloc(tmem, 512);
}

template <int D, bool CAUSAL, bool DROPOUT, bool F16>
__global__ void __launch_bounds__(DROPOUT ? kWThreadsDrop : kWThreads, 1)
    fa_fwd_wide_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ WideParams p) {
  using L = WideSmem<D>;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (!smem_layout_fits(smem_raw, smem, L::kMisc + 16, p.err)) return;
  const WideBars bar = wide_bars<D>(smem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // 1-D grid over (unit group, query tile, unit), heaviest causal tiles first
  // within a group of p.group units
  const int n_qt_grid = (p.seq.Nq + kWBM - 1) / kWBM;
  const int per_group = p.group * n_qt_grid;
  const int grp = blockIdx.x / per_group;
  const int rr = blockIdx.x - grp * per_group;
  const int gsz = min(p.group, p.BH - grp * p.group);
  const int qt_lin = rr / gsz;
  const int unit = grp * p.group + (rr - qt_lin * gsz);
  const SeqUnit su = resolve_unit(p.seq, unit);
  const int N = su.nq;
  const int qt = CAUSAL ? (n_qt_grid - 1 - qt_lin) : qt_lin;
  if (qt * kWBM >= N) return;  // past this unit's queries (shorter packed sequence)
  const int n_kt = (su.nk + kWBN - 1) / kWBN;
  const int delta = su.nk - su.nq;  // query i sits at key position i + delta
  const int last_row = min(N - 1, qt * kWBM + kWBM - 1);
  // key tiles this query tile visits (causal: up to the one holding the last
  // row's last visible key); possibly none
  const int nt = CAUSAL ? min(n_kt, max(0, floor_div(last_row + delta, kWBN) + 1)) : n_kt;

  if (threadIdx.x == 0) {
    mbar_init(bar.q, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&bar.kfull[s], 1);
      mbar_init(&bar.kempty[s], 1);
      mbar_init(&bar.vfull[s], 1);
      mbar_init(&bar.vempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar.s_full[b], 1);
      mbar_init(&bar.p_ready[b], 4);
    }
    mbar_init(bar.pv_done, 1);
    mbar_init(bar.o_ready, 1);
    mbar_init(bar.drain, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar.keep_full[b], 4);
      mbar_init(&bar.keep_empty[b], 4);
    }
    *abort_flag = 0;
    reinterpret_cast<int*>(smem + L::kMisc)[2] = su.q0;
    reinterpret_cast<int*>(smem + L::kMisc)[3] = su.g;
    mbar_fence_init();
  }
  if (warp == kWMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S buffers at 0 and 64 (P over their first 32), O at 128
  constexpr uint32_t kColO = 128;
  const uint32_t sm_q = smem_u32(smem + L::kQ);
  const uint32_t sm_k = smem_u32(smem + L::kK);
  const uint32_t sm_v = smem_u32(smem + L::kV);

  if (warp == kWLoadWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nt > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(bar.q, (D / 64) * L::kQBox);
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(smem + L::kQ + c * L::kQBox, &tmQ, c * 64, su.q0 + qt * kWBM, su.g, bar.q);
      int k_issued = 0, v_issued = 0;
      for (int t = 0; t < nt; ++t) {
        const int s = t % S;
        if (t >= S && !mbar_wait(&bar.kempty[s], ((t / S) - 1) & 1, abort_flag, p.err)) break;
        mbar_expect_tx(&bar.kfull[s], L::kKVTile);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::kK + s * L::kKVTile + c * L::kKVBox, &tmK, c * 64, su.k0 + t * kWBN, su.g,
                      &bar.kfull[s]);
        k_issued = t + 1;
        if (t >= S && !mbar_wait(&bar.vempty[s], ((t / S) - 1) & 1, abort_flag, p.err)) break;
        mbar_expect_tx(&bar.vfull[s], L::kKVTile);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::kV + s * L::kKVTile + c * L::kKVBox, &tmV, c * 64, su.k0 + t * kWBN, su.g,
                      &bar.vfull[s]);
        v_issued = t + 1;
      }
      if (*abort_flag) {
        // copies in flight land before the shared memory goes away
        mbar_wait_drain(bar.q, 0);
        for (int t = max(0, k_issued - S); t < k_issued; ++t) mbar_wait_drain(&bar.kfull[t % S], (t / S) & 1);
        for (int t = max(0, v_issued - S); t < v_issued; ++t) mbar_wait_drain(&bar.vfull[t % S], (t / S) & 1);
      }
    }
    __syncwarp();
    wide_teardown<DROPOUT>(tmem, false);
    return;
  }
  if (warp == kWMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop, so descriptors and counters are
    // warp-uniform values; one elected lane issues the MMAs and commits.
    if (nt > 0) {
      const bool leader = elect_one();
      const uint64_t dq0 = sdesc_sw128(sm_q, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sm_k, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(sm_v, L::kKVBox, 1024);
      // every lane waits; the vote keeps the warp's decision uniform
#define FA_WAIT(b, parity) __all_sync(0xffffffffu, mbar_wait((b), (parity), abort_flag, p.err))
      bool ok = FA_WAIT(bar.q, 0);
      // S_0 and S_1 ahead of the loop
      for (int t = 0; ok && t < min(2, nt); ++t) {
        if (!FA_WAIT(&bar.kfull[t % S], (t / S) & 1)) { ok = false; break; }
        tc_fence_after();
        wide_qk<D, F16>(leader, tmem + 64 * t, dq0, dk0 + static_cast<uint32_t>(((t % S) * L::kKVTile) >> 4));
        if (leader) {
          mma_commit(&bar.s_full[t]);
          mma_commit(&bar.kempty[t % S]);
        }
      }
      for (int t = 0; ok && t < nt; ++t) {
        const int b = t & 1, s = t % S;
        if (!FA_WAIT(&bar.p_ready[b], (t >> 1) & 1) || !FA_WAIT(&bar.vfull[s], (t / S) & 1)) { ok = false; break; }
        tc_fence_after();
        wide_pv<D, F16>(leader, tmem + kColO, tmem + 64 * b, dv0 + static_cast<uint32_t>((s * L::kKVTile) >> 4),
                        t > 0);
        if (leader) {
          mma_commit(bar.pv_done);
          mma_commit(&bar.vempty[s]);
        }
        if (t + 2 < nt) {
          // S_{t+2} into the buffer P_t occupies: issued after the P V product reading it
          const int s2 = (t + 2) % S;
          if (!FA_WAIT(&bar.kfull[s2], ((t + 2) / S) & 1)) { ok = false; break; }
          tc_fence_after();
          wide_qk<D, F16>(leader, tmem + 64 * b, dq0, dk0 + static_cast<uint32_t>((s2 * L::kKVTile) >> 4));
          if (leader) {
            mma_commit(&bar.s_full[b]);
            mma_commit(&bar.kempty[s2]);
          }
        }
      }
#undef FA_WAIT
      if (ok) {
        if (leader) mma_commit(bar.o_ready);
      } else {
        if (leader) mma_commit(bar.drain);  // MMAs already issued finish before TMEM is freed
        mbar_wait_drain(bar.drain, 0);
      }
    }
    __syncwarp();
    wide_teardown<DROPOUT>(tmem, true);
    return;
  }

  if (DROPOUT && warp >= kWKeepWarp0) {
    // ---------------------------------------------------------- keep words
    // One thread per query row draws its 8 Philox calls per 64-key tile (in
    // lockstep) up to two tiles ahead of the softmax, into a two-buffer ring.
    const int kr = (warp - kWKeepWarp0) * 32 + lane;
    const PhiloxFixed123 kphx = philox_fix123(static_cast<uint32_t>(qt * kWBM + kr), static_cast<uint32_t>(su.h),
                                              static_cast<uint32_t>(su.b), p.philox_rk);
    const uint32_t kc2 = make_drop_const(p.drop_t).c2;
    const bool khi = p.drop_t > 0x8000u;
    uint32_t* ring = reinterpret_cast<uint32_t*>(smem + L::kKeep);
    for (int t = 0; t < nt; ++t) {
      const int b = t & 1;
      // the softmax warps have read the buffer's previous tile (t - 2)
      if (t >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bar.keep_empty[b], ((t - 2) >> 1) & 1, abort_flag, p.err)))
        break;
      uint32_t W[2];
      if (khi)
        draw_keep_words<true, kWBN / 8>(static_cast<uint32_t>(t * (kWBN / 8)), kphx, p.philox_rk, kc2, W);
      else
        draw_keep_words<false, kWBN / 8>(static_cast<uint32_t>(t * (kWBN / 8)), kphx, p.philox_rk, kc2, W);
      ring[(b * 2 + 0) * 128 + kr] = W[0];
      ring[(b * 2 + 1) * 128 + kr] = W[1];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.keep_full[b]);
    }
    wide_teardown<DROPOUT>(tmem, false);
    return;
  }

  // ------------------------------------------------------------ softmax warpgroup
  const int r = warp * 32 + lane;  // row within the query tile == TMEM lane
  const int i = qt * kWBM + r;
  const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  const uint32_t t_o = t_lane + kColO;
  const float sl2 = p.scale_log2;
  // masking: key j = t * kWBN + c is visible iff j <= lim0; tiles from t_mask
  // on can hold a masked key for some row of the tile
  const int lim0 = CAUSAL ? min(su.nk - 1, i + delta) : su.nk - 1;
  int t_mask = su.nk / kWBN;
  if (CAUSAL) t_mask = min(t_mask, max(0, floor_div(qt * kWBM + delta - (kWBN - 1), kWBN) + 1));
  float m = -CUDART_INF_F;  // running max of scale*log2(e)*S, possibly stale
  float l = 0.f;            // running sum of exp2(x - m)
  float lc = 0.f;           // sum of (p - p rounded) over each tile's largest P (see fa_fwd.cu)
  bool ok = true;
  for (int t = 0; t < nt; ++t) {
    const int b = t & 1;
    uint32_t W[2] = {0u, 0u};
    if (DROPOUT) {
      // this row's keep words from the keep-word warps' ring
      if (!mbar_wait(&bar.keep_full[b], (t >> 1) & 1, abort_flag, p.err)) { ok = false; break; }
      const uint32_t* ring = reinterpret_cast<const uint32_t*>(smem + L::kKeep);
      W[0] = ring[(b * 2 + 0) * 128 + r];
      W[1] = ring[(b * 2 + 1) * 128 + r];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.keep_empty[b]);
    }
    if (!mbar_wait(&bar.s_full[b], (t >> 1) & 1, abort_flag, p.err)) { ok = false; break; }
    tc_fence_after();
    uint32_t sr[kWBN];
    tmem_ld32(t_lane + 64 * b, sr);
    tmem_ld32(t_lane + 64 * b + 32, sr + 32);
    tmem_ld_wait();
    reg_fence32(sr);
    reg_fence32(sr + 32);
    float s[kWBN];
#pragma unroll
    for (int c = 0; c < kWBN; ++c) s[c] = __uint_as_float(sr[c]);
    if (t >= t_mask) {  // the same for the whole warp
      const int lim = lim0 - t * kWBN;
#pragma unroll
      for (int c = 0; c < kWBN; ++c)
        if (c > lim) s[c] = -CUDART_INF_F;
    }
    float mx0 = fmaxf(s[0], s[1]), mx1 = fmaxf(s[2], s[3]);
#pragma unroll
    for (int c = 4; c < kWBN; c += 4) {
      mx0 = max3f(mx0, s[c], s[c + 1]);
      mx1 = max3f(mx1, s[c + 2], s[c + 3]);
    }
    const float s_max = fmaxf(mx0, mx1);
    const float m_new = fmaxf(m, s_max * sl2);
    const bool rescale = __any_sync(0xffffffffu, m_new > m + kWRescaleTau);
    float alpha = 1.f;
    if (rescale) {
      alpha = ex2_approx(m - m_new);  // 0 on the first tile (m = -inf)
      l *= alpha;
      lc *= alpha;
      m = m_new;
    }
    const float m_use = (m == -CUDART_INF_F) ? 0.f : m;
    {
      const float p_top = ex2_approx(fmaf(s_max, sl2, -m_use));
      lc += p_top - unpack2<F16>(pack2<F16>(p_top, 0.f)).x;
    }
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    const uint64_t negm2 = f2_pack(-m_use, -m_use);
    uint32_t pk[kWBN / 2];
    uint64_t rs0 = 0ull, rs1 = 0ull;
#pragma unroll
    for (int c = 0; c < kWBN / 2; ++c) {
      float x0, x1;
      f2_unpack(fma_f2(f2_pack(s[2 * c], s[2 * c + 1]), sl2x2, negm2), x0, x1);
      const float p0 = ex2_approx(x0);
      const float p1 = ex2_approx(x1);
      const uint64_t pp = f2_pack(p0, p1);
      if (c & 1)
        rs1 = add_f2(rs1, pp);
      else
        rs0 = add_f2(rs0, pp);
      pk[c] = pack2<F16>(p0, p1);
      if (DROPOUT) pk[c] &= keep_mask_pair(W, c);
    }
    {
      float a0, a1;
      f2_unpack(add_f2(rs0, rs1), a0, a1);
      l += a0 + a1;
    }
    if (rescale && t > 0) {
      // S_t was issued before O += P_{t-1} V_{t-1}: wait for that product
      // (at most the phase before the one awaited can be complete, so the
      // parity wait cannot alias)
      if (!mbar_wait(bar.pv_done, (t - 1) & 1, abort_flag, p.err)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t orow[32];
        tmem_ld32(t_o + c * 32, orow);
        tmem_ld_wait();
        reg_fence32(orow);
#pragma unroll
        for (int e = 0; e < 32; ++e) orow[e] = __float_as_uint(__uint_as_float(orow[e]) * alpha);
        tmem_st32(t_o + c * 32, orow);
      }
    }
    tmem_st32(t_lane + 64 * b, pk);
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar.p_ready[b]);
  }
  const bool row_ok = i < N;
  const int q0 = reinterpret_cast<const int*>(smem + L::kMisc)[2];
  const int gq = reinterpret_cast<const int*>(smem + L::kMisc)[3];
  uint16_t* orow_g = p.O + static_cast<size_t>(q0 + i) * p.seq.tok_stride + static_cast<size_t>(gq) * p.seq.q_head_stride;
  float* lse_g = p.LSE + static_cast<size_t>(gq) * p.seq.total_q + q0 + i;
  if (nt == 0) {
    // the tile sees no key: O = 0, LSE = -inf
    if (row_ok) {
      uint4* dst = reinterpret_cast<uint4*>(orow_g);
#pragma unroll
      for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0u, 0u, 0u, 0u);
      *lse_g = -CUDART_INF_F;
    }
  } else if (ok && mbar_wait(bar.o_ready, 0, abort_flag, p.err)) {
    tc_fence_after();
    const float inv = (l > 0.f) ? p.drop_scale / (l - lc) : 0.f;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(t_o + c * 32, o);
      tmem_ld_wait();
      reg_fence32(o);
      uint32_t packed[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        packed[e] = pack2<F16>(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
      if (row_ok) {
        uint4* dst = reinterpret_cast<uint4*>(orow_g + c * 32);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
      }
    }
    if (row_ok) *lse_g = (l > 0.f) ? (m + lg2_approx(l)) * 0.69314718055994531f : -CUDART_INF_F;
  }
  wide_teardown<DROPOUT>(tmem, false);
}

template <int D, bool CAUSAL, bool DROPOUT, bool F16>
cudaError_t launch_wide_t(const FwdArgs& a, cudaStream_t stream) {
  auto kern = fa_fwd_wide_kernel<D, CAUSAL, DROPOUT, F16>;
  const int smem = WideSmem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  WideParams p;
  p.O = static_cast<uint16_t*>(a.O);
  p.LSE = a.LSE;
  p.err = a.err;
  p.seq = a.seq;
  p.scale_log2 = a.scale_log2;
  p.drop_t = a.drop_t;
  p.drop_scale = a.drop_scale;
  for (int r = 0; r < 20; ++r) p.philox_rk[r] = a.philox_rk[r];
  p.BH = a.seq.units;
  const int n_qt = (a.seq.Nq + kWBM - 1) / kWBM;
  // about 256 CTAs per group of units (the heaviest causal tiles of a group first)
  p.group = (256 + n_qt / 2) / n_qt;
  if (p.group < 1) p.group = 1;
  if (p.group > p.BH) p.group = p.BH;
  dim3 grid(static_cast<unsigned>(p.BH) * n_qt);
  kern<<<grid, DROPOUT ? kWThreadsDrop : kWThreads, smem, stream>>>(a.tmQ, a.tmK, a.tmV, p);
  return cudaGetLastError();
}

template <int D, bool F16>
cudaError_t launch_wide_d(const FwdArgs& a, cudaStream_t stream) {
  const bool drop = a.drop_t != 0;
  if (a.causal)
    return drop ? launch_wide_t<D, true, true, F16>(a, stream) : launch_wide_t<D, true, false, F16>(a, stream);
  return drop ? launch_wide_t<D, false, true, F16>(a, stream) : launch_wide_t<D, false, false, F16>(a, stream);
}

}  // namespace

cudaError_t launch_fwd_wide(const FwdArgs& a, cudaStream_t stream) {
  if (a.d == 192) return a.f16 ? launch_wide_d<192, true>(a, stream) : launch_wide_d<192, false>(a, stream);
  if (a.d == 256) return a.f16 ? launch_wide_d<256, true>(a, stream) : launch_wide_d<256, false>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace fa
