// fa_fwd.cu -- fused attention forward for sm_100a.
//
// What it computes: O = dropout(softmax(scale * Q K^T + causal mask)) V and
// LSE_i = ln sum_j exp(scale * Q_i . K_j), tile by tile, never writing the
// N x N scores or probabilities to device memory ("FlashAttention" glossary,
// Tiling; "Flash Attention" glossary, How Flash Attention Works, steps 1-5).
// The row statistics follow the online-softmax recurrence of "DL0056
// FlashAttention", Mathematical Formulation: a running maximum m_i and
// denominator l_i, with exp(m_old - m_new) rescaling the earlier partial sums
// of l and of the output accumulator.
//
// Design (B200):
//  * one CTA owns two 128-row query tiles (Q0, Q1) of one (b, h) and streams
//    128-key K/V tiles through a multi-stage TMA + mbarrier ring;
//  * S_q = Q_q K_t^T and O_q += P_q V_t run on the 5th-generation tensor cores
//    (tcgen05.mma, bf16 or fp16 in, fp32 accumulators in tensor memory).
//    TMEM holds S0 | S1 | O0 | O1 (512 columns); P_q (in the input type) is
//    written back over S_q and read by the PV MMA directly from TMEM;
//  * warp roles: warps 0-3 and 4-7 are the softmax warpgroups of Q0 and Q1
//    (one thread per query row: causal mask on the diagonal tile, running
//    max / sum, exp2, Philox dropout, P to TMEM, and the epilogue); warp 8
//    issues the MMAs (the whole warp runs the loop, so descriptors are
//    warp-uniform values, and one elected lane issues); warp 9 issues the
//    TMA loads.  While one warpgroup turns S into P, the tensor core works
//    on the other query tile;
//  * the O rescale is lazy: the stale maximum is kept until a row's maximum
//    grows by more than 8 (log2 units).  l and O share the stale maximum, so
//    the result is unchanged; P stays <= 2^8;
//  * dropout never stores a mask: keep decisions come from Philox keyed on
//    (seed, b, h, i, j), 16 calls per row and 128-key tile, 4 in lockstep.
//    The first 8 (d = 128) or 4 (d = 64) run while the tensor core computes
//    S and become byte-sign masks (an integer test, an AND per pair of P);
//    the others run inside the exponential loop, one chunk of 32 keys ahead,
//    and are tested on the FMA pipe: one byte permute makes the exact float
//    2^23 + u of a 16-bit draw u, one saturating add turns it into the
//    0.0 / 1.0 keep multiplier.  Kept P are left unscaled and 1/(1-p) is
//    folded into the final normalisation.
//  * a causal CTA processes only key tiles up to its diagonal; the grid puts
//    the heaviest query blocks first;
//  * queries and keys may differ in number (Nq != Nk, causal alignment
//    bottom-right: query i sits at key position i + Nk - Nq) and, with
//    packed sequence offsets, per sequence.  A row that sees no key gets
//    O = 0 and LSE = -inf.
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

constexpr int kBM = 128;             // query rows per tile
constexpr int kBN = 128;             // keys per tile
constexpr int kFwdThreads = 384;     // 2 softmax warpgroups + 1 control warpgroup
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
// Register split (setmaxnreg): the kernel launches with kFwdLaunchRegs per
// thread; softmax warpgroups grow to kSoftmaxRegs, the control warpgroup
// (MMA, TMA, two idle warps) shrinks to kControlRegs.  The split must fit the
// launch pool: 2*128*216 + 128*56 = 62464 <= 384*168 = 64512.
constexpr int kFwdLaunchRegs = 168;
constexpr int kSoftmaxRegs = 216;
constexpr int kControlRegs = 56;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kFwdThreads * kFwdLaunchRegs, "register split");
constexpr float kRescaleTau = 8.0f;  // lazy-rescale threshold, log2 units

template <int D>
struct FwdSmem {
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kTileBytes = kBN * D * 2;  // one 128 x D tile of 16-bit elements
  static constexpr int kBoxBytes = 128 * 128;     // one 128-row x 64-col box (128B rows)
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + 2 * kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kBar = kV + kStages * kTileBytes;
  // barriers: q, kfull[S], vfull[S], kvempty[S], s_ready[2], p_ready[2], o_ready[2], drain
  static constexpr int kNumBars = 1 + 3 * kStages + 7;
  // tmem slot (4 B), abort flag (4 B), the unit's first query row and head coordinate (4 B each)
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16 + 1024;   // + slack for 1024-byte alignment
};

struct FwdBars {
  uint64_t* q;
  uint64_t* kfull;
  uint64_t* vfull;
  uint64_t* kvempty;
  uint64_t* s_ready;
  uint64_t* p_ready;
  uint64_t* o_ready;
  uint64_t* drain;
};

template <int D>
__device__ __forceinline__ FwdBars fwd_bars(uint8_t* smem) {
  using L = FwdSmem<D>;
  uint64_t* b = reinterpret_cast<uint64_t*>(smem + L::kBar);
  FwdBars r;
  r.q = b;
  r.kfull = b + 1;
  r.vfull = b + 1 + L::kStages;
  r.kvempty = b + 1 + 2 * L::kStages;
  r.s_ready = b + 1 + 3 * L::kStages;
  r.p_ready = r.s_ready + 2;
  r.o_ready = r.s_ready + 4;
  r.drain = r.s_ready + 6;
  return r;
}

struct FwdParams {
  uint16_t* O;  // bf16 or fp16 bits
  float* LSE;
  unsigned* err;
  SeqLayout seq;
  int dh;  // head dimension of the tensors (D, or 32 / 96 padded to D = 64 / 128)
  float scale_log2;
  uint32_t drop_t;
  float drop_scale;
  uint32_t philox_rk[20];  // Philox round keys (read from the constant bank)
  int group, BH;
};

// S_q = Q_q K^T : M = 128 query rows, N = 128 keys, K = D (both K-major).
// a0 / b0 are the descriptors of the Q tile and the K stage; each K-step
// adds its box / swizzle-atom offset (bytes / 16) to the start address.
template <int D, bool F16>
__device__ __forceinline__ void issue_qk(bool leader, uint32_t tmem_s, uint64_t a0, uint64_t b0) {
  constexpr uint32_t idesc = idesc_f32acc(128, 128, false, false, F16);
  if (leader) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = static_cast<uint32_t>(((kk / 4) * FwdSmem<D>::kBoxBytes + (kk % 4) * 32) >> 4);
      mma_ss(tmem_s, a0 + off, b0 + off, idesc, kk > 0);
    }
  }
}

// O_q (+)= P_q V : M = 128, N = D, K = 128 keys.  P (16-bit, packed in pairs)
// lives in TMEM over S_q; V is MN-major in shared memory (D contiguous,
// 64-column boxes kBoxBytes apart), b0 the descriptor of its stage.
template <int D, bool F16>
__device__ __forceinline__ void issue_pv(bool leader, uint32_t tmem_o, uint32_t tmem_p, uint64_t b0, bool accumulate) {
  constexpr uint32_t idesc = idesc_f32acc(128, D, false, true, F16);
  if (leader) {
#pragma unroll
    for (int kk = 0; kk < kBN / 16; ++kk)
      mma_ts(tmem_o, tmem_p + kk * 8, b0 + static_cast<uint32_t>((kk * 2048) >> 4), idesc,
             (accumulate || kk > 0) ? 1u : 0u);
  }
}

// All 384 threads meet here once their role is done; the MMA warp then frees TMEM.
__device__ __forceinline__ void cta_teardown(uint32_t tmem, bool dealloc) {
  tc_fence_before();
  asm volatile("bar.sync 1, %0;" ::"n"(kFwdThreads) : "memory");
  tc_fence_after();
  if (dealloc) tmem_dealloc(tmem, 512);
}

template <int D, bool CAUSAL, bool DROPOUT, bool F16>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ FwdParams p) {
  using L = FwdSmem<D>;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (!smem_layout_fits(smem_raw, smem, L::kMisc + 16, p.err)) return;
  const FwdBars bar = fwd_bars<D>(smem);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // 1-D grid over (head group, query block, unit): within a group of
  // p.group units the heaviest causal blocks come first, and the blocks that
  // run together share their units' K and V through L2.
  const int n_qb_grid = ((p.seq.Nq + kBM - 1) / kBM + 1) / 2;
  const int per_group = p.group * n_qb_grid;
  const int grp = blockIdx.x / per_group;
  const int rr = blockIdx.x - grp * per_group;
  const int gsz = min(p.group, p.BH - grp * p.group);
  const int qb_lin = rr / gsz;
  const int unit = grp * p.group + (rr - qb_lin * gsz);  // b * H + h
  const SeqUnit su = resolve_unit(p.seq, unit);
  const int N = su.nq;                   // queries of this unit
  const int n_qt = (N + kBM - 1) / kBM;  // the last tile may be partial
  const int qb = CAUSAL ? (n_qb_grid - 1 - qb_lin) : qb_lin;
  const int qt0 = 2 * qb;
  // a block past this unit's queries (shorter packed sequence) has no work
  if (qt0 >= n_qt) return;
  const int nq = min(2, n_qt - qt0);
  // key tiles each query tile visits: all of them, or (causal) up to the one
  // holding the last valid row's last visible key i + Nk - Nq; possibly none
  const int n_kt = (su.nk + kBN - 1) / kBN;
  const int delta = su.nk - su.nq;
  // (two scalars rather than an indexed array, which would live in local memory)
  auto key_tiles = [&](int q) {
    const int last_row = min(N - 1, (qt0 + q) * kBM + kBM - 1);
    return CAUSAL ? min(n_kt, max(0, floor_div(last_row + delta, kBN) + 1)) : n_kt;
  };
  const int nt0 = key_tiles(0);
  const int nt1 = (nq == 2) ? key_tiles(1) : 0;
  const int nt_all = (nq == 2) ? nt1 : nt0;

  if (threadIdx.x == 0) {
    mbar_init(bar.q, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&bar.kfull[s], 1);
      mbar_init(&bar.vfull[s], 1);
      mbar_init(&bar.kvempty[s], 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&bar.s_ready[q], 1);
      mbar_init(&bar.p_ready[q], 4);
      mbar_init(&bar.o_ready[q], 1);
    }
    mbar_init(bar.drain, 1);
    *abort_flag = 0;
    // the epilogue reads these back instead of keeping them in registers
    // through the softmax loop
    reinterpret_cast<int*>(smem + L::kMisc)[2] = su.q0;
    reinterpret_cast<int*>(smem + L::kMisc)[3] = su.g;
    mbar_fence_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sm_q = smem_u32(smem + L::kQ);
  const uint32_t sm_k = smem_u32(smem + L::kK);
  const uint32_t sm_v = smem_u32(smem + L::kV);

  if (warp >= 8) {
    // control warpgroup: MMA issuer, TMA producer, two idle warps
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs));
    if (warp == kLoadWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nt_all > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      // 3-D coordinates (column, token row, head coordinate): rows past the
      // tensor read as zeros, rows of the next packed sequence are masked
      mbar_expect_tx(bar.q, nq * L::kTileBytes);
      for (int q = 0; q < nq; ++q)
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::kQ + q * L::kTileBytes + c * L::kBoxBytes, &tmQ, c * 64,
                      su.q0 + (qt0 + q) * kBM, su.g, bar.q);
      int issued = 0;
      for (int t = 0; t < nt_all; ++t) {
        const int s = t % S;
        if (t >= S && !mbar_wait(&bar.kvempty[s], ((t / S) - 1) & 1, abort_flag, p.err)) break;
        mbar_expect_tx(&bar.kfull[s], L::kTileBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::kK + s * L::kTileBytes + c * L::kBoxBytes, &tmK, c * 64, su.k0 + t * kBN, su.g,
                      &bar.kfull[s]);
        mbar_expect_tx(&bar.vfull[s], L::kTileBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::kV + s * L::kTileBytes + c * L::kBoxBytes, &tmV, c * 64, su.k0 + t * kBN, su.g,
                      &bar.vfull[s]);
        issued = t + 1;
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA's shared memory goes away
        mbar_wait_drain(bar.q, 0);
        for (int t = max(0, issued - S); t < issued; ++t) {
          mbar_wait_drain(&bar.kfull[t % S], (t / S) & 1);
          mbar_wait_drain(&bar.vfull[t % S], (t / S) & 1);
        }
      }
    }
    } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // Per key tile t and query tile q: O_q += P_{q,t} V_t, then S_{q,t+1}
    // into the columns P_{q,t} occupied (the tensor core runs the products in
    // issue order).  The whole warp runs the loop, so descriptors and
    // counters are warp-uniform values; one elected lane issues the MMAs and
    // commits.
    if (nt_all > 0) {
      const bool leader = elect_one();
      // descriptor bases; a tile, stage, box or K-step offset (bytes / 16) is
      // added to the start-address field
      const uint64_t dq0 = sdesc_sw128(sm_q, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sm_k, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(sm_v, L::kBoxBytes, 1024);
      // every lane waits; the vote keeps the warp's decision uniform
#define FA_WAIT(b, parity) __all_sync(0xffffffffu, mbar_wait((b), (parity), abort_flag, p.err))
      bool ok = FA_WAIT(bar.q, 0) && FA_WAIT(&bar.kfull[0], 0);
      if (ok) {
        tc_fence_after();
        for (int q = 0; q < nq; ++q) {
          if ((q ? nt1 : nt0) == 0) continue;  // a query tile that sees no key
          issue_qk<D, F16>(leader, tmem + q * 128, dq0 + static_cast<uint32_t>((q * L::kTileBytes) >> 4), dk0);
          if (leader) mma_commit(&bar.s_ready[q]);
        }
      }
      for (int t = 0; ok && t < nt_all; ++t) {
        const int s = t % S;
        if (!FA_WAIT(&bar.vfull[s], (t / S) & 1)) { ok = false; break; }
        bool next_k_ready = false;
        const int s1 = (t + 1) % S;
        for (int q = 0; q < nq; ++q) {
          const int ntq = q ? nt1 : nt0;
          if (t >= ntq) continue;
          if (!FA_WAIT(&bar.p_ready[q], t & 1)) { ok = false; break; }
          tc_fence_after();
          issue_pv<D, F16>(leader, tmem + 256 + q * D, tmem + q * 128,
                           dv0 + static_cast<uint32_t>((s * L::kTileBytes) >> 4), t > 0);
          if (t == ntq - 1) {
            if (leader) mma_commit(&bar.o_ready[q]);
          } else {
            if (!next_k_ready) {
              if (!FA_WAIT(&bar.kfull[s1], ((t + 1) / S) & 1)) { ok = false; break; }
              tc_fence_after();
              next_k_ready = true;
            }
            issue_qk<D, F16>(leader, tmem + q * 128, dq0 + static_cast<uint32_t>((q * L::kTileBytes) >> 4),
                             dk0 + static_cast<uint32_t>((s1 * L::kTileBytes) >> 4));
            if (leader) mma_commit(&bar.s_ready[q]);
          }
        }
        if (!ok) break;
        if (leader) mma_commit(&bar.kvempty[s]);
      }
#undef FA_WAIT
      if (!ok) {
        if (leader) mma_commit(bar.drain);  // wait for MMAs already issued before TMEM is freed
        mbar_wait_drain(bar.drain, 0);
      }
    }
    __syncwarp();
    }
    cta_teardown(tmem, warp == kMmaWarp);
    return;
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    const int q = warp >> 2;
    if (q < nq) {
      const int wq = warp & 3;
      const int r = wq * 32 + lane;  // row within the query tile == TMEM lane
      const int i = (qt0 + q) * kBM + r;
      const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
      const uint32_t t_s = t_lane + q * 128;
      const uint32_t t_o = t_lane + 256 + q * D;
      const float sl2 = p.scale_log2;
      // dropout: the Philox counter of this row is (j >> 3, i, h, b); the
      // parts of its first two rounds that do not depend on j are fixed here
      const PhiloxFixed123 phx = philox_fix123(static_cast<uint32_t>(i), static_cast<uint32_t>(su.h),
                                               static_cast<uint32_t>(su.b), p.philox_rk);
      const float drop_bias = -(8388608.0f + static_cast<float>(p.drop_t) - 1.0f);
      // dropout: Philox calls drawn before S is ready (while the tensor core
      // computes S); the rest run inside the exponential loop.  At d = 128 the
      // wait for S is long enough for 8, at d = 64 for 4.
      constexpr int kPre = (D == 128) ? 8 : 4;
      const uint32_t drop_c2 = make_drop_const(p.drop_t).c2;
      const uint32_t drop_m0 = make_drop_const(p.drop_t).m0;
      // masking: key j = t * kBN + c is visible to this row iff j <= lim0 (the
      // last key, and under the causal mask the row's position i + Nk - Nq);
      // tiles from t_mask on are the first that can hold a masked key for
      // some row of the tile
      const int lim0 = CAUSAL ? min(su.nk - 1, i + delta) : su.nk - 1;
      int t_mask = su.nk / kBN;  // first tile running past the keys
      if (CAUSAL) t_mask = min(t_mask, max(0, floor_div((qt0 + q) * kBM + delta - (kBN - 1), kBN) + 1));
      float m = -CUDART_INF_F;  // running max of scale*log2(e)*S, possibly stale
      float l = 0.f;            // running sum of exp2(x - m)
      // running sum of (p - p rounded to 16 bits) over the largest P of each
      // tile: l - lc is the sum the rounded P actually carry into O (exact
      // for the elements that dominate a row), while l itself gives LSE
      float lc = 0.f;
      bool ok = true;
      const int ntq = q ? nt1 : nt0;
      for (int t = 0; t < ntq; ++t) {
        // dropout draws: the first kPre calls (8 kPre keys, 4 in lockstep)
        // before S is ready, while the tensor core computes S.  Their keep
        // test is the two-lane integer test of keep_mask_2x16 (m0 selects the
        // threshold side at run time), gathered into byte-sign words: kz[2g]
        // holds keys 8g .. 8g+3 in the signs of its bytes, kz[2g+1] keys
        // 8g+4 .. 8g+7.
        uint32_t kz[2 * kPre];
        if (DROPOUT) {
#pragma unroll
          for (int g0 = 0; g0 < kPre; g0 += 4) {
            uint32_t w[4][4];
            philox4x32_10_c0_batch<4>(static_cast<uint32_t>(t * (kBN / 8) + g0), phx, p.philox_rk, w);
#pragma unroll
            for (int n = 0; n < 4; ++n) {
              uint32_t z[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const uint32_t y = (w[n][e] & 0x7FFF7FFFu) + drop_c2;
                z[e] = (w[n][e] & y) | ((w[n][e] | y) & drop_m0);
              }
              kz[2 * (g0 + n)] = prmt(z[0], z[1], 0x7531u);
              kz[2 * (g0 + n) + 1] = prmt(z[2], z[3], 0x7531u);
            }
          }
        }
        if (!mbar_wait(&bar.s_ready[q], t & 1, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(t_s + c * 32, sr + c * 32);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 4; ++c) reg_fence32(sr + c * 32);
        float s[kBN];
#pragma unroll
        for (int c = 0; c < kBN; ++c) s[c] = __uint_as_float(sr[c]);
        // masked columns: keys after this row's position i + Nk - Nq (causal)
        // and keys past the unit's last key; both are c > lim for one limit
        if (t >= t_mask) {  // the same for the whole warp
          const int lim = lim0 - t * kBN;
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (c > lim) s[c] = -CUDART_INF_F;
        }
        // row max over the 128 columns: four independent 3-input max chains
        float mx0 = fmaxf(s[0], s[1]), mx1 = fmaxf(s[2], s[3]);
        float mx2 = fmaxf(s[4], s[5]), mx3 = fmaxf(s[6], s[7]);
#pragma unroll
        for (int c = 8; c < kBN; c += 8) {
          mx0 = max3f(mx0, s[c], s[c + 1]);
          mx1 = max3f(mx1, s[c + 2], s[c + 3]);
          mx2 = max3f(mx2, s[c + 4], s[c + 5]);
          mx3 = max3f(mx3, s[c + 6], s[c + 7]);
        }
        static_assert(kBN % 8 == 0, "row max covers the tile in steps of 8");
        const float s_max = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        const float m_tile = s_max * sl2;
        const float m_new = fmaxf(m, m_tile);
        // lazy rescale: the warp moves to the new maximum only when some row's
        // maximum grew by more than kRescaleTau (warp-uniform decision)
        const bool rescale = __any_sync(0xffffffffu, m_new > m + kRescaleTau);
        float alpha = 1.f;
        if (rescale) {
          alpha = ex2_approx(m - m_new);  // 0 on the first tile (m = -inf)
          l *= alpha;
          lc *= alpha;
          m = m_new;
        }
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        // a row that has seen no key yet keeps m = -inf: its P is exp2(-inf) = 0
        const float m_use = (m == -CUDART_INF_F) ? 0.f : m;
        {
          // the tile's largest P, computed exactly as in the loop below, minus
          // its 16-bit rounding (0 when the whole tile is masked for this row)
          const float p_top = ex2_approx(fmaf(s_max, sl2, -m_use));
          lc += p_top - unpack2<F16>(pack2<F16>(p_top, 0.f)).x;
        }
        const uint64_t negm2 = f2_pack(-m_use, -m_use);
        uint32_t pk[64];
        // the exponent arguments, row sums and keep products in packed f32x2
        // operations, or (d = 128 with dropout) as pairs of scalar ones: the
        // same per-lane arithmetic, fewer registers next to the keep words
        constexpr bool kScalarFp = (D == 128) && DROPOUT;
        uint64_t rs0 = 0ull, rs1 = 0ull;
        float r0a = 0.f, r0b = 0.f, r1a = 0.f, r1b = 0.f;
        // the other calls inside the exponential loop, 4 at a time, 32 keys
        // ahead of the pairs that use them (chunk k = pairs 16k .. 16k + 15)
        uint32_t wn[4][4], wc[4][4];
#pragma unroll
        for (int c = 0; c < kBN / 2; ++c) {
          if (DROPOUT && (c & 15) == 0) {
            const int k = c >> 4;  // chunk of this pair
            if (k >= kPre / 4) {
#pragma unroll
              for (int n = 0; n < 4; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) wc[n][e] = wn[n][e];
            }
            // the next chunk's words are drawn while this chunk is
            // exponentiated (chunks from kPre / 4 on come from here)
            const int kd = (k + 1 >= kPre / 4) ? k + 1 : -1;
            if (kd >= kPre / 4 && kd < kBN / 32)
              philox4x32_10_c0_batch<4>(static_cast<uint32_t>(t * (kBN / 8) + 4 * kd), phx, p.philox_rk, wn);
          }
          const float sv0 = s[2 * c], sv1 = s[2 * c + 1];
          float x0, x1;
          if constexpr (kScalarFp) {
            x0 = fmaf(sv0, sl2, -m_use);
            x1 = fmaf(sv1, sl2, -m_use);
          } else {
            f2_unpack(fma_f2(f2_pack(sv0, sv1), sl2x2, negm2), x0, x1);
          }
          const float p0 = ex2_approx(x0);
          const float p1 = ex2_approx(x1);
          const uint64_t pp = f2_pack(p0, p1);
          if constexpr (kScalarFp) {
            if (c & 1) {
              r1a += p0;
              r1b += p1;
            } else {
              r0a += p0;
              r0b += p1;
            }
          } else if (c & 1) {
            rs1 = add_f2(rs1, pp);
          } else {
            rs0 = add_f2(rs0, pp);
          }
          if (DROPOUT && c < 4 * kPre) {
            // keys of the calls drawn before S: the byte signs of kz spread
            // over 16-bit lanes (PRMT sign mode) zero the dropped P
            pk[c] = pack2<F16>(p0, p1) & prmt(kz[c >> 1], 0u, (c & 1) ? 0xBBAAu : 0x9988u);
          } else if (DROPOUT) {
            // keep test on the FMA pipe: the float 2^23 + u16 is exact, and
            // sat((2^23 + u) - (2^23 + t - 1)) is 1.0 when u >= t, else 0.0;
            // dropped keys get P = 0 (the row sum l keeps them)
            const uint32_t wv = wc[(c & 15) >> 2][c & 3];
            float k0, k1;
            asm("add.rn.sat.f32 %0, %1, %2;" : "=f"(k0) : "f"(__uint_as_float(prmt(wv, 0x4B000000u, 0x7610u))),
                "f"(drop_bias));
            asm("add.rn.sat.f32 %0, %1, %2;" : "=f"(k1) : "f"(__uint_as_float(prmt(wv, 0x4B000000u, 0x7632u))),
                "f"(drop_bias));
            float q0, q1;
            if constexpr (kScalarFp) {
              q0 = p0 * k0;
              q1 = p1 * k1;
            } else {
              f2_unpack(mul_f2(pp, f2_pack(k0, k1)), q0, q1);
            }
            pk[c] = pack2<F16>(q0, q1);
          } else {
            pk[c] = pack2<F16>(p0, p1);
          }
          if (c == kBN / 4 - 1) tmem_st32(t_s, pk);  // the first half of P (S is all in registers)
        }
        {
          float a0, a1;
          if constexpr (kScalarFp) {
            a0 = r0a + r1a;
            a1 = r0b + r1b;
          } else {
            f2_unpack(add_f2(rs0, rs1), a0, a1);
          }
          l += a0 + a1;
        }

        if (rescale && t > 0) {
          // O accumulator of this row, after the S row is consumed (fewer live
          // registers); every earlier PV MMA completed before S_t was committed
          // and the next one waits for p_ready
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
        tmem_st32(t_s + 32, pk + 32);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.p_ready[q]);
      }
      const bool row_ok = i < N;  // rows of a partial last tile past N are computed but not stored
      const int q0 = reinterpret_cast<const int*>(smem + L::kMisc)[2];
      const int gq = reinterpret_cast<const int*>(smem + L::kMisc)[3];
      uint16_t* orow_g = p.O + static_cast<size_t>(q0 + i) * p.seq.tok_stride +
                         static_cast<size_t>(gq) * p.seq.q_head_stride;
      float* lse_g = p.LSE + static_cast<size_t>(gq) * p.seq.total_q + q0 + i;
      if (ntq == 0) {
        // the whole tile sees no key: O = 0, LSE = -inf
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow_g);
#pragma unroll
          for (int e = 0; e < D / 8; ++e)
            if (e * 8 < p.dh) dst[e] = make_uint4(0u, 0u, 0u, 0u);
          *lse_g = -CUDART_INF_F;
        }
      } else if (ok && mbar_wait(&bar.o_ready[q], 0, abort_flag, p.err)) {
        // ---------------------------------------------------------- epilogue
        tc_fence_after();
        // l = 0: the row saw no key (O = 0, LSE = -inf)
        // O is normalised by the sum of the P it was built from (l - lc),
        // the LSE by the exact sum l
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
          if (row_ok && c * 32 < p.dh) {  // padded columns are not stored
            uint4* dst = reinterpret_cast<uint4*>(orow_g + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
          }
        }
        if (row_ok) *lse_g = (l > 0.f) ? (m + lg2_approx(l)) * 0.69314718055994531f : -CUDART_INF_F;
      }
    }
    cta_teardown(tmem, false);
  }
}

template <int D, bool CAUSAL, bool DROPOUT, bool F16>
cudaError_t launch_fwd_t(const FwdArgs& a, cudaStream_t stream) {
  auto kern = fa_fwd_kernel<D, CAUSAL, DROPOUT, F16>;
  const int smem = FwdSmem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // setmaxnreg.inc only succeeds if the launch reserved the pool the split assumes
  cudaFuncAttributes attr;
  e = cudaFuncGetAttributes(&attr, kern);
  if (e != cudaSuccess) return e;
  if (attr.numRegs < kFwdLaunchRegs) return cudaErrorInvalidConfiguration;
  FwdParams p;
  p.O = static_cast<uint16_t*>(a.O);
  p.LSE = a.LSE;
  p.err = a.err;
  p.seq = a.seq;
  p.dh = a.d;
  p.scale_log2 = a.scale_log2;
  p.drop_t = a.drop_t;
  p.drop_scale = a.drop_scale;
  for (int r = 0; r < 20; ++r) p.philox_rk[r] = a.philox_rk[r];
  p.BH = a.seq.units;
  const int n_qb = ((a.seq.Nq + kBM - 1) / kBM + 1) / 2;
  {
    // units per group: about 256 work units (~2 waves on 148 SMs) per group,
    // so the blocks running together share their units' K and V in L2 while
    // the heaviest causal blocks of the group still start first
    p.group = (256 + n_qb / 2) / n_qb;
    if (p.group < 1) p.group = 1;
    if (p.group > p.BH) p.group = p.BH;
  }
  dim3 grid(static_cast<unsigned>(p.BH) * n_qb);
  kern<<<grid, kFwdThreads, smem, stream>>>(a.tmQ, a.tmK, a.tmV, p);
  return cudaGetLastError();
}

template <bool F16>
cudaError_t launch_fwd_typed(const FwdArgs& a, cudaStream_t stream) {
  const bool drop = a.drop_t != 0;
  if (a.d <= 64) {
    if (a.causal)
      return drop ? launch_fwd_t<64, true, true, F16>(a, stream) : launch_fwd_t<64, true, false, F16>(a, stream);
    return drop ? launch_fwd_t<64, false, true, F16>(a, stream) : launch_fwd_t<64, false, false, F16>(a, stream);
  }
  if (a.causal)
    return drop ? launch_fwd_t<128, true, true, F16>(a, stream) : launch_fwd_t<128, true, false, F16>(a, stream);
  return drop ? launch_fwd_t<128, false, true, F16>(a, stream) : launch_fwd_t<128, false, false, F16>(a, stream);
}

}  // namespace

cudaError_t launch_fwd(const FwdArgs& a, cudaStream_t stream) {
  if (a.d > 128) return launch_fwd_wide(a, stream);  // head dimensions 192 and 256 (fa_fwd_wide.cu)
  return a.f16 ? launch_fwd_typed<true>(a, stream) : launch_fwd_typed<false>(a, stream);
}

}  // namespace fa
