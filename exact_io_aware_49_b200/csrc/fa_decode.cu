// fa_decode.cu -- attention over a paged key/value cache for decoding (sm_100a).
//
// Serving systems keep the key/value cache in non-contiguous fixed-size pages
// and run FlashAttention-style kernels over it while decoding ("FlashAttention"
// glossary, the inference-server bullets on vLLM and the PagedAttention
// entry).  The result is exact attention of the few newest queries of each
// sequence over all of its cached positions:
//   * cache [num_pages, page_size, H_kv, d]; block_table[b, n] = page holding
//     positions n*page_size .. of sequence b; seqlens[b] = its cached length;
//   * Q, O [B, H, Nq, d]; LSE [B, H, Nq]; query head h reads key/value head
//     h / (H / H_kv); the queries are the last Nq positions (causal mask
//     bottom-right aligned);
//   * a row that sees no key gets O = 0, LSE = -inf.
//
// Design (B200).  Decoding reads every cached key and value once and does
// ~2 * rows FLOPs per element; the arithmetic is a pair of small products per
// 128-key tile, so it runs on the tensor cores in the transposed form where
// the 128 keys are the M = 128 side and the (up to 16) query rows the N = 16
// side, leaving the CUDA cores only the softmax:
//   * S^T = K_tile Q^T   (tcgen05, A = K tile, B = Q rows, fp32 in TMEM:
//     lane = key, column = query row);
//   * softmax over keys, i.e. across TMEM lanes: each of 128 threads holds
//     one key's scores of the CTA's rows (4, 8 or 16 columns: the kernel is
//     instantiated for the row count, the products keep N = 16), a
//     reduce-scatter of shuffles per warp and one exchange through shared
//     memory give every row's tile max and sum; the
//     O rescale is lazy (stale max kept until a row's max grows by more than
//     8 in log2 units, as in the forward kernel); P goes to shared memory as
//     16-bit [16 rows x 128 keys];
//   * O^T += V_tile^T P^T (tcgen05, A = V tile read MN-major, B = P; lane =
//     dimension, column = query row);
//   * warp 4 streams the tiles (1 to 8 pages each, located through the block
//     table) with TMA through a 3-stage (d = 128) / 4-stage (d = 64) mbarrier
//     ring and issues the MMAs (the whole warp runs the loop, one elected lane
//     issues); warps 0-3 do the softmax, the rescale and the epilogue.
// For d = 64 the V tile carries a second, all-zero 64-column box so the P V
// product keeps M = 128 (dimensions 64..127 come out as zeros).
// grid = (split, key/value head x block of up to 16 query rows, sequence): all
// query heads sharing a key/value head are done together, so each cached byte
// is read once per row block; long sequences are cut into splits that run on
// different SMs, written as fp32 partials with their LSE and combined by a
// merge kernel with the log-sum-exp weights (one split writes the final
// output directly).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kDecThreads = 160;  // 4 softmax warps + 1 producer warp
constexpr int kProducerWarp = 4;
constexpr int kTileKeys = 128;    // keys per tile = TMEM lanes of S^T
constexpr int kMaxRows = 16;      // query rows per CTA = N of both products
constexpr float kDecRescaleTau = 8.0f;

template <int D>
struct DecSmem {
  static constexpr int kStages = (D == 128) ? 3 : 4;
  static constexpr int kBox = kTileKeys * 128;  // one 64-column, 128-byte-row box of a tile (16 KB)
  static constexpr int kKBytes = kTileKeys * D * 2;
  static constexpr int kVBytes = 2 * kBox;       // two boxes; for d = 64 the second stays zero
  static constexpr int kStage = kKBytes + kVBytes;
  static constexpr int kQ = kStages * kStage;    // Q rows: [16][D] 16-bit, 128B-swizzled K-major
  static constexpr int kP = kQ + kMaxRows * D * 2;  // P: 2 x [16][128] 16-bit, 128B-swizzled K-major
  static constexpr int kPBytes = kMaxRows * kTileKeys * 2;
  static constexpr int kRed = kP + 2 * kPBytes;  // fp32 [2 parities][max, sum][16 rows][4 warps]
  static constexpr int kBar = kRed + 2 * 2 * kMaxRows * 4 * 4;
  // kfull[kStages], vfull[kStages], s_ready[2], p_ready[2], pv_done[2], drain (the pairs by
  // tile parity: a role may run one tile ahead of the role that waits, never two)
  static constexpr int kNumBars = 2 * kStages + 7;
  static constexpr int kMisc = kBar + kNumBars * 8;  // tmem slot, abort flag
  static constexpr int kUsed = kMisc + 16;
};

// Reduce-scatter of kRows per-lane values over a warp (kRows = 4, 8 or 16):
// log2(kRows) exchange steps (lane bits 4, 3, ...) each halve the values a
// lane holds, then plain butterfly steps over the remaining lane bits finish
// the reduction.  Afterwards every lane holds the warp-wide max (kMax) or sum
// of column scatter_col<kRows>(lane).
template <bool kMax, int kRows>
__device__ __forceinline__ float warp_reduce_scatter(float (&v)[kRows], int lane) {
  static_assert(kRows == 4 || kRows == 8 || kRows == 16, "rows per CTA");
#pragma unroll
  for (int lvl = 0; (kRows >> lvl) > 1; ++lvl) {
    const int half = kRows >> (lvl + 1);
    const int sh = 16 >> lvl;
    const bool up = lane & sh;
#pragma unroll
    for (int k = 0; k < half; ++k) {
      const float send = up ? v[k] : v[k + half];
      const float keep = up ? v[k + half] : v[k];
      const float recv = __shfl_xor_sync(0xffffffffu, send, sh);
      v[k] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  float d = v[0];
#pragma unroll
  for (int sh = 16 / kRows; sh >= 1; sh >>= 1) {
    const float recv = __shfl_xor_sync(0xffffffffu, d, sh);
    d = kMax ? fmaxf(d, recv) : d + recv;
  }
  return d;
}

template <int kRows>
__device__ __forceinline__ int scatter_col(int lane) {
  constexpr int kShift = (kRows == 16) ? 1 : ((kRows == 8) ? 2 : 3);
  return (lane >> kShift) & (kRows - 1);
}

// kN consecutive TMEM columns of this warp's 32 lanes (32x32b shape, kN = 4, 8, 16).
template <int kN>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[kN]) {
  if constexpr (kN == 16) {
    tmem_ld16(taddr, r);
  } else if constexpr (kN == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  } else {
    static_assert(kN == 4, "columns");
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
  }
}

template <int kN>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&r)[kN]) {
  if constexpr (kN == 16) {
    tmem_st16(taddr, r);
  } else if constexpr (kN == 8) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
  } else {
    static_assert(kN == 4, "columns");
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
                 "r"(r[2]), "r"(r[3])
                 : "memory");
  }
}

// Keeps the consumers of r after the preceding tmem_ld_wait() (see reg_fence32).
template <int kN>
__device__ __forceinline__ void reg_fence_cols(uint32_t (&r)[kN]) {
#pragma unroll
  for (int k = 0; k < kN; ++k) asm volatile("" : "+r"(r[k]));
}

template <int D, bool F16, int kRows>
__global__ void __launch_bounds__(kDecThreads, 1) fa_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                  const __grid_constant__ CUtensorMap tmV,
                                                                  const __grid_constant__ DecodeParams p) {
  using L = DecSmem<D>;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (!smem_layout_fits(smem_raw, smem, L::kUsed, p.err)) return;
  uint64_t* kfull = reinterpret_cast<uint64_t*>(smem + L::kBar);  // K of a stage landed
  uint64_t* vfull = kfull + S;                                      // V of a stage landed
  uint64_t* s_ready = vfull + S;  // [2], by tile parity
  uint64_t* p_ready = s_ready + 2;  // [2], by tile parity
  uint64_t* pv_done = p_ready + 2;  // [2], by tile parity
  uint64_t* drain = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  float* red = reinterpret_cast<float*>(smem + L::kRed);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x;
  const int g = blockIdx.y / p.row_chunks;  // key/value head
  const int r0 = (blockIdx.y - g * p.row_chunks) * kMaxRows;
  const int R = min(kMaxRows, p.rows - r0);  // rows of this CTA: row r is query head
  const int b = blockIdx.z;                  // g * group + (r0 + r) / Nq, query (r0 + r) % Nq
  // cached length, clamped to what the block table can address
  const int Lk = min(max(p.seqlens[b], 0), p.max_pages * p.page);
  const int n_tiles = (Lk + kTileKeys - 1) / kTileKeys;
  const int t_begin = split * p.tiles_per_split;
  const int n = max(0, min(n_tiles, t_begin + p.tiles_per_split) - t_begin);  // tiles of this split

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&vfull[s], 1);
    }
    mbar_init(&s_ready[0], 1);
    mbar_init(&s_ready[1], 1);
    mbar_init(&p_ready[0], 4);
    mbar_init(&p_ready[1], 4);
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  // Q rows -> the B operand of S^T: [16][D], 128-byte rows in 64-column boxes
  // (2 KB each), 16-byte chunks swizzled by row; rows past R are zero
  uint8_t* qsm = smem + L::kQ;
  for (int idx = tid; idx < kMaxRows * (D / 8); idx += kDecThreads) {
    const int r = idx / (D / 8), c8 = idx - r * (D / 8);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);  // rows past R and padded columns stay zero
    if (r < R && c8 * 8 < p.dh) {
      const int rr = r0 + r;
      const int h = g * p.group + rr / p.Nq, i = rr - (rr / p.Nq) * p.Nq;
      v = *reinterpret_cast<const uint4*>(p.Q + ((static_cast<size_t>(b) * p.H + h) * p.Nq + i) * p.dh + c8 * 8);
    }
    *reinterpret_cast<uint4*>(qsm + (c8 / 8) * (kMaxRows * 128) + r * 128 + (((c8 % 8) ^ (r & 7)) << 4)) = v;
  }
  // P rows from kRows on are never written by the softmax: zero both buffers
  // once, so the P V product reads zeros there
  if (kRows < kMaxRows)
    for (int idx = tid; idx < 2 * L::kPBytes / 16; idx += kDecThreads)
      *reinterpret_cast<uint4*>(smem + L::kP + idx * 16) = make_uint4(0u, 0u, 0u, 0u);
  if (D == 64) {
    // the second V box of every stage stays zero
    for (int idx = tid; idx < S * (L::kBox / 16); idx += kDecThreads) {
      const int s = idx / (L::kBox / 16), o = idx - s * (L::kBox / 16);
      *reinterpret_cast<uint4*>(smem + s * L::kStage + L::kKBytes + L::kBox + o * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  fence_proxy_async_smem();
  if (warp == kProducerWarp) {
    tmem_alloc(tmem_slot, 64);  // S^T double buffer: columns [0, 16) and [16, 32); O^T [32, 48)
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_o = tmem + 32;  // S^T of tile it: tmem + (it & 1) * 16

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA + MMA
    // The whole warp runs the loop, so descriptors and counters are
    // warp-uniform values; one elected lane issues the copies, the MMAs and
    // the commits.
    if (n > 0) {
      const bool leader = elect_one();
      if (leader) {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
      }
      // a tile's page ids are read from the block table one refill ahead of
      // its copies, so the copies never wait for those reads
      constexpr int kMaxPagesPerTile = kTileKeys / 16;
      auto pages_of = [&](int it) {
        const int first = (t_begin + it) * kTileKeys;
        return min(kTileKeys / p.page, (Lk - first + p.page - 1) / p.page);
      };
      auto read_pids = [&](int it, int (&ids)[kMaxPagesPerTile]) {
        const int first = (t_begin + it) * kTileKeys;
        const int pages_here = pages_of(it);
        const int* bt = p.block_table + static_cast<size_t>(b) * p.max_pages + first / p.page;
#pragma unroll
        for (int pg = 0; pg < kMaxPagesPerTile; ++pg) ids[pg] = (pg < pages_here) ? bt[pg] : 0;
      };
      auto issue = [&](int it, const int (&pids)[kMaxPagesPerTile]) {
        if (!leader) return;
        const int st = it % S;
        const int pages_here = pages_of(it);
        // K and V complete separately: S^T needs only K, so it starts while V is still arriving
        mbar_expect_tx(&kfull[st], static_cast<uint32_t>(pages_here * (D / 64) * p.page * 128));
        mbar_expect_tx(&vfull[st], static_cast<uint32_t>(pages_here * (D / 64) * p.page * 128));
#pragma unroll
        for (int pg = 0; pg < kMaxPagesPerTile; ++pg) {
          if (pg >= pages_here) break;
          const int pid = pids[pg];
          for (int c = 0; c < D / 64; ++c) {
            // an out-of-range page id reads zeros (outside the tensor map)
            uint8_t* kd = smem + st * L::kStage + c * L::kBox + pg * p.page * 128;
            tma_load_3d(kd, &tmK, c * 64, g, pid * p.page, &kfull[st]);
            tma_load_3d(kd + L::kKBytes, &tmV, c * 64, g, pid * p.page, &vfull[st]);
          }
        }
      };
      // descriptor bases; a stage, box, buffer or K-step offset (bytes / 16)
      // is added to the start-address field
      const uint64_t dk0 = sdesc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t dq0 = sdesc_sw128(smem_u32(qsm), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(smem) + L::kKBytes, L::kBox, 1024);
      const uint64_t dp0 = sdesc_sw128(smem_u32(smem + L::kP), 16, 1024);
      constexpr uint32_t idesc_s = idesc_f32acc(128, kMaxRows, false, false, F16);
      constexpr uint32_t idesc_o = idesc_f32acc(128, kMaxRows, true, false, F16);
      int issued = 0;
      int pids_next[kMaxPagesPerTile];
      for (; issued < min(S - 1, n); ++issued) {
        read_pids(issued, pids_next);
        issue(issued, pids_next);
      }
      if (issued < n) read_pids(issued, pids_next);
      // every lane waits; the vote keeps the warp's decision uniform
#define FA_WAIT(bar_, parity) __all_sync(0xffffffffu, mbar_wait((bar_), (parity), abort_flag, p.err))
      bool ok = true;
      int consumed = 0;  // tiles whose copies have landed
      // S^T = K Q^T of tile it into its TMEM buffer: M = 128 keys, N = 16 rows, K = D (both K-major)
      auto issue_s = [&](int it) -> bool {
        const int st = it % S;
        if (!FA_WAIT(&kfull[st], (it / S) & 1)) return false;
        consumed = it + 1;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off_k = st * L::kStage + (kk / 4) * L::kBox + (kk % 4) * 32;
            const uint32_t off_q = (kk / 4) * (kMaxRows * 128) + (kk % 4) * 32;
            mma_ss(tmem + (it & 1) * 16, dk0 + (off_k >> 4), dq0 + (off_q >> 4), idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(&s_ready[it & 1]);
        }
        return true;
      };
      ok = issue_s(0);
      for (int it = 0; ok && it < n; ++it) {
        // refill the stage of tile it - 1 once its P V product has read it
        // (before waiting for the next tile's K, so the copies go out early)
        if (issued < n) {
          if (it >= 1 && !FA_WAIT(&pv_done[(it - 1) & 1], ((it - 1) >> 1) & 1)) {
            ok = false;
            break;
          }
          issue(issued, pids_next);
          ++issued;
          if (issued < n) read_pids(issued, pids_next);
        }
        // the next tile's S^T runs while the softmax warps work on this one; its
        // buffer was last read by the softmax of tile it - 1 (p_ready seen below)
        if (it + 1 < n && !issue_s(it + 1)) { ok = false; break; }
        if (!FA_WAIT(&p_ready[it & 1], (it >> 1) & 1) || !FA_WAIT(&vfull[it % S], (it / S) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // O^T += V^T P^T: M = 128 dimensions (V read MN-major), N = 16 rows, K = 128 keys
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < kTileKeys / 16; ++kk) {
            const uint32_t off_v = (it % S) * L::kStage + kk * 2048;
            const uint32_t off_p = (it & 1) * L::kPBytes + (kk / 4) * (kMaxRows * 128) + (kk % 4) * 32;
            mma_ss(tm_o, dv0 + (off_v >> 4), dp0 + (off_p >> 4), idesc_o, (it > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&pv_done[it & 1]);
        }
      }
#undef FA_WAIT
      if (!ok) {
        // copies and products in flight finish before shared and tensor memory go away
        if (leader) mma_commit(drain);
        mbar_wait_drain(drain, 0);
        if (leader) {
          for (int it2 = consumed; it2 < issued; ++it2) mbar_wait_drain(&kfull[it2 % S], (it2 / S) & 1);
          for (int it2 = max(0, consumed - 1); it2 < issued; ++it2)
            mbar_wait_drain(&vfull[it2 % S], (it2 / S) & 1);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    // only the first kRows >= R columns of S^T and O^T carry rows of this CTA
    float m_st[kRows], l_r[kRows];  // per row: stale max (log2 units) and sum, same in every thread
#pragma unroll
    for (int c = 0; c < kRows; ++c) {
      m_st[c] = -CUDART_INF_F;
      l_r[c] = 0.f;
    }
    const int col = scatter_col<kRows>(lane);
    // last visible position of each row: the cached length, and under the
    // causal mask the row's own position Lk - Nq + i; rows past R see nothing
    int lim[kRows];
#pragma unroll
    for (int c = 0; c < kRows; ++c) {
      const int i = (r0 + c) % p.Nq;
      lim[c] = (c >= R) ? -1 : (p.causal ? min(Lk - 1, Lk - p.Nq + i) : Lk - 1);
    }
    // Every wait below is bounded and may end differently in different
    // threads; the named barriers AND the outcomes, so the 128 threads leave
    // the loop together and tensor-memory instructions only run when all
    // agree.
    bool ok = true;
    for (int it = 0; it < n; ++it) {
      const int first = (t_begin + it) * kTileKeys;
      const int j = warp * 32 + lane;  // this thread's key in the tile
      const int pos = first + j;
      ok = named_bar_and(1, 128, mbar_wait(&s_ready[it & 1], (it >> 1) & 1, abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[kRows];
      tmem_ld_cols<kRows>(tmem + (it & 1) * 16 + lane_base, sr);
      tmem_ld_wait();
      reg_fence_cols<kRows>(sr);
      float s[kRows];
#pragma unroll
      for (int c = 0; c < kRows; ++c) s[c] = (pos <= lim[c]) ? __uint_as_float(sr[c]) * p.scale_log2 : -CUDART_INF_F;
      // tile max per row: reduce over this warp's keys, then over the 4 warps
      float* rmax = red + ((it & 1) * 2 + 0) * kMaxRows * 4;
      float* rsum = red + ((it & 1) * 2 + 1) * kMaxRows * 4;
      {
        float v[kRows];
#pragma unroll
        for (int c = 0; c < kRows; ++c) v[c] = s[c];
        const float wm = warp_reduce_scatter<true, kRows>(v, lane);
        if ((lane & (32 / kRows - 1)) == 0) rmax[col * 4 + warp] = wm;
      }
      // V rows of positions past the sequence (or of pages not loaded) may
      // hold anything, NaN included, and 0 * NaN would reach O through the
      // tensor core: once the tile's V has landed, zero them
      bool v_ok = true;
      if (first + kTileKeys > Lk) {
        v_ok = mbar_wait(&vfull[it % S], (it / S) & 1, abort_flag, p.err);
        if (v_ok && pos >= Lk) {
          uint8_t* vrow = smem + (it % S) * L::kStage + L::kKBytes + j * 128;
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<uint4*>(vrow + c * L::kBox + q * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      // (this barrier also covers the P buffer: the product of tile it - 2 has read it)
      const bool p_free = (it < 2) || mbar_wait(&pv_done[it & 1], ((it - 2) >> 1) & 1, abort_flag, p.err);
      ok = named_bar_and(1, 128, p_free && v_ok);
      if (!ok) break;
      float alpha[kRows];
      bool rescale = false;  // the same in every thread: computed from the same shared values
#pragma unroll
      for (int c = 0; c < kRows; ++c) {
        const float4 w4 = *reinterpret_cast<const float4*>(rmax + c * 4);
        const float m_tile = fmaxf(fmaxf(w4.x, w4.y), fmaxf(w4.z, w4.w));
        const float m_new = fmaxf(m_st[c], m_tile);
        alpha[c] = 1.f;
        if (m_new > m_st[c] + kDecRescaleTau) {  // also the first visible key of the row (m_st = -inf)
          alpha[c] = ex2_approx(m_st[c] - m_new);  // 0 when m_st = -inf
          m_st[c] = m_new;
          rescale = true;
        }
      }
      float pv[kRows];
#pragma unroll
      for (int c = 0; c < kRows; ++c) {
        const float mu = (m_st[c] == -CUDART_INF_F) ? 0.f : m_st[c];
        pv[c] = ex2_approx(s[c] - mu);  // 0 for masked keys
      }
      uint8_t* psm = smem + L::kP + (it & 1) * L::kPBytes;
      {
        const int box = j / 64, kin = j % 64;
#pragma unroll
        for (int c = 0; c < kRows; ++c) {
          const uint32_t bits = pack2<F16>(pv[c], 0.f);
          *reinterpret_cast<uint16_t*>(psm + box * (kMaxRows * 128) + c * 128 + (((kin >> 3) ^ (c & 7)) << 4) +
                                       (kin & 7) * 2) = static_cast<uint16_t>(bits & 0xFFFFu);
        }
      }
      {
        float v[kRows];
#pragma unroll
        for (int c = 0; c < kRows; ++c) v[c] = pv[c];
        const float ws = warp_reduce_scatter<false, kRows>(v, lane);
        if ((lane & (32 / kRows - 1)) == 0) rsum[col * 4 + warp] = ws;
      }
      // rescale O^T (lane = dimension) when a row's max moved: the previous
      // P V product must have finished
      const bool prev_done =
          !(rescale && it > 0) || mbar_wait(&pv_done[(it - 1) & 1], ((it - 1) >> 1) & 1, abort_flag, p.err);
      ok = named_bar_and(1, 128, prev_done);  // also: every row sum partial is written
      if (!ok) break;
#pragma unroll
      for (int c = 0; c < kRows; ++c) {
        const float4 w4 = *reinterpret_cast<const float4*>(rsum + c * 4);
        l_r[c] = l_r[c] * alpha[c] + ((w4.x + w4.y) + (w4.z + w4.w));
      }
      if (rescale && it > 0) {
        tc_fence_after();
        uint32_t orow[kRows];
        tmem_ld_cols<kRows>(tm_o + lane_base, orow);
        tmem_ld_wait();
        reg_fence_cols<kRows>(orow);
#pragma unroll
        for (int c = 0; c < kRows; ++c) orow[c] = __float_as_uint(__uint_as_float(orow[c]) * alpha[c]);
        tmem_st_cols<kRows>(tm_o + lane_base, orow);
        tmem_st_wait();
      }
      fence_proxy_async_smem();  // P is read by the tensor core (async proxy)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[it & 1]);
    }
    // ---------------------------------------------------------------- epilogue
    if (ok && n > 0)
      ok = named_bar_and(1, 128, mbar_wait(&pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag, p.err));
    if (ok) {
      float o[kRows];
      if (n > 0) {
        tc_fence_after();
        uint32_t orow[kRows];
        tmem_ld_cols<kRows>(tm_o + lane_base, orow);
        tmem_ld_wait();
        reg_fence_cols<kRows>(orow);
#pragma unroll
        for (int c = 0; c < kRows; ++c) o[c] = __uint_as_float(orow[c]);
      } else {
#pragma unroll
        for (int c = 0; c < kRows; ++c) o[c] = 0.f;
      }
      const int dim = warp * 32 + lane;
#pragma unroll
      for (int c = 0; c < kRows; ++c) {
        if (c >= R) continue;
        const int rr = r0 + c;
        const int h = g * p.group + rr / p.Nq, i = rr - (rr / p.Nq) * p.Nq;
        const size_t row = (static_cast<size_t>(b) * p.H + h) * p.Nq + i;
        const float l = l_r[c];
        const float val = (l > 0.f) ? o[c] / l : 0.f;
        const float lse = (l > 0.f) ? (m_st[c] + lg2_approx(l)) * 0.69314718055994531f : -CUDART_INF_F;
        if (dim < p.dh) {
          if (p.splits == 1)
            p.O[row * p.dh + dim] = static_cast<uint16_t>(pack2<F16>(val, 0.f) & 0xFFFFu);
          else
            p.O_part[(row * p.splits + split) * p.dh + dim] = val;
        }
        if (dim == 0) {
          if (p.splits == 1)
            p.LSE[row] = lse;
          else
            p.LSE_part[row * p.splits + split] = lse;
        }
      }
    }
  }
  // teardown: every role is done with tensor memory
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kProducerWarp) tmem_dealloc(tmem, 64);
}

// One warp per output row: O = sum_s w_s O_s / sum_s w_s with w_s = exp(LSE_s - max),
// LSE = max + ln(sum_s w_s); rows whose splits all saw nothing get O = 0, LSE = -inf.
template <int D, bool F16>
__global__ void __launch_bounds__(256) fa_decode_merge_kernel(const float* __restrict__ O_part,
                                                              const float* __restrict__ LSE_part,
                                                              uint16_t* __restrict__ O, float* __restrict__ LSE,
                                                              long long rows, int splits, int dh) {
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long row = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    const float* ls = LSE_part + row * splits;
    float mx = -CUDART_INF_F;
    for (int s = lane; s < splits; s += 32) mx = fmaxf(mx, ls[s]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    constexpr int kPer = D / 32;  // columns per lane
    float acc[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
    float wsum = 0.f;
    if (mx != -CUDART_INF_F) {
      for (int s = 0; s < splits; ++s) {
        const float w = __expf(ls[s] - mx);  // 0 for a split that saw nothing
        wsum += w;
        const float* op = O_part + (row * splits + s) * dh + lane * kPer;
        if (lane * kPer < dh) {
#pragma unroll
          for (int e = 0; e < kPer; ++e) acc[e] = fmaf(w, op[e], acc[e]);
        }
      }
    }
    const float inv = (wsum > 0.f) ? 1.f / wsum : 0.f;
    if (lane * kPer < dh) {  // dh is a multiple of 32: a lane's columns are all in or all out
#pragma unroll
      for (int e = 0; e < kPer; e += 2) {
        const uint32_t packed = pack2<F16>(acc[e] * inv, acc[e + 1] * inv);
        *reinterpret_cast<uint32_t*>(O + row * dh + lane * kPer + e) = packed;
      }
    }
    if (lane == 0) LSE[row] = (wsum > 0.f) ? mx + __logf(wsum) : -CUDART_INF_F;
  }
}

template <int D, bool F16, int kRows>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t stream) {
  auto kern = fa_decode_kernel<D, F16, kRows>;
  const int smem = DecSmem<D>::kUsed + 1024;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const DecodeParams& p = a.p;
  dim3 grid(p.splits, a.H_kv * p.row_chunks, a.B);
  kern<<<grid, kDecThreads, smem, stream>>>(a.tmK, a.tmV, p);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.splits == 1) return e;
  const long long rows = static_cast<long long>(a.B) * p.H * p.Nq;
  long long blocks = (rows + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  fa_decode_merge_kernel<D, F16><<<static_cast<int>(blocks), 256, 0, stream>>>(p.O_part, p.LSE_part, p.O, p.LSE,
                                                                                rows, p.splits, p.dh);
  return cudaGetLastError();
}

}  // namespace

template <int D, bool F16>
cudaError_t launch_decode_rows(const DecodeArgs& a, cudaStream_t stream) {
  // the softmax handles only as many S^T / O^T columns as a CTA has rows
  // (query heads per key/value head times queries, up to 16 per CTA)
  const int rows = a.p.row_chunks > 1 ? kMaxRows : a.p.rows;
  if (rows <= 4) return launch_decode_t<D, F16, 4>(a, stream);
  if (rows <= 8) return launch_decode_t<D, F16, 8>(a, stream);
  return launch_decode_t<D, F16, 16>(a, stream);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  if (a.d <= 64) return a.f16 ? launch_decode_rows<64, true>(a, stream) : launch_decode_rows<64, false>(a, stream);
  return a.f16 ? launch_decode_rows<128, true>(a, stream) : launch_decode_rows<128, false>(a, stream);
}

int decode_rows_per_cta() { return kMaxRows; }
int decode_keys_per_tile() { return kTileKeys; }

}  // namespace fa
