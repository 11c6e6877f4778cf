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
// ~2 * rows FLOPs per element, so for the few query rows per key/value head
// that decoding has, the kernel is HBM-bound: it streams 128-key tiles (1 to
// 8 pages each, located through the block table) with TMA into 128-byte-
// swizzled shared memory through a 3- or 4-stage mbarrier ring and does the
// arithmetic on the CUDA cores in fp32.
//   * grid = (split, key/value head x block of up to 16 query rows, sequence):
//     the rows of all query heads sharing a key/value head are done together,
//     so each cached byte is read once per row block; long sequences are cut
//     into splits that run on different SMs;
//   * per tile (512 threads): four lanes per key compute the scores of all
//     rows, one warp per row updates the running max / sum and turns scores
//     into probabilities, and each thread accumulates P V for a column pair
//     over a group of the tile's keys (packed f32x2 FMAs); the key groups are
//     added once at the end;
//   * splits write fp32 partial outputs with their LSE; a merge kernel
//     combines them with the log-sum-exp weights (one split writes the final
//     output directly).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kDecThreads = 512;
constexpr int kTileKeys = 128;  // keys per tile
constexpr int kMaxRows = 8;     // query rows per CTA (one softmax warp each)
constexpr int kKeyLanes = kDecThreads / kTileKeys;  // lanes per key in the score phase (4)

template <int D>
struct DecSmem {
  static constexpr int kStages = (D == 128) ? 3 : 4;
  static constexpr int kHalf = kTileKeys * D * 2;  // K or V tile: 128 keys x D 16-bit
  static constexpr int kBox = kTileKeys * 128;     // one 64-column, 128-byte-row box of a tile
  static constexpr int kStage = 2 * kHalf;         // K then V
  // query rows, fp32, pre-scaled to log2 units; each of the kKeyLanes dimension
  // parts of a row is padded by 4 floats so the lanes of a key read different banks
  static constexpr int kQPart = D / kKeyLanes + 4;
  static constexpr int kQ = kStages * kStage;
  static constexpr int kS = kQ + kMaxRows * kKeyLanes * kQPart * 4;  // fp32 [kMaxRows][kTileKeys]
  static constexpr int kStat = kS + kMaxRows * kTileKeys * 4;         // m, l, alpha: fp32 [kMaxRows] each
  static constexpr int kBar = kStat + 3 * kMaxRows * 4;
  static constexpr int kMisc = kBar + kStages * 8;  // abort flag
  static constexpr int kUsed = kMisc + 16;
  // P V: each thread owns a column pair and a group of the tile's keys; the
  // groups' partial sums are added once at the end (through the stage buffers)
  static constexpr int kColPairs = D / 2;
  static constexpr int kKeyGroups = kDecThreads / kColPairs;  // 8 (D = 128) or 16 (D = 64)
  static constexpr int kKeysPerGroup = kTileKeys / kKeyGroups;
  static_assert(kKeyGroups * kMaxRows * D * 4 <= kStages * kStage, "partial sums fit the stage buffers");
};

template <int D, bool F16>
__global__ void __launch_bounds__(kDecThreads, 1) fa_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                  const __grid_constant__ CUtensorMap tmV,
                                                                  const __grid_constant__ DecodeParams p) {
  using L = DecSmem<D>;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (!smem_layout_fits(smem_raw, smem, L::kUsed, p.err)) return;
  float* qs = reinterpret_cast<float*>(smem + L::kQ);
  float* ss = reinterpret_cast<float*>(smem + L::kS);
  float* m_s = reinterpret_cast<float*>(smem + L::kStat);
  float* l_s = m_s + kMaxRows;
  float* a_s = l_s + kMaxRows;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc);

  const int tid = threadIdx.x;
  const int split = blockIdx.x;
  const int g = blockIdx.y / p.row_chunks;  // key/value head
  const int r0 = (blockIdx.y - g * p.row_chunks) * kMaxRows;
  const int R = min(kMaxRows, p.rows - r0);  // rows of this CTA: row r is query head
  const int b = blockIdx.z;                  // g * group + (r0 + r) / Nq, query (r0 + r) % Nq
  // cached length, clamped to what the block table can address
  const int Lk = min(max(p.seqlens[b], 0), p.max_pages * p.page);
  const int n_tiles = (Lk + kTileKeys - 1) / kTileKeys;
  const int t_begin = split * p.tiles_per_split;
  const int t_end = min(n_tiles, t_begin + p.tiles_per_split);

  if (tid == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  // query rows in fp32, multiplied by scale * log2(e) so scores come out in log2 units
  for (int idx = tid; idx < R * (D / 8); idx += kDecThreads) {
    const int r = idx / (D / 8), c8 = idx - r * (D / 8);
    const int rr = r0 + r;
    const int h = g * p.group + rr / p.Nq, i = rr - (rr / p.Nq) * p.Nq;
    const uint4 v = *reinterpret_cast<const uint4*>(p.Q + ((static_cast<size_t>(b) * p.H + h) * p.Nq + i) * D + c8 * 8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const int dim0 = c8 * 8, part = dim0 / (D / kKeyLanes), within = dim0 - part * (D / kKeyLanes);
    float* dst = qs + (r * kKeyLanes + part) * L::kQPart + within;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack2<F16>(w[e]);
      dst[2 * e] = f.x * p.scale_log2;
      dst[2 * e + 1] = f.y * p.scale_log2;
    }
  }
  if (tid < kMaxRows) {
    m_s[tid] = -CUDART_INF_F;
    l_s[tid] = 0.f;
  }
  __syncthreads();

  // thread 0 streams the tiles: the pages of tile t that hold valid positions
  auto issue = [&](int t, int st) {
    const int pages_per_tile = kTileKeys / p.page;
    const int first = t * kTileKeys;
    const int pages_here = min(pages_per_tile, (Lk - first + p.page - 1) / p.page);
    mbar_expect_tx(&full[st], static_cast<uint32_t>(pages_here * 2 * (D / 64) * p.page * 128));
    for (int n = 0; n < pages_here; ++n) {
      const int pid = p.block_table[static_cast<size_t>(b) * p.max_pages + first / p.page + n];
      for (int c = 0; c < D / 64; ++c) {
        uint8_t* kd = smem + st * L::kStage + c * L::kBox + n * p.page * 128;
        // an out-of-range page id reads zeros (outside the tensor map)
        tma_load_3d(kd, &tmK, c * 64, g, pid * p.page, &full[st]);
        tma_load_3d(kd + L::kHalf, &tmV, c * 64, g, pid * p.page, &full[st]);
      }
    }
  };
  int issued = 0;
  if (tid == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    for (int k = 0; k < S - 1 && t_begin + k < t_end; ++k) issue(t_begin + k, k);
    issued = max(0, min(S - 1, t_end - t_begin));
  }

  // score phase mapping: key j, dimension part (kKeyLanes adjacent lanes per key)
  const int sj = tid / kKeyLanes, spart = tid % kKeyLanes;
  constexpr int kChunksPer = D / kKeyLanes / 8;  // 16-byte chunks per lane
  // P V mapping: column pair cp, key group kg
  const int cp = tid % L::kColPairs, kg = tid / L::kColPairs;
  const int vcol = 2 * cp;
  const int vbox = vcol / 64, vchunk = (vcol % 64) / 8, vbyte = (vcol % 8) * 2;
  float acc[kMaxRows][2];
#pragma unroll
  for (int r = 0; r < kMaxRows; ++r) acc[r][0] = acc[r][1] = 0.f;

  bool ok = true;
  int stop_it = 0;  // first tile not consumed when the loop stops early
  for (int t = t_begin, it = 0; t < t_end; ++t, ++it) {
    const int st = it % S;
    // the stage of tile t + S - 1 was last read in the previous iteration,
    // which every thread has left (barrier at the end of the loop)
    if (tid == 0 && t + S - 1 < t_end) {
      issue(t + S - 1, (it + S - 1) % S);
      ++issued;
    }
    if (!mbar_wait(&full[st], (it / S) & 1, abort_flag, p.err)) {
      ok = false;
      stop_it = it;
      break;
    }
    const int first = t * kTileKeys;
    const int nvalid = min(kTileKeys, Lk - first);
    const uint8_t* kt = smem + st * L::kStage;
    const uint8_t* vt = kt + L::kHalf;

    // ---- scores: kKeyLanes lanes per key, each a part of the dimensions
    {
      float s[kMaxRows];
#pragma unroll
      for (int r = 0; r < kMaxRows; ++r) s[r] = 0.f;
#pragma unroll
      for (int cc = 0; cc < kChunksPer; ++cc) {
        const int c = spart * kChunksPer + cc;  // 16-byte chunk of the row
        const uint4 kv = *reinterpret_cast<const uint4*>(kt + (c / 8) * L::kBox + sj * 128 +
                                                         (((c % 8) ^ (sj & 7)) << 4));
        const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
        float kf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack2<F16>(w[e]);
          kf[2 * e] = f.x;
          kf[2 * e + 1] = f.y;
        }
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r) {
          if (r < R) {
            const float* qr = qs + (r * kKeyLanes + spart) * L::kQPart + cc * 8;
            const float4 q0 = *reinterpret_cast<const float4*>(qr);
            const float4 q1 = *reinterpret_cast<const float4*>(qr + 4);
            uint64_t a2 = fma_f2(f2_pack(q0.x, q0.y), f2_pack(kf[0], kf[1]), f2_pack(s[r], 0.f));
            a2 = fma_f2(f2_pack(q0.z, q0.w), f2_pack(kf[2], kf[3]), a2);
            a2 = fma_f2(f2_pack(q1.x, q1.y), f2_pack(kf[4], kf[5]), a2);
            a2 = fma_f2(f2_pack(q1.z, q1.w), f2_pack(kf[6], kf[7]), a2);
            float lo, hi;
            f2_unpack(a2, lo, hi);
            s[r] = lo + hi;
          }
        }
      }
      const int pos = first + sj;
#pragma unroll
      for (int r = 0; r < kMaxRows; ++r) {
        if (r < R) {
          float v = s[r];
#pragma unroll
          for (int o = 1; o < kKeyLanes; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (spart == 0) {
            const int i = (r0 + r) % p.Nq;
            const bool visible = sj < nvalid && (!p.causal || pos <= Lk - p.Nq + i);
            ss[r * kTileKeys + sj] = visible ? v : -CUDART_INF_F;
          }
        }
      }
    }
    __syncthreads();

    // ---- online softmax: warp r takes row r
    {
      const int r = tid >> 5, lane = tid & 31;
      if (r < R) {
        float4 x = *reinterpret_cast<const float4*>(ss + r * kTileKeys + lane * 4);
        float mx = fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float m_old = m_s[r];
        const float m_new = fmaxf(m_old, mx);
        const float m_use = (m_new == -CUDART_INF_F) ? 0.f : m_new;  // nothing visible yet: P = 0
        x.x = ex2_approx(x.x - m_use);
        x.y = ex2_approx(x.y - m_use);
        x.z = ex2_approx(x.z - m_use);
        x.w = ex2_approx(x.w - m_use);
        float sum = (x.x + x.y) + (x.z + x.w);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        *reinterpret_cast<float4*>(ss + r * kTileKeys + lane * 4) = x;
        if (lane == 0) {
          const float alpha = (m_old == -CUDART_INF_F) ? 0.f : ex2_approx(m_old - m_use);
          a_s[r] = alpha;
          m_s[r] = m_new;
          l_s[r] = l_s[r] * alpha + sum;
        }
      }
    }
    __syncthreads();

    // ---- O += P V for this thread's column pair and key group
    {
#pragma unroll
      for (int r = 0; r < kMaxRows; ++r) {
        if (r < R) {
          const float a = a_s[r];
          acc[r][0] *= a;
          acc[r][1] *= a;
        }
      }
      const int j_lo = kg * L::kKeysPerGroup;
      const int j_hi = min(j_lo + L::kKeysPerGroup, nvalid);
      const uint8_t* vb = vt + vbox * L::kBox + vbyte;
      for (int j0 = j_lo; j0 < j_hi; j0 += 4) {
        float2 v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = j0 + e;
          // rows past the sequence may hold anything: read them as 0
          const uint32_t bits = *reinterpret_cast<const uint32_t*>(vb + j * 128 + ((vchunk ^ (j & 7)) << 4));
          v[e] = (j < j_hi) ? unpack2<F16>(bits) : make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r) {
          if (r < R) {
            const float4 pr = *reinterpret_cast<const float4*>(ss + r * kTileKeys + j0);
            uint64_t a2 = f2_pack(acc[r][0], acc[r][1]);
            a2 = fma_f2(f2_pack(pr.x, pr.x), f2_pack(v[0].x, v[0].y), a2);
            a2 = fma_f2(f2_pack(pr.y, pr.y), f2_pack(v[1].x, v[1].y), a2);
            a2 = fma_f2(f2_pack(pr.z, pr.z), f2_pack(v[2].x, v[2].y), a2);
            a2 = fma_f2(f2_pack(pr.w, pr.w), f2_pack(v[3].x, v[3].y), a2);
            f2_unpack(a2, acc[r][0], acc[r][1]);
          }
        }
      }
    }
    __syncthreads();  // the stage and the probabilities may be overwritten now
  }

  if (!ok) {
    // let the copies already in flight land before the CTA's shared memory goes away
    if (tid == 0)
      for (int it = stop_it; it < issued; ++it) mbar_wait_drain(&full[it % S], (it / S) & 1);
    __syncthreads();
    return;
  }

  // ---- add the key groups' partial sums (the stage buffers are idle now)
  float* part = reinterpret_cast<float*>(smem);  // [kKeyGroups][kMaxRows][D]
#pragma unroll
  for (int r = 0; r < kMaxRows; ++r)
    if (r < R)
      *reinterpret_cast<float2*>(part + (kg * kMaxRows + r) * D + vcol) = make_float2(acc[r][0], acc[r][1]);
  __syncthreads();

  // ---- outputs: the final row (one split) or an fp32 partial with its LSE
  for (int idx = tid; idx < R * D; idx += kDecThreads) {
    const int r = idx / D, col = idx - r * D;
    float o = 0.f;
#pragma unroll
    for (int q = 0; q < L::kKeyGroups; ++q) o += part[(q * kMaxRows + r) * D + col];
    const int rr = r0 + r;
    const int h = g * p.group + rr / p.Nq, i = rr - (rr / p.Nq) * p.Nq;
    const size_t row = (static_cast<size_t>(b) * p.H + h) * p.Nq + i;
    const float l = l_s[r];
    o = (l > 0.f) ? o / l : 0.f;
    const float lse = (l > 0.f) ? (m_s[r] + lg2_approx(l)) * 0.69314718055994531f : -CUDART_INF_F;
    if (p.splits == 1) {
      p.O[row * D + col] = static_cast<uint16_t>(pack2<F16>(o, 0.f) & 0xFFFFu);
      if (col == 0) p.LSE[row] = lse;
    } else {
      p.O_part[(row * p.splits + split) * D + col] = o;
      if (col == 0) p.LSE_part[row * p.splits + split] = lse;
    }
  }
}

// One warp per output row: O = sum_s w_s O_s / sum_s w_s with w_s = exp(LSE_s - max),
// LSE = max + ln(sum_s w_s); rows whose splits all saw nothing get O = 0, LSE = -inf.
template <int D, bool F16>
__global__ void __launch_bounds__(256) fa_decode_merge_kernel(const float* __restrict__ O_part,
                                                              const float* __restrict__ LSE_part,
                                                              uint16_t* __restrict__ O, float* __restrict__ LSE,
                                                              long long rows, int splits) {
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
        const float* op = O_part + (row * splits + s) * D + lane * kPer;
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[e] = fmaf(w, op[e], acc[e]);
      }
    }
    const float inv = (wsum > 0.f) ? 1.f / wsum : 0.f;
#pragma unroll
    for (int e = 0; e < kPer; e += 2) {
      const uint32_t packed = pack2<F16>(acc[e] * inv, acc[e + 1] * inv);
      *reinterpret_cast<uint32_t*>(O + row * D + lane * kPer + e) = packed;
    }
    if (lane == 0) LSE[row] = (wsum > 0.f) ? mx + __logf(wsum) : -CUDART_INF_F;
  }
}

template <int D, bool F16>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t stream) {
  auto kern = fa_decode_kernel<D, F16>;
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
                                                                                rows, p.splits);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  if (a.d == 64) return a.f16 ? launch_decode_t<64, true>(a, stream) : launch_decode_t<64, false>(a, stream);
  return a.f16 ? launch_decode_t<128, true>(a, stream) : launch_decode_t<128, false>(a, stream);
}

int decode_rows_per_cta() { return kMaxRows; }
int decode_keys_per_tile() { return kTileKeys; }

}  // namespace fa
