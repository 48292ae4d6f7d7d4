// pbs_select kernels: block pooling and per-query-block selection.
//
// "Sparser Block-Sparse Attention via Token Permutation", Technical Summary,
// 4. Implementation: block importance is estimated by mean pooling on the
// permuted keys.  Here the block score is S = (sum of the query block's
// rows) . (sum of the permuted key block's rows), which is blk^2 * sqrt(D)
// times the mean scaled logit of the tile.  Selection keeps the block's own
// segment (handled densely by the attention kernel), forces sink / band
// blocks, and then either takes the top blocks to reach a density budget or
// adds blocks by descending score until a cumulative attention mass is
// reached ("SampleAttention", Technical Deep Dive: the minimum attention mass
// to keep per query).
#include "pbs_common.cuh"
#include "pbs_internal.h"

#include <algorithm>

namespace pbs {
namespace {

// Sum of the `blk` rows of query block i: one CTA per (block, head, batch);
// thread = (16-byte chunk, row lane); fp32.  The rows are i*blk .. i*blk +
// blk - 1, or with a query permutation (qperm, [B, H, N]) the positions
// qperm[i*blk + r]; an entry outside block i's segment sets the error word
// and is skipped.
__global__ void __launch_bounds__(256) pool_query_blocks_kernel(
    const __nv_bfloat16* __restrict__ Q, int64_t sB, int64_t sH, int64_t sN, int D, int blk,
    const int32_t* __restrict__ qperm, int64_t N, int seg, int* err, float* __restrict__ qbar) {
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nb = gridDim.x, H = gridDim.y;
  const int nchunk = D / 8, chunk = threadIdx.x % nchunk;
  const int lanes = blockDim.x / nchunk, rl = threadIdx.x / nchunk;
  const int64_t p0 = static_cast<int64_t>(i) * blk;
  const __nv_bfloat16* base = Q + b * sB + h * sH;
  const int32_t* qrow = qperm ? qperm + (static_cast<int64_t>(b) * H + h) * N + p0 : nullptr;
  const int64_t seg_lo = (p0 / seg) * seg, seg_hi = min(seg_lo + seg, N);
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int r = rl; r < blk; r += lanes) {
    int64_t n = p0 + r;
    if (qrow) {
      n = qrow[r];
      if (n < seg_lo || n >= seg_hi) {
        set_error(err, kErrDeviceCheck);
        continue;
      }
    }
    const uint4 v = *reinterpret_cast<const uint4*>(base + n * sN + chunk * 8);
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __bfloat1622float2(p[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  }
  __shared__ float red[256 * 8];
#pragma unroll
  for (int e = 0; e < 8; ++e) red[threadIdx.x * 8 + e] = acc[e];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    const int ch = c / 8, e = c % 8;
    float t = 0.f;
    for (int l = 0; l < lanes; ++l) t += red[(l * nchunk + ch) * 8 + e];
    qbar[((static_cast<int64_t>(b) * H + h) * nb + i) * D + c] = t;
  }
}

// Per (permuted block pb, hkv, b): Kbar_perm = sum of rows perm[pb*blk+r];
// optionally Kbar_nat = sum of rows pb*blk+r; and the inverse permutation
// inv[perm[p]] = p.  A perm entry outside its segment sets the error word
// and is skipped.
// perm, inv and kbar_perm rows of consecutive (b, h) are perm_stride elements
// (inv likewise) and kbar_stride blocks apart: one permutation per KV head,
// or one per (KV head, query segment) launched segment by segment.
__global__ void __launch_bounds__(256) pool_key_blocks_kernel(
    const __nv_bfloat16* __restrict__ K, int64_t sB, int64_t sH, int64_t sN, int64_t N, int D,
    int blk, int seg, const int32_t* __restrict__ perm, int64_t perm_stride, int natural,
    float* __restrict__ kbar_perm, int64_t kbar_stride, float* __restrict__ kbar_nat,
    int32_t* __restrict__ inv, int* err) {
  const int pb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nb = gridDim.x, H = gridDim.y;
  __shared__ int32_t rows[256];
  __shared__ float red[256 * 8];
  const int64_t p0 = static_cast<int64_t>(pb) * blk;
  const int64_t seg_lo = (p0 / seg) * seg;
  const int64_t seg_hi = min(seg_lo + seg, N);
  const int32_t* prow = perm + (static_cast<int64_t>(b) * H + h) * perm_stride;
  int32_t* irow = inv + (static_cast<int64_t>(b) * H + h) * perm_stride;
  for (int r = threadIdx.x; r < blk; r += blockDim.x) {
    int32_t x = prow[p0 + r];
    if (x < seg_lo || x >= seg_hi) {
      set_error(err, kErrDeviceCheck);
      x = -1;
    } else {
      irow[x] = static_cast<int32_t>(p0 + r);
    }
    rows[r] = x;
  }
  __syncthreads();
  const int nchunk = D / 8, chunk = threadIdx.x % nchunk;
  const int lanes = blockDim.x / nchunk, rl = threadIdx.x / nchunk;
  const __nv_bfloat16* base = K + b * sB + h * sH;
  for (int pass = 0; pass < (natural ? 2 : 1); ++pass) {
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int r = rl; r < blk; r += lanes) {
      const int64_t x = pass == 0 ? rows[r] : p0 + r;
      if (x < 0) continue;
      const uint4 v = *reinterpret_cast<const uint4*>(base + x * sN + chunk * 8);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(p[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[threadIdx.x * 8 + e] = acc[e];
    __syncthreads();
    float* out = pass == 0 ? kbar_perm + ((static_cast<int64_t>(b) * H + h) * kbar_stride + pb) * D
                           : kbar_nat + ((static_cast<int64_t>(b) * H + h) * nb + pb) * D;
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
      const int ch = c / 8, e = c % 8;
      float t = 0.f;
      for (int l = 0; l < lanes; ++l) t += red[(l * nchunk + ch) * 8 + e];
      out[c] = t;
    }
    __syncthreads();
  }
}

// Block scores with one permutation per query segment: S[row, pb] =
// Qbar[row] . Kbar[s(row), pb] for the row's candidates pb < ncand.  One warp
// per (b, hq, i) row; each lane takes candidates lane, lane + 32, ... and
// reads that block's pooled key row as float4s against the row's pooled
// query held in shared memory.  Exact in fp32 on lattice inputs (every
// partial sum is a multiple of 2^-6 below 2^18), like the tiled kernel.
constexpr int kSegScoreWarps = 8;
__global__ void __launch_bounds__(kSegScoreWarps * 32) block_scores_seg_kernel(
    SelectParams p, const float* __restrict__ qbar, const float* __restrict__ kbar4,
    float* __restrict__ scores) {
  __shared__ __align__(16) float qs[kSegScoreWarps][128];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kSegScoreWarps + warp;
  if (row >= static_cast<int64_t>(p.B) * p.Hq * p.nb) return;
  const int i = static_cast<int>(row % p.nb);
  const int h = static_cast<int>((row / p.nb) % p.Hq);
  const int b = static_cast<int>(row / (static_cast<int64_t>(p.nb) * p.Hq));
  const int hk = h / (p.Hq / p.Hkv);
  const int spb = p.seg / p.blk;
  const int s = i / spb, ncand = s * spb;
  if (ncand == 0) return;
  for (int c = lane; c < p.D; c += 32) qs[warp][c] = qbar[row * p.D + c];
  __syncwarp();
  const float* kb = kbar4 + ((static_cast<int64_t>(b) * p.Hkv + hk) * p.perm_nseg + s) * p.nb * p.D;
  float* out = scores + row * p.nb;
  for (int pb = lane; pb < ncand; pb += 32) {
    const float4* kr = reinterpret_cast<const float4*>(kb + static_cast<int64_t>(pb) * p.D);
    float acc = 0.f;
    for (int c = 0; c < p.D / 4; ++c) {
      const float4 k4 = kr[c];
      acc = fmaf(qs[warp][4 * c], k4.x, acc);
      acc = fmaf(qs[warp][4 * c + 1], k4.y, acc);
      acc = fmaf(qs[warp][4 * c + 2], k4.z, acc);
      acc = fmaf(qs[warp][4 * c + 3], k4.w, acc);
    }
    out[pb] = acc;
  }
}

constexpr int kSelThreads = 256;

__device__ __forceinline__ double block_sum_f64(double v, double* red) {
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  for (int w = 0; w < kSelThreads / 32; ++w) t += red[w];
  __syncthreads();
  return t;
}

__device__ __forceinline__ double block_max_f64(double v, double* red) {
  for (int off = 16; off > 0; off >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, off));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = red[0];
  for (int w = 1; w < kSelThreads / 32; ++w) t = fmax(t, red[w]);
  __syncthreads();
  return t;
}

// Block scores S[b, hq, i, pb] = Qbar_i . Kbar_pb for every candidate
// pb < candidates(i), as a register-tiled fp32 GEMM per (batch, query head):
// 128 x 128 output tiles, 8 x 8 per thread (four 16-byte shared loads per
// 64 FMAs), d in chunks of 32, accumulated in d order.  Tiles wholly above
// the candidate triangle are skipped.  On lattice inputs every partial sum
// is exact, so any accumulation order gives the same scores.
constexpr int kTile = 128;

__global__ void __launch_bounds__(256, 2) block_scores_kernel(SelectParams p, const float* __restrict__ qbar,
                                                              const float* __restrict__ kbar_perm,
                                                              float* __restrict__ S) {
  const int ct = blockIdx.x, rt = blockIdx.y, bh = blockIdx.z;
  const int b = bh / p.Hq, h = bh % p.Hq, hk = h / (p.Hq / p.Hkv);
  const int spb = p.seg / p.blk;
  const int i_last = min((rt + 1) * kTile, p.nb) - 1;
  const int pb0 = ct * kTile;
  if (pb0 >= (i_last / spb) * spb) return;
  __shared__ __align__(16) float qs[32][kTile + 4];     // [d][row]
  __shared__ __align__(16) float ks[32][kTile + 4];     // [d][candidate]
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[8][8];
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int v = 0; v < 8; ++v) acc[u][v] = 0.f;
  const float* qsrc = qbar + (static_cast<int64_t>(b) * p.Hq + h) * p.nb * p.D;
  const float* ksrc = kbar_perm + (static_cast<int64_t>(b) * p.Hkv + hk) * p.nb * p.D;
  for (int d0 = 0; d0 < p.D; d0 += 32) {
    for (int x = threadIdx.x; x < kTile * 8; x += 256) {
      const int r = x / 8, d4 = x % 8;
      const int i = rt * kTile + r, pb = pb0 + r;
      const float4 qv = i < p.nb ? *reinterpret_cast<const float4*>(qsrc + static_cast<int64_t>(i) * p.D + d0 + 4 * d4)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 kv = pb < p.nb ? *reinterpret_cast<const float4*>(ksrc + static_cast<int64_t>(pb) * p.D + d0 + 4 * d4)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
      qs[4 * d4 + 0][r] = qv.x; qs[4 * d4 + 1][r] = qv.y; qs[4 * d4 + 2][r] = qv.z; qs[4 * d4 + 3][r] = qv.w;
      ks[4 * d4 + 0][r] = kv.x; ks[4 * d4 + 1][r] = kv.y; ks[4 * d4 + 2][r] = kv.z; ks[4 * d4 + 3][r] = kv.w;
    }
    __syncthreads();
#pragma unroll 4
    for (int dd = 0; dd < 32; ++dd) {
      // rows ty*4 .. +3 and 64 + ty*4 .. +3; candidates tx*4 .. +3 and 64 + tx*4 .. +3
      const float4 a0 = *reinterpret_cast<const float4*>(&qs[dd][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&qs[dd][64 + ty * 4]);
      const float4 c0 = *reinterpret_cast<const float4*>(&ks[dd][tx * 4]);
      const float4 c1 = *reinterpret_cast<const float4*>(&ks[dd][64 + tx * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[u][v] = fmaf(av[u], cv[v], acc[u][v]);
    }
    __syncthreads();
  }
  float* out = S + (static_cast<int64_t>(b) * p.Hq + h) * p.nb * p.nb;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int i = rt * kTile + (u < 4 ? ty * 4 + u : 64 + ty * 4 + u - 4);
    if (i >= p.nb) continue;
    const int nc = (i / spb) * spb;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int pb = pb0 + (v < 4 ? tx * 4 + v : 64 + tx * 4 + v - 4);
      if (pb < nc) out[static_cast<int64_t>(i) * p.nb + pb] = acc[u][v];
    }
  }
}

// Forced blocks of row i as a bitmap over candidates (one warp).
__device__ __forceinline__ void forced_bitmap(const SelectParams& p, const int32_t* irow, int i, int ncand,
                                              uint32_t* fbits, int lane) {
  const int words = (ncand + 31) >> 5;
  for (int w = lane; w < words; w += 32) fbits[w] = 0u;
  __syncwarp();
  const int spb = p.seg / p.blk;
  const int64_t s_start = static_cast<int64_t>(i / spb) * p.seg;
  const int64_t sink_hi = min(static_cast<int64_t>(p.n_sink), s_start);
  for (int64_t pos = lane; pos < sink_hi; pos += 32) {
    const int32_t lp = irow[pos];
    if (lp >= 0 && lp < static_cast<int64_t>(ncand) * p.blk) atomicOr(&fbits[(lp / p.blk) >> 5], 1u << ((lp / p.blk) & 31));
  }
  if (p.band > 0) {
    const int64_t band_lo = max(static_cast<int64_t>(0), static_cast<int64_t>(i) * p.blk - p.band + 1);
    for (int64_t pos = band_lo + lane; pos < s_start; pos += 32) {
      const int32_t lp = irow[pos];
      if (lp >= 0 && lp < static_cast<int64_t>(ncand) * p.blk) atomicOr(&fbits[(lp / p.blk) >> 5], 1u << ((lp / p.blk) & 31));
    }
  }
  __syncwarp();
}

// Top-k selection, one warp per (b, hq, i) row: radix select of the `want`
// smallest sort keys, where a forced block's key is 0 and any other block's
// is the order-inverted score (descending score); ties at the threshold go
// to the lowest block ids.  The chosen ids are written in ascending order.
constexpr int kWarpsPerCta = 8;

__global__ void __launch_bounds__(kWarpsPerCta * 32) select_topk_kernel(
    SelectParams p, const float* __restrict__ S_all, const int32_t* __restrict__ inv,
    int32_t* __restrict__ counts, int32_t* __restrict__ idx, int* err) {
  extern __shared__ __align__(16) uint32_t fb_all[];                 // kWarpsPerCta x nbw
  __shared__ uint32_t hist_all[kWarpsPerCta][256];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nbw = p.nb / 32 + 1;
  uint32_t* fbits = fb_all + warp * nbw;
  uint32_t* hist = hist_all[warp];
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + warp;
  if (row >= static_cast<int64_t>(p.B) * p.Hq * p.nb) return;
  const int i = static_cast<int>(row % p.nb);
  const int h = static_cast<int>((row / p.nb) % p.Hq);
  const int b = static_cast<int>(row / (static_cast<int64_t>(p.nb) * p.Hq));
  const int hk = h / (p.Hq / p.Hkv);
  const int spb = p.seg / p.blk;
  const int s = i / spb, ncand = s * spb, Di = i - s * spb + 1;
  if (ncand == 0) {
    if (lane == 0) counts[row] = 0;
    return;
  }
  const float* S = S_all + row * p.nb;
  forced_bitmap(p, inv + ((static_cast<int64_t>(b) * p.Hkv + hk) * p.perm_nseg + (p.perm_nseg > 1 ? s : 0)) * p.N,
                i, ncand, fbits, lane);
  const int words = (ncand + 31) >> 5;
  int nf = 0;
  for (int w = lane; w < words; w += 32) nf += __popc(fbits[w]);
  for (int off = 16; off > 0; off >>= 1) nf += __shfl_xor_sync(0xffffffffu, nf, off);
  const int64_t target = (p.rho_permille * (i + 1) + 999) / 1000;
  const int want = static_cast<int>(min(max(static_cast<int64_t>(Di + nf), target) - Di, static_cast<int64_t>(ncand)));
  if (want > p.cap) {
    if (lane == 0) {
      set_error(err, kErrDeviceCheck);
      counts[row] = 0;
    }
    return;
  }
  auto key_hi = [&](int t) -> uint32_t {
    return ((fbits[t >> 5] >> (t & 31)) & 1u) ? 0u : ~ordered_u32(S[t]);
  };
  // Rows of up to 32 * kCache candidates keep their keys in registers
  // (lane l holds candidates l, l + 32, ...), so the row is read once.
  constexpr int kCache = 32;
  const bool cached = ncand <= 32 * kCache;
  uint32_t kr[kCache];
  if (cached) {
#pragma unroll
    for (int j = 0; j < kCache; ++j) {
      const int t = lane + 32 * j;
      kr[j] = t < ncand ? key_hi(t) : 0xffffffffu;
    }
  }
  uint32_t prefix = 0, pmask = 0;
  int rank = want;
  if (want > 0) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int q = lane; q < 256; q += 32) hist[q] = 0u;
      __syncwarp();
      if (cached) {
#pragma unroll
        for (int j = 0; j < kCache; ++j) {
          const uint32_t k = kr[j];
          if (lane + 32 * j < ncand && (k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
        }
      } else {
        for (int t = lane; t < ncand; t += 32) {
          const uint32_t k = key_hi(t);
          if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
        }
      }
      __syncwarp();
      uint32_t loc[8], sum = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        loc[q] = hist[lane * 8 + q];
        sum += loc[q];
      }
      uint32_t incl = sum;
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const uint32_t excl = incl - sum;
      const bool mine = excl < static_cast<uint32_t>(rank) && static_cast<uint32_t>(rank) <= incl;
      const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
      uint32_t bucket = 0, below = 0;
      if (lane == src) {
        uint32_t c = excl;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (c + loc[q] >= static_cast<uint32_t>(rank)) {
            bucket = lane * 8 + q;
            below = c;
            break;
          }
          c += loc[q];
        }
      }
      bucket = __shfl_sync(0xffffffffu, bucket, src);
      below = __shfl_sync(0xffffffffu, below, src);
      prefix |= bucket << shift;
      pmask |= 255u << shift;
      rank -= static_cast<int>(below);
      __syncwarp();
    }
  }
  int32_t* out = idx + row * p.cap;
  int written = 0, ties = 0;
  // Write the chosen ids in ascending order: keys below the threshold, and
  // the first `rank` keys equal to it.
  auto emit = [&](int t, uint32_t k) {
    const bool lt = t < ncand && k < prefix;
    const bool eq = t < ncand && k == prefix;
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const int my_tie = ties + __popc(eqm & ((1u << lane) - 1u));
    const bool take = lt || (eq && my_tie < rank);
    const uint32_t tm = __ballot_sync(0xffffffffu, take);
    if (take) out[written + __popc(tm & ((1u << lane) - 1u))] = t;
    written += __popc(tm);
    ties += __popc(eqm);
  };
  if (want > 0 && cached) {
#pragma unroll
    for (int j = 0; j < kCache; ++j) {
      if (32 * j >= ncand) break;
      emit(lane + 32 * j, kr[j]);
    }
  } else if (want > 0) {
    for (int base = 0; base < ncand; base += 32) {
      const int t = base + lane;
      emit(t, t < ncand ? key_hi(t) : 0xffffffffu);
    }
  }
  if (lane == 0) counts[row] = want;
}

// Cumulative-mass selection, one CTA per (query block, query head, batch):
// the row's candidates are sorted by (forced first, descending score, lower
// block id) and taken in that order while the accumulated softmax mass (fp64,
// own segment included) is below tau.  The same kernel serves top-k when the
// lists are wanted in that visiting order (the first `want` sorted keys).
__global__ void __launch_bounds__(kSelThreads) select_tau_kernel(
    SelectParams p, const float* __restrict__ S_all, const float* __restrict__ qbar,
    const float* __restrict__ kbar_nat, const int32_t* __restrict__ inv,
    int32_t* __restrict__ counts, int32_t* __restrict__ idx, int* err) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (p.Hq / p.Hkv);
  const int spb = p.seg / p.blk;
  const int s = i / spb;
  const int ncand = s * spb;
  const int Di = i - s * spb + 1;
  const int64_t row = (static_cast<int64_t>(b) * p.Hq + h) * p.nb + i;
  if (ncand == 0) {
    if (threadIdx.x == 0) counts[row] = 0;
    return;
  }
  int n2 = 1;
  while (n2 < ncand) n2 <<= 1;
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem_raw);           // n2
  double* ev = reinterpret_cast<double*>(keys + n2);                 // n2
  float* S = reinterpret_cast<float*>(ev + n2);                      // n2
  float* q = S + n2;                                                 // D
  int* flag = reinterpret_cast<int*>(q + p.D);                       // n2
  __shared__ double red[kSelThreads / 32];
  __shared__ int sh_int[4];
  const float* srow = S_all + row * p.nb;
  for (int t = threadIdx.x; t < ncand; t += blockDim.x) S[t] = srow[t];
  const float* qsrc = qbar + row * p.D;
  for (int c = threadIdx.x; c < p.D; c += blockDim.x) q[c] = qsrc[c];
  for (int t = threadIdx.x; t < n2; t += blockDim.x) flag[t] = 0;
  if (threadIdx.x == 0) {
    sh_int[0] = 0;
    sh_int[1] = ncand;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // Forced blocks: sinks and the recent-key band that fall before the own segment.
  const int64_t s_start = static_cast<int64_t>(s) * p.seg;
  const int32_t* irow = inv + ((static_cast<int64_t>(b) * p.Hkv + hk) * p.perm_nseg + (p.perm_nseg > 1 ? s : 0)) * p.N;
  const int64_t sink_hi = min(static_cast<int64_t>(p.n_sink), s_start);
  for (int64_t pos = threadIdx.x; pos < sink_hi; pos += blockDim.x) {
    const int32_t lp = irow[pos];
    if (lp >= 0 && lp < static_cast<int64_t>(ncand) * p.blk) flag[lp / p.blk] = 1;
  }
  if (p.band > 0) {
    const int64_t band_lo = max(static_cast<int64_t>(0), static_cast<int64_t>(i) * p.blk - p.band + 1);
    for (int64_t pos = band_lo + threadIdx.x; pos < s_start; pos += blockDim.x) {
      const int32_t lp = irow[pos];
      if (lp >= 0 && lp < static_cast<int64_t>(ncand) * p.blk) flag[lp / p.blk] = 1;
    }
  }
  __syncthreads();
  int nf_local = 0;
  for (int t = threadIdx.x; t < ncand; t += blockDim.x) nf_local += flag[t];
  const int nf = static_cast<int>(block_sum_f64(static_cast<double>(nf_local), red));

  // Sort key: forced blocks first, then descending score, ties to lower pb.
  for (int t = threadIdx.x; t < n2; t += blockDim.x) {
    uint64_t key = ~0ull;
    if (t < ncand) {
      const uint32_t hi = flag[t] ? 0u : ~ordered_u32(S[t]);
      key = (static_cast<uint64_t>(hi) << 32) | static_cast<uint32_t>(t);
    }
    keys[t] = key;
  }
  __syncthreads();
  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int t = threadIdx.x; t < n2; t += blockDim.x) {
        const int txj = t ^ j;
        if (txj > t) {
          const uint64_t a = keys[t], c = keys[txj];
          const bool up = (t & k) == 0;
          if ((a > c) == up) {
            keys[t] = c;
            keys[txj] = a;
          }
        }
      }
      __syncthreads();
    }
  }

  int want;
  if (p.mode == PBS_SELECT_TOPK) {
    const int64_t target = (p.rho_permille * (i + 1) + 999) / 1000;
    const int64_t k = max(static_cast<int64_t>(Di + nf), target);
    want = static_cast<int>(min(k - Di, static_cast<int64_t>(ncand)));
  } else if (p.tau >= 1.0) {
    want = ncand;
  } else {
    // Softmax mass over (candidates + natural blocks of the own segment),
    // fp64, logits = S / (blk^2 sqrt(D)).
    const double sc = 1.0 / (static_cast<double>(p.blk) * p.blk * sqrt(static_cast<double>(p.D)));
    const float* kn = kbar_nat + (static_cast<int64_t>(b) * p.Hkv + hk) * p.nb * p.D;
    __shared__ double dlog[128];   // D_i <= seg/blk <= 128
    for (int jj = warp; jj < Di; jj += kSelThreads / 32) {
      const int j = s * spb + jj;
      float acc = 0.f;
      for (int c = lane; c < p.D; c += 32) acc = fmaf(q[c], kn[static_cast<int64_t>(j) * p.D + c], acc);
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) dlog[jj] = static_cast<double>(acc) * sc;
    }
    __syncthreads();
    double mloc = -INFINITY;
    for (int t = threadIdx.x; t < ncand; t += blockDim.x) mloc = fmax(mloc, static_cast<double>(S[t]) * sc);
    for (int jj = threadIdx.x; jj < Di; jj += blockDim.x) mloc = fmax(mloc, dlog[jj]);
    const double m = block_max_f64(mloc, red);
    double dl = 0.0;
    for (int jj = threadIdx.x; jj < Di; jj += blockDim.x) dl += exp(dlog[jj] - m);
    const double ediag = block_sum_f64(dl, red);
    // e in sorted order
    double cl = 0.0;
    for (int t = threadIdx.x; t < ncand; t += blockDim.x) {
      const uint32_t pb = static_cast<uint32_t>(keys[t] & 0xffffffffu);
      const double e = exp(static_cast<double>(S[pb]) * sc - m);
      ev[t] = e;
      cl += e;
    }
    const double Z = ediag + block_sum_f64(cl, red);
    const double goal = p.tau * Z;
    // exclusive prefix over the sorted order: each thread owns a contiguous chunk
    const int per = (ncand + kSelThreads - 1) / kSelThreads;
    const int t0 = threadIdx.x * per, t1 = min(ncand, t0 + per);
    double local = 0.0;
    for (int t = t0; t < t1; ++t) local += ev[t];
    __shared__ double part[kSelThreads];
    part[threadIdx.x] = local;
    __syncthreads();
    if (threadIdx.x == 0) {
      double run = ediag;
      for (int u = 0; u < kSelThreads; ++u) {
        const double x = part[u];
        part[u] = run;
        run += x;
      }
    }
    __syncthreads();
    double c = part[threadIdx.x];
    for (int t = t0; t < t1; ++t) {
      if (t >= nf && c >= goal) {
        atomicMin(&sh_int[1], t);
        break;
      }
      c += ev[t];
    }
    __syncthreads();
    want = max(nf, sh_int[1]);
  }

  if (p.score_order) {
    // Visiting order: the chosen blocks are the first `want` of the sorted
    // keys (forced first, then descending score, ties to the lower block).
    if (want > p.cap) {
      if (threadIdx.x == 0) {
        set_error(err, kErrDeviceCheck);
        counts[row] = 0;
      }
      return;
    }
    int32_t* out = idx + row * p.cap;
    for (int t = threadIdx.x; t < want; t += blockDim.x) out[t] = static_cast<int32_t>(keys[t] & 0xffffffffu);
    if (threadIdx.x == 0) counts[row] = want;
    return;
  }
  // Mark the chosen blocks and write them in ascending order.
  for (int t = threadIdx.x; t < n2; t += blockDim.x) flag[t] = 0;
  __syncthreads();
  for (int t = threadIdx.x; t < want; t += blockDim.x)
    flag[static_cast<uint32_t>(keys[t] & 0xffffffffu)] = 1;
  __syncthreads();
  const int per = (ncand + kSelThreads - 1) / kSelThreads;
  const int t0 = threadIdx.x * per, t1 = min(ncand, t0 + per);
  int cnt = 0;
  for (int t = t0; t < t1; ++t) cnt += flag[t];
  __shared__ int offs[kSelThreads];
  offs[threadIdx.x] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int u = 0; u < kSelThreads; ++u) {
      const int x = offs[u];
      offs[u] = run;
      run += x;
    }
  }
  __syncthreads();
  if (want > p.cap) {
    if (threadIdx.x == 0) {
      set_error(err, kErrDeviceCheck);
      counts[row] = 0;
    }
    return;
  }
  int o = offs[threadIdx.x];
  int32_t* out = idx + row * p.cap;
  for (int t = t0; t < t1; ++t)
    if (flag[t]) out[o++] = t;
  if (threadIdx.x == 0) counts[row] = want;
}

}  // namespace

cudaError_t launch_pool_query_blocks(const TensorDesc& Q, int blk, const int32_t* qperm, int seg, int* err,
                                     float* qbar, cudaStream_t s) {
  dim3 grid(static_cast<unsigned>(Q.N / blk), static_cast<unsigned>(Q.H), static_cast<unsigned>(Q.B));
  pool_query_blocks_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(Q.ptr), Q.sB,
                                                 Q.sH, Q.sN, static_cast<int>(Q.D), blk, qperm, Q.N, seg, err,
                                                 qbar);
  return cudaGetLastError();
}

cudaError_t launch_pool_key_blocks(const TensorDesc& K, const int32_t* perm, int perm_nseg, int blk,
                                   int seg, bool natural, float* kbar_perm, float* kbar_nat, int32_t* inv,
                                   int* err, cudaStream_t s) {
  dim3 grid(static_cast<unsigned>(K.N / blk), static_cast<unsigned>(K.H), static_cast<unsigned>(K.B));
  const int64_t nb = K.N / blk;
  for (int q = 0; q < perm_nseg; ++q) {      // one launch per query segment's permutation
    pool_key_blocks_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(K.ptr), K.sB, K.sH, K.sN,
                                                 K.N, static_cast<int>(K.D), blk, seg, perm + q * K.N,
                                                 perm_nseg * K.N, (natural && q == 0) ? 1 : 0,
                                                 kbar_perm + q * nb * K.D, perm_nseg * nb, kbar_nat,
                                                 inv + q * K.N, err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_select_blocks(const SelectParams& p, const float* qbar, const float* kbar_perm,
                                 const float* kbar_nat, const int32_t* inv, float* scores, int32_t* counts,
                                 int32_t* idx, int* err, cudaStream_t s) {
  cudaError_t e;
  if (p.perm_nseg > 1) {
    const int64_t rows = static_cast<int64_t>(p.B) * p.Hq * p.nb;
    block_scores_seg_kernel<<<static_cast<unsigned>((rows + kSegScoreWarps - 1) / kSegScoreWarps),
                              kSegScoreWarps * 32, 0, s>>>(p, qbar, kbar_perm, scores);
  } else {
    const int tiles = (p.nb + kTile - 1) / kTile;
    dim3 g1(static_cast<unsigned>(tiles), static_cast<unsigned>(tiles), static_cast<unsigned>(p.B * p.Hq));
    block_scores_kernel<<<g1, 256, 0, s>>>(p, qbar, kbar_perm, scores);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (p.mode == PBS_SELECT_TOPK && !p.score_order) {
    const size_t smem = static_cast<size_t>(kWarpsPerCta) * (p.nb / 32 + 1) * 4;
    e = cudaFuncSetAttribute(select_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int64_t rows = static_cast<int64_t>(p.B) * p.Hq * p.nb;
    select_topk_kernel<<<static_cast<unsigned>((rows + kWarpsPerCta - 1) / kWarpsPerCta), kWarpsPerCta * 32, smem, s>>>(
        p, scores, inv, counts, idx, err);
    return cudaGetLastError();
  }
  int n2 = 1;
  while (n2 < p.nb) n2 <<= 1;
  const size_t smem = static_cast<size_t>(n2) * (8 + 8 + 4 + 4) + static_cast<size_t>(p.D) * 4;
  e = cudaFuncSetAttribute(select_tau_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 g2(static_cast<unsigned>(p.nb), static_cast<unsigned>(p.Hq), static_cast<unsigned>(p.B));
  select_tau_kernel<<<g2, kSelThreads, smem, s>>>(p, scores, qbar, kbar_nat, inv, counts, idx, err);
  return cudaGetLastError();
}

}  // namespace pbs
