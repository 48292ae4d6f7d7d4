// pbs_select mode PBS_SELECT_SAMPLE: a SampleAttention-style selector over
// natural key blocks.
//
// "SampleAttention" (MLSys 2025 talk), Technical Deep Dive:
//   Stage 1, Trunk Sampling -- estimate attention scores from queries sampled
//     in chunks (trunks) across the sequence;
//   Stage 2, Score-Based Filtering -- keep the key-column and slash patterns
//     needed to preserve the target attention mass (CIA), the two families
//     filtered separately ("decoupled"), and turn them into a block mask.
// Here the trunks are the last query block of every segment.  Per query
// head, their softmax probabilities are summed per key column and per slash
// offset q - k (fp64 accumulation); each family keeps its highest entries up
// to and including the one at which the accumulated score reaches alpha of
// its total (ties to the lower index); query block i lists every key block
// of earlier segments that holds a kept column, or a key q - d for one of
// its queries q and a kept offset d.
#include <math.h>

#include "pbs_common.cuh"
#include "pbs_internal.h"

namespace pbs {
namespace {

constexpr int kSampleWarps = 8;

// Stage 1.  One warp per (sampled row, hq, b); lanes own keys.  The raw q.k
// of bf16 inputs is accumulated in fp32; the probabilities are
// 2^(x - m) / l with x the scaled logit in log2 units.
__global__ void __launch_bounds__(kSampleWarps * 32) sample_scores_kernel(
    const __nv_bfloat16* __restrict__ Q, int64_t qsB, int64_t qsH, int64_t qsN,
    const __nv_bfloat16* __restrict__ K, int64_t ksB, int64_t ksH, int64_t ksN, int64_t N, int D, int G,
    int blk, int seg, float scale_log2, double* __restrict__ col, double* __restrict__ sl) {
  __shared__ float qs[kSampleWarps][128];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rrow = blockIdx.x * kSampleWarps + warp;            // sampled row index
  const int nseg = static_cast<int>((N + seg - 1) / seg);
  if (rrow >= nseg * blk) return;
  const int hq = blockIdx.y, b = blockIdx.z, Hq = gridDim.y;
  const int s = rrow / blk;
  const int64_t seg_end = min(static_cast<int64_t>(s + 1) * seg, N);
  const int64_t q = seg_end - blk + (rrow % blk);
  const __nv_bfloat16* qrow = Q + b * qsB + hq * qsH + q * qsN;
  for (int c = lane; c < D; c += 32) qs[warp][c] = __bfloat162float(qrow[c]);
  __syncwarp();
  const __nv_bfloat16* kb = K + b * ksB + (hq / G) * ksH;
  auto logit = [&](int64_t k) -> float {
    const uint4* kr = reinterpret_cast<const uint4*>(kb + k * ksN);
    float acc = 0.f;
    for (int c = 0; c < D / 8; ++c) {
      const uint4 v = kr[c];
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p[e]);
        acc = fmaf(f.x, qs[warp][c * 8 + 2 * e], acc);
        acc = fmaf(f.y, qs[warp][c * 8 + 2 * e + 1], acc);
      }
    }
    return acc * scale_log2;
  };
  // pass 1: running max and sum per lane, then across the warp
  float m = -INFINITY, l = 0.f;
  for (int64_t k = lane; k <= q; k += 32) {
    const float x = logit(k);
    if (x > m) {
      l = l * ex2(m - x) + 1.f;
      m = x;
    } else {
      l += ex2(x - m);
    }
  }
  for (int off = 16; off > 0; off >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, off), l2 = __shfl_xor_sync(0xffffffffu, l, off);
    const float mn = fmaxf(m, m2);
    l = (m == -INFINITY ? 0.f : l * ex2(m - mn)) + (m2 == -INFINITY ? 0.f : l2 * ex2(m2 - mn));
    m = mn;
  }
  const float inv_l = 1.f / l;
  // pass 2: probabilities into the column and slash sums
  double* cb = col + (static_cast<int64_t>(b) * Hq + hq) * N;
  double* sb = sl + (static_cast<int64_t>(b) * Hq + hq) * N;
  for (int64_t k = lane; k <= q; k += 32) {
    const double p = static_cast<double>(ex2(logit(k) - m) * inv_l);
    atomicAdd(cb + k, p);
    atomicAdd(sb + (q - k), p);
  }
}

__device__ __forceinline__ uint64_t ordered_f64(double x) {
  const uint64_t u = static_cast<uint64_t>(__double_as_longlong(x));
  return (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
}

// Block-wide fp64 sum (blockDim.x = 1024).
__device__ double block_sum(double v, double* red) {
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x < 32) {
    t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
    for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    if (threadIdx.x == 0) red[32] = t;
  }
  __syncthreads();
  return red[32];
}

// Stage 2, one family.  One CTA per (family, hq, b): the largest score
// threshold whose upper set reaches alpha of the total (a bisection on the
// order-preserving 64-bit image of the scores), then the entries at the
// threshold in ascending index until the target is met.  Writes a bitmap.
__global__ void __launch_bounds__(1024) sample_cut_kernel(const double* __restrict__ col,
                                                          const double* __restrict__ sl, int64_t N,
                                                          double alpha, uint32_t* __restrict__ keep_col,
                                                          uint32_t* __restrict__ keep_sl) {
  __shared__ double red[33];
  const int fam = blockIdx.x, hq = blockIdx.y, b = blockIdx.z, Hq = gridDim.y;
  const int64_t row = static_cast<int64_t>(b) * Hq + hq;
  const double* sc = (fam == 0 ? col : sl) + row * N;
  uint32_t* keep = (fam == 0 ? keep_col : keep_sl) + row * ((N + 31) / 32);
  const int64_t words = (N + 31) / 32;
  for (int64_t w = threadIdx.x; w < words; w += blockDim.x) keep[w] = 0u;
  double loc = 0.0;
  for (int64_t k = threadIdx.x; k < N; k += blockDim.x) loc += sc[k];
  const double total = block_sum(loc, red);
  __syncthreads();
  if (alpha >= 1.0) {
    for (int64_t k = threadIdx.x; k < N; k += blockDim.x)
      if (sc[k] > 0.0) atomicOr(&keep[k >> 5], 1u << (k & 31));
    return;
  }
  const double goal = alpha * total;
  // bisection for the largest t with mass(score image >= t) >= goal
  uint64_t lo = 0, hi = ~0ull;             // invariant: mass(>= lo) >= goal
  while (lo < hi) {
    const uint64_t mid = lo + (hi - lo) / 2 + 1;
    double part = 0.0;
    for (int64_t k = threadIdx.x; k < N; k += blockDim.x)
      if (ordered_f64(sc[k]) >= mid) part += sc[k];
    const double mass = block_sum(part, red);
    if (mass >= goal) lo = mid; else hi = mid - 1;
  }
  // strictly above the threshold: always kept
  double part = 0.0;
  for (int64_t k = threadIdx.x; k < N; k += blockDim.x) {
    if (ordered_f64(sc[k]) > lo) {
      atomicOr(&keep[k >> 5], 1u << (k & 31));
      part += sc[k];
    }
  }
  const double above = block_sum(part, red);
  // at the threshold: ascending index while the accumulated score is below the goal
  if (threadIdx.x == 0) {
    double acc = above;
    for (int64_t k = 0; k < N && acc < goal; ++k) {
      if (ordered_f64(sc[k]) == lo) {
        keep[k >> 5] |= 1u << (k & 31);
        acc += sc[k];
      }
    }
  }
}

// Block lists.  One warp per (b, hq, i): mark the candidate blocks that hold
// a kept column or meet a kept slash for one of block i's queries, then write
// them in ascending order.
__global__ void __launch_bounds__(kSampleWarps * 32) sample_lists_kernel(
    SelectParams p, const uint32_t* __restrict__ keep_col, const uint32_t* __restrict__ keep_sl,
    int32_t* __restrict__ counts, int32_t* __restrict__ idx, int* err) {
  __shared__ uint32_t mark[kSampleWarps][256];                  // ncand <= 8192 blocks
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kSampleWarps + warp;
  if (row >= static_cast<int64_t>(p.B) * p.Hq * p.nb) return;
  const int i = static_cast<int>(row % p.nb);
  const int64_t bh = row / p.nb;
  const int spb = p.seg / p.blk;
  const int ncand = (i / spb) * spb;
  if (ncand == 0) {
    if (lane == 0) counts[row] = 0;
    return;
  }
  const int64_t words = (p.N + 31) / 32;
  const uint32_t* kc = keep_col + bh * words;
  const uint32_t* ks = keep_sl + bh * words;
  uint32_t* mk = mark[warp];
  const int mwords = (ncand + 31) >> 5;
  for (int w = lane; w < mwords; w += 32) mk[w] = 0u;
  __syncwarp();
  // columns: block j holds a kept key
  const int wpb = p.blk / 32;                                   // bitmap words per block
  for (int j = lane; j < ncand; j += 32) {
    uint32_t any = 0u;
    for (int w = 0; w < wpb; ++w) any |= kc[static_cast<int64_t>(j) * wpb + w];
    if (any) atomicOr(&mk[j >> 5], 1u << (j & 31));
  }
  // slashes: offset d meets keys q0 - d .. q0 + blk - 1 - d
  const int64_t q0 = static_cast<int64_t>(i) * p.blk;
  const int64_t dmax = q0 + p.blk - 1;                          // larger offsets see no key
  const int64_t dwords = dmax / 32 + 1;
  for (int64_t w = lane; w < dwords; w += 32) {
    uint32_t bits = ks[w];
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      const int64_t d = w * 32 + bit;
      if (d > dmax) break;
      const int64_t klo = q0 - d, khi = q0 + p.blk - 1 - d;
      const int64_t jlo = klo < 0 ? 0 : klo / p.blk;
      const int64_t jhi = min(khi / p.blk, static_cast<int64_t>(ncand) - 1);
      for (int64_t j = jlo; j <= jhi; ++j) atomicOr(&mk[j >> 5], 1u << (j & 31));
    }
  }
  __syncwarp();
  int total = 0;
  int32_t* out = idx + row * p.cap;
  for (int base = 0; base < mwords; base += 32) {
    const int w = base + lane;
    uint32_t u = w < mwords ? mk[w] : 0u;
    const int c = __popc(u);
    int incl = c;
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    int o = total + incl - c;
    while (u) {
      const int bit = __ffs(u) - 1;
      u &= u - 1;
      if (o < p.cap) out[o] = w * 32 + bit;
      ++o;
    }
    total += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) {
    if (total > p.cap) {
      set_error(err, kErrDeviceCheck);
      counts[row] = 0;
    } else {
      counts[row] = total;
    }
  }
}

}  // namespace

cudaError_t launch_select_sample(const SelectParams& p, const TensorDesc& Q, const TensorDesc& K,
                                 float scale_log2, double* col, double* sl, uint32_t* keep_col,
                                 uint32_t* keep_sl, int32_t* counts, int32_t* idx, int* err, cudaStream_t s) {
  const size_t nsc = static_cast<size_t>(p.B) * p.Hq * p.N;
  cudaError_t e = cudaMemsetAsync(col, 0, nsc * sizeof(double), s);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(sl, 0, nsc * sizeof(double), s);
  if (e != cudaSuccess) return e;
  const int nseg = static_cast<int>((p.N + p.seg - 1) / p.seg);
  const int nrows = nseg * p.blk;
  dim3 g1(static_cast<unsigned>((nrows + kSampleWarps - 1) / kSampleWarps), static_cast<unsigned>(p.Hq),
          static_cast<unsigned>(p.B));
  sample_scores_kernel<<<g1, kSampleWarps * 32, 0, s>>>(
      static_cast<const __nv_bfloat16*>(Q.ptr), Q.sB, Q.sH, Q.sN, static_cast<const __nv_bfloat16*>(K.ptr),
      K.sB, K.sH, K.sN, p.N, p.D, p.Hq / p.Hkv, p.blk, p.seg, scale_log2, col, sl);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(2, static_cast<unsigned>(p.Hq), static_cast<unsigned>(p.B));
  sample_cut_kernel<<<g2, 1024, 0, s>>>(col, sl, p.N, p.tau, keep_col, keep_sl);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t rows = static_cast<int64_t>(p.B) * p.Hq * p.nb;
  sample_lists_kernel<<<static_cast<unsigned>((rows + kSampleWarps - 1) / kSampleWarps), kSampleWarps * 32, 0,
                        s>>>(p, keep_col, keep_sl, counts, idx, err);
  return cudaGetLastError();
}

}  // namespace pbs
