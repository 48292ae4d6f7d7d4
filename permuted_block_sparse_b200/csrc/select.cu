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

namespace pbs {
namespace {

// Sum of `blk` consecutive rows: one CTA per (block, head, batch); thread =
// (16-byte chunk, row lane); fp32.
__global__ void __launch_bounds__(256) pool_query_blocks_kernel(
    const __nv_bfloat16* __restrict__ Q, int64_t sB, int64_t sH, int64_t sN, int D, int blk,
    float* __restrict__ qbar) {
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nb = gridDim.x, H = gridDim.y;
  const int nchunk = D / 8, chunk = threadIdx.x % nchunk;
  const int lanes = blockDim.x / nchunk, rl = threadIdx.x / nchunk;
  const __nv_bfloat16* base = Q + b * sB + h * sH + static_cast<int64_t>(i) * blk * sN;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int r = rl; r < blk; r += lanes) {
    const uint4 v = *reinterpret_cast<const uint4*>(base + r * sN + chunk * 8);
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
__global__ void __launch_bounds__(256) pool_key_blocks_kernel(
    const __nv_bfloat16* __restrict__ K, int64_t sB, int64_t sH, int64_t sN, int64_t N, int D,
    int blk, int seg, const int32_t* __restrict__ perm, int natural, float* __restrict__ kbar_perm,
    float* __restrict__ kbar_nat, int32_t* __restrict__ inv, int* err) {
  const int pb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nb = gridDim.x, H = gridDim.y;
  __shared__ int32_t rows[256];
  __shared__ float red[256 * 8];
  const int64_t p0 = static_cast<int64_t>(pb) * blk;
  const int64_t seg_lo = (p0 / seg) * seg;
  const int64_t seg_hi = min(seg_lo + seg, N);
  const int32_t* prow = perm + (static_cast<int64_t>(b) * H + h) * N;
  int32_t* irow = inv + (static_cast<int64_t>(b) * H + h) * N;
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
    float* out = pass == 0 ? kbar_perm : kbar_nat;
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
      const int ch = c / 8, e = c % 8;
      float t = 0.f;
      for (int l = 0; l < lanes; ++l) t += red[(l * nchunk + ch) * 8 + e];
      out[((static_cast<int64_t>(b) * H + h) * nb + pb) * D + c] = t;
    }
    __syncthreads();
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

// One CTA per (query block i, query head, batch).
__global__ void __launch_bounds__(kSelThreads) select_blocks_kernel(
    SelectParams p, const float* __restrict__ qbar, const float* __restrict__ kbar_perm,
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
  double* ev = reinterpret_cast<double*>(keys + n2);                 // n2 (tau)
  float* S = reinterpret_cast<float*>(ev + n2);                      // n2
  float* q = S + n2;                                                 // D
  int* flag = reinterpret_cast<int*>(q + p.D);                       // n2
  __shared__ double red[kSelThreads / 32];
  __shared__ int sh_int[4];

  const float* qsrc = qbar + row * p.D;
  for (int c = threadIdx.x; c < p.D; c += blockDim.x) q[c] = qsrc[c];
  for (int t = threadIdx.x; t < n2; t += blockDim.x) flag[t] = 0;
  if (threadIdx.x == 0) {
    sh_int[0] = 0;
    sh_int[1] = ncand;
  }
  __syncthreads();

  // Exact block scores (lattice inputs): one warp per candidate.
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float* kb = kbar_perm + (static_cast<int64_t>(b) * p.Hkv + hk) * p.nb * p.D;
  for (int pb = warp; pb < ncand; pb += kSelThreads / 32) {
    float acc = 0.f;
    for (int c = lane; c < p.D; c += 32) acc = fmaf(q[c], kb[static_cast<int64_t>(pb) * p.D + c], acc);
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) S[pb] = acc;
  }
  // Forced blocks: sinks and the recent-key band that fall before the own segment.
  const int64_t s_start = static_cast<int64_t>(s) * p.seg;
  const int32_t* irow = inv + (static_cast<int64_t>(b) * p.Hkv + hk) * p.N;
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

cudaError_t launch_pool_query_blocks(const TensorDesc& Q, int blk, float* qbar, cudaStream_t s) {
  dim3 grid(static_cast<unsigned>(Q.N / blk), static_cast<unsigned>(Q.H), static_cast<unsigned>(Q.B));
  pool_query_blocks_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(Q.ptr), Q.sB,
                                                 Q.sH, Q.sN, static_cast<int>(Q.D), blk, qbar);
  return cudaGetLastError();
}

cudaError_t launch_pool_key_blocks(const TensorDesc& K, const int32_t* perm, int blk, int seg,
                                   bool natural, float* kbar_perm, float* kbar_nat, int32_t* inv,
                                   int* err, cudaStream_t s) {
  dim3 grid(static_cast<unsigned>(K.N / blk), static_cast<unsigned>(K.H), static_cast<unsigned>(K.B));
  pool_key_blocks_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(K.ptr), K.sB,
                                               K.sH, K.sN, K.N, static_cast<int>(K.D), blk, seg,
                                               perm, natural ? 1 : 0, kbar_perm, kbar_nat, inv, err);
  return cudaGetLastError();
}

size_t select_smem_bytes(int nb, int D) {
  int n2 = 1;
  while (n2 < nb) n2 <<= 1;
  return static_cast<size_t>(n2) * (8 + 8 + 4 + 4) + static_cast<size_t>(D) * 4;
}

cudaError_t launch_select_blocks(const SelectParams& p, const float* qbar, const float* kbar_perm,
                                 const float* kbar_nat, const int32_t* inv, int32_t* counts,
                                 int32_t* idx, int* err, cudaStream_t s) {
  const size_t smem = select_smem_bytes(p.nb, p.D);
  cudaError_t e = cudaFuncSetAttribute(select_blocks_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(p.nb), static_cast<unsigned>(p.Hq), static_cast<unsigned>(p.B));
  select_blocks_kernel<<<grid, kSelThreads, smem, s>>>(p, qbar, kbar_perm, kbar_nat, inv, counts,
                                                       idx, err);
  return cudaGetLastError();
}

}  // namespace pbs
