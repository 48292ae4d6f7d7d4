// pbs_permute kernels: proxy-query pooling, key scoring and the per-segment
// stable descending sort.
//
// "Sparser Block-Sparse Attention via Token Permutation", Technical Summary:
//   2. Segmented Permutation for Causality -- permute only inside fixed-size
//      segments, keep segment order;
//   3. Global-Importance-Based Key Permutation -- score keys with the last
//      block of queries (mean-pooled scores) and sort each segment by
//      descending importance.
// The pooled query is kept as an unscaled fp32 sum; the sort order is
// invariant to the positive pooling divisor and softmax scale.
#include "pbs_common.cuh"
#include "pbs_internal.h"

namespace pbs {
namespace {

// qhat[b, hkv, :] = sum of the last `blk` rows of the G query heads of the
// group.  One CTA per (hkv, b); thread = (16-byte column chunk, row lane).
__global__ void __launch_bounds__(256) pool_proxy_query_kernel(
    const __nv_bfloat16* __restrict__ Q, int64_t sB, int64_t sH, int64_t sN, int64_t N, int D,
    int G, int blk, float* __restrict__ qhat) {
  const int hkv = blockIdx.x, b = blockIdx.y, Hkv = gridDim.x;
  const int nchunk = D / 8;
  const int chunk = threadIdx.x % nchunk;
  const int lanes = blockDim.x / nchunk;
  const int rl = threadIdx.x / nchunk;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const int rows = G * blk;
  for (int r = rl; r < rows; r += lanes) {
    const int h = hkv * G + r / blk;
    const int64_t n = N - blk + (r % blk);
    const uint4 v = *reinterpret_cast<const uint4*>(Q + b * sB + h * sH + n * sN + chunk * 8);
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
  if (threadIdx.x < nchunk) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float t = 0.f;
      for (int l = 0; l < lanes; ++l) t += red[(l * nchunk + threadIdx.x) * 8 + e];
      qhat[(static_cast<int64_t>(b) * Hkv + hkv) * D + threadIdx.x * 8 + e] = t;
    }
  }
}

// One CTA per (segment, hkv, b).  Scores every key of the segment with one
// fp32 dot product against qhat (lanes of a row group read 16 bytes each,
// a row is one coalesced 128/256-byte read), packs (descending score,
// ascending position) into one 64-bit key and bitonic-sorts the keys in
// shared memory.  Sorting unique composite keys is a total order, so the
// result equals a stable descending sort by score.
__global__ void __launch_bounds__(1024) score_sort_kernel(
    const __nv_bfloat16* __restrict__ K, int64_t sB, int64_t sH, int64_t sN, int64_t N, int D,
    int seg, int n_sink, const float* __restrict__ qhat, int32_t* __restrict__ perm) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int t = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z, Hkv = gridDim.y;
  const int64_t lo = static_cast<int64_t>(t) * seg;
  const int len = static_cast<int>(min(static_cast<int64_t>(seg), N - lo));
  int n2 = 1;
  while (n2 < len) n2 <<= 1;
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem_raw);
  float* q = reinterpret_cast<float*>(keys + n2);
  for (int c = threadIdx.x; c < D; c += blockDim.x)
    q[c] = qhat[(static_cast<int64_t>(b) * Hkv + hkv) * D + c];
  __syncthreads();

  const int lanes_per_row = D / 8;           // 16 (D=128) or 8 (D=64)
  const int rows_per_warp = 32 / lanes_per_row;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  const int sub = lane / lanes_per_row, cl = lane % lanes_per_row;
  const __nv_bfloat16* base = K + b * sB + hkv * sH;
  float qv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) qv[e] = q[cl * 8 + e];
  for (int r0 = warp * rows_per_warp; r0 < len; r0 += nwarp * rows_per_warp) {
    const int r = r0 + sub;
    float acc = 0.f;
    if (r < len) {
      const uint4 v = *reinterpret_cast<const uint4*>(base + (lo + r) * sN + cl * 8);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(p[e]);
        acc = fmaf(f.x, qv[2 * e], acc);
        acc = fmaf(f.y, qv[2 * e + 1], acc);
      }
    }
    for (int off = lanes_per_row >> 1; off > 0; off >>= 1)
      acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (r < len && cl == 0) {
      const float s = (lo + r < n_sink) ? __int_as_float(0x7f800000) : acc;
      keys[r] = (static_cast<uint64_t>(~ordered_u32(s)) << 32) | static_cast<uint32_t>(r);
    }
  }
  for (int r = len + threadIdx.x; r < n2; r += blockDim.x) keys[r] = ~0ull;
  __syncthreads();

  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t a = keys[i], c = keys[ixj];
          const bool up = (i & k) == 0;
          if ((a > c) == up) {
            keys[i] = c;
            keys[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  int32_t* out = perm + (static_cast<int64_t>(b) * Hkv + hkv) * N + lo;
  for (int r = threadIdx.x; r < len; r += blockDim.x)
    out[r] = static_cast<int32_t>(lo + static_cast<uint32_t>(keys[r] & 0xffffffffu));
}

}  // namespace

cudaError_t launch_pool_proxy_query(const TensorDesc& Q, int Hkv, int blk, float* qhat,
                                    cudaStream_t s) {
  dim3 grid(Hkv, static_cast<unsigned>(Q.B));
  pool_proxy_query_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(Q.ptr), Q.sB,
                                                Q.sH, Q.sN, Q.N, static_cast<int>(Q.D),
                                                static_cast<int>(Q.H / Hkv), blk, qhat);
  return cudaGetLastError();
}

cudaError_t launch_score_sort(const TensorDesc& K, int seg, int n_sink, const float* qhat,
                              int32_t* perm, int* /*err*/, cudaStream_t s) {
  const int64_t nseg = (K.N + seg - 1) / seg;
  int n2 = 1;
  while (n2 < seg) n2 <<= 1;
  const size_t smem = static_cast<size_t>(n2) * 8 + K.D * 4;
  cudaError_t e = cudaFuncSetAttribute(score_sort_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(nseg), static_cast<unsigned>(K.H), static_cast<unsigned>(K.B));
  score_sort_kernel<<<grid, 1024, smem, s>>>(static_cast<const __nv_bfloat16*>(K.ptr), K.sB,
                                              K.sH, K.sN, K.N, static_cast<int>(K.D), seg, n_sink,
                                              qhat, perm);
  return cudaGetLastError();
}

}  // namespace pbs
