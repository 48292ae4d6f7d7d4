// pbs_permute_segmented kernels: one key permutation per query segment.
//
// "S2O: Early Stopping for Sparse Attention via Online Permutation",
// Technical Summary, 1. Online Permutation via Index-Driven Loading
// (Historical KV Permutation): each query segment ranks the keys that come
// before it by one query standing for the whole segment, and that ranking
// is the order in which the segment loads them.
//
// Here the representative query of segment s is the sum of its query rows
// over the KV head's group; for each key segment j < s the keys of j are
// sorted by descending score against it (ties in ascending position), and
// key segments j >= s keep their natural order (they are not s's history).
// Sums and dot products are taken in fp64: a segment's pooled query grows
// with the segment length, and fp64 keeps lattice-valued (bf16) inputs
// exact, so the order does not depend on the summation order.
#include "pbs_common.cuh"
#include "pbs_internal.h"

namespace pbs {
namespace {

// qs[b, hkv, s, :] (fp64) = sum over the rows of segment s of every query
// head of hkv's group.  One CTA per (s, hkv, b).
__global__ void __launch_bounds__(256) pool_segment_queries_kernel(
    const __nv_bfloat16* __restrict__ Q, int64_t sB, int64_t sH, int64_t sN, int64_t N, int D,
    int G, int seg, double* __restrict__ qs) {
  const int s = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;
  const int nseg = gridDim.x, Hkv = gridDim.y;
  const int nchunk = D / 8;
  const int chunk = threadIdx.x % nchunk;
  const int lanes = blockDim.x / nchunk;
  const int rl = threadIdx.x / nchunk;
  const int64_t lo = static_cast<int64_t>(s) * seg;
  const int len = static_cast<int>(min(static_cast<int64_t>(seg), N - lo));
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const int rows = G * len;
  for (int r = rl; r < rows; r += lanes) {
    const int h = hkv * G + r / len;
    const int64_t n = lo + (r % len);
    const uint4 v = *reinterpret_cast<const uint4*>(Q + b * sB + h * sH + n * sN + chunk * 8);
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(p[e]);
      acc[2 * e] += static_cast<double>(f.x);
      acc[2 * e + 1] += static_cast<double>(f.y);
    }
  }
  __shared__ double red[256 * 8];
#pragma unroll
  for (int e = 0; e < 8; ++e) red[threadIdx.x * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < nchunk) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      double t = 0.0;
      for (int l = 0; l < lanes; ++l) t += red[(l * nchunk + threadIdx.x) * 8 + e];
      qs[((static_cast<int64_t>(b) * Hkv + hkv) * nseg + s) * D + threadIdx.x * 8 + e] = t;
    }
  }
}

// One CTA per (key segment j, query segment s, b * Hkv + hkv).  For j < s:
// fp64 scores of j's keys against s's representative query, then a bitonic
// sort of (descending score, ascending position) pairs in shared memory.
// For j >= s: the natural order.
__global__ void __launch_bounds__(1024) score_sort_seg_kernel(
    const __nv_bfloat16* __restrict__ K, int64_t sB, int64_t sH, int64_t sN, int64_t N, int D,
    int seg, int n_sink, int Hkv, const double* __restrict__ qs, int32_t* __restrict__ perm) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int j = blockIdx.x, s = blockIdx.y, nseg = gridDim.y;
  const int hkv = blockIdx.z % Hkv, b = blockIdx.z / Hkv;
  const int64_t lo = static_cast<int64_t>(j) * seg;
  const int len = static_cast<int>(min(static_cast<int64_t>(seg), N - lo));
  int32_t* out = perm + ((static_cast<int64_t>(b) * Hkv + hkv) * nseg + s) * N + lo;
  if (j >= s) {
    for (int r = threadIdx.x; r < len; r += blockDim.x) out[r] = static_cast<int32_t>(lo + r);
    return;
  }
  int n2 = 1;
  while (n2 < len) n2 <<= 1;
  uint64_t* key = reinterpret_cast<uint64_t*>(smem_raw);
  uint32_t* idx = reinterpret_cast<uint32_t*>(key + n2);
  double* q = reinterpret_cast<double*>(smem_raw + static_cast<size_t>(n2) * 12);   // n2 even: 8-byte aligned
  for (int c = threadIdx.x; c < D; c += blockDim.x)
    q[c] = qs[((static_cast<int64_t>(b) * Hkv + hkv) * nseg + s) * D + c];
  __syncthreads();

  const int lanes_per_row = D / 8;
  const int rows_per_warp = 32 / lanes_per_row;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  const int sub = lane / lanes_per_row, cl = lane % lanes_per_row;
  const __nv_bfloat16* base = K + b * sB + hkv * sH;
  double qv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) qv[e] = q[cl * 8 + e];
  for (int r0 = warp * rows_per_warp; r0 < len; r0 += nwarp * rows_per_warp) {
    const int r = r0 + sub;
    double acc = 0.0;
    if (r < len) {
      const uint4 v = *reinterpret_cast<const uint4*>(base + (lo + r) * sN + cl * 8);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p[e]);
        acc = fma(static_cast<double>(f.x), qv[2 * e], acc);
        acc = fma(static_cast<double>(f.y), qv[2 * e + 1], acc);
      }
    }
    for (int off = lanes_per_row >> 1; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (r < len && cl == 0) {
      const double sc = (lo + r < n_sink) ? __longlong_as_double(0x7ff0000000000000ll) : acc;
      key[r] = ~ordered_u64(sc);                 // ascending key = descending score
      idx[r] = static_cast<uint32_t>(r);
    }
  }
  for (int r = len + threadIdx.x; r < n2; r += blockDim.x) {
    key[r] = ~0ull;
    idx[r] = 0xffffffffu;
  }
  __syncthreads();
  // lexicographic on (key, idx): equal scores keep ascending position
  cta_bitonic_sort(key, idx, n2);
  for (int r = threadIdx.x; r < len; r += blockDim.x) out[r] = static_cast<int32_t>(lo + idx[r]);
}

}  // namespace

cudaError_t launch_permute_segmented(const TensorDesc& Q, const TensorDesc& K, int seg, int n_sink,
                                     double* qs, int32_t* perm, cudaStream_t s) {
  const int nseg = static_cast<int>((K.N + seg - 1) / seg);
  const int Hkv = static_cast<int>(K.H);
  dim3 g1(static_cast<unsigned>(nseg), static_cast<unsigned>(Hkv), static_cast<unsigned>(Q.B));
  pool_segment_queries_kernel<<<g1, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(Q.ptr), Q.sB, Q.sH,
                                                  Q.sN, Q.N, static_cast<int>(Q.D),
                                                  static_cast<int>(Q.H / K.H), seg, qs);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int n2 = 1;
  while (n2 < seg) n2 <<= 1;
  const size_t smem = static_cast<size_t>(n2) * 12 + static_cast<size_t>(K.D) * 8;
  e = cudaFuncSetAttribute(score_sort_seg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 g2(static_cast<unsigned>(nseg), static_cast<unsigned>(nseg), static_cast<unsigned>(K.B * K.H));
  score_sort_seg_kernel<<<g2, 1024, smem, s>>>(static_cast<const __nv_bfloat16*>(K.ptr), K.sB, K.sH, K.sN,
                                                K.N, static_cast<int>(K.D), seg, n_sink, Hkv, qs, perm);
  return cudaGetLastError();
}

}  // namespace pbs
