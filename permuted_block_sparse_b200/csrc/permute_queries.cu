// pbs_permute_queries kernels: S2O's query permutation.
//
// "S2O: Early Stopping for Sparse Attention via Online Permutation",
// Technical Summary, 1. Online Permutation via Index-Driven Loading (Query
// Permutation): queries are reordered inside their segment by their score
// against a guide vector shared by the KV head, so that query blocks group
// queries that attend alike.  The guide vector is read here as the sum of
// every key row of the KV head; a query's score q . g is then the sum of its
// logits over all keys, largest for the queries that attend broadly.  Within
// each (batch, query head, segment) the queries are sorted by descending
// score, equal scores by ascending position; segment order is kept.
//
// Sums and dot products are fp64 with a fixed summation order: the guide
// vector grows with N, and fp64 keeps lattice-valued (bf16) inputs exact, so
// the order does not depend on how the work is split.
#include "pbs_common.cuh"
#include "pbs_internal.h"

namespace pbs {
namespace {

constexpr int kGuideRows = 2048;   // key rows per partial sum

// partial[b, hkv, c, :] = sum of key rows [c * kGuideRows, (c + 1) * kGuideRows)
// of (b, hkv), fp64.  One CTA per (chunk c, hkv, b); thread = (16-byte chunk
// of the row, row lane); each thread sums its rows in order, then the lanes
// are added in lane order.
__global__ void __launch_bounds__(256) guide_partial_kernel(const __nv_bfloat16* __restrict__ K, int64_t sB,
                                                             int64_t sH, int64_t sN, int64_t N, int D,
                                                             double* __restrict__ partial) {
  const int c = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;
  const int nchunk = gridDim.x, Hkv = gridDim.y;
  const int ncol = D / 8, col = threadIdx.x % ncol;
  const int lanes = blockDim.x / ncol, rl = threadIdx.x / ncol;
  const int64_t lo = static_cast<int64_t>(c) * kGuideRows;
  const int64_t hi = min(lo + kGuideRows, N);
  const __nv_bfloat16* base = K + b * sB + hkv * sH;
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (rl < lanes) {
    for (int64_t n = lo + rl; n < hi; n += lanes) {
      const uint4 v = *reinterpret_cast<const uint4*>(base + n * sN + col * 8);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p[e]);
        acc[2 * e] += static_cast<double>(f.x);
        acc[2 * e + 1] += static_cast<double>(f.y);
      }
    }
  }
  __shared__ double red[256 * 8];
#pragma unroll
  for (int e = 0; e < 8; ++e) red[threadIdx.x * 8 + e] = acc[e];
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    const int cc = d / 8, e = d % 8;
    double t = 0.0;
    for (int l = 0; l < lanes; ++l) t += red[(l * ncol + cc) * 8 + e];
    partial[((static_cast<int64_t>(b) * Hkv + hkv) * nchunk + c) * D + d] = t;
  }
}

// g[b, hkv, :] = the partial sums added in chunk order.  One CTA per (hkv, b).
__global__ void guide_final_kernel(const double* __restrict__ partial, int nchunk, int D, double* __restrict__ g) {
  const int hkv = blockIdx.x, b = blockIdx.y, Hkv = gridDim.x;
  const double* src = partial + (static_cast<int64_t>(b) * Hkv + hkv) * nchunk * D;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    double t = 0.0;
    for (int c = 0; c < nchunk; ++c) t += src[static_cast<int64_t>(c) * D + d];
    g[(static_cast<int64_t>(b) * Hkv + hkv) * D + d] = t;
  }
}

// One CTA per (segment s, query head hq, b): fp64 scores q . g of the
// segment's queries, then a bitonic sort of (descending score, ascending
// position) in shared memory; qperm[b, hq, lo + p] = lo + (p-th position).
__global__ void __launch_bounds__(1024) query_sort_kernel(const __nv_bfloat16* __restrict__ Q, int64_t sB,
                                                          int64_t sH, int64_t sN, int64_t N, int D, int seg,
                                                          int G, int Hkv, const double* __restrict__ g,
                                                          int32_t* __restrict__ qperm) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int s = blockIdx.x, hq = blockIdx.y, b = blockIdx.z, Hq = gridDim.y;
  const int hkv = hq / G;
  const int64_t lo = static_cast<int64_t>(s) * seg;
  const int len = static_cast<int>(min(static_cast<int64_t>(seg), N - lo));
  int n2 = 1;
  while (n2 < len) n2 <<= 1;
  uint64_t* key = reinterpret_cast<uint64_t*>(smem_raw);
  uint32_t* idx = reinterpret_cast<uint32_t*>(key + n2);
  double* gv = reinterpret_cast<double*>(smem_raw + static_cast<size_t>(n2) * 12);   // n2 even: 8-byte aligned
  for (int c = threadIdx.x; c < D; c += blockDim.x) gv[c] = g[(static_cast<int64_t>(b) * Hkv + hkv) * D + c];
  __syncthreads();
  const int lanes_per_row = D / 8;
  const int rows_per_warp = 32 / lanes_per_row;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  const int sub = lane / lanes_per_row, cl = lane % lanes_per_row;
  const __nv_bfloat16* base = Q + b * sB + hq * sH;
  double gw[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) gw[e] = gv[cl * 8 + e];
  for (int r0 = warp * rows_per_warp; r0 < len; r0 += nwarp * rows_per_warp) {
    const int r = r0 + sub;
    double acc = 0.0;
    if (r < len) {
      const uint4 v = *reinterpret_cast<const uint4*>(base + (lo + r) * sN + cl * 8);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p[e]);
        acc = fma(static_cast<double>(f.x), gw[2 * e], acc);
        acc = fma(static_cast<double>(f.y), gw[2 * e + 1], acc);
      }
    }
    for (int off = lanes_per_row >> 1; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (r < len && cl == 0) {
      key[r] = ~ordered_u64(acc);                // ascending key = descending score
      idx[r] = static_cast<uint32_t>(r);
    }
  }
  for (int r = len + threadIdx.x; r < n2; r += blockDim.x) {
    key[r] = ~0ull;
    idx[r] = 0xffffffffu;
  }
  __syncthreads();
  cta_bitonic_sort(key, idx, n2);
  int32_t* out = qperm + (static_cast<int64_t>(b) * Hq + hq) * N + lo;
  for (int r = threadIdx.x; r < len; r += blockDim.x) out[r] = static_cast<int32_t>(lo + idx[r]);
}

}  // namespace

size_t permute_queries_ws_bytes(const TensorDesc& K) {
  const int64_t nchunk = (K.N + kGuideRows - 1) / kGuideRows;
  return static_cast<size_t>(K.B * K.H * (nchunk + 1) * K.D) * 8;
}

cudaError_t launch_permute_queries(const TensorDesc& Q, const TensorDesc& K, int seg, double* ws, int32_t* qperm,
                                   cudaStream_t s) {
  const int nchunk = static_cast<int>((K.N + kGuideRows - 1) / kGuideRows);
  const int D = static_cast<int>(K.D);
  double* partial = ws;
  double* g = ws + static_cast<int64_t>(K.B * K.H) * nchunk * D;
  dim3 g1(static_cast<unsigned>(nchunk), static_cast<unsigned>(K.H), static_cast<unsigned>(K.B));
  guide_partial_kernel<<<g1, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(K.ptr), K.sB, K.sH, K.sN, K.N, D,
                                          partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  guide_final_kernel<<<dim3(static_cast<unsigned>(K.H), static_cast<unsigned>(K.B)), 128, 0, s>>>(partial, nchunk,
                                                                                                   D, g);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int n2 = 1;
  while (n2 < seg) n2 <<= 1;
  const size_t smem = static_cast<size_t>(n2) * 12 + static_cast<size_t>(D) * 8;
  e = cudaFuncSetAttribute(query_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int nseg = static_cast<int>((Q.N + seg - 1) / seg);
  dim3 g3(static_cast<unsigned>(nseg), static_cast<unsigned>(Q.H), static_cast<unsigned>(Q.B));
  query_sort_kernel<<<g3, 1024, smem, s>>>(static_cast<const __nv_bfloat16*>(Q.ptr), Q.sB, Q.sH, Q.sN, Q.N, D, seg,
                                           static_cast<int>(Q.H / K.H), static_cast<int>(K.H), g, qperm);
  return cudaGetLastError();
}

}  // namespace pbs
