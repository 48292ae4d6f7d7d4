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

// One CTA per (segment, hkv, b), kSortThreads threads.  Scores every key of
// the segment with one fp32 dot product against qhat (lanes of a row group
// read 16 bytes each, a row is one coalesced 128/256-byte read; eight rows
// per thread in flight), packs (descending score, ascending position) into
// one 64-bit key and sorts the keys: sorting unique composite keys is a
// total order, so the result equals a stable descending sort by score.
//
// The sort is bitonic with E keys per thread in registers (thread t holds
// elements t*E .. t*E+E-1): exchanges between elements of one thread are
// register swaps, between threads of one warp (partner distance below 32*E)
// warp shuffles, and only the longer distances go through shared memory
// with a barrier -- 10 of the 78 stages for a 4096-key segment.
constexpr int kSortThreads = 512;

template <int E>
__device__ __forceinline__ void bitonic_regs(uint64_t (&v)[E], int n2, uint64_t* sm) {
  const int tid = threadIdx.x, lane = tid & 31;
  for (int k = 2; k <= n2; k <<= 1) {
    // partner distances j >= E: another thread
    for (int j = k >> 1; j >= E; j >>= 1) {
      if (j < 32 * E) {
        // partner in another lane of this warp: lane ^ (j / E), same e
        const int lx = j / E;
        const bool lower = (lane & lx) == 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const bool up = ((tid * E + e) & k) == 0;
          const uint64_t o = __shfl_xor_sync(0xffffffffu, v[e], lx);
          const uint64_t mn = v[e] < o ? v[e] : o, mx = v[e] < o ? o : v[e];
          v[e] = (lower == up) ? mn : mx;
        }
      } else {
        // partner in another warp: through shared memory
#pragma unroll
        for (int e = 0; e < E; ++e) sm[tid * E + e] = v[e];
        __syncthreads();
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = tid * E + e;
          const bool up = (i & k) == 0, lower = (i & j) == 0;
          const uint64_t o = sm[i ^ j];
          const uint64_t mn = v[e] < o ? v[e] : o, mx = v[e] < o ? o : v[e];
          v[e] = (lower == up) ? mn : mx;
        }
        __syncthreads();
      }
    }
    // partner distances j < E: this thread's own registers (static indices)
#pragma unroll
    for (int j = E / 2; j > 0; j >>= 1) {
      if (j < k) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          if ((e & j) == 0) {
            const bool up = ((tid * E + e) & k) == 0;
            const uint64_t a = v[e], c = v[e | j];
            if ((a > c) == up) {
              v[e] = c;
              v[e | j] = a;
            }
          }
        }
      }
    }
  }
}

template <int E>
__global__ void __launch_bounds__(kSortThreads, 2) score_sort_kernel(
    const __nv_bfloat16* __restrict__ K, int64_t sB, int64_t sH, int64_t sN, int64_t N, int D,
    int seg, int n_sink, const float* __restrict__ qhat, int32_t* __restrict__ perm) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int t = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z, Hkv = gridDim.y;
  const int64_t lo = static_cast<int64_t>(t) * seg;
  const int len = static_cast<int>(min(static_cast<int64_t>(seg), N - lo));
  // the whole CTA sorts kSortThreads * E >= len keys; the padding keys
  // (all ones) sort after every real one
  const int n2 = kSortThreads * E;
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem_raw);
  float* q = reinterpret_cast<float*>(keys + kSortThreads * E);
  for (int c = threadIdx.x; c < D; c += blockDim.x)
    q[c] = qhat[(static_cast<int64_t>(b) * Hkv + hkv) * D + c];
  for (int r = len + threadIdx.x; r < kSortThreads * E; r += blockDim.x) keys[r] = ~0ull;
  __syncthreads();

  const int lanes_per_row = D / 8;           // 16 (D=128) or 8 (D=64)
  const int rows_per_warp = 32 / lanes_per_row;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  const int sub = lane / lanes_per_row, cl = lane % lanes_per_row;
  const __nv_bfloat16* base = K + b * sB + hkv * sH;
  float qv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) qv[e] = q[cl * 8 + e];
  // kRowsInFlight rows per thread are loaded before any is used, so each
  // thread keeps that many 16-byte reads in flight.
  constexpr int kRowsInFlight = 8;
  const int step = nwarp * rows_per_warp;
  for (int r0 = warp * rows_per_warp; r0 < len; r0 += kRowsInFlight * step) {
    uint4 v[kRowsInFlight];
#pragma unroll
    for (int u = 0; u < kRowsInFlight; ++u) {
      const int r = r0 + u * step + sub;
      v[u] = r < len ? *reinterpret_cast<const uint4*>(base + (lo + r) * sN + cl * 8) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kRowsInFlight; ++u) {
      const int r = r0 + u * step + sub;
      float acc = 0.f;
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(p[e]);
        acc = fmaf(f.x, qv[2 * e], acc);
        acc = fmaf(f.y, qv[2 * e + 1], acc);
      }
      for (int off = lanes_per_row >> 1; off > 0; off >>= 1)
        acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (r < len && cl == 0) {
        const float sc = (lo + r < n_sink) ? __int_as_float(0x7f800000) : acc;
        keys[r] = (static_cast<uint64_t>(~ordered_u32(sc)) << 32) | static_cast<uint32_t>(r);
      }
    }
  }
  __syncthreads();
  uint64_t v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) v[e] = keys[threadIdx.x * E + e];
  __syncthreads();
  bitonic_regs<E>(v, n2, keys);
  int32_t* out = perm + (static_cast<int64_t>(b) * Hkv + hkv) * N + lo;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int r = threadIdx.x * E + e;
    if (r < len) out[r] = static_cast<int32_t>(lo + static_cast<uint32_t>(v[e] & 0xffffffffu));
  }
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
  dim3 grid(static_cast<unsigned>(nseg), static_cast<unsigned>(K.H), static_cast<unsigned>(K.B));
  auto run = [&](auto kernel, int E) -> cudaError_t {
    const size_t smem = static_cast<size_t>(kSortThreads) * E * 8 + K.D * 4;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kernel<<<grid, kSortThreads, smem, s>>>(static_cast<const __nv_bfloat16*>(K.ptr), K.sB, K.sH, K.sN, K.N,
                                           static_cast<int>(K.D), seg, n_sink, qhat, perm);
    return cudaGetLastError();
  };
  if (seg <= kSortThreads) return run(score_sort_kernel<1>, 1);
  if (seg <= 2 * kSortThreads) return run(score_sort_kernel<2>, 2);
  if (seg <= 4 * kSortThreads) return run(score_sort_kernel<4>, 4);
  if (seg <= 8 * kSortThreads) return run(score_sort_kernel<8>, 8);
  return run(score_sort_kernel<16>, 16);      // seg <= 8192
}

}  // namespace pbs
