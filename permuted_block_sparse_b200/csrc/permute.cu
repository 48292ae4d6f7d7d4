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
  // eight rows per thread in flight, then added in row order
  for (int r0 = rl; r0 < rows; r0 += 8 * lanes) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int r = r0 + u * lanes;
      const int h = hkv * G + r / blk;
      const int64_t n = N - blk + (r % blk);
      v[u] = r < rows ? *reinterpret_cast<const uint4*>(Q + b * sB + h * sH + n * sN + chunk * 8) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(p[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
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
// per thread in flight), then sorts the segment by descending score with a
// stable least-significant-digit radix sort of the 32-bit order-inverted
// scores (four passes of 8 bits).  The keys start in ascending position and
// every pass keeps equal digits in their current order, so equal scores end
// in ascending position: a stable descending sort by score.
//
// A pass over n = kSortThreads * E keys: warp w owns positions
// [w*32*E, (w+1)*32*E), element (e, lane) at w*32*E + e*32 + lane.  Each
// warp ranks its keys among equal digits with a match over lanes and
// running per-digit counters (e in order), a block-wide scan over
// (digit, warp) in digit-major order gives every warp's offset for every
// digit, and the keys scatter to offset + rank in a second buffer.
constexpr int kSortThreads = 512;
constexpr int kSortWarps = kSortThreads / 32;

template <int E>
__global__ void __launch_bounds__(kSortThreads, 2) score_sort_kernel(
    const __nv_bfloat16* __restrict__ K, int64_t sB, int64_t sH, int64_t sN, int64_t N, int D,
    int seg, int n_sink, const float* __restrict__ qhat, int32_t* __restrict__ perm) {
  constexpr int n = kSortThreads * E;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint32_t* skey = reinterpret_cast<uint32_t*>(smem_raw);                 // [2][n]
  uint16_t* sidx = reinterpret_cast<uint16_t*>(skey + 2 * n);             // [2][n]
  uint32_t* hist = reinterpret_cast<uint32_t*>(sidx + 2 * n);             // [kSortWarps][256]
  float* q = reinterpret_cast<float*>(hist + kSortWarps * 256);
  __shared__ uint32_t wsum[kSortWarps];
  const int t = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z, Hkv = gridDim.y;
  const int64_t lo = static_cast<int64_t>(t) * seg;
  const int len = static_cast<int>(min(static_cast<int64_t>(seg), N - lo));
  for (int c = threadIdx.x; c < D; c += blockDim.x)
    q[c] = qhat[(static_cast<int64_t>(b) * Hkv + hkv) * D + c];
  // padding keys (all ones) come after every real key in the initial order
  for (int r = threadIdx.x; r < n; r += blockDim.x) {
    skey[r] = 0xffffffffu;
    sidx[r] = static_cast<uint16_t>(r);
  }
  __syncthreads();

  const int lanes_per_row = D / 8;           // 16 (D=128) or 8 (D=64)
  const int rows_per_warp = 32 / lanes_per_row;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / lanes_per_row, cl = lane % lanes_per_row;
  const __nv_bfloat16* base = K + b * sB + hkv * sH;
  float qv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) qv[e] = q[cl * 8 + e];
  // kRowsInFlight rows per thread are loaded before any is used, so each
  // thread keeps that many 16-byte reads in flight.
  constexpr int kRowsInFlight = 8;
  const int step = kSortWarps * rows_per_warp;
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
        skey[r] = ~ordered_u32(sc);                // ascending key = descending score
      }
    }
  }
  __syncthreads();

  const uint32_t lt_mask = (1u << lane) - 1u;
  int cur = 0;
  for (int shift = 0; shift < 32; shift += 8) {
    const uint32_t* kin = skey + cur * n;
    const uint16_t* iin = sidx + cur * n;
    uint32_t* kout = skey + (cur ^ 1) * n;
    uint16_t* iout = sidx + (cur ^ 1) * n;
    uint32_t* h = hist + warp * 256;
    for (int d = lane; d < 256; d += 32) h[d] = 0u;
    __syncwarp();
    uint32_t key[E], rank[E];
    uint16_t ix[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int pos = warp * 32 * E + e * 32 + lane;
      key[e] = kin[pos];
      ix[e] = iin[pos];
      const uint32_t dg = (key[e] >> shift) & 255u;
      const uint32_t peers = __match_any_sync(0xffffffffu, dg);
      const uint32_t before = h[dg];
      rank[e] = before + __popc(peers & lt_mask);
      __syncwarp();
      if ((peers & lt_mask) == 0u) h[dg] = before + __popc(peers);   // the lowest peer lane
      __syncwarp();
    }
    __syncthreads();
    // exclusive scan over (digit, warp), digit-major: thread tid covers
    // digit tid / 2, warps (tid % 2) * 8 .. + 7
    {
      const int dg = threadIdx.x >> 1, w0 = (threadIdx.x & 1) * 8;
      uint32_t c[8], tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[(w0 + j) * 256 + dg];
        tot += c[j];
      }
      uint32_t incl = tot;
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      if (lane == 31) wsum[warp] = incl;
      __syncthreads();
      uint32_t wpre = 0;
      for (int w = 0; w < warp; ++w) wpre += wsum[w];
      uint32_t run = wpre + incl - tot;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        hist[(w0 + j) * 256 + dg] = run;           // now this warp's offset for the digit
        run += c[j];
      }
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const uint32_t dg = (key[e] >> shift) & 255u;
      const uint32_t dst = h[dg] + rank[e];
      kout[dst] = key[e];
      iout[dst] = ix[e];
    }
    __syncthreads();
    cur ^= 1;
  }
  const uint16_t* order = sidx + cur * n;
  int32_t* out = perm + (static_cast<int64_t>(b) * Hkv + hkv) * N + lo;
  for (int r = threadIdx.x; r < len; r += blockDim.x) out[r] = static_cast<int32_t>(lo + order[r]);
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
    const size_t n = static_cast<size_t>(kSortThreads) * E;
    const size_t smem = n * 2 * 4 + n * 2 * 2 + kSortWarps * 256 * 4 + K.D * 4;
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
