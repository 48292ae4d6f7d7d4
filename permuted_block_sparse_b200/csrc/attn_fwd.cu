// pbs_attn_fwd: FlashAttention-style forward over an online key permutation.
//
// "S2O: Early Stopping for Sparse Attention via Online Permutation",
// Technical Summary:
//   1. Online Permutation via Index-Driven Loading -- K/V stay in their HBM
//      layout; an index list says which (non-contiguous) rows to load, and
//      the kernel gathers those rows into shared memory;
//   3. Kernel Implementation -- Pass 1 runs dense causal attention over the
//      query block's own segment and builds the online-softmax state
//      (m, l, acc); Pass 2 continues from that state over prefix key blocks
//      in permuted order.
// "Block Sparse Flash Attention", Approach: the exact tile maximum of QK^T
// is compared with a per-(head, query block) threshold; below it the tile
// is dropped before the V load and the PV product.
//
// sm_100a design (this file): one CTA per (query block, query head, batch),
// 128 threads.  K/V rows of a tile (natural or permuted) are gathered with
// 16-byte cp.async into 128B-swizzled shared-memory tiles; QK^T and PV run
// on the 5th-generation tensor cores (tcgen05.mma, bf16 in, fp32 in tensor
// memory); each thread owns one query row of S / O in tensor memory, so the
// online softmax needs no cross-thread reduction; P is written back to
// tensor memory as bf16 and consumed directly as the A operand of PV.
#include <math.h>

#include "pbs_common.cuh"
#include "pbs_internal.h"

namespace pbs {
namespace {

constexpr int kThreads = 128;
constexpr int kM = 128;               // query rows per MMA tile
constexpr uint32_t kTmemCols = 256;   // S/P: cols [0,128), O: cols [128, 128+D)
constexpr float kRescaleSlack = 8.0f; // keep the running max while within 2^8

template <int D, int BLK>
struct Smem {
  static constexpr int kQBytes = (D / 64) * kM * 128;
  static constexpr int kKVBytes = (D / 64) * BLK * 128;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBytes;
  static constexpr int kV = kK + kKVBytes;
  static constexpr int kEnd = kV + kKVBytes;
  // + alignment slack; at least 90 KB so that no more than two CTAs share an
  // SM, which keeps their tensor-memory allocations (256 columns each) within
  // the SM's 512 columns and tcgen05.alloc never has to wait.
  static constexpr int kTotal = (kEnd + 1024) > 92160 ? (kEnd + 1024) : 92160;
};

__device__ __forceinline__ float warp_max(float v) {
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

template <int D, int BLK>
__global__ void __launch_bounds__(kThreads) attn_fwd_kernel(AttnParams p) {
  using L = Smem<D, BLK>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int32_t rowpos[BLK];
  __shared__ float red[4];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Heavy query blocks (more tiles) first.
  const int i = p.nb - 1 - static_cast<int>(blockIdx.x);
  const int hq = blockIdx.y, b = blockIdx.z;
  const int hk = hq / p.G;
  const int spb = p.seg / BLK;
  const int s = i / spb;
  const int64_t q0 = static_cast<int64_t>(i) * BLK;
  const int64_t N = p.Q.N;

  const uint32_t sQ = smem_u32(smem + L::kQ);
  const uint32_t sK = smem_u32(smem + L::kK);
  const uint32_t sV = smem_u32(smem + L::kV);

  if (warp == 0) {
    tmem_alloc(&tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&mma_bar, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tS = tmem, tP = tmem, tO = tmem + 128;

  // ---- Q tile: rows q0 .. q0+BLK-1, padded with zeros to 128 rows.
  {
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(p.Q.ptr) + b * p.Q.sB + hq * p.Q.sH;
    constexpr int CH = D / 8;
    for (int id = tid; id < kM * CH; id += kThreads) {
      const int r = id / CH, c = id % CH;
      const bool valid = r < BLK;
      const __nv_bfloat16* src = valid ? qb + (q0 + r) * p.Q.sN + c * 8 : qb;
      cp_async16_zfill(sQ + (c / 8) * (kM * 128) + sw128_offset(r, c % 8), src, valid);
    }
    cp_async_commit();
  }

  const int cnt_raw = p.counts[(static_cast<int64_t>(b) * (p.G * p.K.H) + hq) * p.nb + i];
  int cnt = cnt_raw;
  if (cnt < 0 || cnt > p.cap) {
    if (tid == 0) set_error(p.err, kErrDeviceCheck);
    cnt = 0;
  }
  const int32_t* list = p.idx + ((static_cast<int64_t>(b) * (p.G * p.K.H) + hq) * p.nb + i) * p.cap;
  const int32_t* prow = p.perm + (static_cast<int64_t>(b) * p.K.H + hk) * N;
  const int n_diag = i - s * spb + 1;
  const int n_tiles = n_diag + cnt;
  const float thr = p.gate_thr ? p.gate_thr[(static_cast<int64_t>(b) * (p.G * p.K.H) + hq) * p.nb + i]
                               : -INFINITY;

  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(p.K.ptr) + b * p.K.sB + hk * p.K.sH;
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(p.V.ptr) + b * p.V.sB + hk * p.V.sH;

  const int r = warp * 32 + lane;      // this thread's query row in the tile
  float m_run = -INFINITY, l_run = 0.f;
  bool o_init = false;
  uint32_t phase = 0;
  int n_qk = 0, n_gated = 0;
  bool aborted = false;

  for (int t = 0; t < n_tiles && !aborted; ++t) {
    // Pass 1 (t < n_diag): natural blocks of the own segment, from block i
    // down; Pass 2: listed permuted blocks of earlier segments.
    const bool is_diag = t < n_diag;
    const int j = is_diag ? i - t : 0;
    int pb = -1;
    if (!is_diag) {
      pb = list[t - n_diag];
      if (pb < 0 || pb >= s * spb) {
        if (tid == 0) set_error(p.err, kErrDeviceCheck);
        continue;
      }
    }
    if (tid < BLK) {
      int64_t x;
      if (is_diag) {
        x = static_cast<int64_t>(j) * BLK + tid;
      } else {
        const int64_t lp = static_cast<int64_t>(pb) * BLK + tid;
        const int64_t lo = (lp / p.seg) * p.seg;
        x = prow[lp];
        if (x < lo || x >= lo + p.seg || x >= N) {
          set_error(p.err, kErrDeviceCheck);
          x = lo;                      // in bounds, inside the segment
        }
      }
      rowpos[tid] = static_cast<int32_t>(x);
    }
    __syncthreads();
    {
      constexpr int CH = D / 8;
      for (int id = tid; id < BLK * CH; id += kThreads) {
        const int rr = id / CH, c = id % CH;
        const int64_t x = rowpos[rr];
        const uint32_t off = (c / 8) * (BLK * 128) + sw128_offset(rr, c % 8);
        cp_async16(sK + off, kb + x * p.K.sN + c * 8);
        cp_async16(sV + off, vb + x * p.V.sN + c * 8);
      }
      cp_async_commit();
      cp_async_wait_all();
      fence_proxy_async();
    }
    __syncthreads();

    // ---- S = Q K^T into tensor memory.
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(kM, BLK, false);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t half = kk / 4, koff = (kk % 4) * 32;
        const uint64_t a = sdesc_sw128(sQ + half * (kM * 128) + koff, 16, 1024);
        const uint64_t bd = sdesc_sw128(sK + half * (BLK * 128) + koff, 16, 1024);
        mma_ss(tS, a, bd, idesc, kk > 0 ? 1u : 0u);
      }
      tc_commit(&mma_bar);
    }
    const bool ok1 = mbar_wait(&mma_bar, phase, p.err);
    phase ^= 1;
    if (__syncthreads_or(!ok1)) {
      aborted = true;
      break;
    }
    tc_fence_after();
    ++n_qk;

    // ---- softmax on this thread's row.
    float sv[BLK];
#pragma unroll
    for (int c = 0; c < BLK / 32; ++c) {
      uint32_t u[32];
      tmem_ld32(tS + lane_off + c * 32, u);
#pragma unroll
      for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(u[e]);
    }
    const bool causal_tile = is_diag && j == i;
    float rmax = -INFINITY;
#pragma unroll
    for (int c = 0; c < BLK; ++c) {
      const bool vis = !causal_tile || c <= r;
      if (!vis) sv[c] = -INFINITY;
      rmax = fmaxf(rmax, sv[c]);
    }
    if (p.gate_thr && !causal_tile) {
      float wm = warp_max(r < BLK ? rmax : -INFINITY);
      if (lane == 0) red[warp] = wm;
      __syncthreads();
      const float tmax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
      __syncthreads();
      if (tmax < thr) {
        ++n_gated;
        tc_fence_before();             // S reads done before the next QK^T overwrites S
        continue;                      // tile dropped: no V, no PV, no state update
      }
    }
    const float mx = rmax * p.scale_log2;
    const float m_new = (m_run == -INFINITY || mx > m_run + kRescaleSlack) ? fmaxf(mx, m_run) : m_run;
    const float alpha = ex2(m_run - m_new);
    float psum = 0.f;
    uint32_t packed[BLK / 2];
#pragma unroll
    for (int c = 0; c < BLK; c += 2) {
      const float p0 = ex2(fmaf(sv[c], p.scale_log2, -m_new));
      const float p1 = ex2(fmaf(sv[c + 1], p.scale_log2, -m_new));
      psum += p0 + p1;
      packed[c / 2] = pack_bf16x2(p0, p1);
    }
    l_run = l_run * alpha + psum;
    m_run = m_new;
    if (o_init && __any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(tO + lane_off + c * 32, u);
#pragma unroll
        for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
        tmem_st32(tO + lane_off + c * 32, u);
      }
    }
#pragma unroll
    for (int c = 0; c < BLK / 64; ++c) {
      uint32_t u[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) u[e] = packed[c * 32 + e];
      tmem_st32(tP + lane_off + c * 32, u);
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();

    // ---- O += P V.
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16(kM, D, true);
#pragma unroll
      for (int kk = 0; kk < BLK / 16; ++kk) {
        const uint64_t bd = sdesc_sw128(sV + kk * 2048, BLK * 128, 1024);
        mma_ts(tO, tP + kk * 8, bd, idesc, (o_init || kk > 0) ? 1u : 0u);
      }
      tc_commit(&mma_bar);
    }
    const bool ok2 = mbar_wait(&mma_bar, phase, p.err);
    phase ^= 1;
    if (__syncthreads_or(!ok2)) {
      aborted = true;
      break;
    }
    tc_fence_after();
    o_init = true;
  }

  // ---- epilogue: O / l -> bf16, LSE.
  if (!aborted && o_init) {
    const float inv_l = 1.0f / l_run;
    __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(const_cast<void*>(p.O.ptr)) + b * p.O.sB +
                        hq * p.O.sH + (q0 + r) * p.O.sN;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t u[32];
      tmem_ld32(tO + lane_off + c * 32, u);
      if (r < BLK) {
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(u[e + 0]) * inv_l, __uint_as_float(u[e + 1]) * inv_l);
          v.y = pack_bf16x2(__uint_as_float(u[e + 2]) * inv_l, __uint_as_float(u[e + 3]) * inv_l);
          v.z = pack_bf16x2(__uint_as_float(u[e + 4]) * inv_l, __uint_as_float(u[e + 5]) * inv_l);
          v.w = pack_bf16x2(__uint_as_float(u[e + 6]) * inv_l, __uint_as_float(u[e + 7]) * inv_l);
          *reinterpret_cast<uint4*>(ob + c * 32 + e) = v;
        }
      }
    }
    if (p.lse && r < BLK)
      p.lse[(static_cast<int64_t>(b) * (p.G * p.K.H) + hq) * N + q0 + r] =
          (m_run + log2f(l_run)) * 0.69314718055994531f;
  }
  if (tid == 0 && p.stats) {
    atomicAdd(reinterpret_cast<unsigned long long*>(p.stats), static_cast<unsigned long long>(n_qk));
    atomicAdd(reinterpret_cast<unsigned long long*>(p.stats) + 1,
              static_cast<unsigned long long>(n_gated));
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int BLK>
cudaError_t launch_typed(const AttnParams& p, cudaStream_t s) {
  using L = Smem<D, BLK>;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, BLK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(p.nb), static_cast<unsigned>(p.Q.H), static_cast<unsigned>(p.Q.B));
  attn_fwd_kernel<D, BLK><<<grid, kThreads, L::kTotal, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd(const AttnParams& p, cudaStream_t s) {
  const int D = static_cast<int>(p.Q.D);
  if (D == 128 && p.blk == 128) return launch_typed<128, 128>(p, s);
  if (D == 128 && p.blk == 64) return launch_typed<128, 64>(p, s);
  if (D == 64 && p.blk == 128) return launch_typed<64, 128>(p, s);
  if (D == 64 && p.blk == 64) return launch_typed<64, 64>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace pbs
