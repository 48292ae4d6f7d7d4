// pbs_select mode PBS_SELECT_SAMPLE: a SampleAttention-style selector over
// natural key blocks.
//
// "SampleAttention" (MLSys 2025 talk), Technical Deep Dive:
//   Stage 1, Trunk Sampling -- estimate attention scores from queries sampled
//     in chunks (trunks) across the sequence;
//   Stage 2, Score-Based Filtering -- choose the key columns and slash
//     offsets that together hold the required share of the attention mass
//     (the CIA target), each family cut on its own, and turn them into a
//     block mask.
// Here the trunks are the last query block of every segment.  Per query
// head, their softmax probabilities are summed per key column and per slash
// offset q - k (fp64 accumulation); each family keeps its highest entries up
// to and including the one at which the accumulated score reaches alpha of
// its total (ties to the lower index); query block i lists every key block
// of earlier segments that holds a kept column, or a key q - d for one of
// its queries q and a kept offset d.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "pbs_common.cuh"
#include "pbs_internal.h"

namespace pbs {
namespace {

constexpr int kSampleWarps = 8;

// Stage 1 on the tensor cores.  One CTA per (trunk s, hq, b), heaviest
// trunks first.  The trunk's rows (the last blk queries of segment s, zero
// rows up to 128) stay in shared memory; the keys 0 .. seg_end - 1 stream
// through twice in tiles of 128 (pass 1, then pass 2).  Warp-specialized:
//   warp 0      issues S = Q_trunk K_tile^T (tcgen05.mma) into a ring of
//               four tensor-memory buffers, as far ahead as the buffers and
//               the key ring allow;
//   warp 1      loads the trunk's query tile once and the key tiles into a
//               ring of three shared-memory slots with TMA (cp.async.bulk
//               .tensor, 128-byte swizzle, no multicast);
//   warps 4-19  read S: warp 4 + w takes tensor-memory lanes 32 (w mod 4)
//               .. +31 (trunk rows) and columns 32 (w / 4) .. +31.
//   Pass 1: per row and quarter the running maximum m of x = S log2(e) /
//     sqrt(d) over the causal keys, kept rounded up to an integer so that
//     every rescale of the running sum l = sum 2^(x - m) (fp32 within a
//     tile, fp64 across tiles) is an exact power of two; the quarters merge
//     at the end.
//   Pass 2: p = 2^(x - m) / l (fp32) goes to a 128 x 129 fp32 tile in shared
//     memory (one word of padding per row).  Consumer threads 0-255 sum key
//     columns (two per column, one per half of the rows), threads 256-511
//     the diagonals t - c = -u and 128 - u of skew u (two per skew, again by
//     row halves), all without bank conflicts; the halves meet in shared
//     memory and each per-tile sum is added to the key's column score or the
//     offset's slash score with one fp64 atomic.
// The logits q.k of bf16 inputs are accumulated in fp32 by the tensor core.
// Every wait is bounded; a shared abort flag ends the MMA and producer roles
// and turns the consumers' remaining waits into no-ops.
template <int D>
struct SampleCfg {
  static constexpr int kHalfBytes = 128 * 128;               // 128 rows x 64 bf16
  static constexpr int kTileBytes = (D / 64) * kHalfBytes;   // Q or K tile
  static constexpr int kPStride = 129;                       // floats per row of the P tile
  static constexpr int kStages = 3;                           // key tile ring
  static constexpr int kSBufs = 4;                            // S buffers in tensor memory
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kP = kK + kStages * kTileBytes;
  static constexpr int kMl = kP + 128 * kPStride * 4;          // per-quarter (m, l) at the end of pass 1
  static constexpr int kHalf = kMl + 4 * 128 * 12;             // second-half partial sums
  static constexpr int kBar = kHalf + 3 * 128 * 4;
  static constexpr int kNBar = 1 + 2 * kStages + 2 * kSBufs;
  static constexpr int kSlot = kBar + kNBar * 8;
  static constexpr int kBytes = kSlot + 16;
  static constexpr int kSmem = kBytes + 1024;                // alignment slack
};
constexpr int kScoreThreads = 640;                            // warps 2-3 only join the teardown
constexpr int kScoreConsumers = 512;                          // warps 4-19


template <int D>
__global__ void __launch_bounds__(kScoreThreads, 1) sample_scores_kernel(
    const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk, int64_t N, int B, int Hq,
    int G, int blk, int seg, float scale_log2, double* __restrict__ col, double* __restrict__ sl,
    int* __restrict__ err) {
  using C = SampleCfg<D>;
  constexpr int PS = C::kPStride, NK = C::kStages, NS = C::kSBufs;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  float* sP = reinterpret_cast<float*>(smem + C::kP);
  double* sL = reinterpret_cast<double*>(smem + C::kMl);                 // [4][128]
  float* sM = reinterpret_cast<float*>(smem + C::kMl + 4 * 128 * 8);     // [4][128]
  float* sH = reinterpret_cast<float*>(smem + C::kHalf);                 // [3][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBar);
  uint64_t* bar_q = bars;
  uint64_t* bar_kfull = bars + 1;
  uint64_t* bar_kempty = bar_kfull + NK;
  uint64_t* bar_sfull = bar_kempty + NK;
  uint64_t* bar_sfree = bar_sfull + NS;
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + C::kSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kSlot + 4);
  const uint32_t sQ = smem_u32(smem + C::kQ), sK = smem_u32(smem + C::kK);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nseg = static_cast<int>((N + seg - 1) / seg);
  const int BH = B * Hq;
  const int s = nseg - 1 - static_cast<int>(blockIdx.x / BH);
  const int bh = static_cast<int>(blockIdx.x % BH);
  const int b = bh / Hq, hq = bh % Hq;
  const int64_t seg_end = min(static_cast<int64_t>(s + 1) * seg, N);
  const int64_t qbase = seg_end - blk;
  const int T = static_cast<int>((seg_end + 127) / 128);
  const int n_it = 2 * T;                                      // MMAs: pass 1 then pass 2

  if (warp == 0) {
    tmem_alloc(slot, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < NK; ++i) {
      mbar_init(&bar_kfull[i], 1);
      mbar_init(&bar_kempty[i], 1);
    }
    for (int i = 0; i < NS; ++i) {
      mbar_init(&bar_sfull[i], 1);
      mbar_init(&bar_sfree[i], kScoreConsumers / 32);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- MMA
    constexpr uint32_t idesc = idesc_bf16(128, 128, false);
    // every lane waits; the warp goes on only if all of them saw the phase
    bool ok = __all_sync(0xffffffffu, mbar_wait_or_abort(bar_q, 0, err, abort_flag));
    for (int it = 0; ok && it < n_it; ++it) {
      const int ks = it % NK, sb = it % NS;
      ok = mbar_wait_or_abort(&bar_kfull[ks], (it / NK) & 1, err, abort_flag);
      if (ok && it >= NS) ok = mbar_wait_or_abort(&bar_sfree[sb], ((it / NS) - 1) & 1, err, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint64_t a0 = sdesc_sw128(sQ, 16, 1024);
      const uint64_t b0 = sdesc_sw128(sK + ks * C::kTileBytes, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk / 4) * C::kHalfBytes + (kk % 4) * 32;
        if (elect_one()) mma_ss(tmem + sb * 128, sdesc_add(a0, off), sdesc_add(b0, off), idesc, kk > 0 ? 1u : 0u);
      }
      if (elect_one()) {
        tc_commit(&bar_sfull[sb]);
        tc_commit(&bar_kempty[ks]);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      constexpr uint32_t kTileTx = 128 * D * 2;
      mbar_expect_tx(bar_q, kTileTx);
      for (int h = 0; h < D / 64; ++h) tma_rows_4d(sQ + h * C::kHalfBytes, &mq, 64 * h, static_cast<int>(qbase), hq, b, bar_q);
      for (int it = 0; it < n_it; ++it) {
        const int ks = it % NK;
        if (it >= NK && !mbar_wait_or_abort(&bar_kempty[ks], ((it / NK) - 1) & 1, err, abort_flag)) break;
        const int k0 = (it % T) * 128;
        mbar_expect_tx(&bar_kfull[ks], kTileTx);
        for (int h = 0; h < D / 64; ++h)
          tma_rows_4d(sK + ks * C::kTileBytes + h * C::kHalfBytes, &mk, 64 * h, k0, hq / G, b, &bar_kfull[ks]);
      }
    }
    __syncwarp();
  } else if (warp < 4) {
    // warps 2-3 have no role
  } else {
    // ----------------------------------------------------------- consumers
    const int ct = tid - 128, cw = ct >> 5;
    const int t = (cw & 3) * 32 + lane;                        // trunk row of this thread
    const int qc = cw >> 2;                                    // column quarter
    const uint32_t lane_base = static_cast<uint32_t>((cw & 3) * 32) << 16;
    const int64_t q_t = qbase + t;
    const bool row_ok = t < blk;
    float m = -INFINITY;                                       // integer-valued running maximum
    double l = 0.0;
    float w = 0.f;                                             // 1 / l of this row (pass 2)
    float* prow = sP + t * PS + qc * 32;
    const int role = ct >> 7, x = ct & 127;                    // reduction role and its index
    const int64_t base = static_cast<int64_t>(bh) * N;
    for (int it = 0; it < n_it; ++it) {
      const int sb = it % NS, j = it % T;
      // After an abort (the wait gave up) the loop still runs to its end, so
      // that every consumer takes the same named barriers; the results are
      // then meaningless and the error word says so.
      mbar_wait_or_abort(&bar_sfull[sb], (it / NS) & 1, err, abort_flag);
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32(tmem + lane_base + sb * 128 + qc * 32, r);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_sfree[sb]);
      const int64_t k0 = static_cast<int64_t>(j) * 128;
      // every key of the tile is causal for every trunk row
      const bool full = k0 + 127 <= qbase;
      // otherwise keys k0 + 32 qc + c with c <= lim are causal for this row
      const int64_t lim64 = q_t - k0 - 32 * qc;
      const int lim = static_cast<int>(lim64 > 31 ? 31 : (lim64 < -1 ? -1 : lim64));
      if (it < T) {
        float mr = -INFINITY;                                  // max of the raw logits
        if (full) {
#pragma unroll
          for (int c = 0; c < 31; c += 2) mr = fmax3(mr, __uint_as_float(r[c]), __uint_as_float(r[c + 1]));
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c <= lim) mr = fmaxf(mr, __uint_as_float(r[c]));
        }
        if (mr > -INFINITY) {
          const float mn = fmaxf(m, ceilf(mr * scale_log2));
          if (mn > m) {
            l = (m == -INFINITY) ? 0.0 : ldexp(l, static_cast<int>(m - mn));
            m = mn;
          }
          float a[4] = {0.f, 0.f, 0.f, 0.f};
          if (full) {
#pragma unroll
            for (int c = 0; c < 32; ++c) a[c % 4] += ex2(fmaf(__uint_as_float(r[c]), scale_log2, -m));
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c <= lim) a[c % 4] += ex2(fmaf(__uint_as_float(r[c]), scale_log2, -m));
          }
          l += static_cast<double>((a[0] + a[1]) + (a[2] + a[3]));
        }
        if (it == T - 1) {
          // merge the quarters: the largest maximum, every sum rescaled by
          // an exact power of two
          sM[qc * 128 + t] = m;
          sL[qc * 128 + t] = l;
          named_sync(1, kScoreConsumers);
          float mm = -INFINITY;
#pragma unroll
          for (int q = 0; q < 4; ++q) mm = fmaxf(mm, sM[q * 128 + t]);
          double lt = 0.0;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float mq = sM[q * 128 + t];
            if (mq > -INFINITY) lt += ldexp(sL[q * 128 + t], static_cast<int>(mq - mm));
          }
          m = mm;
          w = row_ok && lt > 0.0 ? static_cast<float>(1.0 / lt) : 0.f;
        }
      } else {
        if (full) {
#pragma unroll
          for (int c = 0; c < 32; ++c) prow[c] = ex2(fmaf(__uint_as_float(r[c]), scale_log2, -m)) * w;
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            prow[c] = c <= lim ? ex2(fmaf(__uint_as_float(r[c]), scale_log2, -m)) * w : 0.f;
        }
        named_sync(1, kScoreConsumers);
        const int u0 = (role & 1) * 64, u1 = u0 + 64;          // this thread's half of the rows
        float ca = 0.f, cb = 0.f;                              // column, or the two diagonals
        if (role < 2) {
          // key column x: rows u at u * PS + x
          const float* pc = sP + x;
          float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 4
          for (int u = u0; u < u1; u += 4) {
            a0 += pc[u * PS];
            a1 += pc[(u + 1) * PS];
            a2 += pc[(u + 2) * PS];
            a3 += pc[(u + 3) * PS];
          }
          ca = (a0 + a1) + (a2 + a3);
        } else {
          // skew x: element (u, (u + x) mod 128) lies on offset d0 - x for
          // u < 128 - x and on d0 + 128 - x after
          const int split = min(max(128 - x, u0), u1);
          const float* pd = sP + x;
          const float* pe = pd - 128;
          float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
          int u = u0;
          for (; u + 1 < split; u += 2) {
            a0 += pd[u * (PS + 1)];
            a1 += pd[(u + 1) * (PS + 1)];
          }
          if (u < split) a0 += pd[u * (PS + 1)], ++u;
          for (; u + 1 < u1; u += 2) {
            b0 += pe[u * (PS + 1)];
            b1 += pe[(u + 1) * (PS + 1)];
          }
          if (u < u1) b0 += pe[u * (PS + 1)];
          ca = a0 + a1;
          cb = b0 + b1;
        }
        // second row halves hand their sums to the first; after this barrier
        // the P tile is free again
        if (role == 1) sH[x] = ca;
        if (role == 3) {
          sH[128 + x] = ca;
          sH[256 + x] = cb;
        }
        named_sync(1, kScoreConsumers);
        if (role == 0) {
          const double cs = static_cast<double>(ca + sH[x]);
          if (cs != 0.0 && k0 + x < N) atomicAdd(col + base + k0 + x, cs);
        } else if (role == 2) {
          const double da = static_cast<double>(ca + sH[128 + x]), db = static_cast<double>(cb + sH[256 + x]);
          const int64_t d0 = qbase - k0;
          if (da != 0.0 && d0 - x >= 0 && d0 - x < N) atomicAdd(sl + base + d0 - x, da);
          if (db != 0.0 && d0 + 128 - x >= 0 && d0 + 128 - x < N) atomicAdd(sl + base + d0 + 128 - x, db);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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

// Stage 2, one family.  One CTA of 1024 threads per (family, hq, b): the
// largest score threshold whose upper set reaches alpha of the total (a
// bisection on the order-preserving 64-bit image of the scores), then the
// entries at the threshold in ascending index until the target is met.
// Writes a bitmap.  With CACHED (N <= 32768) each thread keeps its 32
// scores for the 64 bisection steps, 4 in registers and 28 in shared memory
// (entries past N hold -1, which no threshold counts); otherwise every step
// re-reads them from global memory.  Both visit a thread's entries in the
// same order, so the result does not depend on the variant.
constexpr int kCutThreads = 1024;
constexpr int kCutRegs = 4;
constexpr int kCutSmem = 28;
constexpr int64_t kCutCachedMax = static_cast<int64_t>(kCutThreads) * (kCutRegs + kCutSmem);

template <bool CACHED>
__global__ void __launch_bounds__(kCutThreads) sample_cut_kernel(const double* __restrict__ col,
                                                                 const double* __restrict__ sl, int64_t N,
                                                                 double alpha, uint32_t* __restrict__ keep_col,
                                                                 uint32_t* __restrict__ keep_sl) {
  extern __shared__ double cache[];                            // CACHED: [kCutSmem][kCutThreads]
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
  double rv[kCutRegs];
  if (CACHED) {
#pragma unroll
    for (int i = 0; i < kCutRegs + kCutSmem; ++i) {
      const int64_t k = threadIdx.x + static_cast<int64_t>(i) * kCutThreads;
      const double v = k < N ? sc[k] : -1.0;
      if (i < kCutRegs) rv[i] = v;
      else cache[(i - kCutRegs) * kCutThreads + threadIdx.x] = v;
    }
  }
  // bisection for the largest t with mass(score image >= t) >= goal
  uint64_t lo = 0, hi = ~0ull;             // invariant: mass(>= lo) >= goal
  while (lo < hi) {
    const uint64_t mid = lo + (hi - lo) / 2 + 1;
    double part = 0.0;
    if (CACHED) {
#pragma unroll
      for (int i = 0; i < kCutRegs + kCutSmem; ++i) {
        const double v = i < kCutRegs ? rv[i] : cache[(i - kCutRegs) * kCutThreads + threadIdx.x];
        if (ordered_f64(v) >= mid) part += v;
      }
    } else {
      for (int64_t k = threadIdx.x; k < N; k += blockDim.x)
        if (ordered_f64(sc[k]) >= mid) part += sc[k];
    }
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
  // at the threshold: equal scores in ascending index while the accumulated
  // score is below the goal.  The number taken follows from the tie count
  // and the tie value; a block-wide scan then ranks the ties by index.
  double nt = 0.0;
  for (int64_t k = threadIdx.x; k < N; k += blockDim.x) nt += ordered_f64(sc[k]) == lo ? 1.0 : 0.0;
  const int64_t ntie = static_cast<int64_t>(block_sum(nt, red));
  const uint64_t ubits = (lo & 0x8000000000000000ull) ? (lo & ~0x8000000000000000ull) : ~lo;
  const double v = __longlong_as_double(static_cast<long long>(ubits));
  __shared__ int64_t need_sh;
  __shared__ int wcnt[32];
  if (threadIdx.x == 0) {
    double acc = above;
    int64_t n = 0;
    while (n < ntie && acc < goal) {
      acc += v;
      ++n;
    }
    need_sh = n;
  }
  __syncthreads();
  const int64_t need = need_sh;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  int64_t running = 0;
  for (int64_t base = 0; base < N && running < need; base += blockDim.x) {
    const int64_t k = base + threadIdx.x;
    const bool f = k < N && ordered_f64(sc[k]) == lo;
    const uint32_t bal = __ballot_sync(0xffffffffu, f);
    if (lane == 0) wcnt[warp] = __popc(bal);
    __syncthreads();
    int before = 0, tot = 0;
    for (int w = 0; w < nwarp; ++w) {
      before += w < warp ? wcnt[w] : 0;
      tot += wcnt[w];
    }
    const int64_t rank = running + before + __popc(bal & ((1u << lane) - 1u));
    if (f && rank < need) atomicOr(&keep[k >> 5], 1u << (k & 31));
    running += tot;
    __syncthreads();
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

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

// Tensor map of a [B, H, N, D] bf16 tensor for 64-column x 128-row boxes,
// 128-byte swizzle, rows past N read as zeros.  The stride of an extent-1
// dimension is never used, so it is replaced by a valid one; a zero stride
// over several heads or batches (a broadcast view) is not supported.
bool encode_rows_map(CUtensorMap* map, const TensorDesc& t) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t sn = static_cast<cuuint64_t>(t.sN) * 2;
  cuuint64_t sh = t.H > 1 ? static_cast<cuuint64_t>(t.sH) * 2 : sn * static_cast<cuuint64_t>(t.N);
  cuuint64_t sb = t.B > 1 ? static_cast<cuuint64_t>(t.sB) * 2 : sh * static_cast<cuuint64_t>(t.H);
  if (sh == 0 || sb == 0) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(t.D), static_cast<cuuint64_t>(t.N), static_cast<cuuint64_t>(t.H),
                        static_cast<cuuint64_t>(t.B)};
  cuuint64_t strides[3] = {sn, sh, sb};
  cuuint32_t box[4] = {64, 128, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(t.ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_select_sample(const SelectParams& p, const TensorDesc& Q, const TensorDesc& K,
                                 float scale_log2, double* col, double* sl, uint32_t* keep_col,
                                 uint32_t* keep_sl, int32_t* counts, int32_t* idx, int* err, cudaStream_t s) {
  const size_t nsc = static_cast<size_t>(p.B) * p.Hq * p.N;
  cudaError_t e = cudaMemsetAsync(col, 0, nsc * sizeof(double), s);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(sl, 0, nsc * sizeof(double), s);
  if (e != cudaSuccess) return e;
  const int nseg = static_cast<int>((p.N + p.seg - 1) / p.seg);
  const unsigned nblk = static_cast<unsigned>(static_cast<int64_t>(nseg) * p.B * p.Hq);   // < 2^31, checked
  CUtensorMap mq, mk;
  if (!encode_rows_map(&mq, Q) || !encode_rows_map(&mk, K)) return cudaErrorNotSupported;
  auto run = [&](auto kernel, int smem_bytes) -> cudaError_t {
    cudaError_t e2 = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e2 != cudaSuccess) return e2;
    kernel<<<nblk, kScoreThreads, smem_bytes, s>>>(mq, mk, p.N, p.B, p.Hq, p.Hq / p.Hkv, p.blk, p.seg, scale_log2,
                                                    col, sl, err);
    return cudaGetLastError();
  };
  e = p.D == 64 ? run(sample_scores_kernel<64>, SampleCfg<64>::kSmem)
                : run(sample_scores_kernel<128>, SampleCfg<128>::kSmem);
  if (e != cudaSuccess) return e;
  dim3 g2(2, static_cast<unsigned>(p.Hq), static_cast<unsigned>(p.B));
  if (p.N <= kCutCachedMax) {
    const int cache_bytes = kCutSmem * kCutThreads * static_cast<int>(sizeof(double));
    e = cudaFuncSetAttribute(sample_cut_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, cache_bytes);
    if (e != cudaSuccess) return e;
    sample_cut_kernel<true><<<g2, kCutThreads, cache_bytes, s>>>(col, sl, p.N, p.tau, keep_col, keep_sl);
  } else {
    sample_cut_kernel<false><<<g2, kCutThreads, 0, s>>>(col, sl, p.N, p.tau, keep_col, keep_sl);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t rows = static_cast<int64_t>(p.B) * p.Hq * p.nb;
  sample_lists_kernel<<<static_cast<unsigned>((rows + kSampleWarps - 1) / kSampleWarps), kSampleWarps * 32, 0,
                        s>>>(p, keep_col, keep_sl, counts, idx, err);
  return cudaGetLastError();
}

}  // namespace pbs
