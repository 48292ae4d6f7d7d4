// pbs_attn_fwd: FlashAttention-style forward over an online key permutation.
//
// "S2O: Early Stopping for Sparse Attention via Online Permutation",
// Technical Summary:
//   1. Online Permutation via Index-Driven Loading -- K/V stay in their HBM
//      layout; an index list says which (non-contiguous) rows to load, and
//      the kernel gathers those rows into on-chip memory;
//   3. Kernel Implementation -- Pass 1 runs dense causal attention over the
//      query block's own segment and builds the online-softmax state
//      (m, l, acc); Pass 2 continues from that state over earlier key blocks
//      in permuted order.
// "Block Sparse Flash Attention", Approach: the exact tile maximum of QK^T
// is compared with a per-(head, query block) threshold; below it the tile
// adds nothing (no PV product, no softmax update).
// S2O page, 2. Early-Stopping Rule (pbs_attn_fwd_early_stop): Pass 2 visits
// each head's listed blocks in the order given and ends once every row's
// marginal gain (the tile's exponential mass over the accumulated mass) is
// below a threshold.
//
// sm_100a design.  One CTA per work item = (query block i, batch b, a pair
// of query heads h0, h0+1 of the same GQA group).  The two heads share K/V,
// so the CTA walks the UNION of their tile lists (the own segment's natural
// blocks, then the listed permuted blocks in ascending order) and gathers
// every K/V tile once for both heads.  (With early stopping the two heads'
// ordered lists are interleaved instead, each tile serving one head.)
// Roles (384 threads):
//   warp 0       tcgen05 MMA issuer (one thread) and tensor-memory owner;
//   warps 1-3    producer: Q once and the K and V tiles into 2-stage rings
//                of 128B-swizzled tiles -- by TMA where a tile's rows are
//                contiguous (Q, natural blocks, in-order permuted blocks),
//                else by 16-byte cp.async row gathers;
//   warps 4-7    softmax for head slot 0, warps 8-11 for head slot 1: each
//                thread owns one query row of S and O in tensor memory.
// Tensor memory (512 columns): S0 | S1 | O0 | O1, 128 columns each; P (bf16)
// overwrites the first half of S and feeds PV as the A operand straight
// from tensor memory.  K and V have separate 2-stage rings: a K stage is
// released as soon as the QK^T of its tile are done, a V stage after the
// PVs, so each gather has about two tiles of time to land.  The MMA thread
// is event driven: it issues whichever QK^T or PV is ready, so that while
// one softmax warpgroup works on its tile the tensor core works for the
// other head.  Causal tiles only mask columns to -inf and then take the
// same softmax pass as every other tile.  All waits are bounded; a shared
// abort flag makes every role of the CTA give up together.
#include <math.h>

#include <algorithm>

#include "pbs_common.cuh"
#include "pbs_internal.h"

namespace pbs {
namespace {

constexpr int kThreads = 384;
constexpr int kM = 128;               // query rows per MMA tile
constexpr int kProducerThreads = 96;  // warps 1-3
constexpr int kStages = 2;
constexpr float kRescaleSlack = 8.0f; // keep the running max while within 2^8

template <int D, int BLK>
struct Cfg {
  static constexpr int kQBytes = (D / 64) * kM * 128;
  static constexpr int kKVBytes = (D / 64) * BLK * 128;
  static constexpr int kQ0 = 0;
  static constexpr int kK = 2 * kQBytes;
  static constexpr int kV = kK + kStages * kKVBytes;
  static constexpr int kEnd = kV + kStages * kKVBytes;
  // Above half the SM's shared memory, so one CTA per SM: its 512 tensor-
  // memory columns are then always available and tcgen05.alloc never waits.
  static constexpr int kMinSmem = 120 * 1024;
};

// Rare softmax paths, kept out of line so that the softmax loop's
// instruction footprint stays small (called by whole warps).
// Rescale the first n16 x 16 P columns of this tile (bf16 pairs) by beta,
// after this thread's earlier P stores have landed.
__device__ __noinline__ void rescale_p(uint32_t tS, int n16, float beta) {
  tmem_st_wait();
  for (int q = 0; q < n16; ++q) {
    uint32_t w[16];
    tmem_ld16(tS + q * 16, w);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
      w[e] = pack_bf16x2(f.x * beta, f.y * beta);
    }
    tmem_st16(tS + q * 16, w);
  }
}
// Rescale this row's O accumulator (D fp32 columns) by alpha.
template <int D>
__device__ __noinline__ void rescale_o(uint32_t tO, float alpha) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t u[32];
    tmem_ld32(tO + c * 32, u);
#pragma unroll
    for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
    tmem_st32(tO + c * 32, u);
  }
}

__device__ __forceinline__ float warp_max(float v) {
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

struct Shared {
  uint64_t bar_q;
  uint64_t bar_k[kStages], bar_v[kStages], bar_kempty[kStages], bar_vempty[kStages];
  uint64_t bar_s[2], bar_p[2], bar_o[2], bar_fin;
  uint64_t bar_sched;      // the schedule is built (the LAZY kernels)
  uint32_t tmem_base;
  int abort;
  int n_union;
  int jtop;                // last natural block of Pass 1
  int skip[2][2];
  float red[2][4];
  int vote[2][4];          // early stopping: per-warp "every row's gain is small"
  int limit[2];            // early stopping: a head runs none of its tiles >= limit
  int n_list[2];           // early stopping: listed tiles per head slot
};

// QP: S2O query permutation -- row r of query block i is the query at
// qperm[i*BLK + r] (both heads' rows from their own qperm rows), Pass 1 runs
// the natural blocks of the own segment up to the last of those queries
// with an element-wise causal mask, and O / LSE go back to the queries'
// positions.
// ES: S2O early stopping -- each head's listed blocks are visited in the
// order given and its Pass 2 is cut once a tile's gain is small.  The two
// heads' lists are interleaved (one tile of each in turn, every tile for one
// head); tiles of a head that has stopped are not loaded and only passed
// through the rings.
template <int D, int BLK, bool ES, bool QP, bool GT, bool LZ>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(AttnParams p, const __grid_constant__ CUtensorMap mq,
                                                                const __grid_constant__ CUtensorMap mk,
                                                                const __grid_constant__ CUtensorMap mv) {
  using C = Cfg<D, BLK>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint32_t* sched = reinterpret_cast<uint32_t*>(smem + C::kEnd);
  __shared__ Shared sh;
  __shared__ uint32_t bm[2][256];          // candidate bitmaps (ncand <= 8192)
  __shared__ int32_t rowbuf[kStages][BLK];
  __shared__ int32_t qpos[2][QP ? BLK : 1];  // QP: the query position of each row

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hq = p.G * static_cast<int>(p.K.H);
  const int npair = (p.G + 1) / 2;
  // Work order: all items of one (batch, KV head) before the next, so that
  // head's K/V (the tiles every item gathers) stays resident in L2; within
  // it, heavy query blocks (more tiles) first, then the head pair.
  const int per_bh = p.nb * npair;
  const int bh = static_cast<int>(blockIdx.x) / per_bh;
  const int rem = static_cast<int>(blockIdx.x) % per_bh;
  const int i = p.nb - 1 - rem / npair;
  const int pr = rem % npair;
  const int b = bh / static_cast<int>(p.K.H);
  const int hk = bh % static_cast<int>(p.K.H);
  const int h0 = hk * p.G + 2 * pr;
  const bool has1 = 2 * pr + 1 < p.G;
  const int spb = p.seg / BLK;
  const int s = i / spb;
  const int ncand = s * spb;
  const int64_t q0 = static_cast<int64_t>(i) * BLK;
  const int64_t N = p.Q.N;

  const uint32_t sQ0 = smem_u32(smem + C::kQ0);
  const uint32_t sK = smem_u32(smem + C::kK);
  const uint32_t sV = smem_u32(smem + C::kV);

  // ------------------------------------------------------------------ setup
  // Barriers first, so that the loads that need no schedule -- Q and, in
  // natural query order, the diagonal block's K and V (tile 0) -- start by
  // TMA while the schedule is being built.
  if (tid == 32) {
    sh.abort = 0;
    sh.limit[0] = 0x7fffffff;
    sh.limit[1] = 0x7fffffff;
    mbar_init(&sh.bar_q, kProducerThreads);
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&sh.bar_k[st], kProducerThreads);
      mbar_init(&sh.bar_v[st], kProducerThreads);
      mbar_init(&sh.bar_kempty[st], 1);
      mbar_init(&sh.bar_vempty[st], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&sh.bar_s[h], 1);
      mbar_init(&sh.bar_p[h], 4);               // one arrival per softmax warp
      mbar_init(&sh.bar_o[h], 1);
    }
    mbar_init(&sh.bar_fin, 1);
    mbar_init(&sh.bar_sched, 32);               // every lane of the building warp
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  // (the failure-path test hook withholds the Q loads; with early stopping
  // warp 0 compacts the lists in the V ring during set-up, so tile 0 waits)
  const bool early = p.tma && !QP && !p.test_wait_limit;
  const bool early_kv = early && !ES;
  if (tid == 32 && early) {
    mbar_expect_tx(&sh.bar_q, static_cast<uint32_t>((has1 ? 2 : 1) * C::kQBytes));
    for (int h = 0; h < (has1 ? 2 : 1); ++h)
      for (int c = 0; c < D / 64; ++c)
        tma_rows_4d(sQ0 + h * C::kQBytes + c * (kM * 128), &mq, c * 64, static_cast<int>(q0), h0 + h, b, &sh.bar_q);
  }
  if (tid == 32 && early_kv) {
    mbar_expect_tx(&sh.bar_k[0], static_cast<uint32_t>(C::kKVBytes));
    for (int c = 0; c < D / 64; ++c)
      tma_rows_4d(sK + c * (BLK * 128), &mk, c * 64, i * BLK, hk, b, &sh.bar_k[0]);
    mbar_expect_tx(&sh.bar_v[0], static_cast<uint32_t>(C::kKVBytes));
    for (int c = 0; c < D / 64; ++c)
      tma_rows_4d(sV + c * (BLK * 128), &mv, c * 64, i * BLK, hk, b, &sh.bar_v[0]);
  }
  // LAZY (natural query order, no early stopping, no gate): a producer warp builds
  // the schedule while the diagonal tile -- block i itself, natural, both
  // heads, needing no schedule -- already runs: its QK^T, softmax and PV go
  // ahead, and each role waits for the schedule only when it needs the tiles
  // after it.  Otherwise warp 0 builds it before anything starts.
  // (chosen by the launcher where the own segment holds more than the
  // diagonal block; with one block per segment, as in the gate workloads and
  // the dense run, and with the gate it measured slower)
  constexpr bool LAZY = LZ && !QP && !ES && !GT;
  auto build_schedule = [&]() {
    // union of the two heads' lists as a bitmap, then an ascending schedule
    int cnt[2] = {0, 0};
    for (int h = 0; h < 2; ++h) {
      if (h == 1 && !has1) break;
      const int64_t row = (static_cast<int64_t>(b) * Hq + h0 + h) * p.nb + i;
      int c = p.counts[row];
      if (c < 0 || c > p.cap) {
        if (lane == 0) set_error(p.err, kErrDeviceCheck);
        c = 0;
      }
      cnt[h] = c;
    }
    const int words = (ncand + 31) >> 5;
    for (int w = lane; w < words; w += 32) {
      bm[0][w] = 0u;
      bm[1][w] = 0u;
    }
    __syncwarp();
    int total = 0;
    if (ES) {
      // Each head's list in the order given (out-of-range and repeated
      // entries dropped and flagged), compacted into the V ring, which is
      // free until the producer starts; then interleaved: the k-th tiles of
      // the two heads at 2k and 2k+1 while both lists last.
      int32_t* scratch = reinterpret_cast<int32_t*>(smem + C::kV);
      int nl[2] = {0, 0};
      for (int h = 0; h < 2; ++h) {
        const int32_t* list = p.idx + ((static_cast<int64_t>(b) * Hq + h0 + h) * p.nb + i) * p.cap;
        for (int base = 0; base < cnt[h]; base += 32) {
          const int e = base + lane;
          bool keep = false;
          int pb = 0;
          if (e < cnt[h]) {
            pb = list[e];
            if (pb < 0 || pb >= ncand) {
              set_error(p.err, kErrDeviceCheck);
            } else if (atomicOr(&bm[h][pb >> 5], 1u << (pb & 31)) & (1u << (pb & 31))) {
              set_error(p.err, kErrDeviceCheck);
            } else {
              keep = true;
            }
          }
          const uint32_t km = __ballot_sync(0xffffffffu, keep);
          if (keep) scratch[h * p.cap + nl[h] + __popc(km & ((1u << lane) - 1u))] = pb;
          nl[h] += __popc(km);
        }
      }
      __syncwarp();
      const int m = min(nl[0], nl[1]);
      for (int h = 0; h < 2; ++h)
        for (int e = lane; e < nl[h]; e += 32)
          sched[e < m ? 2 * e + h : m + e] = static_cast<uint32_t>(scratch[h * p.cap + e]) | ((1u << h) << 30);
      total = nl[0] + nl[1];
      if (lane == 0) {
        sh.n_list[0] = nl[0];
        sh.n_list[1] = nl[1];
      }
    }
    if (!ES) {
      // both heads' entries in batches of 8 per lane, all loads in flight
      // before the first is used (one memory round trip per 256 entries)
      constexpr int kBatch = 8;
      const int32_t* list0 = p.idx + ((static_cast<int64_t>(b) * Hq + h0) * p.nb + i) * p.cap;
      const int32_t* list1 = list0 + static_cast<int64_t>(p.nb) * p.cap;   // next head's row (read only if cnt[1] > 0)
      for (int base = 0; base < max(cnt[0], cnt[1]); base += 32 * kBatch) {
        int pb[2][kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
          const int e = base + lane + 32 * j;
          pb[0][j] = e < cnt[0] ? list0[e] : 0;
          pb[1][j] = e < cnt[1] ? list1[e] : 0;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int j = 0; j < kBatch; ++j) {
            if (base + lane + 32 * j >= cnt[h]) continue;
            const int v = pb[h][j];
            if (v < 0 || v >= ncand) {
              set_error(p.err, kErrDeviceCheck);
              continue;
            }
            atomicOr(&bm[h][v >> 5], 1u << (v & 31));
          }
        }
      }
    }
    __syncwarp();
    for (int base = 0; base < words && !ES; base += 32) {
      const int w = base + lane;
      const uint32_t m0 = w < words ? bm[0][w] : 0u, m1 = w < words ? bm[1][w] : 0u;
      uint32_t u = m0 | m1;
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
        const uint32_t mask = ((m0 >> bit) & 1u) | (((m1 >> bit) & 1u) << 1);
        sched[o++] = static_cast<uint32_t>(w * 32 + bit) | (mask << 30);
      }
      total += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      sh.n_union = total;
      sh.jtop = i;
    }
    if (QP) {
      // Rows' query positions (each must lie in the block's segment; an
      // entry outside it sets the error word and is replaced by the
      // segment's first position) and the last natural block they reach.
      const int64_t seg_lo = static_cast<int64_t>(s) * p.seg, seg_hi = min(seg_lo + p.seg, N);
      int64_t mx = seg_lo;
      for (int h = 0; h < (has1 ? 2 : 1); ++h) {
        const int32_t* qrow = p.qperm + (static_cast<int64_t>(b) * Hq + h0 + h) * N + q0;
        for (int r = lane; r < BLK; r += 32) {
          int64_t x = qrow[r];
          if (x < seg_lo || x >= seg_hi) {
            set_error(p.err, kErrDeviceCheck);
            x = seg_lo;
          }
          qpos[h][r] = static_cast<int32_t>(x);
          mx = max(mx, x);
        }
      }
      for (int off = 16; off > 0; off >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      if (lane == 0) sh.jtop = static_cast<int>(mx / BLK);
    }
    if (LAZY) {
      __syncwarp();
      mbar_arrive(&sh.bar_sched);               // each lane: its schedule writes are released
    }
  };
  if (!LAZY && warp == 0) build_schedule();
  if (!LAZY) {
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  // Pass 1 runs natural blocks jtop, jtop - 1, ..., down to the segment's
  // first; jtop is i itself unless queries are permuted.
  const int jtop = QP ? sh.jtop : i;
  const int n_diag = jtop - s * spb + 1;
  // tiles of the item (LAZY: known to each role once it has waited for the schedule)
  int T = LAZY ? 0 : n_diag + sh.n_union;
  // Poll limit of the role waits (the drain before tensor memory is freed
  // keeps the full limit).
  const uint32_t lim = p.test_wait_limit ? p.test_wait_limit : kSpinLimit;
  const uint32_t both = has1 ? 3u : 1u;
  volatile int* abort_flag = &sh.abort;
  volatile int* limit = sh.limit;
  // tile t: natural block i-t for t < n_diag, else sched[t - n_diag]
  auto tile_mask = [&](int t) -> uint32_t { return t < n_diag ? both : (sched[t - n_diag] >> 30); };
  // Early stopping: does tile t still serve a head (t below that head's
  // stop point)?  Heads that stopped have limit <= t.
  auto live = [&](int t) -> bool {
    const uint32_t m = tile_mask(t);
    return ((m & 1u) && t < limit[0]) || ((m & 2u) && t < limit[1]);
  };
  // ... and is tile t, and every tile after it, past every head's stop point?
  auto past_all = [&](int t) -> bool { return t >= limit[0] && (!has1 || t >= limit[1]); };

  if (warp >= 1 && warp <= 3) {
    // ============================================================ producer
    const int pt = tid - 32;
    const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(p.K.ptr) + b * p.K.sB + hk * p.K.sH;
    const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(p.V.ptr) + b * p.V.sB + hk * p.V.sH;
    // the key permutation this query block reads: its KV head's, or with one
    // permutation per query segment, its segment's
    const int32_t* prow =
        p.perm + ((static_cast<int64_t>(b) * p.K.H + hk) * p.perm_nseg + (p.perm_nseg > 1 ? s : 0)) * N;
    constexpr int CH = D / 8;
    // Tile gathers: thread pt always copies 16-byte chunk c of rows r0,
    // r0 + RPP, r0 + 2 RPP, ... (RPP rows per pass of the 96 threads).  A
    // tile's row indices are read from shared memory all at once before its
    // copies are issued, so the copies go out back to back instead of each
    // waiting on its own index load.
    constexpr int RPP = kProducerThreads / CH, NIT = (BLK + RPP - 1) / RPP;
    static_assert(kProducerThreads % CH == 0, "producer threads cover whole rows");
    const int cc = pt % CH, r0 = pt / CH;
    const uint32_t cc_off = static_cast<uint32_t>((cc / 8) * (BLK * 128));
    auto gather_tile = [&](uint32_t dst, const __nv_bfloat16* base, int64_t sN, const int32_t* rows) {
      int32_t x[NIT];
#pragma unroll
      for (int k = 0; k < NIT; ++k) x[k] = r0 + RPP * k < BLK ? rows[r0 + RPP * k] : 0;
#pragma unroll
      for (int k = 0; k < NIT; ++k) {
        const int r = r0 + RPP * k;
        if (r < BLK) cp_async16(dst + cc_off + sw128_offset(r, cc % 8), base + x[k] * sN + cc * 8);
      }
    };
    // Q tiles of both heads: by TMA (one thread, 64-column boxes) where the
    // rows are contiguous, else by cp.async (rows >= BLK zero-filled when
    // BLK < 128; with permuted queries each row from its own position).
    const bool tma_q = p.tma && !QP;
    if (tma_q) {
      // thread 0 issued the Q boxes during set-up; the others arrive
      if (pt != 0 && !p.test_wait_limit) mbar_arrive(&sh.bar_q);
    }
    for (int h = 0; h < (has1 ? 2 : 1) && !tma_q; ++h) {
      const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(p.Q.ptr) + b * p.Q.sB + (h0 + h) * p.Q.sH;
      const uint32_t dst = sQ0 + h * C::kQBytes;
      for (int id = pt; id < kM * CH; id += kProducerThreads) {
        const int r = id / CH, c = id % CH;
        const bool valid = r < BLK;
        cp_async16_zfill(dst + (c / 8) * (kM * 128) + sw128_offset(r, c % 8),
                         valid ? qb + (QP ? static_cast<int64_t>(qpos[h][r]) : q0 + r) * p.Q.sN + c * 8 : qb,
                         valid);
      }
    }
    // (the failure-path test hook withholds this arrival, so the MMA role's
    // wait for Q runs out)
    if (!p.test_wait_limit && !tma_q) cp_async_mbar_arrive(&sh.bar_q);
    if constexpr (LAZY) {
      if (warp == 2) build_schedule();
      named_sync(1, kProducerThreads);          // the schedule is built
      T = n_diag + sh.n_union;
    }
    // A tile of BLK contiguous rows (from row0) by TMA: one thread announces
    // the bytes and issues the 64-column boxes; the other producer threads
    // arrive.
    auto tma_tile = [&](uint64_t* bar, uint32_t dst, const CUtensorMap* map, int row0, bool issued) {
      if (pt == 0) {
        if (issued) return;                  // tile 0's boxes went out during set-up
        mbar_expect_tx(bar, static_cast<uint32_t>(C::kKVBytes));
        for (int c = 0; c < D / 64; ++c) tma_rows_4d(dst + c * (BLK * 128), map, c * 64, row0, hk, b, bar);
      } else {
        mbar_arrive(bar);
      }
    };
    // Row indices of a tile: natural rows, or the permutation's entries for
    // a permuted block.  Loaded one tile ahead into registers and checked
    // when used, so the load latency overlaps the previous tile.
    constexpr int RPT = (BLK + kProducerThreads - 1) / kProducerThreads;
    int32_t nxt[RPT];
    auto fetch_rows = [&](int t) {
#pragma unroll
      for (int q = 0; q < RPT; ++q) {
        const int r = pt + q * kProducerThreads;
        if (r < BLK && t >= n_diag)
          nxt[q] = prow[static_cast<int64_t>(sched[t - n_diag] & 0x3FFFFFFFu) * BLK + r];
      }
    };
    if (T > 0) fetch_rows(0);
    // Bounded wait for a ring slot.  With early stopping it also ends once
    // the tile to be loaded is past every head's stop point: from there on
    // nothing is run.
    auto wait_slot = [&](uint64_t* bar, uint32_t parity, int t) -> bool {
      if constexpr (!ES) {
        return mbar_wait_or_abort(bar, parity, p.err, abort_flag, lim);
      } else {
        for (uint32_t it = 0; it < lim; ++it) {
          if (mbar_try_wait(bar, parity)) return true;
          if ((it & 15u) == 15u && (*abort_flag || past_all(t))) return false;
        }
        set_error(p.err, kErrTimeout);
        *abort_flag = 1;
        return false;
      }
    };
    // V of tile t is gathered right after its K, also under gating: the
    // gate decides only after the tile's QK^T, and waiting for the decision
    // would put the gather's latency in front of every kept tile's PV.
    // (A dropped tile's V is gathered but never multiplied.)
    for (int t = 0; t < T; ++t) {
      // first row of the tile when its rows are contiguous (natural blocks;
      // a permuted block whose entries happen to run in order, as with the
      // identity permutation), loaded by TMA; else -1 and gathered row by row
      int row0 = -1;
      {                                           // K of tile t
        const int st = t & 1;
        const bool ok = t < kStages || wait_slot(&sh.bar_kempty[st], ((t >> 1) - 1) & 1, t);
        if (named_sync_or(1, kProducerThreads, !ok)) break;   // all producer threads leave together
        const bool nat = t < n_diag;
        const int id0 = nat ? jtop - t : static_cast<int>(sched[t - n_diag] & 0x3FFFFFFFu);
        // a permuted block lies inside one segment (seg is a multiple of BLK)
        const int64_t lo = static_cast<int64_t>((id0 * BLK) / p.seg) * p.seg;
#pragma unroll
        for (int q = 0; q < RPT; ++q) {
          const int r = pt + q * kProducerThreads;
          if (r >= BLK) continue;
          int64_t x;
          if (nat) {
            x = static_cast<int64_t>(id0) * BLK + r;
          } else {
            x = nxt[q];
            if (x < lo || x >= lo + p.seg || x >= N) {
              set_error(p.err, kErrDeviceCheck);
              x = lo;
            }
          }
          rowbuf[st][r] = static_cast<int32_t>(x);
        }
        named_sync(1, kProducerThreads);
        if (nat) row0 = id0 * BLK;
        if constexpr (!ES) {
          if (p.tma && !nat) {
            const int32_t x0 = rowbuf[st][0];
            bool run = true;
#pragma unroll
            for (int q = 0; q < RPT; ++q) {
              const int r = pt + q * kProducerThreads;
              if (r < BLK) run = run && rowbuf[st][r] == x0 + r;
            }
            if (!named_sync_or(1, kProducerThreads, !run)) row0 = x0;
          }
        }
        if (p.tma && row0 >= 0) {
          tma_tile(&sh.bar_k[st], sK + st * C::kKVBytes, &mk, row0, early_kv && t == 0);
        } else {
          if (!ES || live(t)) gather_tile(sK + st * C::kKVBytes, kb, p.K.sN, rowbuf[st]);
          cp_async_mbar_arrive(&sh.bar_k[st]);    // arrives when this thread's copies land
        }
      }
      {                                           // V of tile t
        const int sv = t & 1;
        const bool okv = t < kStages || wait_slot(&sh.bar_vempty[sv], ((t >> 1) - 1) & 1, t);
        if (named_sync_or(1, kProducerThreads, !okv)) break;
        if (p.tma && row0 >= 0) {
          tma_tile(&sh.bar_v[sv], sV + sv * C::kKVBytes, &mv, row0, early_kv && t == 0);
        } else {
          if (!ES || live(t)) gather_tile(sV + sv * C::kKVBytes, vb, p.V.sN, rowbuf[sv]);
          cp_async_mbar_arrive(&sh.bar_v[sv]);
        }
      }
      if (t + 1 < T) fetch_rows(t + 1);
    }
    cp_async_wait_all();
  } else if (warp == 0) {
    // ========================================================= MMA issuer
    // The whole warp runs the issue loop with warp-uniform state, so MMA
    // descriptors stay warp-uniform; lane 0 observes each barrier (and so
    // acquires the data) and alone issues the MMAs and commits.
    const bool leader = lane == 0;
    auto test = [&](uint64_t* bar, uint32_t parity) -> bool {
      bool v = false;
      if (leader) v = mbar_test_wait(bar, parity);
      return __shfl_sync(0xffffffffu, v, 0);
    };
    bool ok = true;
    {
      bool v = true;
      if (leader) v = mbar_wait_or_abort(&sh.bar_q, 0, p.err, abort_flag, lim);
      ok = __shfl_sync(0xffffffffu, v, 0);
      if (leader) fence_proxy_async();   // cp.async (generic proxy) writes -> tensor-core reads
      tc_fence_after();
    }
    {
      constexpr uint32_t idesc_qk = idesc_bf16(kM, BLK, false);
      constexpr uint32_t idesc_pv = idesc_bf16(kM, D, true);
      const int nh = has1 ? 2 : 1;
      // All loop state lives in registers: per-head arrays are indexed only
      // by the unrolled head loop's constant, per-stage values are separate
      // scalars chosen by the stage bit.
      // LAZY: a first pass of the event loop runs tile 0 alone (T = 1 here),
      // then the schedule is awaited and the loop goes on over every tile.
      bool phase_a = LAZY;
      if (phase_a) T = 1;
      // Per head: next tile needing QK^T, tile whose PV is pending, QK count.
      int nq[2] = {T, T}, pend[2] = {-1, -1}, kh[2] = {0, 0};
      bool o_init[2] = {false, false};
      // Early stopping: head stopped; its next tile's K fill already passed on.
      bool hstop[2] = {false, false}, kpassed[2] = {false, false};
      auto next_tile = [&](int h, int from) {
        int t = from;
        while (t < T && !((tile_mask(t) >> h) & 1u)) ++t;
        return t;
      };
#pragma unroll
      for (int h = 0; h < 2; ++h)
        if (h < nh) nq[h] = next_tile(h, 0);
      // Per ring stage: the tile it holds and how many heads still need it,
      // and how many of its fill phases have been observed.  A stage holds
      // tiles st, st+2, st+4, ... in turn; a tile's phase is tested only when
      // it is the next one due on its stage, since a parity test cannot tell
      // a phase two fills ahead from the current one.
      int kt0 = -1, kt1 = -1, kl0 = 0, kl1 = 0, ks0 = 0, ks1 = 0;
      int vt0 = -1, vt1 = -1, vl0 = 0, vl1 = 0, vs0 = 0, vs1 = 0;
      auto landed = [&](uint64_t* bars, int& seen0, int& seen1, int t) -> bool {
        const int st = t & 1;
        const int seen = st ? seen1 : seen0;
        const int due = st + 2 * seen;
        if (t < due) return true;                        // observed earlier, still held
        if (t > due) return false;                       // an earlier fill is not observed yet
        if (!test(&bars[st], seen & 1)) return false;
        if (st) seen1 = seen + 1; else seen0 = seen + 1;
        if (leader) fence_proxy_async();                 // fill's cp.async writes -> tensor-core reads
        return true;
      };
      // One more head done with tile t on its stage; true when it was the
      // last head that needed it (the stage may then be refilled).
      auto release = [&](int& tile0, int& tile1, int& left0, int& left1, int t) -> bool {
        const int st = t & 1;
        int left = st ? left1 : left0;
        if ((st ? tile1 : tile0) != t) {
          if (st) tile1 = t; else tile0 = t;
          left = __popc(tile_mask(t));
        }
        --left;
        if (st) left1 = left; else left0 = left;
        return left == 0;
      };
      uint32_t idle = 0;
      // Event-driven issue: whichever of PV_h (P ready, V landed) or QK_h
      // (previous PV_h issued, K landed) can go, goes.  QK_h(t) is always
      // issued after PV_h of the head's previous tile, so P (which lives in
      // S's columns) has been consumed before S is overwritten.
      for (;;) {
      while (ok) {
        bool pending = false, progress = false;
        const bool all_stopped = ES && hstop[0] && (nh < 2 || hstop[1]);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h >= nh) break;
          if (ES && hstop[h]) {
            // A stopped head runs nothing more, but each of its remaining
            // tiles still occupies a ring slot in turn: pass the K and then
            // the V fill on as they land (until every head has stopped).
            if (nq[h] < T && !all_stopped) {
              pending = true;
              const int t = nq[h], st = t & 1;
              if (!kpassed[h] && landed(sh.bar_k, ks0, ks1, t)) {
                if (release(kt0, kt1, kl0, kl1, t) && elect_one()) tc_commit(&sh.bar_kempty[st]);
                kpassed[h] = true;
                progress = true;
              }
              if (kpassed[h] && landed(sh.bar_v, vs0, vs1, t)) {
                if (release(vt0, vt1, vl0, vl1, t) && elect_one()) tc_commit(&sh.bar_vempty[st]);
                kpassed[h] = false;
                nq[h] = next_tile(h, t + 1);
                progress = true;
              }
            }
            continue;
          }
          if (pend[h] >= 0) {
            pending = true;
            const int t = pend[h], st = t & 1;
            if (test(&sh.bar_p[h], (kh[h] - 1) & 1) && landed(sh.bar_v, vs0, vs1, t)) {
              tc_fence_after();
              int skip = 0;
              if (leader) skip = sh.skip[h][(kh[h] - 1) & 1];      // lane 0 acquired bar_p
              if (!__shfl_sync(0xffffffffu, skip, 0)) {
                const uint32_t tP = tmem + h * 128;
                const uint32_t tO = tmem + 256 + h * 128;
                const uint32_t vbase = sV + st * C::kKVBytes;
                const uint64_t bd0 = sdesc_sw128(vbase, BLK * 128, 1024);
                const uint32_t acc0 = o_init[h] ? 1u : 0u;
#pragma unroll
                for (int kk = 0; kk < BLK / 16; ++kk) {
                  const uint64_t bd = sdesc_add(bd0, kk * 2048);
                  if (elect_one()) mma_ts(tO, tP + kk * 8, bd, idesc_pv, kk > 0 ? 1u : acc0);
                }
                o_init[h] = true;
              }
              if (release(vt0, vt1, vl0, vl1, t) && elect_one()) tc_commit(&sh.bar_vempty[st]);
              pend[h] = -1;
              progress = true;
              if (ES) {
                // lane 0 acquired bar_p, after which the stop point this
                // tile's softmax pass may have set is visible
                int lim = 0;
                if (leader) lim = limit[h];
                hstop[h] = __shfl_sync(0xffffffffu, lim, 0) <= t + 1;
              }
            }
          }
          if (pend[h] < 0 && nq[h] < T && !(ES && hstop[h])) {
            pending = true;
            const int t = nq[h], st = t & 1;
            if (landed(sh.bar_k, ks0, ks1, t)) {
              tc_fence_after();
              const uint32_t qbase = sQ0 + h * C::kQBytes;
              const uint32_t kbase = sK + st * C::kKVBytes;
              const uint32_t tS = tmem + h * 128;
              const uint64_t a0 = sdesc_sw128(qbase, 16, 1024);
              const uint64_t b0 = sdesc_sw128(kbase, 16, 1024);
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t half = kk / 4, koff = (kk % 4) * 32;
                const uint64_t ad = sdesc_add(a0, half * (kM * 128) + koff);
                const uint64_t bd = sdesc_add(b0, half * (BLK * 128) + koff);
                if (elect_one()) mma_ss(tS, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
              }
              if (elect_one()) tc_commit(&sh.bar_s[h]);
              ++kh[h];
              if (release(kt0, kt1, kl0, kl1, t) && elect_one()) tc_commit(&sh.bar_kempty[st]);
              pend[h] = t;
              nq[h] = next_tile(h, t + 1);
              progress = true;
            }
          }
        }
        if (!pending) break;
        if (progress) {
          idle = 0;
        } else if (++idle >= 4u * lim) {
          if (leader) {
            set_error(p.err, kErrTimeout);
            *abort_flag = 1;
          }
          ok = false;
        } else if ((idle & 63u) == 0) {
          ok = !__shfl_sync(0xffffffffu, *abort_flag, 0);
        }
      }
      if (phase_a && ok) {
        // tile 0 is done (its PV issued): wait for the schedule, go on from tile 1
        phase_a = false;
        // (every lane waits, so each has acquired the schedule)
        ok = __all_sync(0xffffffffu, mbar_wait_or_abort(&sh.bar_sched, 0, p.err, abort_flag, lim));
        if (ok) {
          T = n_diag + sh.n_union;
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (h < nh) nq[h] = next_tile(h, 1);
          continue;
        }
      }
      break;
      }
      if (leader) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
          if (h < nh && kh[h] > 0) tc_commit(&sh.bar_o[h]);
        tc_commit(&sh.bar_fin);
        // drain: every MMA of this CTA has completed before tensor memory is freed
        mbar_wait(&sh.bar_fin, 0, p.err);
      }
    }
    __syncwarp();
  } else {
    // ============================================================ softmax
    const int h = (warp - 4) >> 2;                  // head slot
    const int r = tid - 128 - h * 128;              // query row = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + h * 128 + lane_off;
    const uint32_t tO = tmem + 256 + h * 128 + lane_off;
    const int hq = h0 + h;
    // this row's query position (rows r >= BLK, present when BLK < 128, are never written)
    const int64_t qp = QP ? static_cast<int64_t>(qpos[h][r < BLK ? r : 0]) : q0 + r;
    const bool active = h == 0 || has1;
    const float thr =
        (GT && active) ? p.gate_thr[(static_cast<int64_t>(b) * Hq + hq) * p.nb + i] : -INFINITY;
    float m_run = -INFINITY, l_run = 0.f;
    bool o_init = false;
    int k = 0, n_qk = 0, n_gated = 0;
    // ok turns false once a wait gave up (after an abort); the loop then runs
    // to its end with every wait returning at once, so the warpgroup takes
    // the same named barriers without a vote each tile.
    bool ok = true;
    // LAZY: tile 0 first (T = 1 here), then the schedule is awaited
    bool sched_seen = !LAZY;
    if (!sched_seen) T = 1;
    for (int t = 0; active; ++t) {
      if (t >= T) {
        if (sched_seen) break;
        sched_seen = true;
        // one vote, so the warpgroup stays together on its named barriers
        const bool w = mbar_wait_or_abort(&sh.bar_sched, 0, p.err, abort_flag, lim);
        if (named_sync_or(2 + h, 128, !w)) {
          ok = false;
          break;                                    // (after an abort the schedule may be unwritten)
        }
        T = n_diag + sh.n_union;
        if (t >= T) break;
      }
      if (!((tile_mask(t) >> h) & 1u)) continue;
      if (!mbar_wait_or_abort(&sh.bar_s[h], k & 1, p.err, abort_flag, lim)) ok = false;
      tc_fence_after();
      ++n_qk;
      // Block-max gate first: the tile's raw maximum over all rows decides
      // before any exponential is taken, so a dropped tile costs one read of
      // S and a reduction.  A dropped tile leaves m, l and O as they were;
      // the diagonal tile (t == 0) is never gated.  A row whose threshold is
      // -inf (no more causal tiles than the calibration keeps) can never drop
      // a tile, so its warpgroup skips the gate altogether: thr is the same
      // for every thread of the warpgroup, so this costs no divergence.
      if (GT && t != 0 && thr > -INFINITY) {
        float rm = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < BLK / 64; ++c) {
          uint32_t x[64];
          tmem_ld64(tS + c * 64, x);
          float mm[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            mm[q] = fmax3(__uint_as_float(x[q]), __uint_as_float(x[8 + q]), __uint_as_float(x[16 + q]));
            mm[q] = fmax3(mm[q], __uint_as_float(x[24 + q]), __uint_as_float(x[32 + q]));
            mm[q] = fmax3(mm[q], __uint_as_float(x[40 + q]), __uint_as_float(x[48 + q]));
            mm[q] = fmaxf(mm[q], __uint_as_float(x[56 + q]));
          }
          rm = fmaxf(rm, fmax3(fmax3(mm[0], mm[1], mm[2]), fmax3(mm[3], mm[4], mm[5]), fmaxf(mm[6], mm[7])));
        }
        const float wm = warp_max(r < BLK ? rm : -INFINITY);
        if (lane == 0) sh.red[h][warp & 3] = wm;
        named_sync(2 + h, 128);
        const float tmax = fmaxf(fmaxf(sh.red[h][0], sh.red[h][1]), fmaxf(sh.red[h][2], sh.red[h][3]));
        named_sync(2 + h, 128);
        if (tmax < thr) {
          ++n_gated;
          if (r == 0) sh.skip[h][k & 1] = 1;
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.bar_p[h]);     // one arrival per warp
          ++k;
          continue;
        }
      }
      // One pass over S in 64-column chunks.  P = 2^(s*scale - m) is taken
      // against a running max m that starts at the row's max so far; when a
      // chunk's max exceeds m by more than 2^8, m moves up and the P columns
      // already written for this tile are rescaled in place (rare after the
      // first tile).  So P stays below 2^8 and S is read once here.
      // Causal mask: columns above `vis` are not visible to this row.  In
      // natural order only the diagonal tile (t == 0) needs it; with permuted
      // queries every Pass-1 tile does, against the row's own position.
      int vis = BLK;
      if (QP) {
        if (t < n_diag) vis = static_cast<int>(qp - static_cast<int64_t>(jtop - t) * BLK);
      } else if (t == 0) {
        vis = r;
      }
      const bool causal = QP ? __any_sync(0xffffffffu, vis < BLK - 1) : t == 0;
      float psum = 0.f, m_t = m_run;
#pragma unroll 1
      for (int c = 0; c < BLK / 64; ++c) {
        uint32_t x[64], u[32];
        tmem_ld64(tS + c * 64, x);
        float cmax = -INFINITY;
        // Causal tiles: columns above the row's last visible key become -inf
        // (exponential 0), then the same pass as every other tile.
        if (causal) {
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (c * 64 + e > vis) x[e] = __float_as_uint(-INFINITY);
        }
        // Eight independent 3-input max chains (a single chain is latency bound).
        float mm[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          mm[q] = fmax3(__uint_as_float(x[q]), __uint_as_float(x[8 + q]), __uint_as_float(x[16 + q]));
          mm[q] = fmax3(mm[q], __uint_as_float(x[24 + q]), __uint_as_float(x[32 + q]));
          mm[q] = fmax3(mm[q], __uint_as_float(x[40 + q]), __uint_as_float(x[48 + q]));
          mm[q] = fmaxf(mm[q], __uint_as_float(x[56 + q]));
        }
        cmax = fmax3(fmax3(mm[0], mm[1], mm[2]), fmax3(mm[3], mm[4], mm[5]), fmaxf(mm[6], mm[7]));
        const float cm = cmax * p.scale_log2;
        const bool up = cm > (m_t == -INFINITY ? -INFINITY : m_t + kRescaleSlack);
        if (__any_sync(0xffffffffu, up)) {
          const float m_new = up ? cm : m_t;
          // 0 when m_t was -inf; 1 for a row that still has no visible key
          const float beta = m_new == -INFINITY ? 1.0f : ex2(m_t - m_new);
          if (c > 0 && __any_sync(0xffffffffu, beta != 1.0f)) rescale_p(tS, 2 * c, beta);
          psum *= beta;
          m_t = m_new;
        }
        const float m_use = m_t == -INFINITY ? 0.f : m_t;
        // Pairs of columns in packed fp32x2 arithmetic (scale-and-shift and
        // the row sums), four independent packed partial sums.
        unsigned long long ps2[4] = {0ull, 0ull, 0ull, 0ull};   // +0.0f is all zero bits
        const unsigned long long sc2 = f2_pack(p.scale_log2, p.scale_log2);
        const unsigned long long nm2 = f2_pack(-m_use, -m_use);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const unsigned long long y =
              f2_fma(f2_pack(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1])), sc2, nm2);
          float y0, y1;
          f2_unpack(y, y0, y1);
          const float a0 = ex2(y0), a1 = ex2(y1);
          ps2[e & 3] = f2_add(ps2[e & 3], f2_pack(a0, a1));
          u[e] = cvt_bf16x2(a0, a1);
        }
        float s0, s1, s2, s3, s4, s5, s6, s7;
        f2_unpack(ps2[0], s0, s1);
        f2_unpack(ps2[1], s2, s3);
        f2_unpack(ps2[2], s4, s5);
        f2_unpack(ps2[3], s6, s7);
        psum += ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
        tmem_st32(tS + c * 32, u);
      }
      const float m_new = m_t;
      // (a row that has seen no visible key yet keeps m = -inf and l = 0)
      const float alpha = m_new == -INFINITY ? 1.0f : ex2(m_run - m_new);
      // (PV of this head's previous tile has completed: the S-ready barrier
      // tracks every MMA issued before this tile's QK^T)
      if (o_init && __any_sync(0xffffffffu, alpha != 1.0f)) rescale_o<D>(tO, alpha);
      l_run = l_run * alpha + psum;
      m_run = m_new;
      // Early stopping (Pass 2 only): this tile's gain per row is psum / l,
      // its exponential mass over the accumulated mass, both in the frame
      // of m; when every row's gain is below stop_tau the later tiles are
      // not run.  The stop point is published before P is, so the MMA
      // thread sees it when it takes this tile's PV.
      bool stop_now = false;
      if (ES && t >= n_diag) {
        const bool small = !(r < BLK) || psum < p.stop_tau * l_run;
        const bool wsmall = __all_sync(0xffffffffu, small);
        if (lane == 0) sh.vote[h][warp & 3] = wsmall ? 1 : 0;
        named_sync(2 + h, 128);
        stop_now = (sh.vote[h][0] & sh.vote[h][1] & sh.vote[h][2] & sh.vote[h][3]) != 0;
        if (stop_now) {
          if (r == 0) sh.limit[h] = t + 1;
          n_gated += n_diag + sh.n_list[h] - (k + 1);   // listed tiles left out
        }
      }
      tmem_st_wait();
      if (r == 0) sh.skip[h][k & 1] = 0;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.bar_p[h]);         // one arrival per warp
      o_init = true;
      ++k;
      if (stop_now) break;
    }
    // ---- epilogue: O / l -> bf16, LSE
    if (active) ok = !named_sync_or(2 + h, 128, !ok);  // one vote for the whole loop
    if (active && ok && k > 0) {
      ok = mbar_wait_or_abort(&sh.bar_o[h], 0, p.err, abort_flag, lim);
      ok = !named_sync_or(2 + h, 128, !ok);
      tc_fence_after();
    }
    if (active && ok && o_init) {
      const float inv_l = 1.0f / l_run;
      __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(const_cast<void*>(p.O.ptr)) + b * p.O.sB +
                          hq * p.O.sH + qp * p.O.sN;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(tO + c * 32, u);
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
        p.lse[(static_cast<int64_t>(b) * Hq + hq) * N + qp] = (m_run + log2f(l_run)) * 0.69314718055994531f;
    }
    if (active && r == 0 && p.stats) {
      atomicAdd(reinterpret_cast<unsigned long long*>(p.stats), static_cast<unsigned long long>(n_qk));
      atomicAdd(reinterpret_cast<unsigned long long*>(p.stats) + 1, static_cast<unsigned long long>(n_gated));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, int BLK, bool ES, bool QP, bool GT, bool LZ = false>
cudaError_t launch_typed(const AttnParams& p0, cudaStream_t s) {
  // Tensor maps for the TMA loads of Q and of natural K/V tiles (128-row
  // boxes, so BLK = 128 only); without them every tile is gathered.
  AttnParams p = p0;
  CUtensorMap mq{}, mk{}, mv{};
  p.tma = BLK == 128 && encode_rows_map(&mk, p.K) && encode_rows_map(&mv, p.V) && (QP || encode_rows_map(&mq, p.Q));
  if (!p.tma || QP) mq = mk;                       // unused
  using C = Cfg<D, BLK>;
  // schedule: at most min(candidates, 2 * cap) permuted tiles per item
  // (with early stopping both lists in full, compacted first in the V ring)
  const int max_union = ES ? 2 * p.cap : std::min(p.nb, 2 * p.cap);
  if (ES && 2 * p.cap * 4 > kStages * C::kKVBytes) return cudaErrorInvalidValue;
  int smem = 1024 + C::kEnd + 4 * max_union;
  smem = smem < C::kMinSmem ? C::kMinSmem : smem;
  if (smem + 4096 > 227 * 1024) return cudaErrorInvalidValue;   // + static shared memory
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, BLK, ES, QP, GT, LZ>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int npair = (p.G + 1) / 2;
  const int64_t items = static_cast<int64_t>(p.nb) * p.Q.B * p.K.H * npair;
  if (items >= (1ll << 31)) return cudaErrorInvalidValue;
  attn_fwd_kernel<D, BLK, ES, QP, GT, LZ><<<static_cast<unsigned>(items), kThreads, smem, s>>>(p, mq, mk, mv);
  return cudaGetLastError();
}

template <int D, int BLK>
cudaError_t launch_mode(const AttnParams& p, cudaStream_t s) {
  // (the gate's code is compiled only into the kernel that gates)
  if (p.qperm)
    return p.early_stop || p.gate_thr ? cudaErrorInvalidValue : launch_typed<D, BLK, false, true, false>(p, s);
  if (p.early_stop) return p.gate_thr ? cudaErrorInvalidValue : launch_typed<D, BLK, true, false, false>(p, s);
  if (p.gate_thr) return launch_typed<D, BLK, false, false, true>(p, s);
  return p.seg > p.blk ? launch_typed<D, BLK, false, false, false, true>(p, s)
                       : launch_typed<D, BLK, false, false, false, false>(p, s);
}

}  // namespace

cudaError_t launch_attn_fwd(const AttnParams& p, cudaStream_t s) {
  const int D = static_cast<int>(p.Q.D);
  if (p.nb > 8192) return cudaErrorInvalidValue;
  if (attn_fwd_pair_applies(p)) return launch_attn_fwd_pair(p, s);
  if (D == 128 && p.blk == 128) return launch_mode<128, 128>(p, s);
  if (D == 128 && p.blk == 64) return launch_mode<128, 64>(p, s);
  if (D == 64 && p.blk == 128) return launch_mode<64, 128>(p, s);
  if (D == 64 && p.blk == 64) return launch_mode<64, 64>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace pbs
