// pbs_attn_fwd on CTA pairs: the same forward pass as attn_fwd.cu (own
// segment in natural order, then the listed permuted blocks gathered through
// the index list -- "S2O: Early Stopping for Sparse Attention via Online
// Permutation", Technical Summary, 1. Online Permutation via Index-Driven
// Loading and 3. Kernel Implementation), with the tensor-core work of four
// query heads of one GQA group spread over a cluster of two CTAs.
//
// Why pairs.  A K/V tile is 64 KB and every query head that lists it needs
// all of it.  On one CTA (two heads) the row gathers (16-byte cp.async) of
// that 64 KB per tile, and its two-stage rings, set the pace.  A tcgen05 MMA
// with .cta_group::2 spans two CTAs: M = 256 rows, 128 from each CTA's
// shared and tensor memory, and the B operand's N columns split between the
// two CTAs' shared memory.  So a pair runs four heads (two per CTA, as head
// "slots" 0 and 1) against one K/V tile while each CTA gathers only half of
// it: K rows 64*rank .. 64*rank+63 (QK^T splits N = keys), and the d-half
// 64*rank .. 64*rank+63 of every V row (PV splits N = d).  Half the bytes
// per CTA leave room for four ring stages, and one MMA instruction now
// drives both SMs' tensor cores.
//
// The pair walks the union of its four heads' tile lists (natural blocks of
// the own segment, then the listed permuted blocks in ascending order).  The
// MMA of slot s covers the slot-s heads of both CTAs, so it runs whenever
// either of them lists the tile; the PV of a head that does not list the
// tile leaves that head's O rows untouched (the MMA's per-row output mask)
// and its softmax state is left alone, so the head takes nothing from it.
//
// Roles (384 threads per CTA):
//   warp 0    even CTA: tcgen05 MMA issuer for the pair (one thread);
//             odd CTA: relay -- waits for its own CTA's gathers to land and
//             arrives on the even CTA's barriers, which the MMAs wait on;
//   warps 1-3 producer: cp.async of Q (this CTA's two heads) and of this
//             CTA's half of every K/V tile into 4-stage rings;
//   warps 4-11 softmax, one warpgroup per head slot, as in attn_fwd.cu.
// Tensor memory per CTA (512 columns): S0 | S1 | O0 | O1.
// Every wait is bounded; a timeout raises the abort flag of both CTAs, every
// role leaves its loop, and both CTAs meet at a final cluster barrier before
// tensor memory is freed, so neither exits while the other can still touch
// its shared or tensor memory.
#include <math.h>

#include <algorithm>

#include "pbs_common.cuh"
#include "pbs_internal.h"

namespace pbs {
namespace {

constexpr int kThreads = 384;
constexpr int kD = 128, kBlk = 128, kM = 128;
constexpr int kProducerThreads = 96;
constexpr int kStages = 4;
constexpr float kRescaleSlack = 8.0f;
// Per-CTA shared memory (1024-byte aligned regions):
//   Q: two head slots x [2 d-halves x (128 rows x 128 B)]
//   K ring: kStages x [2 d-halves x (64 rows x 128 B)]  -- this CTA's 64 keys
//   V ring: kStages x [128 rows x 128 B]                 -- this CTA's d-half
constexpr int kQBytes = 2 * kM * 128;
constexpr int kKBytes = 2 * 64 * 128;
constexpr int kVBytes = kBlk * 128;
constexpr int kQ0 = 0;
constexpr int kK0 = 2 * kQBytes;
constexpr int kV0 = kK0 + kStages * kKBytes;
constexpr int kEnd = kV0 + kStages * kVBytes;


struct PairShared {
  uint64_t bar_q;
  uint64_t bar_k[kStages], bar_v[kStages], bar_kempty[kStages], bar_vempty[kStages];
  uint64_t bar_s[2], bar_p[2], bar_o[2], bar_fin;
  uint32_t tmem_base;
  int abort;
  int n_union;
};

__global__ void __launch_bounds__(kThreads, 1) attn_fwd_pair_kernel(AttnParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint32_t* sched = reinterpret_cast<uint32_t*>(smem + kEnd);
  __shared__ PairShared sh;
  __shared__ uint32_t bm[4][256];          // per-head candidate bitmaps (ncand <= 8192)
  __shared__ int32_t rowbuf[kStages][kBlk];

  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs; 1: relays its gathers
  const uint32_t peer = rank ^ 1u;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hq = p.G * static_cast<int>(p.K.H);
  const int nquad = p.G / 4;
  // Work order as in attn_fwd.cu: all items of one (batch, KV head) first,
  // heavy query blocks first within it; one item per CTA pair.
  const int item = static_cast<int>(blockIdx.x >> 1);
  const int per_bh = p.nb * nquad;
  const int bh = item / per_bh;
  const int rem = item % per_bh;
  const int i = p.nb - 1 - rem / nquad;
  const int qd = rem % nquad;
  const int b = bh / static_cast<int>(p.K.H);
  const int hk = bh % static_cast<int>(p.K.H);
  const int h0 = hk * p.G + 4 * qd;         // the pair's heads h0 .. h0+3
  const int hmine = h0 + 2 * static_cast<int>(rank);   // this CTA's slot-0 head
  const int spb = p.seg / kBlk;
  const int s = i / spb;
  const int ncand = s * spb;
  const int n_diag = i - s * spb + 1;
  const int64_t q0 = static_cast<int64_t>(i) * kBlk;
  const int64_t N = p.Q.N;

  const uint32_t sQ0 = smem_u32(smem + kQ0);
  const uint32_t sK = smem_u32(smem + kK0);
  const uint32_t sV = smem_u32(smem + kV0);

  // ------------------------------------------------------------------ setup
  if (warp == 0) {
    tmem_alloc_pair(&sh.tmem_base, 512);
    tmem_relinquish_pair();
    // Union of the four heads' lists (same in both CTAs): a bitmap per head,
    // then an ascending schedule, each entry tagged with its 4-bit head mask.
    int cnt[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
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
#pragma unroll
      for (int h = 0; h < 4; ++h) bm[h][w] = 0u;
    }
    __syncwarp();
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int32_t* list = p.idx + ((static_cast<int64_t>(b) * Hq + h0 + h) * p.nb + i) * p.cap;
      for (int e = lane; e < cnt[h]; e += 32) {
        const int pb = list[e];
        if (pb < 0 || pb >= ncand) {
          set_error(p.err, kErrDeviceCheck);
          continue;
        }
        atomicOr(&bm[h][pb >> 5], 1u << (pb & 31));
      }
    }
    __syncwarp();
    int total = 0;
    for (int base = 0; base < words; base += 32) {
      const int w = base + lane;
      uint32_t m[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) m[h] = w < words ? bm[h][w] : 0u;
      uint32_t u = m[0] | m[1] | m[2] | m[3];
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
        uint32_t mask = 0;
#pragma unroll
        for (int h = 0; h < 4; ++h) mask |= ((m[h] >> bit) & 1u) << h;
        sched[o++] = static_cast<uint32_t>(w * 32 + bit) | (mask << 28);
      }
      total += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      sh.n_union = total;
      sh.abort = 0;
      // The even CTA's "landed" barriers also take one arrival from the odd
      // CTA's relay; its P barriers take the four softmax warps of each CTA.
      const uint32_t extra = rank == 0 ? 1u : 0u;
      mbar_init(&sh.bar_q, kProducerThreads + extra);
      for (int st = 0; st < kStages; ++st) {
        mbar_init(&sh.bar_k[st], kProducerThreads + extra);
        mbar_init(&sh.bar_v[st], kProducerThreads + extra);
        mbar_init(&sh.bar_kempty[st], 1);
        mbar_init(&sh.bar_vempty[st], 1);
      }
      for (int h = 0; h < 2; ++h) {
        mbar_init(&sh.bar_s[h], 1);
        mbar_init(&sh.bar_p[h], rank == 0 ? 8 : 4);
        mbar_init(&sh.bar_o[h], 1);
      }
      mbar_init(&sh.bar_fin, 1);
      fence_mbar_init();
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();      // both CTAs' barriers exist before any signal crosses
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const int T = n_diag + sh.n_union;
  volatile int* abort_flag = &sh.abort;
  const uint32_t peer_abort = mapa_shared(smem_u32(&sh.abort), peer);
  auto raise_abort = [&]() {
    *abort_flag = 1;
    st_cluster_u32(peer_abort, 1u);
  };
  // Bounded wait on a barrier of this CTA (acquire at cluster scope, as some
  // arrivals come from the other CTA).  Gives up once either CTA aborted.
  const uint32_t lim = p.test_wait_limit ? p.test_wait_limit : kSpinLimit;
  auto wait_bar = [&](uint64_t* bar, uint32_t parity, uint32_t limit) -> bool {
    for (uint32_t it = 0; it < limit; ++it) {
      if (mbar_try_wait_cl(bar, parity)) return true;
      if ((it & 63u) == 63u && *abort_flag) return false;
    }
    set_error(p.err, kErrTimeout);
    raise_abort();
    return false;
  };
  // 4-bit head mask of tile t (bit j: head h0 + j lists it).
  auto tile_mask = [&](int t) -> uint32_t { return t < n_diag ? 0xFu : (sched[t - n_diag] >> 28); };

  if (warp >= 1 && warp <= 3) {
    // ============================================================ producer
    const int pt = tid - 32;
    const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(p.K.ptr) + b * p.K.sB + hk * p.K.sH;
    const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(p.V.ptr) + b * p.V.sB + hk * p.V.sH;
    const int32_t* prow =
        p.perm + ((static_cast<int64_t>(b) * p.K.H + hk) * p.perm_nseg + (p.perm_nseg > 1 ? s : 0)) * N;
    // Q of this CTA's two heads.
    for (int h = 0; h < 2; ++h) {
      const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(p.Q.ptr) + b * p.Q.sB + (hmine + h) * p.Q.sH;
      const uint32_t dst = sQ0 + h * kQBytes;
      for (int id = pt; id < kM * 16; id += kProducerThreads) {
        const int r = id / 16, c = id % 16;
        cp_async16(dst + (c / 8) * (kM * 128) + sw128_offset(r, c % 8), qb + (q0 + r) * p.Q.sN + c * 8);
      }
    }
    if (!p.test_wait_limit) cp_async_mbar_arrive(&sh.bar_q);   // withheld by the failure-path test hook
    // Row indices of a tile, one tile ahead in registers (rows pt, pt + 96).
    int32_t nxt[2] = {0, 0};
    auto fetch_rows = [&](int t) {
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int r = pt + q * kProducerThreads;
        if (r < kBlk && t >= n_diag)
          nxt[q] = prow[static_cast<int64_t>(sched[t - n_diag] & 0x0FFFFFFFu) * kBlk + r];
      }
    };
    if (T > 0) fetch_rows(0);
    // K: this CTA's 64 keys, full rows: thread pt copies 16-byte chunk pt % 16
    // of rows pt / 16 + 6k.  V: every key, this CTA's d-half: chunk pt % 8 of
    // rows pt / 8 + 12k.  Row indices are read from shared memory first so
    // the copies go out back to back.
    const int kc = pt % 16, kr0 = pt / 16;
    const int vc = pt % 8, vr0 = pt / 8;
    const int rbase = 64 * static_cast<int>(rank);
    for (int t = 0; t < T; ++t) {
      const int st = t % kStages;
      const uint32_t ph = static_cast<uint32_t>(t / kStages);
      {                                           // K of tile t
        const bool ok = t < kStages || wait_bar(&sh.bar_kempty[st], (ph - 1) & 1u, lim);
        if (named_sync_or(1, kProducerThreads, !ok)) break;   // all producer threads leave together
        const bool nat = t < n_diag;
        const int id0 = nat ? i - t : static_cast<int>(sched[t - n_diag] & 0x0FFFFFFFu);
        const int64_t lo = static_cast<int64_t>((id0 * kBlk) / p.seg) * p.seg;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int r = pt + q * kProducerThreads;
          if (r >= kBlk) continue;
          int64_t x;
          if (nat) {
            x = static_cast<int64_t>(id0) * kBlk + r;
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
        const uint32_t dst = sK + st * kKBytes + (kc / 8) * (64 * 128);
        int32_t x[11];
#pragma unroll
        for (int k = 0; k < 11; ++k) x[k] = kr0 + 6 * k < 64 ? rowbuf[st][rbase + kr0 + 6 * k] : 0;
#pragma unroll
        for (int k = 0; k < 11; ++k) {
          const int r = kr0 + 6 * k;
          if (r < 64) cp_async16(dst + sw128_offset(r, kc % 8), kb + x[k] * p.K.sN + kc * 8);
        }
        cp_async_mbar_arrive(&sh.bar_k[st]);
      }
      {                                           // V of tile t
        const bool okv = t < kStages || wait_bar(&sh.bar_vempty[st], (ph - 1) & 1u, lim);
        if (named_sync_or(1, kProducerThreads, !okv)) break;
        const uint32_t dst = sV + st * kVBytes;
        const __nv_bfloat16* vsrc = vb + (rbase + vc * 8);
        int32_t x[11];
#pragma unroll
        for (int k = 0; k < 11; ++k) x[k] = vr0 + 12 * k < kBlk ? rowbuf[st][vr0 + 12 * k] : 0;
#pragma unroll
        for (int k = 0; k < 11; ++k) {
          const int r = vr0 + 12 * k;
          if (r < kBlk) cp_async16(dst + sw128_offset(r, vc), vsrc + x[k] * p.V.sN);
        }
        cp_async_mbar_arrive(&sh.bar_v[st]);
      }
      if (t + 1 < T) fetch_rows(t + 1);
    }
    cp_async_wait_all();
  } else if (warp == 0 && rank == 1) {
    // ============================================================== relay
    // The MMAs read this CTA's shared memory; the MMA issuer waits on the
    // even CTA's barriers only.  One thread observes each of this CTA's
    // fills land, makes the cp.async writes visible to the tensor core
    // (async proxy) and arrives on the even CTA's barrier for that fill.
    if (lane == 0) {
      const uint32_t r_q = mapa_shared(smem_u32(&sh.bar_q), 0);
      if (wait_bar(&sh.bar_q, 0, lim)) {
        fence_proxy_async();
        mbar_arrive_cluster(r_q);
        for (int t = 0; t < T; ++t) {
          const int st = t % kStages;
          const uint32_t ph = static_cast<uint32_t>(t / kStages) & 1u;
          if (!wait_bar(&sh.bar_k[st], ph, lim)) break;
          fence_proxy_async();
          mbar_arrive_cluster(mapa_shared(smem_u32(&sh.bar_k[st]), 0));
          if (!wait_bar(&sh.bar_v[st], ph, lim)) break;
          fence_proxy_async();
          mbar_arrive_cluster(mapa_shared(smem_u32(&sh.bar_v[st]), 0));
        }
      }
    }
    __syncwarp();
  } else if (warp == 0) {
    // ========================================================= MMA issuer
    // Event driven as in attn_fwd.cu: whichever of PV_h (P of both CTAs
    // ready, V landed in both) or QK_h (previous PV_h issued, K landed in
    // both) can go, goes.  Slot h serves tile t if either CTA's slot-h head
    // lists it (mask bits h and h + 2).
    const bool leader = lane == 0;
    auto test = [&](uint64_t* bar, uint32_t parity) -> bool {
      bool v = false;
      if (leader) v = mbar_test_wait_cl(bar, parity);
      return __shfl_sync(0xffffffffu, v, 0);
    };
    bool ok = true;
    {
      bool v = true;
      if (leader) v = wait_bar(&sh.bar_q, 0, lim);
      ok = __shfl_sync(0xffffffffu, v, 0);
      if (leader) fence_proxy_async();
      tc_fence_after();
    }
    constexpr uint32_t idesc_qk = idesc_bf16(2 * kM, kBlk, false);
    constexpr uint32_t idesc_pv = idesc_bf16(2 * kM, kD, true);
    auto serves = [&](int t, int h) -> bool { return (tile_mask(t) >> h) & 5u; };
    auto next_tile = [&](int h, int from) {
      int t = from;
      while (t < T && !serves(t, h)) ++t;
      return t;
    };
    int nq[2] = {next_tile(0, 0), next_tile(1, 0)};   // next tile needing QK_h
    int pend[2] = {-1, -1};                          // tile whose PV_h is due
    int kh[2] = {0, 0};                              // QK_h issued
    bool o_init[2] = {false, false};
    // Fills land in tile order on each ring; k_land / v_land count the fills
    // observed, k_rel / v_rel the stages handed back to the producers.
    int k_land = 0, v_land = 0, k_rel = 0, v_rel = 0;
    auto landed = [&](uint64_t* bars, int& nland, int t) -> bool {
      while (nland <= t) {
        if (!test(&bars[nland % kStages], static_cast<uint32_t>(nland / kStages) & 1u)) return false;
        ++nland;
        if (leader) fence_proxy_async();
      }
      return true;
    };
    // Hand back every landed stage that both slots have moved past.
    auto release_k = [&]() {
      const int lim = min(nq[0], nq[1]);
      while (k_rel < k_land && k_rel < lim) {
        if (elect_one()) tc_commit_pair(&sh.bar_kempty[k_rel % kStages], 3);
        ++k_rel;
      }
    };
    auto release_v = [&]() {
      const int a = pend[0] >= 0 ? pend[0] : nq[0];
      const int c = pend[1] >= 0 ? pend[1] : nq[1];
      const int lim = min(a, c);
      while (v_rel < v_land && v_rel < lim) {
        if (elect_one()) tc_commit_pair(&sh.bar_vempty[v_rel % kStages], 3);
        ++v_rel;
      }
    };
    uint32_t idle = 0;
    while (ok) {
      bool pending = false, progress = false;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (pend[h] >= 0) {
          pending = true;
          const int t = pend[h];
          if (test(&sh.bar_p[h], static_cast<uint32_t>(kh[h] - 1) & 1u) && landed(sh.bar_v, v_land, t)) {
            tc_fence_after();
            const uint32_t tP = tmem + h * 128;
            const uint32_t tO = tmem + 256 + h * 128;
            const uint64_t bd0 = sdesc_sw128(sV + (t % kStages) * kVBytes, kBlk * 128, 1024);
            const uint32_t acc0 = o_init[h] ? 1u : 0u;
            // a head that does not list the tile keeps its O rows untouched
            const uint32_t msk = tile_mask(t);
            const uint32_t off_even = (msk >> h) & 1u ? 0u : 0xFFFFFFFFu;
            const uint32_t off_odd = (msk >> (h + 2)) & 1u ? 0u : 0xFFFFFFFFu;
#pragma unroll
            for (int kk = 0; kk < kBlk / 16; ++kk) {
              const uint64_t bd = sdesc_add(bd0, kk * 2048);
              if (elect_one()) mma_pair_ts_masked(tO, tP + kk * 8, bd, idesc_pv, kk > 0 ? 1u : acc0, off_even, off_odd);
            }
            o_init[h] = true;
            pend[h] = -1;
            progress = true;
            release_v();
          }
        }
        if (pend[h] < 0 && nq[h] < T) {
          pending = true;
          const int t = nq[h];
          if (landed(sh.bar_k, k_land, t)) {
            tc_fence_after();
            const uint32_t qbase = sQ0 + h * kQBytes;
            const uint32_t kbase = sK + (t % kStages) * kKBytes;
            const uint32_t tS = tmem + h * 128;
            const uint64_t a0 = sdesc_sw128(qbase, 16, 1024);
            const uint64_t b0 = sdesc_sw128(kbase, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
              const uint32_t half = kk / 4, koff = (kk % 4) * 32;
              const uint64_t ad = sdesc_add(a0, half * (kM * 128) + koff);
              const uint64_t bd = sdesc_add(b0, half * (64 * 128) + koff);
              if (elect_one()) mma_pair_ss(tS, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
            }
            if (elect_one()) tc_commit_pair(&sh.bar_s[h], 3);
            ++kh[h];
            pend[h] = t;
            nq[h] = next_tile(h, t + 1);
            progress = true;
            release_k();
          }
        }
      }
      if (!pending) break;
      if (progress) {
        idle = 0;
      } else if (++idle >= 4u * lim) {
        if (leader) {
          set_error(p.err, kErrTimeout);
          raise_abort();
        }
        ok = false;
      } else if ((idle & 63u) == 0) {
        ok = !__shfl_sync(0xffffffffu, *abort_flag, 0);
      }
    }
    if (leader) {
#pragma unroll
      for (int h = 0; h < 2; ++h)
        if (kh[h] > 0) tc_commit_pair(&sh.bar_o[h], 3);
      tc_commit_pair(&sh.bar_fin, 3);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ============================================================ softmax
    const int h = (warp - 4) >> 2;                  // head slot
    const int r = tid - 128 - h * 128;              // query row = tensor-memory lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + h * 128 + lane_off;
    const uint32_t tO = tmem + 256 + h * 128 + lane_off;
    const int hq = hmine + h;
    const uint32_t own_bit = 1u << (2 * rank + h);
    const uint32_t p_bar = rank == 0 ? smem_u32(&sh.bar_p[h]) : mapa_shared(smem_u32(&sh.bar_p[h]), 0);
    float m_run = -INFINITY, l_run = 0.f;
    bool o_init = false;
    int k = 0, n_qk = 0;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const uint32_t msk = tile_mask(t);
      if (!((msk >> h) & 5u)) continue;             // the slot does not run this tile
      if (!wait_bar(&sh.bar_s[h], static_cast<uint32_t>(k) & 1u, lim)) ok = false;
      tc_fence_after();
      if (!(msk & own_bit)) {
        // Run for the other CTA's slot-h head only: the PV leaves this
        // head's O rows untouched and its softmax state stays as it is.
      } else {
        ++n_qk;
        const bool causal = t == 0;
        float psum = 0.f, m_t = m_run;
#pragma unroll 1
        for (int c = 0; c < kBlk / 64; ++c) {
          uint32_t x[64], u[32];
          tmem_ld64(tS + c * 64, x);
          float cmax = -INFINITY;
          // Causal tiles: columns above the row's last visible key become -inf
          // (exponential 0), then the same pass as every other tile.
          if (causal) {
#pragma unroll
            for (int e = 0; e < 64; ++e)
              if (c * 64 + e > r) x[e] = __float_as_uint(-INFINITY);
          }
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
            const float beta = ex2(m_t - m_new);
            if (c > 0 && __any_sync(0xffffffffu, beta != 1.0f)) {
              tmem_st_wait();
              for (int q = 0; q < 2 * c; ++q) {
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
            psum *= beta;
            m_t = m_new;
          }
          const float m_use = m_t == -INFINITY ? 0.f : m_t;
          unsigned long long ps2[4] = {0ull, 0ull, 0ull, 0ull};
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
        const float alpha = ex2(m_run - m_new);
        if (o_init && __any_sync(0xffffffffu, alpha != 1.0f)) {
          // every MMA issued before this tile's QK^T has completed (the
          // S-ready commit tracks them), so O holds all earlier PVs
#pragma unroll 1
          for (int c = 0; c < kD / 32; ++c) {
            uint32_t u[32];
            tmem_ld32(tO + c * 32, u);
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
            tmem_st32(tO + c * 32, u);
          }
        }
        l_run = l_run * alpha + psum;
        m_run = m_new;
        o_init = true;
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {                              // one arrival per warp, on the even CTA's barrier
        if (rank == 0) mbar_arrive(&sh.bar_p[h]);
        else mbar_arrive_cluster(p_bar);
      }
      ++k;
    }
    // ---- epilogue: O / l -> bf16, LSE
    ok = !named_sync_or(2 + h, 128, !ok);
    if (ok && k > 0) {
      ok = wait_bar(&sh.bar_o[h], 0, lim);
      ok = !named_sync_or(2 + h, 128, !ok);
      tc_fence_after();
    }
    if (ok && o_init) {
      const float inv_l = 1.0f / l_run;
      __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(const_cast<void*>(p.O.ptr)) + b * p.O.sB +
                          hq * p.O.sH + (q0 + r) * p.O.sN;
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(tO + c * 32, u);
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
      if (p.lse)
        p.lse[(static_cast<int64_t>(b) * Hq + hq) * N + q0 + r] = (m_run + log2f(l_run)) * 0.69314718055994531f;
    }
    if (r == 0 && p.stats)
      atomicAdd(reinterpret_cast<unsigned long long*>(p.stats), static_cast<unsigned long long>(n_qk));
  }
  // ---- teardown: the even CTA drains every MMA of the pair; then both CTAs
  // meet, so neither frees tensor memory or exits while an MMA or an
  // arrival of the pair can still reach it.
  if (warp == 0 && rank == 0) {
    if (lane == 0) wait_bar(&sh.bar_fin, 0, kSpinLimit);
    __syncwarp();
  }
  tc_fence_before();
  __syncwarp();
  __syncthreads();
  cluster_sync_all();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace

// Whether the CTA-pair kernel serves these parameters.
bool attn_fwd_pair_applies(const AttnParams& p) {
  if (!p.cta_pair || p.Q.D != kD || p.blk != kBlk || p.early_stop || p.gate_thr || p.qperm) return false;
  if (p.G % 4 != 0) return false;
  const int max_union = std::min(p.nb, 4 * p.cap);
  const int smem = 1024 + kEnd + 4 * max_union;
  return smem + 8192 <= 227 * 1024;              // + static shared memory
}

cudaError_t launch_attn_fwd_pair(const AttnParams& p, cudaStream_t s) {
  const int max_union = std::min(p.nb, 4 * p.cap);
  const int smem = 1024 + kEnd + 4 * max_union;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t items = static_cast<int64_t>(p.nb) * p.Q.B * p.K.H * (p.G / 4);
  if (2 * items >= (1ll << 31)) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * items));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, attn_fwd_pair_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pbs
