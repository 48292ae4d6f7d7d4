/*
 * pbs.h -- C ABI of the permuted block-sparse attention prefill library
 * (libpbs.so, sm_100a).
 *
 * Three calls make up one prefill-attention pass:
 *
 *   pbs_permute   per-segment stable sort of keys by a pooled-query score.
 *                 "Sparser Block-Sparse Attention via Token Permutation",
 *                 Technical Summary, 2. Segmented Permutation for Causality
 *                 and 3. Global-Importance-Based Key Permutation.
 *   pbs_select    per-query-block lists of permuted key blocks, by top-k
 *                 density or by cumulative attention mass on block-pooled
 *                 scores.  Same page, 4. Implementation (Block Selection);
 *                 cumulative mass as in "SampleAttention", Technical Deep Dive.
 *   pbs_attn_fwd  FlashAttention-style forward over the block's own segment
 *                 (dense, causal, natural order) and the listed permuted
 *                 blocks of earlier segments, gathered through the index
 *                 list; optional exact in-tile block-max gating.
 *                 "S2O: Early Stopping for Sparse Attention via Online
 *                 Permutation", Technical Summary, 1. Online Permutation via
 *                 Index-Driven Loading and 3. Kernel Implementation;
 *                 "Block Sparse Flash Attention", Approach.
 *   pbs_attn_fwd_early_stop
 *                 the same two passes, the listed blocks visited in the order
 *                 given, stopping once a tile's marginal attention mass falls
 *                 below a fraction of the accumulated mass.  S2O page,
 *                 2. Early-Stopping Rule.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Tensors are described by pbs_tensor: a DEVICE pointer to bfloat16
 *    elements with logical shape [B, H, N, D] and element strides sB, sH,
 *    sN; the D stride is 1.  Q is [B, Hq, N, D]; K, V and O are
 *    [B, Hkv, N, D] / [B, Hq, N, D].  Hq must be a multiple of Hkv; query
 *    head h uses KV head h / (Hq / Hkv).
 *  - Supported: D in {64, 128}; blk in {64, 128}; seg a multiple of blk,
 *    seg <= 8192; N a multiple of blk, N < 2^31; pointers 16-byte aligned;
 *    strides multiples of 8 elements.  Anything else returns
 *    PBS_ERR_UNSUPPORTED or PBS_ERR_INVALID_ARG and leaves outputs untouched.
 *  - Index arrays are DEVICE int32, dense row-major, shapes as stated.
 *  - Ownership: the caller owns every buffer, the stream and the workspace.
 *    The library allocates no memory, never synchronises the stream (except
 *    pbs_check_device) and never throws across this boundary.  Work is
 *    enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) of
 *    the current device.
 *  - Workspace: `ws` is a DEVICE buffer of at least pbs_workspace_size()
 *    bytes, 256-byte aligned, used as scratch for the duration of the
 *    enqueued work only.  Concurrent calls need distinct workspaces.
 *  - Errors: every call returns PBS_OK (0) or a negative pbs_status; the
 *    message of the most recent failure on the calling host thread is
 *    returned by pbs_get_last_error().  Host-side checks happen before
 *    anything is enqueued.  Device-side checks (an index outside its
 *    segment or causal range, a list count above capacity, a bounded wait
 *    that gave up) never fault: the offending access is skipped and a
 *    sticky device error word is set, which pbs_check_device() reports.
 */
#ifndef PBS_H_
#define PBS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pbs_tensor {
  void* ptr;              /* device pointer to bf16 elements                 */
  int64_t B, H, N, D;     /* logical shape                                    */
  int64_t sB, sH, sN;     /* element strides of B, H, N (D stride is 1)       */
} pbs_tensor;

typedef enum pbs_status {
  PBS_OK = 0,
  PBS_ERR_INVALID_ARG = -1,   /* null pointer, inconsistent shapes          */
  PBS_ERR_UNSUPPORTED = -2,   /* valid but outside the supported envelope   */
  PBS_ERR_CAPACITY = -3,      /* idx capacity below the required bound      */
  PBS_ERR_CUDA = -4,          /* a CUDA runtime call failed                 */
  PBS_ERR_TIMEOUT = -5,       /* device: a bounded wait gave up             */
  PBS_ERR_DEVICE_CHECK = -6   /* device: an index failed its bounds check   */
} pbs_status;

enum { PBS_OP_PERMUTE = 0, PBS_OP_SELECT = 1, PBS_OP_ATTN = 2, PBS_OP_PERMUTE_SEGMENTED = 3,
       PBS_OP_SELECT_SEGMENTED = 4, PBS_OP_SELECT_SAMPLE = 5, PBS_OP_PERMUTE_QUERIES = 6 };
enum { PBS_SELECT_TOPK = 0, PBS_SELECT_TAU = 1, PBS_SELECT_SAMPLE = 2 };
/* OR-ed into pbs_select's mode: write lists in visiting order, and/or read
 * one permutation per query segment (see there). */
enum { PBS_SELECT_SCORE_ORDER = 0x10, PBS_SELECT_PERM_PER_SEGMENT = 0x20 };
/* pbs_attn_fwd_ex flags. */
enum { PBS_ATTN_EARLY_STOP = 1, PBS_ATTN_PERM_PER_SEGMENT = 2, PBS_ATTN_CTA_PAIR = 4 };

/* Bytes of workspace the given op needs for these shapes (0 if none).
 * Q and K may not be NULL; only their shapes are read.                     */
size_t pbs_workspace_size(int op, const pbs_tensor* Q, const pbs_tensor* K,
                          int blk, int seg);

/* pbs_permute: perm[b, hkv, p] = original key position at logical position
 * p, for every (b, hkv).
 *   1. proxy query qhat[b,hkv] = sum of the last `blk` query rows of every
 *      query head of KV head hkv's group (fp32);
 *   2. score s_j = qhat . K[b,hkv,j] (fp32); positions j < n_sink get +inf;
 *   3. within each segment [t*seg, (t+1)*seg) keys are ordered by descending
 *      score, equal scores by ascending position.  Segment order is kept, so
 *      perm maps each segment onto itself.
 * perm: device int32 [B, Hkv, N].  Requires N >= blk.                      */
int pbs_permute(const pbs_tensor* Q, const pbs_tensor* K, int blk, int seg,
                int n_sink, int32_t* perm, void* ws, size_t ws_bytes,
                void* stream);

/* pbs_permute_noalloc: the same permutation as pbs_permute, for callers
 * that cannot allocate device memory when they call (for example a runtime
 * whose device memory is all reserved by its own allocator, or a plugin
 * interface that passes a kernel its inputs and outputs but no workspace).
 * The pages have no counterpart: this is a deployment convenience.
 * Its scratch is a fixed 256 KiB device array inside libpbs.so (held by
 * every GPU that loads the library until the process exits), so
 * B * Hkv * D must not exceed 65536; larger inputs return PBS_ERR_CAPACITY.
 * The call allocates nothing.  Its first call on a device looks up the
 * array's device address with that device current and keeps it for the
 * life of the process; make that first call before any stream capture.  The
 * kept address belongs to the device's primary context: do not use this
 * entry point from another context of the device, or after
 * cudaDeviceReset() on it.  All calls on a device share the array and it
 * keeps the last call's contents (each call overwrites what it reads), so
 * calls whose GPU work may overlap race and must not be issued together.    */
int pbs_permute_noalloc(const pbs_tensor* Q, const pbs_tensor* K, int blk, int seg,
                        int n_sink, int32_t* perm, void* stream);

/* pbs_permute_segmented: one key permutation per query segment,
 * perm[b, hkv, s, p] = original key position at logical position p as read
 * by query segment s ("S2O ...", Technical Summary, 1. Online Permutation
 * via Index-Driven Loading: each query segment ranks the keys that precede
 * it by one query standing for the whole segment).
 *   1. qbar_s[b,hkv] = sum of every query row of segment s of every query
 *      head of KV head hkv's group (fp64);
 *   2. score s_j = qbar_s . K[b,hkv,j] (fp64); positions j < n_sink get +inf;
 *   3. each key segment t < s is sorted by descending score, equal scores by
 *      ascending position; key segments t >= s keep their natural order.
 * perm: device int32 [B, Hkv, nseg, N] with nseg = ceil(N / seg).
 * ws: pbs_workspace_size(PBS_OP_PERMUTE_SEGMENTED, ...) bytes.
 * Select with mode | PBS_SELECT_PERM_PER_SEGMENT and attend with
 * PBS_ATTN_PERM_PER_SEGMENT to use it; each query block then reads its
 * segment's permutation.  Fp64 keeps the order exact on inputs whose values
 * are multiples of 1/8 (any bf16 input sorts by its fp64-rounded scores). */
int pbs_permute_segmented(const pbs_tensor* Q, const pbs_tensor* K, int blk, int seg, int n_sink,
                          int32_t* perm, void* ws, size_t ws_bytes, void* stream);

/* pbs_permute_queries: S2O's query permutation ("S2O ...", Technical
 * Summary, 1. Online Permutation via Index-Driven Loading, Query
 * Permutation: queries are reordered by their score against a guide vector
 * shared by the head).  qperm[b, hq, p] = original query position at
 * permuted position p:
 *   1. guide vector g[b, hkv] = sum of every key row of KV head hkv (fp64);
 *   2. score of query n of head hq: Q[b, hq, n] . g[b, hq / G] (fp64);
 *   3. within each segment [t*seg, (t+1)*seg) the queries of (b, hq) are
 *      ordered by descending score, equal scores by ascending position;
 *      segment order is kept, so qperm maps each segment onto itself.
 * qperm: device int32 [B, Hq, N].  blk only takes part in the shape checks.
 * ws: pbs_workspace_size(PBS_OP_PERMUTE_QUERIES, ...) bytes (partial and
 * final guide vectors).  Select with pbs_select_qperm and attend with
 * pbs_attn_fwd_qperm to use it.                                            */
int pbs_permute_queries(const pbs_tensor* Q, const pbs_tensor* K, int blk, int seg, int32_t* qperm,
                        void* ws, size_t ws_bytes, void* stream);

/* Upper bound on the list length pbs_select can produce for these settings
 * (host-only arithmetic).  Pass at least this as `cap`.  For
 * PBS_SELECT_TAU and PBS_SELECT_SAMPLE it is the largest number of
 * candidate blocks (the permuted or natural blocks of earlier segments);
 * for PBS_SELECT_TOPK the top-k budget plus the forced band and sink
 * blocks, capped by the candidates.  The flag bits of mode are ignored.
 * Returns PBS_ERR_INVALID_ARG for a bad geometry.                          */
int pbs_select_capacity(int64_t N, int blk, int seg, int mode,
                        double density_or_tau, int band, int n_sink);

/* pbs_select: for each query block i of every (b, hq), the ascending list
 * of permuted key blocks pb (blocks of segments before block i's own) that
 * pbs_attn_fwd shall visit besides block i's own segment.
 *   Qbar_i = sum of the rows of query block i; Kbar_pb = sum of K rows
 *   perm[pb*blk .. pb*blk+blk-1]; block score S = Qbar_i . Kbar_pb (fp32).
 *   Forced blocks: those holding a sink position (< n_sink) or one of the
 *   `band` most recent keys of any query of the block.
 *   mode PBS_SELECT_TOPK: listed count = max(|forced|, ceil(rho*(i+1)) - D_i)
 *     with rho = density rounded to per-mille, D_i = causal blocks of block
 *     i's own segment; forced first, then highest S, ties to lower pb.
 *   mode PBS_SELECT_TAU: softmax (fp64) over S/(blk^2 sqrt(D)) of the
 *     candidates and of the natural blocks of the own segment; after the
 *     forced blocks, add candidates by descending S while the accumulated
 *     mass (own segment included) is below tau.  tau >= 1 lists all.
 * counts: device int32 [B, Hq, N/blk]; idx: device int32
 * [B, Hq, N/blk, cap]; entries at and after counts[...] are unspecified.
 *   mode PBS_SELECT_SAMPLE: a SampleAttention-style selector over natural
 *     key blocks ("SampleAttention", Technical Deep Dive, Stage 1 Trunk
 *     Sampling and Stage 2 Score-Based Filtering).  The sampled queries are
 *     the last block of every segment; their softmax probabilities (scale
 *     1/sqrt(D)) are summed per key column and per slash offset q - k; each
 *     family keeps its highest entries up to the one at which the
 *     accumulated score reaches density_or_tau (the CIA target, > 0) of its
 *     total, ties to the lower index; block i lists every earlier-segment
 *     block holding a kept column, or a key q - d for one of its queries q
 *     and a kept offset d.  perm is not read (may be NULL): the lists index
 *     natural key blocks, to be attended with the identity permutation.
 *     band, n_sink and the flags do not apply.  ws: pbs_workspace_size(
 *     PBS_OP_SELECT_SAMPLE, ...) bytes.  The probabilities and their sums
 *     within a 128-key tile are fp32, the sums across tiles fp64, so a
 *     column or slash whose accumulated score lies within about 1e-6
 *     (relative) of the cut may be decided differently from an fp64
 *     reference.  Q and K are read through TMA tensor maps: a zero head
 *     or batch stride over more than one head or batch entry (a broadcast
 *     view) returns PBS_ERR_UNSUPPORTED.
 * With mode | PBS_SELECT_PERM_PER_SEGMENT, perm is [B, Hkv, nseg, N] from
 * pbs_permute_segmented and block i pools and scores the keys of its own
 * segment's permutation; ws then needs pbs_workspace_size(
 * PBS_OP_SELECT_SEGMENTED, ...) bytes.
 * With mode | PBS_SELECT_SCORE_ORDER the same blocks are listed in visiting
 * order instead of ascending: the forced blocks first (ascending), then the
 * others by descending S, ties to the lower pb -- the descending estimated
 * importance in which S2O's Pass 2 processes candidates ("S2O ...",
 * Technical Summary, 2. Early-Stopping Rule); pbs_attn_fwd_early_stop
 * consumes lists in this order.
 * Returns PBS_ERR_CAPACITY if cap < pbs_select_capacity(...).               */
int pbs_select(const pbs_tensor* Q, const pbs_tensor* K, const int32_t* perm,
               int blk, int seg, int mode, double density_or_tau, int band,
               int n_sink, int32_t* counts, int32_t* idx, int cap, void* ws,
               size_t ws_bytes, void* stream);

/* pbs_attn_fwd: O[b,hq,q] = sum_k softmax_k(scale * Q[q].K[k]) V[k] over the
 * key set of q's block i: the keys of i's own segment up to q (natural
 * order, causal) plus, for each listed pb, keys perm[b,hkv,pb*blk + r].
 *   perm: device int32 [B, Hkv, N] (any source; each permuted block must
 *     map into its own segment); counts/idx as produced by pbs_select.
 *   gate_thr: NULL, or device fp32 [B, Hq, N/blk] in raw q.k units: a tile
 *     other than block i's own whose largest visible raw q.k is below
 *     gate_thr[b,hq,i] adds nothing (no PV product, no softmax update;
 *     its V rows are still gathered, ahead of the decision).
 *   O: bf16 output, same shape as Q.  lse: NULL or device fp32 [B, Hq, N],
 *     natural-log normaliser of the scaled logits.
 *   stats: NULL or device int64[2], incremented by (tiles whose QK^T was
 *     computed, tiles gated off); the caller zeroes it.
 * Result depends on the set of listed blocks, not on their order.          */
int pbs_attn_fwd(const pbs_tensor* Q, const pbs_tensor* K, const pbs_tensor* V,
                 const int32_t* perm, const int32_t* counts, const int32_t* idx,
                 int cap, int blk, int seg, const float* gate_thr,
                 float softmax_scale, pbs_tensor* O, float* lse,
                 long long* stats, void* ws, size_t ws_bytes, void* stream);

/* pbs_attn_fwd_early_stop: pbs_attn_fwd without gating, where Pass 2
 * visits each block's listed permuted blocks in the order given (entries
 * must be distinct; a repeated entry is dropped and sets the device error
 * word) and stops early ("S2O ...", Technical Summary, 2. Early-Stopping
 * Rule and 3. Kernel Implementation):
 *   after each Pass-2 tile, every query row r of the block has a marginal
 *   gain dl_r / l_r -- the tile's exponential mass over the row's mass
 *   accumulated so far (own segment included), both in the running-max
 *   frame; when the gains of all rows of the block are below stop_tau, the
 *   remaining listed blocks are skipped (the tile just run stays in).
 *   stop_tau = 0 never stops; stop_tau > 1 stops after the first listed
 *   block.  Pass 1 (the own segment) always runs in full.
 *   stop_tau: finite, >= 0.  Other arguments as for pbs_attn_fwd.
 *   stats: NULL or device int64[2], incremented by (tiles whose QK^T was
 *     computed, listed tiles the rule skipped); the caller zeroes it.
 * The stop decisions are taken in fp32 on the kernel's running sums.       */
int pbs_attn_fwd_early_stop(const pbs_tensor* Q, const pbs_tensor* K, const pbs_tensor* V,
                            const int32_t* perm, const int32_t* counts, const int32_t* idx,
                            int cap, int blk, int seg, float stop_tau, float softmax_scale,
                            pbs_tensor* O, float* lse, long long* stats, void* stream);

/* pbs_select_qperm: pbs_select over permuted query blocks.  Query block i
 * is made of the queries at positions qperm[b, hq, i*blk .. i*blk+blk-1]
 * (all in block i's segment; an entry outside it sets the device error word
 * and is left out of the pooled sum); its pooled query is their sum, and
 * candidates, budget and rule are those of pbs_select for block i.  mode is
 * PBS_SELECT_TOPK or PBS_SELECT_TAU, with no flag bits; no band.  Other
 * arguments as for pbs_select; `cap` as pbs_select_capacity gives with
 * band = 0.                                                                */
int pbs_select_qperm(const pbs_tensor* Q, const pbs_tensor* K, const int32_t* perm, const int32_t* qperm,
                     int blk, int seg, int mode, double density_or_tau, int n_sink, int32_t* counts,
                     int32_t* idx, int cap, void* ws, size_t ws_bytes, void* stream);

/* pbs_attn_fwd_qperm: pbs_attn_fwd over permuted query blocks ("S2O ...",
 * Technical Summary, 1. Online Permutation via Index-Driven Loading, Query
 * Permutation and Coordinate-Planned Loading).  Row r of query block i is
 * the query at q = qperm[b, hq, i*blk + r]; it attends the keys of its own
 * segment up to q (Pass 1: natural blocks with an element-wise causal mask)
 * and the keys of block i's listed permuted blocks (Pass 2).  O[b, hq, q]
 * and lse[b, hq, q] are written at the query's original position.  No
 * gating, no early stopping.  Other arguments as for pbs_attn_fwd.        */
int pbs_attn_fwd_qperm(const pbs_tensor* Q, const pbs_tensor* K, const pbs_tensor* V, const int32_t* perm,
                       const int32_t* qperm, const int32_t* counts, const int32_t* idx, int cap, int blk, int seg,
                       float softmax_scale, pbs_tensor* O, float* lse, long long* stats, void* stream);

/* pbs_attn_fwd_ex: pbs_attn_fwd and pbs_attn_fwd_early_stop in one call.
 *   flags: PBS_ATTN_EARLY_STOP -- lists in visiting order, stop_tau as for
 *            pbs_attn_fwd_early_stop (gate_thr must then be NULL);
 *          PBS_ATTN_PERM_PER_SEGMENT -- perm is [B, Hkv, nseg, N] from
 *            pbs_permute_segmented and each query block reads its segment's;
 *          PBS_ATTN_CTA_PAIR -- where D = blk = 128, Hq / Hkv is a multiple
 *            of 4 and neither gating nor early stopping is asked for, run
 *            the CTA-pair kernel: four query heads of a KV head per cluster
 *            of two CTAs, tensor-core MMAs spanning both (M = 256), each CTA
 *            gathering half of every K/V tile.  Same results (the same
 *            arithmetic per head, bit for bit); elsewhere the flag is
 *            ignored.
 *   Other arguments as for pbs_attn_fwd; unknown flags are rejected.       */
int pbs_attn_fwd_ex(const pbs_tensor* Q, const pbs_tensor* K, const pbs_tensor* V, const int32_t* perm,
                    const int32_t* counts, const int32_t* idx, int cap, int blk, int seg, unsigned flags,
                    const float* gate_thr, float stop_tau, float softmax_scale, pbs_tensor* O, float* lse,
                    long long* stats, void* stream);

/* Synchronises `stream`, then returns and clears the sticky device error
 * word of the current device (PBS_OK if no device-side check failed).      */
int pbs_check_device(void* stream);

/* pbs_test_inject_timeout: a test hook for the failure path; the pages have
 * no counterpart.  With limit_polls > 0, every later pbs_attn_fwd* launch
 * (from any host thread) withholds the "query tile landed" arrival that its
 * MMA role waits for, and bounds the waits of the producer, MMA and softmax
 * roles by limit_polls polls: the wait for the query tile runs out, the
 * kernel raises its abort flag, every role leaves its loop, the tensor core
 * is drained (that wait keeps its normal bound), tensor memory is freed and
 * PBS_ERR_TIMEOUT is left in the device error word, with no fault.
 * limit_polls = 0 (the default) turns the hook off.  Not for production
 * use: outputs of a launch made while it is on are undefined.             */
void pbs_test_inject_timeout(unsigned limit_polls);

/* Message of the most recent failing call on this host thread ("" if none). */
const char* pbs_get_last_error(void);

/* Library version string. */
const char* pbs_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PBS_H_ */
