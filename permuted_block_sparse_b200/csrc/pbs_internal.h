// Internal launcher interface between the C-ABI front end (api.cu) and the
// kernel translation units.  Host-only; not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pbs.h"

namespace pbs {

struct TensorDesc {       // validated pbs_tensor, strides in elements
  const void* ptr;
  int64_t B, H, N, D, sB, sH, sN;
};

// Tensor map of a [B, H, N, D] bf16 tensor for boxes of 64 columns x 128
// rows, 128-byte swizzle, rows past N read as zeros; false if the tensor
// cannot be described (a zero head or batch stride over several heads or
// batches) or the driver entry point is missing.  (select_sample.cu)
bool encode_rows_map(CUtensorMap* map, const TensorDesc& t);

// pbs_permute launchers ---------------------------------------------------
cudaError_t launch_pool_proxy_query(const TensorDesc& Q, int Hkv, int blk, float* qhat,
                                    cudaStream_t s);
cudaError_t launch_score_sort(const TensorDesc& K, int seg, int n_sink, const float* qhat,
                              int32_t* perm, int* err, cudaStream_t s);

// pbs_select launchers ----------------------------------------------------
cudaError_t launch_pool_query_blocks(const TensorDesc& Q, int blk, const int32_t* qperm, int seg, int* err,
                                     float* qbar, cudaStream_t s);
// pbs_permute_queries: guide vectors and the per-segment query sort.
size_t permute_queries_ws_bytes(const TensorDesc& K);
cudaError_t launch_permute_queries(const TensorDesc& Q, const TensorDesc& K, int seg, double* ws, int32_t* qperm,
                                   cudaStream_t s);
cudaError_t launch_pool_key_blocks(const TensorDesc& K, const int32_t* perm, int perm_nseg, int blk,
                                   int seg, bool natural, float* kbar_perm, float* kbar_nat,
                                   int32_t* inv, int* err, cudaStream_t s);
cudaError_t launch_permute_segmented(const TensorDesc& Q, const TensorDesc& K, int seg, int n_sink,
                                     double* qs, int32_t* perm, cudaStream_t s);
struct SelectParams {
  int B, Hq, Hkv, D, blk, seg, nb, mode, band, n_sink, cap;
  int score_order;        // lists in visiting order instead of ascending
  int perm_nseg;          // 1: one permutation per KV head; else one per query segment
  int64_t N;
  int64_t rho_permille;   // top-k density in per-mille
  double tau;
};
cudaError_t launch_select_sample(const SelectParams& p, const TensorDesc& Q, const TensorDesc& K,
                                 float scale_log2, double* col, double* sl, uint32_t* keep_col,
                                 uint32_t* keep_sl, int32_t* counts, int32_t* idx, int* err, cudaStream_t s);
cudaError_t launch_select_blocks(const SelectParams& p, const float* qbar, const float* kbar_perm,
                                 const float* kbar_nat, const int32_t* inv, float* scores, int32_t* counts,
                                 int32_t* idx, int* err, cudaStream_t s);

// Front-end helpers shared by C-ABI entry points defined outside api.cu.
// They set the calling thread's last-error message like the entry points in
// api.cu do.
int api_fail(int code, const char* msg);
int api_ok();
int* api_device_error_word();
int api_validate_permute(const pbs_tensor* Qt, const pbs_tensor* Kt, int blk, int seg, int n_sink,
                         const int32_t* perm, TensorDesc* Q, TensorDesc* K);

// pbs_attn_fwd launcher ---------------------------------------------------
struct AttnParams {
  TensorDesc Q, K, V, O;
  const int32_t* perm;
  const int32_t* counts;
  const int32_t* idx;
  const int32_t* qperm;   // NULL, or S2O's query permutation [B, Hq, N]
  int cap, blk, seg, nb, G;
  const float* gate_thr;
  int early_stop;         // S2O early stopping: lists in visiting order, cut by stop_tau
  int perm_nseg;          // 1: one permutation per KV head; else one per query segment
  int cta_pair;           // run the CTA-pair kernel where it applies
  int tma;                // set by the launcher: Q and natural K/V tiles by TMA
  // Failure-path test hook (0 in normal use): bound the role waits by this
  // many polls and withhold the "Q landed" arrival, so the kernel times out.
  uint32_t test_wait_limit;
  float stop_tau;
  float scale_log2;       // softmax scale * log2(e)
  float* lse;
  long long* stats;
  int* err;
};
cudaError_t launch_attn_fwd(const AttnParams& p, cudaStream_t s);
// The CTA-pair forward (four query heads per pair of CTAs); used by
// launch_attn_fwd where it applies.
bool attn_fwd_pair_applies(const AttnParams& p);
cudaError_t launch_attn_fwd_pair(const AttnParams& p, cudaStream_t s);

}  // namespace pbs
