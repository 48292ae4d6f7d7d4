// C-ABI front end of libpbs.so: argument validation, workspace carving,
// the sticky device error word, and kernel launches.  See include/pbs.h for
// the contract of every entry point.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "pbs_internal.h"

namespace pbs {
// Sticky device error word (0 = no error), set by kernels' bounds checks and
// bounded waits; read and cleared by pbs_check_device.
__device__ int g_device_error = 0;
}  // namespace pbs

namespace {

thread_local std::string g_last_error;

// Failure-path test hook (pbs_test_inject_timeout): 0 in normal use.
std::atomic<unsigned> g_test_wait_limit{0};

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int ok() {
  g_last_error.clear();
  return PBS_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(PBS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Device address of the error word, cached per device.
int* device_error_word() {
  static std::mutex mu;
  static int* cache[128] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, pbs::g_device_error) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<int*>(ptr);
  }
  return cache[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_tensor(const pbs_tensor* t, const char* name, pbs::TensorDesc* out) {
  if (!t) return fail(PBS_ERR_INVALID_ARG, "%s: null descriptor", name);
  if (!t->ptr) return fail(PBS_ERR_INVALID_ARG, "%s: null data pointer", name);
  if (t->B <= 0 || t->H <= 0 || t->N <= 0 || t->D <= 0)
    return fail(PBS_ERR_INVALID_ARG, "%s: non-positive shape [%lld,%lld,%lld,%lld]", name,
                (long long)t->B, (long long)t->H, (long long)t->N, (long long)t->D);
  if (t->D != 64 && t->D != 128)
    return fail(PBS_ERR_UNSUPPORTED, "%s: head dim %lld not in {64,128}", name, (long long)t->D);
  if (t->N >= (1ll << 31)) return fail(PBS_ERR_UNSUPPORTED, "%s: N >= 2^31", name);
  if (!aligned16(t->ptr)) return fail(PBS_ERR_UNSUPPORTED, "%s: pointer not 16-byte aligned", name);
  if (t->sN < t->D || (t->sN % 8) || (t->sH % 8) || (t->sB % 8) || t->sH < 0 || t->sB < 0)
    return fail(PBS_ERR_UNSUPPORTED,
                "%s: strides (%lld,%lld,%lld) must be non-negative multiples of 8 with sN >= D",
                name, (long long)t->sB, (long long)t->sH, (long long)t->sN);
  *out = pbs::TensorDesc{t->ptr, t->B, t->H, t->N, t->D, t->sB, t->sH, t->sN};
  return PBS_OK;
}

int check_geometry(const pbs::TensorDesc& Q, const pbs::TensorDesc& K, int blk, int seg) {
  if (blk != 64 && blk != 128) return fail(PBS_ERR_UNSUPPORTED, "blk %d not in {64,128}", blk);
  if (seg < blk || seg % blk) return fail(PBS_ERR_INVALID_ARG, "seg %d must be a positive multiple of blk %d", seg, blk);
  if (seg > 8192) return fail(PBS_ERR_UNSUPPORTED, "seg %d > 8192", seg);
  if (Q.B != K.B || Q.N != K.N || Q.D != K.D)
    return fail(PBS_ERR_INVALID_ARG, "Q and K disagree on B, N or D");
  if (Q.H % K.H) return fail(PBS_ERR_INVALID_ARG, "Hq %lld not a multiple of Hkv %lld", (long long)Q.H, (long long)K.H);
  if (Q.N % blk) return fail(PBS_ERR_UNSUPPORTED, "N %lld not a multiple of blk %d", (long long)Q.N, blk);
  if (Q.B > 65535 || Q.H > 65535) return fail(PBS_ERR_UNSUPPORTED, "B or H above 65535");
  return PBS_OK;
}

struct SelectWs {
  size_t qbar, kperm, knat, inv, scores, total;
};

// perm_nseg permutations per KV head (1, or one per query segment).
SelectWs select_ws(const pbs::TensorDesc& Q, const pbs::TensorDesc& K, int blk, int64_t perm_nseg = 1) {
  const size_t nb = static_cast<size_t>(Q.N / blk);
  const size_t np = static_cast<size_t>(perm_nseg);
  SelectWs w;
  w.qbar = 0;
  w.kperm = w.qbar + align256(static_cast<size_t>(Q.B * Q.H) * nb * Q.D * 4);
  w.knat = w.kperm + align256(static_cast<size_t>(K.B * K.H) * np * nb * K.D * 4);
  w.inv = w.knat + align256(static_cast<size_t>(K.B * K.H) * nb * K.D * 4);
  w.scores = w.inv + align256(static_cast<size_t>(K.B * K.H) * np * K.N * 4);
  w.total = w.scores + align256(static_cast<size_t>(Q.B * Q.H) * nb * nb * 4);
  return w;
}

// The sample selector's workspace: column and slash scores (fp64) and the
// two kept-entry bitmaps per (b, hq), in the SelectWs slots qbar, kperm,
// knat and inv.
SelectWs sample_ws(const pbs::TensorDesc& Q) {
  const size_t rows = static_cast<size_t>(Q.B * Q.H);
  const size_t words = static_cast<size_t>((Q.N + 31) / 32);
  SelectWs w;
  w.qbar = 0;
  w.kperm = w.qbar + align256(rows * Q.N * 8);
  w.knat = w.kperm + align256(rows * Q.N * 8);
  w.inv = w.knat + align256(rows * words * 4);
  w.scores = w.inv + align256(rows * words * 4);
  w.total = w.scores;
  return w;
}

int check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return PBS_OK;
  if (!ws) return fail(PBS_ERR_INVALID_ARG, "workspace is null but %zu bytes are needed", need);
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(PBS_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if (ws_bytes < need) return fail(PBS_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", ws_bytes, need);
  return PBS_OK;
}

int64_t rho_permille(double density) { return static_cast<int64_t>(std::llround(density * 1000.0)); }

}  // namespace

namespace pbs {

int api_fail(int code, const char* msg) { return fail(code, "%s", msg); }

int api_ok() { return ok(); }

int* api_device_error_word() { return device_error_word(); }

int api_validate_permute(const pbs_tensor* Qt, const pbs_tensor* Kt, int blk, int seg, int n_sink,
                         const int32_t* perm, TensorDesc* Q, TensorDesc* K) {
  int rc;
  if ((rc = check_tensor(Qt, "Q", Q)) || (rc = check_tensor(Kt, "K", K))) return rc;
  if ((rc = check_geometry(*Q, *K, blk, seg))) return rc;
  if (!perm) return fail(PBS_ERR_INVALID_ARG, "perm is null");
  if (n_sink < 0) return fail(PBS_ERR_INVALID_ARG, "n_sink %d < 0", n_sink);
  return PBS_OK;
}

}  // namespace pbs

namespace {
int attn_common(const pbs_tensor* Qt, const pbs_tensor* Kt, const pbs_tensor* Vt,
                const int32_t* perm, const int32_t* counts, const int32_t* idx, int cap, int blk,
                int seg, const float* gate_thr, int early_stop, float stop_tau, int per_segment,
                float softmax_scale, pbs_tensor* Ot, float* lse, long long* stats, void* stream,
                int cta_pair = 0, const int32_t* qperm = nullptr) {
  pbs::TensorDesc Q, K, V, O;
  int rc;
  if ((rc = check_tensor(Qt, "Q", &Q)) || (rc = check_tensor(Kt, "K", &K)) ||
      (rc = check_tensor(Vt, "V", &V)) || (rc = check_tensor(Ot, "O", &O)))
    return rc;
  if ((rc = check_geometry(Q, K, blk, seg))) return rc;
  if (V.B != K.B || V.H != K.H || V.N != K.N || V.D != K.D)
    return fail(PBS_ERR_INVALID_ARG, "V shape differs from K");
  if (O.B != Q.B || O.H != Q.H || O.N != Q.N || O.D != Q.D)
    return fail(PBS_ERR_INVALID_ARG, "O shape differs from Q");
  if (!perm || !counts || !idx) return fail(PBS_ERR_INVALID_ARG, "perm, counts or idx is null");
  if (cap < 1) return fail(PBS_ERR_INVALID_ARG, "cap %d < 1", cap);
  if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale))
    return fail(PBS_ERR_INVALID_ARG, "softmax_scale must be positive and finite");
  int* err = device_error_word();
  if (!err) return fail(PBS_ERR_CUDA, "cannot resolve the device error word");
  pbs::AttnParams p;
  p.Q = Q;
  p.K = K;
  p.V = V;
  p.O = O;
  p.perm = perm;
  p.counts = counts;
  p.idx = idx;
  p.qperm = qperm;
  p.cap = cap;
  p.blk = blk;
  p.seg = seg;
  p.nb = static_cast<int>(Q.N / blk);
  p.G = static_cast<int>(Q.H / K.H);
  p.gate_thr = gate_thr;
  p.early_stop = early_stop;
  p.stop_tau = stop_tau;
  p.perm_nseg = per_segment ? static_cast<int>((Q.N + seg - 1) / seg) : 1;
  p.cta_pair = cta_pair;
  p.test_wait_limit = g_test_wait_limit.load();
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.lse = lse;
  p.stats = stats;
  p.err = err;
  cudaError_t e = pbs::launch_attn_fwd(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attn_fwd launch");
  return ok();
}
}  // namespace

namespace {
int select_impl(const pbs_tensor* Qt, const pbs_tensor* Kt, const int32_t* perm, const int32_t* qperm, int blk,
                int seg, int mode, double density_or_tau, int band, int n_sink, int32_t* counts, int32_t* idx,
                int cap, void* ws, size_t ws_bytes, void* stream);
}  // namespace

extern "C" {

const char* pbs_version(void) { return "pbs 0.1 (sm_100a)"; }

const char* pbs_get_last_error(void) { return g_last_error.c_str(); }

size_t pbs_workspace_size(int op, const pbs_tensor* Qt, const pbs_tensor* Kt, int blk, int seg) {
  pbs::TensorDesc Q, K;
  if (check_tensor(Qt, "Q", &Q) || check_tensor(Kt, "K", &K)) return 0;
  if (blk != 64 && blk != 128) return 0;
  const int64_t nseg = seg > 0 ? (K.N + seg - 1) / seg : 0;
  switch (op) {
    case PBS_OP_PERMUTE:
      return align256(static_cast<size_t>(K.B * K.H * K.D) * 4);
    case PBS_OP_SELECT:
      return select_ws(Q, K, blk).total;
    case PBS_OP_PERMUTE_SEGMENTED:
      return nseg > 0 ? align256(static_cast<size_t>(K.B * K.H * nseg * K.D) * 8) : 0;
    case PBS_OP_SELECT_SEGMENTED:
      return nseg > 0 ? select_ws(Q, K, blk, nseg).total : 0;
    case PBS_OP_SELECT_SAMPLE:
      return sample_ws(Q).total;
    case PBS_OP_PERMUTE_QUERIES:
      return align256(pbs::permute_queries_ws_bytes(K));
    default:
      return 0;
  }
}

int pbs_permute_segmented(const pbs_tensor* Qt, const pbs_tensor* Kt, int blk, int seg, int n_sink,
                          int32_t* perm, void* ws, size_t ws_bytes, void* stream) {
  pbs::TensorDesc Q, K;
  int rc;
  if ((rc = pbs::api_validate_permute(Qt, Kt, blk, seg, n_sink, perm, &Q, &K))) return rc;
  const int64_t nseg = (K.N + seg - 1) / seg;
  if (nseg > 65535 || K.B * K.H > 65535) return fail(PBS_ERR_UNSUPPORTED, "too many segments or heads");
  if ((rc = check_ws(ws, ws_bytes, align256(static_cast<size_t>(K.B * K.H * nseg * K.D) * 8)))) return rc;
  cudaError_t e = pbs::launch_permute_segmented(Q, K, seg, n_sink, static_cast<double*>(ws), perm,
                                                static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "permute_segmented launch");
  return ok();
}

int pbs_permute_queries(const pbs_tensor* Qt, const pbs_tensor* Kt, int blk, int seg, int32_t* qperm, void* ws,
                        size_t ws_bytes, void* stream) {
  pbs::TensorDesc Q, K;
  int rc;
  if ((rc = pbs::api_validate_permute(Qt, Kt, blk, seg, 0, qperm, &Q, &K))) return rc;
  const int64_t nseg = (Q.N + seg - 1) / seg;
  if (nseg > 65535) return fail(PBS_ERR_UNSUPPORTED, "too many segments");
  if ((rc = check_ws(ws, ws_bytes, align256(pbs::permute_queries_ws_bytes(K))))) return rc;
  cudaError_t e = pbs::launch_permute_queries(Q, K, seg, static_cast<double*>(ws), qperm,
                                              static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "permute_queries launch");
  return ok();
}

int pbs_permute(const pbs_tensor* Qt, const pbs_tensor* Kt, int blk, int seg, int n_sink,
                int32_t* perm, void* ws, size_t ws_bytes, void* stream) {
  pbs::TensorDesc Q, K;
  int rc;
  if ((rc = check_tensor(Qt, "Q", &Q)) || (rc = check_tensor(Kt, "K", &K))) return rc;
  if ((rc = check_geometry(Q, K, blk, seg))) return rc;
  if (!perm) return fail(PBS_ERR_INVALID_ARG, "perm is null");
  if (n_sink < 0) return fail(PBS_ERR_INVALID_ARG, "n_sink %d < 0", n_sink);
  const size_t need = align256(static_cast<size_t>(K.B * K.H * K.D) * 4);
  if ((rc = check_ws(ws, ws_bytes, need))) return rc;
  int* err = device_error_word();
  if (!err) return fail(PBS_ERR_CUDA, "cannot resolve the device error word");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* qhat = static_cast<float*>(ws);
  cudaError_t e = pbs::launch_pool_proxy_query(Q, static_cast<int>(K.H), blk, qhat, s);
  if (e != cudaSuccess) return cuda_fail(e, "pool_proxy_query launch");
  e = pbs::launch_score_sort(K, seg, n_sink, qhat, perm, err, s);
  if (e != cudaSuccess) return cuda_fail(e, "score_sort launch");
  return ok();
}

int pbs_select_capacity(int64_t N, int blk, int seg, int mode, double density_or_tau, int band,
                        int n_sink) {
  if (blk <= 0 || seg < blk || seg % blk || N <= 0 || N % blk)
    return fail(PBS_ERR_INVALID_ARG, "bad geometry for capacity");
  mode &= ~(PBS_SELECT_SCORE_ORDER | PBS_SELECT_PERM_PER_SEGMENT);
  const int64_t nb = N / blk, spb = seg / blk;
  int64_t best = 0;
  const int64_t r = rho_permille(density_or_tau);
  for (int64_t i = 0; i < nb; ++i) {
    const int64_t s = i / spb, ncand = s * spb;
    if (ncand == 0) continue;
    int64_t need;
    if (mode == PBS_SELECT_TAU || mode == PBS_SELECT_SAMPLE) {
      need = ncand;
    } else {
      const int64_t Di = i - s * spb + 1;
      const int64_t sink_ub = n_sink > 0 ? (n_sink + blk - 1) / blk + (n_sink + seg - 1) / seg : 0;
      const int64_t band_ub =
          band > 1 ? std::min<int64_t>(band - 1, spb * (1 + (band - 1 + seg - 1) / seg)) : 0;
      const int64_t target = (r * (i + 1) + 999) / 1000;
      need = std::max<int64_t>(sink_ub + band_ub, target - Di);
    }
    best = std::max(best, std::min(need, ncand));
  }
  return static_cast<int>(best);
}

int pbs_select(const pbs_tensor* Qt, const pbs_tensor* Kt, const int32_t* perm, int blk, int seg,
               int mode, double density_or_tau, int band, int n_sink, int32_t* counts,
               int32_t* idx, int cap, void* ws, size_t ws_bytes, void* stream) {
  return select_impl(Qt, Kt, perm, nullptr, blk, seg, mode, density_or_tau, band, n_sink, counts, idx, cap, ws,
                     ws_bytes, stream);
}

int pbs_select_qperm(const pbs_tensor* Qt, const pbs_tensor* Kt, const int32_t* perm, const int32_t* qperm,
                     int blk, int seg, int mode, double density_or_tau, int n_sink, int32_t* counts,
                     int32_t* idx, int cap, void* ws, size_t ws_bytes, void* stream) {
  if (!qperm) return fail(PBS_ERR_INVALID_ARG, "qperm is null");
  if (mode != PBS_SELECT_TOPK && mode != PBS_SELECT_TAU)
    return fail(PBS_ERR_UNSUPPORTED, "permuted queries take PBS_SELECT_TOPK or PBS_SELECT_TAU without flags");
  return select_impl(Qt, Kt, perm, qperm, blk, seg, mode, density_or_tau, 0, n_sink, counts, idx, cap, ws,
                     ws_bytes, stream);
}

}  // extern "C"

namespace {
int select_impl(const pbs_tensor* Qt, const pbs_tensor* Kt, const int32_t* perm, const int32_t* qperm, int blk,
                int seg, int mode, double density_or_tau, int band, int n_sink, int32_t* counts, int32_t* idx,
                int cap, void* ws, size_t ws_bytes, void* stream) {
  pbs::TensorDesc Q, K;
  int rc;
  if ((rc = check_tensor(Qt, "Q", &Q)) || (rc = check_tensor(Kt, "K", &K))) return rc;
  if ((rc = check_geometry(Q, K, blk, seg))) return rc;
  if (!counts || !idx) return fail(PBS_ERR_INVALID_ARG, "counts or idx is null");
  if (!perm && (mode & 0xF) != PBS_SELECT_SAMPLE) return fail(PBS_ERR_INVALID_ARG, "perm is null");
  const int score_order = (mode & PBS_SELECT_SCORE_ORDER) ? 1 : 0;
  const int per_segment = (mode & PBS_SELECT_PERM_PER_SEGMENT) ? 1 : 0;
  mode &= ~(PBS_SELECT_SCORE_ORDER | PBS_SELECT_PERM_PER_SEGMENT);
  if (mode != PBS_SELECT_TOPK && mode != PBS_SELECT_TAU && mode != PBS_SELECT_SAMPLE)
    return fail(PBS_ERR_INVALID_ARG, "mode %d unknown", mode);
  if (mode == PBS_SELECT_SAMPLE && (score_order || per_segment))
    return fail(PBS_ERR_UNSUPPORTED, "the sample selector lists natural blocks in ascending order only");
  if (mode == PBS_SELECT_SAMPLE && !(density_or_tau > 0.0))
    return fail(PBS_ERR_INVALID_ARG, "CIA target %g must be positive", density_or_tau);
  if (mode == PBS_SELECT_SAMPLE &&
      (Q.B * Q.H * ((Q.N + seg - 1) / seg) >= (1ll << 31) || Q.B * Q.H * (Q.N / blk) >= (1ll << 31)))
    return fail(PBS_ERR_UNSUPPORTED, "B * Hq * segments or B * Hq * blocks above 2^31");
  if (mode == PBS_SELECT_SAMPLE && ((Q.H > 1 && Q.sH == 0) || (Q.B > 1 && Q.sB == 0) ||
                                    (K.H > 1 && K.sH == 0) || (K.B > 1 && K.sB == 0)))
    return fail(PBS_ERR_UNSUPPORTED, "the sample selector reads Q and K by TMA: zero head/batch strides "
                                     "(broadcast views) are not supported");
  if (!(density_or_tau >= 0.0) || (mode == PBS_SELECT_TOPK && density_or_tau > 1.0))
    return fail(PBS_ERR_INVALID_ARG, "density/tau %g out of range", density_or_tau);
  if (band < 0 || n_sink < 0) return fail(PBS_ERR_INVALID_ARG, "band/n_sink negative");
  const int64_t nb = Q.N / blk;
  if (nb > 8192) return fail(PBS_ERR_UNSUPPORTED, "N/blk = %lld > 8192 blocks", (long long)nb);
  const int need_cap = pbs_select_capacity(Q.N, blk, seg, mode, density_or_tau, band, n_sink);
  if (cap < need_cap || cap < 1)
    return fail(PBS_ERR_CAPACITY, "cap %d < required %d", cap, std::max(need_cap, 1));
  const int64_t perm_nseg = per_segment ? (Q.N + seg - 1) / seg : 1;
  const SelectWs w = mode == PBS_SELECT_SAMPLE ? sample_ws(Q) : select_ws(Q, K, blk, perm_nseg);
  if ((rc = check_ws(ws, ws_bytes, w.total))) return rc;
  int* err = device_error_word();
  if (!err) return fail(PBS_ERR_CUDA, "cannot resolve the device error word");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(ws);
  float* qbar = reinterpret_cast<float*>(base + w.qbar);
  float* kperm = reinterpret_cast<float*>(base + w.kperm);
  float* knat = reinterpret_cast<float*>(base + w.knat);
  int32_t* inv = reinterpret_cast<int32_t*>(base + w.inv);
  float* scores = reinterpret_cast<float*>(base + w.scores);
  if (mode == PBS_SELECT_SAMPLE) {
    pbs::SelectParams p;
    p.B = static_cast<int>(Q.B);
    p.Hq = static_cast<int>(Q.H);
    p.Hkv = static_cast<int>(K.H);
    p.D = static_cast<int>(Q.D);
    p.blk = blk;
    p.seg = seg;
    p.nb = static_cast<int>(nb);
    p.mode = mode;
    p.score_order = 0;
    p.perm_nseg = 1;
    p.band = 0;
    p.n_sink = 0;
    p.cap = cap;
    p.N = Q.N;
    p.rho_permille = 0;
    p.tau = density_or_tau;
    const float scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(Q.D)));
    cudaError_t e = pbs::launch_select_sample(p, Q, K, scale_log2, reinterpret_cast<double*>(base + w.qbar),
                                              reinterpret_cast<double*>(base + w.kperm),
                                              reinterpret_cast<uint32_t*>(base + w.knat),
                                              reinterpret_cast<uint32_t*>(base + w.inv), counts, idx, err, s);
    if (e != cudaSuccess) return cuda_fail(e, "select_sample launch");
    return ok();
  }
  cudaError_t e = pbs::launch_pool_query_blocks(Q, blk, qperm, seg, err, qbar, s);
  if (e != cudaSuccess) return cuda_fail(e, "pool_query_blocks launch");
  e = pbs::launch_pool_key_blocks(K, perm, static_cast<int>(perm_nseg), blk, seg, mode == PBS_SELECT_TAU, kperm,
                                  knat, inv, err, s);
  if (e != cudaSuccess) return cuda_fail(e, "pool_key_blocks launch");
  pbs::SelectParams p;
  p.B = static_cast<int>(Q.B);
  p.Hq = static_cast<int>(Q.H);
  p.Hkv = static_cast<int>(K.H);
  p.D = static_cast<int>(Q.D);
  p.blk = blk;
  p.seg = seg;
  p.nb = static_cast<int>(nb);
  p.mode = mode;
  p.score_order = score_order;
  p.perm_nseg = static_cast<int>(perm_nseg);
  p.band = band;
  p.n_sink = n_sink;
  p.cap = cap;
  p.N = Q.N;
  p.rho_permille = rho_permille(density_or_tau);
  p.tau = density_or_tau;
  e = pbs::launch_select_blocks(p, qbar, kperm, knat, inv, scores, counts, idx, err, s);
  if (e != cudaSuccess) return cuda_fail(e, "select_blocks launch");
  return ok();
}

}  // namespace

extern "C" {

int pbs_attn_fwd(const pbs_tensor* Qt, const pbs_tensor* Kt, const pbs_tensor* Vt,
                 const int32_t* perm, const int32_t* counts, const int32_t* idx, int cap, int blk,
                 int seg, const float* gate_thr, float softmax_scale, pbs_tensor* Ot, float* lse,
                 long long* stats, void* ws, size_t ws_bytes, void* stream) {
  (void)ws;
  (void)ws_bytes;
  return attn_common(Qt, Kt, Vt, perm, counts, idx, cap, blk, seg, gate_thr, 0, 0.0f, 0, softmax_scale,
                     Ot, lse, stats, stream);
}

int pbs_attn_fwd_early_stop(const pbs_tensor* Qt, const pbs_tensor* Kt, const pbs_tensor* Vt,
                            const int32_t* perm, const int32_t* counts, const int32_t* idx,
                            int cap, int blk, int seg, float stop_tau, float softmax_scale,
                            pbs_tensor* Ot, float* lse, long long* stats, void* stream) {
  if (!(stop_tau >= 0.0f) || !std::isfinite(stop_tau))
    return fail(PBS_ERR_INVALID_ARG, "stop_tau must be finite and >= 0");
  return attn_common(Qt, Kt, Vt, perm, counts, idx, cap, blk, seg, nullptr, 1, stop_tau, 0, softmax_scale,
                     Ot, lse, stats, stream);
}

int pbs_attn_fwd_ex(const pbs_tensor* Qt, const pbs_tensor* Kt, const pbs_tensor* Vt, const int32_t* perm,
                    const int32_t* counts, const int32_t* idx, int cap, int blk, int seg, unsigned flags,
                    const float* gate_thr, float stop_tau, float softmax_scale, pbs_tensor* Ot, float* lse,
                    long long* stats, void* stream) {
  if (flags & ~static_cast<unsigned>(PBS_ATTN_EARLY_STOP | PBS_ATTN_PERM_PER_SEGMENT | PBS_ATTN_CTA_PAIR))
    return fail(PBS_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  const int early = (flags & PBS_ATTN_EARLY_STOP) ? 1 : 0;
  if (early) {
    if (gate_thr) return fail(PBS_ERR_UNSUPPORTED, "early stopping with a gate is not supported");
    if (!(stop_tau >= 0.0f) || !std::isfinite(stop_tau))
      return fail(PBS_ERR_INVALID_ARG, "stop_tau must be finite and >= 0");
  }
  return attn_common(Qt, Kt, Vt, perm, counts, idx, cap, blk, seg, gate_thr, early, early ? stop_tau : 0.0f,
                     (flags & PBS_ATTN_PERM_PER_SEGMENT) ? 1 : 0, softmax_scale, Ot, lse, stats, stream,
                     (flags & PBS_ATTN_CTA_PAIR) ? 1 : 0);
}

void pbs_test_inject_timeout(unsigned limit_polls) { g_test_wait_limit.store(limit_polls); }

int pbs_attn_fwd_qperm(const pbs_tensor* Qt, const pbs_tensor* Kt, const pbs_tensor* Vt, const int32_t* perm,
                       const int32_t* qperm, const int32_t* counts, const int32_t* idx, int cap, int blk, int seg,
                       float softmax_scale, pbs_tensor* Ot, float* lse, long long* stats, void* stream) {
  if (!qperm) return fail(PBS_ERR_INVALID_ARG, "qperm is null");
  return attn_common(Qt, Kt, Vt, perm, counts, idx, cap, blk, seg, nullptr, 0, 0.0f, 0, softmax_scale, Ot, lse,
                     stats, stream, 0, qperm);
}

int pbs_check_device(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, pbs::g_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(pbs::g_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
    return fail(v, v == PBS_ERR_TIMEOUT ? "device: a bounded wait gave up"
                                        : "device: an index failed its bounds check");
  }
  return ok();
}

}  // extern "C"
