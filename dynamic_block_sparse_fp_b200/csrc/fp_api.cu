// fp_api.cu -- the extern "C" entry points of include/fp.h: argument
// validation (on the host, before any launch), workspace layout, dispatch to
// the stage launchers, and the per-device status word.
#include <math.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "fp_internal.cuh"

#define FP_API extern "C" __attribute__((visibility("default")))

namespace fpi {

__device__ int g_fp_status;  // first device-side error since the last read

int *device_status_ptr() {
  static int *ptrs[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fp_status) == cudaSuccess) ptrs[dev] = static_cast<int *>(p);
  }
  return ptrs[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  // a function-local static is initialised once, under the C++ runtime's lock
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    cudaDriverEntryPointQueryResult qr;
    void *p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) !=
            cudaSuccess ||
        qr != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// The streams of fp_prefill_attn_host besides the caller's: host-to-device
// copies, device-to-host copies, and a second compute stream for every other
// unit; created once per device on first use and kept for the life of the
// process, like the status word.
bool host_streams(cudaStream_t *in, cudaStream_t *out, cudaStream_t *comp) {
  static std::mutex mu;
  static cudaStream_t s_in[64] = {nullptr}, s_out[64] = {nullptr}, s_comp[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(mu);
  for (cudaStream_t *s : {&s_in[dev], &s_out[dev], &s_comp[dev]})
    if (!*s && cudaStreamCreateWithFlags(s, cudaStreamNonBlocking) != cudaSuccess) return false;
  *in = s_in[dev];
  *out = s_out[dev];
  *comp = s_comp[dev];
  return true;
}

namespace {

fp_status check_shape(const fp_shape *s, Dims *D) {
  if (!s) return FP_ERR_NULL;
  if (s->dtype != FP_BF16 && s->dtype != FP_F32) return FP_ERR_DTYPE;
  if (s->batch < 1 || s->n_q_heads < 1 || s->n_kv_heads < 1 || s->seq_len < 1)
    return FP_ERR_SHAPE;
  if (s->n_q_heads % s->n_kv_heads != 0) return FP_ERR_SHAPE;
  if (s->block_size != 64 && s->block_size != 128) return FP_ERR_SHAPE;
  if (s->head_dim != 64 && s->head_dim != 128) return FP_ERR_SHAPE;
  // a partial last block holds the seq_len - (nb - 1) * block_size tokens left
  const long long nb = (s->seq_len + s->block_size - 1) / s->block_size;
  if (nb > 4096) return FP_ERR_SHAPE;
  // row coordinates of every (batch, head, token) must fit in int32
  if ((long long)s->batch * s->n_q_heads * s->seq_len >= (1ll << 31)) return FP_ERR_SHAPE;
  D->bt = s->batch;
  D->hq = s->n_q_heads;
  D->hkv = s->n_kv_heads;
  D->n = s->seq_len;
  D->d = s->head_dim;
  D->bs = s->block_size;
  D->nb = int(nb);
  D->g = s->n_q_heads / s->n_kv_heads;
  D->t_pairs = nb * (nb + 1) / 2;
  D->dtype = s->dtype;
  return FP_OK;
}

fp_status check_attn_shape(const Dims &D) {
  if (D.dtype == FP_BF16 && D.d != 128) return FP_ERR_SHAPE;
  return FP_OK;
}

fp_status check_params(const fp_params *p) {
  if (!p) return FP_ERR_NULL;
  if (!(p->gamma > 0.f) || !(p->gamma <= 1.f)) return FP_ERR_PARAM;
  if (!(p->tau >= 0.f) || isinf(p->tau)) return FP_ERR_PARAM;
  if (p->min_budget < 0) return FP_ERR_PARAM;
  if (p->qa_mode != FP_QA_FLATTENED && p->qa_mode != FP_QA_QUERYWISE) return FP_ERR_PARAM;
  if (p->vs_mode != FP_VS_TOKENS && p->vs_mode != FP_VS_BLOCKS) return FP_ERR_PARAM;
  return FP_OK;
}

SelectBudgets budgets(const Dims &D, const fp_params &p) {
  SelectBudgets b;
  const long long T = D.t_pairs, nb = D.nb, bs = D.bs;
  long long lo = nb * ((p.min_budget + bs - 1) / bs);
  if (lo > T) lo = T;
  long long hi = p.max_budget <= 0 ? T : nb * (p.max_budget / bs);
  if (hi > T) hi = T;
  b.qa_lo = lo < hi ? lo : hi;
  b.qa_hi = hi;
  int vlo = p.min_budget < D.n ? p.min_budget : D.n;
  int vhi = p.max_budget <= 0 ? D.n : (p.max_budget < D.n ? p.max_budget : D.n);
  b.vs_lo = vlo < vhi ? vlo : vhi;
  b.vs_hi = vhi;
  b.qa_mode = p.qa_mode;
  b.row_lo = int((p.min_budget + bs - 1) / bs);
  b.row_hi = p.max_budget <= 0 ? -1 : int(p.max_budget / bs);
  b.vs_mode = p.vs_mode;
  long long blo = (p.min_budget + bs - 1) / bs;
  if (blo > nb) blo = nb;
  long long bhi = p.max_budget <= 0 ? nb : p.max_budget / bs;
  if (bhi > nb) bhi = nb;
  b.vsb_lo = int(blo < bhi ? blo : bhi);
  b.vsb_hi = int(bhi);
  return b;
}

fp_status check_ws(void *ws, size_t have, size_t need) {
  if (need == 0) return FP_OK;
  if (!ws) return FP_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return FP_ERR_WORKSPACE;
  if (have < need) return FP_ERR_WORKSPACE;
  return FP_OK;
}

fp_status check_device() {
  static std::atomic<int> cc[64];  // compute capability major, 0 = not yet read
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP_ERR_CUDA;
  int major = cc[dev].load(std::memory_order_relaxed);
  if (major == 0) {
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return FP_ERR_CUDA;
    cc[dev].store(major, std::memory_order_relaxed);
  }
  return major == 10 ? FP_OK : FP_ERR_UNSUPPORTED;
}

fp_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FP_OK : FP_ERR_CUDA; }

// q, k, v, out, qbar and kbar are moved with 16-byte vector accesses and
// tensor-map copies (whose base must be 16-byte aligned); the other arrays
// with accesses of their element size.  A null pointer passes (the null
// checks come first, and optional outputs may be null).
bool al(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool qkvo_aligned(const void *q, const void *k, const void *v, const void *out) {
  return al(q, 16) && al(k, 16) && al(v, 16) && al(out, 16);
}

// One thread waits on an mbarrier that nothing arrives at, with the bounded
// wait of the pipelined kernels, and records FP_ERR_TIMEOUT when it gives up.
__global__ void watchdog_selftest_kernel(int *status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort_flag, limit_ns))
    report(status, FP_ERR_TIMEOUT);
}

// Intermediates of the whole path, carved from a workspace.
struct Prefill {
  float *qbar, *kbar, *kbar_hi, *kbar_lo, *map, *est_last, *true_last, *vert, *slash, *djs;
  int32_t *pattern, *counts, *indices;
  void *stage_ws;
};

constexpr int kHostMidUnits = 3;  // fp_prefill_attn_host: middle units per batch entry

// One unit of fp_prefill_attn_host: consecutive heads of one batch entry.
struct Unit {
  int kv0, nk;  // kv heads [kv0, kv0 + nk)
  int q0, nq;   // their query heads [kv0 g + q0, kv0 g + q0 + nq)
  bool kv_in;   // this unit copies the kv heads' K and V in
};

// The units of one batch entry.  Only the first unit's copy in and the last
// unit's copy out are not hidden, so those two units hold one query head each
// (with the first, its kv head's K and V come in; the second unit then brings
// only the rest of that kv head's Q), the next to them the rest of the first
// and last kv heads' query heads, and the kv heads between go in three middle
// units.
std::vector<Unit> host_plan(const Dims &D) {
  std::vector<Unit> plan;
  auto whole = [&](int kv0, int nk) { plan.push_back({kv0, nk, 0, nk * D.g, true}); };
  auto middle = [&]() {
    const int mid = D.hkv - 2;
    for (int i = 0, kv = 1; i < kHostMidUnits; ++i) {
      const int n = mid / kHostMidUnits + (i < mid % kHostMidUnits ? 1 : 0);
      if (n > 0) whole(kv, n);
      kv += n;
    }
  };
  if (D.hkv >= 4 && D.g >= 2) {
    plan.push_back({0, 1, 0, 1, true});
    plan.push_back({0, 1, 1, D.g - 1, false});
    middle();
    plan.push_back({D.hkv - 1, 1, 0, D.g - 1, true});
    plan.push_back({D.hkv - 1, 1, D.g - 1, 1, false});
  } else if (D.hkv >= 4) {
    whole(0, 1);
    middle();
    whole(D.hkv - 1, 1);
  } else {
    for (int kv = 0; kv < D.hkv; ++kv) whole(kv, 1);
  }
  return plan;
}

// The shape of one unit (batch 1, the unit's heads).
bool unit_dims(const fp_shape &shape, const Unit &un, Dims *Du);

size_t carve_prefill(const Dims &D, void *ws, Prefill *P) {
  Carver c{static_cast<char *>(ws), 0};
  const size_t heads = size_t(D.bt) * D.hq;
  P->qbar = c.take<float>(heads * D.nb * D.d);
  P->kbar = c.take<float>(size_t(D.bt) * D.hkv * D.nb * D.d);
  P->kbar_hi = c.take<float>(size_t(D.bt) * D.hkv * D.nb * D.d);
  P->kbar_lo = c.take<float>(size_t(D.bt) * D.hkv * D.nb * D.d);
  P->map = c.take<float>(heads * D.t_pairs);
  P->est_last = c.take<float>(heads * D.nb);
  P->true_last = c.take<float>(heads * D.nb);
  P->vert = c.take<float>(heads * D.n);
  P->slash = c.take<float>(heads * D.n);
  P->djs = c.take<float>(heads);
  P->pattern = c.take<int32_t>(heads);
  P->counts = c.take<int32_t>(heads * D.nb);
  P->indices = c.take<int32_t>(heads * D.nb * size_t(D.nb));
  const size_t stage = std::max(estimate_ws_bytes(D), std::max(select_ws_bytes(D),
                                                               attn_ws_bytes(D)));
  P->stage_ws = c.take<char>(stage);
  return c.off + 256;
}

bool unit_dims(const fp_shape &shape, const Unit &un, Dims *Du) {
  fp_shape us = shape;
  us.batch = 1;
  us.n_kv_heads = un.nk;
  us.n_q_heads = un.nq;
  return check_shape(&us, Du) == FP_OK;
}

// Workspace of fp_prefill_attn_host: device copies of q, k, v and out, and two
// unit regions (units alternate between two compute streams), each sized for
// the largest unit.
struct HostWs {
  char *q, *k, *v, *out, *unit[2];
  size_t bytes;
};
HostWs carve_host(const fp_shape &shape, const Dims &D, void *ws) {
  const size_t eb = D.dtype == FP_BF16 ? 2 : 4;
  Carver c{static_cast<char *>(ws), 0};
  HostWs h;
  h.q = c.take<char>(size_t(D.bt) * D.hq * D.n * D.d * eb);
  h.k = c.take<char>(size_t(D.bt) * D.hkv * D.n * D.d * eb);
  h.v = c.take<char>(size_t(D.bt) * D.hkv * D.n * D.d * eb);
  h.out = c.take<char>(size_t(D.bt) * D.hq * D.n * D.d * eb);
  size_t unit_bytes = 0;
  for (const Unit &un : host_plan(D)) {
    Dims Du;
    Prefill P;
    if (unit_dims(shape, un, &Du)) unit_bytes = std::max(unit_bytes, carve_prefill(Du, nullptr, &P));
  }
  h.unit[0] = c.take<char>(unit_bytes);
  h.unit[1] = c.take<char>(unit_bytes);
  h.bytes = c.off + 256;
  return h;
}

size_t elem_bytes(const Dims &D) { return D.dtype == FP_BF16 ? 2 : 4; }

fp_status run_attn(const Dims &D, const void *q, const void *k, const void *v,
                   const int32_t *counts, const int32_t *indices, void *out, float *lse,
                   bool dense, void *ws, cudaStream_t st) {
  if (D.dtype == FP_F32)
    return cuda_status(launch_attn_f32(D, static_cast<const float *>(q),
                                       static_cast<const float *>(k),
                                       static_cast<const float *>(v), counts, indices,
                                       static_cast<float *>(out), lse, dense, st));
  return cuda_status(launch_attn_bf16(D, q, k, v, counts, indices, out, lse, dense, ws, st));
}

// The whole path, pattern-aware: the inputs of the pattern test first, for every
// head; then Q pooling and the block map only for the query-aware heads, and
// the vertical / slash line sums only for the vertical-slash heads (each
// head's selection reads one or the other).  Every value a head's selection
// reads is bitwise the one the separate fp_estimate / fp_pattern / fp_select
// calls produce.  `v_ready` (may be null): an event the attention stage waits
// for, the only stage that reads v (the host path's copy of v in lands
// behind it).
fp_status run_prefill(const Dims &D, const fp_params &p, const void *q, const void *k,
                      const void *v, void *out, float *lse, int64_t *stats, const Prefill &P,
                      cudaStream_t st, cudaEvent_t v_ready = nullptr) {
  cudaError_t e = launch_estimate_decision(D, q, k, P.qbar, P.kbar, P.kbar_hi, P.kbar_lo, P.map,
                                           P.est_last, P.true_last, P.stage_ws, st);
  if (e != cudaSuccess) return FP_ERR_CUDA;
  e = launch_pattern(D, p.tau, P.est_last, P.true_last, P.djs, P.pattern, st);
  if (e != cudaSuccess) return FP_ERR_CUDA;
  e = launch_estimate_map_qa(D, q, P.qbar, P.kbar_hi, P.kbar_lo, P.map, P.est_last, P.pattern,
                             st);
  if (e != cudaSuccess) return FP_ERR_CUDA;
  e = launch_estimate_lines_vs(D, q, k, P.vert, P.slash, P.pattern, P.stage_ws, st);
  if (e != cudaSuccess) return FP_ERR_CUDA;
  e = launch_select(D, p.gamma, budgets(D, p), P.pattern, P.map, P.vert, P.slash, P.counts,
                    P.indices, P.stage_ws, st);
  if (e != cudaSuccess) return FP_ERR_CUDA;
  if (stats && launch_stats(D, P.counts, P.pattern, stats, st) != cudaSuccess)
    return FP_ERR_CUDA;
  if (v_ready && cudaStreamWaitEvent(st, v_ready, 0) != cudaSuccess) return FP_ERR_CUDA;
  return run_attn(D, q, k, v, P.counts, P.indices, out, lse, false, P.stage_ws, st);
}

}  // namespace
}  // namespace fpi

using namespace fpi;

FP_API size_t fp_workspace_size(const fp_shape *shape, int which_call) {
  Dims D;
  if (check_shape(shape, &D) != FP_OK) return 0;
  switch (which_call) {
    case FP_CALL_ESTIMATE:
      return estimate_ws_bytes(D);
    case FP_CALL_SELECT:
      return select_ws_bytes(D);
    case FP_CALL_SPARSE_ATTN:
      return attn_ws_bytes(D);
    case FP_CALL_PREFILL: {
      Prefill P;
      return carve_prefill(D, nullptr, &P);
    }
    case FP_CALL_PREFILL_HOST:
      return carve_host(*shape, D, nullptr).bytes;
    default:
      return 0;
  }
}

FP_API fp_status fp_estimate(const fp_shape *shape, const void *q, const void *k, float *qbar,
                             float *kbar, float *map, float *est_last, float *true_last,
                             float *vert, float *slash, void *ws, size_t ws_bytes,
                             fp_stream_t stream) {
  Dims D;
  fp_status s = check_shape(shape, &D);
  if (s != FP_OK) return s;
  if (!q || !k || !qbar || !kbar || !map || !est_last || !true_last || !vert || !slash)
    return FP_ERR_NULL;
  if (!al(q, 16) || !al(k, 16) || !al(qbar, 16) || !al(kbar, 16) || !al(map, 4) ||
      !al(est_last, 4) || !al(true_last, 4) || !al(vert, 4) || !al(slash, 4))
    return FP_ERR_ALIGN;
  if ((s = check_ws(ws, ws_bytes, estimate_ws_bytes(D))) != FP_OK) return s;
  if ((s = check_device()) != FP_OK) return s;
  return cuda_status(launch_estimate(D, q, k, qbar, kbar, map, est_last, true_last, vert, slash,
                                     ws, reinterpret_cast<cudaStream_t>(stream)));
}

FP_API fp_status fp_pattern(const fp_shape *shape, const fp_params *params,
                            const float *est_last, const float *true_last, float *djs,
                            int32_t *pattern, fp_stream_t stream) {
  Dims D;
  fp_status s = check_shape(shape, &D);
  if (s != FP_OK) return s;
  if ((s = check_params(params)) != FP_OK) return s;
  if (!est_last || !true_last || !djs || !pattern) return FP_ERR_NULL;
  if (!al(est_last, 4) || !al(true_last, 4) || !al(djs, 4) || !al(pattern, 4))
    return FP_ERR_ALIGN;
  if ((s = check_device()) != FP_OK) return s;
  return cuda_status(launch_pattern(D, params->tau, est_last, true_last, djs, pattern,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

FP_API fp_status fp_select(const fp_shape *shape, const fp_params *params,
                           const int32_t *pattern, const float *map, const float *vert,
                           const float *slash, int32_t *counts, int32_t *indices, void *ws,
                           size_t ws_bytes, fp_stream_t stream) {
  Dims D;
  fp_status s = check_shape(shape, &D);
  if (s != FP_OK) return s;
  if ((s = check_params(params)) != FP_OK) return s;
  if (!pattern || !map || !vert || !slash || !counts || !indices) return FP_ERR_NULL;
  if (!al(pattern, 4) || !al(map, 4) || !al(vert, 4) || !al(slash, 4) || !al(counts, 4) ||
      !al(indices, 4))
    return FP_ERR_ALIGN;
  if ((s = check_ws(ws, ws_bytes, select_ws_bytes(D))) != FP_OK) return s;
  if ((s = check_device()) != FP_OK) return s;
  return cuda_status(launch_select(D, params->gamma, budgets(D, *params), pattern, map, vert,
                                   slash, counts, indices, ws,
                                   reinterpret_cast<cudaStream_t>(stream)));
}

FP_API fp_status fp_select_noalloc(const fp_shape *shape, const fp_params *params,
                                   const int32_t *pattern, const float *map, const float *vert,
                                   const float *slash, int32_t *counts, int32_t *indices,
                                   fp_stream_t stream) {
  Dims D;
  fp_status s = check_shape(shape, &D);
  if (s != FP_OK) return s;
  if ((s = check_params(params)) != FP_OK) return s;
  if (!pattern || !map || !vert || !slash || !counts || !indices) return FP_ERR_NULL;
  if (!al(pattern, 4) || !al(map, 4) || !al(vert, 4) || !al(slash, 4) || !al(counts, 4) ||
      !al(indices, 4))
    return FP_ERR_ALIGN;
  if (select_ws_bytes(D) > FP_SELECT_NOALLOC_SCRATCH_BYTES) return FP_ERR_WORKSPACE;
  if ((s = check_device()) != FP_OK) return s;
  return cuda_status(launch_select_noalloc(D, params->gamma, budgets(D, *params), pattern, map,
                                           vert, slash, counts, indices,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

FP_API fp_status fp_sparse_attn(const fp_shape *shape, const void *q, const void *k,
                                const void *v, const int32_t *counts, const int32_t *indices,
                                void *out, float *lse, void *ws, size_t ws_bytes,
                                fp_stream_t stream) {
  Dims D;
  fp_status s = check_shape(shape, &D);
  if (s != FP_OK) return s;
  if ((s = check_attn_shape(D)) != FP_OK) return s;
  if (!q || !k || !v || !counts || !indices || !out) return FP_ERR_NULL;
  if (!qkvo_aligned(q, k, v, out) || !al(counts, 4) || !al(indices, 4) || !al(lse, 4))
    return FP_ERR_ALIGN;
  if ((s = check_ws(ws, ws_bytes, attn_ws_bytes(D))) != FP_OK) return s;
  if ((s = check_device()) != FP_OK) return s;
  return run_attn(D, q, k, v, counts, indices, out, lse, false, ws,
                  reinterpret_cast<cudaStream_t>(stream));
}

FP_API fp_status fp_dense_attn(const fp_shape *shape, const void *q, const void *k,
                               const void *v, void *out, float *lse, fp_stream_t stream) {
  Dims D;
  fp_status s = check_shape(shape, &D);
  if (s != FP_OK) return s;
  if ((s = check_attn_shape(D)) != FP_OK) return s;
  if (!q || !k || !v || !out) return FP_ERR_NULL;
  if (!qkvo_aligned(q, k, v, out) || !al(lse, 4)) return FP_ERR_ALIGN;
  if ((s = check_device()) != FP_OK) return s;
  // dense lists are implicit: counts / indices are never read
  static const int32_t dummy = 0;
  return run_attn(D, q, k, v, &dummy, &dummy, out, lse, true, nullptr,
                  reinterpret_cast<cudaStream_t>(stream));
}

FP_API fp_status fp_prefill_attn(const fp_shape *shape, const fp_params *params, const void *q,
                                 const void *k, const void *v, void *out, float *lse,
                                 int64_t *stats, void *ws, size_t ws_bytes,
                                 fp_stream_t stream) {
  Dims D;
  fp_status s = check_shape(shape, &D);
  if (s != FP_OK) return s;
  if ((s = check_attn_shape(D)) != FP_OK) return s;
  if ((s = check_params(params)) != FP_OK) return s;
  if (!q || !k || !v || !out) return FP_ERR_NULL;
  if (!qkvo_aligned(q, k, v, out) || !al(lse, 4) || !al(stats, 8)) return FP_ERR_ALIGN;
  Prefill P;
  if ((s = check_ws(ws, ws_bytes, carve_prefill(D, nullptr, &P))) != FP_OK) return s;
  if ((s = check_device()) != FP_OK) return s;
  carve_prefill(D, ws, &P);
  return run_prefill(D, *params, q, k, v, out, lse, stats, P,
                     reinterpret_cast<cudaStream_t>(stream));
}

FP_API fp_status fp_prefill_attn_varlen(const fp_shape *shape, const fp_params *params,
                                        int n_seqs, const int32_t *seq_lens, const void *q,
                                        const void *k, const void *v, void *out, float *lse,
                                        int64_t *stats, void *ws, size_t ws_bytes,
                                        fp_stream_t stream) {
  Dims D;
  fp_status s = check_shape(shape, &D);
  if (s != FP_OK) return s;
  if (D.bt != 1) return FP_ERR_SHAPE;
  if ((s = check_attn_shape(D)) != FP_OK) return s;
  if ((s = check_params(params)) != FP_OK) return s;
  if (!q || !k || !v || !out || !seq_lens) return FP_ERR_NULL;
  // a sequence starts at a multiple of Hq d (or Hkv d) elements: aligned with the base
  if (!qkvo_aligned(q, k, v, out) || !al(lse, 4) || !al(stats, 8)) return FP_ERR_ALIGN;
  if (n_seqs < 1) return FP_ERR_SHAPE;
  for (int i = 0; i < n_seqs; ++i)
    if (seq_lens[i] <= 0 || seq_lens[i] > D.n) return FP_ERR_SHAPE;
  Prefill Pmax;
  if ((s = check_ws(ws, ws_bytes, carve_prefill(D, nullptr, &Pmax))) != FP_OK) return s;
  if ((s = check_device()) != FP_OK) return s;
  const size_t eb = elem_bytes(D);
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  size_t tok = 0;  // tokens of the sequences before this one
  for (int i = 0; i < n_seqs; ++i) {
    fp_shape one = *shape;
    one.seq_len = seq_lens[i];
    Dims Ds;
    if ((s = check_shape(&one, &Ds)) != FP_OK) return s;
    Prefill P;
    carve_prefill(Ds, ws, &P);  // fits: a shorter sequence needs less than N_max
    const size_t qo = tok * D.hq * D.d * eb, kvo = tok * D.hkv * D.d * eb;
    s = run_prefill(Ds, *params, static_cast<const char *>(q) + qo,
                    static_cast<const char *>(k) + kvo, static_cast<const char *>(v) + kvo,
                    static_cast<char *>(out) + qo, lse ? lse + tok * D.hq : nullptr,
                    stats ? stats + 2 * i : nullptr, P, st);
    if (s != FP_OK) return s;
    tok += size_t(seq_lens[i]);
  }
  return FP_OK;
}

FP_API fp_status fp_prefill_attn_host(const fp_shape *shape, const fp_params *params,
                                      const void *q_host, const void *k_host,
                                      const void *v_host, void *out_host, void *ws,
                                      size_t ws_bytes, fp_stream_t stream) {
  Dims D;
  fp_status s = check_shape(shape, &D);
  if (s != FP_OK) return s;
  if ((s = check_attn_shape(D)) != FP_OK) return s;
  if ((s = check_params(params)) != FP_OK) return s;
  if (!q_host || !k_host || !v_host || !out_host) return FP_ERR_NULL;
  if ((s = check_ws(ws, ws_bytes, fp_workspace_size(shape, FP_CALL_PREFILL_HOST))) != FP_OK)
    return s;
  if ((s = check_device()) != FP_OK) return s;
  const size_t eb = elem_bytes(D);
  const HostWs hw = carve_host(*shape, D, ws);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream), sin = nullptr, sout = nullptr,
               scomp = nullptr;
  if (!host_streams(&sin, &sout, &scomp)) return FP_ERR_CUDA;
  // Every stage is independent per query head (a query head reads only its
  // kv head's K and V), so the call runs as units of consecutive heads
  // (host_plan): the inputs of unit u+1 are copied in while unit u computes,
  // and each unit's output is copied out while the next one computes.  Units
  // alternate between `stream` and a second compute stream, each with its own
  // workspace region, so that one unit's latency-bound estimate and selection
  // overlap the other's attention.  `stream` forks to the library's streams
  // and joins them at the end through events, so it still orders the whole
  // call.
  const std::vector<Unit> plan = host_plan(D);
  const int units_per_batch = int(plan.size());
  const int nunits = D.bt * units_per_batch;
  std::vector<cudaEvent_t> ev;
  auto event = [&](cudaEvent_t *e) {
    if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return false;
    ev.push_back(*e);
    return true;
  };
  auto finish = [&](fp_status r) {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);  // released once they complete
    return r;
  };
  cudaEvent_t e_start, e_end;
  if (!event(&e_start) || cudaEventRecord(e_start, st) != cudaSuccess ||
      cudaStreamWaitEvent(sin, e_start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(sout, e_start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(scomp, e_start, 0) != cudaSuccess)
    return finish(FP_ERR_CUDA);
  const cudaStream_t comp[2] = {st, scomp};
  const size_t head_bytes = size_t(D.n) * D.d * eb;
  const char *qh = static_cast<const char *>(q_host);
  const char *kh = static_cast<const char *>(k_host);
  const char *vh = static_cast<const char *>(v_host);
  char *oh = static_cast<char *>(out_host);
  cudaEvent_t e_v = nullptr;  // the current kv head's V is in
  for (int u = 0; u < nunits; ++u) {
    const int b = u / units_per_batch;
    const Unit &un = plan[u % units_per_batch];
    Dims Du;
    if (!unit_dims(*shape, un, &Du)) return finish(FP_ERR_SHAPE);
    const cudaStream_t cs = comp[u % 2];
    const size_t qoff = (size_t(b) * D.hq + size_t(un.kv0) * D.g + un.q0) * head_bytes;
    const size_t kvoff = (size_t(b) * D.hkv + un.kv0) * head_bytes;
    const size_t qlen = size_t(un.nq) * head_bytes, kvlen = size_t(un.nk) * head_bytes;
    // Q and K first: the unit's estimate can start on them, while V (read only
    // by the attention stage) is still coming in behind its own event, which
    // the kv heads' later units wait for too
    cudaEvent_t e_in, e_comp;
    if (!event(&e_in) || !event(&e_comp) ||
        cudaMemcpyAsync(hw.q + qoff, qh + qoff, qlen, cudaMemcpyHostToDevice, sin) != cudaSuccess)
      return finish(FP_ERR_CUDA);
    if (un.kv_in &&
        cudaMemcpyAsync(hw.k + kvoff, kh + kvoff, kvlen, cudaMemcpyHostToDevice, sin) !=
            cudaSuccess)
      return finish(FP_ERR_CUDA);
    if (cudaEventRecord(e_in, sin) != cudaSuccess || cudaStreamWaitEvent(cs, e_in, 0) != cudaSuccess)
      return finish(FP_ERR_CUDA);
    if (un.kv_in &&
        (!event(&e_v) ||
         cudaMemcpyAsync(hw.v + kvoff, vh + kvoff, kvlen, cudaMemcpyHostToDevice, sin) !=
             cudaSuccess ||
         cudaEventRecord(e_v, sin) != cudaSuccess))
      return finish(FP_ERR_CUDA);
    Prefill Pu;
    carve_prefill(Du, hw.unit[u % 2], &Pu);  // a region's units run in order on one stream
    const fp_status r = run_prefill(Du, *params, hw.q + qoff, hw.k + kvoff, hw.v + kvoff,
                                    hw.out + qoff, nullptr, nullptr, Pu, cs, e_v);
    if (r != FP_OK) return finish(r);
    if (cudaEventRecord(e_comp, cs) != cudaSuccess ||
        cudaStreamWaitEvent(sout, e_comp, 0) != cudaSuccess ||
        cudaMemcpyAsync(oh + qoff, hw.out + qoff, qlen, cudaMemcpyDeviceToHost, sout) !=
            cudaSuccess)
      return finish(FP_ERR_CUDA);
  }
  // every unit's copy out follows its compute on the copy-out stream, so its
  // last event covers both compute streams
  if (!event(&e_end) || cudaEventRecord(e_end, sout) != cudaSuccess ||
      cudaStreamWaitEvent(st, e_end, 0) != cudaSuccess)
    return finish(FP_ERR_CUDA);
  return finish(FP_OK);
}

FP_API fp_status fp_last_device_status(fp_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FP_ERR_CUDA;
  int *p = device_status_ptr();
  if (!p) return FP_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FP_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return FP_ERR_CUDA;
  return static_cast<fp_status>(v);
}

FP_API fp_status fp_selftest_watchdog(unsigned int limit_us, fp_stream_t stream) {
  if (limit_us == 0 || limit_us > 1000000u) return FP_ERR_PARAM;
  fp_status s = check_device();
  if (s != FP_OK) return s;
  watchdog_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      device_status_ptr(), 1000ull * limit_us);
  return cuda_status(cudaGetLastError());
}

FP_API const char *fp_status_string(fp_status status) {
  switch (status) {
    case FP_OK: return "FP_OK";
    case FP_ERR_NULL: return "FP_ERR_NULL: a required pointer is NULL";
    case FP_ERR_SHAPE: return "FP_ERR_SHAPE: unsupported or inconsistent shape";
    case FP_ERR_DTYPE: return "FP_ERR_DTYPE: unsupported dtype";
    case FP_ERR_PARAM: return "FP_ERR_PARAM: gamma, tau or budget out of range";
    case FP_ERR_WORKSPACE: return "FP_ERR_WORKSPACE: workspace NULL, misaligned or too small";
    case FP_ERR_CUDA: return "FP_ERR_CUDA: a CUDA call or launch failed";
    case FP_ERR_TIMEOUT: return "FP_ERR_TIMEOUT: a device pipeline wait ran out of time";
    case FP_ERR_DEVICE_CHECK: return "FP_ERR_DEVICE_CHECK: an argument failed a device check";
    case FP_ERR_UNSUPPORTED: return "FP_ERR_UNSUPPORTED: the device is not sm_100";
    case FP_ERR_ALIGN: return "FP_ERR_ALIGN: a data pointer is not aligned as required";
  }
  return "unknown fp_status";
}
