// fp_internal.cuh -- shared declarations of the CUDA implementation of fp.h.
//
// Device status word: every kernel gets a pointer to one int per device.  A
// kernel that detects a problem (an index outside the causal range, a wait
// that ran out of time) stores the first error code there with atomicCAS and
// carries on or returns; no kernel traps or asserts.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "../../include/fp.h"

namespace fpi {

// ----------------------------------------------------------------- host API --

struct Dims {
  int bt, hq, hkv, n, d, bs, nb, g;
  long long t_pairs;  // nb (nb + 1) / 2
  fp_dtype dtype;
};

// Workspace carving: each region 256-byte aligned.
struct Carver {
  char *base;
  size_t off;
  template <class T>
  T *take(size_t count) {
    off = (off + 255) & ~size_t(255);
    T *p = reinterpret_cast<T *>(base ? base + off : nullptr);
    off += count * sizeof(T);
    return p;
  }
};

int *device_status_ptr();  // per-device status word (fp_api.cu)
// The driver's cuTensorMapEncodeTiled (looked up once, thread-safe), or null.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Stage launchers (each returns cudaGetLastError() of its launches).
size_t estimate_ws_bytes(const Dims &D);
cudaError_t launch_estimate(const Dims &D, const void *q, const void *k, float *qbar,
                            float *kbar, float *map, float *est_last, float *true_last,
                            float *vert, float *slash, void *ws, cudaStream_t st);
// Pattern-aware parts of launch_estimate (fp_prefill_attn): everything the
// pattern test reads, for every head (K pooled, with its tf32 halves in
// kbar_hi / kbar_lo, map_split_bytes() / 2 each; Q pooled over the last block;
// the map's last row; true_last) ...
cudaError_t launch_estimate_decision(const Dims &D, const void *q, const void *k, float *qbar,
                                     float *kbar, float *kbar_hi, float *kbar_lo, float *map,
                                     float *est_last, float *true_last, void *ws,
                                     cudaStream_t st);
// ... then Q pooling and the map for the query-aware heads of `pattern` ...
cudaError_t launch_estimate_map_qa(const Dims &D, const void *q, float *qbar,
                                   const float *kbar_hi, const float *kbar_lo, float *map,
                                   float *est_last, const int32_t *pattern, cudaStream_t st);

// The map's logits on the tensor cores (map_tc.cu), 3xTF32 products of the
// pooled vectors: for every causal block pair (or, with `last_only`, the last
// row only) of every head (or the query-aware heads of `qa_only`).
// kbar_hi / kbar_lo: the pooled keys split as tf32_hi(x) and x - tf32_hi(x).
size_t map_split_bytes(const Dims &D);  // both halves, with carving slack
cudaError_t launch_map_logits_tc(const Dims &D, const float *qbar, const float *kbar_hi,
                                 const float *kbar_lo, float *map, const int32_t *qa_only,
                                 bool last_only, cudaStream_t st);
// ... and vert and slash for its vertical-slash heads (on the workspace the
// decision part left).
cudaError_t launch_estimate_lines_vs(const Dims &D, const void *q, const void *k, float *vert,
                                     float *slash, const int32_t *pattern, void *ws,
                                     cudaStream_t st);

// Tensor-core passes over the last query block (estimate_tc.cu): bf16,
// block 128, head dim 128.
bool last_block_tc_supported(const Dims &D);
int last_block_tc_tiles(const Dims &D);
size_t last_block_tc_ws_bytes(const Dims &D);
// (with kbar non-null, pass 1 also writes the block means of K with their
// tf32 halves, in place of a separate pooling of K)
cudaError_t launch_last_block_rows_tc(const Dims &D, const void *q, const void *k,
                                      float *true_last, float *kbar, float *kbar_hi,
                                      float *kbar_lo, void *ws, cudaStream_t st);
cudaError_t launch_last_block_lines_tc(const Dims &D, const void *q, const void *k, float *vert,
                                       const int32_t *vs_only, float **sp_out, void *ws,
                                       cudaStream_t st);

cudaError_t launch_pattern(const Dims &D, float tau, const float *est_last,
                           const float *true_last, float *djs, int32_t *pattern,
                           cudaStream_t st);

struct SelectBudgets {
  long long qa_lo, qa_hi;  // in block pairs (flattened rule)
  int vs_lo, vs_hi;        // in lines
  int qa_mode;             // FP_QA_FLATTENED or FP_QA_QUERYWISE
  int row_lo, row_hi;      // query-wise rule: blocks per row before the row-length
                           // cap; row_hi < 0 means uncapped
  int vs_mode;             // FP_VS_TOKENS or FP_VS_BLOCKS
  int vsb_lo, vsb_hi;      // block-pooled lines: budgets in blocks
};
size_t select_ws_bytes(const Dims &D);
cudaError_t launch_select(const Dims &D, float gamma, const SelectBudgets &bud,
                          const int32_t *pattern, const float *map, const float *vert,
                          const float *slash, int32_t *counts, int32_t *indices, void *ws,
                          cudaStream_t st);
cudaError_t launch_select_noalloc(const Dims &D, float gamma, const SelectBudgets &bud,
                                  const int32_t *pattern, const float *map, const float *vert,
                                  const float *slash, int32_t *counts, int32_t *indices,
                                  cudaStream_t st);
cudaError_t launch_stats(const Dims &D, const int32_t *counts, const int32_t *pattern,
                         int64_t *stats, cudaStream_t st);

size_t attn_ws_bytes(const Dims &D);
cudaError_t launch_attn_f32(const Dims &D, const float *q, const float *k, const float *v,
                            const int32_t *counts, const int32_t *indices, float *out,
                            float *lse, bool dense, cudaStream_t st);
cudaError_t launch_attn_bf16(const Dims &D, const void *q, const void *k, const void *v,
                             const int32_t *counts, const int32_t *indices, void *out,
                             float *lse, bool dense, void *ws, cudaStream_t st);

// --------------------------------------------------------------- device API --

__device__ __forceinline__ void report(int *status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// x with its low 13 mantissa bits cleared: exact in tf32, the high half of a
// 3xTF32 split (x - tf32_hi(x) is exact in fp32).
__device__ __forceinline__ float tf32_hi(float x) {
  return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
}

// Two-lane fp32 arithmetic (one f32x2 instruction for both lanes).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// bar.sync on a named barrier (ids 1-15; 0 is __syncthreads) for `count`
// threads, a multiple of 32.
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// mbarrier ------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: true when the phase with `parity` completed; false when the
// CTA-wide abort flag is raised or `limit_ns` of wall time passed (the caller
// then records FP_ERR_TIMEOUT and unwinds).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          volatile int *abort_flag,
                                          uint64_t limit_ns = 2000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > limit_ns) return false;
    }
  }
}

// TMA -------------------------------------------------------------------------

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// tcgen05 ---------------------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void tc_mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem], kind::f16.  A is M lanes (one row each)
// by K elements, two 16-bit elements per 32-bit column, the lower index in the
// low half; one K = 16 step spans 8 columns.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp gets lane
// (warp%4)*32 + t, columns col .. col+31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32"
      " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32"
      " [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// UMMA shared-memory descriptor, SWIZZLE_128B, sm100 version bits.
//   K-major operand: rows of 128 B (64 bf16 of K), 8-row atoms 1024 B apart
//     (SBO = 1024 B); LBO unused.
//   MN-major operand: 64 MN-elements per 128-B row, rows along K, 8-row atoms
//     SBO apart, 64-element MN chunks LBO apart.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFF);
  d |= uint64_t((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= uint64_t((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= uint64_t(1) << 46;  // descriptor version (sm100)
  d |= uint64_t(2) << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: bf16 A/B, fp32 D, M x N, K-major A,
// B K-major (b_mn_major = 0) or MN-major (1).
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int m, int n, int b_mn_major) {
  return (1u << 4)                    // D fp32
         | (1u << 7)                  // A bf16
         | (1u << 10)                 // B bf16
         | (uint32_t(b_mn_major) << 16)
         | (uint32_t(n >> 3) << 17)
         | (uint32_t(m >> 4) << 24);
}

}  // namespace fpi
