// attn_f32.cu -- fp32 block-sparse causal attention on CUDA cores (the debug
// path of fp_sparse_attn / fp_dense_attn for fp32 inputs).
//
// FlexPrefill (atlas.scime.ai summary, "Approach" and "Experimental setup"):
// causal attention over the selected query-key blocks, built on
// FlashAttention's online softmax.  Every product and sum is fp32, so the
// result tracks an fp64 reference to ~1e-6.
//
// One CTA per (query block, head, batch); 4 threads per query row, each
// owning every 4th feature of the row's q and output accumulator
// (interleaved, so the 4 threads hit distinct shared-memory banks).
#include <math.h>

#include "fp_internal.cuh"

namespace fpi {
namespace {

template <int BS, int D>
struct F32Smem {
  float K[BS][D];
  float V[BS][D];
  float S[BS][BS + 1];
};

template <int BS, int D>
__global__ void __launch_bounds__(BS * 4) attn_f32_kernel(
    const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
    const int32_t *__restrict__ counts, const int32_t *__restrict__ indices,
    float *__restrict__ out, float *__restrict__ lse, int hq, int g, int n, bool dense,
    int *status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  auto &sm = *reinterpret_cast<F32Smem<BS, D> *>(smem_raw);
  constexpr int DP = D / 4;
  const int nb = gridDim.x;
  const int qi = nb - 1 - blockIdx.x;  // longest rows first
  const int h = blockIdx.y, b = blockIdx.z, kv = h / g, hkv = hq / g;
  const size_t bh = size_t(b) * hq + h;
  const int r = threadIdx.x / 4, part = threadIdx.x % 4;
  const float scale = 1.f / sqrtf(float(D));
  // a partial last block (N not a multiple of BS): rows and keys at or past
  // N are not read or written (their keys come in as zeros, which the causal
  // mask hides from every real row)
  const bool row_ok = size_t(qi) * BS + r < size_t(n);
  const float *qrow = q + (bh * n + size_t(qi) * BS + r) * D;
  float qv[DP], acc[DP];
#pragma unroll
  for (int i = 0; i < DP; ++i) {
    qv[i] = row_ok ? qrow[part + 4 * i] : 0.f;
    acc[i] = 0.f;
  }
  const float *kbase = k + (size_t(b) * hkv + kv) * n * D;
  const float *vbase = v + (size_t(b) * hkv + kv) * n * D;
  const int cnt = dense ? qi + 1 : counts[bh * nb + qi];
  const int32_t *list = indices + (bh * nb + qi) * size_t(nb);
  float m = -INFINITY, l = 0.f;
  for (int t = 0; t < cnt; ++t) {
    int j = dense ? t : list[t];
    const bool valid = j >= 0 && j <= qi;
    if (!valid) {
      if (threadIdx.x == 0) report(status, FP_ERR_DEVICE_CHECK);
      continue;
    }
    __syncthreads();
    const float4 *ks = reinterpret_cast<const float4 *>(kbase + size_t(j) * BS * D);
    const float4 *vs = reinterpret_cast<const float4 *>(vbase + size_t(j) * BS * D);
    float4 *kd = reinterpret_cast<float4 *>(&sm.K[0][0]);
    float4 *vd = reinterpret_cast<float4 *>(&sm.V[0][0]);
    const int keys = min(BS, n - j * BS);  // real keys of block j
    for (int e = threadIdx.x; e < BS * D / 4; e += BS * 4) {
      const bool in = e / (D / 4) < keys;
      kd[e] = in ? ks[e] : make_float4(0.f, 0.f, 0.f, 0.f);
      vd[e] = in ? vs[e] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    const bool diag = j == qi;
    for (int c = 0; c < BS; ++c) {
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < DP; ++i) s = fmaf(qv[i], sm.K[c][part + 4 * i], s);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (part == 0) sm.S[r][c] = (diag && c > r) ? -INFINITY : s * scale;
    }
    __syncwarp();
    float tmax = -INFINITY;
    for (int c = part; c < BS; c += 4) tmax = fmaxf(tmax, sm.S[r][c]);
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    const float mnew = fmaxf(m, tmax);
    const float alpha = expf(m - mnew);  // 0 on the first tile
    float ps = 0.f;
    __syncwarp();
    for (int c = part; c < BS; c += 4) {
      const float p = expf(sm.S[r][c] - mnew);
      sm.S[r][c] = p;
      ps += p;
    }
    ps += __shfl_xor_sync(0xffffffffu, ps, 1);
    ps += __shfl_xor_sync(0xffffffffu, ps, 2);
    __syncwarp();
    l = l * alpha + ps;
#pragma unroll
    for (int i = 0; i < DP; ++i) acc[i] *= alpha;
    for (int c = 0; c < BS; ++c) {
      const float p = sm.S[r][c];
#pragma unroll
      for (int i = 0; i < DP; ++i) acc[i] = fmaf(p, sm.V[c][part + 4 * i], acc[i]);
    }
    m = mnew;
  }
  if (!row_ok) return;
  float *orow = out + (bh * n + size_t(qi) * BS + r) * D;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int i = 0; i < DP; ++i) orow[part + 4 * i] = acc[i] * inv;
  if (lse && part == 0) lse[bh * n + size_t(qi) * BS + r] = l > 0.f ? m + logf(l) : -INFINITY;
}

template <int BS, int D>
cudaError_t run(const Dims &Dm, const float *q, const float *k, const float *v,
                const int32_t *counts, const int32_t *indices, float *out, float *lse,
                bool dense, cudaStream_t st) {
  const size_t smem = sizeof(F32Smem<BS, D>);
  cudaFuncSetAttribute(attn_f32_kernel<BS, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       int(smem));
  attn_f32_kernel<BS, D><<<dim3(Dm.nb, Dm.hq, Dm.bt), BS * 4, smem, st>>>(
      q, k, v, counts, indices, out, lse, Dm.hq, Dm.g, Dm.n, dense, device_status_ptr());
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_f32(const Dims &D, const float *q, const float *k, const float *v,
                            const int32_t *counts, const int32_t *indices, float *out,
                            float *lse, bool dense, cudaStream_t st) {
  if (D.bs == 64 && D.d == 64) return run<64, 64>(D, q, k, v, counts, indices, out, lse, dense, st);
  if (D.bs == 64 && D.d == 128)
    return run<64, 128>(D, q, k, v, counts, indices, out, lse, dense, st);
  if (D.bs == 128 && D.d == 64)
    return run<128, 64>(D, q, k, v, counts, indices, out, lse, dense, st);
  return run<128, 128>(D, q, k, v, counts, indices, out, lse, dense, st);
}

}  // namespace fpi
