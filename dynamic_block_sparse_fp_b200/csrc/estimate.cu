// estimate.cu -- fp_estimate: block pooling, the estimated block map, and the
// true attention of the last query block with its vertical / slash sums.
//
// FlexPrefill (atlas.scime.ai summary, "Approach"): per head, a block-pooled
// attention estimate from the last query block is compared with the true
// distribution; the vertical-slash fallback is driven by column and diagonal
// attention sums of the same last block.
//
// Kernels (all reductions in a fixed order, so results are reproducible):
//   pool_kernel          mean of each B-token block of q and k (HBM stream);
//                        for k also its tf32 halves
//   (map_tc.cu)          scaled qbar.kbar^T for the causal block pairs, on the
//                        tensor cores
//   map_softmax_kernel   in-place row softmax of the packed map, + est_last
//   map_last_softmax_kernel  the same for the last row alone
//   last_pass1_kernel    per (head, key block): row max / sum of exp of the
//                        last query block's logits (online-softmax partials)
//   last_lse_kernel      combine partials -> log-sum-exp of each last-block row
//   block_mass_kernel    the partials scaled by exp(max - lse), summed over the
//                        rows: the pooled true distribution (true_last)
//   last_pass2_kernel    per (head, key block): P = exp(logit - lse); column
//                        sums (vert) and diagonal partials
//   slash_combine_kernel diagonal partials of neighbouring key blocks -> slash
// The line sums (pass 2 and the slash combine) are read only by the
// selection of vertical-slash heads, so the whole-path call runs them after
// the pattern test, for those heads alone.
#include <math.h>

#include <algorithm>

#include "fp_internal.cuh"

namespace fpi {
namespace {

template <class T>
__device__ __forceinline__ float ld_f(const T *p);
template <>
__device__ __forceinline__ float ld_f<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat162float(*p);
}

// 8 consecutive elements as fp32 (16 B for bf16, 32 B for fp32).
__device__ __forceinline__ void ld8(const float *p, float (&x)[8]) {
  float4 a = *reinterpret_cast<const float4 *>(p);
  float4 b = *reinterpret_cast<const float4 *>(p + 4);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void ld8(const __nv_bfloat16 *p, float (&x)[8]) {
  uint4 u = *reinterpret_cast<const uint4 *>(p);
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

// ------------------------------------------------------------------ pooling --
// grid (blocks, heads, Bt), 256 threads.  x [Bt, heads, N, d] -> out [Bt, heads,
// nb, d], blocks blk0 .. blk0 + gridDim.x - 1; a partial last block is the
// mean of its real tokens.  With `qa_only` (a pattern array, or null), heads
// whose pattern is not query-aware are skipped.  With `hi_out` / `lo_out`
// (both or neither), each mean is also written split into its tf32 high half
// and the fp32 rest (the operands of the tensor-core map).
template <class T>
__global__ void __launch_bounds__(256) pool_kernel(const T *__restrict__ x, float *__restrict__ out,
                                                   int n, int d, int bs, int nb, int blk0,
                                                   const int32_t *__restrict__ qa_only,
                                                   float *__restrict__ hi_out = nullptr,
                                                   float *__restrict__ lo_out = nullptr) {
  __shared__ float part[32][128];
  const int blk = blk0 + int(blockIdx.x), head = blockIdx.y, b = blockIdx.z;
  const int heads = gridDim.y;
  if (qa_only && qa_only[size_t(b) * heads + head] != FP_PATTERN_QA) return;
  const int vec_per_row = d / 8;
  const int rows_per_it = 256 / vec_per_row;
  const int tv = threadIdx.x % vec_per_row, tr = threadIdx.x / vec_per_row;
  const T *base = x + ((size_t(b) * heads + head) * n + size_t(blk) * bs) * d;
  const int rows = min(bs, n - blk * bs);  // a partial last block: its real tokens
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int r = tr; r < rows; r += rows_per_it) {
    float v[8];
    ld8(base + size_t(r) * d + tv * 8, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += v[i];
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[tr][tv * 8 + i] = acc[i];
  __syncthreads();
  if (threadIdx.x < d) {
    float s = 0.f;
    for (int r = 0; r < rows_per_it; ++r) s += part[r][threadIdx.x];
    const size_t o = ((size_t(b) * heads + head) * nb + blk) * d + threadIdx.x;
    const float mean = s / float(rows);
    out[o] = mean;
    if (hi_out) {
      const float hi = tf32_hi(mean);
      hi_out[o] = hi;
      lo_out[o] = mean - hi;
    }
  }
}

// ------------------------------------------------------------ block map --
// Softmax of one map row in place (one warp; the same steps for every row,
// whichever kernel runs them); the last row also goes to est_last.
__device__ __forceinline__ void map_row_softmax(float *r, int len, float *est_last_row,
                                                int lane) {
  float mx = -INFINITY;
  for (int j = lane; j < len; j += 32) mx = fmaxf(mx, r[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float s = 0.f;
  for (int j = lane; j < len; j += 32) s += expf(r[j] - mx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float inv = 1.f / s;
  for (int j = lane; j < len; j += 32) {
    float p = expf(r[j] - mx) * inv;
    r[j] = p;
    if (est_last_row) est_last_row[j] = p;
  }
}

// One warp per map row; 8 rows per CTA, every head's longest rows first (the
// short rows fill the tail).  `qa_only`: as for pool_kernel.
__global__ void __launch_bounds__(256) map_softmax_kernel(float *__restrict__ map,
                                                          float *__restrict__ est_last,
                                                          long long rows_total, int nb,
                                                          const int32_t *__restrict__ qa_only) {
  const long long row = (long long)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows_total) return;
  const long long heads = rows_total / nb;
  const long long bh = row % heads;
  if (qa_only && qa_only[bh] != FP_PATTERN_QA) return;
  const int i = nb - 1 - int(row / heads);
  float *r = map + bh * ((long long)nb * (nb + 1) / 2) + (long long)i * (i + 1) / 2;
  map_row_softmax(r, i + 1, i == nb - 1 ? est_last + bh * nb : nullptr, lane);
}

// The softmax of the map's last row alone (the estimate a-hat that the
// pattern test needs; its logits from launch_map_logits_tc with last_only),
// for every head: grid (Bt*Hq), one warp.  The same map_row_softmax as every
// row of map_softmax_kernel, so the row is bitwise the full map's.
__global__ void __launch_bounds__(32) map_last_softmax_kernel(float *__restrict__ map,
                                                              float *__restrict__ est_last,
                                                              int nb) {
  const size_t bh = blockIdx.x;
  float *r = map + bh * (size_t(nb) * (nb + 1) / 2) + size_t(nb - 1) * nb / 2;
  map_row_softmax(r, nb, est_last + bh * nb, threadIdx.x);
}

// ---------------------------------------------------- last query block --
// S tile: scale * q_last[BS x D] . k_tile[BS x D]^T into smem S[BS][BS+1],
// causally masked (-inf) when the key tile is the diagonal one.
template <int BS, int D, class T>
struct LastTile {
  static constexpr int KC = 32;
  static constexpr int TPR = BS / 16;  // outputs per thread along each axis
  float A[KC][BS + 1];
  float Bm[KC][BS + 1];
  float S[BS][BS + 1];
};

// Rows of q_last at or past qrows and keys at or past krows (a partial last
// block) are read as zeros; the causal mask hides such keys from every real
// query row.
template <int BS, int D, class T>
__device__ void last_tile_scores(LastTile<BS, D, T> &sm, const T *__restrict__ qlast,
                                 const T *__restrict__ ktile, float scale, bool diagonal,
                                 int qrows, int krows) {
  constexpr int KC = LastTile<BS, D, T>::KC;
  constexpr int TPR = LastTile<BS, D, T>::TPR;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[TPR][TPR];
#pragma unroll
  for (int u = 0; u < TPR; ++u)
#pragma unroll
    for (int w = 0; w < TPR; ++w) acc[u][w] = 0.f;
  for (int k0 = 0; k0 < D; k0 += KC) {
    for (int e = threadIdx.x; e < BS * KC; e += 256) {
      int r = e / KC, c = e % KC;
      sm.A[c][r] = r < qrows ? ld_f(qlast + size_t(r) * D + k0 + c) : 0.f;
      sm.Bm[c][r] = r < krows ? ld_f(ktile + size_t(r) * D + k0 + c) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < KC; ++c) {
      float a[TPR], bb[TPR];
#pragma unroll
      for (int u = 0; u < TPR; ++u) a[u] = sm.A[c][ty + 16 * u];
#pragma unroll
      for (int u = 0; u < TPR; ++u) bb[u] = sm.Bm[c][tx + 16 * u];
#pragma unroll
      for (int u = 0; u < TPR; ++u)
#pragma unroll
        for (int w = 0; w < TPR; ++w) acc[u][w] = fmaf(a[u], bb[w], acc[u][w]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < TPR; ++u)
#pragma unroll
    for (int w = 0; w < TPR; ++w) {
      int r = ty + 16 * u, c = tx + 16 * w;
      sm.S[r][c] = (diagonal && c > r) ? -INFINITY : acc[u][w] * scale;
    }
  __syncthreads();
}

// grid (nb, Hq, Bt), 256 threads.
template <int BS, int D, class T>
__global__ void __launch_bounds__(256) last_pass1_kernel(const T *__restrict__ q,
                                                         const T *__restrict__ k, int hq, int g,
                                                         int n, float scale,
                                                         float *__restrict__ pm,
                                                         float *__restrict__ pl) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  auto &sm = *reinterpret_cast<LastTile<BS, D, T> *>(smem_raw);
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z, nb = gridDim.x;
  const int kv = h / g, hkv = hq / g;
  const int q0 = (nb - 1) * BS;  // the last block's first query
  const T *qlast = q + ((size_t(b) * hq + h) * n + q0) * D;
  const T *kt = k + ((size_t(b) * hkv + kv) * n + size_t(j) * BS) * D;
  last_tile_scores<BS, D, T>(sm, qlast, kt, scale, j == nb - 1, n - q0, min(BS, n - j * BS));
  // 256 threads, BS rows: 256/BS threads per row
  constexpr int TPRW = 256 / BS;
  const int r = threadIdx.x / TPRW, part = threadIdx.x % TPRW;
  float mx = -INFINITY;
  for (int c = part; c < BS; c += TPRW) mx = fmaxf(mx, sm.S[r][c]);
#pragma unroll
  for (int o = TPRW / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float s = 0.f;
  if (mx > -INFINITY)
    for (int c = part; c < BS; c += TPRW) s += expf(sm.S[r][c] - mx);
#pragma unroll
  for (int o = TPRW / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (part == 0) {
    size_t o = ((size_t(b) * hq + h) * nb + j) * BS + r;
    pm[o] = mx;
    pl[o] = s;
  }
}

// one thread per (b, h, r): lse over the nb partials, in key-block order.
__global__ void last_lse_kernel(const float *__restrict__ pm, const float *__restrict__ pl,
                                float *__restrict__ lse, int rows, int nb, int bs) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= rows) return;
  const int bh = t / bs, r = t % bs;
  float mx = -INFINITY;
  for (int j = 0; j < nb; ++j) mx = fmaxf(mx, pm[(size_t(bh) * nb + j) * bs + r]);
  float s = 0.f;
  for (int j = 0; j < nb; ++j) {
    size_t o = (size_t(bh) * nb + j) * bs + r;
    if (pm[o] > -INFINITY) s += pl[o] * expf(pm[o] - mx);
  }
  lse[t] = mx + logf(s);
}

// grid (ceil(nb/8), Bt*Hq), 256 threads, one warp per key block j:
// true_last[j] = (1/R) sum over the last block's R rows r of pl[j][r] *
// exp(pm[j][r] - lse[r]), the rows summed in a fixed order (BS/32 per lane,
// then a xor tree).
template <int BS>
__global__ void __launch_bounds__(256) block_mass_kernel(const float *__restrict__ pm,
                                                         const float *__restrict__ pl,
                                                         const float *__restrict__ lse,
                                                         float *__restrict__ true_last, int nb,
                                                         int rows) {
  const int j = blockIdx.x * 8 + threadIdx.x / 32, lane = threadIdx.x % 32;
  if (j >= nb) return;
  const size_t bh = blockIdx.y;
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < BS / 32; ++k) {
    const int r = lane + 32 * k;
    const size_t o = (bh * nb + j) * BS + r;
    if (r < rows) s = fmaf(pl[o], expf(pm[o] - lse[bh * BS + r]), s);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) true_last[bh * nb + j] = s / float(rows);
}

// grid (nb, Hq, Bt), 256 threads; with `vs_only` (a pattern array) heads
// whose pattern is not vertical-slash are skipped.
template <int BS, int D, class T>
__global__ void __launch_bounds__(256) last_pass2_kernel(
    const T *__restrict__ q, const T *__restrict__ k, int hq, int g, int n, float scale,
    const float *__restrict__ lse, float *__restrict__ vert, float *__restrict__ sp,
    const int32_t *__restrict__ vs_only) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  auto &sm = *reinterpret_cast<LastTile<BS, D, T> *>(smem_raw);
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z, nb = gridDim.x;
  const int kv = h / g, hkv = hq / g;
  const size_t bh = size_t(b) * hq + h;
  if (vs_only && vs_only[bh] != FP_PATTERN_VS) return;
  const int q0 = (nb - 1) * BS, rows = n - q0;  // the last block's queries
  const T *qlast = q + (bh * n + q0) * D;
  const T *kt = k + ((size_t(b) * hkv + kv) * n + size_t(j) * BS) * D;
  const int keys = min(BS, n - j * BS);
  last_tile_scores<BS, D, T>(sm, qlast, kt, scale, j == nb - 1, rows, keys);
  for (int e = threadIdx.x; e < BS * BS; e += 256) {
    int r = e / BS, c = e % BS;
    float s = sm.S[r][c];
    sm.S[r][c] = (s == -INFINITY || r >= rows) ? 0.f : expf(s - lse[bh * BS + r]);
  }
  __syncthreads();
  if (threadIdx.x < keys) {
    const int c = threadIdx.x;
    float s = 0.f;
    for (int r = 0; r < BS; ++r) s += sm.S[r][c];
    vert[bh * n + size_t(j) * BS + c] = s;
  }
  // diagonal partials: delta = r - c + BS - 1 in [0, 2BS-2]
  if (threadIdx.x < 2 * BS - 1) {
    const int delta = threadIdx.x;
    float s = 0.f;
    int r0 = delta - (BS - 1) > 0 ? delta - (BS - 1) : 0;
    int r1 = delta < BS - 1 ? delta : BS - 1;
    for (int r = r0; r <= r1; ++r) s += sm.S[r][r - delta + BS - 1];
    sp[(bh * nb + j) * (2 * BS - 1) + delta] = s;
  }
}

// grid (ceil(n/256), Bt*Hq), one thread per (b, h, o): slash[o] from the (at
// most two) key blocks whose diagonal partials hold offset o (q0: the first
// query of the partials' query rows); with `vs_only`, vertical-slash heads
// only.
__global__ void slash_combine_kernel(const float *__restrict__ sp, float *__restrict__ slash,
                                     int n, int q0, int nb, int bs,
                                     const int32_t *__restrict__ vs_only) {
  const size_t bh = blockIdx.y;  // (a head whose pattern skips the lines exits at once)
  if (vs_only && vs_only[bh] != FP_PATTERN_VS) return;
  const int o = blockIdx.x * blockDim.x + threadIdx.x;
  if (o >= n) return;
  const size_t t = bh * n + o;
  // query row c (position q0 + c) and key r of tile j (position j bs + r) sit
  // at delta = c - r + bs - 1 = (j + 1) bs - 1 - u with u = q0 - o, valid in
  // [0, 2bs-2]: (j + 1) bs in [u + 1, u + 2bs - 1], i.e. j + 1 = m1 or m1 + 1
  // with m1 = ceil((u + 1) / bs) (u + 2bs > 0 keeps the division positive)
  const long long u = (long long)q0 - o;
  const long long m1 = (u + 2ll * bs) / bs - 1;
  float s = 0.f;
  for (long long j = m1 - 1; j <= m1; ++j) {  // ascending, a fixed order
    if (j < 0 || j >= nb) continue;
    const long long delta = (j + 1) * bs - 1 - u;
    if (delta >= 0 && delta <= 2 * bs - 2) s += sp[(bh * nb + j) * (2 * bs - 1) + delta];
  }
  slash[t] = s;
}

// CUDA-core workspace: pass-1 partials per (row, key block), the rows'
// log-sum-exps and the diagonal partials.
struct CoreWs {
  float *pm, *pl, *lse, *sp;
  size_t bytes;
};
CoreWs carve_core(const Dims &Dm, void *ws) {
  Carver c{static_cast<char *>(ws), 0};
  const size_t rows = size_t(Dm.bt) * Dm.hq;
  CoreWs w;
  w.pm = c.take<float>(rows * Dm.nb * Dm.bs);
  w.pl = c.take<float>(rows * Dm.nb * Dm.bs);
  w.lse = c.take<float>(rows * Dm.bs);
  w.sp = c.take<float>(rows * Dm.nb * (2 * Dm.bs - 1));
  w.bytes = c.off + 256;
  return w;
}

// Pass 1, the log-sum-exps and true_last (every head).
template <int BS, int D, class T>
cudaError_t run_last_rows(const Dims &Dm, const T *q, const T *k, float *true_last, void *ws,
                          cudaStream_t st) {
  const CoreWs w = carve_core(Dm, ws);
  const size_t rows = size_t(Dm.bt) * Dm.hq;
  const float scale = 1.f / sqrtf(float(D));
  const size_t smem = sizeof(LastTile<BS, D, T>);
  cudaFuncSetAttribute(last_pass1_kernel<BS, D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       int(smem));
  last_pass1_kernel<BS, D, T><<<dim3(Dm.nb, Dm.hq, Dm.bt), 256, smem, st>>>(q, k, Dm.hq, Dm.g,
                                                                            Dm.n, scale, w.pm,
                                                                            w.pl);
  const int lrows = int(rows * BS);
  last_lse_kernel<<<(lrows + 127) / 128, 128, 0, st>>>(w.pm, w.pl, w.lse, lrows, Dm.nb, BS);
  block_mass_kernel<BS><<<dim3((Dm.nb + 7) / 8, unsigned(rows)), 256, 0, st>>>(
      w.pm, w.pl, w.lse, true_last, Dm.nb, Dm.n - (Dm.nb - 1) * BS);
  return cudaGetLastError();
}

// Pass 2 and the slash combine (after run_last_rows on the same workspace);
// with `vs_only`, vertical-slash heads only.
template <int BS, int D, class T>
cudaError_t run_last_lines(const Dims &Dm, const T *q, const T *k, float *vert, float *slash,
                           const int32_t *vs_only, void *ws, cudaStream_t st) {
  const CoreWs w = carve_core(Dm, ws);
  const size_t rows = size_t(Dm.bt) * Dm.hq;
  const float scale = 1.f / sqrtf(float(D));
  const size_t smem = sizeof(LastTile<BS, D, T>);
  cudaFuncSetAttribute(last_pass2_kernel<BS, D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       int(smem));
  last_pass2_kernel<BS, D, T><<<dim3(Dm.nb, Dm.hq, Dm.bt), 256, smem, st>>>(
      q, k, Dm.hq, Dm.g, Dm.n, scale, w.lse, vert, w.sp, vs_only);
  slash_combine_kernel<<<dim3((Dm.n + 255) / 256, unsigned(rows)), 256, 0, st>>>(
      w.sp, slash, Dm.n, (Dm.nb - 1) * BS, Dm.nb, BS, vs_only);
  return cudaGetLastError();
}

// Q pooling and the block map (logits on the tensor cores, then the row
// softmax); with `qa_only`, for query-aware heads only.
template <class T>
cudaError_t run_map(const Dims &Dm, const T *q, float *qbar, const float *kbar_hi,
                    const float *kbar_lo, float *map, float *est_last, const int32_t *qa_only,
                    cudaStream_t st) {
  pool_kernel<T><<<dim3(Dm.nb, Dm.hq, Dm.bt), 256, 0, st>>>(q, qbar, Dm.n, Dm.d, Dm.bs, Dm.nb,
                                                             0, qa_only);
  cudaError_t e = launch_map_logits_tc(Dm, qbar, kbar_hi, kbar_lo, map, qa_only, false, st);
  if (e != cudaSuccess) return e;
  const long long rows = (long long)Dm.bt * Dm.hq * Dm.nb;
  map_softmax_kernel<<<unsigned((rows + 7) / 8), 256, 0, st>>>(map, est_last, rows, Dm.nb,
                                                               qa_only);
  return cudaGetLastError();
}

// The true last-block distribution (every head), and K pooled into kbar with
// its tf32 halves: by the tensor-core pass from the key tiles it streams, or
// by its own pooling launch before the CUDA-core passes.
template <class T>
cudaError_t run_true_last(const Dims &Dm, const T *q, const T *k, float *true_last, float *kbar,
                          float *kbar_hi, float *kbar_lo, void *ws, cudaStream_t st) {
  if (last_block_tc_supported(Dm))
    return launch_last_block_rows_tc(Dm, q, k, true_last, kbar, kbar_hi, kbar_lo, ws, st);
  pool_kernel<T><<<dim3(Dm.nb, Dm.hkv, Dm.bt), 256, 0, st>>>(k, kbar, Dm.n, Dm.d, Dm.bs, Dm.nb,
                                                              0, nullptr, kbar_hi, kbar_lo);
  if (Dm.bs == 128 && Dm.d == 128) return run_last_rows<128, 128, T>(Dm, q, k, true_last, ws, st);
  if (Dm.bs == 128 && Dm.d == 64) return run_last_rows<128, 64, T>(Dm, q, k, true_last, ws, st);
  if (Dm.bs == 64 && Dm.d == 128) return run_last_rows<64, 128, T>(Dm, q, k, true_last, ws, st);
  return run_last_rows<64, 64, T>(Dm, q, k, true_last, ws, st);
}

// The vertical and slash sums (after run_true_last on the same workspace); with
// `vs_only`, for the vertical-slash heads of that pattern array only.
template <class T>
cudaError_t run_lines(const Dims &Dm, const T *q, const T *k, float *vert, float *slash,
                      const int32_t *vs_only, void *ws, cudaStream_t st) {
  if (last_block_tc_supported(Dm)) {
    float *sp = nullptr;
    cudaError_t e = launch_last_block_lines_tc(Dm, q, k, vert, vs_only, &sp, ws, st);
    if (e != cudaSuccess) return e;
    // the passes' partials are per 128-key tile, whatever the block size
    const int nt = last_block_tc_tiles(Dm);
    slash_combine_kernel<<<dim3((Dm.n + 255) / 256, unsigned(Dm.bt * Dm.hq)), 256, 0, st>>>(
        sp, slash, Dm.n, (nt - 1) * 128, nt, 128, vs_only);
    return cudaGetLastError();
  }
  if (Dm.bs == 128 && Dm.d == 128)
    return run_last_lines<128, 128, T>(Dm, q, k, vert, slash, vs_only, ws, st);
  if (Dm.bs == 128 && Dm.d == 64)
    return run_last_lines<128, 64, T>(Dm, q, k, vert, slash, vs_only, ws, st);
  if (Dm.bs == 64 && Dm.d == 128)
    return run_last_lines<64, 128, T>(Dm, q, k, vert, slash, vs_only, ws, st);
  return run_last_lines<64, 64, T>(Dm, q, k, vert, slash, vs_only, ws, st);
}

// The pooled keys' tf32 halves in the staged estimate's workspace, after the
// last-block passes' region (both are live at once: the first pass writes
// them and the map reads them).
size_t passes_ws_bytes(const Dims &D) {
  return last_block_tc_supported(D) ? last_block_tc_ws_bytes(D) : carve_core(D, nullptr).bytes;
}
struct Split {
  float *hi, *lo;
};
Split carve_split(const Dims &Dm, void *ws) {
  Carver c{static_cast<char *>(ws), (passes_ws_bytes(Dm) + 255) & ~size_t(255)};
  const size_t n = size_t(Dm.bt) * Dm.hkv * Dm.nb * Dm.d;
  Split sp;
  sp.hi = c.take<float>(n);
  sp.lo = c.take<float>(n);
  return sp;
}

template <class T>
cudaError_t run_estimate(const Dims &Dm, const T *q, const T *k, float *qbar, float *kbar,
                         float *map, float *est_last, float *true_last, float *vert,
                         float *slash, void *ws, cudaStream_t st) {
  const Split sp = carve_split(Dm, ws);
  cudaError_t e = run_true_last<T>(Dm, q, k, true_last, kbar, sp.hi, sp.lo, ws, st);
  if (e != cudaSuccess) return e;
  e = run_map<T>(Dm, q, qbar, sp.hi, sp.lo, map, est_last, nullptr, st);
  if (e != cudaSuccess) return e;
  return run_lines<T>(Dm, q, k, vert, slash, nullptr, ws, st);
}

// Pattern-aware first part: everything the pattern test reads, for every head
// (K pooled, Q pooled over the last block only, the map's last row and the
// true last-block distribution), and nothing else.
template <class T>
cudaError_t run_decision(const Dims &Dm, const T *q, const T *k, float *qbar, float *kbar,
                         float *kbar_hi, float *kbar_lo, float *map, float *est_last,
                         float *true_last, void *ws, cudaStream_t st) {
  cudaError_t e = run_true_last<T>(Dm, q, k, true_last, kbar, kbar_hi, kbar_lo, ws, st);
  if (e != cudaSuccess) return e;
  pool_kernel<T><<<dim3(1, Dm.hq, Dm.bt), 256, 0, st>>>(q, qbar, Dm.n, Dm.d, Dm.bs, Dm.nb,
                                                         Dm.nb - 1, nullptr);
  e = launch_map_logits_tc(Dm, qbar, kbar_hi, kbar_lo, map, nullptr, true, st);
  if (e != cudaSuccess) return e;
  map_last_softmax_kernel<<<unsigned(Dm.bt * Dm.hq), 32, 0, st>>>(map, est_last, Dm.nb);
  return cudaGetLastError();
}

}  // namespace

size_t estimate_ws_bytes(const Dims &D) {
  return ((passes_ws_bytes(D) + 255) & ~size_t(255)) + map_split_bytes(D);
}

cudaError_t launch_estimate_decision(const Dims &D, const void *q, const void *k, float *qbar,
                                     float *kbar, float *kbar_hi, float *kbar_lo, float *map,
                                     float *est_last, float *true_last, void *ws,
                                     cudaStream_t st) {
  if (D.dtype == FP_F32)
    return run_decision<float>(D, static_cast<const float *>(q), static_cast<const float *>(k),
                               qbar, kbar, kbar_hi, kbar_lo, map, est_last, true_last, ws, st);
  return run_decision<__nv_bfloat16>(D, static_cast<const __nv_bfloat16 *>(q),
                                     static_cast<const __nv_bfloat16 *>(k), qbar, kbar, kbar_hi,
                                     kbar_lo, map, est_last, true_last, ws, st);
}

cudaError_t launch_estimate_lines_vs(const Dims &D, const void *q, const void *k, float *vert,
                                     float *slash, const int32_t *pattern, void *ws,
                                     cudaStream_t st) {
  if (D.dtype == FP_F32)
    return run_lines<float>(D, static_cast<const float *>(q), static_cast<const float *>(k),
                            vert, slash, pattern, ws, st);
  return run_lines<__nv_bfloat16>(D, static_cast<const __nv_bfloat16 *>(q),
                                  static_cast<const __nv_bfloat16 *>(k), vert, slash, pattern,
                                  ws, st);
}

cudaError_t launch_estimate_map_qa(const Dims &D, const void *q, float *qbar,
                                   const float *kbar_hi, const float *kbar_lo, float *map,
                                   float *est_last, const int32_t *pattern, cudaStream_t st) {
  if (D.dtype == FP_F32)
    return run_map<float>(D, static_cast<const float *>(q), qbar, kbar_hi, kbar_lo, map,
                          est_last, pattern, st);
  return run_map<__nv_bfloat16>(D, static_cast<const __nv_bfloat16 *>(q), qbar, kbar_hi,
                                kbar_lo, map, est_last, pattern, st);
}

cudaError_t launch_estimate(const Dims &D, const void *q, const void *k, float *qbar,
                            float *kbar, float *map, float *est_last, float *true_last,
                            float *vert, float *slash, void *ws, cudaStream_t st) {
  if (D.dtype == FP_F32)
    return run_estimate<float>(D, static_cast<const float *>(q), static_cast<const float *>(k),
                               qbar, kbar, map, est_last, true_last, vert, slash, ws, st);
  return run_estimate<__nv_bfloat16>(D, static_cast<const __nv_bfloat16 *>(q),
                                     static_cast<const __nv_bfloat16 *>(k), qbar, kbar, map,
                                     est_last, true_last, vert, slash, ws, st);
}

}  // namespace fpi
