// pattern.cu -- fp_pattern: square-root Jensen-Shannon distance per head and
// the query-aware / vertical-slash switch.
//
// FlexPrefill (atlas.scime.ai summary, "Approach"): the estimate is accurate
// when the square-root JS divergence to the true distribution is below tau;
// the "Measured effects" table (tau = 0 turns query-aware mode off) makes the
// comparison strict.  Natural log; both inputs renormalised; 0 log 0 = 0.
#include "fp_internal.cuh"

namespace fpi {
namespace {

__device__ double block_sum(double v, double *red) {
  // fixed-shape tree over 256 threads: deterministic
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  double s = 0.0;
  if (threadIdx.x == 0)
    for (int i = 0; i < 8; ++i) s += red[i];
  __syncthreads();
  if (threadIdx.x == 0) red[0] = s;
  __syncthreads();
  return red[0];
}

// grid (Hq, Bt), 256 threads.
__global__ void __launch_bounds__(256) pattern_kernel(const float *__restrict__ est,
                                                      const float *__restrict__ tru, int nb,
                                                      double tau, float *__restrict__ djs,
                                                      int32_t *__restrict__ pattern) {
  __shared__ double red[8];
  const size_t bh = size_t(blockIdx.y) * gridDim.x + blockIdx.x;
  const float *p = est + bh * nb;
  const float *q = tru + bh * nb;
  double sp = 0.0, sq = 0.0;
  for (int i = threadIdx.x; i < nb; i += 256) {
    sp += double(p[i]);
    sq += double(q[i]);
  }
  sp = block_sum(sp, red);
  sq = block_sum(sq, red);
  double acc = 0.0;
  for (int i = threadIdx.x; i < nb; i += 256) {
    const double a = double(p[i]) / sp, b = double(q[i]) / sq;
    const double m = 0.5 * (a + b);
    if (a > 0.0) acc += 0.5 * a * log(a / m);
    if (b > 0.0) acc += 0.5 * b * log(b / m);
  }
  acc = block_sum(acc, red);
  if (threadIdx.x == 0) {
    const double d = sqrt(acc > 0.0 ? acc : 0.0);
    djs[bh] = float(d);
    pattern[bh] = d < tau ? FP_PATTERN_QA : FP_PATTERN_VS;
  }
}

}  // namespace

cudaError_t launch_pattern(const Dims &D, float tau, const float *est_last,
                           const float *true_last, float *djs, int32_t *pattern,
                           cudaStream_t st) {
  pattern_kernel<<<dim3(D.hq, D.bt), 256, 0, st>>>(est_last, true_last, D.nb, double(tau), djs,
                                                   pattern);
  return cudaGetLastError();
}

}  // namespace fpi
