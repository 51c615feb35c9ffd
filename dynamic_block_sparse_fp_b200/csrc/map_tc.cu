// map_tc.cu -- the logits of the estimated block map, scale * qbar_i . kbar_j
// for the causal block pairs j <= i of every head, on the sm_100a tensor cores.
//
// FlexPrefill (atlas.scime.ai summary, "Approach"): block-pooled queries and
// keys give the estimated block attention of every query block.  Its logits
// are a dense product of the pooled matrices (nb x d times d x nb per head), so
// they run as tcgen05 MMAs.  fp32 accuracy from the tf32 tensor cores: each
// operand is split as x = hi + lo, hi = x with its low 13 mantissa bits
// cleared (exact in tf32) and lo = x - hi (exact in fp32), and the product is
// hi.hi + hi.lo + lo.hi accumulated in fp32 (the dropped lo.lo term and lo's
// own tf32 rounding are below 2^-19 of |x| |y|, so a logit is off by at most
// about 2^-19 of sum_k |qbar_k kbar_k| times the scale).  The keys' halves come from
// the K pooling (pool_kernel writes them beside kbar); the queries' are formed
// here on the way into TMEM.
//
// One CTA per (head, row tile ti of 128 query blocks) walks the key tiles
// tj = 0 .. ti (the longest strips first); with `last_only` a CTA takes one key
// tile of the last row tile, and only the map's last row is computed (every
// other query row is zero in A and never written: a row's logits depend on
// its own A row only, so they are bitwise those of the full map).
// TMEM (512 columns): pooled queries hi [0, d), lo [d, 2d) (A operand, one
// fp32 per column); two 128-column accumulators at 256 and 384, so the MMAs of
// tile t + 1 run while the epilogue writes tile t.
// Shared memory: a 5-slot ring of key chunks (128 key blocks x 32 d, hi and
// lo, 128-B swizzled, by TMA) and a 128 x 128 staging tile through which a
// warp writes 128 consecutive floats of one map row.
// Warps: 0-7 epilogue (thread = tile row = TMEM lane of its quarter, each
// warp of a quarter taking half of the columns), 8 TMA producer, 9 MMA
// issuer.  Every wait is bounded; on expiry the kernel records FP_ERR_TIMEOUT,
// raises a CTA abort flag, drains its loads and frees TMEM.
// The kernel is held by the key-tile stream (128 KB of hi and lo per 128 x 128
// tile, from L2), not by the tensor pipe: at 128k the pipe is busy about 40 %.
#include "fp_internal.cuh"

namespace fpi {
namespace {

constexpr int MT = 128;                     // query / key blocks per tile
constexpr int KC = 32;                      // fp32 elements of d per 128-B row
constexpr int NCH = 5;                      // chunk slots
constexpr uint32_t CH_BYTES = MT * KC * 4;  // 16 KB: [128 key blocks x 32 d]
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 256;

struct MapSmem {
  uint8_t khi[NCH][CH_BYTES];
  uint8_t klo[NCH][CH_BYTES];
  float stage[MT * MT];  // 16-B chunks swizzled by row (see the epilogue)
  uint64_t full[NCH], empty[NCH];
  uint64_t q_ready, acc_full[2], acc_empty[2], st_full, st_free;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(MapSmem) <= 227 * 1024, "shared memory");

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::tf32 (fp32 operands read as tf32,
// fp32 accumulate); A: one element per TMEM column, a K = 8 step spans 8.
__device__ __forceinline__ void tc_mma_ts_tf32(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::tf32: tf32 A and B (both K-major), fp32 D.
constexpr uint32_t idesc_tf32(int m, int n) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(n >> 3) << 17) |
         (uint32_t(m >> 4) << 24);
}

template <int D>
__global__ void __launch_bounds__(320, 1) map_logits_tc_kernel(
    const __grid_constant__ CUtensorMap tm_hi, const __grid_constant__ CUtensorMap tm_lo,
    const float *__restrict__ qbar, float *__restrict__ map, int hq, int g, int nb, float scale,
    const int32_t *__restrict__ qa_only, int last_only, int *status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the swizzled chunks need a 1024-B aligned window (no slack to realign)
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) report(status, FP_ERR_UNSUPPORTED);
    return;
  }
  const int bh = blockIdx.x;  // batch * hq + head
  if (qa_only && qa_only[bh] != FP_PATTERN_QA) return;
  MapSmem &sm = *reinterpret_cast<MapSmem *>(smem_raw);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int b = bh / hq, h = bh % hq, hkv = hq / g, kv = h / g;
  const int nbt = (nb + MT - 1) / MT;
  // blockIdx.y = 0 first: the longest strips of every head start first
  const int ti = last_only ? nbt - 1 : nbt - 1 - int(blockIdx.y);
  const int tj0 = last_only ? int(blockIdx.y) : 0;
  const int ntile = last_only ? 1 : ti + 1;
  constexpr int NC = D / KC;  // chunks per key tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < NCH; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.q_ready, 256);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.acc_full[a], 1);
      mbar_init(&sm.acc_empty[a], 256);
    }
    mbar_init(&sm.st_full, 256);
    mbar_init(&sm.st_free, 256);
    sm.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 9) {
    tmem_alloc(&sm.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int *abort_flag = &sm.abort_flag;
  auto fail = [&](int code) {
    report(status, code);
    *abort_flag = 1;
  };

  if (warp == 8) {
    // ------------------------------------------------------- TMA producer --
    if (lane == 0) {
      prefetch_tmap(&tm_hi);
      prefetch_tmap(&tm_lo);
      const int row0 = (b * hkv + kv) * nb;  // first pooled key row of this kv head
      int issued = 0;
      for (int t = 0; t < ntile && !*abort_flag; ++t) {
        // rows past this head's nb belong to the next head or are zero-filled;
        // the epilogue never writes their columns
        const int y = row0 + (tj0 + t) * MT;
        for (int c = 0; c < NC; ++c) {
          const int u = t * NC + c, s = u % NCH;
          if (!mbar_wait(&sm.empty[s], ((u / NCH) & 1) ^ 1, abort_flag)) {
            fail(FP_ERR_TIMEOUT);
            break;
          }
          mbar_arrive_expect_tx(&sm.full[s], 2 * CH_BYTES);
          tma_load_2d(sm.khi[s], &tm_hi, &sm.full[s], c * KC, y);
          tma_load_2d(sm.klo[s], &tm_lo, &sm.full[s], c * KC, y);
          issued = u + 1;
        }
      }
      if (*abort_flag) {
        // drain: wait (bounded) for the loads still in flight, the last of each slot
        volatile int never = 0;
        for (int u = issued - NCH > 0 ? issued - NCH : 0; u < issued; ++u)
          mbar_wait(&sm.full[u % NCH], (u / NCH) & 1, &never, 100000000ull);
      }
    }
  } else if (warp == 9) {
    // --------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_tf32(MT, MT);
      bool ok = mbar_wait(&sm.q_ready, 0, abort_flag);
      for (int t = 0; ok && t < ntile; ++t) {
        const int a = t & 1;
        if (!mbar_wait(&sm.acc_empty[a], ((t >> 1) & 1) ^ 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dacc = tmem + ACC_COL + uint32_t(a * MT);
        for (int c = 0; c < NC && ok; ++c) {
          const int u = t * NC + c, s = u % NCH;
          if (!mbar_wait(&sm.full[s], (u / NCH) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t hi_addr = smem_u32(sm.khi[s]), lo_addr = smem_u32(sm.klo[s]);
#pragma unroll
          for (int ks = 0; ks < KC / 8; ++ks) {
            // K = 8 d: 8 TMEM columns of A, 32 B inside the 128-B rows of B
            const uint32_t qh = tmem + uint32_t(c * KC + ks * 8);
            const uint32_t ql = qh + uint32_t(D);
            const uint64_t bhi = umma_desc_sw128(hi_addr + ks * 32, 16, 1024);
            const uint64_t blo = umma_desc_sw128(lo_addr + ks * 32, 16, 1024);
            tc_mma_ts_tf32(dacc, qh, bhi, idesc, (c > 0 || ks > 0) ? 1u : 0u);
            tc_mma_ts_tf32(dacc, qh, blo, idesc, 1u);
            tc_mma_ts_tf32(dacc, ql, bhi, idesc, 1u);
          }
          tc_commit(&sm.empty[s]);
        }
        if (ok) tc_commit(&sm.acc_full[a]);
      }
      if (!ok) fail(FP_ERR_TIMEOUT);
    }
  } else {
    // ------------------------------------------------- epilogue (warps 0-7) --
    // warp w: TMEM lane quarter w % 4 (tile rows 32(w%4) ..), column half
    // w / 4 (64 of the 128 logits of a tile row, and half of the pooled
    // query's d going in)
    const int quarter = warp & 3, ch = warp >> 2;
    const int r = quarter * 32 + lane;  // tile row, TMEM lane
    const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
    const int i = ti * MT + r;  // this row's query block
    const bool has_row = i < nb && (!last_only || i == nb - 1);
    {
      // pooled query row, split into tf32 hi / lo, into TMEM columns [0, 2d)
      const int ir = i < nb ? i : nb - 1;  // (rows past nb are zero, never read)
      const float4 *src = reinterpret_cast<const float4 *>(qbar + (size_t(bh) * nb + ir) * D);
#pragma unroll
      for (int c0 = ch * (D / 2); c0 < (ch + 1) * (D / 2); c0 += 32) {
        uint32_t hi[32], lo[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const float4 x = has_row ? __ldg(src + c0 / 4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
          const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float hv = tf32_hi(xs[e]);
            hi[4 * v + e] = __float_as_uint(hv);
            lo[4 * v + e] = __float_as_uint(xs[e] - hv);
          }
        }
        tmem_st32(lane_base + uint32_t(c0), hi);
        tmem_st32(lane_base + uint32_t(D + c0), lo);
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.q_ready);
    }
    bool ok = true;
    float *mhead = map + size_t(bh) * (size_t(nb) * (nb + 1) / 2);
    float *stage = sm.stage;
    for (int t = 0; t < ntile; ++t) {
      const int a = t & 1, tj = tj0 + t;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.acc_full[a], (t >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // the staging tile is free once the previous tile's rows were copied out
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.st_free, (t & 1) ^ 1, abort_flag))) {
        ok = false;
        break;
      }
      // row r of the staging tile: 16-B chunk k (columns 4k .. 4k+3) sits at
      // chunk k ^ (r % 8), so both the row-wise 16-B writes here and the
      // column-consecutive reads below are free of bank conflicts
#pragma unroll
      for (int c0 = ch * 64; c0 < ch * 64 + 64; c0 += 32) {
        uint32_t u[32];
        tmem_ld32(lane_base + ACC_COL + uint32_t(a * MT + c0), u);
        tc_wait_ld();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int chunk = (c0 / 4 + k) ^ (r & 7);
          *reinterpret_cast<float4 *>(stage + r * MT + 4 * chunk) =
              make_float4(__uint_as_float(u[4 * k]) * scale, __uint_as_float(u[4 * k + 1]) * scale,
                          __uint_as_float(u[4 * k + 2]) * scale,
                          __uint_as_float(u[4 * k + 3]) * scale);
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.acc_empty[a]);
      mbar_arrive(&sm.st_full);
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.st_full, t & 1, abort_flag))) {
        ok = false;
        break;
      }
      // copy out: warp w writes rows w, w + 8, ..., eight rows per batch (all
      // their shared-memory reads issued before their stores); row ii keeps
      // its causal columns j <= ii of this key tile (ii < nb, so j < nb too)
#pragma unroll
      for (int r0 = warp; r0 < MT; r0 += 64) {
        float val[8][MT / 32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int rr = r0 + 8 * q;
#pragma unroll
          for (int c4 = 0; c4 < MT / 32; ++c4) {
            const int c = lane + 32 * c4;
            val[q][c4] = stage[rr * MT + 4 * ((c / 4) ^ (rr & 7)) + (c & 3)];
          }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int ii = ti * MT + r0 + 8 * q;
          if (ii >= nb || (last_only && ii != nb - 1)) continue;
          const int ncol = min(MT, ii + 1 - tj * MT);
          float *dst = mhead + size_t(ii) * (ii + 1) / 2 + size_t(tj) * MT;
#pragma unroll
          for (int c4 = 0; c4 < MT / 32; ++c4)
            if (lane + 32 * c4 < ncol) dst[lane + 32 * c4] = val[q][c4];
        }
      }
      mbar_arrive(&sm.st_free);
    }
    if (!ok) fail(FP_ERR_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// 2-D fp32 tensor map over [rows x d] with a box of [128 rows x 32].
bool encode_f32(CUtensorMap *m, const void *ptr, uint64_t rows, int d) {
  const PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(d) * 4};
  const cuuint32_t box[2] = {KC, MT};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_d(const Dims &Dm, const CUtensorMap &mh, const CUtensorMap &ml,
                     const float *qbar, float *map, const int32_t *qa_only, bool last_only,
                     cudaStream_t st) {
  const int nbt = (Dm.nb + MT - 1) / MT;
  const float scale = 1.f / sqrtf(float(D));
  cudaFuncSetAttribute(map_logits_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       int(sizeof(MapSmem)));
  map_logits_tc_kernel<D><<<dim3(Dm.bt * Dm.hq, nbt), 320, sizeof(MapSmem), st>>>(
      mh, ml, qbar, map, Dm.hq, Dm.g, Dm.nb, scale, qa_only, last_only ? 1 : 0,
      device_status_ptr());
  return cudaGetLastError();
}

}  // namespace

size_t map_split_bytes(const Dims &D) {
  return 2 * (size_t(D.bt) * D.hkv * D.nb * D.d * sizeof(float) + 256);
}

cudaError_t launch_map_logits_tc(const Dims &D, const float *qbar, const float *kbar_hi,
                                 const float *kbar_lo, float *map, const int32_t *qa_only,
                                 bool last_only, cudaStream_t st) {
  if (D.d != 64 && D.d != 128) return cudaErrorInvalidValue;
  CUtensorMap mh, ml;
  const uint64_t rows = uint64_t(D.bt) * D.hkv * D.nb;
  if (!encode_f32(&mh, kbar_hi, rows, D.d) || !encode_f32(&ml, kbar_lo, rows, D.d))
    return cudaErrorInvalidValue;
  if (D.d == 128) return launch_d<128>(D, mh, ml, qbar, map, qa_only, last_only, st);
  return launch_d<64>(D, mh, ml, qbar, map, qa_only, last_only, st);
}

}  // namespace fpi
