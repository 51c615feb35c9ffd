// estimate_tc.cu -- the true attention of the last query block on the sm_100a
// tensor cores (bf16 inputs, block 128, head dim 128): the two passes of
// fp_estimate that dominate its cost.
//
// FlexPrefill (atlas.scime.ai summary, "Approach"): the block-pooled estimate
// is checked against the true attention distribution of the last query
// block; the vertical-slash pattern is chosen from that block's column and
// diagonal attention sums.
//
// Pass 1 (row statistics): S = Q_last K^T per key tile, thread = query row
//   (= TMEM lane); every CTA keeps an online max / sum of 2^(S*scale*log2e)
//   per row over its chunk of key tiles and writes one partial per row.
// Combine: partials -> log-sum-exp of every last-block row (log2 units).
// Pass 2 (sums): S^T = K Q_last^T per key tile, thread = key (= TMEM lane),
//   so P = 2^(S^T*scale*log2e - lse2[query]) is summed per thread into the
//   vertical score of its key; the tile's mass goes to the pooled true
//   distribution; diagonal (query - key) sums of the tile are formed by a
//   register-systolic shuffle within each warp and combined across warps in
//   a fixed order, giving the slash partials of the tile.
// Every reduction has a fixed order, so results are reproducible.
//
// CTA: one kv head, a pair of its query heads (A, B), a chunk of key tiles.
// 12 warps: 0-3 consumer of head A, 4-7 consumer of head B, 8 TMA producer
// (Q_last of both heads, K tiles through a 3-entry ring), 9 MMA issuer,
// 10-11 idle (registers are granted per warpgroup).  TMEM 512 columns: S
// double-buffered per head, head A [0,256), head B [256,512).
#include <math.h>

#include "fp_internal.cuh"

namespace fpi {
namespace {

constexpr int BS = 128;  // block size = last-block rows = key tile
constexpr int HD = 128;  // head dim
constexpr int RING = 3;
constexpr int kThreads = 384;
constexpr int kChunk = 16;  // key tiles per CTA
constexpr uint32_t TILE_BYTES = BS * HD * 2;
constexpr uint32_t HALF_BYTES = TILE_BYTES / 2;
constexpr int kBins = 2 * BS - 1;  // diagonals of a tile
constexpr int kWarpBins = BS + 31;  // diagonals one warp of keys touches

struct EstSmem {
  uint8_t q[2][TILE_BYTES];
  uint8_t ring[RING][TILE_BYTES];
  float lse2[2][BS];               // pass 2: per-query log2-sum-exp
  float bins[2][4][kWarpBins];     // pass 2: per-warp diagonal sums
  float warp_mass[2][4];
  uint64_t q_full, ring_full[RING], ring_empty[RING], s_full[2], s_free[2];
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kSmemBytes = sizeof(EstSmem) + 1024;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Barrier over the 128 threads of one consumer warpgroup (ids 1 and 2).
__device__ __forceinline__ void wg_sync(int wg) {
  asm volatile("bar.sync %0, 128;" ::"r"(wg + 1) : "memory");
}

// nb counts 128-key tiles.  Block size 64 (QLO = 64) runs the same tiles: the
// queries are the last 128 rows with the first QLO left out of every sum, and
// each tile holds two output blocks (nb_out = 2 nb).  QLO is a template
// parameter so that block size 128 carries no extra compare per element.
template <int PASS, int QLO>
__global__ void __launch_bounds__(kThreads, 1) last_block_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    int hq, int g, int n_tok, int nb, int nb_out, int n_chunks, float *__restrict__ pm,
    float *__restrict__ pl, const float *__restrict__ lse2g, float *__restrict__ vert,
    float *__restrict__ true_last, float *__restrict__ sp, int *status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  EstSmem &sm = *reinterpret_cast<EstSmem *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int hkv = hq / g;
  const int pairs = (g + 1) / 2;
  const int chunk = blockIdx.x;
  const int kv = blockIdx.y / pairs, pair = blockIdx.y % pairs, b = blockIdx.z;
  const int h0 = kv * g + 2 * pair;
  const int nheads = (2 * pair + 1 < g) ? 2 : 1;
  const int j0 = chunk * kChunk;
  const int j1 = min(nb, j0 + kChunk);
  const int ntiles = j1 - j0;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int r = 0; r < RING; ++r) {
      mbar_init(&sm.ring_full[r], 1);
      mbar_init(&sm.ring_empty[r], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.s_free[s], 128 * nheads);
    }
    sm.abort_flag = 0;
    mbar_fence_init();
  }
  if (PASS == 2 && threadIdx.x < 2 * BS) {
    const int hh = threadIdx.x / BS, r = threadIdx.x % BS;
    sm.lse2[hh][r] = hh < nheads ? lse2g[(size_t(b) * hq + h0 + hh) * BS + r] : 0.f;
  }
  if (warp == 9) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int *abort_flag = &sm.abort_flag;

  if (warp == 8) {
    // ------------------------------------------------------- TMA producer --
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      mbar_arrive_expect_tx(&sm.q_full, TILE_BYTES * nheads);
      for (int hh = 0; hh < nheads; ++hh) {
        const int qrow = int((size_t(b) * hq + h0 + hh) * n_tok + (n_tok - BS));
        tma_load_2d(sm.q[hh], &tm_q, &sm.q_full, 0, qrow);
        tma_load_2d(sm.q[hh] + HALF_BYTES, &tm_q, &sm.q_full, 64, qrow);
      }
      const size_t krow0 = (size_t(b) * hkv + kv) * n_tok;
      int t = 0;
      for (; t < ntiles; ++t) {
        const int slot = t % RING;
        if (!mbar_wait(&sm.ring_empty[slot], ((t / RING) & 1) ^ 1, abort_flag)) {
          report(status, FP_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        const int row = int(krow0 + size_t(j0 + t) * BS);
        mbar_arrive_expect_tx(&sm.ring_full[slot], TILE_BYTES);
        tma_load_2d(sm.ring[slot], &tm_k, &sm.ring_full[slot], 0, row);
        tma_load_2d(sm.ring[slot] + HALF_BYTES, &tm_k, &sm.ring_full[slot], 64, row);
      }
      if (*abort_flag) {
        volatile int never = 0;
        mbar_wait(&sm.q_full, 0, &never, 100000000ull);
        for (int p = t - RING > 0 ? t - RING : 0; p < t; ++p)
          mbar_wait(&sm.ring_full[p % RING], (p / RING) & 1, &never, 100000000ull);
      }
    }
  } else if (warp == 9) {
    // --------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(128, 128, 0);
      bool ok = mbar_wait(&sm.q_full, 0, abort_flag);
      for (int t = 0; ok && t < ntiles; ++t) {
        const int slot = t % RING, buf = t & 1;
        if (!mbar_wait(&sm.ring_full[slot], (t / RING) & 1, abort_flag) ||
            !mbar_wait(&sm.s_free[buf], ((t >> 1) & 1) ^ 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sm.ring[slot]);
        for (int hh = 0; hh < nheads; ++hh) {
          const uint32_t q_addr = smem_u32(sm.q[hh]);
          // pass 1: D[query][key] = Q K^T; pass 2: D[key][query] = K Q^T
          const uint32_t a_addr = PASS == 1 ? q_addr : k_addr;
          const uint32_t b_addr = PASS == 1 ? k_addr : q_addr;
          const uint32_t d = tmem + uint32_t(hh * 256 + buf * 128);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = (kk / 4) * HALF_BYTES + (kk % 4) * 32;
            tc_mma_ss(d, umma_desc_sw128(a_addr + off, 16, 1024),
                      umma_desc_sw128(b_addr + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
          }
        }
        tc_commit(&sm.ring_empty[slot]);
        tc_commit(&sm.s_full[buf]);
      }
      if (!ok) {
        report(status, FP_ERR_TIMEOUT);
        *abort_flag = 1;
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ consumers --
    const int hh = warp / 4;  // head of the pair
    const int r = threadIdx.x % 128;  // TMEM lane: query row (pass 1) / key (pass 2)
    const int wq = warp % 4;
    const uint32_t lane_base = tmem + (uint32_t(wq * 32) << 16) + uint32_t(hh * 256);
    const float sl2 = 1.4426950408889634f / sqrtf(float(HD));
    const bool active = hh < nheads;
    const size_t bh = size_t(b) * hq + h0 + hh;
    float m = -INFINITY, l = 0.f;  // pass 1
    bool ok = true;
    for (int t = 0; t < ntiles; ++t) {
      const int buf = t & 1;
      // a failed wait marks the result invalid but the loop (and its
      // warpgroup barriers) still runs to the end with every warp
      if (ok && !__all_sync(0xffffffffu, mbar_wait(&sm.s_full[buf], (t >> 1) & 1, abort_flag)))
        ok = false;
      if (!active) continue;  // second head slot unused (odd group size)
      float x[BS];
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < BS; c0 += 32) {
          uint32_t u[32];
          tmem_ld32(lane_base + uint32_t(buf * 128 + c0), u);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) x[c0 + i] = __uint_as_float(u[i]);
        }
        tc_fence_before();
        mbar_arrive(&sm.s_free[buf]);
      } else {
#pragma unroll
        for (int c = 0; c < BS; ++c) x[c] = 0.f;
      }
      const int j = j0 + t;
      const bool diag = j == nb - 1;
      if (PASS == 1) {
        // row r of the last block sees key c of the diagonal tile iff c <= r
        if (diag) {
#pragma unroll
          for (int c = 0; c < BS; ++c)
            if (c > r) x[c] = -INFINITY;
        }
        // 8 independent chains for the max and the sum, then trees
        float mx[8], sm8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          mx[k] = x[k];
          sm8[k] = 0.f;
        }
#pragma unroll
        for (int c = 8; c < BS; ++c) mx[c % 8] = fmaxf(mx[c % 8], x[c]);
        const float tmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                 fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
        const float mnew = fmaxf(m, tmax * sl2);
#pragma unroll
        for (int c = 0; c < BS; ++c) sm8[c % 8] += ex2(fmaf(x[c], sl2, -mnew));
        const float s = ((sm8[0] + sm8[1]) + (sm8[2] + sm8[3])) +
                        ((sm8[4] + sm8[5]) + (sm8[6] + sm8[7]));
        l = l * ex2(m - mnew) + s;
        m = mnew;
      } else {
        // key r of the tile, query c of the last block: visible iff r <= c.
        // Diagonal sums (query - key) by register-systolic chains per warp:
        // at step c lane l holds the diagonal c - l and passes it one lane up;
        // lane 31 completes one diagonal per step (bins[c] = diagonal c - 31).
        // Two independent chains, over columns 0..63 (A) and 64..127 (B), run
        // interleaved so that each shuffle's latency hides the other's.  A
        // diagonal c - 31 with c in 64..94 takes its lanes whose column is
        // >= 64 from B and the others from A, whose lane l still holds
        // diagonal 63 - l when A ends: that part is added once after the loop
        // (a fixed order).  The vertical sum of the key runs in 4 chains.
        static_assert(BS == 128, "two 64-column chains");
        float v4[4] = {0.f, 0.f, 0.f, 0.f};
        float lqa[4], lqb[4];
        float acc_a = 0.f, acc_b = 0.f;
        float *bins = sm.bins[hh][wq];
#pragma unroll
        for (int c = 0; c < BS / 2; ++c) {
          const int cb = c + BS / 2;
          if (c % 4 == 0) {
            const float4 la = *reinterpret_cast<const float4 *>(&sm.lse2[hh][c]);
            const float4 lb = *reinterpret_cast<const float4 *>(&sm.lse2[hh][cb]);
            lqa[0] = la.x;
            lqa[1] = la.y;
            lqa[2] = la.z;
            lqa[3] = la.w;
            lqb[0] = lb.x;
            lqb[1] = lb.y;
            lqb[2] = lb.z;
            lqb[3] = lb.w;
          }
          const float pa =
              (c < QLO || (diag && r > c)) ? 0.f : ex2(fmaf(x[c], sl2, -lqa[c % 4]));
          const float pb =
              (cb < QLO || (diag && r > cb)) ? 0.f : ex2(fmaf(x[cb], sl2, -lqb[c % 4]));
          v4[c % 4] += pa;
          v4[c % 4] += pb;
          const float ua = __shfl_up_sync(0xffffffffu, acc_a, 1);
          const float ub = __shfl_up_sync(0xffffffffu, acc_b, 1);
          acc_a = (lane == 0 ? 0.f : ua) + pa;
          acc_b = (lane == 0 ? 0.f : ub) + pb;
          if (lane == 31) {
            bins[c] = acc_a;   // diagonal c - 31 (only columns < 64 reach it)
            bins[cb] = acc_b;  // diagonal cb - 31: its columns >= 64
          }
        }
        __syncwarp();
        if (lane < 31) bins[BS / 2 + 30 - lane] += acc_a;  // diagonal 63 - lane: columns < 64
        if (lane < 31) bins[BS + 30 - lane] = acc_b;        // diagonals 127 - lane
        const float v = (v4[0] + v4[1]) + (v4[2] + v4[3]);
        vert[bh * n_tok + size_t(j) * BS + r] = v;
        // tile mass, fixed order: lanes (xor tree), then warps
        float wsum = v;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
        if (lane == 0) sm.warp_mass[hh][wq] = wsum;
        wg_sync(hh);
        if (r == 0) {
          const float *wm = sm.warp_mass[hh];
          if (QLO == 0) {
            true_last[bh * nb_out + j] = (wm[0] + wm[1] + wm[2] + wm[3]) / float(BS);
          } else {  // block 2j: keys 0-63 (warps 0, 1); block 2j + 1: keys 64-127
            const float rows = float(BS - QLO);
            true_last[bh * nb_out + 2 * j] = (wm[0] + wm[1]) / rows;
            true_last[bh * nb_out + 2 * j + 1] = (wm[2] + wm[3]) / rows;
          }
        }
        // tile diagonal D = query - key in [-127, 127] -> partial index D + 127;
        // warp w holds D = (bin - 31) - 32 w
        float *dst = sp + (bh * nb + j) * size_t(kBins);
        for (int i = r; i < kBins; i += 128) {
          float s2 = 0.f;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int bi = i - 96 + 32 * w;
            if (bi >= 0 && bi < kWarpBins) s2 += sm.bins[hh][w][bi];
          }
          dst[i] = s2;
        }
        wg_sync(hh);  // bins are rewritten by the next tile
      }
    }
    if (!ok && active && r == 0) report(status, FP_ERR_TIMEOUT);
    if (PASS == 1 && active) {
      const size_t o = (bh * n_chunks + chunk) * BS + r;
      pm[o] = m;
      pl[o] = l;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// one thread per (b, h, row): log2-sum-exp over the chunk partials
__global__ void lse2_combine_kernel(const float *__restrict__ pm, const float *__restrict__ pl,
                                    float *__restrict__ lse2, int rows, int n_chunks) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= rows) return;
  const int bh = t / BS, r = t % BS;
  float mx = -INFINITY;
  for (int c = 0; c < n_chunks; ++c) mx = fmaxf(mx, pm[(size_t(bh) * n_chunks + c) * BS + r]);
  float s = 0.f;
  for (int c = 0; c < n_chunks; ++c) {
    const size_t o = (size_t(bh) * n_chunks + c) * BS + r;
    if (pm[o] > -INFINITY) s += pl[o] * ex2(pm[o] - mx);
  }
  lse2[t] = mx + log2f(s);
}

bool encode_rows(CUtensorMap *map, const void *ptr, uint64_t rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult qr;
    void *p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) !=
            cudaSuccess ||
        qr != cudaDriverEntryPointSuccess || !p)
      return false;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  const cuuint64_t dims[2] = {cuuint64_t(HD), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(HD) * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool last_block_tc_supported(const Dims &D) {
  return D.dtype == FP_BF16 && D.d == HD && (D.bs == BS || (D.bs == BS / 2 && D.n % BS == 0));
}

// 128-key tiles of the passes (block size 64 runs two blocks per tile)
int last_block_tc_tiles(const Dims &D) { return D.n / BS; }

size_t last_block_tc_ws_bytes(const Dims &D) {
  Carver c{nullptr, 0};
  const size_t heads = size_t(D.bt) * D.hq;
  const int nt = last_block_tc_tiles(D);
  const int n_chunks = (nt + kChunk - 1) / kChunk;
  c.take<float>(heads * n_chunks * BS);
  c.take<float>(heads * n_chunks * BS);
  c.take<float>(heads * BS);
  c.take<float>(heads * nt * size_t(kBins));
  return c.off + 256;
}

// Writes true_last and vert, and the diagonal partials sp [Bt,Hq,n/128,255]
// of the 128-key tiles (combined into slash by the caller's slash_combine
// step with block size 128).
cudaError_t launch_last_block_tc(const Dims &D, const void *q, const void *k, float *true_last,
                                 float *vert, float **sp_out, void *ws, cudaStream_t st) {
  CUtensorMap mq, mk;
  if (!encode_rows(&mq, q, uint64_t(D.bt) * D.hq * D.n) ||
      !encode_rows(&mk, k, uint64_t(D.bt) * D.hkv * D.n))
    return cudaErrorInvalidValue;
  Carver c{static_cast<char *>(ws), 0};
  const size_t heads = size_t(D.bt) * D.hq;
  const int nt = last_block_tc_tiles(D);
  const int q_lo = BS - D.bs;  // block 64: the last 128 rows minus the first 64
  const int n_chunks = (nt + kChunk - 1) / kChunk;
  float *pm = c.take<float>(heads * n_chunks * BS);
  float *pl = c.take<float>(heads * n_chunks * BS);
  float *lse2 = c.take<float>(heads * BS);
  float *sp = c.take<float>(heads * nt * size_t(kBins));
  *sp_out = sp;
  const dim3 grid(n_chunks, D.hkv * ((D.g + 1) / 2), D.bt);
  int *status = device_status_ptr();
  const int rows = int(heads * BS);
  auto passes = [&](auto pass1, auto pass2) {
    cudaFuncSetAttribute(pass1, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes));
    cudaFuncSetAttribute(pass2, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes));
    pass1<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, D.hq, D.g, D.n, nt, D.nb, n_chunks, pm, pl,
                                              nullptr, nullptr, nullptr, nullptr, status);
    lse2_combine_kernel<<<(rows + 127) / 128, 128, 0, st>>>(pm, pl, lse2, rows, n_chunks);
    pass2<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, D.hq, D.g, D.n, nt, D.nb, n_chunks,
                                              nullptr, nullptr, lse2, vert, true_last, sp,
                                              status);
  };
  if (q_lo == 0)
    passes(last_block_tc_kernel<1, 0>, last_block_tc_kernel<2, 0>);
  else
    passes(last_block_tc_kernel<1, BS / 2>, last_block_tc_kernel<2, BS / 2>);
  return cudaGetLastError();
}

}  // namespace fpi
