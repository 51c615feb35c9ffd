// attn_tc.cu -- bf16 block-sparse causal attention on the sm_100a tensor
// cores (tcgen05 + TMEM + TMA), the hot kernel of fp_sparse_attn and
// fp_dense_attn.
//
// FlexPrefill (atlas.scime.ai summary, "Approach" and "Experimental setup"):
// causal attention over the selected query-key blocks, built on
// FlashAttention's online softmax.  Block size 128, head dim 128.
//
// One CTA handles one (query block, head, batch) item; 6 warps, specialised:
//   warps 0-3  softmax + epilogue: thread r owns query row r, which is TMEM
//              lane r (warp w may only touch lanes 32w..32w+31);
//   warp 4     TMA producer: Q once, then K and V tiles of the listed key
//              blocks through a 2-stage ring;
//   warp 5     MMA issuer (one thread): S = Q K^T into one of two TMEM
//              buffers, O += P V into a TMEM accumulator.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O [256,384).
// Shared memory (1024-B aligned, 128-B swizzle everywhere):
//   Q 32 KB | K x2 32 KB | V x2 32 KB | P 32 KB  (+ barriers)
// Each operand tile is two 16-KB halves [128 rows x 64 elements]; Q, K and
// P are K-major operands, V is the MN-major B operand of P V.
//
// Per key tile t the softmax warps read S(t) from TMEM, release the buffer,
// compute p = 2^(s*scale*log2e - m) with a running row max m, rescale O in
// TMEM only when m grows by more than 2^8, write P(t) (bf16) to shared memory
// and signal the MMA warp, which then issues P(t) V(t) while S(t+1) is
// already in flight.
//
// Every wait is bounded (2 s); on expiry the kernel records FP_ERR_TIMEOUT,
// raises a CTA-wide abort flag, drains its outstanding TMA loads and frees
// TMEM before returning.
#include <math.h>

#include "fp_internal.cuh"

namespace fpi {
namespace {

constexpr int BM = 128;  // query rows per tile (= block size)
constexpr int BN = 128;  // keys per tile (= block size)
constexpr int HD = 128;  // head dim
constexpr int NS = 2;    // K/V pipeline stages
constexpr uint32_t TILE_BYTES = BM * HD * 2;  // 32 KB
constexpr uint32_t HALF_BYTES = TILE_BYTES / 2;

struct TcSmem {
  uint8_t q[TILE_BYTES];
  uint8_t k[NS][TILE_BYTES];
  uint8_t v[NS][TILE_BYTES];
  uint8_t p[TILE_BYTES];
  uint64_t bar_q;
  uint64_t k_full[NS], v_full[NS], kv_empty[NS];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, p_empty, o_full;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kSmemBytes = sizeof(TcSmem) + 1024;  // + alignment slack

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

struct Item {
  int qi, h, b, kv, n;
  size_t bh;
  const int32_t *list;
};

__device__ __forceinline__ int list_block(const Item &it, int t, bool dense) {
  return dense ? t : __ldg(it.list + t);
}

// One S tile of one row (TMEM lane): the row max over the tile (read once,
// 8 independent chains), the lazy-rescale decision, then the exponentials
// (S read again 32 columns at a time, so few scores are live), packed to bf16
// pairs, with the row sum in 8 chains.  MASK: keys c > lim contribute 0.
template <bool MASK>
__device__ __forceinline__ void softmax_tile(uint32_t s_addr, int lim, float sl2, float m,
                                             float &muse, float &alpha, float (&sm8)[8],
                                             uint32_t (&pk)[BN / 2]) {
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
  {
    // all four 32-column loads in flight, one wait
    uint32_t u[BN];
#pragma unroll
    for (int c0 = 0; c0 < BN; c0 += 32)
      tmem_ld32(s_addr + uint32_t(c0), *reinterpret_cast<uint32_t(*)[32]>(&u[c0]));
    tc_wait_ld();
#pragma unroll
    for (int c = 0; c < BN; ++c) {
      const float y = (MASK && c > lim) ? -INFINITY : __uint_as_float(u[c]);
      mx[c % 8] = fmaxf(mx[c % 8], y);
    }
  }
  const float tmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                           fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * sl2;
  // lazy rescale: keep the old max unless the row max grew by more than 2^8
  // (p <= 256 is exact enough in fp32 and bf16; the final 1/l uses the same
  // stale max, so the result is unchanged)
  muse = m;
  if (tmax > m + 8.0f || m == -INFINITY) muse = fmaxf(m, tmax);
  if (muse == -INFINITY) muse = 0.f;  // every key so far masked
  alpha = ex2(m - muse);              // 1 when unchanged, 0 on the first tile
#pragma unroll
  for (int c0 = 0; c0 < BN; c0 += 64) {
    // two 32-column loads in flight, one wait
    uint32_t u[64];
    tmem_ld32(s_addr + uint32_t(c0), *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
    tmem_ld32(s_addr + uint32_t(c0 + 32), *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
    tc_wait_ld();
#pragma unroll
    for (int i = 0; i < 64; i += 2) {
      float p0 = ex2(fmaf(__uint_as_float(u[i]), sl2, -muse));
      float p1 = ex2(fmaf(__uint_as_float(u[i + 1]), sl2, -muse));
      if (MASK) {
        p0 = c0 + i > lim ? 0.f : p0;
        p1 = c0 + i + 1 > lim ? 0.f : p1;
      }
      sm8[i % 8] += p0;
      sm8[(i + 1) % 8] += p1;
      pk[(c0 + i) / 2] = pack_bf16(p0, p1);
    }
  }
}

__global__ void __launch_bounds__(192, 1) attn_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const int32_t *__restrict__ counts,
    const int32_t *__restrict__ indices, __nv_bfloat16 *__restrict__ out,
    float *__restrict__ lse, int hq, int g, int n_tok, bool dense, int *status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  TcSmem &sm = *reinterpret_cast<TcSmem *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nb = gridDim.x;

  Item it;
  it.qi = nb - 1 - blockIdx.x;  // longest rows first
  it.h = blockIdx.y;
  it.b = blockIdx.z;
  it.kv = it.h / g;
  it.bh = size_t(it.b) * hq + it.h;
  it.n = dense ? it.qi + 1 : counts[it.bh * nb + it.qi];
  if (it.n < 0 || it.n > it.qi + 1) {  // a row holds at most qi + 1 causal blocks
    if (threadIdx.x == 0) report(status, FP_ERR_DEVICE_CHECK);
    it.n = it.n < 0 ? 0 : it.qi + 1;
  }
  it.list = indices + (it.bh * nb + it.qi) * size_t(nb);
  const int hkv = hq / g;

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_q, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.s_free[s], 128);
    }
    mbar_init(&sm.p_full, 128);
    mbar_init(&sm.p_empty, 1);
    mbar_init(&sm.o_full, 1);
    sm.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 5) {
    tmem_alloc(&sm.tmem_base, 512);
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

  if (warp == 4) {
    // ------------------------------------------------------- TMA producer --
    if (lane == 0 && it.n > 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const int qrow = int((it.bh * n_tok) + size_t(it.qi) * BM);
      mbar_arrive_expect_tx(&sm.bar_q, TILE_BYTES);
      tma_load_2d(sm.q, &tm_q, &sm.bar_q, 0, qrow);
      tma_load_2d(sm.q + HALF_BYTES, &tm_q, &sm.bar_q, 64, qrow);
      const size_t kvrow0 = (size_t(it.b) * hkv + it.kv) * n_tok;
      int issued = 0;
      for (int t = 0; t < it.n; ++t) {
        const int s = t % NS;
        if (!mbar_wait(&sm.kv_empty[s], ((t / NS) & 1) ^ 1, abort_flag)) {
          fail(FP_ERR_TIMEOUT);
          break;
        }
        int j = list_block(it, t, dense);
        j = j < 0 ? 0 : (j > it.qi ? it.qi : j);  // invalid entries are masked by softmax
        const int krow = int(kvrow0 + size_t(j) * BN);
        mbar_arrive_expect_tx(&sm.k_full[s], TILE_BYTES);
        tma_load_2d(sm.k[s], &tm_k, &sm.k_full[s], 0, krow);
        tma_load_2d(sm.k[s] + HALF_BYTES, &tm_k, &sm.k_full[s], 64, krow);
        mbar_arrive_expect_tx(&sm.v_full[s], TILE_BYTES);
        tma_load_2d(sm.v[s], &tm_v, &sm.v_full[s], 0, krow);
        tma_load_2d(sm.v[s] + HALF_BYTES, &tm_v, &sm.v_full[s], 64, krow);
        issued = t + 1;
      }
      if (*abort_flag) {
        // drain: wait (bounded) for the loads still in flight
        mbar_wait(&sm.bar_q, 0, abort_flag, 100000000ull);
        for (int t = issued - NS > 0 ? issued - NS : 0; t < issued; ++t) {
          const int s = t % NS;
          volatile int never = 0;
          mbar_wait(&sm.k_full[s], (t / NS) & 1, &never, 100000000ull);
          mbar_wait(&sm.v_full[s], (t / NS) & 1, &never, 100000000ull);
        }
      }
    }
  } else if (warp == 5) {
    // --------------------------------------------------------- MMA issuer --
    if (lane == 0 && it.n > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(BM, BN, 0);
      constexpr uint32_t idesc_o = umma_idesc_bf16(BM, HD, 1);
      const uint32_t q_addr = smem_u32(sm.q);
      const uint32_t p_addr = smem_u32(sm.p);
      bool ok = mbar_wait(&sm.bar_q, 0, abort_flag);
      auto issue_pv = [&](int u) -> bool {
        const int s = u % NS;
        if (!mbar_wait(&sm.p_full, u & 1, abort_flag)) return false;
        if (!mbar_wait(&sm.v_full[s], (u / NS) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sm.v[s]);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // A = P: K-major, 16 keys = 32 B step inside a 64-key half
          const uint64_t ad = umma_desc_sw128(p_addr + (kk / 4) * HALF_BYTES + (kk % 4) * 32,
                                              16, 1024);
          // B = V: MN-major, 16 keys = 16 rows of 128 B
          const uint64_t bd = umma_desc_sw128(v_addr + kk * 16 * 128, HALF_BYTES, 1024);
          tc_mma_ss(tmem + 256, ad, bd, idesc_o, (u > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&sm.kv_empty[s]);
        tc_commit(&sm.p_empty);
        return true;
      };
      for (int t = 0; ok && t < it.n; ++t) {
        const int s = t % NS, sb = t & 1;
        if (!mbar_wait(&sm.k_full[s], (t / NS) & 1, abort_flag) ||
            !mbar_wait(&sm.s_free[sb], ((t >> 1) & 1) ^ 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sm.k[s]);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk / 4) * HALF_BYTES + (kk % 4) * 32;
          const uint64_t ad = umma_desc_sw128(q_addr + off, 16, 1024);
          const uint64_t bd = umma_desc_sw128(k_addr + off, 16, 1024);
          tc_mma_ss(tmem + uint32_t(sb * BN), ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(&sm.s_full[sb]);
        if (t >= 1 && !issue_pv(t - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && !issue_pv(it.n - 1)) ok = false;
      if (ok) tc_commit(&sm.o_full);
      if (!ok) fail(FP_ERR_TIMEOUT);
    }
  } else {
    // ------------------------------------------------ softmax (warps 0-3) --
    const int r = threadIdx.x;  // query row in the tile, TMEM lane
    const uint32_t lane_base = tmem + (uint32_t(warp * 32) << 16);
    const float sl2 = 1.4426950408889634f / sqrtf(float(HD));  // scale * log2(e)
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < it.n; ++t) {
      const int sb = t & 1;
      // waits are made warp-uniform: tcgen05.ld/st below are .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[sb], (t >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int j = list_block(it, t, dense);
      const bool valid = j >= 0 && j <= it.qi;
      if (!valid && r == 0) report(status, FP_ERR_DEVICE_CHECK);
      // keys c > lim are masked: the diagonal block hides keys after the query
      // row, an invalid entry hides all; other tiles take the unmasked path
      const bool masked = !valid || j == it.qi;
      const int lim = valid ? r : -1;
      const uint32_t s_addr = lane_base + uint32_t(sb * BN);
      float muse, alpha;
      float sm8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      uint32_t pk[BN / 2];
      if (masked)
        softmax_tile<true>(s_addr, lim, sl2, m, muse, alpha, sm8, pk);
      else
        softmax_tile<false>(s_addr, lim, sl2, m, muse, alpha, sm8, pk);
      tc_fence_before();
      mbar_arrive(&sm.s_free[sb]);
      const float ps = ((sm8[0] + sm8[1]) + (sm8[2] + sm8[3])) +
                       ((sm8[4] + sm8[5]) + (sm8[6] + sm8[7]));
      l = l * alpha + ps;
      // wait until P(t-1) V(t-1) finished: P buffer free, O up to date
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.p_empty, (t & 1) ^ 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // the whole warp rescales if any of its rows' max grew (alpha == 1 for
      // the others)
      if (__any_sync(0xffffffffu, t > 0 && alpha != 1.f)) {
#pragma unroll
        for (int c0 = 0; c0 < HD; c0 += 32) {
          uint32_t u[32];
          tmem_ld32(lane_base + uint32_t(256 + c0), u);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
          tmem_st32(lane_base + uint32_t(256 + c0), u);
        }
        tc_wait_st();
      }
      // P row -> shared memory, K-major SW128: half = key/64, 16-B chunk
      // (8 keys) c stored at chunk c ^ (row % 8)
#pragma unroll
      for (int ch = 0; ch < BN / 8; ++ch) {
        const uint4 w = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        const int half = ch / 8, c = ch % 8;
        uint8_t *dst = sm.p + half * HALF_BYTES + r * 128 + ((c ^ (r & 7)) * 16);
        *reinterpret_cast<uint4 *>(dst) = w;
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&sm.p_full);
      m = muse;
    }
    // ------------------------------------------------------------ epilogue --
    const size_t orow = it.bh * n_tok + size_t(it.qi) * BM + r;
    if (ok && it.n > 0 && !__all_sync(0xffffffffu, mbar_wait(&sm.o_full, 0, abort_flag)))
      ok = false;
    if (!ok) fail(FP_ERR_TIMEOUT);
    tc_fence_after();
    const float inv = (ok && l > 0.f) ? 1.f / l : 0.f;
    uint4 *dst = reinterpret_cast<uint4 *>(out + orow * HD);
#pragma unroll
    for (int c0 = 0; c0 < HD; c0 += 32) {
      uint32_t u[32];
      if (ok && it.n > 0) {
        tmem_ld32(lane_base + uint32_t(256 + c0), u);
        tc_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) u[i] = 0u;
      }
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        uint4 w;
        w.x = pack_bf16(__uint_as_float(u[i + 0]) * inv, __uint_as_float(u[i + 1]) * inv);
        w.y = pack_bf16(__uint_as_float(u[i + 2]) * inv, __uint_as_float(u[i + 3]) * inv);
        w.z = pack_bf16(__uint_as_float(u[i + 4]) * inv, __uint_as_float(u[i + 5]) * inv);
        w.w = pack_bf16(__uint_as_float(u[i + 6]) * inv, __uint_as_float(u[i + 7]) * inv);
        dst[(c0 + i) / 8] = w;
      }
    }
    if (lse)
      lse[orow] = (ok && l > 0.f) ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

bool encode_map(CUtensorMap *map, const void *ptr, uint64_t rows) {
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

size_t attn_ws_bytes(const Dims &) { return 0; }

cudaError_t launch_attn_bf16(const Dims &D, const void *q, const void *k, const void *v,
                             const int32_t *counts, const int32_t *indices, void *out,
                             float *lse, bool dense, void *, cudaStream_t st) {
  if (D.bs != BM || D.d != HD) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv;
  if (!encode_map(&mq, q, uint64_t(D.bt) * D.hq * D.n) ||
      !encode_map(&mk, k, uint64_t(D.bt) * D.hkv * D.n) ||
      !encode_map(&mv, v, uint64_t(D.bt) * D.hkv * D.n))
    return cudaErrorInvalidValue;
  cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       int(kSmemBytes));
  attn_tc_kernel<<<dim3(D.nb, D.hq, D.bt), 192, kSmemBytes, st>>>(
      mq, mk, mv, counts, indices, static_cast<__nv_bfloat16 *>(out), lse, D.hq, D.g, D.n,
      dense, device_status_ptr());
  return cudaGetLastError();
}

}  // namespace fpi
