// attn_tc.cu -- bf16 block-sparse causal attention on the sm_100a tensor
// cores (tcgen05 + TMEM + TMA), the hot kernel of fp_sparse_attn and
// fp_dense_attn.
//
// FlexPrefill (atlas.scime.ai summary, "Approach" and "Experimental setup"):
// causal attention over the selected query-key blocks, built on
// FlashAttention's online softmax.  Block size 128, head dim 128.
//
// One CTA handles one (query block, head, batch) item and is small enough
// (96 KB of shared memory, 256 TMEM columns, <= 168 registers per thread)
// that two CTAs share an SM, so one CTA's softmax overlaps the other's MMAs.
// Every listed key block (128 keys) is processed as two 64-key tiles.
// 6 warps, specialised:
//   warps 0-3  softmax + epilogue: thread r owns query row r, which is TMEM
//              lane r (warp w may only touch lanes 32w..32w+31);
//   warp 4     TMA producer: Q once, then K and V tiles through a 2-stage ring;
//   warp 5     MMA issuer (one thread): S = Q K^T (N = 64) into one of two
//              TMEM buffers, O += P V (K = 64) into a TMEM accumulator.
// TMEM (256 columns): S0 [0,64), S1 [64,128), O [128,256).
// Shared memory (1024-B aligned, 128-B swizzle everywhere):
//   Q 32 KB (two halves [128 rows x 64 d]) | K x2 16 KB | V x2 16 KB
// K and V tiles are two 8-KB halves [64 keys x 64 d]; Q and K are K-major
// operands of S, V is the MN-major B operand of P V.  P(t) ([128 rows x 64
// keys], 16 KB, K-major) is written into the shared-memory slot of K(t),
// which S(t) no longer needs: the producer refills that slot only after
// P(t) V(t) has completed.
//
// Per key tile t the softmax warps read S(t) from TMEM, release the buffer,
// compute p = 2^(s*scale*log2e - m) with a running row max m, rescale O in
// TMEM only when m grows by more than 2^8, write P(t) (bf16) and signal the
// MMA warp, which then issues P(t) V(t) while S(t+1) is already in flight.
//
// Every wait is bounded (2 s); on expiry the kernel records FP_ERR_TIMEOUT,
// raises a CTA-wide abort flag, drains its outstanding TMA loads and frees
// TMEM before returning.
#include <math.h>

#include "fp_internal.cuh"

namespace fpi {
namespace {

constexpr int BM = 128;   // query rows per tile (= block size)
constexpr int BLK = 128;  // keys per listed block
constexpr int BN = 64;    // keys per tile (half a block)
constexpr int HD = 128;   // head dim
constexpr int NS = 2;     // K/V pipeline stages
constexpr uint32_t Q_BYTES = BM * HD * 2;   // 32 KB
constexpr uint32_t Q_HALF = Q_BYTES / 2;    // [128 rows x 64 d]
constexpr uint32_t KV_BYTES = BN * HD * 2;  // 16 KB
constexpr uint32_t KV_HALF = KV_BYTES / 2;  // [64 keys x 64 d]
constexpr uint32_t TMEM_COLS = 256;

struct TcSmem {
  uint8_t q[Q_BYTES];
  uint8_t k[NS][KV_BYTES];  // K(t), then P(t)
  uint8_t v[NS][KV_BYTES];
  uint64_t bar_q;
  uint64_t k_full[NS], v_full[NS], kv_empty[NS];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, p_empty, o_full;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kSmemBytes = sizeof(TcSmem) + 1024;  // + alignment slack
static_assert(2 * (kSmemBytes + 1024) <= 233472, "two CTAs must fit in one SM");
static_assert(BM * BN * 2 == KV_BYTES, "P(t) must fit the K(t) slot");

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
  int qi, h, b, kv, n;  // n = listed blocks; 2n tiles
  size_t bh;
  const int32_t *list;
};

__device__ __forceinline__ int list_block(const Item &it, int t, bool dense) {
  return dense ? t : __ldg(it.list + t);
}

// One S tile (64 keys) of one row (TMEM lane): the row max over the tile,
// the lazy-rescale decision, then the exponentials packed to bf16 pairs,
// with the row sum in 8 chains.  MASK: keys c > lim contribute 0.
template <bool MASK>
__device__ __forceinline__ void softmax_tile(uint32_t s_addr, int lim, float sl2, float m,
                                             float &muse, float &alpha, float (&sm8)[8],
                                             uint32_t (&pk)[BN / 2]) {
  uint32_t u[BN];
  tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
  tmem_ld32(s_addr + 32u, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
  tc_wait_ld();
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll
  for (int c = 0; c < BN; ++c) {
    const float y = (MASK && c > lim) ? -INFINITY : __uint_as_float(u[c]);
    mx[c % 8] = fmaxf(mx[c % 8], y);
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
  for (int i = 0; i < BN; i += 2) {
    float p0 = ex2(fmaf(__uint_as_float(u[i]), sl2, -muse));
    float p1 = ex2(fmaf(__uint_as_float(u[i + 1]), sl2, -muse));
    if (MASK) {
      p0 = i > lim ? 0.f : p0;
      p1 = i + 1 > lim ? 0.f : p1;
    }
    sm8[i % 8] += p0;
    sm8[(i + 1) % 8] += p1;
    pk[i / 2] = pack_bf16(p0, p1);
  }
}

__global__ void __launch_bounds__(192, 2) attn_tc_kernel(
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
  const int ntile = 2 * it.n;  // tile t: half (t & 1) of listed block t / 2

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

  if (warp == 4) {
    // ------------------------------------------------------- TMA producer --
    if (lane == 0 && ntile > 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const int qrow = int((it.bh * n_tok) + size_t(it.qi) * BM);
      mbar_arrive_expect_tx(&sm.bar_q, Q_BYTES);
      tma_load_2d(sm.q, &tm_q, &sm.bar_q, 0, qrow);
      tma_load_2d(sm.q + Q_HALF, &tm_q, &sm.bar_q, 64, qrow);
      const size_t kvrow0 = (size_t(it.b) * hkv + it.kv) * n_tok;
      int issued = 0;
      for (int t = 0; t < ntile; ++t) {
        const int s = t % NS;
        if (!mbar_wait(&sm.kv_empty[s], ((t / NS) & 1) ^ 1, abort_flag)) {
          fail(FP_ERR_TIMEOUT);
          break;
        }
        int j = list_block(it, t / 2, dense);
        j = j < 0 ? 0 : (j > it.qi ? it.qi : j);  // invalid entries are masked by softmax
        const int krow = int(kvrow0 + size_t(j) * BLK + size_t(t & 1) * BN);
        mbar_arrive_expect_tx(&sm.k_full[s], KV_BYTES);
        tma_load_2d(sm.k[s], &tm_k, &sm.k_full[s], 0, krow);
        tma_load_2d(sm.k[s] + KV_HALF, &tm_k, &sm.k_full[s], 64, krow);
        mbar_arrive_expect_tx(&sm.v_full[s], KV_BYTES);
        tma_load_2d(sm.v[s], &tm_v, &sm.v_full[s], 0, krow);
        tma_load_2d(sm.v[s] + KV_HALF, &tm_v, &sm.v_full[s], 64, krow);
        issued = t + 1;
      }
      if (*abort_flag) {
        // drain: wait (bounded) for the loads still in flight
        volatile int never = 0;
        mbar_wait(&sm.bar_q, 0, &never, 100000000ull);
        for (int t = issued - NS > 0 ? issued - NS : 0; t < issued; ++t) {
          const int s = t % NS;
          mbar_wait(&sm.k_full[s], (t / NS) & 1, &never, 100000000ull);
          mbar_wait(&sm.v_full[s], (t / NS) & 1, &never, 100000000ull);
        }
      }
    }
  } else if (warp == 5) {
    // --------------------------------------------------------- MMA issuer --
    if (lane == 0 && ntile > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(BM, BN, 0);
      constexpr uint32_t idesc_o = umma_idesc_bf16(BM, HD, 1);
      const uint32_t q_addr = smem_u32(sm.q);
      bool ok = mbar_wait(&sm.bar_q, 0, abort_flag);
      auto issue_pv = [&](int u) -> bool {
        const int s = u % NS;
        if (!mbar_wait(&sm.p_full, u & 1, abort_flag)) return false;
        if (!mbar_wait(&sm.v_full[s], (u / NS) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t p_addr = smem_u32(sm.k[s]);  // P(u) sits in K(u)'s slot
        const uint32_t v_addr = smem_u32(sm.v[s]);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // A = P [128 rows x 64 keys]: K-major, 16 keys = 32 B along a row
          const uint64_t ad = umma_desc_sw128(p_addr + kk * 32, 16, 1024);
          // B = V [64 keys x 128 d]: MN-major, 64-d halves KV_HALF apart,
          // 16 keys = 16 rows of 128 B
          const uint64_t bd = umma_desc_sw128(v_addr + kk * 16 * 128, KV_HALF, 1024);
          tc_mma_ss(tmem + 2 * BN, ad, bd, idesc_o, (u > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&sm.kv_empty[s]);
        tc_commit(&sm.p_empty);
        return true;
      };
      for (int t = 0; ok && t < ntile; ++t) {
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
          // 16 d = 32 B inside a 64-d half; Q halves Q_HALF apart, K halves KV_HALF
          const uint64_t ad =
              umma_desc_sw128(q_addr + (kk / 4) * Q_HALF + (kk % 4) * 32, 16, 1024);
          const uint64_t bd =
              umma_desc_sw128(k_addr + (kk / 4) * KV_HALF + (kk % 4) * 32, 16, 1024);
          tc_mma_ss(tmem + uint32_t(sb * BN), ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(&sm.s_full[sb]);
        if (t >= 1 && !issue_pv(t - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && !issue_pv(ntile - 1)) ok = false;
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
    for (int t = 0; t < ntile; ++t) {
      const int sb = t & 1, s = t % NS;
      // waits are made warp-uniform: tcgen05.ld/st below are .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[sb], (t >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int j = list_block(it, t / 2, dense);
      const bool valid = j >= 0 && j <= it.qi;
      if (!valid && r == 0 && (t & 1) == 0) report(status, FP_ERR_DEVICE_CHECK);
      // keys c > lim of this tile are masked: in the diagonal block the tile
      // holds keys 64 (t & 1) + c, hidden after the query row; an invalid
      // entry hides all; other tiles take the unmasked path
      const bool masked = !valid || j == it.qi;
      const int lim = valid ? r - BN * (t & 1) : -1;
      float muse, alpha;
      float sm8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      uint32_t pk[BN / 2];
      const uint32_t s_addr = lane_base + uint32_t(sb * BN);
      if (masked)
        softmax_tile<true>(s_addr, lim, sl2, m, muse, alpha, sm8, pk);
      else
        softmax_tile<false>(s_addr, lim, sl2, m, muse, alpha, sm8, pk);
      tc_fence_before();
      mbar_arrive(&sm.s_free[sb]);
      const float ps = ((sm8[0] + sm8[1]) + (sm8[2] + sm8[3])) +
                       ((sm8[4] + sm8[5]) + (sm8[6] + sm8[7]));
      l = l * alpha + ps;
      // wait until P(t-1) V(t-1) finished: O is up to date.  The slot P(t)
      // goes to held K(t), which S(t) (waited for above) has read.
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
          tmem_ld32(lane_base + uint32_t(2 * BN + c0), u);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
          tmem_st32(lane_base + uint32_t(2 * BN + c0), u);
        }
        tc_wait_st();
      }
      // P row -> the K(t) slot, K-major SW128 [128 rows x 64 keys]: 16-B chunk
      // (8 keys) c of row r stored at chunk c ^ (r % 8)
#pragma unroll
      for (int c = 0; c < BN / 8; ++c) {
        const uint4 w = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4 *>(sm.k[s] + r * 128 + ((c ^ (r & 7)) * 16)) = w;
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&sm.p_full);
      m = muse;
    }
    // ------------------------------------------------------------ epilogue --
    const size_t orow = it.bh * n_tok + size_t(it.qi) * BM + r;
    if (ok && ntile > 0 && !__all_sync(0xffffffffu, mbar_wait(&sm.o_full, 0, abort_flag)))
      ok = false;
    if (!ok) fail(FP_ERR_TIMEOUT);
    tc_fence_after();
    const bool good = ok && ntile > 0 && l > 0.f;
    const float inv = good ? 1.f / l : 0.f;
    uint4 *dst = reinterpret_cast<uint4 *>(out + orow * HD);
#pragma unroll
    for (int c0 = 0; c0 < HD; c0 += 32) {
      uint32_t u[32];
      if (ok && ntile > 0) {
        tmem_ld32(lane_base + uint32_t(2 * BN + c0), u);
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
    if (lse) lse[orow] = good ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// 2-D bf16 tensor map over [rows x 128] with a box of [box_rows x 64].
bool encode_map(CUtensorMap *map, const void *ptr, uint64_t rows, uint32_t box_rows) {
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
  const cuuint32_t box[2] = {64, box_rows};
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
  if (D.bs != BLK || D.d != HD) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv;
  if (!encode_map(&mq, q, uint64_t(D.bt) * D.hq * D.n, BM) ||
      !encode_map(&mk, k, uint64_t(D.bt) * D.hkv * D.n, BN) ||
      !encode_map(&mv, v, uint64_t(D.bt) * D.hkv * D.n, BN))
    return cudaErrorInvalidValue;
  cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       int(kSmemBytes));
  attn_tc_kernel<<<dim3(D.nb, D.hq, D.bt), 192, kSmemBytes, st>>>(
      mq, mk, mv, counts, indices, static_cast<__nv_bfloat16 *>(out), lse, D.hq, D.g, D.n,
      dense, device_status_ptr());
  return cudaGetLastError();
}

}  // namespace fpi
