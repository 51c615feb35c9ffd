// attn_tc.cu -- bf16 block-sparse causal attention on the sm_100a tensor
// cores (tcgen05 + TMEM + TMA), the hot kernel of fp_sparse_attn and
// fp_dense_attn.
//
// FlexPrefill (atlas.scime.ai summary, "Approach" and "Experimental setup"):
// causal attention over the selected query-key blocks, built on
// FlashAttention's online softmax.  Block size 128, head dim 128.
//
// One CTA handles one (query block, head, batch) item and is small enough
// (112 KB of shared memory, 256 TMEM columns, <= 168 registers per thread)
// that two CTAs share an SM, so one CTA's softmax overlaps the other's MMAs.
// Every listed key block (128 keys) is processed as two 64-key tiles.
// 6 warps, specialised:
//   warps 0-3  softmax + epilogue: thread r owns query row r, which is TMEM
//              lane r (warp w may only touch lanes 32w..32w+31);
//   warp 4     TMA producer (one thread): Q's second half once, then K tiles
//              through a 3-slot ring and V tiles through a 3-slot ring;
//   warp 5     MMA issuer (one thread): S = Q K^T (N = 64) into TMEM and
//              O += P V (K = 64, P from TMEM) into a TMEM accumulator.
// TMEM (256 columns): S [0,64) fp32 | P [64,96) bf16 pairs | Q d 0..63
// [96,128) bf16 pairs | O [128,256) fp32.
// Shared memory (1024-B aligned, 128-B swizzle everywhere):
//   Q d 64..127 16 KB [128 rows x 64 d] | K x3 16 KB | V x3 16 KB
// (112 KB in all, with no room for alignment slack: the kernel requires the
// dynamic shared-memory window to start 1024-B aligned, which it is when the
// kernel declares no static shared memory, and checks it).
// K and V tiles are two 8-KB halves [64 keys x 64 d]; K is the K-major B
// operand of S, V the MN-major B operand of P V.  S takes its first 64 d
// with A = Q from TMEM and the other 64 with A = Q from shared memory.  A K
// slot is refilled as soon as S of its tile has completed, a V slot once P V
// of its tile has.
// Why this split: an MMA of N = 64 whose operands both come from shared memory
// reads A (all of Q) for every 64 keys, 192 B per clock at full rate, more
// than the 128 B per clock shared memory delivers, and the K and V tile writes
// share that bandwidth.  Keeping P and half of Q in TMEM cuts the shared
// memory traffic per tile from 128 KB (Q, K, P, V operand reads, P stores,
// K/V writes) to 80 KB; all of Q plus a second P buffer would not fit in 256
// columns.
//
// Per key tile t the softmax warps read S(t) from TMEM into registers and
// release it (so S(t+1) = Q K(t+1)^T runs during the exponentials), compute
// p = 2^(s*scale*log2e - m) with a running row max m, rescale O in TMEM only
// when m grows by more than 2^8, store P(t) (bf16) once P(t-1) V(t-1) has
// read P(t-1), and signal the MMA warp, which issues P(t) V(t).
//
// Every wait is bounded (2 s); on expiry the kernel records FP_ERR_TIMEOUT,
// raises a CTA-wide abort flag, drains its outstanding TMA loads and frees
// TMEM before returning.
#include <math.h>

#include "fp_internal.cuh"

namespace fpi {
namespace {

constexpr int BM = 128;   // query rows per tile (= block size)
constexpr int BN = 64;    // keys per tile (half a block)
constexpr int HD = 128;   // head dim
constexpr int NK = 3;     // K slots
constexpr int NV = 3;     // V slots
constexpr uint32_t Q_BYTES = BM * HD * 2;   // 32 KB
constexpr uint32_t Q_HALF = Q_BYTES / 2;    // [128 rows x 64 d]
constexpr uint32_t KV_BYTES = BN * HD * 2;  // 16 KB
constexpr uint32_t KV_HALF = KV_BYTES / 2;  // [64 keys x 64 d]
constexpr uint32_t TMEM_COLS = 256;

struct TcSmem {
  uint8_t q[Q_HALF];  // Q, d 64..127 (d 0..63 lives in TMEM)
  uint8_t k[NK][KV_BYTES];
  uint8_t v[NV][KV_BYTES];
  uint64_t bar_q, q_tmem;    // Q's shared-memory half loaded / TMEM half stored
  uint64_t k_full[NK], k_empty[NK], v_full[NV], v_empty[NV];
  uint64_t s_full, s_free;   // S(t) written / read out
  uint64_t p_full, p_empty, o_full;  // P(t) stored / P(t) V(t) done / all done
  uint32_t tmem_base;
  int ntile;  // key tiles of this CTA
  int abort_flag;
};
constexpr size_t kSmemBytes = sizeof(TcSmem);  // no slack: the base is 1024-B aligned
// two CTAs per SM: 228 KB of shared memory, 1 KB of it reserved per CTA
static_assert(2 * (kSmemBytes + 1024) <= 233472, "two CTAs must fit in one SM");
// TMEM columns: S fp32, P bf16 pairs, the first 64 d of Q bf16 pairs, O fp32
constexpr uint32_t S_COL = 0, P_COL = BN, Q0_COL = BN + BN / 2, O_COL = 2 * BN;
static_assert(Q0_COL + HD / 4 <= O_COL && O_COL + HD <= TMEM_COLS, "TMEM layout");

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// The key tiles of one CTA, in order.
//  Block size 128 (PAIR = false): the CTA's 128 query rows are one block qa;
//    tile t is half (t & 1) of listed block list_a[t / 2]: 2 n tiles.
//  Block size 64 (PAIR = true): the 128 rows are blocks qa = 2p and qb = 2p+1
//    (qb may be past the end); the tiles are the blocks of the ascending union
//    of both lists, one 64-key block each; in_a / in_b say whose list holds it.
struct Tile {
  int j;     // key block
  int sub;   // 64-key half of a 128-key block (PAIR = false), else 0
  bool in_a, in_b;
};

template <bool PAIR>
struct Walker {
  const int32_t *la, *lb;
  int na, nb2, ia, ib;
  bool dense;
  int t;
  __device__ Walker(const int32_t *la_, int na_, const int32_t *lb_, int nb_, bool dense_)
      : la(la_), lb(lb_), na(na_), nb2(nb_), ia(0), ib(0), dense(dense_), t(0) {}
  __device__ int entry(const int32_t *l, int i) const { return dense ? i : __ldg(l + i); }
  __device__ Tile next() {
    Tile x;
    if (!PAIR) {
      x.j = entry(la, t / 2);
      x.sub = t & 1;
      x.in_a = true;
      x.in_b = false;
    } else {
      const int ja = ia < na ? entry(la, ia) : 0x7fffffff;
      const int jb = ib < nb2 ? entry(lb, ib) : 0x7fffffff;
      x.j = ja < jb ? ja : jb;
      x.sub = 0;
      x.in_a = ja == x.j;
      x.in_b = jb == x.j;
      ia += x.in_a;
      ib += x.in_b;
    }
    ++t;
    return x;
  }
};

// The maximum of one S row over a 64-key tile (raw scores); MASK: keys
// c > lim are left out.
template <bool MASK>
__device__ __forceinline__ float tile_max(const uint32_t (&u)[BN], int lim) {
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll
  for (int c = 0; c < BN; c += 2) {
    const float y0 = (MASK && c > lim) ? -INFINITY : __uint_as_float(u[c]);
    const float y1 = (MASK && c + 1 > lim) ? -INFINITY : __uint_as_float(u[c + 1]);
    mx[(c / 2) % 8] = max3f(mx[(c / 2) % 8], y0, y1);
  }
  return max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
}

// p = 2^(s * sl2 - muse) for one S row over a 64-key tile, packed to bf16
// pairs, and its sum in 4 two-lane chains; MASK: keys c > lim give 0.
template <bool MASK>
__device__ __forceinline__ void tile_exp(const uint32_t (&u)[BN], int lim, float sl2, float muse,
                                         float2 (&acc)[4], uint32_t (&pk)[BN / 2]) {
  const float2 sc = make_float2(sl2, sl2), nm = make_float2(-muse, -muse);
#pragma unroll
  for (int i = 0; i < BN; i += 2) {
    const float2 x = ffma2(make_float2(__uint_as_float(u[i]), __uint_as_float(u[i + 1])), sc, nm);
    float2 p;
    p.x = ex2(x.x);
    p.y = ex2(x.y);
    if (MASK) {
      p.x = i > lim ? 0.f : p.x;
      p.y = i + 1 > lim ? 0.f : p.y;
    }
    acc[(i / 2) % 4] = fadd2(acc[(i / 2) % 4], p);
    pk[i / 2] = pack_bf16(p.x, p.y);
  }
}

// One S tile of one row (TMEM lane): read out (then released); the
// exponentials are computed against the running max m first, and redone only
// if some row of the warp needs a new max: the max grew by more than 2^8
// (lazy rescale: p <= 256 is exact enough in fp32 and bf16, and the final
// 1/l uses the same stale max, so the result is unchanged), or this is the
// first tile.  The tile max itself is computed only when that may be the
// case (it costs a max per pair of scores, a fifth of the softmax's
// instructions).
template <bool MASK>
__device__ __forceinline__ void softmax_tile(uint32_t s_addr, uint64_t *s_free, bool first,
                                             int lim, float sl2, float m, float &muse,
                                             float &alpha, float2 (&acc)[4],
                                             uint32_t (&pk)[BN / 2], float &ps) {
  uint32_t u[BN];
  tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
  tmem_ld32(s_addr + 32u, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
  tc_wait_ld();
  // S is in registers: the next S may overwrite the TMEM buffer
  tc_fence_before();
  mbar_arrive(s_free);
  if (!first) tile_exp<MASK>(u, lim, sl2, m, acc, pk);
  muse = m;
  // the exact tile max is needed only where the lazy rule may move m: on the
  // first tile, or when some key is more than 8 above m, i.e. some p > 2^8,
  // which a tile sum <= 2^8 rules out (a NaN sum takes the exact path too)
  const float ps0 = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                    ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
  const bool need = first || !(ps0 <= 256.f);
  ps = ps0;
  if (__any_sync(0xffffffffu, need)) {
    const float tmax = tile_max<MASK>(u, lim) * sl2;
    if (need && (tmax > m + 8.0f || m == -INFINITY)) muse = fmaxf(m, tmax);
  }
  if (__any_sync(0xffffffffu, first || muse != m)) {
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
    tile_exp<MASK>(u, lim, sl2, muse, acc, pk);
    ps = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
         ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
  }
  alpha = muse != m ? ex2(m - muse) : 1.f;  // 0 on the first tile
}

template <bool PAIR>
__global__ void __launch_bounds__(192, 2) attn_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __nv_bfloat16 *__restrict__ qg,
    const int32_t *__restrict__ counts, const int32_t *__restrict__ indices,
    __nv_bfloat16 *__restrict__ out,
    float *__restrict__ lse, int hq, int g, int n_tok, int nb, bool dense, int *status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the 128-B swizzled operand tiles need 1024-B alignment and there is no
  // slack to realign: refuse (before touching shared memory) if it is missing
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) report(status, FP_ERR_UNSUPPORTED);
    return;
  }
  TcSmem &sm = *reinterpret_cast<TcSmem *>(smem_raw);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  constexpr int KB = PAIR ? 64 : 128;  // tokens per block

  // the CTA's query blocks (longest rows first)
  const int h = blockIdx.y, b = blockIdx.z, kv = h / g, hkv = hq / g;
  const size_t bh = size_t(b) * hq + h;
  const int qa = PAIR ? 2 * (int(gridDim.x) - 1 - int(blockIdx.x)) : nb - 1 - int(blockIdx.x);
  const int qb = qa + 1;
  const bool has_b = PAIR && qb < nb;
  auto row_count = [&](int qblk) {
    int n = dense ? qblk + 1 : counts[bh * nb + qblk];
    if (n < 0 || n > qblk + 1) {  // a row holds at most qblk + 1 causal blocks
      if (threadIdx.x == 0) report(status, FP_ERR_DEVICE_CHECK);
      n = n < 0 ? 0 : qblk + 1;
    }
    return n;
  };
  const int na = row_count(qa);
  const int nbb = has_b ? row_count(qb) : 0;
  const int32_t *la = indices + (bh * nb + qa) * size_t(nb);
  const int32_t *lb = has_b ? indices + (bh * nb + qb) * size_t(nb) : la;
  const int qlast = has_b ? qb : qa;  // largest valid key block of the CTA

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_q, 1);
    mbar_init(&sm.q_tmem, 128);
    for (int s = 0; s < NK; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.s_free, 128);
    mbar_init(&sm.p_full, 128);
    mbar_init(&sm.p_empty, 1);
    mbar_init(&sm.o_full, 1);
    sm.abort_flag = 0;
    int nt = 2 * na;
    if (PAIR) {  // size of the union of the two lists
      Walker<true> w(la, na, lb, nbb, dense);
      nt = 0;
      while (w.ia < w.na || w.ib < w.nb2) {
        w.next();
        ++nt;
      }
    }
    sm.ntile = nt;
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
  const int ntile = sm.ntile;
  volatile int *abort_flag = &sm.abort_flag;

  auto fail = [&](int code) {
    report(status, code);
    *abort_flag = 1;
  };

  if (warp == 4) {
    // ------------------------------------------------------- TMA producer --
    // Q's second half once, then K(i) and V(i - 2) in turn.  K(i) waits for
    // S(i-3) to finish with its slot, V(i-2) for P(i-5) V(i-5), which was
    // issued before S(i-3) and is covered by its commit: by the time K(i) may
    // load, V(i-2) may too, so the interleaving delays neither.
    if (lane == 0 && ntile > 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const int qrow = int((bh * n_tok) + size_t(qa) * KB);
      mbar_arrive_expect_tx(&sm.bar_q, Q_HALF);
      tma_load_2d(sm.q, &tm_q, &sm.bar_q, 64, qrow);
      const size_t kvrow0 = (size_t(b) * hkv + kv) * n_tok;
      Walker<PAIR> walk_k(la, na, lb, nbb, dense), walk_v(la, na, lb, nbb, dense);
      // first row of key tile x: invalid entries load any in-range block (the
      // softmax masks them)
      auto tile_row = [&](const Tile &x) {
        const int j = x.j < 0 ? 0 : (x.j > qlast ? qlast : x.j);
        return int(kvrow0 + size_t(j) * KB + size_t(x.sub) * BN);
      };
      int issued_k = 0, issued_v = 0;
      for (int i = 0; i < ntile + 2 && !*abort_flag; ++i) {
        if (i < ntile) {
          const int sl = i % NK;
          const int row = tile_row(walk_k.next());
          if (!mbar_wait(&sm.k_empty[sl], ((i / NK) & 1) ^ 1, abort_flag)) {
            fail(FP_ERR_TIMEOUT);
            break;
          }
          mbar_arrive_expect_tx(&sm.k_full[sl], KV_BYTES);
          tma_load_2d(sm.k[sl], &tm_k, &sm.k_full[sl], 0, row);
          tma_load_2d(sm.k[sl] + KV_HALF, &tm_k, &sm.k_full[sl], 64, row);
          issued_k = i + 1;
        }
        if (i >= 2) {
          const int t = i - 2, sl = t % NV;
          const int row = tile_row(walk_v.next());
          if (!mbar_wait(&sm.v_empty[sl], ((t / NV) & 1) ^ 1, abort_flag)) {
            fail(FP_ERR_TIMEOUT);
            break;
          }
          mbar_arrive_expect_tx(&sm.v_full[sl], KV_BYTES);
          tma_load_2d(sm.v[sl], &tm_v, &sm.v_full[sl], 0, row);
          tma_load_2d(sm.v[sl] + KV_HALF, &tm_v, &sm.v_full[sl], 64, row);
          issued_v = t + 1;
        }
      }
      if (*abort_flag) {
        // drain: wait (bounded) for the loads still in flight, the last load
        // of each slot
        volatile int never = 0;
        mbar_wait(&sm.bar_q, 0, &never, 100000000ull);
        for (int t = issued_k - NK > 0 ? issued_k - NK : 0; t < issued_k; ++t)
          mbar_wait(&sm.k_full[t % NK], (t / NK) & 1, &never, 100000000ull);
        for (int t = issued_v - NV > 0 ? issued_v - NV : 0; t < issued_v; ++t)
          mbar_wait(&sm.v_full[t % NV], (t / NV) & 1, &never, 100000000ull);
      }
    }
  } else if (warp == 5) {
    // --------------------------------------------------------- MMA issuer --
    if (lane == 0 && ntile > 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(BM, BN, 0);
      constexpr uint32_t idesc_o = umma_idesc_bf16(BM, HD, 1);
      const uint32_t q_addr = smem_u32(sm.q);
      bool ok = mbar_wait(&sm.bar_q, 0, abort_flag) && mbar_wait(&sm.q_tmem, 0, abort_flag);
      auto issue_pv = [&](int u) -> bool {
        const int sv = u % NV;
        if (!mbar_wait(&sm.p_full, u & 1, abort_flag)) return false;
        if (!mbar_wait(&sm.v_full[sv], (u / NV) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sm.v[sv]);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // A = P(u) [128 lanes x 64 keys] in TMEM: 16 keys = 8 columns;
          // B = V [64 keys x 128 d]: MN-major, 64-d halves KV_HALF apart,
          // 16 keys = 16 rows of 128 B
          const uint64_t bd = umma_desc_sw128(v_addr + kk * 16 * 128, KV_HALF, 1024);
          tc_mma_ts(tmem + O_COL, tmem + P_COL + uint32_t(kk * 8), bd, idesc_o,
                    (u > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&sm.v_empty[sv]);
        tc_commit(&sm.p_empty);
        return true;
      };
      for (int t = 0; ok && t < ntile; ++t) {
        const int s = t % NK;
        // S(t) overwrites S(t-1): the softmax must have read it out
        if (!mbar_wait(&sm.k_full[s], (t / NK) & 1, abort_flag) ||
            !mbar_wait(&sm.s_free, (t & 1) ^ 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sm.k[s]);
        // d 0..63: A = Q from TMEM (16 d = 8 columns), B = K's first half;
        // d 64..127: A = Q's second half in shared memory, B = K's second half
        // (16 d = 32 B inside a 64-d half)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_ts(tmem + S_COL, tmem + Q0_COL + uint32_t(kk * 8),
                    umma_desc_sw128(k_addr + kk * 32, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_ss(tmem + S_COL, umma_desc_sw128(q_addr + kk * 32, 16, 1024),
                    umma_desc_sw128(k_addr + KV_HALF + kk * 32, 16, 1024), idesc_s, 1u);
        tc_commit(&sm.s_full);
        tc_commit(&sm.k_empty[s]);
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
    // rows of this warp: block qa (PAIR: rows 0-63) or qb (PAIR: rows 64-127)
    const int half = PAIR ? r / 64 : 0;
    const int qh = PAIR ? qa + half : qa;
    const int rl = r - 64 * half;  // row inside its block
    // (a partial last block: rows at or past N are not read or written)
    const bool row_exists =
        (!PAIR || half == 0 || has_b) && size_t(qa) * KB + size_t(r) < size_t(n_tok);
    {
      // the first 64 d of this row's query -> TMEM (A operand of Q K^T);
      // 32-bit column c holds d 2c (low half) and 2c + 1
      uint32_t qw[32];
      const uint4 *src = reinterpret_cast<const uint4 *>(qg + (bh * n_tok + size_t(qa) * KB + r) * HD);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 w = row_exists ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
        qw[4 * c] = w.x;
        qw[4 * c + 1] = w.y;
        qw[4 * c + 2] = w.z;
        qw[4 * c + 3] = w.w;
      }
      tmem_st32(lane_base + Q0_COL, qw);
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.q_tmem);
    }
    Walker<PAIR> walk(la, na, lb, nbb, dense);
    Tile x = walk.next();  // prefetched one tile ahead
    for (int t = 0; t < ntile; ++t) {
      const Tile cur = x;
      if (t + 1 < ntile) x = walk.next();
      // waits are made warp-uniform: tcgen05.ld/st below are .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full, t & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool mine = PAIR ? (half ? cur.in_b : cur.in_a) : true;
      const bool inrange = cur.j >= 0 && cur.j <= qh;
      if (mine && !inrange && rl == 0 && cur.sub == 0) report(status, FP_ERR_DEVICE_CHECK);
      const bool valid = mine && inrange;
      // keys c > lim of this 64-key tile are masked: the diagonal block hides
      // keys after the query row (tile keys start at 64 sub); a tile off this
      // row's list, or an invalid entry, hides all; other tiles are unmasked
      const bool masked = !valid || cur.j == qh;
      const int lim = valid ? rl - BN * cur.sub : -1;
      float muse, alpha, ps;
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
      uint32_t pk[BN / 2];
      const uint32_t s_addr = lane_base + S_COL;
      // a row's first tile is its first with a key: until then every p is 0
      // and m stays -inf (alpha 1), so m is taken from the row's own scores
      // however low they are
      const bool first = m == -INFINITY;
      if (masked)
        softmax_tile<true>(s_addr, &sm.s_free, first, lim, sl2, m, muse, alpha, acc, pk, ps);
      else
        softmax_tile<false>(s_addr, &sm.s_free, first, lim, sl2, m, muse, alpha, acc, pk, ps);
      l = l * alpha + ps;
      // P(t) overwrites P(t-1), and O may be rescaled: both need P(t-1) V(t-1)
      // finished (for t = 0 the wait is on the phase before the first and
      // returns at once)
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.p_empty, (t & 1) ^ 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // O is rescaled (rarely: lazy) by the whole warp if any of its rows'
      // max grew
      if (__any_sync(0xffffffffu, t > 0 && alpha != 1.f)) {
#pragma unroll
        for (int c0 = 0; c0 < HD; c0 += 32) {
          uint32_t u[32];
          tmem_ld32(lane_base + O_COL + uint32_t(c0), u);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
          tmem_st32(lane_base + O_COL + uint32_t(c0), u);
        }
      }
      tmem_st32(lane_base + P_COL, pk);
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full);
      m = muse;
    }
    // ------------------------------------------------------------ epilogue --
    const size_t orow = bh * n_tok + size_t(qa) * KB + r;
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
        tmem_ld32(lane_base + O_COL + uint32_t(c0), u);
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
        if (row_exists) dst[(c0 + i) / 8] = w;
      }
    }
    if (lse && row_exists) lse[orow] = good ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
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
  const PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (!fn) return false;
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
  if ((D.bs != 128 && D.bs != 64) || D.d != HD) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv;
  if (!encode_map(&mq, q, uint64_t(D.bt) * D.hq * D.n, BM) ||
      !encode_map(&mk, k, uint64_t(D.bt) * D.hkv * D.n, BN) ||
      !encode_map(&mv, v, uint64_t(D.bt) * D.hkv * D.n, BN))
    return cudaErrorInvalidValue;
  int *status = device_status_ptr();
  __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(out);
  if (D.bs == 128) {
    cudaFuncSetAttribute(attn_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         int(kSmemBytes));
    attn_tc_kernel<false><<<dim3(D.nb, D.hq, D.bt), 192, kSmemBytes, st>>>(
        mq, mk, mv, static_cast<const __nv_bfloat16 *>(q), counts, indices, o, lse, D.hq, D.g,
        D.n, D.nb, dense, status);
  } else {
    cudaFuncSetAttribute(attn_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         int(kSmemBytes));
    attn_tc_kernel<true><<<dim3((D.nb + 1) / 2, D.hq, D.bt), 192, kSmemBytes, st>>>(
        mq, mk, mv, static_cast<const __nv_bfloat16 *>(q), counts, indices, o, lse, D.hq, D.g,
        D.n, D.nb, dense, status);
  }
  return cudaGetLastError();
}

}  // namespace fpi
