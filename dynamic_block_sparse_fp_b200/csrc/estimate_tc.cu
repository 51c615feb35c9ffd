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
//   per row over its chunk of key tiles and writes one partial per row, and
//   for every tile the row's running max and the sums over the tile's two
//   64-key halves against it.
// Combine: partials -> log-sum-exp of every last-block row (log2 units); the
//   tile partials scaled by 2^(max - lse) and summed over the rows give the
//   pooled true distribution (no second pass needed for it).
// Pass 2 (line sums): S^T = K Q_last^T per key tile, thread = key (= TMEM
//   lane), so P = 2^(S^T*scale*log2e - lse2[query]) is summed per thread into
//   the vertical score of its key; diagonal (query - key) sums of the tile
//   are formed by a register-systolic shuffle within each warp and combined
//   across warps in a fixed order, giving the slash partials of the tile.
//   Only vertical-slash heads read the line sums, so the whole-path call runs
//   this pass for those heads alone (after the pattern test).
// Every reduction has a fixed order, so results are reproducible.
//
// CTA: one kv head, a pair of its query heads (A, B), a chunk of key tiles.
// 12 warps: 0-3 consumer of head A, 4-7 consumer of head B, 8 TMA producer
// (Q_last of both heads, K tiles through a 3-entry ring), 9 MMA issuer,
// 10-11 pass 1 of a kv head's first pair: the block means of K (kbar and its
// tf32 halves) from the key tiles already in the ring, so K is not streamed
// a second time for its pooling; otherwise idle (registers are granted per
// warpgroup).  TMEM 512 columns: S double-buffered per head, head A [0,256),
// head B [256,512).
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

// nb counts 128-key tiles; the query rows are the 128 from q0 = (nb - 1) 128.
// Block size 64 (QLO = 64) runs the same tiles: the queries are the last 128
// rows with the first QLO left out of every sum, and each tile holds two
// output blocks.  RAG (block 128, N not a multiple of 128): only the first
// qrows = N - q0 query rows are the last block's, and keys at or past N (in
// the last tile) are hidden from them by the causal mask.  QLO and RAG are
// template parameters so that the common case carries no extra compare per
// element.  ptile [Bt,Hq,nb,3,128] (pass 1): per tile and row the running max
// and the two halves' sums.
template <int PASS, int QLO, bool RAG>
__global__ void __launch_bounds__(kThreads, 1) last_block_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    int hq, int g, int n_tok, int nb, int q0, int qrows, int n_chunks, float *__restrict__ pm,
    float *__restrict__ pl, float *__restrict__ ptile, const float *__restrict__ lse2g,
    float *__restrict__ vert, float *__restrict__ sp, const int32_t *__restrict__ vs_only,
    float *__restrict__ kbar, float *__restrict__ kbar_hi, float *__restrict__ kbar_lo,
    int *status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  EstSmem &sm = *reinterpret_cast<EstSmem *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int hkv = hq / g;
  const int pairs = (g + 1) / 2;
  const int chunk = blockIdx.x;
  const int kv = blockIdx.y / pairs, pair = blockIdx.y % pairs, b = blockIdx.z;
  // the pair's query heads, or (pass 2 with vs_only) those of them whose
  // pattern is vertical-slash; a CTA left with none returns at once
  int hs[2] = {0, 0};
  int nheads = 0;
  for (int hh = 0; hh < 2; ++hh) {
    const int h = kv * g + 2 * pair + hh;
    if (2 * pair + hh < g && (!vs_only || vs_only[size_t(b) * hq + h] == FP_PATTERN_VS))
      hs[nheads++] = h;
  }
  if (nheads == 0) return;
  const int j0 = chunk * kChunk;
  const int j1 = min(nb, j0 + kChunk);
  const int ntiles = j1 - j0;
  // pass 1 of the first pair of a kv head also pools the kv head's keys
  const bool pool = PASS == 1 && kbar != nullptr && pair == 0;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int r = 0; r < RING; ++r) {
      mbar_init(&sm.ring_full[r], 1);
      // freed by the MMAs' commit, and by both pooling warps when they pool
      mbar_init(&sm.ring_empty[r], pool ? 3 : 1);
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
    sm.lse2[hh][r] = hh < nheads ? lse2g[(size_t(b) * hq + hs[hh]) * BS + r] : 0.f;
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
        const int qrow = int((size_t(b) * hq + hs[hh]) * n_tok + q0);
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
  } else if (warp >= 10) {
    // ------------------------------------------- K block means (pass 1) --
    // thread p (0..63) takes d = 2p, 2p+1: one 32-bit word per key row of
    // the 128-B swizzled tile half p / 32; the rows of a block are summed in
    // order in fp32, and the mean written with its tf32 halves.
    if (pool) {
      const int p = threadIdx.x - 320;
      // word p % 32 of the 128-B rows of tile half p / 32; its 16-B chunk sits
      // at chunk ^ (row % 8) under the 128-B swizzle
      const uint32_t half_off = uint32_t(p / 32) * HALF_BYTES;
      const int wchunk = (p % 32) / 4, wbyte = (p % 4) * 4;
      constexpr int kBpt = QLO ? 2 : 1;        // blocks per 128-key tile
      constexpr int kBrows = BS / kBpt;        // rows of a block
      const int nbk = (n_tok + kBrows - 1) / kBrows;  // blocks of the sequence
      const size_t kv0 = (size_t(b) * hkv + kv) * nbk;
      for (int t = 0; t < ntiles; ++t) {
        const int slot = t % RING;
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.ring_full[slot], (t / RING) & 1, abort_flag))) {
          if (lane == 0) {
            report(status, FP_ERR_TIMEOUT);
            *abort_flag = 1;
          }
          break;
        }
        const uint32_t base = smem_u32(sm.ring[slot]) + half_off + uint32_t(wbyte);
        const int j = j0 + t;
        const int krows = min(BS, n_tok - j * BS);  // keys of the tile (a partial last tile)
#pragma unroll
        for (int blk = 0; blk < kBpt; ++blk) {
          const int r0 = blk * kBrows, r1 = min(krows, r0 + kBrows);
          if (r1 <= r0) continue;
          float s0 = 0.f, s1 = 0.f;  // d = 2p, 2p + 1
          for (int r = r0; r < r1; ++r) {
            uint32_t w;
            asm volatile("ld.shared.b32 %0, [%1];"
                         : "=r"(w)
                         : "r"(base + uint32_t(r * 128 + ((wchunk ^ (r % 8)) * 16))));
            s0 += __uint_as_float(w << 16);
            s1 += __uint_as_float(w & 0xFFFF0000u);
          }
          const size_t o = (kv0 + size_t(j) * kBpt + blk) * HD + 2 * p;
          const float m0 = s0 / float(r1 - r0), m1 = s1 / float(r1 - r0);
          const float h0 = tf32_hi(m0), h1 = tf32_hi(m1);
          *reinterpret_cast<float2 *>(kbar + o) = make_float2(m0, m1);
          *reinterpret_cast<float2 *>(kbar_hi + o) = make_float2(h0, h1);
          *reinterpret_cast<float2 *>(kbar_lo + o) = make_float2(m0 - h0, m1 - h1);
        }
        // every lane's reads of the slot are done before it may be refilled
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.ring_empty[slot]);
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
    const size_t bh = size_t(b) * hq + (hh == 1 && active ? hs[1] : hs[0]);
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
        // 8 independent chains for the max and the sums (one set per 64-key
        // half), then trees.  Two scores an instruction: a three-input max,
        // and the exponent arguments and the sums as two-lane FMAs and adds
        // (sum chain k, the keys c = k mod 8 in order, is lane k % 2 of pair
        // k / 2), so every lane does what the scalar chains would.
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = x[k];
#pragma unroll
        for (int c = 8; c < BS; c += 2) mx[(c / 2) % 8] = max3f(mx[(c / 2) % 8], x[c], x[c + 1]);
        const float tmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                 fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
        const float mnew = fmaxf(m, tmax * sl2);
        const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-mnew, -mnew);
        float2 sa[4], sb[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) sa[k] = sb[k] = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < BS / 2; c += 2) {
          const float2 e = ffma2(make_float2(x[c], x[c + 1]), sc2, nm2);
          sa[(c % 8) / 2] = fadd2(sa[(c % 8) / 2], make_float2(ex2(e.x), ex2(e.y)));
        }
#pragma unroll
        for (int c = BS / 2; c < BS; c += 2) {
          const float2 e = ffma2(make_float2(x[c], x[c + 1]), sc2, nm2);
          sb[(c % 8) / 2] = fadd2(sb[(c % 8) / 2], make_float2(ex2(e.x), ex2(e.y)));
        }
        const float s0 = ((sa[0].x + sa[0].y) + (sa[1].x + sa[1].y)) +
                         ((sa[2].x + sa[2].y) + (sa[3].x + sa[3].y));
        const float s1 = ((sb[0].x + sb[0].y) + (sb[1].x + sb[1].y)) +
                         ((sb[2].x + sb[2].y) + (sb[3].x + sb[3].y));
        l = l * ex2(m - mnew) + (s0 + s1);
        m = mnew;
        // this tile's mass for row r is (s0 + s1) * 2^(mnew - lse2[r])
        float *pt = ptile + ((bh * nb + j) * 3) * BS + r;
        pt[0] = mnew;
        pt[BS] = s0;
        pt[2 * BS] = s1;
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
          const float pa = (c < QLO || (RAG && c >= qrows) || (diag && r > c))
                               ? 0.f
                               : ex2(fmaf(x[c], sl2, -lqa[c % 4]));
          const float pb = (cb < QLO || (RAG && cb >= qrows) || (diag && r > cb))
                               ? 0.f
                               : ex2(fmaf(x[cb], sl2, -lqb[c % 4]));
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
        if (!RAG || size_t(j) * BS + r < size_t(n_tok)) vert[bh * n_tok + size_t(j) * BS + r] = v;
        wg_sync(hh);  // every warp's diagonal bins are written
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

// The pooled true distribution from pass 1's tile partials: grid (ceil(nt/8),
// Bt*Hq), 256 threads, one warp per 128-key tile.  Row r's mass on the tile's
// key half is s * 2^(m - lse2[r]); the rows' masses are summed in a fixed
// order (4 per lane, then a xor tree) and averaged over the last block's
// rows (the first qrows).  Block size 64 (QLO = 64): rows below QLO are not
// in the last block, and each half is a block of its own.
template <int QLO>
__global__ void __launch_bounds__(256) tile_mass_kernel(const float *__restrict__ ptile,
                                                        const float *__restrict__ lse2,
                                                        float *__restrict__ true_last, int nt,
                                                        int qrows) {
  const int j = blockIdx.x * 8 + threadIdx.x / 32, lane = threadIdx.x % 32;
  if (j >= nt) return;
  const size_t bh = blockIdx.y;
  const float *pt = ptile + (bh * nt + j) * 3 * BS;
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int k = QLO / 32; k < BS / 32; ++k) {
    const int r = lane + 32 * k;
    if (r >= qrows) continue;  // (block 128, N not a multiple of 128)
    const float f = ex2(pt[r] - lse2[bh * BS + r]);
    s0 = fmaf(pt[BS + r], f, s0);
    s1 = fmaf(pt[2 * BS + r], f, s1);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s0 += __shfl_xor_sync(0xffffffffu, s0, o);
    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
  }
  if (lane == 0) {
    if (QLO == 0) {
      true_last[bh * nt + j] = (s0 + s1) / float(qrows);
    } else {
      true_last[bh * 2 * nt + 2 * j] = s0 / float(BS - QLO);
      true_last[bh * 2 * nt + 2 * j + 1] = s1 / float(BS - QLO);
    }
  }
}

bool encode_rows(CUtensorMap *map, const void *ptr, uint64_t rows) {
  const PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (!fn) return false;
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

// 128-key tiles of the passes (block size 64 runs two blocks per tile; a
// partial last block of block size 128 is a partial last tile)
int last_block_tc_tiles(const Dims &D) { return (D.n + BS - 1) / BS; }

namespace {

struct TcWs {
  float *pm, *pl, *lse2, *sp, *ptile;
  size_t bytes;
};

TcWs carve_tc(const Dims &D, void *ws) {
  Carver c{static_cast<char *>(ws), 0};
  const size_t heads = size_t(D.bt) * D.hq;
  const int nt = last_block_tc_tiles(D);
  const int n_chunks = (nt + kChunk - 1) / kChunk;
  TcWs w;
  w.pm = c.take<float>(heads * n_chunks * BS);
  w.pl = c.take<float>(heads * n_chunks * BS);
  w.lse2 = c.take<float>(heads * BS);
  w.sp = c.take<float>(heads * nt * size_t(kBins));
  w.ptile = c.take<float>(heads * nt * size_t(3 * BS));
  w.bytes = c.off + 256;
  return w;
}

bool encode_qk(const Dims &D, const void *q, const void *k, CUtensorMap *mq, CUtensorMap *mk) {
  return encode_rows(mq, q, uint64_t(D.bt) * D.hq * D.n) &&
         encode_rows(mk, k, uint64_t(D.bt) * D.hkv * D.n);
}

}  // namespace

size_t last_block_tc_ws_bytes(const Dims &D) { return carve_tc(D, nullptr).bytes; }

// Pass 1, the log-sum-exps and the pooled true distribution, for every head;
// with kbar (and its halves) non-null, pass 1 also writes the block means of
// K from the key tiles it streams.
cudaError_t launch_last_block_rows_tc(const Dims &D, const void *q, const void *k,
                                      float *true_last, float *kbar, float *kbar_hi,
                                      float *kbar_lo, void *ws, cudaStream_t st) {
  CUtensorMap mq, mk;
  if (!encode_qk(D, q, k, &mq, &mk)) return cudaErrorInvalidValue;
  const TcWs w = carve_tc(D, ws);
  const size_t heads = size_t(D.bt) * D.hq;
  const int nt = last_block_tc_tiles(D);
  const int n_chunks = (nt + kChunk - 1) / kChunk;
  const dim3 grid(n_chunks, D.hkv * ((D.g + 1) / 2), D.bt);
  int *status = device_status_ptr();
  const int rows = int(heads * BS);
  const int q0 = (nt - 1) * BS, qrows = D.n - q0;
  auto run = [&](auto pass1, auto mass) {
    cudaFuncSetAttribute(pass1, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes));
    pass1<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, D.hq, D.g, D.n, nt, q0, qrows, n_chunks,
                                              w.pm, w.pl, w.ptile, nullptr, nullptr, nullptr,
                                              nullptr, kbar, kbar_hi, kbar_lo, status);
    lse2_combine_kernel<<<(rows + 127) / 128, 128, 0, st>>>(w.pm, w.pl, w.lse2, rows, n_chunks);
    mass<<<dim3((nt + 7) / 8, unsigned(heads)), 256, 0, st>>>(w.ptile, w.lse2, true_last, nt,
                                                              qrows);
  };
  if (D.bs == BS && qrows == BS)
    run(last_block_tc_kernel<1, 0, false>, tile_mass_kernel<0>);
  else if (D.bs == BS)  // N not a multiple of 128: a partial last block
    run(last_block_tc_kernel<1, 0, true>, tile_mass_kernel<0>);
  else  // block 64: the last 128 rows minus the first 64
    run(last_block_tc_kernel<1, BS / 2, false>, tile_mass_kernel<BS / 2>);
  return cudaGetLastError();
}

// Pass 2 (after launch_last_block_rows_tc on the same workspace): vert and
// the diagonal partials sp [Bt,Hq,n/128,255] of the 128-key tiles (combined
// into slash by the caller's slash_combine step with block size 128), for
// every head, or with `vs_only` (a pattern array) for its vertical-slash
// heads only.
cudaError_t launch_last_block_lines_tc(const Dims &D, const void *q, const void *k, float *vert,
                                       const int32_t *vs_only, float **sp_out, void *ws,
                                       cudaStream_t st) {
  CUtensorMap mq, mk;
  if (!encode_qk(D, q, k, &mq, &mk)) return cudaErrorInvalidValue;
  const TcWs w = carve_tc(D, ws);
  *sp_out = w.sp;
  const int nt = last_block_tc_tiles(D);
  const int n_chunks = (nt + kChunk - 1) / kChunk;
  const dim3 grid(n_chunks, D.hkv * ((D.g + 1) / 2), D.bt);
  int *status = device_status_ptr();
  const int q0 = (nt - 1) * BS, qrows = D.n - q0;
  auto run = [&](auto pass2) {
    cudaFuncSetAttribute(pass2, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemBytes));
    pass2<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, D.hq, D.g, D.n, nt, q0, qrows, n_chunks,
                                              nullptr, nullptr, nullptr, w.lse2, vert, w.sp,
                                              vs_only, nullptr, nullptr, nullptr, status);
  };
  if (D.bs == BS && qrows == BS)
    run(last_block_tc_kernel<2, 0, false>);
  else if (D.bs == BS)
    run(last_block_tc_kernel<2, 0, true>);
  else
    run(last_block_tc_kernel<2, BS / 2, false>);
  return cudaGetLastError();
}

}  // namespace fpi
