// select.cu -- fp_select: cumulative-attention index selection.
//
// FlexPrefill (atlas.scime.ai summary, "Approach"): keep the smallest set of
// blocks (query-aware heads, over the flattened estimated map) or lines
// (vertical-slash heads, over column and diagonal sums) whose cumulative
// normalised attention reaches gamma; the summary's "Measured effects" table
// adds min / max computational budgets.
//
// Exact rule on a list of fp32 scores s_i (finite, >= 0):
//   order       score descending, then index ascending;
//   mass        w_i = ceil(s_i * 2^32), an integer, summed exactly (W);
//   k_gamma     smallest k with (double)(sum of the first k masses) >=
//               (double)gamma * (double)W; gamma >= 1 keeps everything;
//   k           clamp(k_gamma, lo, hi);
//   kept        the first k entries of the order.
// Because non-negative fp32 scores order like their bit patterns, the kept
// set is {bits_i > b} u {bits_i == b and i <= idx} for one threshold pair
// (b, idx).  select_head_kernel finds it with a three-level radix descent on
// the bit patterns (12 + 12 + 8 bits), weighted by mass to find k_gamma and by
// count when the clamp moves k, and one ordered count for the tie rank.  All
// of it is integer arithmetic, so the result does not depend on thread order.
// emit_rows_kernel then writes every row's ascending block list.
//
// Query-wise rule for query-aware heads ("Measured effects": query-wise index
// selection instead of the flattened map): the same rule on each row
// A[i, 0..i] of the map with the row's own total and per-row budgets.
// select_rows_qa_kernel gives each (row, head) one CTA, which sorts the row's
// (bit pattern, index) keys in shared memory, finds k by an exact uint64
// prefix sum of the masses, and writes the row's list itself.
//
// Block-pooled lines for vertical-slash heads (FP_VS_BLOCKS): pool_lines_kernel
// sums vert per key block and slash per block distance into nb-entry lists,
// which select_head_kernel then selects as lines of a sequence of nb tokens
// with block size 1 (a column is a key block, an offset one block distance).
#include <cooperative_groups.h>

#include <mutex>

#include "fp_internal.cuh"

namespace cg = cooperative_groups;

namespace fpi {
namespace {

constexpr int kMaxBlocks = 4096;  // nb limit (flags live in shared memory)

enum : int { SEL_THRESHOLD = 0, SEL_NONE = 1, SEL_ALL = 2 };

struct HeadSel {
  int mode;
  uint32_t bits;
  uint32_t idx;
  int pad;
};

__device__ __forceinline__ uint32_t score_bits(float s) {
  return s > 0.f ? __float_as_uint(s) : 0u;  // negative zero / NaN / negatives -> 0
}
__device__ __forceinline__ uint64_t score_mass(uint32_t bits) {
  return (uint64_t)ceil((double)__uint_as_float(bits) * 4294967296.0);
}
__device__ __forceinline__ bool kept(uint32_t bits, uint32_t i, const HeadSel &s) {
  if (s.mode == SEL_ALL) return true;
  if (s.mode == SEL_NONE) return false;
  return bits > s.bits || (bits == s.bits && i <= s.idx);
}


// ---------------------------------------------------------------------------
// One selection problem per head, spread over a cluster of kCluster CTAs.
// Rank r of the cluster owns the contiguous slice [r*ceil(n/C), ...) of the
// list.  Each histogram level is built per slice, then every rank sums its
// share of the bins over all ranks (distributed shared memory) into rank 0's
// copy; rank 0 finds the crossing bin and the other ranks read the result.
// Integer arithmetic throughout: the result does not depend on the split.

constexpr int kCluster = 8;
constexpr int kCThreads = 512;
constexpr int kCWarps = kCThreads / 32;

struct SelSmem {
  unsigned long long hmass[4096];
  unsigned int hcnt[4096];
  unsigned long long warp_tot[32];
  unsigned long long res[8];  // [0..2] crossing, [3] scan total, [4] slice count, [5] tie index
  uint8_t colflag[kMaxBlocks];
  uint8_t distflag[kMaxBlocks];
};

struct Ctx {
  cg::cluster_group cl;
  unsigned rank;
  SelSmem *sm;
  __device__ SelSmem *peer(unsigned q) const { return cl.map_shared_rank(sm, int(q)); }
};

// Block-wide exclusive prefix sum (thread order) of one value per thread.
__device__ unsigned long long block_excl_scan(unsigned long long v, SelSmem &sm,
                                              unsigned long long *total) {
  const int lane = threadIdx.x % 32, w = threadIdx.x / 32;
  unsigned long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) sm.warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    unsigned long long t = lane < kCWarps ? sm.warp_tot[lane] : 0ull;
    unsigned long long s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      unsigned long long y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kCWarps) sm.warp_tot[lane] = s - t;  // exclusive over warps
    if (lane == 31) sm.res[3] = s;
  }
  __syncthreads();
  unsigned long long r = sm.warp_tot[w] + x - v;
  *total = sm.res[3];
  __syncthreads();
  return r;
}

// Histogram of (bits >> shift) & (nbins-1) over the slice [i0, i1), entries
// whose masked bits equal `prefix`; mass and count, warp-aggregated
// shared-memory atomics.  Then the cluster-wide merge into rank 0.
__device__ void histogram(const Ctx &cx, const float *__restrict__ s, uint32_t i0, uint32_t i1,
                          uint32_t prefix, uint32_t pmask, int shift, uint32_t nbins) {
  SelSmem &sm = *cx.sm;
  for (uint32_t i = threadIdx.x; i < nbins; i += kCThreads) {
    sm.hmass[i] = 0;
    sm.hcnt[i] = 0;
  }
  __syncthreads();
  const int lane = threadIdx.x % 32;
  // each warp takes kHistU consecutive groups of 32 entries per round and
  // issues all their loads before using any, so the scan is not one load
  // latency per 32 entries
  constexpr uint32_t kHistU = 8;
  constexpr int kHistAggMax = 8;
  for (uint32_t base = i0 + (threadIdx.x / 32) * 32 * kHistU; base < i1;
       base += kCThreads * kHistU) {
    uint32_t bits[kHistU];
#pragma unroll
    for (uint32_t u = 0; u < kHistU; ++u) {
      const uint32_t i = base + u * 32 + lane;
      bits[u] = i < i1 ? score_bits(s[i]) : 0u;
    }
#pragma unroll
    for (uint32_t u = 0; u < kHistU; ++u) {
      const uint32_t i = base + u * 32 + lane;
      uint32_t bin = 0xFFFFFFFFu;
      uint64_t w = 0;
      if (i < i1 && (bits[u] & pmask) == prefix) {
        bin = (bits[u] >> shift) & (nbins - 1);
        w = score_mass(bits[u]);
      }
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      const bool leader = lane == __ffs(peers) - 1;
      // a reduction over one group of peers runs once per distinct group, so
      // when the lanes spread over many bins (the levels below the exponent,
      // where most scores differ) every lane adds its own entry instead; the
      // sums are integers, so both ways give the same bins
      if (__popc(__ballot_sync(0xffffffffu, leader)) > kHistAggMax) {
        if (bin != 0xFFFFFFFFu) {
          atomicAdd(&sm.hmass[bin], (unsigned long long)w);
          atomicAdd(&sm.hcnt[bin], 1u);
        }
      } else {
        const unsigned lo = __reduce_add_sync(peers, unsigned(w & 0xFFFFFFull));
        const unsigned hi = __reduce_add_sync(peers, unsigned(w >> 24));
        if (bin != 0xFFFFFFFFu && leader) {
          atomicAdd(&sm.hmass[bin], ((unsigned long long)hi << 24) + lo);
          atomicAdd(&sm.hcnt[bin], unsigned(__popc(peers)));
        }
      }
    }
  }
  // merge: rank r sums bins [r*nbins/C, (r+1)*nbins/C) of every rank into rank 0
  cx.cl.sync();
  const uint32_t per = nbins / kCluster;
  SelSmem *root = cx.peer(0);
  for (uint32_t b = cx.rank * per + threadIdx.x; b < (cx.rank + 1) * per; b += kCThreads) {
    unsigned long long m = 0;
    unsigned int c = 0;
#pragma unroll
    for (unsigned q = 0; q < kCluster; ++q) {
      const SelSmem *pq = cx.peer(q);
      m += pq->hmass[b];
      c += pq->hcnt[b];
    }
    root->hmass[b] = m;
    root->hcnt[b] = c;
  }
  cx.cl.sync();
}

// Rank 0: scan the merged histogram from the highest bin down and find the
// first bin at which above + (inclusive cumulative) reaches the target.  Every
// rank then reads the bin and the mass / count of the bins strictly higher.
__device__ uint32_t find_crossing(const Ctx &cx, uint32_t nbins, bool by_mass, double target_m,
                                  unsigned long long target_c, unsigned long long *above_m,
                                  unsigned long long *above_c) {
  SelSmem &sm = *cx.sm;
  if (cx.rank == 0) {
    const uint32_t per = nbins >= kCThreads ? nbins / kCThreads : 1;
    const uint32_t p0 = threadIdx.x * per;  // positions in descending-bin order
    unsigned long long lm = 0, lc = 0;
    if (p0 < nbins)
      for (uint32_t p = p0; p < p0 + per; ++p) {
        const uint32_t b = nbins - 1 - p;
        lm += sm.hmass[b];
        lc += sm.hcnt[b];
      }
    unsigned long long tm, tc;
    const unsigned long long em = block_excl_scan(lm, sm, &tm);
    const unsigned long long ec = block_excl_scan(lc, sm, &tc);
    if (threadIdx.x == 0) {
      sm.res[0] = 0;  // fallback: lowest bin (unreachable for valid targets)
      sm.res[1] = tm - sm.hmass[0];
      sm.res[2] = tc - sm.hcnt[0];
    }
    __syncthreads();
    const unsigned long long am = *above_m, ac = *above_c;
    auto reach = [&](unsigned long long m, unsigned long long c) {
      return by_mass ? (double)(am + m) >= target_m : (ac + c) >= target_c;
    };
    if (p0 < nbins && !reach(em, ec) && reach(em + lm, ec + lc)) {
      unsigned long long cm = em, cc = ec;
      for (uint32_t p = p0; p < p0 + per; ++p) {
        const uint32_t b = nbins - 1 - p;
        if (reach(cm + sm.hmass[b], cc + sm.hcnt[b])) {
          sm.res[0] = b;
          sm.res[1] = cm;
          sm.res[2] = cc;
          break;
        }
        cm += sm.hmass[b];
        cc += sm.hcnt[b];
      }
    }
  }
  cx.cl.sync();
  const SelSmem *root = cx.peer(0);
  const uint32_t bin = uint32_t(root->res[0]);
  *above_m += root->res[1];
  *above_c += root->res[2];
  cx.cl.sync();  // rank 0 may reuse res afterwards
  return bin;
}

// Rank 0 sums the merged level-1 histogram (every entry is in it): W.
__device__ unsigned long long total_mass(const Ctx &cx, uint32_t nbins) {
  SelSmem &sm = *cx.sm;
  if (cx.rank == 0) {
    unsigned long long part = 0;
    for (uint32_t b = threadIdx.x; b < nbins; b += kCThreads) part += sm.hmass[b];
    unsigned long long tot;
    block_excl_scan(part, sm, &tot);
    if (threadIdx.x == 0) sm.res[6] = tot;
  }
  cx.cl.sync();
  const unsigned long long w = cx.peer(0)->res[6];
  cx.cl.sync();
  return w;
}

// Radix descent; returns the threshold bit pattern and the mass / count of
// every entry with larger bits.  By mass the target is gamma * W.
__device__ uint32_t descend(const Ctx &cx, const float *s, uint32_t i0, uint32_t i1,
                            bool by_mass, float gamma, unsigned long long target_c,
                            unsigned long long *above_m, unsigned long long *above_c,
                            double *target_m_out) {
  const int shifts[3] = {20, 8, 0};
  const int widths[3] = {12, 12, 8};
  uint32_t prefix = 0, pmask = 0;
  *above_m = 0;
  *above_c = 0;
  double target_m = 0.0;
  for (int lv = 0; lv < 3; ++lv) {
    const uint32_t nbins = 1u << widths[lv];
    histogram(cx, s, i0, i1, prefix, pmask, shifts[lv], nbins);
    if (lv == 0 && by_mass) {
      const unsigned long long tot = total_mass(cx, nbins);
      target_m = (double)gamma * (double)tot;
      *target_m_out = target_m;
    }
    const uint32_t bin = find_crossing(cx, nbins, by_mass, target_m, target_c, above_m, above_c);
    prefix |= bin << shifts[lv];
    pmask |= (nbins - 1) << shifts[lv];
  }
  return prefix;
}

// Index of the m-th (1-based) entry with bit pattern == b, in index order,
// over the whole list (the slices are in index order across ranks).  Warp w
// of a rank scans its contiguous chunk of the rank's slice 32 entries at a
// time (coalesced, kTieU groups in flight) and counts matches by ballot; an
// exclusive scan over the warps and the ranks' totals place the m-th match,
// and the warp holding it rescans its chunk to find it.
__device__ uint32_t tie_index(const Ctx &cx, const float *s, uint32_t n, uint32_t i0,
                              uint32_t i1, uint32_t b, unsigned long long m) {
  SelSmem &sm = *cx.sm;
  constexpr uint32_t kTieU = 8;
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  const uint32_t len = i1 > i0 ? i1 - i0 : 0;
  const uint32_t per = ((len + kCWarps - 1) / kCWarps + 31u) & ~31u;
  const uint32_t w0 = min(i1, i0 + uint32_t(warp) * per), w1 = min(i1, w0 + per);
  auto matches = [&](uint32_t g) -> unsigned {  // ballot of group g (32 entries from w0)
    const uint32_t i = w0 + g * 32 + lane;
    return __ballot_sync(0xffffffffu, i < w1 && score_bits(s[i]) == b);
  };
  const uint32_t ngroups = (w1 - w0 + 31) / 32;
  unsigned long long c = 0;
  for (uint32_t g0 = 0; g0 < ngroups; g0 += kTieU) {
    unsigned bal[kTieU];
#pragma unroll
    for (uint32_t u = 0; u < kTieU; ++u) bal[u] = g0 + u < ngroups ? matches(g0 + u) : 0u;
#pragma unroll
    for (uint32_t u = 0; u < kTieU; ++u) c += __popc(bal[u]);
  }
  unsigned long long tot;
  const unsigned long long e = __shfl_sync(0xffffffffu,
                                           block_excl_scan(lane == 0 ? c : 0ull, sm, &tot), 0);
  if (threadIdx.x == 0) {
    sm.res[4] = tot;
    if (cx.rank == 0) sm.res[5] = n - 1;
  }
  cx.cl.sync();
  unsigned long long off = 0;  // matches in the slices of lower ranks
  for (unsigned q = 0; q < cx.rank; ++q) off += cx.peer(q)->res[4];
  if (off + e < m && m <= off + e + c) {  // warp-uniform
    unsigned long long r = off + e;
    for (uint32_t g = 0; g < ngroups; ++g) {
      const unsigned bal = matches(g);
      const unsigned cnt = __popc(bal);
      if (r + cnt >= m) {
        // the (m - r)-th set bit of bal
        unsigned x = bal;
        for (unsigned long long k = r + 1; k < m; ++k) x &= x - 1;
        if (lane == 0) cx.peer(0)->res[5] = w0 + g * 32 + uint32_t(__ffs(x) - 1);
        break;
      }
      r += cnt;
    }
  }
  cx.cl.sync();
  const uint32_t idx = uint32_t(cx.peer(0)->res[5]);
  cx.cl.sync();
  return idx;
}

__device__ HeadSel select_list(const Ctx &cx, const float *s, uint32_t n, float gamma,
                               unsigned long long lo, unsigned long long hi) {
  HeadSel r{SEL_NONE, 0u, 0u, 0};
  if (n == 0) return r;
  const uint32_t chunk = (n + kCluster - 1) / kCluster;
  const uint32_t i0 = min(n, cx.rank * chunk), i1 = min(n, i0 + chunk);
  unsigned long long am = 0, ac = 0, k;
  double target = 0.0;
  uint32_t b = 0;
  unsigned long long m = 0;
  bool have_threshold = false;
  if (gamma >= 1.f) {
    k = n;
  } else {
    b = descend(cx, s, i0, i1, true, gamma, 0, &am, &ac, &target);
    if (target <= 0.0) {
      k = 0;
    } else {
      const unsigned long long w = score_mass(b);
      // smallest m >= 1 with am + m * w >= target (w >= 1 here: a zero-mass
      // bin cannot be the crossing one for a positive target)
      unsigned long long mm = 1;
      if (w > 0) {
        double need = (target - (double)am) / (double)w;
        mm = need <= 1.0 ? 1ull : (unsigned long long)ceil(need);
        while (mm > 1 && (double)(am + (mm - 1) * w) >= target) --mm;
        while ((double)(am + mm * w) < target) ++mm;
      }
      k = ac + mm;
      m = mm;
      have_threshold = true;
    }
  }
  const unsigned long long kc = k < lo ? lo : (k > hi ? hi : k);
  if (kc == 0) return r;
  if (kc >= n) {
    r.mode = SEL_ALL;
    return r;
  }
  if (!(have_threshold && kc == k)) {
    b = descend(cx, s, i0, i1, false, gamma, kc, &am, &ac, &target);
    m = kc - ac;
  }
  r.mode = SEL_THRESHOLD;
  r.bits = b;
  r.idx = tie_index(cx, s, n, i0, i1, b, m);
  return r;
}

// grid (kCluster * Hq, Bt), clusters of kCluster CTAs along x, kCThreads
// threads, dynamic shared memory SelSmem.  Cluster h selects head h.
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kCThreads)
    select_head_kernel(const int32_t *__restrict__ pattern, const float *__restrict__ map,
                       const float *__restrict__ vert, const float *__restrict__ slash, int n,
                       int nb, int bs, float gamma, long long qa_lo, long long qa_hi, int vs_lo,
                       int vs_hi, int qa_mode, HeadSel *__restrict__ sel,
                       uint8_t *__restrict__ colflag, uint8_t *__restrict__ distflag) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Ctx cx{cg::this_cluster(), 0u, reinterpret_cast<SelSmem *>(smem_raw)};
  cx.rank = cx.cl.block_rank();
  SelSmem &sm = *cx.sm;
  const size_t heads_x = gridDim.x / kCluster;
  const size_t bh = size_t(blockIdx.y) * heads_x + blockIdx.x / kCluster;
  const size_t t_pairs = size_t(nb) * (nb + 1) / 2;
  if (pattern[bh] == FP_PATTERN_QA) {  // uniform over the cluster
    if (qa_mode == FP_QA_QUERYWISE) return;  // rows selected by select_rows_qa_kernel
    HeadSel r = select_list(cx, map + bh * t_pairs, uint32_t(t_pairs), gamma, qa_lo, qa_hi);
    if (cx.rank == 0 && threadIdx.x == 0) sel[2 * bh] = r;
    return;
  }
  for (int i = threadIdx.x; i < nb; i += kCThreads) {
    sm.colflag[i] = 0;
    sm.distflag[i] = 0;
  }
  __syncthreads();
  const float *vv = vert + bh * n;
  const float *ss = slash + bh * n;
  const uint32_t chunk = (uint32_t(n) + kCluster - 1) / kCluster;
  const int s0 = int(min(uint32_t(n), cx.rank * chunk)), s1 = int(min(uint32_t(n), s0 + chunk));
  HeadSel rv = select_list(cx, vv, uint32_t(n), gamma, vs_lo, vs_hi);
  for (int t = s0 + threadIdx.x; t < s1; t += kCThreads)
    if (kept(score_bits(vv[t]), uint32_t(t), rv)) sm.colflag[t / bs] = 1;
  HeadSel rs = select_list(cx, ss, uint32_t(n), gamma, vs_lo, vs_hi);
  for (int o = s0 + threadIdx.x; o < s1; o += kCThreads)
    if (kept(score_bits(ss[o]), uint32_t(o), rs)) {
      const int d0 = o / bs;
      sm.distflag[d0] = 1;
      if (o % bs != 0 && d0 + 1 < nb) sm.distflag[d0 + 1] = 1;
    }
  // OR the slices' flags: rank r writes blocks [r*per, (r+1)*per)
  cx.cl.sync();
  const int per = (nb + kCluster - 1) / kCluster;
  for (int i = int(cx.rank) * per + threadIdx.x; i < min(nb, int(cx.rank + 1) * per);
       i += kCThreads) {
    uint8_t c = 0, d = 0;
#pragma unroll
    for (unsigned q = 0; q < kCluster; ++q) {
      c |= cx.peer(q)->colflag[i];
      d |= cx.peer(q)->distflag[i];
    }
    colflag[bh * nb + i] = c;
    distflag[bh * nb + i] = d;
  }
  if (cx.rank == 0 && threadIdx.x == 0) {
    sel[2 * bh] = rv;
    sel[2 * bh + 1] = rs;
  }
  cx.cl.sync();  // peers' flags stay readable until every rank is done
}

// grid (ceil(nb/8), Hq, Bt), 256 threads: one warp per row.
__global__ void __launch_bounds__(256) emit_rows_kernel(
    const int32_t *__restrict__ pattern, const float *__restrict__ map, int nb,
    const HeadSel *__restrict__ sel, const uint8_t *__restrict__ colflag,
    const uint8_t *__restrict__ distflag, int qa_mode, int32_t *__restrict__ counts,
    int32_t *__restrict__ indices) {
  const int qi = blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (qi >= nb) return;
  const size_t bh = size_t(blockIdx.z) * gridDim.y + blockIdx.y;
  const bool qa = pattern[bh] == FP_PATTERN_QA;
  if (qa && qa_mode == FP_QA_QUERYWISE) return;  // written by select_rows_qa_kernel
  const HeadSel s = sel[2 * bh];
  const size_t rowbase = size_t(qi) * (qi + 1) / 2;
  const float *mrow = map + bh * (size_t(nb) * (nb + 1) / 2) + rowbase;
  const uint8_t *cf = colflag + bh * nb;
  const uint8_t *df = distflag + bh * nb;
  int32_t *out = indices + (bh * nb + qi) * size_t(nb);
  int cnt = 0;
  for (int j0 = 0; j0 <= qi; j0 += 32) {
    const int j = j0 + lane;
    bool keep = false;
    if (j <= qi) {
      if (j == qi)
        keep = true;
      else if (qa)
        keep = kept(score_bits(mrow[j]), uint32_t(rowbase + j), s);
      else
        keep = cf[j] || df[qi - j];
    }
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) out[cnt + __popc(bal & ((1u << lane) - 1u))] = j;
    cnt += __popc(bal);
  }
  if (lane == 0) counts[bh * nb + qi] = cnt;
}

// Block-pooled lines for vertical-slash heads (FP_VS_BLOCKS): grid
// (ceil(nb/256), Hq, Bt), 256 threads; thread c of head bh writes
// pv[bh][c] = sum of vert[bh][c*B .. c*B+B-1] and ps[bh][c] likewise for slash,
// each summed in double, one add at a time in ascending order, and rounded to
// float once.  Query-aware heads are skipped.
__global__ void __launch_bounds__(256) pool_lines_kernel(
    const int32_t *__restrict__ pattern, const float *__restrict__ vert,
    const float *__restrict__ slash, int n, int nb, int bs, float *__restrict__ pv,
    float *__restrict__ ps) {
  const int c = blockIdx.x * 256 + threadIdx.x;
  const size_t bh = size_t(blockIdx.z) * gridDim.y + blockIdx.y;
  if (c >= nb || pattern[bh] == FP_PATTERN_QA) return;
  const float *v = vert + bh * n + size_t(c) * bs;
  const float *s = slash + bh * n + size_t(c) * bs;
  double av = 0.0, as = 0.0;
  for (int t = 0; t < bs; ++t) {
    av += (double)v[t];
    as += (double)s[t];
  }
  pv[bh * nb + c] = __double2float_rn(av);
  ps[bh * nb + c] = __double2float_rn(as);
}

// Query-wise rule: grid (nb, Hq, Bt), kRowThreads threads, dynamic shared
// memory for P = (smallest power of two >= nb) 64-bit keys and P flags.
// Query-aware heads only (others return at once); row qi of head bh:
//   key_j = (bit pattern of score j) << 32 | (0xFFFFFFFF - j), so a descending
//   sort is the rule's order (score descending, then j ascending), with the
//   padding keys (0) last;
//   k_gamma = smallest k whose exact uint64 mass prefix reaches
//   (double)gamma * (double)W; k = clamp(k_gamma, lo, hi) with the row's
//   budgets; the row keeps the first k sorted entries and its diagonal.
constexpr int kRowThreads = 256;

__global__ void __launch_bounds__(kRowThreads) select_rows_qa_kernel(
    const int32_t *__restrict__ pattern, const float *__restrict__ map, int nb, int pmax,
    float gamma, int row_lo, int row_hi, int32_t *__restrict__ counts,
    int32_t *__restrict__ indices) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  unsigned long long *keys = reinterpret_cast<unsigned long long *>(smem_raw);
  uint8_t *flag = smem_raw + size_t(pmax) * 8;
  __shared__ unsigned long long part[kRowThreads];
  __shared__ int kmin;
  __shared__ int wcount[kRowThreads / 32];
  const int qi = blockIdx.x, tid = threadIdx.x;
  const size_t bh = size_t(blockIdx.z) * gridDim.y + blockIdx.y;
  if (pattern[bh] != FP_PATTERN_QA) return;
  const int n = qi + 1;
  int P = 1;
  while (P < n) P <<= 1;
  const float *mrow = map + bh * (size_t(nb) * (nb + 1) / 2) + size_t(qi) * (qi + 1) / 2;
  for (int i = tid; i < P; i += kRowThreads) {
    keys[i] = i < n ? ((unsigned long long)score_bits(mrow[i]) << 32) | (0xFFFFFFFFu - uint32_t(i))
                    : 0ull;
    flag[i] = 0;
  }
  if (tid == 0) kmin = n;
  __syncthreads();
  // bitonic sort, descending
  for (int k = 2; k <= P; k <<= 1)
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < P; i += kRowThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long x = keys[i], y = keys[ixj];
          const bool desc = (i & k) == 0;
          if (desc ? (x < y) : (x > y)) {
            keys[i] = y;
            keys[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  // exact mass prefix: thread t owns sorted entries [t*per, (t+1)*per)
  const int per = (n + kRowThreads - 1) / kRowThreads;
  const int e0 = min(n, tid * per), e1 = min(n, e0 + per);
  unsigned long long loc = 0;
  for (int e = e0; e < e1; ++e) loc += score_mass(uint32_t(keys[e] >> 32));
  part[tid] = loc;
  __syncthreads();
  // inclusive scan of the thread sums (fixed order)
  for (int off = 1; off < kRowThreads; off <<= 1) {
    const unsigned long long v = tid >= off ? part[tid - off] : 0ull;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  const unsigned long long total = part[kRowThreads - 1];
  int kg;
  if (gamma >= 1.f) {
    kg = n;
  } else {
    const double target = (double)gamma * (double)total;
    if (target <= 0.0) {
      kg = 0;
    } else {
      unsigned long long cum = tid > 0 ? part[tid - 1] : 0ull;
      for (int e = e0; e < e1; ++e) {
        cum += score_mass(uint32_t(keys[e] >> 32));
        if ((double)cum >= target) {
          atomicMin(&kmin, e + 1);
          break;
        }
      }
      __syncthreads();
      kg = kmin;
    }
  }
  int lo = row_lo < n ? row_lo : n;
  const int hi = row_hi < 0 ? n : (row_hi < n ? row_hi : n);
  lo = lo < hi ? lo : hi;
  const int kc = kg < lo ? lo : (kg > hi ? hi : kg);
  for (int e = tid; e < kc; e += kRowThreads) flag[0xFFFFFFFFu - uint32_t(keys[e])] = 1;
  if (tid == 0) flag[qi] = 1;
  __syncthreads();
  // ascending compaction of the flags
  int32_t *out = indices + (bh * nb + qi) * size_t(nb);
  const int warp = tid / 32, lane = tid % 32;
  int base = 0;
  for (int j0 = 0; j0 < n; j0 += kRowThreads) {
    const int j = j0 + tid;
    const bool keep = j < n && flag[j];
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) wcount[warp] = __popc(bal);
    __syncthreads();
    int before = base;
    for (int w = 0; w < warp; ++w) before += wcount[w];
    if (keep) out[before + __popc(bal & ((1u << lane) - 1u))] = j;
    for (int w = 0; w < kRowThreads / 32; ++w) base += wcount[w];
    __syncthreads();
  }
  if (tid == 0) counts[bh * nb + qi] = base;
}

size_t rows_qa_smem(int nb, int *pmax) {
  int p = 1;
  while (p < nb) p <<= 1;
  *pmax = p;
  return size_t(p) * 9;
}

__global__ void stats_kernel(const int32_t *__restrict__ counts,
                             const int32_t *__restrict__ pattern, long long rows, int heads,
                             int64_t *__restrict__ stats) {
  __shared__ unsigned long long red[32];
  unsigned long long s = 0, qa = 0;
  for (long long i = threadIdx.x; i < rows; i += blockDim.x) s += (unsigned)counts[i];
  for (int i = threadIdx.x; i < heads; i += blockDim.x) qa += pattern[i] == FP_PATTERN_QA;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    qa += __shfl_xor_sync(0xffffffffu, qa, o);
  }
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = (qa << 40) | s;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long ts = 0, tq = 0;
    for (int w = 0; w < int(blockDim.x / 32); ++w) {
      ts += red[w] & ((1ull << 40) - 1);
      tq += red[w] >> 40;
    }
    stats[0] = (int64_t)ts;
    stats[1] = (int64_t)tq;
  }
}

}  // namespace

size_t select_ws_bytes(const Dims &D) {
  Carver c{nullptr, 0};
  const size_t heads = size_t(D.bt) * D.hq;
  c.take<HeadSel>(2 * heads);
  c.take<uint8_t>(heads * D.nb);
  c.take<uint8_t>(heads * D.nb);
  return c.off + 256;
}

cudaError_t launch_select(const Dims &D, float gamma, const SelectBudgets &bud,
                          const int32_t *pattern, const float *map, const float *vert,
                          const float *slash, int32_t *counts, int32_t *indices, void *ws,
                          cudaStream_t st) {
  if (D.nb > kMaxBlocks) return cudaErrorInvalidValue;
  Carver c{static_cast<char *>(ws), 0};
  const size_t heads = size_t(D.bt) * D.hq;
  HeadSel *sel = c.take<HeadSel>(2 * heads);
  uint8_t *cf = c.take<uint8_t>(heads * D.nb);
  uint8_t *df = c.take<uint8_t>(heads * D.nb);
  const int smem = int(sizeof(SelSmem));
  cudaFuncSetAttribute(select_head_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (bud.vs_mode == FP_VS_BLOCKS) {
    // pooled lines live in the outputs until emit_rows_kernel overwrites them:
    // vert sums in indices (>= Bt*Hq*nb entries), slash sums in counts
    float *pv = reinterpret_cast<float *>(indices);
    float *ps = reinterpret_cast<float *>(counts);
    pool_lines_kernel<<<dim3((D.nb + 255) / 256, D.hq, D.bt), 256, 0, st>>>(
        pattern, vert, slash, D.n, D.nb, D.bs, pv, ps);
    select_head_kernel<<<dim3(kCluster * D.hq, D.bt), kCThreads, smem, st>>>(
        pattern, map, pv, ps, D.nb, D.nb, 1, gamma, bud.qa_lo, bud.qa_hi, bud.vsb_lo,
        bud.vsb_hi, bud.qa_mode, sel, cf, df);
  } else {
    select_head_kernel<<<dim3(kCluster * D.hq, D.bt), kCThreads, smem, st>>>(
        pattern, map, vert, slash, D.n, D.nb, D.bs, gamma, bud.qa_lo, bud.qa_hi, bud.vs_lo,
        bud.vs_hi, bud.qa_mode, sel, cf, df);
  }
  emit_rows_kernel<<<dim3((D.nb + 7) / 8, D.hq, D.bt), 256, 0, st>>>(
      pattern, map, D.nb, sel, cf, df, bud.qa_mode, counts, indices);
  if (bud.qa_mode == FP_QA_QUERYWISE) {
    int pmax;
    const size_t rsm = rows_qa_smem(D.nb, &pmax);
    select_rows_qa_kernel<<<dim3(D.nb, D.hq, D.bt), kRowThreads, rsm, st>>>(
        pattern, map, D.nb, pmax, gamma, bud.row_lo, bud.row_hi, counts, indices);
  }
  return cudaGetLastError();
}

cudaError_t launch_stats(const Dims &D, const int32_t *counts, const int32_t *pattern,
                         int64_t *stats, cudaStream_t st) {
  stats_kernel<<<1, 1024, 0, st>>>(counts, pattern, (long long)D.bt * D.hq * D.nb, D.bt * D.hq,
                                   stats);
  return cudaGetLastError();
}

}  // namespace fpi

// ---------------------------------------------------------------------------
// fp_select without a workspace argument.  Its scratch (the same layout
// select_ws_bytes describes) is one fixed array compiled into the library.
// The array's name is only a host-side stand-in in host code, so the device
// address is looked up with cudaGetSymbolAddress once per device (on the
// first call made with that device current) and cached.  Nothing in the
// scratch has to start at zero: select_head_kernel writes every record and
// flag that emit_rows_kernel later reads.
namespace fpi {

static __device__ __align__(256) unsigned char g_select_scratch[FP_SELECT_NOALLOC_SCRATCH_BYTES];

namespace {

// The array's device address on the current device, looked up on the first
// call made with that device current and cached (under a lock: two host
// threads may make their first calls at the same time).
cudaError_t select_scratch_address(void **out) {
  static std::mutex mu;
  static void *addr[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_select_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace

// The same launches as launch_select, with the fixed array as the workspace.
cudaError_t launch_select_noalloc(const Dims &D, float gamma, const SelectBudgets &bud,
                                  const int32_t *pattern, const float *map, const float *vert,
                                  const float *slash, int32_t *counts, int32_t *indices,
                                  cudaStream_t st) {
  if (D.nb > kMaxBlocks || select_ws_bytes(D) > FP_SELECT_NOALLOC_SCRATCH_BYTES)
    return cudaErrorInvalidValue;
  void *scratch = nullptr;
  cudaError_t e = select_scratch_address(&scratch);
  if (e != cudaSuccess) return e;
  return launch_select(D, gamma, bud, pattern, map, vert, slash, counts, indices, scratch, st);
}

}  // namespace fpi
