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
// (b, idx).  A radix select over the whole GPU finds it: two histogram passes
// over every list (digits of 11 + 11 bits, weighted by mass to find k_gamma
// and by count once the budget clamp decides k), one pass that gathers the
// few entries sharing the crossing 22-bit prefix, and the last digit and the
// tie rank on those.  All of it is integer arithmetic, so the result does not
// depend on thread order.  emit_rows_kernel then writes every row's ascending
// block list.
//
// Query-wise rule for query-aware heads ("Measured effects": query-wise index
// selection instead of the flattened map): the same rule on each row
// A[i, 0..i] of the map with the row's own total and per-row budgets.
// select_rows_qa_kernel gives each (row, head) one warp, which runs the same
// radix select on the row (four digits, warp-private histograms, warp-scan
// decisions) and writes the row's list itself.
//
// Block-pooled lines for vertical-slash heads (FP_VS_BLOCKS): pool_lines_kernel
// sums vert per key block and slash per block distance into nb-entry lists,
// which the radix select then takes as lines of a sequence of nb tokens
// with block size 1 (a column is a key block, an offset one block distance).
#include <algorithm>
#include <atomic>
#include <mutex>

#include "fp_internal.cuh"

namespace fpi {
namespace {

constexpr int kMaxBlocks = 4096;  // nb limit

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
// The flattened rule and the line lists, as a radix select over the whole GPU.
// Every head owns two list slots: slot 2h is its map (query-aware) or its
// vert list (vertical-slash), slot 2h+1 its slash list (vertical-slash only).
// A score's bit pattern (bit 31 is 0 after score_bits) splits into three
// digits: the exponent, bits 30..23 (level 1), bits 22..11 (level 2) and bits
// 10..0 (level 3).
//
//   hist_kernel<1>   every CTA histograms (mass and count) the level-1 digit
//                    of its chunks of one list in shared memory and adds its
//                    non-empty bins to the list's global histogram; the last
//                    CTA of a list to finish (a counter, no waiting) finds the
//                    crossing digit and clears the histogram for level 2.
//   hist_kernel<2>   the same for the level-2 digit of the entries whose
//                    level-1 digit is the crossing one.
//   compact_kernel   entries whose first two digits are the crossing ones go
//                    to a short candidate list; the last CTA of a list finds
//                    the level-3 digit and the tie rank among the candidates
//                    (or, when more than kCand share the prefix, by scans of
//                    the whole list).
// At each level the crossing is found by mass (the gamma rule) until it is
// clear that the budget clamp decides k; from then on by count.  The mass
// crossing bin b bounds k_gamma to (A, A + C] (A entries above the bin, C in
// it): hi <= A means k = hi, lo >= A + C means k = lo, and otherwise a clamped
// k lies in the same bin, so one prefix serves both.  Integer sums
// throughout: the result does not depend on the split into chunks.
//
// Shared-memory histograms of the scanning CTAs hold a mass as two 32-bit
// sums, of its low 16 bits and of the rest (a mass is at most 2^32, so a CTA
// may add up to kMaxCtaEntries entries to one bin): 32-bit shared atomics,
// where 64-bit ones measured several times slower.

constexpr int kSelThreads = 256;
constexpr int kChunk = 2048;         // entries per chunk (16-byte groups of 4)
constexpr int kBins1 = 256;          // level-1 digit (8 bits)
constexpr int kBins2 = 4096;         // level-2 digit (12 bits)
constexpr int kBins3 = 2048;         // level-3 digit (11 bits)
constexpr int kShift1 = 23, kShift2 = 11;
constexpr int kBins = kBins2;        // global histogram bins per list (levels 1, 2)
constexpr int kCand = 1024;          // candidate list length per list slot
constexpr int kHistAggMax = 8;
// scanning CTAs per SM (over every list), per kernel: the first digit's
// 256-bin histograms merge cheaply and gain from more CTAs, the second
// digit's 4096-bin ones pay a merge per CTA (measured at 128k: 24 / 6 / 12)
constexpr int kHist1CtasPerSm = 24, kHist2CtasPerSm = 6, kCompactCtasPerSm = 12;
constexpr int kMaxCtaEntries = 32767;                   // 32767 * 2^17 < 2^32
constexpr int kMaxCtaChunks = kMaxCtaEntries / kChunk;  // chunks a CTA may take
constexpr int kRounds = 4;

struct ListState {
  unsigned long long am, ac;  // mass / count of the entries above the prefix
  unsigned long long target_c;
  double target_m;
  uint32_t prefix;            // digits fixed so far
  int finished;               // the list's HeadSel is written
  int by_mass;                // descending by mass (1) or by count (0)
  int overflow;               // more than kCand entries share the 20-bit prefix
  unsigned int done[3];       // CTAs finished in hist<1>, hist<2>, compact
  unsigned int cand;          // candidates appended
};

struct ListView {
  const float *p;
  uint32_t len;
  unsigned long long lo, hi;
};

struct SelArgs {
  const int32_t *pattern;
  const float *map, *vert, *slash;
  int n, nb, bs;  // line lists: n entries, block size bs
  float gamma;
  long long qa_lo, qa_hi;
  int vs_lo, vs_hi;
  int qa_mode;
  HeadSel *sel;
  ListState *state;
  unsigned long long *hm;  // [slots][kBins]
  unsigned int *hc;        // [slots][kBins]
  uint2 *cand;             // [slots][kCand] (bits, index)
  int ctas;                // CTAs per list in the scanning kernels
};

// The list of `slot`, or false when the slot holds none (the second slot of a
// query-aware head, or a query-aware head under the query-wise rule).
__device__ __forceinline__ bool list_of(const SelArgs &a, int slot, ListView *lv) {
  const size_t bh = size_t(slot) / 2;
  const int which = slot % 2;
  if (a.pattern[bh] == FP_PATTERN_QA) {
    if (which == 1 || a.qa_mode == FP_QA_QUERYWISE) return false;
    const size_t t_pairs = size_t(a.nb) * (a.nb + 1) / 2;
    lv->p = a.map + bh * t_pairs;
    lv->len = uint32_t(t_pairs);
    lv->lo = (unsigned long long)a.qa_lo;
    lv->hi = (unsigned long long)a.qa_hi;
  } else {
    lv->p = (which == 0 ? a.vert : a.slash) + bh * size_t(a.n);
    lv->len = uint32_t(a.n);
    lv->lo = (unsigned long long)a.vs_lo;
    lv->hi = (unsigned long long)a.vs_hi;
  }
  return true;
}

// Element offset of a list inside its 16-byte group: chunks are cut on
// 16-byte boundaries of memory, so every full group is one aligned float4.
__device__ __forceinline__ int group_offset(const float *p) {
  return int((reinterpret_cast<uintptr_t>(p) >> 2) & 3u);
}
__device__ __forceinline__ int list_chunks(const ListView &lv) {
  return int((uint64_t(lv.len) + group_offset(lv.p) + kChunk - 1) / kChunk);
}

// The 4 entries of group g (elements 4g - off .. 4g - off + 3): bit patterns,
// and which are inside the list.  A group that lies wholly inside is one
// aligned 16-byte load; the first and last groups read only their valid
// elements.
__device__ __forceinline__ void load_group(const ListView &lv, int off, uint32_t g,
                                           uint32_t (&bits)[4], bool (&valid)[4]) {
  const long long i0 = (long long)g * 4 - off;
  if (i0 >= 0 && i0 + 3 < (long long)lv.len) {
    const float4 v = __ldg(reinterpret_cast<const float4 *>(lv.p + i0));
    bits[0] = score_bits(v.x);
    bits[1] = score_bits(v.y);
    bits[2] = score_bits(v.z);
    bits[3] = score_bits(v.w);
    valid[0] = valid[1] = valid[2] = valid[3] = true;
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const long long i = i0 + e;
      valid[e] = i >= 0 && i < (long long)lv.len;
      bits[e] = valid[e] ? score_bits(__ldg(lv.p + i)) : 0u;
    }
  }
}

// Adds one entry per lane (bin 0xFFFFFFFF: none) to a shared histogram.  A
// warp groups its lanes by bin; with at most kHistAggMax groups one lane per
// group adds the group's sums (the mass from two 32-bit reductions of its low
// 24 and high bits), with more every lane adds its own (a reduction over one
// group runs once per distinct group).  Integer sums: both give the same bins.
__device__ __forceinline__ void hist_add(unsigned long long *hm, unsigned int *hc, uint32_t bin,
                                         uint64_t w, int lane) {
  const unsigned peers = __match_any_sync(0xffffffffu, bin);
  const bool leader = lane == __ffs(peers) - 1;
  if (__popc(__ballot_sync(0xffffffffu, leader)) > kHistAggMax) {
    if (bin != 0xFFFFFFFFu) {
      atomicAdd(&hm[bin], (unsigned long long)w);
      atomicAdd(&hc[bin], 1u);
    }
  } else {
    const unsigned lo = __reduce_add_sync(peers, unsigned(w & 0xFFFFFFull));
    const unsigned hi = __reduce_add_sync(peers, unsigned(w >> 24));
    if (bin != 0xFFFFFFFFu && leader) {
      atomicAdd(&hm[bin], ((unsigned long long)hi << 24) + lo);
      atomicAdd(&hc[bin], unsigned(__popc(peers)));
    }
  }
}

// A CTA's shared histogram: mass as the sums of its low 16 bits (lo) and of
// the rest (hi), and the count.
struct SmemHist {
  unsigned int *lo, *hi, *cnt;
  __device__ __forceinline__ void add(uint32_t b, uint64_t w, unsigned n) {
    atomicAdd(&lo[b], unsigned(w & 0xFFFFull));
    atomicAdd(&hi[b], unsigned(w >> 16));
    atomicAdd(&cnt[b], n);
  }
};

// Level 1: adds the 4 entries of every lane (bin 0xFFFFFFFF: none).  The warp
// takes its smallest pending bin (a whole-warp minimum), every lane sums its
// entries in that bin, whole-warp reductions add the lanes' sums and one lane
// adds them; neighbouring scores mostly share their exponent, so a round or
// two take every entry.  After kRounds rounds the lanes add what is left one
// entry at a time.  Integer sums: every way gives the same bins.
__device__ __forceinline__ void hist_add4(SmemHist h, const uint32_t (&b)[4],
                                          const uint64_t (&w)[4], int lane) {
  bool pend[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) pend[e] = b[e] != 0xFFFFFFFFu;
#pragma unroll 1
  for (int r = 0; r < kRounds; ++r) {
    uint32_t lmin = 0xFFFFFFFFu;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (pend[e]) lmin = min(lmin, b[e]);
    const uint32_t t = __reduce_min_sync(0xffffffffu, lmin);
    if (t == 0xFFFFFFFFu) return;
    unsigned lo = 0, hi = 0, n = 0;  // 4 entries: lo < 2^18, hi < 2^19
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (pend[e] && b[e] == t) {
        lo += unsigned(w[e] & 0xFFFFull);
        hi += unsigned(w[e] >> 16);
        ++n;
        pend[e] = false;
      }
    lo = __reduce_add_sync(0xffffffffu, lo);
    hi = __reduce_add_sync(0xffffffffu, hi);
    n = __reduce_add_sync(0xffffffffu, n);
    if (lane == 0) {
      atomicAdd(&h.lo[t], lo);
      atomicAdd(&h.hi[t], hi);
      atomicAdd(&h.cnt[t], n);
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (pend[e]) h.add(b[e], w[e], 1u);
}

// Block-wide exclusive prefix sum (thread order) of one value per thread.
__device__ unsigned long long block_excl_scan(unsigned long long v, unsigned long long *warp_tot,
                                              unsigned long long *total) {
  const int lane = threadIdx.x % 32, w = threadIdx.x / 32;
  constexpr int kWarps = kSelThreads / 32;
  unsigned long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    const unsigned long long t = lane < kWarps ? warp_tot[lane] : 0ull;
    unsigned long long s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kWarps) warp_tot[lane] = s - t;
    if (lane == 31) warp_tot[kWarps] = s;
  }
  __syncthreads();
  const unsigned long long r = warp_tot[w] + x - v;
  *total = warp_tot[kWarps];
  __syncthreads();
  return r;
}

struct Crossing {
  uint32_t bin;
  unsigned long long above_m, above_c;  // sums of the bins above `bin`
};

// The first bin, scanning [0, nbins) from the top, at which the cumulative
// mass (by_mass) reaches target_m - base_m, or the cumulative count reaches
// target_c - base_c.  Run by the whole CTA; the result is in *out for every
// thread.  With no crossing (not reached for valid targets) the lowest bin.
__device__ void find_crossing(const unsigned long long *hm, const unsigned int *hc, int nbins,
                              bool by_mass, double target_m, unsigned long long base_m,
                              unsigned long long target_c, unsigned long long base_c,
                              unsigned long long *warp_tot, Crossing *out) {
  const int per = nbins / kSelThreads;
  const int p0 = threadIdx.x * per;  // positions in descending-bin order
  unsigned long long lm = 0, lc = 0;
  for (int p = p0; p < p0 + per; ++p) {
    lm += hm[nbins - 1 - p];
    lc += hc[nbins - 1 - p];
  }
  unsigned long long tm, tc;
  const unsigned long long em = block_excl_scan(lm, warp_tot, &tm);
  const unsigned long long ec = block_excl_scan(lc, warp_tot, &tc);
  if (threadIdx.x == 0) *out = Crossing{0u, tm - hm[0], tc - hc[0]};
  __syncthreads();
  auto reach = [&](unsigned long long m, unsigned long long c) {
    return by_mass ? (double)(base_m + m) >= target_m : (base_c + c) >= target_c;
  };
  if (!reach(em, ec) && reach(em + lm, ec + lc)) {
    unsigned long long cm = em, cc = ec;
    for (int p = p0; p < p0 + per; ++p) {
      const int b = nbins - 1 - p;
      if (reach(cm + hm[b], cc + hc[b])) {
        *out = Crossing{uint32_t(b), cm, cc};
        break;
      }
      cm += hm[b];
      cc += hc[b];
    }
  }
  __syncthreads();
}

__device__ __forceinline__ void finish(ListState &st, HeadSel *sel, int mode, uint32_t bits,
                                       uint32_t idx) {
  st.finished = 1;
  *sel = HeadSel{mode, bits, idx, 0};
}

// Switches to the count rule with target k; k = 0 keeps nothing and k >= len
// everything.
__device__ __forceinline__ void count_mode(ListState &st, HeadSel *sel, unsigned long long k,
                                           uint32_t len) {
  st.by_mass = 0;
  st.target_c = k;
  if (k == 0) finish(st, sel, SEL_NONE, 0u, 0u);
  else if (k >= len) finish(st, sel, SEL_ALL, 0u, 0u);
}

// One level's decision (the whole CTA; st and the histogram in shared memory):
// the crossing digit by mass, or by count once the clamp decides k, appended
// to the prefix.  Returns the crossing bin's count.
__device__ unsigned int decide_level(ListState &st, HeadSel *sel, const ListView &lv,
                                     const unsigned long long *hm, const unsigned int *hc,
                                     int nbins, int shift, unsigned long long *warp_tot,
                                     Crossing *cr) {
  if (st.by_mass) {
    find_crossing(hm, hc, nbins, true, st.target_m, st.am, 0, 0, warp_tot, cr);
    const unsigned long long A = st.ac + cr->above_c, C = hc[cr->bin];
    __syncthreads();
    if (threadIdx.x == 0) {
      if (lv.hi <= A) count_mode(st, sel, lv.hi, lv.len);
      else if (lv.lo >= A + C) count_mode(st, sel, lv.lo, lv.len);
    }
    __syncthreads();
    if (st.finished) return 0;
  }
  if (!st.by_mass) find_crossing(hm, hc, nbins, false, 0.0, 0, st.target_c, st.ac, warp_tot, cr);
  const unsigned int cnt = hc[cr->bin];
  __syncthreads();
  if (threadIdx.x == 0) {
    st.am += cr->above_m;
    st.ac += cr->above_c;
    st.prefix |= cr->bin << shift;
  }
  __syncthreads();
  return cnt;
}

// Clears the histograms and states of every slot and the VS flags; grid
// (slots), kSelThreads threads.
__global__ void __launch_bounds__(kSelThreads) sel_prep_kernel(SelArgs a, uint8_t *colflag,
                                                               uint8_t *distflag) {
  const int slot = blockIdx.x;
  for (int b = threadIdx.x; b < kBins; b += kSelThreads) {
    a.hm[size_t(slot) * kBins + b] = 0ull;
    a.hc[size_t(slot) * kBins + b] = 0u;
  }
  uint8_t *flags = (slot % 2 == 0 ? colflag : distflag) + size_t(slot / 2) * a.nb;
  for (int i = threadIdx.x; i < a.nb; i += kSelThreads) flags[i] = 0;
  if (threadIdx.x == 0) a.state[slot] = ListState{};
}

// Levels 1 and 2: grid (CTAs per list, slots), kSelThreads threads, dynamic
// shared memory hist_smem<LEVEL>(); CTA x of a list takes its chunks x,
// x + nct, ... (at most kMaxCtaChunks of them), the next one's loads issued
// before the current one is added.
template <int LEVEL>
constexpr size_t hist_smem() {
  return (LEVEL == 1 ? kBins1 : kBins2) * 12;
}

template <int LEVEL>
__global__ void __launch_bounds__(kSelThreads) sel_hist_kernel(SelArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  constexpr int NB = LEVEL == 1 ? kBins1 : kBins2;
  __shared__ unsigned long long warp_tot[kSelThreads / 32 + 1];
  __shared__ ListState st;
  __shared__ Crossing cr;
  __shared__ int is_last;
  const int slot = blockIdx.y, lane = threadIdx.x % 32;
  ListView lv;
  if (!list_of(a, slot, &lv)) return;
  const int nch = list_chunks(lv);
  const int nct = min(nch, a.ctas);  // CTAs on this list, each taking every nct-th chunk
  if (int(blockIdx.x) >= nct) return;
  ListState *gst = a.state + slot;
  uint32_t want = 0;  // level 2: the level-1 digit
  if (LEVEL == 2) {
    if (gst->finished) return;
    want = gst->prefix >> kShift1;
  }
  SmemHist h{reinterpret_cast<unsigned int *>(smem_raw),
             reinterpret_cast<unsigned int *>(smem_raw) + NB,
             reinterpret_cast<unsigned int *>(smem_raw) + 2 * NB};
  for (int b = threadIdx.x; b < 3 * NB; b += kSelThreads) h.lo[b] = 0u;
  __syncthreads();
  const int off = group_offset(lv.p);
  constexpr int kG = kChunk / 4 / kSelThreads;  // groups per thread per chunk
  uint32_t bits[kG][4], nbits[kG][4];
  bool valid[kG][4], nvalid[kG][4];
  int chunk = blockIdx.x;
#pragma unroll
  for (int u = 0; u < kG; ++u)
    load_group(lv, off, uint32_t(chunk) * (kChunk / 4) + u * kSelThreads + threadIdx.x, bits[u],
               valid[u]);
  for (; chunk < nch; chunk += nct) {
    const int next = chunk + nct;
    if (next < nch) {
#pragma unroll
      for (int u = 0; u < kG; ++u)
        load_group(lv, off, uint32_t(next) * (kChunk / 4) + u * kSelThreads + threadIdx.x,
                   nbits[u], nvalid[u]);
    }
#pragma unroll
    for (int u = 0; u < kG; ++u) {
      uint32_t bin[4];
      uint64_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t x = bits[u][e];
        bin[e] = 0xFFFFFFFFu;
        w[e] = 0;
        if (valid[u][e] && (LEVEL == 1 || (x >> kShift1) == want)) {
          bin[e] = LEVEL == 1 ? (x >> kShift1) : ((x >> kShift2) & (kBins2 - 1));
          w[e] = score_mass(x);
        }
      }
      if (LEVEL == 1) {
        hist_add4(h, bin, w, lane);
      } else {  // below the exponent nearly every entry has its own bin
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (bin[e] != 0xFFFFFFFFu) h.add(bin[e], w[e], 1u);
      }
    }
#pragma unroll
    for (int u = 0; u < kG; ++u)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        bits[u][e] = nbits[u][e];
        valid[u][e] = nvalid[u][e];
      }
  }
  __syncthreads();
  unsigned long long *ghm = a.hm + size_t(slot) * kBins;
  unsigned int *ghc = a.hc + size_t(slot) * kBins;
  for (int b = threadIdx.x; b < NB; b += kSelThreads)
    if (h.cnt[b]) {
      atomicAdd(&ghm[b], (unsigned long long)h.lo[b] + ((unsigned long long)h.hi[b] << 16));
      atomicAdd(&ghc[b], h.cnt[b]);
    }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(&gst->done[LEVEL - 1], 1u) == unsigned(nct - 1);
  __syncthreads();
  if (!is_last) return;
  // the last CTA of this list: every other CTA's bins are in the global
  // histogram; it is read into this CTA's shared memory (NB * 12 bytes)
  __threadfence();
  unsigned long long *hm = reinterpret_cast<unsigned long long *>(smem_raw);
  unsigned int *hc = reinterpret_cast<unsigned int *>(smem_raw + size_t(NB) * 8);
  for (int b = threadIdx.x; b < NB; b += kSelThreads) {
    hm[b] = __ldcg(&ghm[b]);
    hc[b] = __ldcg(&ghc[b]);
  }
  if (threadIdx.x == 0) st = *gst;
  __syncthreads();
  HeadSel *sel = a.sel + slot;
  if (LEVEL == 1) {
    unsigned long long part = 0, tot;
    for (int b = threadIdx.x; b < NB; b += kSelThreads) part += hm[b];
    block_excl_scan(part, warp_tot, &tot);  // tot = W, the list's total mass
    if (threadIdx.x == 0) {
      st.by_mass = 0;
      if (a.gamma >= 1.f) {
        count_mode(st, sel, lv.hi < lv.len ? lv.hi : lv.len, lv.len);  // k_gamma = len
      } else {
        st.target_m = (double)a.gamma * (double)tot;
        if (st.target_m <= 0.0) count_mode(st, sel, lv.lo, lv.len);  // k_gamma = 0
        else st.by_mass = 1;
      }
    }
    __syncthreads();
  }
  if (!st.finished) {
    const unsigned int cnt = decide_level(st, sel, lv, hm, hc, NB,
                                          LEVEL == 1 ? kShift1 : kShift2, warp_tot, &cr);
    if (LEVEL == 2 && threadIdx.x == 0 && !st.finished) st.overflow = cnt > unsigned(kCand);
  }
  // level 1: the global histogram is reused for level 2
  if (LEVEL == 1)
    for (int b = threadIdx.x; b < NB; b += kSelThreads) {
      ghm[b] = 0ull;
      ghc[b] = 0u;
    }
  if (threadIdx.x == 0) {
    st.done[LEVEL - 1] = gst->done[LEVEL - 1];
    *gst = st;
  }
}

// The m-th (1-based) smallest of the n indices in idx[] (shared memory, n <=
// kCand): a bitonic sort of the padded power of two.
__device__ uint32_t mth_smallest(uint32_t *idx, int n, unsigned long long m) {
  if (m < 1) m = 1;  // (1 <= m <= n by construction)
  if (m > (unsigned long long)n) m = n > 0 ? n : 1;
  int P = 1;
  while (P < n) P <<= 1;
  for (int i = n + threadIdx.x; i < P; i += kSelThreads) idx[i] = 0xFFFFFFFFu;
  __syncthreads();
  for (int k = 2; k <= P; k <<= 1)
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < P; i += kSelThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint32_t x = idx[i], y = idx[ixj];
          if ((i & k) == 0 ? x > y : x < y) {
            idx[i] = y;
            idx[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  return idx[m - 1];
}

// Level 3 and the tie rank: grid (CTAs per list, slots), chunks as above.
__global__ void __launch_bounds__(kSelThreads) sel_compact_kernel(SelArgs a) {
  __shared__ unsigned long long hm[kBins3];
  __shared__ unsigned int hc[kBins3];
  __shared__ uint2 cand[kCand];
  __shared__ uint32_t ties[kCand];
  __shared__ unsigned long long warp_tot[kSelThreads / 32 + 1];
  __shared__ ListState st;
  __shared__ Crossing cr;
  __shared__ int is_last, nties;
  __shared__ unsigned long long found;
  const int slot = blockIdx.y, lane = threadIdx.x % 32;
  ListView lv;
  if (!list_of(a, slot, &lv)) return;
  const int nch = list_chunks(lv);
  const int nct = min(nch, a.ctas);
  if (int(blockIdx.x) >= nct) return;
  ListState *gst = a.state + slot;
  if (gst->finished) return;
  const uint32_t want = gst->prefix >> kShift2;  // the first two digits
  const int off = group_offset(lv.p);
  uint2 *gc = a.cand + size_t(slot) * kCand;
  if (!gst->overflow) {
    constexpr int kG = kChunk / 4 / kSelThreads;
    for (int chunk = blockIdx.x; chunk < nch; chunk += nct) {
      const uint32_t g0 = uint32_t(chunk) * (kChunk / 4);
      uint32_t bits[kG][4];
      bool valid[kG][4];
#pragma unroll
      for (int u = 0; u < kG; ++u)
        load_group(lv, off, g0 + u * kSelThreads + threadIdx.x, bits[u], valid[u]);
#pragma unroll
      for (int u = 0; u < kG; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool hit = valid[u][e] && (bits[u][e] >> kShift2) == want;
          const unsigned bal = __ballot_sync(0xffffffffu, hit);
          if (bal) {
            unsigned base = 0;
            if (lane == __ffs(bal) - 1) base = atomicAdd(&gst->cand, unsigned(__popc(bal)));
            base = __shfl_sync(0xffffffffu, base, __ffs(bal) - 1);
            if (hit) {
              const uint32_t i = (g0 + u * kSelThreads + threadIdx.x) * 4 + e - off;
              gc[base + __popc(bal & ((1u << lane) - 1u))] = make_uint2(bits[u][e], i);
            }
          }
        }
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(&gst->done[2], 1u) == unsigned(nct - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (threadIdx.x == 0) st = *gst;
  for (int b = threadIdx.x; b < kBins3; b += kSelThreads) {
    hm[b] = 0ull;
    hc[b] = 0u;
  }
  __syncthreads();
  HeadSel *sel = a.sel + slot;
  // level 3 over the entries that share the first two digits
  const int nc = st.overflow ? 0 : int(__ldcg(&gst->cand));
  if (!st.overflow) {
    for (int c = threadIdx.x; c < nc; c += kSelThreads) cand[c] = __ldcg(&gc[c]);
    __syncthreads();
    for (int c0 = 0; c0 < nc; c0 += kSelThreads) {
      const int c = c0 + threadIdx.x;
      uint32_t bin = 0xFFFFFFFFu;
      uint64_t w = 0;
      if (c < nc) {
        bin = cand[c].x & (kBins3 - 1);  // (the third digit)
        w = score_mass(cand[c].x);
      }
      hist_add(hm, hc, bin, w, lane);
    }
  } else {  // too many entries share the prefix: scan the whole list
    for (uint32_t i0 = 0; i0 < lv.len; i0 += kSelThreads) {
      const uint32_t i = i0 + threadIdx.x;
      uint32_t bin = 0xFFFFFFFFu;
      uint64_t w = 0;
      if (i < lv.len) {
        const uint32_t x = score_bits(lv.p[i]);
        if ((x >> kShift2) == want) {
          bin = x & (kBins3 - 1);
          w = score_mass(x);
        }
      }
      hist_add(hm, hc, bin, w, lane);
    }
  }
  __syncthreads();
  decide_level(st, sel, lv, hm, hc, kBins3, 0, warp_tot, &cr);
  if (st.finished) {  // (the clamp with k = 0 or k >= len, decided here)
    if (threadIdx.x == 0) *gst = st;
    return;
  }
  const uint32_t b = st.prefix;  // the full threshold pattern
  unsigned long long m;
  if (st.by_mass) {
    // smallest m >= 1 with am + m w >= target (w >= 1: a zero-mass bin cannot
    // be the crossing one for a positive target), then the clamp, which by
    // construction keeps k inside this pattern's entries
    const unsigned long long w = score_mass(b);
    unsigned long long mm = 1;
    if (w > 0) {
      const double need = (st.target_m - (double)st.am) / (double)w;
      mm = need <= 1.0 ? 1ull : (unsigned long long)ceil(need);
      while (mm > 1 && (double)(st.am + (mm - 1) * w) >= st.target_m) --mm;
      while ((double)(st.am + mm * w) < st.target_m) ++mm;
    }
    unsigned long long k = st.ac + mm;
    k = k < lv.lo ? lv.lo : (k > lv.hi ? lv.hi : k);
    m = k - st.ac;
  } else {
    m = st.target_c - st.ac;
  }
  // the m-th entry with pattern b, in index order
  if (!st.overflow) {
    if (threadIdx.x == 0) nties = 0;
    __syncthreads();
    for (int c = threadIdx.x; c < nc; c += kSelThreads)
      if (cand[c].x == b) ties[atomicAdd(&nties, 1)] = cand[c].y;
    __syncthreads();
    const uint32_t idx = mth_smallest(ties, nties, m);
    if (threadIdx.x == 0) finish(st, sel, SEL_THRESHOLD, b, idx);
  } else {
    // ordered count over the whole list, kSelThreads entries at a time
    if (threadIdx.x == 0) found = 0xFFFFFFFFull;
    __syncthreads();
    unsigned long long before = 0;
    for (uint32_t i0 = 0; i0 < lv.len && found == 0xFFFFFFFFull; i0 += kSelThreads) {
      const uint32_t i = i0 + threadIdx.x;
      const bool hit = i < lv.len && score_bits(lv.p[i]) == b;
      unsigned long long tot;
      const unsigned long long e = block_excl_scan(hit ? 1ull : 0ull, warp_tot, &tot);
      if (hit && before + e + 1 == m) found = i;
      before += tot;
      __syncthreads();
    }
    if (threadIdx.x == 0) finish(st, sel, SEL_THRESHOLD, b, uint32_t(found));
  }
  __syncthreads();
  if (threadIdx.x == 0) *gst = st;
}

// Column and distance flags of the vertical-slash heads from their kept
// lines: grid (ceil(n / (256 * kFlagU)), slots), 256 threads, kFlagU lines a
// thread (strided by 256).
constexpr int kFlagU = 16;
__global__ void __launch_bounds__(256) sel_flags_kernel(SelArgs a, uint8_t *__restrict__ colflag,
                                                        uint8_t *__restrict__ distflag) {
  const int slot = blockIdx.y;
  const size_t bh = size_t(slot) / 2;
  if (a.pattern[bh] == FP_PATTERN_QA) return;
  const HeadSel s = a.sel[slot];
  if (s.mode == SEL_NONE) return;
  const float *line = (slot % 2 == 0 ? a.vert : a.slash) + bh * a.n;
  uint8_t *cf = colflag + bh * a.nb;
  uint8_t *df = distflag + bh * a.nb;
#pragma unroll 4
  for (int u = 0; u < kFlagU; ++u) {
    const int t = (blockIdx.x * kFlagU + u) * 256 + threadIdx.x;
    if (t >= a.n || !kept(score_bits(line[t]), uint32_t(t), s)) continue;
    if (slot % 2 == 0) {
      cf[t / a.bs] = 1;
    } else {
      const int d0 = t / a.bs;
      df[d0] = 1;
      if (t % a.bs != 0 && d0 + 1 < a.nb) df[d0 + 1] = 1;
    }
  }
}

// grid (ceil(nb/8), Hq, Bt), 256 threads: one warp per row, kEmitU groups of
// 32 entries in flight.
constexpr int kEmitU = 4;
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
  constexpr int kU = kEmitU;
  for (int j0 = 0; j0 <= qi; j0 += 32 * kU) {
    bool keep[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int j = j0 + u * 32 + lane;
      keep[u] = false;
      if (j <= qi) {
        if (j == qi)
          keep[u] = true;
        else if (qa)
          keep[u] = kept(score_bits(mrow[j]), uint32_t(rowbase + j), s);
        else
          keep[u] = cf[j] || df[qi - j];
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const unsigned bal = __ballot_sync(0xffffffffu, keep[u]);
      if (keep[u]) out[cnt + __popc(bal & ((1u << lane) - 1u))] = j0 + u * 32 + lane;
      cnt += __popc(bal);
    }
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
  const int len = min(bs, n - c * bs);  // a partial last block: its real lines
  double av = 0.0, as = 0.0;
  for (int t = 0; t < len; ++t) {
    av += (double)v[t];
    as += (double)s[t];
  }
  pv[bh * nb + c] = __double2float_rn(av);
  ps[bh * nb + c] = __double2float_rn(as);
}

// Query-wise rule: grid (ceil(nb / kRowWarps), Hq, Bt), kRowWarps warps; warp
// w selects row qi = blockIdx.x * kRowWarps + w of a query-aware head (others
// return at once).  The row A[qi, 0..qi] takes the same radix select as the
// flattened lists, on four digits of its scores' bit patterns (bits 30..23,
// 22..15, 14..7, 6..0), with a warp-private shared histogram per digit and
// the decisions (by mass, or by count once the row's budget clamp decides k)
// taken by the whole warp from warp scans; then the tie rank by an ordered
// count, and the row's ascending list with its diagonal.  Integer sums, so
// the result does not depend on thread order.
constexpr int kRowWarps = 8;
constexpr int kRowLevels = 4;  // digits: bits 30..23, 22..15, 14..7, 6..0

struct RowHist {
  unsigned lo[256], hi[256], cnt[256];  // mass as its low 16 bits and the rest
};

// Warp-inclusive scan of a 64-bit value (lane order).
__device__ __forceinline__ unsigned long long warp_incl_scan(unsigned long long x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// The first bin of h[0, nbins), scanning from the top, at which base + the
// cumulative mass reaches target_m (by_mass) or base_c + the cumulative count
// reaches target_c; the sums of the bins above it.  Whole warp; lane l takes
// bins nbins-1-l*per .. nbins-per-l*per.  With no crossing (not reached for
// valid targets) the lowest bin.
__device__ Crossing row_crossing(const RowHist &h, int nbins, bool by_mass, double target_m,
                                 unsigned long long base_m, unsigned long long target_c,
                                 unsigned long long base_c, int lane) {
  const int per = nbins / 32;
  unsigned long long lm = 0, lc = 0;
  for (int k = 0; k < per; ++k) {
    const int b = nbins - 1 - lane * per - k;
    lm += (unsigned long long)h.lo[b] + ((unsigned long long)h.hi[b] << 16);
    lc += h.cnt[b];
  }
  const unsigned long long im = warp_incl_scan(lm, lane), ic = warp_incl_scan(lc, lane);
  const unsigned long long em = im - lm, ec = ic - lc;
  auto reach = [&](unsigned long long m, unsigned long long c) {
    return by_mass ? (double)(base_m + m) >= target_m : (base_c + c) >= target_c;
  };
  const unsigned hit = __ballot_sync(0xffffffffu, !reach(em, ec) && reach(im, ic));
  Crossing cr;
  if (hit == 0u) {  // fallback: the lowest bin, everything else above it
    const unsigned long long tm = __shfl_sync(0xffffffffu, im, 31);
    const unsigned long long tc = __shfl_sync(0xffffffffu, ic, 31);
    cr.bin = 0u;
    cr.above_m = tm - ((unsigned long long)h.lo[0] + ((unsigned long long)h.hi[0] << 16));
    cr.above_c = tc - h.cnt[0];
    return cr;
  }
  const int src = __ffs(hit) - 1;
  uint32_t bin = 0u;
  unsigned long long am = 0, ac = 0;
  if (lane == src) {
    unsigned long long cm = em, cc = ec;
    for (int k = 0; k < per; ++k) {
      const int b = nbins - 1 - lane * per - k;
      const unsigned long long m = (unsigned long long)h.lo[b] + ((unsigned long long)h.hi[b] << 16);
      if (reach(cm + m, cc + h.cnt[b])) {
        bin = uint32_t(b);
        am = cm;
        ac = cc;
        break;
      }
      cm += m;
      cc += h.cnt[b];
    }
  }
  cr.bin = __shfl_sync(0xffffffffu, bin, src);
  cr.above_m = __shfl_sync(0xffffffffu, am, src);
  cr.above_c = __shfl_sync(0xffffffffu, ac, src);
  return cr;
}

__global__ void __launch_bounds__(kRowWarps * 32) select_rows_qa_kernel(
    const int32_t *__restrict__ pattern, const float *__restrict__ map, int nb, float gamma,
    int row_lo, int row_hi, int32_t *__restrict__ counts, int32_t *__restrict__ indices) {
  __shared__ RowHist hist[kRowWarps];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const size_t bh = size_t(blockIdx.z) * gridDim.y + blockIdx.y;
  if (pattern[bh] != FP_PATTERN_QA) return;
  const int qi = blockIdx.x * kRowWarps + warp;
  if (qi >= nb) return;  // (no CTA-wide barrier below)
  RowHist &h = hist[warp];
  const int n = qi + 1;
  const float *mrow = map + bh * (size_t(nb) * (nb + 1) / 2) + size_t(qi) * (qi + 1) / 2;
  const unsigned long long lo = (unsigned long long)(row_lo < n ? row_lo : n);
  const unsigned long long hi0 = row_hi < 0 ? n : (row_hi < n ? row_hi : n);
  const unsigned long long blo = lo < hi0 ? lo : hi0, bhi = hi0;
  // the rule's state (warp-uniform)
  int mode = -1;  // SEL_* once decided by the clamp alone
  bool by_mass = false;
  double target_m = 0.0;
  unsigned long long target_c = 0, am = 0, ac = 0;
  uint32_t prefix = 0;
  auto count_mode = [&](unsigned long long k) {
    by_mass = false;
    target_c = k;
    if (k == 0) mode = SEL_NONE;
    else if (k >= (unsigned long long)n) mode = SEL_ALL;
  };
  {
    unsigned long long w = 0;
    for (int j = lane; j < n; j += 32) w += score_mass(score_bits(mrow[j]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) w += __shfl_xor_sync(0xffffffffu, w, o);
    if (gamma >= 1.f) {
      count_mode(bhi);  // k_gamma = n, clamped
    } else {
      target_m = (double)gamma * (double)w;
      if (target_m <= 0.0) count_mode(blo);  // k_gamma = 0
      else by_mass = true;
    }
  }
  for (int lv = 0; lv < kRowLevels && mode < 0; ++lv) {
    const int width = lv < 3 ? 8 : 7;
    const int shift = lv < 3 ? 23 - 8 * lv : 0, nbins = 1 << width;
    const int top = shift + width;  // the bits above this digit are fixed
    for (int b = lane; b < 256; b += 32) {
      h.lo[b] = 0u;
      h.hi[b] = 0u;
      h.cnt[b] = 0u;
    }
    __syncwarp();
    for (int j = lane; j < n; j += 32) {
      const uint32_t x = score_bits(mrow[j]);
      if (top >= 31 || (x >> top) == (prefix >> top)) {
        const uint32_t b = (x >> shift) & uint32_t(nbins - 1);
        const uint64_t w = score_mass(x);
        atomicAdd(&h.lo[b], unsigned(w & 0xFFFFull));
        atomicAdd(&h.hi[b], unsigned(w >> 16));
        atomicAdd(&h.cnt[b], 1u);
      }
    }
    __syncwarp();
    Crossing cr;
    if (by_mass) {
      cr = row_crossing(h, nbins, true, target_m, am, 0, 0, lane);
      const unsigned long long A = ac + cr.above_c, C = h.cnt[cr.bin];
      if (bhi <= A) count_mode(bhi);
      else if (blo >= A + C) count_mode(blo);
      if (mode >= 0) break;
    }
    if (!by_mass) cr = row_crossing(h, nbins, false, 0.0, 0, target_c, ac, lane);
    am += cr.above_m;
    ac += cr.above_c;
    prefix |= cr.bin << shift;
    __syncwarp();  // the histogram is cleared for the next digit
  }
  uint32_t tb = 0u, tidx = 0u;  // kept: bits > tb, or bits == tb and j <= tidx
  if (mode < 0) {
    const uint32_t b = prefix;
    unsigned long long m;
    if (by_mass) {
      const unsigned long long w = score_mass(b);
      unsigned long long mm = 1;
      if (w > 0) {
        const double need = (target_m - (double)am) / (double)w;
        mm = need <= 1.0 ? 1ull : (unsigned long long)ceil(need);
        while (mm > 1 && (double)(am + (mm - 1) * w) >= target_m) --mm;
        while ((double)(am + mm * w) < target_m) ++mm;
      }
      unsigned long long k = ac + mm;
      k = k < blo ? blo : (k > bhi ? bhi : k);
      m = k - ac;
    } else {
      m = target_c - ac;
    }
    // the m-th (1-based) entry with pattern b, in index order
    unsigned long long seen = 0;
    uint32_t idx = uint32_t(n - 1);
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      const bool hit = j < n && score_bits(mrow[j]) == b;
      const unsigned bal = __ballot_sync(0xffffffffu, hit);
      const unsigned c = __popc(bal);
      if (seen + c >= m) {
        unsigned x = bal;
        for (unsigned long long r = seen + 1; r < m; ++r) x &= x - 1;
        idx = uint32_t(j0 + __ffs(x) - 1);
        break;
      }
      seen += c;
    }
    tb = b;
    tidx = idx;
  }
  const HeadSel s{mode < 0 ? SEL_THRESHOLD : mode, tb, tidx, 0};
  int32_t *out = indices + (bh * nb + qi) * size_t(nb);
  int cnt = 0;
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    const bool keep = j < n && (j == qi || kept(score_bits(mrow[j]), uint32_t(j), s));
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) out[cnt + __popc(bal & ((1u << lane) - 1u))] = j;
    cnt += __popc(bal);
  }
  if (lane == 0) counts[bh * nb + qi] = cnt;
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

// Streaming multiprocessors of the current device (cached per device).
int sm_count() {
  static std::atomic<int> cache[64];  // 0 = not yet read
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
      n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

size_t select_ws_bytes(const Dims &D) {
  Carver c{nullptr, 0};
  const size_t heads = size_t(D.bt) * D.hq, slots = 2 * heads;
  c.take<HeadSel>(slots);
  c.take<uint8_t>(heads * D.nb);
  c.take<uint8_t>(heads * D.nb);
  c.take<ListState>(slots);
  c.take<unsigned long long>(slots * kBins);
  c.take<unsigned int>(slots * kBins);
  c.take<uint2>(slots * kCand);
  return c.off + 256;
}

cudaError_t launch_select(const Dims &D, float gamma, const SelectBudgets &bud,
                          const int32_t *pattern, const float *map, const float *vert,
                          const float *slash, int32_t *counts, int32_t *indices, void *ws,
                          cudaStream_t st) {
  if (D.nb > kMaxBlocks) return cudaErrorInvalidValue;
  Carver c{static_cast<char *>(ws), 0};
  const size_t heads = size_t(D.bt) * D.hq;
  const int slots = int(2 * heads);
  SelArgs a;
  a.sel = c.take<HeadSel>(slots);
  uint8_t *cf = c.take<uint8_t>(heads * D.nb);
  uint8_t *df = c.take<uint8_t>(heads * D.nb);
  a.state = c.take<ListState>(slots);
  a.hm = c.take<unsigned long long>(size_t(slots) * kBins);
  a.hc = c.take<unsigned int>(size_t(slots) * kBins);
  a.cand = c.take<uint2>(size_t(slots) * kCand);
  a.pattern = pattern;
  a.map = map;
  a.vert = vert;
  a.slash = slash;
  a.n = D.n;
  a.nb = D.nb;
  a.bs = D.bs;
  a.gamma = gamma;
  a.qa_lo = bud.qa_lo;
  a.qa_hi = bud.qa_hi;
  a.vs_lo = bud.vs_lo;
  a.vs_hi = bud.vs_hi;
  a.qa_mode = bud.qa_mode;
  if (bud.vs_mode == FP_VS_BLOCKS) {
    // pooled lines live in the outputs until emit_rows_kernel overwrites them:
    // vert sums in indices (>= Bt*Hq*nb entries), slash sums in counts; they
    // are then lines of nb tokens with block size 1
    float *pv = reinterpret_cast<float *>(indices);
    float *ps = reinterpret_cast<float *>(counts);
    pool_lines_kernel<<<dim3((D.nb + 255) / 256, D.hq, D.bt), 256, 0, st>>>(
        pattern, vert, slash, D.n, D.nb, D.bs, pv, ps);
    a.vert = pv;
    a.slash = ps;
    a.n = D.nb;
    a.bs = 1;
    a.vs_lo = bud.vsb_lo;
    a.vs_hi = bud.vsb_hi;
  }
  long long maxlen = a.n;
  if (bud.qa_mode == FP_QA_FLATTENED && D.t_pairs > maxlen) maxlen = D.t_pairs;
  const int max_chunks = int((maxlen + 3 + kChunk - 1) / kChunk);
  // about `per_sm` CTAs per SM over all slots, each looping over chunks, and
  // enough of them that no CTA takes more than kMaxCtaChunks; every scanning
  // kernel derives its CTAs per list from its own args (the decisions are
  // integer sums, the same for any count)
  auto with_ctas = [&](int per_sm) {
    SelArgs x = a;
    x.ctas = std::max(1, std::min(max_chunks, sm_count() * per_sm / slots));
    x.ctas = std::max(x.ctas, (max_chunks + kMaxCtaChunks - 1) / kMaxCtaChunks);
    return x;
  };
  const SelArgs a1 = with_ctas(kHist1CtasPerSm), a2 = with_ctas(kHist2CtasPerSm),
                a3 = with_ctas(kCompactCtasPerSm);
  cudaFuncSetAttribute(sel_hist_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       int(hist_smem<2>()));
  sel_prep_kernel<<<slots, kSelThreads, 0, st>>>(a1, cf, df);
  sel_hist_kernel<1><<<dim3(unsigned(a1.ctas), slots), kSelThreads, hist_smem<1>(), st>>>(a1);
  sel_hist_kernel<2><<<dim3(unsigned(a2.ctas), slots), kSelThreads, hist_smem<2>(), st>>>(a2);
  sel_compact_kernel<<<dim3(unsigned(a3.ctas), slots), kSelThreads, 0, st>>>(a3);
  sel_flags_kernel<<<dim3((a.n + 256 * kFlagU - 1) / (256 * kFlagU), slots), 256, 0, st>>>(
      a, cf, df);
  emit_rows_kernel<<<dim3((D.nb + 7) / 8, D.hq, D.bt), 256, 0, st>>>(
      pattern, map, D.nb, a.sel, cf, df, bud.qa_mode, counts, indices);
  if (bud.qa_mode == FP_QA_QUERYWISE)
    select_rows_qa_kernel<<<dim3((D.nb + kRowWarps - 1) / kRowWarps, D.hq, D.bt),
                            kRowWarps * 32, 0, st>>>(pattern, map, D.nb, gamma, bud.row_lo,
                                                     bud.row_hi, counts, indices);
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
// first call made with that device current) and cached.  What must start at
// zero (histograms, counters, flags) is cleared by sel_prep_kernel, the
// first launch of every call.
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
