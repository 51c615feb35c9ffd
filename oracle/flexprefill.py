"""CPU oracle for the FlexPrefill prefill-attention hot path.

TEST INFRASTRUCTURE.  This module is a plain, slow, obviously-correct
restatement of what the method computes, used to check the CUDA library.
Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import it.  It shares no code with the CUDA path and imports nothing
from the product package; callers hand it arrays.

Sources (cited by page and section):
  [abstract]  FlexPrefill: A Context-Aware Sparse Attention Mechanism for
              Efficient Long-Sequence Inference -- abstract (codewithpapers and
              OpenReview pages): the two components, "Query-Aware Sparse Pattern
              Determination" via Jensen-Shannon divergence and
              "Cumulative-Attention Based Index Selection".
  [approach]  Same title, atlas.scime.ai AI-extracted summary, section
              "Approach": per head, a block-pooled estimate built from the last
              query block is compared with the true distribution by the square
              root of the JS divergence; query-aware block selection if the
              estimate is accurate, vertical-slash otherwise; then the smallest
              set of blocks/lines whose cumulative normalised attention passes
              gamma.
  [ablations] Same summary, table "Measured effects reported in the paper":
              tau = 0 disables query-aware mode; min budget (1024/2048 tokens);
              max budget (8k/32k tokens); block size 64/128; last (not middle)
              representative queries; the flattened estimated map, with
              query-wise selection as the alternative the ablation compares.

Where the pages are silent the plainest reading is taken; each is named at the
function that makes it.  Floating point runs in float64 except where a float
decides an integer (the selection rule), where the decision is taken on
float32 scores exactly as the kernels receive them.

Every function here is pinned by ``tests/test_oracle_*.py`` against closed
forms, library routines (torch SDPA, scipy's Jensen-Shannon distance) or brute
force; none is "parity unpinned".

Layouts (all C-contiguous):
  q [Bt, Hq, N, d];  k, v [Bt, Hkv, N, d];  g = Hq // Hkv;  kv head of h = h // g
  nb = ceil(N / B);  T = nb (nb + 1) / 2 (causal block pairs).  When B does not
  divide N the last block is partial: it holds the N - (nb - 1) B tokens left
  (reading of a sequence of any length: the pages define the method per
  sequence and never tie N to B), and every block-level step uses that
  block's real tokens only.
  map   [Bt, Hq, T]: row i of the block map stored at i(i+1)/2 .. i(i+1)/2 + i
  counts [Bt, Hq, nb] int32; indices [Bt, Hq, nb, nb] int32, first counts[...]
  entries of each row ascending, the rest unspecified.
"""
from __future__ import annotations

import math

import numpy as np

PATTERN_QA = 0
PATTERN_VS = 1
QA_FLATTENED = 0  # query-aware heads: one cumulative rule over the flattened map
QA_QUERYWISE = 1  # query-aware heads: one cumulative rule per query-block row
VS_TOKENS = 0     # vertical-slash heads: lines chosen per token, then a block cover
VS_BLOCKS = 1     # vertical-slash heads: lines pooled per block before the rule
QUANT_SCALE = 2.0 ** 32  # selection masses are integers: ceil(score * 2^32)


def _f64(x) -> np.ndarray:
    """Upcast a numpy array or torch tensor (fp32 / bf16) to float64 numpy."""
    if hasattr(x, "detach"):  # torch tensor: bf16 has no numpy dtype
        return x.detach().to(dtype=__import__("torch").float64).cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def _f32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        return x.detach().to(dtype=__import__("torch").float32).cpu().numpy()
    return np.asarray(x, dtype=np.float32)


def tri_offset(i: int) -> int:
    """Start of block-map row i in the packed lower triangle."""
    return i * (i + 1) // 2


# ---------------------------------------------------------------- estimate --

def n_blocks_of(n: int, block: int) -> int:
    """ceil(N / B): the blocks of a sequence of N tokens (the last may be partial)."""
    return -(-n // block)


def block_pool(x, block: int) -> np.ndarray:
    """Mean over each run of ``block`` tokens: [..., N, d] -> [..., nb, d].

    [approach] says the estimate is "block-pooled"; the operator is not
    named.  Reading: arithmetic mean, over the real tokens of a partial last
    block.
    """
    x = _f64(x)
    *lead, n, d = x.shape
    nb = n_blocks_of(n, block)
    out = np.empty((*lead, nb, d))
    for c in range(nb):
        out[..., c, :] = x[..., c * block: min((c + 1) * block, n), :].mean(axis=-2)
    return out


def estimated_block_map(qbar: np.ndarray, kbar: np.ndarray, scale: float):
    """Causal softmax over key blocks of the pooled logits, one head.

    qbar [nb, d], kbar [nb, d] -> A [nb, nb] with A[i, j] = 0 for j > i and
    each row i a softmax over j <= i of scale * qbar[i] . kbar[j].
    [approach] "block-pooled attention"; reading: the same 1/sqrt(d) scale as
    attention, causal at block granularity (block j visible to block i iff
    j <= i).
    """
    nb = qbar.shape[0]
    logits = scale * (qbar @ kbar.T)
    a = np.zeros((nb, nb))
    for i in range(nb):
        row = logits[i, : i + 1]
        e = np.exp(row - row.max())
        a[i, : i + 1] = e / e.sum()
    return a


def last_block_attention(q_last: np.ndarray, k: np.ndarray, n_total: int, scale: float):
    """True causal attention probabilities of the last query block, one head.

    q_last [R, d] holds the queries at positions N-R .. N-1 (R = B, or the
    partial last block's length); k [N, d].  Returns P [R, N] with P[r, t] =
    softmax over t <= N-R+r of scale*q.k, and 0 for t > N-R+r.  [approach]
    "the true distribution" of the last query block ([ablations]: last, not
    middle, representative queries).
    """
    bsz = q_last.shape[0]
    logits = scale * (q_last @ k.T)
    p = np.zeros((bsz, n_total))
    for r in range(bsz):
        pos = n_total - bsz + r
        row = logits[r, : pos + 1]
        e = np.exp(row - row.max())
        p[r, : pos + 1] = e / e.sum()
    return p


def estimate(q, k, block: int):
    """All outputs of the estimate step for every (batch, q head).

    Returns a dict of float64 arrays:
      qbar [Bt,Hq,nb,d], kbar [Bt,Hkv,nb,d]   block means (block_pool)
      map [Bt,Hq,T]          packed lower triangle of estimated_block_map
      est_last [Bt,Hq,nb]    last row of the map (the estimate a-hat)
      true_last [Bt,Hq,nb]   true pooled distribution a-bar of the last block:
                             P summed over the keys of each block and averaged
                             over the last block's R query rows (sums to 1).
                             Reading of "true distribution" [approach].
      vert [Bt,Hq,N]         column sums  vert[t]  = sum_r P[r, t]
      slash [Bt,Hq,N]        diagonal sums slash[o] = sum_r P[r, N-R+r-o]
                             (o = query position - key position >= 0)
    R = B, or the partial last block's length when B does not divide N.
    vert and slash are the vertical and slash line scores of the
    vertical-slash pattern [approach], read off the same last-block P.
    """
    qf, kf = _f64(q), _f64(k)
    bt, hq, n, d = qf.shape
    hkv = kf.shape[1]
    g = hq // hkv
    nb = n_blocks_of(n, block)
    q0 = (nb - 1) * block  # first query of the last block
    rows = n - q0
    t_pairs = nb * (nb + 1) // 2
    scale = 1.0 / math.sqrt(d)
    qbar = block_pool(qf, block)
    kbar = block_pool(kf, block)
    amap = np.zeros((bt, hq, t_pairs))
    est_last = np.zeros((bt, hq, nb))
    true_last = np.zeros((bt, hq, nb))
    vert = np.zeros((bt, hq, n))
    slash = np.zeros((bt, hq, n))
    for b in range(bt):
        for h in range(hq):
            kv = h // g
            a = estimated_block_map(qbar[b, h], kbar[b, kv], scale)
            for i in range(nb):
                amap[b, h, tri_offset(i): tri_offset(i) + i + 1] = a[i, : i + 1]
            est_last[b, h] = a[nb - 1]
            p = last_block_attention(qf[b, h, q0:], kf[b, kv], n, scale)
            for j in range(nb):
                true_last[b, h, j] = p[:, j * block: min((j + 1) * block, n)].sum() / rows
            vert[b, h] = p.sum(axis=0)
            for r in range(rows):
                pos = q0 + r
                # key t = pos - o for o = 0..pos
                slash[b, h, : pos + 1] += p[r, pos::-1]
    return {"qbar": qbar, "kbar": kbar, "map": amap, "est_last": est_last,
            "true_last": true_last, "vert": vert, "slash": slash}


# ----------------------------------------------------------------- pattern --

def js_distance(p, q) -> float:
    """Square root of the Jensen-Shannon divergence, natural log.

    [approach] "square-root JS divergence".  Readings: both inputs are first
    renormalised to sum 1 in float64; 0 * log 0 := 0; natural log, so the
    result lies in [0, sqrt(ln 2)].
    """
    p = _f64(p).ravel()
    q = _f64(q).ravel()
    p = p / p.sum()
    q = q / q.sum()
    m = 0.5 * (p + q)
    kl_pm = sum(pi * math.log(pi / mi) for pi, mi in zip(p, m) if pi > 0.0)
    kl_qm = sum(qi * math.log(qi / mi) for qi, mi in zip(q, m) if qi > 0.0)
    return math.sqrt(max(0.0, 0.5 * kl_pm + 0.5 * kl_qm))


def pattern(est_last, true_last, tau: float):
    """Per-head pattern choice: query-aware iff d_JS(a-hat, a-bar) < tau.

    [approach]: query-aware selection when the estimate is accurate,
    vertical-slash otherwise.  [ablations]: tau = 0 turns query-aware mode off,
    which fixes the comparison as strict (d_JS == tau goes to vertical-slash).
    Returns (djs [Bt,Hq] float64, pattern [Bt,Hq] int32).
    """
    e = _f64(est_last)
    t = _f64(true_last)
    bt, hq, _ = e.shape
    djs = np.zeros((bt, hq))
    pat = np.zeros((bt, hq), dtype=np.int32)
    for b in range(bt):
        for h in range(hq):
            djs[b, h] = js_distance(e[b, h], t[b, h])
            pat[b, h] = PATTERN_QA if djs[b, h] < float(np.float32(tau)) else PATTERN_VS
    return djs, pat


# --------------------------------------------------------------- selection --

def quantised_masses(scores_f32: np.ndarray) -> list:
    """Integer masses w = ceil(score * 2^32) (Python ints; exact).

    Reading: the cumulative test "cumulative normalised attention reaches
    gamma" [approach] is made order-independent by summing integers; a
    positive score always weighs at least 1.
    """
    s = np.asarray(scores_f32, dtype=np.float32).astype(np.float64)
    return [int(math.ceil(x * QUANT_SCALE)) for x in s]


def cumulative_count(scores_f32, gamma: float) -> int:
    """Smallest k (0..n) whose top-k quantised mass reaches gamma * total.

    Order: score descending, then index ascending.  target is one float64
    multiply (double)gamma_f32 * (double)W; cum_k >= target ("reaches";
    reading of "exceeds" vs "reaches").  gamma >= 1 selects every entry.
    """
    s = np.asarray(scores_f32, dtype=np.float32)
    n = s.size
    g32 = float(np.float32(gamma))
    if g32 >= 1.0:
        return n
    order = np.argsort(-s, kind="stable")
    w = quantised_masses(s[order])
    total = sum(w)
    target = g32 * float(total)
    cum = 0
    if float(cum) >= target:
        return 0
    for k, wi in enumerate(w, start=1):
        cum += wi
        if float(cum) >= target:
            return k
    return n


def cumulative_select(scores_f32, gamma: float, lo: int, hi: int) -> np.ndarray:
    """Indices of the selected entries, in selection order.

    k = clamp(cumulative_count, lo, hi) with lo <= hi <= n, then the first k
    entries of the (score desc, index asc) order.  [approach] smallest set
    reaching gamma; [ablations] min / max computational budgets.
    """
    s = np.asarray(scores_f32, dtype=np.float32)
    k = cumulative_count(s, gamma)
    k = min(max(k, lo), hi)
    order = np.argsort(-s, kind="stable")
    return order[:k]


def qa_budget(n_blocks: int, block: int, min_budget: int, max_budget: int):
    """(lo, hi) for the flattened query-aware map, counted in block pairs.

    Reading: budgets are tokens per query row, so min_budget tokens buy
    ceil(min_budget / B) key blocks in each of the nb rows; max_budget tokens
    cap at floor(max_budget / B) per row.  max_budget <= 0: uncapped.
    """
    t_pairs = n_blocks * (n_blocks + 1) // 2
    lo = min(t_pairs, n_blocks * (-(-max(min_budget, 0) // block)))
    hi = t_pairs if max_budget <= 0 else min(t_pairs, n_blocks * (max_budget // block))
    return min(lo, hi), hi


def vs_budget(n_tokens: int, min_budget: int, max_budget: int):
    """(lo, hi) for each vertical or slash line list, counted in lines (tokens)."""
    lo = min(n_tokens, max(min_budget, 0))
    hi = n_tokens if max_budget <= 0 else min(n_tokens, max_budget)
    return min(lo, hi), hi


def slash_block_distances(offset: int, block: int) -> list:
    """Block distances qi - j of the block pairs holding a point with i - t == offset."""
    d0 = offset // block
    return [d0] if offset % block == 0 else [d0, d0 + 1]


def select_head_qa(map_row_f32: np.ndarray, n_blocks: int, block: int, gamma: float,
                   min_budget: int, max_budget: int):
    """Per-row block lists of one query-aware head.

    The packed map is flattened [ablations: flattened, not query-wise],
    selected with cumulative_select, and every row also keeps its diagonal
    block (reading: forced so that each causal query row sees a key).
    Returns a list of nb sorted lists.
    """
    lo, hi = qa_budget(n_blocks, block, min_budget, max_budget)
    chosen = cumulative_select(map_row_f32, gamma, lo, hi)
    rows = [set([i]) for i in range(n_blocks)]
    # packed index p -> (i, j): i is the largest with i(i+1)/2 <= p
    for p in chosen.tolist():
        i = int((math.isqrt(8 * p + 1) - 1) // 2)
        j = p - tri_offset(i)
        rows[i].add(j)
    return [sorted(r) for r in rows]


def qa_row_budget(row: int, block: int, min_budget: int, max_budget: int):
    """(lo, hi) for row ``row`` of a query-wise head, counted in its row+1 key blocks.

    Reading: the same tokens-per-query-row budgets as the flattened rule,
    applied to the one row: ceil(min_budget / B) blocks at least and
    floor(max_budget / B) at most, never more than the row holds.
    """
    n = row + 1
    lo = min(n, -(-max(min_budget, 0) // block))
    hi = n if max_budget <= 0 else min(n, max_budget // block)
    return min(lo, hi), hi


def select_head_qa_querywise(map_row_f32: np.ndarray, n_blocks: int, block: int,
                             gamma: float, min_budget: int, max_budget: int):
    """Per-row block lists of one query-aware head, selected row by row.

    [ablations] "query-wise index selection instead of flattening the
    estimated attention map": the cumulative rule (cumulative_select, same
    order, masses and target) runs on each query-block row i of the map,
    A[i, 0..i], with the row's own total, and the row's budgets from
    qa_row_budget; every row also keeps its diagonal block.
    """
    m = np.asarray(map_row_f32, dtype=np.float32)
    rows = []
    for i in range(n_blocks):
        seg = m[tri_offset(i): tri_offset(i) + i + 1]
        lo, hi = qa_row_budget(i, block, min_budget, max_budget)
        chosen = cumulative_select(seg, gamma, lo, hi)
        rows.append(sorted(set(chosen.tolist()) | {i}))
    return rows


def select_head_vs(vert_f32: np.ndarray, slash_f32: np.ndarray, n_blocks: int, block: int,
                   gamma: float, min_budget: int, max_budget: int):
    """Per-row block lists of one vertical-slash head.

    The vertical lines (key columns) and slash lines (query-key offsets) are
    each selected with cumulative_select.  A column t covers key block t // B
    in every row; an offset o covers the block pairs at distance
    slash_block_distances(o).  Reading of "blocks/lines" [approach]: lines
    are chosen at token granularity and mapped to the blocks that hold them.
    """
    n = vert_f32.size
    lo, hi = vs_budget(n, min_budget, max_budget)
    cols = cumulative_select(vert_f32, gamma, lo, hi)
    offs = cumulative_select(slash_f32, gamma, lo, hi)
    col_blocks = set(int(t) // block for t in cols.tolist())
    dists = set()
    for o in offs.tolist():
        dists.update(slash_block_distances(int(o), block))
    rows = []
    for qi in range(n_blocks):
        r = {j for j in range(qi + 1) if j in col_blocks or (qi - j) in dists}
        r.add(qi)
        rows.append(sorted(r))
    return rows


def pool_lines(line_f32: np.ndarray, n_blocks: int, block: int) -> np.ndarray:
    """Block sums of a vertical (per key) or slash (per offset) score line.

    Entry c of the result sums the scores of tokens / offsets c*B .. c*B+B-1:
    a key block's column mass, or the mass of the offsets whose primary block
    distance is c (floor(o / B)).  Reading: the sum runs in float64, one add
    at a time in ascending order, and is rounded to float32 once at the end;
    the kernels take the same steps, so both select on identical scores.
    """
    x = np.asarray(line_f32, dtype=np.float32)
    out = np.empty(n_blocks, dtype=np.float32)
    for c in range(n_blocks):
        acc = 0.0
        for v in x[c * block: (c + 1) * block].tolist():
            acc += v
        out[c] = np.float32(acc)
    return out


def vs_block_budget(n_blocks: int, block: int, min_budget: int, max_budget: int):
    """(lo, hi) for each pooled line list, counted in blocks (tokens / B)."""
    lo = min(n_blocks, -(-max(min_budget, 0) // block))
    hi = n_blocks if max_budget <= 0 else min(n_blocks, max_budget // block)
    return min(lo, hi), hi


def select_head_vs_blocks(vert_f32: np.ndarray, slash_f32: np.ndarray, n_blocks: int,
                          block: int, gamma: float, min_budget: int, max_budget: int):
    """Per-row block lists of one vertical-slash head, from block-pooled lines.

    The block-level reading of "blocks/lines" [approach]: the vertical
    scores are summed per key block and the slash scores per block distance
    (pool_lines) before the cumulative rule, so the rule and its budgets count
    whole blocks.  Column block j is kept in every row; block
    distance d keeps the pairs (qi, qi - d); every row keeps its diagonal.
    """
    vb = pool_lines(vert_f32, n_blocks, block)
    sb = pool_lines(slash_f32, n_blocks, block)
    lo, hi = vs_block_budget(n_blocks, block, min_budget, max_budget)
    cols = set(cumulative_select(vb, gamma, lo, hi).tolist())
    dists = set(cumulative_select(sb, gamma, lo, hi).tolist())
    return [sorted({j for j in range(qi + 1) if j in cols or (qi - j) in dists} | {qi})
            for qi in range(n_blocks)]


def select(pattern_arr, amap, vert, slash, n_blocks: int, block: int, gamma: float,
           min_budget: int, max_budget: int, qa_mode: int = QA_FLATTENED,
           vs_mode: int = VS_TOKENS):
    """Block lists for every (batch, head): counts [Bt,Hq,nb], indices [Bt,Hq,nb,nb].

    Scores are taken as float32 (the precision the kernels decide in).  Unused
    tail entries of each indices row are set to -1 here.  qa_mode picks the
    flattened or the query-wise rule for query-aware heads, vs_mode the token
    or the block-pooled lines for vertical-slash heads.
    """
    pat = np.asarray(pattern_arr)
    m32, v32, s32 = _f32(amap), _f32(vert), _f32(slash)
    bt, hq = pat.shape
    counts = np.zeros((bt, hq, n_blocks), dtype=np.int32)
    indices = np.full((bt, hq, n_blocks, n_blocks), -1, dtype=np.int32)
    for b in range(bt):
        for h in range(hq):
            if pat[b, h] == PATTERN_QA and qa_mode == QA_QUERYWISE:
                rows = select_head_qa_querywise(m32[b, h], n_blocks, block, gamma, min_budget,
                                                max_budget)
            elif pat[b, h] == PATTERN_QA:
                rows = select_head_qa(m32[b, h], n_blocks, block, gamma, min_budget, max_budget)
            elif vs_mode == VS_BLOCKS:
                rows = select_head_vs_blocks(v32[b, h], s32[b, h], n_blocks, block, gamma,
                                             min_budget, max_budget)
            else:
                rows = select_head_vs(v32[b, h], s32[b, h], n_blocks, block, gamma,
                                      min_budget, max_budget)
            for i, r in enumerate(rows):
                counts[b, h, i] = len(r)
                indices[b, h, i, : len(r)] = r
    return counts, indices


# --------------------------------------------------------------- attention --

def sparse_attention(q, k, v, counts, indices, block: int, heads=None, q_blocks=None):
    """Causal attention restricted to the listed key blocks, in float64.

    Row qi of head h attends to the keys of blocks indices[b,h,qi,:counts]
    with key position <= query position; softmax of scale * q.k (scale
    1/sqrt(d)), times V.  GQA: kv head = h // g.  Returns (out, lse) with lse
    the natural-log log-sum-exp of the scaled logits.  ``heads`` /
    ``q_blocks`` restrict the work to a sample (other outputs stay NaN).
    """
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    bt, hq, n, d = qf.shape
    g = hq // kf.shape[1]
    nb = n_blocks_of(n, block)
    scale = 1.0 / math.sqrt(d)
    out = np.full((bt, hq, n, d), np.nan)
    lse = np.full((bt, hq, n), np.nan)
    cnt = np.asarray(counts)
    idx = np.asarray(indices)
    hs = range(hq) if heads is None else heads
    qbs = range(nb) if q_blocks is None else q_blocks
    for b in range(bt):
        for h in hs:
            kv = h // g
            for qi in qbs:
                blocks = [int(j) for j in idx[b, h, qi, : cnt[b, h, qi]]]
                keys = np.concatenate([np.arange(j * block, min((j + 1) * block, n))
                                       for j in blocks])
                q1 = min((qi + 1) * block, n)  # (a partial last block ends at N)
                qrows = qf[b, h, qi * block:q1]
                logits = scale * (qrows @ kf[b, kv, keys].T)
                qpos = np.arange(qi * block, q1)
                logits = np.where(keys[None, :] <= qpos[:, None], logits, -np.inf)
                mx = logits.max(axis=1, keepdims=True)
                e = np.exp(logits - mx)
                s = e.sum(axis=1, keepdims=True)
                out[b, h, qi * block:q1] = (e / s) @ vf[b, kv, keys]
                lse[b, h, qi * block:q1] = (mx + np.log(s))[:, 0]
    return out, lse


def dense_lists(bt: int, hq: int, n_blocks: int):
    """Full causal lists: row qi holds blocks 0..qi."""
    counts = np.tile(np.arange(1, n_blocks + 1, dtype=np.int32), (bt, hq, 1))
    indices = np.full((bt, hq, n_blocks, n_blocks), -1, dtype=np.int32)
    for i in range(n_blocks):
        indices[:, :, i, : i + 1] = np.arange(i + 1, dtype=np.int32)
    return counts, indices


def dense_attention(q, k, v, block: int, heads=None, q_blocks=None):
    """Dense causal attention: sparse_attention over the full causal lists."""
    qf = _f64(q)
    bt, hq, n, _ = qf.shape
    counts, indices = dense_lists(bt, hq, n_blocks_of(n, block))
    return sparse_attention(qf, k, v, counts, indices, block, heads, q_blocks)


# ---------------------------------------------------------------- pipeline --

def flexprefill(q, k, v, block: int, gamma: float, tau: float, min_budget: int,
                max_budget: int, attention: bool = True, heads=None, q_blocks=None,
                qa_mode: int = QA_FLATTENED, vs_mode: int = VS_TOKENS):
    """Whole hot path: estimate -> pattern -> select -> sparse attention.

    The selection stage sees float32 copies of the estimate (the precision the
    kernels store); returns a dict with every intermediate.
    """
    est = estimate(q, k, block)
    e32 = {key: est[key].astype(np.float32) for key in ("map", "est_last", "true_last",
                                                         "vert", "slash")}
    djs, pat = pattern(e32["est_last"], e32["true_last"], tau)
    nb = n_blocks_of(_f64(q).shape[2], block)
    counts, indices = select(pat, e32["map"], e32["vert"], e32["slash"], nb, block, gamma,
                             min_budget, max_budget, qa_mode, vs_mode)
    res = dict(est)
    res.update(djs=djs, pattern=pat, counts=counts, indices=indices)
    if attention:
        out, lse = sparse_attention(q, k, v, counts, indices, block, heads, q_blocks)
        res.update(out=out, lse=lse)
    return res
