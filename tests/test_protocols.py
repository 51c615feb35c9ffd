"""CPU model checks of the mbarrier protocols of the pipelined tensor-core
kernels (csrc/attn_tc.cu, csrc/map_tc.cu and csrc/estimate_tc.cu).

Each role of a kernel (TMA producer, MMA issuer, softmax or epilogue warps) is
a Python generator that takes the kernel's waits, arrivals and buffer accesses
in the kernel's order; a scheduler interleaves them at random, and the tensor
pipe completes issued MMAs (and the arrivals their commits carry) in issue
order at random later times.  Checked, over many seeds and list lengths:
- every role finishes (no deadlock);
- no barrier receives more arrivals than its count in a phase;
- no buffer (ring slot, S, P, accumulator, staging tile) is written while a
  reader of its previous contents has not finished, and none is read while an
  MMA still writes it or before the generation the reader waits for.
The model abstracts the hardware (a TMA copy lands when issued, a 32-thread
warp is one agent); it checks the ordering logic, which a code change can
break without any numerical test noticing.  The last test removes one wait at
a time and checks that the model then reports a violation.
"""
import random

import pytest


class Bar:
    """An mbarrier: `count` arrivals complete a phase."""

    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, count, 0

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, f"{self.name}: more arrivals than its count"
        if self.pending == 0:
            self.done += 1
            self.pending = self.count

    def passes(self, parity):
        # try_wait.parity(P) passes once the phase of parity P has completed,
        # i.e. while the current (incomplete) phase has the other parity
        return (self.done & 1) != parity


class Buf:
    """A buffer's generation, its readers and its in-flight writes."""

    def __init__(self, name):
        self.name, self.gen, self.readers, self.writing = name, -1, 0, 0

    def write_begin(self, gen, fresh=True, exclusive=True):
        assert self.readers == 0, f"{self.name}: written while being read"
        # MMAs into one accumulator queue behind each other in the pipe; any
        # other write must not overlap one in flight
        assert not exclusive or self.writing == 0, f"{self.name}: written during an MMA"
        if fresh:
            assert gen == self.gen + 1, f"{self.name}: generation {gen} after {self.gen}"
            self.gen = gen
        else:
            assert gen == self.gen, f"{self.name}: accumulates into the wrong generation"
        self.writing += 1

    def write_end(self):
        self.writing -= 1

    def write(self, gen, fresh=True):
        self.write_begin(gen, fresh)
        self.write_end()

    def read_begin(self, gen):
        assert self.writing == 0, f"{self.name}: read while being written"
        assert self.gen == gen, f"{self.name}: read generation {gen}, holds {self.gen}"
        self.readers += 1

    def read_end(self):
        self.readers -= 1


class Pipe:
    """The tensor pipe: issued MMAs and commits complete in issue order."""

    def __init__(self):
        self.q = []

    def mma(self, reads, writes):
        for b, g in reads:
            b.read_begin(g)
        for b, g, fresh in writes:
            b.write_begin(g, fresh, exclusive=False)
        self.q.append(("mma", (reads, writes)))

    def commit(self, bar):
        self.q.append(("commit", bar))

    def step(self):
        kind, x = self.q.pop(0)
        if kind == "mma":
            reads, writes = x
            for b, _ in reads:
                b.read_end()
            for b, _, _ in writes:
                b.write_end()
        else:
            x.arrive()


def wait(bar, parity, skip=False):
    """Generator: spin until the phase of `parity` has completed."""
    while not skip and not bar.passes(parity):
        yield


def run(roles, pipe, rng, limit=1_000_000):
    live = list(roles)
    for _ in range(limit):
        if not live and not pipe.q:
            return
        if pipe.q and (not live or rng.random() < 0.3):
            pipe.step()
            continue
        r = rng.choice(live)
        try:
            next(r)
        except StopIteration:
            live.remove(r)
    raise AssertionError(f"deadlock: {len(live)} roles stuck, {len(pipe.q)} MMAs pending")


# ---------------------------------------------------------------- attention --
# attn_tc.cu: S (64 keys) single-buffered in TMEM, P single-buffered, K and V
# rings of 3 slots; the producer loads K(i) and V(i - 2) in turn; the MMA
# issuer runs S(t), then P(t-1) V(t-1); four softmax warps per CTA.

def attention_roles(ntile, NK=3, NV=3, warps=4, drop=None):
    pipe = Pipe()
    k_full = [Bar(f"k_full{s}", 1) for s in range(NK)]
    k_empty = [Bar(f"k_empty{s}", 1) for s in range(NK)]
    v_full = [Bar(f"v_full{s}", 1) for s in range(NV)]
    v_empty = [Bar(f"v_empty{s}", 1) for s in range(NV)]
    s_full, s_free = Bar("s_full", 1), Bar("s_free", warps)
    p_full, p_empty, o_full = Bar("p_full", warps), Bar("p_empty", 1), Bar("o_full", 1)
    K = [Buf(f"K{s}") for s in range(NK)]
    V = [Buf(f"V{s}") for s in range(NV)]
    S, P, O = Buf("S"), Buf("P"), Buf("O")
    p_stores = {}

    def producer():
        for i in range(ntile + 2):
            if i < ntile:
                sl = i % NK
                yield from wait(k_empty[sl], ((i // NK) & 1) ^ 1, drop == "k_empty")
                K[sl].write(i // NK)
                k_full[sl].arrive()
            if i >= 2:
                t = i - 2
                sl = t % NV
                yield from wait(v_empty[sl], ((t // NV) & 1) ^ 1, drop == "v_empty")
                V[sl].write(t // NV)
                v_full[sl].arrive()
            yield

    def mma():
        def issue_pv(u):
            sv = u % NV
            yield from wait(p_full, u & 1, drop == "p_full")
            yield from wait(v_full[sv], (u // NV) & 1)
            pipe.mma([(P, u), (V[sv], u // NV)], [(O, 0, u == 0)])
            pipe.commit(v_empty[sv])
            pipe.commit(p_empty)

        for t in range(ntile):
            s = t % NK
            yield from wait(k_full[s], (t // NK) & 1)
            yield from wait(s_free, (t & 1) ^ 1, drop == "s_free")
            pipe.mma([(K[s], t // NK)], [(S, t, True)])
            pipe.commit(s_full)
            pipe.commit(k_empty[s])
            if t >= 1:
                yield from issue_pv(t - 1)
            yield
        if ntile:
            yield from issue_pv(ntile - 1)
            pipe.commit(o_full)

    def softmax():
        for t in range(ntile):
            yield from wait(s_full, t & 1, drop == "s_full")
            S.read_begin(t)
            yield
            S.read_end()
            s_free.arrive()
            yield
            # P(t) overwrites P(t-1), and O may be rescaled: P(t-1) V(t-1) done
            yield from wait(p_empty, (t & 1) ^ 1, drop == "p_empty")
            if t > 0:
                O.write(0, fresh=False)  # the (rare) rescale of O by this warp's rows
            n = p_stores.get(t, 0)
            P.write(t, fresh=n == 0)  # the first warp's store starts generation t
            p_stores[t] = n + 1
            yield
            p_full.arrive()
        if ntile:
            yield from wait(o_full, 0)
            O.read_begin(0)
            O.read_end()

    return [producer(), mma()] + [softmax() for _ in range(warps)], pipe


@pytest.mark.parametrize("ntile", [0, 1, 2, 3, 4, 7, 16])
@pytest.mark.parametrize("seed", range(40))
def test_attention_protocol(ntile, seed):
    roles, pipe = attention_roles(ntile)
    run(roles, pipe, random.Random(seed * 1000 + ntile))


# ---------------------------------------------------------------------- map --
# map_tc.cu: a ring of NCH key chunks (NC per tile), two TMEM accumulators,
# eight epilogue warps sharing one staging tile.

def map_roles(ntile, NC=4, NCH=5, warps=8, drop=None):
    pipe = Pipe()
    full = [Bar(f"full{s}", 1) for s in range(NCH)]
    empty = [Bar(f"empty{s}", 1) for s in range(NCH)]
    q_ready = Bar("q_ready", warps)
    acc_full = [Bar(f"acc_full{a}", 1) for a in range(2)]
    acc_empty = [Bar(f"acc_empty{a}", warps) for a in range(2)]
    st_full, st_free = Bar("st_full", warps), Bar("st_free", warps)
    chunk = [Buf(f"chunk{s}") for s in range(NCH)]
    acc = [Buf(f"acc{a}") for a in range(2)]
    Q, stage = Buf("Q"), Buf("stage")
    q_stores, stage_stores = {"n": 0}, {}

    def producer():
        for t in range(ntile):
            for c in range(NC):
                u = t * NC + c
                s = u % NCH
                yield from wait(empty[s], ((u // NCH) & 1) ^ 1, drop == "empty")
                chunk[s].write(u // NCH)
                full[s].arrive()
                yield

    def mma():
        yield from wait(q_ready, 0, drop == "q_ready")
        for t in range(ntile):
            a = t & 1
            yield from wait(acc_empty[a], ((t >> 1) & 1) ^ 1, drop == "acc_empty")
            for c in range(NC):
                u = t * NC + c
                s = u % NCH
                yield from wait(full[s], (u // NCH) & 1)
                pipe.mma([(chunk[s], u // NCH), (Q, 0)], [(acc[a], t >> 1, c == 0)])
                pipe.commit(empty[s])
            pipe.commit(acc_full[a])
            yield

    def epilogue():
        Q.write(0, fresh=q_stores["n"] == 0)
        q_stores["n"] += 1
        q_ready.arrive()
        for t in range(ntile):
            a = t & 1
            yield from wait(acc_full[a], (t >> 1) & 1, drop == "acc_full")
            yield from wait(st_free, (t & 1) ^ 1, drop == "st_free")
            acc[a].read_begin(t >> 1)
            yield
            acc[a].read_end()
            n = stage_stores.get(t, 0)
            stage.write(t, fresh=n == 0)  # this warp's rows of tile t
            stage_stores[t] = n + 1
            acc_empty[a].arrive()
            st_full.arrive()
            yield from wait(st_full, t & 1, drop == "st_full")
            stage.read_begin(t)
            yield
            stage.read_end()
            st_free.arrive()

    return [producer(), mma()] + [epilogue() for _ in range(warps)], pipe


@pytest.mark.parametrize("ntile,nc", [(1, 4), (2, 4), (3, 4), (8, 4), (5, 2), (32, 2)])
@pytest.mark.parametrize("seed", range(30))
def test_map_protocol(ntile, nc, seed):
    roles, pipe = map_roles(ntile, NC=nc)
    run(roles, pipe, random.Random(seed * 1000 + ntile))


# -------------------------------------------------------- estimate passes --
# estimate_tc.cu: the last block's queries of two heads loaded once, key tiles
# through a ring of 3, S double-buffered per head in TMEM (both heads' S of a
# tile in one buffer index), four consumer warps per head; in the second pass
# each head's warps exchange diagonal bins through shared memory between two
# warpgroup barriers per tile; in the first pass of a kv head's first pair two
# more warps read every key tile of the ring for the block means of K, and a
# ring slot is free once the MMAs and both of them are done with it.

def estimate_roles(ntile, RING=3, heads=2, warps_per_head=4, line_pass=True, pool=False,
                   drop=None):
    pipe = Pipe()
    q_full = Bar("q_full", 1)
    ring_full = [Bar(f"ring_full{r}", 1) for r in range(RING)]
    ring_empty = [Bar(f"ring_empty{r}", 3 if pool else 1) for r in range(RING)]
    s_full = [Bar(f"s_full{b}", 1) for b in range(2)]
    s_free = [Bar(f"s_free{b}", heads * warps_per_head) for b in range(2)]
    wg = [Bar(f"wg{h}", warps_per_head) for h in range(heads)]  # bar.sync per head
    Q = Buf("Q")
    ring = [Buf(f"ring{r}") for r in range(RING)]
    S = [[Buf(f"S{h}_{b}") for b in range(2)] for h in range(heads)]
    bins = [Buf(f"bins{h}") for h in range(heads)]
    bin_stores = {}

    def producer():
        Q.write(0)
        q_full.arrive()
        for t in range(ntile):
            slot = t % RING
            yield from wait(ring_empty[slot], ((t // RING) & 1) ^ 1, drop == "ring_empty")
            ring[slot].write(t // RING)
            ring_full[slot].arrive()
            yield

    def mma():
        yield from wait(q_full, 0)
        for t in range(ntile):
            slot, buf = t % RING, t & 1
            yield from wait(ring_full[slot], (t // RING) & 1)
            yield from wait(s_free[buf], ((t >> 1) & 1) ^ 1, drop == "s_free")
            for h in range(heads):
                pipe.mma([(Q, 0), (ring[slot], t // RING)], [(S[h][buf], t >> 1, True)])
            pipe.commit(ring_empty[slot])
            pipe.commit(s_full[buf])
            yield

    def bar_sync(b, gen):
        # bar.sync over the head's warps: arrive, then wait for this generation
        b.arrive()
        while b.done <= gen:
            yield

    def consumer(h):
        syncs = 0
        for t in range(ntile):
            buf = t & 1
            yield from wait(s_full[buf], (t >> 1) & 1, drop == "s_full")
            S[h][buf].read_begin(t >> 1)
            yield
            S[h][buf].read_end()
            s_free[buf].arrive()
            if line_pass:
                key = (h, t)
                n = bin_stores.get(key, 0)
                bins[h].write(t, fresh=n == 0)  # this warp's diagonal bins
                bin_stores[key] = n + 1
                yield from bar_sync(wg[h], syncs)  # every warp's bins are written
                syncs += 1
                bins[h].read_begin(t)
                yield
                bins[h].read_end()
                if drop != "wg_after":
                    yield from bar_sync(wg[h], syncs)  # bins are rewritten by the next tile
                    syncs += 1
            yield

    def pooler():
        for t in range(ntile):
            slot = t % RING
            yield from wait(ring_full[slot], (t // RING) & 1, drop == "pool_full")
            ring[slot].read_begin(t // RING)
            yield
            ring[slot].read_end()
            ring_empty[slot].arrive()

    roles = [producer(), mma()]
    roles += [consumer(h) for h in range(heads) for _ in range(warps_per_head)]
    if pool:
        roles += [pooler(), pooler()]
    return roles, pipe


@pytest.mark.parametrize("ntile", [1, 2, 3, 5, 16])
@pytest.mark.parametrize("line_pass,pool", [(False, False), (False, True), (True, False)])
@pytest.mark.parametrize("seed", range(25))
def test_estimate_pass_protocol(ntile, line_pass, pool, seed):
    roles, pipe = estimate_roles(ntile, line_pass=line_pass, pool=pool)
    run(roles, pipe, random.Random(seed * 1000 + ntile + 7 * line_pass + 13 * pool))


@pytest.mark.parametrize("model,drop", [
    ("attention", "k_empty"), ("attention", "v_empty"), ("attention", "s_free"),
    ("attention", "s_full"), ("attention", "p_empty"), ("attention", "p_full"),
    ("map", "empty"), ("map", "q_ready"), ("map", "acc_empty"), ("map", "acc_full"),
    ("map", "st_free"), ("map", "st_full"),
    ("estimate", "ring_empty"), ("estimate", "s_free"), ("estimate", "s_full"),
    ("estimate", "wg_after"), ("estimate_pool", "pool_full"), ("estimate_pool", "ring_empty"),
])
def test_each_wait_is_needed(model, drop):
    """With any one of the kernel's waits taken out, some interleaving
    violates a buffer rule: the model is sensitive to every wait it checks."""
    failures = 0
    for seed in range(60):
        if model == "attention":
            roles, pipe = attention_roles(8, drop=drop)
        elif model == "map":
            roles, pipe = map_roles(6, drop=drop)
        elif model == "estimate":
            roles, pipe = estimate_roles(6, drop=drop)
        else:
            roles, pipe = estimate_roles(6, line_pass=False, pool=True, drop=drop)
        try:
            run(roles, pipe, random.Random(seed))
        except AssertionError:
            failures += 1
    assert failures > 0, f"dropping {drop} went unnoticed"
