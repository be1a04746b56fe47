"""Host-side model of the fused attention kernel's synchronisation protocol.

The kernel's roles (TMA producer lanes, MMA issuer, two softmax warpgroups)
talk only through mbarriers.  An mbarrier wait names a phase by its
parity alone, so a wait is only meaningful while the barrier is within one
phase of the awaited one; a role that falls two phases behind (or waits one
phase early) reads the wrong phase.  This model replays the roles' exact
sequence of arrivals and waits, with the tensor core executing its queue in
order and the TMA unit completing loads in any order, under many random
interleavings, and checks that

* every parity wait is evaluated only while the barrier is at the awaited
  phase or one past it;
* no phase receives more arrivals than its count, and the transaction count
  never goes negative;
* no shared-memory slot, TMEM buffer or the query tile is overwritten while an
  operation that reads it is still in flight, and every consumer reads the
  tile of its own step;
* every role finishes (no deadlock).

It mirrors the step structure of attention_tc.cu: per work item, one step per
selected block followed by one step per 128-cluster chunk; key, value and
bias-row rings (outside the variance-corrected mode a value tile lands on the
P-ready barrier of its score buffer, so one wait covers both); softmax warpgroup
X taking the steps g with g & 1 == X; three
score buffers in TMEM, step g's S (and then P, written over it) in buffer
g mod 3, and one accumulator O shared by both warpgroups, which exponentiate
against a reference max that the item's first step publishes to the other
warpgroup.  Two threads issue to the tensor core: the score issuer (S(g) once
its key tile has landed and P(g - 3) V(g - 3) has completed) and the product
issuer (P(g) V(g) once P(g) is written); each thread's products execute in its
issue order, but nothing orders one thread's products against the other's, so
the model keeps one in-order queue per issuer and completes them in any
interleaving.  At the end of an item the two warpgroups exchange their row sums
through a double-buffered shared array and each reads half of O.  The compensation chunks are written by an earlier kernel, so they
are plain inputs here.

The variance-corrected mode (spread=True) changes three things: a chunk step's
score tile reads two key-ring tiles (the centroid chunk and the chunk of the
scaled spread), so the key ring counts tiles, not steps; the value ring has
two slots; and both softmax warpgroups write their half of the squared query
tile Q2 at the start of each item (after the query tile has landed), which the
first chunk step of the item waits for.
"""
import random

import pytest

KSTAGES = 2   # key / centroid tiles, freed when S is computed
VSTAGES = 3   # value / vbar^U tiles, freed after P V
BSTAGES = 4   # softmax bias rows, freed after the softmax has read them (even: one warpgroup per slot)
SBUFS = 3     # score buffers in TMEM


class Barrier:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending = count
        self.tx = 0
        self.phase = 0          # number of completed phases

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self):
        assert self.pending > 0, f"{self.name}: arrival beyond the count"
        self.pending -= 1
        self._maybe_complete()

    def expect_tx(self, n):
        self.tx += n
        self.arrive()

    def complete_tx(self, n):
        self.tx -= n
        assert self.tx >= 0, f"{self.name}: transaction count below zero"
        self._maybe_complete()

    def test(self, target):
        """Wait for completion of phase `target` (-1: the phase before the first)."""
        assert self.phase in (target, target + 1) or (target == -1 and self.phase == 0), (
            f"{self.name}: parity wait for phase {target} while at phase {self.phase}")
        return self.phase > target


class Machine:
    def __init__(self, items, nchunk, rng, lazy_v_wait=False, skip_b_empty=False, single_xch=False,
                 no_final_wait=False, single_xch_barrier=False, spread=False, q2_no_wait=False,
                 mma_no_q2_wait=False, chunk_frees_one_tile=False, s_before_pv=False, no_mref_wait=False,
                 no_o_free_wait=False, key_on_own_barrier=False):
        self.items = items                     # list of nsel per item of one CTA
        self.nchunk = nchunk
        self.rng = rng
        self.spread = spread                   # variance-corrected mode: two key tiles per chunk step
        self.vstages = 2 if spread else VSTAGES
        self.q2_no_wait = q2_no_wait           # planted: Q2 written without waiting for the query tile
        self.mma_no_q2_wait = mma_no_q2_wait   # planted: chunk scores issued without waiting for Q2
        self.chunk_frees_one_tile = chunk_frees_one_tile   # planted: a chunk step frees only its first key tile
        self.s_before_pv = s_before_pv         # planted: S(g + 3) issued without waiting for P(g) V(g)
        self.no_mref_wait = no_mref_wait       # planted: the second warpgroup reads the reference unpublished
        self.no_o_free_wait = no_o_free_wait   # planted: an item's first product without waiting for O's readers
        self.key_on_own_barrier = key_on_own_barrier   # planted: key tiles land on k_full, not waited
        self.lazy_v_wait = lazy_v_wait         # planted: value lane waits for a free slot only at chunk steps
        self.skip_b_empty = skip_b_empty       # planted: bias rows loaded without waiting for a free slot
        self.single_xch = single_xch           # planted: one (max, sum) exchange buffer for all items
        self.no_final_wait = no_final_wait     # planted: epilogue without waiting for the last product
        self.single_xch_barrier = single_xch_barrier   # planted: one exchange barrier per warpgroup
        B = Barrier
        self.q_full, self.q_empty = B("q_full", 1), B("q_empty", 1)
        self.k_full = [B(f"k_full{i}", 1) for i in range(KSTAGES)]
        self.k_empty = [B(f"k_empty{i}", 1) for i in range(KSTAGES)]
        self.v_full = [B(f"v_full{i}", 1) for i in range(self.vstages)]
        self.v_empty = [B(f"v_empty{i}", 1) for i in range(self.vstages)]
        self.q2_full = B("q2_full", 2)         # one arrival per softmax warpgroup
        self.b_full = [B(f"b_full{i}", 1) for i in range(BSTAGES)]
        self.b_empty = [B(f"b_empty{i}", 1) for i in range(BSTAGES)]
        self.version = {}                      # buffer -> step whose tile it holds
        self.s_full = [B(f"s_full{i}", 1) for i in range(2 * SBUFS)]   # [g mod 6]
        # [g mod 3]; outside the variance-corrected mode the value tile of step g lands on it too
        self.p_ready = [B(f"p_ready{i}", 1 if spread else 2) for i in range(SBUFS)]
        # [g mod 3]; outside the variance-corrected mode the key tile of step g lands on it too,
        # and its first phase stands for a product before the first step
        self.pv_done = [B(f"pv_done{i}", 1 if spread or key_on_own_barrier else 2) for i in range(SBUFS)]
        if not spread:
            for b in self.pv_done:
                b.arrive()
        self.o_full = B("o_full", 1)
        self.o_free = B("o_free", 2)           # one arrival per warpgroup (128 threads each)
        self.mref_full = [B(f"mref_full{i}", 1) for i in range(2)]
        self.mref = [None, None]               # [item parity] -> item whose reference it holds
        # exchange published: [item parity][warpgroup]; one barrier per item parity, so a warpgroup
        # without steps cannot complete a barrier twice before the other has waited on it once
        self.xch_full = [[B(f"xch_full{j}{i}", 1) for i in range(2)] for j in range(2)]
        self.xch = [[None, None], [None, None]]   # [item parity][warpgroup] -> item whose (max, sum) it holds
        self.o_content = None                  # (item, products accumulated), at execution
        self.tc_queues = {"s": [], "pv": []}   # per issuer, in order: ("mma", ...) / ("commit", bar)
        self.tma = []                          # in flight: (bar, buffer written, buffers read)
        self.readers = {}                      # resource -> units with an operation in flight on it

    # ---- resources: in-flight users of each buffer, tagged by unit
    def _start_read(self, res, unit):
        self.readers.setdefault(res, []).append(unit)

    def _end_read(self, res, unit):
        self.readers[res].remove(unit)

    def _write(self, res, who, unit=None):
        """A write by `unit`; an issuer's products execute in its issue order, so its earlier
        operations on the same buffer are not a hazard for its later ones (the other issuer's are)."""
        busy = [u for u in self.readers.get(res, []) if not (unit is not None and unit.startswith("tc") and u == unit)]
        assert not busy, f"{who} overwrites {res} while {busy} use it"

    # ---- asynchronous units
    def tc_issue_mma(self, q, reads, writes, expect=None, produce=None, on_exec=None):
        """Queue a product on issuer q's queue.  expect: {buffer: version it must hold when the
        product executes}; produce: {buffer: version it holds afterwards}; on_exec: a callback run
        at execution."""
        for w in writes:
            self._write(w, "tensor core", unit=f"tc{q}")
        for r in reads:
            assert "tma" not in self.readers.get(r, []), f"a product reads {r} while its copy is in flight"
        for r in reads + writes:     # the destination is busy until the MMA completes
            self._start_read(r, f"tc{q}")
        self.tc_queues[q].append(("mma", (reads + writes, expect or {}, produce or {}, on_exec)))

    def tc_commit(self, q, bar):
        self.tc_queues[q].append(("commit", bar))

    @property
    def tc_busy(self):
        return any(self.tc_queues.values())

    def step_units(self):
        progressed = False
        live = [q for q, v in self.tc_queues.items() if v]
        if live and self.rng.random() < 0.5:
            q = self.rng.choice(live)
            kind, x = self.tc_queues[q].pop(0)
            if kind == "mma":
                bufs, expect, produce, on_exec = x
                for b, v in expect.items():
                    assert self.version.get(b) == v, f"a product reads {b} holding {self.version.get(b)}, wants {v}"
                for b, v in produce.items():
                    self.version[b] = v
                if on_exec:
                    on_exec()
                for r in bufs:
                    self._end_read(r, f"tc{q}")
            else:
                x.arrive()
            progressed = True
        if self.tma and self.rng.random() < 0.5:
            i = self.rng.randrange(len(self.tma))
            bar, dst, srcs = self.tma.pop(i)
            for r in [dst] + srcs:
                self._end_read(r, "tma")
            bar.complete_tx(1)
            progressed = True
        return progressed

    def tma_load(self, bar, res, step, srcs=()):
        """A copy of step `step`'s tile into buffer `res` (busy until it lands) that reads `srcs`."""
        self._write(res, "TMA", unit="tma")
        for r in [res, *srcs]:
            self._start_read(r, "tma")
        self.version[res] = step
        self.tma.append((bar, res, list(srcs)))

    def holds(self, res, step):
        assert self.version.get(res) == step, f"{res} holds step {self.version.get(res)}, read at step {step}"

    # ---- roles (generators yield a predicate to wait on)
    def tiles_of(self, s, nsel):
        """Key-ring tiles of step s: the chunk of the scaled spread follows a centroid chunk."""
        return 2 if self.spread and s >= nsel else 1

    def producer(self):
        """Lane 0 of the producer warp: query tiles, key / centroid tiles, bias rows."""
        g = 0
        kt = 0                                  # key-ring tiles loaded
        for n, nsel in enumerate(self.items):
            T = nsel + self.nchunk
            yield lambda: self.q_empty.test(n - 1)
            self.q_full.expect_tx(1)
            self.tma_load(self.q_full, "Q", n)
            for s in range(T):
                bs = g % BSTAGES
                for _ in range(self.tiles_of(s, nsel)):
                    ks = kt % KSTAGES
                    yield lambda: self.k_empty[ks].test(kt // KSTAGES - 1)
                    landed = self.k_full[ks] if self.spread or self.key_on_own_barrier else self.pv_done[g % SBUFS]
                    landed.expect_tx(1)
                    self.tma_load(landed, f"K{ks}", kt)
                    kt += 1
                if not self.skip_b_empty:
                    yield lambda: self.b_empty[bs].test(g // BSTAGES - 1)
                    self.b_full[bs].expect_tx(1)
                else:
                    self.b_full[bs].tx += 1          # the planted variant: no free-slot wait
                self.tma_load(self.b_full[bs], f"BIAS{bs}", g)
                g += 1

    def producer_v(self):
        """Lane 1 of the producer warp: value / vbar^U tiles."""
        g = 0
        for n, nsel in enumerate(self.items):
            T = nsel + self.nchunk
            for s in range(T):
                vs = g % self.vstages
                if not self.lazy_v_wait or s >= nsel:
                    yield lambda: self.v_empty[vs].test(g // self.vstages - 1)
                landed = self.v_full[vs] if self.spread else self.p_ready[g % SBUFS]
                landed.expect_tx(1)
                self.tma_load(landed, f"V{vs}", g)
                g += 1

    def s_issuer(self):
        g = 0
        kt = 0                                  # key-ring tiles consumed
        for n, nsel in enumerate(self.items):
            T = nsel + self.nchunk
            yield lambda: self.q_full.test(n)
            self.holds("Q", n)
            for s in range(T):
                b = g % SBUFS
                if not self.spread:
                    # the product that read the buffer, and the key tile, in one phase
                    yield lambda: self.pv_done[b].test(g // SBUFS)
                elif g >= SBUFS and not self.s_before_pv:
                    yield lambda: self.pv_done[b].test(g // SBUFS - 1)
                reads = ["Q"]
                for _ in range(self.tiles_of(s, nsel)):
                    t = kt
                    if self.spread:
                        yield lambda: self.k_full[t % KSTAGES].test(t // KSTAGES)
                    self.holds(f"K{t % KSTAGES}", t)
                    reads.append(f"K{t % KSTAGES}")
                    kt += 1
                if self.tiles_of(s, nsel) == 2:
                    if s == nsel and not self.mma_no_q2_wait:
                        yield lambda: self.q2_full.test(n)
                    for h in (0, 1):
                        self.holds(f"Q2h{h}", n)
                        reads.append(f"Q2h{h}")
                self.tc_issue_mma("s", reads, [f"S{b}"], produce={f"S{b}": ("S", g)})
                self.tc_commit("s", self.s_full[g % (2 * SBUFS)])
                freed = reads[1:2] if self.chunk_frees_one_tile else [r for r in reads if r.startswith("K")]
                for r in freed:
                    self.tc_commit("s", self.k_empty[int(r[1:])])
                if s == T - 1:
                    self.tc_commit("s", self.q_empty)
                g += 1

    def pv_issuer(self):
        g = 0
        for n, nsel in enumerate(self.items):
            T = nsel + self.nchunk
            for s in range(T):
                vs = g % self.vstages
                yield lambda: self.p_ready[g % SBUFS].test(g // SBUFS)
                if self.spread:
                    yield lambda: self.v_full[vs].test(g // self.vstages)
                if s == 0 and not self.no_o_free_wait:
                    yield lambda: self.o_free.test(n - 1)
                self.holds(f"V{vs}", g)

                def count(n=n, s=s):
                    self.o_content = (n, 1) if s == 0 else (n, self.o_content[1] + 1)
                self.tc_issue_mma("pv", [f"S{g % SBUFS}", f"V{vs}"], ["O"], expect={f"S{g % SBUFS}": ("P", g)},
                                  on_exec=count)
                self.tc_commit("pv", self.v_empty[vs])
                self.tc_commit("pv", self.pv_done[g % SBUFS])
                if s == T - 1:
                    self.tc_commit("pv", self.o_full)
                g += 1

    def softmax(self, X):
        g0 = 0
        for n, nsel in enumerate(self.items):
            T = nsel + self.nchunk
            if self.spread:
                # this warpgroup's half of Q2 = Q o Q (generic stores) once Q has landed
                if not self.q2_no_wait:
                    yield lambda: self.q_full.test(n)
                assert "tma" not in self.readers.get("Q", []), "Q read by the Q2 writer before it landed"
                self.holds("Q", n)
                self._write(f"Q2h{X}", "Q2 writer")
                self.version[f"Q2h{X}"] = n
                self.q2_full.arrive()
            steps = list(range((X - g0) & 1, T, 2))
            for s in steps:
                g = g0 + s
                bs = g % BSTAGES
                b = g % SBUFS
                yield lambda: self.b_full[bs].test(g // BSTAGES)
                yield lambda: self.s_full[g % (2 * SBUFS)].test(g // (2 * SBUFS))
                assert not self.readers.get(f"S{b}"), "S read before its MMA completed"
                assert self.version.get(f"S{b}") == ("S", g), f"S{b} holds {self.version.get(f'S{b}')} at step {g}"
                assert not self.readers.get(f"BIAS{bs}"), "bias row read before it landed"
                self.holds(f"BIAS{bs}", g)
                if s == 0:
                    self.mref[n & 1] = n
                    self.mref_full[n & 1].arrive()
                elif s == 1:
                    if not self.no_mref_wait:
                        yield lambda: self.mref_full[n & 1].test(n >> 1)
                    assert self.mref[n & 1] == n, f"reference of item {self.mref[n & 1]} read for item {n}"
                self._write(f"S{b}", "softmax (P)")
                self.version[f"S{b}"] = ("P", g)
                self.b_empty[bs].arrive()
                self.p_ready[b].arrive()
            # epilogue
            if not self.no_final_wait:
                yield lambda: self.o_full.test(n)
            slot = 0 if self.single_xch else n & 1
            self.xch[slot][X] = n
            if self.single_xch_barrier:
                self.xch_full[0][X].arrive()
                yield lambda: self.xch_full[0][X ^ 1].test(n)
            else:
                self.xch_full[n & 1][X].arrive()
                yield lambda: self.xch_full[n & 1][X ^ 1].test(n >> 1)
            assert self.xch[slot][X ^ 1] == n, f"exchange slot holds item {self.xch[slot][X ^ 1]}, read for item {n}"
            # this warpgroup's half of O is read over a span in which the other roles move on
            assert "tcpv" not in self.readers.get("O", []), "O read while a product into it is in flight"
            assert self.o_content == (n, T), f"O holds {self.o_content} at the end of item {n}"
            self._start_read("O", f"epilogue{X}")
            for _ in range(self.rng.randrange(1, 40)):  # a read of random length
                yield lambda: True
            assert self.o_content == (n, T), f"O changed to {self.o_content} while item {n}'s epilogue read it"
            self._end_read("O", f"epilogue{X}")
            self.o_free.arrive()
            g0 += T

    def run(self, max_iters=200000):
        roles = [self.producer(), self.producer_v(), self.s_issuer(), self.pv_issuer(), self.softmax(0),
                 self.softmax(1)]
        waits = [None] * len(roles)
        done = [False] * len(roles)
        for _ in range(max_iters):
            if all(done) and not self.tc_busy and not self.tma:
                return True
            order = list(range(len(roles)))
            self.rng.shuffle(order)
            progressed = False
            for r in order:
                if done[r]:
                    continue
                if waits[r] is not None and not waits[r]():
                    continue
                try:
                    waits[r] = next(roles[r])
                except StopIteration:
                    done[r] = True
                    waits[r] = None
                progressed = True
                if self.rng.random() < 0.5:
                    break
            progressed = self.step_units() or progressed
            if not progressed and not self.tc_busy and not self.tma:
                raise AssertionError("deadlock: no role can progress")
        raise AssertionError("did not finish")


CASES = [
    ([4], 2), ([37], 2), ([0], 2), ([0, 37, 2, 0, 5], 2), ([30, 30, 30], 4), ([1, 0, 0, 1], 1),
    ([9, 3, 0, 12], 8), ([2], 1), ([0, 0, 0], 3), ([40, 1], 4),
]


@pytest.mark.parametrize("items,nchunk", CASES)
def test_protocol_random_interleavings(items, nchunk):
    for seed in range(60):
        Machine(items, nchunk, random.Random(seed)).run()


@pytest.mark.parametrize("items,nchunk", [c for c in CASES if c[1] >= 1])
def test_protocol_random_interleavings_variance_corrected(items, nchunk):
    for seed in range(60):
        Machine(items, nchunk, random.Random(seed), spread=True).run()


def _caught(items, nchunk, **planted):
    caught = 0
    for seed in range(40):
        try:
            Machine(items, nchunk, random.Random(seed), **planted).run()
        except AssertionError:
            caught += 1
    return caught


def test_model_catches_a_lane_that_skips_ring_phases():
    """A value lane waiting for a free slot only at its chunk steps runs ahead of the ring by
    several phases when many exact steps precede a chunk."""
    assert _caught([37], 2, lazy_v_wait=True) > 0


def test_model_catches_bias_rows_loaded_without_a_free_slot():
    assert _caught([3, 3, 3, 3, 3], 2, skip_b_empty=True) > 0


def test_a_single_exchange_buffer_is_safe_with_the_shared_accumulator():
    """Both warpgroups wait for the item's last product before the exchange, and that product
    waits for both warpgroups' previous epilogue (o_free), so the exchange of item n + 1 cannot be
    written before item n's has been read: one buffer would do; two are kept."""
    assert _caught([0, 0, 0, 0, 0, 0], 1, single_xch=True) == 0
    assert _caught([2, 0, 1, 0, 3], 1, single_xch=True) == 0


def test_model_catches_an_epilogue_that_does_not_wait_for_the_last_product():
    assert _caught([3, 4, 1], 2, no_final_wait=True) > 0


def test_model_catches_a_score_tile_issued_before_the_product_that_reads_its_buffer_completes():
    """S(g + 3) goes into the buffer that holds P(g); the two issuers' products are not ordered, so
    without waiting for P(g) V(g) to complete it can overwrite P(g) first.  (Outside the
    variance-corrected mode that wait is also the key tile's, so the variant is planted there.)"""
    assert _caught([5, 2, 4], 2, spread=True, s_before_pv=True) > 0


def test_model_catches_a_reference_max_read_before_it_is_published():
    assert _caught([2, 3, 1, 4], 1, no_mref_wait=True) > 0


def test_model_catches_a_first_product_that_does_not_wait_for_the_epilogue():
    """An item's first product overwrites O: without waiting on o_free it can land while the other
    item's epilogue still reads O."""
    assert _caught([1, 0, 2, 1], 1, no_o_free_wait=True) > 0


def test_one_exchange_barrier_per_warpgroup_is_safe_with_the_shared_accumulator():
    """With one accumulator the warpgroups meet at every item's last product (o_full) and at the
    next item's first product (o_free), so a warpgroup without steps can no longer complete an
    exchange barrier twice before the other's wait: the per-item-parity barriers are kept anyway."""
    assert _caught([1, 0, 0, 1], 1, single_xch_barrier=True) == 0
    assert _caught([0, 0, 2, 0, 0, 1], 1, single_xch_barrier=True) == 0


def test_model_catches_a_key_tile_that_lands_on_a_barrier_the_score_issuer_does_not_wait():
    """Outside the variance-corrected mode the score issuer waits only on pv_done, which the key
    tile's bytes must complete; a tile landing on its own barrier is read while it is in flight."""
    assert _caught([4, 3, 5], 2, key_on_own_barrier=True) > 0
