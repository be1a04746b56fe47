"""Host-side model of the fused attention kernel's synchronisation protocol.

The kernel's roles (TMA producers, MMA issuer, two softmax warpgroups) talk only
through mbarriers.  An mbarrier wait names a phase by its parity alone, so a
wait is only meaningful while the barrier is within one phase of the awaited
one; a role that falls two phases behind (or waits one phase early) reads the
wrong phase.  This model replays the roles' exact sequence of arrivals and
waits, with the tensor core executing its queue in order and the TMA unit
completing loads in any order, under many random interleavings, and checks that

* every parity wait is evaluated only while the barrier is at the awaited
  phase or one past it;
* no phase receives more arrivals than its count, and the transaction count
  never goes negative;
* no shared-memory slot, TMEM buffer or query tile is overwritten while an
  operation that reads it is still in flight, and every consumer reads the
  tile (and the published running max) of its own step;
* every role finishes (no deadlock).

It mirrors the step structure of attention_tc.cu: per work item, one step per
selected block, one per 128-cluster chunk, then one per entry tile of the
selected blocks' cluster entries; double-buffered query tiles; key, value and
bias-row rings; two MMA issuing threads, one for S = Q K^T (the query tile
copied into tensor memory at an item's start, S(g) into the one score buffer
once softmax(g - 1) has read it) and one for O += P V, each with its own
commits; softmax warpgroup X taking the steps
g with g & 1 == X, with its own score buffer S_X and probability tile P_X; one
output accumulator O shared by both, with the running max passed between the
warpgroups at every step and O rescaled by whichever raises it; at the end of
an item the two warpgroups exchange (max, sum) through a double-buffered shared
array and each reads half of O.  Chunk and entry tiles are written by the
Reassign Cache before the kernel starts, so they are plain inputs here; an entry
tile arrives as several copies on one barrier, which the model counts as one
transaction.
"""
import random

import pytest

QSTAGES = 1   # query tiles, freed when the item's last S is computed
KSTAGES = 3   # key / centroid tiles, freed when S is computed
VSTAGES = 2   # value / mean tiles, freed after P V
BSTAGES = 4   # softmax bias rows, freed after the softmax has read them (even: one warpgroup per slot)


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
                 no_final_wait=False, single_xch_barrier=False, s_before_read=False, no_pfree_wait=False,
                 no_rescale_wait=False, single_q=False, skip_m_wait=False, s_early=False):
        # per item of one CTA: nsel, or (nsel, entry tiles)
        self.items = [(x, 0) if isinstance(x, int) else tuple(x) for x in items]
        self.nchunk = nchunk
        self.rng = rng
        self.lazy_v_wait = lazy_v_wait         # planted: value producer waits for a free slot only at chunk steps
        self.skip_b_empty = skip_b_empty       # planted: bias rows loaded without waiting for a free slot
        self.single_xch = single_xch           # planted: one (max, sum) exchange buffer for all items
        self.no_final_wait = no_final_wait     # planted: epilogue without waiting for the last product
        self.single_xch_barrier = single_xch_barrier   # planted: one exchange barrier per warpgroup
        self.s_before_read = s_before_read     # planted: softmax releases S before reading it
        self.no_pfree_wait = no_pfree_wait     # planted: P written without waiting for P V(g - 2)
        self.no_rescale_wait = no_rescale_wait  # planted: O rescaled without waiting for P V(g - 1)
        self.single_q = single_q               # planted: one query buffer, with the waits of two
        self.skip_m_wait = skip_m_wait         # planted: the running max read without its barrier
        self.s_early = s_early                 # planted: S(g) issued without waiting for softmax(g - 1)
        B = Barrier
        self.q_full = [B(f"q_full{i}", 1) for i in range(QSTAGES)]
        self.q_empty = [B(f"q_empty{i}", 1) for i in range(QSTAGES)]
        self.k_full = [B(f"k_full{i}", 1) for i in range(KSTAGES)]
        self.k_empty = [B(f"k_empty{i}", 1) for i in range(KSTAGES)]
        self.v_full = [B(f"v_full{i}", 1) for i in range(VSTAGES)]
        self.v_empty = [B(f"v_empty{i}", 1) for i in range(VSTAGES)]
        self.b_full = [B(f"b_full{i}", 1) for i in range(BSTAGES)]
        self.b_empty = [B(f"b_empty{i}", 1) for i in range(BSTAGES)]
        self.version = {}                      # buffer -> step whose tile it holds
        self.s_full = [B(f"s_full{i}", 1) for i in range(2)]
        self.s_free = [B(f"s_free{i}", 1) for i in range(2)]     # 128 threads, one arrival here
        self.p_ready = [B(f"p_ready{i}", 1) for i in range(2)]
        self.p_free = [B(f"p_free{i}", 1) for i in range(2)]
        self.m_pub = [B(f"m_pub{i}", 1) for i in range(2)]
        self.mrow = [None, None]               # warpgroup -> step whose running max it holds
        self.o_free = B("o_free", 2)           # one arrival per warpgroup (128 threads each)
        # exchange published: [item parity][warpgroup]; one barrier per item parity, so a warpgroup
        # without steps cannot complete a barrier twice before the other has waited on it once
        self.xch_full = [[B(f"xch_full{j}{i}", 1) for i in range(2)] for j in range(2)]
        self.xch = [[None, None], [None, None]]   # [item parity][warpgroup] -> item whose (max, sum) it holds
        self.o_content = None                  # (item, last step accumulated), at issue
        self.o_scaled = None                   # (item, step) of the last rescale of O
        # per issuing thread, in order: ("mma", buffers) / ("commit", bar); a commit arrives once that
        # thread's earlier products are done (the two threads' products interleave in any order)
        self.tc_queues = {"s": [], "pv": []}
        self.tma = []                          # in flight: (bar, buffer written, buffers read)
        self.readers = {}                      # resource -> units with an operation in flight on it

    def T(self, n):
        nsel, nent = self.items[n]
        return nsel + self.nchunk + nent

    # ---- resources: in-flight users of each buffer, tagged by unit
    def _start_read(self, res, unit):
        self.readers.setdefault(res, []).append(unit)

    def _end_read(self, res, unit):
        self.readers[res].remove(unit)

    def _write(self, res, who, unit=None):
        """A write by `unit`; the tensor core executes its own queue in issue order, so its earlier
        operations on the same buffer are not a hazard for its later ones."""
        busy = [u for u in self.readers.get(res, []) if not (unit == "tc" and u == "tc")]
        assert not busy, f"{who} overwrites {res} while {busy} use it"

    # ---- asynchronous units
    def tc_issue_mma(self, q, reads, writes):
        for w in writes:
            self._write(w, "tensor core", unit="tc")
        for r in reads + writes:     # the destination is busy until the MMA completes
            self._start_read(r, "tc")
        self.tc_queues[q].append(("mma", reads + writes))

    def tc_commit(self, q, bar):
        self.tc_queues[q].append(("commit", bar))

    @property
    def tc_busy(self):
        return any(self.tc_queues.values())

    def step_units(self):
        progressed = False
        live = [q for q in self.tc_queues.values() if q]
        if live and self.rng.random() < 0.6:
            q = self.rng.choice(live)
            kind, x = q.pop(0)
            if kind == "mma":
                for r in x:
                    self._end_read(r, "tc")
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

    def qbuf(self, n):
        return 0 if self.single_q else n % QSTAGES

    # ---- roles (generators yield a predicate to wait on)
    def producer(self):
        """The producer of keys: query tiles, key / centroid / entry tiles, bias rows."""
        g = 0
        for n in range(len(self.items)):
            qb = self.qbuf(n)
            qs = n % QSTAGES
            yield lambda: self.q_empty[qs].test(n // QSTAGES - 1)
            self.q_full[qs].expect_tx(1)
            self.tma_load(self.q_full[qs], f"Q{qb}", ("q", n))
            for s in range(self.T(n)):
                ks, bs = g % KSTAGES, g % BSTAGES
                yield lambda: self.k_empty[ks].test(g // KSTAGES - 1)
                self.k_full[ks].expect_tx(1)
                self.tma_load(self.k_full[ks], f"K{ks}", g)
                if not self.skip_b_empty:
                    yield lambda: self.b_empty[bs].test(g // BSTAGES - 1)
                    self.b_full[bs].expect_tx(1)
                else:
                    self.b_full[bs].tx += 1          # the planted variant: no free-slot wait
                self.tma_load(self.b_full[bs], f"BIAS{bs}", g)
                g += 1

    def producer_v(self):
        """The producer of values / means / entry means."""
        g = 0
        for n in range(len(self.items)):
            nsel = self.items[n][0]
            for s in range(self.T(n)):
                vs = g % VSTAGES
                if not self.lazy_v_wait or s >= nsel:
                    yield lambda: self.v_empty[vs].test(g // VSTAGES - 1)
                self.v_full[vs].expect_tx(1)
                self.tma_load(self.v_full[vs], f"V{vs}", g)
                g += 1

    def _steps(self):
        """(item, step in item, global step) of every step of the CTA, in order."""
        g = 0
        for n in range(len(self.items)):
            for s in range(self.T(n)):
                yield n, s, g
                g += 1

    def mma_s(self):
        """The issuer of S = Q K^T: at an item's start it copies the query tile into tensor memory
        (buffer n & 1; in order with its products), then S(g) into the one score buffer once
        softmax(g - 1) has read it."""
        for n, s, g in self._steps():
            qb = self.qbuf(n)
            if s == 0:
                yield lambda: self.q_full[n % QSTAGES].test(n // QSTAGES)
                self.holds(f"Q{qb}", ("q", n))
                self.tc_issue_mma("s", [f"Q{qb}"], [f"QT{n & 1}"])    # tcgen05.cp into tensor memory
                self.version[f"QT{n & 1}"] = n
                self.tc_commit("s", self.q_empty[n % QSTAGES])
            if g >= 1 and not self.s_early:
                yield lambda: self.s_free[(g - 1) & 1].test((g - 1) >> 1)
            yield lambda: self.k_full[g % KSTAGES].test(g // KSTAGES)
            self.holds(f"QT{n & 1}", n)
            self.holds(f"K{g % KSTAGES}", g)
            self.tc_issue_mma("s", [f"QT{n & 1}", f"K{g % KSTAGES}"], ["S"])
            self.version["S"] = g
            self.tc_commit("s", self.s_full[g & 1])
            self.tc_commit("s", self.k_empty[g % KSTAGES])

    def mma_pv(self):
        """The issuer of O += P V: P V(g) once P(g) is written."""
        for n, s, g in self._steps():
            yield lambda: self.p_ready[g & 1].test(g >> 1)
            yield lambda: self.v_full[g % VSTAGES].test(g // VSTAGES)
            if s == 0:
                yield lambda: self.o_free.test(n - 1)
            self.holds(f"V{g % VSTAGES}", g)
            self.holds(f"P{g & 1}", g)
            if s > 0:
                assert self.o_content == (n, g - 1), f"O holds {self.o_content} before P V of step {g}"
            self.tc_issue_mma("pv", [f"P{g & 1}", f"V{g % VSTAGES}"], ["O"])
            self.o_content = (n, g)
            self.tc_commit("pv", self.v_empty[g % VSTAGES])
            self.tc_commit("pv", self.p_free[g & 1])

    def softmax(self, X):
        g0 = 0
        for n in range(len(self.items)):
            T = self.T(n)
            for s in range((X - g0) & 1, T, 2):
                g = g0 + s
                bs = g % BSTAGES
                yield lambda: self.b_full[bs].test(g // BSTAGES)
                yield lambda: self.s_full[X].test(g >> 1)
                assert not self.readers.get(f"BIAS{bs}"), "bias row read before it landed"
                self.holds(f"BIAS{bs}", g)
                if self.s_before_read:
                    self.s_free[X].arrive()
                    yield lambda: True                 # the row is read from TMEM after the release
                assert not self.readers.get("S"), "S read before its MMA completed or while it is rewritten"
                self.holds("S", g)
                if not self.s_before_read:
                    self.s_free[X].arrive()
                yield lambda: True                     # the row max and the exponentials
                if g >= 1:
                    if not self.skip_m_wait:
                        yield lambda: self.m_pub[X ^ 1].test((g - 1) >> 1)
                    assert self.mrow[X ^ 1] == g - 1, f"running max of step {self.mrow[X ^ 1]} read at step {g}"
                if g >= 2:
                    assert self.mrow[X] is None or self.mrow[X] == g - 2
                self.mrow[X] = g
                self.m_pub[X].arrive()
                if g >= 2 and not self.no_pfree_wait:
                    yield lambda: self.p_free[X].test((g - 2) >> 1)
                self._write(f"P{X}", "softmax (P)")
                self.version[f"P{X}"] = g
                self.b_empty[bs].arrive()
                # a rescale of O (only when the running max moved: here at random, and always at an
                # item's second step) waits for P V(g - 1) first
                if s > 0 and (s == 1 or self.rng.random() < 0.3):
                    if not self.no_rescale_wait:
                        yield lambda: self.p_free[X ^ 1].test((g - 1) >> 1)
                    self._write("O", "softmax (rescale)")
                    assert self.o_content == (n, g - 1), f"O holds {self.o_content} at the rescale of step {g}"
                self.p_ready[X].arrive()
            # epilogue
            gl = g0 + T - 1
            if not self.no_final_wait:
                if gl >= 1:
                    yield lambda: self.p_free[(gl - 1) & 1].test((gl - 1) >> 1)
                yield lambda: self.p_free[gl & 1].test(gl >> 1)
            slot = 0 if self.single_xch else n & 1
            self.xch[slot][X] = n
            if self.single_xch_barrier:
                self.xch_full[0][X].arrive()
                yield lambda: self.xch_full[0][X ^ 1].test(n)
            else:
                self.xch_full[n & 1][X].arrive()
                yield lambda: self.xch_full[n & 1][X ^ 1].test(n >> 1)
            assert self.xch[slot][X ^ 1] == n, f"exchange slot holds item {self.xch[slot][X ^ 1]}, read for item {n}"
            assert not self.readers.get("O"), "O read while a product into it is in flight"
            assert self.o_content == (n, gl), f"O holds {self.o_content} at the end of item {n}"
            self.o_free.arrive()
            g0 += T

    def run(self, max_iters=400000):
        roles = [self.producer(), self.producer_v(), self.mma_s(), self.mma_pv(), self.softmax(0), self.softmax(1)]
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
    # with entry tiles: a block's entries always fill at least one tile row, so nsel > 0 => tiles > 0
    ([(30, 8), (26, 7), (30, 8)], 4), ([(1, 1), (0, 0), (2, 1), (0, 0)], 1), ([(9, 3), (1, 1)], 8),
    ([(3, 1), (3, 1), (3, 1), (3, 1)], 2),
]


@pytest.mark.parametrize("items,nchunk", CASES)
def test_protocol_random_interleavings(items, nchunk):
    for seed in range(60):
        Machine(items, nchunk, random.Random(seed)).run()


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


def test_model_catches_an_epilogue_that_does_not_wait_for_the_last_product():
    assert _caught([3, 4, 1], 2, no_final_wait=True) > 0


def test_one_exchange_barrier_per_warpgroup_is_now_safe():
    """With one accumulator, the first product of item n + 1 waits for item n's epilogue (o_free),
    and item n + 1's epilogue waits for that product, so a warpgroup cannot complete a single
    exchange barrier twice before the other has waited on it; the double buffer stays as a margin."""
    assert _caught([1, 0, 0, 1], 1, single_xch_barrier=True) == 0


def test_model_catches_s_released_before_it_is_read():
    assert _caught([5, 5], 2, s_before_read=True) > 0


def test_model_catches_p_written_during_its_product():
    assert _caught([6, 4], 2, no_pfree_wait=True) > 0


def test_model_catches_a_rescale_during_the_previous_product():
    assert _caught([6, 4], 2, no_rescale_wait=True) > 0


@pytest.mark.skipif(QSTAGES < 2, reason="one query buffer is the design: its waits are those of one buffer")
def test_model_catches_a_single_query_buffer():
    """Two query buffers waited as two while one is used: the next item's query tile would
    overwrite the one the current item's S still reads."""
    assert _caught([1, 1, 1, 1, 2, 1], 1, single_q=True) > 0


def test_model_catches_the_running_max_read_without_its_barrier():
    caught = 0
    for seed in range(400):
        try:
            Machine([6, 6, 3], 2, random.Random(seed), skip_m_wait=True).run()
        except AssertionError:
            caught += 1
    assert caught > 0


def test_model_catches_s_issued_before_the_previous_softmax_read_it():
    assert _caught([5, 5], 2, s_early=True) > 0
