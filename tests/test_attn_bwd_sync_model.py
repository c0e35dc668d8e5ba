"""Randomised models of the synchronisation of the one-pass attention backward kernels in
csrc/attn_tc_bwd.cu, run on the CPU. They check the protocols, not the kernels: the TMA thread,
the MMA issuers, the compute warps (two stand for all of them) and, at d = 64, the copy engine
that adds dQ, under random interleavings.

d = 64 (`attn_bwd_fused64_tc`):
per 128-query step j the issuer runs dV(j), S^T(j+1), dP^T(j+1), dQ(j), dK(j) on one in-order
tensor queue. Tensor memory holds S^T (then P^T over it), dP^T, and two dQ buffers; shared
memory holds two Q/dO stages, one dS^T tile and one dQ staging tile. The model asserts that no
MMA or warp overwrites one of them before its last reader is done, that every parity wait which
passes sees the phase it means, and that every named barrier completes.

d = 128 (`attn_bwd_fused_tc`): per 64-query step one issuer runs S^T and dP^T, the other the
accumulations dV, dK and dQ^T, on the same in-order tensor queue. S^T/dP^T, P^T, dS^T and dQ^T
are single buffers; the Q/dO stages form a ring of three.
"""
import random

import pytest

from sync_model import MBar, Named, schedule

WARPS = 2  # compute warps modelled; every per-warp barrier counts them


class Clocked:
    """Bounded waits and an abort clock shared by the models. After any wait has run out
    (`aborted`), every wait returns at once, true only if its phase is already complete."""

    def start_clock(self, abort_after):
        self.aborted = False
        self.clock = [None] * abort_after if abort_after else []

    def on_tick(self, _):
        if not self.clock:
            self.aborted = True

    def wait(self, cond):
        yield lambda: cond() or self.aborted
        return cond()

    def drain(self):  # mma_drain: a commit of the issuer's own MMAs, then a wait for it
        bar = MBar(1)
        self.tensor.append(("commit", bar))
        yield lambda: bar.phase >= 1


class Fused64(Clocked):
    def __init__(self, nit, seed, staging_wait=True, dqr_wait=True, abort_after=None):
        self.nit, self.R = nit, random.Random(seed)
        self.start_clock(abort_after)
        self.staging_wait, self.dqr_wait = staging_wait, dqr_wait
        self.kv = MBar(1)
        self.st = [MBar(1), MBar(1)]
        self.stfree = [MBar(1), MBar(1)]
        self.s, self.dp, self.vdone, self.kdone = MBar(1), MBar(1), MBar(1), MBar(1)
        self.p, self.ds = MBar(WARPS), MBar(WARPS)
        self.dq = [MBar(1), MBar(1)]
        self.dqr = [MBar(WARPS), MBar(WARPS)]
        self.sync = Named()  # the compute warps' named barrier around the staging
        self.tensor, self.tma, self.copy = [], [], []
        self.done = set()             # ("S", j), ("dP", j), ("dV", j), ("dQ", j), ("dK", j)
        self.loaded = set()           # stages loaded, by step
        self.s_cols = None            # what the S^T columns hold: ("S", j) or ("P", j)
        self.p_read = {}              # warps that have read S^T(j) / dP^T(j) / dQ(j)
        self.dp_read, self.dq_read = {}, {}
        self.ds_tile = None           # the step whose dS^T the tile holds
        self.staging = None           # the step whose sigma dQ the staging tile holds
        self.staging_reads = 0        # reductions issued that have not read the staging yet
        self.added = []               # steps the copy engine added, in order

    # ---- roles
    def tma_thread(self):
        yield lambda: True
        self.tma.append(("kv", 0))
        for j in range(self.nit):
            if j >= 2:
                ok = yield from self.wait(lambda j=j: self.stfree[j & 1].passes(((j - 2) >> 1) & 1))
                if not ok:
                    break
                assert self.stfree[j & 1].phase >= (j - 2) // 2 + 1, "stale stage-free pass"
                assert ("dK", j - 2) in self.done, "stage reloaded under its readers"
                assert self.dp_read.get(j - 2) == WARPS, "stage reloaded before the warps read its vectors"
            self.tma.append(("st", j))
        yield lambda: not self.tma  # every issued load lands before the thread leaves

    def issuer(self):
        ok = yield from self.wait(lambda: self.kv.passes(0) and self.st[0].passes(0))
        if ok:
            self.tensor += [("S", 0), ("commit", self.s), ("dP", 0), ("commit", self.dp)]
        j = 0
        while j < self.nit and ok:
            if not (yield from self.wait(lambda j=j: self.p.passes(j & 1))):
                break
            assert self.p.phase >= j + 1 and self.s_cols == ("P", j)
            self.tensor += [("dV", j), ("commit", self.vdone)]
            if j + 1 < self.nit:
                n = j + 1
                ok = (yield from self.wait(lambda n=n: self.st[n & 1].passes((n >> 1) & 1))) and (
                    yield from self.wait(lambda j=j: self.vdone.passes(j & 1)))
                if not ok:
                    break
                assert self.st[n & 1].phase >= n // 2 + 1 and self.vdone.phase >= j + 1
                self.tensor += [("S", n), ("commit", self.s)]
            if not (yield from self.wait(lambda j=j: self.ds.passes(j & 1))):
                break
            assert self.ds.phase >= j + 1 and self.ds_tile == j
            if j + 1 < self.nit:
                self.tensor += [("dP", j + 1), ("commit", self.dp)]
            if j >= 2 and self.dqr_wait:
                if not (yield from self.wait(lambda j=j: self.dqr[j & 1].passes(((j - 2) >> 1) & 1))):
                    break
                assert self.dqr[j & 1].phase >= (j - 2) // 2 + 1
            self.tensor += [("dQ", j), ("commit", self.dq[j & 1]),
                            ("dK", j), ("commit", self.stfree[j & 1]), ("commit", self.kdone)]
            j += 1
        yield from self.drain()

    def compute_warp(self, w):
        # `ok` turns false at the first wait that fails; the warp then goes on through every named
        # barrier of the remaining steps without touching tensor memory, the tiles or the barriers
        # the other roles wait on.
        ok = True

        def flush(i):
            nonlocal ok
            if ok:
                ok = yield from self.wait(lambda i=i: self.dq[i & 1].passes((i >> 1) & 1))
            if ok:
                assert self.dq[i & 1].phase >= i // 2 + 1 and ("dQ", i) in self.done
                self.dq_read[i] = self.dq_read.get(i, 0) + 1
                self.dqr[i & 1].arrive()
            if w == 0 and self.staging_wait:  # bulk_wait_read_all: the last reduction has read it
                yield lambda: self.staging_reads == 0
            ph = self.sync.join(("stage", i), 32 * WARPS)
            yield lambda ph=ph: self.sync.phase > ph
            assert self.staging_reads == 0, "staging overwritten before the copy engine read it"
            if ok:
                self.staging = i
            ph = self.sync.join(("issue", i), 32 * WARPS)
            yield lambda ph=ph: self.sync.phase > ph
            if w == 0 and ok:
                self.staging_reads += 1
                self.copy.append(i)

        for j in range(self.nit):
            if ok:
                ok = yield from self.wait(lambda j=j: self.s.passes(j & 1) and self.st[j & 1].passes((j >> 1) & 1))
            if ok:
                assert self.s.phase >= j + 1 and self.st[j & 1].phase >= j // 2 + 1
                assert self.s_cols in (("S", j), ("P", j)) and j in self.loaded
                self.p_read[j] = self.p_read.get(j, 0) + 1
                if self.p_read[j] == WARPS:
                    self.s_cols = ("P", j)  # every warp's columns now hold P^T(j)
                self.p.arrive()
                ok = yield from self.wait(lambda j=j: self.dp.passes(j & 1) and (
                    j == 0 or self.kdone.passes((j - 1) & 1)))
            if ok:
                assert ("dP", j) in self.done and (j == 0 or ("dK", j - 1) in self.done)
                assert ("dQ", j - 1) in self.done or j == 0, "dS^T overwritten under dQ"
                self.dp_read[j] = self.dp_read.get(j, 0) + 1
                self.ds_tile = j
                self.ds.arrive()
            if j > 0:
                yield from flush(j - 1)
        yield from flush(self.nit - 1)
        if ok and not self.aborted:
            ok = yield from self.wait(lambda: self.kdone.passes((self.nit - 1) & 1))
            if ok:
                assert ("dK", self.nit - 1) in self.done
        if w == 0:  # bulk_wait_all
            yield lambda: not self.copy

    # ---- the units that complete work in order
    def on_tensor(self, item):
        op, x = item
        if op == "commit":
            x.arrive()
            return
        j = x
        if op == "S":
            assert j == 0 or ("dV", j - 1) in self.done, "S^T over a P^T that dV has not read"
            assert j == 0 or self.p_read.get(j - 1) == WARPS
            self.s_cols = ("S", j)
        elif op == "dP":
            assert j == 0 or self.dp_read.get(j - 1) == WARPS, "dP^T overwritten before the warps read it"
        elif op == "dV":
            assert self.s_cols == ("P", j)
        elif op == "dQ":
            assert self.ds_tile == j
            assert j < 2 or self.dq_read.get(j - 2) == WARPS, "dQ buffer overwritten before the warps read it"
        elif op == "dK":
            assert self.ds_tile == j
        self.done.add((op, j))

    def on_tma(self, item):
        op, j = item
        if op == "kv":
            self.kv.arrive()
        else:
            self.loaded.add(j)
            self.st[j & 1].arrive()

    def on_copy(self, i):
        assert self.staging == i, "the copy engine read another step's staging"
        self.staging_reads -= 1
        self.added.append(i)

    def run(self):
        actors = [self.tma_thread(), self.issuer()] + [self.compute_warp(w) for w in range(WARPS)]
        schedule(self.R, actors, [(self.tensor, self.on_tensor), (self.tma, self.on_tma),
                                  (self.copy, self.on_copy), (self.clock, self.on_tick)])
        if not self.aborted:
            assert self.added == list(range(self.nit)), "a step's dQ was not added exactly once"
        assert len(set(self.added)) == len(self.added), "a step's dQ was added twice"


@pytest.mark.parametrize("nit", list(range(1, 10)) + [24, 48])
def test_fused64_protocol(nit):
    for seed in range(60):
        Fused64(nit, seed).run()


def test_model_catches_a_staging_overwrite():
    """Without the wait for the copy engine to have read the staging, a warp can overwrite it."""
    with pytest.raises(AssertionError, match="staging"):
        for nit in range(2, 10):
            for seed in range(300):
                Fused64(nit, seed, staging_wait=False).run()


def test_dq_buffer_wait_is_implied_by_the_step_order():
    """The issuer's wait for the warps to have read dQ(j - 2) before dQ(j) is a guard the step
    order already implies: dQ(j) follows dS^T(j), which every warp writes only after its flush
    of step j - 2 has read dQ(j - 2). Without the wait the model finds no overwrite."""
    for nit in range(3, 10):
        for seed in range(100):
            Fused64(nit, seed, dqr_wait=False).run()


class Fused128(Clocked):
    def __init__(self, nit, seed, stages=3, sfree_wait=True, abort_after=None):
        self.nit, self.R, self.ks = nit, random.Random(seed), stages
        self.start_clock(abort_after)
        self.sfree_wait = sfree_wait
        self.kv = MBar(1)
        self.st = [MBar(1) for _ in range(stages)]
        self.stfree = [MBar(1) for _ in range(stages)]
        self.s, self.acc = MBar(1), MBar(1)
        self.sfree, self.p = MBar(WARPS), MBar(WARPS)
        self.tensor, self.tma = [], []
        self.done, self.loaded = set(), set()
        self.sdp = None          # the step whose S^T/dP^T the columns hold
        self.sdp_read = {}       # warps that have read S^T/dP^T(n)
        self.pds = None          # the step whose P^T and dS^T the warps last wrote
        self.pds_writes = {}
        self.dqt = None          # the step whose dQ^T the columns hold
        self.dqt_read = {}

    def tma_thread(self):
        yield lambda: True
        self.tma.append(("kv", 0))
        for it in range(self.nit):
            if it >= self.ks:
                n = it - self.ks
                ok = yield from self.wait(lambda it=it, n=n: self.stfree[it % self.ks].passes((n // self.ks) & 1))
                if not ok:
                    break
                assert self.stfree[it % self.ks].phase >= n // self.ks + 1, "stale stage-free pass"
                assert ("acc", n) in self.done and self.sdp_read.get(n) == WARPS
            self.tma.append(("st", it))
        yield lambda: not self.tma

    def s_issuer(self):
        ok = yield from self.wait(lambda: self.kv.passes(0))
        n = 0
        while n < self.nit and ok:
            ok = yield from self.wait(lambda n=n: self.st[n % self.ks].passes((n // self.ks) & 1) and (
                n == 0 or not self.sfree_wait or self.sfree.passes((n - 1) & 1)))
            if not ok:
                break
            assert self.st[n % self.ks].phase >= n // self.ks + 1 and n in self.loaded
            assert n == 0 or not self.sfree_wait or self.sfree.phase >= n
            self.tensor += [("S", n), ("commit", self.s)]
            n += 1
        yield from self.drain()

    def acc_issuer(self):
        for it in range(self.nit):
            if not (yield from self.wait(lambda it=it: self.p.passes(it & 1))):
                break
            assert self.p.phase >= it + 1 and self.pds_writes.get(it) == WARPS
            self.tensor += [("acc", it), ("commit", self.acc), ("commit", self.stfree[it % self.ks])]
        yield from self.drain()

    def compute_warp(self, w):
        # a failed wait ends the warp's loop (this kernel has no named barrier in it)
        for it in range(self.nit):
            ok = yield from self.wait(lambda it=it: self.s.passes(it & 1) and self.st[it % self.ks].passes((it // self.ks) & 1))
            if not ok:
                break
            assert self.s.phase >= it + 1 and self.sdp == it and it in self.loaded
            self.sdp_read[it] = self.sdp_read.get(it, 0) + 1
            self.sfree.arrive()
            if it > 0:
                if not (yield from self.wait(lambda it=it: self.acc.passes((it - 1) & 1))):
                    break
                assert self.acc.phase >= it and ("acc", it - 1) in self.done
                assert self.dqt == it - 1
                self.dqt_read[it - 1] = self.dqt_read.get(it - 1, 0) + 1
            assert it == 0 or ("acc", it - 1) in self.done, "P^T or dS^T overwritten under its MMAs"
            self.pds_writes[it] = self.pds_writes.get(it, 0) + 1
            self.pds = it
            self.p.arrive()
        if not self.aborted:
            ok = yield from self.wait(lambda: self.acc.passes((self.nit - 1) & 1))
            if ok:
                assert ("acc", self.nit - 1) in self.done and self.dqt == self.nit - 1

    def on_tensor(self, item):
        op, x = item
        if op == "commit":
            x.arrive()
            return
        if op == "S":
            assert x == 0 or self.sdp_read.get(x - 1) == WARPS, "S^T/dP^T overwritten before the warps read it"
            self.sdp = x
        else:
            assert self.pds == x and self.pds_writes.get(x) == WARPS
            assert x == 0 or self.dqt_read.get(x - 1) == WARPS, "dQ^T overwritten before the warps read it"
            self.dqt = x
        self.done.add((op, x))

    def on_tma(self, item):
        op, j = item
        if op == "kv":
            self.kv.arrive()
        else:
            self.loaded.add(j)
            self.st[j % self.ks].arrive()

    def run(self):
        actors = [self.tma_thread(), self.s_issuer(), self.acc_issuer()] + [
            self.compute_warp(w) for w in range(WARPS)]
        schedule(self.R, actors, [(self.tensor, self.on_tensor), (self.tma, self.on_tma),
                                  (self.clock, self.on_tick)])


@pytest.mark.parametrize("nit", list(range(1, 10)) + [32, 128])
def test_fused128_protocol(nit):
    for seed in range(60):
        Fused128(nit, seed).run()


def test_model_catches_s_over_unread_scores():
    """Without the S issuer's wait for the warps to have read S^T/dP^T(n - 1), S^T(n) can
    overwrite them."""
    with pytest.raises(AssertionError, match="before the warps read it"):
        for nit in range(2, 10):
            for seed in range(300):
                Fused128(nit, seed, sfree_wait=False).run()


@pytest.mark.parametrize("nit", [1, 2, 3, 5, 9, 24])
def test_abort_at_any_point_ends_every_role(nit):
    """A wait that runs out at a random moment: every role of both kernels takes its abort path
    and ends (at d = 64 the compute warps still meet at both named barriers of every dQ
    staging), with issued loads, MMAs and reductions drained and no dQ added twice."""
    rng = random.Random(nit)
    for seed in range(80):
        Fused64(nit, seed, abort_after=rng.randint(1, 12 * nit)).run()
        Fused128(nit, seed, abort_after=rng.randint(1, 12 * nit)).run()
