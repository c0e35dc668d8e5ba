"""A randomised model of the attention forward's synchronisation (csrc/attn_tc_fwd.cu), run on
the CPU. It checks the protocol, not the kernel: every wait and barrier of the kernel's roles,
for one lane quarter, with every interleaving a seeded scheduler picks.

Modelled:
  - mbarriers with phase-parity waits. A wait passes when the phase of the other parity is the
    current one, exactly as the hardware test does. So a waiter two phases behind passes on a
    stale phase, and the model reports that.
  - The tensor core as one in-order queue, each commit arriving once the operations before it
    are done, and TMA loads landing in issue order.
  - Named barriers as phases of a fixed count. An arrival that joins an open phase with another
    tag or count is an error, and so is a barrier that never completes (a deadlock).
  - The shared-memory slots that carry the block maxima between warps.
Roles: the TMA thread (independent K and V rings), the S and PV issuers, and two softmax sets
(even and odd key blocks) of two warps each (the two key halves of a block).
"""
import random

import pytest

from sync_model import MBar, Named, schedule


class Protocol:
    """One CTA of the forward at nkb key blocks. `xc_slots` and `epilogue_on_last_pv` select the
    design (4 slots and a dedicated last-PV barrier) or a flawed alternative."""

    def __init__(self, nkb, seed, kStV=2, xc_slots=4, epilogue_on_last_pv=True, abort_after=None):
        self.nkb, self.R, self.kStV = nkb, random.Random(seed), kStV
        self.aborted = False
        # a wait runs out after this many ticks of a clock the scheduler advances at random
        self.clock = [None] * abort_after if abort_after else []
        self.kStages = self.kSBuf = 3
        self.xc_slots, self.fin_bar = xc_slots, epilogue_on_last_pv
        self.q = MBar(1)
        self.K = [MBar(1) for _ in range(3)]
        self.V = [MBar(1) for _ in range(kStV)]
        self.KF = [MBar(1) for _ in range(3)]
        self.VF = [MBar(1) for _ in range(kStV)]
        self.SB = [MBar(1) for _ in range(3)]
        self.PB = [MBar(2) for _ in range(3)]  # the set's two warps of this lane quarter
        self.PVB = [MBar(1) for _ in range(3)]
        self.FIN = MBar(1)
        self.named = [Named(), Named()]  # the incoming barrier of set 0 and of set 1
        self.epi = Named()
        self.xm, self.xc = {}, {}
        self.tensor, self.tma = [], []
        self.S_done, self.PV_done, self.P_written = set(), set(), {}

    def seen(self, bar, phases):  # a wait that passed must see at least this many phases
        assert bar.phase >= phases, "a wait passed on a stale phase"

    def wait(self, cond):
        """A bounded mbarrier wait: passes once cond() holds. After any wait has run out
        (self.aborted) every wait returns at once, true only if its phase is already complete."""
        yield lambda: cond() or self.aborted
        return cond()

    def drain(self):  # mma_drain: a commit of the issuer's own MMAs, then a wait for it
        bar = MBar(1)
        self.tensor.append(("commit", bar))
        yield lambda: bar.phase >= 1

    def tma_thread(self):
        yield lambda: True
        self.tma.append(("q", 0))
        nk = nv = 0
        ks, kv = self.kStages, self.kStV
        k_ok = lambda: nk < self.nkb and (nk < ks or self.KF[nk % ks].passes(((nk - ks) // ks) & 1))
        v_ok = lambda: nv < nk and (nv < kv or self.VF[nv % kv].passes(((nv - kv) // kv) & 1))
        while nk < self.nkb or nv < self.nkb:
            if not (k_ok() or v_ok()):
                yield lambda: k_ok() or v_ok() or self.aborted
                if not (k_ok() or v_ok()):
                    break  # no stage freed and the CTA has aborted
                continue
            if k_ok():
                if nk >= ks:
                    self.seen(self.KF[nk % ks], (nk - ks) // ks + 1)
                    assert nk - ks in self.S_done, "K stage reloaded before S read it"
                self.tma.append(("k", nk))
                nk += 1
            if v_ok():
                if nv >= kv:
                    self.seen(self.VF[nv % kv], (nv - kv) // kv + 1)
                    assert nv - kv in self.PV_done, "V stage reloaded before PV read it"
                self.tma.append(("v", nv))
                nv += 1
            yield lambda: True
        yield lambda: not self.tma  # every issued load lands before the thread leaves

    def s_issuer(self):
        ok = yield from self.wait(lambda: self.q.passes(0))
        n = 0
        while n < self.nkb and ok:
            ok = yield from self.wait(lambda n=n: self.K[n % 3].passes((n // 3) & 1))
            if ok:
                self.seen(self.K[n % 3], n // 3 + 1)
            if ok and n >= 3:
                ok = yield from self.wait(lambda n=n: self.PVB[n % 3].passes(((n // 3) - 1) & 1))
                if ok:
                    self.seen(self.PVB[n % 3], n // 3)
                    assert n - 3 in self.PV_done, "S written over a P that PV has not read"
            if not ok:
                break
            self.tensor += [("S", n), ("commit", self.SB[n % 3]), ("commit", self.KF[n % 3])]
            n += 1
        yield from self.drain()

    def pv_issuer(self):
        j = 0
        while j < self.nkb:
            ok = yield from self.wait(lambda j=j: self.PB[j % 3].passes((j // 3) & 1))
            if ok:
                self.seen(self.PB[j % 3], j // 3 + 1)
                assert self.P_written.get(j) == 2
                ok = yield from self.wait(lambda j=j: self.V[j % self.kStV].passes((j // self.kStV) & 1))
            if not ok:
                break
            self.seen(self.V[j % self.kStV], j // self.kStV + 1)
            self.tensor += [("PV", j), ("commit", self.PVB[j % 3]),
                            ("commit", self.VF[j % self.kStV])]
            j += 1
        if j == self.nkb:
            self.tensor.append(("commit", self.FIN))
        yield from self.drain()

    def softmax_warp(self, st, half):
        ok = True
        for j in range(st, self.nkb, 2):
            if ok:
                ok = yield from self.wait(lambda j=j: self.SB[j % 3].passes((j // 3) & 1))
                if ok:
                    self.seen(self.SB[j % 3], j // 3 + 1)
                    assert j in self.S_done
            yield lambda: True  # load S_j (when ok), take this half's max
            self.xc[(j % self.xc_slots, half)] = j
            ph = self.named[st].join(j, 64 if j == 0 else 128)
            yield lambda ph=ph, st=st: self.named[st].phase > ph
            assert self.xc[(j % self.xc_slots, half ^ 1)] == j, "the other half's max was overwritten"
            if j > 0:
                assert self.xm[(j - 1) & 1] == j - 1, "the max of block j - 1 was overwritten"
            yield lambda: True
            if j + 1 < self.nkb:
                if half == 0:
                    self.xm[j & 1] = j
                self.named[st ^ 1].join(j + 1, 128)
            if j > 0 and self.R.random() < 0.3 and ok:  # a row max grew: rescale O after PV_{j-1}
                ok = yield from self.wait(lambda j=j: self.PVB[(j - 1) % 3].passes(((j - 1) // 3) & 1))
                if ok:
                    self.seen(self.PVB[(j - 1) % 3], (j - 1) // 3 + 1)
                    assert j - 1 in self.PV_done and j not in self.PV_done
            yield lambda: True
            if ok:
                self.P_written[j] = self.P_written.get(j, 0) + 1
                self.PB[j % 3].arrive()
        if ok:
            if self.fin_bar:
                ok = yield from self.wait(lambda: self.FIN.passes(0))
                if ok:
                    self.seen(self.FIN, 1)
            else:  # the flawed alternative: the last block's own PV barrier
                last = self.nkb - 1
                ok = yield from self.wait(lambda: self.PVB[last % 3].passes((last // 3) & 1))
                if ok:
                    self.seen(self.PVB[last % 3], last // 3 + 1)
            if ok:
                assert self.nkb - 1 in self.PV_done, "epilogue before the last PV"
        ph = self.epi.join("epilogue", 128)
        yield lambda ph=ph: self.epi.phase > ph

    def on_tensor(self, item):
        op, x = item
        if op == "S":
            self.S_done.add(x)
        elif op == "PV":
            assert self.P_written.get(x) == 2
            self.PV_done.add(x)
        else:
            x.arrive()

    def on_tma(self, item):
        op, n = item
        {"q": lambda: self.q, "k": lambda: self.K[n % 3], "v": lambda: self.V[n % self.kStV]}[op]().arrive()

    def run(self):
        actors = [self.tma_thread(), self.s_issuer(), self.pv_issuer()] + [
            self.softmax_warp(st, h) for st in (0, 1) for h in (0, 1)]
        schedule(self.R, actors, [(self.tensor, self.on_tensor), (self.tma, self.on_tma),
                                  (self.clock, self.on_tick)])

    def on_tick(self, _):
        if not self.clock:
            self.aborted = True


@pytest.mark.parametrize("kStV", [2, 3])  # V stages at d = 128 and d = 64
@pytest.mark.parametrize("nkb", list(range(1, 12)) + [31, 64])
def test_forward_protocol_never_deadlocks_or_reads_stale(nkb, kStV):
    for seed in range(40):
        Protocol(nkb, seed, kStV).run()


@pytest.mark.parametrize("nkb", [1, 2, 3, 5, 8, 13, 31])
def test_forward_abort_at_any_point_ends_every_role(nkb):
    """A wait that runs out at a random moment: every role takes its abort path (issuers and the
    TMA thread stop, softmax warps keep meeting at their named barriers without touching tensor
    memory) and every one of them ends, with its issued loads and MMAs drained."""
    rng = random.Random(nkb)
    for seed in range(80):
        Protocol(nkb, seed, abort_after=rng.randint(1, 8 * nkb)).run()


def test_model_catches_the_epilogue_on_a_per_buffer_barrier():
    """The set that does not own the last block can reach the epilogue while the last block's
    PV barrier is two phases behind: its parity wait would pass at once."""
    with pytest.raises(AssertionError, match="stale phase"):
        for nkb in range(2, 12):
            for seed in range(200):
                Protocol(nkb, seed, epilogue_on_last_pv=False).run()


def test_model_catches_two_slots_for_the_halves_maxima():
    """With the halves' block maxima in two slots, a warp can store block j + 2's max before its
    partner has read block j's."""
    with pytest.raises(AssertionError, match="other half"):
        for nkb in range(3, 16):
            for seed in range(200):
                Protocol(nkb, seed, xc_slots=2).run()
