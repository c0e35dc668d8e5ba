"""Building blocks of the randomised synchronisation models in test_attn_*_sync_model.py: an
mbarrier with phase-parity waits, a named barrier with counted phases, and a scheduler that runs
role generators against an in-order tensor queue and an in-order copy queue."""


class MBar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, 0, 0  # phase = completed phases

    def arrive(self):
        self.pending += 1
        assert self.pending <= self.count
        if self.pending == self.count:
            self.pending, self.phase = 0, self.phase + 1

    def passes(self, parity):  # mbarrier.try_wait.parity
        return (self.phase & 1) != parity


class Named:
    def __init__(self):
        self.phase, self.n, self.tag, self.count = 0, 0, None, None

    def join(self, tag, threads):
        if self.n == 0:
            self.tag, self.count = tag, threads
        assert (self.tag, self.count) == (tag, threads), "arrival joins another phase"
        self.n += 32
        ph = self.phase
        if self.n == self.count:
            self.n, self.phase = 0, self.phase + 1
        return ph


def schedule(rng, actors, queues, limit=200000):
    """Runs role generators until all are done and every queue is empty. A role yields a predicate
    (what it waits for); the scheduler steps a random ready role or pops the head of a random
    non-empty queue (`queues`: list of (list, handler)). No ready choice is a deadlock."""
    waiting = [next(a) for a in actors]
    done = [False] * len(actors)
    for _ in range(limit):
        if all(done) and not any(q for q, _ in queues):
            return
        ready = [("actor", i) for i, a in enumerate(actors) if not done[i] and waiting[i]()]
        ready += [("queue", i) for i, (q, _) in enumerate(queues) if q]
        assert ready, "deadlock"
        kind, i = rng.choice(ready)
        if kind == "queue":
            q, handler = queues[i]
            handler(q.pop(0))
        else:
            try:
                waiting[i] = next(actors[i])
            except StopIteration:
                done[i] = True
    raise AssertionError("livelock")
