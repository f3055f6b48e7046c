"""A CPU model of the decode chain's synchronisation protocol (csrc/chain.cu),
run under random schedules.

Every role of one CTA is a coroutine that yields wherever the kernel may be
overtaken by another warp: the weight producer (stages of the stream, one
arrival per stage, transaction bytes landing at random times), the activation
loader and the quantiser warps (staging slots, rows quantised into int8
buffers), the MMA warps (one ring slot each, every record of their stages,
projections opened and closed through monotonic counters) and the epilogue.
The model checks what the kernel relies on:
  * a parity wait never sees a barrier more than one phase away from the
    round it waits for (else the hardware would answer for the wrong round);
  * an MMA warp reads stage bytes only after they landed, and int8 codes only
    after every row of the projection was quantised;
  * the epilogue takes a projection only after every record of it was run,
    and finds its own scale in the scale slot;
  * nothing deadlocks.
Sizes are in records (one 16x64 weight record = one unit), so stages, shares
and projections are small integers.
"""
import random

import pytest


class _Bar:
    """An mbarrier: pending arrivals and transaction bytes of the current phase."""

    def __init__(self, name, count):
        self.name, self.count, self.pending, self.tx, self.phases = name, count, count, 0, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, f"{self.name}: too many arrivals"
        self._complete()

    def expect_tx(self, n):
        self.tx += n
        self.arrive()

    def complete_tx(self, n):
        self.tx -= n
        self._complete()

    def _complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phases += 1
            self.pending = self.count

    def done(self, rnd):
        assert self.phases in (rnd, rnd + 1), f"{self.name}: wait for round {rnd} with {self.phases} phases done"
        return self.phases == rnd + 1


def run_chain(T, nb, shares, stage, seed, n_mma=4, n_quant=4, n_acc=4, slots=None):
    """One CTA's chain: shares[j] records of projection j (0: no rows here)."""
    slots = nb + n_acc if slots is None else slots
    rng = random.Random(seed)
    ns = n_mma
    full = [_Bar(f"full{i}", 1) for i in range(ns)]
    empty = [_Bar(f"empty{i}", 1) for i in range(ns)]
    xs_full = [_Bar(f"xs_full{i}", 1) for i in range(n_quant)]
    xs_empty = [_Bar(f"xs_empty{i}", 1) for i in range(n_quant)]
    rows_q, recs_x = [0] * nb, [0] * nb
    recs_a, freed = [0] * n_acc, [0] * n_acc
    inflight, landed, scale, codes, runs = [], {}, {}, {}, {}
    uses = [b for b in shares if b > 0]
    n = len(uses)
    ustart = [0]
    for b in uses:
        ustart.append(ustart[-1] + b)
    total = ustart[-1]
    cum_x = [sum(uses[v] for v in range(u - nb, -1, -nb)) for u in range(n)]
    cum_a = [sum(uses[v] for v in range(u - n_acc, -1, -n_acc)) for u in range(n)]

    def wait(bar, rnd):
        while not bar.done(rnd):
            yield

    def producer():
        it = ps = fill = 0
        opened = False
        for b in uses:
            off = 0
            while off < b:
                if not opened:
                    if it >= ns:
                        yield from wait(empty[ps], it // ns - 1)
                    opened, fill = True, 0
                m = min(b - off, stage - fill)
                full[ps].tx += m
                inflight.append((full[ps], m, it))
                fill += m
                off += m
                yield
                if fill == stage:
                    full[ps].arrive()
                    opened = False
                    it += 1
                    ps = it % ns
        if opened:
            full[ps].arrive()

    def loader():
        item = 0
        for _ in uses:
            for _t in range(T):
                slot, r = item % n_quant, item // n_quant
                if r >= 1:
                    yield from wait(xs_empty[slot], r - 1)
                xs_full[slot].expect_tx(1)
                inflight.append((xs_full[slot], 1, None))
                item += 1
                yield

    def quantiser(q):
        item = 0
        for u in range(n):
            xb = u % nb
            waited = False
            for t in range(T):
                if item % n_quant == q:
                    if not waited and u >= nb:
                        while recs_x[xb] < cum_x[u]:
                            yield
                    waited = True
                    yield from wait(xs_full[q], item // n_quant)
                    yield
                    if t == 0:
                        scale[u % slots] = u
                    codes[u] = codes.get(u, 0) + 1
                    rows_q[xb] += 1
                    xs_empty[q].arrive()
                item += 1

    def mma(w):
        s, opened, mine = w, None, 0

        def open_(u):
            while freed[u % n_acc] < u // n_acc:
                yield
            while rows_q[u % nb] < T * (u // nb + 1):
                yield

        def close(u, cnt):
            runs[u] = runs.get(u, 0) + cnt
            recs_a[u % n_acc] += cnt
            recs_x[u % nb] += cnt

        while s * stage < total:
            a, b = s * stage, min((s + 1) * stage, total)
            yield from wait(full[s % ns], s // ns)
            pos = a
            u = max(i for i in range(n) if ustart[i] <= pos)
            while pos < b:
                seg = min(b, ustart[u + 1])
                if opened != u:
                    if opened is not None:
                        close(opened, mine)
                    yield from open_(u)
                    opened, mine = u, 0
                assert landed.get(s, 0) >= seg - a, "records read before they landed"
                assert codes.get(u, 0) == T, f"projection {u}: codes read before every row was quantised"
                yield
                mine += seg - pos
                pos = seg
                if pos == ustart[u + 1]:
                    close(u, mine)
                    opened, mine = None, 0
                    u += 1
            empty[s % ns].arrive()
            s += n_mma
        if opened is not None:
            close(opened, mine)

    def epilogue():
        for u in range(n):
            ab = u % n_acc
            while recs_a[ab] < cum_a[u] + uses[u]:
                yield
            assert runs.get(u, 0) == uses[u], f"projection {u}: taken before every record ran"
            assert scale.get(u % slots) == u, f"projection {u}: scale slot overwritten"
            yield
            freed[ab] += 1

    alive = [producer(), loader(), epilogue()] + [quantiser(q) for q in range(n_quant)] + \
        [mma(w) for w in range(n_mma)]
    steps = 0
    while alive:
        steps += 1
        assert steps < 2_000_000, "no progress (deadlock)"
        if inflight and rng.random() < 0.3:
            bar, m, st = inflight.pop(rng.randrange(len(inflight)))
            if st is not None:
                landed[st] = landed.get(st, 0) + m
            bar.complete_tx(m)
            continue
        g = rng.choice(alive)
        try:
            next(g)
        except StopIteration:
            alive.remove(g)


def _case(seed):
    rng = random.Random(seed)
    T = rng.randint(1, 8)
    nb = rng.choice([1, 2, 4, 8])
    shares = [rng.choice([0, 1, 2, 3, 5, 8, 13, 30]) for _ in range(rng.randint(1, 24))]
    return dict(T=T, nb=nb, shares=shares, stage=rng.choice([1, 2, 3, 4, 8]), seed=seed,
                n_mma=rng.choice([2, 3, 4, 6]), n_acc=rng.choice([2, 4, 8]))


@pytest.mark.parametrize("block", range(4))
def test_protocol_random_schedules(block):
    for seed in range(block * 40, (block + 1) * 40):
        run_chain(**_case(seed))


def test_protocol_model_catches_too_few_scale_slots():
    # with fewer scale slots than int8 buffers + partial-sum buffers, a quantiser
    # may overwrite a scale the epilogue has not read yet: the model must see it
    hits = 0
    for seed in range(60):
        rng = random.Random(seed)
        try:
            run_chain(1, 8, [rng.choice([1, 2, 3]) for _ in range(24)], 2, seed, n_mma=3, n_acc=4, slots=6)
        except AssertionError as e:
            assert "scale slot" in str(e)
            hits += 1
    assert hits > 0
