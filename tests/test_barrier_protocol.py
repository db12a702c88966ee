"""A model of the prefill kernel's barrier protocol, checked on the CPU.

csrc/prefill_bf16.cuh synchronises its roles (TMA producer, S-MMA issuer,
PV-MMA issuer, output store, two softmax warpgroups) with mbarriers waited by
parity. A parity wait for phase k is only right while the barrier has
completed k or k+1 phases: with k+2 or more completed it aliases and spins
until its time limit; with k-1 or fewer (of the other parity) it passes
early. This file restates each role's sequence of waits and arrivals, lets
asynchronous completions (TMA loads, MMA commits) land at random later
times, runs many random interleavings over random item sizes, and checks that
every wait is satisfied with exactly k+1 phases completed and that every role
finishes.

What it shows:
  * the kernel's protocol (K tiles in a ring of two stages, V tiles in a
    ring of one, each stage with its own full and empty barriers, each full
    barrier waited in consecutive phases by its one consumer) is correct with
    asynchronous completions landing in any order: it does not rely on TMA
    loads completing in the order they were issued, which PTX does not
    promise; so is the previous form (one shared ring, full barriers split by
    tile kind);
  * the earliest form, where K and V tiles shared one full barrier per stage
    and each MMA issuer waited only on its own tiles' phases, relied on that
    order: a later load landing first lets a wait pass early;
  * the S issuer's wait for the softmax's Q-ready arrival is needed even
    when the queries arrive already rotated: without it, a run of one-tile
    items lets the next Q load complete before a softmax warpgroup has
    waited for the current one, and that wait aliases;
  * the model is sharp: the earlier one-arrival Q-free barrier without the
    Q-ready handshake aliases, as a GPU variant of that kind did.
"""
import random

import pytest

NSTAGE = 3


class Barrier:
    def __init__(self, count):
        self.count, self.pending, self.completed = count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending, self.completed = 0, self.completed + 1


class ProtocolError(AssertionError):
    pass


def kv_ring(n):
    """The producer's load order for one item: K0, K1, V0, K2, V1, ..., V(n-1)."""
    order = [("K", 0)]
    for j in range(1, n):
        order += [("K", j), ("V", j - 1)]
    order.append(("V", n - 1))
    return order


def k_index(j):
    return 0 if j == 0 else 2 * j - 1


def v_index(j, n):
    return 2 * j + 2 if j < n - 1 else 2 * n - 1


def roles(items, q_free_count, s_waits_q_ready, split_full=False, rings=None):
    """Generators yielding ('wait', name, phase) / ('arrive', name) /
    ('async', name) steps, one per role; the item list ends with a sentinel.
    rings=(NK, NV): K and V tiles in rings of their own (NK and NV stages),
    each with its own full and empty barriers."""
    NH = 2
    if rings is not None:
        return _ring_roles(items, q_free_count, s_waits_q_ready, rings)

    def producer():
        idx = 0
        for it, n in enumerate(items + [None]):
            if it > 0:
                yield ("wait", "Q_FREE", it - 1)
            if n is None:
                yield ("arrive", "Q_FULL")  # sentinel: a plain arrival
                return
            yield ("async", "Q_FULL")        # the Q tiles' TMA completion
            for kind, _ in kv_ring(n):
                st, use = idx % NSTAGE, idx // NSTAGE
                if use > 0:
                    yield ("wait", f"KV_EMPTY{st}", use - 1)
                yield ("async", f"FULL_{kind}{st}" if split_full else f"KV_FULL{st}")
                idx += 1

    def s_issuer():
        ring = tiles = 0
        kph = [0] * NSTAGE
        for it, n in enumerate(items + [None]):
            yield ("wait", "Q_FULL", it)
            if n is None:
                return
            if s_waits_q_ready:
                for s in range(NH):
                    yield ("wait", f"Q_READY{s}", it)
            for j in range(n):
                idx = ring + k_index(j)
                T = tiles + j
                if split_full:  # the K loads of this stage, counted by this issuer
                    yield ("wait", f"FULL_K{idx % NSTAGE}", kph[idx % NSTAGE])
                    kph[idx % NSTAGE] += 1
                else:
                    yield ("wait", f"KV_FULL{idx % NSTAGE}", idx // NSTAGE)
                for s in range(NH):
                    if T > 0:
                        yield ("wait", f"S_FREE{s}", T - 1)
                    yield ("async", f"S_READY{s}")
                yield ("async", f"KV_EMPTY{idx % NSTAGE}")
            yield ("async", "Q_FREE")
            ring += 2 * n
            tiles += n

    def pv_issuer():
        ring = tiles = 0
        vph = [0] * NSTAGE
        for it, n in enumerate(items + [None]):
            yield ("wait", "Q_FULL", it)
            if q_free_count == 2:
                yield ("arrive", "Q_FREE")
            if n is None:
                return
            for j in range(n):
                idx = ring + v_index(j, n)
                T = tiles + j
                if split_full:  # the V loads of this stage, counted by this issuer
                    yield ("wait", f"FULL_V{idx % NSTAGE}", vph[idx % NSTAGE])
                    vph[idx % NSTAGE] += 1
                else:
                    yield ("wait", f"KV_FULL{idx % NSTAGE}", idx // NSTAGE)
                for s in range(NH):
                    yield ("wait", f"P_READY{s}", T)
                    yield ("async", f"PV_DONE{s}")
                yield ("async", f"KV_EMPTY{idx % NSTAGE}")
            ring += 2 * n
            tiles += n

    def store():
        for it, n in enumerate(items + [None]):
            yield ("wait", "O_STAGED0", it)
            if n is None:
                return
            for s in range(NH):
                if s > 0:
                    yield ("wait", f"O_STAGED{s}", it)
                yield ("arrive", f"O_READ{s}")

    def softmax(s):
        tiles = 0

        def begin(it):
            yield ("wait", "Q_FULL", it)
            yield ("arrive", f"Q_READY{s}")

        more_items = items + [None]
        if more_items[0] is not None:
            yield from begin(0)
        for it, n in enumerate(items):
            for j in range(n):
                T = tiles + j
                yield ("wait", f"S_READY{s}", T)
                yield ("arrive", f"S_FREE{s}")
                if j > 0:
                    yield ("wait", f"PV_DONE{s}", T - 1)
                elif it > 0:
                    yield ("wait", f"O_READ{s}", it - 1)
                yield ("arrive", f"P_READY{s}")
            nxt = more_items[it + 1]
            if nxt is not None:  # at the end the ring says so before any Q wait
                yield from begin(it + 1)
            yield ("wait", f"PV_DONE{s}", tiles + n - 1)
            yield ("arrive", f"O_STAGED{s}")
            tiles += n
            if nxt is None and s == 0:
                yield ("wait", "O_READ0", it)
                yield ("arrive", "O_STAGED0")
        if not items and s == 0:
            yield ("arrive", "O_STAGED0")

    return {"producer": producer(), "s_issuer": s_issuer(), "pv_issuer": pv_issuer(), "store": store(),
            "softmax0": softmax(0), "softmax1": softmax(1)}


def _ring_roles(items, q_free_count, s_waits_q_ready, rings):
    NH = 2
    NK, NV = rings
    base = roles(items, q_free_count, s_waits_q_ready)  # store and softmax roles are unchanged

    def producer():
        kt = vt = 0
        for it, n in enumerate(items + [None]):
            if it > 0:
                yield ("wait", "Q_FREE", it - 1)
            if n is None:
                yield ("arrive", "Q_FULL")
                return
            yield ("async", "Q_FULL")
            for kind, _ in kv_ring(n):
                if kind == "K":
                    st, use = kt % NK, kt // NK
                    if use > 0:
                        yield ("wait", f"K_EMPTY{st}", use - 1)
                    yield ("async", f"K_FULL{st}")
                    kt += 1
                else:
                    st, use = vt % NV, vt // NV
                    if use > 0:
                        yield ("wait", f"V_EMPTY{st}", use - 1)
                    yield ("async", f"V_FULL{st}")
                    vt += 1

    def s_issuer():
        tiles = 0
        for it, n in enumerate(items + [None]):
            yield ("wait", "Q_FULL", it)
            if n is None:
                return
            if s_waits_q_ready:
                for s in range(NH):
                    yield ("wait", f"Q_READY{s}", it)
            for j in range(n):
                T = tiles + j
                yield ("wait", f"K_FULL{T % NK}", T // NK)
                for s in range(NH):
                    if T > 0:
                        yield ("wait", f"S_FREE{s}", T - 1)
                    yield ("async", f"S_READY{s}")
                yield ("async", f"K_EMPTY{T % NK}")
            yield ("async", "Q_FREE")
            tiles += n

    def pv_issuer():
        tiles = 0
        for it, n in enumerate(items + [None]):
            yield ("wait", "Q_FULL", it)
            if q_free_count == 2:
                yield ("arrive", "Q_FREE")
            if n is None:
                return
            for j in range(n):
                T = tiles + j
                yield ("wait", f"V_FULL{T % NV}", T // NV)
                for s in range(NH):
                    yield ("wait", f"P_READY{s}", T)
                    yield ("async", f"PV_DONE{s}")
                yield ("async", f"V_EMPTY{T % NV}")
            tiles += n

    base.update(producer=producer(), s_issuer=s_issuer(), pv_issuer=pv_issuer())
    return base


def barriers(q_free_count):
    b = {"Q_FULL": Barrier(1), "Q_FREE": Barrier(q_free_count)}
    for st in range(NSTAGE):
        for name in ("K_FULL", "K_EMPTY", "V_FULL", "V_EMPTY"):
            b[f"{name}{st}"] = Barrier(1)
        b[f"KV_FULL{st}"] = Barrier(1)
        b[f"FULL_K{st}"] = Barrier(1)
        b[f"FULL_V{st}"] = Barrier(1)
        b[f"KV_EMPTY{st}"] = Barrier(1)
    for s in range(2):
        for name in ("Q_READY", "S_FREE", "P_READY", "O_STAGED"):
            b[f"{name}{s}"] = Barrier(1)  # one arrival stands for the slot's 128 threads
        for name in ("S_READY", "PV_DONE", "O_READ"):
            b[f"{name}{s}"] = Barrier(1)
    return b


def simulate(items, seed, q_free_count=2, s_waits_q_ready=True, in_order=True, split_full=False,
             max_steps=200000, rings=None):
    """in_order: each asynchronous source completes in the order it issued
    (the producer's TMA loads; each MMA issuer's commits); sources interleave
    freely. in_order=False lets any in-flight completion land first."""
    rng = random.Random(seed)
    bars = barriers(q_free_count)
    gens = roles(items, q_free_count, s_waits_q_ready, split_full, rings)
    current = {name: next(g, None) for name, g in gens.items()}
    inflight = []  # (source, barrier) of completions not yet landed (MMA commits, TMA bytes)
    for _ in range(max_steps):
        runnable = []
        for name, step in current.items():
            if step is None:
                continue
            if step[0] == "wait":
                _, bname, k = step
                c = bars[bname].completed
                if c >= k + 2:
                    raise ProtocolError(f"{name} waits for phase {k} of {bname} with {c} phases done (aliased)")
                if c <= k - 1 and (c & 1) != (k & 1):
                    raise ProtocolError(f"{name}'s wait for phase {k} of {bname} would pass with {c} phases done")
                if c == k + 1:
                    runnable.append(name)
            else:
                runnable.append(name)
        choices = runnable + (["<async>"] if inflight else [])
        if not choices:
            if all(v is None for v in current.values()):
                return
            raise ProtocolError(f"deadlock: {[(n, s) for n, s in current.items() if s]}")
        pick = rng.choice(choices)
        if pick == "<async>":
            if in_order:  # the oldest completion of a randomly chosen source
                src = rng.choice(sorted({q for q, _ in inflight}))
                i = next(i for i, (q, _) in enumerate(inflight) if q == src)
            else:
                i = rng.randrange(len(inflight))
            bars[inflight.pop(i)[1]].arrive()
            continue
        step = current[pick]
        if step[0] == "arrive":
            bars[step[1]].arrive()
        elif step[0] == "async":
            inflight.append((pick, step[1]))
        current[pick] = next(gens[pick], None)
    raise ProtocolError("did not finish")


def _random_items(seed):
    rng = random.Random(1000 + seed)
    sizes = rng.choice([[1, 1, 2, 3, 5, 8], [1, 1, 1, 2]])
    return [rng.choice(sizes) for _ in range(rng.randint(0, 9))]


@pytest.mark.parametrize("seed", range(80))
def test_committed_protocol_needs_no_completion_order(seed):
    """The kernel's protocol: separate K (two stages) and V (one stage) rings,
    Q-ready handshake kept."""
    simulate(_random_items(seed), seed, in_order=False, rings=(2, 1))
    simulate(_random_items(seed), seed + 7, in_order=True, rings=(2, 1))


@pytest.mark.parametrize("seed", range(40))
def test_other_ring_splits_and_the_split_barrier_form(seed):
    """The other division of the three stages, and the previous revision's
    shared ring with full barriers split by tile kind, are correct too."""
    simulate(_random_items(seed), seed + 11, in_order=False, rings=(1, 2))
    simulate(_random_items(seed), seed + 13, in_order=False, split_full=True)


def test_shared_full_barriers_rely_on_tma_completion_order():
    hits = 0
    for seed in range(400):
        try:
            simulate(_random_items(seed), seed, in_order=False)
        except ProtocolError:
            hits += 1
    assert hits > 0, "expected an interleaving where a later TMA load landing first breaks a parity wait"


def test_dropping_the_q_ready_handshake_aliases():
    """Even with split full barriers, an S issuer that does not wait for the
    softmax's Q-ready arrival lets a softmax Q_FULL wait alias on runs of
    one-tile items."""
    hits = 0
    for seed in range(1500):
        rng = random.Random(seed)
        items = [rng.choice([1, 1, 2]) for _ in range(rng.randint(3, 8))]
        try:
            simulate(items, seed, in_order=False, split_full=True, s_waits_q_ready=False)
        except ProtocolError:
            hits += 1
    assert hits > 0, "the model did not find the aliasing Q_FULL wait"


def test_old_q_free_protocol_without_the_handshake_aliases():
    """The earlier Q-free barrier (one arrival) with the S issuer no longer
    waiting for the softmax's Q-ready: some interleaving must alias."""
    hits = 0
    for seed in range(400):
        rng = random.Random(seed)
        items = [rng.choice([1, 1, 2]) for _ in range(rng.randint(3, 7))]
        try:
            simulate(items, seed, q_free_count=1, s_waits_q_ready=False)
        except ProtocolError:
            hits += 1
    assert hits > 0, "the model did not reproduce the known hazard"
