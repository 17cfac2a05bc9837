"""CPU model of the query-absorption kernel's work split and mbarrier protocol (q_absorb_kernel,
more than 64 tokens).

Work split: (head, 128-token tile) items, head-major, CTA c of G running items
[c F / G, (c + 1) F / G) of F = 128 * ntiles. Every item must run exactly once, and a CTA loads a
head's weights once per run of that head's items.

Protocol, per CTA: one TMA thread loads the head's weights (barrier w_full) when a new head
starts, after the MMAs of the previous head's last item have completed (w_empty), and the item's
q_nope tile into the single A stage after the previous item's MMAs have completed (a_empty); one
MMA thread waits w_full (new head) and a_full, then per half n waits acc_empty[n] (the epilogue
drained half n of the previous item), issues the half's MMAs and commits acc_full[n], then
commits a_empty and, before a new head, w_empty; the epilogue waits acc_full[n], reads half n and
arrives on acc_empty[n]. TMA loads land in any order; MMAs and commits retire in issue order.
An mbarrier parity wait returns once the barrier's current phase parity differs from the one
waited for, so a wait on a barrier one phase behind returns at once: the model plays random
interleavings and reports any read of data that is not (or no longer) the item's, and any
deadlock. A mutant protocol (w_empty committed before the item's A-stage release) is shown to
be caught.
"""
import random

HEADS = 128


def _ranges(ntiles, grid):
    items = HEADS * ntiles
    return [(c * items // grid, (c + 1) * items // grid) for c in range(grid)]


def test_item_ranges_cover_every_item_once():
    for ntiles in range(1, 41):
        items = HEADS * ntiles
        for grid in {1, 7, 128, 148, min(148, items)}:
            if grid > items:
                continue
            seen = [0] * items
            for lo, hi in _ranges(ntiles, grid):
                assert hi > lo                                  # no CTA without work
                for i in range(lo, hi):
                    seen[i] += 1
            assert all(v == 1 for v in seen)


def test_weight_loads_are_one_per_head_run():
    for ntiles in (1, 2, 5, 33):
        for lo, hi in _ranges(ntiles, 148):
            heads = {i // ntiles for i in range(lo, hi)}
            loads = sum(1 for i in range(lo, hi) if i == lo or i % ntiles == 0)
            assert loads == len(heads)


def _parity_complete(completed, phase):
    return (completed & 1) != (phase & 1)


def _run(lo, hi, ntiles, seed, mutant=False):
    """Returns 'ok', 'hazard' or 'deadlock' for one CTA's items [lo, hi)."""
    rnd = random.Random(seed)
    n_items = hi - lo
    head = lambda j: (lo + j) // ntiles
    new_head = lambda j: j == 0 or (lo + j) % ntiles == 0
    h0 = head(0)
    done = {"w_full": 0, "w_empty": 0, "a_full": 0, "a_empty": 0,
            "acc_full0": 0, "acc_full1": 0, "acc_empty0": 0, "acc_empty1": 0}
    wbuf = abuf = None                      # what the weight buffer / A stage hold (landed)
    acc = [None, None]                      # item whose half n the accumulator holds
    drained = [-1, -1]                      # last item whose half n the epilogue has read
    in_flight = []                          # TMA loads: ("w", head) / ("a", item)
    pipe = []                               # tensor pipe, in issue order
    # agent program counters
    prod = {"j": 0, "step": 0}
    mma = {"j": 0, "step": 0}
    epi = {"j": 0, "n": 0}

    def producer():
        j = prod["j"]
        if j >= n_items:
            return False
        if prod["step"] == 0:
            if new_head(j):
                seg = head(j) - h0
                if seg > 0 and not _parity_complete(done["w_empty"], seg - 1):
                    return False
                in_flight.append(("w", head(j)))
            prod["step"] = 1
            return True
        if j >= 1 and not _parity_complete(done["a_empty"], j - 1):
            return False
        in_flight.append(("a", j))
        prod["j"] += 1
        prod["step"] = 0
        return True

    def mma_thread():
        j = mma["j"]
        if j >= n_items:
            return False
        st = mma["step"]
        if st == 0:
            if new_head(j) and not _parity_complete(done["w_full"], head(j) - h0):
                return False
            mma["step"] = 1
            return True
        if st == 1:
            if not _parity_complete(done["a_full"], j):
                return False
            mma["step"] = 2
            return True
        if st in (2, 3):
            n = st - 2
            if j >= 1 and not _parity_complete(done[f"acc_empty{n}"], j - 1):
                return False
            pipe.append(("mma", j, n))
            pipe.append(("commit", f"acc_full{n}"))
            mma["step"] += 1
            return True
        last_of_head = j + 1 < n_items and new_head(j + 1)
        if mutant and last_of_head:
            pipe.insert(len(pipe) - 4, ("commit", "w_empty"))   # released before the item's MMAs
            pipe.append(("commit", "a_empty"))
        else:
            pipe.append(("commit", "a_empty"))
            if last_of_head:
                pipe.append(("commit", "w_empty"))
        mma["j"] += 1
        mma["step"] = 0
        return True

    def epilogue():
        j, n = epi["j"], epi["n"]
        if j >= n_items:
            return False
        if not _parity_complete(done[f"acc_full{n}"], j):
            return False
        if acc[n] != j:
            raise AssertionError("hazard")
        drained[n] = j
        done[f"acc_empty{n}"] += 1
        epi["n"] = 1 - n
        if n == 1:
            epi["j"] += 1
        return True

    def land():
        nonlocal wbuf, abuf
        if not in_flight:
            return False
        kind, v = in_flight.pop(rnd.randrange(len(in_flight)))
        if kind == "w":
            if any(op[0] == "mma" for op in pipe):             # overwrites weights still to be read
                raise AssertionError("hazard")
            wbuf = v
            done["w_full"] += 1
        else:
            if any(op[0] == "mma" for op in pipe):
                raise AssertionError("hazard")
            abuf = v
            done["a_full"] += 1
        return True

    def retire():
        if not pipe:
            return False
        op = pipe.pop(0)
        if op[0] == "mma":
            _, j, n = op
            if wbuf != head(j) or abuf != j or drained[n] < j - 1:
                raise AssertionError("hazard")
            acc[n] = j
        else:
            done[op[1]] += 1
        return True

    agents = [producer, mma_thread, epilogue, land, retire]
    try:
        idle = 0
        while idle < 200:
            if epi["j"] >= n_items and not pipe and not in_flight:
                return "ok"
            progressed = rnd.choice(agents)()
            idle = 0 if progressed else idle + 1
            if idle >= 200 and not any(a() for a in agents):
                return "deadlock"
            elif idle >= 200:
                idle = 0
    except AssertionError:
        return "hazard"
    return "deadlock"


def _cases():
    for ntiles in (1, 2, 3, 5, 33):
        for lo, hi in _ranges(ntiles, 148)[:6] + _ranges(ntiles, 7)[:2]:
            yield lo, hi, ntiles


def test_kernel_protocol_has_no_hazard_or_deadlock():
    for lo, hi, ntiles in _cases():
        for seed in range(40):
            assert _run(lo, hi, ntiles, seed) == "ok", (lo, hi, ntiles, seed)


def test_the_model_catches_an_early_weight_release():
    # a CTA whose range crosses heads: releasing the weights before the item's MMAs retire lets
    # the next head's weights land under them
    lo, hi, ntiles = 3 * 5 - 2, 3 * 5 + 3, 5          # items of heads 2 and 3
    results = {_run(lo, hi, ntiles, seed, mutant=True) for seed in range(200)}
    assert "hazard" in results
