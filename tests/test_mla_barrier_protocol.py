"""CPU model of the sparse-MLA exchange kernel's mbarrier protocol for the gathered key data.

The kernel has two data slots and three Q K^T issuers (issuer e takes pair-tiles e, e+3, ...), so
the previous user of a slot's barrier phase is another issuer. An mbarrier parity wait returns as
soon as the phase with that parity is complete relative to the barrier's current phase: on a
barrier still one phase behind, the wait for parity P returns at once (the "preceding phase" has
parity P). The model plays random interleavings of gathers completing, gathers being issued (only
once Q K^T of the pair-tile two earlier has read the slot) and issuers waiting, with that parity
rule, and checks that no Q K^T starts before its own gather has landed: true with the kernel's
two-step wait (the slot's previous phase, then its own), false with a single wait.
"""
import random


def _parity_complete(completed_phases: int, phase: int) -> bool:
    # the barrier's current (incomplete) phase is `completed_phases`; a parity wait for `phase`
    # returns when the current phase's parity differs from the wanted one
    return (completed_phases & 1) != (phase & 1)


def _run(ntiles: int, seed: int, two_step: bool) -> bool:
    rnd = random.Random(seed)
    kv_full = [0, 0]                       # completed phases per slot barrier
    issued = landed = 0                    # gathers issued / landed (they land in order)
    qk_done = [False] * ntiles
    stage = {}
    todo = {e: list(range(e, ntiles, 3)) for e in range(3)}
    for _ in range(20000):
        if not any(todo.values()):
            return True
        r = rnd.random()
        if r < 0.3:
            if issued < ntiles and (issued < 2 or qk_done[issued - 2]):
                issued += 1
        elif r < 0.6:
            if landed < issued:
                kv_full[landed % 2] += 1
                landed += 1
        else:
            e = rnd.randrange(3)
            if not todo[e]:
                continue
            j = todo[e][0]
            if j >= 3 and not qk_done[j - 3]:          # the issuer's wait for P V of pair-tile j - 3
                continue
            s = j % 2
            if two_step and j >= 2 and stage.get(j, 0) == 0:
                if _parity_complete(kv_full[s], j // 2 - 1):
                    stage[j] = 1
                continue
            if _parity_complete(kv_full[s], j // 2):
                if landed <= j:                        # Q K^T would read a slot still being filled
                    return False
                qk_done[j] = True
                todo[e].pop(0)
    return True


def test_two_step_wait_never_reads_early():
    assert all(_run(n, seed, two_step=True) for n in range(1, 12) for seed in range(200))


def test_single_wait_would_read_early():
    # the model does reach the hazard the two-step wait removes
    assert not all(_run(n, seed, two_step=False) for n in range(1, 12) for seed in range(200))
