"""CPU model of the sparse-MLA kernel's mbarrier protocol for the gathered key data.

The kernel's three Q K^T issuers take the 32-key tiles round robin (issuer e: tiles e, e+3, ...),
and the gather fills a ring of slots whose "full" barrier a later tile's issuer waits on with a
parity wait. An mbarrier parity wait returns as soon as the phase with that parity is complete
relative to the barrier's current phase, so on a barrier still one phase behind, a wait for the
next phase returns at once. What keeps each issuer's wait on its own phase is the ordering around
it. The model plays random interleavings of gathers landing (in order), gathers being issued (once
the tile that last used the slot has been read) and issuers waiting, with that parity rule, and
reports whether a Q K^T could start before its own tile's data has landed.

- The kernel's configuration: four slots in the ring Q K^T reads for three issuers. A slot's previous
  user is tile j - 4, which landed before tile j - 3, the issuer's own previous tile, whose data it
  has already waited for: never early, with or without the issuer's wait for P V of tile j - 3.
- Two slots with three issuers and a single wait (a layout tried while developing the kernel) does
  start early; waiting first for the slot's previous phase closes it. The model shows the hazard is
  real, so the slot count and the ordering are load-bearing.
"""
import random


def _parity_complete(completed_phases: int, phase: int) -> bool:
    # the barrier's current (incomplete) phase is `completed_phases`; a parity wait for `phase`
    # returns when the current phase's parity differs from the wanted one
    return (completed_phases & 1) != (phase & 1)


def _run(ntiles, seed, slots, two_step=False, order_after_pv=True) -> bool:
    rnd = random.Random(seed)
    full = [0] * slots                     # completed phases per slot barrier
    issued = landed = 0                    # gathers issued / landed (they land in order)
    qk_done = [False] * ntiles
    stage = {}
    todo = {e: list(range(e, ntiles, 3)) for e in range(3)}
    for _ in range(20000):
        if not any(todo.values()):
            return True
        r = rnd.random()
        if r < 0.3:
            if issued < ntiles and (issued < slots or qk_done[issued - slots]):
                issued += 1
        elif r < 0.6:
            if landed < issued:
                full[landed % slots] += 1
                landed += 1
        else:
            e = rnd.randrange(3)
            if not todo[e]:
                continue
            j = todo[e][0]
            # the issuer first waits for P V of tile j - 3 (modelled as that tile's Q K^T, which
            # P V follows), whose data landed before tile j - 2's
            if order_after_pv and j >= 3 and not qk_done[j - 3]:
                continue
            s = j % slots
            if two_step and j >= slots and stage.get(j, 0) == 0:
                if _parity_complete(full[s], j // slots - 1):
                    stage[j] = 1
                continue
            if _parity_complete(full[s], j // slots):
                if landed <= j:                        # Q K^T would read a slot still being filled
                    return False
                qk_done[j] = True
                todo[e].pop(0)
    return True


def test_kernel_configuration_never_reads_early():
    assert all(_run(n, seed, slots=4) for n in range(1, 14) for seed in range(200))


def test_two_slots_need_the_two_step_wait():
    assert not all(_run(n, seed, slots=2) for n in range(1, 12) for seed in range(200))
    assert all(_run(n, seed, slots=2, two_step=True) for n in range(1, 12) for seed in range(200))


def test_four_slots_are_ordered_by_the_issuers_own_waits():
    assert all(_run(n, seed, slots=4, order_after_pv=False) for n in range(1, 14) for seed in range(200))
