"""Host model of the W4A16 GEMM's code-stage protocol (csrc/gemm_tc.cu).

Two groups of dequant warps take alternate k-blocks i (group i % 2) from a
ring of S code stages (stage i % S). One producer fills stage s with k-block i
only after the stage's previous use was consumed, but copies land out of
order. A consumer waits with mbarrier.try_wait.parity(u % 2) for use u of its
stage, which passes whenever the barrier's current phase parity differs, so
the wait is only sound if the barrier is at phase u or u + 1 then.

With an odd S the uses of a stage alternate between the groups, and a group
can arrive two phases early (its own previous k-block landed, the other
group's use of this stage did not): the model finds reads of stages whose copy
had not landed. With an even S (the kernel's 4 or 2) every stage belongs to
one group, the waits are sound, and every k-block is read only after it
landed."""
import random

import pytest


def simulate(kblocks: int, stages: int, seed: int):
    """Returns (reads of a not-yet-landed stage, whether every k-block was consumed)."""
    rng = random.Random(seed)
    landed = [False] * kblocks
    consumed = [False] * kblocks
    full_phases = [0] * stages    # completed phases of each stage's full barrier
    empty_phases = [0] * stages   # completed phases of each stage's empty barrier
    pos = [0, 1]                  # next k-block of each group
    issue, inflight, bad = 0, [], 0
    for _ in range(400000):
        if all(consumed):
            break
        if issue < kblocks:  # the producer, in k-block order
            s, u = issue % stages, issue // stages
            if u == 0 or empty_phases[s] >= u:
                inflight.append(issue)
                issue += 1
        if inflight and rng.random() < 0.5:  # some copy in flight lands
            i = inflight.pop(rng.randrange(len(inflight)))
            landed[i] = True
            s = i % stages
            while full_phases[s] * stages + s < kblocks and landed[full_phases[s] * stages + s]:
                full_phases[s] += 1
        g = rng.randrange(2)  # one group tries its next k-block
        i = pos[g]
        if i >= kblocks:
            continue
        s, u = i % stages, i // stages
        if (full_phases[s] & 1) != (u & 1):  # try_wait.parity(u % 2) passes
            bad += not landed[i]
            consumed[i] = True
            while empty_phases[s] * stages + s < kblocks and consumed[empty_phases[s] * stages + s]:
                empty_phases[s] += 1
            pos[g] += 2
    return bad, all(consumed)


@pytest.mark.parametrize("stages", [2, 4])
@pytest.mark.parametrize("seed", range(10))
def test_an_even_ring_reads_every_stage_after_its_copy_landed(stages, seed):
    assert simulate(96, stages, seed) == (0, True)


def test_an_odd_ring_shared_by_alternating_groups_can_read_before_the_copy_lands():
    assert sum(simulate(96, 3, s)[0] for s in range(10)) > 0
