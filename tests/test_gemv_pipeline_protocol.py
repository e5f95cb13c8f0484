"""Host model of the decode GEMV's stage protocol (csrc/gemv.cu).

A CTA streams its units through a ring of NS shared-memory stages (unit i in
stage i % NS, use u = i // NS of that stage). Per stage there are three
mbarriers:
- full: 32 cp.async arrivals (one per producer lane, when that lane's scale
  and zero copies have landed), the producer's arrive.expect_tx carrying the
  code bytes (and the x bytes when there is no x-prep warp), and, with an x-prep
  warp, that warp's arrival once it has written the stage's x sums;
- xland (with an x-prep warp): the producer's arrive.expect_tx carrying the x
  bytes;
- empty: one arrival from each consumer warp when it is done with the stage.
The producer issues use u of a stage after waiting on empty with parity
(u - 1) % 2 (not for u = 0); the x-prep warp waits on xland and the consumers on
full with parity u % 2. A parity wait passes whenever the barrier's phase
parity differs, so it is only sound if the barrier is at phase u or u + 1 when
the waiter asks.

The model runs random interleavings of the producer, the copies landing in any
order, the x-prep warp and the consumer warps, with mbarriers that count
arrivals and transaction bytes as the hardware does, and checks that
- no copy lands in a stage that a warp is still reading (a previous use);
- the x-prep warp reads x only after it landed, and writes its sums only after
  every consumer is done with the stage's previous use;
- a consumer reads codes, scales, zeros and x sums (or x) of use u only after
  all of them landed or were written for use u;
- every unit is consumed by every consumer warp.
A planted mistake (one arrival too few expected on full, or a producer that
does not wait for empty) must produce a violation, so the model is not vacuous.
"""
import random

import pytest


class Bar:
    """An mbarrier: a phase completes when its pending arrival count reaches
    zero and its transaction count is zero. An arrival beyond the expected
    count while the phase still waits for bytes is undefined on the hardware;
    the model records it."""

    def __init__(self, expected):
        self.expected, self.count, self.tx, self.phases = expected, 0, 0, 0
        self.overflow = False

    def _settle(self):
        if self.count == self.expected and self.tx == 0:
            self.phases += 1
            self.count = 0

    def arrive(self, tx=0):
        self.tx += tx
        self.count += 1
        if self.count > self.expected:
            self.overflow = True
        self._settle()

    def complete_tx(self, b):
        self.tx -= b
        self._settle()

    def passes(self, parity):
        # try_wait.parity(p) passes once the phase with parity p completed,
        # i.e. whenever the current phase's parity differs from p
        return (self.phases & 1) != parity


def simulate(units, NS, consumers, xwarp, seed, full_extra=0, producer_waits=True):
    rng = random.Random(seed)
    full = [Bar(33 + (1 if xwarp else 0) + full_extra) for _ in range(NS)]
    xland = [Bar(1) for _ in range(NS)]
    empty = [Bar(consumers) for _ in range(NS)]
    CODE, X = 1000, 7  # transaction bytes of one use (any positive sizes)
    landed = [dict(code=False, small=0, x=False, xs=False) for _ in range(units)]
    reading = {}          # warp -> (stage, unit) it is reading now
    inflight = []         # (unit, kind) copies issued, not landed
    issued = 0
    xpos, cpos = 0, [0] * consumers
    done = [[False] * units for _ in range(consumers)]
    violations = []

    def check_stage_free(s, i, what):
        for w, (rs, ri) in reading.items():
            if rs == s and ri != i:
                violations.append(f"{what} of unit {i} lands in stage {s} while {w} reads unit {ri}")

    for _ in range(200000):
        if all(all(d) for d in done) and not reading and not inflight:
            break
        r = rng.random()
        if r < 0.2 and issued < units:  # producer: issue the next unit
            i, s = issued, issued % NS
            u = i // NS
            if u == 0 or not producer_waits or empty[s].passes((u - 1) & 1):
                full[s].arrive(tx=CODE + (0 if xwarp else X))
                if xwarp:
                    xland[s].arrive(tx=X)
                inflight += [(i, "code"), (i, "x")] + [(i, "small")] * 32
                issued += 1
        elif r < 0.5 and inflight:  # some copy lands
            i, kind = inflight.pop(rng.randrange(len(inflight)))
            s = i % NS
            check_stage_free(s, i, kind)
            if kind == "code":
                landed[i]["code"] = True
                full[s].complete_tx(CODE)
            elif kind == "small":
                landed[i]["small"] += 1
                full[s].arrive()          # cp.async.mbarrier.arrive.noinc
            else:
                landed[i]["x"] = True
                (xland[s] if xwarp else full[s]).complete_tx(X)
        elif r < 0.6 and xwarp:  # the x-prep warp
            if "xprep" in reading:  # finish: write the sums, arrive on full
                s, i = reading.pop("xprep")
                for c in range(consumers):
                    if i >= NS and not done[c][i - NS]:
                        violations.append(f"x sums of unit {i} written while consumer {c} reads unit {i - NS}")
                landed[i]["xs"] = True
                full[s].arrive()
                xpos += 1
            elif xpos < units:
                s, u = xpos % NS, xpos // NS
                if xland[s].passes(u & 1):
                    if not landed[xpos]["x"]:
                        violations.append(f"x-prep reads x of unit {xpos} before it landed")
                    reading["xprep"] = (s, xpos)
        else:  # one consumer warp
            c = rng.randrange(consumers)
            w = f"consumer{c}"
            if w in reading:  # finish reading: release the stage
                s, i = reading.pop(w)
                done[c][i] = True
                cpos[c] += 1
                empty[s].arrive()
            elif cpos[c] < units:
                i = cpos[c]
                s, u = i % NS, i // NS
                if full[s].passes(u & 1):
                    st = landed[i]
                    ok = st["code"] and st["small"] == 32 and st["x"] and (st["xs"] or not xwarp)
                    if not ok:
                        violations.append(f"consumer {c} reads unit {i} before its data is in: {st}")
                    reading[w] = (s, i)
    complete = all(all(d) for d in done)
    if any(b.overflow for b in full + xland + empty):
        violations.append("an arrival beyond a barrier's expected count")
    return violations, complete


@pytest.mark.parametrize("xwarp", [True, False])
@pytest.mark.parametrize("NS", [1, 2, 3, 4, 7])
@pytest.mark.parametrize("seed", range(4))
def test_every_stage_is_read_after_it_landed_and_rewritten_after_release(xwarp, NS, seed):
    violations, complete = simulate(units=24, NS=NS, consumers=8, xwarp=xwarp, seed=seed)
    assert violations == []
    assert complete


def test_one_arrival_too_few_on_full_lets_consumers_read_early():
    found = []
    for seed in range(20):
        found += simulate(units=24, NS=3, consumers=8, xwarp=True, seed=seed, full_extra=-1)[0]
    assert any("before its data is in" in v for v in found)


def test_a_producer_that_does_not_wait_for_empty_breaks_the_protocol():
    # it overwrites a stage in use, or its arrivals run past a phase
    for seed in range(20):
        violations, complete = simulate(units=24, NS=2, consumers=8, xwarp=True, seed=seed, producer_waits=False)
        assert violations or not complete
