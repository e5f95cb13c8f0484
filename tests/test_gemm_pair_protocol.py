"""Host model of the CTA-pair GEMM's barrier protocol (gemm_pair_kernel in
csrc/gemm_tc.cu).

Two CTAs (rank 0 = leader, rank 1) share each tcgen05 MMA. Per CTA:
- the x producer waits on its own x-empty barrier of stage s, then loads its
  128 tokens of x; the copy completes on the LEADER's x-full barrier, which
  only the leader arms (one arrive.expect_tx for both CTAs' bytes);
- the code producer fills its own code stages (full: copies + one arrival);
- two dequant groups take alternate k-blocks (code stages: 2, so each code stage
  belongs to one group), wait for their code stage, release it, wait on their
  own W-empty barrier, write their CTA's half of the W stage (3 stages, so W
  stages alternate between the groups) and arrive on the LEADER's W-full barrier
  (one group of each CTA completes a phase);
- the epilogue waits on its own accumulator-full barrier, reads its half of the
  accumulator and arrives on the LEADER's accumulator-empty barrier (both CTAs'
  epilogues complete a phase).
The leader's MMA thread waits for accumulator-empty, W-full and x-full (all on
the leader), issues the pair MMA and commits to x-empty, W-empty and
accumulator-full of BOTH CTAs; a commit arrives once every MMA issued before it
has completed, in issue order.

The model runs random interleavings of all roles, copies that land in any
order and a tensor pipe that completes MMAs and commits in order, with
mbarriers that count arrivals and bytes, and checks that no stage or
accumulator is read before it holds what the reader wants, nor overwritten
while a reader still needs its previous contents, and that every tile
finishes. Planted mistakes (a W-full or accumulator-empty barrier that expects
one CTA's arrivals only) must be caught.
"""
import random

import pytest


class Bar:
    def __init__(self, expected):
        self.expected, self.count, self.tx, self.phases, self.overflow = expected, 0, 0, 0, False

    def _settle(self):
        if self.count == self.expected and self.tx == 0:
            self.phases += 1
            self.count = 0

    def arrive(self, tx=0):
        self.tx += tx
        self.count += 1
        self.overflow |= self.count > self.expected
        self._settle()

    def complete_tx(self, b):
        self.tx -= b
        self._settle()

    def passes(self, parity):
        return (self.phases & 1) != parity


def simulate(ntiles, KB, seed, XS=6, WS=3, QS=2, wfull_ctas=2, accempty_ctas=2):
    rng = random.Random(seed)
    XB = 16  # bytes of one CTA's x half-stage (any positive size)
    bars = []
    for c in range(2):
        bars.append(dict(
            xfull=[Bar(1) for _ in range(XS)], xempty=[Bar(1) for _ in range(XS)],
            wfull=[Bar(wfull_ctas) for _ in range(WS)], wempty=[Bar(1) for _ in range(WS)],
            qfull=[Bar(1) for _ in range(QS)], qempty=[Bar(1) for _ in range(QS)],
            accfull=[Bar(1) for _ in range(2)], accempty=[Bar(accempty_ctas) for _ in range(2)]))
    lead = bars[0]
    xstage = [[None] * XS for _ in range(2)]       # x index whose copy landed in the stage
    wstage = [[None] * WS for _ in range(2)]       # k-block whose dequantized W is in the stage
    qstage = [[None] * QS for _ in range(2)]       # k-block whose codes landed in the stage
    inflight = []                                  # copies: (kind, cta, stage, index)
    pipe = []                                      # tensor pipe, in order: ("mma", reads) / ("commit", targets)
    mma_reads = []                                 # (kind, stage, index) read by MMAs not yet complete
    acc_tile = [None, None]                        # tile accumulating (or done) in each accumulator
    acc_mmas_left = {}                             # tile -> MMAs issued but not complete
    epi_reading = {}                               # cta -> (acc, tile)
    deq_reading = {}                               # (cta, group) -> (qstage, kb)
    epi_done = [[False] * ntiles for _ in range(2)]
    violations = []

    def bad(msg):
        violations.append(msg)

    def x_producer(c):
        i = 0
        for _ in range(ntiles):
            for h in range(2 * KB):
                s = i % XS
                while not bars[c]["xempty"][s].passes(((i // XS) & 1) ^ 1):
                    yield
                if c == 0:
                    lead["xfull"][s].arrive(tx=2 * XB)
                inflight.append(("x", c, s, i))
                i += 1
                yield

    def q_producer(c):
        i = 0
        for _ in range(ntiles):
            for _kb in range(KB):
                s = i % QS
                while not bars[c]["qempty"][s].passes(((i // QS) & 1) ^ 1):
                    yield
                inflight.append(("q", c, s, i))
                i += 1
                yield

    def dequant(c, grp):
        for i in range(ntiles * KB):
            if (i & 1) != grp:
                continue
            qs = i % QS
            while not bars[c]["qfull"][qs].passes((i // QS) & 1):
                yield
            if qstage[c][qs] != i:
                bad(f"cta {c} group {grp} reads codes of k-block {i} from stage {qs} holding {qstage[c][qs]}")
            deq_reading[(c, grp)] = (qs, i)
            yield
            del deq_reading[(c, grp)]
            bars[c]["qempty"][qs].arrive()
            ws = i % WS
            while not bars[c]["wempty"][ws].passes(((i // WS) & 1) ^ 1):
                yield
            for kind, st, idx in mma_reads:
                if kind == "w" and st == ws and idx != i:
                    bad(f"cta {c} writes W of k-block {i} into stage {ws} while an MMA reads k-block {idx}")
            wstage[c][ws] = i
            lead["wfull"][ws].arrive()
            yield

    def mma():
        wi = xi = 0
        for j in range(ntiles):
            a = j & 1
            while not lead["accempty"][a].passes(((j >> 1) & 1) ^ 1):
                yield
            for c, (ea, et) in epi_reading.items():
                if ea == a:
                    bad(f"MMA of tile {j} starts in accumulator {a} while cta {c} reads tile {et}")
            if j >= 2 and not all(epi_done[c][j - 2] for c in range(2)):
                bad(f"MMA of tile {j} overwrites accumulator {a} before both epilogues read tile {j - 2}")
            acc_tile[a] = j
            acc_mmas_left[j] = 0
            for _kb in range(KB):
                ws = wi % WS
                while not lead["wfull"][ws].passes((wi // WS) & 1):
                    yield
                for c in range(2):
                    if wstage[c][ws] != wi:
                        bad(f"MMA reads W of k-block {wi} from cta {c} stage {ws} holding {wstage[c][ws]}")
                for _h in range(2):
                    s = xi % XS
                    while not lead["xfull"][s].passes((xi // XS) & 1):
                        yield
                    for c in range(2):
                        if xstage[c][s] != xi:
                            bad(f"MMA reads x {xi} from cta {c} stage {s} holding {xstage[c][s]}")
                    reads = [("w", ws, wi), ("x", s, xi)]
                    mma_reads.extend(reads)
                    acc_mmas_left[j] += 1
                    pipe.append(("mma", reads, j))
                    pipe.append(("commit", [("xempty", s)], None))
                    xi += 1
                    yield
                pipe.append(("commit", [("wempty", ws)], None))
                wi += 1
            pipe.append(("commit", [("accfull", a)], None))
            yield

    def epilogue(c):
        for j in range(ntiles):
            a = j & 1
            while not bars[c]["accfull"][a].passes((j >> 1) & 1):
                yield
            if acc_tile[a] != j or acc_mmas_left.get(j, 1) != 0:
                bad(f"cta {c} reads accumulator {a} for tile {j}: holds {acc_tile[a]}, "
                    f"{acc_mmas_left.get(j)} MMAs outstanding")
            epi_reading[c] = (a, j)
            yield
            del epi_reading[c]
            epi_done[c][j] = True
            lead["accempty"][a].arrive()

    agents = [x_producer(0), x_producer(1), q_producer(0), q_producer(1), dequant(0, 0), dequant(0, 1),
              dequant(1, 0), dequant(1, 1), mma(), epilogue(0), epilogue(1)]
    live = list(agents)
    for _ in range(400000):
        if not live and not inflight and not pipe:
            break
        r = rng.random()
        if r < 0.25 and inflight:  # a copy lands
            kind, c, s, i = inflight.pop(rng.randrange(len(inflight)))
            if kind == "x":
                for k, st, idx in mma_reads:
                    if k == "x" and st == s and idx != i:
                        bad(f"x {i} lands in cta {c} stage {s} while an MMA reads x {idx}")
                xstage[c][s] = i
                lead["xfull"][s].complete_tx(XB)
            else:
                for (cc, _g), (qs, idx) in deq_reading.items():
                    if cc == c and qs == s and idx != i:
                        bad(f"codes of k-block {i} land in cta {c} stage {s} while k-block {idx} is read")
                qstage[c][s] = i
                bars[c]["qfull"][s].arrive()
        elif r < 0.45 and pipe:  # the tensor pipe completes its oldest operation
            op, arg, j = pipe.pop(0)
            if op == "mma":
                for rd in arg:
                    mma_reads.remove(rd)
                acc_mmas_left[j] -= 1
            else:
                for name, idx in arg:  # commit with a multicast to both CTAs
                    for c in range(2):
                        bars[c][name][idx].arrive()
        elif live:
            ag = rng.choice(live)
            try:
                next(ag)
            except StopIteration:
                live.remove(ag)
    finished = not live and all(all(d) for d in epi_done)
    for b in bars:
        for lst in b.values():
            if any(x.overflow for x in lst):
                violations.append("an arrival beyond a barrier's expected count")
    return violations, finished


@pytest.mark.parametrize("ntiles,KB", [(1, 1), (1, 5), (3, 2), (4, 7), (6, 3)])
@pytest.mark.parametrize("seed", range(4))
def test_the_pair_protocol_reads_every_stage_and_accumulator_in_time(ntiles, KB, seed):
    violations, finished = simulate(ntiles, KB, seed)
    assert violations == []
    assert finished


def test_a_w_full_barrier_counting_one_cta_lets_the_mma_read_the_peers_half_early():
    found = []
    for seed in range(20):
        v, _ = simulate(4, 7, seed, wfull_ctas=1)
        found += v
    assert any("MMA reads W" in v for v in found)


def test_an_accumulator_empty_barrier_counting_one_cta_lets_the_mma_overwrite_a_tile_being_read():
    found = []
    for seed in range(20):
        v, _ = simulate(6, 1, seed, accempty_ctas=1)
        found += v
    assert any("MMA of tile" in v for v in found)
