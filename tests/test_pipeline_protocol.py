"""The staged kernels' copy pipeline (tma_begin / tma_run in
fp8adam_step_tma.cuh), replayed on the CPU as a sequence of events.  For
every sub-tile count and every point at which a wait could give up it checks
the protocol's invariants: each sub-tile is issued once, into stage k %
kStages, only after that stage's previous sub-tile was consumed; each wait
uses the parity of the barrier phase it waits for; and the drain after a
timeout waits for exactly the copies issued and not consumed, so no copy is
in flight when the CTA exits.  The constants are read from the source."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = open(os.path.join(ROOT, "fp8_quantized_adam_b200", "csrc", "fp8adam_step_tma.cuh")).read()
K_STAGES = int(re.search(r"constexpr int kStages = (\d+);", SRC).group(1))
K_SUB = int(re.search(r"constexpr int kSub = (\d+);", SRC).group(1))


def run(nsub, abort_at=None):
    """Events of one CTA: ('issue', k), ('wait', k, stage, parity),
    ('consume', k), ('drain', k, stage, parity); the barrier phase each stage
    is in as the protocol advances."""
    ev = []
    phase = [0] * K_STAGES         # completed phases of each stage's barrier
    in_flight = set()
    consumed = set()

    def issue(k):
        s = k % K_STAGES
        assert k - K_STAGES < 0 or k - K_STAGES in consumed, "stage reused before it was consumed"
        in_flight.add(k)
        ev.append(("issue", k))

    # tma_begin: thread 0 issues the first kStages sub-tiles
    for k in range(min(K_STAGES, nsub)):
        issue(k)
    # tma_run
    for k in range(nsub):
        s, parity = k % K_STAGES, (k // K_STAGES) & 1
        assert parity == phase[s] & 1, "wait parity is not the pending phase"
        if k == abort_at:  # the wait gives up: drain what was issued and not consumed
            last = min(k + K_STAGES, nsub)
            for q in range(k, last):
                ev.append(("drain", q, q % K_STAGES, (q // K_STAGES) & 1))
                in_flight.discard(q)
            return ev, in_flight
        ev.append(("wait", k, s, parity))
        in_flight.discard(k)
        phase[s] += 1
        consumed.add(k)
        ev.append(("consume", k))
        if k + K_STAGES < nsub:
            issue(k + K_STAGES)
    return ev, in_flight


def test_every_subtile_is_issued_once_and_consumed_in_order():
    for nsub in range(0, 40):
        ev, left = run(nsub)
        issued = [e[1] for e in ev if e[0] == "issue"]
        consumed = [e[1] for e in ev if e[0] == "consume"]
        assert sorted(issued) == list(range(nsub)) and consumed == list(range(nsub))
        assert not left


def test_drain_after_a_timeout_leaves_no_copy_in_flight():
    for nsub in range(1, 40):
        for k in range(nsub):
            ev, left = run(nsub, abort_at=k)
            assert not left, (nsub, k)
            drained = [e[1] for e in ev if e[0] == "drain"]
            issued = {e[1] for e in ev if e[0] == "issue"}
            consumed = {e[1] for e in ev if e[0] == "consume"}
            assert set(drained) == issued - consumed, (nsub, k)


def test_stage_geometry():
    # a stage holds kSub elements of p (4 B), g (2 B), m and v (1 B each), and
    # 2 groups of 4 elements for each of the 256 threads
    assert K_SUB == 2 * 4 * 256
    assert "kTmaSmemBytes = kStages * (int)sizeof(TmaStage)" in SRC
    assert K_STAGES * K_SUB * (4 + 2 + 1 + 1) == 48 * 1024
