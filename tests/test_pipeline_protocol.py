"""The forward kernel's pipeline arithmetic, checked on the host (no GPU).

hstu_fwd_kernel streams K and V through a ring of shared-memory slots in the order its MMA warp
consumes them: group g issues the P.V of tile g-3 (reading V_{g-3}) and then the scores of tile g
(reading K_g), so the loads run K_0 K_1 K_2 | V_0 K_3 | V_1 K_4 | ... and end with the last (up to)
three V tiles.  The producer reuses the slot of load j once the group that consumed load
j - kStages has completed, found with group_of_load(e) = e for e < 3, (e + 3) // 2 otherwise, and
waits on that group's score commit, which rotates over kSCommits barriers; each group's inputs
arrive on one of kGroupBars ready barriers.

This module restates those rules in Python and replays them on random sequences of tile counts, to
show that (1) group_of_load names the group that really consumed each load, (2) a slot is never
reused before its previous tile was consumed, (3) no parity wait can see a barrier two phases
ahead, for the ring depths the kernel uses (6 slots at d = 128, 10 at d <= 64), and (4) the
constraint kStages <= 2 kSCommits - 2 stated beside the kernel's configuration is the exact limit.
An event-level model of the group barriers then replays random interleavings of the roles, with
and without an abort, to show that no arrival ever lands on a phase with no pending arrivals, and
that the abort path's earlier stand-in arrivals could.  Last, the Q-buffer waits (one buffer at
d = 128, two at d <= 64) are checked against the MMA warp's per-query-tile commits.
"""
import numpy as np
import pytest

K_SCOMMITS = 6
K_GROUP_BARS = 8


def group_of_load(e):
    return e if e < 3 else (e + 3) // 2


def load_sequence(tiles):
    """(kind, tile) of every K/V load in producer order, for `tiles` score tiles in all."""
    seq = []
    for g in range(tiles):
        if g >= 3:
            seq.append(("V", g - 3))
        seq.append(("K", g))
    for t in range(max(tiles - 3, 0), tiles):
        seq.append(("V", t))
    return seq


def consuming_group(kind, tile):
    """The MMA group that reads a K or V tile: S_t in group t, P.V of tile t in group t + 3."""
    return tile if kind == "K" else tile + 3


def replay(tiles, stages):
    """Check the reuse and phase rules for one CTA's stream of `tiles` score tiles."""
    seq = load_sequence(tiles)
    groups = [consuming_group(k, t) for k, t in seq]
    # Each group reads at most one K and one V, in the order the producer loads them.
    assert groups == sorted(groups)
    last_s_group = tiles - 1  # groups after this one issue P.V only and commit no scores
    for j in range(len(seq)):
        g_j = groups[j]
        if j < stages:
            continue
        e = j - stages
        G = group_of_load(e)
        # (1) the lookup names the consumer of the slot's previous tile (it is never a P.V-only group)
        assert G == groups[e] and G <= last_s_group, (tiles, stages, j)
        # (2) load j comes after load e was consumed: its own consumer is a later group
        assert g_j > G
        # (3) score commits: waiting on barrier G % K_SCOMMITS for phase G // K_SCOMMITS is unambiguous
        # only if group G + K_SCOMMITS cannot have committed yet, i.e. its K tile is not loaded yet.
        k_late = 2 * (G + K_SCOMMITS) - 2 if G + K_SCOMMITS >= 3 else G + K_SCOMMITS
        assert k_late >= j, (tiles, stages, j, G)
        # (4) group-ready barriers: the producer arms group g_j only after group G completed, so group
        # g_j - K_GROUP_BARS (same barrier, previous phase) was consumed long before.
        assert g_j - K_GROUP_BARS < G + 1
    return True


@pytest.mark.parametrize("stages", [5, 6, 10])
def test_ring_rules_hold_for_random_streams(stages):
    rng = np.random.default_rng(100 + stages)
    for tiles in list(range(1, 40)) + list(rng.integers(40, 400, 20)):
        assert replay(int(tiles), stages)


def test_group_of_load_matches_the_load_order():
    seq = load_sequence(50)
    for e, (kind, t) in enumerate(seq[:-3]):
        assert group_of_load(e) == consuming_group(kind, t)


def test_ring_depth_limit_is_exact():
    """kStages <= 2 kSCommits - 2: the deepest ring the score-commit rotation can track."""
    limit = 2 * K_SCOMMITS - 2
    assert replay(200, limit)
    with pytest.raises(AssertionError):
        replay(200, limit + 1)


def test_three_commit_barriers_would_not_cover_the_deep_ring():
    """With one score-commit barrier per score buffer (3), a 10-slot ring lets a group two phases
    ahead complete before the producer checks: the failure the rotating commits avoid."""
    global K_SCOMMITS
    saved = K_SCOMMITS
    try:
        K_SCOMMITS = 3
        with pytest.raises(AssertionError):
            replay(200, 10)
        assert replay(200, 4)
    finally:
        K_SCOMMITS = saved


# ---------------------------------------------------------------------------------------------
# Event-level model of the group barriers, with an abort at a random moment.
#
# Group g of the MMA warp waits on g_ready[g mod 8]: the producer's expect-tx arrival plus the
# bytes of the group's copies (Q on a query tile's first tile, V_{g-3}, K_g), and, for g >= 3, the
# arrivals of the four SiLU warps that wrote P_{g-3} (the producer stands in for them when g < 3).
# On abort every role leaves its loop; SiLU warps that already read a tile may still arrive, and
# copies in flight still land.  The producer then lets its copies land before the CTA ends.
#
# An mbarrier arrival on a phase with no arrivals pending while bytes are still outstanding is not
# defined; the model flags it.  An earlier drain added the four SiLU arrivals to each barrier still
# in use and then waited for its phase, which can do exactly that when the SiLU warps did arrive.
# The kernel's drain only waits (within a time budget, as a phase whose SiLU arrivals never come
# cannot complete).
# ---------------------------------------------------------------------------------------------
class Barrier:
    def __init__(self, count):
        self.count, self.phase, self.pending, self.tx = count, 0, count, 0

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self, phase_expected, n=1, tx=0, check_phase=True):
        for i in range(n):
            if self.pending == 0:
                raise AssertionError("arrival on a phase with no pending arrivals (bytes outstanding: %d)" % self.tx)
            if check_phase:
                assert self.phase == phase_expected, ("arrival for the wrong phase", self.phase, phase_expected)
            self.pending -= 1
            if i == 0:
                self.tx += tx
            self._maybe_complete()

    def bytes_landed(self, nbytes):
        self.tx -= nbytes
        self._maybe_complete()

    def done(self, phase):
        return self.phase > phase


def simulate(tiles, rng, abort_at=None, stand_in_on_abort=False, lag=2):
    """One CTA's groups 0 .. tiles+2 under a random interleaving; returns the number of steps.
    After an abort the producer's drain runs interleaved with the copies still landing and the
    SiLU arrivals still to come."""
    nbar = K_GROUP_BARS
    bars = [Barrier(1 + 4) for _ in range(nbar)]
    closing = list(range(max(tiles - 3, 0), tiles))
    arm_order = list(range(tiles)) + [t + 3 for t in closing]  # groups in the order the producer arms them
    armed, mma_next, in_flight, silu_todo = 0, 0, [], []
    mma_done = set()
    aborted, step = False, 0
    drain, drain_i, drain_arrived = [], 0, False
    while True:
        step += 1
        if abort_at is not None and step == abort_at:
            aborted = True
            drain = arm_order[max(armed - nbar, 0):armed]
        actions = []
        if not aborted and armed < len(arm_order):
            # ring slots free once the group armed `lag` places earlier has completed
            if armed - lag < 0 or arm_order[armed - lag] in mma_done:
                actions.append("arm")
        if not aborted and mma_next < len(arm_order):
            x = arm_order[mma_next]
            if bars[x % nbar].done(x // nbar):
                actions.append("mma")
        if in_flight:
            actions.append("land")
        if silu_todo:
            actions.append("silu")  # may run after abort: a warp past its score wait still arrives
        if drain_i < len(drain):
            x = drain[drain_i]
            if (stand_in_on_abort and not drain_arrived) or bars[x % nbar].done(x // nbar):
                actions.append("drain")
        if not actions:
            break
        a = actions[rng.integers(len(actions))]
        if a == "arm":
            x = arm_order[armed]
            armed += 1
            bars[x % nbar].arrive(x // nbar, tx=1)
            in_flight.append(x)
            if x < 3:
                bars[x % nbar].arrive(x // nbar, n=4)
        elif a == "mma":
            x = arm_order[mma_next]
            mma_next += 1
            mma_done.add(x)
            if x < tiles:
                silu_todo.append(x)  # S_x computed: its SiLU tile feeds group x + 3
        elif a == "land":
            x = in_flight.pop(rng.integers(len(in_flight)))
            bars[x % nbar].bytes_landed(1)
        elif a == "silu":
            t = silu_todo.pop(0)
            # after a stand-in drain a late arrival may meet a phase the drain already opened
            bars[(t + 3) % nbar].arrive((t + 3) // nbar, n=4, check_phase=not stand_in_on_abort)
        else:
            x = drain[drain_i]
            if stand_in_on_abort and not drain_arrived:
                bars[x % nbar].arrive(x // nbar, n=4, check_phase=False)  # the earlier drain's stand-ins
                drain_arrived = True
            else:
                drain_i += 1  # this phase completed: its copies landed
                drain_arrived = False
    if not aborted:
        assert mma_next == len(arm_order) and not in_flight
    return step, drain, drain_i


def test_group_barriers_hold_under_random_interleavings_and_aborts():
    """No arrival ever meets a phase with none pending, with or without an abort, and once every
    copy has landed a drained phase is either complete or still waits for SiLU arrivals that will
    never come (the case the drain's time budget covers)."""
    rng = np.random.default_rng(7)
    for trial in range(800):
        tiles = int(rng.integers(1, 30))
        total, _, _ = simulate(tiles, rng)  # no abort: every group runs
        simulate(tiles, rng, abort_at=int(rng.integers(1, total + 1)))


def test_stand_in_arrivals_on_abort_can_meet_a_phase_with_none_pending():
    """The earlier drain (four stand-in arrivals, then a wait) reaches an arrival on a phase with
    no arrivals pending while bytes are outstanding in some interleavings."""
    hit = 0
    for trial in range(600):
        rng = np.random.default_rng(trial)
        tiles = int(rng.integers(4, 30))
        total, _, _ = simulate(tiles, np.random.default_rng(trial))
        try:
            simulate(tiles, np.random.default_rng(trial + 1000), abort_at=int(rng.integers(1, total + 1)),
                     stand_in_on_abort=True)
        except AssertionError as e:
            if "no pending arrivals" in str(e):
                hit += 1
    assert hit > 0


# ---------------------------------------------------------------------------------------------
# Q buffers.  Query tile s (the s-th the CTA takes) goes into buffer s mod kQBufs.  The MMA warp
# commits q_empty[b] after a query tile's last score MMA; before loading tile s the producer waits
# on q_empty[s mod kQBufs] with parity ((s / kQBufs) & 1) ^ 1.  An mbarrier parity wait succeeds once
# the phase of that parity has completed, and a fresh barrier counts its phase before phase 0 as
# completed with parity 1.
# ---------------------------------------------------------------------------------------------
def q_wait_passes(completions, parity):
    """try_wait.parity on a barrier that has completed `completions` phases: it passes while the
    current phase's parity differs from the one asked for, so it cannot tell phases two apart."""
    return (completions & 1) != parity


@pytest.mark.parametrize("qbufs", [1, 2])
def test_q_buffer_waits_release_exactly_after_the_previous_user_of_the_buffer(qbufs):
    """For every query tile s, the producer's wait passes exactly when tile s - kQBufs (the buffer's
    previous user) has committed.  Tiles commit in order, and the producer reached tile s only after
    its wait for tile s - 1 passed, so tiles up to s - 1 - kQBufs have committed: `done`, the number of
    committed tiles, is at least s - kQBufs, which keeps the parity wait unambiguous."""
    for s in range(12):
        b = s % qbufs
        parity = ((s // qbufs) & 1) ^ 1
        for done in range(max(0, s - qbufs), s + 1):
            completions = sum(1 for t in range(done) if t % qbufs == b)
            ok = q_wait_passes(completions, parity)
            assert ok == (s < qbufs or done > s - qbufs), (qbufs, s, done)


def test_q_buffer_parity_is_what_catches_a_wrong_buffer_count():
    """A planted mistake: the parity of two buffers with a single buffer's commits (kQBufs changed in
    one place only) lets the wait for tile 2 pass before tile 1 has committed."""
    s, done = 2, 1  # one buffer: tile 2 must wait for tile 1, which has not committed
    completions = done  # every tile commits on the one barrier
    parity_two_buffer_formula = ((s // 2) & 1) ^ 1
    assert q_wait_passes(completions, parity_two_buffer_formula)  # would pass too early
