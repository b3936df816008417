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
ahead, for the ring depths the kernel uses (5 slots at d = 128, 10 at d <= 64), and (4) the
constraint kStages <= 2 kSCommits - 2 stated beside the kernel's configuration is the exact limit.
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


@pytest.mark.parametrize("stages", [5, 10])
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
