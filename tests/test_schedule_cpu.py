"""Pins for the split-KV schedule of the oracle: structural validity on random batches
and a schedule worked out by hand."""

import numpy as np
import pytest

from oracle import mla_oracle as O


def check_valid(seqlens, s_q, H, workers):
    sc = O.schedule_ref(seqlens, s_q, H, workers)
    B = len(seqlens)
    P = sc["num_parts"]
    T = sc["num_tiles"]
    assert T == -(-(s_q * H) // 128)
    assert P == max(1, workers // T)
    nblk = sc["nblk"]
    assert np.array_equal(nblk, [(n + 63) // 64 if n > 0 else 0 for n in seqlens])
    covered = {b: [] for b in range(B)}
    costs = []
    for p in range(P):
        pieces = O.pieces_of_partition(sc, p)
        cost = 0
        for b, lo, hi, s in pieces:
            assert 0 <= lo < hi <= nblk[b]
            # cuts fall on whole key tiles: a piece starts on a tile boundary and
            # ends on one or at the sequence end
            assert lo % O.SCHED_BLOCKS_PER_TILE == 0
            assert hi % O.SCHED_BLOCKS_PER_TILE == 0 or hi == nblk[b]
            covered[b].append((s, lo, hi, p))
            cost += -(-(hi - lo) // O.SCHED_BLOCKS_PER_TILE)
        costs.append(cost)
    for b in range(B):
        parts = sorted(covered[b])
        # every block exactly once, contiguous, split indices 0..num_splits-1 in order
        assert len(parts) == sc["num_splits"][b]
        k = 0
        for i, (s, lo, hi, p) in enumerate(parts):
            assert s == i and lo == k
            assert p == sc["first_part"][b] + i
            k = hi
        assert k == nblk[b]
    assert sc["total_slots"] == int(np.sum(sc["num_splits"]))
    assert np.array_equal(sc["split_prefix"], np.concatenate([[0], np.cumsum(sc["num_splits"])[:-1]]))
    # each sequence is cut at most once per partition boundary
    assert sc["total_slots"] <= B + P - 1
    # balance: no partition exceeds the cap (tiles only; the overhead sits before tiles)
    assert max(costs) <= sc["cap"]
    return sc


@pytest.mark.parametrize("seed", range(12))
def test_random_schedules_valid(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 300))
    seqlens = rng.integers(0, 5000, size=B)
    seqlens[rng.random(B) < 0.1] = 0
    s_q = int(rng.integers(1, 5))
    H = int(rng.choice([16, 32, 64, 128]))
    workers = int(rng.choice([1, 7, 74, 256]))
    check_valid(seqlens, s_q, H, workers)


@pytest.mark.parametrize("name", ["tiny", "decode_b64", "mtp_b128_sq2", "serving_b256", "long_b4"])
def test_workload_schedules_valid(name):
    from deepseek_mla_decode_b200.workloads import WORKLOADS

    w = WORKLOADS[name]
    check_valid(w.seqlens(), w.s_q, w.H, 74)


def test_hand_worked_schedule():
    """Two sequences of 16 and 3 blocks (n = 1000, 129), 2 partitions, tiles of 4
    blocks, overhead 1 tile: 4 and 1 tiles, costs 5 and 2, total 7,
    cap = max(2, ceil(7/2)) = 4.  Positions: seq0 tiles at 1..4, seq1's tile at 6.
    Tile->partition: seq0 tiles 0..2 -> 0 (pos 1..3), tile 3 -> 1 (pos 4); seq1 -> 1.
    Partition 1 starts at position 4 = seq0 tile 3 = block 12."""
    sc = O.schedule_ref(np.array([1000, 129]), 1, 128, 2)
    assert sc["cap"] == 4 and sc["num_parts"] == 2
    assert sc["part_start"].tolist() == [[0, 0], [0, 12]]
    assert sc["part_end"].tolist() == [[0, 12], [2, 0]]
    assert sc["num_splits"].tolist() == [2, 1]
    assert sc["first_part"].tolist() == [0, 1]
    assert sc["split_prefix"].tolist() == [0, 2]
    assert O.pieces_of_partition(sc, 0) == [(0, 0, 12, 0)]
    assert O.pieces_of_partition(sc, 1) == [(0, 12, 16, 1), (1, 0, 3, 0)]


def test_min_cap_keeps_tiny_problems_whole():
    sc = O.schedule_ref(np.array([37, 130]), 1, 16, 74)
    # 1 and 3 blocks = 1 tile each, costs 2 and 2, total 4 -> cap = max(2, 1) = 2:
    # seq0's tile at position 1 -> partition 0, seq1's tile at 3 -> partition 1
    assert sc["cap"] == 2
    assert sc["num_splits"].tolist() == [1, 1]
    assert sc["first_part"].tolist() == [0, 1]


def test_split_decode_equals_unsplit():
    """The oracle computed the split-KV way (schedule + partials + merge) equals the
    plain definition."""
    from deepseek_mla_decode_b200.workloads import make_inputs

    inp = make_inputs(3, 2, 4, [700, 65, 1290], seed=3, causal=True)
    qn, qp, kv = O.bf16_to_f64(inp.q_nope), O.bf16_to_f64(inp.q_pe), O.bf16_to_f64(inp.kv_cache)
    sc = O.schedule_ref(inp.cache_seqlens, inp.s_q, inp.H, 5)
    assert sc["total_slots"] > 3  # really split
    a = O.mla_decode_split_ref(qn, qp, kv, inp.block_table, inp.cache_seqlens, inp.softmax_scale, True, sc)
    b = O.mla_decode_ref(qn, qp, kv, inp.block_table, inp.cache_seqlens, inp.softmax_scale, True)
    assert np.max(np.abs(a[0] - b[0])) < 1e-12 and np.max(np.abs(a[1] - b[1])) < 1e-12
