"""The benchmark's algorithmic work counts (the numerators of its roofline figures),
checked against closed forms and against each other.  CPU only."""

import os
import sys

import numpy as np

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

PER_KEY_FLOPS = 2 * (576 + 512)  # per head, query token and visible key
ROW_BYTES = 1152                 # one bf16 cache row of 576 values


def test_uniform_counts_closed_form():
    f, cache, algo = bench.algorithmic_work(np.array([4096, 4096]), 1, 128, False)
    assert f == 2 * 4096 * 128 * PER_KEY_FLOPS
    assert cache == 2 * 4096 * ROW_BYTES
    # + q (576 bf16) + out (512 bf16) + lse (fp32) per query row
    assert algo == cache + 2 * 128 * (576 * 2 + 512 * 2 + 4)
    # causal s_q = 2 over 10 keys: the tokens see 9 and 10 keys
    f2, _, _ = bench.algorithmic_work(np.array([10]), 2, 1, True)
    assert f2 == (9 + 10) * PER_KEY_FLOPS
    # the packed FP8 row only changes the cache bytes
    f3, c3, _ = bench.algorithmic_work(np.array([100]), 1, 16, False, row_bytes=656)
    assert f3 == 100 * 16 * PER_KEY_FLOPS and c3 == 100 * 656


def test_ragged_counts_reduce_to_the_uniform_ones():
    rng = np.random.default_rng(7)
    lens = rng.integers(1, 3000, size=17)
    for s_q in (1, 2, 4):
        for causal in (False, True):
            full = bench.algorithmic_work(lens, s_q, 128, causal)
            rag = bench.ragged_work(lens, np.full(17, s_q), 128, causal)
            assert rag == full
    # one token per sequence is the s_q = 1 call, causal or not
    assert bench.ragged_work(lens, np.ones(17, dtype=int), 64, True) == bench.algorithmic_work(lens, 1, 64, False)


def test_ragged_counts_hand_worked():
    # n = 10 with 2 tokens (sees 9 and 10 keys), n = 7 with 1 token (7 keys), n = 5 with
    # none (no cache rows read, no q / out)
    f, cache, algo = bench.ragged_work(np.array([10, 7, 5]), np.array([2, 1, 0]), 2, True)
    assert f == (9 + 10 + 7) * 2 * PER_KEY_FLOPS
    assert cache == (10 + 7) * ROW_BYTES
    assert algo == cache + 3 * 2 * (576 * 2 + 512 * 2 + 4)


def test_prefill_work_closed_form():
    # causal: S (S + 1) / 2 visible pairs per head, 2 (192 + 128) operations each
    assert bench.prefill_work(4, 3) == 2 * 320 * 3 * 10
