"""GPU parity tests: the CUDA path (through the C ABI) against the float64 oracle on
identical seeded inputs.  Tolerances: out max-abs <= 2e-2, mean-abs <= 2e-3; lse
max-abs <= 1e-3; the integer schedule must match the oracle word for word."""

import math

import numpy as np
import pytest

from oracle import mla_oracle as O
from deepseek_mla_decode_b200.workloads import make_inputs, make_workload, WORKLOADS
from mla_testlib import to_device, run_cuda, oracle, compare

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import deepseek_mla_decode_b200 as mla  # noqa: E402


def check(inp, seqs=None, status_expect=0):
    import torch

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, meta = run_cuda(inp, status=status)
    assert int(status.item()) == status_expect, int(status.item())
    ref_out, ref_lse = oracle(inp, seqs)
    if seqs is not None:
        out, lse = out[seqs], lse[seqs]
    return compare(out, lse, ref_out, ref_lse, what=f"B={inp.B} s_q={inp.s_q} H={inp.H}")


# ---------------------------------------------------------------------------
# small cases: several 256-key tiles, ragged tails, all head counts
# ---------------------------------------------------------------------------
def test_tiny_config():
    check(make_workload("tiny"))


@pytest.mark.parametrize("H", [16, 32, 64, 128])
@pytest.mark.parametrize("s_q,causal", [(1, False), (2, True), (2, False)])
def test_ragged_lengths(H, s_q, causal):
    lens = [1, 63, 64, 65, 255, 256, 257, 1000]
    check(make_inputs(len(lens), s_q, H, lens, seed=100 + H + 7 * s_q, causal=causal))


@pytest.mark.parametrize("s_q", [3, 4])
def test_more_draft_tokens(s_q):
    check(make_inputs(3, s_q, 64, [5, 300, 777], seed=40 + s_q, causal=True))
    check(make_inputs(2, s_q, 128, [129, 1030], seed=50 + s_q, causal=True))


@pytest.mark.parametrize("H,s_q,q_lens,lens", [
    (64, 4, [4, 1, 2, 0, 3], [300, 1000, 77, 500, 2000]),   # two row tiles: tokens {0,1} and {2,3}
    (128, 2, [1, 2, 0, 1, 2], [5000, 129, 64, 9000, 1]),    # one row tile per token; long splits
    (16, 3, [3, 2, 1], [1, 2, 700]),                        # fewer keys than query tokens
])
def test_ragged_query_counts(H, s_q, q_lens, lens):
    inp = make_inputs(len(lens), s_q, H, lens, seed=80 + H + s_q, causal=True)
    dev = to_device(inp)
    ql = torch.tensor(q_lens, dtype=torch.int32, device="cuda")
    meta = mla.get_metadata(dev["cache_seqlens"], s_q, H)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = mla.decode_ragged(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"],
                                 dev["cache_seqlens"], ql, inp.softmax_scale, True, meta, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_out, ref_lse = oracle(inp, q_lens=np.array(q_lens))
    compare(out.float().cpu().double().numpy(), lse.cpu().double().numpy(), ref_out, ref_lse,
            what=f"ragged H={H} s_q={s_q}")


def test_ragged_invalid_query_count():
    inp = make_inputs(3, 2, 64, [100, 300, 50], seed=90, causal=True)
    dev = to_device(inp)
    ql = torch.tensor([2, 3, 1], dtype=torch.int32, device="cuda")  # 3 > s_q
    meta = mla.get_metadata(dev["cache_seqlens"], 2, 64)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = mla.decode_ragged(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"],
                                 dev["cache_seqlens"], ql, inp.softmax_scale, True, meta, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == mla.MLA_DEVICE_ERR_SEQLEN
    out, lse = out.float().cpu().double().numpy(), lse.cpu().double().numpy()
    assert np.all(np.isnan(out[1])) and np.all(np.isnan(lse[1]))
    ref_out, ref_lse = oracle(inp, [0, 2], q_lens=np.array([2, 2, 1]))
    compare(out[[0, 2]], lse[[0, 2]], ref_out, ref_lse)


def test_single_long_sequence_split():
    # one sequence long enough to be cut into many pieces + LSE combine
    check(make_inputs(1, 1, 128, [20000], seed=61))


@pytest.mark.parametrize("extra", [-1, 0, 1])
def test_combine_grid_forms_at_the_partition_count(extra):
    """The combine's grid runs over sequences while B <= P (partitions per row tile) and
    over partitions beyond: batches of P - 1, P and P + 1 sequences, lengths mixed so
    that some sequences are cut into two or more pieces and some are whole."""
    P = min(mla.device_sm_count() // 2, 256)  # CTA pairs = partitions of the single row tile
    B = P + extra
    rng = np.random.default_rng(300 + extra)
    lens = rng.integers(1, 6000, size=B).astype(np.int32)
    lens[::7] = rng.integers(9000, 20000, size=len(lens[::7]))
    check(make_inputs(B, 1, 128, lens, seed=301 + extra))


def test_nan_poison_outside_visible_range():
    inp = make_inputs(4, 1, 32, [37, 100, 129, 200], seed=62, nan_poison=True)
    check(inp)


def test_zero_length_and_short_causal_rows():
    # n = 0: out 0 / lse -inf; causal with n < s_q: first token sees nothing
    check(make_inputs(4, 2, 16, [0, 1, 2, 70], seed=63, causal=True))


def test_weights_sum_to_one_on_gpu():
    inp = make_inputs(3, 1, 64, [90, 700, 1500], seed=64)
    from deepseek_mla_decode_b200.workloads import f32_to_bf16_bits

    inp.kv_cache[:, :, :512] = f32_to_bf16_bits(np.ones(1, np.float32))[0]
    out, lse, _ = run_cuda(inp)
    assert np.max(np.abs(out - 1.0)) == 0.0  # bf16 sum of bf16 weights normalises exactly


def test_deterministic():
    inp = make_inputs(5, 2, 128, [3000, 17, 900, 4100, 640], seed=65, causal=True)
    dev = to_device(inp)
    a = run_cuda(inp, dev)
    b = run_cuda(inp, dev)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1], equal_nan=True)


# ---------------------------------------------------------------------------
# schedule: bit-exact against the oracle
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("B", [1023, 1024, 1025, 3000])
def test_metadata_matches_oracle_large_batch(B):
    """Batches around and beyond one pass of the scheduler block (1024 sequences):
    the single-pass and multi-pass paths give the oracle's schedule word for word."""
    rng = np.random.default_rng(B)
    seqlens = rng.integers(0, 3000, size=B).astype(np.int64)
    seqlens[rng.random(B) < 0.05] = 0
    t = torch.from_numpy(seqlens.astype(np.int32)).cuda()
    meta = mla.get_metadata(t, 1, 128).cpu().numpy()
    workers = min(mla.device_sm_count() // 2, 256)
    sc = O.schedule_ref(seqlens, 1, 128, workers)
    P = sc["num_parts"]
    assert list(meta[1:9]) == [B, 1, 128, P, sc["num_tiles"], sc["cap"], sc["total_slots"], workers]
    assert np.array_equal(meta[16 : 16 + 512].reshape(256, 2)[:P], sc["part_start"])
    assert np.array_equal(meta[16 + 512 : 16 + 1024].reshape(256, 2)[:P], sc["part_end"])
    base = 16 + 1024
    for i, key in enumerate(["nblk", "first_part", "num_splits", "split_prefix"]):
        assert np.array_equal(meta[base + i * B : base + (i + 1) * B], sc[key]), key


@pytest.mark.parametrize("name", ["tiny", "decode_b64", "mtp_b128_sq2", "serving_b256", "long_b4"])
def test_metadata_matches_oracle(name):
    w = WORKLOADS[name]
    seqlens = w.seqlens()
    t = torch.from_numpy(seqlens.astype(np.int32)).cuda()
    meta = mla.get_metadata(t, w.s_q, w.H).cpu().numpy()
    workers = min(mla.device_sm_count() // 2, 256)
    sc = O.schedule_ref(seqlens, w.s_q, w.H, workers)
    B = w.B
    P = sc["num_parts"]
    assert meta[0] == 0x4D4C4131
    assert list(meta[1:10]) == [B, w.s_q, w.H, P, sc["num_tiles"], sc["cap"], sc["total_slots"], workers,
                             O.SCHED_OVERHEAD_TILES]
    ps = meta[16 : 16 + 512].reshape(256, 2)[:P]
    pe = meta[16 + 512 : 16 + 1024].reshape(256, 2)[:P]
    assert np.array_equal(ps, sc["part_start"]) and np.array_equal(pe, sc["part_end"])
    base = 16 + 1024
    assert np.array_equal(meta[base : base + B], sc["nblk"])
    assert np.array_equal(meta[base + B : base + 2 * B], sc["first_part"])
    assert np.array_equal(meta[base + 2 * B : base + 3 * B], sc["num_splits"])
    assert np.array_equal(meta[base + 3 * B : base + 4 * B], sc["split_prefix"])


# ---------------------------------------------------------------------------
# device-detected errors: never fault, NaN rows + status bits
# ---------------------------------------------------------------------------
def test_bad_block_id_gives_nan_rows_and_status():
    inp = make_inputs(3, 1, 64, [100, 300, 50], seed=66)
    inp.block_table[1, 2] = inp.kv_cache.shape[0] + 5  # out of range, inside seq 1's range
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, _ = run_cuda(inp, status=status)
    assert int(status.item()) & mla.MLA_DEVICE_ERR_BLOCK_ID
    assert np.all(np.isnan(out[1])) and np.all(np.isnan(lse[1]))
    ref_out, ref_lse = oracle(inp, [0, 2])
    compare(out[[0, 2]], lse[[0, 2]], ref_out, ref_lse)


def test_bad_seqlen_gives_nan_rows_and_status():
    inp = make_inputs(3, 1, 64, [100, 300, 50], seed=67)
    dev = to_device(inp)
    dev["cache_seqlens"][1] = 64 * inp.block_table.shape[1] + 1  # beyond the table
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, _ = run_cuda(inp, dev=dev, status=status)
    assert int(status.item()) & mla.MLA_DEVICE_ERR_SEQLEN
    assert np.all(np.isnan(out[1])) and np.all(np.isnan(lse[1]))
    ref_out, ref_lse = oracle(inp, [0, 2])
    compare(out[[0, 2]], lse[[0, 2]], ref_out, ref_lse)


def test_metadata_for_other_shape_rejected_on_device():
    inp = make_inputs(2, 1, 64, [100, 300], seed=68)
    dev = to_device(inp)
    meta = mla.get_metadata(dev["cache_seqlens"], 1, 32)  # wrong H
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.decode(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"], dev["cache_seqlens"],
               inp.softmax_scale, False, meta, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & mla.MLA_DEVICE_ERR_METADATA


def test_metadata_for_other_lengths():
    """A schedule built for other lengths of the same shape (a serving loop that reuses
    last step's metadata): sequences whose block count changed get NaN rows and the
    metadata bit, and no block-table entry past their blocks is read; sequences whose
    block count is unchanged are still exact."""
    old_lens = [100, 300, 50, 700, 5000]
    new_lens = [100, 400, 50, 650, 200]  # seq 1: 5 -> 7 blocks, seq 3: 11 -> 11, seq 4: 79 -> 4
    inp = make_inputs(5, 1, 128, new_lens, seed=70, extra_table_cols=0)
    dev = to_device(inp)
    stale = mla.get_metadata(torch.tensor(old_lens, dtype=torch.int32, device="cuda"), 1, 128)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = mla.decode(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"], dev["cache_seqlens"],
                          inp.softmax_scale, False, stale, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == mla.MLA_DEVICE_ERR_METADATA, int(status.item())
    out = out.float().cpu().double().numpy()
    lse = lse.cpu().double().numpy()
    for b in (1, 4):
        assert np.all(np.isnan(out[b])) and np.all(np.isnan(lse[b]))
    good = [0, 2, 3]
    ref_out, ref_lse = oracle(inp, good)
    compare(out[good], lse[good], ref_out, ref_lse)


def test_wait_timeout_sets_status_and_returns():
    """The MMA warp waits on a barrier nothing completes (a test hook), bounded by
    1 ms: the kernel must set the timeout bit, stop every role, drain what the pair
    had in flight and return, leaving the context usable -- the next call, with the
    default bound, is exact."""
    inp = make_inputs(3, 1, 128, [3000, 700, 5000], seed=71)
    dev = to_device(inp)
    meta = mla.get_metadata(dev["cache_seqlens"], 1, 128)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        mla.set_wait_timeout_ns(1_000_000)
        mla.set_stall_injection(True)
        mla.decode(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"], dev["cache_seqlens"],
                   inp.softmax_scale, False, meta, status=status)
        torch.cuda.synchronize()
    finally:
        mla.set_stall_injection(False)
        mla.set_wait_timeout_ns(0)
    assert int(status.item()) & mla.MLA_DEVICE_ERR_TIMEOUT
    check(inp)


def test_host_argument_errors():
    inp = make_inputs(2, 1, 64, [100, 300], seed=69)
    dev = to_device(inp)
    meta = mla.get_metadata(dev["cache_seqlens"], 1, 64)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(mla.MLAError) as e:
        mla.decode(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"], dev["cache_seqlens"],
                   inp.softmax_scale, False, meta, workspace=ws)
    assert e.value.code == 4
    with pytest.raises(mla.MLAError) as e:
        mla.decode(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"], dev["cache_seqlens"],
                   -1.0, False, meta)
    assert e.value.code == 1


# ---------------------------------------------------------------------------
# full-size workloads, in the launch configuration bench.py times: every sequence of
# the batch against the oracle (converted to float64 one sequence at a time)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["decode_b64", "mtp_b128_sq2", "serving_b256", "long_b4"])
def test_full_size_whole_batch(name):
    inp = make_workload(name)
    stats = check(inp, seqs=list(range(inp.B)))
    print(f"{name}: {stats}")
