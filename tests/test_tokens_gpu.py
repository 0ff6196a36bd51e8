"""GPU tests of the token schedule (mla_get_metadata_tokens with mla_decode_tokens /
mla_decode_fp8_tokens): the ragged decode run as an s_q = 1 decode over one sequence
per query token.  Parity with the float64 oracles on ragged query counts, the schedule
word for word against the oracle's schedule over the tokens' key counts, error paths,
determinism.  Tolerances as in test_decode_gpu.py."""

import numpy as np
import pytest

from oracle import mla_oracle as O
from deepseek_mla_decode_b200.workloads import make_inputs, make_workload
from mla_testlib import to_device, oracle, oracle_fp8, compare

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import deepseek_mla_decode_b200 as mla  # noqa: E402


def token_key_counts(seqlens, q_lens, s_q, causal):
    """Keys each query token sees (the ragged decode's definition: the tokens are the
    last q cache positions, token t sees keys 0 .. n - q + t with the causal mask, all n
    without it, none when t >= q); -1 for an invalid count or length."""
    out = []
    for n, q in zip(np.asarray(seqlens).tolist(), np.asarray(q_lens).tolist()):
        for t in range(s_q):
            if q < 0 or q > s_q or n < 0:
                out.append(-1)
            elif t >= q:
                out.append(0)
            elif not causal:
                out.append(n)
            else:
                out.append(max(0, n - q + t + 1))
    return np.array(out, dtype=np.int64)


def run_tokens(inp, q_lens, fp8=False, status=None, causal=None):
    dev = to_device(inp)
    causal = inp.causal if causal is None else causal
    ql = None if q_lens is None else torch.tensor(np.asarray(q_lens, dtype=np.int32), device="cuda")
    meta = mla.get_metadata_tokens(dev["cache_seqlens"], ql, inp.s_q, inp.H, causal)
    if fp8:
        kv8 = mla.quantize_kv_fp8(dev["kv_cache"])
        out, lse = mla.decode_fp8_tokens(dev["q_nope"], dev["q_pe"], kv8, dev["block_table"], dev["cache_seqlens"],
                                         ql, inp.softmax_scale, causal, meta, status=status)
    else:
        out, lse = mla.decode_tokens(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"],
                                     dev["cache_seqlens"], ql, inp.softmax_scale, causal, meta, status=status)
    torch.cuda.synchronize()
    return out.float().cpu().double().numpy(), lse.cpu().double().numpy(), meta


@pytest.mark.parametrize("H,s_q,q_lens,lens,causal", [
    (64, 4, [4, 1, 2, 0, 3], [300, 1000, 77, 500, 2000], True),
    (128, 2, [1, 2, 0, 1, 2], [5000, 129, 64, 9000, 1], True),   # long sequences cut into pieces
    (16, 3, [3, 2, 1], [1, 2, 700], True),                       # fewer keys than query tokens
    (128, 4, [2, 4, 1], [3000, 257, 40000], False),              # every token sees every key
])
def test_tokens_match_oracle(H, s_q, q_lens, lens, causal):
    inp = make_inputs(len(lens), s_q, H, lens, seed=120 + H + s_q, causal=causal)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, _ = run_tokens(inp, q_lens, status=status)
    assert int(status.item()) == 0
    ref_out, ref_lse = oracle(inp, q_lens=np.array(q_lens))
    compare(out, lse, ref_out, ref_lse, what=f"tokens H={H} s_q={s_q}")


def test_tokens_uniform_mtp_whole_batch():
    """Every sequence of the MTP workload (s_q = 2, causal) through the token schedule."""
    inp = make_workload("mtp_b128_sq2")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, _ = run_tokens(inp, None, status=status)
    assert int(status.item()) == 0
    ref_out, ref_lse = oracle(inp)
    compare(out, lse, ref_out, ref_lse, what="mtp_b128_sq2 via tokens")


def ragged_bench_config():
    """The benchmark's ragged MTP verification: B = 128, s_q <= 4, q_lens U{1..4},
    causal, lengths U[1024, 8192] (seed 1005)."""
    rng = np.random.default_rng(1005 + 7919)
    lens = rng.integers(1024, 8192 + 1, size=128, dtype=np.int64).astype(np.int32)
    q_lens = rng.integers(1, 5, size=128, dtype=np.int64).astype(np.int32)
    return make_inputs(128, 4, 128, lens, 1005, causal=True), q_lens


def test_tokens_ragged_full_size_whole_batch():
    inp, q_lens = ragged_bench_config()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, _ = run_tokens(inp, q_lens, status=status)
    assert int(status.item()) == 0
    ref_out, ref_lse = oracle(inp, q_lens=q_lens)
    compare(out, lse, ref_out, ref_lse, what="ragged B=128 s_q<=4 via tokens")


@pytest.mark.parametrize("causal", [True, False])
def test_tokens_schedule_matches_oracle(causal):
    rng = np.random.default_rng(17 + causal)
    B, s_q, H = 200, 4, 128
    lens = rng.integers(0, 6000, size=B).astype(np.int64)
    q_lens = rng.integers(0, s_q + 1, size=B).astype(np.int64)
    q_lens[3] = 7   # invalid count: the sequence's tokens get no keys in the schedule
    lens[5] = -2    # invalid length: likewise
    meta = mla.get_metadata_tokens(torch.from_numpy(lens.astype(np.int32)).cuda(),
                                   torch.from_numpy(q_lens.astype(np.int32)).cuda(), s_q, H, causal).cpu().numpy()
    workers = min(mla.device_sm_count() // 2, 256)
    keys = token_key_counts(lens, q_lens, s_q, causal)
    sc = O.schedule_ref(keys, 1, H, workers)
    Bt = B * s_q
    P = sc["num_parts"]
    assert meta[0] == 0x4D4C4131
    assert list(meta[1:12]) == [Bt, 1, H, P, sc["num_tiles"], sc["cap"], sc["total_slots"], workers,
                                O.SCHED_OVERHEAD_TILES, s_q, int(causal)]
    assert np.array_equal(meta[16 : 16 + 512].reshape(256, 2)[:P], sc["part_start"])
    assert np.array_equal(meta[16 + 512 : 16 + 1024].reshape(256, 2)[:P], sc["part_end"])
    base = 16 + 1024
    for i, key in enumerate(["nblk", "first_part", "num_splits", "split_prefix"]):
        assert np.array_equal(meta[base + i * Bt : base + (i + 1) * Bt], sc[key]), key


def test_tokens_invalid_query_count_and_length():
    inp = make_inputs(4, 2, 64, [100, 300, 50, 400], seed=91, causal=True)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, _ = run_tokens(inp, [2, 3, 1, 2], status=status)  # 3 > s_q
    assert int(status.item()) == mla.MLA_DEVICE_ERR_SEQLEN
    assert np.all(np.isnan(out[1])) and np.all(np.isnan(lse[1]))
    ref_out, ref_lse = oracle(inp, [0, 2, 3], q_lens=np.array([2, 2, 1, 2]))
    compare(out[[0, 2, 3]], lse[[0, 2, 3]], ref_out, ref_lse)


def test_tokens_schedule_of_another_kind_is_rejected_on_device():
    """Token metadata built for the causal call, used without the mask: the kernel
    refuses it (MLA_DEVICE_ERR_METADATA) instead of computing other lengths."""
    inp = make_inputs(3, 2, 128, [500, 900, 70], seed=92, causal=True)
    dev = to_device(inp)
    ql = torch.tensor([2, 1, 2], dtype=torch.int32, device="cuda")
    meta = mla.get_metadata_tokens(dev["cache_seqlens"], ql, 2, 128, True)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.decode_tokens(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"], dev["cache_seqlens"], ql,
                      inp.softmax_scale, False, meta, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & mla.MLA_DEVICE_ERR_METADATA


def test_tokens_deterministic():
    inp = make_inputs(6, 4, 128, [3000, 10, 777, 5000, 1, 2048], seed=93, causal=True)
    q_lens = [4, 1, 3, 2, 1, 4]
    a_out, a_lse, _ = run_tokens(inp, q_lens)
    b_out, b_lse, _ = run_tokens(inp, q_lens)
    assert np.array_equal(a_out, b_out, equal_nan=True) and np.array_equal(a_lse, b_lse, equal_nan=True)


def test_fp8_tokens_match_oracle():
    inp = make_inputs(5, 3, 128, [2000, 64, 6000, 300, 1], seed=94, causal=True)
    q_lens = [3, 1, 2, 0, 1]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, _ = run_tokens(inp, q_lens, fp8=True, status=status)
    assert int(status.item()) == 0
    ref_out, ref_lse = oracle_fp8(inp, q_lens=np.array(q_lens))
    compare(out, lse, ref_out, ref_lse, what="fp8 tokens")
