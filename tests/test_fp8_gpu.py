"""GPU parity of the FP8 latent-cache path against the FP8 oracle.

mla_quantize_kv_fp8 must reproduce the oracle's packed rows byte for byte: the scale,
the e4m3 codes and the scaled bf16 k_pe are decided in fp32 on both sides (IEEE
division, round to nearest even)."""

import numpy as np
import pytest

from oracle import mla_fp8_oracle as F
from deepseek_mla_decode_b200.workloads import make_inputs, f32_to_bf16_bits

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import deepseek_mla_decode_b200 as mla  # noqa: E402


def bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("lens,seed", [([37, 130], 1), ([4096] * 3, 2), ([1, 64, 65, 2000], 3)])
def test_quantize_matches_oracle_bit_exact(lens, seed):
    inp = make_inputs(len(lens), 1, 16, lens, seed=seed)
    kv = inp.kv_cache.copy()
    kv[0, 0, :] = 0                                             # a zero row: scale 0, all zeros
    kv[0, 1, :] = f32_to_bf16_bits(np.full(576, -3.0, np.float32))  # constant row: codes -448, k_pe' -448
    kv[0, 2, 512:] = f32_to_bf16_bits(np.full(64, 40.0, np.float32))  # k_pe sets the row's scale
    kv[0, 3, :512] = 0                                          # only k_pe non-zero: codes 0
    got = mla.quantize_kv_fp8(bf16(kv)).cpu().numpy()
    ref = F.pack_cache(kv)
    assert got.shape == ref.shape
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} bytes differ, first at {bad[:5].tolist()}: got {got[tuple(bad[0])]} ref {ref[tuple(bad[0])]}"


# ---------------------------------------------------------------------------
# mla_decode_fp8 against the FP8 oracle (each side packs the cache with its own
# quantiser; the two are byte-identical by the test above).  Tolerances as for the
# bf16 path: out max-abs <= 2e-2, mean-abs <= 2e-3; lse max-abs <= 1e-3.
# ---------------------------------------------------------------------------
from deepseek_mla_decode_b200.workloads import make_workload  # noqa: E402
from mla_testlib import run_cuda_fp8, oracle_fp8, compare  # noqa: E402


def check_fp8(inp, seqs=None, q_lens=None, status_expect=0):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, _ = run_cuda_fp8(inp, status=status, q_lens=q_lens)
    assert int(status.item()) == status_expect, int(status.item())
    ref_out, ref_lse = oracle_fp8(inp, seqs, q_lens=q_lens)
    if seqs is not None:
        out, lse = out[seqs], lse[seqs]
    return compare(out, lse, ref_out, ref_lse, what=f"fp8 B={inp.B} s_q={inp.s_q} H={inp.H}")


def test_fp8_tiny_config():
    check_fp8(make_workload("tiny"))


@pytest.mark.parametrize("H", [16, 64, 128])
@pytest.mark.parametrize("s_q,causal", [(1, False), (2, True)])
def test_fp8_ragged_lengths(H, s_q, causal):
    lens = [1, 63, 64, 65, 255, 256, 257, 1000]
    check_fp8(make_inputs(len(lens), s_q, H, lens, seed=300 + H + 7 * s_q, causal=causal))


@pytest.mark.parametrize("s_q", [3, 4])
def test_fp8_more_draft_tokens(s_q):
    check_fp8(make_inputs(3, s_q, 64, [5, 300, 777], seed=340 + s_q, causal=True))


def test_fp8_ragged_query_counts():
    check_fp8(make_inputs(5, 4, 64, [300, 1000, 77, 500, 2000], seed=350, causal=True), q_lens=[4, 1, 2, 0, 3])


def test_fp8_single_long_sequence_split():
    check_fp8(make_inputs(1, 1, 128, [20000], seed=361))


def test_fp8_nan_poison_outside_visible_range():
    check_fp8(make_inputs(4, 1, 32, [37, 100, 129, 200], seed=362, nan_poison=True))


def test_fp8_zero_length_and_short_causal_rows():
    check_fp8(make_inputs(4, 2, 16, [0, 1, 2, 70], seed=363, causal=True))


def test_fp8_single_key_reproduces_every_code():
    # One visible key per sequence: its softmax weight is exactly 1, so the output row is
    # the dequantised value row itself.  The rows hold every finite e4m3 value (the
    # subnormals and both zeros included) and reach 448, so the scale is exactly 1 and
    # each output element must equal its code's value bit for bit.
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = F.e4m3_decode(finite)
    inp = make_inputs(4, 1, 16, [1, 1, 1, 1], seed=364)
    rng = np.random.default_rng(365)
    expect = np.empty((4, 512))
    for b in range(4):
        row = np.concatenate([rng.permutation(vals), rng.choice(vals, 512 - vals.size)])
        row[rng.integers(512)] = 448.0
        kpe = rng.choice(vals[np.abs(vals) <= 448], 64)
        blk = inp.block_table[b, 0]
        inp.kv_cache[blk, 0, :512] = f32_to_bf16_bits(row.astype(np.float32))
        inp.kv_cache[blk, 0, 512:] = f32_to_bf16_bits(kpe.astype(np.float32))
        expect[b] = row
    out, lse, _ = run_cuda_fp8(inp)
    got = out[:, 0]  # [B, H, 512]
    assert np.array_equal(got, np.broadcast_to(expect[:, None, :], got.shape)), \
        f"max diff {np.max(np.abs(got - expect[:, None, :]))}"
    ref_out, ref_lse = oracle_fp8(inp)
    assert np.array_equal(got, ref_out[:, 0])
    assert np.max(np.abs(lse - ref_lse)) <= 1e-3


def test_fp8_deterministic():
    inp = make_inputs(5, 2, 128, [3000, 17, 900, 4100, 640], seed=366, causal=True)
    from mla_testlib import to_device

    dev = to_device(inp)
    a = run_cuda_fp8(inp, dev)
    b = run_cuda_fp8(inp, dev)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1], equal_nan=True)


@pytest.mark.parametrize("name", ["serving_b256", "decode_b64", "mtp_b128_sq2", "long_b4"])
def test_fp8_full_size_whole_batch(name):
    inp = make_workload(name)
    stats = check_fp8(inp, seqs=list(range(inp.B)))
    print(f"fp8 {name}: {stats}")


def test_fp8_wait_timeout_sets_status_and_returns():
    """The failure path of the FP8 instantiation: the MMA warp waits on a barrier nothing
    completes (a test hook), bounded by 1 ms; converters and producers then stop at their
    next bounded wait, the pair drains and returns, and the next call is exact."""
    from mla_testlib import to_device

    inp = make_inputs(3, 1, 128, [3000, 700, 5000], seed=371)
    dev = to_device(inp)
    kv8 = mla.quantize_kv_fp8(dev["kv_cache"])
    meta = mla.get_metadata(dev["cache_seqlens"], 1, 128)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        mla.set_wait_timeout_ns(1_000_000)
        mla.set_stall_injection(True)
        mla.decode_fp8(dev["q_nope"], dev["q_pe"], kv8, dev["block_table"], dev["cache_seqlens"],
                       inp.softmax_scale, False, meta, status=status)
        torch.cuda.synchronize()
    finally:
        mla.set_stall_injection(False)
        mla.set_wait_timeout_ns(0)
    assert int(status.item()) & mla.MLA_DEVICE_ERR_TIMEOUT
    check_fp8(inp)
