"""The seeded input recipe: shapes and length distributions of the five workloads,
bf16 rounding, determinism, and the placement of the poison that makes any read
outside a sequence's visible keys detectable."""

import numpy as np
import pytest

from deepseek_mla_decode_b200 import workloads as W


def test_workload_shapes_and_lengths():
    w = W.WORKLOADS
    assert (w["tiny"].B, w["tiny"].s_q, w["tiny"].H) == (2, 1, 16)
    assert w["tiny"].seqlens().tolist() == [37, 130]
    assert (w["decode_b64"].B, w["decode_b64"].H) == (64, 128)
    assert set(w["decode_b64"].seqlens().tolist()) == {4096}
    m = w["mtp_b128_sq2"]
    assert (m.B, m.s_q, m.H, m.causal) == (128, 2, 128, True)
    n = m.seqlens()
    assert n.min() >= 1024 and n.max() <= 8192
    s = w["serving_b256"]
    assert (s.B, s.s_q, s.H) == (256, 1, 128)
    n = s.seqlens()
    assert n.min() >= 1812 and n.max() <= 1812 + 978
    assert abs(n.mean() - (1812 + 978 / 2)) < 80  # uniform offset: mean near the middle
    assert w["long_b4"].seqlens().tolist() == [65536, 65536, 32768, 8192]


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 65504.0], dtype=np.float32)
    bits = W.f32_to_bf16_bits(x)
    back = (bits.astype(np.uint32) << 16).view(np.float32)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: rounds to the even mantissa (1.0);
    # 1 + 3*2^-8 is a tie between 1 + 2^-7 and 1 + 2^-6: rounds to 1 + 2^-6
    assert back.tolist() == [1.0, 1.0, 1.0 + 2 ** -6, -2.5, 65536.0]


def test_inputs_are_deterministic_per_seed():
    a = W.make_inputs(3, 2, 16, [70, 5, 200], seed=11, causal=True)
    b = W.make_inputs(3, 2, 16, [70, 5, 200], seed=11, causal=True)
    c = W.make_inputs(3, 2, 16, [70, 5, 200], seed=12, causal=True)
    for f in ("q_nope", "q_pe", "kv_cache", "block_table"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f
    assert not np.array_equal(a.q_nope, c.q_nope)


@pytest.mark.parametrize("nan", [False, True])
def test_poison_placement(nan):
    seqlens = [70, 5, 200, 128]
    inp = W.make_inputs(4, 1, 16, seqlens, seed=3, nan_poison=nan)
    nblk = [(n + 63) // 64 for n in seqlens]
    kv = (inp.kv_cache.astype(np.uint32) << 16).view(np.float32)
    # the poison as stored: POISON rounded to bf16 (1e4 -> 9984)
    pv = float((W.f32_to_bf16_bits(np.array([W.POISON], np.float32)).astype(np.uint32) << 16).view(np.float32)[0])
    used = set()
    for b, n in enumerate(seqlens):
        ids = inp.block_table[b, : nblk[b]].tolist()
        assert len(set(ids)) == nblk[b] and inp.spare_block not in ids
        used |= set(ids)
        # entries past the last block point at the spare block
        assert set(inp.block_table[b, nblk[b]:].tolist()) == {inp.spare_block}
        # visible rows are finite N(0, 1) draws, rows past n in the last block poisoned
        rows = np.concatenate([kv[i] for i in ids])
        assert np.isfinite(rows[:n]).all() and np.abs(rows[:n]).max() < 10
        tail = rows[n:]
        if len(tail):
            assert (np.isnan(tail).all() if nan else (np.abs(tail) == pv).all())
    assert len(used) == sum(nblk)  # every physical block handed out once
    spare = kv[inp.spare_block]
    assert (np.isnan(spare).all() if nan else (np.abs(spare) == pv).all())
    assert inp.kv_cache.shape[0] == sum(nblk) + 1
