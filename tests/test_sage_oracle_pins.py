"""Pins of the quantised-prefill oracle (oracle/sage_oracle.py) against facts that do
not come from the oracle itself: hand-checked quantiser codes, closed forms in exact
cases, invariants of causal attention and of the per-channel V scale, and a derived
error bound against exact softmax attention on the unquantised inputs."""

import numpy as np
import pytest

from oracle import sage_oracle as SA
from oracle import mla_fp8_oracle as F
from deepseek_mla_decode_b200.workloads import f32_to_bf16_bits


def bits(x):
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def rand_bf16(rng, shape, scale=1.0):
    return bits(rng.standard_normal(shape) * scale)


# ---------------------------------------------------------------------------
# quantisers
# ---------------------------------------------------------------------------
def test_int8_hand_codes():
    x = np.zeros((2, 192), np.float32)
    x[0, :5] = [127.0, -63.5, 0.5, 1.5, -2.5]  # scale 1: rint with ties to even
    codes, scale = SA.quantize_int8_rows(x)
    assert scale[0] == 1.0 and scale[1] == 0.0
    assert codes[0, :5].tolist() == [127, -64, 0, 2, -2]
    assert np.all(codes[1] == 0)


def test_int8_bounds_random():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((64, 192)) * rng.uniform(0.01, 100, (64, 1))).astype(np.float32)
    codes, s = SA.quantize_int8_rows(x)
    assert codes.dtype == np.int8 and np.all(np.abs(codes.astype(int)) <= 127)
    # the row maximum maps to +-127, and every value is within half a step (plus the
    # fp32 quotient's rounding) of its dequantised code
    assert np.all(np.max(np.abs(codes.astype(int)), axis=1) == 127)
    err = np.abs(x.astype(np.float64) - codes * s[:, None].astype(np.float64))
    assert np.all(err <= s[:, None] * (0.5 + 2.0 ** -16))


def test_v_channel_quantiser():
    rng = np.random.default_rng(2)
    v = (rng.standard_normal((300, 2, 128)) * 3).astype(np.float32)
    v[:, 1, 5] = 0.0  # a zero channel
    codes, s = SA.quantize_v_channels(v)
    assert s.shape == (2, 128) and s[1, 5] == 0 and np.all(codes[:, 1, 5] == 0)
    amax = np.abs(v).max(axis=0)
    assert np.array_equal(s, (amax / np.float32(448.0)).astype(np.float32))
    # the channel maximum maps to +-448 (code 0x7E / 0xFE)
    top = np.argmax(np.abs(v), axis=0)
    c_top = np.take_along_axis(codes, top[None], axis=0)[0]
    assert np.all((c_top[s > 0] & 0x7F) == 0x7E)
    # half-spacing bound of e4m3 (relative 2^-4 for normal values, 2^-10 absolute below)
    vh = F.e4m3_decode(codes) * s[None].astype(np.float64)
    q = v / np.where(s > 0, s, 1)[None]
    bound = np.maximum(np.abs(q) * 2.0 ** -4, 2.0 ** -10) * s[None] * (1 + 2.0 ** -20)
    assert np.all(np.abs(vh - v) <= bound + 1e-30)


# ---------------------------------------------------------------------------
# exact cases
# ---------------------------------------------------------------------------
def grid_values(rng, shape):
    """e4m3-exact values whose channels reach +-448, so V's scale is exactly 1."""
    finite = F.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    vals = rng.choice(finite, shape) * rng.choice([-1.0, 1.0], shape)
    vals[0] = 448.0
    return vals


@pytest.mark.parametrize("S", [1, 5, 130, 300])
def test_equal_logits_give_mean_of_visible_values(S):
    # every key row is the same, so a query's logits are all equal: p = 1 for every
    # visible key (code 448, weight exactly 1) and the output is the plain mean of the
    # visible value rows; lse = logit + log(i + 1)
    rng = np.random.default_rng(3 + S)
    H = 2
    q = rand_bf16(rng, (S, H, 192))
    krow = rand_bf16(rng, (1, H, 192))
    k = np.repeat(krow, S, axis=0)
    v = grid_values(rng, (S, H, 128))
    out, lse = SA.sage_prefill_ref(q, k, bits(v))
    mean = np.cumsum(v, axis=0) / np.arange(1, S + 1)[:, None, None]
    assert np.allclose(out, mean, rtol=1e-12, atol=1e-12)
    assert np.all(np.isfinite(lse))
    # lse - log(i + 1) is the (common) logit of row i: the same for every key
    logit = lse - np.log(np.arange(1, S + 1))[:, None]
    qc, sq = SA.quantize_int8_rows(F.O.bf16_to_f64(q).astype(np.float32))
    kc, sk = SA.quantize_int8_rows(F.O.bf16_to_f64(krow).astype(np.float32))
    direct = (qc.astype(np.int64) * kc.astype(np.int64)).sum(-1) * sq.astype(np.float64) * sk.astype(np.float64) \
        * SA.SCALE_192
    assert np.allclose(logit, direct, rtol=1e-12, atol=1e-12)


def test_first_row_sees_only_itself():
    rng = np.random.default_rng(4)
    S, H = 40, 3
    q, k = rand_bf16(rng, (S, H, 192)), rand_bf16(rng, (S, H, 192))
    v = grid_values(rng, (S, H, 128))
    out, _ = SA.sage_prefill_ref(q, k, bits(v))
    assert np.array_equal(out[0], v[0])


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------
def test_causal_outputs_ignore_later_keys():
    rng = np.random.default_rng(5)
    S, H, cut = 260, 2, 150
    q, k = rand_bf16(rng, (S, H, 192)), rand_bf16(rng, (S, H, 192))
    v = rng.standard_normal((S, H, 128)).astype(np.float32)
    v[0] = 10.0  # channel maxima at token 0: later V changes below it keep the scales
    out1, lse1 = SA.sage_prefill_ref(q, k, bits(v))
    k2 = k.copy()
    k2[cut:] = rand_bf16(rng, (S - cut, H, 192), 5.0)
    v2 = v.copy()
    v2[cut:] = rng.uniform(-1, 1, (S - cut, H, 128))
    out2, lse2 = SA.sage_prefill_ref(q, k2, bits(v2))
    assert np.array_equal(out1[:cut], out2[:cut]) and np.array_equal(lse1[:cut], lse2[:cut])
    assert not np.array_equal(out1[cut:], out2[cut:])


def test_v_scaling_and_channel_permutation():
    rng = np.random.default_rng(6)
    S, H = 200, 2
    q, k = rand_bf16(rng, (S, H, 192)), rand_bf16(rng, (S, H, 192))
    v = rng.standard_normal((S, H, 128)).astype(np.float32)
    out, lse = SA.sage_prefill_ref(q, k, bits(v))
    vb = F.O.bf16_to_f64(bits(v))
    out2, lse2 = SA.sage_prefill_ref(q, k, bits(vb * 4.0))  # exact in bf16: scales x4, codes equal
    assert np.array_equal(out2, out * 4.0) and np.array_equal(lse2, lse)
    perm = rng.permutation(128)
    out3, _ = SA.sage_prefill_ref(q, k, bits(vb[:, :, perm]))
    assert np.array_equal(out3, out[:, :, perm])


# ---------------------------------------------------------------------------
# derived bound against exact attention
# ---------------------------------------------------------------------------
def test_close_to_exact_attention():
    """|O_quant - O_exact| <= (e^d - e^-d) max|v| + max|v^ - v| + tiny-weight term,
    with d = 2 eps + 2 log(1 + 2^-4): eps bounds the logit error of the INT8 Q/K
    (half a step per element), 2^-4 the relative e4m3 rounding of P; weights below the
    e4m3 normal range (p * 448 < 2^-6) carry an absolute error of at most 2^-10 / 448."""
    rng = np.random.default_rng(7)
    S, H = 384, 2
    qb, kb, vb = rand_bf16(rng, (S, H, 192)), rand_bf16(rng, (S, H, 192)), rand_bf16(rng, (S, H, 128))
    out, lse = SA.sage_prefill_ref(qb, kb, vb)
    ex, ex_lse = SA.exact_prefill_ref(qb, kb, vb)
    q, k, v = (F.O.bf16_to_f64(b) for b in (qb, kb, vb))
    _, sq = SA.quantize_int8_rows(q.astype(np.float32))
    _, sk = SA.quantize_int8_rows(k.astype(np.float32))
    vc, sv = SA.quantize_v_channels(v.astype(np.float32))
    vh = F.e4m3_decode(vc) * sv[None].astype(np.float64)
    for h in range(H):
        # eps_ij <= scale * (s_q/2 * sum|k_j| + s_k/2 * sum|q_i| + 192 s_q s_k / 4)
        aq, ak = np.abs(q[:, h]).sum(-1), np.abs(k[:, h]).sum(-1)
        eps = SA.SCALE_192 * (sq[:, h, None] / 2 * ak[None] + sk[None, :, h] / 2 * aq[:, None]
                              + 192 * sq[:, h, None] * sk[None, :, h] / 4)
        eps_row = np.where(np.tril(np.ones((S, S), bool)), eps, 0).max(axis=1)
        d = 2 * eps_row + 2 * np.log1p(2.0 ** -4)
        vmax = np.abs(v[:, h]).max()
        n = np.arange(1, S + 1)
        bound = (np.exp(d) - np.exp(-d)) * vmax + np.abs(vh[:, h] - v[:, h]).max() \
            + 2 * n * (2.0 ** -10 / 448) * vmax
        err = np.abs(out[:, h] - ex[:, h]).max(axis=1)
        assert np.all(err <= bound), (h, float((err - bound).max()))
        assert np.all(np.abs(lse[:, h] - ex_lse[:, h]) <= d + 1e-12)
        # and the quantised method is far from trivially loose here
        assert err.mean() < 0.05


def test_running_max_rescale_closed_form():
    # Keys of block 0 all equal k_a, keys of block 1 all equal 2 k_a (same INT8 codes,
    # twice the scale: logit 2 L for logit L).  Every weight quantises exactly (p = 1 at
    # the block's running maximum); when block 1 raises the maximum, block 0's sums are
    # rescaled by r = exp(L - 2L), so rows i >= 128 give
    #   O_i = (r sum_{j<128} v_j + sum_{128<=j<=i} v_j) / (128 r + i - 127).
    rng = np.random.default_rng(8)
    S, H = 200, 1
    q0 = rng.standard_normal((1, H, 192)).astype(np.float32)
    ka = q0 * 0.02  # positive logit L
    q = np.repeat(bits(q0), S, axis=0)
    k = np.concatenate([np.repeat(bits(ka), 128, axis=0), np.repeat(bits(2 * ka), S - 128, axis=0)])
    v = grid_values(rng, (S, H, 128))
    out, lse = SA.sage_prefill_ref(q, k, bits(v))
    qc, sq = SA.quantize_int8_rows(F.O.bf16_to_f64(bits(q0)).astype(np.float32))
    kc, sk = SA.quantize_int8_rows(F.O.bf16_to_f64(bits(ka)).astype(np.float32))
    L = float((qc.astype(np.int64) * kc.astype(np.int64)).sum() * np.float64(sq[0, 0]) * np.float64(sk[0, 0])
              * SA.SCALE_192)
    assert L > 0
    r = np.exp(-L)
    i = np.arange(128, S)
    num = r * v[:128].sum(axis=0) + np.cumsum(v[128:], axis=0)
    den = (128 * r + (i - 127))[:, None, None]
    assert np.allclose(out[128:], num / den, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse[128:, 0], 2 * L + np.log(128 * r + (i - 127)), rtol=1e-12, atol=1e-12)
    assert np.allclose(out[:128], np.cumsum(v[:128], axis=0) / np.arange(1, 129)[:, None, None], rtol=1e-12)


def test_row_subset_follows_the_same_steps():
    # a subset of query rows gives exactly those rows of the full computation
    rng = np.random.default_rng(9)
    S, H = 333, 2
    q, k, v = rand_bf16(rng, (S, H, 192)), rand_bf16(rng, (S, H, 192)), rand_bf16(rng, (S, H, 128))
    out, lse = SA.sage_prefill_ref(q, k, v)
    rows = [0, 1, 127, 128, 200, 255, 256, 332]
    o2, l2 = SA.sage_prefill_ref(q, k, v, rows=rows)
    assert np.array_equal(o2, out[rows]) and np.array_equal(l2, lse[rows])
