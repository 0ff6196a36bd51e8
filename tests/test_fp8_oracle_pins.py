"""Pins of the FP8 (e4m3) latent-cache oracle against facts fixed independently of
its own code: the e4m3 encoding's defining values, exact round trips, the tie and
saturation rules, the half-spacing error bound of the quantiser, and bit-exact
agreement with the bf16 oracle on rows the format holds exactly."""

import math

import numpy as np
import pytest

from oracle import mla_oracle as O
from oracle import mla_fp8_oracle as F
from deepseek_mla_decode_b200.workloads import f32_to_bf16_bits, make_inputs


def test_e4m3_defining_values():
    # by the format's definition: bias 7, 3 mantissa bits, no infinities
    assert F.e4m3_decode(np.uint8(0x00)) == 0.0
    assert F.e4m3_decode(np.uint8(0x01)) == 2.0 ** -9  # smallest subnormal
    assert F.e4m3_decode(np.uint8(0x07)) == 7 * 2.0 ** -9  # largest subnormal
    assert F.e4m3_decode(np.uint8(0x08)) == 2.0 ** -6  # smallest normal
    assert F.e4m3_decode(np.uint8(0x38)) == 1.0
    assert F.e4m3_decode(np.uint8(0x3C)) == 1.5
    assert F.e4m3_decode(np.uint8(0x7E)) == 448.0  # largest finite
    assert F.e4m3_decode(np.uint8(0xFE)) == -448.0
    assert F.e4m3_decode(np.uint8(0xB8)) == -1.0
    assert math.isnan(F.e4m3_decode(np.uint8(0x7F))) and math.isnan(F.e4m3_decode(np.uint8(0xFF)))
    finite = F.E4M3_VALUES[np.isfinite(F.E4M3_VALUES)]
    assert finite.size == 254 and np.unique(finite).size == 253  # +0 and -0 coincide


def test_encode_decode_round_trip():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = F.e4m3_decode(codes).astype(np.float32)
    vals[codes == 0x80] = np.float32(-0.0)
    assert np.array_equal(F.e4m3_encode(vals), codes)


def test_ties_go_to_even_code_and_saturation():
    pos = F.E4M3_VALUES[:127]
    for c in range(0, 126):
        mid = (pos[c] + pos[c + 1]) / 2  # exactly representable in float32
        want = c if c % 2 == 0 else c + 1
        assert F.e4m3_encode(np.float32(mid)) == want, c
        assert F.e4m3_encode(np.nextafter(np.float32(mid), np.float32(0))) == c
        assert F.e4m3_encode(np.nextafter(np.float32(mid), np.float32(1e9))) == c + 1
    for big in (448.0, 449.0, 464.0, 480.0, 1e9):
        assert F.e4m3_encode(np.float32(big)) == 0x7E
        assert F.e4m3_encode(np.float32(-big)) == 0xFE
    assert F.e4m3_encode(np.float32(2.0 ** -10)) == 0x00  # tie with 2^-9 -> even code 0
    assert F.e4m3_encode(np.float32(-(2.0 ** -11))) == 0x80  # sign of zero kept


def test_quantiser_error_bound_and_scale():
    inp = make_inputs(2, 1, 16, [300, 200], seed=5)
    rows = inp.kv_cache
    codes, kpe, scale = F.quantize_rows(rows)
    r = O.bf16_to_f64(rows)
    amax = np.max(np.abs(r), axis=-1)
    assert np.array_equal(scale, (amax.astype(np.float32) / np.float32(448.0)).astype(np.float32))
    # k_pe' = k_pe / scale to within half a bf16 ulp (2^-8 relative: 8 significant
    # bits) plus the fp32 quotient's rounding
    kq = r[..., 512:] / scale[..., None].astype(np.float64)
    kd = O.bf16_to_f64(kpe)
    assert np.all(np.abs(kd - kq) <= np.abs(kq) * (2.0 ** -8 + 2.0 ** -23) + 1e-30)
    c = r[..., :512]
    x = c / scale[..., None].astype(np.float64)  # exact quotient
    deq = F.e4m3_decode(codes)
    a = np.abs(deq)
    # spacing of e4m3 around |value|: 2^-9 below 2^-6, else 2^(floor(log2 a) - 3)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    spacing = np.where(a < 2.0 ** -6, 2.0 ** -9, 2.0 ** (e - 3))
    # quotient rounded to fp32 first, then to e4m3: half a spacing plus the fp32 rounding
    assert np.all(np.abs(x - deq) <= spacing / 2 * (1 + 2.0 ** -20) + np.abs(x) * 2.0 ** -23)
    # where the row maximum lies in c_kv it maps to +-448 exactly
    in_c = np.max(np.abs(c), axis=-1) == amax
    arg = np.argmax(np.abs(c), axis=-1)
    top = np.take_along_axis(codes, arg[..., None], axis=-1)[..., 0]
    assert in_c.any() and np.all(((top == 0x7E) | (top == 0xFE))[in_c])


def test_zero_row_has_zero_scale_and_codes():
    rows = np.zeros((1, 64, 576), dtype=np.uint16)
    codes, kpe, scale = F.quantize_rows(rows)
    assert np.all(scale == 0) and np.all(codes == 0) and np.all(kpe == 0)


def test_packed_row_layout():
    inp = make_inputs(1, 1, 16, [64], seed=6)
    packed = F.pack_cache(inp.kv_cache)
    assert packed.shape == (inp.kv_cache.shape[0], 64, 656)
    codes, kpe, scale = F.unpack_cache(packed)
    assert np.all(packed[..., 644:] == 0)
    c2, k2, s2 = F.quantize_rows(inp.kv_cache)
    assert np.array_equal(codes, c2) and np.array_equal(kpe, k2) and np.array_equal(scale, s2)


def test_fp8_decode_equals_bf16_decode_on_exact_rows():
    """Rows whose latent values are e4m3 values with a 448 in each row (and k_pe
    within +-448) quantise with scale 1, codes equal to the values and k_pe stored
    unchanged, so the FP8 decode must equal the bf16 decode bit for bit."""
    inp = make_inputs(3, 2, 16, [70, 130, 5], seed=7, causal=True, poison=False)
    rng = np.random.default_rng(8)
    grid = F.E4M3_VALUES[:127][F.E4M3_VALUES[:127] <= 8.0]
    vals = rng.choice(grid, size=inp.kv_cache[..., :512].shape) * rng.choice([-1.0, 1.0], size=inp.kv_cache[..., :512].shape)
    vals[..., 17] = 448.0
    inp.kv_cache[..., :512] = f32_to_bf16_bits(vals.astype(np.float32))  # exact in bf16
    packed = F.pack_cache(inp.kv_cache)
    _, _, scale = F.unpack_cache(packed)
    assert np.all(scale == 1.0)
    args = (O.bf16_to_f64(inp.q_nope), O.bf16_to_f64(inp.q_pe))
    o8, l8 = F.mla_decode_fp8_ref(*args, packed, inp.block_table, inp.cache_seqlens, inp.softmax_scale, True)
    o16, l16 = O.mla_decode_ref(*args, O.bf16_to_f64(inp.kv_cache), inp.block_table, inp.cache_seqlens,
                                inp.softmax_scale, True)
    assert np.array_equal(o8, o16) and np.array_equal(l8, l16)


def test_fp8_decode_within_perturbation_bound_of_bf16_decode():
    """Quantisation moves each stored value by delta (latent and RoPE parts); a score
    moves by at most Delta = scale * sum |q| |delta|, so every weight changes by a
    factor within exp(+-2 Delta) and the weights' total variation is at most
    exp(2 Delta) - 1.  Hence |out - out8| <= max |delta_c| + (exp(2 Delta) - 1) max |c|
    per query row, and |lse - lse8| <= Delta."""
    inp = make_inputs(2, 1, 32, [500, 900], seed=9)
    packed = F.pack_cache(inp.kv_cache)
    qn, qp = O.bf16_to_f64(inp.q_nope), O.bf16_to_f64(inp.q_pe)
    o8, l8 = F.mla_decode_fp8_ref(qn, qp, packed, inp.block_table, inp.cache_seqlens, inp.softmax_scale, False)
    o16, l16 = O.mla_decode_ref(qn, qp, O.bf16_to_f64(inp.kv_cache), inp.block_table, inp.cache_seqlens,
                                inp.softmax_scale, False)
    deq = F.dequantize_cache(packed)
    orig = O.bf16_to_f64(inp.kv_cache)
    for b in range(inp.B):
        n = int(inp.cache_seqlens[b])
        r16 = O.gather_rows(orig, inp.block_table[b], n)
        r8 = O.gather_rows(deq, inp.block_table[b], n)
        delta = np.abs(r8 - r16)
        q = np.concatenate([qn[b, 0], qp[b, 0]], axis=-1)
        big_delta = inp.softmax_scale * (np.abs(q) @ delta.T).max(axis=-1)  # [H]
        bound = delta[:, :512].max() + (np.exp(2 * big_delta) - 1) * np.abs(r16[:, :512]).max()
        err = np.abs(o8[b, 0] - o16[b, 0]).max(axis=-1)
        assert np.all(err <= bound), (err.max(), bound.min())
        assert np.all(np.abs(l8[b, 0] - l16[b, 0]) <= big_delta * (1 + 1e-12))
