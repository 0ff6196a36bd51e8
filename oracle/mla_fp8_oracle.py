"""Plain CPU oracle for MLA decode over an FP8 (e4m3) latent cache.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or run this
module: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs use
it.  It shares no code with the CUDA library and imports nothing from it.

Sources (page titles and sections):

* 8-bit (and 4-bit) KV-cache inference is listed among the serving capabilities of
  the Paddle 3.0 inference upgrade article (closing capabilities list), beside the
  FP8 deployment of DeepSeek-R1 (same article, overview).
* A quantised KV cache scaled per token by its max-abs value: "DeepSeek speed test"
  article, section 3.1 (per-token INT8 KV).

The pages give no FP8 cache format.  The readings taken here (this library's own):

1. One fp32 scale per token (per cache row) for the whole 576-wide row:
   ``scale = amax / 448`` with ``amax = max |row|`` over c_kv and k_pe, and 448 the
   largest finite e4m3 value; both computed in fp32.
2. The 512-wide latent ``c_kv`` is quantised: the code of value ``c`` is
   ``e4m3(c / scale)``, the fp32 quotient (IEEE division, round to nearest even)
   rounded to e4m3 to nearest even, saturating to +-448.  The 64-wide RoPE key
   ``k_pe`` keeps 16 bits (it is 11 % of the row and carries position
   information) and is stored in the same scaled units: ``bf16(k_pe / scale)``,
   the fp32 quotient rounded to bf16 to nearest even.  A row with ``amax = 0`` has
   scale 0 and stores zeros.  Every stored row is then ``scale * [codes | k_pe']``.
3. e4m3 is the OCP "E4M3FN" encoding: 1 sign, 4 exponent (bias 7), 3 mantissa
   bits, no infinities, NaN = S.1111.111, largest finite 448, smallest subnormal
   2^-9.  The sign of zero is kept (-0 encodes as 0x80).
4. A cache row is packed into 656 bytes: bytes [0, 512) the e4m3 codes of c_kv,
   [512, 640) the scaled k_pe as 64 bf16, [640, 644) the fp32 scale, [644, 656)
   zero.
5. The dequantised row is ``scale * [e4m3_value(codes) | k_pe']`` (exact in
   float64), and decode over the FP8 cache is the bf16 definition
   (``mla_oracle.mla_decode_ref``) applied to the dequantised rows.

Parity: the decode table, the encoder and the quantiser are pinned in
``tests/test_fp8_oracle_pins.py`` by hand-checked codes, round trips, tie and
saturation cases and the half-spacing error bound; the decode is pinned by its
bit-exact agreement with the bf16 oracle on rows whose values the format holds
exactly.
"""

from __future__ import annotations

from typing import Tuple

import numpy as np

from . import mla_oracle as O

E4M3_MAX = 448.0
ROW_BYTES = 656  # packed FP8 cache row
OFF_KPE = 512
OFF_SCALE = 640


def _e4m3_table() -> np.ndarray:
    """float64 value of every e4m3 code 0..255 (NaN for S.1111.111)."""
    vals = np.empty(256, dtype=np.float64)
    for code in range(256):
        s = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = s * m * 2.0 ** -9  # subnormal: (m / 8) * 2^(1 - 7)
        else:
            vals[code] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


E4M3_VALUES = _e4m3_table()
_POS = E4M3_VALUES[:127]  # codes 0..126: the finite non-negative values, ascending


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Exact float64 values of e4m3 codes (uint8)."""
    return E4M3_VALUES[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Round float32 values to e4m3 codes: nearest, ties to the even code, saturating
    to +-448; NaN gives 0x7F (with the sign bit of the input)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    sign = np.signbit(x).astype(np.uint8) << 7
    a = np.abs(x)
    hi = np.clip(np.searchsorted(_POS, a, side="left"), 0, 126)  # first value >= a
    lo = np.clip(hi - 1, 0, 126)
    d_lo = a - _POS[lo]
    d_hi = _POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    mag = np.where(pick_hi, hi, lo)
    mag = np.where(a >= E4M3_MAX, 126, mag)  # saturate
    mag = np.where(np.isnan(a), 127, mag)
    return (sign | mag.astype(np.uint8)).astype(np.uint8)


def f32_to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)).astype(np.uint16)


def quantize_rows(rows_bf16: np.ndarray) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Per-token quantisation of bf16 cache rows [..., 576] (uint16 bit patterns).

    Returns (codes uint8 [..., 512], k_pe' uint16 [..., 64], scale float32 [...]):
    scale = amax / 448 over the whole row, codes = e4m3(c / scale) and
    k_pe' = bf16(k_pe / scale), every step in float32 as stated above."""
    r = O.bf16_to_f64(rows_bf16).astype(np.float32)  # exact
    amax = np.max(np.abs(r), axis=-1)  # float32, exact
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)  # IEEE fp32 division
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    q = (r / safe[..., None]).astype(np.float32)  # IEEE fp32 division
    live = (scale > 0)[..., None]
    codes = np.where(live, e4m3_encode(q[..., : O.D_LATENT]), np.uint8(0)).astype(np.uint8)
    kpe = np.where(live, f32_to_bf16_rne(q[..., O.D_LATENT :]), np.uint16(0)).astype(np.uint16)
    return codes, kpe, scale


def pack_cache(kv_cache_bf16: np.ndarray) -> np.ndarray:
    """bf16 cache [num_blocks, 64, 576] (uint16) -> packed FP8 cache
    [num_blocks, 64, 656] (uint8) in the row format stated above."""
    nb, bs, d = kv_cache_bf16.shape
    assert bs == O.BLOCK_SIZE and d == O.D_QK
    codes, kpe, scale = quantize_rows(kv_cache_bf16)
    out = np.zeros((nb, bs, ROW_BYTES), dtype=np.uint8)
    out[..., :OFF_KPE] = codes
    out[..., OFF_KPE:OFF_SCALE] = np.ascontiguousarray(kpe).view(np.uint8).reshape(nb, bs, 2 * O.D_ROPE)
    out[..., OFF_SCALE : OFF_SCALE + 4] = np.ascontiguousarray(scale, dtype=np.float32).view(np.uint8).reshape(nb, bs, 4)
    return out


def unpack_cache(packed: np.ndarray) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Packed FP8 cache -> (codes uint8 [..., 512], scaled k_pe uint16 [..., 64],
    scale float32 [...])."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    codes = packed[..., :OFF_KPE]
    kpe = np.ascontiguousarray(packed[..., OFF_KPE:OFF_SCALE]).view(np.uint16)
    scale = np.ascontiguousarray(packed[..., OFF_SCALE : OFF_SCALE + 4]).view(np.float32)[..., 0]
    return codes, kpe, scale


def dequantize_cache(packed: np.ndarray) -> np.ndarray:
    """Packed FP8 cache -> float64 rows [..., 576] = scale * [e4m3(codes) | k_pe']."""
    codes, kpe, scale = unpack_cache(packed)
    s = scale.astype(np.float64)[..., None]
    return np.concatenate([e4m3_decode(codes) * s, O.bf16_to_f64(kpe) * s], axis=-1)


def mla_decode_fp8_ref(q_nope, q_pe, kv_fp8_packed, block_table, cache_seqlens, softmax_scale, causal,
                       q_lens=None):
    """Decode over the packed FP8 cache: the float64 definition of ``mla_decode_ref``
    applied to the dequantised rows (q_nope / q_pe float64 as there; q_lens, the
    per-sequence query counts, as there)."""
    return O.mla_decode_ref(q_nope, q_pe, dequantize_cache(kv_fp8_packed), block_table, cache_seqlens,
                            softmax_scale, causal, q_lens=q_lens)
