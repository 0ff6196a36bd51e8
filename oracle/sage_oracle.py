"""Plain CPU oracle for quantised (SageAttention-style) causal prefill attention with
head dimension 192.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or run this
module: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs use
it.  It shares no code with the CUDA library and imports nothing from it.

Source: Paddle 3.0 inference upgrade article, long-sequence section.  For long-prompt
prefill the attention is computed with SageAttention's dynamic quantisation: Q and K
are quantised to INT8 and V to FP8; the INT32 products Q K^T are converted to FP32 and
dequantised, then an online softmax runs; its weights P are quantised to FP8 and
multiplied with the FP8 V, and the product is dequantised by V's scale.  DeepSeek's
case is a head dimension of 192 (128 without RoPE + 64 RoPE) for Q and K; V has 128.

Readings where the page is silent (this library's own; each is stated here):

1. Q and K are quantised per (token, head): ``s = max|x| / 127`` over the 192 values,
   ``code = round-half-even(x / s)``, scale and quotient in IEEE fp32; a zero row has
   ``s = 0`` and codes 0.  (Per-token scales factor out of the score as a row factor
   times a column factor.)
2. V is quantised per (head, channel) over all tokens: ``s_v = max_t |v| / 448`` (448
   = the largest finite e4m3), ``code = e4m3(v / s_v)`` (fp32 quotient, nearest even,
   saturating); a zero channel has ``s_v = 0``.  The dequantised V is
   ``code_value * s_v`` -- a per-channel factor applied after the product, as the page
   describes.
3. Logits ``S_ij = (sum_d Qc_id Kc_jd) * s_q[i] * s_k[j] * softmax_scale`` with the
   integer dot product exact, ``softmax_scale = 1/sqrt(192)`` and the causal mask
   ``j <= i`` (a prefill over one sequence: query i is token i).
4. The online softmax walks the keys in blocks of 128 (``[128 b, 128 b + 128)``); for
   each row, ``m_b = max(m_{b-1}, max of the block's visible logits)`` (the running
   maximum, updated at every block), ``p = exp(S - m_b)`` in (0, 1], and P is quantised
   as ``Pc = e4m3(p * 448)`` (nearest even) with ``P^ = Pc / 448``.  The running sums
   are rescaled by ``exp(m_{b-1} - m_b)``: ``l = l * r + sum P^``, ``A = A * r +
   sum P^ V^``.  The output is ``O = A / l`` -- normalised by the quantised weights that
   entered the product, so the weights of a row sum to one -- and ``lse = m + log l``
   (natural log, softmax scale included).

Parity: pinned in ``tests/test_sage_oracle_pins.py`` by the quantisers' bounds and
hand-checked codes, exact cases (equal logits give the mean of the visible dequantised
V rows; row 0 sees only its own key), invariants (causality, per-channel scaling of V,
permutation of V's channels) and a derived error bound against exact float64 softmax
attention on the unquantised inputs.
"""

from __future__ import annotations

from typing import Tuple

import numpy as np

from . import mla_fp8_oracle as F

D_QK = 192
D_V = 128
KEY_BLOCK = 128
INT8_MAX = 127.0
E4M3_MAX = 448.0
SCALE_192 = 1.0 / np.sqrt(192.0)


def quantize_int8_rows(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per-row symmetric INT8: x float32 [..., D] -> (codes int8 [..., D], scale float32
    [...]) with scale = max|x| / 127 and code = rint(x / scale) (ties to even), both in
    IEEE fp32."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=-1)
    scale = (amax / np.float32(INT8_MAX)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    q = (x / safe[..., None]).astype(np.float32)
    codes = np.where((scale > 0)[..., None], np.rint(q), 0.0)
    codes = np.clip(codes, -INT8_MAX, INT8_MAX).astype(np.int8)
    return codes, scale


def quantize_v_channels(v: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """V float32 [S, H, 128] -> (e4m3 codes uint8 [S, H, 128], scale float32 [H, 128])
    with one scale per (head, channel) over all tokens: max|v| / 448."""
    v = np.asarray(v, dtype=np.float32)
    amax = np.max(np.abs(v), axis=0)  # [H, 128]
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    q = (v / safe[None]).astype(np.float32)
    codes = np.where((scale > 0)[None], F.e4m3_encode(q), np.uint8(0)).astype(np.uint8)
    return codes, scale


def sage_prefill_ref(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray,
                     softmax_scale: float = SCALE_192, rows=None) -> Tuple[np.ndarray, np.ndarray]:
    """Quantised causal prefill attention.  q, k: bf16 bits [S, H, 192]; v: bf16 bits
    [S, H, 128].  Returns (out float64 [R, H, 128], lse float64 [R, H]) for the query
    rows ``rows`` (all S rows when None); each row follows the same steps whether or not
    the others are computed (the quantisation scales still come from every token)."""
    q = F.O.bf16_to_f64(q_bits).astype(np.float32)
    k = F.O.bf16_to_f64(k_bits).astype(np.float32)
    v = F.O.bf16_to_f64(v_bits).astype(np.float32)
    S, H, d = q.shape
    assert d == D_QK and k.shape == (S, H, D_QK) and v.shape == (S, H, D_V)
    qc, sq = quantize_int8_rows(q)  # [S, H, 192], [S, H]
    kc, sk = quantize_int8_rows(k)
    vc, sv = quantize_v_channels(v)
    v_hat = F.e4m3_decode(vc) * sv.astype(np.float64)[None]  # [S, H, 128]
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    R = rows.size
    out = np.zeros((R, H, D_V))
    lse = np.zeros((R, H))
    last = int(rows.max()) + 1 if R else 0  # keys past the last row are never visible
    for h in range(H):
        # exact integer scores (int64 accumulation of int8 products)
        s_int = qc[rows, h, :].astype(np.int64) @ kc[:last, h, :].astype(np.int64).T  # [R, last]
        logits = s_int.astype(np.float64) * sq[rows, h].astype(np.float64)[:, None] \
            * sk[:last, h].astype(np.float64)[None, :] * softmax_scale
        m = np.full(R, -np.inf)
        l = np.zeros(R)
        acc = np.zeros((R, D_V))
        for b0 in range(0, last, KEY_BLOCK):
            cols = np.arange(b0, min(b0 + KEY_BLOCK, last))
            live = rows >= b0  # rows that see at least one key of this block
            blk = logits[:, b0:b0 + cols.size]
            vis = cols[None, :] <= rows[:, None]
            blk_max = np.where(vis, blk, -np.inf).max(axis=1)
            m_new = np.where(live, np.maximum(m, blk_max), m)
            r = np.where(live & np.isfinite(m), np.exp(m - m_new), np.where(live, 0.0, 1.0))
            p = np.where(vis, np.exp(blk - np.where(live, m_new, 0.0)[:, None]), 0.0)
            p_hat = F.e4m3_decode(F.e4m3_encode((p * E4M3_MAX).astype(np.float32))) / E4M3_MAX
            p_hat = np.where(vis, p_hat, 0.0)
            l = l * r + p_hat.sum(axis=1)
            acc = acc * r[:, None] + p_hat @ v_hat[cols, h, :]
            m = m_new
        out[:, h, :] = acc / l[:, None]
        lse[:, h] = m + np.log(l)
    return out, lse


def exact_prefill_ref(q_bits, k_bits, v_bits, softmax_scale: float = SCALE_192):
    """Unquantised float64 causal softmax attention on the same bf16 inputs (the
    quantity the quantised method approximates)."""
    q = F.O.bf16_to_f64(q_bits)
    k = F.O.bf16_to_f64(k_bits)
    v = F.O.bf16_to_f64(v_bits)
    S, H, _ = q.shape
    out = np.zeros((S, H, D_V))
    lse = np.zeros((S, H))
    mask = np.tril(np.ones((S, S), dtype=bool))
    for h in range(H):
        s = (q[:, h, :] @ k[:, h, :].T) * softmax_scale
        s = np.where(mask, s, -np.inf)
        m = s.max(axis=1)
        e = np.exp(s - m[:, None])
        l = e.sum(axis=1)
        out[:, h, :] = (e @ v[:, h, :]) / l[:, None]
        lse[:, h] = m + np.log(l)
    return out, lse
