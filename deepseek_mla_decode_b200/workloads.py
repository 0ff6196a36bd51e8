"""Seeded synthetic inputs for MLA decode (shared by tests, bench and smoke).

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic.  Values are drawn as float32 N(0, 1) from numpy's PCG64
``default_rng(seed)`` and rounded to bf16 (round-to-nearest-even on the bit
pattern), so the CUDA library and the float64 oracle see identical bits.

Workload shapes follow the decode configurations this library is measured on:
a tiny two-sequence case, a uniform decode batch, an MTP draft-verification batch
(s_q = 2, causal), a high-concurrency serving mix whose lengths follow the
1812-token-prompt / 978-token-output request mix of the KsanaLLM 0.6.0 release
notes (section 2.3), and a long-context split-KV stress case.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

BLOCK_SIZE = 64
D_LATENT = 512
D_ROPE = 64
D_QK = D_LATENT + D_ROPE
POISON = 1.0e4  # finite value planted in cache rows / blocks that must never be read


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    s_q: int
    H: int
    causal: bool
    seed: int
    lengths: str  # "fixed:<list>", "uniform:<lo>:<hi>" or "offset:<base>:<span>"

    def seqlens(self) -> np.ndarray:
        rng = np.random.default_rng(self.seed + 7919)
        kind, *args = self.lengths.split(":")
        if kind == "fixed":
            vals = [int(v) for v in args[0].split(",")]
            if len(vals) == 1:
                vals = vals * self.B
            assert len(vals) == self.B
            return np.asarray(vals, dtype=np.int32)
        if kind == "uniform":
            lo, hi = int(args[0]), int(args[1])
            return rng.integers(lo, hi + 1, size=self.B, dtype=np.int64).astype(np.int32)
        if kind == "offset":
            base, span = int(args[0]), int(args[1])
            return (base + rng.integers(0, span + 1, size=self.B, dtype=np.int64)).astype(np.int32)
        raise ValueError(self.lengths)


SCALE_192 = 1.0 / math.sqrt(192.0)

WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 2, 1, 16, False, 1000, "fixed:37,130"),
    "decode_b64": Workload("decode_b64", 64, 1, 128, False, 1001, "fixed:4096"),
    "mtp_b128_sq2": Workload("mtp_b128_sq2", 128, 2, 128, True, 1002, "uniform:1024:8192"),
    "serving_b256": Workload("serving_b256", 256, 1, 128, False, 1003, "offset:1812:978"),
    "long_b4": Workload("long_b4", 4, 1, 128, False, 1004, "fixed:65536,65536,32768,8192"),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest-even) and return the uint16 patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def _normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal(size=shape, dtype=np.float32))


@dataclass
class DecodeInputs:
    """Host arrays for one decode call.  bf16 tensors are raw uint16 bit patterns."""

    q_nope: np.ndarray  # [B, s_q, H, 512] uint16
    q_pe: np.ndarray  # [B, s_q, H, 64] uint16
    kv_cache: np.ndarray  # [num_blocks, 64, 576] uint16
    block_table: np.ndarray  # [B, max_blocks] int32
    cache_seqlens: np.ndarray  # [B] int32
    softmax_scale: float
    causal: bool
    spare_block: int  # physical block id that holds only poison (-1 if none)

    @property
    def B(self):
        return self.q_nope.shape[0]

    @property
    def s_q(self):
        return self.q_nope.shape[1]

    @property
    def H(self):
        return self.q_nope.shape[2]


def make_inputs(
    B: int,
    s_q: int,
    H: int,
    seqlens,
    seed: int,
    causal: bool = False,
    softmax_scale: float = SCALE_192,
    poison: bool = True,
    nan_poison: bool = False,
    extra_table_cols: int = 1,
    shuffle_blocks: bool = True,
) -> DecodeInputs:
    """Build a paged decode problem.

    Physical blocks: sum_b ceil(n_b / 64) used blocks plus one spare block, shuffled
    by a seeded permutation and handed to sequences in order.  Block-table entries
    past a sequence's last block point at the spare block; the spare block and the
    rows past n_b in each sequence's last block hold ``POISON`` (or NaN), so reading
    anything outside the visible range corrupts the result detectably.
    """
    rng = np.random.default_rng(seed)
    seqlens = np.asarray(seqlens, dtype=np.int32)
    assert seqlens.shape == (B,)
    nblk = [(int(n) + BLOCK_SIZE - 1) // BLOCK_SIZE for n in seqlens]
    used = int(sum(nblk))
    num_blocks = used + 1
    max_blocks = max(1, max(nblk) + extra_table_cols)

    q_nope = _normal_bf16(rng, (B, s_q, H, D_LATENT))
    q_pe = _normal_bf16(rng, (B, s_q, H, D_ROPE))
    kv = _normal_bf16(rng, (num_blocks, BLOCK_SIZE, D_QK))

    perm = rng.permutation(num_blocks) if shuffle_blocks else np.arange(num_blocks)
    spare = int(perm[-1])
    table = np.full((B, max_blocks), spare, dtype=np.int32)
    cursor = 0
    for b in range(B):
        table[b, : nblk[b]] = perm[cursor : cursor + nblk[b]]
        cursor += nblk[b]

    if poison:
        pv = np.float32(np.nan) if nan_poison else np.float32(POISON)
        pbits = f32_to_bf16_bits(np.asarray([pv]))[0]
        nbits = f32_to_bf16_bits(np.asarray([-pv]))[0]
        kv[spare, :, :] = pbits
        kv[spare, 1::2, :] = nbits
        for b in range(B):
            n = int(seqlens[b])
            if n % BLOCK_SIZE and nblk[b] > 0:
                last = table[b, nblk[b] - 1]
                kv[last, n % BLOCK_SIZE :, :] = pbits
    return DecodeInputs(q_nope, q_pe, kv, table, seqlens, float(softmax_scale), bool(causal), spare)


def make_workload(name: str, **kw) -> DecodeInputs:
    w = WORKLOADS[name]
    return make_inputs(w.B, w.s_q, w.H, w.seqlens(), w.seed, causal=w.causal, **kw)


def make_up_projections(H: int, seed: int, scale: float = 0.05):
    """Per-head up-projection weights W_UK, W_UV [H, 128, 512] as bf16 bit patterns,
    drawn N(0, scale^2) (random stand-ins for trained weights)."""
    rng = np.random.default_rng(seed)
    w_uk = f32_to_bf16_bits(rng.standard_normal((H, 128, D_LATENT), dtype=np.float32) * np.float32(scale))
    w_uv = f32_to_bf16_bits(rng.standard_normal((H, 128, D_LATENT), dtype=np.float32) * np.float32(scale))
    return w_uk, w_uv


def make_rows(shape, seed: int):
    """bf16 bit patterns of N(0, 1) draws with the given shape."""
    return _normal_bf16(np.random.default_rng(seed), shape)


# ---------------------------------------------------------------------------
# quantised prefill (SageAttention-style, head dim 192)
# ---------------------------------------------------------------------------
# The long-prompt prefill of the Paddle 3.0 inference article's long-sequence section:
# a 64K-token prompt with DeepSeek's head dimension 192 (V 128).  16 heads is one GPU's
# share of the 128 query heads under 8-way tensor parallelism.
PREFILL_S, PREFILL_H, PREFILL_SEED = 65536, 16, 2024


def make_prefill(S: int, H: int, seed: int):
    """q, k as bf16 bits [S, H, 192] and v [S, H, 128], N(0, 1)."""
    rng = np.random.default_rng(seed)
    q = _normal_bf16(rng, (S, H, 192))
    k = _normal_bf16(rng, (S, H, 192))
    v = _normal_bf16(rng, (S, H, 128))
    return q, k, v
