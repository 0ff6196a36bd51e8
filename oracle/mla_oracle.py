"""Plain float64 CPU oracle for weight-absorbed MLA decode over a paged latent cache.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or run this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the CUDA
library in ``deepseek_mla_decode_b200/`` and imports nothing from it.

What is computed (sources, by page title and section):

* Weight-absorbed MLA ("WA-MLA") -- KsanaLLM 0.6.0 release notes, section 2.1
  (DP attention / WA-MLA): in decode the per-head key/value up-projections are folded
  into the query and output, so every head attends directly over one shared latent
  cache row per token instead of per-head K/V.
* The cache row is 576 wide: a 512-d latent ``c_kv`` followed by a 64-d decoupled
  RoPE key ``k_pe``; the score of head h against token t is
  ``scale * (q_nope[h] . c_kv[t] + q_pe[h] . k_pe[t])`` and the value is ``c_kv[t]``.
  The softmax scale is 1/sqrt(192) because DeepSeek's attention head dimension is 192
  (128 no-RoPE + 64 RoPE) -- Paddle 3.0 inference upgrade article, long-sequence
  section (SageAttention, head dim 192).
* Several query tokens per sequence in one decode call (draft-token verification
  keeps the batch size) -- Paddle 3.0 article, speculative-decoding section.  The new
  tokens are the last ``s_q`` cache positions (bottom-right causal alignment).
* ``softmax_lse`` is returned beside the output (natural log, scale included) --
  "DeepSeek speed test / FA3" article, section 2.1.
* Paged KV: fixed 64-row physical blocks addressed through a per-sequence block
  table -- Dewu deployment slides (PagedAttention); "DeepSeek speed test" article 4.1.
* Split-KV: a sequence's keys are split into disjoint ranges whose normalised partial
  outputs are merged by their log-sum-exp -- "DeepSeek speed test" article 2.1
  ("split-K parallelism"); the merge identity is exact algebra.

Readings where the pages are silent (this library's own; each is stated here):
V is the first 512 columns of the same cache row; lse uses the natural log and
includes the scale; rows with no visible key give out = 0 and lse = -inf; block-table
entries past ceil(n/64) and rows past n in the last block are never read.

Parity status: every function here is pinned by tests in ``tests/test_oracle_pins.py``
against closed forms, invariants, an independent non-absorbed formulation and scalar
brute force.  ``schedule_ref`` is a deterministic integer algorithm of this library's
own design (the pages only name split-K); it is pinned by structural validity checks
and hand-worked schedules.
"""

from __future__ import annotations

import math
from typing import Dict, List, Tuple

import numpy as np

BLOCK_SIZE = 64  # cache rows per physical block
D_LATENT = 512  # c_kv width (= value width = output width)
D_ROPE = 64  # k_pe / q_pe width
D_QK = D_LATENT + D_ROPE  # 576, width of one cache row


# ----------------------------------------------------------------------------
# bf16 bits -> float64 (exact: a bf16 is the upper half of an IEEE binary32)
# ----------------------------------------------------------------------------
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Convert raw bf16 bit patterns (uint16) to float64 exactly."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------
# the definition
# ----------------------------------------------------------------------------
def visible_key_count(n: int, s_q: int, i: int, causal: bool) -> int:
    """Number of keys query token ``i`` (0-based among the s_q new tokens) may see.

    The s_q new tokens occupy cache positions n-s_q .. n-1, so with the causal mask
    token i sees positions 0 .. n-s_q+i (Paddle 3.0 article, speculative decoding:
    draft tokens are verified in one pass; bottom-right alignment is the plain
    reading).  Without the mask every token sees all n keys.
    """
    if n <= 0:
        return 0
    if not causal:
        return n
    return max(0, min(n, n - s_q + i + 1))


def gather_rows(kv_cache: np.ndarray, block_table_row: np.ndarray, n: int) -> np.ndarray:
    """Logical rows 0..n-1 of one sequence: row t lives at
    kv_cache[block_table_row[t // 64], t % 64, :] (PagedAttention block table)."""
    if n == 0:
        return np.zeros((0, kv_cache.shape[-1]), dtype=kv_cache.dtype)
    t = np.arange(n)
    return kv_cache[block_table_row[t // BLOCK_SIZE], t % BLOCK_SIZE, :]


def mla_decode_ref(
    q_nope: np.ndarray,
    q_pe: np.ndarray,
    kv_cache: np.ndarray,
    block_table: np.ndarray,
    cache_seqlens: np.ndarray,
    softmax_scale: float,
    causal: bool,
    q_lens=None,
) -> Tuple[np.ndarray, np.ndarray]:
    """Weight-absorbed MLA decode attention, float64, no tiling or online softmax.

    q_nope [B, s_q, H, 512], q_pe [B, s_q, H, 64], kv_cache [num_blocks, 64, 576]
    (all float64 holding the bf16 input values), block_table [B, max_blocks] int,
    cache_seqlens [B] int.  Returns out [B, s_q, H, 512] and lse [B, s_q, H]:

        s_t   = scale * (q_nope . c_kv[t] + q_pe . k_pe[t])   for visible t
        lse   = ln sum_t exp(s_t)            (computed as m + ln sum exp(s_t - m))
        out   = sum_t exp(s_t - lse) * c_kv[t]

    ``q_lens`` [B] (optional) gives sequence b its own number of query tokens
    q_lens[b] <= s_q (draft tokens accepted per sequence differ in speculative
    decoding: Paddle 3.0 article, speculative-decoding section).  Its new tokens are
    the last q_lens[b] cache positions, so with the causal mask token i sees keys
    0 .. n - q_lens[b] + i; tokens i >= q_lens[b] are padding and give out = 0,
    lse = -inf.  Without q_lens every sequence has s_q tokens.
    """
    B, s_q, H, dl = q_nope.shape
    assert dl == D_LATENT and q_pe.shape == (B, s_q, H, D_ROPE)
    assert kv_cache.shape[1:] == (BLOCK_SIZE, D_QK)
    out = np.zeros((B, s_q, H, D_LATENT), dtype=np.float64)
    lse = np.full((B, s_q, H), -np.inf, dtype=np.float64)
    for b in range(B):
        n = int(cache_seqlens[b])
        s_b = s_q if q_lens is None else int(q_lens[b])
        assert 0 <= s_b <= s_q
        rows = gather_rows(kv_cache, block_table[b], n)  # [n, 576]
        q = np.concatenate([q_nope[b], q_pe[b]], axis=-1)  # [s_q, H, 576]
        scores = softmax_scale * (q @ rows.T)  # [s_q, H, n]
        for i in range(s_b):
            nv = visible_key_count(n, s_b, i, causal)
            if nv == 0:
                continue  # out stays 0, lse stays -inf
            s = scores[i, :, :nv]
            m = s.max(axis=-1, keepdims=True)
            e = np.exp(s - m)
            z = e.sum(axis=-1, keepdims=True)
            out[b, i] = (e @ rows[:nv, :D_LATENT]) / z
            lse[b, i] = (m + np.log(z))[:, 0]
    return out, lse


# ----------------------------------------------------------------------------
# weight absorption either side of the decode
# ----------------------------------------------------------------------------
D_NOPE = 128  # per-head no-RoPE query / value width of DeepSeek's attention head


def absorb_q_ref(q_heads: np.ndarray, w_uk: np.ndarray) -> np.ndarray:
    """Absorbed latent query: q_nope[b,i,h,:] = W_UK[h]^T q[b,i,h,:].

    q_heads [B, s_q, H, 128] (the per-head no-RoPE queries), w_uk [H, 128, 512] (the
    key up-projection of each head, k_h = W_UK[h] c).  Folding W_UK into the query
    lets every head score the shared 512-d latent directly (KsanaLLM 0.6.0 release
    notes, section 2.1, WA-MLA).  Returns [B, s_q, H, 512], float64."""
    return np.einsum("bihd,hdc->bihc", q_heads, w_uk)


def absorb_out_ref(o_latent: np.ndarray, w_uv: np.ndarray) -> np.ndarray:
    """Per-head output from the latent one: y[b,i,h,:] = W_UV[h] o[b,i,h,:].

    o_latent [B, s_q, H, 512] (the decode output), w_uv [H, 128, 512] (the value
    up-projection of each head, v_h = W_UV[h] c); the attention-weighted sum of
    v_h is W_UV[h] applied to the weighted sum of latents (same section).  Returns
    [B, s_q, H, 128], float64."""
    return np.einsum("bihc,hdc->bihd", o_latent, w_uv)


# ----------------------------------------------------------------------------
# split-KV partials and their log-sum-exp merge
# ----------------------------------------------------------------------------
def partial_ref(
    q_nope_b: np.ndarray,
    q_pe_b: np.ndarray,
    rows: np.ndarray,
    key_lo: int,
    key_hi: int,
    softmax_scale: float,
    causal: bool,
    n: int,
) -> Tuple[np.ndarray, np.ndarray]:
    """Attention of one sequence restricted to keys [key_lo, key_hi).

    Returns the partial output normalised by its own softmax sum, O_s [s_q, H, 512],
    and its lse_s [s_q, H] (-inf, with O_s = 0, where no key of the range is
    visible).  ``rows`` are the sequence's gathered cache rows, ``n`` its length.
    """
    s_q, H, _ = q_nope_b.shape
    q = np.concatenate([q_nope_b, q_pe_b], axis=-1)
    o = np.zeros((s_q, H, D_LATENT))
    l = np.full((s_q, H), -np.inf)
    for i in range(s_q):
        hi = min(key_hi, visible_key_count(n, s_q, i, causal))
        if hi <= key_lo:
            continue
        r = rows[key_lo:hi]
        s = softmax_scale * (q[i] @ r.T)
        m = s.max(axis=-1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=-1, keepdims=True)
        o[i] = (e @ r[:, :D_LATENT]) / z
        l[i] = (m + np.log(z))[:, 0]
    return o, l


def lse_combine_ref(o_parts: List[np.ndarray], lse_parts: List[np.ndarray]):
    """Merge normalised partials: lse = ln sum_s exp(lse_s);
    out = sum_s exp(lse_s - lse) * O_s.  Rows where every lse_s is -inf give
    out = 0 and lse = -inf."""
    L = np.stack(lse_parts)  # [S, ...]
    O = np.stack(o_parts)  # [S, ..., 512]
    m = L.max(axis=0)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    w = np.where(np.isfinite(L), np.exp(L - m_safe), 0.0)
    z = w.sum(axis=0)
    lse = np.where(finite, m_safe + np.log(np.where(finite, z, 1.0)), -np.inf)
    coef = np.where(finite, w / np.where(finite, z, 1.0), 0.0)
    out = (coef[..., None] * O).sum(axis=0)
    return out, lse


# ----------------------------------------------------------------------------
# split-KV schedule (integer; bit-exact target for the device scheduler)
# ----------------------------------------------------------------------------
SCHED_KEYS_PER_TILE = 256  # scheduling unit: a key tile of 4 blocks
SCHED_BLOCKS_PER_TILE = SCHED_KEYS_PER_TILE // 64
SCHED_OVERHEAD_TILES = 1  # cost of starting a sequence, in key tiles
SCHED_MIN_CAP = 2  # smallest partition cost (tiles), so tiny problems are not shattered
ROWS_PER_TILE = 128  # query rows (heads x draft tokens) handled by one worker


def schedule_ref(cache_seqlens: np.ndarray, s_q: int, H: int, num_workers: int) -> Dict:
    """Split-KV schedule: cut the concatenation of all sequences' key tiles into
    contiguous ranges of near-equal cost, one per partition.  Cuts fall on whole
    tiles of SCHED_BLOCKS_PER_TILE blocks, so a split never leaves a ragged tile
    except at a sequence's end.

    Cost model: every key tile (up to 4 blocks) costs 1, and every sequence with at
    least one block costs SCHED_OVERHEAD_TILES extra, placed just before its first
    tile.  Let pre[b] be the total cost of sequences before b; tile j of sequence b
    sits at cost position pos = pre[b] + OVERHEAD + j.  With P = num_workers // T
    partitions (T = ceil(s_q*H / 128) row tiles, each row tile scheduled
    identically) and cap = max(SCHED_MIN_CAP, ceil(total_cost / P)), tile (b, j)
    and its blocks belong to partition floor(pos / cap).

    Returns a dict of int arrays:
      num_parts, num_tiles, cap, total_slots (scalars)
      part_start [P, 2]  (b, k) of the partition's first block ((B, 0) if empty)
      part_end   [P, 2]  exclusive end (next partition's start)
      nblk [B], first_part [B], num_splits [B], split_prefix [B]
    A sequence's piece in partition p has split index p - first_part[b]; its
    workspace slot is split_prefix[b] + that index.
    """
    seqlens = np.asarray(cache_seqlens, dtype=np.int64)
    B = seqlens.shape[0]
    T = -(-(s_q * H) // ROWS_PER_TILE)
    P = max(1, num_workers // T)
    nblk = np.where(seqlens > 0, -(-seqlens // BLOCK_SIZE), 0)
    ntile = -(-nblk // SCHED_BLOCKS_PER_TILE)
    cost = np.where(nblk > 0, ntile + SCHED_OVERHEAD_TILES, 0)
    pre = np.concatenate([[0], np.cumsum(cost)])  # [B+1]
    total = int(pre[-1])
    cap = max(SCHED_MIN_CAP, -(-total // P))

    first_part = np.zeros(B, dtype=np.int64)
    num_splits = np.zeros(B, dtype=np.int64)
    for b in range(B):
        if nblk[b] == 0:
            continue
        p0 = (pre[b] + SCHED_OVERHEAD_TILES) // cap
        p1 = (pre[b] + SCHED_OVERHEAD_TILES + ntile[b] - 1) // cap
        first_part[b] = p0
        num_splits[b] = p1 - p0 + 1
    split_prefix = np.concatenate([[0], np.cumsum(num_splits)])[:B]
    total_slots = int(num_splits.sum())

    # start of partition p: the first tile whose position is >= p * cap
    part_start = np.tile(np.array([B, 0], dtype=np.int64), (P, 1))
    for p in range(P):
        target = p * cap
        for b in range(B):
            if nblk[b] == 0:
                continue
            first_pos = pre[b] + SCHED_OVERHEAD_TILES
            last_pos = first_pos + ntile[b] - 1
            if last_pos >= target:
                j = max(0, target - first_pos)
                part_start[p] = (b, j * SCHED_BLOCKS_PER_TILE)
                break
    part_end = np.empty_like(part_start)
    part_end[:-1] = part_start[1:]
    part_end[-1] = (B, 0)
    return dict(
        num_parts=P,
        num_tiles=T,
        cap=cap,
        total_slots=total_slots,
        part_start=part_start,
        part_end=part_end,
        nblk=nblk,
        first_part=first_part,
        num_splits=num_splits,
        split_prefix=split_prefix,
    )


def pieces_of_partition(sched: Dict, p: int) -> List[Tuple[int, int, int, int]]:
    """(b, k_lo, k_hi, split_index) for every piece of partition p, in order."""
    (b, k), (be, ke) = sched["part_start"][p], sched["part_end"][p]
    nblk = sched["nblk"]
    B = nblk.shape[0]
    out = []
    while b < B and (b < be or (b == be and k < ke)):
        hi = ke if b == be else nblk[b]
        if k < hi:
            out.append((int(b), int(k), int(hi), int(p - sched["first_part"][b])))
        b, k = b + 1, 0
    return out


def mla_decode_split_ref(q_nope, q_pe, kv_cache, block_table, cache_seqlens, softmax_scale,
                         causal, sched: Dict):
    """The decode computed the split-KV way: every piece of the schedule produces a
    normalised partial over its key range, and each sequence's partials are merged
    with ``lse_combine_ref``.  Mathematically identical to ``mla_decode_ref``."""
    B, s_q, H, _ = q_nope.shape
    parts: Dict[int, List] = {b: [] for b in range(B)}
    for p in range(sched["num_parts"]):
        for b, k_lo, k_hi, s in pieces_of_partition(sched, p):
            n = int(cache_seqlens[b])
            rows = gather_rows(kv_cache, block_table[b], n)
            lo, hi = k_lo * BLOCK_SIZE, min(n, k_hi * BLOCK_SIZE)
            parts[b].append((s, partial_ref(q_nope[b], q_pe[b], rows, lo, hi, softmax_scale,
                                            causal, n)))
    out = np.zeros((B, s_q, H, D_LATENT))
    lse = np.full((B, s_q, H), -np.inf)
    for b in range(B):
        if not parts[b]:
            continue
        parts[b].sort(key=lambda x: x[0])
        o, l = lse_combine_ref([x[1][0] for x in parts[b]], [x[1][1] for x in parts[b]])
        out[b], lse[b] = o, l
    return out, lse


def flops_and_bytes(cache_seqlens: np.ndarray, s_q: int, H: int, causal: bool) -> Tuple[int, int]:
    """Algorithmic work of one decode call: FLOPs = sum over (sequence, query token,
    visible key, head) of 2*(576+512); cache bytes = every visible cache row read once
    (576 bf16 = 1152 B per (sequence, key)), independent of H and s_q."""
    flops = 0
    rows = 0
    for n in np.asarray(cache_seqlens).tolist():
        rows += int(n)
        for i in range(s_q):
            flops += visible_key_count(int(n), s_q, i, causal) * H * 2 * (D_QK + D_LATENT)
    return flops, rows * D_QK * 2
