"""Pins for the float64 oracle: every check here ties the oracle to something other
than itself -- an independent non-absorbed MLA formulation, closed forms, algebraic
invariants of attention, scalar brute force, or hand-derived golden values."""

import json
import math
import os

import numpy as np
import pytest

from oracle import mla_oracle as O
from deepseek_mla_decode_b200.workloads import make_inputs, f32_to_bf16_bits, SCALE_192

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f64(inp):
    return (O.bf16_to_f64(inp.q_nope), O.bf16_to_f64(inp.q_pe), O.bf16_to_f64(inp.kv_cache))


def run(inp, **kw):
    qn, qp, kv = f64(inp)
    return O.mla_decode_ref(qn, qp, kv, inp.block_table, inp.cache_seqlens,
                            kw.get("scale", inp.softmax_scale), kw.get("causal", inp.causal))


# ---------------------------------------------------------------------------
# bf16 conversion
# ---------------------------------------------------------------------------
def test_bf16_roundtrip_exact():
    x = np.array([0.0, -0.0, 1.0, -2.5, 3.140625, 1e4, -1e-3, 65504.0], dtype=np.float32)
    bits = f32_to_bf16_bits(x)
    back = O.bf16_to_f64(bits)
    # every value is representable after rounding; converting back is exact and
    # equals float32 rounding to 8 significant bits
    for v, b in zip(x.tolist(), back.tolist()):
        if v == 0:
            assert b == 0
            continue
        e = math.floor(math.log2(abs(v)))
        ulp = 2.0 ** (e - 7)
        assert abs(b - v) <= ulp / 2 + 1e-30
    assert O.bf16_to_f64(np.array([0x3F80], dtype=np.uint16))[0] == 1.0
    assert O.bf16_to_f64(np.array([0xC040], dtype=np.uint16))[0] == -3.0


# ---------------------------------------------------------------------------
# independent formulation: non-absorbed MLA with explicit up-projections
# ---------------------------------------------------------------------------
def test_equals_nonabsorbed_mla():
    """Weight absorption is an algebraic identity.  With explicit per-head
    up-projections W_UK, W_UV (128 x 512), ordinary attention over
    k_h = [W_UK c ; k_pe], v_h = W_UV c with queries [q_h ; q_pe] and scale
    1/sqrt(192) equals W_UV applied to the absorbed output with
    q_nope = W_UK^T q_h."""
    rng = np.random.default_rng(5)
    B, s_q, H, n = 1, 1, 3, 11
    d_nope = 128
    c = rng.standard_normal((n, 512)) * 0.2
    k_pe = rng.standard_normal((n, 64))
    q_h = rng.standard_normal((H, d_nope))
    q_pe = rng.standard_normal((H, 64))
    W_UK = rng.standard_normal((H, d_nope, 512)) * 0.05
    W_UV = rng.standard_normal((H, d_nope, 512)) * 0.05
    scale = 1 / math.sqrt(192)

    # non-absorbed: explicit keys and values per head, textbook attention
    out_full = np.zeros((H, d_nope))
    lse_full = np.zeros(H)
    for h in range(H):
        K = np.concatenate([c @ W_UK[h].T, k_pe], axis=1)  # [n, 192]
        V = c @ W_UV[h].T  # [n, 128]
        qv = np.concatenate([q_h[h], q_pe[h]])
        s = scale * K @ qv
        w = np.exp(s - s.max())
        out_full[h] = (w / w.sum()) @ V
        lse_full[h] = s.max() + math.log(w.sum())

    # absorbed through the oracle: one block, identity table
    kv = np.zeros((1, 64, 576))
    kv[0, :n, :512] = c
    kv[0, :n, 512:] = k_pe
    q_nope = np.einsum("hd,hdc->hc", q_h, W_UK)[None, None]
    out_abs, lse_abs = O.mla_decode_ref(q_nope, q_pe[None, None], kv, np.zeros((1, 1), int),
                                        np.array([n]), scale, False)
    up = np.einsum("hc,hdc->hd", out_abs[0, 0], W_UV)
    assert np.max(np.abs(up - out_full)) < 1e-12
    assert np.max(np.abs(lse_abs[0, 0] - lse_full)) < 1e-12


def test_absorption_gemms_equal_nonabsorbed_mla():
    """absorb_q_ref -> mla_decode_ref -> absorb_out_ref equals textbook attention
    with explicit per-head keys [W_UK c ; k_pe] and values W_UV c (to 1e-12), on a
    paged batch with two query tokens, causal."""
    rng = np.random.default_rng(6)
    inp = make_inputs(2, 2, 4, [9, 70], seed=24, causal=True)
    qn_lat, qp, kv = f64(inp)
    q_h = rng.standard_normal((2, 2, 4, 128))
    W_UK = rng.standard_normal((4, 128, 512)) * 0.05
    W_UV = rng.standard_normal((4, 128, 512)) * 0.05
    q_abs = O.absorb_q_ref(q_h, W_UK)
    out_lat, lse = O.mla_decode_ref(q_abs, qp, kv, inp.block_table, inp.cache_seqlens, inp.softmax_scale, True)
    y = O.absorb_out_ref(out_lat, W_UV)
    for b in range(2):
        n = int(inp.cache_seqlens[b])
        rows = O.gather_rows(kv, inp.block_table[b], n)
        c, k_pe = rows[:, :512], rows[:, 512:]
        for i in range(2):
            nv = n - 2 + i + 1
            for h in range(4):
                K = np.concatenate([c[:nv] @ W_UK[h].T, k_pe[:nv]], axis=1)
                V = c[:nv] @ W_UV[h].T
                sc = inp.softmax_scale * K @ np.concatenate([q_h[b, i, h], qp[b, i, h]])
                w = np.exp(sc - sc.max())
                assert np.max(np.abs((w / w.sum()) @ V - y[b, i, h])) < 1e-12
                assert abs(sc.max() + math.log(w.sum()) - lse[b, i, h]) < 1e-12


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------
def test_weights_sum_to_one():
    """c_kv == 1 in every row (k_pe random) => out == 1 exactly up to rounding."""
    inp = make_inputs(2, 2, 4, [70, 129], seed=11, causal=True)
    one = f32_to_bf16_bits(np.ones(1, np.float32))[0]
    inp.kv_cache[:, :, :512] = one
    out, lse = run(inp)
    assert np.max(np.abs(out - 1.0)) < 1e-13
    assert np.all(np.isfinite(lse))


def test_zero_query_uniform_weights():
    """q = 0 => every score is 0: out = mean of the visible c_kv rows, lse = ln n."""
    inp = make_inputs(2, 1, 3, [1, 77], seed=12, poison=True)
    inp.q_nope[:] = 0
    inp.q_pe[:] = 0
    out, lse = run(inp)
    qn, qp, kv = f64(inp)
    for b, n in enumerate(inp.cache_seqlens):
        rows = np.stack([kv[inp.block_table[b, t // 64], t % 64, :512] for t in range(n)])
        assert np.max(np.abs(out[b, 0] - rows.mean(axis=0))) < 1e-12
        assert np.max(np.abs(lse[b, 0] - math.log(n))) < 1e-12


def test_single_key():
    """n = 1 => out = that row's c_kv and lse = its scaled score."""
    inp = make_inputs(1, 1, 5, [1], seed=13)
    out, lse = run(inp)
    qn, qp, kv = f64(inp)
    row = kv[inp.block_table[0, 0], 0]
    for h in range(5):
        s = inp.softmax_scale * (qn[0, 0, h] @ row[:512] + qp[0, 0, h] @ row[512:])
        assert abs(lse[0, 0, h] - s) < 1e-12
        assert np.max(np.abs(out[0, 0, h] - row[:512])) == 0.0


def test_identical_keys_give_mean_of_values():
    """All keys score equally (q_nope = 0 and one k_pe shared by all rows) =>
    out = mean of c_kv rows whatever q_pe is."""
    inp = make_inputs(1, 1, 4, [150], seed=14)
    inp.q_nope[:] = 0
    shared = inp.kv_cache[0, 0, 512:].copy()
    inp.kv_cache[:, :, 512:] = shared
    out, lse = run(inp)
    qn, qp, kv = f64(inp)
    rows = np.stack([kv[inp.block_table[0, t // 64], t % 64, :512] for t in range(150)])
    assert np.max(np.abs(out[0, 0] - rows.mean(axis=0))) < 1e-12
    s = inp.softmax_scale * (qp[0, 0] @ O.bf16_to_f64(shared))
    assert np.max(np.abs(lse[0, 0] - (s + math.log(150)))) < 1e-12


def test_golden_two_key_closed_form():
    """Hand-derived fixture (tests/golden/two_keys.json): two keys whose scores are
    set through single nonzero coordinates; out and lse follow from the two-term
    softmax in closed form."""
    with open(os.path.join(GOLDEN, "two_keys.json")) as f:
        g = json.load(f)
    H = len(g["heads"])
    q_nope = np.zeros((1, 1, H, 512))
    q_pe = np.zeros((1, 1, H, 64))
    kv = np.zeros((2, 64, 576))
    for h, head in enumerate(g["heads"]):
        q_nope[0, 0, h, 0] = head["q_nope0"]
        q_pe[0, 0, h, 0] = head["q_pe0"]
    for t, row in enumerate(g["rows"]):
        blk, off = g["block_table"][t // 64], t % 64
        for idx, val in row.items():
            kv[blk, off, int(idx)] = val
    out, lse = O.mla_decode_ref(q_nope, q_pe, kv, np.array([g["block_table"]]),
                                np.array([len(g["rows"])]), g["scale"], False)
    for h, head in enumerate(g["heads"]):
        assert abs(lse[0, 0, h] - head["lse"]) < 1e-12
        for idx, val in head["out"].items():
            assert abs(out[0, 0, h, int(idx)] - val) < 1e-12


# ---------------------------------------------------------------------------
# layout invariants
# ---------------------------------------------------------------------------
def test_paged_equals_contiguous_bit_exact():
    inp = make_inputs(3, 1, 8, [64, 200, 129], seed=15, shuffle_blocks=True)
    out_p, lse_p = run(inp)
    # rebuild the same rows contiguously with an identity block table
    qn, qp, kv = f64(inp)
    nblk = [(n + 63) // 64 for n in inp.cache_seqlens]
    kv_c = np.zeros((sum(nblk), 64, 576))
    table = np.zeros((3, max(nblk)), dtype=np.int64)
    cur = 0
    for b in range(3):
        for k in range(nblk[b]):
            kv_c[cur] = kv[inp.block_table[b, k]]
            table[b, k] = cur
            cur += 1
    out_c, lse_c = O.mla_decode_ref(qn, qp, kv_c, table, inp.cache_seqlens, inp.softmax_scale, False)
    assert np.array_equal(out_p, out_c) and np.array_equal(lse_p, lse_c)


def test_unused_table_entries_and_tail_rows_ignored():
    """Entries past ceil(n/64) point at a poisoned block and rows past n hold poison;
    replacing the poison with NaN changes nothing."""
    a = make_inputs(2, 1, 4, [37, 130], seed=16, poison=True)
    b = make_inputs(2, 1, 4, [37, 130], seed=16, poison=True, nan_poison=True)
    oa, la = run(a)
    ob, lb = run(b)
    assert np.array_equal(oa, ob) and np.array_equal(la, lb)
    assert np.all(np.isfinite(oa))


def test_causal_sq2_equals_two_sq1_calls():
    """s_q = 2 causal over n keys == s_q = 1 over n-1 keys (first token) and over n
    keys (second token)."""
    inp = make_inputs(3, 2, 6, [2, 65, 300], seed=17, causal=True)
    out, lse = run(inp)
    qn, qp, kv = f64(inp)
    for i, delta in ((0, 1), (1, 0)):
        o1, l1 = O.mla_decode_ref(qn[:, i : i + 1], qp[:, i : i + 1], kv, inp.block_table,
                                  inp.cache_seqlens - delta, inp.softmax_scale, False)
        assert np.array_equal(out[:, i], o1[:, 0]) and np.array_equal(lse[:, i], l1[:, 0])


def test_ragged_query_counts_equal_single_token_calls():
    """Per-sequence query counts: token i of sequence b with q_lens[b] = L, causal,
    over n keys == an s_q = 1 call over n - L + i + 1 keys (bit-exact); tokens
    i >= L are padding (out 0, lse -inf); q_lens = s_q everywhere is the uniform call."""
    inp = make_inputs(4, 4, 6, [3, 70, 300, 9], seed=23, causal=True)
    qn, qp, kv = f64(inp)
    q_lens = np.array([2, 4, 1, 0])
    out, lse = O.mla_decode_ref(qn, qp, kv, inp.block_table, inp.cache_seqlens, inp.softmax_scale, True,
                                q_lens=q_lens)
    for b in range(inp.B):
        L, n = int(q_lens[b]), int(inp.cache_seqlens[b])
        for i in range(4):
            if i >= L:
                assert np.all(out[b, i] == 0) and np.all(np.isneginf(lse[b, i]))
                continue
            o1, l1 = O.mla_decode_ref(qn[b : b + 1, i : i + 1], qp[b : b + 1, i : i + 1], kv,
                                      inp.block_table[b : b + 1], np.array([n - L + i + 1]), inp.softmax_scale,
                                      False)
            assert np.array_equal(out[b, i], o1[0, 0]) and np.array_equal(lse[b, i], l1[0, 0])
    u = O.mla_decode_ref(qn, qp, kv, inp.block_table, inp.cache_seqlens, inp.softmax_scale, True,
                         q_lens=np.full(4, 4))
    v = O.mla_decode_ref(qn, qp, kv, inp.block_table, inp.cache_seqlens, inp.softmax_scale, True)
    assert np.array_equal(u[0], v[0]) and np.array_equal(u[1], v[1])


def test_causal_sq1_equals_noncausal():
    inp = make_inputs(2, 1, 4, [5, 99], seed=18)
    a = run(inp, causal=True)
    b = run(inp, causal=False)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_no_visible_key_rows():
    """n = 0, or causal with n < s_q: rows with nothing visible give out = 0 and
    lse = -inf; other rows are unaffected."""
    inp = make_inputs(3, 2, 2, [0, 1, 5], seed=19, causal=True)
    out, lse = run(inp)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(out[1, 0] == 0) and np.all(np.isneginf(lse[1, 0]))
    assert np.all(np.isfinite(lse[1, 1])) and np.all(np.isfinite(lse[2]))


def test_scale_enters_lse():
    """lse is computed on scaled scores: doubling the scale with half the query is
    the identical problem."""
    inp = make_inputs(1, 1, 3, [40], seed=20)
    qn, qp, kv = f64(inp)
    a = O.mla_decode_ref(qn, qp, kv, inp.block_table, inp.cache_seqlens, 0.1, False)
    b = O.mla_decode_ref(qn / 2, qp / 2, kv, inp.block_table, inp.cache_seqlens, 0.2, False)
    assert np.max(np.abs(a[0] - b[0])) < 1e-13 and np.max(np.abs(a[1] - b[1])) < 1e-13


# ---------------------------------------------------------------------------
# brute force
# ---------------------------------------------------------------------------
def _scalar_attention(q576, rows, scale):
    scores = []
    for r in rows:
        acc = 0.0
        for d in range(576):
            acc += q576[d] * r[d]
        scores.append(scale * acc)
    m = max(scores)
    z = sum(math.exp(s - m) for s in scores)
    out = [0.0] * 512
    for s, r in zip(scores, rows):
        w = math.exp(s - m) / z
        for d in range(512):
            out[d] += w * r[d]
    return out, m + math.log(z)


@pytest.mark.parametrize("n", [1, 2, 5, 8])
def test_brute_force_scalar(n):
    inp = make_inputs(1, 1, 1, [n], seed=30 + n)
    out, lse = run(inp)
    qn, qp, kv = f64(inp)
    q = list(qn[0, 0, 0]) + list(qp[0, 0, 0])
    rows = [list(kv[inp.block_table[0, t // 64], t % 64]) for t in range(n)]
    o, l = _scalar_attention(q, rows, inp.softmax_scale)
    assert abs(l - lse[0, 0, 0]) < 1e-12
    assert max(abs(a - b) for a, b in zip(o, out[0, 0, 0])) < 1e-12


# ---------------------------------------------------------------------------
# split-KV merge
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_split_combine_equals_unsplit(causal):
    inp = make_inputs(2, 2, 4, [300, 129], seed=21, causal=causal)
    qn, qp, kv = f64(inp)
    ref_o, ref_l = O.mla_decode_ref(qn, qp, kv, inp.block_table, inp.cache_seqlens,
                                    inp.softmax_scale, causal)
    for b in range(2):
        n = int(inp.cache_seqlens[b])
        rows = O.gather_rows(kv, inp.block_table[b], n)
        cuts = [0, 64, 65, 192, n] if n > 192 else [0, 1, 64, n]
        parts = [O.partial_ref(qn[b], qp[b], rows, lo, hi, inp.softmax_scale, causal, n)
                 for lo, hi in zip(cuts[:-1], cuts[1:])]
        o, l = O.lse_combine_ref([p[0] for p in parts], [p[1] for p in parts])
        assert np.max(np.abs(o - ref_o[b])) < 1e-12
        assert np.max(np.abs(l - ref_l[b])) < 1e-12


def test_combine_with_empty_partials():
    """A partial whose range holds no visible key (lse = -inf) contributes nothing."""
    o1 = np.full((1, 2, 512), 3.0)
    l1 = np.array([[0.5, -np.inf]])
    o2 = np.zeros((1, 2, 512))
    l2 = np.array([[-np.inf, -np.inf]])
    o, l = O.lse_combine_ref([o1, o2], [l1, l2])
    assert np.all(o[0, 0] == 3.0) and l[0, 0] == 0.5
    assert np.all(o[0, 1] == 0.0) and np.isneginf(l[0, 1])


def test_combine_two_equal_halves():
    """Two partials with equal lse and outputs a, b merge to (a+b)/2 and lse + ln 2."""
    a = np.random.default_rng(1).standard_normal((1, 1, 512))
    b = np.random.default_rng(2).standard_normal((1, 1, 512))
    o, l = O.lse_combine_ref([a, b], [np.array([[0.3]]), np.array([[0.3]])])
    assert np.max(np.abs(o - (a + b) / 2)) < 1e-15
    assert abs(l[0, 0] - (0.3 + math.log(2))) < 1e-15


def test_flops_and_bytes_closed_form():
    f, by = O.flops_and_bytes(np.array([4096, 4096]), 1, 128, False)
    assert f == 2 * 4096 * 128 * 2 * (576 + 512)
    assert by == 2 * 4096 * 1152
    f2, _ = O.flops_and_bytes(np.array([10]), 2, 1, True)
    assert f2 == (9 + 10) * 2 * 1088
