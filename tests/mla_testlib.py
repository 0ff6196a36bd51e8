"""Helpers shared by the test files: device transfer of seeded inputs, the CUDA path
through the C ABI, and the tolerance check against the float64 oracle."""

from __future__ import annotations

import numpy as np

from oracle import mla_oracle as O
from oracle import mla_fp8_oracle as F

# Tolerances against the float64 oracle (the acceptance bar of this library):
# out max-abs <= 2e-2 and mean-abs <= 2e-3, lse max-abs <= 1e-3.
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3


def to_device(inp):
    import torch

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()

    return dict(
        q_nope=bf16(inp.q_nope),
        q_pe=bf16(inp.q_pe),
        kv_cache=bf16(inp.kv_cache),
        block_table=torch.from_numpy(np.ascontiguousarray(inp.block_table, dtype=np.int32)).cuda(),
        cache_seqlens=torch.from_numpy(np.ascontiguousarray(inp.cache_seqlens, dtype=np.int32)).cuda(),
    )


def run_cuda(inp, dev=None, status=None):
    """mla_get_metadata + mla_decode through the C ABI; returns (out f64, lse f64, meta)."""
    import torch
    import deepseek_mla_decode_b200 as mla

    dev = dev or to_device(inp)
    meta = mla.get_metadata(dev["cache_seqlens"], inp.s_q, inp.H)
    out, lse = mla.decode(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"], dev["cache_seqlens"],
                          inp.softmax_scale, inp.causal, meta, status=status)
    torch.cuda.synchronize()
    return out.float().cpu().double().numpy(), lse.cpu().double().numpy(), meta


def oracle(inp, seqs=None, q_lens=None):
    """Oracle outputs, optionally for a subset of sequences only, optionally with
    per-sequence query counts."""
    qn, qp = O.bf16_to_f64(inp.q_nope), O.bf16_to_f64(inp.q_pe)
    kv = O.bf16_to_f64(inp.kv_cache) if seqs is None else None
    if seqs is None:
        return O.mla_decode_ref(qn, qp, kv, inp.block_table, inp.cache_seqlens, inp.softmax_scale, inp.causal,
                                q_lens=q_lens)
    outs, lses = [], []
    for b in seqs:
        n = int(inp.cache_seqlens[b])
        nblk = (n + 63) // 64
        ids = inp.block_table[b, :nblk]
        kv_b = O.bf16_to_f64(inp.kv_cache[ids])  # only this sequence's blocks
        table = np.arange(max(nblk, 1))[None, :]
        o, l = O.mla_decode_ref(qn[b : b + 1], qp[b : b + 1], kv_b if nblk else np.zeros((1, 64, 576)), table,
                                np.array([n]), inp.softmax_scale, inp.causal,
                                q_lens=None if q_lens is None else np.asarray(q_lens)[b : b + 1])
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.stack(lses)


def run_cuda_fp8(inp, dev=None, status=None, q_lens=None):
    """The FP8 path: mla_quantize_kv_fp8 of the bf16 cache, then mla_get_metadata +
    mla_decode_fp8; returns (out f64, lse f64, meta)."""
    import torch
    import deepseek_mla_decode_b200 as mla

    dev = dev or to_device(inp)
    kv8 = mla.quantize_kv_fp8(dev["kv_cache"])
    meta = mla.get_metadata(dev["cache_seqlens"], inp.s_q, inp.H)
    ql = None if q_lens is None else torch.tensor(np.asarray(q_lens, dtype=np.int32)).cuda()
    out, lse = mla.decode_fp8(dev["q_nope"], dev["q_pe"], kv8, dev["block_table"], dev["cache_seqlens"],
                              inp.softmax_scale, inp.causal, meta, q_lens=ql, status=status)
    torch.cuda.synchronize()
    return out.float().cpu().double().numpy(), lse.cpu().double().numpy(), meta


def oracle_fp8(inp, seqs=None, q_lens=None):
    """FP8 oracle: the oracle's own quantiser packs the bf16 cache, then the decode
    over the dequantised rows; per sequence (its blocks only) when seqs is given."""
    qn, qp = O.bf16_to_f64(inp.q_nope), O.bf16_to_f64(inp.q_pe)
    if seqs is None:
        return F.mla_decode_fp8_ref(qn, qp, F.pack_cache(inp.kv_cache), inp.block_table, inp.cache_seqlens,
                                    inp.softmax_scale, inp.causal, q_lens=q_lens)
    outs, lses = [], []
    for b in seqs:
        n = int(inp.cache_seqlens[b])
        nblk = (n + 63) // 64
        ids = inp.block_table[b, :nblk]
        packed = F.pack_cache(inp.kv_cache[ids]) if nblk else np.zeros((1, 64, F.ROW_BYTES), np.uint8)
        table = np.arange(max(nblk, 1))[None, :]
        o, l = F.mla_decode_fp8_ref(qn[b : b + 1], qp[b : b + 1], packed, table, np.array([n]), inp.softmax_scale,
                                    inp.causal, q_lens=None if q_lens is None else np.asarray(q_lens)[b : b + 1])
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.stack(lses)


def compare(out, lse, ref_out, ref_lse, what=""):
    """Assert the tolerance bar; -inf lse rows must match exactly (and out = 0 there)."""
    ninf = np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(lse), ninf), f"{what}: -inf rows differ"
    assert np.all(np.isfinite(lse[~ninf])), f"{what}: non-finite lse"
    assert np.all(out[ninf] == 0), f"{what}: rows without visible keys must be 0"
    err = np.abs(out - ref_out)
    lerr = np.abs(lse[~ninf] - ref_lse[~ninf]) if (~ninf).any() else np.zeros(1)
    stats = dict(out_max=float(err.max()), out_mean=float(err.mean()), lse_max=float(lerr.max()))
    assert stats["out_max"] <= OUT_MAX_ABS, f"{what}: {stats}"
    assert stats["out_mean"] <= OUT_MEAN_ABS, f"{what}: {stats}"
    assert stats["lse_max"] <= LSE_MAX_ABS, f"{what}: {stats}"
    return stats
