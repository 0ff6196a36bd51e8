"""GPU parity of the quantised causal prefill attention (mla_sage_*) against the
oracle in oracle/sage_oracle.py.

The INT8 / e4m3 codes and their scales are decided in fp32 on both sides (IEEE
division, nearest even) and must match byte for byte.  The attention itself follows
the oracle's steps in fp32 with ex2.approx, so a weight whose P * 448 lies within
rounding distance of an e4m3 midpoint may land one code apart; tolerances: out
max-abs <= 2e-2 and mean-abs <= 2e-3 (bf16 output), lse max-abs <= 1e-3."""

import numpy as np
import pytest

from oracle import sage_oracle as SA
from oracle import mla_fp8_oracle as F
from deepseek_mla_decode_b200.workloads import f32_to_bf16_bits

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import deepseek_mla_decode_b200 as mla  # noqa: E402


def make(S, H, seed, kscale=1.0):
    rng = np.random.default_rng(seed)
    q = f32_to_bf16_bits(rng.standard_normal((S, H, 192)).astype(np.float32))
    k = f32_to_bf16_bits((rng.standard_normal((S, H, 192)) * kscale).astype(np.float32))
    v = f32_to_bf16_bits(rng.standard_normal((S, H, 128)).astype(np.float32))
    return q, k, v


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def workspace_views(ws, S, H):
    """Split the workspace as documented in include/mla_decode.h."""
    sp = (S + 127) // 128 * 128
    b = ws.cpu().numpy()
    o = 0
    q8 = b[o:o + H * sp * 192].view(np.int8).reshape(H, sp, 192); o += H * sp * 192
    k8 = b[o:o + H * sp * 192].view(np.int8).reshape(H, sp, 192); o += H * sp * 192
    vt8 = b[o:o + H * 128 * sp].reshape(H, 128, sp); o += H * 128 * sp
    sq = b[o:o + 4 * H * sp].view(np.float32).reshape(H, sp); o += 4 * H * sp
    sk = b[o:o + 4 * H * sp].view(np.float32).reshape(H, sp); o += 4 * H * sp
    sv = b[o:o + 4 * H * 128].view(np.float32).reshape(H, 128)
    return q8, k8, vt8, sq, sk, sv, sp


@pytest.mark.parametrize("S,H", [(1, 1), (130, 2), (1000, 3)])
def test_quantizers_match_oracle_bit_exact(S, H):
    q, k, v = make(S, H, seed=10 + S)
    ws = mla.sage_quantize(dev(q), dev(k), dev(v))
    torch.cuda.synchronize()
    q8, k8, vt8, sq, sk, sv, sp = workspace_views(ws, S, H)
    for codes, scale, x in ((q8, sq, q), (k8, sk, k)):
        rc, rs = SA.quantize_int8_rows(F.O.bf16_to_f64(x).astype(np.float32))  # [S, H, 192], [S, H]
        assert np.array_equal(codes[:, :S], rc.transpose(1, 0, 2))
        assert np.array_equal(scale[:, :S], rs.T)
        assert np.all(codes[:, S:] == 0) and np.all(scale[:, S:] == 0)
    rv, rsv = SA.quantize_v_channels(F.O.bf16_to_f64(v).astype(np.float32))  # [S, H, 128], [H, 128]
    assert np.array_equal(vt8[:, :, :S], rv.transpose(1, 2, 0))
    assert np.all(vt8[:, :, S:] == 0)
    assert np.array_equal(sv, rsv)


def run(q, k, v, S, H, status=None):
    out, lse = mla.sage_prefill(dev(q), dev(k), dev(v), SA.SCALE_192, status=status)
    torch.cuda.synchronize()
    return out.float().cpu().double().numpy(), lse.cpu().double().numpy()


def check(S, H, seed, kscale=1.0):
    q, k, v = make(S, H, seed, kscale)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = run(q, k, v, S, H, status)
    assert int(status.item()) == 0
    ref, ref_lse = SA.sage_prefill_ref(q, k, v)
    err = np.abs(out - ref)
    stats = dict(out_max=float(err.max()), out_mean=float(err.mean()), lse_max=float(np.abs(lse - ref_lse).max()))
    assert stats["out_max"] <= 2e-2 and stats["out_mean"] <= 2e-3 and stats["lse_max"] <= 1e-3, stats
    return stats


@pytest.mark.parametrize("S,H", [(1, 1), (2, 1), (127, 2), (128, 1), (129, 2), (300, 3), (1000, 2)])
def test_prefill_matches_oracle(S, H):
    check(S, H, seed=20 + S + H)


def test_prefill_long_sequence():
    print(check(4096, 2, seed=31))


def test_prefill_peaked_scores():
    # larger keys: sharper softmax rows, the running maximum moves across many blocks
    check(700, 2, seed=32, kscale=4.0)


def test_prefill_equal_logits_rows_are_means():
    # identical key rows: every visible weight is coded 448, the output is the mean of
    # the visible dequantised value rows (the oracle's closed-form pin, on the GPU)
    S, H = 300, 2
    q, k, v = make(S, H, seed=33)
    k[:] = k[:1]
    out, lse = run(q, k, v, S, H)
    vh = SA.quantize_v_channels(F.O.bf16_to_f64(v).astype(np.float32))
    vhat = F.e4m3_decode(vh[0]) * vh[1][None].astype(np.float64)
    mean = np.cumsum(vhat, axis=0) / np.arange(1, S + 1)[:, None, None]
    assert np.max(np.abs(out - mean)) <= 1e-2 * max(1.0, np.abs(mean).max())


def test_prefill_deterministic():
    q, k, v = make(777, 2, seed=34)
    a = run(q, k, v, 777, 2)
    b = run(q, k, v, 777, 2)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_sage_host_argument_errors():
    L = mla.load_library()
    import ctypes

    n = ctypes.c_size_t()
    assert L.mla_sage_workspace_size(0, 1, ctypes.byref(n)) != 0
    assert L.mla_sage_workspace_size(10, 0, ctypes.byref(n)) != 0
    assert L.mla_sage_workspace_size(10, 2, ctypes.byref(n)) == 0
    ws = torch.empty(n.value, dtype=torch.uint8, device="cuda")
    out = torch.empty((10, 2, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((10, 2), dtype=torch.float32, device="cuda")
    # too small a workspace, a null output, a non-positive scale
    assert L.mla_sage_attention(10, 2, 0.1, ws.data_ptr(), n.value - 1, out.data_ptr(), lse.data_ptr(), None, None) != 0
    assert L.mla_sage_attention(10, 2, 0.1, ws.data_ptr(), n.value, None, lse.data_ptr(), None, None) != 0
    assert L.mla_sage_attention(10, 2, -1.0, ws.data_ptr(), n.value, out.data_ptr(), lse.data_ptr(), None, None) != 0


def test_prefill_full_size_sampled_rows():
    # the bench's configuration (64K tokens, 16 heads): rows sampled across the whole
    # sequence (first and last rows, block and tile-pair edges, random interior rows)
    # against the oracle, which computes each sampled row on its own
    from deepseek_mla_decode_b200.workloads import make_prefill, PREFILL_S, PREFILL_H

    S, H = PREFILL_S, PREFILL_H
    q, k, v = make_prefill(S, H, seed=41)
    out, lse = mla.sage_prefill(dev(q), dev(k), dev(v), SA.SCALE_192)
    torch.cuda.synchronize()
    rng = np.random.default_rng(42)
    rows = sorted(set([0, 1, 127, 128, 255, 256, 257, 4095, 32767, 32768, S - 129, S - 128, S - 2, S - 1]
                      + rng.integers(0, S, 34).tolist()))
    ref, ref_lse = SA.sage_prefill_ref(q, k, v, rows=rows)
    got = out[rows].float().cpu().double().numpy()
    got_lse = lse[rows].cpu().double().numpy()
    err = np.abs(got - ref)
    stats = dict(out_max=float(err.max()), out_mean=float(err.mean()),
                 lse_max=float(np.abs(got_lse - ref_lse).max()))
    assert stats["out_max"] <= 2e-2 and stats["out_mean"] <= 2e-3 and stats["lse_max"] <= 1e-3, stats
    print(stats)
