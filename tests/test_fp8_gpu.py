"""GPU parity of the FP8 latent-cache path against the FP8 oracle.

mla_quantize_kv_fp8 must reproduce the oracle's packed rows byte for byte: the scale,
the e4m3 codes and the scaled bf16 k_pe are decided in fp32 on both sides (IEEE
division, round to nearest even)."""

import numpy as np
import pytest

from oracle import mla_fp8_oracle as F
from deepseek_mla_decode_b200.workloads import make_inputs, f32_to_bf16_bits

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import deepseek_mla_decode_b200 as mla  # noqa: E402


def bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("lens,seed", [([37, 130], 1), ([4096] * 3, 2), ([1, 64, 65, 2000], 3)])
def test_quantize_matches_oracle_bit_exact(lens, seed):
    inp = make_inputs(len(lens), 1, 16, lens, seed=seed)
    kv = inp.kv_cache.copy()
    kv[0, 0, :] = 0                                             # a zero row: scale 0, all zeros
    kv[0, 1, :] = f32_to_bf16_bits(np.full(576, -3.0, np.float32))  # constant row: codes -448, k_pe' -448
    kv[0, 2, 512:] = f32_to_bf16_bits(np.full(64, 40.0, np.float32))  # k_pe sets the row's scale
    kv[0, 3, :512] = 0                                          # only k_pe non-zero: codes 0
    got = mla.quantize_kv_fp8(bf16(kv)).cpu().numpy()
    ref = F.pack_cache(kv)
    assert got.shape == ref.shape
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} bytes differ, first at {bad[:5].tolist()}: got {got[tuple(bad[0])]} ref {ref[tuple(bad[0])]}"
