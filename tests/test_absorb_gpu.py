"""GPU parity of the weight-absorption GEMMs (mla_absorb_q, mla_absorb_out) against
the float64 oracle, element by element.  Both accumulate in fp32 and round once to
bf16, so every element must satisfy |gpu - ref| <= 2^-8 |ref| + 1e-4 (half a bf16
ulp is 2^-9 relative; the rest covers fp32 accumulation over 128 or 512 terms)."""

import numpy as np
import pytest

from oracle import mla_oracle as O
from deepseek_mla_decode_b200.workloads import make_rows, make_up_projections

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import deepseek_mla_decode_b200 as mla  # noqa: E402


def bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def check_close(gpu, ref, what):
    err = np.abs(gpu - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-4
    worst = float((err / bound).max())
    assert worst <= 1.0, f"{what}: max err {err.max():.3e}, worst err/bound {worst:.3f}"
    return float(err.max())


@pytest.mark.parametrize("B,s_q,H", [(3, 2, 16), (130, 1, 8), (256, 1, 128), (128, 2, 128), (1, 1, 1)])
def test_absorb_q_and_out_match_oracle(B, s_q, H):
    w_uk, w_uv = make_up_projections(H, seed=300 + H)
    q = make_rows((B, s_q, H, 128), seed=301 + B)
    o = make_rows((B, s_q, H, 512), seed=302 + B)
    q_nope = mla.absorb_q(bf16(q), bf16(w_uk))
    y = mla.absorb_out(bf16(o), bf16(w_uv))
    torch.cuda.synchronize()
    ref_q = O.absorb_q_ref(O.bf16_to_f64(q), O.bf16_to_f64(w_uk))
    ref_y = O.absorb_out_ref(O.bf16_to_f64(o), O.bf16_to_f64(w_uv))
    check_close(q_nope.float().cpu().double().numpy(), ref_q, f"absorb_q B={B} s_q={s_q} H={H}")
    check_close(y.float().cpu().double().numpy(), ref_y, f"absorb_out B={B} s_q={s_q} H={H}")


def test_absorb_argument_errors():
    w_uk, _ = make_up_projections(2, seed=1)
    q = bf16(make_rows((2, 1, 2, 128), seed=2))
    with pytest.raises(ValueError):
        mla.absorb_q(q, bf16(w_uk)[:1])
    L = mla.load_library()
    assert L.mla_absorb_q(None, None, None, 1, 1, None) == 1
    assert L.mla_absorb_out(q.data_ptr(), q.data_ptr(), q.data_ptr(), 0, 2, None) == 1
