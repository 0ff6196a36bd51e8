"""mla_decode_noalloc: the decode for callers that cannot allocate device memory (an
engine whose pool already reserved the GPU, a plugin handed only input/output
pointers, a loop that cannot afford cudaMalloc's synchronisation).  It uses the
library's built-in 64 MiB scratch instead of a caller workspace.

Checked through the C ABI against mla_decode (same inputs, the tolerance of the other
GPU tests) on two calls in a row, so the second call runs over the scratch contents
the first one left behind.  This file is collected last on purpose."""

import numpy as np
import pytest

from deepseek_mla_decode_b200.workloads import make_inputs
from mla_testlib import to_device, OUT_MAX_ABS, OUT_MEAN_ABS, LSE_MAX_ABS

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import deepseek_mla_decode_b200 as mla  # noqa: E402


def _close(a_out, a_lse, b_out, b_lse):
    a_out, b_out = a_out.float().cpu().double().numpy(), b_out.float().cpu().double().numpy()
    a_lse, b_lse = a_lse.cpu().double().numpy(), b_lse.cpu().double().numpy()
    ninf = np.isneginf(b_lse)
    assert np.array_equal(np.isneginf(a_lse), ninf)
    err = np.abs(a_out - b_out)
    assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS
    assert np.abs(a_lse[~ninf] - b_lse[~ninf]).max() <= LSE_MAX_ABS


def test_noalloc_matches_decode_twice():
    # two different problems back to back; both need split-KV partials in the scratch
    problems = [
        make_inputs(4, 1, 128, [9000, 130, 4097, 2500], seed=90),
        make_inputs(6, 2, 64, [1, 7000, 333, 64, 5000, 12000], seed=91, causal=True),
    ]
    for inp in problems:
        dev = to_device(inp)
        meta = mla.get_metadata(dev["cache_seqlens"], inp.s_q, inp.H)
        ref_out, ref_lse = mla.decode(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"],
                                      dev["cache_seqlens"], inp.softmax_scale, inp.causal, meta)
        out = torch.empty_like(ref_out)
        lse = torch.empty_like(ref_lse)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        mla.decode_noalloc(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"], dev["cache_seqlens"],
                           inp.softmax_scale, inp.causal, meta, out, lse, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert int(meta[7].item()) > inp.B  # the schedule really split sequences
        _close(out, lse, ref_out, ref_lse)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    inp = make_inputs(256, 1, 128, [64] * 256, seed=92)
    dev = to_device(inp)
    meta = mla.get_metadata(dev["cache_seqlens"], 1, 128)
    out = torch.empty((256, 1, 128, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((256, 1, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(mla.MLAError) as e:
        mla.decode_noalloc(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"], dev["cache_seqlens"],
                           inp.softmax_scale, False, meta, out, lse)
    assert e.value.code == 4
