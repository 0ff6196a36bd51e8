"""mla_decode_noalloc: the decode for callers that cannot allocate device memory (an
engine whose pool already reserved the GPU, a plugin handed only input/output
pointers, a loop that cannot afford cudaMalloc's synchronisation).  It uses the
library's built-in 64 MiB scratch instead of a caller workspace.

Each call goes through the C ABI and is checked two ways: against the float64 oracle
with the tolerance of the other GPU tests, and bit for bit against mla_decode with a
caller workspace on the same inputs (the two run the same kernels and schedule, so any
difference would come from stale scratch contents).  Two different split-KV problems
run back to back, so the second call runs over the scratch the first one left behind.
This file is collected last on purpose."""

import numpy as np
import pytest

from deepseek_mla_decode_b200.workloads import make_inputs
from mla_testlib import to_device, oracle, compare

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import deepseek_mla_decode_b200 as mla  # noqa: E402


def _bits_equal(a, b):
    """Bitwise equality of two tensors (NaN patterns included)."""
    a = a.contiguous().view(torch.int16 if a.dtype == torch.bfloat16 else torch.int32)
    b = b.contiguous().view(torch.int16 if b.dtype == torch.bfloat16 else torch.int32)
    return bool(torch.equal(a, b))


def test_noalloc_matches_oracle_and_decode_twice():
    # two different problems back to back; both need split-KV partials in the scratch
    problems = [
        make_inputs(4, 1, 128, [9000, 130, 4097, 2500], seed=90),
        make_inputs(6, 2, 64, [1, 7000, 333, 64, 5000, 12000], seed=91, causal=True),
    ]
    for inp in problems:
        dev = to_device(inp)
        meta = mla.get_metadata(dev["cache_seqlens"], inp.s_q, inp.H)
        out = torch.empty((inp.B, inp.s_q, inp.H, 512), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((inp.B, inp.s_q, inp.H), dtype=torch.float32, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        mla.decode_noalloc(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"], dev["cache_seqlens"],
                           inp.softmax_scale, inp.causal, meta, out, lse, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert int(meta[7].item()) > inp.B  # the schedule really split sequences
        ref_out, ref_lse = oracle(inp)
        compare(out.float().cpu().double().numpy(), lse.cpu().double().numpy(), ref_out, ref_lse,
                what=f"noalloc B={inp.B} s_q={inp.s_q} H={inp.H}")
        ws_out, ws_lse = mla.decode(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"],
                                    dev["cache_seqlens"], inp.softmax_scale, inp.causal, meta)
        torch.cuda.synchronize()
        assert _bits_equal(out, ws_out) and _bits_equal(lse, ws_lse)


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
