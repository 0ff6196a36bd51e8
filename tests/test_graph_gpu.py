"""The decode step captured in a CUDA graph: mla_get_metadata + mla_decode recorded once
and replayed, as an engine does to launch a step's layers without host overhead.
Replays must equal eager calls bit for bit, and a replay after the lengths changed in
place must follow the new lengths (the schedule is recomputed inside the graph)."""

import numpy as np
import pytest

from deepseek_mla_decode_b200.workloads import make_inputs
from mla_testlib import to_device, oracle, compare

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import deepseek_mla_decode_b200 as mla  # noqa: E402


def test_decode_step_in_cuda_graph():
    lens = [3000, 17, 700, 5000, 1, 2048]
    inp = make_inputs(len(lens), 2, 128, lens, seed=140, causal=True)
    dev = to_device(inp)
    B, s_q, H = inp.B, inp.s_q, inp.H
    meta = torch.empty((mla.metadata_size(B, s_q, H) + 3) // 4, dtype=torch.int32, device="cuda")
    ws = torch.empty(mla.workspace_size(B, s_q, H), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, s_q, H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, s_q, H), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step(stream):
        mla.get_metadata(dev["cache_seqlens"], s_q, H, metadata=meta, stream=stream)
        mla.decode(dev["q_nope"], dev["q_pe"], dev["kv_cache"], dev["block_table"], dev["cache_seqlens"],
                   inp.softmax_scale, True, meta, workspace=ws, out=out, lse=lse, status=status, stream=stream)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step(s)  # eager, also the warm-up before capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    eager_out, eager_lse = out.clone(), lse.clone()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(s)
    out.zero_()
    lse.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(out, eager_out) and torch.equal(lse, eager_lse)

    # new lengths written in place (shorter, so the table still covers them): the
    # replay recomputes the schedule and follows them
    new_lens = np.array([2999, 5, 700, 4000, 1, 100], dtype=np.int32)
    dev["cache_seqlens"].copy_(torch.from_numpy(new_lens))
    g.replay()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    inp.cache_seqlens[:] = new_lens
    ref_out, ref_lse = oracle(inp)
    compare(out.float().cpu().double().numpy(), lse.cpu().double().numpy(), ref_out, ref_lse,
            what="graph replay with new lengths")
