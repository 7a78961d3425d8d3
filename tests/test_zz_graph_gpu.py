"""A decode step (quantise-append + split-K attention + combine) captured once
in a CUDA Graph and replayed, as batched decode is served by the engine the
"knoopx/ninfer" README describes ("Capabilities and limits": decode replayed
from CUDA Graphs).  Every call only enqueues kernels and the split plan is
computed on the device from kv_lens, so one captured graph serves later
steps whose inputs change in place: a replay must equal a direct step on
the same state, bit for bit, before and after new rows, queries and
lengths are written into the captured buffers."""
import numpy as np
import pytest
import torch

import nvfp4_quantized_kv_b200 as nv
from nvfp4_quantized_kv_b200 import workload as W
from nvfp4_quantized_kv_b200.harness import DeviceWorkload, bf16_tensor

pytestmark = pytest.mark.gpu

CASES = [
    # name, batch, hq, hkv, d, T, ctx (the next position stays inside the last page)
    ("graph_tensor_core", 3, 24, 4, 256, 1, [1000, 300, 70]),
    ("graph_cuda_core", 2, 8, 2, 128, 2, [500, 33]),
    ("graph_mtp", 2, 24, 4, 256, 4, [600, 90]),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_replay_equals_direct_step(case):
    name, b, hq, hkv, d, T, ctx = case
    wl = W.small(name, b, hq, hkv, d, T, ctx, seed=41)
    dw = DeviceWorkload(wl)
    dw.fill_context()
    dw.load_step_inputs()
    # a host bound that leaves room for one more step in the last pages
    dw.seqs = nv.Seqs(dw.page_table, dw.kv_lens, dw.page_table.shape[1] * 16, dw.err)
    for _ in range(2):
        dw.step()
    torch.cuda.synchronize()
    direct0 = dw.out.clone()

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        dw.step()
    dw.out.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(dw.out, direct0)

    # the next step: one more position per sequence, new rows and queries,
    # written into the captured buffers
    rng = np.random.default_rng(5)
    last = wl.kv_lens + 1
    pages = dw.page_table.cpu().numpy()
    assert all(pages[i, (int(last[i]) - 1) // 16] >= 0 for i in range(b))
    dw.kv_lens.copy_(torch.from_numpy(last.astype(np.int32)))
    for t in (dw.k_new, dw.v_new, dw.q):
        t.copy_(bf16_tensor(W.to_bf16_bits(rng.standard_normal(tuple(t.shape)).astype(np.float32)),
                            t.device))
    graph.replay()
    torch.cuda.synchronize()
    replayed = dw.out.clone()
    dw.step()  # the same state, direct launches (re-appends the same rows)
    torch.cuda.synchronize()
    assert torch.equal(replayed, dw.out)
    assert not torch.equal(replayed, direct0)
    assert torch.isfinite(replayed.float()).all()
    assert dw.err_bits() == 0
    del graph
