"""The allocation-free decode entry point (nvkv_decode_attn_static).

It exists for callers that cannot allocate device memory where they run
attention (inside a CUDA Graph capture, under a memory pool they do not own,
on paths that must not take allocator locks): instead of a caller workspace
it keeps the split-K partial results in a fixed device array owned by the
library.  This test calls it through the C ABI twice in a row and checks
each result against the workspace entry point (nvkv_decode_attn +
nvkv_combine) on the same inputs, within the attention tolerance the other
tests use.  The file is named to be collected last."""
import pytest
import torch

import nvfp4_quantized_kv_b200 as nv
from nvfp4_quantized_kv_b200 import workload as W
from nvfp4_quantized_kv_b200.harness import DeviceWorkload

from parity_util import ATOL, RTOL

pytestmark = pytest.mark.gpu

CASES = [
    ("tensor_core_path", 3, 24, 4, 256, 2, [1000, 300, 77]),
    ("cuda_core_path", 2, 8, 2, 128, 1, [500, 33]),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_static_scratch_entry_matches_workspace_entry(case):
    name, b, hq, hkv, d, T, ctx = case
    wl = W.small(name, b, hq, hkv, d, T, ctx, seed=31)
    dw = DeviceWorkload(wl)
    dw.fill_context()
    dw.load_step_inputs()
    dw.append()
    dw.attend()  # workspace entry point
    torch.cuda.synchronize()
    ref = dw.out.float().clone()
    for call in range(2):
        out = torch.full_like(dw.out, float("nan"))
        nv.nvkv_decode_attn_static(dw.cache, dw.seqs, dw.q, wl.T, wl.num_q_heads, wl.sm_scale,
                                   0, out)
        torch.cuda.synchronize()
        got = out.float()
        assert torch.isfinite(got).all(), f"call {call}"
        err = (got - ref).abs()
        assert (err <= ATOL + RTOL * ref.abs()).all(), f"call {call}: max err {float(err.max())}"
    assert dw.err_bits() == 0


def test_static_scratch_rejects_oversized_shapes():
    """A shape whose split-K scratch exceeds the fixed array is refused with
    NVKV_ERR_WORKSPACE before anything is launched (q and out are never read,
    so small placeholders suffice)."""
    batch, T, hq, hkv, d = 4096, 16, 96, 12, 256
    need = nv.nvkv_decode_workspace_bytes(batch, T, hq, hkv, d, 0)
    assert need > nv.nvkv_decode_static_scratch_bytes()
    pt = torch.zeros((batch, 1), dtype=torch.int32, device="cuda")
    lens = torch.ones(batch, dtype=torch.int32, device="cuda")
    seqs = nv.Seqs(pt, lens, 1)
    cache = nv.Cache.allocate(2, hkv, d, "cuda")
    q = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.NvkvError) as e:
        nv.nvkv_decode_attn_static(cache, seqs, q, T, hq, 0.1, 0, out)
    assert e.value.status == nv.ERR_WORKSPACE
    torch.cuda.synchronize()
    assert (out == 0).all()
