"""The allocation-free decode entry point (nvkv_decode_attn_static).

It exists for callers that cannot call cudaMalloc or any other allocator
where they run attention (device memory owned by a pool they may not draw
from, plugins inside an application that owns all device memory, paths that
must not take allocator locks): instead of a caller workspace it keeps the
split-K partial results in a fixed device array owned by the library.

These tests call it through the C ABI.  Before the checked calls, a call of
a different shape (more sequences, another T, another split count) leaves
different partial results in the shared array, so a merge that read a slot
the current call did not write would see wrong values.  Then two calls in a
row are each checked against the workspace entry point (nvkv_decode_attn +
nvkv_combine) on the same inputs and against the float64 oracle, within the
attention tolerance the other tests use.  The file is named to be collected
last."""
import pytest
import torch

import nvfp4_quantized_kv_b200 as nv
from nvfp4_quantized_kv_b200 import workload as W
from nvfp4_quantized_kv_b200.harness import DeviceWorkload

from parity_util import ATOL, RTOL, all_rows, assert_close, gpu_rows, oracle_outputs

pytestmark = pytest.mark.gpu

CASES = [
    ("tensor_core_path", 3, 24, 4, 256, 2, [1000, 300, 77]),
    ("cuda_core_path", 2, 8, 2, 128, 1, [500, 33]),
]


def _dirty_the_scratch(d):
    """A call of another shape through the static entry point."""
    wl = W.small("dirty", 5, 24, 4, d, 3, [2000, 900, 40, 1300, 7], seed=77)
    dw = DeviceWorkload(wl)
    dw.fill_context()
    dw.load_step_inputs()
    dw.append()
    out = torch.empty_like(dw.out)
    nv.nvkv_decode_attn_static(dw.cache, dw.seqs, dw.q, wl.T, wl.num_q_heads, wl.sm_scale, 57,
                               out)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_static_scratch_entry_matches_workspace_entry_and_oracle(case):
    name, b, hq, hkv, d, T, ctx = case
    _dirty_the_scratch(d)
    wl = W.small(name, b, hq, hkv, d, T, ctx, seed=31)
    dw = DeviceWorkload(wl)
    dw.fill_context()
    dw.load_step_inputs()
    dw.append()
    dw.attend()  # workspace entry point
    torch.cuda.synchronize()
    ref = dw.out.float().clone()
    rows = all_rows(wl)
    want = oracle_outputs(wl, rows)
    for call in range(2):
        out = torch.full_like(dw.out, float("nan"))
        nv.nvkv_decode_attn_static(dw.cache, dw.seqs, dw.q, wl.T, wl.num_q_heads, wl.sm_scale,
                                   0, out)
        torch.cuda.synchronize()
        got = out.float()
        assert torch.isfinite(got).all(), f"call {call}"
        err = (got - ref).abs()
        assert (err <= ATOL + RTOL * ref.abs()).all(), f"call {call}: max err {float(err.max())}"
        assert_close(gpu_rows(out, wl, rows), want, f"{name} call {call}")
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


def test_static_scratch_rejects_a_misaligned_output_before_launching():
    """A misaligned out is refused with NVKV_ERR_INVALID_ARG up front: the
    device error word, which the partials kernel would report a bad page id
    into, stays clear."""
    dev = torch.device("cuda")
    hkv, hq, d = 2, 4, 128
    cache = nv.Cache.allocate(2, hkv, d, dev, fill=0)
    pt = torch.tensor([[0, 9]], dtype=torch.int32, device=dev)  # page 9 does not exist
    lens = torch.tensor([20], dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    seqs = nv.Seqs(pt, lens, 20, err)
    q = torch.zeros((1, hq, d), dtype=torch.bfloat16, device=dev)
    buf = torch.zeros(hq * d + 8, dtype=torch.bfloat16, device=dev)
    out = buf[1:1 + hq * d]  # 2 bytes past a 16-byte boundary
    with pytest.raises(nv.NvkvError) as e:
        nv.nvkv_decode_attn_static(cache, seqs, q, 1, hq, 0.1, 2, out)
    assert e.value.status == nv.ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert int(err.item()) == 0
