"""GPU parity of chunked-prefill attention (nvkv_prefill_attn and the
key-split nvkv_prefill_attn_split) against the float64 oracle: a chunk of new
queries, appended first, attends causally to the whole cache of its
sequence.  head_dim 256 runs on the tensor-core kernel, head_dim 128 on the
CUDA-core kernel; NVKV_DECODE_KERNEL=simt forces the latter for
cross-checks."""
import zlib

import numpy as np
import pytest
import torch

from nvfp4_quantized_kv_b200 import workload as W
from nvfp4_quantized_kv_b200.harness import DeviceWorkload

from parity_util import (ATOL, RTOL, all_rows, assert_close, gpu_rows, oracle_outputs,
                         oracle_outputs_dense, prefill_sample_queries, sample_rows)

pytestmark = pytest.mark.gpu

SMALL = [
    # name, batch, hq, hkv, d, chunk, ctx
    ("chunk_from_empty", 1, 8, 2, 128, 64, [0]),
    ("chunk_ragged", 2, 24, 4, 256, 37, [300, 5]),
    ("chunk_long", 1, 12, 2, 256, 200, [1500]),
    ("chunk_tiny_tail", 3, 24, 4, 256, 1, [0, 63, 64]),
    ("chunk_mtiles", 1, 24, 4, 256, 90, [700]),
]


def run(wl, prefill_splits=None):
    dw = DeviceWorkload(wl, prefill_splits=prefill_splits)
    dw.fill_context()
    dw.load_step_inputs()
    dw.step()
    torch.cuda.synchronize()
    assert dw.err_bits() == 0
    return dw


def seed_of(name):
    return zlib.crc32(name.encode()) % 1000


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_prefill_small(case):
    name, b, hq, hkv, d, T, ctx = case
    wl = W.small(name, b, hq, hkv, d, T, ctx, mode="prefill", seed=seed_of(name))
    dw = run(wl)
    rows = all_rows(wl) if len(all_rows(wl)) <= 2500 else sample_rows(wl, 400, seed=3)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs(wl, rows), name)


@pytest.mark.parametrize("case", [c for c in SMALL if c[4] == 256], ids=[c[0] for c in SMALL if c[4] == 256])
def test_prefill_kernels_agree(case, monkeypatch):
    name, b, hq, hkv, d, T, ctx = case
    wl = W.small(name, b, hq, hkv, d, T, ctx, mode="prefill", seed=seed_of(name) + 1)
    rows = sample_rows(wl, 200, seed=4)
    ref = oracle_outputs(wl, rows)
    for kernel in ("default", "simt"):
        if kernel == "simt":
            monkeypatch.setenv("NVKV_DECODE_KERNEL", "simt")
        dw = run(wl)
        assert_close(gpu_rows(dw.out, wl, rows), ref, f"{name}/{kernel}")


@pytest.mark.parametrize("splits", [None, 0], ids=["unsplit", "auto_split"])
def test_chunked_prefill_config_sampled(splits):
    """65536 cached tokens + a 2048-token chunk, 24/4 heads, head_dim 256:
    the first 64, the last 64 and every 31st chunk query, all heads; through
    nvkv_prefill_attn and through the key-split call with the automatic
    count (the launch the benchmark times: 5 splits on 148 SMs)."""
    import nvfp4_quantized_kv_b200 as nv
    wl = W.chunked_prefill()
    dw = run(wl, prefill_splits=splits)
    if splits == 0:
        S = nv.nvkv_prefill_num_splits(dw.cache, wl.batch, wl.T, wl.num_q_heads)
        assert 1 <= S <= 8
        if torch.cuda.get_device_properties(0).multi_processor_count == 148:
            assert S == 5
    rows = [(0, t, hq) for t in prefill_sample_queries(wl.T) for hq in range(wl.num_q_heads)]
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs_dense(wl, rows), wl.name)


def test_prefill_tail_matches_decode_verify():
    """The last T positions of a prefill chunk are an MTP-verify block: both
    entry points must agree on the same cache and queries."""
    ctx, T = 1000, 6
    wp = W.small("tail", 2, 24, 4, 256, T, [ctx, 333], mode="prefill", seed=9)
    wd = W.small("tail", 2, 24, 4, 256, T, [ctx, 333], mode="decode", seed=9)
    a = run(wp).out.float()
    b = run(wd).out.float()
    assert ((a - b).abs() <= 2 * (ATOL + RTOL * b.abs())).all()


@pytest.mark.parametrize("kernel", ["default", "simt"])
def test_prefill_reports_bad_page(kernel, monkeypatch):
    """A page id outside the pool is reported through the error word; its
    keys read as absent and nothing outside the pool is touched."""
    import nvfp4_quantized_kv_b200 as nv
    if kernel == "simt":
        monkeypatch.setenv("NVKV_DECODE_KERNEL", "simt")
    dev = torch.device("cuda")
    hkv, hq, d, n = 2, 12, 256, 20
    cache = nv.Cache.allocate(2, hkv, d, dev, fill=0)
    pt = torch.tensor([[0, 9]], dtype=torch.int32, device=dev)  # page 9 does not exist
    lens = torch.tensor([n], dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    seqs = nv.Seqs(pt, lens, n, err)
    q = torch.zeros((n, hq, d), dtype=torch.bfloat16, device=dev)
    cu = torch.tensor([0, n], dtype=torch.int32, device=dev)
    out = torch.empty((n, hq, d), dtype=torch.bfloat16, device=dev)
    nv.nvkv_prefill_attn(cache, seqs, q, cu, n, n, hq, 0.0625, out)
    torch.cuda.synchronize()
    assert int(err.item()) & nv.DEVERR_PAGE_ID
    assert torch.isfinite(out.float()).all()
    assert (out == 0).all()  # an all-zero pool dequantises to 0


SPLIT_CASES = [c for c in SMALL if c[4] == 256]


@pytest.mark.parametrize("splits", [2, 3, 5, 8])
@pytest.mark.parametrize("case", SPLIT_CASES, ids=[c[0] for c in SPLIT_CASES])
def test_prefill_split_small(case, splits):
    """Every key-split count on the small chunks: ragged chunks, several
    m-tiles, and chunks with fewer 64-key tiles than splits (empty splits
    leave lse = -inf, which the merge skips)."""
    name, b, hq, hkv, d, T, ctx = case
    wl = W.small(name, b, hq, hkv, d, T, ctx, mode="prefill", seed=seed_of(name))
    dw = run(wl, prefill_splits=splits)
    rows = all_rows(wl) if len(all_rows(wl)) <= 2500 else sample_rows(wl, 400, seed=3)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs(wl, rows), f"{name}/S{splits}")


@pytest.mark.parametrize("mode", ["default", "split", "simt"])
def test_prefill_chunk_past_total_q_writes_no_row_beyond(mode, monkeypatch):
    """cu_q claims 20 rows but total_q is 12: nothing is written past row 12
    of out (the tensor-core kernels also report the sequence with
    NVKV_DEVERR_LENGTH and leave its rows alone)."""
    import nvfp4_quantized_kv_b200 as nv
    if mode == "simt":
        monkeypatch.setenv("NVKV_DECODE_KERNEL", "simt")
    dev = torch.device("cuda")
    hkv, hq, d, n, total_q = 2, 12, 256, 20, 12
    cache = nv.Cache.allocate(2, hkv, d, dev, fill=0)
    pt = torch.tensor([[0, 1]], dtype=torch.int32, device=dev)
    lens = torch.tensor([n], dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    seqs = nv.Seqs(pt, lens, n, err)
    q = torch.zeros((n, hq, d), dtype=torch.bfloat16, device=dev)
    cu = torch.tensor([0, n], dtype=torch.int32, device=dev)
    out_full = torch.full((n, hq, d), 7.0, dtype=torch.bfloat16, device=dev)
    out = out_full[:total_q]
    if mode == "split":
        ws = torch.empty(nv.nvkv_prefill_workspace_bytes(total_q, hq, d, 2), dtype=torch.uint8,
                         device=dev)
        nv.nvkv_prefill_attn_split(cache, seqs, q, cu, total_q, n, hq, 0.0625, 2, ws, out)
    else:
        nv.nvkv_prefill_attn(cache, seqs, q, cu, total_q, n, hq, 0.0625, out)
    torch.cuda.synchronize()
    assert (out_full[total_q:].float() == 7.0).all()
    if mode != "simt":
        assert int(err.item()) & nv.DEVERR_LENGTH
