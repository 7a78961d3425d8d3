"""GPU parity of the K8V4 cache (K rows of E4M3 bytes with one fp32 scale per
row, V in NVFP4): the pool bytes written by nvkv_append_k8v4 against the
oracle's K8V4 pool image bit for bit, and decode / MTP-verify / chunked
prefill attention over that cache against the float64 oracle with K in the
same 8-bit format (tolerance |err| <= 8e-3 + 8e-3 |ref|, parity_util)."""
import zlib

import numpy as np
import pytest
import torch

import oracle
import nvfp4_quantized_kv_b200 as nv
from nvfp4_quantized_kv_b200 import workload as W
from nvfp4_quantized_kv_b200.harness import DeviceWorkload, bf16_tensor
from nvfp4_quantized_kv_b200.workload import to_bf16_bits

from parity_util import all_rows, assert_close, gpu_rows, oracle_outputs, sample_rows

pytestmark = pytest.mark.gpu
SENTINEL = 0xA5


def k_rows(rng, shape):
    """K rows whose magnitudes span six decades, with a few outlier channels
    that set each row's scale."""
    n, hkv, d = shape
    x = rng.standard_normal(shape) * 10.0 ** rng.uniform(-3, 3, size=(n, hkv, 1))
    x[..., rng.integers(d, size=4)] *= 20
    return to_bf16_bits(x.astype(np.float32))


def run_appends(hkv, d, page_table, calls, num_pages):
    """calls: list of (kv_lens after the call, k rows, v rows, cu) in order.
    Runs them through nvkv_append_k8v4 and the oracle; returns both images."""
    dev = torch.device("cuda")
    pb = nv.nvkv_k8v4_page_bytes(hkv, d)
    assert pb == oracle.k8v4_page_bytes(hkv, d)
    cache = nv.Cache.allocate(num_pages, hkv, d, dev, fill=SENTINEL, kv_format="k8v4")
    ref = np.full(num_pages * pb, SENTINEL, np.uint8)
    pt = torch.from_numpy(page_table).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for lens, k, v, cu in calls:
        seqs = nv.Seqs(pt, torch.from_numpy(lens).to(dev), int(lens.max()), err)
        counts = np.diff(cu)
        nv.nvkv_append_k8v4(cache, seqs, bf16_tensor(k, dev), bf16_tensor(v, dev),
                            torch.from_numpy(cu).to(dev), int(cu[-1]), int(counts.max()))
        oracle.append_k8v4(ref, hkv, d, page_table, lens, k, v, cu)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return cache.pool.cpu().numpy(), ref


@pytest.mark.parametrize("hkv,d,batch,seed", [(2, 128, 1, 0), (4, 256, 3, 1), (1, 256, 5, 2),
                                              (3, 128, 4, 3)])
def test_append_k8v4_matches_oracle(hkv, d, batch, seed):
    rng = np.random.default_rng(100 + seed)
    maxp = 12
    num_pages = batch * maxp + 5
    page_table = rng.permutation(num_pages)[: batch * maxp].reshape(batch, maxp).astype(np.int32)
    lens = np.zeros(batch, np.int32)
    calls = []
    for step in range(6):
        counts = rng.integers(0, 40, size=batch).astype(np.int32)
        if step == 5:
            counts[:] = 1
        counts = np.minimum(counts, maxp * 16 - lens)
        lens = lens + counts
        cu = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        n = int(cu[-1])
        calls.append((lens.copy(), k_rows(rng, (n, hkv, d)),
                      to_bf16_bits(rng.standard_normal((n, hkv, d)).astype(np.float32)), cu))
    got, ref = run_appends(hkv, d, page_table, calls, num_pages)
    assert np.array_equal(got, ref), f"{(got != ref).sum()} bytes differ"


def test_append_k8v4_special_rows():
    """All-zero rows (scale 0, codes 0), a negative element that rounds to
    zero (stored as +0), rows of bf16 subnormals (a subnormal fp32 scale),
    rows near the bf16 maximum, and a row whose maximum is negative."""
    hkv, d = 2, 128
    rng = np.random.default_rng(7)
    n = 8
    x = np.zeros((n, hkv, d), np.float32)
    x[1, :, 5] = 1.0
    x[1, :, 6] = -1e-30
    x[3] = rng.standard_normal((hkv, d)).astype(np.float32) * 3e37
    x[4] = -np.abs(rng.standard_normal((hkv, d)).astype(np.float32))
    x[4, :, 9] = -50.0
    x[5] = rng.standard_normal((hkv, d)).astype(np.float32) * 1e-3
    k = to_bf16_bits(x)
    # row 2: bf16 subnormals (bit patterns 0x0001 .. 0x007f with random signs)
    sub = rng.integers(1, 0x80, size=(hkv, d)).astype(np.uint16)
    k[2] = sub | np.where(rng.random((hkv, d)) < 0.5, 0x8000, 0).astype(np.uint16)
    k[6] = sub  # all positive
    v = to_bf16_bits(rng.standard_normal((n, hkv, d)).astype(np.float32))
    page_table = np.array([[2, 0]], np.int32)
    lens = np.array([n], np.int32)
    cu = np.array([0, n], np.int32)
    got, ref = run_appends(hkv, d, page_table, [(lens, k, v, cu)], 3)
    assert np.array_equal(got, ref), f"{(got != ref).sum()} bytes differ"
    pb = nv.nvkv_k8v4_page_bytes(hkv, d)
    blk = got[2 * pb: 2 * pb + 25 * d + 64]  # page 2, kv-head 0
    assert (blk[0:d] == 0).all()                                            # zero row: codes
    assert blk[16 * d: 16 * d + 4].view(np.float32)[0] == 0                 # and its scale
    assert blk[d + 5] == 0x7E and blk[d + 6] == 0x00                        # 448 and +0


def test_k8v4_v_regions_equal_the_nvfp4_cache():
    """V is stored identically in both formats: appending the same rows to an
    NVFP4 cache and a K8V4 cache gives the same V code and V scale bytes."""
    dev = torch.device("cuda")
    rng = np.random.default_rng(8)
    hkv, d, n = 3, 256, 37
    k = k_rows(rng, (n, hkv, d))
    v = to_bf16_bits(rng.standard_normal((n, hkv, d)).astype(np.float32))
    pt = torch.tensor([[1, 0, 2]], dtype=torch.int32, device=dev)
    lens = torch.tensor([n], dtype=torch.int32, device=dev)
    cu = torch.tensor([0, n], dtype=torch.int32, device=dev)
    seqs = nv.Seqs(pt, lens, n)
    a = nv.Cache.allocate(3, hkv, d, dev, fill=0)
    b = nv.Cache.allocate(3, hkv, d, dev, fill=0, kv_format="k8v4")
    nv.nvkv_append(a, seqs, bf16_tensor(k, dev), bf16_tensor(v, dev), cu, n, n)
    nv.nvkv_append_k8v4(b, seqs, bf16_tensor(k, dev), bf16_tensor(v, dev), cu, n, n)
    torch.cuda.synchronize()
    pa, pb_ = a.pool.cpu().numpy(), b.pool.cpu().numpy()
    for page in range(3):
        for h in range(hkv):
            ba = (page * hkv + h) * 18 * d
            bb = (page * hkv + h) * (25 * d + 64)
            assert np.array_equal(pa[ba + 9 * d: ba + 18 * d], pb_[bb + 16 * d + 64: bb + 25 * d + 64])


def run_step(wl, num_splits=0):
    dw = DeviceWorkload(wl, num_splits=num_splits, kv_format="k8v4")
    dw.fill_context()
    dw.load_step_inputs()
    dw.step()
    torch.cuda.synchronize()
    assert dw.err_bits() == 0
    return dw


DECODE = [
    # name, batch, hq, hkv, d, T, ctx
    ("k8_one_token", 1, 8, 2, 128, 1, [0]),
    ("k8_tail_ragged", 2, 8, 2, 128, 1, [17, 300]),
    ("k8_gqa6_d256", 3, 24, 4, 256, 1, [1000, 129, 5]),
    ("k8_mtp4", 2, 24, 4, 256, 4, [127, 520]),
    ("k8_mtp6", 1, 12, 2, 256, 6, [777]),
    ("k8_rows96", 2, 24, 4, 256, 16, [400, 130]),
    ("k8_many_short", 9, 24, 4, 256, 1, [1, 15, 16, 17, 127, 128, 129, 255, 256]),
]


def k8_kernel(d, hq, hkv, T):
    """The kernel nvkv_decode_attn_k8v4 picks: the tensor-core pipeline for
    head_dim 256 and at most 6 query rows per kv-head, else CUDA cores."""
    return "decode_qk4_k8v4" if d == 256 and T * (hq // hkv) <= 6 else "decode_simt"


@pytest.mark.parametrize("case", DECODE, ids=[c[0] for c in DECODE])
@pytest.mark.parametrize("num_splits", [0, 3])
def test_decode_k8v4_all_rows(case, num_splits):
    name, b, hq, hkv, d, T, ctx = case
    wl = W.small(name, b, hq, hkv, d, T, ctx, seed=zlib.crc32(name.encode()) % 1000)
    dw = run_step(wl, num_splits)
    assert nv.nvkv_decode_kernel_name(dw.cache, T, hq) == k8_kernel(d, hq, hkv, T)
    rows = all_rows(wl)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs(wl, rows, k8=True), name)


TC_CASES = [c for c in DECODE if k8_kernel(c[4], c[2], c[3], c[5]) == "decode_qk4_k8v4"]


@pytest.mark.parametrize("case", TC_CASES, ids=[c[0] for c in TC_CASES])
def test_decode_k8v4_cuda_core_kernel_on_the_tensor_core_shapes(case, monkeypatch):
    """The shapes the tensor-core K8V4 decode takes, forced onto the
    CUDA-core kernel: both within tolerance of the oracle."""
    name, b, hq, hkv, d, T, ctx = case
    monkeypatch.setenv("NVKV_DECODE_KERNEL", "simt")
    wl = W.small(name, b, hq, hkv, d, T, ctx, seed=zlib.crc32(name.encode()) % 1000 + 1)
    dw = run_step(wl)
    assert nv.nvkv_decode_kernel_name(dw.cache, T, hq) == "decode_simt"
    rows = all_rows(wl)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs(wl, rows, k8=True), name + "/simt")


def test_decode_k8v4_tensor_core_long_context_sampled():
    """3 x 60000 cached tokens, T=1, on the tensor-core K8V4 decode: many
    units per split, several segments per CTA; sampled rows vs the oracle."""
    wl = W.long_context(T=1, ctx=(60000, 60000, 60000))
    dw = run_step(wl)
    assert nv.nvkv_decode_kernel_name(dw.cache, 1, wl.num_q_heads) == "decode_qk4_k8v4"
    rows = sample_rows(wl, 12, seed=9)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs(wl, rows, k8=True), wl.name + "/k8v4")


def test_decode_k8v4_batch2_verify_config():
    wl = W.batch2_verify()
    dw = run_step(wl)
    rows = sample_rows(wl, 24, seed=5)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs(wl, rows, k8=True), wl.name)


PREFILL = [
    # name, batch, hq, hkv, d, chunk, ctx
    ("k8_chunk_from_empty", 1, 8, 2, 128, 64, [0]),
    ("k8_chunk_ragged", 2, 24, 4, 256, 37, [300, 5]),
    ("k8_chunk_tiny_tail", 3, 24, 4, 256, 1, [0, 63, 64]),
]


@pytest.mark.parametrize("case", PREFILL, ids=[c[0] for c in PREFILL])
def test_prefill_k8v4(case):
    name, b, hq, hkv, d, T, ctx = case
    wl = W.small(name, b, hq, hkv, d, T, ctx, mode="prefill", seed=zlib.crc32(name.encode()) % 1000)
    dw = run_step(wl)
    rows = all_rows(wl) if len(all_rows(wl)) <= 2500 else sample_rows(wl, 400, seed=3)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs(wl, rows, k8=True), name)


def test_decode_k8v4_reports_bad_page():
    dev = torch.device("cuda")
    hkv, hq, d = 2, 4, 128
    cache = nv.Cache.allocate(2, hkv, d, dev, fill=0, kv_format="k8v4")
    pt = torch.tensor([[0, 9]], dtype=torch.int32, device=dev)
    lens = torch.tensor([20], dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    seqs = nv.Seqs(pt, lens, 20, err)
    q = torch.zeros((1, hq, d), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(nv.nvkv_decode_workspace_bytes(1, 1, hq, hkv, d, 2), dtype=torch.uint8,
                     device=dev)
    out = torch.empty((1, hq, d), dtype=torch.bfloat16, device=dev)
    nv.nvkv_decode_attn_k8v4(cache, seqs, q, 1, hq, 0.1, 2, ws)
    nv.nvkv_combine(seqs, ws, 1, hq, hkv, d, 2, out)
    torch.cuda.synchronize()
    assert int(err.item()) & nv.DEVERR_PAGE_ID
    assert torch.isfinite(out.float()).all()


def test_decode_k8v4_tensor_core_reports_bad_page():
    """head_dim 256 on the tensor-core K8V4 decode: an out-of-range page id
    inside the visible range is reported, its tokens are skipped, and the
    outputs equal the oracle over the remaining keys (a fill of 0 makes
    every loaded key and value zero, so each row is the mean of zeros)."""
    dev = torch.device("cuda")
    hkv, hq, d = 4, 24, 256
    cache = nv.Cache.allocate(4, hkv, d, dev, fill=0, kv_format="k8v4")
    pt = torch.tensor([[0, 1, 99, 2]], dtype=torch.int32, device=dev)
    lens = torch.tensor([60], dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    seqs = nv.Seqs(pt, lens, 64, err)
    assert nv.nvkv_decode_kernel_name(cache, 1, hq) == "decode_qk4_k8v4"
    q = torch.randn((1, hq, d), device=dev).bfloat16()
    ws = torch.empty(nv.nvkv_decode_workspace_bytes(1, 1, hq, hkv, d, 3), dtype=torch.uint8,
                     device=dev)
    out = torch.empty((1, hq, d), dtype=torch.bfloat16, device=dev)
    nv.nvkv_decode_attn_k8v4(cache, seqs, q, 1, hq, 0.0625, 3, ws)
    nv.nvkv_combine(seqs, ws, 1, hq, hkv, d, 3, out)
    torch.cuda.synchronize()
    assert int(err.item()) & nv.DEVERR_PAGE_ID
    assert torch.isfinite(out.float()).all()
    assert (out.float() == 0).all()


@pytest.mark.parametrize("kind", ["device", "pinned"])
def test_k8v4_spill_restore_and_attention_after_restore(kind):
    """Whole K8V4 pages (nvkv_k8v4_page_bytes each) move to arena slots and
    back bit for bit; attention over a pool whose pages were destroyed and
    restored equals attention before the spill, bit for bit."""
    wl = W.small("k8_spill", 2, 24, 4, 256, 1, [700, 300], seed=22)
    dw = run_step(wl)
    before = dw.out.clone()
    pb = nv.nvkv_k8v4_page_bytes(4, 256)
    used = np.unique(dw.page_table_np[dw.page_table_np >= 0])
    slots = np.arange(len(used))
    if kind == "device":
        arena = torch.full((len(used) * pb,), 0x3C, dtype=torch.uint8, device="cuda")
        pid = torch.from_numpy(used.astype(np.int32)).cuda()
        sid = torch.from_numpy(slots.astype(np.int32)).cuda()
    else:
        arena = torch.full((len(used) * pb,), 0x3C, dtype=torch.uint8).pin_memory()
        pid = torch.from_numpy(used.astype(np.int32)).pin_memory()
        sid = torch.from_numpy(slots.astype(np.int32)).pin_memory()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvkv_pages_spill(dw.cache, pid, sid, arena, err)
    torch.cuda.synchronize()
    pool = dw.cache.pool.cpu().numpy().reshape(wl.num_pages, pb)
    ar = arena.cpu().numpy().reshape(len(used), pb)
    for p, s in zip(used, slots):
        assert np.array_equal(ar[s], pool[p])
    dw.cache.pool.fill_(0x77)
    nv.nvkv_pages_restore(dw.cache, pid, sid, arena, err)
    torch.cuda.synchronize()
    assert np.array_equal(dw.cache.pool.cpu().numpy().reshape(wl.num_pages, pb)[used], pool[used])
    dw.attend()
    torch.cuda.synchronize()
    assert torch.equal(dw.out, before)
    assert int(err.item()) == 0


@pytest.mark.parametrize("scale", [1e4, 1e-4])
def test_decode_k8v4_query_scale(scale):
    """q scaled by 1e4 and by 1e-4 on the tensor-core K8V4 decode: the query
    terms take any finite scale (power-of-two row prescale), against the
    oracle at the attention tolerance."""
    wl = W.small("k8_qscale", 2, 24, 4, 256, 1, [3000, 1500], seed=78)
    dw = DeviceWorkload(wl, num_splits=5, kv_format="k8v4")
    dw.fill_context()
    dw.load_step_inputs()
    assert nv.nvkv_decode_kernel_name(dw.cache, 1, wl.num_q_heads) == "decode_qk4_k8v4"
    q = to_bf16_bits(W.bf16_bits_to_f32(dw.q_np) * np.float32(scale))
    dw.q = bf16_tensor(q, dw.device)
    dw.step()
    torch.cuda.synchronize()
    assert dw.err_bits() == 0
    rows = all_rows(wl)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs(wl, rows, k8=True, q=q),
                 f"{wl.name} q x {scale:g}")
