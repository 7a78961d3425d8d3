"""GPU parity of the split-K decode / MTP-verify attention (nvkv_decode_attn
+ nvkv_combine) against the float64 oracle, on the seeded synthetic
workloads: all rows for small cases, sampled rows at full size.  The
tolerance is |err| <= 8e-3 + 8e-3 |ref| (parity_util)."""
import zlib

import numpy as np
import pytest
import torch

import nvfp4_quantized_kv_b200 as nv
import oracle
from nvfp4_quantized_kv_b200 import workload as W
from nvfp4_quantized_kv_b200.harness import DeviceWorkload

from parity_util import (all_rows, assert_close, gpu_rows, oracle_outputs, oracle_outputs_dense,
                         sample_rows)

pytestmark = pytest.mark.gpu


def run_step(wl, num_splits=0):
    dw = DeviceWorkload(wl, num_splits=num_splits)
    dw.fill_context()
    dw.load_step_inputs()
    dw.step()
    torch.cuda.synchronize()
    assert dw.err_bits() == 0
    return dw


SMALL = [
    # name, batch, hq, hkv, d, T, ctx
    ("one_token", 1, 8, 2, 128, 1, [0]),
    ("tail_ragged", 2, 8, 2, 128, 1, [17, 300]),
    ("gqa6_d256", 3, 24, 4, 256, 1, [1000, 129, 5]),
    ("mtp4_short", 2, 24, 4, 256, 4, [127, 520]),
    ("mtp6", 1, 12, 2, 256, 6, [777]),
    ("mha", 2, 4, 4, 128, 2, [250, 33]),
    ("t16_g8", 1, 8, 1, 128, 16, [300]),
    ("rows80_d256", 1, 8, 1, 256, 10, [1000]),
    ("rows96_d256", 2, 24, 4, 256, 16, [400, 130]),
    ("many_short", 9, 24, 4, 256, 1, [1, 15, 16, 17, 127, 128, 129, 255, 256]),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
@pytest.mark.parametrize("num_splits", [0, 3])
def test_decode_small_all_rows(case, num_splits):
    name, b, hq, hkv, d, T, ctx = case
    wl = W.small(name, b, hq, hkv, d, T, ctx, seed=zlib.crc32(name.encode()) % 1000)
    dw = run_step(wl, num_splits)
    rows = all_rows(wl)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs(wl, rows), name)


def test_tiny_decode_config():
    wl = W.tiny_decode()
    dw = run_step(wl)
    rows = all_rows(wl)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs(wl, rows), wl.name)


def test_batch2_verify_config():
    wl = W.batch2_verify()
    dw = run_step(wl)
    rows = sample_rows(wl, 40, seed=1)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs(wl, rows), wl.name)


def test_ragged_batch_config():
    wl = W.ragged_batch()
    dw = run_step(wl)
    rows = sample_rows(wl, 48, seed=2)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs(wl, rows), wl.name)


@pytest.mark.parametrize("T", [1, 6])
def test_long_context_config_sampled(T):
    """3 x {330k, 420k, 470k}: every head of the last query of each
    sequence, and for T=6 every head of the first query too."""
    wl = W.long_context(T=T)
    dw = run_step(wl)
    assert nv.nvkv_decode_kernel_name(dw.cache, T, wl.num_q_heads) == (
        "decode_qk4" if T == 1 else "decode_tc")
    ts = sorted({0, T - 1})
    rows = [(b, t, hq) for b in range(wl.batch) for t in ts for hq in range(wl.num_q_heads)]
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs_dense(wl, rows), wl.name)


@pytest.mark.parametrize("T", [1, 6])
@pytest.mark.parametrize("num_splits", [0, 12, 1502])
def test_rows_ending_on_page_unit_and_split_boundaries(T, num_splits):
    """Visible ranges that end exactly on a page, a 128-token unit and a
    split boundary.  Every pair has 500 or 501 units; 12 splits put
    boundaries at pair ends, 1502 (= units of all pairs / 4) at every fourth
    unit, so the last row of sequence 0 ends where a split ends and rows of
    sequences 1 and 2 end on the unit boundary at 64000 keys.  All rows."""
    ctx = {1: [63999, 64002, 64000], 6: [63994, 63997, 63995]}[T]
    wl = W.small(f"bounds_T{T}", 3, 24, 4, 256, T, ctx, seed=41)
    dw = run_step(wl, num_splits)
    ends = {(b, t): wl.query_position(b, t) + 1 for b in range(3) for t in range(T)}
    assert 64000 in ends.values()
    rows = all_rows(wl)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs_dense(wl, rows), wl.name)


def split_count_bound(wl, rows, f16_exponent: bool):
    """Largest difference the split count can make to an output element.

    Split boundaries change which running maximum m each weight
    p = 2^(x - m) is rounded against; the scores x (log2 units) themselves
    do not change.  The combine merges the splits exactly up to fp32
    rounding, so every split count computes o = sum_j P~_j v_j / sum_j P~_j
    with P~_j the rounded weights in one global scale, and
        o~ - o = sum_j (P~_j - P_j)(v_j - o) / sum_j P~_j.
    A weight's error is at most e_j * p_j + 2^-25 (f16 subnormals, absolute
    in units where the split's largest weight is >= 1, i.e. the lazy maximum
    is at most 8 below the top score), with
      e_j = 2^-11 + 2^-22             (fp32 exp2, one rounding to f16), or
      e_j = 2^-9 + ln2 * 2^-11 * |x_j - m|,  |x_j - m| <= x_max - x_j + 8
                                      (exponent argument rounded to f16, f16
                                       exp2 and its rounding within 2^-9).
    So |o~_d - o_d| <= sum_j w_j e_j |v_jd - o_d| + 2^-25 sum_j |v_jd - o_d|
    (w_j the exact weights), plus fp32 accumulation (2^-20 of sum_j w_j
    |v_jd|).  Two split counts differ by at most twice that, plus the two
    bf16 roundings of the outputs (unit roundoff 2^-8, bf16 having 8
    significant bits: 2^-8 |o| each).  All terms from the oracle's
    dequantised keys and values in float64."""
    q = wl.queries()
    G = wl.group
    bounds = np.zeros((len(rows), wl.head_dim))
    cache = {}
    for i, (b, t, hq) in enumerate(rows):
        h = hq // G
        if (b, h) not in cache:
            k, v = wl.kv_rows(b, 0, int(wl.kv_lens[b]))
            cache[(b, h)] = (oracle.qdq_rows(np.ascontiguousarray(k[:, h])),
                             oracle.qdq_rows(np.ascontiguousarray(v[:, h])))
        k_hat, v_hat = cache[(b, h)]
        n = wl.query_position(b, t) + 1
        qf = W.bf16_bits_to_f32(q[b * wl.T + t, hq]).astype(np.float64)
        s = (k_hat[:n] @ qf) * wl.sm_scale
        w = np.exp(s - s.max())
        w /= w.sum()
        o = w @ v_hat[:n]
        x = s * np.log2(np.e)
        if f16_exponent:
            e = 2.0 ** -9 + np.log(2) * 2.0 ** -11 * (x.max() - x + 8)
        else:
            e = np.full(n, 2.0 ** -11 + 2.0 ** -22)
        dev = np.abs(v_hat[:n] - o)
        one = (w * e) @ dev + 2.0 ** -25 * dev.sum(axis=0) + 2.0 ** -20 * (w @ np.abs(v_hat[:n]))
        bounds[i] = 2 * one + 2 * 2.0 ** -8 * np.abs(o) + 1e-7
    return bounds


@pytest.mark.parametrize("T,kernel", [(1, "decode_qk4"), (3, "decode_tc")])
def test_split_count_does_not_change_the_result(T, kernel):
    """Combine metamorphic check: 1 split per pair up to more splits than
    units give the same outputs within the bound derived in
    split_count_bound (far tighter than the attention tolerance when the
    weights are spread over many keys)."""
    wl = W.small(f"splits_T{T}", 3, 24, 4, 256, T, [2000, 50, 900], seed=4)
    dw = DeviceWorkload(wl, num_splits=1)
    dw.fill_context()
    dw.load_step_inputs()
    assert nv.nvkv_decode_kernel_name(dw.cache, T, wl.num_q_heads) == kernel
    dw.append()
    outs = []
    for S in (1, 2, 7, 64, 296, 5000):
        dw.num_splits = S
        dw.workspace = torch.empty(
            nv.nvkv_decode_workspace_bytes(wl.batch, wl.T, wl.num_q_heads, wl.num_kv_heads,
                                           wl.head_dim, S), dtype=torch.uint8, device="cuda")
        dw.attend()
        torch.cuda.synchronize()
        assert dw.err_bits() == 0
        outs.append(dw.out.float().cpu().numpy().astype(np.float64))
    rows = all_rows(wl)
    bound = split_count_bound(wl, rows, f16_exponent=False)  # both: fp32 exp2, f16 weights
    ref = np.stack([outs[0][b * wl.T + t, hq] for b, t, hq in rows])
    for S, o in zip((2, 7, 64, 296, 5000), outs[1:]):
        got = np.stack([o[b * wl.T + t, hq] for b, t, hq in rows])
        ratio = np.abs(got - ref) / bound
        assert ratio.max() <= 1.0, (S, float(ratio.max()))
    # the bound is several times tighter than the parity tolerance
    assert np.median(bound) < 2e-3


def test_queries_without_keys_give_zeros():
    """kv_len < T: the first queries of the block see no key."""
    dev = torch.device("cuda")
    hkv, hq, d, T = 2, 4, 128, 4
    cache = nv.Cache.allocate(2, hkv, d, dev, fill=0)
    pt = torch.tensor([[0, 1]], dtype=torch.int32, device=dev)
    lens = torch.tensor([2], dtype=torch.int32, device=dev)
    seqs = nv.Seqs(pt, lens, 2)
    rng = np.random.default_rng(0)
    q = torch.from_numpy(rng.standard_normal((T, hq, d)).astype(np.float32)).to(dev).bfloat16()
    S = 4
    ws = torch.empty(nv.nvkv_decode_workspace_bytes(1, T, hq, hkv, d, S), dtype=torch.uint8,
                     device=dev)
    out = torch.full((T, hq, d), 7.0, dtype=torch.bfloat16, device=dev)
    nv.nvkv_decode_attn(cache, seqs, q, T, hq, 0.1, S, ws)
    nv.nvkv_combine(seqs, ws, T, hq, hkv, d, S, out)
    torch.cuda.synchronize()
    assert (out[:2] == 0).all()          # positions -2, -1: no key
    assert torch.isfinite(out[2:]).all()  # positions 0 and 1 see the (zero) cache
    assert (out[2:] == 0).all()           # an all-zero pool dequantises to 0


def test_decode_reports_bad_page():
    dev = torch.device("cuda")
    hkv, hq, d = 2, 4, 128
    cache = nv.Cache.allocate(2, hkv, d, dev, fill=0)
    pt = torch.tensor([[0, 9]], dtype=torch.int32, device=dev)
    lens = torch.tensor([20], dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    seqs = nv.Seqs(pt, lens, 20, err)
    q = torch.zeros((1, hq, d), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(nv.nvkv_decode_workspace_bytes(1, 1, hq, hkv, d, 2), dtype=torch.uint8,
                     device=dev)
    out = torch.empty((1, hq, d), dtype=torch.bfloat16, device=dev)
    nv.nvkv_decode_attn(cache, seqs, q, 1, hq, 0.1, 2, ws)
    nv.nvkv_combine(seqs, ws, 1, hq, hkv, d, 2, out)
    torch.cuda.synchronize()
    assert int(err.item()) & nv.DEVERR_PAGE_ID
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("case", [c for c in SMALL if c[4] == 256], ids=[c[0] for c in SMALL if c[4] == 256])
def test_tensor_core_and_cuda_core_kernels_agree(case, monkeypatch):
    """The same workload through both decode kernels (the tensor-core one is
    the default for head_dim 256; NVKV_DECODE_KERNEL=simt forces the other):
    both within tolerance of the oracle."""
    name, b, hq, hkv, d, T, ctx = case
    wl = W.small(name, b, hq, hkv, d, T, ctx, seed=zlib.crc32(name.encode()) % 1000 + 1)
    rows = all_rows(wl)
    ref = oracle_outputs(wl, rows)
    for kernel in ("default", "simt"):
        if kernel == "simt":
            monkeypatch.setenv("NVKV_DECODE_KERNEL", "simt")
        dw = run_step(wl)
        assert_close(gpu_rows(dw.out, wl, rows), ref, f"{name}/{kernel}")


@pytest.mark.parametrize("T,kernel", [(1, "decode_qk4"), (4, "decode_tc")])
def test_tensor_core_kernels_report_bad_page_and_stay_finite(T, kernel):
    """head_dim 256: an out-of-range page id in a visible range is reported
    through the error word by the tensor-core kernels, its tokens are
    skipped, and every output stays finite."""
    dev = torch.device("cuda")
    hkv, hq, d = 4, 24, 256
    cache = nv.Cache.allocate(4, hkv, d, dev, fill=0)
    pt = torch.tensor([[0, 1, 99, 2]], dtype=torch.int32, device=dev)  # page 99 does not exist
    lens = torch.tensor([60], dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    seqs = nv.Seqs(pt, lens, 64, err)
    assert nv.nvkv_decode_kernel_name(cache, T, hq) == kernel
    q = torch.randn((T, hq, d), device=dev).bfloat16()
    S = 3
    ws = torch.empty(nv.nvkv_decode_workspace_bytes(1, T, hq, hkv, d, S), dtype=torch.uint8,
                     device=dev)
    out = torch.empty((T, hq, d), dtype=torch.bfloat16, device=dev)
    nv.nvkv_decode_attn(cache, seqs, q, T, hq, 0.0625, S, ws)
    nv.nvkv_combine(seqs, ws, T, hq, hkv, d, S, out)
    torch.cuda.synchronize()
    assert int(err.item()) & nv.DEVERR_PAGE_ID
    assert torch.isfinite(out.float()).all()
    # the loaded pages are all zero (fill 0), so every row is a mean of zeros
    assert (out.float() == 0).all()


@pytest.mark.parametrize("T,kernel", [(1, "decode_qk4"), (4, "decode_tc")])
def test_tensor_core_kernels_empty_sequence_gives_zeros(T, kernel):
    """head_dim 256, a batch whose first sequence has no key at all and
    whose second has fewer keys than queries: rows without a visible key
    are zeros, the others match the oracle."""
    wl = W.small(f"empty_T{T}", 2, 24, 4, 256, T, [0, 700], seed=12)
    dw = DeviceWorkload(wl, num_splits=7)
    dw.fill_context()
    dw.load_step_inputs()
    assert nv.nvkv_decode_kernel_name(dw.cache, T, wl.num_q_heads) == kernel
    # no step append: sequence 0 has kv_len 0 (every row sees no key),
    # sequence 1 its 700 cached rows
    dw.kv_lens.copy_(torch.tensor([0, 700], dtype=torch.int32))
    dw.attend()
    torch.cuda.synchronize()
    assert dw.err_bits() == 0
    out = dw.out.float().cpu().numpy()
    assert (out[:T] == 0).all()
    rows = [(1, t, hq) for t in range(T) for hq in range(wl.num_q_heads)]
    q = wl.queries()
    got = np.stack([out[T + t, hq] for _, t, hq in rows]).astype(np.float64)
    k, v = wl.kv_rows(1, 0, 700)
    jobs = [(k, v, hq // wl.group, 700 - T + t + 1, q[T + t, hq]) for _, t, hq in rows]
    ref, _, _ = oracle.attention_rows(jobs, wl.num_kv_heads, wl.head_dim, wl.sm_scale)
    assert_close(got, ref, wl.name)
