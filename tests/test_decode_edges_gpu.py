"""GPU parity at the edges of the decode kernels' arithmetic, against the
float64 oracle (|err| <= 8e-3 + 8e-3 |ref|, parity_util):

* query rows scaled by 1e4 and by 1e-4 (the tensor-core kernels take q
  through a prescaled NVFP4 expansion or through f16; the CUDA-core kernel
  in fp32);
* keys that raise the running maximum by more than the lazy-rescale
  threshold (8 in log2 units) in the middle of a split, three times by
  about 12 and once by about 230;
* all-equal scores (q = 0) over the 3 x {330k, 420k, 470k} pool, where the
  output is the mean of the dequantised values.

Each case states the kernel the dispatcher picks for its shape and checks
that nvkv_decode_kernel_name agrees.  The source of the path is the decode
half of the "knoopx/ninfer" README, "Capabilities and limits" (batched
decode, MTP verify), over the NVFP4 cache of the "gzenz/ninfer" README,
"Fork changes vs upstream" -> "Context and model"."""
import numpy as np
import pytest
import torch

import nvfp4_quantized_kv_b200 as nv
from nvfp4_quantized_kv_b200 import workload as W
from nvfp4_quantized_kv_b200.harness import DeviceWorkload, bf16_tensor

import oracle
from parity_util import ATOL, RTOL, all_rows, assert_close, gpu_rows, oracle_outputs_dense

pytestmark = pytest.mark.gpu

# (T, kernel the default dispatch picks for 24 q / 4 kv heads, head_dim 256)
KERNELS = [(1, "decode_qk4"), (6, "decode_tc")]


def scaled_bits(bits: np.ndarray, s: float) -> np.ndarray:
    """bf16 bits of bf16(x * s): the scaled query both sides receive."""
    return W.to_bf16_bits(W.bf16_bits_to_f32(bits) * np.float32(s))


def run(dw: DeviceWorkload, q_bits=None):
    if q_bits is not None:
        dw.q = bf16_tensor(q_bits, dw.device)
    dw.step()
    torch.cuda.synchronize()
    assert dw.err_bits() == 0


def expect_kernel(dw: DeviceWorkload, name: str, monkeypatch, simt: bool):
    if simt:
        monkeypatch.setenv("NVKV_DECODE_KERNEL", "simt")
        name = "decode_simt"
    assert nv.nvkv_decode_kernel_name(dw.cache, dw.wl.T, dw.wl.num_q_heads) == name


def score_accumulation_bound(wl, rows, q_bits, steps: int):
    """Output change the fp32 accumulation of the scores can cause.

    The tensor-core kernels accumulate each score over `steps` MMA steps in
    fp32; each step may move it by up to 2^-23 of the sum of the magnitudes
    of its products, so |dx_j| <= steps * 2^-23 * sum_d |q'_d k_jd| (log2
    units, q' = q * sm_scale * log2(e)).  A weight 2^(x_j - max x) then
    changes by at most a factor 2^(|dx_j| + max_i |dx_i|), so
    |do_d| <= sum_j w_j * ln2 * (|dx_j| + max|dx|) * |v_jd - o_d| to first
    order (doubled for the higher orders).  From the oracle's dequantised keys
    and values in float64; zero wherever the scores are small."""
    G = wl.group
    out = np.zeros((len(rows), wl.head_dim))
    kv = {}
    for i, (b, t, hq) in enumerate(rows):
        h = hq // G
        if (b, h) not in kv:
            k, v = wl.kv_rows(b, 0, int(wl.kv_lens[b]))
            kv[(b, h)] = (oracle.qdq_rows(np.ascontiguousarray(k[:, h])),
                          oracle.qdq_rows(np.ascontiguousarray(v[:, h])))
        k_hat, v_hat = kv[(b, h)]
        n = wl.query_position(b, t) + 1
        qp = W.bf16_bits_to_f32(q_bits[b * wl.T + t, hq]).astype(np.float64) * wl.sm_scale * \
            np.log2(np.e)
        x = k_hat[:n] @ qp
        dx = steps * 2.0 ** -23 * (np.abs(k_hat[:n]) @ np.abs(qp))
        w = np.exp2(x - x.max())
        w /= w.sum()
        o = w @ v_hat[:n]
        out[i] = 2 * ((w * np.log(2) * (dx + dx.max())) @ np.abs(v_hat[:n] - o))
    return out


@pytest.mark.parametrize("simt", [False, True], ids=["default", "simt"])
@pytest.mark.parametrize("T,kernel", KERNELS, ids=[k for _, k in KERNELS])
@pytest.mark.parametrize("scale", [1e4, 1e-4])
def test_query_scale(T, kernel, scale, simt, monkeypatch):
    """At q x 1e4 the scores reach about 2e4 log2 units.  decode_qk4 and the
    CUDA-core kernel meet the attention tolerance there; decode_tc, whose
    scores accumulate over 32 f16 MMA steps (two f16 terms of q, 16 head_dim
    steps each), is checked against the tolerance plus the bound its fp32
    score accumulation allows (score_accumulation_bound): rows with keys
    within a few hundredths of a log2 unit of the top score move by more
    than the tolerance alone."""
    wl = W.small(f"qscale_T{T}", 2, 24, 4, 256, T, [3000, 1500], seed=77)
    dw = DeviceWorkload(wl, num_splits=5)
    dw.fill_context()
    dw.load_step_inputs()
    expect_kernel(dw, kernel, monkeypatch, simt)
    q = scaled_bits(dw.q_np, scale)
    run(dw, q)
    rows = all_rows(wl)
    got = gpu_rows(dw.out, wl, rows)
    ref = oracle_outputs_dense(wl, rows, q=q)
    if kernel == "decode_tc" and not simt and scale > 1:
        extra = score_accumulation_bound(wl, rows, q, steps=32)
        err = np.abs(got - ref)
        bound = ATOL + RTOL * np.abs(ref) + extra
        assert np.isfinite(got).all()
        assert (err <= bound).all(), float((err / bound).max())
        # the extra allowance only matters where scores nearly tie
        assert np.mean(extra > ATOL) < 0.05
    else:
        assert_close(got, ref, f"{wl.name} q x {scale:g}")


def plant_keys(wl: W.Workload, plants):
    """Replace K rows of kv-head 0 at the given positions by c times the
    head-0 row of the sequence's last query (plants: {b: [(pos, c), ...]});
    every consumer of wl.kv_rows (the device fill, the step's new rows and
    the oracle) sees the same keys."""
    q = wl.queries()
    orig = wl.kv_rows

    def kv_rows(b, start, stop, threads=None):
        k, v = orig(b, start, stop, threads)
        qrow = W.bf16_bits_to_f32(q[b * wl.T + wl.T - 1, 0])
        for pos, c in plants.get(b, []):
            if start <= pos < stop:
                k[pos - start, 0] = W.to_bf16_bits(qrow * np.float32(c))
        return k, v

    wl.kv_rows = kv_rows
    return wl


@pytest.mark.parametrize("simt", [False, True], ids=["default", "simt"])
@pytest.mark.parametrize("T,kernel", KERNELS, ids=[k for _, k in KERNELS])
@pytest.mark.parametrize("num_splits", [0, 12])
def test_running_max_raised_mid_split(T, kernel, num_splits, simt, monkeypatch):
    """A key c*q has score c*|q|^2*sm_scale*log2(e), about 23c in log2
    units for |q|^2 ~ 256, against about 10 for the largest random key of
    20000: c = 1, 1.5, 2 raise the running maximum by about 12 each, c = 12
    by about 230 (the old sums then scale by 2^-230, i.e. vanish).  With 12
    splits a split covers about 9,700 tokens, so every planted position is
    inside a split and inside a 128-token unit."""
    wl = W.small(f"raise_T{T}", 2, 24, 4, 256, T, [20000, 9000], seed=5)
    plant_keys(wl, {0: [(3000, 1.0), (7777, 1.5), (12345, 2.0), (19950, 12.0)],
                    1: [(1000, 1.0), (4321, 1.5), (8100, 2.0)]})
    dw = DeviceWorkload(wl, num_splits=num_splits)
    dw.fill_context()
    dw.load_step_inputs()
    expect_kernel(dw, kernel, monkeypatch, simt)
    run(dw)
    rows = all_rows(wl)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs_dense(wl, rows), wl.name)


def test_all_equal_scores_long_context():
    """q = 0 over the 3 x {330k, 420k, 470k} pool: every weight is 1, so each
    row is the plain mean of the dequantised V rows it sees (a property of
    the definition at any size); all 72 rows against the oracle."""
    wl = W.long_context(T=1)
    dw = DeviceWorkload(wl)
    dw.fill_context()
    dw.load_step_inputs()
    assert nv.nvkv_decode_kernel_name(dw.cache, 1, wl.num_q_heads) == "decode_qk4"
    q0 = np.zeros_like(dw.q_np)
    run(dw, q0)
    rows = all_rows(wl)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs_dense(wl, rows, q=q0), wl.name)
