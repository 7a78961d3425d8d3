"""GPU parity of chunked-prefill attention (nvkv_prefill_attn) against the
float64 oracle: a chunk of new queries, appended first, attends causally to
the whole cache of its sequence."""
import zlib

import pytest
import torch

from nvfp4_quantized_kv_b200 import workload as W
from nvfp4_quantized_kv_b200.harness import DeviceWorkload

from parity_util import all_rows, assert_close, gpu_rows, oracle_outputs, sample_rows

pytestmark = pytest.mark.gpu

SMALL = [
    # name, batch, hq, hkv, d, chunk, ctx
    ("chunk_from_empty", 1, 8, 2, 128, 64, [0]),
    ("chunk_ragged", 2, 24, 4, 256, 37, [300, 5]),
    ("chunk_long", 1, 12, 2, 256, 200, [1500]),
]


def run(wl):
    dw = DeviceWorkload(wl)
    dw.fill_context()
    dw.load_step_inputs()
    dw.step()
    torch.cuda.synchronize()
    assert dw.err_bits() == 0
    return dw


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_prefill_small(case):
    name, b, hq, hkv, d, T, ctx = case
    wl = W.small(name, b, hq, hkv, d, T, ctx, mode="prefill", seed=zlib.crc32(name.encode()) % 1000)
    dw = run(wl)
    rows = all_rows(wl) if len(all_rows(wl)) <= 2000 else sample_rows(wl, 400, seed=3)
    assert_close(gpu_rows(dw.out, wl, rows), oracle_outputs(wl, rows), name)
