"""The seeded input generator that feeds both the kernels and the oracle
(CPU): rows regenerate identically whatever range or thread count asks for
them, a step's new rows are the rows of their positions, page tables are
permutations of the pool, values are bf16 round-to-nearest-even of the
drawn floats with the K outlier channels scaled, and the algorithmic byte
count of a step is the closed form the metric is defined by."""
import numpy as np
import pytest
import torch

from nvfp4_quantized_kv_b200 import workload as W


def test_rows_do_not_depend_on_the_requested_range_or_threads():
    wl = W.small("gen", 2, 24, 4, 256, 3, [20000, 9000], seed=77)
    full_k, full_v = wl.kv_rows(0, 0, 12000, threads=1)
    for a, b in [(0, 5), (4090, 4100), (4096, 8192), (8000, 12000), (11999, 12000)]:
        k, v = wl.kv_rows(0, a, b, threads=4)
        assert np.array_equal(k, full_k[a:b]) and np.array_equal(v, full_v[a:b])
    k1, _ = wl.kv_rows(1, 100, 200)
    k0, _ = wl.kv_rows(0, 100, 200)
    assert not np.array_equal(k0, k1)  # sequences draw different rows


def test_new_rows_are_the_rows_of_their_positions():
    wl = W.small("gen2", 3, 8, 2, 128, 4, [10, 4095, 0], seed=3)
    k, v, cu = wl.new_rows()
    assert list(cu) == [0, 4, 8, 12]
    for b, c in enumerate(wl.ctx):
        kk, vv = wl.kv_rows(b, c, c + wl.T)
        assert np.array_equal(k[cu[b]:cu[b + 1]], kk) and np.array_equal(v[cu[b]:cu[b + 1]], vv)
    assert list(wl.kv_lens) == [14, 4099, 4]


def test_page_tables_are_permutations_of_the_pool():
    for wl in (W.small("gen3", 4, 8, 2, 128, 1, [0, 15, 16, 1000], seed=5), W.tiny_decode()):
        pt = wl.page_table()
        used = pt[pt >= 0]
        assert len(used) == wl.num_pages and len(np.unique(used)) == wl.num_pages
        assert used.min() == 0 and used.max() == wl.num_pages - 1
        for b, n in enumerate(wl.pages_per_seq):
            assert (pt[b, :n] >= 0).all() and (pt[b, n:] == -1).all()
            assert n * 16 >= wl.kv_lens[b] > (n - 1) * 16
    tiny = W.tiny_decode()
    assert np.array_equal(tiny.page_table()[0], np.arange(tiny.num_pages))  # contiguous
    assert np.array_equal(W.small("x", 2, 8, 2, 128, 1, [500, 70], seed=9).page_table(),
                          W.small("x", 2, 8, 2, 128, 1, [500, 70], seed=9).page_table())


def test_bf16_rounding_is_round_to_nearest_even():
    x = np.random.default_rng(1).standard_normal(200000).astype(np.float32)
    x = np.concatenate([x, np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, -0.0],
                                    np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(W.to_bf16_bits(x), want)


def test_outlier_channels_scale_k_only():
    wl = W.small("gen4", 1, 8, 2, 128, 1, [4096], seed=11)
    k, v = wl.kv_rows(0, 0, 4096)
    kf = W.bf16_bits_to_f32(k).reshape(-1, 128)
    vf = W.bf16_bits_to_f32(v).reshape(-1, 128)
    kstd, vstd = kf.std(axis=0), vf.std(axis=0)
    out = np.zeros(128, bool)
    out[wl.outliers] = True
    assert out.sum() == 4
    assert (kstd[out] > 8).all() and (kstd[~out] < 1.2).all()
    assert (vstd < 1.2).all()


def test_kv_bytes_per_step_is_the_metric_closed_form():
    wl = W.long_context(T=1)
    assert wl.kv_bytes_per_step() == 1405443456
    # K and V of every visible token and kv-head: 4.5 bits per element each,
    # 1.125 * D bytes per token per kv-head for the pair
    assert wl.kv_bytes_per_step() == int(sum(int(c) + 1 for c in wl.ctx) * 4 * 256 * 1.125)
    w6 = W.long_context(T=6)
    assert w6.kv_bytes_per_step() == int(sum(int(c) + 6 for c in w6.ctx) * 4 * 256 * 1.125)


def test_device_workload_refuses_an_unknown_cache_format():
    from nvfp4_quantized_kv_b200.harness import DeviceWorkload
    with pytest.raises(ValueError, match="kv_format"):
        DeviceWorkload(W.tiny_decode(), device="cpu", kv_format="int8")
