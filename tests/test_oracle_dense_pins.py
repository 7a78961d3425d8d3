"""Pins of the oracle's bulk helpers (CPU): qdq_rows over many rows at once
equals the per-row quantise-dequantise, and attention_dense over
pre-dequantised rows equals the per-row oracle (attention_rows, itself
pinned by closed forms and brute force in test_oracle_pins.py) on random
cases with ragged visibility, to float64 summation-order accuracy."""
import numpy as np

import oracle


def _bits(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_bulk_qdq_equals_row_by_row():
    rng = np.random.default_rng(1)
    x = _bits(rng.standard_normal((300, 256)) * 10.0 ** rng.uniform(-3, 3, (300, 1)))
    bulk = oracle.qdq_rows(x)
    one = np.stack([oracle.qdq_rows(x[i:i + 1])[0] for i in range(x.shape[0])])
    assert np.array_equal(bulk, one)
    # and the row helper agrees with the group quantiser + dequantiser
    codes, sb = oracle.quantize_group(x[7, :16])
    assert np.array_equal(bulk[7, :16], [oracle.dequant(int(c), sb) for c in codes])


def test_dense_attention_equals_per_row_oracle():
    rng = np.random.default_rng(2)
    Hkv, D, n = 3, 128, 700
    k = _bits(rng.standard_normal((n, Hkv, D)) * np.where(rng.random(D) < 0.03, 10.0, 1.0))
    v = _bits(rng.standard_normal((n, Hkv, D)))
    h = 2
    k_hat = oracle.qdq_rows(k[:, h])
    v_hat = oracle.qdq_rows(v[:, h])
    qs = _bits(rng.standard_normal((9, D)) * 3)
    nvis = np.array([1, 2, 16, 17, 127, 128, 129, 699, 700])
    out, lse = oracle.attention_dense(k_hat, v_hat, qs, nvis, 0.07)
    jobs = [(k, v, h, int(nv), qs[i]) for i, nv in enumerate(nvis)]
    ref, ref_lse, _ = oracle.attention_rows(jobs, Hkv, D, 0.07)
    assert np.allclose(out, ref, rtol=1e-11, atol=1e-12)
    assert np.allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)
    # a row that sees no key gets zeros and lse -inf
    z, zl = oracle.attention_dense(k_hat, v_hat, qs[:1], [0], 0.07)
    assert (z == 0).all() and zl[0] == -np.inf
