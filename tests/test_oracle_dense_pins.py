"""Pins of the oracle's bulk helpers (CPU): qdq_rows over many rows at once
equals the per-row quantise-dequantise, and attention_dense over
pre-dequantised rows equals the per-row oracle (attention_rows, itself
pinned by closed forms and brute force in test_oracle_pins.py) on random
cases with ragged visibility, to float64 summation-order accuracy; and
attention over runs of the keys merged by log-sum-exp equals one pass."""
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


def _merge(parts):
    """Log-sum-exp merge of (normalised output, lse) partials of one set of
    rows: out = sum_s e^(lse_s - M) o_s / sum_s e^(lse_s - M), M = max lse_s;
    partials with lse = -inf (no visible key) drop out."""
    outs = np.stack([o for o, _ in parts])           # [S][m][D]
    lses = np.stack([l for _, l in parts])           # [S][m]
    top = lses.max(axis=0)
    ok = np.isfinite(top)
    w = np.zeros_like(lses)
    w[:, ok] = np.exp(lses[:, ok] - top[None, ok])
    den = w.sum(axis=0)
    out = np.zeros(outs.shape[1:])
    out[ok] = (w[:, ok, None] * outs[:, ok]).sum(axis=0) / den[ok, None]
    lse = np.full(top.shape, -np.inf)
    lse[ok] = top[ok] + np.log(den[ok])
    return out, lse


def test_key_runs_merged_by_log_sum_exp_equal_one_pass():
    """Attention over runs of the keys, each run on its own (its softmax
    normalised over the run, and its log-sum-exp), merged by log-sum-exp,
    equals attention over all the keys: the identity the split-K decode and
    the prefill's key splits rest on.  Runs split at arbitrary places (a
    run of one key, runs past a row's last visible key, empty runs) and
    rows that see no key at all."""
    rng = np.random.default_rng(3)
    D, n = 256, 900
    k_hat = oracle.qdq_rows(_bits(rng.standard_normal((n, D))))
    v_hat = oracle.qdq_rows(_bits(rng.standard_normal((n, D))))
    qs = _bits(rng.standard_normal((8, D)) * 2)
    nvis = np.array([0, 1, 2, 63, 64, 65, 600, 900])
    sm = 256 ** -0.5
    full, full_lse = oracle.attention_dense(k_hat, v_hat, qs, nvis, sm)
    for cuts in ([0, 900], [0, 1, 900], [0, 64, 128, 600, 601, 900], [0, 300, 300, 900],
                 list(range(0, 901, 180))):
        parts = []
        for a, b in zip(cuts[:-1], cuts[1:]):
            vis = np.clip(nvis - a, 0, b - a)
            if b > a:
                parts.append(oracle.attention_dense(k_hat[a:b], v_hat[a:b], qs, vis, sm))
            else:  # an empty run sees no key
                parts.append((np.zeros((len(qs), D)), np.full(len(qs), -np.inf)))
        out, lse = _merge(parts)
        assert np.allclose(out, full, rtol=1e-12, atol=1e-13), cuts
        assert np.allclose(lse[1:], full_lse[1:], rtol=1e-13, atol=1e-13), cuts
        assert (out[0] == 0).all() and lse[0] == -np.inf and full_lse[0] == -np.inf
