"""Helpers shared by the GPU parity tests: oracle references for sampled
output rows of a synthetic workload, and the attention tolerance."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from nvfp4_quantized_kv_b200.workload import Workload

# Attention output tolerance against the float64 oracle computed on the same
# dequantised values: |gpu - ref| <= ATOL + RTOL * |ref| element-wise.
ATOL = 8e-3
RTOL = 8e-3


def oracle_outputs(wl: Workload, rows, nthreads=None, k8=False, q=None):
    """rows: list of (b, t, hq).  Returns float64 [len(rows)][D]: the exact
    attention of query t of sequence b, head hq, over the sequence's keys
    0 .. ctx_b + t (all rows of the workload, quantised by the oracle; K in
    the K8V4 cache's 8-bit row format when k8).  q: bf16 bits
    [batch*T][Hq][D] replacing the workload's queries."""
    q = wl.queries() if q is None else q
    G = wl.group
    kv = {}
    for b in sorted({r[0] for r in rows}):
        kv[b] = wl.kv_rows(b, 0, int(wl.kv_lens[b]))
    jobs = []
    for b, t, hq in rows:
        k, v = kv[b]
        jobs.append((k, v, hq // G, wl.query_position(b, t) + 1, q[b * wl.T + t, hq]))
    out, _, psum = oracle.attention_rows(jobs, wl.num_kv_heads, wl.head_dim, wl.sm_scale, nthreads,
                                         k8=k8)
    assert np.all(np.abs(psum - 1) < 1e-9)
    return out


def oracle_outputs_dense(wl: Workload, rows, q=None):
    """As oracle_outputs, for many rows over long caches: the keys and values
    of each (sequence, kv-head) are quantised and dequantised once by the
    oracle (qdq_rows) and the rows are computed by oracle.attention_dense
    (pinned against the per-row oracle in test_oracle_dense_pins.py)."""
    q = wl.queries() if q is None else q
    G = wl.group
    out = np.zeros((len(rows), wl.head_dim), np.float64)
    by = {}
    for i, (b, t, hq) in enumerate(rows):
        by.setdefault((b, hq // G), []).append((i, t, hq))
    for b in sorted({b for b, _ in by}):
        k, v = wl.kv_rows(b, 0, int(wl.kv_lens[b]))
        for h in sorted(h for bb, h in by if bb == b):
            items = by[(b, h)]
            k_hat = oracle.qdq_rows(np.ascontiguousarray(k[:, h]))
            v_hat = oracle.qdq_rows(np.ascontiguousarray(v[:, h]))
            qs = np.stack([q[b * wl.T + t, hq] for _, t, hq in items])
            nvis = [wl.query_position(b, t) + 1 for _, t, _ in items]
            o, _ = oracle.attention_dense(k_hat, v_hat, qs, nvis, wl.sm_scale)
            for (i, _, _), row in zip(items, o):
                out[i] = row
            del k_hat, v_hat
    return out


def prefill_sample_queries(n: int):
    """The deterministic sample of a prefill chunk's queries: the first 64,
    the last 64 and every 31st."""
    return sorted(set(range(min(64, n))) | set(range(max(0, n - 64), n)) | set(range(0, n, 31)))


def gpu_rows(out: torch.Tensor, wl: Workload, rows) -> np.ndarray:
    o = out.float().cpu().numpy()
    return np.stack([o[b * wl.T + t, hq] for b, t, hq in rows]).astype(np.float64)


def assert_close(got: np.ndarray, ref: np.ndarray, what: str):
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; "
                           f"max err {err.max():.3e}, worst ratio {(err / bound).max():.2f}")
    return float((err / bound).max())


def all_rows(wl: Workload):
    return [(b, t, hq) for b in range(wl.batch) for t in range(wl.T) for hq in range(wl.num_q_heads)]


def sample_rows(wl: Workload, n: int, seed: int = 0):
    """n distinct rows (all of them when the workload has no more than n)."""
    if wl.batch * wl.T * wl.num_q_heads <= n:
        return all_rows(wl)
    rng = np.random.default_rng(seed)
    rows = set()
    # always the last query of every sequence and the first and last head
    for b in range(wl.batch):
        rows.add((b, wl.T - 1, 0))
        rows.add((b, 0, wl.num_q_heads - 1))
    while len(rows) < n:
        rows.add((int(rng.integers(wl.batch)), int(rng.integers(wl.T)),
                  int(rng.integers(wl.num_q_heads))))
    return sorted(rows)
