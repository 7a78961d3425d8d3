"""GPU check of the split-K merge alone (nvkv_combine) against the float64
oracle, tight enough to see errors of the order of 1e-5.

Each split range of the plan gets the oracle's exact partial result for the
keys it owns -- the normalised output o_c and the base-2 log-sum-exp of the
scaled scores -- written in float32 into the workspace layout that
nvkv_decode_attn fills (slot c + b*Hkv + h; lse after the 256-byte aligned
output block).  The merged output is then compared with the oracle's
attention over the whole visible range.

What the merge may add before its final bf16 rounding (fp32 arithmetic), as
a multiple of A = sum_c w_c |o_c| / sum_c w_c (w_c = 2^lse_c, per element):
the float32 rounding of every lse (|lse| < 32 here, half an ulp <= 2^-20
absolute, a relative weight error ln2 * 2^-20 < 7e-7) and exp2f (<= 2 ulp,
2.4e-7) perturb the weights by eps < 1e-6 relative, which moves the
weighted mean by at most 2 * eps * A; the float32 sums of the weights and of
the weighted outputs over n <= 16 ranges and the final division add at most
(2n + 2) * 2^-24 * A < 2.1e-6 A.  Together that is below 4.2e-6 * A; the
test allows delta = 1.2e-5 * A.  Rounding to bf16 (nearest, ties to even)
is monotone, so the bf16 output must lie in [RNE(ref - delta), RNE(ref +
delta)]: for almost every element both ends are the same bf16 value and the
output must be exactly the correctly rounded oracle value; only elements
within delta of a rounding midpoint, or smaller than delta, have more than
one admissible value.  A weighting error of 1e-5 relative moves about 1
element in 400 across a rounding boundary at these magnitudes; the check
covers tens of thousands of elements."""
import numpy as np
import pytest
import torch

import nvfp4_quantized_kv_b200 as nv
import oracle
from nvfp4_quantized_kv_b200 import workload as W

pytestmark = pytest.mark.gpu

LOG2E = 1.4426950408889634


def _bf16_rne(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even of float64 x to bf16, decided in float64: the
    candidates are the bf16 value t obtained by truncating float32(x) and
    its neighbour u away from zero (when float32 rounding carried x onto a
    bf16 value, that value is t and is the nearer one)."""
    f = x.astype(np.float32)
    trunc = (f.view(np.uint32) & 0xFFFF0000).astype(np.uint32)
    t = trunc.view(np.float32).astype(np.float64)
    up = ((trunc.astype(np.uint64) + 0x10000) & 0xFFFFFFFF).astype(np.uint32)
    u = up.view(np.float32).astype(np.float64)
    dt, du = np.abs(x - t), np.abs(x - u)
    even_t = ((trunc >> 16) & 1) == 0
    return np.where((dt < du) | ((dt == du) & even_t), t, u)


def _partials(wl, S):
    """Oracle partials of every split range for every pair and query row."""
    B, Hkv, Hq, D, T, G = wl.batch, wl.num_kv_heads, wl.num_q_heads, wl.head_dim, wl.T, wl.group
    R = T * G
    lens = [int(x) for x in wl.kv_lens]
    units = [(l + 127) // 128 for l in lens]
    U = sum(units) * Hkv
    assert U >= S, "every range must own a unit"
    q = wl.queries()
    slots = S + B * Hkv - 1
    ws_o = np.zeros((slots, R, D), np.float32)
    ws_lse = np.full((slots, R), -np.inf, np.float32)
    wsum = np.zeros((B, T, Hq))
    wabs = np.zeros((B, T, Hq, D))
    jobs, where = [], []
    start = 0
    for b in range(B):
        k, v = wl.kv_rows(b, 0, lens[b])
        for h in range(Hkv):
            ps = start + h * units[b]
            c0 = ((ps + 1) * S - 1) // U
            c1 = ((ps + units[b]) * S - 1) // U
            assert c1 - c0 + 1 <= 16  # the error bound above counts on it
            for c in range(c0, c1 + 1):
                u_lo = max(c * U // S, ps) - ps
                u_hi = min((c + 1) * U // S, ps + units[b]) - ps
                for r in range(R):
                    t, g = divmod(r, G)
                    vis = lens[b] - T + t + 1
                    lo, hi = u_lo * 128, min(u_hi * 128, vis)
                    if hi <= lo:
                        continue
                    jobs.append((k[lo:], v[lo:], h, hi - lo, q[b * T + t, h * G + g]))
                    where.append((c + b * Hkv + h, r, b, t, h * G + g))
        start += units[b] * Hkv
    out, lse, psum = oracle.attention_rows(jobs, Hkv, D, wl.sm_scale)
    assert np.all(np.abs(psum - 1) < 1e-9)
    top = np.full((B, T, Hq), -np.inf)
    for (slot, r, b, t, hq), l in zip(where, lse):
        top[b, t, hq] = max(top[b, t, hq], l)
    for (slot, r, b, t, hq), o, l in zip(where, out, lse):
        ws_o[slot, r] = o
        ws_lse[slot, r] = l * LOG2E
        w = np.exp(l - top[b, t, hq])
        wsum[b, t, hq] += w
        wabs[b, t, hq] += w * np.abs(o)
    return ws_o, ws_lse, wabs / wsum[..., None]


@pytest.mark.parametrize("S", [3, 8, 37])
def test_combine_of_exact_partials_is_correctly_rounded(S):
    wl = W.small("combine", 2, 12, 2, 256, 3, [2100, 700], seed=21)
    B, Hkv, Hq, D, T = wl.batch, wl.num_kv_heads, wl.num_q_heads, wl.head_dim, wl.T
    ws_o, ws_lse, A = _partials(wl, S)
    total = nv.nvkv_decode_workspace_bytes(B, T, Hq, Hkv, D, S)
    o_bytes = (ws_o.nbytes + 255) // 256 * 256
    host = np.zeros(total, np.uint8)
    host[:ws_o.nbytes] = ws_o.reshape(-1).view(np.uint8)
    host[o_bytes:o_bytes + ws_lse.nbytes] = ws_lse.reshape(-1).view(np.uint8)
    dev = torch.device("cuda")
    ws = torch.from_numpy(host).to(dev)
    max_len = int(max(wl.kv_lens))
    pt = torch.zeros((B, (max_len + 15) // 16), dtype=torch.int32, device=dev)  # unread by the merge
    lens = torch.from_numpy(np.asarray(wl.kv_lens, np.int32)).to(dev)
    seqs = nv.Seqs(pt, lens, max_len)
    out = torch.full((B * T, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    nv.nvkv_combine(seqs, ws, T, Hq, Hkv, D, S, out)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().astype(np.float64).reshape(B, T, Hq, D)

    q = wl.queries()
    jobs = []
    for b in range(B):
        k, v = wl.kv_rows(b, 0, int(wl.kv_lens[b]))
        for t in range(T):
            for hq in range(Hq):
                jobs.append((k, v, hq // wl.group, wl.query_position(b, t) + 1, q[b * T + t, hq]))
    ref, _, _ = oracle.attention_rows(jobs, Hkv, D, wl.sm_scale)
    ref = ref.reshape(B, T, Hq, D)
    delta = 1.2e-5 * A
    lo = _bf16_rne(ref - delta)
    hi = _bf16_rne(ref + delta)
    assert np.isfinite(got).all()
    ok = (got >= lo) & (got <= hi)
    assert ok.all(), (f"{int((~ok).sum())} elements outside the correctly rounded interval; "
                      f"worst |got-ref| / delta {(np.abs(got - ref) / delta).max():.2f}")
    # the check is not vacuous: almost every element has exactly one
    # admissible bf16 value, the correctly rounded oracle value
    assert (lo == hi).mean() > 0.95
