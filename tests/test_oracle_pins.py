"""Pins for the float64 oracle (CPU only).

Each test checks the oracle against something other than itself: the
E2M1 / E4M3 definitions and torch's float8 decoding, a table-scan
formulation of round-to-nearest-even that never divides, closed-form
attention cases, and a pure-Python brute force on tiny inputs.  The pages
print no worked example for the NVFP4 KV path (see
tests/golden/nvfp4_format.txt for everything they do state).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

E2M1_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def torch_e4m3_table():
    """All 256 E4M3FN byte values, decoded by torch (a library routine)."""
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def bf16_vals(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16_bits_exact(x):
    """float64 -> bf16 bits, asserting the value is exactly representable."""
    f = np.asarray(x, np.float64).astype(np.float32)
    assert np.array_equal(f.astype(np.float64), np.asarray(x, np.float64))
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(bf16_vals(bits), np.asarray(x, np.float64))
    return bits


def scan_e4m3(targets):
    """Nearest finite non-negative E4M3 byte to each target >= 0, ties to
    the even byte, by scanning the torch-decoded table (no division)."""
    tab = torch_e4m3_table()[:0x7F]  # bytes 0x00..0x7E, 0 .. 448
    t = np.asarray(targets, np.float64)[:, None]
    dist = np.abs(tab[None, :] - t)
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    # among the (at most two) nearest, prefer the even byte
    even = cand & ((np.arange(0x7F) % 2) == 0)[None, :]
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    return pick.astype(np.uint8)


def scan_scale_from_amax(amax):
    """Scale byte nearest to amax/6, compared as |6 v - amax| (no division).
    Targets far above the largest value (448) are clipped first: the nearest
    value of a sorted table to anything above its top is the top, and the
    clip keeps the float64 distances from collapsing for amax ~ 1e38."""
    tab = torch_e4m3_table()[:0x7F]
    a = np.minimum(np.asarray(amax, np.float64), 1e6)[:, None]
    dist = np.abs(6.0 * tab[None, :] - a)
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    even = cand & ((np.arange(0x7F) % 2) == 0)[None, :]
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    return pick.astype(np.uint8)


def scan_codes(x, scale):
    """E2M1 code for x given the group scale, by scanning |m*scale - |x||
    over the eight magnitudes; ties to the even index; sign from x unless
    the magnitude index is 0."""
    x = np.asarray(x, np.float64)
    s = np.asarray(scale, np.float64)
    dist = np.abs(E2M1_MAGS[None, :] * s[:, None] - np.abs(x)[:, None])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    even = cand & ((np.arange(8) % 2) == 0)[None, :]
    idx = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    idx = np.where(s == 0, 0, idx)
    neg = np.signbit(x)
    return np.where(idx == 0, 0, idx + 8 * neg).astype(np.uint8)


# ---------------------------------------------------------------------------
# formats
# ---------------------------------------------------------------------------
def test_e2m1_table_is_the_e2m1_value_set():
    vals = [oracle.e2m1_value(c) for c in range(16)]
    assert vals[:8] == list(E2M1_MAGS)
    assert vals[8:] == [-v for v in E2M1_MAGS]
    assert math.copysign(1.0, vals[8]) == -1.0  # code 8 decodes to -0


def test_e4m3_table_matches_torch_float8():
    tab = torch_e4m3_table()
    mine = np.array([oracle.e4m3_value(b) for b in range(256)])
    nan = np.isnan(tab)
    assert np.array_equal(nan, np.isnan(mine))
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(tab[~nan], mine[~nan])
    assert mine[0x7E] == 448.0 and mine[0x08] == 2.0 ** -6 and mine[0x01] == 2.0 ** -9


def test_bf16_decoding():
    bits = np.arange(0, 65536, 97, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    mine = np.array([oracle.bf16_value(b) for b in bits])
    fin = np.isfinite(ref)
    assert np.array_equal(ref[fin], mine[fin])


# ---------------------------------------------------------------------------
# rounding
# ---------------------------------------------------------------------------
def all_nonneg_finite_bf16():
    return np.arange(0, 0x7F80, dtype=np.uint32).astype(np.uint16)


def test_scale_exhaustive_over_every_bf16_amax():
    """Every non-negative finite bf16 amax: oracle scale byte (through the
    quantiser) == table scan of |6 v - amax|."""
    amax_bits = all_nonneg_finite_bf16()
    groups = np.zeros((amax_bits.size, 16), np.uint16)
    groups[:, 5] = amax_bits  # amax anywhere in the group
    _, scales = oracle.quantize_rows(groups)
    expect = scan_scale_from_amax(bf16_vals(amax_bits))
    assert np.array_equal(scales[:, 0], expect)


def test_scale_rounding_matches_torch_below_overflow():
    """torch's float64 -> float8_e4m3fn conversion is round-to-nearest-even;
    it overflows to NaN above 464, so compare below that and check the
    saturating reading separately."""
    amax = bf16_vals(all_nonneg_finite_bf16())
    x = amax / 6.0
    keep = x < 448.0
    ref = torch.from_numpy(x[keep]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([oracle.e4m3_round(v) for v in x[keep]], np.uint8)
    assert np.array_equal(ref, mine)
    for v in (448.0, 449.0, 464.0, 465.0, 1e6, 3.3e38 / 6):
        assert oracle.e4m3_round(v) == 0x7E


def test_e4m3_ties_go_to_even_mantissa():
    tab = torch_e4m3_table()[:0x7F]
    mids = (tab[:-1] + tab[1:]) / 2.0
    got = np.array([oracle.e4m3_round(m) for m in mids], np.uint8)
    lo = np.arange(0x7E, dtype=np.uint8)
    expect = np.where(lo % 2 == 0, lo, lo + 1)
    assert np.array_equal(got, expect)
    # just off the midpoint goes to the nearer neighbour
    up = np.array([oracle.e4m3_round(np.nextafter(m, np.inf)) for m in mids], np.uint8)
    dn = np.array([oracle.e4m3_round(np.nextafter(m, -np.inf)) for m in mids], np.uint8)
    assert np.array_equal(up, lo + 1) and np.array_equal(dn, lo)
    assert np.array_equal(scan_e4m3(mids), expect)


def test_e2m1_rounding_ties_and_neighbours():
    mids = (E2M1_MAGS[:-1] + E2M1_MAGS[1:]) / 2  # .25 .75 1.25 1.75 2.5 3.5 5
    got = [oracle.e2m1_round_index(m) for m in mids]
    assert [E2M1_MAGS[i] for i in got] == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    for i, m in enumerate(mids):
        assert oracle.e2m1_round_index(np.nextafter(m, np.inf)) == i + 1
        assert oracle.e2m1_round_index(np.nextafter(m, -np.inf)) == i
    for i, v in enumerate(E2M1_MAGS):
        assert oracle.e2m1_round_index(v) == i
    for v in (6.0, 6.5, 7.0, 8.0, 100.0):
        assert oracle.e2m1_round_index(v) == 7


def test_e2m1_rounding_random_vs_scan():
    rng = np.random.default_rng(5)
    r = np.concatenate([rng.uniform(0, 8, 20000), rng.uniform(0, 1, 5000)])
    got = np.array([oracle.e2m1_round_index(v) for v in r])
    expect = scan_codes(r, np.ones_like(r))
    assert np.array_equal(got, expect)


def test_codes_exhaustive_every_bf16_under_every_scale():
    """For every positive finite scale s, a group whose amax is 6 s (so its
    scale is s) and whose other 15 entries sweep every bf16 x with
    |x| <= 6 s, both signs: oracle codes == table scan."""
    tab = torch_e4m3_table()
    all_pos = bf16_vals(all_nonneg_finite_bf16())
    all_bits = all_nonneg_finite_bf16()
    total = 0
    for sb in range(1, 0x7F):
        s = tab[sb]
        amax_bits = f64_to_bf16_bits_exact(np.array([6.0 * s]))[0]
        xs = all_bits[all_pos <= 6.0 * s]
        xs = np.concatenate([xs, xs | np.uint16(0x8000)])
        n = -(-xs.size // 15)
        fill = np.zeros(n * 15, np.uint16)
        fill[:xs.size] = xs
        groups = np.concatenate([np.full((n, 1), amax_bits, np.uint16), fill.reshape(n, 15)], 1)
        codes, scales = oracle.quantize_rows(groups)
        assert np.all(scales == sb)
        expect = scan_codes(bf16_vals(groups.reshape(-1)), np.full(groups.size, s))
        assert np.array_equal(codes.reshape(-1), expect), f"scale byte {sb:#x}"
        total += groups.size
    assert total > 4_000_000  # ~4.5M (x, scale) pairs


def test_hand_worked_group():
    """amax = 6 gives scale 1.0 (byte 0x38); the E2M1 midpoints then land
    exactly on ties."""
    x = np.array([6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -5, -0.25, -0.0, 0.0,
                  5.5, -3.0, 0.5, 0.1875], np.float64)
    bits = f64_to_bf16_bits_exact(x)
    codes, sb = oracle.quantize_group(bits)
    assert sb == 0x38 and oracle.e4m3_value(sb) == 1.0
    #            6  .25 .75 1.25 1.75 2.5 3.5 5   -5   -.25 -0 0 5.5 -3 .5  .1875
    expect = [7, 0, 2, 2, 4, 4, 6, 6, 14, 0, 0, 0, 7, 13, 1, 0]
    assert list(codes) == expect


def test_zero_and_tiny_groups():
    codes, sb = oracle.quantize_group(np.zeros(16, np.uint16))
    assert sb == 0 and not codes.any()
    neg0 = np.full(16, 0x8000, np.uint16)
    codes, sb = oracle.quantize_group(neg0)
    assert sb == 0 and not codes.any()
    # amax/6 == 2^-10 exactly: a tie between 0 and 2^-9 -> 0 (even)
    x = np.zeros(16, np.uint16)
    x[0] = f64_to_bf16_bits_exact(np.array([6 * 2.0 ** -10]))[0]
    codes, sb = oracle.quantize_group(x)
    assert sb == 0 and not codes.any()
    # just above the tie -> scale 2^-9, code of 6*2^-10 / 2^-9 = 3 -> index 5
    x[0] = f64_to_bf16_bits_exact(np.array([6 * 2.0 ** -10 * (1 + 2 ** -6)]))[0]
    codes, sb = oracle.quantize_group(x)
    assert sb == 0x01 and codes[0] == 5


def test_round_trip_requantisation():
    """Requantising a dequantised group returns the same codes and scale
    whenever its largest code magnitude is 6 or it is all zero; that always
    holds for a normal scale.  The exception lives in the subnormal-scale
    corner."""
    rng = np.random.default_rng(11)
    n = 50000
    x = rng.standard_normal((n, 16)).astype(np.float32)
    x[: n // 4, 3] *= 10.0
    x *= (2.0 ** rng.integers(-14, 9, size=(n, 1))).astype(np.float32)
    x[::97] = 0.0
    bits = (torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    codes, scales = oracle.quantize_rows(bits)
    tab = torch_e4m3_table()
    deq = E2M1_MAGS[codes & 7] * np.where(codes & 8, -1.0, 1.0) * tab[scales]
    codes2, scales2 = oracle.quantize_rows(f64_to_bf16_bits_exact(deq))
    maxidx = (codes & 7).max(axis=1)
    pre = (maxidx == 7) | (scales[:, 0] == 0)
    assert np.all(pre[scales[:, 0] >= 0x08])  # normal scale => max code 6
    assert np.array_equal(codes[pre], codes2[pre]) and np.array_equal(scales[pre], scales2[pre])
    # the known exception: amax = 3.0625 * 2^-9 -> scale 2^-9, top code 3;
    # requantised amax/6 = 2^-10 ties to scale 0
    g = np.zeros(16, np.uint16)
    g[0] = f64_to_bf16_bits_exact(np.array([3.0625 * 2.0 ** -9]))[0]
    c, s = oracle.quantize_group(g)
    assert s == 0x01 and c[0] == 5
    g2 = np.zeros(16, np.uint16)
    g2[0] = f64_to_bf16_bits_exact(np.array([3 * 2.0 ** -9]))[0]
    c2, s2 = oracle.quantize_group(g2)
    assert s2 == 0 and not c2.any()


def test_dequantised_values_fit_bf16_and_f16_exactly():
    tab = torch_e4m3_table()
    for sb in range(0x7F):
        for c in range(16):
            v = oracle.dequant(c, sb)
            assert v == E2M1_MAGS[c & 7] * (-1 if c & 8 else 1) * tab[sb]
            assert float(torch.tensor(v, dtype=torch.float64).to(torch.bfloat16).double()) == v
            assert float(torch.tensor(v, dtype=torch.float64).to(torch.float16).double()) == v


# ---------------------------------------------------------------------------
# format arithmetic vs the pages' statement
# ---------------------------------------------------------------------------
def read_golden(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            out[k] = v
    return out


def test_bits_per_element_and_saving_vs_int8():
    g = read_golden("nvfp4_format.txt")
    for hkv, d in ((2, 128), (4, 256), (8, 64)):
        pb = oracle.page_bytes(hkv, d)
        bits = pb * 8 / (16 * hkv * d * 2)
        assert bits == int(g["code_bits"]) + int(g["scale_bits"]) / int(g["group_size"]) == 4.5
    int8_bits = 8 + int(g["int8_scale_bits"]) / int(g["int8_group_size"])
    saving = 100 * (1 - 4.5 / int8_bits)
    assert round(saving) == int(g["kv_saving_vs_int8_percent"])


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------
def rand_bits(rng, shape, scale=1.0):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def run(k, v, h, nvis, q, D, Hkv, sm=None):
    sm = 1 / math.sqrt(D) if sm is None else sm
    out, lse, psum = oracle.attention_rows([(k, v, h, nvis, q)], Hkv, D, sm, nthreads=1)
    return out[0], lse[0], psum[0]


def test_softmax_weights_sum_to_one():
    rng = np.random.default_rng(1)
    Hkv, D, n = 2, 64, 300
    k, v = rand_bits(rng, (n, Hkv, D), 3.0), rand_bits(rng, (n, Hkv, D))
    q = rand_bits(rng, (D,), 2.0)
    for nvis in (1, 2, 17, 300):
        _, _, psum = run(k, v, 1, nvis, q, D, Hkv)
        assert abs(psum - 1.0) < 1e-12


def test_single_visible_key_returns_its_value_row():
    rng = np.random.default_rng(2)
    Hkv, D = 2, 32
    k, v = rand_bits(rng, (5, Hkv, D)), rand_bits(rng, (5, Hkv, D))
    q = rand_bits(rng, (D,))
    out, lse, _ = run(k, v, 1, 1, q, D, Hkv)
    assert np.array_equal(out, oracle.qdq_rows(v[0, 1]))
    s = np.dot(bf16_vals(q), oracle.qdq_rows(k[0, 1])) / math.sqrt(D)
    assert abs(lse - s) < 1e-12


def test_zero_query_averages_values():
    rng = np.random.default_rng(3)
    Hkv, D, n = 1, 48, 40
    k, v = rand_bits(rng, (n, Hkv, D), 5.0), rand_bits(rng, (n, Hkv, D))
    q = np.zeros(D, np.uint16)
    out, _, _ = run(k, v, 0, n, q, D, Hkv)
    assert np.allclose(out, oracle.qdq_rows(v[:, 0]).mean(axis=0), rtol=0, atol=1e-13)


def test_equal_keys_average_values():
    rng = np.random.default_rng(4)
    Hkv, D, n = 2, 32, 25
    k = np.repeat(rand_bits(rng, (1, Hkv, D), 4.0), n, axis=0)
    v = rand_bits(rng, (n, Hkv, D))
    q = rand_bits(rng, (D,))
    out, _, _ = run(k, v, 0, n, q, D, Hkv)
    assert np.allclose(out, oracle.qdq_rows(v[:, 0]).mean(axis=0), rtol=0, atol=1e-13)


def test_one_dominant_key_selects_its_value():
    rng = np.random.default_rng(5)
    Hkv, D, n = 1, 32, 30
    k = rand_bits(rng, (n, Hkv, D), 0.01)
    v = rand_bits(rng, (n, Hkv, D))
    q = f64_to_bf16_bits_exact(np.full(D, 4.0))
    k[13, 0] = f64_to_bf16_bits_exact(np.full(D, 8.0))  # score 32*32/sqrt(32) ~ 181
    out, _, _ = run(k, v, 0, n, q, D, Hkv)
    assert np.allclose(out, oracle.qdq_rows(v[13, 0]), rtol=0, atol=1e-60)


def test_causal_visibility_ignores_later_rows():
    rng = np.random.default_rng(6)
    Hkv, D, n = 2, 32, 40
    k, v = rand_bits(rng, (n, Hkv, D)), rand_bits(rng, (n, Hkv, D))
    q = rand_bits(rng, (D,))
    a, _, _ = run(k, v, 1, 23, q, D, Hkv)
    k2, v2 = k.copy(), v.copy()
    k2[23:] = rand_bits(rng, (n - 23, Hkv, D), 9.0)
    v2[23:] = rand_bits(rng, (n - 23, Hkv, D), 9.0)
    b, _, _ = run(k2, v2, 1, 23, q, D, Hkv)
    assert np.array_equal(a, b)


def py_quant_group(xs):
    """Pure-Python quantiser for the brute force: table scans, no division."""
    tab = [v for v in torch_e4m3_table()[:0x7F]]
    amax = max(abs(x) for x in xs)
    best = None
    for b, v in enumerate(tab):
        d = abs(6 * v - amax)
        if best is None or d < best[0] or (d == best[0] and b % 2 == 0):
            best = (d, b, v)
    s = best[2]
    out = []
    for x in xs:
        if s == 0:
            out.append(0.0)
            continue
        bi = None
        for i, m in enumerate(E2M1_MAGS):
            d = abs(m * s - abs(x))
            if bi is None or d < bi[0] or (d == bi[0] and i % 2 == 0):
                bi = (d, i, m)
        out.append(math.copysign(bi[2] * s, x) if bi[2] else 0.0)
    return out


def test_brute_force_tiny_attention():
    rng = np.random.default_rng(8)
    D, Hkv = 16, 1
    for trial in range(40):
        n = int(rng.integers(1, 6))
        k = rand_bits(rng, (n, Hkv, D), float(rng.choice([0.01, 1.0, 30.0])))
        v = rand_bits(rng, (n, Hkv, D), float(rng.choice([0.001, 1.0, 100.0])))
        q = rand_bits(rng, (D,), 2.0)
        nvis = int(rng.integers(1, n + 1))
        out, lse, _ = run(k, v, 0, nvis, q, D, Hkv)
        qv = [float(x) for x in bf16_vals(q)]
        K = [py_quant_group([float(x) for x in bf16_vals(k[j, 0])]) for j in range(nvis)]
        V = [py_quant_group([float(x) for x in bf16_vals(v[j, 0])]) for j in range(nvis)]
        s = [sum(a * b for a, b in zip(qv, K[j])) / 4.0 for j in range(nvis)]
        m = max(s)
        w = [math.exp(x - m) for x in s]
        z = sum(w)
        ref = [sum(w[j] * V[j][d] for j in range(nvis)) / z for d in range(D)]
        assert np.allclose(out, ref, rtol=1e-12, atol=1e-300), trial
        assert abs(lse - (m + math.log(z))) < 1e-12


# ---------------------------------------------------------------------------
# page layout
# ---------------------------------------------------------------------------
def layout_reader(pool, Hkv, D, page, h, slot):
    """Independent restatement of the documented page layout."""
    base = page * 18 * Hkv * D + h * 18 * D
    kc = pool[base + slot * D // 2: base + (slot + 1) * D // 2]
    kcodes = np.empty(D, np.uint8)
    kcodes[0::2], kcodes[1::2] = kc & 15, kc >> 4
    ks = pool[base + 8 * D + slot * D // 16: base + 8 * D + (slot + 1) * D // 16]
    vc = pool[base + 9 * D: base + 17 * D].reshape(D, 8)[:, slot // 2]
    vcodes = (vc >> 4) if slot % 2 else (vc & 15)
    vs = pool[base + 17 * D: base + 18 * D].reshape(D // 16, 16)[:, slot]
    return kcodes, ks, vcodes.astype(np.uint8), vs


def test_pool_append_layout_and_untouched_bytes():
    rng = np.random.default_rng(9)
    Hkv, D, B = 2, 64, 3
    lens0 = [5, 16, 0]
    adds = [[6, 3], [1, 17], [33, 2]]  # two append calls per sequence
    maxp = 8
    npages = B * maxp + 3
    pt = rng.permutation(npages)[: B * maxp].reshape(B, maxp).astype(np.int32)
    pool = np.full(npages * oracle.page_bytes(Hkv, D), 0xA5, np.uint8)
    rows = {b: [] for b in range(B)}
    written = set()
    lens = list(lens0)
    # positions below lens0 are never written (treated as pre-existing)
    for step in range(2):
        ks, vs, cu = [], [], [0]
        for b in range(B):
            n = adds[b][step]
            k, v = rand_bits(rng, (n, Hkv, D), 2.0), rand_bits(rng, (n, Hkv, D))
            for i in range(n):
                rows[b].append((lens[b] + i, k[i], v[i]))
            ks.append(k)
            vs.append(v)
            lens[b] += n
            cu.append(cu[-1] + n)
        oracle.append(pool, Hkv, D, pt, np.array(lens, np.int32), np.concatenate(ks),
                      np.concatenate(vs), np.array(cu, np.int32))
    vbyte_nibbles = {}
    for b in range(B):
        for pos, k, v in rows[b]:
            page, slot = pt[b, pos // 16], pos % 16
            for h in range(Hkv):
                kcodes, ks, vcodes, vsc = layout_reader(pool, Hkv, D, page, h, slot)
                ck, sk = oracle.quantize_rows(k[h])
                cv, sv = oracle.quantize_rows(v[h])
                assert np.array_equal(kcodes, ck) and np.array_equal(ks, sk)
                assert np.array_equal(vcodes, cv) and np.array_equal(vsc, sv)
                assert np.array_equal(oracle.pool_read_row(pool, Hkv, D, pt[b], pos, h, False),
                                      oracle.qdq_rows(k[h]))
                assert np.array_equal(oracle.pool_read_row(pool, Hkv, D, pt[b], pos, h, True),
                                      oracle.qdq_rows(v[h]))
                base = page * 18 * Hkv * D + h * 18 * D
                written.update(range(base + slot * D // 2, base + (slot + 1) * D // 2))
                written.update(range(base + 8 * D + slot * D // 16, base + 8 * D + (slot + 1) * D // 16))
                for d in range(D):
                    off = base + 9 * D + d * 8 + slot // 2
                    vbyte_nibbles.setdefault(off, set()).add(slot % 2)
                written.update(base + 17 * D + g * 16 + slot for g in range(D // 16))
    for off, nibs in vbyte_nibbles.items():
        if nibs == {0}:
            assert pool[off] >> 4 == 0xA
        elif nibs == {1}:
            assert pool[off] & 15 == 0x5
        written.add(off)
    untouched = np.ones(pool.size, bool)
    untouched[list(written)] = False
    assert np.all(pool[untouched] == 0xA5)


def test_attention_over_pool_equals_attention_over_rows():
    rng = np.random.default_rng(10)
    Hkv, D, n = 2, 32, 45
    maxp = 3
    pt = np.array([[4, 0, 2]], np.int32)
    k, v = rand_bits(rng, (n, Hkv, D), 3.0), rand_bits(rng, (n, Hkv, D))
    pool = np.full(5 * oracle.page_bytes(Hkv, D), 0xA5, np.uint8)
    oracle.append(pool, Hkv, D, pt, np.array([n], np.int32), k, v, np.array([0, n], np.int32))
    jobs_r, jobs_p = [], []
    for h in range(Hkv):
        for nvis in (1, 16, 17, 45):
            q = rand_bits(rng, (D,))
            jobs_r.append((k, v, h, nvis, q))
            jobs_p.append((pt[0], h, nvis, q))
    a = oracle.attention_rows(jobs_r, Hkv, D, 0.3, nthreads=3)
    b = oracle.attention_pool(pool, Hkv, D, jobs_p, 0.3, nthreads=2)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
