"""Pins of the oracle's K8V4 cache (CPU): K rows in E4M3 with one float
scale per row, V in NVFP4.  Checked against an independent float32 table
scan, the E4M3 error bound, the row-maximum rule, a restated reader of the
documented page layout, and attention consistency between the row and the
pool forms."""
import numpy as np
import pytest

import oracle

E4M3_POS = np.array([oracle.e4m3_value(b) for b in range(127)])  # 0x00 .. 0x7E


def _bits(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _scan_k8(bits):
    """Independent formulation: float32 scale amax/448 and float32 quotients
    (numpy float32 arithmetic is IEEE round-to-nearest-even), then the E4M3
    value nearest to |q| by scanning the finite values, ties to the even
    byte (even mantissa), saturating at 448."""
    x = _f32(bits)
    amax = np.float32(np.max(np.abs(x)))
    sc = np.float32(amax / np.float32(448.0))
    codes = np.zeros(len(x), np.uint8)
    if sc == 0:
        return codes, float(sc)
    q = (x / sc).astype(np.float32)
    for i, qi in enumerate(q):
        a = abs(float(qi))
        if a >= 448:
            b = 0x7E
        else:
            dist = np.abs(E4M3_POS - a)
            cand = np.flatnonzero(dist == dist.min())
            b = int(cand[0]) if len(cand) == 1 else int([c for c in cand if c % 2 == 0][0])
        codes[i] = 0 if b == 0 else (b | (0x80 if qi < 0 else 0))
    return codes, float(sc)


def test_row_quantiser_matches_table_scan():
    rng = np.random.default_rng(31)
    for _ in range(300):
        D = int(rng.choice([128, 256]))
        x = rng.standard_normal(D) * 10.0 ** rng.uniform(-3, 3)
        x[rng.integers(D, size=3)] *= 20  # outliers set the scale
        bits = _bits(x)
        c, s = oracle.k8_quantize_row(bits)
        c2, s2 = _scan_k8(bits)
        assert s == s2 and np.array_equal(c, c2)


def test_row_maximum_codes_to_448_and_error_bound():
    rng = np.random.default_rng(32)
    for _ in range(300):
        x = _bits(rng.standard_normal(256) * 10.0 ** rng.uniform(-4, 4))
        c, s = oracle.k8_quantize_row(x)
        xf = _f32(x).astype(np.float64)
        i = int(np.argmax(np.abs(xf)))
        assert (c[i] & 0x7F) == 0x7E
        deq = np.array([oracle.k8_dequant(int(b), s) for b in c])
        err = np.abs(deq - xf)
        # E4M3: 3 mantissa bits (relative half-ulp 2^-4) above 2^-6, absolute
        # half-ulp 2^-10 below, in units of the scale; plus the float quotient
        assert (err <= np.abs(xf) * (2 ** -4 + 2 ** -20) + s * 2 ** -10 * 1.0001).all()


def test_zero_row_and_negative_zero():
    c, s = oracle.k8_quantize_row(np.zeros(128, np.uint16))
    assert s == 0.0 and (c == 0).all()
    x = np.zeros(128, np.float32)
    x[5] = 1.0
    x[6] = -1e-30  # rounds to zero against the row's scale
    c, s = oracle.k8_quantize_row(_bits(x))
    assert c[6] == 0 and c[5] == 0x7E
    assert (np.delete(c, 5) == 0).all()


def _layout_read(pool, Hkv, D, page, h, s):
    """Restated reader of the documented K8V4 page layout."""
    base = (page * Hkv + h) * (25 * D + 64)
    kc = pool[base + s * D: base + s * D + D]
    ks = pool[base + 16 * D + 4 * s: base + 16 * D + 4 * s + 4].view(np.float32)[0]
    k = np.array([oracle.e4m3_value(int(b)) for b in kc]) * np.float64(ks)
    vbytes = pool[base + 16 * D + 64 + np.arange(D) * 8 + (s >> 1)]
    vcode = (vbytes >> 4) if (s & 1) else (vbytes & 15)
    vs = pool[base + 24 * D + 64 + (np.arange(D) // 16) * 16 + s]
    v = np.array([oracle.dequant(int(c), int(b)) for c, b in zip(vcode, vs)])
    return k, v


def test_append_layout_and_reader():
    rng = np.random.default_rng(33)
    Hkv, D, B, n = 2, 128, 2, 7
    ctx = [30, 9]
    lens = np.array([c + n for c in ctx], np.int32)
    pages_per = [(int(l) + 15) // 16 for l in lens]
    num_pages = sum(pages_per) + 1
    perm = rng.permutation(num_pages).astype(np.int32)
    pt = np.full((B, max(pages_per)), -1, np.int32)
    pt[0, :pages_per[0]] = perm[:pages_per[0]]
    pt[1, :pages_per[1]] = perm[pages_per[0]:pages_per[0] + pages_per[1]]
    cu = np.array([0, n, 2 * n], np.int32)
    k = _bits(rng.standard_normal((B * n, Hkv, D)))
    v = _bits(rng.standard_normal((B * n, Hkv, D)))
    assert oracle.k8v4_page_bytes(Hkv, D) == Hkv * (25 * D + 64)
    pool = np.full(num_pages * oracle.k8v4_page_bytes(Hkv, D), 0xA5, np.uint8)
    oracle.append_k8v4(pool, Hkv, D, pt, lens, k, v, cu)
    touched = np.zeros_like(pool, dtype=bool)
    for b in range(B):
        for i in range(n):
            pos = int(lens[b]) - n + i
            row = cu[b] + i
            page, s = pt[b, pos // 16], pos % 16
            for h in range(Hkv):
                kr, vr = _layout_read(pool, Hkv, D, page, h, s)
                c, sc = oracle.k8_quantize_row(k[row, h])
                want_k = np.array([oracle.k8_dequant(int(x), sc) for x in c])
                assert np.array_equal(kr, want_k)
                assert np.array_equal(vr, oracle.qdq_rows(v[row, h][None])[0])
                assert np.array_equal(oracle.k8v4_read_row(pool, Hkv, D, pt[b], pos, h, False), kr)
                assert np.array_equal(oracle.k8v4_read_row(pool, Hkv, D, pt[b], pos, h, True), vr)
                base = (page * Hkv + h) * (25 * D + 64)
                touched[base + s * D: base + s * D + D] = True
                touched[base + 16 * D + 4 * s: base + 16 * D + 4 * s + 4] = True
                touched[base + 16 * D + 64 + np.arange(D) * 8 + (s >> 1)] = True
                touched[base + 24 * D + 64 + np.arange(D // 16) * 16 + s] = True
    # every byte outside the written slots keeps the sentinel (shared V bytes
    # of a half-written pair keep the other slot's nibble: 0x5 of 0xA5)
    assert (pool[~touched] == 0xA5).all()


def test_attention_rows_and_pool_forms_agree():
    rng = np.random.default_rng(34)
    Hkv, D, T = 2, 128, 1
    L = 70
    k = _bits(rng.standard_normal((L, Hkv, D)))
    v = _bits(rng.standard_normal((L, Hkv, D)))
    pages = (L + 15) // 16
    pt = rng.permutation(pages).astype(np.int32)[None]
    pool = np.zeros(pages * oracle.k8v4_page_bytes(Hkv, D), np.uint8)
    oracle.append_k8v4(pool, Hkv, D, pt, np.array([L], np.int32), k, v, np.array([0, L], np.int32))
    q = [_bits(rng.standard_normal(D)) for _ in range(4)]
    jobs_r = [(k, v, j % Hkv, L - 3 * j, q[j]) for j in range(4)]
    jobs_p = [(pt[0], j % Hkv, L - 3 * j, q[j]) for j in range(4)]
    a, la, pa = oracle.attention_rows(jobs_r, Hkv, D, 0.088, k8=True)
    b, lb, pb = oracle.attention_pool(pool, Hkv, D, jobs_p, 0.088, k8=True)
    assert np.array_equal(a, b) and np.array_equal(la, lb)
    assert np.all(np.abs(pa - 1) < 1e-12)
    # one visible key returns its (dequantised) value row
    one, _, _ = oracle.attention_rows([(k, v, 1, 1, q[0])], Hkv, D, 0.088, k8=True)
    assert np.array_equal(one[0], oracle.qdq_rows(v[0, 1][None])[0])
    # K in the 8-bit format differs from NVFP4 K, V is the same format
    c, _, _ = oracle.attention_rows(jobs_r, Hkv, D, 0.088, k8=False)
    assert not np.array_equal(a, c)


def test_attention_invariants_with_8bit_keys():
    """Closed forms of softmax attention that hold whatever the key format:
    a zero query and equal key rows both give the mean of the dequantised
    values; one key whose score dominates gives its value row; the lse of a
    single key is its score, computed here from the 8-bit dequantised row."""
    rng = np.random.default_rng(35)
    Hkv, D, n = 2, 128, 33
    k = _bits(rng.standard_normal((n, Hkv, D)) * 4)
    v = _bits(rng.standard_normal((n, Hkv, D)))
    vmean = oracle.qdq_rows(v[:, 1]).mean(axis=0)
    zero_q = np.zeros(D, np.uint16)
    out, _, _ = oracle.attention_rows([(k, v, 1, n, zero_q)], Hkv, D, 0.088, k8=True)
    assert np.allclose(out[0], vmean, rtol=0, atol=1e-13)
    keq = np.repeat(k[:1], n, axis=0)
    q = _bits(rng.standard_normal(D))
    out, _, _ = oracle.attention_rows([(keq, v, 1, n, q)], Hkv, D, 0.088, k8=True)
    assert np.allclose(out[0], vmean, rtol=0, atol=1e-13)
    kd = _bits(rng.standard_normal((n, Hkv, D)) * 0.01)
    kd[13, 0] = _bits(np.full(D, 8.0))
    qd = _bits(np.full(D, 4.0))
    out, _, _ = oracle.attention_rows([(kd, v, 0, n, qd)], Hkv, D, 1 / np.sqrt(D), k8=True)
    assert np.allclose(out[0], oracle.qdq_rows(v[13, 0][None])[0], rtol=0, atol=1e-60)
    out, lse, _ = oracle.attention_rows([(k, v, 1, 1, q)], Hkv, D, 0.088, k8=True)
    c, sc = oracle.k8_quantize_row(k[0, 1])
    krow = np.array([oracle.k8_dequant(int(x), sc) for x in c])
    qf = _f32(q).astype(np.float64)
    assert abs(lse[0] - 0.088 * float(np.dot(qf, krow))) < 1e-12
