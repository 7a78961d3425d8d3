"""Pins of the oracle's rotary-embedding additions (CPU): the (cos, sin)
table, the float rotation the fused append applies to K, the float-input
group quantiser, and the rotating append.  Each is checked against something
other than its own formula: special positions and frequencies in closed
form, the relative-position property of rotations, the bf16 quantiser and an
independent table-scan quantiser, and the plain append."""
import numpy as np
import pytest

import oracle

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])


def test_table_position_zero_is_identity_and_rows_are_unit():
    cs = oracle.rope_table(64, 128, 1e6, 3.0)
    assert (cs[0, :, 0] == 1).all() and (cs[0, :, 1] == 0).all()
    n = cs[..., 0].astype(np.float64) ** 2 + cs[..., 1].astype(np.float64) ** 2
    assert np.abs(n - 1).max() < 2 ** -22


def test_table_linear_scaling_divides_positions():
    """Scale s at position s*p is the unscaled table at position p."""
    a = oracle.rope_table(200, 64, 1e4, 2.0)
    b = oracle.rope_table(100, 64, 1e4, 1.0)
    assert np.array_equal(a[0::2], b)


def test_table_frequencies_in_closed_form():
    base, r, s = 1e4, 64, 1.0
    cs = oracle.rope_table(300, r, base, s)
    # pair 0 turns by one radian per position; pair r/4 by base^(-1/2) = 1/100
    p = np.arange(300)
    assert np.allclose(cs[:, 0, 0], np.cos(p), atol=1e-7)
    assert np.allclose(cs[:, 0, 1], np.sin(p), atol=1e-7)
    assert np.allclose(cs[:, r // 4, 0], np.cos(p / 100.0), atol=1e-7)
    assert np.allclose(cs[:, r // 4, 1], np.sin(p / 100.0), atol=1e-7)


def _bits(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_rotation_direction_and_pass_through():
    D, r = 256, 64
    cs = oracle.rope_table(10, r, 1e4, 1.0)
    row = np.zeros(D, np.float32)
    row[0] = 1.0   # unit vector along element 0 (paired with element r/2)
    row[200] = 5.0  # beyond rotary_dim: untouched
    out = oracle.rope_rotate_f32(_bits(row), r, cs[3])
    c, s = cs[3, 0]
    assert out[0] == c and out[r // 2] == s  # x' = x cos - y sin, y' = y cos + x sin
    assert out[200] == 5.0
    assert (out[r:200] == 0).all() and (out[201:] == 0).all()
    assert np.array_equal(oracle.rope_rotate_f32(_bits(row), r, cs[0]), row)  # position 0


def test_rotation_keeps_relative_position_scores():
    """<R(p) q, R(p') k> depends on p - p' only (the property RoPE exists for):
    a wrong pairing or sign breaks it."""
    rng = np.random.default_rng(5)
    D, r = 256, 128
    cs = oracle.rope_table(2000, r, 1e4, 2.0)
    q = _bits(rng.standard_normal(D))
    k = _bits(rng.standard_normal(D))
    def score(p, pk):
        return float(np.dot(oracle.rope_rotate_f32(q, r, cs[p]).astype(np.float64),
                            oracle.rope_rotate_f32(k, r, cs[pk]).astype(np.float64)))
    base = score(17, 5)
    for shift in (1, 100, 1500):
        assert abs(score(17 + shift, 5 + shift) - base) < 1e-4 * (1 + abs(base))
    # and it does depend on the difference
    assert abs(score(17, 6) - base) > 1e-3


def test_rotation_preserves_pair_norms():
    rng = np.random.default_rng(6)
    D, r = 256, 256
    cs = oracle.rope_table(500, r, 1e6, 2.12)
    row = _bits(rng.standard_normal(D) * 3)
    x = row.astype(np.uint32) << 16
    x = x.view(np.float32).astype(np.float64)
    out = oracle.rope_rotate_f32(row, r, cs[457]).astype(np.float64)
    h = r // 2
    n0 = x[:h] ** 2 + x[h:r] ** 2
    n1 = out[:h] ** 2 + out[h:r] ** 2
    assert np.allclose(n0, n1, rtol=1e-6, atol=1e-12)


def test_float_rotation_is_within_two_roundings_of_the_exact_rotation():
    """The float rotation against the rotation evaluated in float64 from the
    same (float) bf16 inputs and table entries, element by element.  The
    float evaluation x' = fma(x, c, -(y*s)) rounds twice: the product y*s
    (at most half an ulp of |y*s|) and the fused multiply-add (at most half
    an ulp of the result), so |x'_float - x'_exact| <= 2^-24 (|y*s| + |x'|)
    (half an ulp of v is at most 2^-24 |v| for normal floats); the same holds
    for y' = fma(y, c, x*s) with x*s.  A wrong pairing, sign or table index
    misses by far more than this bound."""
    rng = np.random.default_rng(11)
    D = 256
    for r, base, scale in ((256, 1e7, 2.12), (64, 1e4, 1.0), (128, 5e5, 3.0)):
        cs = oracle.rope_table(3000, r, base, scale)
        h = r // 2
        for pos in (0, 1, 17, 999, 2999):
            bits = _bits(rng.standard_normal(D) * 10.0 ** rng.uniform(-2, 2, D))
            x = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            c = cs[pos, :, 0].astype(np.float64)
            s = cs[pos, :, 1].astype(np.float64)
            got = oracle.rope_rotate_f32(bits, r, cs[pos]).astype(np.float64)
            a, b = x[:h], x[h:r]
            want_a = a * c - b * s
            want_b = b * c + a * s
            bound_a = 2.0 ** -24 * (np.abs(b * s) + np.abs(want_a)) * (1 + 2.0 ** -20) + 2.0 ** -140
            bound_b = 2.0 ** -24 * (np.abs(a * s) + np.abs(want_b)) * (1 + 2.0 ** -20) + 2.0 ** -140
            assert (np.abs(got[:h] - want_a) <= bound_a).all()
            assert (np.abs(got[h:r] - want_b) <= bound_b).all()
            assert np.array_equal(got[r:], x[r:])


def _scan_quantize(x):
    """Independent formulation: the E4M3 value nearest to amax/6 by scanning
    the finite E4M3 values (ties to the even mantissa), then the E2M1 value
    nearest to |x|/scale by scanning (ties to the even code)."""
    vals = np.array([oracle.e4m3_value(b) for b in range(127)])  # 0x00..0x7E
    amax = float(np.max(np.abs(np.asarray(x, np.float64))))
    t = amax / 6.0
    dist = np.abs(vals - t)
    cand = np.flatnonzero(dist == dist.min())
    sb = int(cand[0]) if len(cand) == 1 else int([c for c in cand if c % 2 == 0][0])
    if t > 448:
        sb = 0x7E
    scale = vals[sb]
    codes = np.zeros(16, np.uint8)
    if scale > 0:
        for i, xv in enumerate(np.asarray(x, np.float64)):
            d = np.abs(E2M1 * scale - abs(xv))
            c = np.flatnonzero(d == d.min())
            idx = int(c[0]) if len(c) == 1 else int([j for j in c if j % 2 == 0][0])
            codes[i] = 0 if idx == 0 else ((8 if xv < 0 else 0) | idx)
    return codes, sb


def test_float_quantiser_matches_bf16_quantiser_on_bf16_values():
    rng = np.random.default_rng(7)
    for _ in range(3000):
        bits = _bits(rng.standard_normal(16) * 10.0 ** rng.uniform(-3, 2))
        f = (bits.astype(np.uint32) << 16).view(np.float32)
        c1, s1 = oracle.quantize_group(bits)
        c2, s2 = oracle.quantize_group_f32(f)
        assert s1 == s2 and np.array_equal(c1, c2)


def test_float_quantiser_matches_table_scan_on_float_values():
    rng = np.random.default_rng(8)
    for _ in range(1500):
        x = (rng.standard_normal(16) * 10.0 ** rng.uniform(-2, 2)).astype(np.float32)
        c, s = oracle.quantize_group_f32(x)
        c2, s2 = _scan_quantize(x)
        assert s == s2 and np.array_equal(c, c2), (x, c, c2, s, s2)
    for x in (np.zeros(16, np.float32), np.full(16, 3000.0, np.float32)):
        c, s = oracle.quantize_group_f32(x)
        c2, s2 = _scan_quantize(x)
        assert s == s2 and np.array_equal(c, c2)


def _append_case(rng, Hkv=2, D=128, B=2, n=5, ctx=(40, 17)):
    pages_per = [(c + n + 15) // 16 for c in ctx]
    num_pages = sum(pages_per) + 2
    perm = rng.permutation(num_pages).astype(np.int32)
    pt = np.full((B, max(pages_per)), -1, np.int32)
    k0 = 0
    for b in range(B):
        pt[b, :pages_per[b]] = perm[k0:k0 + pages_per[b]]
        k0 += pages_per[b]
    lens = np.array([c + n for c in ctx], np.int32)
    cu = np.arange(B + 1, dtype=np.int32) * n
    k = _bits(rng.standard_normal((B * n, Hkv, D)))
    v = _bits(rng.standard_normal((B * n, Hkv, D)))
    return num_pages, pt, lens, cu, k, v


def test_rotating_append_with_no_rotary_dims_is_the_plain_append():
    rng = np.random.default_rng(9)
    Hkv, D = 2, 128
    num_pages, pt, lens, cu, k, v = _append_case(rng, Hkv, D)
    pb = oracle.page_bytes(Hkv, D)
    a = np.full(num_pages * pb, 0xA5, np.uint8)
    b = a.copy()
    oracle.append(a, Hkv, D, pt, lens, k, v, cu)
    oracle.append_rope(b, Hkv, D, pt, lens, k, v, cu, 0, oracle.rope_table(64, 32, 1e4, 1.0))
    assert np.array_equal(a, b)


def test_rotating_append_writes_the_rotated_rows_at_their_positions():
    rng = np.random.default_rng(10)
    Hkv, D, r = 2, 128, 64
    num_pages, pt, lens, cu, k, v = _append_case(rng, Hkv, D)
    cs = oracle.rope_table(128, r, 1e4, 2.0)
    pool = np.full(num_pages * oracle.page_bytes(Hkv, D), 0xA5, np.uint8)
    oracle.append_rope(pool, Hkv, D, pt, lens, k, v, cu, r, cs)
    n = cu[1] - cu[0]
    for b in range(2):
        for i in range(n):
            pos = lens[b] - n + i
            row = cu[b] + i
            for h in range(Hkv):
                rot = oracle.rope_rotate_f32(k[row, h], r, cs[pos])
                want = np.concatenate([
                    [oracle.dequant(c, s) for c in cc]
                    for cc, s in (oracle.quantize_group_f32(rot[16 * g:16 * g + 16])
                                  for g in range(D // 16))])
                got_k = oracle.pool_read_row(pool, Hkv, D, pt[b], pos, h, False)
                assert np.array_equal(got_k, want)
                got_v = oracle.pool_read_row(pool, Hkv, D, pt[b], pos, h, True)
                assert np.array_equal(got_v, oracle.qdq_rows(v[row, h][None])[0])
