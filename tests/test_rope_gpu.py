"""GPU parity of the fused RoPE + quantise-append (nvkv_rope_table,
nvkv_append_rope) against the float64 oracle: the (cos, sin) table within
one float ulp, and the pool written by the rotating append bit-exact against
the oracle's rotating append.  The append test builds its table with the
oracle and uploads it, so both sides rotate with the oracle's table and no
value computed on the GPU reaches the oracle; the GPU table kernel is
checked on its own by test_table_matches_oracle."""
import numpy as np
import pytest
import torch

import nvfp4_quantized_kv_b200 as nv
import oracle

pytestmark = pytest.mark.gpu


def _ulps(a, b):
    ai = a.astype(np.float32).view(np.int32).astype(np.int64)
    bi = b.astype(np.float32).view(np.int32).astype(np.int64)
    ai = np.where(ai < 0, np.int64(-2 ** 31) - ai, ai)
    bi = np.where(bi < 0, np.int64(-2 ** 31) - bi, bi)
    return np.abs(ai - bi)


@pytest.mark.parametrize("r,base,scale", [(64, 1e7, 2.12), (256, 1e4, 1.0), (128, 5e5, 3.0)])
def test_table_matches_oracle(r, base, scale):
    max_pos = 8192
    cs = torch.empty((max_pos, r // 2, 2), dtype=torch.float32, device="cuda")
    nv.nvkv_rope_table(cs, r, base, scale)
    torch.cuda.synchronize()
    got = cs.cpu().numpy()
    want = oracle.rope_table(max_pos, r, base, scale)
    # cos and sin are at most 1 in magnitude: the two double-precision
    # evaluations (GPU and host libraries) may differ by a few double ulps of
    # the angle, which after rounding to float is at most about one float ulp
    # of 1 -- measured as an absolute difference (near a zero of cos or sin a
    # count of float ulps of the tiny value is meaningless).
    assert np.abs(got.astype(np.float64) - want.astype(np.float64)).max() <= 2.0 ** -23
    assert (_ulps(got, want) == 0).mean() > 0.99
    assert (got[0, :, 0] == 1).all() and (got[0, :, 1] == 0).all()


def _bits(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _case(rng, Hkv, D, ctx, n):
    B = len(ctx)
    lens = np.array([c + k for c, k in zip(ctx, n)], np.int32)
    pages_per = [(int(l) + 15) // 16 for l in lens]
    num_pages = sum(pages_per) + 3
    perm = rng.permutation(num_pages).astype(np.int32)
    pt = np.full((B, max(pages_per)), -1, np.int32)
    k0 = 0
    for b in range(B):
        pt[b, :pages_per[b]] = perm[k0:k0 + pages_per[b]]
        k0 += pages_per[b]
    cu = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    rows = int(cu[-1])
    k = _bits(rng.standard_normal((rows, Hkv, D)) * np.where(rng.random(D) < 0.02, 10.0, 1.0))
    v = _bits(rng.standard_normal((rows, Hkv, D)))
    return num_pages, pt, lens, cu, k, v


def _run(rng, Hkv, D, ctx, n, r, max_pos, base=1e6, scale=2.12):
    num_pages, pt, lens, cu, k, v = _case(rng, Hkv, D, ctx, n)
    dev = torch.device("cuda")
    cache = nv.Cache.allocate(num_pages, Hkv, D, dev, fill=0xA5)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    seqs = nv.Seqs(torch.from_numpy(pt).to(dev), torch.from_numpy(lens).to(dev), int(lens.max()), err)
    table = oracle.rope_table(max_pos, r, base, scale)
    cs = torch.from_numpy(np.ascontiguousarray(table, dtype=np.float32)).to(dev)
    kt = torch.from_numpy(k.view(np.int16)).to(dev).view(torch.bfloat16)
    vt = torch.from_numpy(v.view(np.int16)).to(dev).view(torch.bfloat16)
    nv.nvkv_append_rope(cache, seqs, kt, vt, torch.from_numpy(cu).to(dev), int(cu[-1]), int(max(n)),
                        cs, r)
    torch.cuda.synchronize()
    want = np.full(num_pages * oracle.page_bytes(Hkv, D), 0xA5, np.uint8)
    oracle.append_rope(want, Hkv, D, pt, lens, k, v, cu, r, table)
    return cache.pool.cpu().numpy(), want, int(err.item())


@pytest.mark.parametrize("Hkv,D,r", [(4, 256, 256), (4, 256, 64), (2, 128, 32), (2, 128, 128)])
def test_rotating_append_is_bit_exact(Hkv, D, r):
    rng = np.random.default_rng(100 + r + D)
    got, want, err = _run(rng, Hkv, D, ctx=[301, 1000, 0], n=[37, 5, 16], r=r, max_pos=4096)
    assert err == 0
    assert np.array_equal(got, want)


def test_positions_without_a_table_row_are_reported_and_skipped():
    rng = np.random.default_rng(7)
    # sequence 1's new rows sit at positions 60..64; the table has 62 rows
    got, want, err = _run(rng, 2, 128, ctx=[10, 60], n=[3, 5], r=64, max_pos=62)
    assert err & nv.DEVERR_LENGTH
    assert np.array_equal(got, want)
