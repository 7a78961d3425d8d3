"""GPU parity of nvkv_append: the pool bytes written by the CUDA kernel must
equal the oracle's pool image bit for bit (codes, scales, page placement,
untouched bytes and untouched V-code nibbles)."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_quantized_kv_b200 as nv
from nvfp4_quantized_kv_b200.harness import bf16_tensor
from nvfp4_quantized_kv_b200.workload import to_bf16_bits

pytestmark = pytest.mark.gpu
SENTINEL = 0xA5


def rand_bits(rng, shape, scale=1.0):
    return to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def run_appends(hkv, d, page_table, calls, num_pages):
    """calls: list of (kv_lens after the call, k rows, v rows, cu) in order.
    Runs them on the GPU and in the oracle; returns both pool images."""
    dev = torch.device("cuda")
    pb = nv.nvkv_page_bytes(hkv, d)
    cache = nv.Cache.allocate(num_pages, hkv, d, dev, fill=SENTINEL)
    ref = np.full(num_pages * pb, SENTINEL, np.uint8)
    pt = torch.from_numpy(page_table).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for lens, k, v, cu in calls:
        seqs = nv.Seqs(pt, torch.from_numpy(lens).to(dev), int(lens.max()), err)
        counts = np.diff(cu)
        nv.nvkv_append(cache, seqs, bf16_tensor(k, dev), bf16_tensor(v, dev),
                       torch.from_numpy(cu).to(dev), int(cu[-1]), int(counts.max()))
        oracle.append(ref, hkv, d, page_table, lens, k, v, cu)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return cache.pool.cpu().numpy(), ref


@pytest.mark.parametrize("hkv,d,batch,seed", [(2, 128, 1, 0), (4, 256, 3, 1), (1, 256, 5, 2),
                                              (3, 128, 4, 3)])
def test_append_sequence_matches_oracle(hkv, d, batch, seed):
    rng = np.random.default_rng(seed)
    maxp = 12
    num_pages = batch * maxp + 5
    page_table = rng.permutation(num_pages)[: batch * maxp].reshape(batch, maxp).astype(np.int32)
    lens = np.zeros(batch, np.int32)
    calls = []
    for step in range(6):
        counts = rng.integers(0, 40, size=batch).astype(np.int32)
        if step == 5:
            counts[:] = 1
        counts = np.minimum(counts, maxp * 16 - lens)
        lens = lens + counts
        cu = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        n = int(cu[-1])
        k = rand_bits(rng, (n, hkv, d), 3.0)
        v = rand_bits(rng, (n, hkv, d))
        calls.append((lens.copy(), k, v, cu))
    got, ref = run_appends(hkv, d, page_table, calls, num_pages)
    assert np.array_equal(got, ref), f"{(got != ref).sum()} bytes differ"


def test_append_every_bf16_amax():
    """One group per bf16 amax value (all 32640 non-negative finite ones),
    with both signs and random companions in the group."""
    rng = np.random.default_rng(5)
    hkv, d = 1, 256
    amax = np.arange(0, 0x7F80, dtype=np.uint32).astype(np.uint16)
    ngroups = amax.size
    rows = -(-ngroups // (d // 16))
    groups = np.zeros((rows * (d // 16), 16), np.uint16)
    frac = rng.uniform(-1, 1, size=(ngroups, 15)).astype(np.float32)
    amax_f = (amax.astype(np.uint32) << 16).view(np.float32)
    comp = to_bf16_bits(frac * amax_f[:, None])
    # keep |companion| <= amax after rounding
    comp_f = (comp.astype(np.uint32) << 16).view(np.float32)
    comp = np.where(np.abs(comp_f) <= amax_f[:, None], comp, np.uint16(0))
    groups[:ngroups, 0] = amax | np.where(rng.random(ngroups) < 0.5, 0x8000, 0).astype(np.uint16)
    groups[:ngroups, 1:] = comp
    rng.shuffle(groups[:ngroups].T)  # move the amax element around within groups
    k = groups.reshape(rows, hkv, d)
    v = k[::-1].copy()
    maxp = -(-rows // 16)
    pt = np.arange(maxp, dtype=np.int32)[None]
    calls = [(np.array([rows], np.int32), k, v, np.array([0, rows], np.int32))]
    got, ref = run_appends(hkv, d, pt, calls, maxp)
    assert np.array_equal(got, ref)


def test_append_every_code_decision():
    """For every positive finite scale s: groups whose amax is 6 s and whose
    other entries sweep every bf16 with |x| <= 6 s, both signs."""
    hkv, d = 2, 256
    e4m3 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    allpos = np.arange(0, 0x7F80, dtype=np.uint32).astype(np.uint16)
    allpos_f = (allpos.astype(np.uint32) << 16).view(np.float32)
    groups = []
    for sb in range(1, 0x7F):
        top = np.float32(6.0 * e4m3[sb])
        top_bits = (np.array([top]).view(np.uint32) >> 16).astype(np.uint16)[0]
        xs = allpos[allpos_f <= top]
        xs = np.concatenate([xs, xs | np.uint16(0x8000)])
        n = -(-xs.size // 15)
        fill = np.zeros(n * 15, np.uint16)
        fill[: xs.size] = xs
        groups.append(np.concatenate([np.full((n, 1), top_bits, np.uint16), fill.reshape(n, 15)], 1))
    groups = np.concatenate(groups)
    per_row = hkv * d // 16
    rows = -(-groups.shape[0] // per_row)
    pad = np.zeros((rows * per_row - groups.shape[0], 16), np.uint16)
    k = np.concatenate([groups, pad]).reshape(rows, hkv, d)
    v = np.roll(k, 1, axis=0)
    maxp = -(-rows // 16)
    pt = np.arange(maxp, dtype=np.int32)[None]
    calls = [(np.array([rows], np.int32), k, v, np.array([0, rows], np.int32))]
    got, ref = run_appends(hkv, d, pt, calls, maxp)
    assert np.array_equal(got, ref)


def test_append_reports_bad_page_and_skips_it():
    dev = torch.device("cuda")
    hkv, d = 2, 128
    cache = nv.Cache.allocate(4, hkv, d, dev, fill=SENTINEL)
    pt = torch.tensor([[0, 7, 2]], dtype=torch.int32, device=dev)  # page 7 does not exist
    lens = torch.tensor([40], dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    seqs = nv.Seqs(pt, lens, 40, err)
    rng = np.random.default_rng(0)
    k = bf16_tensor(rand_bits(rng, (40, hkv, d)), dev)
    cu = torch.tensor([0, 40], dtype=torch.int32, device=dev)
    nv.nvkv_append(cache, seqs, k, k, cu, 40, 40)
    torch.cuda.synchronize()
    assert int(err.item()) & nv.DEVERR_PAGE_ID
    pool = cache.pool.cpu().numpy().reshape(4, -1)
    assert (pool[1] == SENTINEL).all() and (pool[3] == SENTINEL).all()
    assert (pool[0] != SENTINEL).any() and (pool[2] != SENTINEL).any()
