"""GPU tests of host KV spill / restore (nvkv_pages_spill / _restore): whole
page blocks move between the pool and an arena of page-sized slots, bit-exact,
in device memory or pinned host memory; bad ids are reported and skipped;
attention over restored pages is bit-identical to attention before the spill."""
import numpy as np
import pytest
import torch

import nvfp4_quantized_kv_b200 as nv
from nvfp4_quantized_kv_b200 import workload as W
from nvfp4_quantized_kv_b200.harness import DeviceWorkload

pytestmark = pytest.mark.gpu


def _arena(slots, pb, kind, fill):
    if kind == "device":
        return torch.full((slots * pb,), fill, dtype=torch.uint8, device="cuda")
    return torch.full((slots * pb,), fill, dtype=torch.uint8).pin_memory()


def _ids(a, kind):
    t = torch.tensor(np.asarray(a, np.int32))
    return t.cuda() if kind == "device" else t.pin_memory()


@pytest.mark.parametrize("kind", ["device", "pinned"])
def test_spill_then_restore_moves_exact_bytes(kind):
    wl = W.small("spill", 2, 24, 4, 256, 1, [700, 300], seed=21)
    dw = DeviceWorkload(wl)
    dw.fill_context()
    torch.cuda.synchronize()
    pb = nv.nvkv_page_bytes(4, 256)
    rng = np.random.default_rng(3)
    used = np.unique(dw.page_table_np[dw.page_table_np >= 0])
    pages = rng.choice(used, size=20, replace=False)
    slots = rng.choice(64, size=20, replace=False)
    arena = _arena(64, pb, kind, 0x3C)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvkv_pages_spill(dw.cache, _ids(pages, kind), _ids(slots, kind), arena, err)
    torch.cuda.synchronize()
    pool = dw.cache.pool.cpu().numpy().reshape(wl.num_pages, pb)
    ar = arena.cpu().numpy().reshape(64, pb)
    for p, s in zip(pages, slots):
        assert np.array_equal(ar[s], pool[p])
    untouched = np.setdiff1d(np.arange(64), slots)
    assert (ar[untouched] == 0x3C).all()
    # restore into a different pool: exactly the listed pages change
    other = nv.Cache.allocate(wl.num_pages, 4, 256, "cuda", fill=0x5A)
    nv.nvkv_pages_restore(other, _ids(pages, kind), _ids(slots, kind), arena, err)
    torch.cuda.synchronize()
    got = other.pool.cpu().numpy().reshape(wl.num_pages, pb)
    for p in pages:
        assert np.array_equal(got[p], pool[p])
    rest = np.setdiff1d(np.arange(wl.num_pages), pages)
    assert (got[rest] == 0x5A).all()
    assert int(err.item()) == 0


def test_bad_ids_are_reported_and_skipped():
    pb = nv.nvkv_page_bytes(2, 128)
    cache = nv.Cache.allocate(4, 2, 128, "cuda", fill=0x11)
    arena = _arena(2, pb, "device", 0x22)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvkv_pages_spill(cache, _ids([9, 1, 2], "device"), _ids([0, -1, 1], "device"), arena, err)
    torch.cuda.synchronize()
    assert int(err.item()) & nv.DEVERR_PAGE_ID
    ar = arena.cpu().numpy().reshape(2, pb)
    assert (ar[0] == 0x22).all()  # pair (9 -> 0): no page 9
    assert (ar[1] == 0x11).all()  # pair (2 -> 1) moved
    err.zero_()
    nv.nvkv_pages_restore(cache, _ids([0, 3], "device"), _ids([5, 0], "device"), arena, err)
    torch.cuda.synchronize()
    assert int(err.item()) & nv.DEVERR_PAGE_ID
    pool = cache.pool.cpu().numpy().reshape(4, pb)
    assert (pool[0] == 0x11).all() and (pool[3] == 0x22).all()


def test_pageable_arena_is_refused():
    cache = nv.Cache.allocate(4, 2, 128, "cuda", fill=0)
    arena = torch.zeros(2 * nv.nvkv_page_bytes(2, 128), dtype=torch.uint8)  # not pinned
    ids = _ids([0], "device")
    with pytest.raises((ValueError, nv.NvkvError)):
        nv.nvkv_pages_spill(cache, ids, ids, arena)


def test_attention_after_spill_and_restore_is_bit_identical():
    wl = W.small("spill_rt", 2, 24, 4, 256, 1, [900, 400], seed=22)
    dw = DeviceWorkload(wl)
    dw.fill_context()
    dw.load_step_inputs()
    dw.step()
    torch.cuda.synchronize()
    before = dw.out.clone()
    pages = np.unique(dw.page_table_np[0][dw.page_table_np[0] >= 0])  # every page of sequence 0
    pb = nv.nvkv_page_bytes(4, 256)
    arena = _arena(len(pages), pb, "pinned", 0)
    pid, sid = _ids(pages, "device"), _ids(np.arange(len(pages)), "device")
    nv.nvkv_pages_spill(dw.cache, pid, sid, arena)
    pool2d = dw.cache.pool.view(wl.num_pages, pb)
    pool2d[torch.as_tensor(pages, device="cuda").long()] = 0xFF  # the device copy is gone
    dw.attend()
    torch.cuda.synchronize()
    assert not torch.equal(dw.out, before)
    nv.nvkv_pages_restore(dw.cache, pid, sid, arena)
    dw.attend()
    torch.cuda.synchronize()
    assert torch.equal(dw.out, before)
    assert dw.err_bits() == 0
