"""C-ABI checks that need no GPU: the library loads, exports every function
include/nvkv.h declares, rejects bad arguments before launching anything,
and its split plan covers every unit exactly once."""
import ctypes
import os
import re

import numpy as np
import pytest

import nvfp4_quantized_kv_b200 as nv
from nvfp4_quantized_kv_b200 import build as nvbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    nvbuild.build()
    return nv.library()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "nvkv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nvkv_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"nvkv_append", "nvkv_decode_attn", "nvkv_combine", "nvkv_prefill_attn"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_page_bytes(lib):
    assert nv.nvkv_page_bytes(4, 256) == 18432
    assert nv.nvkv_page_bytes(2, 128) == 4608
    assert lib.nvkv_page_bytes(0, 128) == 0 and lib.nvkv_page_bytes(2, -1) == 0


def test_status_strings(lib):
    for s in range(5):
        assert nv.nvkv_status_string(s)
    assert "unknown" in nv.nvkv_status_string(99)


def cache(pool=0x1000, num_pages=4, hkv=2, d=128):
    return nv._CacheC(pool, num_pages, hkv, d)


def seqs(batch=1, maxp=4, max_len=64, pt=0x2000, lens=0x3000):
    return nv._SeqsC(pt, maxp, lens, batch, max_len, None)


def test_append_rejects_bad_arguments_without_launch(lib):
    c, s = cache(), seqs()
    f = lib.nvkv_append
    B = ctypes.byref
    assert f(None, B(s), 0x10, 0x20, 0x30, 1, 1, None) == nv.ERR_INVALID_ARG
    assert f(B(c), None, 0x10, 0x20, 0x30, 1, 1, None) == nv.ERR_INVALID_ARG
    assert f(B(cache(d=64)), B(s), 0x10, 0x20, 0x30, 1, 1, None) == nv.ERR_UNSUPPORTED
    assert f(B(cache(pool=0x1001)), B(s), 0x10, 0x20, 0x30, 1, 1, None) == nv.ERR_INVALID_ARG
    assert f(B(c), B(seqs(max_len=65)), 0x10, 0x20, 0x30, 1, 1, None) == nv.ERR_INVALID_ARG
    assert f(B(c), B(s), None, 0x20, 0x30, 1, 1, None) == nv.ERR_INVALID_ARG
    assert f(B(c), B(s), 0x18, 0x20, 0x30, 1, 1, None) == nv.ERR_INVALID_ARG  # misaligned
    assert f(B(c), B(s), 0x10, 0x20, 0x30, -1, 1, None) == nv.ERR_INVALID_ARG
    assert f(B(c), B(s), None, None, None, 0, 0, None) == nv.OK  # nothing to do


def test_decode_rejects_bad_arguments_without_launch(lib):
    c, s = cache(hkv=4, d=256), seqs()
    f = lib.nvkv_decode_attn
    B = ctypes.byref
    need = lib.nvkv_decode_workspace_bytes(1, 1, 24, 4, 256, 8)
    assert need > 0
    assert f(B(c), B(s), 0x100, 1, 25, 0.1, 8, 0x1000, need, None) == nv.ERR_INVALID_ARG  # Hq % Hkv
    assert f(B(c), B(s), 0x100, 17, 24, 0.1, 8, 0x1000, need, None) == nv.ERR_UNSUPPORTED  # T
    assert f(B(c), B(s), 0x100, 6, 96, 0.1, 8, 0x1000, need, None) == nv.ERR_UNSUPPORTED  # rows
    assert f(B(c), B(s), 0x100, 0, 24, 0.1, 8, 0x1000, need, None) == nv.ERR_INVALID_ARG
    assert f(B(c), B(s), None, 1, 24, 0.1, 8, 0x1000, need, None) == nv.ERR_INVALID_ARG
    assert f(B(c), B(s), 0x100, 1, 24, float("nan"), 8, 0x1000, need, None) == nv.ERR_INVALID_ARG
    assert f(B(c), B(s), 0x100, 1, 24, 0.1, 8, None, need, None) == nv.ERR_WORKSPACE
    assert f(B(c), B(s), 0x100, 1, 24, 0.1, 8, 0x1000, need - 1, None) == nv.ERR_WORKSPACE
    assert f(B(c), B(s), 0x100, 1, 24, 0.1, 8, 0x1008, need, None) == nv.ERR_WORKSPACE


def test_combine_and_prefill_reject_bad_arguments(lib):
    B = ctypes.byref
    s = seqs()
    assert lib.nvkv_combine(B(s), 0x1000, 1, 24, 4, 256, 8, None, None) == nv.ERR_INVALID_ARG
    assert lib.nvkv_combine(B(s), None, 1, 24, 4, 256, 8, 0x100, None) == nv.ERR_WORKSPACE
    assert lib.nvkv_combine(B(s), 0x1000, 1, 24, 5, 256, 8, 0x100, None) == nv.ERR_INVALID_ARG
    c = cache(hkv=4, d=256)
    f = lib.nvkv_prefill_attn
    assert f(B(c), B(s), 0x100, 0x200, 10, 10, 25, 0.1, 0x300, None) == nv.ERR_INVALID_ARG
    assert f(B(c), B(s), None, 0x200, 10, 10, 24, 0.1, 0x300, None) == nv.ERR_INVALID_ARG
    assert f(B(c), B(s), None, None, 0, 0, 24, 0.1, None, None) == nv.OK


def test_workspace_size_formula(lib):
    for batch, T, hq, hkv, d, S in [(3, 1, 24, 4, 256, 296), (64, 1, 24, 4, 256, 100),
                                     (1, 1, 8, 2, 128, 5), (2, 4, 24, 4, 256, 1)]:
        R = T * hq // hkv
        slots = S + batch * hkv - 1
        a256 = lambda x: (x + 255) // 256 * 256
        assert lib.nvkv_decode_workspace_bytes(batch, T, hq, hkv, d, S) == \
            a256(slots * R * d * 4) + a256(slots * R * 4)
    assert lib.nvkv_decode_workspace_bytes(0, 1, 24, 4, 256, 8) == 0


def test_split_prefill_host_logic(lib):
    """Workspace bytes of the key-split prefill, its argument checks (before
    any launch) and the automatic split count (148 SMs when no GPU is
    visible): the chunked-prefill grid of 96 m-tiles x 4 kv-heads = 384 CTAs
    fills 2.59 of 3 waves, 3 splits fill 7.78 of 8 (0.973), 5 splits 12.97
    of 13 (0.998); a 148-CTA grid stays whole; a 100-CTA grid fills 0.68
    whole, 0.90 in 4 splits, 0.95 in 7."""
    B = ctypes.byref
    a256 = lambda x: (x + 255) // 256 * 256
    for tq, hq, d, S in [(2048, 24, 256, 3), (37, 12, 256, 2), (1, 8, 128, 4)]:
        rows = tq * hq * S
        assert lib.nvkv_prefill_workspace_bytes(tq, hq, d, S) == a256(rows * d * 4) + a256(rows * 4)
    assert lib.nvkv_prefill_workspace_bytes(2048, 24, 256, 0) == \
        lib.nvkv_prefill_workspace_bytes(2048, 24, 256, 8)
    assert lib.nvkv_prefill_workspace_bytes(2048, 24, 256, 1) == 0
    assert lib.nvkv_prefill_workspace_bytes(2048, 24, 256, 9) == 0
    assert lib.nvkv_prefill_workspace_bytes(-1, 24, 256, 2) == 0
    c, s = cache(hkv=4, d=256), seqs()
    f = lib.nvkv_prefill_attn_split
    need = lib.nvkv_prefill_workspace_bytes(10, 24, 256, 2)
    assert f(B(c), B(s), 0x100, 0x200, 10, 10, 24, 0.1, 9, None, 0, 0x300, None) == nv.ERR_INVALID_ARG
    assert f(B(c), B(s), 0x100, 0x200, 10, 10, 24, 0.1, -1, None, 0, 0x300, None) == nv.ERR_INVALID_ARG
    assert f(B(c), B(s), 0x100, 0x200, 10, 10, 25, 0.1, 2, None, 0, 0x300, None) == nv.ERR_INVALID_ARG
    assert f(B(c), B(s), 0x100, 0x200, 10, 10, 24, 0.1, 2, None, 0, 0x300, None) == nv.ERR_WORKSPACE
    assert f(B(c), B(s), 0x100, 0x200, 10, 10, 24, 0.1, 2, 0x1000, need - 1, 0x300, None) == \
        nv.ERR_WORKSPACE
    assert f(B(c), B(s), 0x100, 0x200, 10, 10, 24, 0.1, 2, 0x1008, need, 0x300, None) == \
        nv.ERR_WORKSPACE
    assert f(B(c), B(s), None, None, 0, 0, 24, 0.1, 2, None, 0, None, None) == nv.OK
    n = lib.nvkv_prefill_num_splits
    assert n(B(c), 1, 2048, 24) == 5
    assert n(B(c), 1, 789, 24) == 1      # ceil(789 * 6 / 128) = 37 m-tiles x 4 = 148 CTAs
    assert n(B(c), 1, 533, 24) == 7      # 25 m-tiles x 4 = 100 CTAs
    assert n(B(cache(hkv=4, d=128)), 1, 2048, 24) == 1  # CUDA-core kernel
    assert n(B(c), 1, 2048, 25) == 0 and n(None, 1, 2048, 24) == 0


@pytest.mark.parametrize("seed", range(6))
def test_split_plan_partitions_units(lib, seed):
    """Every 128-token unit of every (b, h) pair lies in exactly one split
    range; ranges are contiguous and balanced to within one unit; the
    workspace slots c + b*Hkv + h written by a range are unique."""
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 40))
    hkv = int(rng.integers(1, 6))
    lens = rng.integers(0, 5000, size=B).astype(np.int32)
    lens[rng.random(B) < 0.2] = 0
    S = int(rng.choice([1, 3, 7, 148, 296, 1000]))
    first, last = nv.nvkv_split_plan(lens, hkv, S)
    units = [(int(l) + 127) // 128 for l in lens]
    U = sum(u * hkv for u in units)
    begin = [c * U // S for c in range(S + 1)]
    owner = np.full(U, -1)
    for c in range(S):
        owner[begin[c]:begin[c + 1]] = c
        assert begin[c + 1] - begin[c] in (U // S, -(-U // S)) or U == 0
    assert (owner >= 0).all() or U == 0
    start = 0
    slots = set()
    for b in range(B):
        for h in range(hkv):
            bh = b * hkv + h
            if units[b] == 0:
                assert first[bh] > last[bh]
                continue
            touched = sorted(set(owner[start:start + units[b]]))
            assert first[bh] == touched[0] and last[bh] == touched[-1]
            for c in touched:
                assert (c, bh) not in slots
                slots.add((c, bh))
            start += units[b]
    used = {c + bh for c, bh in slots}
    assert len(used) == len(slots)
    assert max(used, default=0) <= S + B * hkv - 2


def test_pages_spill_restore_reject_bad_arguments_without_launch(lib):
    c = cache()
    B = ctypes.byref
    for f in (lib.nvkv_pages_spill, lib.nvkv_pages_restore):
        assert f(None, 0x10, 0x20, 1, 0x1000, 4, None, None) == nv.ERR_INVALID_ARG
        assert f(B(c), 0x10, 0x20, -1, 0x1000, 4, None, None) == nv.ERR_INVALID_ARG
        assert f(B(c), None, 0x20, 1, 0x1000, 4, None, None) == nv.ERR_INVALID_ARG
        assert f(B(c), 0x10, None, 1, 0x1000, 4, None, None) == nv.ERR_INVALID_ARG
        assert f(B(c), 0x10, 0x20, 1, None, 4, None, None) == nv.ERR_INVALID_ARG
        assert f(B(c), 0x10, 0x20, 1, 0x1008, 4, None, None) == nv.ERR_INVALID_ARG  # unaligned arena
        assert f(B(c), 0x10, 0x20, 1, 0x1000, 0, None, None) == nv.ERR_INVALID_ARG  # no slots
        assert f(B(c), 0x10, 0x20, 0, 0x1000, 4, None, None) == nv.OK  # nothing to move
        # pointers no kernel can reach (here: not CUDA memory at all) are refused
        buf = (ctypes.c_uint8 * 4096)()
        ids = (ctypes.c_int32 * 1)()
        a = (ctypes.addressof(buf) + 15) & ~15
        assert f(B(c), ctypes.addressof(ids), ctypes.addressof(ids), 1, a, 1, None, None) == \
            nv.ERR_INVALID_ARG


def test_rope_calls_reject_bad_arguments_without_launch(lib):
    c, s = cache(), seqs()
    B = ctypes.byref
    t = lib.nvkv_rope_table
    assert t(None, 16, 64, 1e4, 1.0, None) == nv.ERR_INVALID_ARG
    assert t(0x1004, 16, 64, 1e4, 1.0, None) == nv.ERR_INVALID_ARG   # not 8-byte aligned
    assert t(0x1000, 0, 64, 1e4, 1.0, None) == nv.ERR_INVALID_ARG
    assert t(0x1000, 16, 48, 1e4, 1.0, None) == nv.ERR_INVALID_ARG   # not a multiple of 32
    assert t(0x1000, 16, 64, -1.0, 1.0, None) == nv.ERR_INVALID_ARG
    assert t(0x1000, 16, 64, 1e4, 0.0, None) == nv.ERR_INVALID_ARG
    a = lib.nvkv_append_rope
    ok = (0x10, 0x20, 0x30, 1, 1)
    assert a(B(c), B(s), *ok, None, 16, 64, None) == nv.ERR_INVALID_ARG
    assert a(B(c), B(s), *ok, 0x1000, 16, 0, None) == nv.ERR_INVALID_ARG
    assert a(B(c), B(s), *ok, 0x1000, 16, 160, None) == nv.ERR_INVALID_ARG  # > head_dim 128
    assert a(B(c), B(s), *ok, 0x1000, 16, 40, None) == nv.ERR_INVALID_ARG
    assert a(B(c), B(s), *ok, 0x1000, 0, 64, None) == nv.ERR_INVALID_ARG
    assert a(B(c), B(s), 0x10, 0x20, 0x30, 0, 0, 0x1000, 16, 64, None) == nv.OK  # nothing new


def test_k8v4_page_bytes(lib):
    import oracle
    for hkv, d in [(4, 256), (2, 128), (1, 128), (8, 256)]:
        assert nv.nvkv_k8v4_page_bytes(hkv, d) == hkv * (25 * d + 64) == \
            oracle.k8v4_page_bytes(hkv, d)
        assert (25 * d + 64) % 16 == 0  # every kv-head block starts 16-byte aligned
    assert lib.nvkv_k8v4_page_bytes(0, 128) == 0 and lib.nvkv_k8v4_page_bytes(2, 0) == 0


def test_k8v4_calls_reject_bad_arguments_without_launch(lib):
    B = ctypes.byref
    c, s = cache(), seqs()
    a = lib.nvkv_append_k8v4
    assert a(None, B(s), 0x10, 0x20, 0x30, 1, 1, None) == nv.ERR_INVALID_ARG
    assert a(B(cache(d=64)), B(s), 0x10, 0x20, 0x30, 1, 1, None) == nv.ERR_UNSUPPORTED
    assert a(B(c), B(s), 0x18, 0x20, 0x30, 1, 1, None) == nv.ERR_INVALID_ARG  # misaligned
    assert a(B(c), B(seqs(max_len=65)), 0x10, 0x20, 0x30, 1, 1, None) == nv.ERR_INVALID_ARG
    assert a(B(c), B(s), None, None, None, 0, 0, None) == nv.OK  # nothing to do
    c4 = cache(hkv=4, d=256)
    f = lib.nvkv_decode_attn_k8v4
    need = lib.nvkv_decode_workspace_bytes(1, 1, 24, 4, 256, 8)
    assert f(B(c4), B(s), 0x100, 1, 25, 0.1, 8, 0x1000, need, None) == nv.ERR_INVALID_ARG
    assert f(B(c4), B(s), 0x100, 17, 24, 0.1, 8, 0x1000, need, None) == nv.ERR_UNSUPPORTED
    assert f(B(c4), B(s), 0x100, 1, 24, float("inf"), 8, 0x1000, need, None) == \
        nv.ERR_INVALID_ARG
    assert f(B(c4), B(s), 0x100, 1, 24, 0.1, 8, 0x1000, need - 1, None) == nv.ERR_WORKSPACE
    assert f(B(c4), B(s), 0x100, 1, 24, 0.1, 8, None, need, None) == nv.ERR_WORKSPACE
    p = lib.nvkv_prefill_attn_k8v4
    assert p(B(c4), B(s), 0x100, 0x200, 10, 10, 25, 0.1, 0x300, None) == nv.ERR_INVALID_ARG
    assert p(B(c4), B(s), None, 0x200, 10, 10, 24, 0.1, 0x300, None) == nv.ERR_INVALID_ARG
    assert p(B(c4), B(s), 0x100, 0x200, 10, 10, 24, 0.1, 0x308, None) == nv.ERR_INVALID_ARG
    assert p(B(c4), B(s), None, None, 0, 0, 24, 0.1, None, None) == nv.OK


def test_calls_refuse_a_cache_of_the_other_format():
    """The Python binding keeps the two layouts apart: an NVFP4 call given a
    K8V4 cache (and the reverse) raises before any argument is marshalled."""
    import types
    k8 = types.SimpleNamespace(kv_format="k8v4")
    fp4 = types.SimpleNamespace(kv_format="nvfp4")
    for call in (lambda: nv.nvkv_append(k8, None, None, None, None, 1, 1),
                 lambda: nv.nvkv_decode_attn(k8, None, None, 1, 8, 0.1, 0, None),
                 lambda: nv.nvkv_prefill_attn(k8, None, None, None, 1, 1, 8, 0.1, None),
                 lambda: nv.nvkv_decode_attn_static(k8, None, None, 1, 8, 0.1, 0, None),
                 lambda: nv.nvkv_append_rope(k8, None, None, None, None, 1, 1, None, 64),
                 lambda: nv.nvkv_append_k8v4(fp4, None, None, None, None, 1, 1),
                 lambda: nv.nvkv_decode_attn_k8v4(fp4, None, None, 1, 8, 0.1, 0, None),
                 lambda: nv.nvkv_prefill_attn_k8v4(fp4, None, None, None, 1, 1, 8, 0.1, None)):
        with pytest.raises(ValueError, match="cache"):
            call()
    with pytest.raises(ValueError):
        nv._page_bytes_of("int8", 2, 128)


def test_k8v4_pages_calls_reject_bad_arguments_without_launch(lib):
    c = cache()
    B = ctypes.byref
    for f in (lib.nvkv_pages_spill_k8v4, lib.nvkv_pages_restore_k8v4):
        assert f(None, 0x10, 0x20, 1, 0x1000, 4, None, None) == nv.ERR_INVALID_ARG
        assert f(B(c), 0x10, 0x20, -1, 0x1000, 4, None, None) == nv.ERR_INVALID_ARG
        assert f(B(c), 0x10, 0x20, 1, 0x1008, 4, None, None) == nv.ERR_INVALID_ARG
        assert f(B(cache(d=64)), 0x10, 0x20, 1, 0x1000, 4, None, None) == nv.ERR_UNSUPPORTED
        assert f(B(c), 0x10, 0x20, 0, 0x1000, 4, None, None) == nv.OK


def test_appends_refuse_item_counts_beyond_32_bits(lib):
    """The append kernels index (slot pair, kv-head, group) items with 32-bit
    integers; a max_new whose item count would overflow is refused."""
    B = ctypes.byref
    c, s = cache(hkv=64, d=256), seqs()
    big = 2 ** 31 - 1  # (big/2 + 1) * 64 * 16 items > 2^31
    assert lib.nvkv_append(B(c), B(s), 0x10, 0x20, 0x30, 1, big, None) == nv.ERR_UNSUPPORTED
    assert lib.nvkv_append_k8v4(B(c), B(s), 0x10, 0x20, 0x30, 1, big, None) == \
        nv.ERR_UNSUPPORTED
    assert lib.nvkv_append_rope(B(c), B(s), 0x10, 0x20, 0x30, 1, big, 0x1000, 16, 64, None) == \
        nv.ERR_UNSUPPORTED


def test_the_library_is_usable_from_plain_c(lib, tmp_path):
    """A C program compiled against include/nvkv.h and linked with libnvkv.so
    runs the size functions, the split plan and the argument checks."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path / "abi_from_c")
    libdir = os.path.dirname(nv.library_path)
    subprocess.run([cc, "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_from_c.c"), "-L", libdir, "-lnvkv",
                    "-Wl,-rpath," + libdir, "-o", exe], check=True, capture_output=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"


def test_decode_kernel_name_without_launch(lib):
    """The dispatch query launches nothing; invalid shapes give "none",
    valid ones one of the three kernel names (on a host without a GPU the
    tensor-map encoder is missing, so it reports the CUDA-core kernel)."""
    B = ctypes.byref
    f = lib.nvkv_decode_kernel_name
    assert f(None, 1, 24) == b"none"
    assert f(B(cache(hkv=4, d=256)), 1, 25) == b"none"  # Hq % Hkv
    assert f(B(cache(hkv=4, d=256)), 0, 24) == b"none"
    for T in (1, 6, 16):
        assert f(B(cache(hkv=4, d=256)), T, 24) in (b"decode_qk4", b"decode_tc", b"decode_simt")
    assert f(B(cache(hkv=2, d=128)), 1, 8) == b"decode_simt"  # head_dim 128: CUDA cores only
