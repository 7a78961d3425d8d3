"""Python binding of libnvkv: attention over an NVFP4-quantised paged KV
cache on B200 (sm_100a).

Argument marshalling only.  Every step of the path (quantise-append, split-K
decode / MTP-verify attention, combine, chunked prefill) runs in the CUDA
kernels of ``libnvkv.so``; the functions here take torch tensors (device
memory and streams come from PyTorch), check dtypes and devices, and pass raw
pointers to the C ABI declared in ``include/nvkv.h``.  There is no CPU or
PyTorch fallback: if the library is missing, every call raises.

Build the library with ``python -m nvfp4_quantized_kv_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "NvkvError", "Cache", "Seqs", "library", "library_path",
    "nvkv_page_bytes", "nvkv_default_num_splits", "nvkv_decode_workspace_bytes",
    "nvkv_split_plan", "nvkv_append", "nvkv_decode_attn", "nvkv_combine",
    "nvkv_prefill_attn", "nvkv_status_string", "nvkv_decode_attn_static",
    "nvkv_decode_static_scratch_bytes", "nvkv_rope_table", "nvkv_append_rope",
    "nvkv_pages_spill", "nvkv_pages_restore", "nvkv_k8v4_page_bytes", "nvkv_append_k8v4",
    "nvkv_decode_attn_k8v4", "nvkv_prefill_attn_k8v4", "nvkv_pages_spill_k8v4",
    "nvkv_pages_restore_k8v4", "nvkv_prefill_attn_split", "nvkv_prefill_workspace_bytes",
    "nvkv_prefill_num_splits",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libnvkv.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA = range(5)
DEVERR_PAGE_ID, DEVERR_LENGTH, DEVERR_TIMEOUT = 1, 2, 4


class NvkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {nvkv_status_string(status)} (status {status})")


class _CacheC(ctypes.Structure):
    _fields_ = [("pool", ctypes.c_void_p), ("num_pages", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


class _SeqsC(ctypes.Structure):
    _fields_ = [("page_table", ctypes.c_void_p), ("max_pages_per_seq", ctypes.c_int32),
                ("kv_lens", ctypes.c_void_p), ("batch", ctypes.c_int32),
                ("max_kv_len", ctypes.c_int32), ("err_word", ctypes.c_void_p)]


_lib = None


def library():
    """Load libnvkv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise ImportError(
                f"{library_path} is missing: build it with "
                "`python -m nvfp4_quantized_kv_b200.build` (needs nvcc); there is no fallback")
        L = ctypes.CDLL(library_path)
        vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
        cp, sp = ctypes.POINTER(_CacheC), ctypes.POINTER(_SeqsC)
        sig = {
            "nvkv_page_bytes": (sz, [i32, i32]),
            "nvkv_default_num_splits": (i32, []),
            "nvkv_decode_workspace_bytes": (sz, [i32, i32, i32, i32, i32, i32]),
            "nvkv_split_plan": (ctypes.c_int, [vp, i32, i32, i32, vp, vp]),
            "nvkv_append": (ctypes.c_int, [cp, sp, vp, vp, vp, i32, i32, vp]),
            "nvkv_decode_attn": (ctypes.c_int, [cp, sp, vp, i32, i32, f32, i32, vp, sz, vp]),
            "nvkv_decode_kernel_name": (ctypes.c_char_p, [cp, i32, i32]),
            "nvkv_decode_kernel_name_k8v4": (ctypes.c_char_p, [cp, i32, i32]),
            "nvkv_combine": (ctypes.c_int, [sp, vp, i32, i32, i32, i32, i32, vp, vp]),
            "nvkv_prefill_attn": (ctypes.c_int, [cp, sp, vp, vp, i32, i32, i32, f32, vp, vp]),
            "nvkv_prefill_workspace_bytes": (sz, [i32, i32, i32, i32]),
            "nvkv_prefill_num_splits": (i32, [cp, i32, i32, i32]),
            "nvkv_prefill_attn_split": (ctypes.c_int, [cp, sp, vp, vp, i32, i32, i32, f32, i32, vp,
                                                       sz, vp, vp]),
            "nvkv_decode_static_scratch_bytes": (sz, []),
            "nvkv_decode_attn_static": (ctypes.c_int, [cp, sp, vp, i32, i32, f32, i32, vp, vp]),
            "nvkv_rope_table": (ctypes.c_int, [vp, i32, i32, ctypes.c_double, ctypes.c_double, vp]),
            "nvkv_append_rope": (ctypes.c_int, [cp, sp, vp, vp, vp, i32, i32, vp, i32, i32, vp]),
            "nvkv_pages_spill": (ctypes.c_int, [cp, vp, vp, i32, vp, ctypes.c_int64, vp, vp]),
            "nvkv_pages_restore": (ctypes.c_int, [cp, vp, vp, i32, vp, ctypes.c_int64, vp, vp]),
            "nvkv_k8v4_page_bytes": (sz, [i32, i32]),
            "nvkv_pages_spill_k8v4": (ctypes.c_int, [cp, vp, vp, i32, vp, ctypes.c_int64, vp, vp]),
            "nvkv_pages_restore_k8v4": (ctypes.c_int, [cp, vp, vp, i32, vp, ctypes.c_int64, vp,
                                                       vp]),
            "nvkv_append_k8v4": (ctypes.c_int, [cp, sp, vp, vp, vp, i32, i32, vp]),
            "nvkv_decode_attn_k8v4": (ctypes.c_int, [cp, sp, vp, i32, i32, f32, i32, vp, sz, vp]),
            "nvkv_prefill_attn_k8v4": (ctypes.c_int, [cp, sp, vp, vp, i32, i32, i32, f32, vp, vp]),
            "nvkv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def nvkv_status_string(status: int) -> str:
    return library().nvkv_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != OK:
        raise NvkvError(status, what)


def _dev(t: torch.Tensor, dtype: torch.dtype, name: str) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


KV_FORMATS = ("nvfp4", "k8v4")


def _page_bytes_of(kv_format: str, num_kv_heads: int, head_dim: int) -> int:
    if kv_format == "nvfp4":
        return nvkv_page_bytes(num_kv_heads, head_dim)
    if kv_format == "k8v4":
        return nvkv_k8v4_page_bytes(num_kv_heads, head_dim)
    raise ValueError(f"kv_format must be one of {KV_FORMATS}, got {kv_format!r}")


class Cache:
    """The paged pool: ``pool`` is a uint8 CUDA tensor of num_pages pages of
    nvkv_page_bytes(num_kv_heads, head_dim) bytes (kv_format "nvfp4") or
    nvkv_k8v4_page_bytes(...) bytes ("k8v4": 8-bit K, NVFP4 V).  A K8V4
    cache is used only with the *_k8v4 calls."""

    def __init__(self, pool: torch.Tensor, num_pages: int, num_kv_heads: int, head_dim: int,
                 kv_format: str = "nvfp4"):
        self.pool, self.num_pages, self.num_kv_heads, self.head_dim = pool, num_pages, num_kv_heads, head_dim
        self.kv_format = kv_format
        need = num_pages * _page_bytes_of(kv_format, num_kv_heads, head_dim)
        if pool.numel() < need:
            raise ValueError(f"pool has {pool.numel()} bytes, needs {need}")
        self._c = _CacheC(_dev(pool, torch.uint8, "pool"), num_pages, num_kv_heads, head_dim)

    @staticmethod
    def allocate(num_pages: int, num_kv_heads: int, head_dim: int, device="cuda", fill=None,
                 kv_format: str = "nvfp4"):
        n = num_pages * _page_bytes_of(kv_format, num_kv_heads, head_dim)
        pool = torch.empty(n, dtype=torch.uint8, device=device)
        if fill is not None:
            pool.fill_(fill)
        return Cache(pool, num_pages, num_kv_heads, head_dim, kv_format)


def _fmt(cache: "Cache", want: str, what: str) -> None:
    if cache.kv_format != want:
        raise ValueError(f"{what} needs a {want} cache, got a {cache.kv_format} cache")


class Seqs:
    """The batch: page_table int32 [batch][max_pages_per_seq] and kv_lens
    int32 [batch] on the device; max_kv_len a host bound; err_word an
    optional int32 device tensor of one element."""

    def __init__(self, page_table: torch.Tensor, kv_lens: torch.Tensor, max_kv_len: int,
                 err_word: torch.Tensor | None = None):
        if page_table.dim() != 2 or kv_lens.dim() != 1 or kv_lens.numel() != page_table.shape[0]:
            raise ValueError("page_table must be [batch][max_pages], kv_lens [batch]")
        self.page_table, self.kv_lens, self.max_kv_len, self.err_word = page_table, kv_lens, max_kv_len, err_word
        self.batch = page_table.shape[0]
        self._c = _SeqsC(_dev(page_table, torch.int32, "page_table"), page_table.shape[1],
                         _dev(kv_lens, torch.int32, "kv_lens"), self.batch, int(max_kv_len),
                         _dev(err_word, torch.int32, "err_word") if err_word is not None else None)


def nvkv_page_bytes(num_kv_heads: int, head_dim: int) -> int:
    return int(library().nvkv_page_bytes(num_kv_heads, head_dim))


def nvkv_default_num_splits() -> int:
    return int(library().nvkv_default_num_splits())


def nvkv_decode_workspace_bytes(batch: int, T: int, num_q_heads: int, num_kv_heads: int,
                                head_dim: int, num_splits: int = 0) -> int:
    n = int(library().nvkv_decode_workspace_bytes(batch, T, num_q_heads, num_kv_heads, head_dim,
                                                  num_splits))
    if n == 0:
        raise NvkvError(ERR_INVALID_ARG, "nvkv_decode_workspace_bytes")
    return n


def nvkv_split_plan(kv_lens_host, num_kv_heads: int, num_splits: int):
    """Host copy of the split plan: (first_split, last_split) per (b, h)."""
    import numpy as np
    kl = np.ascontiguousarray(kv_lens_host, dtype=np.int32)
    n = kl.size * num_kv_heads
    first = np.zeros(n, np.int32)
    last = np.zeros(n, np.int32)
    _check(library().nvkv_split_plan(kl.ctypes.data, kl.size, num_kv_heads, num_splits,
                                     first.ctypes.data, last.ctypes.data), "nvkv_split_plan")
    return first, last


def nvkv_append(cache: Cache, seqs: Seqs, k_new: torch.Tensor, v_new: torch.Tensor,
                cu_new: torch.Tensor, total_new: int, max_new: int, stream=None) -> None:
    _fmt(cache, "nvfp4", "nvkv_append")
    _check(library().nvkv_append(
        ctypes.byref(cache._c), ctypes.byref(seqs._c), _dev(k_new, torch.bfloat16, "k_new"),
        _dev(v_new, torch.bfloat16, "v_new"), _dev(cu_new, torch.int32, "cu_new"), int(total_new),
        int(max_new), _stream(stream)), "nvkv_append")


def nvkv_rope_table(cs: torch.Tensor, rotary_dim: int, base: float, scale: float,
                    stream=None) -> None:
    """Fill cs (float32 CUDA [max_pos][rotary_dim/2][2]) with (cos, sin) of
    (pos / scale) * base^(-2i / rotary_dim)."""
    if cs.dim() != 3 or cs.shape[1] * 2 != rotary_dim or cs.shape[2] != 2:
        raise ValueError("cs must be [max_pos][rotary_dim/2][2]")
    _check(library().nvkv_rope_table(_dev(cs, torch.float32, "cs"), int(cs.shape[0]),
                                     int(rotary_dim), float(base), float(scale), _stream(stream)),
           "nvkv_rope_table")


def nvkv_append_rope(cache: Cache, seqs: Seqs, k_new: torch.Tensor, v_new: torch.Tensor,
                     cu_new: torch.Tensor, total_new: int, max_new: int, rope_cs: torch.Tensor,
                     rotary_dim: int, stream=None) -> None:
    """nvkv_append with K rotated at its position by the rope_cs table."""
    _fmt(cache, "nvfp4", "nvkv_append_rope")
    _check(library().nvkv_append_rope(
        ctypes.byref(cache._c), ctypes.byref(seqs._c), _dev(k_new, torch.bfloat16, "k_new"),
        _dev(v_new, torch.bfloat16, "v_new"), _dev(cu_new, torch.int32, "cu_new"), int(total_new),
        int(max_new), _dev(rope_cs, torch.float32, "rope_cs"), int(rope_cs.shape[0]),
        int(rotary_dim), _stream(stream)), "nvkv_append_rope")


def nvkv_decode_attn(cache: Cache, seqs: Seqs, q: torch.Tensor, T: int, num_q_heads: int,
                     sm_scale: float, num_splits: int, workspace: torch.Tensor,
                     stream=None) -> None:
    _fmt(cache, "nvfp4", "nvkv_decode_attn")
    _check(library().nvkv_decode_attn(
        ctypes.byref(cache._c), ctypes.byref(seqs._c), _dev(q, torch.bfloat16, "q"), int(T),
        int(num_q_heads), float(sm_scale), int(num_splits), _dev(workspace, torch.uint8, "workspace"),
        workspace.numel(), _stream(stream)), "nvkv_decode_attn")


def nvkv_decode_kernel_name(cache: Cache, T: int, num_q_heads: int) -> str:
    """The decode kernel the decode call of this cache's format launches for
    this step shape: "decode_qk4", "decode_tc" or "decode_simt" (NVFP4);
    "decode_qk4_k8v4" or "decode_simt" (K8V4)."""
    if cache.kv_format == "k8v4":
        fn = library().nvkv_decode_kernel_name_k8v4
    else:
        fn = library().nvkv_decode_kernel_name
    return fn(ctypes.byref(cache._c), int(T), int(num_q_heads)).decode()


def nvkv_combine(seqs: Seqs, workspace: torch.Tensor, T: int, num_q_heads: int,
                 num_kv_heads: int, head_dim: int, num_splits: int, out: torch.Tensor,
                 stream=None) -> None:
    _check(library().nvkv_combine(
        ctypes.byref(seqs._c), _dev(workspace, torch.uint8, "workspace"), int(T), int(num_q_heads),
        int(num_kv_heads), int(head_dim), int(num_splits), _dev(out, torch.bfloat16, "out"),
        _stream(stream)), "nvkv_combine")


def nvkv_prefill_attn(cache: Cache, seqs: Seqs, q: torch.Tensor, cu_q: torch.Tensor,
                      total_q: int, max_q: int, num_q_heads: int, sm_scale: float,
                      out: torch.Tensor, stream=None) -> None:
    _fmt(cache, "nvfp4", "nvkv_prefill_attn")
    _check(library().nvkv_prefill_attn(
        ctypes.byref(cache._c), ctypes.byref(seqs._c), _dev(q, torch.bfloat16, "q"),
        _dev(cu_q, torch.int32, "cu_q"), int(total_q), int(max_q), int(num_q_heads),
        float(sm_scale), _dev(out, torch.bfloat16, "out"), _stream(stream)), "nvkv_prefill_attn")


def nvkv_prefill_workspace_bytes(total_q: int, num_q_heads: int, head_dim: int,
                                 num_splits: int) -> int:
    return int(library().nvkv_prefill_workspace_bytes(int(total_q), int(num_q_heads),
                                                      int(head_dim), int(num_splits)))


def nvkv_prefill_num_splits(cache: Cache, batch: int, max_q: int, num_q_heads: int) -> int:
    """The key-split count nvkv_prefill_attn_split takes for num_splits = 0."""
    return int(library().nvkv_prefill_num_splits(ctypes.byref(cache._c), int(batch), int(max_q),
                                                 int(num_q_heads)))


def nvkv_prefill_attn_split(cache: Cache, seqs: Seqs, q: torch.Tensor, cu_q: torch.Tensor,
                            total_q: int, max_q: int, num_q_heads: int, sm_scale: float,
                            num_splits: int, workspace: "torch.Tensor | None", out: torch.Tensor,
                            stream=None) -> None:
    """Chunked prefill with the keys of each query tile split over num_splits
    (1..8) CTAs (0: automatic) and merged; workspace: uint8 device tensor of at least
    nvkv_prefill_workspace_bytes(...) bytes (None when the count is 1)."""
    _fmt(cache, "nvfp4", "nvkv_prefill_attn_split")
    ws = _dev(workspace, torch.uint8, "workspace") if workspace is not None else None
    nbytes = workspace.numel() if workspace is not None else 0
    _check(library().nvkv_prefill_attn_split(
        ctypes.byref(cache._c), ctypes.byref(seqs._c), _dev(q, torch.bfloat16, "q"),
        _dev(cu_q, torch.int32, "cu_q"), int(total_q), int(max_q), int(num_q_heads),
        float(sm_scale), int(num_splits), ws, nbytes, _dev(out, torch.bfloat16, "out"),
        _stream(stream)), "nvkv_prefill_attn_split")


def nvkv_decode_static_scratch_bytes() -> int:
    return int(library().nvkv_decode_static_scratch_bytes())


def nvkv_decode_attn_static(cache: Cache, seqs: Seqs, q: torch.Tensor, T: int, num_q_heads: int,
                            sm_scale: float, num_splits: int, out: torch.Tensor,
                            stream=None) -> None:
    """Decode attention + combine with the library's own device scratch (no
    workspace argument, nothing allocated); see include/nvkv.h."""
    _fmt(cache, "nvfp4", "nvkv_decode_attn_static")
    _check(library().nvkv_decode_attn_static(
        ctypes.byref(cache._c), ctypes.byref(seqs._c), _dev(q, torch.bfloat16, "q"), int(T),
        int(num_q_heads), float(sm_scale), int(num_splits), _dev(out, torch.bfloat16, "out"),
        _stream(stream)), "nvkv_decode_attn_static")


def _dev_or_pinned(t: torch.Tensor, dtype: torch.dtype, name: str) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not (t.is_cuda or t.is_pinned()):
        raise ValueError(f"{name} must be on a CUDA device or in pinned host memory")
    return t.data_ptr()


def _pages_args(cache: Cache, page_ids, slot_ids, arena, err_word):
    n = page_ids.numel()
    if slot_ids.numel() != n:
        raise ValueError("page_ids and slot_ids must have the same length")
    pb = _page_bytes_of(cache.kv_format, cache.num_kv_heads, cache.head_dim)
    return (ctypes.byref(cache._c), _dev_or_pinned(page_ids, torch.int32, "page_ids"),
            _dev_or_pinned(slot_ids, torch.int32, "slot_ids"), int(n),
            _dev_or_pinned(arena, torch.uint8, "arena"), arena.numel() // pb,
            _dev(err_word, torch.int32, "err_word") if err_word is not None else None)


def nvkv_pages_spill(cache: Cache, page_ids: torch.Tensor, slot_ids: torch.Tensor,
                     arena: torch.Tensor, err_word: torch.Tensor | None = None, stream=None) -> None:
    """Pool page page_ids[i] -> arena slot slot_ids[i] (arena: uint8, device
    or pinned host, a whole number of page-sized slots of the cache's
    format)."""
    fn = library().nvkv_pages_spill_k8v4 if cache.kv_format == "k8v4" else library().nvkv_pages_spill
    _check(fn(*_pages_args(cache, page_ids, slot_ids, arena, err_word), _stream(stream)),
           "nvkv_pages_spill")


def nvkv_pages_restore(cache: Cache, page_ids: torch.Tensor, slot_ids: torch.Tensor,
                       arena: torch.Tensor, err_word: torch.Tensor | None = None,
                       stream=None) -> None:
    """Arena slot slot_ids[i] -> pool page page_ids[i]."""
    fn = (library().nvkv_pages_restore_k8v4 if cache.kv_format == "k8v4"
          else library().nvkv_pages_restore)
    _check(fn(*_pages_args(cache, page_ids, slot_ids, arena, err_word), _stream(stream)),
           "nvkv_pages_restore")


# ---- K8V4 cache (8-bit K rows with one fp32 scale per row, NVFP4 V) --------

def nvkv_k8v4_page_bytes(num_kv_heads: int, head_dim: int) -> int:
    return int(library().nvkv_k8v4_page_bytes(num_kv_heads, head_dim))


def nvkv_append_k8v4(cache: Cache, seqs: Seqs, k_new: torch.Tensor, v_new: torch.Tensor,
                     cu_new: torch.Tensor, total_new: int, max_new: int, stream=None) -> None:
    _fmt(cache, "k8v4", "nvkv_append_k8v4")
    _check(library().nvkv_append_k8v4(
        ctypes.byref(cache._c), ctypes.byref(seqs._c), _dev(k_new, torch.bfloat16, "k_new"),
        _dev(v_new, torch.bfloat16, "v_new"), _dev(cu_new, torch.int32, "cu_new"), int(total_new),
        int(max_new), _stream(stream)), "nvkv_append_k8v4")


def nvkv_decode_attn_k8v4(cache: Cache, seqs: Seqs, q: torch.Tensor, T: int, num_q_heads: int,
                          sm_scale: float, num_splits: int, workspace: torch.Tensor,
                          stream=None) -> None:
    """Split-K partial results over a K8V4 cache; merge with nvkv_combine."""
    _fmt(cache, "k8v4", "nvkv_decode_attn_k8v4")
    _check(library().nvkv_decode_attn_k8v4(
        ctypes.byref(cache._c), ctypes.byref(seqs._c), _dev(q, torch.bfloat16, "q"), int(T),
        int(num_q_heads), float(sm_scale), int(num_splits), _dev(workspace, torch.uint8, "workspace"),
        workspace.numel(), _stream(stream)), "nvkv_decode_attn_k8v4")


def nvkv_prefill_attn_k8v4(cache: Cache, seqs: Seqs, q: torch.Tensor, cu_q: torch.Tensor,
                           total_q: int, max_q: int, num_q_heads: int, sm_scale: float,
                           out: torch.Tensor, stream=None) -> None:
    _fmt(cache, "k8v4", "nvkv_prefill_attn_k8v4")
    _check(library().nvkv_prefill_attn_k8v4(
        ctypes.byref(cache._c), ctypes.byref(seqs._c), _dev(q, torch.bfloat16, "q"),
        _dev(cu_q, torch.int32, "cu_q"), int(total_q), int(max_q), int(num_q_heads),
        float(sm_scale), _dev(out, torch.bfloat16, "out"), _stream(stream)), "nvkv_prefill_attn_k8v4")
