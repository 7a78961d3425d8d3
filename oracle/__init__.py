"""Float64 CPU oracle for the NVFP4 paged KV path.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it; the product library never does.
It shares no code with the CUDA path: the arithmetic lives in
``nvkv_oracle.c`` (plain C, IEEE double), and this module only builds it
with gcc and marshals numpy arrays into it.

Sources (page titles and sections of the pages this path is built from):
  * "gzenz/ninfer" README, "Fork changes vs upstream" -> "Context and model",
    NVFP4 KV cache bullet: 4-bit E2M1 codes plus one E4M3 scale per group
    of 16, here groups along head_dim.
  * "knoopx/ninfer" README, "Capabilities and limits": chunked prefill,
    batched decode, MTP verify with one to five drafts, one shared KV pool;
    K8V4 among the KV storage formats (8-bit K rows, NVFP4 V).
  * "gzenz/ninfer" README, "Fork changes vs upstream" -> "Context and
    model": linear RoPE scaling of the context extension (the rotating
    append).

Parity of every function here is pinned by ``tests/test_oracle_pins.py``
(format tables, exhaustive rounding sweeps against an independent
table-scan formulation and torch's float8 conversion, round-trip
invariants, closed-form attention cases and pure-Python brute force),
``tests/test_oracle_rope_pins.py`` (rotary table and rotation: closed-form
angles, linear scaling, the relative-position property, norms) and
``tests/test_oracle_k8v4_pins.py`` (8-bit K rows: table scan, error bound,
layout reader, attention closed forms).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvkv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile nvkv_oracle.c into liboracle.so next to it (gcc -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
             "-ffp-contract=off", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            d, i32, u8, u16 = ctypes.c_double, ctypes.c_int, ctypes.c_uint8, ctypes.c_uint16
            vp = ctypes.c_void_p
            L.oracle_bf16_value.restype = d
            L.oracle_bf16_value.argtypes = [u16]
            L.oracle_e2m1_value.restype = d
            L.oracle_e2m1_value.argtypes = [i32]
            L.oracle_e4m3_value.restype = d
            L.oracle_e4m3_value.argtypes = [i32]
            L.oracle_e4m3_round.restype = u8
            L.oracle_e4m3_round.argtypes = [d]
            L.oracle_e2m1_round_index.restype = i32
            L.oracle_e2m1_round_index.argtypes = [d]
            L.oracle_quantize_group.restype = None
            L.oracle_quantize_group.argtypes = [vp, vp, vp]
            L.oracle_quantize_groups.restype = None
            L.oracle_quantize_groups.argtypes = [vp, ctypes.c_long, vp, vp]
            L.oracle_dequant.restype = d
            L.oracle_dequant.argtypes = [i32, i32]
            L.oracle_qdq_row.restype = None
            L.oracle_qdq_row.argtypes = [vp, i32, vp]
            L.oracle_qdq_rows.restype = None
            L.oracle_qdq_rows.argtypes = [vp, ctypes.c_long, i32, vp]
            L.oracle_page_bytes.restype = ctypes.c_size_t
            L.oracle_page_bytes.argtypes = [i32, i32]
            L.oracle_append.restype = None
            L.oracle_append.argtypes = [vp, i32, i32, vp, i32, vp, i32, vp, vp, vp]
            L.oracle_pool_read_row.restype = None
            L.oracle_pool_read_row.argtypes = [vp, i32, i32, vp, i32, i32, i32, vp]
            L.oracle_rope_table.restype = None
            L.oracle_rope_table.argtypes = [i32, i32, d, d, vp]
            L.oracle_rope_rotate_f32.restype = None
            L.oracle_rope_rotate_f32.argtypes = [vp, i32, i32, vp, vp]
            L.oracle_quantize_group_f32.restype = None
            L.oracle_quantize_group_f32.argtypes = [vp, vp, vp]
            L.oracle_append_rope.restype = None
            L.oracle_append_rope.argtypes = [vp, i32, i32, vp, i32, vp, i32, vp, vp, vp, i32, vp, i32]
            L.oracle_k8_quantize_row.restype = None
            L.oracle_k8_quantize_row.argtypes = [vp, i32, vp, vp]
            L.oracle_k8_dequant.restype = d
            L.oracle_k8_dequant.argtypes = [i32, ctypes.c_float]
            L.oracle_k8v4_page_bytes.restype = ctypes.c_size_t
            L.oracle_k8v4_page_bytes.argtypes = [i32, i32]
            L.oracle_append_k8v4.restype = None
            L.oracle_append_k8v4.argtypes = [vp, i32, i32, vp, i32, vp, i32, vp, vp, vp]
            L.oracle_k8v4_read_row.restype = None
            L.oracle_k8v4_read_row.argtypes = [vp, i32, i32, vp, i32, i32, i32, vp]
            for fn in (L.oracle_attention_rows_k8v4, L.oracle_attention_pool_k8v4):
                fn.restype = None
            L.oracle_attention_rows_k8v4.argtypes = [i32, vp, vp, i32, i32, vp, vp, vp, d, vp, vp,
                                                     vp, i32]
            L.oracle_attention_pool_k8v4.argtypes = [i32, vp, i32, i32, vp, vp, vp, vp, d, vp, vp,
                                                     vp, i32]
            L.oracle_attention_rows.restype = None
            L.oracle_attention_rows.argtypes = [i32, vp, vp, i32, i32, vp, vp, vp, d, vp, vp, vp, i32]
            L.oracle_attention_pool.restype = None
            L.oracle_attention_pool.argtypes = [i32, vp, i32, i32, vp, vp, vp, vp, d, vp, vp, vp, i32]
            _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _u16(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 inputs are passed as their raw uint16 bits")
    return np.ascontiguousarray(a)


# --------------------------------------------------------------------------
# formats
# --------------------------------------------------------------------------
def bf16_value(bits: int) -> float:
    return lib().oracle_bf16_value(int(bits))


def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(int(code))


def e4m3_value(byte: int) -> float:
    return lib().oracle_e4m3_value(int(byte))


def e4m3_round(x: float) -> int:
    return int(lib().oracle_e4m3_round(float(x)))


def e2m1_round_index(r: float) -> int:
    return int(lib().oracle_e2m1_round_index(float(r)))


def dequant(code: int, scale_byte: int) -> float:
    return lib().oracle_dequant(int(code), int(scale_byte))


def quantize_group(x_bits) -> tuple[np.ndarray, int]:
    """16 bf16 values (uint16 bits) -> (16 E2M1 codes as uint8, E4M3 scale byte)."""
    x = _u16(x_bits).reshape(16)
    codes = np.zeros(16, np.uint8)
    sb = np.zeros(1, np.uint8)
    lib().oracle_quantize_group(_ptr(x), _ptr(codes), _ptr(sb))
    return codes, int(sb[0])


def quantize_rows(x_bits) -> tuple[np.ndarray, np.ndarray]:
    """[..., D] bf16 bits -> codes [..., D] (uint8, one per element) and
    scales [..., D/16] (uint8)."""
    x = _u16(x_bits)
    D = x.shape[-1]
    flat = np.ascontiguousarray(x.reshape(-1, 16))
    codes = np.zeros(flat.shape, np.uint8)
    scales = np.zeros(flat.shape[0], np.uint8)
    lib().oracle_quantize_groups(_ptr(flat), flat.shape[0], _ptr(codes), _ptr(scales))
    return codes.reshape(x.shape), scales.reshape(x.shape[:-1] + (D // 16,))


def qdq_rows(x_bits) -> np.ndarray:
    """Quantise and dequantise rows of bf16 bits ([..., D]) -> float64."""
    x = _u16(x_bits)
    D = x.shape[-1]
    flat = np.ascontiguousarray(x.reshape(-1, D))
    out = np.zeros(flat.shape, np.float64)
    n = flat.shape[0]
    L = lib()

    def run(lo, hi):  # ctypes releases the GIL: blocks of rows run in parallel
        L.oracle_qdq_rows(flat[lo:hi].ctypes.data, ctypes.c_long(hi - lo), D, out[lo:hi].ctypes.data)

    nthreads = min(os.cpu_count() or 1, max(1, n // 4096))
    if nthreads <= 1:
        run(0, n)
    else:
        bounds = [n * i // nthreads for i in range(nthreads + 1)]
        ts = [threading.Thread(target=run, args=(bounds[i], bounds[i + 1]))
              for i in range(nthreads)]
        for t in ts:
            t.start()
        for t in ts:
            t.join()
    return out.reshape(x.shape)


def attention_dense(k_hat: np.ndarray, v_hat: np.ndarray, q_bits, n_visible, sm_scale: float):
    """Exact softmax attention of several query rows of one kv-head over
    already dequantised keys and values (float64 [n][D], e.g. from
    qdq_rows), straight from the definition with numpy's float64 matrix
    product as the dot-product step: row i sees keys 0 .. n_visible[i]-1,
    s = sm_scale * q.k, p = exp(s - max s) / sum, out = sum p v.  Used where
    many rows share one long cache (the per-row oracle re-quantises every key
    for every row).  Returns (out [m][D], lse [m] natural log)."""
    qb = _u16(q_bits).reshape(-1, k_hat.shape[1])
    q = (qb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)  # bf16 -> f64, exact
    nvis = np.asarray(n_visible, np.int64).reshape(-1)
    m = q.shape[0]
    out = np.zeros((m, k_hat.shape[1]), np.float64)
    lse = np.full(m, -np.inf)
    n = int(nvis.max()) if m else 0
    if n <= 0:
        return out, lse
    s = (q @ k_hat[:n].T) * float(sm_scale)          # [m][n]
    s[np.arange(n)[None, :] >= nvis[:, None]] = -np.inf
    top = s.max(axis=1)
    ok = np.isfinite(top)
    p = np.zeros_like(s)
    p[ok] = np.exp(s[ok] - top[ok, None])
    denom = p.sum(axis=1)
    out[ok] = (p[ok] @ v_hat[:n]) / denom[ok, None]
    lse[ok] = top[ok] + np.log(denom[ok])
    return out, lse


# --------------------------------------------------------------------------
# pool
# --------------------------------------------------------------------------
def page_bytes(num_kv_heads: int, head_dim: int) -> int:
    return int(lib().oracle_page_bytes(num_kv_heads, head_dim))


def append(pool: np.ndarray, num_kv_heads: int, head_dim: int, page_table: np.ndarray,
           kv_lens: np.ndarray, k_new, v_new, cu_new: np.ndarray) -> None:
    """Quantise k_new / v_new ([rows][Hkv][D] bf16 bits) into the pool image
    in place; see oracle_append in nvkv_oracle.c for the position rule."""
    assert pool.dtype == np.uint8 and pool.flags["C_CONTIGUOUS"]
    pt = np.ascontiguousarray(page_table, np.int32)
    kl = np.ascontiguousarray(kv_lens, np.int32)
    cu = np.ascontiguousarray(cu_new, np.int32)
    k = _u16(k_new)
    v = _u16(v_new)
    lib().oracle_append(_ptr(pool), num_kv_heads, head_dim, _ptr(pt), pt.shape[1], _ptr(kl),
                        kl.shape[0], _ptr(k), _ptr(v), _ptr(cu))


def pool_read_row(pool: np.ndarray, num_kv_heads: int, head_dim: int, page_row: np.ndarray,
                  pos: int, h: int, is_v: bool) -> np.ndarray:
    pr = np.ascontiguousarray(page_row, np.int32)
    out = np.zeros(head_dim, np.float64)
    lib().oracle_pool_read_row(_ptr(pool), num_kv_heads, head_dim, _ptr(pr), int(pos), int(h),
                               int(bool(is_v)), _ptr(out))
    return out


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------
def _ptr_array(arrs) -> np.ndarray:
    return np.array([a.ctypes.data for a in arrs], dtype=np.uint64)


def attention_rows(jobs, num_kv_heads: int, head_dim: int, sm_scale: float,
                   nthreads: int | None = None, k8: bool = False):
    """Exact softmax attention for a list of output rows over a logical cache
    (K in NVFP4, or in the 8-bit row format of the K8V4 cache when k8).

    jobs: iterable of (k_rows, v_rows, h, n_visible, q) with k_rows / v_rows
    the sequence's bf16 bits [rows][Hkv][D] in position order, h the kv-head,
    n_visible the number of visible keys (position + 1) and q the [D] bf16
    bits of the query row.  Returns (out [n][D] f64, lse [n], psum [n])."""
    jobs = list(jobs)
    n = len(jobs)
    keep = []
    ks, vs, qs = [], [], []
    hs = np.zeros(n, np.int32)
    nv = np.zeros(n, np.int32)
    for i, (k, v, h, nvis, q) in enumerate(jobs):
        k = _u16(k)
        v = _u16(v)
        q = _u16(q).reshape(head_dim)
        keep += [k, v, q]
        ks.append(k)
        vs.append(v)
        qs.append(q)
        hs[i] = h
        nv[i] = nvis
    kp, vp_, qp = _ptr_array(ks), _ptr_array(vs), _ptr_array(qs)
    out = np.zeros((n, head_dim), np.float64)
    lse = np.zeros(n, np.float64)
    psum = np.zeros(n, np.float64)
    fn = lib().oracle_attention_rows_k8v4 if k8 else lib().oracle_attention_rows
    fn(n, _ptr(kp), _ptr(vp_), num_kv_heads, head_dim, _ptr(hs), _ptr(nv), _ptr(qp),
       float(sm_scale), _ptr(out), _ptr(lse), _ptr(psum), int(nthreads or os.cpu_count() or 1))
    del keep
    return out, lse, psum


def attention_pool(pool: np.ndarray, num_kv_heads: int, head_dim: int, jobs, sm_scale: float,
                   nthreads: int | None = None, k8: bool = False):
    """As attention_rows, but the cache is a pool image (the K8V4 layout when
    k8); jobs are (page_row, h, n_visible, q)."""
    jobs = list(jobs)
    n = len(jobs)
    keep, prs, qs = [], [], []
    hs = np.zeros(n, np.int32)
    nv = np.zeros(n, np.int32)
    for i, (pr, h, nvis, q) in enumerate(jobs):
        pr = np.ascontiguousarray(pr, np.int32)
        q = _u16(q).reshape(head_dim)
        keep += [pr, q]
        prs.append(pr)
        qs.append(q)
        hs[i] = h
        nv[i] = nvis
    pp, qp = _ptr_array(prs), _ptr_array(qs)
    out = np.zeros((n, head_dim), np.float64)
    lse = np.zeros(n, np.float64)
    psum = np.zeros(n, np.float64)
    fn = lib().oracle_attention_pool_k8v4 if k8 else lib().oracle_attention_pool
    fn(n, _ptr(pool), num_kv_heads, head_dim, _ptr(pp), _ptr(hs), _ptr(nv), _ptr(qp),
       float(sm_scale), _ptr(out), _ptr(lse), _ptr(psum), int(nthreads or os.cpu_count() or 1))
    del keep
    return out, lse, psum


# --------------------------------------------------------------------------
# rotary position embedding of K fused with quantise-append
# --------------------------------------------------------------------------
def rope_table(max_pos: int, rotary_dim: int, base: float, scale: float) -> np.ndarray:
    """float32 [max_pos][rotary_dim/2][2]: (cos, sin) of
    (pos / scale) * base^(-2i / rotary_dim), from double."""
    cs = np.zeros((max_pos, rotary_dim // 2, 2), np.float32)
    lib().oracle_rope_table(int(max_pos), int(rotary_dim), float(base), float(scale), _ptr(cs))
    return cs


def rope_rotate_f32(row_bits, rotary_dim: int, cs_pos) -> np.ndarray:
    """One bf16 row (uint16 bits [D]) rotated in float by one table row."""
    row = _u16(row_bits).reshape(-1)
    cs_pos = np.ascontiguousarray(cs_pos, np.float32).reshape(-1)
    out = np.zeros(row.shape[0], np.float32)
    lib().oracle_rope_rotate_f32(_ptr(row), int(row.shape[0]), int(rotary_dim), _ptr(cs_pos),
                                 _ptr(out))
    return out


def quantize_group_f32(x) -> tuple[np.ndarray, int]:
    """16 float32 values -> (16 E2M1 codes, E4M3 scale byte)."""
    x = np.ascontiguousarray(x, np.float32).reshape(16)
    codes = np.zeros(16, np.uint8)
    sb = np.zeros(1, np.uint8)
    lib().oracle_quantize_group_f32(_ptr(x), _ptr(codes), _ptr(sb))
    return codes, int(sb[0])


def append_rope(pool: np.ndarray, Hkv: int, D: int, page_table, kv_lens, k_new_bits, v_new_bits,
                cu_new, rotary_dim: int, cs) -> None:
    """oracle.append with K rotated at its position by table cs (in place)."""
    pt = np.ascontiguousarray(page_table, np.int32)
    lens = np.ascontiguousarray(kv_lens, np.int32)
    cu = np.ascontiguousarray(cu_new, np.int32)
    k, v = _u16(k_new_bits), _u16(v_new_bits)
    cs = np.ascontiguousarray(cs, np.float32)
    lib().oracle_append_rope(_ptr(pool), int(Hkv), int(D), _ptr(pt), int(pt.shape[1]), _ptr(lens),
                             int(pt.shape[0]), _ptr(k), _ptr(v), _ptr(cu), int(rotary_dim), _ptr(cs),
                             int(cs.shape[0]))


# --------------------------------------------------------------------------
# K8V4 cache: 8-bit K rows (E4M3 codes, one float scale per row), NVFP4 V
# --------------------------------------------------------------------------
def k8_quantize_row(x_bits) -> tuple[np.ndarray, float]:
    """One K row (bf16 bits [D]) -> (E4M3 code bytes [D], float32 scale)."""
    x = _u16(x_bits).reshape(-1)
    codes = np.zeros(x.shape[0], np.uint8)
    sc = np.zeros(1, np.float32)
    lib().oracle_k8_quantize_row(_ptr(x), int(x.shape[0]), _ptr(codes), _ptr(sc))
    return codes, float(sc[0])


def k8_dequant(code: int, scale: float) -> float:
    return lib().oracle_k8_dequant(int(code), float(np.float32(scale)))


def k8v4_page_bytes(num_kv_heads: int, head_dim: int) -> int:
    return int(lib().oracle_k8v4_page_bytes(num_kv_heads, head_dim))


def append_k8v4(pool: np.ndarray, num_kv_heads: int, head_dim: int, page_table, kv_lens, k_new,
                v_new, cu_new) -> None:
    """oracle.append for a K8V4 pool image (in place)."""
    assert pool.dtype == np.uint8 and pool.flags["C_CONTIGUOUS"]
    pt = np.ascontiguousarray(page_table, np.int32)
    kl = np.ascontiguousarray(kv_lens, np.int32)
    cu = np.ascontiguousarray(cu_new, np.int32)
    k, v = _u16(k_new), _u16(v_new)
    lib().oracle_append_k8v4(_ptr(pool), num_kv_heads, head_dim, _ptr(pt), pt.shape[1], _ptr(kl),
                             kl.shape[0], _ptr(k), _ptr(v), _ptr(cu))


def k8v4_read_row(pool: np.ndarray, num_kv_heads: int, head_dim: int, page_row, pos: int, h: int,
                  is_v: bool) -> np.ndarray:
    pr = np.ascontiguousarray(page_row, np.int32)
    out = np.zeros(head_dim, np.float64)
    lib().oracle_k8v4_read_row(_ptr(pool), num_kv_heads, head_dim, _ptr(pr), int(pos), int(h),
                               int(bool(is_v)), _ptr(out))
    return out
