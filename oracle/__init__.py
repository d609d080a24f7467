"""CPU oracle for mixed-precision KV-cache quantization and decode attention.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The product library never
imports, links or runs anything in this directory.

The arithmetic lives in ``kvq_oracle.c`` (plain C, binary32 quantizer steps with
no FMA contraction, binary64 attention); this module is a thin ctypes wrapper
over numpy arrays.  ``build()`` compiles the shared library in place.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkvq_oracle.so")
_lib = None

PER_CHANNEL = 0
PER_TOKEN = 1


def build(force: bool = False) -> str:
    """Compile kvq_oracle.c -> libkvq_oracle.so (gcc, -O2 -ffp-contract=off, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fopenmp",
           "-fPIC", "-shared", "-Wall", "-o", _LIB_PATH + ".tmp", _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int, ctypes.c_long
        L.orc_record_bytes.restype = i64
        L.orc_record_bytes.argtypes = [i32, i32, i32]
        L.orc_unit_image_bytes.restype = i64
        L.orc_unit_image_bytes.argtypes = [i32, i32, i32, i32, i32]
        L.orc_get_code.restype = ctypes.c_uint
        L.orc_get_code.argtypes = [P, i32, i32, i32, i32, i32]
        L.orc_code_position.restype = None
        L.orc_code_position.argtypes = [i32, i32, i32, i32, i32, P, P]
        L.orc_sz_position.restype = None
        L.orc_sz_position.argtypes = [i32, i32, i32, i32, P, P]
        L.orc_unit.restype = i32
        L.orc_unit.argtypes = [P, P, i32, i32, i32, i32, i32, P, P, P]
        L.orc_attention_partial.restype = None
        L.orc_attention_partial.argtypes = [P, P, P, i32, i32, i32, i32, P, P, P]
        L.orc_merge_partials.restype = None
        L.orc_merge_partials.argtypes = [i32, i32, i32, P, P, P, P]
        L.orc_attention.restype = None
        L.orc_attention.argtypes = [P, P, P, i32, i32, i32, P]
        L.orc_layer.restype = i32
        L.orc_layer.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, i32, i32, P, P]
        L.orc_paged_unit.restype = i32
        L.orc_paged_unit.argtypes = [P, P, P, i32, i32, P, P, P]
        L.orc_paged_unit_bytes.restype = i64
        L.orc_paged_unit_bytes.argtypes = [P, i32, i32]
        L.orc_paged_layer.restype = i32
        L.orc_paged_layer.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, P, P]
        L.orc_paged_page4_bytes.restype = i64
        L.orc_paged_page4_bytes.argtypes = [i32]
        L.orc_paged_rec2_bytes.restype = i64
        L.orc_paged_rec2_bytes.argtypes = [i32]
        L.orc_f32_to_f16_array.restype = None
        L.orc_f32_to_f16_array.argtypes = [P, P, i64]
        L.orc_f16_to_f64_array.restype = None
        L.orc_f16_to_f64_array.argtypes = [P, P, i64]
        L.orc_set_threads.restype = i32
        L.orc_set_threads.argtypes = [i32]
        L.orc_quant_groups.restype = None
        L.orc_quant_groups.argtypes = [P, i64, i32, P, P, P]
        L.orc_format_version.restype = i32
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    """bf16 / fp16 bit patterns as a contiguous uint16 array."""
    a = np.asarray(a)
    if a.dtype != np.uint16:
        a = a.view(np.uint16)
    return np.ascontiguousarray(a)


# ---------------------------------------------------------------- scalars
def f32_to_f16_bits(x) -> np.ndarray:
    x = np.ascontiguousarray(np.asarray(x, np.float32))
    out = np.empty(x.shape, np.uint16)
    lib().orc_f32_to_f16_array(_p(x), _p(out), x.size)
    return out


def f16_bits_to_f64(h) -> np.ndarray:
    h = _u16(h)
    out = np.empty(h.shape, np.float64)
    lib().orc_f16_to_f64_array(_p(h), _p(out), h.size)
    return out


def bf16_bits_to_f32(b) -> np.ndarray:
    b = _u16(b)
    return (b.astype(np.uint32) << 16).view(np.float32)


def set_threads(n: int) -> int:
    """Threads of the oracle's OpenMP loops (n <= 0: default); returns the count in use.
    Timing only: results do not depend on it."""
    return int(lib().orc_set_threads(int(n)))


def quant_groups(x, bits: int):
    """Quantize rows of 32 binary32 values: returns (s16 bits, z16 bits, codes uint8)."""
    x = np.ascontiguousarray(np.asarray(x, np.float32).reshape(-1, 32))
    n = x.shape[0]
    s = np.empty(n, np.uint16)
    z = np.empty(n, np.uint16)
    c = np.empty((n, 32), np.uint8)
    lib().orc_quant_groups(_p(x), n, bits, _p(s), _p(z), _p(c))
    return s, z, c


# ---------------------------------------------------------------- format
def record_bytes(D: int, bk: int, bv: int) -> int:
    return int(lib().orc_record_bytes(D, bk, bv))


def unit_image_bytes(L: int, D: int, bk: int, bv: int, kmode: int) -> int:
    return int(lib().orc_unit_image_bytes(L, D, bk, bv, kmode))


def get_code(area: np.ndarray, role: int, u: int, d: int, D: int, bits: int) -> int:
    area = np.ascontiguousarray(area, np.uint8)
    return int(lib().orc_get_code(_p(area), role, u, d, D, bits))


def code_position(role: int, u: int, d: int, D: int, bits: int):
    """(byte offset, bit offset) of the code of token u, channel d in a block's code area."""
    b = ctypes.c_long()
    t = ctypes.c_int()
    lib().orc_code_position(role, u, d, D, bits, ctypes.byref(b), ctypes.byref(t))
    return b.value, t.value


def sz_position(kind: int, index: int, j: int, nj: int):
    """(scale offset, zero offset) inside an s/z area: kind 0 per-channel (index =
    channel), kind 1 per-token (index = token in block, j = channel group)."""
    so = ctypes.c_long()
    zo = ctypes.c_long()
    lib().orc_sz_position(kind, index, j, nj, ctypes.byref(so), ctypes.byref(zo))
    return so.value, zo.value


# ---------------------------------------------------------------- units / layers
def unit(K, V, D: int, bk: int, bv: int, kmode: int, want_image=True, want_dequant=True):
    """One (batch, kv head) unit. K, V: [L, D] bf16 bits.  Returns (image, Kh, Vh)."""
    K = _u16(K).reshape(-1, D)
    V = _u16(V).reshape(-1, D)
    L = K.shape[0]
    img = np.empty(unit_image_bytes(L, D, bk, bv, kmode), np.uint8) if want_image else None
    Kh = np.empty((L, D), np.float64) if want_dequant else None
    Vh = np.empty((L, D), np.float64) if want_dequant else None
    rc = lib().orc_unit(_p(K), _p(V), L, D, bk, bv, kmode,
                        _p(img) if img is not None else None,
                        _p(Kh) if Kh is not None else None,
                        _p(Vh) if Vh is not None else None)
    if rc != 0:
        raise ValueError("orc_unit rejected its arguments")
    return img, Kh, Vh


def attention(q, Kh, Vh):
    """q: [G, D] bf16 bits; Kh, Vh: [L, D] float64 -> out [G, D] float64."""
    q = _u16(q)
    G, D = q.shape
    Kh = np.ascontiguousarray(Kh, np.float64)
    Vh = np.ascontiguousarray(Vh, np.float64)
    out = np.empty((G, D), np.float64)
    lib().orc_attention(_p(q), _p(Kh), _p(Vh), Kh.shape[0], D, G, _p(out))
    return out


def attention_partial(q, Kh, Vh, t0: int, t1: int):
    q = _u16(q)
    G, D = q.shape
    Kh = np.ascontiguousarray(Kh, np.float64)
    Vh = np.ascontiguousarray(Vh, np.float64)
    m = np.empty(G)
    l = np.empty(G)
    acc = np.empty((G, D))
    lib().orc_attention_partial(_p(q), _p(Kh), _p(Vh), t0, t1, D, G, _p(m), _p(l), _p(acc))
    return m, l, acc


def merge_partials(m, l, acc):
    """m, l: [S, G]; acc: [S, G, D] -> out [G, D]."""
    m = np.ascontiguousarray(m, np.float64)
    l = np.ascontiguousarray(l, np.float64)
    acc = np.ascontiguousarray(acc, np.float64)
    S, G, D = acc.shape
    out = np.empty((G, D))
    lib().orc_merge_partials(S, G, D, _p(m), _p(l), _p(acc), _p(out))
    return out


def layer(K, V, Q, G: int, bk: int, bv: int, kmode: int, want_image=True, want_out=True):
    """K, V: [B, Hkv, L, D] bf16 bits; Q: [B, Hkv*G, D] bf16 bits.
    Returns (image bytes concatenated over (b, h) units, out [B, Hq, D] float64)."""
    K = _u16(K)
    V = _u16(V)
    B, Hkv, L, D = K.shape
    img = None
    if want_image:
        img = np.empty(B * Hkv * unit_image_bytes(L, D, bk, bv, kmode), np.uint8)
    out = None
    Qp = None
    if want_out:
        Q = _u16(Q)
        assert Q.shape == (B, Hkv * G, D)
        out = np.empty((B, Hkv * G, D), np.float64)
        Qp = _p(Q)
    rc = lib().orc_layer(_p(K), _p(V), Qp, B, Hkv, G, L, D, bk, bv, kmode,
                         _p(img) if img is not None else None,
                         _p(out) if out is not None else None)
    if rc != 0:
        raise ValueError("orc_layer rejected its arguments")
    return img, out


# ---------------------------------------------------------------- paged INT2/INT4
def paged_unit(K, V, tags, D: int, want_image=True, want_dequant=True):
    """One (batch, kv head) unit of the paged cache. K, V: [L, D] bf16 bits; tags: [L]
    uint8 (2 or 4).  Returns (image, Kh, Vh) with Kh/Vh in token order."""
    K = _u16(K).reshape(-1, D)
    V = _u16(V).reshape(-1, D)
    tags = np.ascontiguousarray(tags, np.uint8)
    L = K.shape[0]
    n = int(lib().orc_paged_unit_bytes(_p(tags), L, D))
    img = np.empty(n, np.uint8) if want_image else None
    Kh = np.empty((L, D), np.float64) if want_dequant else None
    Vh = np.empty((L, D), np.float64) if want_dequant else None
    rc = lib().orc_paged_unit(_p(K), _p(V), _p(tags), L, D, _p(img) if img is not None else None,
                              _p(Kh) if Kh is not None else None, _p(Vh) if Vh is not None else None)
    if rc != 0:
        raise ValueError("orc_paged_unit rejected its arguments")
    return img, Kh, Vh


def paged_layer(K, V, tags, Q, G: int, want_image=True, want_out=True):
    """K, V: [B, Hkv, L, D] bf16 bits; tags [B, L]; Q [B, Hkv*G, D].  Returns (image, out)."""
    K = _u16(K)
    V = _u16(V)
    tags = np.ascontiguousarray(tags, np.uint8)
    B, Hkv, L, D = K.shape
    img = None
    if want_image:
        tot = sum(int(lib().orc_paged_unit_bytes(_p(np.ascontiguousarray(tags[b])), L, D)) for b in range(B)) * Hkv
        img = np.empty(tot, np.uint8)
    out = None
    Qp = None
    if want_out:
        Q = _u16(Q)
        out = np.empty((B, Hkv * G, D), np.float64)
        Qp = _p(Q)
    rc = lib().orc_paged_layer(_p(K), _p(V), _p(tags), Qp, B, Hkv, G, L, D,
                               _p(img) if img is not None else None, _p(out) if out is not None else None)
    if rc != 0:
        raise ValueError("orc_paged_layer rejected its arguments")
    return img, out


def paged_page4_bytes(D: int) -> int:
    return int(lib().orc_paged_page4_bytes(D))


def paged_rec2_bytes(D: int) -> int:
    return int(lib().orc_paged_rec2_bytes(D))
