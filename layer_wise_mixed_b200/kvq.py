"""Python binding of the C ABI in include/kvq.h (ctypes; argument marshalling only).

Every function keeps the C name and forwards to libkvq.so; all computation runs in
the library's CUDA kernels.  There is no fallback: if libkvq.so is missing this module
raises on first use.  PyTorch appears only to pass device pointers and the current
CUDA stream, and (in ``Cache``) to allocate the caller-owned workspace.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import List, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "kvq.h")

KVQ_OK = 0
KVQ_EINVAL = -1
KVQ_EUNSUPPORTED = -2
KVQ_ECAPACITY = -3
KVQ_EUNBOUND = -4
KVQ_EALIGN = -5
KVQ_ECUDA = -6
KVQ_EDEVICE = -7
KVQ_PER_CHANNEL = 0
KVQ_PER_TOKEN = 1
KVQ_DECODE_MMA_SYNC = 0
KVQ_DECODE_TCGEN05 = 1

_NAMES = {0: "KVQ_OK", -1: "KVQ_EINVAL", -2: "KVQ_EUNSUPPORTED", -3: "KVQ_ECAPACITY",
          -4: "KVQ_EUNBOUND", -5: "KVQ_EALIGN", -6: "KVQ_ECUDA", -7: "KVQ_EDEVICE"}


class KvqError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{_NAMES.get(code, code)}: {msg}")
        self.code = code


class kvq_layer_cfg(ctypes.Structure):
    _fields_ = [("bk", ctypes.c_int), ("bv", ctypes.c_int), ("kmode", ctypes.c_int), ("vmode", ctypes.c_int)]


class kvq_plan_desc(ctypes.Structure):
    _fields_ = [("num_layers", ctypes.c_int), ("batch", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
                ("n_q_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("group", ctypes.c_int),
                ("max_ctx", ctypes.c_int), ("layers", ctypes.POINTER(kvq_layer_cfg)),
                ("paged", ctypes.c_int), ("page_tokens", ctypes.c_int), ("avg_bits", ctypes.c_float),
                ("pool_blocks", ctypes.c_int)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libkvq.so (raises FileNotFoundError if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise FileNotFoundError(f"{LIB_PATH} is missing: build it with `python -m layer_wise_mixed_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sig = {
        "kvq_plan": (I, [ctypes.POINTER(kvq_plan_desc), ctypes.POINTER(P)]),
        "kvq_workspace_bytes": (I, [P, ctypes.POINTER(SZ)]),
        "kvq_bind": (I, [P, P, SZ]),
        "kvq_append": (I, [P, I, P, P, I, P]),
        "kvq_append_tagged": (I, [P, I, P, P, I, P, P, P]),
        "kvq_append_ragged": (I, [P, I, P, P, P, I, P]),
        "kvq_seq_lens": (I, [P, I, P]),
        "kvq_decode_attn": (I, [P, I, P, P, I, P]),
        "kvq_append_decode": (I, [P, I, P, P, P, P, I, P]),
        "kvq_decode_attn_noalloc": (I, [P, I, P, P, I, P]),
        "kvq_set_num_splits": (I, [P, I]),
        "kvq_set_decode_path": (I, [P, I]),
        "kvq_get_num_splits": (I, [P, I, ctypes.POINTER(I)]),
        "kvq_export_layer": (I, [P, I, P, SZ, ctypes.POINTER(SZ)]),
        "kvq_seq_len": (I, [P, I, ctypes.POINTER(I)]),
        "kvq_truncate": (I, [P, I, I]),
        "kvq_reset_sequences": (I, [P, P, I]),
        "kvq_device_status": (I, [P, P, ctypes.POINTER(ctypes.c_uint)]),
        "kvq_tag_distortion": (I, [I, I, I, I, I, I, P, P, P, P, I, P, P, P]),
        "kvq_tag_allocate": (I, [I, P, P, P, ctypes.c_double, P, P]),
        "kvq_tag_distortion_workspace_bytes": (I, [I, I, I, I, I, I, I, ctypes.POINTER(SZ)]),
        "kvq_tag_distortion_device": (I, [I, I, I, I, I, I, P, P, P, P, I, P, SZ, P, P, P, P]),
        "kvq_destroy": (None, [P]),
        "kvq_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def header_functions() -> List[str]:
    """Names of the functions declared in include/kvq.h."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*KVQ_API\s+(?:int|void|const char)\s*\*?\s*(kvq_\w+)\s*\(", text, re.M)))


def _check(rc: int):
    if rc != KVQ_OK:
        raise KvqError(rc, load().kvq_last_error().decode())
    return rc


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr(x) -> int:
    return x if isinstance(x, int) else x.data_ptr()


# ------------------------------------------------------------------ C names
def kvq_plan(desc: kvq_plan_desc) -> int:
    h = ctypes.c_void_p()
    _check(load().kvq_plan(ctypes.byref(desc), ctypes.byref(h)))
    return h.value


def kvq_workspace_bytes(h: int) -> int:
    n = ctypes.c_size_t()
    _check(load().kvq_workspace_bytes(h, ctypes.byref(n)))
    return n.value


def kvq_bind(h: int, dev_ptr: int, nbytes: int):
    _check(load().kvq_bind(h, dev_ptr, nbytes))


def kvq_append(h: int, layer: int, K, V, n_new: int, stream=None):
    _check(load().kvq_append(h, layer, _ptr(K), _ptr(V), n_new, _stream(stream)))


def kvq_append_tagged(h: int, layer: int, K, V, n_new: int, host_tags, dev_tags, stream=None):
    """host_tags: contiguous uint8 numpy array [B, n_new]; dev_tags: the same bytes on the device."""
    host_tags = np.ascontiguousarray(host_tags, np.uint8)
    _check(load().kvq_append_tagged(h, layer, _ptr(K), _ptr(V), n_new, host_tags.ctypes.data_as(ctypes.c_void_p),
                                    _ptr(dev_tags), _stream(stream)))


def kvq_append_ragged(h: int, layer: int, K, V, n_new, stream=None):
    """K, V [B, Hkv, n_max, D]; request b appends its first n_new[b] tokens."""
    import numpy as np
    n = np.ascontiguousarray(n_new, np.int32)
    _check(load().kvq_append_ragged(h, layer, _ptr(K), _ptr(V), n.ctypes.data_as(ctypes.c_void_p), K.shape[2],
                                    _stream(stream)))


def kvq_seq_lens(h: int, layer: int, batch: int):
    import numpy as np
    out = np.zeros(batch, np.int32)
    _check(load().kvq_seq_lens(h, layer, out.ctypes.data_as(ctypes.c_void_p)))
    return out


def kvq_decode_attn(h: int, layer: int, q, out, out_fp32: bool, stream=None):
    _check(load().kvq_decode_attn(h, layer, _ptr(q), _ptr(out), int(bool(out_fp32)), _stream(stream)))


def kvq_append_decode(h: int, layer: int, K, V, q, out, out_fp32: bool, stream=None):
    _check(load().kvq_append_decode(h, layer, _ptr(K), _ptr(V), _ptr(q), _ptr(out), int(bool(out_fp32)),
                                    _stream(stream)))


def kvq_decode_attn_noalloc(h: int, layer: int, q, out, out_fp32: bool, stream=None):
    _check(load().kvq_decode_attn_noalloc(h, layer, _ptr(q), _ptr(out), int(bool(out_fp32)), _stream(stream)))


def kvq_set_num_splits(h: int, n: int):
    _check(load().kvq_set_num_splits(h, n))


def kvq_set_decode_path(h: int, path: int):
    _check(load().kvq_set_decode_path(h, path))


def kvq_get_num_splits(h: int, layer: int) -> int:
    n = ctypes.c_int()
    _check(load().kvq_get_num_splits(h, layer, ctypes.byref(n)))
    return n.value


def kvq_export_layer(h: int, layer: int) -> np.ndarray:
    need = ctypes.c_size_t()
    _check(load().kvq_export_layer(h, layer, None, 0, ctypes.byref(need)))
    buf = np.empty(need.value, np.uint8)
    _check(load().kvq_export_layer(h, layer, buf.ctypes.data_as(ctypes.c_void_p), buf.nbytes,
                                   ctypes.byref(need)))
    return buf


def kvq_seq_len(h: int, layer: int) -> int:
    n = ctypes.c_int()
    _check(load().kvq_seq_len(h, layer, ctypes.byref(n)))
    return n.value


def kvq_truncate(h: int, layer: int, L: int):
    _check(load().kvq_truncate(h, layer, L))


def kvq_reset_sequences(h: int, seqs):
    n = np.ascontiguousarray(seqs, np.int32)
    _check(load().kvq_reset_sequences(h, n.ctypes.data_as(ctypes.c_void_p), n.size))


def kvq_device_status(h: int, stream=None) -> int:
    f = ctypes.c_uint()
    rc = load().kvq_device_status(h, _stream(stream), ctypes.byref(f))
    _check(rc)
    return f.value


def kvq_destroy(h: int):
    load().kvq_destroy(h)


def kvq_last_error() -> str:
    return load().kvq_last_error().decode()


def kvq_tag_distortion(Q, K, V, tags, num_tags: int):
    """Per-tag distortion from calibration prefills (host numpy arrays): Q uint16 (bf16
    bits) [NL, R, Hq, T, D], K/V [NL, R, Hkv, T, D], tags int32 [R, T].
    Returns (D2, D4, counts)."""
    import numpy as np
    Q = np.ascontiguousarray(Q, np.uint16)
    K = np.ascontiguousarray(K, np.uint16)
    V = np.ascontiguousarray(V, np.uint16)
    tags = np.ascontiguousarray(tags, np.int32)
    NL, R, Hq, T, D = Q.shape
    Hkv = K.shape[2]
    if K.shape != (NL, R, Hkv, T, D) or V.shape != K.shape or tags.shape != (R, T):
        raise ValueError("shape mismatch")
    D2 = np.zeros(num_tags, np.float64)
    D4 = np.zeros(num_tags, np.float64)
    counts = np.zeros(num_tags, np.int64)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _check(load().kvq_tag_distortion(NL, R, Hq, Hkv, D, T, p(Q), p(K), p(V), p(tags), num_tags, p(D2), p(D4),
                                     p(counts)))
    return D2, D4, counts


def kvq_tag_distortion_workspace_bytes(NL: int, R: int, Hq: int, Hkv: int, D: int, T: int, num_tags: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load().kvq_tag_distortion_workspace_bytes(NL, R, Hq, Hkv, D, T, num_tags, ctypes.byref(n)))
    return n.value


def kvq_tag_distortion_device(Q, K, V, tags, num_tags: int, workspace=None, stream=None):
    """kvq_tag_distortion on the GPU: Q, K, V CUDA tensors (bf16 or int16/uint16 holding bf16
    bits) [NL, R, Hq, T, D] / [NL, R, Hkv, T, D]; tags host int32 [R, T].  The workspace
    (a CUDA uint8 tensor) is allocated here when not given.  Returns (D2, D4, counts)."""
    import numpy as np
    import torch
    for a in (Q, K, V):
        if not (a.is_cuda and a.is_contiguous() and a.element_size() == 2):
            raise ValueError("Q, K, V must be contiguous 2-byte CUDA tensors")
    tags = np.ascontiguousarray(tags, np.int32)
    NL, R, Hq, T, D = Q.shape
    Hkv = K.shape[2]
    if tuple(K.shape) != (NL, R, Hkv, T, D) or tuple(V.shape) != tuple(K.shape) or tags.shape != (R, T):
        raise ValueError("shape mismatch")
    need = kvq_tag_distortion_workspace_bytes(NL, R, Hq, Hkv, D, T, num_tags)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    D2 = np.zeros(num_tags, np.float64)
    D4 = np.zeros(num_tags, np.float64)
    counts = np.zeros(num_tags, np.int64)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    st = _stream(stream)
    _check(load().kvq_tag_distortion_device(NL, R, Hq, Hkv, D, T, Q.data_ptr(), K.data_ptr(), V.data_ptr(), p(tags),
                                            num_tags, workspace.data_ptr(), workspace.numel(), p(D2), p(D4),
                                            p(counts), st))
    return D2, D4, counts


def kvq_tag_allocate(D2, D4, counts, avg_bits: float):
    """INT2/INT4 per tag under the average-bit budget: (bits int32 [K], total distortion)."""
    import numpy as np
    D2 = np.ascontiguousarray(D2, np.float64)
    D4 = np.ascontiguousarray(D4, np.float64)
    counts = np.ascontiguousarray(counts, np.int64)
    bits = np.zeros(len(counts), np.int32)
    total = ctypes.c_double(0.0)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _check(load().kvq_tag_allocate(len(counts), p(D2), p(D4), p(counts), float(avg_bits), p(bits),
                                   ctypes.byref(total)))
    return bits, total.value


# ------------------------------------------------------------------ convenience owner
def make_paged_desc(num_layers: int, batch: int, n_kv_heads: int, n_q_heads: int, head_dim: int, max_ctx: int,
                    avg_bits: float):
    return kvq_plan_desc(num_layers, batch, n_kv_heads, n_q_heads, head_dim, 32, max_ctx, None, 1, 16, avg_bits, 0)


def make_desc(num_layers: int, batch: int, n_kv_heads: int, n_q_heads: int, head_dim: int, max_ctx: int,
              layer_bits: Sequence[Tuple[int, int]], kmodes: Optional[Sequence[int]] = None, pool_blocks: int = 0):
    cfgs = (kvq_layer_cfg * num_layers)()
    for i, (bk, bv) in enumerate(layer_bits):
        cfgs[i] = kvq_layer_cfg(bk, bv, KVQ_PER_CHANNEL if kmodes is None else kmodes[i], KVQ_PER_TOKEN)
    d = kvq_plan_desc(num_layers, batch, n_kv_heads, n_q_heads, head_dim, 32, max_ctx, cfgs, 0, 16, 0.0, pool_blocks)
    d._cfgs = cfgs   # keep the array alive with the descriptor
    return d


class Cache:
    """A plan plus a torch-allocated workspace on the current CUDA device.  Pass
    avg_bits (and no layer_bits) for a paged INT2/INT4 plan."""

    def __init__(self, num_layers, batch, n_kv_heads, n_q_heads, head_dim, max_ctx, layer_bits=None,
                 kmodes=None, device="cuda", avg_bits=None, pool_blocks=0):
        import torch
        if avg_bits is not None:
            self.desc = make_paged_desc(num_layers, batch, n_kv_heads, n_q_heads, head_dim, max_ctx, avg_bits)
        else:
            self.desc = make_desc(num_layers, batch, n_kv_heads, n_q_heads, head_dim, max_ctx, layer_bits, kmodes,
                                  pool_blocks)
        self.h = kvq_plan(self.desc)
        self._destroy = load().kvq_destroy   # held so that teardown at interpreter exit still works
        self.nbytes = kvq_workspace_bytes(self.h)
        self.ws = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device)
        base = self.ws.data_ptr()
        self.ws_ptr = (base + 255) // 256 * 256
        kvq_bind(self.h, self.ws_ptr, self.nbytes)
        self.B, self.Hkv, self.Hq, self.D = batch, n_kv_heads, n_q_heads, head_dim

    def append(self, layer, K, V, stream=None):
        assert K.is_contiguous() and V.is_contiguous() and K.shape == V.shape
        kvq_append(self.h, layer, K, V, K.shape[2], stream)

    def append_tagged(self, layer, K, V, tags, stream=None):
        """tags: uint8 torch tensor [B, n] (2 or 4) on the device."""
        assert K.is_contiguous() and V.is_contiguous() and K.shape == V.shape
        kvq_append_tagged(self.h, layer, K, V, K.shape[2], tags.cpu().numpy(), tags, stream)

    def decode_attn(self, layer, q, out=None, out_fp32=False, stream=None):
        import torch
        if out is None:
            out = torch.empty((self.B, self.Hq, self.D), dtype=torch.float32 if out_fp32 else torch.bfloat16,
                              device=q.device)
        kvq_decode_attn(self.h, layer, q, out, out_fp32, stream)
        return out

    def append_decode(self, layer, K, V, q, out=None, out_fp32=False, stream=None):
        """One decode step: append the token K, V [B, Hkv, 1, D] and attend with q."""
        import torch
        assert K.is_contiguous() and V.is_contiguous() and K.shape == V.shape and K.shape[2] == 1
        if out is None:
            out = torch.empty((self.B, self.Hq, self.D), dtype=torch.float32 if out_fp32 else torch.bfloat16,
                              device=q.device)
        kvq_append_decode(self.h, layer, K, V, q, out, out_fp32, stream)
        return out

    def append_ragged(self, layer, K, V, n_new, stream=None):
        """K, V [B, Hkv, n_max, D] (contiguous); request b appends its first n_new[b] tokens."""
        assert K.is_contiguous() and V.is_contiguous() and K.shape == V.shape
        kvq_append_ragged(self.h, layer, K, V, n_new, stream)

    def seq_lens(self, layer):
        return kvq_seq_lens(self.h, layer, self.B)

    def export_layer(self, layer):
        return kvq_export_layer(self.h, layer)

    def seq_len(self, layer):
        return kvq_seq_len(self.h, layer)

    def __del__(self):
        h = getattr(self, "h", None)
        destroy = getattr(self, "_destroy", None)
        if h and destroy is not None:
            destroy(h)
            self.h = None
