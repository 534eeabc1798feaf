"""ORACLE - test infrastructure only.

ctypes front-end of ``oracle.c``: the fp64 CPU statement of the padding-free
varlen GPT-3 layer stack (offsets, transpose_padding_remove,
transpose_padding_rebuild, pre-LN decoder layer, stack).  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` use it.
It imports nothing from the CUDA package; the seeded input generator is the
one piece both sides share, and it holds none of the method's arithmetic.

Weights are handed over in their storage type (f32 / f16 / bf16 bits) and
decoded exactly to double inside the C code; activations are float64 arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

# Storage codes understood by oracle.c.
OR_F32, OR_F16, OR_BF16, OR_F64 = 0, 1, 2, 3
_NP_CODE = {np.dtype(np.float32): OR_F32, np.dtype(np.float16): OR_F16,
            np.dtype(np.uint16): OR_BF16, np.dtype(np.float64): OR_F64}
WEIGHT_FIELDS = ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o",
                 "ln2_g", "ln2_b", "w_1", "b_1", "w_2", "b_2")


# A test may point the wrapper at a deliberately broken copy of the oracle
# (mutation testing of the pins); nothing else sets this.
_OVERRIDE = os.environ.get("ORACLE_LIB_OVERRIDE")


def compile_to(src: str, out: str) -> None:
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                           "-ffp-contract=off", "-o", out, src, "-lm"])


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` (gcc -O2, OpenMP; no fast-math, no FMA contraction)."""
    if _OVERRIDE:
        return _OVERRIDE
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        compile_to(_SRC, tmp)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Cfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_heads", ctypes.c_int), ("ffn", ctypes.c_int),
                ("wdtype", ctypes.c_int), ("ln_eps", ctypes.c_double), ("gelu_tanh", ctypes.c_int)]


class _Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_FIELDS]


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        vp, i64, ci, dbl = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        sig = {
            "oracle_decode": [vp, ci, i64, vp],
            "oracle_offsets": [vp, ci, ci, vp, vp],
            "oracle_remove_padding": [vp, vp, ci, ci, i64, vp],
            "oracle_rebuild_padding": [vp, vp, ci, ci, i64, vp],
            "oracle_transpose_padding_rebuild": [vp, vp, ci, ci, ci, ci, i64, vp],
            "oracle_transpose_padding_remove": [vp, vp, ci, ci, ci, ci, i64, vp],
            "oracle_layernorm": [vp, i64, ci, vp, vp, ci, dbl, vp],
            "oracle_linear": [vp, i64, ci, vp, vp, ci, ci, vp],
            "oracle_gelu": [vp, i64, ci, vp],
            "oracle_causal_attention": [vp, ci, ci, ci, vp],
            "oracle_layer_sequence": [ctypes.POINTER(_Cfg), ctypes.POINTER(_Weights), vp, ci, vp],
            "oracle_layer_padded": [ctypes.POINTER(_Cfg), ctypes.POINTER(_Weights), vp, vp, ci, ci, vp],
        }
        for name, args in sig.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise RuntimeError(f"{what}: oracle status {rc}")


def code_of(a: np.ndarray) -> int:
    """Storage code of a numpy array (uint16 means bf16 bits)."""
    return _NP_CODE[a.dtype]


def decode(a: np.ndarray) -> np.ndarray:
    """Exact float64 values of a storage array (f32, f16, bf16-as-uint16, f64)."""
    a = np.ascontiguousarray(a)
    out = np.empty(a.shape, dtype=np.float64)
    _check(_L().oracle_decode(_ptr(a), code_of(a), a.size, _ptr(out)), "decode")
    return out


def offsets(lengths: np.ndarray, pad_len: int):
    """(cu_seqlens[int32, batch+1], status) - exclusive prefix sum of the lengths."""
    lengths = np.ascontiguousarray(lengths, dtype=np.int32)
    cu = np.empty(lengths.size + 1, dtype=np.int32)
    st = np.zeros(1, dtype=np.int32)
    _check(_L().oracle_offsets(_ptr(lengths), lengths.size, pad_len, _ptr(cu), _ptr(st)), "offsets")
    return cu, int(st[0])


def remove_padding(padded: np.ndarray, cu: np.ndarray, out: np.ndarray | None = None) -> np.ndarray:
    """padded [B, S, ...] -> packed [capacity, ...] (rows >= cu[B] of ``out`` untouched)."""
    padded = np.ascontiguousarray(padded)
    B, S = padded.shape[:2]
    row_bytes = padded.itemsize * int(np.prod(padded.shape[2:]))
    cu = np.ascontiguousarray(cu, dtype=np.int32)
    if out is None:
        out = np.zeros((B * S,) + padded.shape[2:], dtype=padded.dtype)
    _check(_L().oracle_remove_padding(_ptr(padded), _ptr(cu), B, S, row_bytes, _ptr(out)), "remove")
    return out


def rebuild_padding(packed: np.ndarray, cu: np.ndarray, batch: int, pad_len: int,
                    out: np.ndarray | None = None) -> np.ndarray:
    """packed [>=cu[B], ...] -> padded [B, S, ...] with all-zero pad rows."""
    packed = np.ascontiguousarray(packed)
    row_bytes = packed.itemsize * int(np.prod(packed.shape[1:]))
    cu = np.ascontiguousarray(cu, dtype=np.int32)
    if out is None:
        out = np.empty((batch, pad_len) + packed.shape[1:], dtype=packed.dtype)
    _check(_L().oracle_rebuild_padding(_ptr(packed), _ptr(cu), batch, pad_len, row_bytes, _ptr(out)),
           "rebuild")
    return out


def transpose_padding_rebuild(packed: np.ndarray, cu: np.ndarray, batch: int, pad_len: int, parts: int,
                              n_heads: int, out: np.ndarray | None = None) -> np.ndarray:
    """packed [>=cu[B], parts * n_heads * d] -> head-major [parts, B, n_heads, S, d], zero pads."""
    packed = np.ascontiguousarray(packed)
    width = packed.shape[1]
    assert width % (parts * n_heads) == 0
    d = width // (parts * n_heads)
    cu = np.ascontiguousarray(cu, dtype=np.int32)
    if out is None:
        out = np.empty((parts, batch, n_heads, pad_len, d), dtype=packed.dtype)
    _check(_L().oracle_transpose_padding_rebuild(_ptr(packed), _ptr(cu), batch, pad_len, parts, n_heads,
                                                 d * packed.itemsize, _ptr(out)), "transpose rebuild")
    return out


def transpose_padding_remove(heads: np.ndarray, cu: np.ndarray, out: np.ndarray | None = None) -> np.ndarray:
    """head-major [parts, B, n_heads, S, d] -> packed [capacity, parts * n_heads * d]
    (rows >= cu[B] of ``out`` untouched)."""
    heads = np.ascontiguousarray(heads)
    parts, B, nh, S, d = heads.shape
    cu = np.ascontiguousarray(cu, dtype=np.int32)
    if out is None:
        out = np.zeros((B * S, parts * nh * d), dtype=heads.dtype)
    _check(_L().oracle_transpose_padding_remove(_ptr(heads), _ptr(cu), B, S, parts, nh, d * heads.itemsize,
                                                _ptr(out)), "transpose remove")
    return out


def layernorm(x: np.ndarray, g: np.ndarray, b: np.ndarray, eps: float = 1e-5) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    g, b = np.ascontiguousarray(g), np.ascontiguousarray(b)
    assert g.dtype == b.dtype
    H = x.shape[-1]
    y = np.empty_like(x)
    _check(_L().oracle_layernorm(_ptr(x), x.size // H, H, _ptr(g), _ptr(b), code_of(g), eps, _ptr(y)),
           "layernorm")
    return y


def linear(x: np.ndarray, W: np.ndarray, bias: np.ndarray | None = None) -> np.ndarray:
    """y = x W^T + bias with W in [out, in] layout (storage type)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    W = np.ascontiguousarray(W)
    N, K = W.shape
    assert x.shape[-1] == K
    rows = x.size // K
    y = np.empty(x.shape[:-1] + (N,), dtype=np.float64)
    bp = None
    if bias is not None:
        bias = np.ascontiguousarray(bias)
        assert bias.dtype == W.dtype
        bp = _ptr(bias)
    _check(_L().oracle_linear(_ptr(x), rows, K, _ptr(W), bp, N, code_of(W), _ptr(y)), "linear")
    return y


def gelu(x: np.ndarray, tanh_form: bool = True) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    _check(_L().oracle_gelu(_ptr(x), x.size, int(tanh_form), _ptr(y)), "gelu")
    return y


def causal_attention(qkv: np.ndarray, n_heads: int) -> np.ndarray:
    """One sequence: qkv [L, 3H] ([Q | K | V], head-major) -> o [L, H]."""
    qkv = np.ascontiguousarray(qkv, dtype=np.float64)
    L, H3 = qkv.shape
    H = H3 // 3
    o = np.empty((L, H), dtype=np.float64)
    _check(_L().oracle_causal_attention(_ptr(qkv), L, H, n_heads, _ptr(o)), "attention")
    return o


def _structs(weights: dict, hidden: int, n_heads: int, ffn: int, eps: float, gelu_tanh: bool):
    arrs = {n: np.ascontiguousarray(weights[n]) for n in WEIGHT_FIELDS}
    codes = {code_of(a) for a in arrs.values()}
    if len(codes) != 1:
        raise ValueError("all weight tensors of a layer must share one storage type")
    cfg = _Cfg(hidden, n_heads, ffn, codes.pop(), eps, int(gelu_tanh))
    w = _Weights(*[_ptr(arrs[n]) for n in WEIGHT_FIELDS])
    return cfg, w, arrs


def layer_sequence(x: np.ndarray, weights: dict, n_heads: int, eps: float = 1e-5,
                   gelu_tanh: bool = True) -> np.ndarray:
    """One pre-LN GPT layer on the valid tokens of one sequence: x [L, H] float64."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    L, H = x.shape
    ffn = weights["w_1"].shape[0]
    cfg, w, keep = _structs(weights, H, n_heads, ffn, eps, gelu_tanh)
    y = np.empty_like(x)
    _check(_L().oracle_layer_sequence(ctypes.byref(cfg), ctypes.byref(w), _ptr(x), L, _ptr(y)),
           "layer_sequence")
    return y


def layer_padded(x_padded: np.ndarray, lengths: np.ndarray, weights: dict, n_heads: int,
                 eps: float = 1e-5, gelu_tanh: bool = True) -> np.ndarray:
    """The layer on a padded batch [B, S, H] (float64); pad rows of the result are 0."""
    x = np.ascontiguousarray(x_padded, dtype=np.float64)
    B, S, H = x.shape
    lengths = np.ascontiguousarray(lengths, dtype=np.int32)
    ffn = weights["w_1"].shape[0]
    cfg, w, keep = _structs(weights, H, n_heads, ffn, eps, gelu_tanh)
    y = np.empty_like(x)
    _check(_L().oracle_layer_padded(ctypes.byref(cfg), ctypes.byref(w), _ptr(x), _ptr(lengths), B, S,
                                    _ptr(y)), "layer_padded")
    return y


def stack_padded(x_padded: np.ndarray, lengths: np.ndarray, layer_weights, n_layers: int,
                 n_heads: int, eps: float = 1e-5, gelu_tanh: bool = True) -> np.ndarray:
    """``n_layers`` layers on a padded batch; ``layer_weights(l)`` returns layer l's tensors
    (called once per layer, so weights can be regenerated one layer at a time).
    No final LayerNorm; pad rows are 0."""
    y = np.ascontiguousarray(x_padded, dtype=np.float64)
    for l in range(n_layers):
        y = layer_padded(y, lengths, layer_weights(l), n_heads, eps, gelu_tanh)
    return y
