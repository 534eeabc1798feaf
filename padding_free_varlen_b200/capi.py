"""Thin ctypes binding of ``libenergon_rce.so`` (the C ABI in ``include/energon_rce.h``).

Each function has the name of the C entry point it calls and only marshals
arguments: torch tensors become device pointers (after a check that each
holds the bytes the call will touch, since the C ABI takes sizes on trust),
streams become ``cudaStream_t`` handles, and a nonzero return code raises
``EnergonError`` with the library's message.  Every step of the path runs in
the CUDA library; if it is missing, the first call fails loudly.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libenergon_rce.so")

ENERGON_OK = 0
ENERGON_ERR_INVALID_ARGUMENT = 1
ENERGON_ERR_UNSUPPORTED = 2
ENERGON_ERR_MISALIGNED = 3
ENERGON_ERR_CUDA = 4
ENERGON_ERR_WORKSPACE_TOO_SMALL = 5
ENERGON_ERR_DEVICE_TIMEOUT = 6

ENERGON_DEVICE_OK = 0
ENERGON_DEVICE_BAD_LENGTH = 1
ENERGON_DEVICE_TIMEOUT = 2

ENERGON_F32, ENERGON_F16, ENERGON_BF16 = 0, 1, 2
TORCH_DTYPE = {ENERGON_F32: torch.float32, ENERGON_F16: torch.float16, ENERGON_BF16: torch.bfloat16}
DTYPE_OF = {v: k for k, v in TORCH_DTYPE.items()}

EXPORTED = ("energon_rce_offsets", "energon_rce_remove_padding", "energon_rce_rebuild_padding",
            "energon_workspace_bytes", "energon_layer_forward", "energon_stack_forward",
            "energon_selftest_bounded_wait", "energon_set_wait_timeout_us", "energon_last_error",
            "energon_trace_start", "energon_trace_stop", "energon_rce_remove_padding_noalloc",
            "energon_rce_transpose_padding_rebuild", "energon_rce_transpose_padding_remove",
            "energon_sched_plan", "energon_sched_fifo", "energon_kernel_binary_version",
            "energon_layer_fold_weights")
ENERGON_NOALLOC_MAX_BATCH = 16384
WEIGHT_FIELDS = ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o",
                 "ln2_g", "ln2_b", "w_1", "b_1", "w_2", "b_2")


class EnergonError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(msg)
        self.code = code


class energon_layer_config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_heads", ctypes.c_int), ("ffn", ctypes.c_int),
                ("dtype", ctypes.c_int), ("ln_eps", ctypes.c_float), ("gelu_tanh", ctypes.c_int)]


class energon_layer_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_FIELDS] + [("ln1_fold", ctypes.c_void_p)]


class energon_request(ctypes.Structure):
    _fields_ = [("length", ctypes.c_int32), ("arrival_s", ctypes.c_double)]


class energon_trace_entry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int), ("total_ms", ctypes.c_double)]


_lib = None


def load() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m padding_free_varlen_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, ci, sz, u32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint32
        cfgp, wp = ctypes.POINTER(energon_layer_config), ctypes.POINTER(energon_layer_weights)
        sigs = {
            "energon_rce_offsets": ([vp, ci, ci, vp, vp, vp], ci),
            "energon_rce_remove_padding": ([vp, vp, ci, ci, ci, ci, vp, vp], ci),
            "energon_rce_rebuild_padding": ([vp, vp, ci, ci, ci, ci, vp, vp], ci),
            "energon_rce_transpose_padding_rebuild": ([vp, vp, ci, ci, ci, ci, ci, ci, vp, vp], ci),
            "energon_rce_transpose_padding_remove": ([vp, vp, ci, ci, ci, ci, ci, ci, vp, vp], ci),
            "energon_workspace_bytes": ([cfgp, ci, ci], sz),
            "energon_layer_forward": ([cfgp, wp, vp, vp, ci, ci, vp, vp, vp, sz, vp], ci),
            "energon_stack_forward": ([cfgp, wp, ci, vp, vp, ci, ci, ci, vp, vp, vp, sz, vp], ci),
            "energon_selftest_bounded_wait": ([vp, u32, vp], ci),
            "energon_kernel_binary_version": ([ctypes.POINTER(ci)], ci),
            "energon_layer_fold_weights": ([cfgp, wp, vp, vp], ci),
            "energon_set_wait_timeout_us": ([u32], None),
            "energon_last_error": ([], ctypes.c_char_p),
            "energon_trace_start": ([], ci),
            "energon_rce_remove_padding_noalloc": ([vp, vp, ci, ci, ci, ci, vp, vp, vp], ci),
            "energon_trace_stop": ([ctypes.POINTER(energon_trace_entry), ci, ctypes.POINTER(ci)], ci),
            "energon_sched_plan": ([ctypes.POINTER(energon_request), ci, ctypes.c_double, ci,
                                    ctypes.POINTER(ctypes.c_double), ci, ctypes.c_double, ctypes.POINTER(ctypes.c_int32),
                                    ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)], ci),
            "energon_sched_fifo": ([ctypes.POINTER(energon_request), ci, ci, ctypes.POINTER(ctypes.c_int32),
                                    ctypes.POINTER(ctypes.c_int32)], ci),
        }
        for name, (args, res) in sigs.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _dev(x, what: str) -> int:
    """Device pointer of a CUDA tensor (or a raw integer address)."""
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    if not isinstance(x, torch.Tensor):
        raise TypeError(f"{what}: expected a CUDA tensor")
    if not x.is_cuda:
        raise ValueError(f"{what}: tensor must live on a CUDA device")
    if not x.is_contiguous():
        raise ValueError(f"{what}: tensor must be contiguous")
    return x.data_ptr()


def _need(x, nbytes: int, what: str) -> None:
    """A tensor argument must hold at least the bytes the call will touch (the C ABI takes
    the sizes on trust); raw integer addresses are the caller's responsibility."""
    if isinstance(x, torch.Tensor) and x.numel() * x.element_size() < nbytes:
        raise ValueError(f"{what}: {x.numel() * x.element_size()} bytes, the call needs {nbytes}")


_ELEM_BYTES = {0: 4, 1: 2, 2: 2}  # ENERGON_F32, ENERGON_F16, ENERGON_BF16


def _stream(s) -> int:
    if s is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc: int, name: str) -> None:
    if rc != ENERGON_OK:
        raise EnergonError(rc, f"{name} failed ({rc}): {load().energon_last_error().decode()}")


def energon_last_error() -> str:
    return load().energon_last_error().decode()


def energon_set_wait_timeout_us(timeout_us: int) -> None:
    load().energon_set_wait_timeout_us(int(timeout_us))


def energon_rce_offsets(lengths, batch, pad_len, cu_seqlens, d_status, stream=None) -> None:
    _need(lengths, 4 * batch, "lengths")
    _need(cu_seqlens, 4 * (batch + 1), "cu_seqlens")
    _check(load().energon_rce_offsets(_dev(lengths, "lengths"), batch, pad_len, _dev(cu_seqlens, "cu_seqlens"),
                                      _dev(d_status, "d_status"), _stream(stream)), "energon_rce_offsets")


def energon_rce_remove_padding(padded, cu_seqlens, batch, pad_len, hidden, elem_bytes, packed,
                               stream=None) -> None:
    _need(padded, batch * pad_len * hidden * elem_bytes, "padded")
    _need(packed, batch * pad_len * hidden * elem_bytes, "packed")
    _need(cu_seqlens, 4 * (batch + 1), "cu_seqlens")
    _check(load().energon_rce_remove_padding(_dev(padded, "padded"), _dev(cu_seqlens, "cu_seqlens"), batch,
                                             pad_len, hidden, elem_bytes, _dev(packed, "packed"), _stream(stream)),
           "energon_rce_remove_padding")


def energon_rce_rebuild_padding(packed, cu_seqlens, batch, pad_len, hidden, elem_bytes, padded,
                                stream=None) -> None:
    _need(padded, batch * pad_len * hidden * elem_bytes, "padded")
    _need(cu_seqlens, 4 * (batch + 1), "cu_seqlens")
    _check(load().energon_rce_rebuild_padding(_dev(packed, "packed"), _dev(cu_seqlens, "cu_seqlens"), batch,
                                              pad_len, hidden, elem_bytes, _dev(padded, "padded"), _stream(stream)),
           "energon_rce_rebuild_padding")


def energon_rce_transpose_padding_rebuild(packed, cu_seqlens, batch, pad_len, parts, n_heads, head_dim, elem_bytes,
                                          heads, stream=None) -> None:
    _need(heads, parts * batch * n_heads * pad_len * head_dim * elem_bytes, "heads")
    _need(cu_seqlens, 4 * (batch + 1), "cu_seqlens")
    _check(load().energon_rce_transpose_padding_rebuild(_dev(packed, "packed"), _dev(cu_seqlens, "cu_seqlens"), batch,
                                                        pad_len, parts, n_heads, head_dim, elem_bytes,
                                                        _dev(heads, "heads"), _stream(stream)),
           "energon_rce_transpose_padding_rebuild")


def energon_rce_transpose_padding_remove(heads, cu_seqlens, batch, pad_len, parts, n_heads, head_dim, elem_bytes,
                                         packed, stream=None) -> None:
    _need(heads, parts * batch * n_heads * pad_len * head_dim * elem_bytes, "heads")
    _need(cu_seqlens, 4 * (batch + 1), "cu_seqlens")
    _check(load().energon_rce_transpose_padding_remove(_dev(heads, "heads"), _dev(cu_seqlens, "cu_seqlens"), batch,
                                                       pad_len, parts, n_heads, head_dim, elem_bytes,
                                                       _dev(packed, "packed"), _stream(stream)),
           "energon_rce_transpose_padding_remove")


def energon_rce_remove_padding_noalloc(padded, lengths, batch, pad_len, hidden, elem_bytes, packed, d_status,
                                       stream=None) -> None:
    """Offsets + transpose_padding_remove with the offsets kept in the library's own
    fixed scratch array: for callers that cannot allocate (batch <= ENERGON_NOALLOC_MAX_BATCH)."""
    _need(padded, batch * pad_len * hidden * elem_bytes, "padded")
    _need(packed, batch * pad_len * hidden * elem_bytes, "packed")
    _need(lengths, 4 * batch, "lengths")
    _check(load().energon_rce_remove_padding_noalloc(_dev(padded, "padded"), _dev(lengths, "lengths"), batch, pad_len,
                                                     hidden, elem_bytes, _dev(packed, "packed"),
                                                     _dev(d_status, "d_status"), _stream(stream)),
           "energon_rce_remove_padding_noalloc")


def energon_workspace_bytes(cfg: energon_layer_config, batch: int, pad_len: int) -> int:
    return int(load().energon_workspace_bytes(ctypes.byref(cfg), batch, pad_len))


def energon_layer_forward(cfg, weights, x_packed, cu_seqlens, batch, max_len, y_packed, d_status, workspace,
                          ws_bytes, stream=None) -> None:
    rows_bytes = batch * max_len * cfg.hidden * _ELEM_BYTES.get(cfg.dtype, 4)
    _need(x_packed, rows_bytes, "x_packed")
    _need(y_packed, rows_bytes, "y_packed")
    _need(cu_seqlens, 4 * (batch + 1), "cu_seqlens")
    _need(workspace, ws_bytes, "workspace")
    _check(load().energon_layer_forward(ctypes.byref(cfg), ctypes.byref(weights), _dev(x_packed, "x_packed"),
                                        _dev(cu_seqlens, "cu_seqlens"), batch, max_len, _dev(y_packed, "y_packed"),
                                        _dev(d_status, "d_status"), _dev(workspace, "workspace"), ws_bytes,
                                        _stream(stream)), "energon_layer_forward")


def energon_stack_forward(cfg, layers, n_layers, padded_in, lengths, batch, pad_len, remove_padding, padded_out,
                          d_status, workspace, ws_bytes, stream=None) -> None:
    rows_bytes = batch * pad_len * cfg.hidden * _ELEM_BYTES.get(cfg.dtype, 4)
    _need(padded_in, rows_bytes, "padded_in")
    _need(padded_out, rows_bytes, "padded_out")
    _need(lengths, 4 * batch, "lengths")
    _need(workspace, ws_bytes, "workspace")
    arr = layers if isinstance(layers, ctypes.Array) else (energon_layer_weights * max(1, len(layers)))(*layers)
    _check(load().energon_stack_forward(ctypes.byref(cfg), arr, n_layers, _dev(padded_in, "padded_in"),
                                        _dev(lengths, "lengths"), batch, pad_len, int(remove_padding),
                                        _dev(padded_out, "padded_out"), _dev(d_status, "d_status"),
                                        _dev(workspace, "workspace"), ws_bytes, _stream(stream)),
           "energon_stack_forward")


def energon_selftest_bounded_wait(d_status, timeout_us, stream=None) -> None:
    _check(load().energon_selftest_bounded_wait(_dev(d_status, "d_status"), int(timeout_us), _stream(stream)),
           "energon_selftest_bounded_wait")


def energon_layer_fold_weights(cfg, weights, fold, stream=None) -> None:
    _check(load().energon_layer_fold_weights(ctypes.byref(cfg), ctypes.byref(weights), _dev(fold, "fold"),
                                             _stream(stream)), "energon_layer_fold_weights")


def energon_kernel_binary_version() -> int:
    v = ctypes.c_int(0)
    _check(load().energon_kernel_binary_version(ctypes.byref(v)), "energon_kernel_binary_version")
    return v.value


def energon_trace_start() -> None:
    _check(load().energon_trace_start(), "energon_trace_start")


def energon_trace_stop() -> dict:
    """{kernel name: (launches, total device ms)} of the launches traced since the start."""
    cap = 64
    arr = (energon_trace_entry * cap)()
    n = ctypes.c_int(0)
    _check(load().energon_trace_stop(arr, cap, ctypes.byref(n)), "energon_trace_stop")
    return {arr[i].name.decode(): (arr[i].launches, arr[i].total_ms) for i in range(min(n.value, cap))}


def _requests(lengths, arrivals):
    n = len(lengths)
    if len(arrivals) != n:
        raise ValueError("lengths and arrivals differ in size")
    arr = (energon_request * max(1, n))()
    for i in range(n):
        arr[i].length = int(lengths[i])
        arr[i].arrival_s = float(arrivals[i])
    return arr, n


def energon_sched_plan(lengths, arrivals, now_s, max_batch, cost_table, age_scale_s):
    """Dynamic batching decision for a queue snapshot (host only).  cost_table: nested
    [max_batch][table_max_len] of positive costs.  Returns (group_of, order) as lists."""
    reqs, n = _requests(lengths, arrivals)
    rows = len(cost_table)
    width = len(cost_table[0]) if rows else 0
    flat = (ctypes.c_double * max(1, rows * width))(*[float(v) for row in cost_table for v in row])
    group_of = (ctypes.c_int32 * max(1, n))()
    order = (ctypes.c_int32 * max(1, n))()
    ng = ctypes.c_int32(0)
    if rows < min(max_batch, n):
        raise ValueError("cost_table has fewer rows than the batch sizes it must price")
    _check(load().energon_sched_plan(reqs, n, float(now_s), int(max_batch), flat, width, float(age_scale_s),
                                     group_of, ctypes.byref(ng), order), "energon_sched_plan")
    return [group_of[i] for i in range(n)], [order[g] for g in range(ng.value)]


def energon_sched_fifo(arrivals, max_batch):
    """FIFO packing: group_of for requests in arrival order (host only)."""
    reqs, n = _requests([1] * len(arrivals), arrivals)
    group_of = (ctypes.c_int32 * max(1, n))()
    ng = ctypes.c_int32(0)
    _check(load().energon_sched_fifo(reqs, n, int(max_batch), group_of, ctypes.byref(ng)), "energon_sched_fifo")
    return [group_of[i] for i in range(n)]


# ----------------------------------------------------------------------------- struct helpers


def make_config(hidden: int, n_heads: int, ffn: int, dtype: int, ln_eps: float = 1e-5,
                gelu_tanh: bool = True) -> energon_layer_config:
    return energon_layer_config(hidden, n_heads, ffn, dtype, ln_eps, int(gelu_tanh))


def make_weights(tensors: dict) -> energon_layer_weights:
    """Weight table of one layer from a dict of CUDA tensors (the dict must outlive its use);
    an "ln1_fold" entry (fp32 [6H], from energon_layer_fold_weights) is optional."""
    return energon_layer_weights(*[_dev(tensors[n], n) for n in WEIGHT_FIELDS],
                                 _dev(tensors.get("ln1_fold"), "ln1_fold"))
