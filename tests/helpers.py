"""Shared test helpers: device buffers, the documented workspace layout, comparisons."""
from __future__ import annotations

import numpy as np
import torch

from padding_free_varlen_b200 import capi, synth

SYNTH_TO_ENERGON = {synth.F32: capi.ENERGON_F32, synth.F16: capi.ENERGON_F16, synth.BF16: capi.ENERGON_BF16}
TORCH_OF_SYNTH = {synth.F32: torch.float32, synth.F16: torch.float16, synth.BF16: torch.bfloat16}


def to_device(a: np.ndarray, dtype: int, device="cuda") -> torch.Tensor:
    """Storage array from ``synth`` -> CUDA tensor of the matching torch dtype (same bits)."""
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype == synth.BF16:
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.to(device)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def to_storage(t: torch.Tensor) -> np.ndarray:
    """CUDA tensor -> numpy storage array (bf16 as uint16 bits)."""
    c = t.detach().cpu()
    if c.dtype == torch.bfloat16:
        return c.view(torch.int16).numpy().view(np.uint16)
    return c.numpy()


def align_up(v: int, a: int) -> int:
    return (v + a - 1) // a * a


def layer_ws_offsets(H: int, F: int, batch: int, pad_len: int, elem: int) -> dict:
    """Byte offsets of the intermediates a energon_layer_forward call leaves in its
    workspace (layout stated in include/energon_rce.h)."""
    R = align_up(batch * pad_len, 256)
    off, out = 0, {}
    for name, cols, eb in (("a", H, elem), ("qkv", 3 * H, elem), ("qk_lo", 2 * H if elem != 4 else 0, elem),
                           ("o", H, elem), ("x1", H, 4), ("f", F, elem)):
        out[name] = (off, cols)
        off = align_up(off + R * cols * eb, 1024)
    p32 = 4 * 128 * max(3 * H, F) * 4 if batch * pad_len <= 128 else 0
    out["p32"] = (off, p32)
    off = align_up(off + p32, 1024)
    out["stats"] = (off, 2)                       # float2 per row
    off = align_up(off + R * 8, 1024)
    out["fold"] = (off, 6 * H)                    # c [3H] then d [3H], fp32
    off = align_up(off + 6 * H * 4, 1024)
    out["_layer_bytes"] = off
    return out


def ws_view(ws: torch.Tensor, offs: dict, name: str, rows: int, dtype: torch.dtype) -> torch.Tensor:
    off, cols = offs[name]
    elem = torch.tensor([], dtype=dtype).element_size()
    return ws[off: off + rows * cols * elem].view(dtype).view(rows, cols)


def ulp(x: np.ndarray, dtype: int) -> np.ndarray:
    """Spacing of the storage type at |x| (fp16: 10 stored bits, bf16: 7, fp32: 23)."""
    mant = {synth.F16: 10, synth.BF16: 7, synth.F32: 23}[dtype]
    emin = {synth.F16: -14, synth.BF16: -126, synth.F32: -126}[dtype]
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** emin)))
    return 2.0 ** (e - mant)


MAX_ABS = 2e-2   # stated max-abs bound for fp16/bf16 layer outputs
REL_FRO = 5e-3   # stated relative Frobenius bound


def check_end_to_end(g: np.ndarray, r: np.ndarray, dtype: int, label: str, max_abs: bool = True):
    """Tolerance against the fp64 oracle for fp16 / bf16 layer outputs (fp32 accumulation):
    relative Frobenius error <= 5e-3 and max-abs error <= 2e-2, the latter above one
    rounding unit of the storage type at the reference value (a 16-bit output cannot sit
    closer to an fp64 value than its own rounding): max |g - r| - ulp(r) <= 2e-2.
    max_abs=False gates rel-Frobenius only (outputs of a stack of layers, where the stated
    bound applies to each layer's output, not to their composition); the max-abs figures
    are printed either way."""
    err = np.abs(g - r)
    e_max, e_fro = (float(err.max()) if err.size else 0.0), rel_frobenius(g, r)
    excess = float((err - ulp(r, dtype)).max()) if r.size else 0.0
    print(f"\n[{label}] max-abs {e_max:.3e} (beyond one ulp {excess:.3e}) rel-fro {e_fro:.3e}")
    assert e_fro <= REL_FRO, f"{label}: rel-Frobenius {e_fro:.3e} > {REL_FRO}"
    if max_abs:
        assert excess <= MAX_ABS, f"{label}: max-abs beyond one ulp {excess:.3e} > {MAX_ABS}"
    return e_max, e_fro, excess


def rel_frobenius(g: np.ndarray, r: np.ndarray) -> float:
    d = np.linalg.norm((g - r).ravel())
    n = np.linalg.norm(r.ravel())
    return float(d / n) if n > 0 else float(d)


def gpu_layer_weights(shape, layer, seed, dtype, recipe=None):
    """(numpy storage dict, CUDA tensor dict) of one layer's synthetic weights."""
    host = synth.layer_weights(shape, layer, seed, dtype, recipe)
    dev = {k: to_device(v, dtype) for k, v in host.items()}
    return host, dev
