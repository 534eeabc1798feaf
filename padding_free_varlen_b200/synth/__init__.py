"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module draws random numbers and nothing else: no step of the method
(offsets, packing, LayerNorm, GEMM, attention) is computed here.  The C
generator (``synth.c``) is counter-based, so any slice of any tensor of any
layer is reproducible on its own; that lets the oracle regenerate one layer's
weights at a time and lets the bench write 43.5 GB of weights straight into
pinned buffers.

Workload recipes follow the five workloads the Energon-AI pages measure or
imply (GPT-3 12 layers FP16 with sequence length half the padding length;
random lengths up to 256 padded to the batch maximum) restated as synthetic,
seeded inputs: N(0, 1) activations (pad positions included, as garbage),
N(0, 0.02) weights, zero biases, LayerNorm gamma = 1 and beta = 0.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")

F32, F16, BF16, F64 = 0, 1, 2, 3
DTYPE_NAMES = {F32: "f32", F16: "f16", BF16: "bf16", F64: "f64"}
DTYPE_BYTES = {F32: 4, F16: 2, BF16: 2, F64: 8}
_NP_STORAGE = {F32: np.float32, F16: np.float16, BF16: np.uint16, F64: np.float64}

# Stream identifiers (the "tensor" key of the counter-based generator).
TID_LENGTHS = 1
TID_X = 2
TID_X_ALT_PADS = 3
TID_LAYER_BASE = 1000
WEIGHT_NAMES = ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o",
                "ln2_g", "ln2_b", "w_1", "b_1", "w_2", "b_2")


def build(force: bool = False) -> str:
    """Compile ``libsynth.so`` next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, u64, dbl, vp = ctypes.c_int64, ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p
        lib.synth_normal.argtypes = [u64, u64, i64, i64, dbl, dbl, ctypes.c_int, vp]
        lib.synth_uniform.argtypes = [u64, u64, i64, i64, vp]
        lib.synth_uniform_int.argtypes = [u64, u64, i64, ctypes.c_int32, ctypes.c_int32, vp]
        lib.synth_raw.argtypes = [u64, u64, i64, i64, vp]
        lib.synth_round.argtypes = [vp, i64, ctypes.c_int, vp]
        for f in (lib.synth_normal, lib.synth_uniform, lib.synth_uniform_int, lib.synth_raw, lib.synth_round):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def fill_normal_ptr(ptr: int, n: int, seed: int, tensor: int, dtype: int,
                    mean: float = 0.0, std: float = 1.0, offset: int = 0) -> None:
    """Write n normal draws (rounded to ``dtype``) to the host address ``ptr``."""
    if _L().synth_normal(seed, tensor, offset, n, mean, std, dtype, ptr) != 0:
        raise ValueError("synth_normal: bad arguments")


def normal(shape, seed: int, tensor: int, dtype: int, mean: float = 0.0, std: float = 1.0,
           offset: int = 0) -> np.ndarray:
    """numpy array of N(mean, std^2) draws in storage type ``dtype`` (bf16 as uint16 bits)."""
    out = np.empty(shape, dtype=_NP_STORAGE[dtype])
    fill_normal_ptr(out.ctypes.data, out.size, seed, tensor, dtype, mean, std, offset)
    return out


def uniform(n: int, seed: int, tensor: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _L().synth_uniform(seed, tensor, offset, n, out.ctypes.data)
    return out


def uniform_int(n: int, lo: int, hi: int, seed: int, tensor: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    if _L().synth_uniform_int(seed, tensor, n, lo, hi, out.ctypes.data) != 0:
        raise ValueError("synth_uniform_int: bad arguments")
    return out


def raw(n: int, seed: int, tensor: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _L().synth_raw(seed, tensor, offset, n, out.ctypes.data)
    return out


def round_to(values: np.ndarray, dtype: int) -> np.ndarray:
    """Round float64 values to storage ``dtype`` (RNE) - the generator's rounding."""
    v = np.ascontiguousarray(values, dtype=np.float64)
    out = np.empty(v.shape, dtype=_NP_STORAGE[dtype])
    _L().synth_round(v.ctypes.data, v.size, dtype, out.ctypes.data)
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (upper half of an fp32)."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_f64(a: np.ndarray, dtype: int) -> np.ndarray:
    """Exact float64 value of a storage array produced by this module."""
    if dtype == BF16:
        return bf16_bits_to_f64(a)
    return a.astype(np.float64)


# ----------------------------------------------------------------------------- recipes


@dataclass
class LayerShape:
    hidden: int
    n_heads: int
    ffn: int

    @property
    def head_dim(self) -> int:
        return self.hidden // self.n_heads

    def weight_shapes(self):
        H, F = self.hidden, self.ffn
        return {"ln1_g": (H,), "ln1_b": (H,), "w_qkv": (3 * H, H), "b_qkv": (3 * H,),
                "w_o": (H, H), "b_o": (H,), "ln2_g": (H,), "ln2_b": (H,),
                "w_1": (F, H), "b_1": (F,), "w_2": (H, F), "b_2": (H,)}


@dataclass
class WeightRecipe:
    """Distribution of each weight tensor: (mean, std) per name."""
    w_std: float = 0.02
    bias_std: float = 0.0
    gamma_mean: float = 1.0
    gamma_std: float = 0.0
    beta_std: float = 0.0

    def moments(self, name: str):
        if name.startswith("w_"):
            return 0.0, self.w_std
        if name.startswith("b_"):
            return 0.0, self.bias_std
        if name.endswith("_g"):
            return self.gamma_mean, self.gamma_std
        return 0.0, self.beta_std  # ln*_b


def weight_tensor_id(layer: int, name: str) -> int:
    return TID_LAYER_BASE + 32 * layer + WEIGHT_NAMES.index(name)


def layer_weights(shape: LayerShape, layer: int, seed: int, dtype: int,
                  recipe: WeightRecipe | None = None) -> dict:
    """All twelve tensors of one layer as numpy storage arrays (nn.Linear layout W[out, in])."""
    recipe = recipe or WeightRecipe()
    out = {}
    for name, shp in shape.weight_shapes().items():
        mean, std = recipe.moments(name)
        out[name] = normal(shp, seed, weight_tensor_id(layer, name), dtype, mean, std)
    return out


@dataclass
class Workload:
    """One synthetic workload: shapes, dtype, length recipe, seed."""
    name: str
    dtype: int
    batch: int
    pad_len: int | None            # None: the batch maximum of the drawn lengths
    n_layers: int = 0              # 0: offsets + remove/rebuild only
    shape: LayerShape | None = None
    hidden: int | None = None      # for the remove/rebuild-only workload
    len_lo: int = 1
    len_hi: int = 1
    fixed_len: int | None = None
    seed: int = 20260000
    recipe: WeightRecipe = field(default_factory=WeightRecipe)
    ln_eps: float = 1e-5

    @property
    def H(self) -> int:
        return self.shape.hidden if self.shape else self.hidden

    def lengths(self) -> np.ndarray:
        if self.fixed_len is not None:
            return np.full(self.batch, self.fixed_len, dtype=np.int32)
        return uniform_int(self.batch, self.len_lo, self.len_hi, self.seed, TID_LENGTHS)

    def padded_len(self) -> int:
        return int(self.lengths().max()) if self.pad_len is None else self.pad_len

    def x_padded(self, tensor: int = TID_X) -> np.ndarray:
        """[batch, pad_len, hidden], every position N(0,1) (pad positions are garbage)."""
        return normal((self.batch, self.padded_len(), self.H), self.seed, tensor, self.dtype)

    def layer(self, layer: int) -> dict:
        return layer_weights(self.shape, layer, self.seed, self.dtype, self.recipe)


GPT3 = LayerShape(hidden=12288, n_heads=96, ffn=49152)

WORKLOADS = {
    # 1 pre-LN GPT decoder layer, fp32, hidden 256, 4 heads, FFN 1024; batch 4, pad 32, len U[1,32]
    "tiny": Workload("tiny", F32, batch=4, pad_len=32, n_layers=1,
                     shape=LayerShape(256, 4, 1024), len_lo=1, len_hi=32, seed=20260001),
    # offsets + remove/rebuild only: bf16 [64, 512, 4096], len U[1,512]
    "remove_rebuild": Workload("remove_rebuild", BF16, batch=64, pad_len=512, n_layers=0,
                               hidden=4096, len_lo=1, len_hi=512, seed=20260002),
    # one GPT-3 layer, fp16, batch 1, pad 64, length 32
    "gpt3_layer": Workload("gpt3_layer", F16, batch=1, pad_len=64, n_layers=1, shape=GPT3,
                           fixed_len=32, seed=20260003),
    # GPT-3 12-layer stack, fp16, batch 32, pad 256, every length 128 (half the padding)
    "gpt3_stack_half_pad": Workload("gpt3_stack_half_pad", F16, batch=32, pad_len=256, n_layers=12,
                                    shape=GPT3, fixed_len=128, seed=20260004),
    # dynamic-batching-shaped: 12 layers, batch 64, len U[1,256], padded to the batch maximum
    "gpt3_stack_dynbatch": Workload("gpt3_stack_dynbatch", F16, batch=64, pad_len=None, n_layers=12,
                                    shape=GPT3, len_lo=1, len_hi=256, seed=20260005),
}
