"""The C-ABI library without a GPU: it builds, loads, exports every declared
symbol, and refuses bad arguments on the host before any launch."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

from padding_free_varlen_b200 import build as pbuild
from padding_free_varlen_b200 import capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    pbuild.build()
    return capi.load()


def declared_symbols():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        names += re.findall(r"ENERGON_API\s+[\w\s\*]+?\b(energon_\w+)\s*\(", open(h).read())
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 9
    out = subprocess.run(["nm", "-D", "--defined-only", capi.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (energon_\w+)", out))
    assert set(names) <= exported, set(names) - exported
    assert set(capi.EXPORTED) == set(names)
    for n in names:
        assert hasattr(lib, n)


def test_library_is_built_for_sm100a(lib):
    """Every object is compiled for sm_100a and nothing else (the build's own flags); on a
    GPU, tests/test_gpu_rce.py asks the runtime for the kernels' binary version."""
    assert pbuild.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert all(a in pbuild.NVCC_FLAGS for a in pbuild.ARCH)


def cfg(H=256, nh=2, F=1024, dtype=capi.ENERGON_F16):
    return capi.make_config(H, nh, F, dtype)


def test_workspace_bytes_matches_documented_layout(lib):
    def align(v, a):
        return (v + a - 1) // a * a
    for (H, nh, F, dt, e, B, S) in [(256, 2, 1024, capi.ENERGON_F16, 2, 3, 70),
                                   (12288, 96, 49152, capi.ENERGON_F16, 2, 32, 256),
                                   (12288, 96, 49152, capi.ENERGON_F16, 2, 1, 64),
                                   (256, 4, 1024, capi.ENERGON_F32, 4, 4, 32)]:
        R = align(B * S, 256)
        off = 0
        for cols, eb in ((H, e), (3 * H, e), (2 * H if e == 2 else 0, e), (H, e), (H, 4), (F, e)):
            off = align(off + R * cols * eb, 1024)      # a, qkv, qk_lo (16-bit only), o, x1 (fp32), f
        off = align(off + (4 * 128 * max(3 * H, F) * 4 if B * S <= 128 else 0), 1024)   # split-K partials
        off = align(off + R * 8, 1024)                                                    # LayerNorm statistics
        off = align(off + 6 * H * 4, 1024)                                                # folded c, d
        off = align(off + R * H * e, 1024)                                                # stack: x
        off = align(off + (B + 1) * 4, 1024)
        off = align(off + (B + 1) * 4, 1024)
        assert capi.energon_workspace_bytes(cfg(H, nh, F, dt), B, S) == off


def test_workspace_bytes_invalid_config(lib):
    assert capi.energon_workspace_bytes(cfg(H=250), 2, 8) == 0          # head_dim 125
    assert capi.energon_workspace_bytes(cfg(dtype=7), 2, 8) == 0
    assert capi.energon_workspace_bytes(cfg(), 0, 8) == 0


def test_bad_arguments_fail_before_launch(lib):
    # Each call below is refused by the host-side checks, so no kernel is launched.
    with pytest.raises(capi.EnergonError) as e:
        capi.energon_rce_offsets(None, 4, 8, None, None, stream=0)
    assert e.value.code == capi.ENERGON_ERR_INVALID_ARGUMENT
    with pytest.raises(capi.EnergonError) as e:
        capi.energon_rce_remove_padding(None, None, 1, 1, 1, 2, None, stream=0)
    assert e.value.code == capi.ENERGON_ERR_INVALID_ARGUMENT
    with pytest.raises(capi.EnergonError) as e:
        capi.energon_rce_rebuild_padding(None, None, 1, 1, 1, 2, None, stream=0)
    assert e.value.code == capi.ENERGON_ERR_INVALID_ARGUMENT
    w = capi.energon_layer_weights(*([0] * 12))
    with pytest.raises(capi.EnergonError) as e:
        capi.energon_layer_forward(cfg(), w, 0, 0, 2, 8, 0, 0, 0, 0, stream=0)
    assert e.value.code == capi.ENERGON_ERR_INVALID_ARGUMENT
    assert "weight" in capi.energon_last_error()
    with pytest.raises(capi.EnergonError) as e:
        capi.energon_stack_forward(cfg(H=384, nh=4), [w], 1, 0, 0, 2, 8, 1, 0, 0, 0, 0, stream=0)
    assert e.value.code == capi.ENERGON_ERR_UNSUPPORTED                     # head_dim 96
    with pytest.raises(capi.EnergonError) as e:
        capi.energon_stack_forward(cfg(), [w], 1, 0, 0, 0, 8, 1, 0, 0, 0, 0, stream=0)
    assert e.value.code == capi.ENERGON_ERR_INVALID_ARGUMENT                # batch 0
    fake = capi.energon_layer_weights(*([4096] * 12))
    with pytest.raises(capi.EnergonError) as e:   # workspace of 0 bytes is always too small
        capi.energon_stack_forward(cfg(), [fake], 1, 4096, 8192, 2, 8, 1, 12288, 16384, 20480, 0, stream=0)
    assert e.value.code == capi.ENERGON_ERR_WORKSPACE_TOO_SMALL
    with pytest.raises(capi.EnergonError) as e:
        capi.energon_stack_forward(cfg(), [fake], 1, 4096, 8192, 2, 8, 1, 4096, 16384, 20480, 1 << 40, stream=0)
    assert e.value.code == capi.ENERGON_ERR_INVALID_ARGUMENT                # out aliases in
    for mode in (-1, 3):
        with pytest.raises(capi.EnergonError) as e:
            capi.energon_stack_forward(cfg(), [fake], 1, 4096, 8192, 2, 8, mode, 12288, 16384, 20480, 1 << 40,
                                       stream=0)
        assert e.value.code == capi.ENERGON_ERR_INVALID_ARGUMENT and "remove_padding" in capi.energon_last_error()
    with pytest.raises(capi.EnergonError):
        capi.energon_selftest_bounded_wait(None, 10, stream=0)
    for fn in (capi.energon_rce_transpose_padding_rebuild, capi.energon_rce_transpose_padding_remove):
        for args in ((None, 4096, 2, 8, 3, 2, 64, 2, 8192), (4096, 4096, 2, 8, 0, 2, 64, 2, 8192),
                     (4096, 4096, 2, 8, 3, 2, 64, 3, 8192), (4096, 4096, 2, -1, 3, 2, 64, 2, 8192),
                     (4096, 4096, 2, 8, 3, 1 << 16, 1 << 14, 8, 8192)):
            with pytest.raises(capi.EnergonError) as e:
                fn(*args, stream=0)
            assert e.value.code == capi.ENERGON_ERR_INVALID_ARGUMENT


def test_binding_rejects_host_tensors(lib):
    import torch
    with pytest.raises(ValueError):
        capi.energon_rce_offsets(torch.zeros(4, dtype=torch.int32), 4, 8, torch.zeros(5, dtype=torch.int32),
                                 torch.zeros(1, dtype=torch.int32), stream=0)


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(capi, "_lib", None)
    monkeypatch.setattr(capi, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="missing"):
        capi.load()


def test_header_is_c_and_struct_layouts_match_the_binding(tmp_path):
    """The header compiles as C11, and every struct has the size and field offsets the
    ctypes binding assumes (gcc prints them; no GPU needed)."""
    import ctypes
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    structs = {
        "energon_layer_weights": (capi.energon_layer_weights, list(capi.WEIGHT_FIELDS) + ["ln1_fold"]),
        "energon_layer_config": (capi.energon_layer_config, ["hidden", "n_heads", "ffn", "dtype", "ln_eps",
                                                             "gelu_tanh"]),
        "energon_trace_entry": (capi.energon_trace_entry, ["name", "launches", "total_ms"]),
        "energon_request": (capi.energon_request, ["length", "arrival_s"]),
    }
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "energon_rce.h"', "int main(void) {"]
    for name, (_, fields) in structs.items():
        lines.append(f'    printf("{name} size %zu\\n", sizeof({name}));')
        for f in fields:
            lines.append(f'    printf("{name} {f} %zu\\n", offsetof({name}, {f}));')
    lines += ["    return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    include = os.path.join(ROOT, "include")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", include, str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {tuple(l.split()[:2]): int(l.split()[2]) for l in out if l.strip()}
    for name, (cls, fields) in structs.items():
        assert got[(name, "size")] == ctypes.sizeof(cls), name
        for f in fields:
            assert got[(name, f)] == getattr(cls, f).offset, (name, f)


def test_every_export_has_a_binding_of_the_same_name():
    missing = [n for n in capi.EXPORTED if not callable(getattr(capi, n, None))]
    assert not missing, missing
