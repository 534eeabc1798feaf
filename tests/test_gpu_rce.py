"""Offsets, transpose_padding_remove and transpose_padding_rebuild on the GPU,
bit-exact against the oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

from padding_free_varlen_b200 import capi, synth
from helpers import to_device, to_storage

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from padding_free_varlen_b200 import build
    build.build()
    capi.load()


def gpu_offsets(lengths: np.ndarray, pad_len: int):
    B = lengths.size
    d_len = torch.from_numpy(lengths.astype(np.int32)).cuda()
    cu = torch.full((B + 1,), -7, dtype=torch.int32, device="cuda")
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    capi.energon_rce_offsets(d_len if B else None, B, pad_len, cu, st)
    torch.cuda.synchronize()
    return cu.cpu().numpy(), int(st.item()), cu


@pytest.mark.parametrize("B", [0, 1, 2, 31, 32, 33, 64, 1000, 1024, 1025, 3000])
def test_offsets_match_oracle(oracle_lib, synth_mod, B):
    lengths = synth_mod.uniform_int(B, 0, 300, 77, B) if B else np.zeros(0, np.int32)
    cu, st, _ = gpu_offsets(lengths, 300)
    ref, rst = oracle_lib.offsets(lengths, 300)
    assert st == rst == 0
    assert np.array_equal(cu, ref)


@pytest.mark.parametrize("bad", [[5, 301, 2], [-1], [0] * 40 + [1000]])
def test_offsets_invalid_lengths(oracle_lib, bad):
    lengths = np.array(bad, np.int32)
    cu, st, _ = gpu_offsets(lengths, 300)
    ref, rst = oracle_lib.offsets(lengths, 300)
    assert st == rst == capi.ENERGON_DEVICE_BAD_LENGTH
    assert np.array_equal(cu, ref) and not cu.any()


CASES = [  # (np storage dtype, elem bytes, hidden, batch, pad_len, byte offset of the buffers)
    (np.uint16, 2, 4096, 5, 33, 0),     # 16-byte vector path
    (np.float32, 4, 7, 9, 13, 0),       # 4-byte path (28-byte rows)
    (np.int8, 1, 5, 6, 11, 0),          # byte path
    (np.float64, 8, 3, 4, 10, 0),
    (np.uint16, 2, 64, 7, 20, 2),       # misaligned base pointers -> narrower path
    (np.float16, 2, 8, 3, 1, 0),        # pad_len 1
]


@pytest.mark.parametrize("dt,e,H,B,S,shift", CASES)
def test_remove_rebuild_bit_exact(oracle_lib, synth_mod, dt, e, H, B, S, shift):
    lengths = synth_mod.uniform_int(B, 0, S, 5, H + B)
    lengths[0] = S                                   # a full row and ...
    if B > 2:
        lengths[1] = 0                               # ... an empty one
    rng = np.random.default_rng(H * 31 + B)
    padded = rng.integers(0, 256, size=(B, S, H * e), dtype=np.uint8)
    cu, st, d_cu = gpu_offsets(lengths, S)
    assert st == 0
    T = int(cu[-1])
    nbytes = B * S * H * e
    # buffers carved at a byte offset from a raw allocation to exercise alignment handling
    raw_in = torch.zeros(nbytes + 16, dtype=torch.uint8, device="cuda")
    raw_in[shift:shift + nbytes] = torch.from_numpy(padded.ravel()).cuda()
    raw_pk = torch.full((nbytes + 16,), 0xAB, dtype=torch.uint8, device="cuda")
    capi.energon_rce_remove_padding(raw_in.data_ptr() + shift, d_cu, B, S, H, e, raw_pk.data_ptr() + shift)
    raw_out = torch.full((nbytes + 16,), 0xCD, dtype=torch.uint8, device="cuda")
    capi.energon_rce_rebuild_padding(raw_pk.data_ptr() + shift, d_cu, B, S, H, e, raw_out.data_ptr() + shift)
    torch.cuda.synchronize()
    pk = raw_pk.cpu().numpy()
    out = raw_out.cpu().numpy()
    sentinel_pk = np.full(B * S * H * e, 0xAB, np.uint8).reshape(B * S, H * e)
    ref_pk = oracle_lib.remove_padding(padded, cu, out=sentinel_pk)
    assert np.array_equal(pk[shift:shift + nbytes].reshape(B * S, H * e), ref_pk)   # rows >= T untouched
    ref_out = oracle_lib.rebuild_padding(ref_pk, cu, B, S)
    assert np.array_equal(out[shift:shift + nbytes].reshape(B, S, H * e), ref_out)
    assert (pk[:shift] == 0xAB).all() and (pk[shift + nbytes:] == 0xAB).all()          # no stray writes
    assert (out[:shift] == 0xCD).all() and (out[shift + nbytes:] == 0xCD).all()
    for b in range(B):                                                                 # round trip
        assert np.array_equal(out[shift:shift + nbytes].reshape(B, S, H * e)[b, :lengths[b]],
                              padded[b, :lengths[b]])
    assert T == lengths.sum()


def test_all_empty_lengths():
    B, S, H = 4, 6, 16
    cu, st, d_cu = gpu_offsets(np.zeros(B, np.int32), S)
    assert st == 0 and not cu.any()
    src = torch.randn(B, S, H, device="cuda", dtype=torch.float16)
    pk = torch.full((B * S, H), 3.0, device="cuda", dtype=torch.float16)
    capi.energon_rce_remove_padding(src, d_cu, B, S, H, 2, pk)
    out = torch.full((B, S, H), 5.0, device="cuda", dtype=torch.float16)
    capi.energon_rce_rebuild_padding(pk, d_cu, B, S, H, 2, out)
    torch.cuda.synchronize()
    assert (pk == 3.0).all()
    assert (out.view(torch.int16) == 0).all()


def test_remove_rebuild_workload_full_size(oracle_lib, synth_mod):
    """The bf16 [64, 512, 4096] workload with lengths U[1, 512]: bit-exact remove,
    rebuild, round trip, zero pads; and all-full lengths make remove the identity."""
    wl = synth_mod.WORKLOADS["remove_rebuild"]
    lengths = wl.lengths()
    x = wl.x_padded()
    B, S, H = x.shape
    cu, st, d_cu = gpu_offsets(lengths, S)
    assert st == 0
    d_x = to_device(x, wl.dtype)
    pk = torch.empty((B * S, H), dtype=torch.bfloat16, device="cuda")
    pk.view(torch.int16).fill_(0x7F7F)
    capi.energon_rce_remove_padding(d_x, d_cu, B, S, H, 2, pk)
    out = torch.empty_like(d_x)
    out.view(torch.int16).fill_(-1)
    capi.energon_rce_rebuild_padding(pk, d_cu, B, S, H, 2, out)
    torch.cuda.synchronize()
    ref_pk = oracle_lib.remove_padding(x, cu, out=np.full((B * S, H), 0x7F7F, np.uint16))
    assert np.array_equal(to_storage(pk), ref_pk)
    ref_out = oracle_lib.rebuild_padding(ref_pk, cu, B, S)
    assert np.array_equal(to_storage(out), ref_out)
    full = np.full(B, S, np.int32)
    _, st, d_cu_full = gpu_offsets(full, S)
    capi.energon_rce_remove_padding(d_x, d_cu_full, B, S, H, 2, pk)
    torch.cuda.synchronize()
    assert torch.equal(pk.view(torch.int16), d_x.view(B * S, H).view(torch.int16))


def test_kernels_are_sm100a_binaries():
    """The runtime reports binary version 100 (sm_100a) for the library's kernels."""
    assert capi.energon_kernel_binary_version() == 100
