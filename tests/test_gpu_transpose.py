"""Head-transposing transpose_padding_rebuild / transpose_padding_remove on the GPU,
bit-exact against the oracle through the C ABI: every vector path (16, 4 and 1 bytes),
misaligned buffers, ragged lengths with full and empty sequences, pad length 1, an
empty batch, and the GPT-3 QKV / attention-output shapes at full size."""
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
    cu = torch.empty(B + 1, dtype=torch.int32, device="cuda")
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    capi.energon_rce_offsets(d_len, B, pad_len, cu, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return cu.cpu().numpy(), cu


CASES = [  # (elem bytes, parts, n_heads, head_dim, batch, pad_len, byte offset of the buffers)
    (2, 3, 4, 64, 5, 33, 0),      # 16-byte vectors, Q|K|V blocks
    (2, 1, 3, 6, 7, 9, 0),        # 12-byte heads: 4-byte path
    (1, 3, 2, 5, 6, 11, 0),       # byte path
    (4, 3, 2, 8, 4, 10, 4),       # 32-byte heads on 4-byte aligned buffers: 4-byte path
    (8, 1, 2, 2, 3, 5, 0),        # 16-byte heads of 8-byte elements
    (2, 3, 2, 8, 3, 1, 0),        # pad_len 1
    (2, 1, 96, 128, 2, 40, 0),    # GPT-3 head split (96 heads of 128)
]


@pytest.mark.parametrize("e,parts,nh,d,B,S,shift", CASES)
def test_transpose_forms_bit_exact(oracle_lib, synth_mod, e, parts, nh, d, B, S, shift):
    lengths = synth_mod.uniform_int(B, 0, S, 9, nh * d + B)
    lengths[0] = S
    if B > 2:
        lengths[1] = 0
    cu, d_cu = gpu_offsets(lengths, S)
    T, row = int(cu[-1]), parts * nh * d * e
    n_heads_bytes = parts * B * nh * S * d * e
    rng = np.random.default_rng(parts * 1000 + nh * d + B)
    packed = rng.integers(0, 256, size=(B * S, row), dtype=np.uint8)
    packed[T:] = 0x5A
    # rebuild: packed -> head-major, every element written, nothing outside it
    raw_pk = torch.zeros(B * S * row + 16, dtype=torch.uint8, device="cuda")
    raw_pk[shift:shift + B * S * row] = torch.from_numpy(packed.ravel()).cuda()
    raw_hd = torch.full((n_heads_bytes + 16,), 0xCD, dtype=torch.uint8, device="cuda")
    capi.energon_rce_transpose_padding_rebuild(raw_pk.data_ptr() + shift, d_cu, B, S, parts, nh, d, e,
                                               raw_hd.data_ptr() + shift)
    # remove: head-major with garbage in its pad positions -> packed rows 0..T-1 only
    heads_in = rng.integers(0, 256, size=n_heads_bytes, dtype=np.uint8)
    raw_hin = torch.zeros(n_heads_bytes + 16, dtype=torch.uint8, device="cuda")
    raw_hin[shift:shift + n_heads_bytes] = torch.from_numpy(heads_in).cuda()
    raw_out = torch.full((B * S * row + 16,), 0xAB, dtype=torch.uint8, device="cuda")
    capi.energon_rce_transpose_padding_remove(raw_hin.data_ptr() + shift, d_cu, B, S, parts, nh, d, e,
                                              raw_out.data_ptr() + shift)
    torch.cuda.synchronize()
    hd = raw_hd.cpu().numpy()
    ref_hd = oracle_lib.transpose_padding_rebuild(packed, cu, B, S, parts, nh)
    assert np.array_equal(hd[shift:shift + n_heads_bytes], ref_hd.ravel())
    assert (hd[:shift] == 0xCD).all() and (hd[shift + n_heads_bytes:] == 0xCD).all()
    out = raw_out.cpu().numpy()
    sentinel = np.full((B * S, row), 0xAB, np.uint8)
    ref_out = oracle_lib.transpose_padding_remove(heads_in.reshape(parts, B, nh, S, d * e), cu, out=sentinel)
    assert np.array_equal(out[shift:shift + B * S * row].reshape(B * S, row), ref_out)
    assert (out[:shift] == 0xAB).all() and (out[shift + B * S * row:] == 0xAB).all()


def test_transpose_forms_round_trip_and_empty():
    B, S, nh, d = 4, 16, 2, 64
    lengths = np.array([16, 3, 0, 9], np.int32)
    cu, d_cu = gpu_offsets(lengths, S)
    T = int(cu[-1])
    pk = torch.randn(T, 3 * nh * d, device="cuda", dtype=torch.float16)
    heads = torch.full((3, B, nh, S, d), 7.0, device="cuda", dtype=torch.float16)
    capi.energon_rce_transpose_padding_rebuild(pk, d_cu, B, S, 3, nh, d, 2, heads)
    back = torch.full((B * S, 3 * nh * d), 9.0, device="cuda", dtype=torch.float16)
    capi.energon_rce_transpose_padding_remove(heads, d_cu, B, S, 3, nh, d, 2, back)
    torch.cuda.synchronize()
    assert torch.equal(back[:T].view(torch.int16), pk.view(torch.int16)) and (back[T:] == 9.0).all()
    for b in range(B):
        assert not heads[:, b, :, lengths[b]:].view(torch.int16).any()
    _, d_cu0 = gpu_offsets(np.zeros(B, np.int32), S)                   # every sequence empty
    capi.energon_rce_transpose_padding_rebuild(pk, d_cu0, B, S, 3, nh, d, 2, heads)
    back.fill_(9.0)
    capi.energon_rce_transpose_padding_remove(heads, d_cu0, B, S, 3, nh, d, 2, back)
    capi.energon_rce_transpose_padding_rebuild(pk, d_cu0, 0, S, 3, nh, d, 2, heads)   # batch 0: no-op
    torch.cuda.synchronize()
    assert not heads.view(torch.int16).any() and (back == 9.0).all()


@pytest.mark.slow
def test_transpose_forms_gpt3_dynbatch_full_size(oracle_lib):
    """GPT-3 hidden 12288 (96 heads of 128), fp16, the ragged batch of 64 (lengths U[1, 256],
    pad = batch maximum): Q|K|V rows [T, 3H] -> [3, B, 96, S, 128] and an attention output
    [1, B, 96, S, 128] -> [T, H], bit-exact against the oracle on the whole tensors."""
    wl = synth.WORKLOADS["gpt3_stack_dynbatch"]
    lengths, S = wl.lengths(), wl.padded_len()
    B, H, nh = wl.batch, wl.shape.hidden, wl.shape.n_heads
    d = H // nh
    cu, d_cu = gpu_offsets(lengths, S)
    T = int(cu[-1])
    qkv = synth.normal((T, 3 * H), wl.seed, 91, synth.F16)
    d_qkv = to_device(qkv, synth.F16)
    heads = torch.empty((3, B, nh, S, d), dtype=torch.float16, device="cuda")
    heads.view(torch.int16).fill_(-1)
    capi.energon_rce_transpose_padding_rebuild(d_qkv, d_cu, B, S, 3, nh, d, 2, heads)
    torch.cuda.synchronize()
    ref = oracle_lib.transpose_padding_rebuild(qkv, cu, B, S, 3, nh)
    assert np.array_equal(to_storage(heads).view(np.uint16), ref.view(np.uint16))
    del heads, d_qkv
    attn = synth.normal((1, B, nh, S, d), wl.seed, 92, synth.F16)
    d_attn = to_device(attn, synth.F16)
    out = torch.empty((B * S, H), dtype=torch.float16, device="cuda")
    out.view(torch.int16).fill_(0x3C00)
    capi.energon_rce_transpose_padding_remove(d_attn, d_cu, B, S, 1, nh, d, 2, out)
    torch.cuda.synchronize()
    ref = oracle_lib.transpose_padding_remove(attn, cu, out=np.full((B * S, H), 1.0, np.float16))
    assert np.array_equal(to_storage(out).view(np.uint16), ref.view(np.uint16))
