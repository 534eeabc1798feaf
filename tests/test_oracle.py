"""Pins for the fp64 oracle (CPU only).

Each check ties the oracle to something other than itself: brute-force loops
over tiny inputs, closed forms, invariants the definitions imply, and
independent fp64 library compositions (numpy / torch CPU).  None of these
re-runs the oracle's own routine.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


# ----------------------------------------------------------------------------- helpers


def brute_offsets(lengths):
    return [sum(lengths[:b]) for b in range(len(lengths) + 1)]


def brute_remove(padded, lengths):
    rows = [padded[b, s] for b in range(padded.shape[0]) for s in range(lengths[b])]
    return np.stack(rows) if rows else np.zeros((0,) + padded.shape[2:], padded.dtype)


def brute_rebuild(packed, lengths, pad_len):
    B = len(lengths)
    out = np.zeros((B, pad_len) + packed.shape[1:], packed.dtype)
    r = 0
    for b in range(B):
        for s in range(lengths[b]):
            out[b, s] = packed[r]
            r += 1
    return out


def torch_layer(x, w, n_heads, eps=1e-5, gelu_tanh=True):
    """Independent fp64 composition of a pre-LN GPT layer from torch CPU library ops."""
    t = {k: torch.from_numpy(np.asarray(v, dtype=np.float64)) for k, v in w.items()}
    x = torch.from_numpy(np.asarray(x, dtype=np.float64))
    L, H = x.shape
    d = H // n_heads
    a = F.layer_norm(x, (H,), t["ln1_g"], t["ln1_b"], eps)
    qkv = F.linear(a, t["w_qkv"], t["b_qkv"])
    q, k, v = qkv.split(H, dim=-1)
    heads = lambda z: z.view(L, n_heads, d).transpose(0, 1)
    o = F.scaled_dot_product_attention(heads(q), heads(k), heads(v), is_causal=True)
    o = o.transpose(0, 1).reshape(L, H)
    x1 = x + F.linear(o, t["w_o"], t["b_o"])
    a2 = F.layer_norm(x1, (H,), t["ln2_g"], t["ln2_b"], eps)
    f = F.gelu(F.linear(a2, t["w_1"], t["b_1"]), approximate="tanh" if gelu_tanh else "none")
    return (x1 + F.linear(f, t["w_2"], t["b_2"])).numpy()


def small_weights(synth, H, nh, ffn, dtype, layer=0, seed=7, nonzero=True):
    shape = synth.LayerShape(H, nh, ffn)
    recipe = synth.WeightRecipe(w_std=0.05, bias_std=0.1 if nonzero else 0.0,
                                gamma_std=0.2 if nonzero else 0.0, beta_std=0.1 if nonzero else 0.0)
    return synth.layer_weights(shape, layer, seed, dtype, recipe)


# ----------------------------------------------------------------------------- offsets


def test_offsets_hand_case(oracle_lib):
    cu, st = oracle_lib.offsets(np.array([3, 0, 2, 5]), pad_len=5)
    assert st == 0 and cu.tolist() == [0, 3, 3, 5, 10]


@pytest.mark.parametrize("B", list(range(0, 71)))
def test_offsets_brute_force(oracle_lib, synth_mod, B):
    lengths = synth_mod.uniform_int(B, 0, 40, 11, 100 + B) if B else np.zeros(0, np.int32)
    cu, st = oracle_lib.offsets(lengths, pad_len=40)
    assert st == 0
    assert cu.tolist() == brute_offsets(lengths.tolist())


@pytest.mark.parametrize("bad", [[3, 6, 1], [-1, 2], [0, 0, 9]])
def test_offsets_invalid_lengths(oracle_lib, bad):
    cu, st = oracle_lib.offsets(np.array(bad), pad_len=5)
    assert st == 1 and not cu.any()


def test_offsets_edge_lengths(oracle_lib):
    cu, st = oracle_lib.offsets(np.array([0, 5, 0, 5]), pad_len=5)
    assert st == 0 and cu.tolist() == [0, 0, 5, 5, 10]
    cu, st = oracle_lib.offsets(np.zeros(6, np.int32), pad_len=1)
    assert st == 0 and not cu.any()


# ----------------------------------------------------------------------------- remove / rebuild


def test_remove_rebuild_hand_case(oracle_lib):
    padded = np.array([[[b * 100 + s * 10 + k for k in range(2)] for s in range(3)] for b in range(2)],
                      dtype=np.int16)
    cu, _ = oracle_lib.offsets(np.array([2, 1]), 3)
    packed = oracle_lib.remove_padding(padded, cu)
    assert packed[:3].tolist() == [[0, 1], [10, 11], [100, 101]]
    out = oracle_lib.rebuild_padding(packed, cu, 2, 3)
    assert out.tolist() == [[[0, 1], [10, 11], [0, 0]], [[100, 101], [0, 0], [0, 0]]]


@pytest.mark.parametrize("dtype,H", [(np.float32, 7), (np.float16, 16), (np.uint16, 33), (np.int8, 5)])
def test_remove_rebuild_brute_force(oracle_lib, synth_mod, dtype, H):
    B, S = 9, 13
    lengths = synth_mod.uniform_int(B, 0, S, 3, 4)
    rng = np.random.default_rng(0)
    padded = rng.integers(0, 255, size=(B, S, H * np.dtype(dtype).itemsize), dtype=np.uint8).view(dtype)
    cu, st = oracle_lib.offsets(lengths, S)
    assert st == 0
    sentinel = np.full((B * S, H * np.dtype(dtype).itemsize), 0xFF, np.uint8).view(dtype)
    packed = oracle_lib.remove_padding(padded, cu, out=sentinel.copy())
    T = int(cu[-1])
    assert packed[:T].tobytes() == brute_remove(padded, lengths).tobytes()
    assert (packed[T:].view(np.uint8) == 0xFF).all()          # no stray writes past T
    out = oracle_lib.rebuild_padding(packed, cu, B, S,
                                     out=np.full_like(padded.view(np.uint8), 0xFF).view(dtype))
    assert out.tobytes() == brute_rebuild(packed[:T], lengths, S).tobytes()
    for b in range(B):                                         # round trip + zero pads
        assert out[b, :lengths[b]].tobytes() == padded[b, :lengths[b]].tobytes()
        assert not out[b, lengths[b]:].view(np.uint8).any()


def test_remove_full_lengths_is_identity(oracle_lib, synth_mod):
    B, S, H = 4, 6, 8
    padded = synth_mod.normal((B, S, H), 1, 2, synth_mod.F16)
    cu, _ = oracle_lib.offsets(np.full(B, S), S)
    packed = oracle_lib.remove_padding(padded, cu)
    assert packed.tobytes() == padded.reshape(B * S, H).tobytes()


def test_rebuild_writes_positive_zero(oracle_lib):
    packed = np.array([[-0.0, 1.5]], dtype=np.float32)
    cu, _ = oracle_lib.offsets(np.array([1]), 3)
    out = oracle_lib.rebuild_padding(packed, cu, 1, 3)
    assert out[0, 1:].view(np.uint32).tolist() == [[0, 0], [0, 0]]
    assert out[0, 0].view(np.uint32)[0] == 0x80000000       # valid rows keep their bytes


# ----------------------------------------------------------------------------- head-transposing forms


def test_transpose_rebuild_remove_hand_case(oracle_lib):
    # 2 sequences (lengths 2, 1), pad 2, blocks Q|K (parts 2), 2 heads of 1 element;
    # packed row t holds t*10 + column.  Expected head-major tensor written out by hand.
    packed = np.array([[t * 10 + j for j in range(4)] for t in range(3)], dtype=np.int16)
    cu, _ = oracle_lib.offsets(np.array([2, 1]), 2)
    heads = oracle_lib.transpose_padding_rebuild(packed, cu, 2, 2, parts=2, n_heads=2,
                                                 out=np.full((2, 2, 2, 2, 1), -1, np.int16))
    expect = [[[[[0], [10]], [[1], [11]]], [[[20], [0]], [[21], [0]]]],
              [[[[2], [12]], [[3], [13]]], [[[22], [0]], [[23], [0]]]]]
    assert heads.tolist() == expect
    back = oracle_lib.transpose_padding_remove(heads, cu, out=np.full((4, 4), -1, np.int16))
    assert back[:3].tolist() == packed.tolist() and back[3].tolist() == [-1] * 4


def np_transpose_rebuild(packed, lengths, pad_len, parts, nh):
    """The same map through numpy reshapes and an axis permutation, sequence by sequence."""
    d = packed.shape[1] // (parts * nh)
    out = np.zeros((parts, len(lengths), nh, pad_len, d), packed.dtype)
    r = 0
    for b, n in enumerate(lengths):
        out[:, b, :, :n, :] = packed[r:r + n].reshape(n, parts, nh, d).transpose(1, 2, 0, 3)
        r += n
    return out


@pytest.mark.parametrize("parts,nh,d,dtype", [(3, 4, 8, np.float16), (1, 3, 5, np.float32), (3, 2, 3, np.int8),
                                              (1, 1, 6, np.uint16)])
def test_transpose_forms_brute_force(oracle_lib, synth_mod, parts, nh, d, dtype):
    B, S = 7, 11
    lengths = synth_mod.uniform_int(B, 0, S, 5, 4)
    cu, st = oracle_lib.offsets(lengths, S)
    assert st == 0
    T, width = int(cu[-1]), parts * nh * d
    rng = np.random.default_rng(1)
    isz = np.dtype(dtype).itemsize
    packed = rng.integers(0, 255, size=(T, width * isz), dtype=np.uint8).view(dtype)
    heads = oracle_lib.transpose_padding_rebuild(
        packed, cu, B, S, parts, nh, out=np.full((parts, B, nh, S, d * isz), 0xFF, np.uint8).view(dtype))
    assert heads.tobytes() == np_transpose_rebuild(packed, lengths, S, parts, nh).tobytes()
    sentinel = np.full((B * S, width * isz), 0xFF, np.uint8).view(dtype)
    back = oracle_lib.transpose_padding_remove(heads, cu, out=sentinel)
    assert back[:T].tobytes() == packed.tobytes()                  # round trip
    assert (back[T:].view(np.uint8) == 0xFF).all()                 # nothing written past T
    # remove on a head-major tensor whose pad positions hold garbage ignores them
    noisy = rng.integers(0, 255, size=heads.view(np.uint8).shape, dtype=np.uint8).view(dtype)
    got = oracle_lib.transpose_padding_remove(noisy, cu)
    ref = [noisy[:, b, :, :n, :].transpose(2, 0, 1, 3).reshape(n, width) for b, n in enumerate(lengths)]
    assert got[:T].tobytes() == np.concatenate(ref).tobytes()


def test_transpose_forms_one_block_one_head_are_the_plain_forms(oracle_lib, synth_mod):
    B, S, H = 5, 9, 12
    lengths = synth_mod.uniform_int(B, 0, S, 6, 4)
    cu, _ = oracle_lib.offsets(lengths, S)
    T = int(cu[-1])
    packed = synth_mod.normal((T, H), 2, 3, synth_mod.F16)
    heads = oracle_lib.transpose_padding_rebuild(packed, cu, B, S, 1, 1)
    assert heads.tobytes() == oracle_lib.rebuild_padding(packed, cu, B, S).tobytes()
    padded = synth_mod.normal((B, S, H), 2, 4, synth_mod.F16)
    a = oracle_lib.transpose_padding_remove(padded.reshape(1, B, 1, S, H), cu)
    assert a[:T].tobytes() == oracle_lib.remove_padding(padded, cu)[:T].tobytes()


# ----------------------------------------------------------------------------- decoding


def test_decode_matches_library_conversions(oracle_lib, synth_mod):
    bits = np.arange(0, 1 << 16, dtype=np.uint16)
    h = bits.view(np.float16)
    finite = np.isfinite(h)
    assert np.array_equal(oracle_lib.decode(h)[finite], h[finite].astype(np.float64))
    bf = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    dec = oracle_lib.decode(bits)
    fin = np.isfinite(bf)
    assert np.array_equal(dec[fin], bf[fin])


# ----------------------------------------------------------------------------- LayerNorm


def test_layernorm_hand_case(oracle_lib):
    y = oracle_lib.layernorm(np.array([[1.0, 2.0, 3.0, 4.0]]), np.ones(4), np.zeros(4), eps=0.0)
    # mean 2.5, biased variance 1.25
    expect = (np.array([1, 2, 3, 4]) - 2.5) / math.sqrt(1.25)
    assert np.allclose(y[0], expect, rtol=0, atol=1e-15)


def test_layernorm_invariants_and_torch(oracle_lib, synth_mod):
    x = synth_mod.normal((17, 256), 5, 6, synth_mod.F64, mean=3.0, std=2.0)
    y = oracle_lib.layernorm(x, np.ones(256), np.zeros(256), eps=1e-5)
    assert np.abs(y.mean(axis=1)).max() < 1e-13
    var = (y ** 2).mean(axis=1)
    assert np.allclose(var, 1.0 / (1.0 + 1e-5 / (x.var(axis=1))), rtol=1e-12)
    g = synth_mod.normal((256,), 5, 7, synth_mod.F16, 1.0, 0.3)
    b = synth_mod.normal((256,), 5, 8, synth_mod.F16, 0.0, 0.3)
    y2 = oracle_lib.layernorm(x, g, b, eps=1e-5)
    ref = F.layer_norm(torch.from_numpy(x), (256,), torch.from_numpy(g.astype(np.float64)),
                       torch.from_numpy(b.astype(np.float64)), 1e-5).numpy()
    assert np.abs(y2 - ref).max() < 1e-12


# ----------------------------------------------------------------------------- linear / GELU


@pytest.mark.parametrize("wd", ["F32", "F16", "BF16"])
def test_linear_against_numpy(oracle_lib, synth_mod, wd):
    code = getattr(synth_mod, wd)
    x = synth_mod.normal((13, 96), 1, 2, synth_mod.F64)
    W = synth_mod.normal((40, 96), 1, 3, code, 0.0, 0.1)
    b = synth_mod.normal((40,), 1, 4, code, 0.0, 0.5)
    y = oracle_lib.linear(x, W, b)
    Wd, bd = synth_mod.to_f64(W, code), synth_mod.to_f64(b, code)
    ref = x @ Wd.T + bd
    assert np.abs(y - ref).max() < 1e-13
    # a transposed operand would not even match shape-compatible products
    assert np.abs(oracle_lib.linear(x, W) - x @ Wd.T).max() < 1e-13


def test_gelu_closed_forms(oracle_lib):
    pts = np.array([-3.0, -1.0, -0.5, 0.0, 0.5, 1.0, 3.0])
    c = math.sqrt(2 / math.pi)
    tanh_ref = [0.5 * v * (1 + math.tanh(c * (v + 0.044715 * v ** 3))) for v in pts]
    erf_ref = [0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in pts]
    assert np.allclose(oracle_lib.gelu(pts, True), tanh_ref, rtol=0, atol=1e-15)
    assert np.allclose(oracle_lib.gelu(pts, False), erf_ref, rtol=0, atol=1e-15)
    xs = np.linspace(-8, 8, 20001)
    tg = F.gelu(torch.from_numpy(xs), approximate="tanh").numpy()
    eg = F.gelu(torch.from_numpy(xs)).numpy()
    assert np.abs(oracle_lib.gelu(xs, True) - tg).max() < 1e-14
    assert np.abs(oracle_lib.gelu(xs, False) - eg).max() < 1e-14
    # the two forms differ by at most ~4.7e-4 on the real line
    assert 4.0e-4 < np.abs(tg - eg).max() < 5.0e-4


# ----------------------------------------------------------------------------- attention


def test_attention_first_query_and_length_one(oracle_lib, synth_mod):
    L, H, nh = 9, 64, 4
    qkv = synth_mod.normal((L, 3 * H), 2, 3, synth_mod.F64)
    o = oracle_lib.causal_attention(qkv, nh)
    assert np.abs(o[0] - qkv[0, 2 * H:]).max() < 1e-15         # q0 only sees k0
    o1 = oracle_lib.causal_attention(qkv[:1], nh)
    assert np.abs(o1[0] - qkv[0, 2 * H:]).max() < 1e-15


def test_attention_zero_keys_gives_prefix_mean(oracle_lib, synth_mod):
    L, H, nh = 12, 32, 2
    qkv = synth_mod.normal((L, 3 * H), 2, 4, synth_mod.F64)
    qkv[:, H:2 * H] = 0.0
    o = oracle_lib.causal_attention(qkv, nh)
    v = qkv[:, 2 * H:]
    prefix_mean = np.cumsum(v, axis=0) / np.arange(1, L + 1)[:, None]
    assert np.abs(o - prefix_mean).max() < 1e-14


def test_attention_against_torch_sdpa(oracle_lib, synth_mod):
    L, H, nh = 21, 128, 2
    d = H // nh
    qkv = synth_mod.normal((L, 3 * H), 2, 5, synth_mod.F64, 0.0, 2.0)
    o = oracle_lib.causal_attention(qkv, nh)
    t = torch.from_numpy(qkv)
    q, k, v = (z.view(L, nh, d).transpose(0, 1) for z in t.split(H, dim=-1))
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(0, 1).reshape(L, H).numpy()
    assert np.abs(o - ref).max() < 1e-13
    # heads are independent: scrambling head 1's keys leaves head 0 alone
    qkv2 = qkv.copy()
    qkv2[:, H + d:2 * H] *= -3.0
    o2 = oracle_lib.causal_attention(qkv2, nh)
    assert np.array_equal(o2[:, :d], o[:, :d]) and not np.allclose(o2[:, d:], o[:, d:])


# ----------------------------------------------------------------------------- layer / stack


@pytest.mark.parametrize("wd,nonzero", [("F32", False), ("F32", True), ("F16", True), ("BF16", True)])
def test_layer_against_torch_composition(oracle_lib, synth_mod, wd, nonzero):
    code = getattr(synth_mod, wd)
    H, nh, ffn, L = 128, 2, 512, 11
    w = small_weights(synth_mod, H, nh, ffn, code, nonzero=nonzero)
    x = synth_mod.normal((L, H), 9, 2, synth_mod.F64)
    y = oracle_lib.layer_sequence(x, w, nh)
    ref = torch_layer(x, {k: synth_mod.to_f64(v, code) for k, v in w.items()}, nh)
    assert np.abs(y - ref).max() < 1e-11 * max(1.0, np.abs(ref).max())
    y_erf = oracle_lib.layer_sequence(x, w, nh, gelu_tanh=False)
    ref_erf = torch_layer(x, {k: synth_mod.to_f64(v, code) for k, v in w.items()}, nh, gelu_tanh=False)
    assert np.abs(y_erf - ref_erf).max() < 1e-11 * max(1.0, np.abs(ref).max())


def test_tiny_workload_layer_against_torch(oracle_lib, synth_mod):
    wl = synth_mod.WORKLOADS["tiny"]
    lengths = wl.lengths()
    x = wl.x_padded()
    w = wl.layer(0)
    y = oracle_lib.layer_padded(x.astype(np.float64), lengths, w, wl.shape.n_heads)
    wd = {k: synth_mod.to_f64(v, wl.dtype) for k, v in w.items()}
    for b in range(wl.batch):
        L = lengths[b]
        ref = torch_layer(x[b, :L].astype(np.float64), wd, wl.shape.n_heads)
        assert np.abs(y[b, :L] - ref).max() < 1e-11
        assert not y[b, L:].any()


def test_layer_padded_invariants(oracle_lib, synth_mod):
    H, nh, ffn, B, S = 64, 2, 128, 5, 8
    w = small_weights(synth_mod, H, nh, ffn, synth_mod.F32)
    lengths = np.array([3, 0, 8, 1, 5], np.int32)
    x = synth_mod.normal((B, S, H), 4, synth_mod.TID_X, synth_mod.F64)
    y = oracle_lib.layer_padded(x, lengths, w, nh)
    # garbage in the pad positions does not reach valid outputs
    x2 = synth_mod.normal((B, S, H), 4, synth_mod.TID_X_ALT_PADS, synth_mod.F64)
    for b in range(B):
        x2[b, :lengths[b]] = x[b, :lengths[b]]
    assert np.array_equal(oracle_lib.layer_padded(x2, lengths, w, nh), y)
    # a sequence run alone equals its slice of the batch; batch permutation permutes outputs
    for b in range(B):
        alone = oracle_lib.layer_padded(x[b:b + 1], lengths[b:b + 1], w, nh)
        assert np.array_equal(alone[0], y[b])
    perm = [4, 2, 0, 3, 1]
    yp = oracle_lib.layer_padded(x[perm], lengths[perm], w, nh)
    assert np.array_equal(yp, y[perm])
    # causality: the first p outputs of a sequence depend only on its first p tokens
    b = 2
    for p in (1, 4, 7):
        pre = oracle_lib.layer_padded(x[b:b + 1, :p], np.array([p], np.int32), w, nh)
        assert np.abs(pre[0] - y[b, :p]).max() < 1e-12
    # a length outside [0, pad_len] is refused
    with pytest.raises(RuntimeError):
        oracle_lib.layer_padded(x, np.array([3, 0, 9, 1, 5], np.int32), w, nh)


def test_stack_regenerates_layers(oracle_lib, synth_mod):
    H, nh, ffn, B, S, n_layers = 64, 2, 128, 3, 6, 3
    lengths = np.array([6, 2, 4], np.int32)
    x = synth_mod.normal((B, S, H), 8, 2, synth_mod.F64)
    wfn = lambda l: small_weights(synth_mod, H, nh, ffn, synth_mod.F16, layer=l)
    y = oracle_lib.stack_padded(x, lengths, wfn, n_layers, nh)
    for b in range(B):
        L = lengths[b]
        ref = x[b, :L]
        for l in range(n_layers):
            ref = torch_layer(ref, {k: v.astype(np.float64) for k, v in wfn(l).items()}, nh)
        assert np.abs(y[b, :L] - ref).max() < 1e-10
        assert not y[b, L:].any()
