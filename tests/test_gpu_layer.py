"""The GPT-3 decoder layer and the stack on the GPU against the fp64 oracle.

Two kinds of checks, all through the C ABI:
  * step parity: every step's GPU output (read from the documented workspace
    regions) against the oracle applied to the GPU's own inputs of that step,
    so each step is checked alone: within one unit in the last place of the
    output type plus an fp32-accumulation allowance.  The first LayerNorm is
    folded into the QKV GEMM: the GEMM's operand is u = x * ln1_g rounded to
    the storage type, so the QKV step is held to the oracle's LN(x) W^T + b
    plus the exact effect of that one rounding (zero when ln1_g is 1).  Q and
    K are two-term values (high and low halves), checked as their sum;
  * end to end: the layer output against the oracle on the original inputs,
    relative Frobenius error <= 5e-3 and max-abs error <= 2e-2 above one
    rounding unit of the storage type (helpers.check_end_to_end), the
    tolerance stated for fp16 / bf16 layer outputs with fp32 accumulation.
"""
import numpy as np
import pytest
import torch

from padding_free_varlen_b200 import capi, synth
from helpers import (SYNTH_TO_ENERGON, TORCH_OF_SYNTH, check_end_to_end, gpu_layer_weights, layer_ws_offsets,
                     to_device, to_f64, ulp, ws_view)

pytestmark = pytest.mark.gpu

@pytest.fixture(scope="module", autouse=True)
def _lib():
    from padding_free_varlen_b200 import build
    build.build()
    capi.load()


def acc_tol(r: np.ndarray, K: int) -> np.ndarray:
    """fp32 accumulation over K terms, relative to the output's scale."""
    scale = np.sqrt(np.mean(r ** 2)) + 1e-30
    return 8 * np.sqrt(K) * 2.0 ** -24 * scale


def step_tol(r: np.ndarray, dtype: int, K: int) -> np.ndarray:
    """One ulp of the storage type at |r| plus fp32 accumulation over K terms."""
    return ulp(r, dtype) + acc_tol(r, K)


def check_step(name, g, r, dtype, K, report, extra=0.0):
    err = np.abs(g - r)
    tol = step_tol(r, dtype, K) + extra
    ratio = float((err / tol).max()) if err.size else 0.0
    report[name] = ratio
    assert ratio <= 1.0, f"{name}: max err/tol {ratio:.3f} (max err {err.max():.3e})"


def pack(x_padded: np.ndarray, lengths: np.ndarray) -> np.ndarray:
    return np.concatenate([x_padded[b, :lengths[b]] for b in range(len(lengths))], axis=0)


def read_intermediates(ws, H, F, B, S, T, tdt):
    """Host copies of the workspace regions a layer call leaves behind (float64)."""
    e = torch.tensor([], dtype=tdt).element_size()
    offs = layer_ws_offsets(H, F, B, S, e)
    it = {k: to_f64(ws_view(ws, offs, k, T, tdt)) for k in ("a", "qkv", "o", "f")}
    it["x1"] = to_f64(ws_view(ws, offs, "x1", T, torch.float32))
    if tdt != torch.float32:
        it["qk_lo"] = to_f64(ws_view(ws, offs, "qk_lo", T, tdt))
    off, _ = offs["stats"]
    it["stats"] = ws[off: off + T * 8].view(torch.float32).view(T, 2).double().cpu().numpy()
    return it


def run_layer(shape, dtype, lengths, S, seed, recipe, layer=0, x_pk=None):
    """Packs the synthetic batch (or takes x_pk), runs energon_layer_forward, returns host copies."""
    B = len(lengths)
    H, F = shape.hidden, shape.ffn
    if x_pk is None:
        x_pad = synth.normal((B, S, H), seed, synth.TID_X, dtype)
        x_pk = pack(x_pad, lengths)
    T = x_pk.shape[0]
    tdt = TORCH_OF_SYNTH[dtype]
    d_x = torch.empty((B * S, H), dtype=tdt, device="cuda")
    d_x.view(torch.uint8).fill_(0x3C)                      # garbage beyond T
    if T:
        d_x[:T] = to_device(x_pk, dtype)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    d_cu = torch.from_numpy(cu).cuda()
    host_w, dev_w = gpu_layer_weights(shape, layer, seed, dtype, recipe)
    cfg = capi.make_config(H, shape.n_heads, F, SYNTH_TO_ENERGON[dtype])
    ws_bytes = capi.energon_workspace_bytes(cfg, B, S)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    d_y = torch.empty_like(d_x)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    w = capi.make_weights(dev_w)
    capi.energon_layer_forward(cfg, w, d_x, d_cu, B, S, d_y, st, ws, ws_bytes)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    inter = read_intermediates(ws, H, F, B, S, T, tdt)
    return dict(x_pk=x_pk, T=T, cu=cu, y=to_f64(d_y[:T]), inter=inter, w=host_w)


def qkv_reference(x, w, dtype, oracle_lib):
    """LN(x) W_qkv^T + b_qkv from the oracle, and the exact effect on it of the folded
    LayerNorm's one rounding: the QKV GEMM reads u = round(x * g) instead of x * g, which
    moves output n of row r by rstd_r * sum_k (u - x g)[r][k] W[n][k]."""
    g = synth.to_f64(w["ln1_g"], dtype)
    ref = oracle_lib.linear(oracle_lib.layernorm(x, w["ln1_g"], w["ln1_b"]), w["w_qkv"], w["b_qkv"])
    xg = x * g[None, :]
    du = synth.to_f64(synth.round_to(xg, dtype), dtype) - xg
    if not du.any():
        return ref, np.zeros_like(ref)
    mean = x.mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(((x - mean) ** 2).mean(axis=1, keepdims=True) + 1e-5)
    return ref, rstd * oracle_lib.linear(du, w["w_qkv"], None)


def layer_step_checks(res, shape, dtype, oracle_lib):
    x = synth.to_f64(res["x_pk"], dtype)
    w, it, cu = res["w"], res["inter"], res["cu"]
    H, F, nh = shape.hidden, shape.ffn, shape.n_heads
    report = {}
    # LN1 folded into QKV: Q and K as hi + lo, V as one rounding
    qkv_ref, shift = qkv_reference(x, w, dtype, oracle_lib)
    qkv = it["qkv"].copy()
    two_term = dtype != synth.F32
    if two_term:
        qkv[:, :2 * H] += it["qk_lo"]
    want = qkv_ref + shift                                # the result on the GPU's own operand u
    err = np.abs(qkv - want)
    tol = np.full_like(want, acc_tol(want, H))
    tol[:, 2 * H:] += ulp(want[:, 2 * H:], dtype)         # V: one rounding of the storage type
    if two_term:                                          # Q, K: the low half's own rounding
        tol[:, :2 * H] += ulp(it["qk_lo"], dtype) + 2.0 ** -22 * np.abs(want[:, :2 * H])
    else:
        tol += ulp(want, dtype)
    report["qkv"] = float((err / tol).max()) if err.size else 0.0
    assert report["qkv"] <= 1.0, report
    # attention on the GPU's q, k (hi + lo) and v, one sequence at a time.  The tensor-core
    # kernel (16-bit, head_dim 128) rounds the probabilities P to the storage type before
    # P V: allow that rounding (unit roundoff times the largest |v| the row can weight).
    o_ref = np.concatenate([oracle_lib.causal_attention(qkv[cu[b]:cu[b + 1]], nh)
                            for b in range(len(cu) - 1)], axis=0)
    extra = np.zeros_like(o_ref)
    if dtype in (synth.F16, synth.BF16) and H // nh == 128:
        u = 2.0 ** -11 if dtype == synth.F16 else 2.0 ** -8
        d = H // nh
        for b in range(len(cu) - 1):
            v = np.abs(qkv[cu[b]:cu[b + 1], 2 * H:])
            for j in range(nh):
                extra[cu[b]:cu[b + 1], j * d:(j + 1) * d] = u * (v[:, j * d:(j + 1) * d].max() if len(v) else 0)
    check_step("attention", it["o"], o_ref, dtype, max(1, int(np.diff(cu).max())), report, extra)
    # out-projection + residual, kept in fp32
    x1_ref = x + oracle_lib.linear(it["o"], w["w_o"], w["b_o"])
    check_step("out_proj_residual", it["x1"], x1_ref, synth.F32, H, report)
    check_step("ln2", it["a"], oracle_lib.layernorm(it["x1"], w["ln2_g"], w["ln2_b"]), dtype, H, report)
    check_step("ffn1_gelu", it["f"], oracle_lib.gelu(oracle_lib.linear(it["a"], w["w_1"], w["b_1"])), dtype, H,
               report)
    check_step("ffn2_residual", res["y"], it["x1"] + oracle_lib.linear(it["f"], w["w_2"], w["b_2"]), dtype, F,
               report)
    return report


NONZERO = synth.WeightRecipe(w_std=0.02, bias_std=0.1, gamma_std=0.2, beta_std=0.1)


@pytest.mark.parametrize("dtype,nh", [(synth.F16, 2), (synth.BF16, 2), (synth.F16, 4), (synth.F32, 2)])
def test_layer_steps_and_end_to_end(oracle_lib, dtype, nh):
    shape = synth.LayerShape(256, nh, 1024)
    lengths = np.array([70, 1, 33, 0, 129], np.int32)       # ragged, a length-1 and an empty sequence
    S = 130
    res = run_layer(shape, dtype, lengths, S, seed=31 + nh, recipe=NONZERO)
    report = layer_step_checks(res, shape, dtype, oracle_lib)
    x = synth.to_f64(res["x_pk"], dtype)
    ref = np.concatenate([oracle_lib.layer_sequence(x[res["cu"][b]:res["cu"][b + 1]], res["w"], nh)
                          for b in range(len(lengths)) if lengths[b] > 0], axis=0)
    print(f"\n[layer {synth.DTYPE_NAMES[dtype]} nh={nh}] step err/tol {report}")
    check_end_to_end(res["y"], ref, dtype, f"layer {synth.DTYPE_NAMES[dtype]} nh={nh}")


@pytest.mark.parametrize("T_target", [1, 127, 128, 129, 300])
def test_layer_row_tails(oracle_lib, T_target):
    """M tails around the 128-row GEMM tile, one sequence of T tokens."""
    shape = synth.LayerShape(256, 2, 512)
    lengths = np.array([T_target], np.int32)
    res = run_layer(shape, synth.F16, lengths, T_target, seed=5, recipe=NONZERO)
    layer_step_checks(res, shape, synth.F16, oracle_lib)


def stack_run(wl_dtype, shape, n_layers, x_pad, lengths, seed, recipe, remove_padding, lengths_dev=None):
    B, S, H = x_pad.shape
    cfg = capi.make_config(H, shape.n_heads, shape.ffn, SYNTH_TO_ENERGON[wl_dtype])
    ws_bytes = capi.energon_workspace_bytes(cfg, B, S)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    keep = [gpu_layer_weights(shape, l, seed, wl_dtype, recipe) for l in range(n_layers)]
    tables = [capi.make_weights(d) for _, d in keep]
    d_in = to_device(x_pad, wl_dtype)
    d_out = torch.empty_like(d_in)
    d_out.view(torch.uint8).fill_(0xEE)
    d_len = lengths_dev if lengths_dev is not None else torch.from_numpy(lengths.astype(np.int32)).cuda()
    st = torch.full((1,), -5, dtype=torch.int32, device="cuda")
    capi.energon_stack_forward(cfg, tables, n_layers, d_in, d_len, B, S, remove_padding, d_out, st, ws, ws_bytes)
    torch.cuda.synchronize()
    return d_out, int(st.item()), [h for h, _ in keep]


def test_tiny_workload_stack(oracle_lib):
    """The tiny fp32 workload (1 layer, hidden 256, 4 heads, FFN 1024, batch 4, pad 32)."""
    wl = synth.WORKLOADS["tiny"]
    lengths, x = wl.lengths(), wl.x_padded()
    out, st, hw = stack_run(wl.dtype, wl.shape, 1, x, lengths, wl.seed, wl.recipe, 1)
    assert st == 0
    ref = oracle_lib.layer_padded(x.astype(np.float64), lengths, hw[0], wl.shape.n_heads)
    check_end_to_end(to_f64(out), ref, synth.F32, "tiny fp32")
    for b in range(wl.batch):
        assert (out[b, lengths[b]:].view(torch.int32) == 0).all()


@pytest.mark.parametrize("dtype", [synth.F16, synth.BF16])
def test_stack_packed_equals_padded_and_oracle(oracle_lib, dtype):
    shape = synth.LayerShape(256, 2, 1024)
    lengths = np.array([17, 64, 1, 0, 40, 64], np.int32)
    B, S, L = len(lengths), 64, 3
    x = synth.normal((B, S, shape.hidden), 12, synth.TID_X, dtype)
    out_pk, st1, hw = stack_run(dtype, shape, L, x, lengths, 12, NONZERO, 1)
    out_pd, st2, _ = stack_run(dtype, shape, L, x, lengths, 12, NONZERO, 0)
    out_mlp, st6, _ = stack_run(dtype, shape, L, x, lengths, 12, NONZERO, 2)
    assert st1 == st2 == st6 == 0
    # the padded run computes pad rows too, yet every valid row must agree bit for bit; so must
    # the run that packs only around each MLP (attention on the padded rows)
    assert torch.equal(out_pk.view(torch.int16), out_pd.view(torch.int16))
    assert torch.equal(out_pk.view(torch.int16), out_mlp.view(torch.int16))
    # The stated tolerance is for a layer output.  fp16 meets it through 3 layers; bf16 (unit
    # roundoff 8x fp16's) is held to it over one layer, its 3-layer run to the exact checks.
    L_ref = L if dtype == synth.F16 else 1
    if L_ref != L:
        out_pk1, st0, _ = stack_run(dtype, shape, L_ref, x, lengths, 12, NONZERO, 1)
        assert st0 == 0
    else:
        out_pk1 = out_pk
    ref = oracle_lib.stack_padded(synth.to_f64(x, dtype), lengths, lambda l: hw[l], L_ref, shape.n_heads)
    check_end_to_end(to_f64(out_pk1), ref, dtype, f"stack {synth.DTYPE_NAMES[dtype]} L={L_ref}")
    # garbage in the pad positions does not reach valid outputs
    x2 = synth.normal((B, S, shape.hidden), 12, synth.TID_X_ALT_PADS, dtype)
    for b in range(B):
        x2[b, :lengths[b]] = x[b, :lengths[b]]
    out2, st3, _ = stack_run(dtype, shape, L, x2, lengths, 12, NONZERO, 1)
    assert st3 == 0 and torch.equal(out2.view(torch.int16), out_pk.view(torch.int16))
    # a sequence run alone equals its slice of the batch: bit for bit when the launch shape
    # is the same (the other sequences given length 0); as a batch of one, the buffer holds
    # <= 128 rows and the weight-streaming GEMMs split K, so the sums are ordered
    # differently and the rows agree within the tolerance instead
    for b in (0, 2):
        only = np.zeros_like(lengths)
        only[b] = lengths[b]
        same_shape, st4, _ = stack_run(dtype, shape, L, x, only, 12, NONZERO, 1)
        assert st4 == 0 and torch.equal(same_shape[b].view(torch.int16), out_pk[b].view(torch.int16))
        alone, st5, _ = stack_run(dtype, shape, L, x[b:b + 1], lengths[b:b + 1], 12, NONZERO, 1)
        assert st5 == 0
        if lengths[b]:
            check_end_to_end(to_f64(alone[0, :lengths[b]]), to_f64(out_pk[b, :lengths[b]]), dtype,
                             f"alone vs batch seq {b}")


@pytest.mark.parametrize("S,lens", [(512, [192, 320]), (256, [96, 160]), (256, [240, 240])])
def test_gemm_wave_tail_cut_does_not_change_rows(oracle_lib, S, lens):
    """Hidden 1024, FFN 2560, 16 sequences.  On 148 SMs (74 CTA pairs) the last, partly
    filled round of 512 x 256 pair tiles is cut into half units (one row tile) or quarter
    units (one row tile, 128 columns) depending on how many tiles it holds: with 4096
    valid tokens the packed QKV and FFN1 GEMMs (96 and 80 tiles) cut their tail in halves;
    with 2048 the out-projection and FFN2 (16 tiles) and FFN1 (40) cut it in quarters.
    With 3840 (15 row tiles of 256) the last pair row holds one row tile, and the full
    tiles of that row skip the empty one.  The padded runs (more rows) cut differently or
    not at all.  Valid rows must agree bit for bit across the three modes, and match the
    oracle."""
    shape = synth.LayerShape(1024, 8, 2560)
    B = 16
    lengths = np.array(lens * 8, np.int32)
    x = synth.normal((B, S, shape.hidden), 31, synth.TID_X, synth.F16)
    out1, st1, hw = stack_run(synth.F16, shape, 1, x, lengths, 31, NONZERO, 1)
    out0, st0, _ = stack_run(synth.F16, shape, 1, x, lengths, 31, NONZERO, 0)
    out2, st2, _ = stack_run(synth.F16, shape, 1, x, lengths, 31, NONZERO, 2)
    assert st0 == st1 == st2 == 0
    assert torch.equal(out1.view(torch.int16), out0.view(torch.int16))
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    sel = [0, 1]
    ref = oracle_lib.layer_padded(synth.to_f64(x[sel], synth.F16), lengths[sel], hw[0], shape.n_heads)
    for j, b in enumerate(sel):
        n = int(lengths[b])
        check_end_to_end(to_f64(out1[b, :n]), ref[j, :n], synth.F16, f"wave-tail layer seq {b}")


def test_workspace_offset_by_16_bytes_gives_the_same_rows():
    """FFN2's epilogue reads its fp32 residual rows in 32-byte loads when they start on
    32-byte boundaries and in 16-byte loads otherwise (the out-projection's fp32 output goes
    out by TMA either way).  A workspace that starts 16 bytes past a 32-byte boundary takes
    the second path; the results must be bit-identical to an aligned workspace's."""
    shape = synth.LayerShape(1024, 8, 2560)
    H = shape.hidden
    lengths = np.array([96, 160] * 8, np.int32)
    B, S = len(lengths), 256
    x = synth.normal((B, S, H), 33, synth.TID_X, synth.F16)
    keep = [gpu_layer_weights(shape, 0, 33, synth.F16, NONZERO)]
    cfg = capi.make_config(H, shape.n_heads, shape.ffn, capi.ENERGON_F16)
    ws_bytes = capi.energon_workspace_bytes(cfg, B, S)
    big = torch.empty(ws_bytes + 1024, dtype=torch.uint8, device="cuda")
    assert big.data_ptr() % 256 == 0
    d_in = to_device(x, synth.F16)
    d_len = torch.from_numpy(lengths).cuda()
    tables = [capi.make_weights(d) for _, d in keep]
    outs = []
    for off in (0, 16):
        ws = big[off:off + ws_bytes]
        out = torch.empty_like(d_in)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        capi.energon_stack_forward(cfg, tables, 1, d_in, d_len, B, S, 1, out, st, ws, ws_bytes)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        outs.append(out)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))


def test_prepared_fold_vectors_match_the_per_call_ones(oracle_lib):
    """energon_layer_fold_weights writes c = W_qkv ln1_g and d = b_qkv + W_qkv ln1_b (checked
    against the oracle's linear map); a stack given them returns, bit for bit, what it
    returns when every layer computes them itself."""
    shape = synth.LayerShape(256, 2, 1024)
    H = shape.hidden
    lengths = np.array([17, 64, 1, 0, 40, 64], np.int32)
    B, S, L = len(lengths), 64, 2
    x = synth.normal((B, S, H), 12, synth.TID_X, synth.F16)
    out_call, st1, hw = stack_run(synth.F16, shape, L, x, lengths, 12, NONZERO, 1)
    cfg = capi.make_config(H, shape.n_heads, shape.ffn, capi.ENERGON_F16)
    keep = [gpu_layer_weights(shape, l, 12, synth.F16, NONZERO) for l in range(L)]
    for host, dev in keep:
        fold = torch.full((6 * H,), float("nan"), dtype=torch.float32, device="cuda")
        capi.energon_layer_fold_weights(cfg, capi.make_weights(dev), fold)
        dev["ln1_fold"] = fold
        torch.cuda.synchronize()
        g = synth.to_f64(host["ln1_g"], synth.F16)[None, :]
        beta = synth.to_f64(host["ln1_b"], synth.F16)[None, :]
        c_ref = oracle_lib.linear(g, host["w_qkv"])[0]
        d_ref = oracle_lib.linear(beta, host["w_qkv"], host["b_qkv"])[0]
        got = fold.double().cpu().numpy()
        scale = 8 * np.sqrt(H) * 2.0 ** -24
        assert np.abs(got[:3 * H] - c_ref).max() <= scale * np.abs(c_ref).max() + 1e-30
        assert np.abs(got[3 * H:] - d_ref).max() <= scale * np.abs(d_ref).max() + 1e-30
    ws_bytes = capi.energon_workspace_bytes(cfg, B, S)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    d_in = to_device(x, synth.F16)
    out_prep = torch.empty_like(d_in)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tables = [capi.make_weights(d) for _, d in keep]
    capi.energon_trace_start()
    capi.energon_stack_forward(cfg, tables, L, d_in, torch.from_numpy(lengths).cuda(), B, S, 1, out_prep, st, ws,
                               ws_bytes)
    trace = capi.energon_trace_stop()
    assert st1 == 0 and int(st.item()) == 0
    assert "ln_fold_weights" not in trace                 # nothing recomputed per call
    assert torch.equal(out_prep.view(torch.int16), out_call.view(torch.int16))


def test_stack_invalid_lengths_and_empty_batch():
    shape = synth.LayerShape(256, 2, 512)
    x = synth.normal((3, 16, 256), 4, synth.TID_X, synth.F16)
    out, st, _ = stack_run(synth.F16, shape, 2, x, np.array([3, 17, 2], np.int32), 4, NONZERO, 1)
    assert st == capi.ENERGON_DEVICE_BAD_LENGTH
    assert (out.view(torch.int16) == 0).all()
    out, st, _ = stack_run(synth.F16, shape, 2, x, np.array([3, -1, 2], np.int32), 4, NONZERO, 0)
    assert st == capi.ENERGON_DEVICE_BAD_LENGTH and (out.view(torch.int16) == 0).all()
    out, st, _ = stack_run(synth.F16, shape, 2, x, np.array([3, 17, 2], np.int32), 4, NONZERO, 2)
    assert st == capi.ENERGON_DEVICE_BAD_LENGTH and (out.view(torch.int16) == 0).all()
    for mode in (0, 1, 2):
        out, st, _ = stack_run(synth.F16, shape, 2, x, np.zeros(3, np.int32), 4, NONZERO, mode)
        assert st == 0 and (out.view(torch.int16) == 0).all()


@pytest.mark.parametrize("S", [16, 64])
def test_stack_modes_launch_their_own_schedules(S):
    """The three modes agree on valid rows by design, so their schedules are told apart by
    the launch trace.  Mode 1 packs inside the first LayerNorm and, when the last FFN2 runs
    on the CTA-pair GEMM (more than 128 buffer rows), scatters back inside its epilogue;
    mode 0 never packs; mode 2 packs around every MLP with the standalone operators."""
    shape = synth.LayerShape(256, 2, 512)
    lengths = np.array([5, S, 9], np.int32)
    x = synth.normal((3, S, 256), 3, synth.TID_X, synth.F16)
    L = 3
    pair = 3 * S > 128
    want = {1: {"remove_padding": 0, "layernorm_remove": 1, "zero_pads": 1, "padded_starts": 0,
                "rebuild_padding": 0 if pair else 1, "gemm_ffn2_rebuild": 1 if pair else 0},
            0: {"remove_padding": 0, "layernorm_remove": 0, "rebuild_padding": 1, "padded_starts": 1,
                "gemm_ffn2_rebuild": 0},
            2: {"remove_padding": L, "layernorm_remove": 0, "rebuild_padding": L, "padded_starts": 1,
                "gemm_ffn2_rebuild": 0}}
    outs = {}
    for mode, counts in want.items():
        capi.energon_trace_start()
        outs[mode], st, _ = stack_run(synth.F16, shape, L, x, lengths, 3, NONZERO, mode)
        trace = capi.energon_trace_stop()
        assert st == 0
        got = {k: trace.get(k, (0, 0.0))[0] for k in counts}
        assert got == counts, (mode, trace)
        n_ffn2 = trace.get("gemm_ffn2", (0, 0.0))[0] + trace.get("gemm_ffn2_rebuild", (0, 0.0))[0]
        assert trace["gemm_qkv"][0] == n_ffn2 == L
    assert torch.equal(outs[1].view(torch.int16), outs[0].view(torch.int16))
    assert torch.equal(outs[1].view(torch.int16), outs[2].view(torch.int16))


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_stack_without_layers_repacks_input(mode):
    """Zero layers: every mode returns the valid rows of the input unchanged and zero pads."""
    shape = synth.LayerShape(256, 2, 512)
    lengths = np.array([5, 16, 0, 9], np.int32)
    x = synth.normal((4, 16, 256), 8, synth.TID_X, synth.F16)
    out, st, _ = stack_run(synth.F16, shape, 0, x, lengths, 8, NONZERO, mode)
    assert st == 0
    got = out.cpu().view(torch.int16).numpy()
    for b in range(4):
        assert np.array_equal(got[b, :lengths[b]], x[b, :lengths[b]].view(np.int16))
        assert not got[b, lengths[b]:].any()


def test_bounded_wait_times_out_and_context_survives():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    capi.energon_selftest_bounded_wait(st, 20000)          # 20 ms, nobody arrives
    torch.cuda.synchronize()
    assert int(st.item()) == capi.ENERGON_DEVICE_TIMEOUT
    cu = torch.empty(3, dtype=torch.int32, device="cuda")
    st2 = torch.empty(1, dtype=torch.int32, device="cuda")
    capi.energon_rce_offsets(torch.tensor([2, 5], dtype=torch.int32, device="cuda"), 2, 8, cu, st2)
    torch.cuda.synchronize()
    assert cu.tolist() == [0, 2, 7] and int(st2.item()) == 0
