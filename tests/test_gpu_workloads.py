"""The GPT-3 workloads at full size, in the launch configuration bench.py times.

* gpt3_layer (1 layer, hidden 12288, batch 1, pad 64, length 32): every valid output
  against the fp64 oracle, under the stated tolerance (max-abs 2e-2 above one fp16
  rounding unit, rel-Frobenius 5e-3).
* gpt3_stack_half_pad (12 layers, batch 32, pad 256, every length 128) and
  gpt3_stack_dynbatch (12 layers, batch 64, lengths U[1,256], pad = batch maximum):
  - layer by layer: energon_layer_forward runs every layer on all packed tokens, and
    each layer's output is held to the stated tolerance against the oracle applied to
    that layer's GPU input, on sampled sequence prefixes (causal attention makes the
    first p outputs of a sequence a function of its first p tokens only);
  - the whole stack: energon_stack_forward's sampled outputs against the oracle's
    12-layer composition (relative Frobenius gated; the max-abs figure reported), and
    properties that hold at any size on the full output: pad rows are zero, the padded
    path and the path that packs only around each MLP give the same valid rows bit for
    bit, and different garbage in the pad positions changes no valid row.
* attention at hidden 12288 / 96 heads on sequences of 256 and 129 tokens (two query
  tiles, two key blocks): every position and head against the oracle on the GPU's own
  Q, K, V.
"""
import numpy as np
import pytest
import torch

from padding_free_varlen_b200 import capi, synth
from helpers import check_end_to_end, layer_ws_offsets, to_device, to_f64, ulp, ws_view

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from padding_free_varlen_b200 import build
    build.build()
    capi.load()
    yield
    torch.cuda.empty_cache()


def upload_and_sample(wl, x, plan, oracle_lib):
    """Generates each layer's weights once: uploads them and advances the oracle's samples
    (the first plan[b] tokens of sequence b, as one padded float64 batch) through that layer.
    Returns the device weights and {b: oracle output [plan[b], H]}."""
    seqs = list(plan)
    pmax = max(plan.values())
    lens = np.array([plan[b] for b in seqs], np.int32)
    y = np.zeros((len(seqs), pmax, wl.shape.hidden))
    for i, b in enumerate(seqs):
        y[i, :plan[b]] = x[b, :plan[b]].astype(np.float64)
    dev_layers = []
    for l in range(wl.n_layers):
        hw = wl.layer(l)
        dev_layers.append({k: to_device(v, wl.dtype) for k, v in hw.items()})
        y = oracle_lib.layer_padded(y, lens, hw, wl.shape.n_heads)
        del hw
    return dev_layers, {b: y[i, :plan[b]] for i, b in enumerate(seqs)}


def run_stack(wl, dev_layers, x, lengths, S, remove_padding):
    B, H = wl.batch, wl.shape.hidden
    cfg = capi.make_config(H, wl.shape.n_heads, wl.shape.ffn, capi.ENERGON_F16, wl.ln_eps)
    ws_bytes = capi.energon_workspace_bytes(cfg, B, S)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    tables = [capi.make_weights(d) for d in dev_layers]
    d_in = to_device(x, wl.dtype)
    d_out = torch.empty_like(d_in)
    d_out.view(torch.uint8).fill_(0xEE)
    st = torch.full((1,), -3, dtype=torch.int32, device="cuda")
    capi.energon_stack_forward(cfg, tables, wl.n_layers, d_in, torch.from_numpy(lengths).cuda(), B, S,
                               remove_padding, d_out, st, ws, ws_bytes)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    del ws
    return d_out


def check(g, r, label, max_abs=True):
    check_end_to_end(g, r, synth.F16, label, max_abs=max_abs)


def full_size_case(wl, oracle_lib, sample_plan):
    lengths, S = wl.lengths(), wl.padded_len()
    x = wl.x_padded()
    dev_layers, refs = upload_and_sample(wl, x, sample_plan, oracle_lib)
    out = run_stack(wl, dev_layers, x, lengths, S, 1)
    g_all = out.float().cpu().numpy()
    for b, ref in refs.items():
        p = sample_plan[b]
        # one layer: the stated bound on the layer output; a stack: rel-Frobenius gated
        check(g_all[b, :p].astype(np.float64), ref, f"{wl.name} seq {b} positions 0..{p - 1}",
              max_abs=wl.n_layers == 1)
    for b in range(wl.batch):                                     # pad rows are zero
        assert not out[b, lengths[b]:].view(torch.int16).any()
    out_pad = run_stack(wl, dev_layers, x, lengths, S, 0)         # padded path: same valid rows
    assert torch.equal(out.view(torch.int16), out_pad.view(torch.int16))
    del out_pad
    out_mlp = run_stack(wl, dev_layers, x, lengths, S, 2)         # packing around each MLP only
    assert torch.equal(out.view(torch.int16), out_mlp.view(torch.int16))
    del out_mlp
    x2 = wl.x_padded(synth.TID_X_ALT_PADS)                        # other pad garbage: same rows
    for b in range(wl.batch):
        x2[b, :lengths[b]] = x[b, :lengths[b]]
    out2 = run_stack(wl, dev_layers, x2, lengths, S, 1)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    del out2, out, dev_layers


def test_gpt3_layer_full(oracle_lib):
    wl = synth.WORKLOADS["gpt3_layer"]
    full_size_case(wl, oracle_lib, {0: 32})                       # every valid row


def test_gpt3_stack_half_pad_sampled(oracle_lib):
    wl = synth.WORKLOADS["gpt3_stack_half_pad"]
    full_size_case(wl, oracle_lib, {0: 4, 13: 4, 31: 4})


def test_gpt3_stack_dynbatch_sampled(oracle_lib):
    wl = synth.WORKLOADS["gpt3_stack_dynbatch"]
    lengths = wl.lengths()
    order = np.argsort(lengths, kind="stable")
    plan = {int(b): int(lengths[b]) for b in order[:3]}           # the three shortest, whole
    plan[int(order[-1])] = 2                                      # the longest: first 2 positions
    full_size_case(wl, oracle_lib, plan)


def per_layer_case(wl, oracle_lib, plan):
    """energon_layer_forward layer by layer on all packed tokens; each layer's output on the
    sampled prefixes (plan: sequence -> tokens) against the oracle on the GPU's own input of
    that layer, under the stated tolerance."""
    lengths, S = wl.lengths(), wl.padded_len()
    B, H, nh = wl.batch, wl.shape.hidden, wl.shape.n_heads
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    d_x = to_device(wl.x_padded(), wl.dtype)
    d_len = torch.from_numpy(lengths).cuda()
    d_cu = torch.empty(B + 1, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    capi.energon_rce_offsets(d_len, B, S, d_cu, st)
    xa = torch.zeros((B * S, H), dtype=torch.float16, device="cuda")
    capi.energon_rce_remove_padding(d_x, d_cu, B, S, H, 2, xa)
    del d_x
    ya = torch.empty_like(xa)
    cfg = capi.make_config(H, nh, wl.shape.ffn, capi.ENERGON_F16, wl.ln_eps)
    ws_bytes = capi.energon_workspace_bytes(cfg, B, S)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    worst = 0.0
    for l in range(wl.n_layers):
        hw = wl.layer(l)
        dev = {k: to_device(v, wl.dtype) for k, v in hw.items()}
        capi.energon_layer_forward(cfg, capi.make_weights(dev), xa, d_cu, B, S, ya, st, ws, ws_bytes)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for b, p in plan.items():
            rows = slice(int(cu[b]), int(cu[b]) + p)
            xin = xa[rows].double().cpu().numpy()
            ref = oracle_lib.layer_sequence(xin, hw, nh)
            g = ya[rows].double().cpu().numpy()
            _, _, excess = check_end_to_end(g, ref, synth.F16, f"{wl.name} layer {l} seq {b} positions 0..{p - 1}")
            worst = max(worst, excess)
        xa, ya = ya, xa
        del dev, hw
    print(f"\n[{wl.name}] worst max-abs beyond one ulp over {wl.n_layers} layers: {worst:.3e}")


def test_gpt3_stack_half_pad_per_layer(oracle_lib):
    wl = synth.WORKLOADS["gpt3_stack_half_pad"]
    per_layer_case(wl, oracle_lib, {0: 24, 31: 24})


def test_gpt3_stack_dynbatch_per_layer(oracle_lib):
    wl = synth.WORKLOADS["gpt3_stack_dynbatch"]
    lengths = wl.lengths()
    order = np.argsort(lengths, kind="stable")
    per_layer_case(wl, oracle_lib, {int(order[-1]): 24, int(order[0]): int(lengths[order[0]]),
                                    int(order[len(order) // 2]): 16})


def test_gpt3_attention_long_sequences(oracle_lib):
    """Attention at hidden 12288 / 96 heads on sequences of 256 and 129 tokens: the second
    query tile and the second key block at full size, every position and every head,
    against the oracle on the GPU's own Q, K (two-term) and V."""
    shape = synth.GPT3
    H, F, nh, d = shape.hidden, shape.ffn, shape.n_heads, shape.head_dim
    lengths = np.array([256, 129], np.int32)
    B, S, seed = 2, 256, 20260007
    x = synth.normal((B, S, H), seed, synth.TID_X, synth.F16)
    x_pk = np.concatenate([x[b, :lengths[b]] for b in range(B)], axis=0)
    T = x_pk.shape[0]
    d_x = torch.zeros((B * S, H), dtype=torch.float16, device="cuda")
    d_x[:T] = to_device(x_pk, synth.F16)
    cu = np.array([0, 256, 385], np.int32)
    d_cu = torch.from_numpy(cu).cuda()
    hw = synth.layer_weights(shape, 0, seed, synth.F16)
    dev = {k: to_device(v, synth.F16) for k, v in hw.items()}
    cfg = capi.make_config(H, nh, F, capi.ENERGON_F16)
    ws_bytes = capi.energon_workspace_bytes(cfg, B, S)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    d_y = torch.empty_like(d_x)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    capi.energon_layer_forward(cfg, capi.make_weights(dev), d_x, d_cu, B, S, d_y, st, ws, ws_bytes)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    offs = layer_ws_offsets(H, F, B, S, 2)
    qkv = to_f64(ws_view(ws, offs, "qkv", T, torch.float16))
    qkv[:, :2 * H] += to_f64(ws_view(ws, offs, "qk_lo", T, torch.float16))
    o = to_f64(ws_view(ws, offs, "o", T, torch.float16))
    for b in range(B):
        rows = slice(int(cu[b]), int(cu[b + 1]))
        ref = oracle_lib.causal_attention(qkv[rows], nh)
        v = np.abs(qkv[rows, 2 * H:]).reshape(-1, nh, d).max(axis=(0, 2))
        # one fp16 rounding of the output, fp32 accumulation, and the rounding of P to fp16
        # before P V (unit roundoff times the largest |v| of the head)
        tol = ulp(ref, synth.F16) + 8 * np.sqrt(int(lengths[b])) * 2.0 ** -24 * np.abs(ref).max() + \
            np.repeat(2.0 ** -11 * v, d)[None, :]
        ratio = np.abs(o[rows] - ref) / tol
        worst = np.unravel_index(int(ratio.argmax()), ratio.shape)
        print(f"\n[attention seq {b} len {lengths[b]}] max err/tol {ratio.max():.3f} at position {worst[0]}, "
              f"column {worst[1]}; positions >= 128 max {ratio[128:].max() if lengths[b] > 128 else 0:.3f}")
        assert ratio.max() <= 1.0
