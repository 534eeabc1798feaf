"""The GPT-3 workloads at full size, in the launch configuration bench.py times.

* gpt3_layer (1 layer, hidden 12288, batch 1, pad 64, length 32): every valid output
  against the fp64 oracle.
* gpt3_stack_half_pad (12 layers, batch 32, pad 256, every length 128) and
  gpt3_stack_dynbatch (12 layers, batch 64, lengths U[1,256], pad = batch maximum): sampled
  outputs.  Causal attention makes the first p outputs of a sequence a function of its
  first p tokens only, so the oracle computes them exactly from a p-token prefix: whole
  short sequences and the first positions of long ones.  Properties that hold at any size
  are checked on the full output: pad rows are zero, the padded path and the path that
  packs only around each MLP give the same valid rows bit for bit, and different garbage
  in the pad positions changes no valid row.
"""
import numpy as np
import pytest
import torch

from padding_free_varlen_b200 import capi, synth
from helpers import check_end_to_end, to_device

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


def check(g, r, label):
    check_end_to_end(g, r, synth.F16, label)


def full_size_case(wl, oracle_lib, sample_plan):
    lengths, S = wl.lengths(), wl.padded_len()
    x = wl.x_padded()
    dev_layers, refs = upload_and_sample(wl, x, sample_plan, oracle_lib)
    out = run_stack(wl, dev_layers, x, lengths, S, 1)
    g_all = out.float().cpu().numpy()
    for b, ref in refs.items():
        p = sample_plan[b]
        check(g_all[b, :p].astype(np.float64), ref, f"{wl.name} seq {b} positions 0..{p - 1}")
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
