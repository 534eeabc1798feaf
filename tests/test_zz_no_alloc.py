"""energon_rce_remove_padding_noalloc: packing for callers that cannot allocate.

Some callers have no way to allocate device memory where they pack a batch
(for example an inference runtime's per-request hook that forbids allocation
after start-up), so this entry point keeps the per-sequence offsets in a
fixed scratch array inside the library instead of a caller workspace.  The
test calls it several times in a row through the C ABI, with different
batches, and compares each packed result bit for bit with the allocating
pair energon_rce_offsets + energon_rce_remove_padding and with the oracle's
remove_padding (bit-exact is the tolerance the packing tests use).  It also
covers the documented edges: an empty batch, a batch that fills the scratch
array, a length outside [0, pad_len] (status set, nothing gathered), and a
batch above the scratch limit (refused on the host).  The file is named so
that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from padding_free_varlen_b200 import capi, synth

pytestmark = pytest.mark.gpu


def _reference_pack(d_x, d_len, B, S, H):
    cu = torch.empty(B + 1, dtype=torch.int32, device="cuda")
    st = torch.empty(1, dtype=torch.int32, device="cuda")
    capi.energon_rce_offsets(d_len, B, S, cu, st)
    out = torch.full((max(1, B * S), H), -7.0, dtype=d_x.dtype, device="cuda")
    capi.energon_rce_remove_padding(d_x, cu, B, S, H, d_x.element_size(), out)
    return out, st


def _noalloc_pack(d_x, d_len, B, S, H):
    got = torch.full((max(1, B * S), H), -7.0, dtype=torch.bfloat16, device="cuda")
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    capi.energon_rce_remove_padding_noalloc(d_x, d_len, B, S, H, 2, got, st)
    return got, st


def _case(B, S, H, seed, lo, hi):
    lengths = synth.uniform_int(B, lo, hi, seed, synth.TID_LENGTHS)
    x = synth.normal((B, S, H), seed, synth.TID_X, synth.BF16)
    d_x = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    return lengths, x, d_x, torch.from_numpy(lengths).cuda()


def test_noalloc_pack_matches_allocating_pack_and_oracle(oracle_lib):
    from padding_free_varlen_b200 import build
    build.build()
    capi.load()
    # (B, S, H, seed, lo, hi): the bf16 [64, 512, 4096] workload, a ragged batch with empty
    # sequences, and a batch that fills the scratch array (ENERGON_NOALLOC_MAX_BATCH offsets)
    cases = [(64, 512, 4096, 20260002, 1, 512), (300, 37, 24, 77, 0, 37),
             (capi.ENERGON_NOALLOC_MAX_BATCH, 3, 8, 5, 0, 3)]
    for B, S, H, seed, lo, hi in cases + cases[:1]:                        # calls in a row
        lengths, x, d_x, d_len = _case(B, S, H, seed, lo, hi)
        got, st = _noalloc_pack(d_x, d_len, B, S, H)
        ref, st_ref = _reference_pack(d_x, d_len, B, S, H)
        torch.cuda.synchronize()
        assert int(st.item()) == int(st_ref.item()) == 0
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
        cu, ost = oracle_lib.offsets(lengths, S)
        assert ost == 0
        want = np.full((B * S, H), -7.0, dtype=np.float32)
        want = synth.round_to(want.astype(np.float64), synth.BF16)       # the sentinel's bf16 bits
        want = oracle_lib.remove_padding(x, cu, out=want)
        assert np.array_equal(got.cpu().view(torch.int16).numpy().view(np.uint16), want)


def test_noalloc_empty_batch_and_bad_length():
    from padding_free_varlen_b200 import build
    build.build()
    capi.load()
    # batch 0: nothing to gather, status OK, the output untouched
    d_x = torch.zeros((1, 4, 8), dtype=torch.bfloat16, device="cuda")
    got, st = _noalloc_pack(d_x, torch.zeros(1, dtype=torch.int32, device="cuda"), 0, 4, 8)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and bool((got == -7.0).all())
    # a length of pad_len + 1: status BAD_LENGTH and nothing gathered
    lengths, x, d_x, _ = _case(5, 6, 16, 3, 1, 6)
    bad = lengths.copy()
    bad[2] = 7
    got, st = _noalloc_pack(d_x, torch.from_numpy(bad).cuda(), 5, 6, 16)
    torch.cuda.synchronize()
    assert int(st.item()) == capi.ENERGON_DEVICE_BAD_LENGTH
    assert bool((got == -7.0).all())
    # a valid call afterwards is unaffected by the failed one
    got, st = _noalloc_pack(d_x, torch.from_numpy(lengths).cuda(), 5, 6, 16)
    ref, _ = _reference_pack(d_x, torch.from_numpy(lengths).cuda(), 5, 6, 16)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_noalloc_refuses_batch_above_the_scratch_limit():
    from padding_free_varlen_b200 import build
    build.build()
    capi.load()
    B = capi.ENERGON_NOALLOC_MAX_BATCH + 1
    d_x = torch.zeros((B, 1, 8), dtype=torch.bfloat16, device="cuda")
    d_len = torch.ones(B, dtype=torch.int32, device="cuda")
    got = torch.zeros((B, 8), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(capi.EnergonError) as e:
        capi.energon_rce_remove_padding_noalloc(d_x, d_len, B, 1, 8, 2, got, st)
    assert e.value.code == capi.ENERGON_ERR_INVALID_ARGUMENT and "MAX_BATCH" in capi.energon_last_error()
