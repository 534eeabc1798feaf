"""energon_rce_remove_padding_noalloc: packing for callers that cannot allocate.

Some callers have no way to allocate device memory where they pack a batch
(for example an inference runtime's per-request hook that forbids allocation
after start-up), so this entry point keeps the per-sequence offsets in a
fixed scratch array inside the library instead of a caller workspace.  The
test calls it twice in a row through the C ABI, with different batches, and
compares each packed result bit for bit with the allocating pair
energon_rce_offsets + energon_rce_remove_padding (bit-exact is the tolerance
the packing tests use).  It also checks that a batch above the scratch limit
is refused on the host.  The file is named so that pytest collects it last.
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
    out = torch.full((B * S, H), -7.0, dtype=d_x.dtype, device="cuda")
    capi.energon_rce_remove_padding(d_x, cu, B, S, H, d_x.element_size(), out)
    return out, st


def test_noalloc_pack_matches_allocating_pack_twice():
    from padding_free_varlen_b200 import build
    build.build()
    capi.load()
    cases = [(64, 512, 4096, 20260002, 1, 512), (300, 37, 24, 77, 0, 37)]  # (B, S, H, seed, lo, hi)
    for B, S, H, seed, lo, hi in cases:                                     # two calls in a row
        lengths = synth.uniform_int(B, lo, hi, seed, synth.TID_LENGTHS)
        x = synth.normal((B, S, H), seed, synth.TID_X, synth.BF16)
        d_x = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
        d_len = torch.from_numpy(lengths).cuda()
        got = torch.full((B * S, H), -7.0, dtype=torch.bfloat16, device="cuda")
        st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        capi.energon_rce_remove_padding_noalloc(d_x, d_len, B, S, H, 2, got, st)
        ref, st_ref = _reference_pack(d_x, d_len, B, S, H)
        torch.cuda.synchronize()
        assert int(st.item()) == int(st_ref.item()) == 0
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    with pytest.raises(capi.EnergonError) as e:
        capi.energon_rce_remove_padding_noalloc(d_x, d_len, capi.ENERGON_NOALLOC_MAX_BATCH + 1, S, H, 2, got, st)
    assert e.value.code == capi.ENERGON_ERR_INVALID_ARGUMENT and "MAX_BATCH" in capi.energon_last_error()
