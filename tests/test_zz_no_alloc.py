"""basiskv_decode_noalloc: the fused decode step for callers that cannot
allocate device memory (a runtime that owns every device allocation through
its own pool, a plug-in that runs where allocation is forbidden, a service
with a footprint fixed at start-up).  It uses the library's static device
scratch array instead of a workspace.

Checked through the C-ABI against basiskv_decode with a caller workspace, on
two steps in a row (each appending a token), within the tolerance the other
parity tests use.  This file sorts last so that a run stopping at the first
failure has run every other test already; it also passes on its own in a
fresh process.
"""
import numpy as np
import pytest
import torch

import sparse_decode_attention_basiskv_b200 as bkv
from sparse_decode_attention_basiskv_b200 import synth
from sparse_decode_attention_basiskv_b200.layer import DecodeLayer

pytestmark = pytest.mark.gpu

Y_REL, Y_ABS = 1e-2, 1e-3


def _max_err_ok(y, ref):
    err = (y.float() - ref.float()).abs().max().item()
    bound = Y_REL * ref.float().abs().max().item() + Y_ABS
    return err <= bound, err, bound


@pytest.mark.parametrize("base", [synth.LLAMA8B_T32K_B16, synth.LLAMA8B_T32K_B16_FP8],
                         ids=["bf16", "e4m3"])
def test_noalloc_decode_matches_workspace_decode_two_steps(base):
    wl = synth.with_sizes(base, B=4, T=3000, top_k=32, steps=2)
    pb = synth.make_problem(wl, device="cuda")
    ref = DecodeLayer.from_problem(pb)  # basiskv_decode with its own workspace
    nal = DecodeLayer.from_problem(pb)  # same state, driven through the no-alloc entry
    assert bkv.workspace_size(ref.dims, wl.top_k, ref.max_seq_len) <= bkv.NOALLOC_SCRATCH_BYTES
    T = wl.T
    for step in range(2):
        k, v = synth.make_tokens(wl, pb.factors, 1, device="cuda", stream_id=50 + step)
        k, v = k[:, 0].contiguous(), v[:, 0].contiguous()
        q, _ = synth.make_query(wl, pb.cache["K"], T, step=step)
        sel_ref = torch.empty(wl.B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda")
        sel_nal = torch.full_like(sel_ref, -7)
        y_ref = ref.decode(q, k, v, sel=sel_ref, max_seq_len=T + 1).clone()
        y_nal = torch.empty_like(y_ref)
        bkv.basiskv_decode_noalloc(nal.dims, q, k, v, nal.seq_lens, T + 1, nal.block_table,
                                   nal.A_V, nal.P_K, nal.U_K, nal.W_fold, nal.K, nal.Z, nal.E,
                                   wl.top_k, sel_nal, y_nal)
        torch.cuda.synchronize()
        assert bkv.read_device_status() == 0
        ok, err, bound = _max_err_ok(y_nal, y_ref)
        assert ok, f"step {step}: max err {err:.3e} > {bound:.3e}"
        assert torch.equal(sel_nal, sel_ref)
        assert torch.equal(nal.seq_lens, ref.seq_lens)
        for name in ("K", "Z", "E"):  # byte views: the caches may hold E4M3
            assert torch.equal(getattr(nal, name).view(torch.uint8),
                               getattr(ref, name).view(torch.uint8)), name
        T += 1


def test_noalloc_rejects_oversized_problem():
    """A shape whose workspace exceeds the static array is refused before
    anything is launched."""
    d = bkv.Dims(B=64, Hq=32, Hkv=8, d=128, hidden=4096, r_v=96, r_k=32, page_size=16,
                 max_pages_per_seq=8200, num_phys_pages=64 * 8200)
    assert bkv.workspace_size(d, 2048, 8200 * 16) > bkv.NOALLOC_SCRATCH_BYTES
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    i = torch.zeros(64, dtype=torch.int32, device="cuda")
    with pytest.raises(bkv.BasisKVError) as e:
        bkv.basiskv_decode_noalloc(d, x, None, None, i, 8200 * 16, i, x, x, x, x, x, x, x, 2048,
                                   None, x)
    assert e.value.status == bkv.ERR_SCRATCH_LIMIT
