"""Tensor-parallel layer (Figure 1) on one GPU: the ranks' shares are built
side by side on the device and run one after another (no rank waits on
another); each writes its heads' latents into its slot of one source-major
buffer — what the AllGather leaves on every rank — and the out-projection
over all sources rebuilds the complete output, compared with the oracle's
unsharded step.  A one-rank NCCL group runs the in-place AllGather call."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

from oracle import basiskv_oracle as O
from sparse_decode_attention_basiskv_b200 import synth
from sparse_decode_attention_basiskv_b200.tp import LatentGather, TPDecodeLayer, head_shard

from harness import StepChecker, Y_ABS, Y_REL, assert_within, factors_np, np64, status_clean

pytestmark = pytest.mark.gpu

CASES = {
    "llama_tp2": (synth.with_sizes(synth.LLAMA8B_T32K_B16, B=4, T=1500, top_k=24), 2),
    "llama_tp4": (synth.with_sizes(synth.LLAMA8B_T32K_B16, B=4, T=1500, top_k=24), 4),
    "llama_v96_tp8": (synth.with_sizes(synth.LLAMA8B_T4K, B=2, T=1000, top_k=16), 8),
    "qwen_tp2": (synth.with_sizes(synth.QWEN32B_T64K_B8, B=2, T=1200, prefill_tokens=0,
                                  top_k=16), 2),
    "llama_tp2_e4m3": (synth.with_sizes(synth.LLAMA8B_T32K_B16_FP8, B=4, T=1500, top_k=24), 2),
    # the pages' narrow router (split tiles) across two ranks
    "llama_b16r16_tp2": (synth.with_sizes(synth.LLAMA8B_T32K_B16_B16R16, B=4, T=1500, top_k=24),
                         2),
}


@pytest.mark.parametrize("case", list(CASES))
def test_sharded_step_matches_unsharded_oracle(case):
    wl, world = CASES[case]
    pb = synth.make_problem(wl, device="cuda")
    f = factors_np(pb)
    Hq_l = wl.Hq // world
    a_src = torch.empty(world, wl.B, Hq_l, wl.r_v, dtype=torch.bfloat16, device="cuda")
    ranks = [TPDecodeLayer.from_problem(pb, world, r, a_src=a_src) for r in range(world)]
    k_new, v_new = synth.make_tokens(wl, pb.factors, 1, device="cuda")
    k_new, v_new = k_new[:, 0].contiguous(), v_new[:, 0].contiguous()
    sel = torch.empty(wl.B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda")
    for r, L in enumerate(ranks):
        g0, g1, h0, h1 = head_shard(wl.Hq, wl.Hkv, world, r)
        sel_r = torch.empty(wl.B, g1 - g0, wl.top_k, dtype=torch.int32, device="cuda")
        L.compute.latents(L, pb.q[:, h0:h1].contiguous(), k_new[:, g0:g1].contiguous(),
                          v_new[:, g0:g1].contiguous(), wl.T + 1, sel_r, a_src[r], None)
        sel[:, g0:g1] = sel_r
    y = torch.empty(wl.B, wl.hidden, dtype=torch.bfloat16, device="cuda")
    ranks[0].compute.outproj(ranks[0], a_src, y, None)
    status_clean()
    for L in ranks:
        assert L.seq_lens.tolist() == [wl.T + 1] * wl.B
    W = O.fold_outproj(f["B_V"], f["W_O"], wl.Hq)
    chk = StepChecker(wl, W, case)
    for b in range(wl.B):
        c = {k: np64(v[b]) for k, v in pb.cache.items()}
        out = O.decode_sequence(np64(pb.q[b]), c["K"], c["Z"], c["E"], wl.T, wl.page_size,
                                wl.top_k, f["P_K"], f["U_K"], W, k_new=np64(k_new[b]),
                                v_new=np64(v_new[b]), A_V=f["A_V"], fp8=bool(wl.cache_fp8),
                                **wl.router)
        gsel = sel[b].cpu().numpy()
        a_ref, y_ref = chk.expected(out, np64(pb.q[b]), gsel, chk.selection(b, out, gsel))
        a = np64(a_src[:, b].reshape(wl.Hq, wl.r_v))
        assert_within(a, a_ref, 1e-2, what=f"latents b{b}")  # one bf16 rounding
        assert_within(np64(y[b]), y_ref, Y_REL, Y_ABS, what=f"y b{b}")
    chk.report()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_nccl_group_runs_the_allgather():
    """world = 1 through an NCCL process group: latents, the in-place
    AllGather call, the out-projection; equal to the fused single-GPU step."""
    import torch.distributed as dist
    from sparse_decode_attention_basiskv_b200.layer import DecodeLayer
    wl = synth.with_sizes(synth.LLAMA8B_T32K_B16, B=4, T=1500, top_k=24)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        pb = synth.make_problem(wl, device="cuda")
        tp = TPDecodeLayer.from_problem(pb, 1, 0, gather=LatentGather())
        y_tp = tp.decode(pb.q, max_seq_len=wl.T).clone()
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref = DecodeLayer.from_problem(pb).decode(pb.q, max_seq_len=wl.T).clone()
    status_clean()
    # same latents (bf16) and projection; the K split of the two calls may
    # differ, so compare within the output tolerance
    assert_within(np64(y_tp), np64(ref), 1e-3, 1e-3, what="tp vs fused")
