"""Host logic of the tensor-parallel layer (Figure 1): two or four gloo ranks
on the CPU, each holding its share of the KV heads, compute their heads' latents, gather
them source-major and rebuild the complete output.  The per-rank compute is
the oracle standing in for the kernels (no GPU here), so the test checks the
head split, the factor and cache slicing, the gather order and the
source-major reassembly against the unsharded oracle."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp



def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload(world):
    from sparse_decode_attention_basiskv_b200 import synth
    return synth.with_sizes(synth.TINY, Hq=2 * world * 2, Hkv=2 * world, T=200, top_k=6,
                            n_planted=2)


class OracleCompute:
    """Stand-in for the kernels: the oracle on this rank's heads."""

    def __init__(self, pb, world, rank):
        from oracle import basiskv_oracle as O
        from sparse_decode_attention_basiskv_b200.tp import head_shard
        self.O, self.pb = O, pb
        wl = pb.wl
        self.g0, self.g1, self.h0, self.h1 = head_shard(wl.Hq, wl.Hkv, world, rank)
        f = {k: v.double().numpy() for k, v in pb.factors.items()}
        self.f = f
        self.W = O.fold_outproj(f["B_V"], f["W_O"], wl.Hq)  # all heads

    def latents(self, layer, q, k_new, v_new, max_seq_len, sel, out, stream):
        O, wl = self.O, self.pb.wl
        g0, g1 = self.g0, self.g1
        Wl = np.zeros((q.shape[1], wl.r_v, wl.hidden))
        for b in range(wl.B):
            c = {k: v[b, g0:g1].double().numpy() for k, v in self.pb.cache.items()}
            r = self.O.decode_sequence(q[b].double().numpy(), c["K"], c["Z"], c["E"], wl.T,
                                       wl.page_size, wl.top_k, self.f["P_K"][g0:g1],
                                       self.f["U_K"][g0:g1], Wl)
            out[b] = torch.from_numpy(r["a"]).bfloat16()

    def outproj(self, layer, a_src, y, stream):
        O, wl = self.O, self.pb.wl
        for b in range(wl.B):
            a = a_src[:, b].reshape(wl.Hq, wl.r_v).double().numpy()  # sources in head order
            y[b] = torch.from_numpy(O.outproj(a, self.W)).bfloat16()


def _rank(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from sparse_decode_attention_basiskv_b200 import synth
        from sparse_decode_attention_basiskv_b200.tp import LatentGather, TPDecodeLayer, head_shard
        wl = _workload(world)
        pb = synth.make_problem(wl)
        layer = TPDecodeLayer.from_problem(pb, world, rank, gather=LatentGather(),
                                           compute=OracleCompute(pb, world, rank), device="cpu")
        _, _, h0, h1 = head_shard(wl.Hq, wl.Hkv, world, rank)
        assert layer.dims.Hq == wl.Hq // world and layer.dims.Hkv == wl.Hkv // world
        assert layer.K.shape[1] == wl.Hkv // world and layer.A_V.shape[0] == wl.Hkv // world
        y = layer.decode(pb.q[:, h0:h1].contiguous())
        out[rank] = (y.float().numpy(), layer.a_src.float().numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_tensor_parallel_gloo_ranks(world):
    from oracle import basiskv_oracle as O
    from sparse_decode_attention_basiskv_b200 import synth
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    wl = _workload(world)
    pb = synth.make_problem(wl)
    f = {k: v.double().numpy() for k, v in pb.factors.items()}
    W = O.fold_outproj(f["B_V"], f["W_O"], wl.Hq)
    y0, a0 = out[0]
    for r in range(1, world):
        y1, a1 = out[r]
        np.testing.assert_array_equal(a0, a1)  # every rank holds every source's latents
        np.testing.assert_array_equal(y0, y1)  # and rebuilds the same output
    for b in range(wl.B):  # the unsharded step
        c = {k: v[b].double().numpy() for k, v in pb.cache.items()}
        r = O.decode_sequence(pb.q[b].double().numpy(), c["K"], c["Z"], c["E"], wl.T,
                              wl.page_size, wl.top_k, f["P_K"], f["U_K"], W)
        a_ref = r["a"].reshape(world, wl.Hq // world, wl.r_v)
        np.testing.assert_allclose(a0[:, b], a_ref, rtol=1e-2, atol=1e-2)  # bf16 latents
        ref = np.abs(r["y"]).max()
        assert np.abs(y0[b] - r["y"]).max() <= 1e-2 * ref + 1e-3
