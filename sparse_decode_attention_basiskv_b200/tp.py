"""Tensor-parallel BasisKV attention layer (Figure 1 of the BasisKV pages).

Each rank holds Hkv / world KV heads of the layer (with their query heads),
runs the fused decode step up to those heads' Value latents
(``basiskv_decode_latents``), all-gathers every rank's latents into one
source-major buffer [world][B][Hq / world][r_v] (NCCL over NVLink when the
process group is NCCL), and rebuilds the complete output from all latents
with the full folded projection (``basiskv_outproj_sources``).  The latents
are what crosses the links: B * Hq * r_v bf16 per step instead of the dense
output's B * H.

Allocation and the collective are PyTorch's; every step of the compute is
the library's.
"""
from __future__ import annotations

import torch

from . import (Dims, basiskv_decode_latents, basiskv_fold_outproj, basiskv_outproj_sources,
               workspace_size)


def head_shard(Hq: int, Hkv: int, world: int, rank: int) -> tuple:
    """(g0, g1, h0, h1): the KV heads [g0, g1) and query heads [h0, h1) of a
    rank; the KV heads are split evenly, each keeps its G query heads."""
    if Hkv % world:
        raise ValueError(f"{Hkv} KV heads do not split over {world} ranks")
    n, G = Hkv // world, Hq // Hkv
    g0 = rank * n
    return g0, g0 + n, g0 * G, (g0 + n) * G


def local_dims(full: Dims, world: int) -> Dims:
    """A rank's dims: the layer's with Hq / world query and Hkv / world KV heads."""
    d = Dims()
    for name, _ in Dims._fields_:
        setattr(d, name, getattr(full, name))
    d.Hq, d.Hkv = full.Hq // world, full.Hkv // world
    return d


def shard_factors(factors: dict, Hq: int, Hkv: int, d: int, world: int, rank: int) -> dict:
    """A rank's factors: per-KV-head factors of its KV heads, W_O rows of its
    query heads."""
    g0, g1, h0, h1 = head_shard(Hq, Hkv, world, rank)
    out = {k: factors[k][g0:g1] for k in ("A_V", "P_K", "U_K", "B_V")}
    out["W_O"] = factors["W_O"][h0 * d:h1 * d]
    return out


class LatentGather:
    """All-gather of the ranks' latents into one source-major buffer: in
    place (each rank's latents already sit in its own slot)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group

    def __call__(self, a_src: torch.Tensor, rank: int) -> None:
        dist = self.dist
        if dist.get_backend(self.group) == "nccl":
            dist.all_gather_into_tensor(a_src, a_src[rank], group=self.group)
        else:
            dist.all_gather(list(a_src.unbind(0)), a_src[rank].clone(), group=self.group)


class CudaCompute:
    """The per-rank compute of a tensor-parallel step through the C-ABI."""

    @staticmethod
    def latents(layer, q, k_new, v_new, max_seq_len, sel, out, stream) -> None:
        basiskv_decode_latents(layer.dims, q, k_new, v_new, layer.seq_lens, max_seq_len,
                               layer.block_table, layer.A_V, layer.P_K, layer.U_K, layer.K,
                               layer.Z, layer.E, layer.top_k, sel, out, layer.workspace, stream)

    @staticmethod
    def outproj(layer, a_src, y, stream) -> None:
        basiskv_outproj_sources(layer.full, a_src, layer.world, layer.W_fold, y, layer.workspace,
                                stream)


class TPDecodeLayer:
    """One rank's share of a tensor-parallel BasisKV attention layer."""

    def __init__(self, full: Dims, world: int, rank: int, factors_local: dict, caches_local: dict,
                 block_table: torch.Tensor, seq_lens: torch.Tensor, top_k: int, max_seq_len: int,
                 W_fold: torch.Tensor, gather=None, compute=None, a_src=None):
        self.full, self.world, self.rank = full, world, rank
        self.dims = local_dims(full, world)
        self.top_k, self.max_seq_len = top_k, max_seq_len
        self.A_V, self.P_K, self.U_K = (factors_local[k] for k in ("A_V", "P_K", "U_K"))
        self.K, self.Z, self.E = caches_local["K"], caches_local["Z"], caches_local["E"]
        self.block_table, self.seq_lens = block_table, seq_lens
        self.W_fold = W_fold
        dev = self.K.device
        self.gather = gather
        self.compute = compute or CudaCompute()
        B, r_v = full.B, full.r_v
        self.a_src = (a_src if a_src is not None else
                      torch.empty(world, B, self.dims.Hq, r_v, dtype=torch.bfloat16, device=dev))
        self.y = torch.empty(B, full.hidden, dtype=torch.bfloat16, device=dev)
        n = 0
        if dev.type == "cuda":
            n = max(workspace_size(self.dims, top_k, max_seq_len),
                    workspace_size(full, top_k, max_seq_len))
            if n == 0:
                raise ValueError("unsupported dims for the BasisKV library")
        self.workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=dev)

    @classmethod
    def from_problem(cls, pb, world: int, rank: int, gather=None, compute=None, a_src=None,
                     device="cuda", W_fold=None) -> "TPDecodeLayer":
        """A rank's share of a synthetic workload (``synth.Problem``): its KV
        heads' caches and factors, the full folded projection."""
        from . import synth
        wl = pb.wl
        pc = wl.pages_capacity()
        full = Dims(B=wl.B, Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, hidden=wl.hidden, r_v=wl.r_v,
                    r_k=wl.r_k, page_size=wl.page_size, max_pages_per_seq=pc,
                    num_phys_pages=wl.B * pc, route_r_v=wl.route_r_v, route_r_k=wl.route_r_k,
                    sink_pages=wl.sink_pages, recent_pages=wl.recent_pages,
                    cache_fp8=wl.cache_fp8, route_page=wl.route_page)
        g0, g1, _, _ = head_shard(wl.Hq, wl.Hkv, world, rank)
        fl = {k: v.to(device).contiguous()
              for k, v in shard_factors(pb.factors, wl.Hq, wl.Hkv, wl.d, world, rank).items()}
        lead = wl.tile_lead()
        table = pb.table.to(device).contiguous()
        caches = {k: synth.storage(wl, synth.paginate(v[:, g0:g1].to(device), table,
                                                      wl.page_size, wl.B * pc,
                                                      lead.get(k, 0))).contiguous()
                  for k, v in pb.cache.items()}
        if W_fold is None and torch.device(device).type == "cuda":
            W_fold = torch.empty(wl.hidden, wl.Hq * wl.r_v, dtype=torch.bfloat16, device=device)
            basiskv_fold_outproj(full, pb.factors["B_V"].to(device).contiguous(),
                                 pb.factors["W_O"].to(device).contiguous(), W_fold)
        return cls(full, world, rank, fl, caches, table, pb.seq_lens.to(device).clone(),
                   wl.top_k, pc * wl.page_size, W_fold, gather, compute, a_src)

    def decode(self, q_local, k_new=None, v_new=None, sel=None, max_seq_len=None, y=None,
               stream=None) -> torch.Tensor:
        """One tensor-parallel decode step of this rank: its heads' latents,
        the AllGather, and the complete output y [B][H] (the same on every
        rank).  q_local [B][Hq/world][d]; k_new, v_new [B][Hkv/world][d]."""
        y = self.y if y is None else y
        msl = self.max_seq_len if max_seq_len is None else max_seq_len
        self.compute.latents(self, q_local, k_new, v_new, msl, sel, self.a_src[self.rank], stream)
        if self.gather is not None:
            self.gather(self.a_src, self.rank)
        self.compute.outproj(self, self.a_src, y, stream)
        return y
