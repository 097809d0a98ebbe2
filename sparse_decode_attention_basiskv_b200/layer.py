"""Device state of one BasisKV attention layer and its decode call.

Holds the paged caches, block table, lengths, factors, folded out-projection
and workspace of one layer on one GPU, and forwards each decode step to the
C-ABI (``basiskv_decode``).  Allocation is PyTorch's; all compute is the
library's.
"""
from __future__ import annotations

import torch

from . import (Dims, basiskv_append, basiskv_decode, basiskv_fold_append, basiskv_fold_outproj,
               workspace_size)


class DecodeLayer:
    def __init__(self, dims: Dims, factors: dict, caches: dict, block_table: torch.Tensor,
                 seq_lens: torch.Tensor, top_k: int, max_seq_len: int, stream=None):
        self.dims = dims
        self.top_k = top_k
        self.max_seq_len = max_seq_len
        self.A_V, self.P_K, self.U_K = factors["A_V"], factors["P_K"], factors["U_K"]
        self.K, self.Z, self.E = caches["K"], caches["Z"], caches["E"]
        self.block_table = block_table
        self.seq_lens = seq_lens
        dev = self.K.device
        self.W_fold = torch.empty(dims.hidden, dims.Hq * dims.r_v, dtype=torch.bfloat16,
                                  device=dev)
        basiskv_fold_outproj(dims, factors["B_V"], factors["W_O"], self.W_fold, stream)
        self.W_app = torch.empty(dims.Hkv, dims.r_v + dims.r_k, 2 * dims.d, dtype=torch.bfloat16,
                                 device=dev)
        basiskv_fold_append(dims, self.A_V, self.P_K, self.U_K, self.W_app, stream)
        n = workspace_size(dims, top_k, max_seq_len)
        if n == 0:
            raise ValueError("unsupported dims for the BasisKV library")
        self.workspace = torch.empty(n, dtype=torch.uint8, device=dev)
        self.y = torch.empty(dims.B, dims.hidden, dtype=torch.bfloat16, device=dev)

    @classmethod
    def from_problem(cls, pb, device="cuda", stream=None) -> "DecodeLayer":
        """Builds the layer of a synthetic workload (``synth.Problem``)."""
        return cls.from_parts(pb.wl, pb.factors, pb.paged(), pb.table, pb.seq_lens, device,
                              stream)

    @classmethod
    def from_parts(cls, wl, factors: dict, paged: dict, table, seq_lens=None, device="cuda",
                   stream=None) -> "DecodeLayer":
        """Builds the layer of workload ``wl`` from its factors, its paged
        caches (``synth.make_paged_cache`` or ``Problem.paged``) and block
        table; lengths default to wl.T for every sequence."""
        pc = wl.pages_capacity()
        dims = Dims(B=wl.B, Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, hidden=wl.hidden, r_v=wl.r_v,
                    r_k=wl.r_k, page_size=wl.page_size, max_pages_per_seq=pc,
                    num_phys_pages=wl.B * pc, route_r_v=wl.route_r_v, route_r_k=wl.route_r_k,
                    sink_pages=wl.sink_pages, recent_pages=wl.recent_pages,
                    cache_fp8=wl.cache_fp8, route_page=wl.route_page)
        factors = {k: v.to(device).contiguous() for k, v in factors.items()}
        caches = {k: v.contiguous() for k, v in paged.items()}
        if seq_lens is None:
            seq_lens = torch.full((wl.B,), wl.T, dtype=torch.int32)
        return cls(dims, factors, caches, table.to(device).contiguous(),
                   seq_lens.to(device).clone(), wl.top_k, pc * wl.page_size, stream)

    def append(self, k_new, v_new, n_new: int, stream=None) -> None:
        """Appends n_new tokens ([B][n_new][Hkv][d] bf16) to every sequence
        (a prefill chunk runs on the tensor cores with the folded factor)."""
        basiskv_append(self.dims, k_new, v_new, n_new, self.seq_lens, self.block_table, self.A_V,
                       self.P_K, self.U_K, self.K, self.Z, self.E, self.workspace, stream,
                       W_app=self.W_app)

    def capture(self, q, k_new=None, v_new=None, max_seq_len=None) -> "DecodeGraph":
        """Captures one decode step reading q (and k_new, v_new) as static
        buffers into a CUDA graph; replaying it runs the step again with
        whatever those buffers hold.  Run one eager step first (the library
        looks up its device state on its first call)."""
        msl = self.max_seq_len if max_seq_len is None else max_seq_len
        return DecodeGraph(lambda: self.decode(q, k_new, v_new, max_seq_len=msl))

    def decode(self, q, k_new=None, v_new=None, sel=None, max_seq_len=None, y=None,
               stream=None) -> torch.Tensor:
        """One decode step: optional append of (k_new, v_new), then routing,
        exact attention on the selected pages and the latent out-projection.
        Returns y [B][hidden] (bf16, on the device)."""
        y = self.y if y is None else y
        basiskv_decode(self.dims, q, k_new, v_new, self.seq_lens,
                       self.max_seq_len if max_seq_len is None else max_seq_len,
                       self.block_table, self.A_V, self.P_K, self.U_K, self.W_fold, self.K,
                       self.Z, self.E, self.top_k, sel, y, self.workspace, stream)
        return y


class DecodeGraph:
    """A CUDA graph of decode steps replayed without host launch overhead.

    The captured step reads its inputs from static device buffers (copy the
    step's q, k_new, v_new into them before each replay) and writes y into a
    static buffer; the sequence lengths live on the device and advance inside
    the step, so one graph serves every step while the lengths stay within
    the max_seq_len it was captured with."""

    def __init__(self, fn, warmup_stream=None):
        import torch
        s = torch.cuda.Stream() if warmup_stream is None else warmup_stream
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            self.graph.capture_begin()
            try:
                self.out = fn()
            finally:
                self.graph.capture_end()
        torch.cuda.current_stream().wait_stream(s)

    def replay(self):
        self.graph.replay()
        return self.out


class DecodeStack:
    """The attention blocks of a layer stack run in order on one stream, each
    layer with its own Value width (and so its own cache widths, factors and
    workspace): the per-layer Value ranks of Table 12 ("Avg. V rank")."""

    def __init__(self, layers: list):
        self.layers = layers

    @property
    def widths(self) -> list:
        return [L.dims.r_v for L in self.layers]

    def capture(self, qs, ks=None, vs=None, max_seq_len=None) -> DecodeGraph:
        """One CUDA graph of a decode step through every layer (static input
        buffers qs, ks, vs; see DecodeLayer.capture)."""
        return DecodeGraph(lambda: self.decode(qs, ks, vs, max_seq_len=max_seq_len))

    def decode(self, qs, ks=None, vs=None, max_seq_len=None, ys=None, stream=None) -> list:
        """One decode step of every layer: layer l gets qs[l] (and ks[l],
        vs[l] when appending).  Returns the layers' y (views of their output
        buffers unless ys is given)."""
        out = []
        for i, L in enumerate(self.layers):
            out.append(L.decode(qs[i], None if ks is None else ks[i],
                                None if vs is None else vs[i], max_seq_len=max_seq_len,
                                y=None if ys is None else ys[i], stream=stream))
        return out
