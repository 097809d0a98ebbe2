"""Seeded synthetic workloads for the BasisKV decode-attention block.

This module only draws random numbers and lays data out; it contains none of
the method's own arithmetic (no append projection, no routing, no selection,
no attention, no out-projection).  Both the CUDA path (through the C-ABI) and
the CPU oracle receive the tensors produced here.

Input recipe (BasisKV, "Value Latents for Communication and Key Routing":
per-token state of Table 4; model shapes of Figure 3's caption):

* Factors, per KV head g, drawn on the CPU from ``torch.Generator(seed)`` in
  this order: A_V [d][r_v] ~ N(0, 1/d); P_K [r_v][d] ~ N(0, 1/r_v);
  U_K [d][r_k] = Q of a QR of an N(0,1) matrix (columns orthonormal, the sign
  of each column fixed so diag(R) > 0); B_V [r_v][d] ~ N(0, 1/r_v);
  W_O [Hq*d][hidden] ~ N(0, 1/(Hq*d)).  Every factor is rounded to bf16 once.
* Cache contents for tokens t < T of every (sequence b, KV head g), drawn
  per sequence with ``torch.Generator(device).manual_seed(seed*1000 + 1 +
  100003*layer + 7919*b)`` (so one sequence can be drawn alone): z ~ N(0,1),
  e ~ N(0,1) (both bf16), and the exact key
  K = z.P_K + e.U_K^T + N(0, 0.1^2), rounded to bf16.  This makes part of
  each key predictable from the Value latent, the structure BasisKV's router
  relies on.  Slots at t >= T hold a large finite filler so that a kernel
  that forgets the length mask is caught.
* Planted pages and queries (CPU generator seed*1000 + 2 for the choices):
  per (b, g) ``n_planted`` distinct pages from 1..P-2; each query head h of
  group g sums the keys of one uniform token in each of 2 distinct planted
  pages of its group, plus N(0, 0.1^2) noise.  Retrieval-style attention:
  the planted pages should win the routing.
* New tokens for decode step ``s`` (generator seed*1000 + 3 + s on the
  device): v ~ N(0,1); k = (v.A_V).P_K + e'.U_K^T + N(0, 0.1^2) with
  e' ~ N(0,1); both bf16.  The same recipe draws a prefill chunk.
* Paging: physical pages are a random permutation (CPU generator
  seed*1000 + 4) of ``B * pages_capacity`` slots, so every logical page is
  fetched through the block table from a scattered location.

The public benchmarks of the pages (RULER, LongBench, ...) need datasets and
trained checkpoints; these synthetic inputs stand in for them at the pages'
model shapes (Llama-3.1-8B and Qwen3-32B attention layers).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

FILLER = 64.0  # value stored in cache slots beyond a sequence's length


@dataclass(frozen=True)
class Workload:
    """Shape and seed of one synthetic decode-attention workload."""

    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    hidden: int
    T: int
    page_size: int
    r_v: int
    r_k: int
    top_k: int
    n_planted: int
    seed: int
    append_tokens: int = 0  # decode tokens appended per sequence per step
    prefill_tokens: int = 0  # tokens of one prefill chunk (sequence 0)
    layers: int = 1
    steps: int = 1
    # router and budget (0 = the defaults: full widths, sink page, newest page)
    route_r_v: int = 0
    route_r_k: int = 0
    sink_pages: int = 0
    recent_pages: int = 0
    cache_fp8: int = 0  # 1: the K, Z and E caches hold FP8 E4M3 values
    route_page: int = 0  # tokens per routing page (0 = page_size)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def sel_page(self) -> int:
        """Tokens per selected (routing) page: the oracle's page size."""
        return self.route_page or self.page_size

    @property
    def pages(self) -> int:
        return -(-self.T // self.page_size)

    def capacity_tokens(self) -> int:
        """Token slots per sequence: context, every token appended, and one
        page of slack (room for an extra decode token in any workload)."""
        return (self.T + self.append_tokens * self.steps + self.prefill_tokens
                + self.page_size)

    def pages_capacity(self) -> int:
        return -(-self.capacity_tokens() // self.page_size)

    @property
    def router(self) -> dict:
        """Effective router widths and forced pages."""
        return {"r_b": self.route_r_v or self.r_v, "r_q": self.route_r_k or self.r_k,
                "n_sink": 1 if self.sink_pages == 0 else max(self.sink_pages, 0),
                "n_recent": self.recent_pages or 1}

    def tile_lead(self) -> dict:
        """Columns stored first in each cache tile (a narrow router's)."""
        return {"Z": self.route_r_v or self.r_v, "E": self.route_r_k or self.r_k}

    def describe(self) -> dict:
        out = {k: getattr(self, k) for k in (
            "name", "B", "Hq", "Hkv", "d", "hidden", "T", "page_size", "r_v",
            "r_k", "top_k", "append_tokens", "prefill_tokens", "layers",
            "steps")}
        if (self.route_r_v, self.route_r_k, self.sink_pages, self.recent_pages) != (0, 0, 0, 0):
            out["router"] = self.router
        if self.route_page:
            out["route_page"] = self.route_page
        out["cache"] = "e4m3" if self.cache_fp8 else "bf16"
        return out


# The five workloads.  Names say what they are; sizes follow the pages' model
# shapes (Llama-3.1-8B: 32 query / 8 KV heads, d 128, hidden 4096; Qwen3-32B:
# 64 query / 8 KV heads, hidden 5120) and Value widths V96 / V64.
TINY = Workload("tiny_b1_t512", B=1, Hq=4, Hkv=1, d=64, hidden=256, T=512,
                page_size=16, r_v=32, r_k=16, top_k=8, n_planted=2, seed=0)
LLAMA8B_T4K = Workload("llama8b_layer_b1_t4k_v96", B=1, Hq=32, Hkv=8, d=128,
                       hidden=4096, T=4096, page_size=16, r_v=96, r_k=32,
                       top_k=64, n_planted=8, seed=1)
LLAMA8B_T32K_B16 = Workload("llama8b_layer_b16_t32k_v64_append1", B=16, Hq=32,
                            Hkv=8, d=128, hidden=4096, T=32768, page_size=16,
                            r_v=64, r_k=32, top_k=128, n_planted=8, seed=2,
                            append_tokens=1)
# The headline shape with the pages' narrow router and budget (Table 9's
# B16R16 router: 16 latent + 16 residual dimensions read per token; 2048
# routed tokens plus a 64-token recent window, no sink page), at page 16.
LLAMA8B_T32K_B16_B16R16 = replace(
    LLAMA8B_T32K_B16, name="llama8b_layer_b16_t32k_v64_router_b16r16_recent64", top_k=132,
    route_r_v=16, route_r_k=16, sink_pages=-1, recent_pages=4)
# The headline shape with FP8 E4M3 caches (Table 13's KV format).
LLAMA8B_T32K_B16_FP8 = replace(LLAMA8B_T32K_B16, name="llama8b_layer_b16_t32k_v64_append1_e4m3",
                               cache_fp8=1)
# The pages' adopted router configuration (Table 10's Page4; Table 9's
# budget of 2048 routed tokens plus a 64-token recent window; Table 13's
# B16R16): 4-token routing pages over the cache's 16-token pages, 512 routed
# pages + a 16-page recent window, no sink page.
LLAMA8B_T32K_B16_B16R16_PAGE4 = replace(
    LLAMA8B_T32K_B16, name="llama8b_layer_b16_t32k_v64_router_b16r16_page4_recent64",
    top_k=528, route_r_v=16, route_r_k=16, sink_pages=-1, recent_pages=16, route_page=4)
QWEN32B_T64K_B8 = Workload("qwen32b_layer_b8_t64k_v96_prefill4k", B=8, Hq=64,
                           Hkv=8, d=128, hidden=5120, T=65536, page_size=32,
                           r_v=96, r_k=32, top_k=64, n_planted=8, seed=3,
                           prefill_tokens=4096)


def sweep_point(B: int, T: int, r_v: int, layers: int = 32,
                steps: int = 128) -> Workload:
    """One point of the 32-layer decode sweep at the Llama-3.1-8B layer shape:
    top-k = T/64 pages of 16 tokens (a quarter of the context), one token
    appended per sequence per step."""
    return Workload(f"llama8b_sweep_b{B}_t{T // 1024}k_v{r_v}", B=B, Hq=32,
                    Hkv=8, d=128, hidden=4096, T=T, page_size=16, r_v=r_v,
                    r_k=32, top_k=T // 64, n_planted=8, seed=4,
                    append_tokens=1, layers=layers, steps=steps)


def v_rank_schedule(avg: int, layers: int = 32, seed: int = 0) -> list:
    """Per-layer Value widths with average `avg` over `layers` layers (Table
    12 reports an average V rank per model, the widths chosen per layer):
    half the layers at the average, a quarter 32 below, a quarter 32 above,
    in a seeded order.  avg in {64, 96}; layers a multiple of 4."""
    if avg not in (64, 96) or layers % 4:
        raise ValueError("schedules exist for avg 64 / 96 and layers % 4 == 0")
    q = layers // 4
    widths = [avg - 32] * q + [avg] * (2 * q) + [avg + 32] * q
    order = torch.randperm(layers, generator=torch.Generator().manual_seed(seed + 17))
    return [widths[i] for i in order.tolist()]


def stack_layers(wl: Workload, widths: list) -> list:
    """The per-layer workloads of a layer stack: wl with layer l's Value
    width (and its own seeds through the layer index of make_problem)."""
    return [replace(wl, name=f"{wl.name}_layer{l}_v{r}", r_v=r) for l, r in enumerate(widths)]


# The 32 attention layers of Llama-3.1-8B at the headline batch and context,
# Value widths varying per layer with average 64.
LLAMA8B_32L_T32K_B16_AVG64 = replace(LLAMA8B_T32K_B16, name="llama8b_32layers_b16_t32k_avg_v64_append1",
                                     layers=32)


SWEEP = [sweep_point(B, T, r_v) for B in (1, 8, 32, 64)
         for T in (4096, 32768, 131072) for r_v in (96, 64)]

WORKLOADS = {w.name: w for w in (TINY, LLAMA8B_T4K, LLAMA8B_T32K_B16,
                                  QWEN32B_T64K_B8)}


def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def make_factors(wl: Workload, layer: int = 0) -> dict:
    """Per-KV-head factors and W_O, drawn on the CPU (device independent)."""
    g = torch.Generator().manual_seed(wl.seed * 7919 + layer)
    Hkv, d, r_v, r_k = wl.Hkv, wl.d, wl.r_v, wl.r_k
    A_V = torch.randn(Hkv, d, r_v, generator=g, dtype=torch.float64) / math.sqrt(d)
    P_K = torch.randn(Hkv, r_v, d, generator=g, dtype=torch.float64) / math.sqrt(r_v)
    raw = torch.randn(Hkv, d, r_k, generator=g, dtype=torch.float64)
    U_K = torch.empty_like(raw)
    for h in range(Hkv):
        qm, rm = torch.linalg.qr(raw[h])
        U_K[h] = qm * torch.sign(torch.diagonal(rm)).unsqueeze(0)
    B_V = torch.randn(Hkv, r_v, d, generator=g, dtype=torch.float64) / math.sqrt(r_v)
    W_O = torch.randn(wl.Hq * d, wl.hidden, generator=g,
                      dtype=torch.float64) / math.sqrt(wl.Hq * d)
    return {"A_V": _bf16(A_V), "P_K": _bf16(P_K), "U_K": _bf16(U_K),
            "B_V": _bf16(B_V), "W_O": _bf16(W_O)}


def as_cache_values(wl: Workload, x: torch.Tensor) -> torch.Tensor:
    """The values a cache of this workload holds for x, as bf16: x rounded to
    bf16, or for E4M3 caches to E4M3 (nearest even, clamped to +-448), every
    E4M3 value being a bf16 value."""
    if not wl.cache_fp8:
        return x.bfloat16()
    return x.float().clamp(-448.0, 448.0).to(torch.float8_e4m3fn).to(torch.bfloat16)


def storage(wl: Workload, x: torch.Tensor) -> torch.Tensor:
    """A cache tensor of as_cache_values in the workload's element type (E4M3
    bytes or bf16)."""
    return x.to(torch.float8_e4m3fn) if wl.cache_fp8 else x


def _dev_gen(device, seed: int) -> torch.Generator:
    return torch.Generator(device=device).manual_seed(seed)


def _draw_sequence(wl: Workload, factors: dict, dev, layer: int, b: int) -> tuple:
    """Cache values (z, e, K) [Hkv][T][*] of sequence b, as the cache holds
    them (bf16 values, or E4M3 values for E4M3 caches)."""
    P_K = factors["P_K"].to(dev, torch.float32)
    U_K = factors["U_K"].to(dev, torch.float32)
    gen = _dev_gen(dev, wl.seed * 1000 + 1 + 100003 * layer + 7919 * b)
    z = torch.randn(wl.Hkv, wl.T, wl.r_v, generator=gen, device=dev).bfloat16()
    e = torch.randn(wl.Hkv, wl.T, wl.r_k, generator=gen, device=dev).bfloat16()
    noise = torch.randn(wl.Hkv, wl.T, wl.d, generator=gen, device=dev) * 0.1
    k = torch.bmm(z.float(), P_K) + torch.bmm(e.float(), U_K.transpose(1, 2)) + noise
    return as_cache_values(wl, z), as_cache_values(wl, e), as_cache_values(wl, k)


def make_cache(wl: Workload, factors: dict, device="cpu", layer: int = 0,
               seqs=None) -> dict:
    """Logical caches [len(seqs)][Hkv][capacity][*] holding T tokens for each
    sequence in ``seqs`` (default: all B)."""
    dev = torch.device(device)
    seqs = list(range(wl.B)) if seqs is None else list(seqs)
    Hkv, T, cap = wl.Hkv, wl.T, wl.capacity_tokens()
    n = len(seqs)
    Z = torch.full((n, Hkv, cap, wl.r_v), FILLER, dtype=torch.bfloat16, device=dev)
    E = torch.full((n, Hkv, cap, wl.r_k), FILLER, dtype=torch.bfloat16, device=dev)
    K = torch.full((n, Hkv, cap, wl.d), FILLER, dtype=torch.bfloat16, device=dev)
    for i, b in enumerate(seqs):  # one sequence at a time bounds the temporaries
        Z[i, :, :T], E[i, :, :T], K[i, :, :T] = _draw_sequence(wl, factors, dev, layer, b)
    return {"Z": Z, "E": E, "K": K}


def make_paged_cache(wl: Workload, factors: dict, table: torch.Tensor, device="cpu",
                     layer: int = 0) -> dict:
    """The paged caches of ``Problem.paged()`` (same values, same layout and
    element type) drawn one sequence at a time straight into the pages,
    without the logical copy: for workloads whose cache is tens of GB."""
    dev = torch.device(device)
    S, pc, T = wl.page_size, wl.pages_capacity(), wl.T
    n_phys = wl.B * pc
    lead = wl.tile_lead()
    widths = {"Z": wl.r_v, "E": wl.r_k, "K": wl.d}
    dt = torch.float8_e4m3fn if wl.cache_fp8 else torch.bfloat16
    out = {k: torch.full((n_phys, wl.Hkv, S, w), FILLER, dtype=torch.bfloat16,
                         device=dev).to(dt) for k, w in widths.items()}
    full = T // S  # whole pages; the partial last page keeps its filler rows
    for b in range(wl.B):
        vals = dict(zip(("Z", "E", "K"), _draw_sequence(wl, factors, dev, layer, b)))
        phys = table[b].long().to(dev)
        for name, x in vals.items():
            w = widths[name]
            if full:
                tiles = x[:, :full * S].reshape(wl.Hkv, full, S, w).permute(1, 0, 2, 3)
                out[name][phys[:full]] = storage(wl, split_tiles(tiles, lead.get(name, w)))
            if T % S:
                tail = torch.full((wl.Hkv, S, w), FILLER, dtype=torch.bfloat16, device=dev)
                tail[:, :T % S] = x[:, full * S:T]
                out[name][phys[full]] = storage(wl, split_tiles(tail, lead.get(name, w)))
    return out


class PagedKeys:
    """Logical indexing K[b, g, t] of a paged Key cache through the block
    table (what ``make_query`` reads when no logical cache exists)."""

    def __init__(self, K_paged: torch.Tensor, table: torch.Tensor, page_size: int):
        self.K, self.table, self.S = K_paged, table, page_size
        self.device = K_paged.device

    def __getitem__(self, idx) -> torch.Tensor:
        b, g, t = idx
        row = self.K[int(self.table[b, t // self.S]), g, t % self.S]
        return row.float() if row.dtype == torch.float8_e4m3fn else row


def planted_pages(wl: Workload, P: int | None = None) -> torch.Tensor:
    """[B][Hkv][n_planted] distinct pages drawn from 1..P-2 (CPU)."""
    P = wl.pages if P is None else P
    g = torch.Generator().manual_seed(wl.seed * 1000 + 2)
    n = min(wl.n_planted, max(P - 2, 0))
    out = torch.empty(wl.B, wl.Hkv, n, dtype=torch.int64)
    for b in range(wl.B):
        for h in range(wl.Hkv):
            out[b, h] = torch.randperm(P - 2, generator=g)[:n] + 1
    return out


def make_query(wl: Workload, K: torch.Tensor, T: int, step: int = 0) -> tuple:
    """Planted queries q [B][Hq][d] (bf16) built from cached keys.

    Returns (q, used) where used[b][h] lists the two planted pages that
    query head h drew from."""
    dev = K.device
    P = -(-T // wl.page_size)
    planted = planted_pages(wl, P)
    g = torch.Generator().manual_seed(wl.seed * 1000 + 2 + 7 * (step + 1))
    gen = _dev_gen(dev, wl.seed * 1000 + 5 + step)
    S = wl.page_size
    q = torch.empty(wl.B, wl.Hq, wl.d, dtype=torch.float32, device=dev)
    used = torch.zeros(wl.B, wl.Hq, 2, dtype=torch.int64)
    for b in range(wl.B):
        for h in range(wl.Hq):
            grp = h // wl.G
            cand = planted[b, grp]
            if len(cand) >= 2:
                pick = cand[torch.randperm(len(cand), generator=g)[:2]]
            else:  # too few pages to plant: any two tokens of the context
                pick = torch.tensor([0, P - 1])
            acc = torch.zeros(wl.d, dtype=torch.float32, device=dev)
            for j, p in enumerate(pick.tolist()):
                lo, hi = p * S, min((p + 1) * S, T)
                t = lo + int(torch.randint(hi - lo, (1,), generator=g))
                acc += K[b, grp, t].float()
                used[b, h, j] = p
            q[b, h] = acc
    q += torch.randn(q.shape, generator=gen, device=dev) * 0.1
    return q.bfloat16(), used


def make_tokens(wl: Workload, factors: dict, n: int, device="cpu",
                stream_id: int = 0) -> tuple:
    """n new tokens per sequence: (k, v) each [B][n][Hkv][d] bf16."""
    dev = torch.device(device)
    gen = _dev_gen(dev, wl.seed * 1000 + 3 + stream_id)
    A_V = factors["A_V"].to(dev, torch.float32)
    P_K = factors["P_K"].to(dev, torch.float32)
    U_K = factors["U_K"].to(dev, torch.float32)
    B, Hkv, d = wl.B, wl.Hkv, wl.d
    v = torch.randn(B, n, Hkv, d, generator=gen, device=dev).bfloat16()
    ep = torch.randn(B, n, Hkv, wl.r_k, generator=gen, device=dev)
    noise = torch.randn(B, n, Hkv, d, generator=gen, device=dev) * 0.1
    lat = torch.einsum("bnhd,hdr->bnhr", v.float(), A_V)
    k = (torch.einsum("bnhr,hrd->bnhd", lat, P_K)
         + torch.einsum("bnhr,hdr->bnhd", ep, U_K) + noise)
    return k.bfloat16().contiguous(), v


def block_table(wl: Workload, device="cpu") -> torch.Tensor:
    """[B][pages_capacity] int32 logical->physical page map (a permutation)."""
    pc = wl.pages_capacity()
    g = torch.Generator().manual_seed(wl.seed * 1000 + 4)
    perm = torch.randperm(wl.B * pc, generator=g).to(torch.int32)
    return perm.view(wl.B, pc).to(device)


def split_tiles(tiles: torch.Tensor, lead: int) -> torch.Tensor:
    """Tiles [..., S, r] stored with their first `lead` columns first: the
    memory of each tile holds [S][lead] then [S][r - lead] (the layout the
    C-ABI uses for a narrow router's columns).  lead == r: unchanged."""
    S, r = tiles.shape[-2:]
    if lead == r:
        return tiles
    flat = torch.cat([tiles[..., :lead].reshape(*tiles.shape[:-2], S * lead),
                      tiles[..., lead:].reshape(*tiles.shape[:-2], S * (r - lead))], -1)
    return flat.reshape(tiles.shape)


def unsplit_tiles(tiles: torch.Tensor, lead: int) -> torch.Tensor:
    """Inverse of split_tiles."""
    S, r = tiles.shape[-2:]
    if lead == r:
        return tiles
    flat = tiles.reshape(*tiles.shape[:-2], S * r)
    a = flat[..., :S * lead].reshape(*tiles.shape[:-2], S, lead)
    b = flat[..., S * lead:].reshape(*tiles.shape[:-2], S, r - lead)
    return torch.cat([a, b], -1)


def paginate(logical: torch.Tensor, table: torch.Tensor, page_size: int,
             num_phys: int, lead: int = 0) -> torch.Tensor:
    """Scatter a logical cache [B][Hkv][cap][r] into the paged layout
    [num_phys][Hkv][page_size][r] through the block table (each tile with
    its first `lead` columns first when 0 < lead < r)."""
    B, Hkv, cap, r = logical.shape
    pc = table.shape[1]
    pad = pc * page_size - cap
    if pad:
        logical = torch.cat([logical, torch.full((B, Hkv, pad, r), FILLER,
                            dtype=logical.dtype, device=logical.device)], 2)
    tiles = logical.view(B, Hkv, pc, page_size, r).permute(0, 2, 1, 3, 4)
    tiles = split_tiles(tiles, lead or r)
    out = torch.full((num_phys, Hkv, page_size, r), FILLER, dtype=logical.dtype,
                     device=logical.device)
    out[table.long().reshape(-1).to(logical.device)] = tiles.reshape(B * pc, Hkv, page_size, r)
    return out


def logical_view(paged: torch.Tensor, table: torch.Tensor, b: int, g: int,
                 n_tokens: int) -> torch.Tensor:
    """Gather tokens [0, n_tokens) of (sequence b, KV head g) from a paged
    cache, in logical order (used to hand the CUDA path's outputs to a
    comparison)."""
    S = paged.shape[2]
    n_pages = -(-n_tokens // S)
    phys = table[b, :n_pages].long().to(paged.device)
    return paged[phys, g].reshape(n_pages * S, -1)[:n_tokens]


@dataclass
class Problem:
    """Everything one decode-attention workload needs, on one device."""

    wl: Workload
    factors: dict
    cache: dict
    table: torch.Tensor
    seq_lens: torch.Tensor
    q: torch.Tensor
    used_pages: torch.Tensor
    extra: dict = field(default_factory=dict)

    def paged(self) -> dict:
        n = self.wl.B * self.wl.pages_capacity()
        lead = self.wl.tile_lead()
        return {k: storage(self.wl, paginate(v, self.table.to(v.device), self.wl.page_size, n,
                                             lead.get(k, 0)))
                for k, v in self.cache.items()}


def make_problem(wl: Workload, device="cpu", layer: int = 0) -> Problem:
    factors = make_factors(wl, layer)
    cache = make_cache(wl, factors, device, layer)
    table = block_table(wl, device)
    seq_lens = torch.full((wl.B,), wl.T, dtype=torch.int32, device=device)
    q, used = make_query(wl, cache["K"], wl.T)
    return Problem(wl, factors, cache, table, seq_lens, q, used)


def with_sizes(wl: Workload, **kw) -> Workload:
    """A copy of a workload with some sizes changed (ragged / edge cases)."""
    return replace(wl, **kw)
