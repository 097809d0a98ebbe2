"""Host-side checks of the C-ABI library (no GPU needed).

The library must load, export every entry point include/basiskv.h declares,
and reject invalid calls on the host, before any CUDA call, with the status
the header documents.  Only fake (aligned, never dereferenced) addresses are
passed, so nothing reaches a device.
"""
import ctypes
import subprocess

import pytest
import torch

import sparse_decode_attention_basiskv_b200 as bkv

FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def _dims(**kw):
    base = dict(B=2, Hq=8, Hkv=2, d=128, hidden=256, r_v=64, r_k=32, page_size=16,
                max_pages_per_seq=64, num_phys_pages=128)
    base.update(kw)
    return bkv.Dims(**base)


@pytest.fixture(scope="module")
def lib():
    return bkv.load_library()


def test_header_symbols_are_exported(lib):
    names = bkv.header_symbols()
    assert len(names) == 15
    out = subprocess.run(["nm", "-D", "--defined-only", bkv.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for n in names:
        assert n in exported, n
        assert getattr(lib, n)


def test_strerror_every_status(lib):
    for s in range(-7, 1):
        assert bkv.strerror(s) and "unknown" not in bkv.strerror(s)
    assert "unknown" in bkv.strerror(-99)


def test_workspace_size(lib):
    d = _dims()
    n = bkv.workspace_size(d, 8, 1000)
    assert n > 0 and n % 256 == 0
    assert bkv.workspace_size(d, 1, 1000) == 0           # top_k < 2
    assert bkv.workspace_size(d, 8, 64 * 16 + 1) == 0    # longer than a block-table row
    assert bkv.workspace_size(_dims(d=96), 8, 100) == 0  # unsupported head dim
    assert bkv.workspace_size(_dims(Hq=6), 8, 100) == 0  # G = 3
    assert bkv.workspace_size(d, 16, 1000) >= n


@pytest.mark.parametrize("field,value,status", [
    ("d", 80, bkv.ERR_UNSUPPORTED_SHAPE),
    ("r_v", 48, bkv.ERR_UNSUPPORTED_SHAPE),
    ("r_k", 8, bkv.ERR_UNSUPPORTED_SHAPE),
    ("page_size", 12, bkv.ERR_UNSUPPORTED_SHAPE),
    ("hidden", 200, bkv.ERR_UNSUPPORTED_SHAPE),
    ("Hq", 3, bkv.ERR_UNSUPPORTED_SHAPE),
    ("B", 0, bkv.ERR_INVALID_ARG),
    ("num_phys_pages", 0, bkv.ERR_INVALID_ARG),
])
def test_route_rejects_bad_dims(lib, field, value, status):
    d = _dims(**{field: value})
    rc = lib.basiskv_route(ctypes.byref(d), FAKE, FAKE, 100, FAKE, FAKE, FAKE, FAKE, FAKE, 8,
                           None, FAKE, FAKE, 1 << 30, None)
    assert rc == status


@pytest.mark.parametrize("field,value,status", [
    ("route_r_v", 8, bkv.ERR_INVALID_ARG),      # not a multiple of 16
    ("route_r_v", 80, bkv.ERR_INVALID_ARG),     # wider than r_v
    ("route_r_k", -16, bkv.ERR_INVALID_ARG),
    ("recent_pages", -1, bkv.ERR_INVALID_ARG),
])
def test_router_fields_validated(lib, field, value, status):
    d = _dims(**{field: value})
    rc = lib.basiskv_route(ctypes.byref(d), FAKE, FAKE, 100, FAKE, FAKE, FAKE, FAKE, FAKE, 8,
                           None, FAKE, FAKE, 1 << 30, None)
    assert rc == status


def test_narrow_router_shapes_and_budget(lib):
    # no instance of the scoring kernel for a narrow router at G = 1
    d = _dims(Hq=2, route_r_v=16)
    assert lib.basiskv_route(ctypes.byref(d), FAKE, FAKE, 100, FAKE, FAKE, FAKE, FAKE, FAKE, 8,
                             None, FAKE, FAKE, 1 << 30, None) == bkv.ERR_UNSUPPORTED_SHAPE
    # the forced pages must fit in top_k
    d = _dims(route_r_v=16, route_r_k=16, sink_pages=2, recent_pages=4)
    assert lib.basiskv_route(ctypes.byref(d), FAKE, FAKE, 100, FAKE, FAKE, FAKE, FAKE, FAKE, 5,
                             None, FAKE, FAKE, 1 << 30, None) == bkv.ERR_INVALID_ARG
    # a supported narrow router passes validation (then fails on the tiny workspace)
    d = _dims(route_r_v=16, route_r_k=16, sink_pages=-1, recent_pages=4)
    assert lib.basiskv_route(ctypes.byref(d), FAKE, FAKE, 100, FAKE, FAKE, FAKE, FAKE, FAKE, 8,
                             None, FAKE, FAKE, 64, None) == bkv.ERR_WORKSPACE_TOO_SMALL


def test_route_rejects_bad_args(lib):
    d = _dims()
    args = [ctypes.byref(d), FAKE, FAKE, 100, FAKE, FAKE, FAKE, FAKE, FAKE, 8, None, FAKE, FAKE,
            1 << 30, None]

    def call(i, v):
        a = list(args)
        a[i] = v
        return lib.basiskv_route(*a)

    assert call(1, None) == bkv.ERR_INVALID_ARG          # q null
    assert call(1, FAKE + 2) == bkv.ERR_INVALID_ARG      # q misaligned
    assert call(11, None) == bkv.ERR_INVALID_ARG         # sel and page scores both null
    assert call(11, FAKE + 2) == bkv.ERR_INVALID_ARG     # sel misaligned
    assert call(9, 1) == bkv.ERR_INVALID_ARG             # top_k < 2
    assert call(3, 0) == bkv.ERR_INVALID_ARG             # empty context bound
    assert call(3, 64 * 16 + 1) == bkv.ERR_INVALID_ARG   # past the block-table row
    assert call(12, FAKE + 16) == bkv.ERR_INVALID_ARG    # workspace not 256-aligned
    assert call(13, 64) == bkv.ERR_WORKSPACE_TOO_SMALL


def test_other_entry_points_validate(lib):
    d = _dims()
    big = 1 << 30
    assert lib.basiskv_attend(ctypes.byref(d), FAKE, FAKE, 100, FAKE, FAKE, FAKE, None, 8, FAKE,
                              FAKE, big, None) == bkv.ERR_INVALID_ARG
    assert lib.basiskv_outproj(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, 16,
                               None) == bkv.ERR_WORKSPACE_TOO_SMALL
    assert lib.basiskv_append(ctypes.byref(d), FAKE, FAKE, 0, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                              FAKE, FAKE, FAKE, FAKE, big, None) == bkv.ERR_INVALID_ARG
    assert lib.basiskv_append(ctypes.byref(d), FAKE, FAKE, 1, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                              FAKE, None, FAKE, FAKE, big, None) == bkv.ERR_INVALID_ARG
    # a chunk for the tensor-core path with a misaligned folded factor
    assert lib.basiskv_append(ctypes.byref(d), FAKE, FAKE, 64, FAKE, FAKE, FAKE, FAKE, FAKE,
                              FAKE + 2, FAKE, FAKE, FAKE, FAKE, big,
                              None) == bkv.ERR_INVALID_ARG
    assert lib.basiskv_fold_append(ctypes.byref(d), FAKE, None, FAKE, FAKE,
                                   None) == bkv.ERR_INVALID_ARG
    assert lib.basiskv_decode(ctypes.byref(d), FAKE, FAKE, None, FAKE, 100, FAKE, FAKE, FAKE,
                              FAKE, FAKE, FAKE, FAKE, FAKE, 8, None, FAKE, FAKE, big,
                              None) == bkv.ERR_INVALID_ARG  # k_new without v_new
    assert lib.basiskv_decode(ctypes.byref(d), FAKE, None, None, FAKE, 100, FAKE, FAKE, FAKE,
                              FAKE, FAKE, FAKE, FAKE, FAKE, 8, None, None, FAKE, big,
                              None) == bkv.ERR_INVALID_ARG  # y null
    assert lib.basiskv_fold_outproj(ctypes.byref(_dims(d=72)), FAKE, FAKE, FAKE,
                                    None) == bkv.ERR_UNSUPPORTED_SHAPE
    flags = ctypes.c_uint32(7)
    assert lib.basiskv_read_device_status(None, None) == bkv.ERR_INVALID_ARG


def test_e4m3_cache_validation(lib):
    """cache_fp8 is 0 or 1; E4M3 caches need an E4M3 router and attention
    instance (validated before any launch)."""
    assert bkv.workspace_size(_dims(cache_fp8=1), 8, 1000) > 0          # G 4, r_v 64, S 16
    assert bkv.workspace_size(_dims(cache_fp8=1, Hq=16, Hkv=2, page_size=32, r_v=96), 8,
                              1000) > 0                                  # G 8, S 32
    assert bkv.workspace_size(_dims(cache_fp8=1, route_r_v=16, route_r_k=16, sink_pages=-1,
                                    recent_pages=4), 8, 1000) > 0        # narrow router
    assert bkv.workspace_size(_dims(cache_fp8=2), 8, 1000) == 0          # not a type
    assert bkv.workspace_size(_dims(cache_fp8=-1), 8, 1000) == 0
    assert bkv.workspace_size(_dims(cache_fp8=1, Hq=2), 8, 1000) == 0   # G 1: no instance
    assert bkv.workspace_size(_dims(cache_fp8=1, page_size=8), 8, 1000) == 0
    assert bkv.workspace_size(_dims(cache_fp8=1, r_k=16), 8, 1000) == 0
    d = _dims(cache_fp8=1, Hq=2)
    assert lib.basiskv_route(ctypes.byref(d), FAKE, FAKE, 100, FAKE, FAKE, FAKE, FAKE, FAKE, 8,
                             None, FAKE, FAKE, 1 << 30, None) == bkv.ERR_UNSUPPORTED_SHAPE
    d = _dims(cache_fp8=3)
    assert lib.basiskv_decode(ctypes.byref(d), FAKE, None, None, FAKE, 100, FAKE, FAKE, FAKE,
                              FAKE, FAKE, FAKE, FAKE, FAKE, 8, None, FAKE, FAKE, 1 << 30,
                              None) == bkv.ERR_INVALID_ARG


def test_tensor_parallel_entry_points_validate(lib):
    big = 1 << 30
    d = _dims()
    # sources must divide the query heads
    assert lib.basiskv_outproj_sources(ctypes.byref(d), FAKE, 3, FAKE, FAKE, FAKE, big,
                                       None) == bkv.ERR_INVALID_ARG
    assert lib.basiskv_outproj_sources(ctypes.byref(d), FAKE, 0, FAKE, FAKE, FAKE, big,
                                       None) == bkv.ERR_INVALID_ARG
    # (Hq / n_src) * r_v = 1 * 32 is not a multiple of 64
    assert lib.basiskv_outproj_sources(ctypes.byref(_dims(r_v=32)), FAKE, 8, FAKE, FAKE, FAKE,
                                       big, None) == bkv.ERR_UNSUPPORTED_SHAPE
    assert lib.basiskv_outproj_sources(ctypes.byref(d), None, 2, FAKE, FAKE, FAKE, big,
                                       None) == bkv.ERR_INVALID_ARG
    assert lib.basiskv_outproj_sources(ctypes.byref(d), FAKE, 2, FAKE, FAKE, FAKE, 16,
                                       None) == bkv.ERR_WORKSPACE_TOO_SMALL
    # latents: output buffer required, k_new without v_new refused
    assert lib.basiskv_decode_latents(ctypes.byref(d), FAKE, None, None, FAKE, 100, FAKE, FAKE,
                                      FAKE, FAKE, FAKE, FAKE, FAKE, 8, None, None, FAKE, big,
                                      None) == bkv.ERR_INVALID_ARG
    assert lib.basiskv_decode_latents(ctypes.byref(d), FAKE, FAKE, None, FAKE, 100, FAKE, FAKE,
                                      FAKE, FAKE, FAKE, FAKE, FAKE, 8, None, FAKE, FAKE, big,
                                      None) == bkv.ERR_INVALID_ARG
    assert lib.basiskv_decode_latents(ctypes.byref(d), FAKE, None, None, FAKE, 100, FAKE, FAKE,
                                      FAKE, FAKE, FAKE, FAKE, FAKE, 8, None, FAKE, FAKE, 64,
                                      None) == bkv.ERR_WORKSPACE_TOO_SMALL


def test_head_shard_covers_every_head_once():
    from sparse_decode_attention_basiskv_b200.tp import head_shard, local_dims, shard_factors
    for Hq, Hkv, world in ((32, 8, 2), (32, 8, 4), (32, 8, 8), (64, 8, 8), (8, 2, 2)):
        hs, gs = [], []
        for r in range(world):
            g0, g1, h0, h1 = head_shard(Hq, Hkv, world, r)
            gs += range(g0, g1)
            hs += range(h0, h1)
            assert h0 == g0 * (Hq // Hkv) and h1 == g1 * (Hq // Hkv)
        assert gs == list(range(Hkv)) and hs == list(range(Hq))
    with pytest.raises(ValueError):
        head_shard(32, 8, 3, 0)
    ld = local_dims(_dims(), 2)
    assert (ld.Hq, ld.Hkv, ld.d, ld.r_v) == (4, 1, 128, 64)
    f = {"A_V": torch.arange(2)[:, None], "P_K": torch.arange(2)[:, None],
         "U_K": torch.arange(2)[:, None], "B_V": torch.arange(2)[:, None],
         "W_O": torch.arange(8 * 3)[:, None]}
    s1 = shard_factors(f, 8, 2, 3, 2, 1)
    assert s1["A_V"].tolist() == [[1]] and s1["W_O"][:, 0].tolist() == list(range(12, 24))


def test_selftest_wait_limit_validated(lib):
    """The bounded-wait self-test refuses a limit of 0 or above one second
    before any CUDA call."""
    for bad in (0, 1_000_000_001, 2**63):
        assert lib.basiskv_selftest_bounded_wait(bad, None) == bkv.ERR_INVALID_ARG


def _noalloc(lib, dims, top_k, max_seq_len):
    return lib.basiskv_decode_noalloc(ctypes.byref(dims), FAKE, FAKE, FAKE, FAKE, max_seq_len,
                                      FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, top_k,
                                      None, FAKE, None)


def test_noalloc_reports_the_validation_status(lib):
    """The no-allocation entry returns the same shape / argument status as
    basiskv_decode, and refuses workspaces above its static array, all
    before any CUDA call."""
    assert _noalloc(lib, _dims(d=100), 8, 256) == bkv.ERR_UNSUPPORTED_SHAPE
    assert _noalloc(lib, _dims(Hq=7), 8, 256) == bkv.ERR_UNSUPPORTED_SHAPE
    assert _noalloc(lib, _dims(), 1, 256) == bkv.ERR_INVALID_ARG  # top_k below sink + newest
    assert _noalloc(lib, _dims(), 8, 0) == bkv.ERR_INVALID_ARG
    assert _noalloc(lib, _dims(), 8, 64 * 16 + 1) == bkv.ERR_INVALID_ARG  # above the table
    big = _dims(B=256, Hq=32, Hkv=8, hidden=4096, max_pages_per_seq=25000,
                num_phys_pages=256 * 25000 // 8)
    assert lib.basiskv_workspace_size(ctypes.byref(big), 64, 400000) > bkv.NOALLOC_SCRATCH_BYTES
    assert _noalloc(lib, big, 64, 400000) == bkv.ERR_SCRATCH_LIMIT


def test_route_page_validation(lib):
    """Routing pages of 4 or 8 tokens (Table 10's Page4) over cache pages of
    16 or 32: accepted for routers with such an instance, bf16 or E4M3
    (Table 13's B16R16 Page4 over FP8 caches); other values and routers
    without an instance are refused; the standalone attention takes cache
    pages only."""
    nar = dict(Hq=8, Hkv=2, r_v=64, r_k=32, route_r_v=16, route_r_k=16, sink_pages=-1,
               recent_pages=4)
    ok = _dims(**nar, route_page=4)
    assert lib.basiskv_workspace_size(ctypes.byref(ok), 64, 1024) > 0
    assert lib.basiskv_workspace_size(ctypes.byref(_dims(**nar, route_page=8)), 64, 1024) > 0
    assert lib.basiskv_workspace_size(ctypes.byref(_dims(**nar, route_page=16)), 64, 1024) > 0
    # the scores hold one entry per routing page
    plain = lib.basiskv_workspace_size(ctypes.byref(_dims(**nar)), 64, 1024)
    assert lib.basiskv_workspace_size(ctypes.byref(ok), 64, 1024) > plain
    for bad, status in ((3, bkv.ERR_INVALID_ARG), (2, bkv.ERR_INVALID_ARG)):
        d = _dims(**nar, route_page=bad)
        assert lib.basiskv_route(ctypes.byref(d), FAKE, FAKE, 256, FAKE, FAKE, FAKE, FAKE, FAKE,
                                 64, None, FAKE, FAKE, 1 << 20, None) == status
    assert lib.basiskv_workspace_size(ctypes.byref(_dims(**nar, route_page=4, cache_fp8=1)),
                                      64, 1024) > 0
    for d in (_dims(**dict(nar, r_v=96), route_page=8, cache_fp8=1),  # no E4M3 instance
              _dims(route_page=4, r_v=32, r_k=16),      # no routing-page instance
              _dims(**nar, route_page=8, page_size=8)):  # not smaller than the page
        assert lib.basiskv_workspace_size(ctypes.byref(d), 64, 1024) == 0
    a = lib.basiskv_attend(ctypes.byref(ok), FAKE, FAKE, 1024, FAKE, FAKE, FAKE, FAKE, 64, FAKE,
                           FAKE, 1 << 20, None)
    assert a == bkv.ERR_UNSUPPORTED_SHAPE


def test_binding_refuses_strided_tensors():
    """The library reads every array as dense row-major memory: the binding
    refuses a strided view instead of passing its base address."""
    import torch
    strided = torch.zeros(4, 6)[:, ::2]
    with pytest.raises(ValueError, match="not contiguous"):
        bkv._ptr(strided)
    dense = torch.zeros(4, 6)
    assert bkv._ptr(dense) == dense.data_ptr() and bkv._ptr(None) is None
