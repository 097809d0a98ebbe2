"""BasisKV decode-attention block on NVIDIA B200 (sm_100a).

A thin ctypes binding over the C-ABI library ``libbasiskv.so`` built from
``csrc/`` (see ``include/basiskv.h`` for the contract of every call).  The
functions here only marshal arguments: every step of the decode path runs in
the library's CUDA kernels.  PyTorch supplies device memory and streams.

There is no CPU fallback: if the library has not been built, the first call
raises.
"""
from __future__ import annotations

import ctypes
import os
import re

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbasiskv.so")
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "basiskv.h")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED_SHAPE = -2
ERR_WORKSPACE_TOO_SMALL = -3
ERR_LAUNCH_FAILED = -4
ERR_DEVICE = -5
ERR_CUDA = -6
ERR_SCRATCH_LIMIT = -7
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024

DEV_BAD_PAGE = 0x1
DEV_OVERFLOW = 0x2
DEV_TIMEOUT = 0x4
DEV_BAD_LENGTH = 0x8


class Dims(ctypes.Structure):
    """Mirror of ``basiskv_dims``."""

    _fields_ = [(n, ctypes.c_int32) for n in (
        "B", "Hq", "Hkv", "d", "hidden", "r_v", "r_k", "page_size",
        "max_pages_per_seq", "num_phys_pages",
        "route_r_v", "route_r_k", "sink_pages", "recent_pages", "cache_fp8", "route_page")]

    @classmethod
    def of(cls, B, Hq, Hkv, d, hidden, r_v, r_k, page_size, max_pages_per_seq,
           num_phys_pages) -> "Dims":
        return cls(B, Hq, Hkv, d, hidden, r_v, r_k, page_size, max_pages_per_seq,
                   num_phys_pages)


class BasisKVError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {strerror(status)} (status {status})")
        self.status = status


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_DIMS = ctypes.POINTER(Dims)
_SIGNATURES = {
    "basiskv_workspace_size": (_SZ, [_DIMS, _I, _I]),
    "basiskv_fold_outproj": (_I, [_DIMS, _P, _P, _P, _P]),
    "basiskv_fold_append": (_I, [_DIMS, _P, _P, _P, _P, _P]),
    "basiskv_append": (_I, [_DIMS, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "basiskv_route": (_I, [_DIMS, _P, _P, _I, _P, _P, _P, _P, _P, _I, _P, _P, _P, _SZ, _P]),
    "basiskv_attend": (_I, [_DIMS, _P, _P, _I, _P, _P, _P, _P, _I, _P, _P, _SZ, _P]),
    "basiskv_outproj": (_I, [_DIMS, _P, _P, _P, _P, _SZ, _P]),
    "basiskv_decode": (_I, [_DIMS, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I,
                            _P, _P, _P, _SZ, _P]),
    "basiskv_decode_noalloc": (_I, [_DIMS, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P,
                                    _I, _P, _P, _P]),
    "basiskv_decode_latents": (_I, [_DIMS, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _I,
                                    _P, _P, _P, _SZ, _P]),
    "basiskv_outproj_sources": (_I, [_DIMS, _P, _I, _P, _P, _P, _SZ, _P]),
    "basiskv_read_device_status": (_I, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "basiskv_strerror": (ctypes.c_char_p, [_I]),
    "basiskv_launch_count": (ctypes.c_uint64, []),
    "basiskv_selftest_bounded_wait": (_I, [ctypes.c_uint64, _P]),
}

_lib = None


def header_symbols() -> list:
    """Names of the entry points declared in include/basiskv.h."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"BASISKV_API\s+[\w\s\*]*?\b(basiskv_\w+)\s*\(", text)))


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads the C-ABI library (once) and declares every signature."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(
                f"{path} is missing: build it with "
                "`python -m sparse_decode_attention_basiskv_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def strerror(status: int) -> str:
    return load_library().basiskv_strerror(status).decode()


def _ptr(t) -> int | None:
    """Device (or host) address of a tensor, None for None.  The library
    reads every array as dense row-major memory, so a strided view is
    refused rather than read in the wrong order."""
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError(f"tensor of shape {tuple(t.shape)} is not contiguous "
                         "(call .contiguous() first)")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != OK:
        raise BasisKVError(status, where)


def workspace_size(dims: Dims, top_k: int, max_seq_len: int) -> int:
    return load_library().basiskv_workspace_size(ctypes.byref(dims), top_k, max_seq_len)


def basiskv_fold_outproj(dims: Dims, B_V, W_O, W_fold, stream=None) -> None:
    _check(load_library().basiskv_fold_outproj(
        ctypes.byref(dims), _ptr(B_V), _ptr(W_O), _ptr(W_fold), _stream(stream)),
        "basiskv_fold_outproj")


def basiskv_fold_append(dims: Dims, A_V, P_K, U_K, W_app, stream=None) -> None:
    _check(load_library().basiskv_fold_append(
        ctypes.byref(dims), _ptr(A_V), _ptr(P_K), _ptr(U_K), _ptr(W_app), _stream(stream)),
        "basiskv_fold_append")


def basiskv_append(dims: Dims, k_new, v_new, n_new: int, seq_lens, block_table, A_V, P_K,
                   U_K, K_cache, Z_cache, E_cache, workspace, stream=None, W_app=None) -> None:
    _check(load_library().basiskv_append(
        ctypes.byref(dims), _ptr(k_new), _ptr(v_new), n_new, _ptr(seq_lens),
        _ptr(block_table), _ptr(A_V), _ptr(P_K), _ptr(U_K), _ptr(W_app), _ptr(K_cache),
        _ptr(Z_cache), _ptr(E_cache), _ptr(workspace), _nbytes(workspace), _stream(stream)),
        "basiskv_append")


def basiskv_route(dims: Dims, q, seq_lens, max_seq_len: int, block_table, P_K, U_K,
                  Z_cache, E_cache, top_k: int, page_scores, sel, workspace,
                  stream=None) -> None:
    _check(load_library().basiskv_route(
        ctypes.byref(dims), _ptr(q), _ptr(seq_lens), max_seq_len, _ptr(block_table),
        _ptr(P_K), _ptr(U_K), _ptr(Z_cache), _ptr(E_cache), top_k, _ptr(page_scores),
        _ptr(sel), _ptr(workspace), _nbytes(workspace), _stream(stream)), "basiskv_route")


def basiskv_attend(dims: Dims, q, seq_lens, max_seq_len: int, block_table, K_cache, Z_cache,
                   sel, top_k: int, a_lat, workspace, stream=None) -> None:
    _check(load_library().basiskv_attend(
        ctypes.byref(dims), _ptr(q), _ptr(seq_lens), max_seq_len, _ptr(block_table),
        _ptr(K_cache), _ptr(Z_cache), _ptr(sel), top_k, _ptr(a_lat), _ptr(workspace),
        _nbytes(workspace), _stream(stream)), "basiskv_attend")


def basiskv_outproj(dims: Dims, a_lat, W_fold, y, workspace, stream=None) -> None:
    _check(load_library().basiskv_outproj(
        ctypes.byref(dims), _ptr(a_lat), _ptr(W_fold), _ptr(y), _ptr(workspace),
        _nbytes(workspace), _stream(stream)), "basiskv_outproj")


def basiskv_decode(dims: Dims, q, k_new, v_new, seq_lens, max_seq_len: int, block_table, A_V,
                   P_K, U_K, W_fold, K_cache, Z_cache, E_cache, top_k: int, sel, y,
                   workspace, stream=None) -> None:
    _check(load_library().basiskv_decode(
        ctypes.byref(dims), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(seq_lens), max_seq_len,
        _ptr(block_table), _ptr(A_V), _ptr(P_K), _ptr(U_K), _ptr(W_fold), _ptr(K_cache),
        _ptr(Z_cache), _ptr(E_cache), top_k, _ptr(sel), _ptr(y), _ptr(workspace),
        _nbytes(workspace), _stream(stream)), "basiskv_decode")


def basiskv_decode_noalloc(dims: Dims, q, k_new, v_new, seq_lens, max_seq_len: int,
                           block_table, A_V, P_K, U_K, W_fold, K_cache, Z_cache, E_cache,
                           top_k: int, sel, y, stream=None) -> None:
    """basiskv_decode without a workspace, for callers that cannot allocate:
    the scratch is the library's static device array (see the header)."""
    _check(load_library().basiskv_decode_noalloc(
        ctypes.byref(dims), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(seq_lens), max_seq_len,
        _ptr(block_table), _ptr(A_V), _ptr(P_K), _ptr(U_K), _ptr(W_fold), _ptr(K_cache),
        _ptr(Z_cache), _ptr(E_cache), top_k, _ptr(sel), _ptr(y), _stream(stream)),
        "basiskv_decode_noalloc")


def basiskv_decode_latents(dims: Dims, q, k_new, v_new, seq_lens, max_seq_len: int, block_table,
                           A_V, P_K, U_K, K_cache, Z_cache, E_cache, top_k: int, sel, a_out,
                           workspace, stream=None) -> None:
    """The fused step up to the Value latents a_out (bf16 [B][Hq][r_v]) of
    the heads in dims: one GPU's share of a tensor-parallel layer."""
    _check(load_library().basiskv_decode_latents(
        ctypes.byref(dims), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(seq_lens), max_seq_len,
        _ptr(block_table), _ptr(A_V), _ptr(P_K), _ptr(U_K), _ptr(K_cache), _ptr(Z_cache),
        _ptr(E_cache), top_k, _ptr(sel), _ptr(a_out), _ptr(workspace), _nbytes(workspace),
        _stream(stream)), "basiskv_decode_latents")


def basiskv_outproj_sources(dims: Dims, a_src, n_src: int, W_fold, y, workspace,
                            stream=None) -> None:
    """y from the latents of n_src sources stored source-major
    ([n_src][B][Hq/n_src][r_v] bf16, as an AllGather leaves them)."""
    _check(load_library().basiskv_outproj_sources(
        ctypes.byref(dims), _ptr(a_src), n_src, _ptr(W_fold), _ptr(y), _ptr(workspace),
        _nbytes(workspace), _stream(stream)), "basiskv_outproj_sources")


def read_device_status(stream=None) -> int:
    """Waits for the stream; returns and clears the device status bits."""
    flags = ctypes.c_uint32(0)
    rc = load_library().basiskv_read_device_status(_stream(stream), ctypes.byref(flags))
    if rc not in (OK, ERR_DEVICE):
        raise BasisKVError(rc, "basiskv_read_device_status")
    return flags.value


def basiskv_selftest_bounded_wait(limit_ns: int, stream=None) -> None:
    """Launches the bounded-wait self-test (a wait that cannot complete,
    given up after limit_ns); read_device_status() then shows DEV_TIMEOUT."""
    _check(load_library().basiskv_selftest_bounded_wait(limit_ns, _stream(stream)),
           "basiskv_selftest_bounded_wait")


def launch_count() -> int:
    """Kernels the library has launched in this process so far."""
    return load_library().basiskv_launch_count()


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()
