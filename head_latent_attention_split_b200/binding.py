"""ctypes binding of libmla_decode.so (include/mla_decode.h).

Argument marshalling only: every step of the decode runs in the library's CUDA
kernels. torch is used for device memory and streams. There is no fallback: the
library is loaded on first use, and a missing or stale library raises then.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmla_decode.so")

F32, BF16, E4M3 = 0, 1, 2
KERNELS = {"auto": 0, "simt": 1, "tcgen05": 2, "tc_pair": 3}
KERNEL_NAMES = {v: k for k, v in KERNELS.items()}

MLA_OK = 0
STATUS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_ALIGNMENT",
          4: "MLA_ERR_WORKSPACE_TOO_SMALL", 5: "MLA_ERR_CUDA", 6: "MLA_ERR_BAD_BLOCK_ID",
          7: "MLA_ERR_BAD_SEQ_LEN", 8: "MLA_ERR_TIMEOUT"}

EXPORTED = ("mla_decode_workspace_size", "mla_decode_resolve", "mla_decode", "mla_decode_timed",
            "mla_decode_host_io_workspace_size", "mla_decode_host_io", "mla_plan_host", "mla_plan_probe",
            "mla_get_device_status", "mla_status_string", "mla_abi_version", "mla_decode_noalloc",
            "mla_decode_noalloc_max_workspace", "mla_cache_append", "mla_head_gemm", "mla_dsa_index",
            "mla_dsa_topk", "mla_sparse_decode", "mla_set_wait_timeout_ns", "mla_get_wait_timeout_ns")


class MlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class Params(ctypes.Structure):
    """mla_decode_params_t."""
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "q_len", "num_heads", "kv_rank", "rope_dim", "block_size", "num_blocks",
        "max_blocks_per_seq", "q_dtype", "cache_dtype", "out_dtype", "causal")] + [
        ("softmax_scale", ctypes.c_float), ("num_workers", ctypes.c_int32), ("kernel", ctypes.c_int32),
        ("reserved", ctypes.c_int32)]


class HeadGemmParams(ctypes.Structure):
    """mla_head_gemm_params_t."""
    _fields_ = [("rows", ctypes.c_int32), ("heads", ctypes.c_int32), ("k", ctypes.c_int32), ("n", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class AppendParams(ctypes.Structure):
    """mla_append_params_t."""
    _fields_ = [("batch", ctypes.c_int32), ("q_len", ctypes.c_int32), ("kv_rank", ctypes.c_int32),
                ("rope_dim", ctypes.c_int32), ("block_size", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
                ("max_blocks_per_seq", ctypes.c_int32), ("in_dtype", ctypes.c_int32),
                ("cache_dtype", ctypes.c_int32), ("rope", ctypes.c_int32), ("rope_base", ctypes.c_float),
                ("reserved", ctypes.c_int32)]


class DsaParams(ctypes.Structure):
    """mla_dsa_params_t."""
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "q_len", "index_heads", "index_dim", "block_size", "num_blocks", "max_blocks_per_seq",
        "max_seq_len", "top_k", "causal", "reserved")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built: run `python -m head_latent_attention_split_b200.build` "
                          "(the decode has no CPU or Python fallback)")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(Params)
    vp, i32p, sz = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.c_size_t
    L.mla_decode_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
    L.mla_decode_resolve.argtypes = [P, i32p, i32p]
    L.mla_decode.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.mla_decode_timed.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, ctypes.POINTER(vp)]
    L.mla_decode_host_io_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
    L.mla_decode_host_io.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.mla_decode_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.mla_decode_noalloc_max_workspace.argtypes = []
    L.mla_decode_noalloc_max_workspace.restype = ctypes.c_size_t
    L.mla_plan_host.argtypes = [P, vp, vp, vp, vp]
    L.mla_plan_probe.argtypes = [P, vp, vp, vp, vp, vp, vp]
    L.mla_get_device_status.argtypes = [vp, i32p]
    L.mla_status_string.argtypes = [ctypes.c_int32]
    L.mla_status_string.restype = ctypes.c_char_p
    L.mla_abi_version.argtypes = []
    L.mla_cache_append.argtypes = [ctypes.POINTER(AppendParams), vp, vp, vp, vp, vp, vp, vp, vp]
    L.mla_head_gemm.argtypes = [ctypes.POINTER(HeadGemmParams), vp, vp, vp, vp]
    D = ctypes.POINTER(DsaParams)
    L.mla_dsa_index.argtypes = [D, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.mla_dsa_topk.argtypes = [D, vp, vp, vp, vp, vp]
    L.mla_sparse_decode.argtypes = [P, ctypes.c_int32, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.mla_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    L.mla_get_wait_timeout_ns.argtypes = []
    for name in EXPORTED:
        if not hasattr(L, name):
            raise ImportError(f"{LIB_PATH} lacks {name}: rebuild it")
        f = getattr(L, name)
        if f.restype is ctypes.c_int and name != "mla_decode_noalloc_max_workspace":   # default
            f.restype = ctypes.c_int32
    L.mla_status_string.restype = ctypes.c_char_p
    L.mla_get_wait_timeout_ns.restype = ctypes.c_uint64
    return L


class _Lib:
    """Loads libmla_decode.so on first attribute access (so the package imports, and the
    build script runs, before the library exists)."""
    _handle = None

    def __getattr__(self, name):
        if _Lib._handle is None:
            _Lib._handle = _load()
        return getattr(_Lib._handle, name)


lib = _Lib()


def _check(st, where):
    if st != MLA_OK:
        raise MlaError(st, where)


def make_params(B, Sq, H, r, d_r, block_size, num_blocks, max_blocks_per_seq, q_dtype, cache_dtype,
                out_dtype, causal, softmax_scale, num_workers=0, kernel="auto") -> Params:
    return Params(batch=B, q_len=Sq, num_heads=H, kv_rank=r, rope_dim=d_r, block_size=block_size,
                  num_blocks=num_blocks, max_blocks_per_seq=max_blocks_per_seq, q_dtype=q_dtype,
                  cache_dtype=cache_dtype, out_dtype=out_dtype, causal=int(bool(causal)),
                  softmax_scale=float(softmax_scale), num_workers=int(num_workers),
                  kernel=KERNELS[kernel] if isinstance(kernel, str) else int(kernel), reserved=0)


def workspace_size(p: Params) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.mla_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)), "mla_decode_workspace_size")
    return n.value


def host_io_workspace_size(p: Params) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.mla_decode_host_io_workspace_size(ctypes.byref(p), ctypes.byref(n)),
           "mla_decode_host_io_workspace_size")
    return n.value


def resolve(p: Params):
    k, w = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib.mla_decode_resolve(ctypes.byref(p), ctypes.byref(k), ctypes.byref(w)), "mla_decode_resolve")
    return KERNEL_NAMES[k.value], w.value


def _addr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    raise TypeError(type(x))


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def mla_decode(p: Params, q_lat, q_rope, kv_cache, k_rope_cache, kv_scale, block_table, seq_lens, out, lse,
               workspace, workspace_bytes=None, stream=None, check=True) -> int:
    """Raw C-ABI call. Tensors are torch CUDA tensors (or integer device addresses)."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib.mla_decode(ctypes.byref(p), _addr(q_lat), _addr(q_rope), _addr(kv_cache), _addr(k_rope_cache),
                        _addr(kv_scale), _addr(block_table), _addr(seq_lens), _addr(out), _addr(lse),
                        _addr(workspace), workspace_bytes, _stream(stream))
    if check:
        _check(st, "mla_decode")
    return st


def mla_decode_timed(p: Params, q_lat, q_rope, kv_cache, k_rope_cache, kv_scale, block_table, seq_lens, out,
                     lse, workspace, events, stream=None) -> None:
    """mla_decode that records events[0..2] (torch.cuda.Event, already recorded once so
    that they exist) before the decode kernel, before the combine kernel and after it."""
    handles = (ctypes.c_void_p * 3)(*[e.cuda_event for e in events])
    st = lib.mla_decode_timed(ctypes.byref(p), _addr(q_lat), _addr(q_rope), _addr(kv_cache), _addr(k_rope_cache),
                              _addr(kv_scale), _addr(block_table), _addr(seq_lens), _addr(out), _addr(lse),
                              _addr(workspace), workspace.numel() * workspace.element_size(), _stream(stream),
                              handles)
    _check(st, "mla_decode_timed")


def mla_decode_host_io(p: Params, q_lat_host, q_rope_host, kv_cache, k_rope_cache, kv_scale, block_table_host,
                       seq_lens_host, out_host, lse_host, workspace, workspace_bytes=None, stream=None,
                       check=True) -> int:
    """C-ABI call with per-step tensors in (pinned) host memory; the cache is on the device."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    st = lib.mla_decode_host_io(ctypes.byref(p), _addr(q_lat_host), _addr(q_rope_host), _addr(kv_cache),
                                _addr(k_rope_cache), _addr(kv_scale), _addr(block_table_host),
                                _addr(seq_lens_host), _addr(out_host), _addr(lse_host), _addr(workspace),
                                workspace_bytes, _stream(stream))
    if check:
        _check(st, "mla_decode_host_io")
    return st


def mla_decode_noalloc(p: Params, q_lat, q_rope, kv_cache, k_rope_cache, kv_scale, block_table, seq_lens, out,
                       lse, stream=None, check=True) -> int:
    """C-ABI call that takes no workspace: the library's own device scratch array is used."""
    st = lib.mla_decode_noalloc(ctypes.byref(p), _addr(q_lat), _addr(q_rope), _addr(kv_cache), _addr(k_rope_cache),
                                _addr(kv_scale), _addr(block_table), _addr(seq_lens), _addr(out), _addr(lse),
                                _stream(stream))
    if check:
        _check(st, "mla_decode_noalloc")
    return st


def noalloc_max_workspace() -> int:
    return lib.mla_decode_noalloc_max_workspace()


def device_status(stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(lib.mla_get_device_status(_stream(stream), ctypes.byref(v)), "mla_get_device_status")
    return v.value


def plan_host(p: Params, seq_lens) -> dict:
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B = p.batch
    begin = np.zeros(B + 1, np.int32)
    first = np.zeros(B, np.int32)
    splits = np.zeros(B, np.int32)
    _check(lib.mla_plan_host(ctypes.byref(p), sl.ctypes.data, begin.ctypes.data, first.ctypes.data,
                             splits.ctypes.data), "mla_plan_host")
    return dict(block_begin=begin, first_worker=first, splits=splits)


def plan_probe(p: Params, block_table, seq_lens, stream=None):
    """Device plan walk: (token_slot, token_worker, seq_meta) torch int32 tensors."""
    import torch
    n = p.batch * p.max_blocks_per_seq * p.block_size
    dev = block_table.device
    slot = torch.full((n,), -1, dtype=torch.int32, device=dev)
    worker = torch.full((n,), -1, dtype=torch.int32, device=dev)
    meta = torch.full((p.batch, 2), -1, dtype=torch.int32, device=dev)
    _check(lib.mla_plan_probe(ctypes.byref(p), _addr(block_table), _addr(seq_lens), _addr(slot), _addr(worker),
                              _addr(meta), _stream(stream)), "mla_plan_probe")
    return slot.view(p.batch, -1), worker.view(p.batch, -1), meta


def set_wait_timeout_ns(ns: int) -> None:
    """Limit of the kernels' bounded pipeline waits, process-wide (0 restores the 2 s default)."""
    _check(lib.mla_set_wait_timeout_ns(int(ns)), "mla_set_wait_timeout_ns")


def wait_timeout_ns() -> int:
    return lib.mla_get_wait_timeout_ns()


def status_string(st: int) -> str:
    return lib.mla_status_string(st).decode()


def abi_version() -> int:
    return lib.mla_abi_version()


def make_append_params(B, Sq, r, d_r, block_size, num_blocks, max_blocks_per_seq, in_dtype, cache_dtype,
                       rope=False, rope_base=10000.0) -> AppendParams:
    return AppendParams(batch=B, q_len=Sq, kv_rank=r, rope_dim=d_r, block_size=block_size, num_blocks=num_blocks,
                        max_blocks_per_seq=max_blocks_per_seq, in_dtype=in_dtype, cache_dtype=cache_dtype,
                        rope=int(bool(rope)), rope_base=float(rope_base), reserved=0)


def mla_cache_append(p: AppendParams, c_new, k_rope_new, kv_cache, k_rope_cache, kv_scale, block_table, seq_lens,
                     stream=None, check=True) -> int:
    """Raw C-ABI call of the paged cache append (device tensors or integer addresses)."""
    st = lib.mla_cache_append(ctypes.byref(p), _addr(c_new), _addr(k_rope_new), _addr(kv_cache),
                              _addr(k_rope_cache), _addr(kv_scale), _addr(block_table), _addr(seq_lens),
                              _stream(stream))
    if check:
        _check(st, "mla_cache_append")
    return st


def mla_head_gemm(p: HeadGemmParams, x, w, y, stream=None, check=True) -> int:
    """Raw C-ABI call of the per-head GEMM y[m, h] = x[m, h] . w[h] (device tensors or addresses)."""
    st = lib.mla_head_gemm(ctypes.byref(p), _addr(x), _addr(w), _addr(y), _stream(stream))
    if check:
        _check(st, "mla_head_gemm")
    return st


def make_dsa_params(B, Sq, index_heads, index_dim, block_size, num_blocks, max_blocks_per_seq, max_seq_len, top_k,
                    causal=False) -> DsaParams:
    return DsaParams(batch=B, q_len=Sq, index_heads=index_heads, index_dim=index_dim, block_size=block_size,
                     num_blocks=num_blocks, max_blocks_per_seq=max_blocks_per_seq, max_seq_len=max_seq_len,
                     top_k=top_k, causal=int(bool(causal)), reserved=0)


def mla_dsa_index(p: DsaParams, q_codes, q_scale, weights, k_codes, k_scale, block_table, seq_lens, scores,
                  stream=None, check=True) -> int:
    """Raw C-ABI call of the lightning indexer (device tensors or integer addresses)."""
    st = lib.mla_dsa_index(ctypes.byref(p), _addr(q_codes), _addr(q_scale), _addr(weights), _addr(k_codes),
                           _addr(k_scale), _addr(block_table), _addr(seq_lens), _addr(scores), _stream(stream))
    if check:
        _check(st, "mla_dsa_index")
    return st


def mla_dsa_topk(p: DsaParams, scores, seq_lens, indices, counts, stream=None, check=True) -> int:
    """Raw C-ABI call of the top-k selection."""
    st = lib.mla_dsa_topk(ctypes.byref(p), _addr(scores), _addr(seq_lens), _addr(indices), _addr(counts),
                          _stream(stream))
    if check:
        _check(st, "mla_dsa_topk")
    return st


def mla_sparse_decode(p: Params, top_k: int, q_lat, q_rope, kv_cache, block_table, indices, counts, out, lse,
                      workspace, workspace_bytes=None, stream=None, check=True) -> int:
    """Raw C-ABI call of the decode over selected positions."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib.mla_sparse_decode(ctypes.byref(p), int(top_k), _addr(q_lat), _addr(q_rope), _addr(kv_cache),
                               _addr(block_table), _addr(indices), _addr(counts), _addr(out), _addr(lse),
                               _addr(workspace), workspace_bytes, _stream(stream))
    if check:
        _check(st, "mla_sparse_decode")
    return st
