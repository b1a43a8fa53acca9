"""fp64 CPU oracle for absorbed MLA decode -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package. The product path (``head_latent_attention_split_b200``) never
does, and the two share no code: the oracle is ``mla_oracle.c`` (plain C, fp64,
OpenMP over heads) plus the small ctypes wrapper below.

What it computes is stated in ``mla_oracle.c``: the absorbed MLA decode score of
"TransMLA: Multi-Head Latent Attention Is All You Need" (sec. 3.4.5) with the
decoupled RoPE term of the TPLA page (sec. 3.4, "The RoPE handling"), a two-pass
fp64 softmax, and the latent itself as the value.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(worked examples of the "TransMLA & Sparse Latent Attention" lesson, the
absorbed == explicit identity, GQA == GQA-as-MLA, closed forms, a 50-digit mpmath
brute force, and library decoders for bf16 / e4m3).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_LIB = os.path.join(_HERE, "libmla_oracle.so")

F32, BF16, E4M3, F64 = 0, 1, 2, 3

ERRORS = {0: "ok", 1: "invalid argument", 2: "block id out of range", 3: "seq_len out of range",
          4: "out of memory"}


class Problem(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("Sq", ctypes.c_int32), ("H", ctypes.c_int32),
        ("r", ctypes.c_int32), ("d_r", ctypes.c_int32),
        ("block_size", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32),
        ("q_dtype", ctypes.c_int32), ("cache_dtype", ctypes.c_int32),
        ("causal", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("softmax_scale", ctypes.c_double),
        ("q_lat", ctypes.c_void_p), ("q_rope", ctypes.c_void_p), ("kv_cache", ctypes.c_void_p),
        ("k_rope_cache", ctypes.c_void_p), ("kv_scale", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
    ]


def build(force: bool = False) -> str:
    """Compile mla_oracle.c into libmla_oracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.POINTER(Problem)
        dp = ctypes.POINTER(ctypes.c_double)
        L.mla_oracle_decode.argtypes = [P, dp, dp, ctypes.c_int]
        L.mla_oracle_decode_window.argtypes = [P, ctypes.c_void_p, ctypes.c_void_p, dp, dp, ctypes.c_int]
        L.mla_oracle_decode_rows.argtypes = [P, ctypes.c_int, ctypes.c_void_p, dp, dp, ctypes.c_int]
        L.mla_oracle_merge.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, dp, dp, dp, dp]
        L.mla_oracle_merge.restype = None
        L.mla_oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.mla_oracle_bf16_to_double.restype = ctypes.c_double
        L.mla_oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        L.mla_oracle_e4m3_to_double.restype = ctypes.c_double
        L.mla_oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.mla_oracle_e4m3_encode.restype = ctypes.c_uint8
        L.mla_oracle_e4m3_encode_n.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64]
        L.mla_oracle_e4m3_encode_n.restype = None
        L.mla_oracle_cache_append.argtypes = [ctypes.c_int] * 10 + [ctypes.c_double] + [ctypes.c_void_p] * 7
        L.mla_oracle_cache_append.restype = ctypes.c_int
        L.mla_oracle_head_gemm.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                                                 ctypes.c_void_p]
        L.mla_oracle_head_gemm.restype = None
        L.mla_oracle_dsa_index.argtypes = [ctypes.c_int] * 9 + [ctypes.c_void_p] * 8 + [ctypes.c_int]
        L.mla_oracle_dsa_index.restype = ctypes.c_int
        L.mla_oracle_decode_sparse.argtypes = [P, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, dp, dp,
                                               ctypes.c_int]
        L.mla_oracle_decode_sparse.restype = ctypes.c_int
        _lib = L
    return _lib


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float64:
        return F64
    if a.dtype == np.uint8:
        return E4M3
    raise TypeError(f"unsupported oracle input dtype {a.dtype}")


def _ptr(a):
    return None if a is None else a.ctypes.data


class _Bound:
    """Keeps the numpy inputs alive while the C problem struct points at them."""

    def __init__(self, q_lat, q_rope, kv_cache, block_table, seq_lens, softmax_scale, causal,
                 k_rope_cache=None, kv_scale=None, block_size=64):
        self.arrays = [np.ascontiguousarray(x) if x is not None else None
                       for x in (q_lat, q_rope, kv_cache, k_rope_cache, kv_scale, block_table, seq_lens)]
        q_lat, q_rope, kv_cache, k_rope_cache, kv_scale, block_table, seq_lens = self.arrays
        block_table = block_table.astype(np.int32, copy=False)
        seq_lens = seq_lens.astype(np.int32, copy=False)
        self.arrays[5], self.arrays[6] = block_table, seq_lens
        B, Sq, H, r = q_lat.shape
        d_r = q_rope.shape[-1]
        cd = _dtype_code(kv_cache)
        if cd == E4M3:
            assert kv_scale is not None and kv_scale.dtype == np.float32
            assert d_r == 0 or (k_rope_cache is not None and k_rope_cache.dtype == np.uint16)
        qd = _dtype_code(q_lat)
        assert _dtype_code(q_rope) == qd or q_rope.size == 0
        self.shape = (B, Sq, H, r, d_r)
        self.p = Problem(B=B, Sq=Sq, H=H, r=r, d_r=d_r, block_size=block_size,
                         num_blocks=kv_cache.shape[0], max_blocks_per_seq=block_table.shape[1],
                         q_dtype=qd, cache_dtype=cd, causal=int(bool(causal)), reserved=0,
                         softmax_scale=float(softmax_scale),
                         q_lat=_ptr(q_lat), q_rope=_ptr(q_rope), kv_cache=_ptr(kv_cache),
                         k_rope_cache=_ptr(k_rope_cache), kv_scale=_ptr(kv_scale),
                         block_table=_ptr(block_table), seq_lens=_ptr(seq_lens))


def _check(rc):
    if rc != 0:
        raise RuntimeError(f"oracle error {rc}: {ERRORS.get(rc, '?')}")


def _dp(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def decode(q_lat, q_rope, kv_cache, block_table, seq_lens, softmax_scale, causal=False,
           k_rope_cache=None, kv_scale=None, block_size=64, tok_begin=None, tok_end=None,
           nthreads=0):
    """Absorbed MLA decode in fp64. Returns (out [B,Sq,H,r] f64, lse [B,Sq,H] f64).

    Inputs are numpy arrays in their storage format: float32 / float64, uint16 bf16
    patterns, or uint8 e4m3 codes (cache only, with k_rope_cache bf16 + kv_scale f32).
    tok_begin / tok_end (int64 [B]) restrict each sequence to a token window.
    """
    bd = _Bound(q_lat, q_rope, kv_cache, block_table, seq_lens, softmax_scale, causal,
                k_rope_cache, kv_scale, block_size)
    B, Sq, H, r, _ = bd.shape
    out = np.zeros((B, Sq, H, r), dtype=np.float64)
    lse = np.zeros((B, Sq, H), dtype=np.float64)
    if tok_begin is None and tok_end is None:
        rc = lib().mla_oracle_decode(ctypes.byref(bd.p), _dp(out), _dp(lse), nthreads)
    else:
        tb = np.ascontiguousarray(tok_begin, dtype=np.int64) if tok_begin is not None else None
        te = np.ascontiguousarray(tok_end, dtype=np.int64) if tok_end is not None else None
        rc = lib().mla_oracle_decode_window(ctypes.byref(bd.p), _ptr(tb), _ptr(te), _dp(out),
                                            _dp(lse), nthreads)
    _check(rc)
    return out, lse


def decode_rows(rows, q_lat, q_rope, kv_cache, block_table, seq_lens, softmax_scale, causal=False,
                k_rope_cache=None, kv_scale=None, block_size=64, nthreads=0):
    """fp64 decode of selected (b, s, h) rows only. Returns (out [n, r], lse [n])."""
    bd = _Bound(q_lat, q_rope, kv_cache, block_table, seq_lens, softmax_scale, causal,
                k_rope_cache, kv_scale, block_size)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
    n = rows.shape[0]
    r = bd.shape[3]
    out = np.zeros((n, r), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    _check(lib().mla_oracle_decode_rows(ctypes.byref(bd.p), n, rows.ctypes.data, _dp(out), _dp(lse),
                                        nthreads))
    return out, lse


def merge(o_parts, lse_parts):
    """Log-sum-exp merge of partials over disjoint token windows.

    o_parts [P, ..., r], lse_parts [P, ...] -> (out [..., r], lse [...]).
    """
    o_parts = np.ascontiguousarray(o_parts, dtype=np.float64)
    lse_parts = np.ascontiguousarray(lse_parts, dtype=np.float64)
    P = o_parts.shape[0]
    r = o_parts.shape[-1]
    rest = lse_parts.shape[1:]
    n_rows = int(np.prod(rest)) if rest else 1
    out = np.zeros(rest + (r,), dtype=np.float64)
    lse = np.zeros(rest, dtype=np.float64)
    lib().mla_oracle_merge(P, n_rows, r, _dp(o_parts), _dp(lse_parts), _dp(out), _dp(lse))
    return out, lse


def bf16_to_double(bits: int) -> float:
    return lib().mla_oracle_bf16_to_double(int(bits))


def e4m3_to_double(code: int) -> float:
    return lib().mla_oracle_e4m3_to_double(int(code))


def decode_inputs(inp: dict, nthreads=0, **kw):
    """Convenience: run ``decode`` on a dict produced by ``workloads.make_inputs``."""
    w = inp["workload"]
    return decode(inp["q_lat"], inp["q_rope"], inp["kv_cache"], inp["block_table"], inp["seq_lens"],
                  w.scale, w.causal, inp.get("k_rope_cache"), inp.get("kv_scale"), w.block_size,
                  nthreads=nthreads, **kw)


def decode_rows_inputs(inp: dict, rows, nthreads=0):
    w = inp["workload"]
    return decode_rows(rows, inp["q_lat"], inp["q_rope"], inp["kv_cache"], inp["block_table"],
                       inp["seq_lens"], w.scale, w.causal, inp.get("k_rope_cache"),
                       inp.get("kv_scale"), w.block_size, nthreads=nthreads)


def e4m3_encode(x) -> np.ndarray:
    """fp32 values -> OCP e4m3 codes (nearest, ties to even, saturated to +-448)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    codes = np.empty(x.shape, dtype=np.uint8)
    lib().mla_oracle_e4m3_encode_n(x.ctypes.data, codes.ctypes.data, x.size)
    return codes


def cache_append(*, B, Sq, r, d_r, block_size, num_blocks, max_blocks_per_seq, in_dtype, cache_dtype,
                 c_new, k_new, kv_cache, block_table, seq_lens, k_rope_cache=None, kv_scale=None,
                 rope=False, rope_base=10000.0) -> int:
    """Write the new tokens into the paged cache arrays in place (see mla_oracle.c).

    c_new / k_new: [B, Sq, r] / [B, Sq, d_r] as float32 (in_dtype F32) or bf16 bit
    patterns in uint16 (BF16). kv_cache: float32 / uint16 [num_blocks, bs, r + d_r], or
    uint8 codes [num_blocks, bs, r] with k_rope_cache uint16 [num_blocks, bs, d_r] and
    kv_scale float32 [num_blocks, bs] for E4M3. Returns the oracle status (0 = ok).
    """
    c_new = np.ascontiguousarray(c_new)
    k_new = np.ascontiguousarray(k_new)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    for a in (kv_cache, k_rope_cache, kv_scale):
        if a is not None:
            assert a.flags["C_CONTIGUOUS"]
    ptr = lambda a: None if a is None else a.ctypes.data  # noqa: E731
    return lib().mla_oracle_cache_append(
        B, Sq, r, d_r, block_size, num_blocks, max_blocks_per_seq, in_dtype, cache_dtype, int(bool(rope)),
        float(rope_base), c_new.ctypes.data, k_new.ctypes.data, kv_cache.ctypes.data, ptr(k_rope_cache),
        ptr(kv_scale), bt.ctypes.data, sl.ctypes.data)


def _dtype_of(a):
    if a.dtype == np.float64:
        return F64
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(a.dtype)


def head_gemm(x, w) -> np.ndarray:
    """y[m, h, :] = x[m, h, :] . w[h] in fp64. x [..., H, k], w [H, k, n]: float32 / float64
    arrays or bf16 bit patterns (uint16). Returns float64 [..., H, n]."""
    x = np.ascontiguousarray(x)
    w = np.ascontiguousarray(w)
    H, k = x.shape[-2], x.shape[-1]
    n = w.shape[-1]
    assert w.shape == (H, k, n), (w.shape, (H, k, n))
    rows = x.size // (H * k)
    y = np.empty((*x.shape[:-2], H, n), dtype=np.float64)
    lib().mla_oracle_head_gemm(rows, H, k, n, _dtype_of(x), x.ctypes.data, _dtype_of(w), w.ctypes.data,
                               y.ctypes.data)
    return y


# ---------------------------------------------------------------------------------------
# DeepSeek Sparse Attention: "TransMLA & Sparse Latent Attention" lesson, Chapter 6 ("The
# lightning indexer", "Fine-grained token selection") and Chapter 7 ("DSA runs in MLA's
# MQA mode"). Parity status: pinned by tests/test_dsa_pins.py.

def attended_counts(seq_lens, Sq, causal) -> np.ndarray:
    """Tokens each query row (b, s) may see: [B, Sq] int64 (the decode's causal rule)."""
    L = np.asarray(seq_lens, dtype=np.int64)[:, None]
    s = np.arange(Sq, dtype=np.int64)[None, :]
    n = L - Sq + 1 + s if causal else np.broadcast_to(L, (L.shape[0], Sq))
    return np.maximum(n, 0)


def dsa_index(q_codes, q_scale, weights, k_codes, k_scale, block_table, seq_lens, *, causal=False,
              max_seq_len=None, block_size=64, nthreads=0) -> np.ndarray:
    """Lightning-indexer scores in fp64 (see mla_oracle.c).

    q_codes uint8 e4m3 [B, Sq, HI, dI], q_scale / weights float32 [B, Sq, HI], k_codes
    uint8 e4m3 [num_blocks, bs, dI], k_scale float32 [num_blocks, bs]. Returns float64
    [B, Sq, max_seq_len]; entries past a row's attended count are NaN.
    """
    q_codes = np.ascontiguousarray(q_codes, dtype=np.uint8)
    q_scale = np.ascontiguousarray(q_scale, dtype=np.float32)
    weights = np.ascontiguousarray(weights, dtype=np.float32)
    k_codes = np.ascontiguousarray(k_codes, dtype=np.uint8)
    k_scale = np.ascontiguousarray(k_scale, dtype=np.float32)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Sq, HI, dI = q_codes.shape
    num_blocks = k_codes.shape[0]
    if max_seq_len is None:
        max_seq_len = int(sl.max()) if sl.size else 0
    out = np.full((B, Sq, max_seq_len), np.nan, dtype=np.float64)
    _check(lib().mla_oracle_dsa_index(B, Sq, HI, dI, block_size, num_blocks, bt.shape[1], int(bool(causal)),
                                      max_seq_len, q_codes.ctypes.data, q_scale.ctypes.data,
                                      weights.ctypes.data, k_codes.ctypes.data, k_scale.ctypes.data,
                                      bt.ctypes.data, sl.ctypes.data, out.ctypes.data, nthreads))
    return out


def dsa_counts(n_rows, k: int) -> np.ndarray:
    """Tokens a query row keeps: all of its n candidates while n <= k, else k
    (Chapter 6, "Worked arithmetic": min(t, k) per query)."""
    return np.minimum(np.maximum(np.asarray(n_rows, dtype=np.int64), 0), k)


def dsa_topk(scores, n_rows, k: int):
    """Top-k selection ("Fine-grained token selection"): for each row, the positions of
    the k highest of its first n scores (all n when n <= k). Equal scores are taken
    lowest position first, so the set is unique. Returns (indices int32 [..., k] in
    ascending position order, -1 past the count; counts int32 [...]).
    A stable sort of (-score, position) is the selection step."""
    scores = np.asarray(scores)
    n_rows = np.asarray(n_rows, dtype=np.int64)
    lead = scores.shape[:-1]
    assert n_rows.shape == lead, (n_rows.shape, lead)
    flat = scores.reshape(-1, scores.shape[-1])
    nf = n_rows.reshape(-1)
    idx = np.full((flat.shape[0], k), -1, dtype=np.int32)
    cnt = dsa_counts(nf, k).astype(np.int32)
    for i in range(flat.shape[0]):
        n = int(nf[i])
        if n <= 0:
            continue
        pos = np.arange(n)
        if n > k:
            order = np.lexsort((pos, -flat[i, :n]))   # score descending, then position
            pos = np.sort(order[:k])
        idx[i, :len(pos)] = pos
    return idx.reshape(lead + (k,)), cnt.reshape(lead)


def decode_sparse(q_lat, q_rope, kv_cache, block_table, seq_lens, softmax_scale, indices, counts,
                  k_rope_cache=None, kv_scale=None, block_size=64, nthreads=0):
    """MLA decode of each query row over its selected tokens only, fp64.

    indices int32 [B, Sq, top_k] (positions of sequence b), counts int32 [B, Sq]. Returns
    (out [B, Sq, H, r] f64, lse [B, Sq, H] f64)."""
    bd = _Bound(q_lat, q_rope, kv_cache, block_table, seq_lens, softmax_scale, False,
                k_rope_cache, kv_scale, block_size)
    B, Sq, H, r, _ = bd.shape
    indices = np.ascontiguousarray(indices, dtype=np.int32)
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    assert indices.shape[:2] == (B, Sq) and counts.shape == (B, Sq)
    out = np.zeros((B, Sq, H, r), dtype=np.float64)
    lse = np.zeros((B, Sq, H), dtype=np.float64)
    _check(lib().mla_oracle_decode_sparse(ctypes.byref(bd.p), indices.shape[2], indices.ctypes.data,
                                          counts.ctypes.data, _dp(out), _dp(lse), nthreads))
    return out, lse
