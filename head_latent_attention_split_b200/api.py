"""torch-tensor front end of the C ABI: shape/dtype inference and output allocation."""
from __future__ import annotations

from . import binding as _b


def _dtype_code(t, what):
    import torch
    if t.dtype == torch.float32:
        return _b.F32
    if t.dtype == torch.bfloat16:
        return _b.BF16
    if t.dtype in (torch.uint8, getattr(torch, "float8_e4m3fn", None)):
        return _b.E4M3
    raise TypeError(f"{what}: unsupported dtype {t.dtype}")


def params_for(q_lat, q_rope, kv_cache, block_table, softmax_scale, causal=False, out_dtype=None,
               num_workers=0, kernel="auto") -> _b.Params:
    """Build mla_decode_params_t from tensor shapes.

    q_lat [B, Sq, H, r], q_rope [B, Sq, H, d_r], kv_cache [num_blocks, block_size, r + d_r]
    (f32 / bf16) or e4m3 codes [num_blocks, block_size, r], block_table [B, max_blocks].
    """
    B, Sq, H, r = q_lat.shape
    d_r = q_rope.shape[-1] if q_rope is not None else 0
    qd = _dtype_code(q_lat, "q_lat")
    cd = _dtype_code(kv_cache, "kv_cache")
    od = qd if out_dtype is None else out_dtype
    nb, bs = kv_cache.shape[0], kv_cache.shape[1]
    return _b.make_params(B, Sq, H, r, d_r, bs, nb, block_table.shape[1], qd, cd, od, causal, softmax_scale,
                          num_workers, kernel)


def decode(q_lat, q_rope, kv_cache, block_table, seq_lens, softmax_scale, causal=False, k_rope_cache=None,
           kv_scale=None, out=None, lse=None, workspace=None, out_dtype=None, num_workers=0, kernel="auto",
           stream=None):
    """One MLA decode step on the current CUDA device. Returns (out, lse).

    out [B, Sq, H, r] (dtype of q unless out_dtype), lse [B, Sq, H] float32 (natural log).
    """
    import torch
    p = params_for(q_lat, q_rope, kv_cache, block_table, softmax_scale, causal, out_dtype, num_workers, kernel)
    dev = q_lat.device
    if out is None:
        od = {_b.F32: torch.float32, _b.BF16: torch.bfloat16}[p.out_dtype]
        out = torch.empty(q_lat.shape, dtype=od, device=dev)
    if lse is None:
        lse = torch.empty(q_lat.shape[:3], dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(_b.workspace_size(p), 1), dtype=torch.uint8, device=dev)
    _b.mla_decode(p, q_lat, q_rope, kv_cache, k_rope_cache, kv_scale, block_table, seq_lens, out, lse, workspace,
                  stream=stream)
    return out, lse


def decode_host_io(q_lat_host, q_rope_host, kv_cache, block_table_host, seq_lens_host, softmax_scale,
                   causal=False, k_rope_cache=None, kv_scale=None, out_host=None, lse_host=None, workspace=None,
                   out_dtype=None, num_workers=0, kernel="auto", stream=None):
    """Decode step with per-step tensors in pinned host memory (see mla_decode_host_io)."""
    import torch
    p = params_for(q_lat_host, q_rope_host, kv_cache, block_table_host, softmax_scale, causal, out_dtype,
                   num_workers, kernel)
    if out_host is None:
        od = {_b.F32: torch.float32, _b.BF16: torch.bfloat16}[p.out_dtype]
        out_host = torch.empty(q_lat_host.shape, dtype=od, pin_memory=True)
    if lse_host is None:
        lse_host = torch.empty(q_lat_host.shape[:3], dtype=torch.float32, pin_memory=True)
    if workspace is None:
        workspace = torch.empty(_b.host_io_workspace_size(p), dtype=torch.uint8, device=kv_cache.device)
    _b.mla_decode_host_io(p, q_lat_host, q_rope_host, kv_cache, k_rope_cache, kv_scale, block_table_host,
                          seq_lens_host, out_host, lse_host, workspace, stream=stream)
    return out_host, lse_host


def cache_append(c_new, k_rope_new, kv_cache, block_table, seq_lens, k_rope_cache=None, kv_scale=None,
                 rope=False, rope_base=10000.0, stream=None):
    """Write the Sq new tokens of each sequence into the paged cache (see mla_cache_append).

    c_new [B, Sq, r] and k_rope_new [B, Sq, d_r] (float32 for an f32 cache, bf16 otherwise);
    kv_cache [num_blocks, block_size, r + d_r] (f32 / bf16), or e4m3 codes
    [num_blocks, block_size, r] (uint8) with k_rope_cache bf16 [num_blocks, block_size, d_r]
    and kv_scale float32 [num_blocks, block_size]. Token s of sequence b lands at position
    seq_lens[b] - Sq + s. With rope, the RoPE key is rotated for that position first.
    """
    B, Sq, r = c_new.shape
    d_r = k_rope_new.shape[-1] if k_rope_new is not None else 0
    p = _b.make_append_params(B, Sq, r, d_r, kv_cache.shape[1], kv_cache.shape[0], block_table.shape[1],
                              _dtype_code(c_new, "c_new"), _dtype_code(kv_cache, "kv_cache"), rope, rope_base)
    _b.mla_cache_append(p, c_new, k_rope_new, kv_cache, k_rope_cache, kv_scale, block_table, seq_lens, stream=stream)


def head_gemm(x, w, y=None, stream=None):
    """y[m, h, :] = x[m, h, :] @ w[h] on the tensor cores (bf16 in and out, fp32 accumulation).

    x [rows, H, k] (or [B, Sq, H, k]), w [H, k, n]; k and n multiples of 64. Query absorption:
    head_gemm(q_nope, W_UK) -> q_lat; output projection: head_gemm(out, W_UV.transpose(1, 2)).
    """
    import torch
    lead = x.shape[:-2]
    H, k = x.shape[-2], x.shape[-1]
    n = w.shape[-1]
    rows = int(x.numel() // (H * k))
    if y is None:
        y = torch.empty((*lead, H, n), dtype=torch.bfloat16, device=x.device)
    p = _b.HeadGemmParams(rows=rows, heads=H, k=k, n=n, reserved=0)
    _b.mla_head_gemm(p, x, w, y, stream=stream)
    return y


def dsa_params_for(q_codes, k_codes, block_table, max_seq_len, top_k, causal=False) -> _b.DsaParams:
    """mla_dsa_params_t from tensor shapes: q_codes [B, Sq, H^I, d^I], k_codes
    [num_blocks, block_size, d^I], block_table [B, max_blocks]."""
    B, Sq, HI, dI = q_codes.shape
    nb, bs = k_codes.shape[0], k_codes.shape[1]
    return _b.make_dsa_params(B, Sq, HI, dI, bs, nb, block_table.shape[1], max_seq_len, top_k, causal)


def dsa_index(q_codes, q_scale, weights, k_codes, k_scale, block_table, seq_lens, max_seq_len, scores=None,
              causal=False, stream=None):
    """Lightning-indexer scores [B, Sq, max_seq_len] float32 (see mla_dsa_index). Code
    tensors are uint8 (or float8_e4m3fn) e4m3 codes."""
    import torch
    p = dsa_params_for(q_codes, k_codes, block_table, max_seq_len, 1, causal)
    if scores is None:
        scores = torch.empty((q_codes.shape[0], q_codes.shape[1], max_seq_len), dtype=torch.float32,
                             device=q_codes.device)
    _b.mla_dsa_index(p, q_codes, q_scale, weights, k_codes, k_scale, block_table, seq_lens, scores, stream=stream)
    return scores


def dsa_topk(scores, seq_lens, top_k, causal=False, indices=None, counts=None, stream=None):
    """Top-k positions per query row: (indices int32 [B, Sq, top_k] ascending, -1 padded;
    counts int32 [B, Sq]) (see mla_dsa_topk)."""
    import torch
    B, Sq, max_seq_len = scores.shape
    p = _b.make_dsa_params(B, Sq, 64, 128, 64, 1, max(1, (max_seq_len + 63) // 64), max_seq_len, top_k, causal)
    if indices is None:
        indices = torch.empty((B, Sq, top_k), dtype=torch.int32, device=scores.device)
    if counts is None:
        counts = torch.empty((B, Sq), dtype=torch.int32, device=scores.device)
    _b.mla_dsa_topk(p, scores, seq_lens, indices, counts, stream=stream)
    return indices, counts


def sparse_decode(q_lat, q_rope, kv_cache, block_table, indices, counts, softmax_scale, out=None, lse=None,
                  workspace=None, num_workers=0, stream=None, kernel="auto"):
    """MLA decode over selected positions (q_len 1, bf16 cache): indices [B, top_k] (or
    [B, 1, top_k]) int32, counts [B] (or [B, 1]) int32. Returns (out, lse)."""
    import torch
    p = params_for(q_lat, q_rope, kv_cache, block_table, softmax_scale, False, None, num_workers, kernel)
    top_k = indices.shape[-1]
    dev = q_lat.device
    if out is None:
        out = torch.empty(q_lat.shape, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(q_lat.shape[:3], dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(_b.workspace_size(p), 1), dtype=torch.uint8, device=dev)
    _b.mla_sparse_decode(p, top_k, q_lat, q_rope, kv_cache, block_table, indices, counts, out, lse, workspace,
                         stream=stream)
    return out, lse
