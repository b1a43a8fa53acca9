"""Absorbed multi-head latent attention (MLA) decode for B200 (sm_100a).

One decode step over a paged, compressed latent KV cache: every query head scores its
absorbed query against each cached token's latent c_t (plus the decoupled RoPE key)
and sums the latents back with the softmax weights, so one latent tile serves as both
key and value. The kernels live in libmla_decode.so (C ABI: include/mla_decode.h);
this package is a thin binding over it. The sparse variant (DeepSeek Sparse Attention:
FP8 lightning indexer, top-k selection, decode over the selected tokens) shares the cache.
"""
from .binding import (BF16, E4M3, F32, KERNELS, AppendParams, MlaError, Params, abi_version,  # noqa: F401
                      HeadGemmParams, device_status, make_append_params, mla_cache_append, mla_head_gemm,
                      host_io_workspace_size, make_params, mla_decode, mla_decode_host_io, mla_decode_timed, plan_host,
                      mla_decode_noalloc, noalloc_max_workspace, DsaParams, make_dsa_params, mla_dsa_index,
                      mla_dsa_topk, mla_sparse_decode,
                      plan_probe, resolve, set_wait_timeout_ns, status_string, wait_timeout_ns, workspace_size)
from .api import (cache_append, decode, decode_host_io, dsa_index, dsa_params_for, dsa_topk,  # noqa: F401
                  head_gemm, params_for, sparse_decode)
