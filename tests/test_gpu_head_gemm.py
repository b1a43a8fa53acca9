"""GPU parity of the per-head tensor-core GEMM (query absorption / output projection)
against the oracle's fp64 products, and of the whole absorbed layer (absorb -> decode ->
project) against the oracle chain."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workloads as W
from parity_util import TOL, compare

pytestmark = pytest.mark.gpu


def _bf16(a):
    import torch
    return torch.from_numpy(W.f32_to_bf16_bits(a.astype(np.float32)).view(np.int16)).cuda().view(torch.bfloat16)


def _np(t):
    import torch
    return t.float().cpu().numpy().astype(np.float64) if t.dtype != torch.bfloat16 else \
        W.bf16_bits_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)


@pytest.mark.parametrize("rows,H,k,n", [(64, 128, 128, 512), (64, 128, 512, 128), (200, 4, 128, 512),
                                        (1, 3, 64, 64), (130, 2, 192, 320), (256, 8, 512, 256)])
def test_head_gemm_matches_oracle(rows, H, k, n):
    import torch
    import head_latent_attention_split_b200 as mla
    rng = np.random.default_rng(rows * 7 + H + k + n)
    x = rng.normal(size=(rows, H, k)).astype(np.float32)
    w = (rng.normal(size=(H, k, n)) / np.sqrt(k)).astype(np.float32)
    xt, wt = _bf16(x), _bf16(w)
    y = mla.head_gemm(xt, wt)
    torch.cuda.synchronize()
    assert mla.device_status() == 0
    ref = oracle.head_gemm(W.f32_to_bf16_bits(x), W.f32_to_bf16_bits(w))
    got = _np(y)
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert err <= TOL[W.BF16], err
    # rows never touched beyond `rows`: y was allocated exactly [rows, H, n]
    assert got.shape == (rows, H, n)


def test_head_gemm_rejects_bad_shapes():
    from head_latent_attention_split_b200 import binding
    for bad in (dict(k=48), dict(n=100), dict(heads=0), dict(rows=-1), dict(reserved=1)):
        kw = dict(rows=4, heads=2, k=64, n=64, reserved=0)
        kw.update(bad)
        p = binding.HeadGemmParams(**kw)
        assert binding.mla_head_gemm(p, 1 << 20, 1 << 20, 1 << 20, stream=0, check=False) == 1


def test_absorbed_layer_matches_oracle_chain():
    """q_nope -> W^UK -> decode (tcgen05) -> W^UV^T, against the same chain in the oracle."""
    import torch
    import head_latent_attention_split_b200 as mla
    w = W.WORKLOADS[2].with_(B=2, H=16, seq_lens=(300, 77))
    inp = W.make_inputs(w)
    rng = np.random.default_rng(21)
    d_h, d_v = 128, 128
    q_nope = rng.normal(size=(w.B, w.Sq, w.H, d_h)).astype(np.float32)
    w_uk = (rng.normal(size=(w.H, d_h, 512)) / np.sqrt(d_h)).astype(np.float32)
    w_uv_t = (rng.normal(size=(w.H, 512, d_v)) / np.sqrt(512)).astype(np.float32)
    t = W.to_torch(inp)
    q_lat = mla.head_gemm(_bf16(q_nope), _bf16(w_uk))
    out, lse = mla.decode(q_lat, t["q_rope"], t["kv_cache"], t["block_table"], t["seq_lens"], w.scale, w.causal,
                          kernel="tcgen05")
    y = mla.head_gemm(out, _bf16(w_uv_t))
    torch.cuda.synchronize()
    assert mla.device_status() == 0
    # oracle chain on the GPU's own intermediate roundings (q_lat and out are bf16 there)
    q_lat_bits = q_lat.view(torch.int16).cpu().numpy().view(np.uint16)
    ref_out, ref_lse = oracle.decode(q_lat_bits, inp["q_rope"], inp["kv_cache"], inp["block_table"],
                                     inp["seq_lens"], w.scale, w.causal)
    compare(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_out, ref_lse, TOL[W.BF16], "decode")
    ref_y = oracle.head_gemm(out.view(torch.int16).cpu().numpy().view(np.uint16), W.f32_to_bf16_bits(w_uv_t))
    err = np.abs(_np(y) - ref_y).max() / np.abs(ref_y).max()
    assert err <= TOL[W.BF16], err
    # and the absorption itself
    ref_q = oracle.head_gemm(W.f32_to_bf16_bits(q_nope), W.f32_to_bf16_bits(w_uk))
    assert np.abs(_np(q_lat) - ref_q).max() / np.abs(ref_q).max() <= TOL[W.BF16]
