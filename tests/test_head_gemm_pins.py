"""Pins of the oracle's per-head products (query absorption, output up-projection).

Brute force on small integer operands (exact in fp64), and the absorbed path composed of
these products and the oracle decode against the explicit up-projected attention
("TransMLA: Multi-Head Latent Attention Is All You Need", sec. 3.4.5: with k_t,i = W^UK_i c_t
and v_t,i = W^UV_i c_t, q_i . k_t,i = (q_i W^UK_i) . c_t and sum_t p_t v_t,i = W^UV_i sum_t p_t c_t).
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle


def test_head_gemm_bruteforce_integers():
    rng = np.random.default_rng(3)
    rows, H, k, n = 3, 2, 5, 4
    x = rng.integers(-4, 5, size=(rows, H, k)).astype(np.float64)
    w = rng.integers(-4, 5, size=(H, k, n)).astype(np.float64)
    y = oracle.head_gemm(x, w)
    for m in range(rows):
        for h in range(H):
            for j in range(n):
                assert y[m, h, j] == sum(x[m, h, kk] * w[h, kk, j] for kk in range(k))


def test_head_gemm_reads_bf16_patterns():
    import workloads as W
    rng = np.random.default_rng(4)
    x = W.f32_to_bf16_bits(rng.normal(size=(4, 3, 8)).astype(np.float32))
    w = W.f32_to_bf16_bits(rng.normal(size=(3, 8, 6)).astype(np.float32))
    xd = W.bf16_bits_to_f32(x).astype(np.float64)
    wd = W.bf16_bits_to_f32(w).astype(np.float64)
    np.testing.assert_allclose(oracle.head_gemm(x, w), oracle.head_gemm(xd, wd), rtol=0, atol=0)


@pytest.mark.parametrize("causal", [False, True])
def test_absorbed_layer_equals_explicit_attention(causal):
    rng = np.random.default_rng(9 + causal)
    B, Sq, H, d_h, d_v, r, d_r, bs = 2, 2, 3, 6, 5, 8, 4, 4
    lens = np.array([7, 3], np.int32)
    mb = 2
    bt = np.array([[3, 0], [1, 2]], np.int32)
    cache = rng.normal(size=(4, bs, r + d_r))
    w_uk = rng.normal(size=(H, d_h, r))          # W^UK_i: d_h x r
    w_uv = rng.normal(size=(H, d_v, r))          # W^UV_i: d_v x r
    q_nope = rng.normal(size=(B, Sq, H, d_h))
    q_rope = rng.normal(size=(B, Sq, H, d_r))
    scale = 0.7
    # absorbed path: q_lat = q_nope W^UK, decode over the latent, then W^UV on the result
    q_lat = oracle.head_gemm(q_nope, w_uk)
    out_lat, _ = oracle.decode(q_lat, q_rope, cache, bt, lens, scale, causal, block_size=bs)
    y = oracle.head_gemm(out_lat, np.ascontiguousarray(w_uv.transpose(0, 2, 1)))
    # explicit path: per-head keys and values up-projected from every cached latent
    for b in range(B):
        L = int(lens[b])
        toks = np.stack([cache[bt[b, t // bs], t % bs] for t in range(L)])
        c, kr = toks[:, :r], toks[:, r:]
        for s in range(Sq):
            n_att = L - Sq + 1 + s if causal else L
            for h in range(H):
                K = c[:n_att] @ w_uk[h].T            # [n, d_h]
                V = c[:n_att] @ w_uv[h].T            # [n, d_v]
                sc = scale * (K @ q_nope[b, s, h] + kr[:n_att] @ q_rope[b, s, h])
                p = np.exp(sc - sc.max())
                p /= p.sum()
                np.testing.assert_allclose(y[b, s, h], p @ V, rtol=1e-11, atol=1e-12)
