"""GPU parity of the paged cache append (mla_cache_append) against the oracle's append.

The latent bytes and per-token scales must match the oracle bit for bit (copies, and
e4m3 codes decided in fp32 on both sides); the RoPE key matches bit for bit when stored
as given and within one unit in the last place of the cache type when rotated (fp64 sin
and cos of two libraries). Then a decode over the appended cache matches the oracle's
decode of the oracle-appended cache.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workloads as W
from parity_util import LSE_TOL, TOL, compare

pytestmark = pytest.mark.gpu


def _ulp_diff_f32(a, b):
    ai = a.view(np.int32).astype(np.int64)
    bi = b.view(np.int32).astype(np.int64)
    return np.abs(ai - bi)


def _setup(cache_dtype, B, Sq, r, d_r, bs, lens, seed):
    rng = np.random.default_rng(seed)
    mb = max((L + bs - 1) // bs for L in lens) + 1
    nb = B * mb + 2
    perm = rng.permutation(nb).astype(np.int32)
    bt = perm[:B * mb].reshape(B, mb).copy()
    cf = (rng.normal(size=(B, Sq, r)) * rng.uniform(0.05, 20, size=(B, Sq, 1))).astype(np.float32)
    kf = rng.normal(size=(B, Sq, d_r)).astype(np.float32)
    if cache_dtype == W.F32:
        c, k = cf, kf
        cache = rng.normal(size=(nb, bs, r + d_r)).astype(np.float32)
        kr = sc = None
    else:
        c, k = W.f32_to_bf16_bits(cf), W.f32_to_bf16_bits(kf)
        if cache_dtype == W.BF16:
            cache = rng.integers(0, 1 << 16, size=(nb, bs, r + d_r)).astype(np.uint16)
            kr = sc = None
        else:
            cache = rng.integers(0, 256, size=(nb, bs, r)).astype(np.uint8)
            kr = rng.integers(0, 1 << 16, size=(nb, bs, d_r)).astype(np.uint16)
            sc = rng.normal(size=(nb, bs)).astype(np.float32)
    return dict(B=B, Sq=Sq, r=r, d_r=d_r, bs=bs, nb=nb, mb=mb, bt=bt, lens=np.array(lens, np.int32), c=c, k=k,
                cache=cache, kr=kr, sc=sc, cache_dtype=cache_dtype,
                in_dtype=W.F32 if cache_dtype == W.F32 else W.BF16)


def _oracle_append(S, rope):
    cache = S["cache"].copy()
    kr = None if S["kr"] is None else S["kr"].copy()
    sc = None if S["sc"] is None else S["sc"].copy()
    st = oracle.cache_append(B=S["B"], Sq=S["Sq"], r=S["r"], d_r=S["d_r"], block_size=S["bs"], num_blocks=S["nb"],
                             max_blocks_per_seq=S["mb"], in_dtype=S["in_dtype"], cache_dtype=S["cache_dtype"],
                             c_new=S["c"], k_new=S["k"], kv_cache=cache, k_rope_cache=kr, kv_scale=sc,
                             block_table=S["bt"], seq_lens=S["lens"], rope=rope, rope_base=10000.0)
    return st, cache, kr, sc


def _gpu_append(S, rope):
    import torch
    import head_latent_attention_split_b200 as mla
    dev = "cuda"
    t = lambda a: None if a is None else torch.from_numpy(a.copy()).to(dev)  # noqa: E731
    tt = lambda a: None if a is None else torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(dev)  # noqa: E731
    c = torch.from_numpy(S["c"]).to(dev) if S["in_dtype"] == W.F32 else \
        torch.from_numpy(S["c"].view(np.int16)).to(dev).view(torch.bfloat16)
    k = torch.from_numpy(S["k"]).to(dev) if S["in_dtype"] == W.F32 else \
        torch.from_numpy(S["k"].view(np.int16)).to(dev).view(torch.bfloat16)
    if S["cache_dtype"] == W.F32:
        cache = t(S["cache"])
    elif S["cache_dtype"] == W.BF16:
        cache = tt(S["cache"].copy()).view(torch.bfloat16)
    else:
        cache = t(S["cache"])
    kr = None if S["kr"] is None else tt(S["kr"].copy()).view(torch.bfloat16)
    sc = t(S["sc"])
    mla.cache_append(c, k, cache, t(S["bt"]), t(S["lens"]), k_rope_cache=kr, kv_scale=sc, rope=rope,
                     rope_base=10000.0)
    torch.cuda.synchronize()
    st = mla.device_status()
    back = lambda x: None if x is None else (x.view(torch.int16).cpu().numpy().view(np.uint16)  # noqa: E731
                                             if x.dtype == torch.bfloat16 else x.cpu().numpy())
    return st, back(cache), back(kr), back(sc)


CASES = [
    (W.F32, 2, 1, 16, 8, 8, (5, 17)),
    (W.F32, 3, 2, 40, 6, 4, (3, 9, 21)),
    (W.BF16, 3, 2, 512, 64, 64, (70, 130, 2)),
    (W.E4M3, 3, 1, 512, 64, 64, (1, 64, 65)),
    (W.E4M3, 2, 2, 512, 64, 64, (200, 4096)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{W.DTYPE_NAMES[c[0]]}-B{c[1]}-Sq{c[2]}-r{c[3]}")
@pytest.mark.parametrize("rope", [False, True])
def test_append_matches_oracle(case, rope):
    cache_dtype, B, Sq, r, d_r, bs, lens = case
    S = _setup(cache_dtype, B, Sq, r, d_r, bs, lens, seed=hash((case, rope)) % 1000)
    st_o, cache_o, kr_o, sc_o = _oracle_append(S, rope)
    st_g, cache_g, kr_g, sc_g = _gpu_append(S, rope)
    assert st_o == 0 and st_g == 0
    if cache_dtype == W.E4M3:
        np.testing.assert_array_equal(cache_g, cache_o)          # codes, bit for bit
        np.testing.assert_array_equal(sc_g.view(np.int32), sc_o.view(np.int32))
        rope_g, rope_o = kr_g, kr_o
    else:
        np.testing.assert_array_equal(cache_g[..., :r], cache_o[..., :r])
        rope_g, rope_o = cache_g[..., r:], cache_o[..., r:]
    if not rope:
        np.testing.assert_array_equal(rope_g, rope_o)
    elif cache_dtype == W.F32:
        assert _ulp_diff_f32(np.ascontiguousarray(rope_g), np.ascontiguousarray(rope_o)).max() <= 1
    else:
        d = np.abs(rope_g.astype(np.int32) - rope_o.astype(np.int32))
        assert d.max() <= 1   # bf16 patterns of the same sign: one unit in the last place


def test_append_reports_bad_block_and_position():
    import torch
    import head_latent_attention_split_b200 as mla
    dev = "cuda"
    cache = torch.zeros((2, 4, 6), dtype=torch.float32, device=dev)
    c = torch.ones((1, 1, 4), device=dev)
    k = torch.ones((1, 1, 2), device=dev)
    bt = torch.tensor([[0, 9]], dtype=torch.int32, device=dev)
    mla.cache_append(c, k, cache, bt, torch.tensor([6], dtype=torch.int32, device=dev))
    assert mla.device_status() == 6    # MLA_ERR_BAD_BLOCK_ID
    mla.cache_append(c, k, cache, bt, torch.tensor([9], dtype=torch.int32, device=dev))
    assert mla.device_status() == 7    # MLA_ERR_BAD_SEQ_LEN
    assert not cache.any()


@pytest.mark.parametrize("cache_dtype", [W.BF16, W.E4M3])
def test_decode_after_append_matches_oracle(cache_dtype):
    """Append two new tokens per sequence (rotated RoPE keys), then decode them causally."""
    import torch
    import head_latent_attention_split_b200 as mla
    base = W.WORKLOADS[3] if cache_dtype == W.BF16 else W.WORKLOADS[4]
    w = base.with_(B=3, Sq=2, causal=True, H=16, seq_lens=(70, 300, 129))
    inp = W.make_inputs(w)
    rng = np.random.default_rng(77)
    S = dict(B=w.B, Sq=2, r=512, d_r=64, bs=64, nb=inp["num_blocks"], mb=inp["max_blocks_per_seq"],
             bt=inp["block_table"], lens=inp["seq_lens"], cache_dtype=cache_dtype, in_dtype=W.BF16,
             c=W.f32_to_bf16_bits((rng.normal(size=(w.B, 2, 512)) / 20).astype(np.float32)),
             k=W.f32_to_bf16_bits((rng.normal(size=(w.B, 2, 64)) / 20).astype(np.float32)),
             cache=inp["kv_cache"], kr=inp.get("k_rope_cache"), sc=inp.get("kv_scale"))
    st_o, cache_o, kr_o, sc_o = _oracle_append(S, True)
    st_g, cache_g, kr_g, sc_g = _gpu_append(S, True)
    assert st_o == 0 and st_g == 0
    # decode the GPU-appended cache on the GPU, the oracle-appended cache on the oracle
    inp_g = dict(inp, kv_cache=cache_g, k_rope_cache=kr_g, kv_scale=sc_g)
    t = W.to_torch(inp_g)
    out, lse = mla.decode(t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], t["seq_lens"], w.scale, True,
                          t["k_rope_cache"], t["kv_scale"], kernel="tcgen05")
    torch.cuda.synchronize()
    assert mla.device_status() == 0
    ref_out, ref_lse = oracle.decode(inp["q_lat"], inp["q_rope"], cache_o, inp["block_table"], inp["seq_lens"],
                                     w.scale, True, kr_o, sc_o)
    compare(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_out, ref_lse, TOL[cache_dtype],
            "decode after append")
    assert LSE_TOL > 0
