"""Pins of the oracle's cache append (the producer of the cache the decode reads).

The e4m3 encoder is pinned against the bit definition (every finite code round-trips,
ties go to the even code, saturation at 448) and against torch's float8_e4m3fn cast; the
RoPE rotation against the two-position toy of the TransMLA & Sparse Latent Attention
lesson (tests/golden/rope_toy.json), read back through the oracle's own decode; the copy
paths against the slot arithmetic of the paged layout.
"""
from __future__ import annotations

import json
import os

import numpy as np
import pytest

import oracle
import workloads as W


def _finite_codes():
    return [c for c in range(256) if c not in (0x7F, 0xFF)]


def test_e4m3_encoder_round_trips_every_finite_code():
    codes = np.array(_finite_codes(), dtype=np.uint8)
    vals = np.array([oracle.e4m3_to_double(int(c)) for c in codes], dtype=np.float32)
    got = oracle.e4m3_encode(vals)
    # +0 and -0 keep their sign bit; every other code maps back to itself
    np.testing.assert_array_equal(got, codes)


def test_e4m3_encoder_ties_to_even_and_saturates():
    pos = [c for c in range(0x7E)]   # consecutive finite positive codes c, c + 1
    for c in pos:
        lo, hi = oracle.e4m3_to_double(c), oracle.e4m3_to_double(c + 1)
        mid = np.float32((lo + hi) / 2)
        if float(mid) != (lo + hi) / 2:
            continue   # midpoint not representable in fp32
        want = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode([mid])[0] == want, (c, lo, hi)
        assert oracle.e4m3_encode([-mid])[0] == (want | 0x80)
    assert oracle.e4m3_encode([1000.0, -1e30, 449.0, 470.0])[0] == 0x7E
    assert list(oracle.e4m3_encode([1000.0, -1e30, 449.0, 470.0])) == [0x7E, 0xFE, 0x7E, 0x7E]
    assert oracle.e4m3_encode([np.nan])[0] == 0x7F


def test_e4m3_encoder_matches_torch_below_overflow():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 100, 20000), rng.uniform(-2 ** -6, 2 ** -6, 5000),
                        rng.uniform(-460, 460, 5000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode(x), ref)


def _paged(B, Sq, lens, bs, rng, spare=3):
    mb = max((L + bs - 1) // bs for L in lens)
    nb = B * mb + spare
    perm = rng.permutation(nb).astype(np.int32)
    bt = np.full((B, mb), -1, np.int32)
    for b in range(B):
        bt[b] = perm[b * mb:(b + 1) * mb]
    return bt, nb, mb


def test_rope_toy_through_append_and_decode(golden_dir):
    G = json.load(open(os.path.join(golden_dir, "rope_toy.json")))
    for t, want in zip(G["positions"], G["scores"]):
        # one sequence whose new token sits at position t; f32 cache with r = 1 latent
        # channel (zero) and a d_r = 2 RoPE key; theta_0 = base^0 = 1 rad per position
        bs = 8
        bt = np.array([[0, 1]], np.int32)
        cache = np.zeros((2, bs, 1 + 2), np.float32)
        st = oracle.cache_append(B=1, Sq=1, r=1, d_r=2, block_size=bs, num_blocks=2, max_blocks_per_seq=2,
                                 in_dtype=oracle.F32, cache_dtype=oracle.F32,
                                 c_new=np.zeros((1, 1, 1), np.float32),
                                 k_new=np.array([[G["k"]]], np.float32), kv_cache=cache, block_table=bt,
                                 seq_lens=np.array([t + 1], np.int32), rope=True, rope_base=10000.0)
        assert st == 0
        # score against q = [1, 0] over the appended token alone (a one-token window): lse = score
        q_lat = np.zeros((1, 1, 1, 1))
        q_rope = np.array(G["q"], np.float64).reshape(1, 1, 1, 2)
        out, lse = oracle.decode(q_lat, q_rope, cache, bt, np.array([t + 1], np.int32), 1.0, block_size=bs,
                                 tok_begin=np.array([t], np.int64), tok_end=np.array([t + 1], np.int64))
        assert round(float(lse[0, 0, 0]), G["digits"]) == want
        assert abs(float(lse[0, 0, 0]) - np.cos(t)) < 1e-7


@pytest.mark.parametrize("Sq", [1, 2])
def test_bf16_append_copies_into_the_right_slots(Sq):
    rng = np.random.default_rng(11)
    B, r, d_r, bs = 3, 8, 4, 4
    lens = [5, 9, 2]
    bt, nb, mb = _paged(B, Sq, lens, bs, rng)
    cache = np.full((nb, bs, r + d_r), 0x7FC0, np.uint16)
    c = W.f32_to_bf16_bits(rng.normal(size=(B, Sq, r)).astype(np.float32))
    k = W.f32_to_bf16_bits(rng.normal(size=(B, Sq, d_r)).astype(np.float32))
    st = oracle.cache_append(B=B, Sq=Sq, r=r, d_r=d_r, block_size=bs, num_blocks=nb, max_blocks_per_seq=mb,
                             in_dtype=oracle.BF16, cache_dtype=oracle.BF16, c_new=c, k_new=k, kv_cache=cache,
                             block_table=bt, seq_lens=np.array(lens, np.int32))
    assert st == 0
    written = 0
    for b in range(B):
        for s in range(Sq):
            pos = lens[b] - Sq + s
            row = cache[bt[b, pos // bs], pos % bs]
            np.testing.assert_array_equal(row[:r], c[b, s])
            np.testing.assert_array_equal(row[r:], k[b, s])
            written += 1
    assert (cache != 0x7FC0).any(axis=-1).sum() == written   # nothing else touched


def test_e4m3_append_quantises_within_half_a_step():
    rng = np.random.default_rng(5)
    B, Sq, r, d_r, bs = 2, 2, 16, 4, 4
    lens = [6, 11]
    bt, nb, mb = _paged(B, Sq, lens, bs, rng)
    codes = np.zeros((nb, bs, r), np.uint8)
    kr = np.zeros((nb, bs, d_r), np.uint16)
    sc = np.full((nb, bs), -1.0, np.float32)
    cf = (rng.normal(size=(B, Sq, r)) * rng.uniform(0.01, 50, size=(B, Sq, 1))).astype(np.float32)
    c = W.f32_to_bf16_bits(cf)
    cb = c.astype(np.uint32) << 16
    cv = cb.view(np.float32)
    k = W.f32_to_bf16_bits(rng.normal(size=(B, Sq, d_r)).astype(np.float32))
    st = oracle.cache_append(B=B, Sq=Sq, r=r, d_r=d_r, block_size=bs, num_blocks=nb, max_blocks_per_seq=mb,
                             in_dtype=oracle.BF16, cache_dtype=oracle.E4M3, c_new=c, k_new=k, kv_cache=codes,
                             k_rope_cache=kr, kv_scale=sc, block_table=bt, seq_lens=np.array(lens, np.int32))
    assert st == 0
    for b in range(B):
        for s in range(Sq):
            pos = lens[b] - Sq + s
            blk, o = bt[b, pos // bs], pos % bs
            v = cv[b, s].astype(np.float64)
            scale = sc[blk, o]
            assert scale == np.float32(np.float32(np.abs(cv[b, s]).max()) / np.float32(448.0))
            dec = np.array([oracle.e4m3_to_double(int(x)) for x in codes[blk, o]]) * float(scale)
            # nearest e4m3: half a step (2^-4 relative for normals, 2^-10 absolute below 2^-6)
            bound = np.maximum(np.abs(v) * 2.0 ** -4, 2.0 ** -10 * float(scale)) * (1 + 1e-6)
            assert np.all(np.abs(dec - v) <= bound)
            assert np.abs(codes[blk, o].astype(np.int32) & 0x7F).max() == 0x7E   # amax maps to 448
            np.testing.assert_array_equal(kr[blk, o], k[b, s])


def test_append_reports_bad_positions_and_blocks():
    bt = np.array([[0, 9]], np.int32)
    cache = np.zeros((2, 4, 6), np.float32)
    common = dict(B=1, Sq=1, r=4, d_r=2, block_size=4, num_blocks=2, max_blocks_per_seq=2, in_dtype=oracle.F32,
                  cache_dtype=oracle.F32, c_new=np.ones((1, 1, 4), np.float32), k_new=np.ones((1, 1, 2), np.float32),
                  kv_cache=cache, block_table=bt)
    assert oracle.cache_append(seq_lens=np.array([6], np.int32), **common) == 2   # block 9 does not exist
    assert oracle.cache_append(seq_lens=np.array([9], np.int32), **common) == 3   # past the table
    assert oracle.cache_append(seq_lens=np.array([0], np.int32), **common) == 3   # no room for the new token
    assert not cache.any()
