"""Pins for the fp64 oracle: what the pages and the mathematics fix, independent of it.

Each test checks the oracle against something other than its own formula:
  * worked examples printed in the "TransMLA & Sparse Latent Attention" lesson
    (tests/golden/*.json, each with its citation);
  * GQA computed head by head, which the pages prove equal to the same GQA written
    as MLA with identity-selector up-projections (TransMLA sec. 3.4.1, eqs. 11-15);
  * the explicit, non-absorbed form with per-head up-projected keys and values,
    which the absorb identity equates to the absorbed score (TransMLA sec. 3.4.2,
    TPLA sec. 3.4 eq. 5 and "The RoPE handling");
  * closed forms (scale 0 gives the mean, one token gives itself), row sums of the
    softmax, the log-sum-exp merge of disjoint windows;
  * a 50-digit mpmath brute force on tiny paged causal inputs;
  * torch's bf16 / float8_e4m3fn decoders for every code.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(20240521)


# ----------------------------------------------------------------------------- helpers
def paged(c_dense, kr_dense, lens, block_size, rng, spare=1, dtype=np.float64):
    """Scatter dense per-sequence tokens into a shuffled paged cache.

    c_dense [B, Lmax, r], kr_dense [B, Lmax, d_r]. Unused slots are NaN.
    Returns (cache [num_blocks, bs, r+d_r], block_table [B, max_blocks]).
    """
    B, Lmax, r = c_dense.shape
    d_r = kr_dense.shape[-1]
    nblk = [(int(L) + block_size - 1) // block_size for L in lens]
    num_blocks = sum(nblk) + spare
    perm = rng.permutation(num_blocks)
    mb = max(1, max(nblk))
    bt = np.full((B, mb), -1, dtype=np.int32)
    cache = np.full((num_blocks, block_size, r + d_r), np.nan, dtype=dtype)
    off = 0
    for b in range(B):
        for i in range(nblk[b]):
            blk = perm[off + i]
            bt[b, i] = blk
            for o in range(block_size):
                t = i * block_size + o
                if t < lens[b]:
                    cache[blk, o, :r] = c_dense[b, t]
                    cache[blk, o, r:] = kr_dense[b, t]
        off += nblk[b]
    return cache, bt


def selector(i0, h, g, d):
    """Identity-selector up-projection W_i (d x g*d) for 0-based head i0.

    0-based group = i0 // (h // g), the same map as the 1-based ceil(i/(h/g)).
    """
    j = i0 // (h // g)
    W = np.zeros((d, g * d))
    W[:, j * d:(j + 1) * d] = np.eye(d)
    return W


def gqa_attention(q, K, V, h, g):
    """Plain GQA for one query step, head by head (TransMLA eqs. 2-6).

    q [h, d], K [g, n, d], V [g, n, d] -> o [h, d]; scale 1/sqrt(d).
    """
    d = q.shape[1]
    o = np.zeros((h, d))
    for i in range(h):
        j = i // (h // g)
        s = K[j] @ q[i] / math.sqrt(d)
        w = np.exp(s - s.max())
        w /= w.sum()
        o[i] = w @ V[j]
    return o


# ----------------------------------------------------------------------------- golden toys
def test_gqa_toy_single_token(golden_dir):
    """Chapter 1 toy: heads 1,2 -> group 1 -> 10; heads 3,4 -> group 2 -> 20."""
    G = json.load(open(os.path.join(golden_dir, "gqa_toy.json")))
    h, g, d = G["h"], G["g"], G["d"]
    k, v = G["keys"], G["values"]
    latent = np.array(k + v, dtype=np.float64)          # [K_1, K_2, V_1, V_2], r = 2 g d
    r = latent.size
    qs = {int(i): x for i, x in G["queries"].items()}
    qs[4] = 0.625                                       # not printed; any value works
    q_lat = np.zeros((1, 1, h, r))
    for i in range(1, h + 1):
        WK = selector(i - 1, h, g, d)                   # d x g d over the K half
        q_lat[0, 0, i - 1, :g * d] = WK.T @ np.array([qs[i]])
        assert (i - 1) // (h // g) + 1 == G["expected_group"][str(i)] == math.ceil(i / (h / g))
    cache = latent.reshape(1, 1, r)
    out, lse = oracle.decode(q_lat, np.zeros((1, 1, h, 0)), cache, np.zeros((1, 1), np.int32),
                             np.array([1], np.int32), 1.0 / math.sqrt(d), block_size=1)
    for i in range(1, h + 1):
        WV = selector(i - 1, h, g, d)
        got = (WV @ out[0, 0, i - 1, g * d:])[0]        # value read out through W^UV_i
        assert got == G["expected_output"][str(i)]
        # one token: lse equals its own score
        assert lse[0, 0, i - 1] == pytest.approx(q_lat[0, 0, i - 1] @ latent / math.sqrt(d), abs=1e-15)


def test_selector_toy(golden_dir):
    """Chapter 2 toy: the selector recovers group keys/values from the concatenated latent."""
    G = json.load(open(os.path.join(golden_dir, "selector_toy.json")))
    h, g, d = G["h"], G["g"], G["d"]
    latent = np.array(G["latent"])
    assert list(latent) == sum(G["keys"], []) + sum(G["values"], [])
    K, V = latent[:g * d], latent[g * d:]
    assert list(selector(0, h, g, d) @ K) == G["head1_key_value"][0]
    assert list(selector(0, h, g, d) @ V) == G["head1_key_value"][1]
    assert list(selector(2, h, g, d) @ K) == G["head3_key"]
    L = G["listing_check"]
    assert L["head_index_0_based"] // (L["h"] // L["g"]) == L["group_0_based"]


# ----------------------------------------------------------------------------- identities
@pytest.mark.parametrize("h,g,d,n", [(4, 2, 3, 5), (8, 8, 4, 9), (6, 1, 5, 17), (12, 3, 8, 70)])
def test_gqa_equals_gqa_written_as_mla(h, g, d, n):
    """GQA with g groups == the oracle run on the concatenated latent with selector queries."""
    q = RNG.standard_normal((h, d))
    K = RNG.standard_normal((g, n, d))
    V = RNG.standard_normal((g, n, d))
    ref = gqa_attention(q, K, V, h, g)
    r = 2 * g * d
    lat = np.concatenate([K.transpose(1, 0, 2).reshape(n, g * d), V.transpose(1, 0, 2).reshape(n, g * d)], 1)
    q_lat = np.zeros((1, 1, h, r))
    for i in range(h):
        q_lat[0, 0, i, :g * d] = selector(i, h, g, d).T @ q[i]
    cache, bt = paged(lat[None], np.zeros((1, n, 0)), [n], 4, RNG)
    out, _ = oracle.decode(q_lat, np.zeros((1, 1, h, 0)), cache, bt, np.array([n], np.int32),
                           1.0 / math.sqrt(d), block_size=4)
    for i in range(h):
        got = selector(i, h, g, d) @ out[0, 0, i, g * d:]
        np.testing.assert_allclose(got, ref[i], rtol=0, atol=1e-12)


def _explicit(q, qr, c, kr, WUK, WUV, scale, n):
    """Non-absorbed MLA for one head: k_t = W^UK c_t, v_t = W^UV c_t, decoupled RoPE term."""
    k = c[:n] @ WUK.T
    v = c[:n] @ WUV.T
    s = scale * (k @ q + kr[:n] @ qr)
    m = s.max()
    lse = m + math.log(np.exp(s - m).sum())
    return np.exp(s - lse) @ v, lse, s


@pytest.mark.parametrize("causal", [False, True])
def test_absorbed_equals_explicit(causal):
    """q.(W^UK c) + qR.kR with values W^UV c  ==  W^UV (absorbed output), lse equal."""
    B, Sq, H, r, d_r, dh, bs = 3, 2 if causal else 1, 5, 12, 4, 6, 8
    lens = [1 + Sq, 29, 40]
    Lmax = max(lens)
    c = RNG.standard_normal((B, Lmax, r))
    kr = RNG.standard_normal((B, Lmax, d_r))
    WUK = RNG.standard_normal((H, dh, r))
    WUV = RNG.standard_normal((H, dh, r))
    q = RNG.standard_normal((B, Sq, H, dh))
    qr = RNG.standard_normal((B, Sq, H, d_r))
    scale = 1.0 / math.sqrt(dh + d_r)
    q_lat = np.einsum("bshd,hdr->bshr", q, WUK)            # absorbed query (W^UK)^T q
    cache, bt = paged(c, kr, lens, bs, RNG)
    out, lse = oracle.decode(q_lat, qr, cache, bt, np.array(lens, np.int32), scale, causal, block_size=bs)
    for b in range(B):
        for s in range(Sq):
            n = lens[b] - Sq + 1 + s if causal else lens[b]
            for h in range(H):
                o_ref, l_ref, _ = _explicit(q[b, s, h], qr[b, s, h], c[b], kr[b], WUK[h], WUV[h], scale, n)
                np.testing.assert_allclose(WUV[h] @ out[b, s, h], o_ref, rtol=0, atol=1e-11)
                assert abs(lse[b, s, h] - l_ref) < 1e-12


def test_softmax_rows_sum_to_one():
    B, H, r, d_r, bs = 2, 7, 16, 8, 16
    lens = [33, 100]
    c = RNG.standard_normal((B, 100, r))
    kr = RNG.standard_normal((B, 100, d_r))
    q = RNG.standard_normal((B, 1, H, r)) * 2
    qr = RNG.standard_normal((B, 1, H, d_r)) * 2
    scale = 0.37
    cache, bt = paged(c, kr, lens, bs, RNG)
    out, lse = oracle.decode(q, qr, cache, bt, np.array(lens, np.int32), scale, block_size=bs)
    for b in range(B):
        n = lens[b]
        for h in range(H):
            sig = scale * (c[b, :n] @ q[b, 0, h] + kr[b, :n] @ qr[b, 0, h])
            assert abs(np.exp(sig - lse[b, 0, h]).sum() - 1.0) < 1e-12


def test_closed_forms():
    """scale = 0: out = mean of latents, lse = ln n.  n = 1: out = c_0, lse = its score."""
    B, H, r, d_r, bs = 2, 3, 9, 3, 4
    lens = [1, 23]
    c = RNG.standard_normal((B, 23, r))
    kr = RNG.standard_normal((B, 23, d_r))
    q = RNG.standard_normal((B, 1, H, r))
    qr = RNG.standard_normal((B, 1, H, d_r))
    cache, bt = paged(c, kr, lens, bs, RNG)
    out, lse = oracle.decode(q, qr, cache, bt, np.array(lens, np.int32), 0.0, block_size=bs)
    for b in range(B):
        for h in range(H):
            np.testing.assert_allclose(out[b, 0, h], c[b, :lens[b]].mean(0), rtol=0, atol=1e-13)
            assert abs(lse[b, 0, h] - math.log(lens[b])) < 1e-14
    out, lse = oracle.decode(q, qr, cache, bt, np.array(lens, np.int32), 0.25, block_size=bs)
    for h in range(H):
        np.testing.assert_array_equal(out[0, 0, h], c[0, 0])
        assert abs(lse[0, 0, h] - 0.25 * (q[0, 0, h] @ c[0, 0] + qr[0, 0, h] @ kr[0, 0])) < 1e-13


def test_empty_rows():
    """Rows that see no token: out = 0, lse = -inf (L = 0, and causal L < Sq)."""
    B, Sq, H, r, d_r, bs = 3, 2, 2, 4, 2, 4
    lens = [0, 1, 5]
    c = RNG.standard_normal((B, 5, r))
    kr = RNG.standard_normal((B, 5, d_r))
    cache, bt = paged(c, kr, lens, bs, RNG)
    q = RNG.standard_normal((B, Sq, H, r))
    qr = RNG.standard_normal((B, Sq, H, d_r))
    out, lse = oracle.decode(q, qr, cache, bt, np.array(lens, np.int32), 0.5, True, block_size=bs)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(out[1, 0] == 0) and np.all(np.isneginf(lse[1, 0]))      # sees L-Sq+1 = 0 tokens
    assert np.all(np.isfinite(lse[1, 1])) and np.all(np.isfinite(lse[2]))


def test_window_merge_equals_full():
    """Partials over disjoint token windows, merged by log-sum-exp, equal the full decode."""
    B, Sq, H, r, d_r, bs = 3, 2, 4, 10, 4, 8
    lens = [70, 9, 130]
    c = RNG.standard_normal((B, 130, r))
    kr = RNG.standard_normal((B, 130, d_r))
    cache, bt = paged(c, kr, lens, bs, RNG)
    q = RNG.standard_normal((B, Sq, H, r))
    qr = RNG.standard_normal((B, Sq, H, d_r))
    L = np.array(lens, np.int32)
    full_o, full_l = oracle.decode(q, qr, cache, bt, L, 0.3, True, block_size=bs)
    cuts = [np.zeros(B, np.int64), np.array([16, 8, 40]), np.array([64, 8, 41]), np.array(lens, np.int64)]
    parts = [oracle.decode(q, qr, cache, bt, L, 0.3, True, block_size=bs, tok_begin=cuts[i], tok_end=cuts[i + 1])
             for i in range(3)]
    mo, ml = oracle.merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    np.testing.assert_allclose(mo, full_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(ml, full_l, rtol=0, atol=1e-12)


def test_causal_rows_equal_shorter_sequences():
    """Causal query s of Sq sees exactly the first L - Sq + 1 + s tokens."""
    B, Sq, H, r, d_r, bs = 2, 3, 3, 8, 4, 4
    lens = np.array([11, 30], np.int32)
    c = RNG.standard_normal((B, 30, r))
    kr = RNG.standard_normal((B, 30, d_r))
    cache, bt = paged(c, kr, lens, bs, RNG)
    q = RNG.standard_normal((B, Sq, H, r))
    qr = RNG.standard_normal((B, Sq, H, d_r))
    o, l = oracle.decode(q, qr, cache, bt, lens, 0.4, True, block_size=bs)
    for s in range(Sq):
        o1, l1 = oracle.decode(q[:, s:s + 1], qr[:, s:s + 1], cache, bt, lens - Sq + 1 + s, 0.4, False,
                               block_size=bs)
        np.testing.assert_array_equal(o[:, s], o1[:, 0])
        np.testing.assert_array_equal(l[:, s], l1[:, 0])


def test_paging_is_invisible():
    """The same sequences under two different physical layouts give identical results."""
    B, H, r, d_r = 3, 4, 6, 2
    lens = [5, 17, 33]
    c = RNG.standard_normal((B, 33, r))
    kr = RNG.standard_normal((B, 33, d_r))
    q = RNG.standard_normal((B, 1, H, r))
    qr = RNG.standard_normal((B, 1, H, d_r))
    L = np.array(lens, np.int32)
    res = []
    for bs, seed in [(4, 1), (4, 2), (8, 3), (64, 4)]:
        cache, bt = paged(c, kr, lens, bs, np.random.default_rng(seed), spare=3)
        res.append(oracle.decode(q, qr, cache, bt, L, 0.5, block_size=bs))
    for o, l in res[1:]:
        np.testing.assert_array_equal(o, res[0][0])
        np.testing.assert_array_equal(l, res[0][1])


def test_rows_api_matches_full():
    import workloads as W
    inp = W.make_inputs(W.WORKLOADS[3].with_(B=3, seq_lens=(70, 2, 129)))
    o, l = oracle.decode_inputs(inp)
    rows = [(0, 0, 5), (1, 0, 0), (1, 1, 127), (2, 1, 64), (2, 0, 3)]
    ro, rl = oracle.decode_rows_inputs(inp, rows)
    for i, (b, s, h) in enumerate(rows):
        np.testing.assert_array_equal(ro[i], o[b, s, h])
        assert rl[i] == l[b, s, h] or (np.isneginf(rl[i]) and np.isneginf(l[b, s, h]))


# ----------------------------------------------------------------------------- brute force
def test_mpmath_bruteforce_tiny():
    """50-digit brute force on paged causal inputs; oracle agrees to 1e-13.

    The reference rebuilds each sequence from the physical blocks by inverting the
    block table, and evaluates softmax as exp(s_t) / sum exp(s_u) without shifting.
    """
    mp = pytest.importorskip("mpmath")
    mp.mp.dps = 50
    B, Sq, H, r, d_r, bs = 2, 2, 3, 5, 3, 4
    lens = [7, 3]
    c = RNG.standard_normal((B, 7, r)).astype(np.float32).astype(np.float64)
    kr = RNG.standard_normal((B, 7, d_r)).astype(np.float32).astype(np.float64)
    cache, bt = paged(c, kr, lens, bs, RNG, spare=2)
    cache32 = cache.astype(np.float32)
    q = RNG.standard_normal((B, Sq, H, r)).astype(np.float32)
    qr = RNG.standard_normal((B, Sq, H, d_r)).astype(np.float32)
    scale = 0.61
    out, lse = oracle.decode(q, qr, cache32, bt, np.array(lens, np.int32), scale, True, block_size=bs)
    # invert the block table: physical block -> (sequence, logical block)
    owner = {}
    for b in range(B):
        for i in range(bt.shape[1]):
            if bt[b, i] >= 0:
                owner[int(bt[b, i])] = (b, i)
    seqs = {b: {} for b in range(B)}
    for blk in range(cache32.shape[0]):
        if blk not in owner:
            continue
        b, i = owner[blk]
        for o in range(bs):
            t = i * bs + o
            if t < lens[b]:
                seqs[b][t] = [mp.mpf(float(x)) for x in cache32[blk, o]]
    for b in range(B):
        for s in range(Sq):
            n = lens[b] - (Sq - 1 - s)
            for h in range(H):
                qv = [mp.mpf(float(x)) for x in q[b, s, h]] + [mp.mpf(float(x)) for x in qr[b, s, h]]
                sc = [mp.mpf(scale) * mp.fsum(qv[k] * seqs[b][t][k] for k in range(r + d_r)) for t in range(n)]
                den = mp.fsum(mp.exp(x) for x in sc)
                for k in range(r):
                    ref = mp.fsum(mp.exp(sc[t]) * seqs[b][t][k] for t in range(n)) / den
                    assert abs(float(ref) - out[b, s, h, k]) < 1e-13
                assert abs(float(mp.log(den)) - lse[b, s, h]) < 1e-13


# ----------------------------------------------------------------------------- storage decoders
def test_bf16_decoder_matches_torch():
    torch = pytest.importorskip("torch")
    bits = np.arange(0, 1 << 16, 97, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().double().numpy()
    got = np.array([oracle.bf16_to_double(int(x)) for x in bits])
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.all(both_nan | (ref == got))


def test_e4m3_decoder_matches_torch_all_codes():
    torch = pytest.importorskip("torch")
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().double().numpy()
    got = np.array([oracle.e4m3_to_double(int(x)) for x in codes])
    nan = np.isnan(ref)
    assert set(np.nonzero(nan)[0]) == {0x7F, 0xFF}
    assert np.all(np.isnan(got[nan]))
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_fp8_cache_equals_dequantized_cache():
    """The e4m3 path equals the f64 path run on code * scale (torch-decoded), k_rope from its plane."""
    torch = pytest.importorskip("torch")
    import workloads as W
    inp = W.make_inputs(W.WORKLOADS[4].with_(B=2, seq_lens=(75, 130), H=6))
    codes, kr, sc = inp["kv_cache"], inp["k_rope_cache"], inp["kv_scale"]
    lat = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy() * sc.astype(np.float64)[..., None]
    rope = torch.from_numpy(kr.view(np.int16)).view(torch.bfloat16).double().numpy()
    dense = np.concatenate([lat, rope], -1)
    w = inp["workload"]
    o8, l8 = oracle.decode_inputs(inp)
    of, lf = oracle.decode(inp["q_lat"], inp["q_rope"], dense, inp["block_table"], inp["seq_lens"],
                           w.scale, w.causal)
    np.testing.assert_array_equal(o8, of)
    np.testing.assert_array_equal(l8, lf)
    assert np.isfinite(o8).all()          # poisoned slots were never read


def test_rejects_bad_indices():
    inp = dict(q_lat=np.zeros((1, 1, 1, 4)), q_rope=np.zeros((1, 1, 1, 0)),
               kv_cache=np.zeros((2, 4, 4)), block_table=np.array([[0, 5]], np.int32))
    with pytest.raises(RuntimeError, match="block id"):
        oracle.decode(inp["q_lat"], inp["q_rope"], inp["kv_cache"], inp["block_table"],
                      np.array([6], np.int32), 1.0, block_size=4)
    with pytest.raises(RuntimeError, match="seq_len"):
        oracle.decode(inp["q_lat"], inp["q_rope"], inp["kv_cache"], inp["block_table"],
                      np.array([9], np.int32), 1.0, block_size=4)


# ----------------------------------------------------------------------------- byte accounting
def test_byte_accounting(golden_dir):
    import workloads as W
    G = json.load(open(os.path.join(golden_dir, "byte_accounting.json")))
    per_tok = W.cache_bytes_per_token(G["d_c"], G["d_r"], W.BF16)
    assert per_tok == 1152
    assert round(per_tok * G["layers"] / 1024, 1) == G["per_token_kib_all_layers"]
    assert round(G["tpla_tokens"] * per_tok / 1e6, 1) == G["tpla_mb"]
    # FLOPs per (head, token) = 2 (r + d_r) for the score + 2 r for the weighted sum
    ai = G["h_q"] * 2 * (2 * G["d_c"] + G["d_r"]) / per_tok
    assert abs(ai - G["ai_approx"]) / G["ai_approx"] < 0.07
