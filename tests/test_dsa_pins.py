"""Pins of the sparse-attention (DSA) oracle functions, on the CPU.

Pages: "TransMLA & Sparse Latent Attention" lesson, Chapter 6 ("The lightning indexer",
"Fine-grained token selection", "Worked arithmetic", "A sanity check on the formula
itself") and Chapter 7 ("DSA runs in MLA's MQA mode").

Each oracle function is held to something other than itself: the pages' worked counts,
closed forms, special cases that reduce to a library matmul, invariants (paging,
linearity, homogeneity), a brute-force subset search, and the dense decode (pinned in
test_oracle_pins.py) where the selection keeps every token.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W


def e4m3_lib(codes):
    """e4m3 codes -> float64 through torch's float8_e4m3fn (a library decoder)."""
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).to(
        torch.float64).numpy()


def small_index_problem(seed, B=2, Sq=1, HI=4, dI=16, lens=(70, 130), bs=64, sign_q=None, sign_k=None,
                        contiguous=False):
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, dtype=np.int32)
    nb = [(int(L) + bs - 1) // bs for L in lens]
    num_blocks = sum(nb) + 1
    perm = np.arange(num_blocks, dtype=np.int32) if contiguous else rng.permutation(num_blocks).astype(np.int32)
    bt = np.full((B, max(nb)), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        bt[b, :nb[b]] = perm[off:off + nb[b]]
        off += nb[b]

    def codes(shape, sign):
        c = rng.integers(0, 256, size=shape, dtype=np.uint16).astype(np.uint8)
        c[(c & 0x7F) == 0x7F] &= 0xB0            # no NaN codes (S.1111.111)
        if sign == "+":
            c &= 0x7F
        elif sign == "-":
            c |= 0x80
        return c

    q = codes((B, Sq, HI, dI), sign_q)
    k = codes((num_blocks, bs, dI), sign_k)
    qs = rng.uniform(0.5, 2.0, size=(B, Sq, HI)).astype(np.float32)
    ks = rng.uniform(0.5, 2.0, size=(num_blocks, bs)).astype(np.float32)
    w = rng.standard_normal((B, Sq, HI)).astype(np.float32)
    return dict(q_codes=q, q_scale=qs, weights=w, k_codes=k, k_scale=ks, block_table=bt, seq_lens=lens)


def logical_keys(P, b, n, bs=64):
    """Decoded keys of positions [0, n) of sequence b, [n, dI], via the library decoder."""
    t = np.arange(n)
    blk = P["block_table"][b, t // bs]
    slot = t % bs
    return e4m3_lib(P["k_codes"][blk, slot]) * P["k_scale"][blk, slot].astype(np.float64)[:, None]


# ----------------------------------------------------------------------------- counts

def test_pairs_toy_from_the_pages():
    # Chapter 6, "A sanity check on the formula itself": a 10-token causal generation with a
    # top-3 budget compares 55 query-key pairs densely and 27 under DSA.
    n = oracle.attended_counts([10], Sq=10, causal=True)        # query t sees t tokens
    assert n.tolist() == [list(range(1, 11))]
    assert int(n.sum()) == 55
    assert int(oracle.dsa_counts(n, 3).sum()) == 27


@pytest.mark.parametrize("L,ratio", [(16384, 4.3), (131072, 32.3)])
def test_pairs_ratio_from_the_pages(L, ratio):
    # Chapter 6: with k = 2048, a whole causal generation compares ~4.3x fewer pairs at 16K
    # and ~32.3x fewer at 128K; the last step alone compares L / k = 64x fewer at 128K.
    n = np.arange(1, L + 1)
    dense = int(n.sum())
    sparse = int(oracle.dsa_counts(n, 2048).sum())
    assert round(dense / sparse, 1) == ratio
    assert int(oracle.dsa_counts([131072], 2048)[0]) * 64 == 131072


# ----------------------------------------------------------------------------- indexer

def test_index_relu_zeroes_negative_dots():
    # every q code >= 0 and every k code <= 0: all dots are <= 0, ReLU clamps them, I = 0
    P = small_index_problem(1, sign_q="+", sign_k="-")
    I = oracle.dsa_index(**P)
    for b, L in enumerate(P["seq_lens"]):
        assert np.all(I[b, 0, :L] == 0.0)


def test_index_nonnegative_dots_is_a_matmul():
    # all codes >= 0: ReLU is the identity and I = K (Q^T w), a library matmul
    P = small_index_problem(2, sign_q="+", sign_k="+")
    I = oracle.dsa_index(**P)
    for b, L in enumerate(P["seq_lens"]):
        Q = e4m3_lib(P["q_codes"][b, 0]) * P["q_scale"][b, 0].astype(np.float64)[:, None]   # [HI, dI]
        K = logical_keys(P, b, int(L))
        ref = K @ (Q.T @ P["weights"][b, 0].astype(np.float64))
        np.testing.assert_allclose(I[b, 0, :L], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_index_single_head_is_relu_of_a_matvec():
    P = small_index_problem(3, HI=1)
    P["weights"][:] = 1.0
    I = oracle.dsa_index(**P)
    for b, L in enumerate(P["seq_lens"]):
        q = e4m3_lib(P["q_codes"][b, 0, 0]) * float(P["q_scale"][b, 0, 0])
        ref = np.maximum(0.0, logical_keys(P, b, int(L)) @ q)
        assert (ref > 0).any() and (ref == 0).any()        # both sides of the ReLU are exercised
        np.testing.assert_allclose(I[b, 0, :L], ref, rtol=1e-12, atol=1e-300)


def test_index_linear_in_weights_and_homogeneous_in_scales():
    P = small_index_problem(4)
    rng = np.random.default_rng(5)
    # weights on a 1/8 grid so that their sum is exact in fp32
    P["weights"] = (rng.integers(-16, 17, size=P["weights"].shape) / 8.0).astype(np.float32)
    I = oracle.dsa_index(**P)
    w2 = (rng.integers(-16, 17, size=P["weights"].shape) / 8.0).astype(np.float32)
    Ia = oracle.dsa_index(**{**P, "weights": w2})
    Ib = oracle.dsa_index(**{**P, "weights": (P["weights"] + w2).astype(np.float32)})
    Ik = oracle.dsa_index(**{**P, "k_scale": (P["k_scale"] * np.float32(4.0))})
    for b, L in enumerate(P["seq_lens"]):
        s = slice(0, int(L))
        np.testing.assert_allclose(Ib[b, 0, s], I[b, 0, s] + Ia[b, 0, s], rtol=1e-9, atol=1e-9)
        np.testing.assert_allclose(Ik[b, 0, s], 4.0 * I[b, 0, s], rtol=1e-12, atol=0)


def test_index_paging_and_causal_window():
    # the same logical keys in a contiguous and in a permuted block layout score the same;
    # with Sq = 3 causal, row s sees L - 2 + s tokens and nothing past them is written
    Pc = small_index_problem(6, Sq=3, contiguous=True)
    Pp = dict(Pc)
    rng = np.random.default_rng(7)
    nbk = Pc["k_codes"].shape[0]
    perm = rng.permutation(nbk)               # physical block p of Pp holds block perm[p] of Pc
    inv = np.argsort(perm)
    Pp["k_codes"] = Pc["k_codes"][perm]
    Pp["k_scale"] = Pc["k_scale"][perm]
    bt = Pc["block_table"].copy()
    Pp["block_table"] = np.where(bt >= 0, inv[np.maximum(bt, 0)], -1).astype(np.int32)
    Ic = oracle.dsa_index(**Pc, causal=True)
    Ip = oracle.dsa_index(**Pp, causal=True)
    n = oracle.attended_counts(Pc["seq_lens"], 3, True)
    for b in range(2):
        for s in range(3):
            k = int(n[b, s])
            assert k == int(Pc["seq_lens"][b]) - 2 + s
            np.testing.assert_array_equal(Ic[b, s, :k], Ip[b, s, :k])
            assert np.all(np.isnan(Ic[b, s, k:]))
            assert not np.any(np.isnan(Ic[b, s, :k]))


# ----------------------------------------------------------------------------- top-k

def brute_topk(scores, k):
    """The k-subset of largest sum; among equal sums the smallest sorted position tuple."""
    n = len(scores)
    best, best_key = None, None
    for sub in itertools.combinations(range(n), k):
        key = (-sum(scores[i] for i in sub), sub)
        if best_key is None or key < best_key:
            best, best_key = sub, key
    return list(best)


@pytest.mark.parametrize("seed", range(6))
def test_topk_is_the_largest_sum_subset(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 10))
    scores = rng.integers(-3, 4, size=n).astype(np.float64)     # many ties
    for k in range(1, n + 1):
        idx, cnt = oracle.dsa_topk(scores[None], np.array([n]), k)
        assert int(cnt[0]) == k
        assert idx[0].tolist() == brute_topk(scores.tolist(), k)


def test_topk_short_rows_keep_everything():
    # Chapter 6: below k candidates "the top-k step selects everything"
    s = np.array([[5.0, -1.0, 2.0, 0.0, 9.0, 9.0]])
    idx, cnt = oracle.dsa_topk(s, np.array([4]), 8)
    assert cnt.tolist() == [4] and idx[0].tolist() == [0, 1, 2, 3, -1, -1, -1, -1]
    idx, cnt = oracle.dsa_topk(s, np.array([0]), 2)
    assert cnt.tolist() == [0] and idx[0].tolist() == [-1, -1]
    # +0 and -0 are one value: the tie goes to the lower position
    z = np.array([[-0.0, 0.0, -1.0]])
    idx, _ = oracle.dsa_topk(z, np.array([3]), 1)
    assert idx[0].tolist() == [0]


# ----------------------------------------------------------------------------- sparse decode

@pytest.fixture(scope="module")
def small_mla():
    w = W.WORKLOADS[2].with_(B=2, H=8, seq_lens=(150, 97), seed=77)
    return W.make_inputs(w)


def sparse(inp, idx, cnt):
    w = inp["workload"]
    return oracle.decode_sparse(inp["q_lat"], inp["q_rope"], inp["kv_cache"], inp["block_table"],
                                inp["seq_lens"], w.scale, idx, cnt)


def test_sparse_over_every_token_is_the_dense_decode(small_mla):
    inp = small_mla
    L = inp["seq_lens"]
    k = 160
    idx = np.full((2, 1, k), -1, dtype=np.int32)
    for b in range(2):
        idx[b, 0, :L[b]] = np.arange(L[b])
    cnt = L.reshape(2, 1).astype(np.int32)
    o, l = sparse(inp, idx, cnt)
    od, ld = oracle.decode_inputs(inp)
    np.testing.assert_allclose(o, od, rtol=0, atol=1e-12 * np.abs(od).max())
    np.testing.assert_allclose(l, ld, rtol=0, atol=1e-12)


def test_sparse_contiguous_range_is_the_window_decode_and_order_free(small_mla):
    inp = small_mla
    a, e = np.array([10, 40]), np.array([75, 97])
    k = 70
    idx = np.full((2, 1, k), -1, dtype=np.int32)
    rng = np.random.default_rng(3)
    for b in range(2):
        idx[b, 0, :e[b] - a[b]] = rng.permutation(np.arange(a[b], e[b]))   # any order
    cnt = (e - a).reshape(2, 1).astype(np.int32)
    o, l = sparse(inp, idx, cnt)
    ow, lw = oracle.decode_inputs(inp, tok_begin=a, tok_end=e)
    np.testing.assert_allclose(o, ow, rtol=0, atol=1e-12 * np.abs(ow).max())
    np.testing.assert_allclose(l, lw, rtol=0, atol=1e-12)


def test_sparse_single_token_and_empty_lists(small_mla):
    inp = small_mla
    idx = np.array([[[33, -1]], [[-1, -1]]], dtype=np.int32)
    cnt = np.array([[1], [0]], dtype=np.int32)
    o, l = sparse(inp, idx, cnt)
    # one token: softmax weight 1, out = its latent exactly
    bt, bs = inp["block_table"], 64
    c = W.bf16_bits_to_f32(inp["kv_cache"][bt[0, 33 // bs], 33 % bs, :512]).astype(np.float64)
    np.testing.assert_array_equal(o[0, 0], np.broadcast_to(c, o[0, 0].shape))
    # its lse is the single score: the dense decode of the one-token window
    _, lw = oracle.decode_inputs(inp, tok_begin=np.array([33, 0]), tok_end=np.array([34, 0]))
    np.testing.assert_allclose(l[0, 0], lw[0, 0], rtol=0, atol=1e-12)
    # no token: out = 0, lse = -inf
    assert np.all(o[1] == 0) and np.all(np.isneginf(l[1]))


def test_dsa_with_k_at_least_the_context_is_dense(small_mla):
    # Chapter 6: a context shorter than k leaves nothing to filter, so DSA equals dense
    # attention. Index -> select -> sparse decode against the dense decode.
    inp = small_mla
    rng = np.random.default_rng(9)
    nb = inp["num_blocks"]
    qc = W.quantize_e4m3_per_token(rng.standard_normal((2, 1, 4, 16)).astype(np.float32))
    kc = W.quantize_e4m3_per_token(rng.standard_normal((nb, 64, 16)).astype(np.float32))
    wts = rng.standard_normal((2, 1, 4)).astype(np.float32)
    I = oracle.dsa_index(qc[0], qc[1], wts, kc[0], kc[1], inp["block_table"], inp["seq_lens"])
    n = oracle.attended_counts(inp["seq_lens"], 1, False)
    idx, cnt = oracle.dsa_topk(np.nan_to_num(I, nan=-np.inf), n, 256)
    o, l = sparse(inp, idx, cnt)
    od, ld = oracle.decode_inputs(inp)
    np.testing.assert_allclose(o, od, rtol=0, atol=1e-12 * np.abs(od).max())
    np.testing.assert_allclose(l, ld, rtol=0, atol=1e-12)
    # and with k below the context, each row keeps exactly k of its tokens
    idx, cnt = oracle.dsa_topk(np.nan_to_num(I, nan=-np.inf), n, 64)
    assert cnt.ravel().tolist() == [64, 64]
    assert all(len(set(idx[b, 0].tolist())) == 64 for b in range(2))
    assert math.isfinite(float(sparse(inp, idx, cnt)[1].max()))
