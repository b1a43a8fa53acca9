"""GPU parity of the sparse-attention (DSA) path against the oracle: the FP8 lightning
indexer (mla_dsa_index), the top-k selection (mla_dsa_topk) and the decode over the
selected tokens (mla_sparse_decode).

Tolerances:
  * indexer scores: the kernel sums 128 exact e4m3 products per head on the tensor cores
    (4 MMAs of 32) and the 64 weighted heads in fp32. With S_t = sum_j |w_j| |q_scale_j
    k_scale_t| sum_d |q_jd k_td|, a full fp32 accumulator gives |I_gpu - I| <= ~200 u S_t
    (u = 2^-24). FP8 MMAs could align their products to a narrower accumulator (about 14
    mantissa bits on the previous generation); on B200 the worst error measured over the
    small workloads is 1.4e-8 S_t, below u S_t, so the sum is full fp32 and the test allows
    2e-5 S_t (about 330 u) and prints the worst observed fraction of it.
    With small-integer codes, unit scales and integer weights every partial sum is an
    integer below 2^24, so the scores are exact and compared bit for bit.
  * top-k: bit-exact against the oracle's selection on the same fp32 scores (seeded inputs,
    with ties, -0/+0 and -inf), and, on the indexer's own scores, a valid selection of the
    oracle's scores within the score tolerance (near-ties may go either way).
  * sparse decode: the decode's bf16 bound (max|d|/max|ref| <= 1e-2, lse within 1e-3) on
    lists chosen by the oracle or drawn by the seeded generator.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workloads as W
from parity_util import LSE_TOL, TOL, compare

pytestmark = pytest.mark.gpu

SCORE_TOL = 2e-5   # of S_t (module docstring)


def _torch():
    import torch
    return torch


def _dev(a):
    torch = _torch()
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _mla():
    import head_latent_attention_split_b200 as mla
    return mla


def _status_ok():
    mla = _mla()
    _torch().cuda.synchronize()
    st = mla.device_status()
    assert st == 0, mla.status_string(st)


def e4m3_lib(codes):
    torch = _torch()
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def score_bound(inp, b, s, n):
    """S_t for tokens [0, n) of query row (b, s) (see the module docstring)."""
    bt = inp["block_table"]
    t = np.arange(n)
    blk, slot = bt[b, t // 64], t % 64
    K = np.abs(e4m3_lib(inp["ik_codes"][blk, slot])) * np.abs(inp["ik_scale"][blk, slot]).astype(np.float64)[:, None]
    Q = np.abs(e4m3_lib(inp["iq_codes"][b, s])) * np.abs(inp["iq_scale"][b, s]).astype(np.float64)[:, None]
    return K @ (Q.T @ np.abs(inp["iw"][b, s]).astype(np.float64))


def gpu_index(inp, causal=False, sentinel=-12345.0):
    torch = _torch()
    mla = _mla()
    w = inp["workload"]
    L = inp["max_seq_len"]
    scores = torch.full((w.B, w.Sq, L), sentinel, dtype=torch.float32, device="cuda")
    mla.dsa_index(_dev(inp["iq_codes"]), _dev(inp["iq_scale"]), _dev(inp["iw"]), _dev(inp["ik_codes"]),
                  _dev(inp["ik_scale"]), _dev(inp["block_table"]), _dev(inp["seq_lens"]), L, scores=scores,
                  causal=causal)
    _status_ok()
    return scores


def oracle_index(inp, causal=False):
    return oracle.dsa_index(inp["iq_codes"], inp["iq_scale"], inp["iw"], inp["ik_codes"], inp["ik_scale"],
                            inp["block_table"], inp["seq_lens"], causal=causal, max_seq_len=inp["max_seq_len"])


@pytest.fixture(scope="module")
def small():
    return W.make_dsa_inputs(W.DSA_BY_NAME["dsa_small"])


@pytest.fixture(scope="module")
def small_causal():
    w = W.DSA_BY_NAME["dsa_small"]
    w2 = W.DsaWorkload("dsa_small_mtp", w.mla.with_(Sq=2, causal=True, seed=1102), top_k=w.top_k)
    return W.make_dsa_inputs(w2)


# ----------------------------------------------------------------------------- indexer
@pytest.mark.parametrize("which", ["small", "small_causal"])
def test_index_parity(which, request):
    inp = request.getfixturevalue(which)
    w = inp["workload"]
    g = gpu_index(inp, causal=w.causal).cpu().numpy().astype(np.float64)
    ref = oracle_index(inp, causal=w.causal)
    n = oracle.attended_counts(inp["seq_lens"], w.Sq, w.causal)
    for b in range(w.B):
        for s in range(w.Sq):
            k = int(n[b, s])
            gr, rr = g[b, s, :k], ref[b, s, :k]
            assert np.isfinite(gr).all()
            tol = SCORE_TOL * score_bound(inp, b, s, k) + 1e-30
            err = np.abs(gr - rr)
            print(f"indexer row {(b, s)}: worst error {np.max(err / tol):.3g} of the bound")
            assert (err <= tol).all(), f"row {(b, s)}: worst {np.max(err / tol):.2f} x tolerance"
            assert np.all(g[b, s, k:] == -12345.0), "wrote past the row's attended tokens"


def integer_problem(seed, B=3, lens=(200, 1300, 777), Sq=1):
    """Codes of small integers, unit scales, integer weights: every score is exact in fp32."""
    torch = _torch()
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, np.int32)
    nb_seq = [(int(L) + 63) // 64 for L in lens]
    nb = sum(nb_seq) + 2
    perm = rng.permutation(nb).astype(np.int32)
    bt = np.full((B, max(nb_seq)), -1, np.int32)
    off = 0
    for b in range(B):
        bt[b, :nb_seq[b]] = perm[off:off + nb_seq[b]]
        off += nb_seq[b]

    def codes(shape):
        v = rng.integers(-4, 5, size=shape).astype(np.float32)
        return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()

    return dict(iq_codes=codes((B, Sq, 64, 128)), iq_scale=np.ones((B, Sq, 64), np.float32),
                iw=rng.integers(-2, 3, size=(B, Sq, 64)).astype(np.float32), ik_codes=codes((nb, 64, 128)),
                ik_scale=np.ones((nb, 64), np.float32), block_table=bt, seq_lens=lens, max_seq_len=int(lens.max()),
                num_blocks=nb, workload=W.Workload(name="int", B=B, Sq=Sq, H=1, r=2, d_r=0, seq_lens=tuple(lens)))


def test_index_and_topk_integer_scores_bit_exact():
    inp = integer_problem(5)
    g = gpu_index(inp).cpu().numpy()
    ref = oracle_index(inp)
    n = oracle.attended_counts(inp["seq_lens"], 1, False)
    for b in range(3):
        k = int(n[b, 0])
        np.testing.assert_array_equal(g[b, 0, :k].astype(np.float64), ref[b, 0, :k])
    # many equal scores: the tie rule decides; both sides see the same values
    mla = _mla()
    for top_k in (1, 64, 700, 2048):
        idx, cnt = mla.dsa_topk(_dev(g), _dev(inp["seq_lens"]), top_k)
        _status_ok()
        ridx, rcnt = oracle.dsa_topk(np.nan_to_num(ref.astype(np.float32), nan=-np.inf), n, top_k)
        np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
        np.testing.assert_array_equal(idx.cpu().numpy(), ridx)


# ----------------------------------------------------------------------------- top-k
def topk_case(seed, rows, L, tie_levels=None):
    rng = np.random.default_rng(seed)
    if tie_levels:
        s = rng.integers(0, tie_levels, size=(rows, 1, L)).astype(np.float32) - tie_levels / 2
    else:
        s = rng.standard_normal((rows, 1, L)).astype(np.float32)
    return s


@pytest.mark.parametrize("L,top_k,ties", [(70000, 2048, None), (70000, 2048, 50), (5000, 1, None), (5000, 4999, 7),
                                          (9000, 4096, 3), (300, 512, None),
                                          (140000, 2048, 9)])   # slices beyond the register-resident size
def test_topk_bit_exact(L, top_k, ties):
    mla = _mla()
    s = topk_case(L + top_k, 4, L, ties)
    s[0, 0, 17] = -0.0
    s[0, 0, 18] = 0.0
    s[1, 0, :5] = -np.inf
    lens = np.array([L, L - 1, max(L // 3, 0), 0], np.int32)
    idx, cnt = mla.dsa_topk(_dev(s), _dev(lens), top_k)
    _status_ok()
    ridx, rcnt = oracle.dsa_topk(s, lens.reshape(4, 1), top_k)
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)


def test_topk_causal_rows():
    mla = _mla()
    s = topk_case(3, 2, 3000).reshape(1, 2, 3000)
    lens = np.array([3000], np.int32)
    idx, cnt = mla.dsa_topk(_dev(s), _dev(lens), 2999, causal=True)
    _status_ok()
    ridx, rcnt = oracle.dsa_topk(s, oracle.attended_counts(lens, 2, True), 2999)
    assert rcnt.tolist() == [[2999, 2999]]
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)


# ----------------------------------------------------------------------------- sparse decode
SPARSE_KERNELS = ["tcgen05", "tc_pair"]


def gpu_sparse(inp, idx, cnt, kernel="auto"):
    mla = _mla()
    w = inp["workload"]
    t = W.to_torch(inp)
    out, lse = mla.sparse_decode(t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], _dev(idx), _dev(cnt),
                                 w.scale, kernel=kernel)
    _status_ok()
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


def oracle_sparse(inp, idx, cnt):
    w = inp["workload"]
    return oracle.decode_sparse(inp["q_lat"], inp["q_rope"], inp["kv_cache"], inp["block_table"], inp["seq_lens"],
                                w.scale, idx.reshape(w.B, 1, -1), cnt.reshape(w.B, 1))


@pytest.mark.parametrize("kernel", SPARSE_KERNELS)
def test_sparse_decode_on_the_oracle_selection(small, kernel):
    inp = small
    k = inp["top_k"]
    ref_scores = oracle_index(inp)
    n = oracle.attended_counts(inp["seq_lens"], 1, False)
    idx, cnt = oracle.dsa_topk(np.nan_to_num(ref_scores, nan=-np.inf), n, k)
    assert cnt.ravel().tolist() == [300, 512, 512]    # one row keeps all of its tokens
    out, lse = gpu_sparse(inp, idx[:, 0], cnt[:, 0], kernel)
    ro, rl = oracle_sparse(inp, idx[:, 0], cnt[:, 0])
    compare(out, lse, ro, rl, TOL[W.BF16], "sparse decode")


@pytest.mark.parametrize("kernel", SPARSE_KERNELS)
def test_sparse_decode_random_lists_and_edges(small, kernel):
    inp = small
    rng = np.random.default_rng(11)
    k = 200
    lens = inp["seq_lens"]
    idx = np.full((3, k), -1, np.int32)
    cnt = np.array([0, k, 77], np.int32)                # empty list, full list, ragged tail
    for b in range(3):
        if cnt[b]:
            idx[b, :cnt[b]] = rng.choice(int(lens[b]), size=int(cnt[b]), replace=False)   # any order
    out, lse = gpu_sparse(inp, idx, cnt, kernel)
    ro, rl = oracle_sparse(inp, idx, cnt)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    compare(out, lse, ro, rl, TOL[W.BF16], "sparse decode, random lists")


@pytest.mark.parametrize("kernel", SPARSE_KERNELS)
def test_sparse_decode_wait_timeout_expires_cleanly(small, kernel):
    """A pipeline wait limit far below a tile's time makes the sparse decode's waits run out
    (both copy warps and the consumers): the call returns, the status reads MLA_ERR_TIMEOUT
    once, every row is NaN throughout or right, and the next call at the default limit
    matches the oracle."""
    torch = _torch()
    mla = _mla()
    inp = small
    rng = np.random.default_rng(5)
    k = 512
    lens = inp["seq_lens"]
    cnt = np.minimum(lens, k).astype(np.int32)
    idx = np.full((3, k), -1, np.int32)
    for b in range(3):
        idx[b, :cnt[b]] = rng.choice(int(lens[b]), size=int(cnt[b]), replace=False)
    ro, rl = oracle_sparse(inp, idx, cnt)
    w = inp["workload"]
    t = W.to_torch(inp)
    assert mla.wait_timeout_ns() == 2_000_000_000
    mla.set_wait_timeout_ns(200)
    try:
        out, lse = mla.sparse_decode(t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], _dev(idx),
                                     _dev(cnt), w.scale, kernel=kernel)
        torch.cuda.synchronize()
    finally:
        mla.set_wait_timeout_ns(0)
    assert mla.wait_timeout_ns() == 2_000_000_000
    assert mla.device_status() == 8           # MLA_ERR_TIMEOUT
    assert mla.device_status() == 0
    o = out.double().cpu().numpy()
    l = lse.double().cpu().numpy()
    assert np.isnan(l).any()
    for b in range(w.B):
        for h in range(w.H):
            if np.isnan(l[b, 0, h]):
                assert np.isnan(o[b, 0, h]).all()
            else:
                assert abs(l[b, 0, h] - rl[b, 0, h]) <= LSE_TOL
    out2, lse2 = gpu_sparse(inp, idx, cnt, kernel)
    compare(out2, lse2, ro, rl, TOL[W.BF16], "sparse decode after the timeout")


@pytest.mark.parametrize("kernel", SPARSE_KERNELS)
def test_sparse_decode_every_token_is_dense(small, kernel):
    # a list holding every position equals the dense decode (the oracle's dense decode)
    inp = small
    lens = inp["seq_lens"]
    k = int(lens.max())
    idx = np.full((3, k), -1, np.int32)
    for b in range(3):
        idx[b, :lens[b]] = np.arange(lens[b])
    out, lse = gpu_sparse(inp, idx, lens.astype(np.int32), kernel)
    ro, rl = oracle.decode_inputs(inp)
    compare(out, lse, ro, rl, TOL[W.BF16], "sparse == dense")


def test_pipeline_integer_scores_matches_oracle_pipeline(small):
    # index -> top-k -> sparse decode on the GPU, against the same three steps of the
    # oracle; the indexer inputs are small integers so both sides select identical sets
    mla = _mla()
    torch = _torch()
    inp = dict(small)
    ip = integer_problem(8, B=3, lens=tuple(int(x) for x in small["seq_lens"]))
    ip["block_table"] = inp["block_table"]
    ip["ik_codes"] = np.resize(ip["ik_codes"], (inp["num_blocks"], 64, 128))
    ip["ik_scale"] = np.ones((inp["num_blocks"], 64), np.float32)
    inp.update({k: ip[k] for k in ("iq_codes", "iq_scale", "iw", "ik_codes", "ik_scale")})
    k = 512
    g = gpu_index(inp)
    idx, cnt = mla.dsa_topk(g, _dev(inp["seq_lens"]), k)
    t = W.to_torch(inp)
    out, lse = mla.sparse_decode(t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], idx[:, 0], cnt[:, 0],
                                 inp["workload"].scale)
    _status_ok()
    ref = oracle_index(inp)
    n = oracle.attended_counts(inp["seq_lens"], 1, False)
    ridx, rcnt = oracle.dsa_topk(np.nan_to_num(ref, nan=-np.inf), n, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    ro, rl = oracle_sparse(inp, ridx[:, 0], rcnt[:, 0])
    compare(out.double().cpu().numpy(), lse.double().cpu().numpy(), ro, rl, TOL[W.BF16], "pipeline")
    assert torch.equal(cnt.cpu(), torch.from_numpy(rcnt))


# ----------------------------------------------------------------------------- full size
@pytest.fixture(scope="module")
def full():
    return W.make_dsa_inputs(W.DSA_BY_NAME["dsa_v32"])


def test_full_size_sampled_rows(full):
    """DeepSeek-V3.2 shapes (B=32, 128K context, 64 x 128 indexer, k=2048): indexer scores
    and selection validity on sampled rows; the decode on seeded lists, sampled rows."""
    mla = _mla()
    inp = full
    w = inp["workload"]
    k = inp["top_k"]
    g = gpu_index(inp)
    idx, cnt = mla.dsa_topk(g, _dev(inp["seq_lens"]), k)
    _status_ok()
    gi = idx.cpu().numpy()
    assert (cnt.cpu().numpy() == k).all()
    rows = [0, w.B - 1]
    for b in rows:
        L = int(inp["seq_lens"][b])
        sub = dict(inp)
        sub["seq_lens"] = inp["seq_lens"][b:b + 1]
        sub["block_table"] = inp["block_table"][b:b + 1]
        for key in ("iq_codes", "iq_scale", "iw"):
            sub[key] = inp[key][b:b + 1]
        ref = oracle.dsa_index(sub["iq_codes"], sub["iq_scale"], sub["iw"], sub["ik_codes"], sub["ik_scale"],
                               sub["block_table"], sub["seq_lens"], max_seq_len=L)[0, 0]
        tol = SCORE_TOL * score_bound(inp, b, 0, L) + 1e-30
        gr = g[b, 0, :L].cpu().numpy().astype(np.float64)
        assert (np.abs(gr - ref) <= tol).all()
        sel = gi[b, 0]
        assert len(set(sel.tolist())) == k and sel.min() >= 0 and sel.max() < L and (np.diff(sel) > 0).all()
        mask = np.zeros(L, bool)
        mask[sel] = True
        assert (ref[mask] + tol[mask]).min() >= (ref[~mask] - tol[~mask]).max(), "selection not a top-k"
    # decode over seeded lists (sorted distinct positions), compared on sampled rows
    rng = np.random.default_rng(21)
    lst = np.stack([np.sort(rng.choice(int(L), size=k, replace=False)) for L in inp["seq_lens"]]).astype(np.int32)
    cnts = np.full(w.B, k, np.int32)
    outs = {kern: gpu_sparse(inp, lst, cnts, kern) for kern in SPARSE_KERNELS}
    for b in rows:
        sub = {key: inp[key] for key in ("kv_cache", "k_rope_cache", "kv_scale")}
        ro, rl = oracle.decode_sparse(inp["q_lat"][b:b + 1], inp["q_rope"][b:b + 1], sub["kv_cache"],
                                      inp["block_table"][b:b + 1], inp["seq_lens"][b:b + 1], w.scale,
                                      lst[b:b + 1].reshape(1, 1, k), cnts[b:b + 1].reshape(1, 1))
        for kern, (out, lse) in outs.items():
            compare(out[b:b + 1], lse[b:b + 1], ro, rl, TOL[W.BF16], f"full-size sparse decode ({kern}) b={b}")


# ----------------------------------------------------------------------------- error paths
def test_index_bad_block_id_and_seq_len_set_status(small):
    """A block id outside [0, num_blocks) marks its tokens NaN and sets MLA_ERR_BAD_BLOCK_ID; a
    seq_len above max_seq_len skips the row and sets MLA_ERR_BAD_SEQ_LEN. Neither loads past the
    cache (the bad block is not fetched)."""
    torch = _torch()
    mla = _mla()
    inp = dict(small)
    bt = inp["block_table"].copy()
    bt[1, 3] = inp["num_blocks"] + 7               # tokens [192, 256) of sequence 1
    inp["block_table"] = bt
    w = inp["workload"]
    L = inp["max_seq_len"]
    scores = torch.full((w.B, 1, L), -12345.0, dtype=torch.float32, device="cuda")
    mla.dsa_index(_dev(inp["iq_codes"]), _dev(inp["iq_scale"]), _dev(inp["iw"]), _dev(inp["ik_codes"]),
                  _dev(inp["ik_scale"]), _dev(bt), _dev(inp["seq_lens"]), L, scores=scores)
    torch.cuda.synchronize()
    assert mla.device_status() == 6                 # MLA_ERR_BAD_BLOCK_ID (read and cleared)
    assert mla.device_status() == 0
    g = scores.cpu().numpy()
    assert np.isnan(g[1, 0, 192:256]).all() and np.isfinite(g[1, 0, :192]).all()
    assert np.isfinite(g[1, 0, 256:4100]).all() and np.isfinite(g[0, 0, :300]).all()
    sl = inp["seq_lens"].copy()
    sl[2] = L + 1                                   # longer than the score rows
    scores.fill_(-12345.0)
    mla.dsa_index(_dev(inp["iq_codes"]), _dev(inp["iq_scale"]), _dev(inp["iw"]), _dev(inp["ik_codes"]),
                  _dev(inp["ik_scale"]), _dev(small["block_table"]), _dev(sl), L, scores=scores)
    idx, cnt = mla.dsa_topk(scores, _dev(sl), 64)
    torch.cuda.synchronize()
    assert mla.device_status() == 7                 # MLA_ERR_BAD_SEQ_LEN
    g = scores.cpu().numpy()
    assert (g[2] == -12345.0).all() and np.isfinite(g[0, 0, :300]).all()
    assert cnt.cpu().numpy()[2, 0] == 0 and (idx.cpu().numpy()[2] == -1).all()


@pytest.mark.parametrize("kernel", SPARSE_KERNELS)
def test_sparse_decode_bad_position_sets_status(small, kernel):
    """A listed position outside the block table's range sets MLA_ERR_BAD_BLOCK_ID and turns that
    sequence's rows NaN; the other sequences are unaffected."""
    torch = _torch()
    inp = small
    rng = np.random.default_rng(5)
    k = 64
    idx = np.stack([np.sort(rng.choice(int(L), size=k, replace=False)) for L in inp["seq_lens"]]).astype(np.int32)
    cnt = np.full(3, k, np.int32)
    bad = idx.copy()
    bad[1, 10] = inp["block_table"].shape[1] * 64 + 3
    mla = _mla()
    w = inp["workload"]
    t = W.to_torch(inp)
    out, lse = mla.sparse_decode(t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], _dev(bad), _dev(cnt),
                                 w.scale, kernel=kernel)
    torch.cuda.synchronize()
    assert mla.device_status() == 6
    o, l = out.double().cpu().numpy(), lse.double().cpu().numpy()
    assert np.isnan(o[1]).all() and np.isnan(l[1]).all()
    ro, rl = oracle_sparse(inp, idx, cnt)
    keep = [0, 2]
    compare(o[keep], l[keep], ro[keep], rl[keep], TOL[W.BF16], "sequences without the bad position")


@pytest.mark.parametrize("kernel", SPARSE_KERNELS)
def test_sparse_decode_count_above_top_k_sets_status(small, kernel):
    """A count above top_k (the list's row stride) is an error: MLA_ERR_BAD_SEQ_LEN, that
    sequence's rows NaN, nothing read past its list; the other sequences are unaffected."""
    torch = _torch()
    inp = small
    rng = np.random.default_rng(6)
    k = 64
    idx = np.stack([np.sort(rng.choice(int(L), size=k, replace=False)) for L in inp["seq_lens"]]).astype(np.int32)
    cnt = np.full(3, k, np.int32)
    bad = cnt.copy()
    bad[2] = k + 5          # the last row: a read past the count would run off the indices buffer
    mla = _mla()
    w = inp["workload"]
    t = W.to_torch(inp)
    out, lse = mla.sparse_decode(t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], _dev(idx), _dev(bad),
                                 w.scale, kernel=kernel)
    torch.cuda.synchronize()
    assert mla.device_status() == 7
    o, l = out.double().cpu().numpy(), lse.double().cpu().numpy()
    assert np.isnan(o[2]).all() and np.isnan(l[2]).all()
    ro, rl = oracle_sparse(inp, idx, cnt)
    keep = [0, 1]
    compare(o[keep], l[keep], ro[keep], rl[keep], TOL[W.BF16], "sequences with a valid count")
