"""CPU-only checks of the C-ABI library: it loads, exports what include/mla_decode.h
declares, rejects bad arguments before touching the GPU, and plans splits as defined."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla_decode.h")


@pytest.fixture(scope="module")
def m():
    from head_latent_attention_split_b200 import build as B
    B.build()
    import head_latent_attention_split_b200 as mod
    return mod


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(mla_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("mla_decode", "mla_decode_workspace_size", "mla_get_device_status", "mla_plan_host"):
        assert n in names


def test_library_exports_every_declared_symbol(m):
    from head_latent_attention_split_b200 import binding
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (mla_\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(binding.lib, name)
    assert set(binding.EXPORTED) <= exported
    assert m.abi_version() == 1


def test_library_has_no_torch_or_libcuda_dependency(m):
    from head_latent_attention_split_b200 import binding
    out = subprocess.run(["readelf", "-d", binding.LIB_PATH], capture_output=True, text=True).stdout
    needed = re.findall(r"\(NEEDED\).*\[(.*)\]", out)
    assert not any("torch" in n or n.startswith("libcuda.so") or "c10" in n for n in needed), needed


def _p(m, **kw):
    base = dict(B=2, Sq=1, H=4, r=16, d_r=8, block_size=64, num_blocks=2, max_blocks_per_seq=1,
                q_dtype=0, cache_dtype=0, out_dtype=0, causal=False, softmax_scale=0.2, num_workers=3,
                kernel="simt")
    base.update(kw)
    return m.make_params(**base)


FAKE = 1 << 20   # a 256-byte aligned address that is never dereferenced


def _call(m, p, **ptrs):
    from head_latent_attention_split_b200 import binding
    args = dict(q_lat=FAKE, q_rope=FAKE, kv_cache=FAKE, k_rope_cache=None, kv_scale=None, block_table=FAKE,
                seq_lens=FAKE, out=FAKE, lse=FAKE, workspace=FAKE, workspace_bytes=1 << 30)
    args.update(ptrs)
    return binding.mla_decode(p, stream=0, check=False, **args)


@pytest.mark.parametrize("bad", [dict(Sq=0), dict(H=0), dict(r=0), dict(d_r=-1), dict(block_size=0),
                                 dict(max_blocks_per_seq=0), dict(q_dtype=7), dict(q_dtype=1),
                                 dict(cache_dtype=2, q_dtype=0), dict(out_dtype=2, q_dtype=1, cache_dtype=1),
                                 dict(softmax_scale=float("nan")), dict(causal=2), dict(kernel=9),
                                 dict(num_workers=-1), dict(num_blocks=0)])
def test_invalid_params_rejected_on_host(m, bad):
    causal = bad.pop("causal", None)
    p = _p(m, **bad)
    if causal is not None:
        p.causal = causal          # make_params would coerce it to 0/1
    assert _call(m, p) == 1     # MLA_ERR_INVALID_ARG, nothing launched


def test_null_pointers_rejected(m):
    p = _p(m)
    for k in ("q_lat", "kv_cache", "block_table", "seq_lens", "out", "lse", "workspace", "q_rope"):
        assert _call(m, p, **{k: None}) == 1, k
    # e4m3 needs its rope plane and scales; f32/bf16 must not get them
    p8 = _p(m, q_dtype=1, cache_dtype=2, out_dtype=1)
    assert _call(m, p8) == 1
    assert _call(m, p, kv_scale=FAKE) == 1


def test_workspace_and_alignment_checks(m):
    p = _p(m)
    need = m.workspace_size(p)
    assert _call(m, p, workspace_bytes=need - 1) == 4           # MLA_ERR_WORKSPACE_TOO_SMALL
    assert _call(m, p, workspace=FAKE + 16, workspace_bytes=need) == 3   # MLA_ERR_ALIGNMENT
    assert _call(m, p, out=FAKE + 2, workspace_bytes=need) == 3


def test_unsupported_kernel_requests(m):
    # the SIMT kernel is limited to r <= 1024, r + d_r <= 1280
    assert _call(m, _p(m, r=2048)) == 2
    # the tensor-core kernel needs r = 512, d_r = 64, block 64, bf16 queries
    assert _call(m, _p(m, kernel="tcgen05")) == 2
    assert _call(m, _p(m, kernel="tc_pair")) == 2
    # the pair kernel reads bf16 caches only
    tc_shape = dict(r=512, d_r=64, block_size=64, q_dtype=1, cache_dtype=1, out_dtype=1)
    assert _call(m, _p(m, kernel="tc_pair", **{**tc_shape, "cache_dtype": 2})) == 2


def test_batch_zero_is_a_noop(m):
    p = _p(m, B=0)
    assert _call(m, p, q_lat=None, kv_cache=None) == 0


def _host_io(m, p, **ptrs):
    from head_latent_attention_split_b200 import binding
    args = dict(q_lat_host=FAKE, q_rope_host=FAKE, kv_cache=FAKE, k_rope_cache=None, kv_scale=None,
                block_table_host=FAKE, seq_lens_host=FAKE, out_host=FAKE, lse_host=FAKE, workspace=FAKE,
                workspace_bytes=1 << 30)
    args.update(ptrs)
    return binding.mla_decode_host_io(p, stream=0, check=False, **args)


def test_host_io_workspace_size_formula(m):
    # device staging of q_lat, q_rope, block_table, seq_lens, out, lse after mla_decode's own
    # workspace, each region 256-byte aligned (f32 queries and output here)
    B, Sq, H, r, d_r, mb = 5, 2, 8, 32, 8, 3
    p = _p(m, B=B, Sq=Sq, H=H, r=r, d_r=d_r, max_blocks_per_seq=mb, num_blocks=16, num_workers=7)
    rows = B * Sq * H
    al = lambda x: (x + 255) // 256 * 256  # noqa: E731
    want = (al(m.workspace_size(p)) + al(rows * r * 4) + al(rows * d_r * 4) + al(B * mb * 4) + al(B * 4)
            + al(rows * r * 4) + al(rows * 4))
    assert m.host_io_workspace_size(p) == want


def test_host_io_rejects_bad_arguments_on_host(m):
    p = _p(m)
    need = m.host_io_workspace_size(p)
    for k in ("q_lat_host", "q_rope_host", "block_table_host", "seq_lens_host", "out_host", "lse_host", "workspace"):
        assert _host_io(m, p, **{k: None}) == 1, k                  # MLA_ERR_INVALID_ARG
    assert _host_io(m, p, workspace_bytes=need - 1) == 4            # MLA_ERR_WORKSPACE_TOO_SMALL
    assert _host_io(m, p, workspace=FAKE + 16, workspace_bytes=need) == 3   # MLA_ERR_ALIGNMENT
    assert _host_io(m, _p(m, Sq=0)) == 1                            # bad params, nothing enqueued
    assert _host_io(m, _p(m, B=0), q_lat_host=None, workspace=None) == 0   # empty batch: a no-op


def test_workspace_size_formula(m):
    p = _p(m, B=5, Sq=2, H=8, r=32, num_workers=7)
    rows, slots = 2 * 8, 7 + 5 - 1
    al = lambda x: (x + 255) // 256 * 256
    assert m.workspace_size(p) == al(5 * 8) + al(slots * rows * 4) + al(slots * rows * 32 * 4)


def n_b(L, bs):
    return (L + bs - 1) // bs


def _plan_by_definition(lens, bs, W):
    n = [(L + bs - 1) // bs for L in lens]
    P = np.concatenate([[0], np.cumsum(n)]).astype(np.int64)
    T = int(P[-1])
    Wa = min(W, T) if T else W           # active workers
    rng = [(w * T // Wa, (w + 1) * T // Wa) if w < Wa else (T, T) for w in range(W)]
    first, splits = [], []
    for b in range(len(lens)):
        touch = [w for w, (s, e) in enumerate(rng) if n[b] and s < e and s < P[b] + n[b] and e > P[b]]
        first.append(touch[0] if touch else 0)
        splits.append(len(touch))
    return P, first, splits, rng


@pytest.mark.parametrize("W", [1, 2, 5, 74, 300, 5000])
def test_plan_host_matches_definition(m, W):
    rng = np.random.default_rng(W)
    lens = [int(x) for x in rng.integers(0, 3000, size=37)] + [0, 1, 64, 65, 128]
    B = len(lens)
    bs = 64
    p = _p(m, B=B, max_blocks_per_seq=(max(lens) + bs - 1) // bs, num_blocks=10 ** 5, num_workers=W)
    plan = m.plan_host(p, lens)
    P, first, splits, ranges = _plan_by_definition(lens, bs, W)
    np.testing.assert_array_equal(plan["block_begin"], P)
    np.testing.assert_array_equal(plan["splits"], splits)
    for b in range(B):
        if splits[b]:
            assert plan["first_worker"][b] == first[b]
    # balance: active worker ranges differ by at most one block and are never empty
    sizes = [e - s for s, e in ranges[:min(W, int(P[-1]))]]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    # the workers that touch a sequence are consecutive
    for b in range(B):
        touch = [w for w, (s, e) in enumerate(ranges) if n_b(lens[b], bs) and s < e and s < P[b] + n_b(lens[b], bs) and e > P[b]]
        assert touch == list(range(touch[0], touch[0] + len(touch))) if touch else True
    # workspace slots w + b of all (worker, sequence) pairs are distinct and < W + B - 1
    slots = [plan["first_worker"][b] + k + b for b in range(B) if splits[b] > 1 for k in range(splits[b])]
    assert len(slots) == len(set(slots)) and (not slots or max(slots) < W + B - 1)


def test_plan_host_rejects_bad_lengths(m):
    p = _p(m, B=2, max_blocks_per_seq=1)
    with pytest.raises(Exception):
        m.plan_host(p, [65, 3])
    with pytest.raises(Exception):
        m.plan_host(p, [-1, 3])


# ----------------------------------------------------------------------------- cache append
def _append(m, stream=0, **kw):
    from head_latent_attention_split_b200 import binding
    args = dict(B=2, Sq=1, r=512, d_r=64, block_size=64, num_blocks=8, max_blocks_per_seq=4, in_dtype=1,
                cache_dtype=1, rope=False, rope_base=10000.0)
    ptrs = dict(c_new=FAKE, k_rope_new=FAKE, kv_cache=FAKE, k_rope_cache=None, kv_scale=None, block_table=FAKE,
                seq_lens=FAKE)
    for k in list(kw):
        if k in ptrs:
            ptrs[k] = kw.pop(k)
    reserved = kw.pop("reserved", 0)
    args.update(kw)
    p = binding.make_append_params(**args)
    p.reserved = reserved
    return binding.mla_cache_append(p, stream=stream, check=False, **ptrs)


@pytest.mark.parametrize("bad", [dict(Sq=0), dict(r=0), dict(d_r=-1), dict(block_size=0), dict(max_blocks_per_seq=0),
                                 dict(num_blocks=0), dict(in_dtype=0), dict(in_dtype=2), dict(cache_dtype=0),
                                 dict(in_dtype=0, cache_dtype=2), dict(reserved=1),
                                 dict(cache_dtype=2, r=511, k_rope_cache=FAKE, kv_scale=FAKE),
                                 dict(cache_dtype=2), dict(rope=True, d_r=63), dict(rope=True, rope_base=0.0),
                                 dict(rope=True, rope_base=float("inf")), dict(c_new=None), dict(kv_cache=None),
                                 dict(block_table=None), dict(seq_lens=None), dict(k_rope_new=None)])
def test_append_rejects_bad_arguments_on_host(m, bad):
    assert _append(m, **bad) == 1      # MLA_ERR_INVALID_ARG, nothing launched


def test_append_batch_zero_is_a_noop(m):
    assert _append(m, B=0, c_new=None, kv_cache=None, block_table=None, seq_lens=None) == 0


# ----------------------------------------------------------------------------- sparse attention
def _dsa(m, fn="index", **kw):
    from head_latent_attention_split_b200 import binding
    args = dict(B=2, Sq=1, index_heads=64, index_dim=128, block_size=64, num_blocks=8, max_blocks_per_seq=4,
                max_seq_len=256, top_k=64, causal=False)
    reserved = kw.pop("reserved", 0)
    causal_raw = kw.pop("causal_raw", None)
    ptr_names = ("q_codes", "q_scale", "weights", "k_codes", "k_scale", "block_table", "seq_lens", "scores",
                 "indices", "counts")
    ptrs = {k: kw.pop(k, FAKE) for k in ptr_names}
    args.update(kw)
    p = binding.make_dsa_params(**args)
    p.reserved = reserved
    if causal_raw is not None:
        p.causal = causal_raw
    if fn == "index":
        return binding.mla_dsa_index(p, ptrs["q_codes"], ptrs["q_scale"], ptrs["weights"], ptrs["k_codes"],
                                     ptrs["k_scale"], ptrs["block_table"], ptrs["seq_lens"], ptrs["scores"],
                                     stream=0, check=False)
    return binding.mla_dsa_topk(p, ptrs["scores"], ptrs["seq_lens"], ptrs["indices"], ptrs["counts"], stream=0,
                                check=False)


@pytest.mark.parametrize("fn", ["index", "topk"])
@pytest.mark.parametrize("bad,code", [(dict(Sq=0), 1), (dict(top_k=0), 1), (dict(causal_raw=2), 1), (dict(reserved=1), 1),
                                      (dict(max_seq_len=-1), 1), (dict(num_blocks=0), 1), (dict(index_heads=32), 2),
                                      (dict(index_dim=64), 2), (dict(block_size=32), 2), (dict(B=70000), 2),
                                      (dict(scores=None), 1)])
def test_dsa_rejects_bad_arguments_on_host(m, fn, bad, code):
    assert _dsa(m, fn, **bad) == code


def test_dsa_null_and_alignment_checks(m):
    assert _dsa(m, "index", q_codes=None) == 1
    assert _dsa(m, "index", k_codes=FAKE + 8) == 3           # TMA sources: 16-byte aligned
    assert _dsa(m, "index", k_scale=FAKE + 4) == 3
    assert _dsa(m, "topk", indices=None) == 1
    assert _dsa(m, "topk", counts=FAKE + 2) == 3
    assert _dsa(m, "index", B=0, q_codes=None) == 0           # nothing to do
    assert _dsa(m, "topk", B=0, scores=None) == 0


def _sparse(m, **kw):
    from head_latent_attention_split_b200 import binding
    base = dict(B=2, Sq=1, H=128, r=512, d_r=64, block_size=64, num_blocks=8, max_blocks_per_seq=4, q_dtype=1,
                cache_dtype=1, out_dtype=1, causal=False, softmax_scale=0.07, num_workers=4, kernel="tcgen05")
    top_k = kw.pop("top_k", 64)
    ptr_names = ("q_lat", "q_rope", "kv_cache", "block_table", "indices", "counts", "out", "lse", "workspace")
    ptrs = {k: kw.pop(k, FAKE) for k in ptr_names}
    ws_bytes = kw.pop("workspace_bytes", 1 << 30)
    base.update(kw)
    p = m.make_params(**base)
    return binding.mla_sparse_decode(p, top_k, ptrs["q_lat"], ptrs["q_rope"], ptrs["kv_cache"], ptrs["block_table"],
                                     ptrs["indices"], ptrs["counts"], ptrs["out"], ptrs["lse"], ptrs["workspace"],
                                     workspace_bytes=ws_bytes, stream=0, check=False)


@pytest.mark.parametrize("bad,code", [(dict(Sq=2), 2), (dict(causal=True), 2), (dict(cache_dtype=2), 2),
                                      (dict(kernel="simt"), 2), (dict(top_k=0), 1), (dict(indices=None), 1),
                                      (dict(counts=None), 1), (dict(q_rope=None), 1), (dict(workspace_bytes=16), 4),
                                      (dict(q_lat=FAKE + 8), 3), (dict(indices=FAKE + 2), 3)])
def test_sparse_decode_rejects_bad_arguments_on_host(m, bad, code):
    assert _sparse(m, **bad) == code
