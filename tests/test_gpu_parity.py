"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Small cases span several 64-token tiles with ragged tails, empty sequences, causal
two-token queries, every storage type and several worker counts (1 worker = no
split; more workers than tiles = empty workers). Full-size workloads are checked whole,
every row against the oracle, in the launch configuration the bench times.
"""
import math

import numpy as np
import pytest

import oracle
import workloads as W
from parity_util import TOL, compare, run_gpu

pytestmark = pytest.mark.gpu

KERNELS = ["simt", "tcgen05", "tc_pair"]


@pytest.fixture(scope="module")
def mla():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_split_b200 import build
    build.build()
    import head_latent_attention_split_b200 as m
    return m


def kernel_ok(mla, inp, kernel, num_workers=0):
    w = inp["workload"]
    p = mla.make_params(w.B, w.Sq, w.H, w.r, w.d_r, w.block_size, inp["num_blocks"], inp["max_blocks_per_seq"],
                        w.q_dtype, w.cache_dtype, w.out_dtype, w.causal, w.scale, num_workers, kernel)
    try:
        mla.resolve(p)
        return True
    except mla.MlaError as e:
        if e.status == 2:
            return False
        raise


SMALL = {
    "bf16_h128": W.WORKLOADS[2].with_(B=4, seq_lens=(1, 63, 64, 1000)),
    "bf16_h32": W.WORKLOADS[1].with_(B=3, seq_lens=(700, 65, 2049)),
    "bf16_zero_len": W.WORKLOADS[2].with_(B=5, seq_lens=(0, 3, 0, 129, 64), spare_blocks=2),
    "mtp_causal": W.WORKLOADS[3].with_(B=4, seq_lens=(2, 65, 130, 777)),
    "mtp_causal_short": W.WORKLOADS[3].with_(B=3, seq_lens=(1, 0, 64)),
    "fp8": W.WORKLOADS[4].with_(B=4, seq_lens=(5, 64, 200, 1500)),
    "fp8_h32": W.WORKLOADS[4].with_(B=2, H=32, seq_lens=(129, 1000)),
    # all-zero latents (scale 0, what the cache append stores for them) and tiny scales whose
    # reciprocal overflows fp32 (2^-130 latents: scale ~2^-137, subnormal; 2^-120 latents)
    "fp8_zero_tiny130": W.WORKLOADS[4].with_(B=3, seq_lens=(130, 700, 64), zero_every=7, tiny_every=11,
                                             tiny_exp=-130),
    "fp8_zero_tiny120": W.WORKLOADS[4].with_(B=2, seq_lens=(1000, 77), zero_every=3, tiny_every=5,
                                             tiny_exp=-120),
    "bf16_zero_tokens": W.WORKLOADS[2].with_(B=2, seq_lens=(200, 513), zero_every=5),
    "sharp_softmax": W.WORKLOADS[2].with_(B=2, seq_lens=(300, 513), scale=8.0 / math.sqrt(192.0)),
    "scale_zero": W.WORKLOADS[2].with_(B=2, seq_lens=(100, 257), scale=0.0),
}


@pytest.fixture(scope="module")
def small_cases():
    cache = {}

    def get(name):
        if name not in cache:
            inp = W.make_inputs(SMALL[name])
            cache[name] = (inp, oracle.decode_inputs(inp))
        return cache[name]
    return get


def test_tiny_f32_workload(mla):
    inp = W.make_inputs(W.WORKLOADS[0])
    ref_o, ref_l = oracle.decode_inputs(inp)
    for nw in (0, 1, 2, 3):
        o, l = run_gpu(inp, "simt", nw)
        compare(o, l, ref_o, ref_l, TOL[W.F32], f"tiny f32 W={nw}")


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("num_workers", [0, 1, 5, 500])
def test_small_parity(mla, small_cases, name, kernel, num_workers):
    inp, (ref_o, ref_l) = small_cases(name)
    if not kernel_ok(mla, inp, kernel, num_workers):
        pytest.skip(f"{kernel} does not take {name}")
    o, l = run_gpu(inp, kernel, num_workers)
    compare(o, l, ref_o, ref_l, TOL[inp["workload"].cache_dtype], f"{name}/{kernel}/W={num_workers}")


@pytest.mark.parametrize("kernel", KERNELS)
def test_f32_output(mla, small_cases, kernel):
    inp, (ref_o, ref_l) = small_cases("bf16_h128")
    if not kernel_ok(mla, inp, kernel):
        pytest.skip(kernel)
    o, l = run_gpu(inp, kernel, 0, out_dtype=W.F32)
    compare(o, l, ref_o, ref_l, 4e-3, "f32 out")


@pytest.mark.parametrize("kernel", KERNELS)
def test_deterministic(mla, small_cases, kernel):
    inp, _ = small_cases("mtp_causal")
    if not kernel_ok(mla, inp, kernel):
        pytest.skip(kernel)
    t = W.to_torch(inp)
    a = run_gpu(inp, kernel, 7, tensors=t)
    b = run_gpu(inp, kernel, 7, tensors=t)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_integer_latents_exact_mean(mla):
    """F32 path, scale 0, integer latents: every row is the exact mean (power-of-two n)."""
    import torch
    B, H, r, d_r, bs = 3, 5, 40, 8, 16
    lens = np.array([64, 128, 256], np.int32)
    nb = int(sum(lens // bs))
    perm = np.random.default_rng(3).permutation(nb)
    bt = np.full((B, 16), -1, np.int32)
    cache = np.zeros((nb, bs, r + d_r), np.float32)
    off = 0
    for b in range(B):
        for i in range(lens[b] // bs):
            bt[b, i] = perm[off + i]
            for o in range(bs):
                t = i * bs + o
                cache[perm[off + i], o, :r] = (t * 7 + np.arange(r) + 13 * b) % 64
        off += lens[b] // bs
    q = np.random.default_rng(1).standard_normal((B, 1, H, r)).astype(np.float32)
    qr = np.random.default_rng(2).standard_normal((B, 1, H, d_r)).astype(np.float32)
    dev = lambda a: torch.from_numpy(a).cuda()
    out, lse = mla.decode(dev(q), dev(qr), dev(cache), dev(bt), dev(lens), 0.0, num_workers=1, kernel="simt")
    out = out.cpu().numpy()
    for b in range(B):
        t = np.arange(lens[b])[:, None]
        exact = ((t * 7 + np.arange(r) + 13 * b) % 64).sum(0) / lens[b]
        for h in range(H):
            assert np.array_equal(out[b, 0, h], exact.astype(np.float32))
    np.testing.assert_allclose(lse.cpu().numpy()[:, 0, 0], np.log(lens), rtol=0, atol=1e-6)


def test_plan_probe_bit_exact(mla):
    """Every token is read once, from the slot the block table names, by the planned worker."""
    import torch
    inp = W.make_inputs(W.WORKLOADS[3].with_(B=9, seq_lens=(1, 0, 64, 65, 300, 0, 1024, 7, 129)))
    w = inp["workload"]
    t = W.to_torch(inp)
    for nw in (1, 3, 13, 74, 400):
        p = mla.make_params(w.B, w.Sq, w.H, w.r, w.d_r, 64, inp["num_blocks"], inp["max_blocks_per_seq"],
                            w.q_dtype, w.cache_dtype, w.out_dtype, w.causal, w.scale, nw, "simt")
        slot, worker, meta = mla.plan_probe(p, t["block_table"], t["seq_lens"])
        torch.cuda.synchronize()
        slot, worker, meta = slot.cpu().numpy(), worker.cpu().numpy(), meta.cpu().numpy()
        plan = mla.plan_host(p, inp["seq_lens"])
        P = plan["block_begin"].astype(np.int64)
        T = int(P[-1])
        for b, L in enumerate(inp["seq_lens"]):
            tok = np.arange(L)
            exp_slot = inp["block_table"][b, tok // 64] * 64 + tok % 64
            assert np.array_equal(slot[b, :L], exp_slot)
            assert (slot[b, L:] == -1).all()
            Wa = min(nw, T)
            exp_worker = ((P[b] + tok // 64 + 1) * Wa - 1) // T if L else tok
            assert np.array_equal(worker[b, :L], exp_worker)
            if L:
                assert meta[b, 0] == plan["first_worker"][b] and meta[b, 1] == plan["splits"][b]
        assert mla.device_status() == 0


def _check_nan_rows(out, lse, bad, ref_o, ref_l, tol, what):
    """Every row of the sequences in `bad` is NaN (out and lse); the others match the oracle."""
    o = out.double().cpu().numpy()
    l = lse.double().cpu().numpy()
    good = [b for b in range(o.shape[0]) if b not in bad]
    for b in bad:
        assert np.isnan(o[b]).all() and np.isnan(l[b]).all(), f"{what}: sequence {b} not NaN"
    compare(o[good], l[good], ref_o[good], ref_l[good], tol, what)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("num_workers", [0, 1, 7])
def test_bad_block_id_and_seq_len_set_status(mla, small_cases, kernel, num_workers):
    """A bad block id or seq_len sets the sticky status and turns that sequence's rows NaN;
    the other sequences still match the oracle (also when the bad one is split over workers)."""
    import torch
    inp, (ref_o, ref_l) = small_cases("bf16_h128")
    if not kernel_ok(mla, inp, kernel, num_workers):
        pytest.skip(kernel)
    w = inp["workload"]
    tol = TOL[w.cache_dtype]
    t = W.to_torch(inp)
    args = dict(num_workers=num_workers, kernel=kernel)
    for blk in (inp["num_blocks"] + 17, -1):
        bt = t["block_table"].clone()
        bt[3, 2] = blk
        out, lse = mla.decode(t["q_lat"], t["q_rope"], t["kv_cache"], bt, t["seq_lens"], w.scale, **args)
        torch.cuda.synchronize()
        assert mla.device_status() == 6           # MLA_ERR_BAD_BLOCK_ID
        assert mla.device_status() == 0           # cleared by the read
        _check_nan_rows(out, lse, {3}, ref_o, ref_l, tol, f"bad block {blk}")
    sl = t["seq_lens"].clone()
    for bad_len in (inp["max_blocks_per_seq"] * 64 + 1, -5):
        sl[1] = bad_len
        out, lse = mla.decode(t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], sl, w.scale, **args)
        torch.cuda.synchronize()
        assert mla.device_status() == 7           # MLA_ERR_BAD_SEQ_LEN
        _check_nan_rows(out, lse, {1}, ref_o, ref_l, tol, f"bad seq_len {bad_len}")
    # the stream and context stay usable: a clean call still matches
    o, l = run_gpu(inp, kernel, num_workers, tensors=t)
    compare(o, l, ref_o, ref_l, tol, "after the bad calls")


@pytest.mark.parametrize("kernel", ["tcgen05", "tc_pair"])
def test_wait_timeout_expires_cleanly(mla, small_cases, kernel):
    """A pipeline wait limit far below the time a tile takes makes the tensor-core kernel's
    waits run out: the call returns, the status word reads MLA_ERR_TIMEOUT once, the unfinished
    rows are NaN, and the next call with the default limit matches the oracle."""
    import torch
    inp, (ref_o, ref_l) = small_cases("bf16_h128")
    if not kernel_ok(mla, inp, kernel):
        pytest.skip(kernel)
    w = inp["workload"]
    t = W.to_torch(inp)
    assert mla.wait_timeout_ns() == 2_000_000_000
    mla.set_wait_timeout_ns(200)
    try:
        assert mla.wait_timeout_ns() == 200
        out, lse = mla.decode(t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], t["seq_lens"], w.scale,
                              kernel=kernel)
        torch.cuda.synchronize()
    finally:
        mla.set_wait_timeout_ns(0)
    assert mla.wait_timeout_ns() == 2_000_000_000
    assert mla.device_status() == 8           # MLA_ERR_TIMEOUT
    assert mla.device_status() == 0
    o = out.double().cpu().numpy()
    l = lse.double().cpu().numpy()
    assert np.isnan(o).any() and np.isnan(l).any()
    # every row is either NaN throughout or the right answer
    for b in range(w.B):
        for h in range(w.H):
            if np.isnan(l[b, 0, h]):
                assert np.isnan(o[b, 0, h]).all()
    o2, l2 = run_gpu(inp, kernel, 0, tensors=t)
    compare(o2, l2, ref_o, ref_l, TOL[w.cache_dtype], "after the timeout")


@pytest.mark.parametrize("kernel", KERNELS)
def test_host_io_matches_device_call(mla, small_cases, kernel):
    import torch
    inp, (ref_o, ref_l) = small_cases("mtp_causal")
    if not kernel_ok(mla, inp, kernel):
        pytest.skip(kernel)
    w = inp["workload"]
    t = W.to_torch(inp)
    pin = lambda x: x.cpu().pin_memory()
    o_h, l_h = mla.decode_host_io(pin(t["q_lat"]), pin(t["q_rope"]), t["kv_cache"], pin(t["block_table"]),
                                  pin(t["seq_lens"]), w.scale, w.causal, t["k_rope_cache"], t["kv_scale"],
                                  kernel=kernel)
    torch.cuda.synchronize()
    o_d, l_d = run_gpu(inp, kernel, 0, tensors=t)
    assert np.array_equal(o_h.double().numpy(), o_d) and np.array_equal(l_h.double().numpy(), l_d)


@pytest.mark.parametrize("kernel", KERNELS)
def test_host_io_chunked_pipeline(mla, kernel):
    """A host-I/O step large enough to be pipelined (B = 32, 128 heads: 8.5 MiB of per-step
    copies) runs as four chunks of 8 consecutive sequences whose copies overlap the other
    chunks' decodes. Each chunk is its own decode: the result equals, bit for bit, the device
    decode of each 8-sequence slice, and matches the oracle."""
    import torch
    rng = np.random.default_rng(21)
    wl = W.WORKLOADS[2].with_(B=32, seq_lens=tuple(int(x) for x in rng.integers(1, 700, 32)))
    inp = W.make_inputs(wl)
    if not kernel_ok(mla, inp, kernel):
        pytest.skip(kernel)
    ref_o, ref_l = oracle.decode_inputs(inp)
    t = W.to_torch(inp)
    pin = lambda x: x.cpu().pin_memory()  # noqa: E731
    o_h, l_h = mla.decode_host_io(pin(t["q_lat"]), pin(t["q_rope"]), t["kv_cache"], pin(t["block_table"]),
                                  pin(t["seq_lens"]), wl.scale, wl.causal, kernel=kernel)
    torch.cuda.synchronize()
    assert mla.device_status() == 0
    o_h, l_h = o_h.double().numpy(), l_h.double().numpy()
    compare(o_h, l_h, ref_o, ref_l, TOL[wl.cache_dtype], f"chunked host I/O ({kernel})")
    for b0 in range(0, 32, 8):
        sl = slice(b0, b0 + 8)
        o_d, l_d = mla.decode(t["q_lat"][sl].contiguous(), t["q_rope"][sl].contiguous(), t["kv_cache"],
                              t["block_table"][sl].contiguous(), t["seq_lens"][sl].contiguous(), wl.scale,
                              wl.causal, kernel=kernel)
        torch.cuda.synchronize()
        assert np.array_equal(o_h[sl], o_d.double().cpu().numpy()), f"chunk {b0}"
        assert np.array_equal(l_h[sl], l_d.double().cpu().numpy()), f"chunk {b0}"


# ---------------------------------------------------------------------------- full-size workloads
_FULL = {}


def _full_case(idx):
    """Inputs and the fp64 oracle's whole output for full-size workload idx (computed once)."""
    if idx not in _FULL:
        inp = W.make_inputs(W.WORKLOADS[idx])
        _FULL.clear()
        _FULL[idx] = (inp, oracle.decode_inputs(inp))
    return _FULL[idx]


@pytest.mark.parametrize("idx,kernel", [(1, "auto"), (2, "auto"), (2, "tcgen05"), (3, "auto"), (4, "auto")])
def test_full_size_workloads_element_wise(mla, idx, kernel):
    """The full workload in the launch configuration the bench times (default worker count),
    every (b, s, h) row against the fp64 oracle's whole output, element by element."""
    import torch
    inp, (ref_o, ref_l) = _full_case(idx)
    w = inp["workload"]
    t = W.to_torch(inp)
    o, l = run_gpu(inp, kernel, 0, tensors=t)
    compare(o, l, ref_o, ref_l, TOL[w.cache_dtype], f"{w.name} ({kernel})")
    del t
    torch.cuda.empty_cache()
