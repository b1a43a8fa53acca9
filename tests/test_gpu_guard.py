"""Out-of-bounds writes and the rare O-rescale path.

Canaries: out, lse and the workspace live inside larger buffers whose guard bands hold
a NaN pattern; after the decode the bands must be untouched (and the workspace must not
be written past the size the library asked for).

Late spikes: one token near the end of each sequence gets a latent 200x larger, so for
many heads its score exceeds the running maximum by far more than 2^8 (the threshold at
which the kernel rescales O, and in the tensor-core path ships per-row rescale factors
across the CTA pair). The result must still match the oracle.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workloads as W
from parity_util import TOL, compare

pytestmark = pytest.mark.gpu

GUARD = 4096   # elements of each guard band


def _guarded(torch, shape, dtype, dev):
    n = int(np.prod(shape))
    buf = torch.empty(n + 2 * GUARD, dtype=dtype, device=dev)
    if dtype == torch.uint8:
        buf.fill_(0xA5)
    else:
        buf.fill_(float("nan"))
    return buf, buf[GUARD:GUARD + n].view(shape)


def _bands_ok(torch, buf, n, dtype):
    lo, hi = buf[:GUARD], buf[GUARD + n:]
    if dtype == torch.uint8:
        return bool((lo == 0xA5).all()) and bool((hi == 0xA5).all())
    return bool(torch.isnan(lo.float()).all()) and bool(torch.isnan(hi.float()).all())


CASES = [
    ("tcgen05", W.WORKLOADS[2].with_(B=3, seq_lens=(1, 700, 129)), 0),
    ("tcgen05", W.WORKLOADS[3].with_(B=3, seq_lens=(2, 300, 65)), 500),
    ("tcgen05", W.WORKLOADS[4].with_(B=2, seq_lens=(64, 1100)), 1),
    ("tc_pair", W.WORKLOADS[2].with_(B=3, seq_lens=(1, 700, 129)), 0),
    ("tc_pair", W.WORKLOADS[3].with_(B=3, seq_lens=(2, 300, 65)), 500),
    ("simt", W.WORKLOADS[1].with_(B=2, seq_lens=(3, 200)), 7),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-{c[1].name}-W{c[2]}")
def test_decode_writes_nothing_outside_its_buffers(case):
    import torch
    import head_latent_attention_split_b200 as mla
    kernel, w, nw = case
    inp = W.make_inputs(w)
    t = W.to_torch(inp)
    p = mla.params_for(t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], w.scale, w.causal,
                       num_workers=nw, kernel=kernel)
    dev = t["q_lat"].device
    od = torch.bfloat16 if w.out_dtype == W.BF16 else torch.float32
    obuf, out = _guarded(torch, tuple(t["q_lat"].shape), od, dev)
    lbuf, lse = _guarded(torch, tuple(t["q_lat"].shape[:3]), torch.float32, dev)
    need = mla.workspace_size(p)
    wbuf, ws = _guarded(torch, (need,), torch.uint8, dev)
    mla.mla_decode(p, t["q_lat"], t["q_rope"], t["kv_cache"], t["k_rope_cache"], t["kv_scale"], t["block_table"],
                   t["seq_lens"], out, lse, ws, workspace_bytes=need)
    torch.cuda.synchronize()
    assert mla.device_status() == 0
    assert _bands_ok(torch, obuf, out.numel(), od)
    assert _bands_ok(torch, lbuf, lse.numel(), torch.float32)
    assert _bands_ok(torch, wbuf, need, torch.uint8)
    ref_out, ref_lse = oracle.decode_inputs(inp)
    compare(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_out, ref_lse, TOL[w.cache_dtype], "guarded")


def _spike(inp, factor=200.0):
    """Scale the latent of one late token of every sequence (bf16 or e4m3 storage)."""
    w = inp["workload"]
    inp = dict(inp)
    cache = inp["kv_cache"].copy()
    scale = None if inp.get("kv_scale") is None else inp["kv_scale"].copy()
    bt = inp["block_table"]
    for b, L in enumerate(inp["seq_lens"]):
        if L < 70:
            continue
        t = int(L) - 5
        blk, o = bt[b, t // w.block_size], t % w.block_size
        if w.cache_dtype == W.E4M3:
            scale[blk, o] *= np.float32(factor)        # same codes, 200x the values
        else:
            v = W.bf16_bits_to_f32(cache[blk, o, :w.r]) * np.float32(factor)
            cache[blk, o, :w.r] = W.f32_to_bf16_bits(v)
    inp["kv_cache"] = cache
    if scale is not None:
        inp["kv_scale"] = scale
    return inp


@pytest.mark.parametrize("wl", [W.WORKLOADS[2].with_(B=2, seq_lens=(2000, 700)),
                                W.WORKLOADS[3].with_(B=2, seq_lens=(1500, 300)),
                                W.WORKLOADS[4].with_(B=2, seq_lens=(900, 2100))],
                         ids=lambda w: w.name)
@pytest.mark.parametrize("num_workers", [1, 0])
def test_late_spike_forces_rescale(wl, num_workers):
    import torch
    import head_latent_attention_split_b200 as mla
    inp = _spike(W.make_inputs(wl))
    t = W.to_torch(inp)
    out, lse = mla.decode(t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], t["seq_lens"], wl.scale,
                          wl.causal, t["k_rope_cache"], t["kv_scale"], num_workers=num_workers, kernel="tcgen05")
    torch.cuda.synchronize()
    assert mla.device_status() == 0
    ref_out, ref_lse = oracle.decode_inputs(inp)
    # the spike must really move the running maximum by more than 2^8 for some rows
    base_out, base_lse = oracle.decode_inputs(W.make_inputs(wl))
    assert ((ref_lse - base_lse) / np.log(2) > 8).any()
    compare(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_out, ref_lse, TOL[wl.cache_dtype], "spike")
