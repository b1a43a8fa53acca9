"""Helpers for GPU-vs-oracle parity tests (imported by the gpu-marked tests only)."""
import numpy as np

import workloads as W

# max|gpu - ref| / max|ref| over the compared outputs, per cache storage type
TOL = {W.F32: 1e-5, W.BF16: 1e-2, W.E4M3: 2e-2}
LSE_TOL = 1e-3


def run_gpu(inp, kernel="auto", num_workers=0, out_dtype=None, tensors=None):
    import torch
    import head_latent_attention_split_b200 as mla
    t = tensors if tensors is not None else W.to_torch(inp)
    w = inp["workload"]
    out, lse = mla.decode(t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], t["seq_lens"], w.scale,
                          w.causal, t["k_rope_cache"], t["kv_scale"], out_dtype=out_dtype,
                          num_workers=num_workers, kernel=kernel)
    torch.cuda.synchronize()
    st = mla.device_status()
    assert st == 0, mla.status_string(st)
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


def compare(out, lse, ref_out, ref_lse, tol, what=""):
    ref_out = np.asarray(ref_out)
    assert out.shape == ref_out.shape, (out.shape, ref_out.shape)
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    scale = max(np.abs(ref_out).max(), 1e-30)
    err = np.abs(out - ref_out).max() / scale
    assert err <= tol, f"{what}: max|d|/max|ref| = {err:.3e} > {tol:g}"
    inf_ref = np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(lse), inf_ref), f"{what}: -inf lse rows differ"
    if (~inf_ref).any():
        lerr = np.abs(lse[~inf_ref] - ref_lse[~inf_ref]).max()
        assert lerr <= LSE_TOL, f"{what}: lse error {lerr:.3e}"
    return err
