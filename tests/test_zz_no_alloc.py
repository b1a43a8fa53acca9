"""The allocation-free entry point, mla_decode_noalloc, against mla_decode.

mla_decode_noalloc exists for callers that may not allocate device memory while they
decode: a serving engine that reserved the GPU's memory for its cache before the first
step, or a plugin that runs in a memory pool it does not own. It takes the same inputs
and outputs as mla_decode but no workspace; the split workspace is the library's own
fixed-size device array. Calls in a row must each give what mla_decode gives: the array
keeps the previous call's contents, so a large call (more sequences, more workers, more
split partials) runs first and the smaller call after it checks that none of the larger
call's leftovers leak into the result.
"""
import numpy as np
import pytest

import workloads as W
from parity_util import LSE_TOL, TOL


def _mla():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_split_b200 import build
    build.build()
    import head_latent_attention_split_b200 as mla
    return mla


def _noalloc_vs_workspace(mla, wl, num_workers, calls):
    """Run mla_decode_noalloc `calls` times on workload wl and compare each result with
    mla_decode's (same parameters, caller-owned workspace)."""
    import torch
    inp = W.make_inputs(wl)
    t = W.to_torch(inp)
    p = mla.params_for(t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], wl.scale, wl.causal,
                       num_workers=num_workers)
    assert mla.workspace_size(p) <= mla.noalloc_max_workspace()
    ref_o, ref_l = mla.decode(t["q_lat"], t["q_rope"], t["kv_cache"], t["block_table"], t["seq_lens"], wl.scale,
                              wl.causal, t["k_rope_cache"], t["kv_scale"], num_workers=num_workers)
    torch.cuda.synchronize()
    ref_o = ref_o.double().cpu().numpy()
    ref_l = ref_l.double().cpu().numpy()
    for call in range(calls):
        out = torch.full(t["q_lat"].shape, float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full(t["q_lat"].shape[:3], float("nan"), dtype=torch.float32, device="cuda")
        mla.mla_decode_noalloc(p, t["q_lat"], t["q_rope"], t["kv_cache"], t["k_rope_cache"], t["kv_scale"],
                               t["block_table"], t["seq_lens"], out, lse)
        torch.cuda.synchronize()
        assert mla.device_status() == 0
        o = out.double().cpu().numpy()
        l = lse.double().cpu().numpy()
        assert np.isfinite(o).all(), f"{wl.name} call {call}: non-finite output"
        err = np.abs(o - ref_o).max() / np.abs(ref_o).max()
        assert err <= TOL[wl.cache_dtype], f"{wl.name} call {call}: {err}"
        assert np.abs(l - ref_l).max() <= LSE_TOL, f"{wl.name} call {call}: lse"


@pytest.mark.gpu
@pytest.mark.parametrize("wl", [W.WORKLOADS[3].with_(B=4, seq_lens=(2, 65, 300, 777)),
                                W.WORKLOADS[4].with_(B=3, seq_lens=(5, 200, 1500))],
                         ids=["bf16_causal", "fp8"])
def test_noalloc_matches_workspace_entry_point(wl):
    mla = _mla()
    # a larger call first (more sequences and workers: more split partials in the array) ...
    big = wl.with_(B=12, seq_lens=tuple((list(W.resolve_seq_lens(wl)) * 4)[:12]))
    _noalloc_vs_workspace(mla, big, 40, 1)
    # ... then the small one twice: five workers split its longer sequences
    _noalloc_vs_workspace(mla, wl, 5, 2)


def test_noalloc_rejects_workspace_beyond_its_array():
    """Host-side size check: runs without a GPU."""
    from head_latent_attention_split_b200 import binding
    import head_latent_attention_split_b200 as mla
    # 4096 sequences x 128 heads x 512 channels of fp32 partials: far above 64 MiB
    p = mla.make_params(4096, 1, 128, 512, 64, 64, 1 << 20, 1024, W.BF16, W.BF16, W.BF16, False, 0.1,
                        num_workers=74, kernel="simt")
    assert mla.workspace_size(p) > mla.noalloc_max_workspace()
    st = binding.mla_decode_noalloc(p, 1 << 20, 1 << 20, 1 << 20, None, None, 1 << 20, 1 << 20, 1 << 20, 1 << 20,
                                    stream=0, check=False)
    assert st == 4        # MLA_ERR_WORKSPACE_TOO_SMALL, nothing launched
