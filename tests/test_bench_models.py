"""The benchmark's algorithmic-work models (the numerators of its roofline fractions), on CPU,
against counts written out from their definitions for small shapes."""
from __future__ import annotations

import numpy as np

import bench
import workloads as W


def test_decode_work_model_counts():
    # one sequence of 100 tokens, 2 causal query rows, 4 heads, r = 512, d_r = 64, bf16
    w = W.WORKLOADS[3].with_(B=1, Sq=2, H=4, seq_lens=(100,), name="m")
    inp = dict(workload=w, seq_lens=np.array([100], np.int32))
    m = bench.work_model(inp)
    assert m["tokens"] == 100 and m["cache_bytes"] == 100 * 1152
    # query rows see 99 and 100 tokens; 2176 FLOP per (row, head, token)
    assert m["pairs"] == (99 + 100) * 4
    assert m["flops"] == (99 + 100) * 4 * 2176
    assert m["io_bytes"] == 2 * 4 * (576 * 2 + 512 * 2 + 4)


def test_sparse_step_work_model_counts():
    # two sequences of 5000 and 1000 tokens, k = 2048: the second keeps all of its tokens
    dw = W.DsaWorkload("m", W.Workload(name="m_mla", B=2, Sq=1, H=8, r=512, d_r=64, seq_lens=(5000, 1000)),
                       top_k=2048)
    inp = dict(dsa=dw, workload=dw.mla, seq_lens=np.array([5000, 1000], np.int32))
    m = bench.dsa_work_model(inp)
    assert m["tokens"] == 6000 and m["selected"] == 2048 + 1000
    # indexer: 128 B of codes, a 4 B scale and a 4 B score per token; 64 x 128 MACs per token
    assert m["index"]["bytes"] == 6000 * 136 + 2 * 64 * (128 + 8)
    assert m["index"]["flops"] == 6000 * 64 * 128 * 2
    # top-k: the scores in, k positions out per row
    assert m["topk"]["bytes"] == 6000 * 4 + 2 * 2048 * 4
    # decode over the selected tokens: 1152 B each, 2176 FLOP per (head, token)
    assert m["decode"]["bytes"] == 3048 * 1152 + 2 * 8 * (1152 + 1024 + 4)
    assert m["decode"]["flops"] == 3048 * 8 * 2176
