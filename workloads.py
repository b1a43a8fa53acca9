"""Seeded synthetic inputs for absorbed MLA decode over a paged latent cache.

This module only draws random numbers and lays them out in the storage formats the
decode consumes (fp32, bf16 bit patterns, e4m3 codes with a per-token fp32 scale).
It holds none of the attention arithmetic: both the fp64 oracle (``oracle/``) and
the CUDA path (``head_latent_attention_split_b200``) read the arrays it returns.

Shapes follow the pages' workloads:
  * a LLaMA-2-7B model converted by TransMLA keeps a 512-wide latent plus a 64-wide
    RoPE key per token and has 32 query heads ("TransMLA: Multi-Head Latent Attention
    Is All You Need", sec. 3.4.5 "The full MLA structure after conversion"; TPLA
    paper-graph page, sec. 4 experiments on the 512+64 split);
  * DeepSeek-V3 has 128 query heads, d_c = 512 and d_h^R = 64
    ("TransMLA & Sparse Latent Attention" lesson, Chapter 6 "Even MLA's own cache,
    priced out honestly").

Every array is produced on the host with numpy generators derived from one seed, in
fixed-size chunks with their own substreams, so the values do not depend on the
number of threads used to fill them.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace
import os

import numpy as np

BLOCK = 64          # tokens per cache block (paged layout)
F32, BF16, E4M3 = 0, 1, 2   # storage codes shared by both sides' bindings
DTYPE_NAMES = {F32: "f32", BF16: "bf16", E4M3: "e4m3"}

# bf16 NaN bit pattern and e4m3 NaN code, used to poison cache slots that no
# sequence may read (tokens past seq_len inside a sequence's last block).
BF16_NAN = np.uint16(0x7FC0)
E4M3_NAN = np.uint8(0x7F)


@dataclass(frozen=True)
class Workload:
    """One decode problem: shapes, value recipe and seed."""
    name: str
    B: int
    Sq: int
    H: int
    r: int
    d_r: int
    seq_lens: tuple | str          # explicit tuple, or "loguniform:lo:hi"
    q_dtype: int = BF16
    cache_dtype: int = BF16
    out_dtype: int = BF16
    causal: bool = False
    scale: float = 1.0 / math.sqrt(192.0)
    q_std: float = 1.0
    c_std: float = 1.0
    outlier_frac: float = 0.0      # fraction of latent channels multiplied by outlier_gain
    outlier_gain: float = 8.0
    contiguous: bool = False       # block_table = identity layout instead of a permutation
    spare_blocks: int = 0          # physical blocks owned by no sequence (poisoned)
    zero_every: int = 0            # > 0: every zero_every-th cache slot (from slot 1) holds an all-zero latent
    tiny_every: int = 0            # > 0: every tiny_every-th slot (from slot 2) has its latent scaled by 2^tiny_exp
    tiny_exp: int = -130
    seed: int = 0
    block_size: int = BLOCK
    description: str = ""

    @property
    def rows(self) -> int:
        return self.Sq * self.H

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def _wl(idx: int, **kw) -> Workload:
    return Workload(seed=1000 + idx, **kw)


# The five reference workloads (index 0..4); seed = 1000 + index.
WORKLOADS = [
    _wl(0, name="tiny_f32", B=2, Sq=1, H=4, r=16, d_r=8, seq_lens=(64, 64),
        q_dtype=F32, cache_dtype=F32, out_dtype=F32, scale=1.0 / math.sqrt(24.0),
        contiguous=True,
        description="tiny fp32 MLA decode: B=2 H=4 r=16 d_r=8 L=64, contiguous cache"),
    _wl(1, name="llama2_7b_transmla", B=16, Sq=1, H=32, r=512, d_r=64,
        seq_lens=(8192,) * 16, q_std=0.5, c_std=0.5,
        description="LLaMA-2-7B converted by TransMLA, bf16: B=16 H=32 L=8192, 512+64 latent, "
                    "shuffled paged cache"),
    _wl(2, name="deepseek_v3", B=64, Sq=1, H=128, r=512, d_r=64,
        seq_lens=(32768,) * 64, q_std=1.0, c_std=1.0 / math.sqrt(512.0),
        outlier_frac=0.01,
        description="DeepSeek-V3-shaped decode, bf16: B=64 H=128 L=32768, 512+64 latent, "
                    "1% outlier channels x8, shuffled paged cache"),
    _wl(3, name="ragged_mtp", B=128, Sq=2, H=128, r=512, d_r=64,
        seq_lens="loguniform:1024:32768", causal=True, q_std=1.0,
        c_std=1.0 / math.sqrt(512.0), outlier_frac=0.01,
        description="ragged paged batch, 2 causal query tokens per sequence, bf16: B=128 H=128, "
                    "seq_lens log-uniform in [1024, 32768]"),
    _wl(4, name="fp8_cache", B=32, Sq=1, H=128, r=512, d_r=64,
        seq_lens=(65536,) * 32, cache_dtype=E4M3, q_std=1.0, c_std=1.0,
        description="FP8 e4m3 latent cache with per-token fp32 scale (k_rope bf16): "
                    "B=32 H=128 L=65536"),
]
BY_NAME = {w.name: w for w in WORKLOADS}

_CHUNK = 1 << 22      # elements per independently seeded chunk


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even) and return the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _fill_normal(rng_seed: np.random.SeedSequence, n: int, threads: int) -> np.ndarray:
    """n standard normals (float32), chunked with per-chunk substreams."""
    out = np.empty(n, dtype=np.float32)
    nchunks = max(1, (n + _CHUNK - 1) // _CHUNK)
    subs = rng_seed.spawn(nchunks)

    def work(i):
        lo, hi = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        np.random.default_rng(subs[i]).standard_normal(hi - lo, dtype=np.float32, out=out[lo:hi])

    if nchunks == 1 or threads <= 1:
        for i in range(nchunks):
            work(i)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(work, range(nchunks)))
    return out


def resolve_seq_lens(w: Workload) -> np.ndarray:
    if isinstance(w.seq_lens, str):
        kind, lo, hi = w.seq_lens.split(":")
        assert kind == "loguniform"
        rng = np.random.default_rng(np.random.SeedSequence([w.seed, 7]))
        u = rng.uniform(math.log(float(lo)), math.log(float(hi)), size=w.B)
        lens = np.floor(np.exp(u)).astype(np.int64)
        lens = np.clip(lens, max(int(lo), w.Sq), int(hi))
        return lens.astype(np.int32)
    lens = np.asarray(w.seq_lens, dtype=np.int32)
    assert lens.shape == (w.B,)
    return lens


def quantize_e4m3_per_token(c: np.ndarray):
    """Per-token e4m3 storage: scale = amax/448, code = RNE(c/scale) (OCP e4m3, no inf).

    Uses torch's float8_e4m3fn cast as the rounding routine. Tokens whose amax is 0
    get scale 0 and all-zero codes (what the library's cache append stores for them).
    """
    import torch
    amax = np.abs(c).max(axis=-1)
    scale = (amax / np.float32(448.0)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    y = np.clip(c / safe[..., None], -448.0, 448.0).astype(np.float32)
    codes = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, scale


def make_inputs(w: Workload, threads: int | None = None) -> dict:
    """Generate every input array of one decode call for workload ``w`` (host numpy)."""
    threads = threads or min(16, os.cpu_count() or 1)
    root = np.random.SeedSequence(w.seed)
    ss_q, ss_qr, ss_c, ss_kr, ss_perm, ss_out = root.spawn(6)
    bs = w.block_size
    lens = resolve_seq_lens(w)
    nblk_seq = [(int(L) + bs - 1) // bs for L in lens]
    max_blocks = max(1, max(nblk_seq))
    used = int(sum(nblk_seq))
    num_blocks = max(1, used + w.spare_blocks)

    # physical placement: a seeded permutation (or identity) of all blocks
    if w.contiguous:
        perm = np.arange(num_blocks, dtype=np.int32)
    else:
        perm = np.random.default_rng(ss_perm).permutation(num_blocks).astype(np.int32)
    block_table = np.full((w.B, max_blocks), -1, dtype=np.int32)
    off = 0
    for b, nb in enumerate(nblk_seq):
        block_table[b, :nb] = perm[off:off + nb]
        off += nb

    # queries
    q = _fill_normal(ss_q, w.B * w.Sq * w.H * w.r, threads).reshape(w.B, w.Sq, w.H, w.r)
    qr = _fill_normal(ss_qr, w.B * w.Sq * w.H * w.d_r, threads).reshape(w.B, w.Sq, w.H, w.d_r)
    q *= np.float32(w.q_std)
    qr *= np.float32(w.q_std)

    # cache: latent c (r) and rope key k^R (d_r) per token slot
    c = _fill_normal(ss_c, num_blocks * bs * w.r, threads).reshape(num_blocks, bs, w.r)
    kr = _fill_normal(ss_kr, num_blocks * bs * w.d_r, threads).reshape(num_blocks, bs, w.d_r)
    c *= np.float32(w.c_std)
    kr *= np.float32(w.c_std)
    if w.outlier_frac > 0:
        n_out = max(1, int(round(w.outlier_frac * w.r)))
        ch = np.random.default_rng(np.random.SeedSequence([w.seed, 11])).choice(w.r, n_out, replace=False)
        c[:, :, np.sort(ch)] *= np.float32(w.outlier_gain)
    flat = c.reshape(-1, w.r)
    if w.zero_every > 0:
        flat[1::w.zero_every] = 0.0
    if w.tiny_every > 0:
        flat[2::w.tiny_every] *= np.float32(2.0 ** w.tiny_exp)

    # slots no sequence may read: tokens past seq_len in each last block, spare blocks
    poison = np.zeros((num_blocks, bs), dtype=bool)
    for b, L in enumerate(lens):
        nb = nblk_seq[b]
        if nb and L % bs:
            poison[block_table[b, nb - 1], L % bs:] = True
    owned = np.zeros(num_blocks, dtype=bool)
    owned[block_table[block_table >= 0]] = True
    poison[~owned] = True

    res = dict(workload=w, seq_lens=lens, block_table=block_table, num_blocks=num_blocks,
               max_blocks_per_seq=max_blocks, poison=poison)
    if w.q_dtype == F32:
        res["q_lat"], res["q_rope"] = q, qr
    else:
        res["q_lat"], res["q_rope"] = f32_to_bf16_bits(q), f32_to_bf16_bits(qr)

    if w.cache_dtype == F32:
        cache = np.concatenate([c, kr], axis=-1)
        cache[poison] = np.nan
        res["kv_cache"] = cache
        res["k_rope_cache"] = None
        res["kv_scale"] = None
    elif w.cache_dtype == BF16:
        cache = np.empty((num_blocks, bs, w.r + w.d_r), dtype=np.uint16)
        cache[..., :w.r] = f32_to_bf16_bits(c)
        cache[..., w.r:] = f32_to_bf16_bits(kr)
        cache[poison] = BF16_NAN
        res["kv_cache"] = cache
        res["k_rope_cache"] = None
        res["kv_scale"] = None
    elif w.cache_dtype == E4M3:
        codes, scale = quantize_e4m3_per_token(c)
        krb = f32_to_bf16_bits(kr)
        codes[poison] = E4M3_NAN
        krb[poison] = BF16_NAN
        scale[poison] = np.nan
        res["kv_cache"] = codes
        res["k_rope_cache"] = krb
        res["kv_scale"] = scale
    else:
        raise ValueError(w.cache_dtype)
    return res


def cache_bytes_per_token(r: int, d_r: int, cache_dtype: int) -> int:
    """Stored bytes of one cached token (latent + RoPE key [+ scale])."""
    if cache_dtype == F32:
        return 4 * (r + d_r)
    if cache_dtype == BF16:
        return 2 * (r + d_r)
    return r + 2 * d_r + 4


def attended_pairs(w: Workload, lens: np.ndarray) -> int:
    """Sum over (query row, head) of attended tokens."""
    tot = 0
    for L in lens:
        for s in range(w.Sq):
            n = int(L) - w.Sq + 1 + s if w.causal else int(L)
            tot += max(0, n)
    return tot * w.H


def to_torch(inp: dict, device="cuda") -> dict:
    """Move the arrays of ``make_inputs`` to torch tensors on ``device`` (bit-exact)."""
    import torch

    def t(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    out = {k: t(inp[k]) for k in ("q_lat", "q_rope", "kv_cache", "k_rope_cache", "kv_scale", "block_table",
                                   "seq_lens")}
    out["workload"] = inp["workload"]
    return out


# ---------------------------------------------------------------------------------------
# DeepSeek Sparse Attention inputs ("TransMLA & Sparse Latent Attention" lesson, Chapter 6
# "The lightning indexer": H^I = 64 indexer heads of width d^I = 128, top k = 2048 of a
# 128K context). The indexer's query and its key side-cache are stored as e4m3 codes with
# one fp32 scale per vector (per indexer head of a query row; per cached token), the
# per-head weights as fp32. The key side-cache shares the latent cache's block table.

@dataclass(frozen=True)
class DsaWorkload:
    """A sparse decode problem: the latent-cache decode workload plus the indexer's shapes."""
    name: str
    mla: Workload
    HI: int = 64
    dI: int = 128
    top_k: int = 2048
    w_std: float = 1.0 / 8.0
    description: str = ""

    @property
    def seed(self) -> int:
        return self.mla.seed


DSA_WORKLOADS = [
    DsaWorkload(
        "dsa_small",
        Workload(name="dsa_small_mla", B=3, Sq=1, H=32, r=512, d_r=64, seq_lens=(300, 4100, 2500),
                 q_std=1.0, c_std=1.0 / math.sqrt(512.0), outlier_frac=0.01, seed=1100),
        top_k=512,
        description="small sparse decode: B=3 H=32, L = 300 / 4100 / 2500 (one list shorter than k), k=512"),
    DsaWorkload(
        "dsa_v32",
        Workload(name="dsa_v32_mla", B=32, Sq=1, H=128, r=512, d_r=64, seq_lens=(131072,) * 32,
                 q_std=1.0, c_std=1.0 / math.sqrt(512.0), outlier_frac=0.01, seed=1101),
        description="DeepSeek-V3.2-shaped sparse decode: B=32 H=128 at the end of a 128K context, "
                    "indexer 64 heads x 128 (FP8), top 2048"),
]
DSA_BY_NAME = {w.name: w for w in DSA_WORKLOADS}


def make_dsa_inputs(w: DsaWorkload, threads: int | None = None, with_cache: bool = True) -> dict:
    """Inputs of one sparse decode step: the latent-cache decode inputs of ``w.mla`` (unless
    ``with_cache`` is False) plus the indexer query codes / scales / weights and the key
    side-cache (host numpy)."""
    threads = threads or min(16, os.cpu_count() or 1)
    res = make_inputs(w.mla, threads) if with_cache else None
    m = w.mla
    lens = resolve_seq_lens(m)
    bs = m.block_size
    if res is None:
        # the same block table as make_inputs (identical draws), without the latent cache
        tmp = make_inputs(m.with_(r=2, d_r=0, cache_dtype=F32, q_dtype=F32), threads)
        block_table, num_blocks = tmp["block_table"], tmp["num_blocks"]
        res = dict(workload=m, seq_lens=lens, block_table=block_table, num_blocks=num_blocks,
                   max_blocks_per_seq=block_table.shape[1])
    num_blocks = res["num_blocks"]
    ss_q, ss_w, ss_k = np.random.SeedSequence([m.seed, 23]).spawn(3)
    q = _fill_normal(ss_q, m.B * m.Sq * w.HI * w.dI, threads).reshape(m.B, m.Sq, w.HI, w.dI)
    wts = _fill_normal(ss_w, m.B * m.Sq * w.HI, threads).reshape(m.B, m.Sq, w.HI) * np.float32(w.w_std)
    k = _fill_normal(ss_k, num_blocks * bs * w.dI, threads).reshape(num_blocks, bs, w.dI)
    q_codes, q_scale = quantize_e4m3_per_token(q)
    k_codes, k_scale = quantize_e4m3_per_token(k)
    if "poison" in res:   # slots no sequence may read hold NaN here too
        k_codes[res["poison"]] = E4M3_NAN
        k_scale[res["poison"]] = np.nan
    res.update(dsa=w, iq_codes=q_codes, iq_scale=q_scale, iw=wts.astype(np.float32), ik_codes=k_codes,
               ik_scale=k_scale, top_k=w.top_k, max_seq_len=int(lens.max()) if lens.size else 0)
    return res
