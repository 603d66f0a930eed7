"""Seeded synthetic inputs for gated block-sparse decode.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic, so both the CUDA path and the fp64 oracle can be fed from
it. The shapes follow the long-reasoning decode setting of "SeerAttention-R:
Sparse Attention Adaptation for Long Reasoning" (abstract: a 4K-token budget,
sparse block sizes 64/128, high sparsity); there is no public dataset on this
path, so seeded N(0, 1) caches stand in for real activations.

Recipe (the same on every machine for a given device type and seed):
  * q, K, V: float32 N(0, 1) cast to bf16 (round to nearest even). K and V
    are [B, Hkv, Lmax, D]; positions t >= L_b are filled too (with N(0, 1)
    draws, or with ``pad_value`` when given, e.g. NaN to test masking).
  * W_q, W_k: float32 N(0, sigma^2), sigma = 1 / sqrt(D), shape [Hkv, dg, D].
  * salient blocks (large-block workload): per (b, kvh) row, ceil(frac * NB)
    blocks chosen uniformly without replacement get K x ``salient_scale``
    before the bf16 cast.
  * ragged lengths: L_b drawn uniformly from [lo, hi] with numpy's PCG64
    seeded by (seed, b), redrawn while L_b is a multiple of the block size,
    so the last block of every sequence is partial.
Draw order: seq_lens, K, V, salient choice, q, W_q, W_k.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    gate_dim: int
    block_size: int
    max_seq_len: int
    budget_tokens: int
    ragged: tuple = ()             # (lo, hi) inclusive when ragged, else ()
    salient_frac: float = 0.0
    salient_scale: float = 3.0
    description: str = ""

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def nb_max(self) -> int:
        return (self.max_seq_len + self.block_size - 1) // self.block_size

    @property
    def kmax(self) -> int:
        return self.budget_tokens // self.block_size

    def dims(self) -> dict:
        return dict(batch=self.batch, num_q_heads=self.num_q_heads, num_kv_heads=self.num_kv_heads,
                    head_dim=self.head_dim, gate_dim=self.gate_dim, block_size=self.block_size,
                    max_seq_len=self.max_seq_len)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def budget_for_fraction(frac: float, max_seq_len: int, block_size: int) -> int:
    """Token budget that keeps ceil(frac * NB) blocks of a full-length sequence."""
    nb = (max_seq_len + block_size - 1) // block_size
    return int(math.ceil(frac * nb)) * block_size


def _sweep(batch: int, frac: float | None) -> Workload:
    L, blk = 131072, 128
    budget = L if frac is None else budget_for_fraction(frac, L, blk)
    tag = "dense" if frac is None else "keep%02d" % round(frac * 100)
    return Workload(f"sweep_b{batch}_{tag}", batch, 40, 8, 128, 128, blk, L, budget,
                    description=f"batch {batch}, 40 q / 8 kv heads, head_dim 128, context 131072, "
                                f"block 128, " + ("all blocks" if frac is None else f"keep {frac:.0%}"))


WORKLOADS: dict[str, Workload] = {w.name: w for w in [
    Workload("tiny", 1, 4, 1, 64, 64, 64, 2048, 512,
             description="batch 1, 1 kv head, 4 q heads, head_dim 64, context 2048, block 64, "
                         "budget 512 (8 of 32 blocks incl. last), gate dim 64"),
    Workload("decode_b16", 16, 32, 8, 128, 128, 64, 32768, 4096,
             description="batch 16, 32 q / 8 kv heads, head_dim 128, context 32768, block 64, "
                         "budget 4096 (64 of 512 blocks, 87.5% sparsity), gate dim 128"),
    Workload("large_block", 8, 32, 8, 128, 128, 128, 65536, budget_for_fraction(0.10, 65536, 128),
             salient_frac=0.05,
             description="batch 8, 32 q / 8 kv heads, head_dim 128, context 65536, block 128, "
                         "keep 10% (52 of 512 blocks), 5% of K blocks scaled x3"),
    Workload("ragged", 64, 32, 8, 128, 128, 64, 32768, 4096, ragged=(4096, 32768),
             description="64 sequences, lengths uniform in [4096, 32768] with a partial last "
                         "block, 32 q / 8 kv heads, head_dim 128, block 64, budget 4096"),
] + [_sweep(b, f) for b in (1, 4) for f in (0.5, 0.3, 0.1, 0.05, None)]}


def seq_lens_for(wl: Workload, seed: int) -> np.ndarray:
    if not wl.ragged:
        return np.full(wl.batch, wl.max_seq_len, np.int32)
    lo, hi = wl.ragged
    out = np.empty(wl.batch, np.int32)
    for b in range(wl.batch):
        rng = np.random.Generator(np.random.PCG64([seed, b]))
        while True:
            L = int(rng.integers(lo, hi + 1))
            if L % wl.block_size != 0:
                break
        out[b] = L
    return out


def make_inputs(wl: Workload, seed: int = 0, device="cpu", pad_value: float | None = None,
                seq_lens: np.ndarray | None = None) -> dict:
    """Seeded inputs for one decode step of ``wl`` on ``device``.

    Returns q [B,Hq,D] bf16, k_cache / v_cache [B,Hkv,Lmax,D] bf16,
    w_q / w_k [Hkv,dg,D] fp32, seq_lens [B] int32 (on ``device``), plus
    ``seq_lens_host`` (numpy) and the workload.
    """
    device = torch.device(device)
    lens = seq_lens_for(wl, seed) if seq_lens is None else np.asarray(seq_lens, np.int32)
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    B, Hq, Hkv, D, dg, L = (wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.gate_dim,
                            wl.max_seq_len)
    shape = (B, Hkv, L, D)

    def normal(*shp):
        return torch.randn(*shp, generator=g, device=device, dtype=torch.float32)

    k = normal(*shape)
    v = normal(*shape)
    if wl.salient_frac > 0:
        nb = wl.nb_max
        n_sal = int(math.ceil(wl.salient_frac * nb))
        scale = torch.ones(B, Hkv, nb, device=device)
        for r in range(B * Hkv):
            pick = torch.randperm(nb, generator=g, device=device)[:n_sal]
            scale.view(B * Hkv, nb)[r, pick] = wl.salient_scale
        if L % wl.block_size == 0:
            k.view(B, Hkv, nb, wl.block_size, D).mul_(scale[..., None, None])
        else:
            _scale_ragged_blocks(k, scale, wl.block_size)
    k = k.to(torch.bfloat16)
    v = v.to(torch.bfloat16)
    q = normal(B, Hq, D).to(torch.bfloat16)
    sigma = 1.0 / math.sqrt(D)
    w_q = normal(Hkv, dg, D) * sigma
    w_k = normal(Hkv, dg, D) * sigma
    if pad_value is not None:
        for b in range(B):
            if int(lens[b]) < L:
                k[b, :, int(lens[b]):, :] = pad_value
                v[b, :, int(lens[b]):, :] = pad_value
    return dict(q=q, k_cache=k, v_cache=v, w_q=w_q, w_k=w_k,
                seq_lens=torch.from_numpy(lens).to(device), seq_lens_host=lens, workload=wl)


def _scale_ragged_blocks(k, scale, blk):
    nb = scale.shape[-1]
    for j in range(nb):
        k[:, :, j * blk:(j + 1) * blk, :] *= scale[:, :, j, None, None]


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a tensor as a host uint16 array (the oracle's input form)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def identity_block_list(seq_lens_host: np.ndarray, num_kv_heads: int, block_size: int,
                        nb_max: int) -> tuple[np.ndarray, np.ndarray]:
    """Block list of a dense decode: every block 0..NB_b-1 of every row (kmax = NBmax)."""
    B = len(seq_lens_host)
    idx = np.full((B, num_kv_heads, nb_max), -1, np.int32)
    nsel = np.zeros((B, num_kv_heads), np.int32)
    for b in range(B):
        nb = (int(seq_lens_host[b]) + block_size - 1) // block_size
        idx[b, :, :nb] = np.arange(nb, dtype=np.int32)
        nsel[b, :] = nb
    return idx, nsel
