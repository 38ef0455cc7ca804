"""Seeded synthetic inputs for the Elastic Attention prefill path.

This module only draws random numbers and shapes tensors.  It holds none of
the method's arithmetic, so both the CUDA path's tests/bench and the CPU
oracle can take their inputs from it without sharing any computation.

Workloads stand in for the pages' evaluation (Qwen3-4B/8B and Llama-3.1-8B on
LongBench-E/V2 and RULER up to 256K, EA blog (results copy) §4.1): the
datasets and trained weights are not used; only the layer shapes (query/kv
heads, head dim), the sequence lengths and the measured router sparsity of
Figure 6 (about 85% sparse heads on code tasks, about 68% on QA, EA blog
(results copy) §4.2) are taken over.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

__all__ = ["Workload", "WORKLOADS", "get", "make_qkv", "make_router_weights",
           "make_fixed_mask", "sparse_head_set", "layer_seed",
           "layer_sparse_frac", "decode_positions", "packed_lengths"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seq: int
    hq: int
    hkv: int
    d: int
    sink: int
    window: int
    layers: int = 1
    # fraction of heads routed sparse; for multi-layer workloads the per-layer
    # fraction is drawn uniformly from [sparse_lo, sparse_hi]
    sparse_frac: float = 0.0
    sparse_lo: float = 0.0
    sparse_hi: float = 0.0
    use_router: bool = False
    router_hidden: int = 256
    # explicit mask heads (per batch identical), used by the tiny workload
    fixed_sparse_heads: Optional[tuple] = None
    # K drawn as low-rank plus noise (rank, noise std) instead of N(0, 1)
    k_lowrank: Optional[tuple] = None
    index: int = 0

    @property
    def group(self) -> int:
        return self.hq // self.hkv


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny", batch=1, seq=512, hq=4, hkv=2, d=64, sink=16, window=128,
                 fixed_sparse_heads=(1, 3), index=0),
        Workload("llama8b", batch=1, seq=32768, hq=32, hkv=8, d=128, sink=64,
                 window=1024, sparse_frac=0.68, use_router=True, index=1),
        Workload("qwen4b", batch=2, seq=65536, hq=32, hkv=8, d=128, sink=64,
                 window=2048, sparse_frac=0.85, use_router=False, index=2),
        Workload("qwen8b36", batch=4, seq=16384, hq=32, hkv=8, d=128, sink=128,
                 window=512, layers=36, sparse_lo=0.5, sparse_hi=0.9,
                 use_router=True, index=3),
        Workload("ext256k", batch=1, seq=262144, hq=32, hkv=8, d=128, sink=128,
                 window=4096, sparse_frac=0.75, use_router=True,
                 k_lowrank=(16, 0.1), index=4),
    ]
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def layer_seed(w: Workload, layer: int = 0) -> int:
    return 1000 * w.index + layer


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_qkv(w: Workload, seed: int, device="cpu", seq: Optional[int] = None,
             batch: Optional[int] = None):
    """q [B,Hq,N,d], k and v [B,Hkv,N,d] in bf16, contiguous BHSD."""
    n = seq if seq is not None else w.seq
    b = batch if batch is not None else w.batch
    g = _gen(seed, device)
    q = torch.randn((b, w.hq, n, w.d), generator=g, device=device,
                    dtype=torch.float32).to(torch.bfloat16)
    if w.k_lowrank is None:
        k = torch.randn((b, w.hkv, n, w.d), generator=g, device=device,
                        dtype=torch.float32).to(torch.bfloat16)
    else:
        rank, noise = w.k_lowrank
        k = torch.empty((b, w.hkv, n, w.d), device=device, dtype=torch.bfloat16)
        for bi in range(b):
            u = torch.randn((n, rank), generator=g, device=device)
            vv = torch.randn((w.hkv * w.d, rank), generator=g, device=device)
            low = (u @ vv.T) / math.sqrt(rank)          # [n, Hkv*d]
            low = low.view(n, w.hkv, w.d).permute(1, 0, 2)
            k[bi] = (low + noise * torch.randn(low.shape, generator=g,
                                               device=device)).to(torch.bfloat16)
    v = torch.randn((b, w.hkv, n, w.d), generator=g, device=device,
                    dtype=torch.float32).to(torch.bfloat16)
    return q.contiguous(), k.contiguous(), v.contiguous()


def sparse_head_set(hq: int, frac: float, seed: int) -> list:
    """A seeded set of round(frac * hq) head indices."""
    g = _gen(seed + 7, "cpu")
    perm = torch.randperm(hq, generator=g).tolist()
    return sorted(perm[: int(round(frac * hq))])


def make_router_weights(in_dim: int, hidden: int, out_dim: int, sparse_heads,
                        seed: int, bias_mag: float = 0.5, w_std: float = 0.02):
    """Router weights: W ~ N(0, w_std), b1 = 0, b2 = +bias_mag on the chosen
    heads and -bias_mag elsewhere (so those heads route sparse when the data
    term is small).  Returns fp32 CPU tensors (w1 [hidden,in], b1, w2
    [out,hidden], b2)."""
    g = _gen(seed + 13, "cpu")
    w1 = torch.randn((hidden, in_dim), generator=g) * w_std
    b1 = torch.zeros(hidden)
    w2 = torch.randn((out_dim, hidden), generator=g) * w_std
    b2 = torch.full((out_dim,), -bias_mag)
    for h in sparse_heads:
        b2[h] = bias_mag
    return w1.float(), b1.float(), w2.float(), b2.float()


def gumbel_noise(batch: int, hq: int, seed: int, device="cpu"):
    """Two fp32 [batch, hq] draws of standard Gumbel noise, -log(-log U) with
    U uniform in (0, 1): the noise of the FA and SA choices that a
    Gumbel-Softmax training step takes as input."""
    g = _gen(seed + 31, "cpu")
    u = torch.rand((2, batch, hq), generator=g, dtype=torch.float64).clamp(1e-12, 1.0 - 1e-12)
    gum = (-torch.log(-torch.log(u))).float()
    return gum[0].contiguous().to(device), gum[1].contiguous().to(device)


def make_fixed_mask(w: Workload, seed: int) -> torch.Tensor:
    """uint8 [B, Hq] mask (1 = sparse), drawn independently per batch row."""
    m = torch.zeros((w.batch, w.hq), dtype=torch.uint8)
    for b in range(w.batch):
        if w.fixed_sparse_heads is not None:
            heads = list(w.fixed_sparse_heads)
        else:
            heads = sparse_head_set(w.hq, w.sparse_frac, seed + 101 * b)
        m[b, heads] = 1
    return m


def layer_sparse_frac(w: Workload, layer: int) -> float:
    """Per-layer sparse fraction, uniform in [sparse_lo, sparse_hi]."""
    if w.layers == 1:
        return w.sparse_frac
    g = _gen(layer_seed(w, layer) + 29, "cpu")
    u = torch.rand((1,), generator=g, dtype=torch.float64).item()
    return w.sparse_lo + (w.sparse_hi - w.sparse_lo) * u


def decode_positions(w: Workload, batch: int, seed: int) -> torch.Tensor:
    """int32 [batch] decode positions, ragged: uniform in [seq/2, seq - 1]
    (a serving batch whose prompts finished prefill at different lengths)."""
    g = _gen(seed + 211, "cpu")
    lo = max(0, w.seq // 2)
    return torch.randint(lo, w.seq, (batch,), generator=g, dtype=torch.int64).to(torch.int32)


def packed_lengths(w: Workload, nseq: int, seed: int) -> list:
    """Sequence lengths of a packed (ragged) prefill batch: uniform in
    [seq/8, seq], so the batch mixes short prompts with full-length ones."""
    g = _gen(seed + 307, "cpu")
    lo = max(1, w.seq // 8)
    return torch.randint(lo, w.seq + 1, (nseq,), generator=g, dtype=torch.int64).tolist()
