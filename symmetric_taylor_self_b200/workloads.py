"""Seeded synthetic workloads: shapes, seeds and value distributions only.

This module holds no part of the attention arithmetic.  Both the CUDA path
(through the tests and the benchmark) and the float64 oracle receive the same
tensors from here.

Recipe (one per (b, h) head, so any head can be regenerated alone):
  * generator: torch.Generator("cpu").manual_seed(seed * 2**20 + b * H + h)
  * draws, in order: q [T, d_K], k [T, d_K], v [T, d_V], all torch.randn fp32,
    where T = N (+ steps for the decode workload: the decode tokens follow the
    prefill tokens in the same draw)
  * "normalize": q and k rows rescaled to Euclidean norm sqrt(d_K)
  * cast to bf16 (the kernels' input type); the oracle widens these exact bf16
    values to float64.  The small d_K = 8 workload is specified in fp32; its
    draws are rounded to bf16 once so both sides see identical inputs.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d_K: int
    d_V: int
    P: int
    seed: int
    normalize: bool = False
    steps: int = 0                      # decode steps after an N-token prefill
    note: str = ""
    oracle_heads: tuple = field(default=())     # (b, h) heads the oracle checks in full
    oracle_tokens: int = 0                       # 0: all tokens of those heads

    @property
    def F(self) -> int:
        return math.comb(self.d_K + self.P - 1, self.P - 1)


WORKLOADS = {
    "tiny_d8": Workload("tiny_d8", B=1, H=1, N=256, d_K=8, d_V=8, P=4, seed=0,
                        note="fp32 N(0,1) draws, rounded to bf16 once", oracle_heads=((0, 0),)),
    "prefill_d16": Workload("prefill_d16", B=1, H=8, N=4096, d_K=16, d_V=16, P=4, seed=1,
                            oracle_heads=tuple((0, h) for h in range(8))),
    "prefill_d32": Workload("prefill_d32", B=2, H=16, N=16384, d_K=32, d_V=32, P=4, seed=2,
                            normalize=True, oracle_heads=((0, 0), (1, 15))),
    "prefill_d64": Workload("prefill_d64", B=1, H=8, N=65536, d_K=64, d_V=64, P=4, seed=3,
                            oracle_heads=((0, 0),), oracle_tokens=2048),
    "decode_d32": Workload("decode_d32", B=64, H=32, N=8192, d_K=32, d_V=32, P=4, seed=4,
                           steps=1024, oracle_heads=((0, 0), (63, 31), (17, 5), (40, 22))),
    # other head sizes and degrees: d = 128 (the state size worked out on the
    # "Fixed-size hidden state" page), d_K != d_V, and P = 6
    "prefill_d128": Workload("prefill_d128", B=1, H=8, N=16384, d_K=128, d_V=128, P=4, seed=7,
                             oracle_heads=((0, 0),), oracle_tokens=256),
    "prefill_d64_dv32": Workload("prefill_d64_dv32", B=1, H=8, N=32768, d_K=64, d_V=32, P=4, seed=8,
                                 oracle_heads=((0, 0),), oracle_tokens=1024),
    "prefill_d16_p6": Workload("prefill_d16_p6", B=1, H=8, N=4096, d_K=16, d_V=16, P=6, seed=9,
                               oracle_heads=((0, 0),), oracle_tokens=1024),
    # backward pass of the prefill (gradients of q, k, v): the prefill_d64 head
    # shape over 4096 tokens; the upstream gradient dy is N(0, 1) (cotangent())
    "backward_d64": Workload("backward_d64", B=1, H=8, N=4096, d_K=64, d_V=64, P=4, seed=5,
                             oracle_heads=((0, 0),)),
    "backward_d16": Workload("backward_d16", B=1, H=8, N=4096, d_K=16, d_V=16, P=4, seed=6,
                             oracle_heads=((0, 3),)),
    # reduced sizes of the benchmark workloads, for ncu captures
    "prefill_d64_small": Workload("prefill_d64_small", B=1, H=8, N=8192, d_K=64, d_V=64, P=4, seed=3),
    "decode_d32_small": Workload("decode_d32_small", B=8, H=32, N=256, d_K=32, d_V=32, P=4, seed=4,
                                 steps=16),
    "backward_d64_small": Workload("backward_d64_small", B=1, H=4, N=1024, d_K=64, d_V=64, P=4, seed=5),
}


def head_seed(w: Workload, b: int, h: int, H_total: int | None = None) -> int:
    """Seed of head (b, h) of the workload, or of a job of H_total heads per batch
    row made of several copies of its head shape (head h of H_total)."""
    return w.seed * 2 ** 20 + b * (w.H if H_total is None else H_total) + h


def head_inputs(w: Workload, b: int, h: int, dtype=torch.bfloat16, H_total: int | None = None):
    """q, k, v for one head over all N + steps tokens, as ``dtype`` CPU tensors."""
    g = torch.Generator("cpu").manual_seed(head_seed(w, b, h, H_total))
    T = w.N + w.steps
    q = torch.randn(T, w.d_K, generator=g)
    k = torch.randn(T, w.d_K, generator=g)
    v = torch.randn(T, w.d_V, generator=g)
    if w.normalize:
        q = q / q.norm(dim=1, keepdim=True) * math.sqrt(w.d_K)
        k = k / k.norm(dim=1, keepdim=True) * math.sqrt(w.d_K)
    return q.to(dtype), k.to(dtype), v.to(dtype)


def make_inputs(w: Workload, dtype=torch.bfloat16, h0: int = 0, H_total: int | None = None):
    """Prefill tensors [B, H, N, d] and, for decode workloads, per-step tensors
    [steps, B, H, d] (empty when steps == 0).  CPU, ``dtype``.  With H_total, the
    H heads are heads h0 .. h0 + H - 1 of a job of H_total heads per batch row (the
    shard one rank of a head-sharded job owns); by default the workload itself."""
    T = w.N + w.steps
    q = torch.empty(w.B, w.H, T, w.d_K, dtype=dtype)
    k = torch.empty(w.B, w.H, T, w.d_K, dtype=dtype)
    v = torch.empty(w.B, w.H, T, w.d_V, dtype=dtype)

    def fill(bh):
        b, h = divmod(bh, w.H)
        q[b, h], k[b, h], v[b, h] = head_inputs(w, b, h0 + h, dtype, H_total)

    # heads are independent draws (one generator each): fill them on host threads
    with ThreadPoolExecutor(max_workers=min(16, len(os.sched_getaffinity(0)))) as ex:
        list(ex.map(fill, range(w.B * w.H)))
    pre = (q[:, :, :w.N].contiguous(), k[:, :, :w.N].contiguous(), v[:, :, :w.N].contiguous())
    dec = tuple(x[:, :, w.N:].permute(2, 0, 1, 3).contiguous() for x in (q, k, v))
    return pre, dec


def random_cotangent(B, H, N, d_V, seed):
    """Seeded N(0, 1) fp32 [B, H, N, d_V]: an upstream gradient dL/dy for the
    backward pass (any values will do; a loss's gradient has no special form)."""
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randn(B, H, N, d_V, generator=g)


def cotangent(w: Workload):
    """The upstream gradient dy [B, H, N, d_V] (fp32, N(0, 1)) of a backward workload."""
    return random_cotangent(w.B, w.H, w.N, w.d_V, seed=w.seed * 2 ** 20 + 2 ** 19)


def random_inputs(B, H, N, d_K, d_V, seed, dtype=torch.bfloat16, scale=1.0, vscale=1.0):
    """Free-form seeded inputs [B, H, N, d] for edge-case tests: q, k ~ N(0, scale^2),
    v ~ N(0, vscale^2)."""
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn(B, H, N, d_K, generator=g) * scale
    k = torch.randn(B, H, N, d_K, generator=g) * scale
    v = torch.randn(B, H, N, d_V, generator=g) * vscale
    return q.to(dtype), k.to(dtype), v.to(dtype)
