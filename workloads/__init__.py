"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds shapes and random numbers only -- none of the attention
arithmetic.  Both sides of every parity check (the CUDA library and the fp64
oracle) consume the tensors it returns, after the same rounding to the 16-bit
input dtype.

Recipe: every tensor is i.i.d. N(0, 1), drawn in fp32 on the CPU with
``torch.Generator().manual_seed(1000 * config_id + tensor_id)`` (Q=0, K=1,
V=2, dO=3, seqlens=4), then rounded to the workload dtype.  scale = 1/sqrt(d).
For decode, the first half of the batch has Nk = Nk_max and the second half
draws Nk uniformly from [1024, Nk_max] with the seqlens generator.
"""
from __future__ import annotations

import dataclasses
import math

import torch

__all__ = ["Workload", "WORKLOADS", "get", "make_inputs", "make_decode_inputs", "seqlens_for", "workload_inputs",
           "rotation_signs", "block_mask_local", "block_mask_random"]


@dataclasses.dataclass(frozen=True)
class Workload:
    id: int
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    dtype: str  # "fp16" | "bf16"
    causal: tuple  # causal settings exercised
    backward: bool = False
    decode: bool = False

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def torch_dtype(self):
        return torch.float16 if self.dtype == "fp16" else torch.bfloat16


WORKLOADS = {
    1: Workload(1, "tiny forward", 1, 2, 2, 128, 128, 64, "fp16", (False, True)),
    2: Workload(2, "MHA prefill forward", 4, 16, 16, 2048, 2048, 128, "bf16", (False, True)),
    3: Workload(3, "GQA training step", 1, 32, 8, 8192, 8192, 128, "bf16", (True,), backward=True),
    4: Workload(4, "long-context GQA", 1, 32, 8, 16384, 16384, 128, "bf16", (True,), backward=True),
    5: Workload(5, "split-KV decode", 64, 32, 8, 1, 32768, 128, "bf16", (False,), decode=True),
}


def get(i: int) -> Workload:
    return WORKLOADS[i]


def _normal(shape, seed: int, dtype, device="cpu") -> torch.Tensor:
    """N(0,1) drawn in fp32 with a generator seeded ``seed`` on ``device``, then
    rounded to ``dtype``.  CPU and CUDA generators give different streams; a
    workload is always generated on one device and copied from there."""
    g = torch.Generator(device=device).manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float32, device=device).to(dtype)


def make_inputs(B, Hq, Hkv, Nq, Nk, d, dtype=torch.bfloat16, seed_base=0, with_do=False, device="cpu"):
    """q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d] (and dO like q), tensors of ``dtype`` on ``device``."""
    q = _normal((B, Nq, Hq, d), seed_base + 0, dtype, device)
    k = _normal((B, Nk, Hkv, d), seed_base + 1, dtype, device)
    v = _normal((B, Nk, Hkv, d), seed_base + 2, dtype, device)
    if not with_do:
        return q, k, v
    do = _normal((B, Nq, Hq, d), seed_base + 3, dtype, device)
    return q, k, v, do


def rotation_signs(d: int, seed: int, device="cpu") -> torch.Tensor:
    """fp32 [d] of +-1, each sign drawn with probability 1/2 by a generator seeded ``seed``."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    bits = torch.randint(0, 2, (d,), generator=g)
    return (bits.float() * 2 - 1).to(device)


def block_mask_local(B: int, Hq: int, nqb: int, nkb: int, window: int, sink: int = 1) -> torch.Tensor:
    """uint8 [B, Hq, nqb, nkb]: query block I sees key blocks I - window + 1 .. I and the first ``sink``."""
    i = torch.arange(nqb)[:, None]
    j = torch.arange(nkb)[None, :]
    m = ((j <= i) & (j > i - window)) | (j < sink)
    return m.to(torch.uint8).expand(B, Hq, nqb, nkb).contiguous()


def block_mask_random(B: int, Hq: int, nqb: int, nkb: int, density: float, seed: int) -> torch.Tensor:
    """uint8 [B, Hq, nqb, nkb], each block visible with probability ``density`` (seeded)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.rand(B, Hq, nqb, nkb, generator=g) < density).to(torch.uint8)


def seqlens_for(B: int, Nk_max: int, seed: int, lo: int = 1024) -> torch.Tensor:
    """int32 [B]: b < B/2 -> Nk_max; b >= B/2 -> uniform integer in [min(lo, Nk_max), Nk_max]."""
    g = torch.Generator().manual_seed(seed)
    lo = min(lo, Nk_max)
    half = B // 2
    tail = torch.randint(lo, Nk_max + 1, (B - half,), generator=g, dtype=torch.int64)
    return torch.cat([torch.full((half,), Nk_max, dtype=torch.int64), tail]).to(torch.int32)


def make_decode_inputs(B, Hq, Hkv, Nk_max, d, dtype=torch.bfloat16, seed_base=0, lo=1024, device="cpu"):
    """q [B,1,Hq,d], k/v cache [B,Nk_max,Hkv,d] (on ``device``), seqlens_k int32 [B] (CPU)."""
    q = _normal((B, 1, Hq, d), seed_base + 0, dtype, device)
    kc = _normal((B, Nk_max, Hkv, d), seed_base + 1, dtype, device)
    vc = _normal((B, Nk_max, Hkv, d), seed_base + 2, dtype, device)
    sl = seqlens_for(B, Nk_max, seed_base + 4, lo)
    return q, kc, vc, sl


def workload_inputs(w: Workload, with_do=None, device="cpu"):
    """Inputs of a named workload, seeded 1000 * id + tensor id, drawn on ``device``."""
    if w.decode:
        return make_decode_inputs(w.B, w.Hq, w.Hkv, w.Nk, w.d, w.torch_dtype, 1000 * w.id, device=device)
    wd = w.backward if with_do is None else with_do
    return make_inputs(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.torch_dtype, 1000 * w.id, with_do=wd, device=device)
