"""Named attention workloads and their seeded bf16 inputs.

Shapes are per head ``[B, H, N, d]`` (d fastest).  Values are iid N(0, 1)
(times ``std``) drawn in fp32 from a CPU ``torch.Generator`` and rounded to
bf16 (round-to-nearest-even), in the order Q, K, V; the output gradient dO of
the backward workload comes from a second seed.  The workloads follow the
shapes the FlashAttention pages discuss: a tiny smoke case, a GPT-2-like
sequence length (FlashAttention (NL), "Empirische resultaten": GPT-2 at 1K),
a causal LLM shape, its backward with recomputation (memory-optimized flash
attention page, "How it works"), long-context sliding-window cases
(sparse-attention glossary, "Abgrenzung": sliding-window attention), shared
K/V heads, and one generation step over a key/value cache (FlashAttention (NL),
"Gespecialiseerde oplossingen"), where Q has Nq rows and K, V have N.

Nothing in this module computes attention.
"""

from __future__ import annotations

import math
import random
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool = False
    window: int = 0          # 0 = no band; W > 0 keeps keys i-W+1 .. i (causal) or |i-j| <= W-1
    std: float = 1.0
    seed: int = 0
    grad_seed: int | None = None   # seed of dO (backward workloads)
    oracle_heads: int | None = None  # heads the oracle checks (None = all)
    description: str = ""
    H_kv: int | None = None  # K/V heads (None = H); H must be a multiple (shared K/V heads)
    Nq: int | None = None    # query rows (None = N); fewer rows than keys: the last Nq positions

    @property
    def scale(self) -> float:
        # the 1/sqrt(d_k) of the attention formula (FlashAttention (NL),
        # "Problemen met standaard attention")
        return 1.0 / math.sqrt(self.d)

    @property
    def BH(self) -> int:
        return self.B * self.H

    @property
    def kv_heads(self) -> int:
        return self.H if self.H_kv is None else self.H_kv

    @property
    def q_rows(self) -> int:
        return self.N if self.Nq is None else self.Nq

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS: dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 2, 128, 64, seed=1001,
                     description="tiny forward B1 H2 N128 d64 non-causal"),
    "gpt2": Workload("gpt2", 4, 16, 2048, 64, seed=1002,
                     description="GPT-2-like forward B4 H16 N2048 d64 non-causal"),
    "causal": Workload("causal", 2, 32, 4096, 128, causal=True, std=0.5, seed=1003,
                       description="causal LLM-shape forward B2 H32 N4096 d128"),
    "bwd": Workload("bwd", 2, 32, 4096, 128, causal=True, std=0.5, seed=1003,
                    grad_seed=2003,
                    description="causal backward B2 H32 N4096 d128, dO seed 2003"),
    "long": Workload("long", 1, 16, 32768, 128, causal=True, window=4096, seed=1005,
                     oracle_heads=2,
                     description="long-context forward B1 H16 N32768 d128 causal+window 4096"),
    # the same length with the local window on both sides (non-causal sliding-window attention)
    "swa": Workload("swa", 1, 16, 32768, 128, window=4096, seed=1006, grad_seed=2006, oracle_heads=2,
                    description="long-context two-sided window B1 H16 N32768 d128, |i-j| < 4096"),
    # the causal LLM shape with 8 K/V heads for 32 query heads (grouped-query attention)
    "gqa": Workload("gqa", 2, 32, 4096, 128, causal=True, std=0.5, seed=1007, grad_seed=2007, H_kv=8,
                    description="causal B2 H32 (8 K/V heads) N4096 d128"),
    # head dimension 256 (the pages list it among what FlashAttention-2 supports)
    "d256": Workload("d256", 2, 16, 4096, 256, causal=True, std=0.5, seed=1010, grad_seed=2010,
                     description="causal B2 H16 N4096 d256"),
    # one generation step over a key/value cache: one new row per query head, 64 query heads
    # on 8 K/V heads (a 70B-class grouped-query layout), 32768 cached positions
    "decode": Workload("decode", 8, 64, 32768, 128, causal=True, seed=1008, H_kv=8, Nq=1,
                       description="decode B8 H64 (8 K/V heads) N_q 1 over N_k 32768 d128 causal"),
}


def _randn_bf16(gen: torch.Generator, shape, std: float) -> torch.Tensor:
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(torch.bfloat16)


def make_inputs(wl: Workload, seed: int | None = None):
    """Q [B, H, Nq, d] and K, V [B, H_kv, N, d] as contiguous CPU bf16 tensors."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(wl.seed if seed is None else seed)
    q = _randn_bf16(gen, (wl.B, wl.H, wl.q_rows, wl.d), wl.std)
    k = _randn_bf16(gen, (wl.B, wl.kv_heads, wl.N, wl.d), wl.std)
    v = _randn_bf16(gen, (wl.B, wl.kv_heads, wl.N, wl.d), wl.std)
    return q, k, v


def quantize_e4m3(x: torch.Tensor):
    """Per-tensor E4M3 codes of x: scale = max|x| / 448 (the largest E4M3 value), codes =
    x / scale rounded to nearest even by torch's float8_e4m3fn conversion, as uint8.
    Returns (codes, scale)."""
    amax = float(x.float().abs().max())
    scale = amax / 448.0 if amax > 0 else 1.0
    codes = (x.float() / scale).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale


def make_inputs_fp8kv(wl: Workload, seed: int | None = None):
    """make_inputs with K and V quantised to E4M3 per tensor: (Q bf16, K8, V8, s_k, s_v)."""
    q, k, v = make_inputs(wl, seed)
    k8, s_k = quantize_e4m3(k)
    v8, s_v = quantize_e4m3(v)
    return q, k8, v8, s_k, s_v


def make_inputs_fp8(wl: Workload, seed: int | None = None):
    """make_inputs with Q, K and V quantised to E4M3 per tensor, V returned transposed
    ([B, H_kv, d, N], contiguous): (Q8, K8, V8^T, s_q, s_k, s_v)."""
    q, k, v = make_inputs(wl, seed)
    q8, s_q = quantize_e4m3(q)
    k8, s_k = quantize_e4m3(k)
    v8, s_v = quantize_e4m3(v)
    return q8, k8, v8.transpose(-1, -2).contiguous(), s_q, s_k, s_v


def make_grad_output(wl: Workload, seed: int | None = None) -> torch.Tensor:
    """dO as a contiguous CPU bf16 tensor [B, H, N, d], N(0, 1) from the grad seed."""
    s = seed if seed is not None else (wl.grad_seed if wl.grad_seed is not None else wl.seed + 1000)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(s)
    return _randn_bf16(gen, (wl.B, wl.H, wl.N, wl.d), 1.0)


def head_subset(wl: Workload, count: int, seed: int | None = None) -> list[int]:
    """A seeded, sorted sample of flat head indices b*H + h."""
    rng = random.Random(wl.seed if seed is None else seed)
    count = min(count, wl.BH)
    return sorted(rng.sample(range(wl.BH), count))
