"""Seeded synthetic inputs for the attention forward pass.

This module only draws random numbers and describes problem shapes; it holds
none of the attention arithmetic.  It is the one module that both the CUDA
path's callers (tests, bench) and the fp64 oracle's callers share.

Recipe (every workload): a CPU ``torch.Generator`` seeded with ``seed``; Q, K
and V drawn in that order as float32 ``randn`` of shape [B, H, N, d] times the
stated standard deviation, then rounded to bfloat16 (round-to-nearest-even);
for key-padded workloads the per-sequence key lengths are drawn next as
integers uniform in [lo, hi] inclusive.  The scale is the float32 value of
1/sqrt(d).  The shapes stand in for the pages' BERT-large (length 512) and
GPT-2 (length 1K) workloads by shape only; no dataset is involved.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    qk_std: float = 1.0
    kpad: tuple | None = None          # (lo, hi) inclusive range of key lengths, or None
    sample_rows_per_head: int | None = None  # rows the oracle checks per head (None: all)
    H_kv: int | None = None            # key/value heads (grouped attention); None: H
    Nk: int | None = None              # keys (more keys than queries: cached keys); None: N
    splits: int = 0                    # key splits the benchmark uses (0: none, -1: library's choice)
    dtype: str = "bf16"                # element type of Q, K, V: "bf16" or "e4m3"
    pass_: str = "fwd"                 # "fwd" (O and lse) or "bwd" (dQ, dK, dV for a seeded dO)
    seed: int = 0
    notes: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        # the float32 value the kernel receives, as a Python float
        return float(torch.tensor(1.0 / math.sqrt(self.d), dtype=torch.float32).item())

    @property
    def kv_heads(self) -> int:
        return self.H if self.H_kv is None else self.H_kv

    @property
    def keys(self) -> int:
        return self.N if self.Nk is None else self.Nk

    def flops(self) -> float:
        """Nominal attention FLOPs: 4*B*H*N^2*d, halved when causal; with N_k != N,
        4*B*H*d times the allowed (query, key) pairs (bottom-right causal mask).
        The backward pass counts 2.5 times the forward (five products of the
        forward's size instead of two)."""
        if self.pass_ == "bwd":
            return 2.5 * Workload.flops(replace(self, pass_="fwd"))
        if self.Nk is None or self.Nk == self.N:
            f = 4.0 * self.B * self.H * self.N * self.N * self.d
            return f / 2 if self.causal else f
        N, Nk = self.N, self.Nk
        pairs = sum(max(0, min(Nk, i + 1 + Nk - N)) for i in range(N)) if self.causal else N * Nk
        return 4.0 * self.B * self.H * self.d * pairs


# The five workloads; seeds are 52000 + workload number.
WORKLOADS = {
    1: Workload("tiny B1 H1 N128 d64 non-causal", 1, 1, 128, 64, False, seed=52001),
    2: Workload("gpt2-small-shaped B8 H12 N1024 d64 causal", 8, 12, 1024, 64, True, seed=52002),
    3: Workload("bert-large-shaped B16 H16 N512 d64 key-padded L~U[256,512]", 16, 16, 512, 64,
                False, kpad=(256, 512), seed=52003),
    4: Workload("long-context causal B1 H32 N16384 d128", 1, 32, 16384, 128, True,
                sample_rows_per_head=512, seed=52004),
    5: Workload("softmax-stress causal B1 H16 N65536 d128 QK~N(0,4^2)", 1, 16, 65536, 128, True,
                qk_std=4.0, sample_rows_per_head=256, seed=52005),
    # grouped key/value heads (multi-query family): 8 key/value heads serve 32 query heads
    6: Workload("long-context causal grouped-KV B1 H32 Hkv8 N16384 d128", 1, 32, 16384, 128, True,
                sample_rows_per_head=128, seed=52006, H_kv=8),
    # cached keys: 256 new queries per head against 128K keys, key range split across SMs
    7: Workload("cached-keys causal grouped-KV B1 H32 Hkv8 Nq256 Nk131072 d128 split-KV", 1, 32, 256, 128, True,
                sample_rows_per_head=16, seed=52007, H_kv=8, Nk=131072, splits=-1),
    # head dimension 256: the FLOPs of workload 4 with half the heads
    8: Workload("long-context causal B1 H16 N16384 d256", 1, 16, 16384, 256, True,
                sample_rows_per_head=256, seed=52008),
    # FP8: the shape of workload 4 with E4M3 inputs (unit scales)
    9: Workload("long-context causal FP8-E4M3 B1 H32 N16384 d128", 1, 32, 16384, 128, True,
                sample_rows_per_head=64, seed=52009, dtype="e4m3"),
    # the backward pass of workload 4's shape, for a seeded dO ~ N(0, 1)
    10: Workload("backward long-context causal B1 H32 N16384 d128", 1, 32, 16384, 128, True,
                 sample_rows_per_head=64, seed=52010, pass_="bwd"),
    # a small backward case of the same kernel (profiler captures)
    11: Workload("backward causal B1 H8 N4096 d128", 1, 8, 4096, 128, True, seed=52011, pass_="bwd"),
}


def make_dout(w: Workload):
    """The seeded upstream gradient dO ~ N(0, 1), bf16 [B, H, N, d], of a backward workload."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed + 1)
    return torch.randn((w.B, w.H, w.N, w.d), generator=g, dtype=torch.float32).to(torch.bfloat16)


def make_inputs(w: Workload, seed: int | None = None):
    """Draw (q, k, v, k_len) on the CPU for workload ``w``.

    q: [B, H, N, d]; k, v: [B, H_kv, N_k, d] contiguous CPU tensors of bfloat16
    (or float8_e4m3fn, rounded from the same float32 draws, for dtype "e4m3").
    k_len: int32 [B] CPU tensor, or None when the workload has no key padding.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    shape = (w.B, w.H, w.N, w.d)
    kv_shape = (w.B, w.kv_heads, w.keys, w.d)
    dt = torch.float8_e4m3fn if w.dtype == "e4m3" else torch.bfloat16
    q = (torch.randn(shape, generator=g, dtype=torch.float32) * w.qk_std).to(dt)
    k = (torch.randn(kv_shape, generator=g, dtype=torch.float32) * w.qk_std).to(dt)
    v = torch.randn(kv_shape, generator=g, dtype=torch.float32).to(dt)
    k_len = None
    if w.kpad is not None:
        lo, hi = w.kpad
        k_len = torch.randint(lo, hi + 1, (w.B,), generator=g, dtype=torch.int64).to(torch.int32)
    return q, k, v, k_len


def sample_rows(w: Workload, seed: int | None = None):
    """Flat row ids (b*H + h)*N + i the oracle checks for ``w``.

    All rows when ``w.sample_rows_per_head`` is None; otherwise, per (b, h), a
    seeded uniform sample without replacement of that many query rows, plus
    rows 0 and N-1, sorted.
    """
    import numpy as np

    n_bh = w.B * w.H
    if w.sample_rows_per_head is None:
        return np.arange(n_bh * w.N, dtype=np.int64)
    rng = np.random.default_rng((w.seed if seed is None else seed) + 7)
    out = []
    for bh in range(n_bh):
        pick = rng.choice(w.N, size=min(w.sample_rows_per_head, w.N), replace=False)
        pick = np.union1d(pick, [0, w.N - 1])
        out.append(bh * w.N + pick.astype(np.int64))
    return np.concatenate(out)


def custom(B, H, N, d, causal, qk_std=1.0, kpad=None, seed=1, name="custom", H_kv=None, Nk=None,
           splits=0, dtype="bf16") -> Workload:
    """A workload of arbitrary shape (tests of ragged and edge shapes)."""
    return Workload(name, B, H, N, d, causal, qk_std=qk_std, kpad=kpad, seed=seed, H_kv=H_kv, Nk=Nk,
                    splits=splits, dtype=dtype)
