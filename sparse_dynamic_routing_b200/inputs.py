"""Seeded synthetic inputs for the Graph Machine sparse layer.

This module only draws random data. It holds none of the layer's arithmetic, so both the
CUDA library's tests and benchmark and the CPU oracle's tests take their inputs from it.

What it draws, per the workloads of "Graph Machine: Towards Better Pretraining via Edges"
(arXiv 2609.02881), as summarised on ai.info ("Methodology in Plain English": Qwen3-0.6B
backbone, 4,096-token packed sequences; "Main Findings": 2 or 4 positions per KV head):

* node features q, k, v and the upstream gradient dO: i.i.d. N(0, 1), drawn in fp32 and
  rounded to bf16 (round-to-nearest-even) where the workload is bf16;
* edge indices int32 of shape [B, n, k, s]: each slot independently uniform over the causal
  predecessors {0..i} of its position i (position 0 can only point at itself, the padding
  token that sits at the start of every packed sequence), optionally mixed with a local
  window {max(0, i - window + 1)..i};
* edge weights fp32 of shape [B, n, k, s]: one Dirichlet(alpha) draw in fp64 per
  (b, i, channel) row over its s slots, rounded to fp32;
* for the leg sparsification in front of the referral ("Methodology in Plain English",
  referral paragraph: the stored edges are mixed into a pair of legs), the stored edges E
  [B, n, k, s1] drawn as above and two sets of mixing coefficients [B, n, k, k]: one
  Dirichlet(1) draw in fp64 per (b, i, leg channel) over the k stored channels, rounded to
  fp32 (non-negative, summing to one, like a softmax over channel logits).

Every stream (q, k, v, dO, indices, weights, and per layer for the stacked workload) has its
own numpy Generator seeded from (seed, stream id[, layer]), so any one tensor can be redrawn
without drawing the others.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

# stream ids
_Q, _K, _V, _DO, _IDX1, _W1, _IDX2, _W2, _EIDX, _EW, _MIX1, _MIX2 = range(12)


@dataclass(frozen=True)
class Workload:
    """Shape and distribution of one synthetic workload."""

    name: str
    kind: str  # "ser_sea" (SER then SEA forward), "stack" (L layers), "sea_train" (SEA fwd+bwd)
    B: int
    n: int
    hq: int
    hkv: int
    d: int
    s1: int
    s2: int
    s3: int
    dtype: str  # "f32" or "bf16": type of q/k/v/o/dO
    alpha: float = 1.0  # Dirichlet concentration of the edge weights
    local_frac: float = 0.0  # probability that an index is drawn from the local window
    window: int = 64  # local window length (positions i-window+1 .. i)
    layers: int = 1
    seed: int = 1000

    @property
    def s(self) -> int:
        """Edges read by SEA per (token, KV head): the referral output width s1."""
        return self.s1

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def scale(self) -> float:
        return float(np.float32(1.0 / np.sqrt(self.d)))

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


# The five workloads. Sizes follow the Qwen3-0.6B shape (16 query / 8 KV heads, head_dim 128,
# n = 4096) and the 2- and 4-position access budgets of the two model families.
WORKLOADS = {
    "tiny_b1_n128_s2_f32": Workload(
        "tiny_b1_n128_s2_f32", "ser_sea", B=1, n=128, hq=2, hkv=1, d=64,
        s1=2, s2=2, s3=2, dtype="f32", alpha=1.0, seed=1001),
    "layer_b8_n4096_s2": Workload(
        "layer_b8_n4096_s2", "ser_sea", B=8, n=4096, hq=16, hkv=8, d=128,
        s1=2, s2=2, s3=2, dtype="bf16", alpha=1.0, seed=1002),
    "layer_b8_n4096_s4_local": Workload(
        "layer_b8_n4096_s4_local", "ser_sea", B=8, n=4096, hq=16, hkv=8, d=128,
        s1=4, s2=4, s3=4, dtype="bf16", alpha=0.5, local_frac=0.5, window=64, seed=1003),
    "stack21_b16_n4096_s4": Workload(
        "stack21_b16_n4096_s4", "stack", B=16, n=4096, hq=16, hkv=8, d=128,
        s1=4, s2=4, s3=4, dtype="bf16", alpha=1.0, layers=21, seed=1004),
    "long_b1_n32768_s4_train": Workload(
        "long_b1_n32768_s4_train", "sea_train", B=1, n=32768, hq=16, hkv=8, d=128,
        s1=4, s2=4, s3=4, dtype="bf16", alpha=1.0, seed=1005),
}
WORKLOAD_ORDER = list(WORKLOADS)


def _rng(seed: int, stream: int, layer: int = 0) -> np.random.Generator:
    return np.random.default_rng([seed, stream, layer])


def features(seed: int, stream: int, shape, dtype: torch.dtype, layer: int = 0) -> torch.Tensor:
    """N(0,1) features drawn in fp32, rounded to `dtype` (CPU tensor, contiguous)."""
    x = _rng(seed, stream, layer).standard_normal(size=tuple(shape), dtype=np.float32)
    t = torch.from_numpy(x)
    return t if dtype == torch.float32 else t.to(dtype)


def edge_indices(rng: np.random.Generator, B: int, n: int, k: int, s: int,
                 local_frac: float = 0.0, window: int = 64) -> np.ndarray:
    """int32 [B, n, k, s]; slot t ~ U{0..i}, or with prob. local_frac U{max(0,i-window+1)..i}."""
    shape = (B, n, k, s)
    hi = np.broadcast_to(np.arange(1, n + 1, dtype=np.int64)[None, :, None, None], shape)
    t = rng.integers(0, hi)
    if local_frac > 0.0:
        lo = np.maximum(hi - window, 0)
        local = rng.integers(lo, hi)
        pick = rng.random(size=shape) < local_frac
        t = np.where(pick, local, t)
    return np.ascontiguousarray(t.astype(np.int32))


def edge_weights(rng: np.random.Generator, B: int, n: int, k: int, s: int,
                 alpha: float) -> np.ndarray:
    """fp32 [B, n, k, s]: Dirichlet(alpha) over each row's s slots, drawn in fp64."""
    w = rng.dirichlet(np.full(s, alpha, dtype=np.float64), size=(B, n, k))
    return np.ascontiguousarray(w.astype(np.float32))


def edges(wl: Workload, which: int, s: int | None = None, layer: int = 0):
    """(idx int32, w fp32) CPU tensors [B, n, hkv, s] for edge tensor `which` (1 or 2)."""
    s = wl.s1 if s is None else s
    si, sw = (_IDX1, _W1) if which == 1 else (_IDX2, _W2)
    idx = edge_indices(_rng(wl.seed, si, layer), wl.B, wl.n, wl.hkv, s, wl.local_frac, wl.window)
    w = edge_weights(_rng(wl.seed, sw, layer), wl.B, wl.n, wl.hkv, s, wl.alpha)
    return torch.from_numpy(idx), torch.from_numpy(w)


def make(wl: Workload, layer: int = 0, grad: bool = False) -> dict:
    """All inputs of one layer of `wl` as CPU tensors.

    Keys: q [B,n,hq,d], k, v [B,n,hkv,d] (wl.dtype); for "ser_sea", a1_idx/a1_w
    [B,n,hkv,s2] and a2_idx/a2_w [B,n,hkv,s3] (the two referral legs, drawn independently
    with the same law); for "sea_train" and "stack", idx/w [B,n,hkv,s1] (the edges SEA reads
    directly, or the stack's first edge tensor); dout [B,n,hq,d] when grad is set.
    """
    dt = wl.torch_dtype
    out = {
        "q": features(wl.seed, _Q, (wl.B, wl.n, wl.hq, wl.d), dt, layer),
        "k": features(wl.seed, _K, (wl.B, wl.n, wl.hkv, wl.d), dt, layer),
        "v": features(wl.seed, _V, (wl.B, wl.n, wl.hkv, wl.d), dt, layer),
    }
    if wl.kind == "sea_train":
        out["idx"], out["w"] = edges(wl, 1, wl.s1)
    elif wl.kind == "stack":
        # A stack carries one edge tensor E from layer to layer and refers it through
        # itself, E' = SER(E, E); only the first layer's E is drawn.
        out["idx"], out["w"] = edges(wl, 1, wl.s1)
    else:
        out["a1_idx"], out["a1_w"] = edges(wl, 1, wl.s2)
        out["a2_idx"], out["a2_w"] = edges(wl, 2, wl.s3)
    if grad:
        out["dout"] = features(wl.seed, _DO, (wl.B, wl.n, wl.hq, wl.d), dt, layer)
    return out


def layer_features(wl: Workload, layer: int) -> dict:
    """Fresh q/k/v of one layer of a stacked workload (CPU tensors)."""
    dt = wl.torch_dtype
    return {
        "q": features(wl.seed, _Q, (wl.B, wl.n, wl.hq, wl.d), dt, layer),
        "k": features(wl.seed, _K, (wl.B, wl.n, wl.hkv, wl.d), dt, layer),
        "v": features(wl.seed, _V, (wl.B, wl.n, wl.hkv, wl.d), dt, layer),
    }


def mixing(wl: Workload, which: int, layer: int = 0) -> torch.Tensor:
    """fp32 [B, n, hkv, hkv] mixing coefficients of leg `which` (1 or 2): Dirichlet(1) rows."""
    rng = _rng(wl.seed, _MIX1 if which == 1 else _MIX2, layer)
    m = rng.dirichlet(np.ones(wl.hkv, dtype=np.float64), size=(wl.B, wl.n, wl.hkv))
    return torch.from_numpy(np.ascontiguousarray(m.astype(np.float32)))


def leg_inputs(wl: Workload, layer: int = 0) -> dict:
    """Stored edges e_idx/e_w [B, n, hkv, s1] and mix1/mix2 [B, n, hkv, hkv] (CPU tensors).

    The legs built from them have budgets wl.s2 and wl.s3.
    """
    idx = edge_indices(_rng(wl.seed, _EIDX, layer), wl.B, wl.n, wl.hkv, wl.s1,
                       wl.local_frac, wl.window)
    w = edge_weights(_rng(wl.seed, _EW, layer), wl.B, wl.n, wl.hkv, wl.s1, wl.alpha)
    return {"e_idx": torch.from_numpy(idx), "e_w": torch.from_numpy(w),
            "mix1": mixing(wl, 1, layer), "mix2": mixing(wl, 2, layer)}
