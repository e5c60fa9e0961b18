"""Seeded synthetic inputs for the mixed-head causal attention layer.

This module only draws random numbers; it holds none of the layer's
arithmetic.  It is the one piece shared by the fp64 oracle's tests and the
GPU path's tests and benchmark, so both sides always see identical tensors.

Workloads follow the shapes of "When Can Attention Heads Be Statically
Defined?" (reading notes, section 三 "124M 预训练与主要控制": a 12-layer,
12-head, width-768 decoder, so d_h = 64; Table 2 for the 4K/8K contexts and
25%/50% replacement; Table 29 for the batch-64 causal prefill sweep).  The
1B-scale shape (H=32, d_h=64) is an assumption: the pages do not print it.

Recipe (all draws are independent per (tensor, b, h) slice, so any slice can
be regenerated alone for a sampled oracle check):

* Q, K, V, dO: standard normal fp32, rounded to bf16 (round-to-nearest-even).
* replaced heads: a fixed list, or the first ``n_replaced`` entries of a seeded
  permutation of range(H), sorted.
* for each replaced head h: a[j] ~ N(0, 0.5) (0.5 is the standard deviation)
  with a[0] += 4 (a sink); r[k] = -0.05 k + N(0, 0.3) with r[0] += 2.
* rows of a and r that belong to ordinary heads are NaN: the layer must never
  read them.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import torch

HEAD_DIM = 64

# slice-stream identifiers (part of the seeding recipe; never change)
_TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "do": 4, "alpha": 5, "rho": 6, "perm": 7}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    d: int = HEAD_DIM
    n_replaced: int = 0
    fixed_replaced: Optional[Tuple[int, ...]] = None
    backward: bool = True

    @property
    def tokens(self) -> int:
        return self.B * self.T


def _prefill(B: int, T: int) -> Workload:
    return Workload(f"prefill_124m_b{B}_t{T}", B=B, H=12, T=T, n_replaced=3, backward=False)


# The layer shapes exercised by tests and the benchmark.
WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny_b1_h4_t256", B=1, H=4, T=256, fixed_replaced=(2,)),
        Workload("124m_b8_t4096_r25", B=8, H=12, T=4096, n_replaced=3),
        Workload("124m_b4_t8192_r50", B=4, H=12, T=8192, n_replaced=6),
        Workload("1b_b4_h32_t8192_r25", B=4, H=32, T=8192, n_replaced=8),
    ]
    + [_prefill(64, T) for T in (512, 1024, 2048, 4096, 8192, 16384)]
    + [_prefill(B, 4096) for B in (1, 8, 16, 32)]
}

PREFILL_SWEEP = [n for n in WORKLOADS if n.startswith("prefill_")]


def custom(B: int, H: int, T: int, replaced: Sequence[int], backward: bool = True) -> Workload:
    """An ad-hoc shape (edge cases: ragged T, all/none replaced, ...)."""
    return Workload(f"custom_b{B}_h{H}_t{T}", B=B, H=H, T=T,
                    fixed_replaced=tuple(sorted(set(int(h) for h in replaced))), backward=backward)


def _gen(seed: int, tensor: str, b: int = 0, h: int = 0) -> torch.Generator:
    # torch's CPU generator keeps only 32 bits of its seed: hash the slice id
    key = f"{int(seed)}/{_TENSOR_IDS[tensor]}/{int(b)}/{int(h)}".encode()
    s = int.from_bytes(hashlib.blake2b(key, digest_size=4).digest(), "little")
    g = torch.Generator(device="cpu")
    g.manual_seed(s)
    return g


def replaced_heads(w: Workload, seed: int = 0) -> List[int]:
    if w.fixed_replaced is not None:
        return list(w.fixed_replaced)
    perm = torch.randperm(w.H, generator=_gen(seed, "perm"))
    return sorted(int(x) for x in perm[: w.n_replaced])


def replaced_mask(w: Workload, seed: int = 0) -> torch.Tensor:
    m = torch.zeros(w.H, dtype=torch.uint8)
    for h in replaced_heads(w, seed):
        m[h] = 1
    return m


def make_slice(w: Workload, seed: int, tensor: str, b: int, h: int) -> torch.Tensor:
    """One [T, d] bf16 slice of q/k/v/do."""
    x = torch.randn(w.T, w.d, generator=_gen(seed, tensor, b, h), dtype=torch.float32)
    return x.to(torch.bfloat16)


def make_tensor(w: Workload, seed: int, tensor: str, out: Optional[torch.Tensor] = None,
                threads: int = 0) -> torch.Tensor:
    """Full [B, H, T, d] bf16 tensor, built slice by slice (CPU).  `threads`
    > 1 fills slices concurrently (same values: every slice has its own
    generator)."""
    if out is None:
        out = torch.empty(w.B, w.H, w.T, w.d, dtype=torch.bfloat16)
    jobs = [(b, h) for b in range(w.B) for h in range(w.H)]

    def fill(bh):
        b, h = bh
        out[b, h].copy_(make_slice(w, seed, tensor, b, h))

    if threads and threads > 1 and len(jobs) > 1:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(fill, jobs))
    else:
        for bh in jobs:
            fill(bh)
    return out


def make_pattern(w: Workload, seed: int = 0) -> Tuple[torch.Tensor, torch.Tensor]:
    """a, r as [H, T] fp32; NaN rows for ordinary heads."""
    a = torch.full((w.H, w.T), float("nan"), dtype=torch.float32)
    r = torch.full((w.H, w.T), float("nan"), dtype=torch.float32)
    k = torch.arange(w.T, dtype=torch.float32)
    for h in replaced_heads(w, seed):
        ah = torch.randn(w.T, generator=_gen(seed, "alpha", 0, h)) * 0.5
        ah[0] += 4.0
        rh = -0.05 * k + torch.randn(w.T, generator=_gen(seed, "rho", 0, h)) * 0.3
        rh[0] += 2.0
        a[h] = ah
        r[h] = rh
    return a, r


def make_inputs(w: Workload, seed: int = 0, tensors: Iterable[str] = ("q", "k", "v", "do"),
                pin: bool = False, threads: int = 0) -> Dict[str, torch.Tensor]:
    """All inputs of one workload as CPU tensors (optionally pinned)."""
    out: Dict[str, torch.Tensor] = {}
    for t in tensors:
        if t == "do" and not w.backward:
            continue
        buf = torch.empty(w.B, w.H, w.T, w.d, dtype=torch.bfloat16, pin_memory=pin)
        out[t] = make_tensor(w, seed, t, out=buf, threads=threads)
    out["alpha"], out["rho"] = make_pattern(w, seed)
    out["mask"] = replaced_mask(w, seed)
    return out


def flops(w: Workload, backward: Optional[bool] = None, strict: bool = False) -> Dict[str, float]:
    """Algorithmic flop counts, causal T^2/2 convention.

    Ordinary head: forward 2*d*T^2 (QK^T and PV), backward 5*d*T^2 (five
    T x T x d contractions counting the recompute of QK^T; `strict` counts
    the method's own four, 4*d*T^2, without the recompute).  Replaced head:
    forward d*T^2 (PV only), backward d*T^2 (P^T dO only).
    """
    if backward is None:
        backward = w.backward
    n_r = len(replaced_heads(w))
    n_o = w.H - n_r
    unit = float(w.d) * w.T * w.T * w.B
    fwd = unit * (2 * n_o + 1 * n_r)
    bwd = unit * ((4 if strict else 5) * n_o + 1 * n_r) if backward else 0.0
    return {"fwd": fwd, "bwd": bwd, "total": fwd + bwd}
