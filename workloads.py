"""Seeded synthetic inputs for banded log-domain Sinkhorn attention.

This module is the only code shared by the CUDA path's tests/benchmark and the
CPU oracle's tests.  It draws random numbers and builds masks; it holds none
of the method's arithmetic.

Recipe (the same for every named workload): one CPU ``torch.Generator`` seeded
with ``seed`` draws, in this order, Q, K, V and dO as ``randn(B,H,L,d)`` in
float32, then casts them with round-to-nearest-even to bfloat16 when the
workload is bf16.  A masked workload then draws its per-sequence valid lengths
``randint(lo, hi+1, (B,))`` from the same generator and masks out the padded
tail.  The dustbin value vectors are zero.

The pages' experiments ran on Pfam protein embeddings; that data is not used.
Synthetic N(0,1) problems of the stated sizes stand in for it, as they do in
the pages' own exactness checks on synthetic masked problems.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    d: int
    W: int
    eps: float
    T: int
    R: int
    dtype: str                   # "f32" or "bf16": storage type of Q, K, V, dO, O and gradients
    valid_len: tuple | None = None   # (lo, hi) uniform valid lengths, tail padded
    dustbin: bool = False
    dustbin_score: float = -2.0

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    # single small problem: L=512, W=64, eps=1, T=15, fp32, no mask
    "small512": Workload("small512", B=1, H=1, L=512, d=64, W=64, eps=1.0, T=15, R=2, dtype="f32"),
    # synthetic masked problems: valid lengths uniform in [1024, 2048], tail padded
    "masked2k": Workload("masked2k", B=4, H=8, L=2048, d=64, W=128, eps=0.5, T=20, R=2,
                         dtype="f32", valid_len=(1024, 2048)),
    # long-context single layer, bf16 storage, fp32 accumulation and duals
    "long32k": Workload("long32k", B=1, H=16, L=32768, d=64, W=256, eps=1.0, T=20, R=2,
                        dtype="bf16"),
    # gap-aware dustbin path, constant dustbin score -2
    "dustbin4k": Workload("dustbin4k", B=8, H=4, L=4096, d=64, W=128, eps=1.0, T=15, R=2,
                          dtype="f32", dustbin=True, dustbin_score=-2.0),
    # per-device context of the pages' VJP timing, bf16
    "vjp262k": Workload("vjp262k", B=1, H=8, L=262144, d=64, W=128, eps=1.0, T=15, R=2,
                        dtype="bf16"),
}


def draw(B, H, L, d, *, dtype="f32", seed=0, valid_len=None, mask_kind=None, dustbin=False):
    """Draw ``q, k, v, dO`` (CPU tensors of the storage dtype), ``mask`` (uint8
    ``[B,L]`` or None) and ``v_dust`` (zeros ``[H,d]`` float32 when ``dustbin``).

    ``valid_len=(lo, hi)``: tail padding with lengths uniform in [lo, hi].
    ``mask_kind="holes"``: additionally drop a random 10 % of the tokens
    (a mask that is not a prefix; exercised by the small parity cases).
    """
    g = torch.Generator().manual_seed(seed)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    q = torch.randn(B, H, L, d, generator=g, dtype=torch.float32).to(td)
    k = torch.randn(B, H, L, d, generator=g, dtype=torch.float32).to(td)
    v = torch.randn(B, H, L, d, generator=g, dtype=torch.float32).to(td)
    dO = torch.randn(B, H, L, d, generator=g, dtype=torch.float32).to(td)
    mask = None
    if valid_len is not None:
        lo, hi = valid_len
        n = torch.randint(lo, hi + 1, (B,), generator=g)
        mask = (torch.arange(L)[None, :] < n[:, None]).to(torch.uint8)
    if mask_kind == "holes":
        keep = (torch.rand(B, L, generator=g) >= 0.1).to(torch.uint8)
        mask = keep if mask is None else (mask & keep)
    v_dust = torch.zeros(H, d, dtype=torch.float32) if dustbin else None
    return dict(q=q, k=k, v=v, dO=dO, mask=mask, v_dust=v_dust)


def make(name_or_workload, seed=0):
    """Inputs of a named workload (see ``WORKLOADS``)."""
    w = WORKLOADS[name_or_workload] if isinstance(name_or_workload, str) else name_or_workload
    x = draw(w.B, w.H, w.L, w.d, dtype=w.dtype, seed=seed, valid_len=w.valid_len,
             dustbin=w.dustbin)
    return w, x
