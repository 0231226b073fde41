"""Seeded synthetic inputs for the Mixtral sparse-MoE layer.

This is the one module that both the CUDA path's tests/bench and the CPU oracle
consume.  It holds none of the layer's arithmetic: only random draws, scaling by
the stated standard deviations, the structural tweaks of the skewed and
long-context workloads, and rounding to the storage dtype.

Shapes follow the Mixtral-8x7B layer: d = 32 heads x 128 = 4096, h = 14336, E = 8,
k = 2 (atlas "Mixtral", "Design overview"; notion notes "Mixtral of Experts",
"Implementation").  Recipe (the pages fix no data; these are synthetic):

* draws are float32 normals from one ``torch.Generator`` seeded with the
  workload's seed, in the order x, W_g, W1, W3, W2, then scaled and rounded
  (round-to-nearest-even) to the dtype;
* x ~ N(0, 1); W_g, W1, W3 ~ N(0, 1/d); W2 ~ N(0, 1/h);
* ``skew``: a constant input channel carries a per-expert logit offset:
  ``x[:, d-1] = 1`` and ``W_g[d-1, :] = (+2, +1, 0, 0, 0, 0, -4, -4)``, so the
  logits are ``x[:, :d-1] W_g[:d-1] + offset`` while the layer still computes
  exactly ``x . W_g`` (about 60% of first choices land on expert 0 and experts 6
  and 7 get few or no rows);
* ``long``: x = s_t z_t with z ~ N(0, 1) and a per-token scale
  s_t = exp(U[ln 0.5, ln 2]) drawn right after z.

Values are generated on the requested device; the CPU and CUDA generators give
different (but each deterministic) streams, so a test always hands the very same
tensors to both sides.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

MIXTRAL_D = 32 * 128
MIXTRAL_H = 14336


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    h: int
    E: int = 8
    k: int = 2
    dtype: str = "bf16"  # "bf16" or "f32"
    seed: int = 0
    kind: str = "plain"  # "plain", "skew" or "long"
    note: str = ""

    @property
    def P(self) -> int:
        return self.T * self.k

    def with_tokens(self, T: int) -> "Workload":
        return replace(self, T=T)

    def active_flops(self) -> int:
        """Algorithmic flops of the expert FFNs: 2 * k * 3 * d * h per token."""
        return 2 * self.k * 3 * self.d * self.h * self.T


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", T=64, d=128, h=256, dtype="f32", seed=0,
                         note="tiny fp32 layer, T=64 d=128 h=256"),
    "decode": Workload("decode", T=16, d=MIXTRAL_D, h=MIXTRAL_H, seed=1,
                       note="Mixtral-8x7B layer, decode batch T=16, bf16"),
    "prefill": Workload("prefill", T=4096, d=MIXTRAL_D, h=MIXTRAL_H, seed=2,
                        note="Mixtral-8x7B layer, prefill T=4096, bf16"),
    "skew": Workload("skew", T=4096, d=MIXTRAL_D, h=MIXTRAL_H, seed=3, kind="skew",
                     note="Mixtral-8x7B layer, T=4096, skewed routing, bf16"),
    "long": Workload("long", T=32768, d=MIXTRAL_D, h=MIXTRAL_H, seed=4, kind="long",
                     note="Mixtral-8x7B layer, T=32768 (32K context), bf16"),
    # Half-width layer with the prefill's rows per expert, for profiler captures that
    # must hold a few GB on the device at most (backward: about 3 GB).
    "prefill_half": Workload("prefill_half", T=4096, d=MIXTRAL_D // 2, h=MIXTRAL_H // 2,
                             seed=5, note="half-width layer (d=2048, h=7168), T=4096, "
                                          "bf16: profiling case"),
}

SKEW_OFFSETS = (2.0, 1.0, 0.0, 0.0, 0.0, 0.0, -4.0, -4.0)


def torch_dtype(dtype: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[dtype]


def _normal(gen, shape, std, device):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def make_inputs(w: Workload, device="cpu", weights: bool = True) -> dict:
    """Draw the workload's tensors on ``device``.

    Returns a dict with ``x [T,d]``, ``Wg [d,E]``, ``W1 [E,h,d]``, ``W3 [E,h,d]`` and
    ``W2 [E,d,h]`` in the workload's dtype, contiguous.  ``weights=False`` skips the
    expert stacks; x and Wg are unchanged by that because they are drawn first.
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)
    dt = torch_dtype(w.dtype)
    x = _normal(gen, (w.T, w.d), 1.0, dev)
    if w.kind == "long":
        u = torch.rand((w.T, 1), generator=gen, device=dev, dtype=torch.float32)
        s = torch.exp(math.log(0.5) + u * (math.log(2.0) - math.log(0.5)))
        x.mul_(s)
    Wg = _normal(gen, (w.d, w.E), 1.0 / math.sqrt(w.d), dev)
    if w.kind == "skew":
        if w.E != len(SKEW_OFFSETS):
            raise ValueError("the skewed workload is defined for E = 8")
        x[:, w.d - 1] = 1.0
        Wg[w.d - 1, :] = torch.tensor(SKEW_OFFSETS, device=dev)
    out = dict(x=x.to(dt).contiguous(), Wg=Wg.to(dt).contiguous())
    if weights:
        for name, shape, std in (("W1", (w.E, w.h, w.d), 1.0 / math.sqrt(w.d)),
                                 ("W3", (w.E, w.h, w.d), 1.0 / math.sqrt(w.d)),
                                 ("W2", (w.E, w.d, w.h), 1.0 / math.sqrt(w.h))):
            t = _normal(gen, shape, std, dev)
            out[name] = t.to(dt).contiguous()
            del t
    return out


def small(name: str, T: int, d: int, h: int, E: int = 8, dtype: str = "bf16",
          seed: int = 0, kind: str = "plain") -> Workload:
    """A small ad-hoc workload with the same draw recipe (for parity at many shapes)."""
    return Workload(name, T=T, d=d, h=h, E=E, dtype=dtype, seed=seed, kind=kind)
