"""The five workload shapes, as seeded problem lists.

A *problem* is one Hessian and every row that shares it: the q/k/v/o/gate/up
projections of a decoder layer all read the layer input, so their rows form
one stack on one H; down_proj reads SiLU(gate)·up and has its own H.  Layers
are independent (every layer input is drawn from the seeded generator).

Shapes follow the pages' three models ("Warum Geometrie Gewichte nicht
komprimiert", Teil 1 and Table 4) plus a square stress layer.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

from .synth import (cone_activations, gaussian_weights, seed_for,
                    student_t_activations, swiglu_input)

# tensor ids inside one layer's seed block
_TID = {"x": 0, "q": 1, "k": 2, "v": 3, "o": 4, "gate": 5, "up": 6, "down": 7}


@dataclass
class Problem:
    name: str
    X: torch.Tensor            # T × n bf16: the activations the Hessian reads
    W: torch.Tensor            # m × n, bf16 (or float32 for the single layer)
    bits: int = 4
    group: int = 128
    block: int = 128
    damp: float = 0.01
    order: str = "natural"
    parts: tuple = field(default_factory=tuple)   # ((name, rows), ...)

    @property
    def m(self) -> int:
        return int(self.W.shape[0])

    @property
    def n(self) -> int:
        return int(self.W.shape[1])

    @property
    def T(self) -> int:
        return int(self.X.shape[0])

    @property
    def params(self) -> int:
        return self.m * self.n


def _decoder(hidden, kv, inter, layers, T, bits):
    return {"kind": "decoder", "hidden": hidden, "kv": kv, "inter": inter,
            "layers": layers, "T": T, "bits": bits}


CONFIGS = {
    0: {"kind": "single", "name": "single-576", "m": 576, "n": 576, "T": 2048,
        "bits": (4,), "layers": 1},
    1: dict(_decoder(576, 192, 1536, 1, 2048, (4,)), name="smollm135m-layer"),
    2: dict(_decoder(896, 128, 4864, 24, 2048, (4,)), name="qwen2.5-0.5b-24L"),
    3: dict(_decoder(2048, 256, 5632, 22, 2048, (4, 3)),
            name="tinyllama1.1b-22L"),
    4: {"kind": "stress", "name": "stress-8192", "m": 8192, "n": 8192,
        "T": 16384, "bits": (4,), "layers": 1, "orders": ("act", "reverse")},
}


def config_params(cid: int) -> int:
    """Weights quantized by one pass over the whole config (all layers, once)."""
    c = CONFIGS[cid]
    if c["kind"] in ("single", "stress"):
        return c["m"] * c["n"]
    h, kv, it = c["hidden"], c["kv"], c["inter"]
    per_layer = (2 * h + 2 * kv + 2 * it) * h + h * it
    return per_layer * c["layers"]


def problems_for(cid: int, layer: int = 0, bits: int | None = None,
                 order: str | None = None) -> list[Problem]:
    """Seeded problems of one layer of config ``cid`` (CPU tensors)."""
    c = CONFIGS[cid]
    b = bits if bits is not None else c["bits"][0]
    if c["kind"] == "single":
        X = cone_activations(c["T"], c["n"], seed_for(layer, _TID["x"]))
        W = gaussian_weights(c["m"], c["n"], seed_for(layer, _TID["q"]))
        return [Problem("layer", X.to(torch.bfloat16), W, bits=b,
                        order=order or "natural", parts=(("w", c["m"]),))]
    if c["kind"] == "stress":
        X = student_t_activations(c["T"], c["n"], seed_for(layer, _TID["x"]))
        W = gaussian_weights(c["m"], c["n"], seed_for(layer, _TID["q"]))
        return [Problem("stress", X.to(torch.bfloat16), W.to(torch.bfloat16),
                        bits=b, order=order or c["orders"][0],
                        parts=(("w", c["m"]),))]
    h, kv, it, T = c["hidden"], c["kv"], c["inter"], c["T"]
    X = cone_activations(T, h, seed_for(layer, _TID["x"]))
    rows = {"q": h, "k": kv, "v": kv, "o": h, "gate": it, "up": it}
    Ws = {k: gaussian_weights(r, h, seed_for(layer, _TID[k])).to(torch.bfloat16)
          for k, r in rows.items()}
    Wd = gaussian_weights(h, it, seed_for(layer, _TID["down"])).to(torch.bfloat16)
    Xd = swiglu_input(X, Ws["gate"], Ws["up"])
    stack = torch.cat([Ws[k] for k in rows], dim=0).contiguous()
    o = order or "natural"
    return [
        Problem("attn+mlp_in", X.to(torch.bfloat16), stack, bits=b, order=o,
                parts=tuple(rows.items())),
        Problem("down", Xd, Wd, bits=b, order=o, parts=(("down", h),)),
    ]
