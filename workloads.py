"""Seeded synthetic inputs for the routed MoE FFN.

This module is the one place both the CUDA path's tests/bench and the oracle
take their inputs from.  It holds none of the method's arithmetic: it only
draws seeded random tensors in the shapes, value distributions and router
biases of the five synthetic workloads, and converts bf16 tensors to the bit
patterns the oracle reads.

Recipe (every workload): values are drawn in fp32 from torch's seeded normal
generator (one generator per tensor, seed = base + tensor index) and rounded
to bf16 with round-to-nearest-even.  x ~ N(0, 1); every weight ~ N(0, 0.02).
Router bias: none, "+8 on experts 0..15" (load-imbalanced), or the Zipf(1.1)
skew b_e = -1.1 * ln(e + 1) so that softmax(b) is proportional to
(e + 1)^-1.1 (large).
"""
import math
from dataclasses import dataclass, field
from typing import Optional, Tuple

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: Tuple[int, ...]          # token counts the workload is run at
    H: int
    E: int
    top_k: int
    I: int
    I_s: int                    # 0 = no shared expert
    x_dtype: str                # "bf16" or "f32"
    bias: str                   # "none", "plus8_first16", "zipf1.1"
    bands: Tuple[int, ...]
    description: str = field(default="", compare=False)


WORKLOADS = {
    "tiny": Workload("tiny", (4,), 256, 16, 4, 128, 128, "f32", "none", (1, 2, 4),
                     "T=4, H=256, E=16, top_k=4, I=128, shared I=128, fp32 x"),
    "decode": Workload("decode", (1, 4, 8), 4096, 128, 8, 1536, 1536, "bf16", "none", (8,),
                       "T in {1,4,8}, H=4096, E=128, top_k=8, I=1536, shared I=1536"),
    "prefill": Workload("prefill", (512,), 4096, 128, 8, 2048, 2048, "bf16", "none", (4,),
                        "T=512, H=4096, E=128, top_k=8, I=2048, shared I=2048"),
    "imbalanced": Workload("imbalanced", (2048,), 4096, 64, 4, 2048, 0, "bf16", "plus8_first16",
                           (4, 1), "T=2048, H=4096, E=64, top_k=4, I=2048, no shared expert, "
                           "bias +8 on experts 0..15"),
    "large": Workload("large", (4096,), 6144, 256, 8, 2048, 2048, "bf16", "zipf1.1", (8,),
                      "T=4096, H=6144, E=256, top_k=8, I=2048, shared I=2048, Zipf(1.1) bias"),
}

WEIGHT_STD = 0.02
SEED_BASE = 1000


def _normal(shape, seed, device, std=1.0):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        out.mul_(std)
    return out


def _bf16_normal(shape, seed, device, std):
    return _normal(shape, seed, device, std).to(torch.bfloat16)


def _expert_seed(seed, e):
    return seed * 1_000_003 + e


def _expert_stack(E, rows, cols, seed, device):
    """[E, rows, cols] bf16, one seeded draw per expert (bounded temporaries)."""
    out = torch.empty((E, rows, cols), dtype=torch.bfloat16, device=device)
    for e in range(E):
        out[e].copy_(_bf16_normal((rows, cols), _expert_seed(seed, e), device, WEIGHT_STD))
    return out


# tensor index of each expert projection in make_weights' seed sequence
_EXPERT_TENSORS = {"w_gate": 2, "w_up": 3, "w_down": 4}


def make_expert(w: Workload, which: str, e: int, device="cpu", seed=SEED_BASE):
    """One expert's matrix of make_weights (which = "w_gate", "w_up" or
    "w_down"), drawn alone: the same values as make_weights(...)[which][e]
    on the same device type."""
    rows, cols = (w.I, w.H) if which in ("w_gate", "w_up") else (w.H, w.I)
    return _bf16_normal((rows, cols), _expert_seed(seed + _EXPERT_TENSORS[which], e), device,
                        WEIGHT_STD)


def make_router(w: Workload, device="cpu", seed=SEED_BASE):
    """(w_router, bias) of make_weights, without the experts."""
    b = router_bias(w.bias, w.E)
    return (_bf16_normal((w.E, w.H), seed + 1, device, WEIGHT_STD),
            None if b is None else b.to(device))


def make_shared(w: Workload, device="cpu", seed=SEED_BASE):
    """(ws_gate, ws_up, ws_down) of make_weights, or None without a shared expert."""
    if w.I_s == 0:
        return None
    return (_bf16_normal((w.I_s, w.H), seed + 5, device, WEIGHT_STD),
            _bf16_normal((w.I_s, w.H), seed + 6, device, WEIGHT_STD),
            _bf16_normal((w.H, w.I_s), seed + 7, device, WEIGHT_STD))


def router_bias(kind: str, E: int) -> Optional[torch.Tensor]:
    if kind == "none":
        return None
    if kind == "plus8_first16":
        b = torch.zeros(E, dtype=torch.float32)
        b[: min(16, E)] = 8.0
        return b
    if kind == "zipf1.1":
        return torch.tensor([-1.1 * math.log(e + 1.0) for e in range(E)], dtype=torch.float32)
    raise ValueError(kind)


def make_weights(w: Workload, device="cpu", seed=SEED_BASE, H=None, E=None, I=None, I_s=None,
                 bias=None):
    """All weights of one MoE layer.  Sizes may be overridden for small cases."""
    H = H or w.H
    E = E or w.E
    I = I or w.I
    I_s = w.I_s if I_s is None else I_s
    out = {
        "w_router": _bf16_normal((E, H), seed + 1, device, WEIGHT_STD),
        "w_gate": _expert_stack(E, I, H, seed + 2, device),
        "w_up": _expert_stack(E, I, H, seed + 3, device),
        "w_down": _expert_stack(E, H, I, seed + 4, device),
    }
    b = router_bias(bias or w.bias, E)
    out["bias"] = None if b is None else b.to(device)
    if I_s > 0:
        out["ws_gate"] = _bf16_normal((I_s, H), seed + 5, device, WEIGHT_STD)
        out["ws_up"] = _bf16_normal((I_s, H), seed + 6, device, WEIGHT_STD)
        out["ws_down"] = _bf16_normal((H, I_s), seed + 7, device, WEIGHT_STD)
    else:
        out["ws_gate"] = out["ws_up"] = out["ws_down"] = None
    return out


# NVFP4 expert weights are drawn directly as stored bytes: element codes
# uniform over all 16 FP4 codes (two per byte), block-scale bytes uniform over
# the E4M3 codes of 0.5 .. 3.75 (0x30 .. 0x47), and a tensor scale of 2^-7, so
# the weights lie within +-0.18.  Nothing is quantised here.
NVFP4_SCALE_CODES = (0x30, 0x48)
NVFP4_TENSOR_SCALE = 2.0 ** -7


def make_nvfp4_experts(E: int, rows: int, cols: int, seed: int, device="cpu"):
    """{"packed": [E, rows, cols / 2] uint8, "scales": [E, rows, cols / 16]
    uint8, "tensor_scale": float} for one projection of E experts."""
    if cols % 16:
        raise ValueError("NVFP4 rows are whole blocks of 16")
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    packed = torch.randint(0, 256, (E, rows, cols // 2), generator=g, device=device,
                           dtype=torch.int32).to(torch.uint8)
    lo, hi = NVFP4_SCALE_CODES
    scales = torch.randint(lo, hi, (E, rows, cols // 16), generator=g, device=device,
                           dtype=torch.int32).to(torch.uint8)
    return {"packed": packed, "scales": scales, "tensor_scale": NVFP4_TENSOR_SCALE}


def make_x(w: Workload, T: int, device="cpu", seed=SEED_BASE, batch=0, H=None, x_dtype=None):
    """Activations for one batch; `batch` selects one of several distinct draws."""
    H = H or w.H
    x = _normal((T, H), seed + 100 + batch, device)
    return x if (x_dtype or w.x_dtype) == "f32" else x.to(torch.bfloat16)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy); fp32 -> float32."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)


def from_bits(a: np.ndarray) -> torch.Tensor:
    """numpy uint16 bf16 bit patterns -> bf16 tensor (host)."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
