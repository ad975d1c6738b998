"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and the bench.

This module holds no attention arithmetic: it only draws random tensors in a
fixed order and casts them to the workload's storage type.  Both the CUDA path
and the fp64 oracle consume exactly the tensors produced here (the oracle takes
their exact fp64 upcast), so neither side generates data for the other.

Recipe (all workloads): ``torch.Generator('cpu').manual_seed(seed)``, then
``torch.randn`` in fp32 in the order Q, K, V, dO (K and V with the workload's
key/value head count, which equals the query head count unless the workload
shares key/value heads); Q and K are multiplied by
``qk_mult`` in fp32 (the single-query workload uses 40 so that logits reach
the +-1e3 range that a max-free exponential cannot represent); finally the
tensors are cast (round-to-nearest-even) to the workload dtype.  Layout is
``[B, H, N, D]`` contiguous, as in the query-chunking example of "Fast and
memory-efficient exact attention" (the ``batch, heads, seq_len, d_k`` unpacking).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    D: int
    dtype: str  # "f32" or "bf16"
    backward: bool
    qk_mult: float = 1.0
    note: str = ""
    Hkv: int | None = None  # key/value heads (None: one per query head)

    @property
    def H_kv(self) -> int:
        return self.H if self.Hkv is None else self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def fwd_flops(self) -> float:
        # shared key/value heads change the bytes read, not the flops
        # 4 * B * H * Nq * Nk * D: two GEMMs of 2*Nq*Nk*D each per head.
        return 4.0 * self.B * self.H * self.Nq * self.Nk * self.D

    def bwd_flops(self) -> float:
        return 2.5 * self.fwd_flops()


# The five workloads of the method's evaluation, named by what they are.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 1, 256, 256, 64, "f32", False,
                         note="tiny self-attention, fp32 forward"),
    "single_query_f32": Workload("single_query_f32", 1, 8, 1, 16384, 64, "f32", False, qk_mult=40.0,
                                 note="single-query attention over 16384 keys, fp32 forward, logits ~1e3"),
    "mha_4k_bf16": Workload("mha_4k_bf16", 4, 8, 4096, 4096, 64, "bf16", True,
                            note="multi-head self-attention B4 H8 N4096 D64"),
    "encoder_512_bf16": Workload("encoder_512_bf16", 32, 8, 512, 512, 64, "bf16", True,
                                 note="encoder-shaped batch B32 H8 N512 D64"),
}
WORKLOADS["decode_16384_bf16"] = Workload("decode_16384_bf16", 1, 8, 1, 16384, 128, "bf16", False,
                                          note="decode-shaped bf16 forward: one query row over 16384 keys, 8 heads")
# Shared key/value heads, with the grouping that "当注意力成为瓶颈" (section 推理优化：减少KV Cache)
# gives as its example
# (32 query heads in 8 groups of 4).
WORKLOADS["gqa_32x8_4096_bf16"] = Workload("gqa_32x8_4096_bf16", 1, 32, 4096, 4096, 128, "bf16", True, Hkv=8,
                                           note="grouped-query attention: 32 query heads, 8 key/value heads")
WORKLOADS["decode_gqa_32x8_16384_bf16"] = Workload(
    "decode_gqa_32x8_16384_bf16", 1, 32, 1, 16384, 128, "bf16", False, Hkv=8,
    note="decode-shaped grouped-query forward: one query row per head, 32 query heads over 8 key/value heads")
for _n in (256, 1024, 4096, 16384):
    WORKLOADS[f"long_{_n}_bf16"] = Workload(f"long_{_n}_bf16", 1, 16, _n, _n, 128, "bf16", True,
                                             note=f"long-sequence sweep B1 H16 N{_n} D128")


def make_workload(name: str) -> Workload:
    return WORKLOADS[name]


def custom(B: int, H: int, Nq: int, Nk: int, D: int, dtype: str, backward: bool = True,
           qk_mult: float = 1.0, name: str = "custom", Hkv: int | None = None) -> Workload:
    return Workload(name, B, H, Nq, Nk, D, dtype, backward, qk_mult, Hkv=Hkv)


def make_inputs(w: Workload, seed: int, with_grad_output: bool | None = None):
    """Return (q, k, v, do) CPU tensors in the workload's storage dtype.

    ``do`` is None when the workload is forward-only and ``with_grad_output``
    is not forced.  Draw order is always Q, K, V, dO so a forward-only draw
    yields the same Q, K, V as a forward+backward draw.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn((w.B, w.H, w.Nq, w.D), generator=g, dtype=torch.float32)
    k = torch.randn((w.B, w.H_kv, w.Nk, w.D), generator=g, dtype=torch.float32)
    v = torch.randn((w.B, w.H_kv, w.Nk, w.D), generator=g, dtype=torch.float32)
    want_do = w.backward if with_grad_output is None else with_grad_output
    do = torch.randn((w.B, w.H, w.Nq, w.D), generator=g, dtype=torch.float32) if want_do else None
    if w.qk_mult != 1.0:
        q = q * w.qk_mult
        k = k * w.qk_mult
    dt = w.torch_dtype
    q, k, v = q.to(dt).contiguous(), k.to(dt).contiguous(), v.to(dt).contiguous()
    if do is not None:
        do = do.to(dt).contiguous()
    return q, k, v, do


E4M3_MAX = 448.0  # largest finite value of float8 e4m3 (the "fn" variant without infinities)


def make_inputs_fp8(w: Workload, seed: int):
    """Inputs for the FP8 forward: (q8, k8, v, q_descale, k_descale).

    Same draws as ``make_inputs`` (Q, K, V in fp32 from the same generator
    order, scaled by ``qk_mult``); Q and K are then quantised per tensor to
    e4m3: descale = max|x| / 448, x8 = e4m3(x / descale) with round to nearest
    even (clamped to +-448 first).  V is cast to bf16.  The dequantised values
    descale * x8 are what the method computes on; the oracle takes their exact
    fp64 upcast.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn((w.B, w.H, w.Nq, w.D), generator=g, dtype=torch.float32)
    k = torch.randn((w.B, w.H_kv, w.Nk, w.D), generator=g, dtype=torch.float32)
    v = torch.randn((w.B, w.H_kv, w.Nk, w.D), generator=g, dtype=torch.float32)
    if w.qk_mult != 1.0:
        q = q * w.qk_mult
        k = k * w.qk_mult

    def quant(x):
        amax = float(x.abs().max()) if x.numel() else 0.0
        # an fp32 number, as the library takes it
        descale = float(torch.tensor(amax / E4M3_MAX if amax > 0 else 1.0, dtype=torch.float32))
        x8 = (x / descale).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn).contiguous()
        return x8, descale

    q8, qd = quant(q)
    k8, kd = quant(k)
    return q8, k8, v.to(torch.bfloat16).contiguous(), qd, kd


def dequant_f64(x8: torch.Tensor, descale: float):
    """Exact fp64 value of descale * x8 (both factors are exactly representable)."""
    return x8.to(torch.float64).numpy() * float(descale)


def to_f64(t: torch.Tensor):
    """Exact fp64 upcast as a numpy array (bf16 and fp32 values are exactly representable)."""
    return t.detach().to(torch.float64).cpu().numpy()
