"""FP8 forward (e4m3 Q and K, bf16 V and O) against the fp64 oracle, through the C ABI (GPU).

The oracle computes exact attention on the dequantised inputs descale * x8
(exact in fp64).  Each product of two e4m3 values is exact in the fp32
accumulator, so the kernel's error budget is that of the bf16 path (P rounded
to bf16, O rounded to bf16) and the same tolerances apply: O max-abs 2e-2 and
relative Frobenius 5e-3, lse within the bound derived from the arithmetic.
"""

import numpy as np
import pytest
import torch

import oracle
from synthetic_inputs import custom, dequant_f64, make_inputs_fp8, make_workload, to_f64
from tests._parity import BF16_O, assert_close, assert_lse_close, to_np

pytestmark = pytest.mark.gpu


def run_fp8(w, seed):
    import exact_memory_efficient_b200 as m
    q8, k8, v, qd, kd = make_inputs_fp8(w, seed)
    o = torch.empty((w.B, w.H, w.Nq, w.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device="cuda")
    m.mea_attn_fwd_fp8(q8.cuda(), k8.cuda(), v.cuda(), o, lse, w.scale, qd, kd)
    assert m.mea_last_device_error() == m.MEA_OK
    return o, lse, dequant_f64(q8, qd), dequant_f64(k8, kd), to_f64(v)


@pytest.mark.parametrize("B,H,Hkv,Nq,Nk", [
    (1, 1, 1, 128, 128),
    (1, 2, 2, 300, 400),      # ragged tails
    (2, 3, 3, 257, 513),
    (1, 8, 2, 200, 333),      # grouped-query heads
    (1, 4, 4, 1, 3000),       # one query row: single-tile CTAs, keys split over a cluster
])
def test_fp8_full(B, H, Hkv, Nq, Nk):
    w = custom(B, H, Nq, Nk, 128, "bf16", backward=False, Hkv=Hkv)
    o, lse, q, k, v = run_fp8(w, 13)
    ro, rl = oracle.attention_forward_gqa(q, k, v, w.scale)
    assert_close(to_np(o), ro, *BF16_O, what=f"fp8 O {(B, H, Hkv, Nq, Nk)}")
    assert_lse_close(to_np(lse), rl, q, np.repeat(k, H // Hkv, axis=1), w.scale, what="fp8 lse")


def test_fp8_decode_full():
    """Decode shape (8 heads, one row, 16384 keys) with e4m3 Q and K."""
    w = make_workload("decode_16384_bf16")
    o, lse, q, k, v = run_fp8(w, 1)
    ro, rl = oracle.attention_forward(q, k, v, w.scale)
    assert_close(to_np(o), ro, *BF16_O, what="fp8 decode O")
    assert_lse_close(to_np(lse), rl, q, k, w.scale, what="fp8 decode lse")


@pytest.mark.parametrize("seed", [0, 1])
def test_fp8_long_sampled(seed):
    """Full-size launch (B1 H16 N16384 D128); the oracle checks sampled rows of three heads."""
    w = make_workload("long_16384_bf16")
    o, lse, q, k, v = run_fp8(w, seed)
    o, lse = to_np(o), to_np(lse)
    rng = np.random.default_rng(300 + seed)
    for h in sorted({0, w.H - 1, int(rng.integers(w.H))}):
        rows = np.unique(np.concatenate([[0, w.Nq - 1], rng.choice(w.Nq, 32, replace=False)]))
        ro, rl = oracle.attention_forward_rows(q[0, h], k[0, h], v[0, h], w.scale, rows)
        assert_close(o[0, h][rows], ro, *BF16_O, what=f"fp8 O head {h}")
        assert_lse_close(lse[0, h][rows], rl, q[0, h][rows], k[0, h], w.scale, what=f"fp8 lse head {h}")


def test_fp8_descale_folds_into_scale():
    """Doubling q_descale while halving scale leaves the result bit-identical (the kernel
    multiplies the three factors once on the host)."""
    import exact_memory_efficient_b200 as m
    w = custom(1, 2, 200, 300, 128, "bf16", backward=False)
    q8, k8, v, qd, kd = make_inputs_fp8(w, 4)
    q8, k8, v = q8.cuda(), k8.cuda(), v.cuda()
    outs = []
    for sc, a in ((w.scale, qd), (w.scale / 2, 2 * qd)):
        o = torch.empty((1, 2, 200, 128), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((1, 2, 200), dtype=torch.float32, device="cuda")
        m.mea_attn_fwd_fp8(q8, k8, v, o, lse, sc, a, kd)
        outs.append((o, lse))
    torch.cuda.synchronize()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_fp8_negative_scale():
    """scale < 0: the largest scaled score of a block comes from the smallest raw score."""
    import exact_memory_efficient_b200 as m
    w = custom(1, 2, 300, 700, 128, "bf16", backward=False)
    q8, k8, v, qd, kd = make_inputs_fp8(w, 14)
    o = torch.empty((1, 2, 300, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 2, 300), dtype=torch.float32, device="cuda")
    m.mea_attn_fwd_fp8(q8.cuda(), k8.cuda(), v.cuda(), o, lse, -w.scale, qd, kd)
    assert m.mea_last_device_error() == m.MEA_OK
    q, k = dequant_f64(q8, qd), dequant_f64(k8, kd)
    ro, rl = oracle.attention_forward(q, k, to_f64(v), -w.scale)
    assert_close(to_np(o), ro, *BF16_O, what="fp8 negative scale O")
    assert_lse_close(to_np(lse), rl, q, k, -w.scale, what="fp8 negative scale lse")
