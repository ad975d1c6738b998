"""Seeded random shapes through every entry point, against the fp64 oracle (GPU).

Sixty cases drawn from a fixed seed: B in 1..2, H_kv in 1..3 key/value heads
shared by 1, 2 or 4 query heads, Nq in {1, small, large}, Nk in {1, small,
large}, D in {64, 128}.  Each runs the bf16 forward and backward; every third
D = 128 case also runs the FP8 forward and every fourth D = 64 case the fp32
forward and backward.  Every output is held to the max-abs and relative
Frobenius pair of the dedicated tests; the lse to its derived bound.  A
gradient whose reference exceeds order one (few keys shared by many query
rows, so that dV and dK sum many rows) scales its absolute bound
by max|ref| / 4 (the rounding errors of such sums grow with their terms).
"""

import numpy as np
import pytest
import torch

import oracle
from synthetic_inputs import custom, dequant_f64, make_inputs, make_inputs_fp8, to_f64
from tests._parity import BF16_GRAD, BF16_O, F32_O_MAX_ABS, ORDER_ONE, assert_close, assert_lse_close, to_np

pytestmark = pytest.mark.gpu

F32_GRAD = (F32_O_MAX_ABS, 1e-5)


def cases(n=60, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        D = int(rng.choice([64, 128]))
        B = int(rng.integers(1, 3))
        Hkv = int(rng.integers(1, 4))
        G = int(rng.choice([1, 1, 2, 4]))
        Nq = int(rng.choice([1, int(rng.integers(1, 40)), int(rng.integers(100, 1200))]))
        Nk = int(rng.choice([1, int(rng.integers(2, 300)), int(rng.integers(300, 2500))]))
        out.append((i, B, Hkv * G, Hkv, Nq, Nk, D))
    return out


def _large(r):
    return bool(np.abs(r).max() > ORDER_ONE)


def _grad_check(g, r, tols, what):
    # relative Frobenius is undefined for a gradient that is exactly zero (one key: dQ = dK = 0)
    rel = tols[1] if np.linalg.norm(r) > tols[0] else None
    assert_close(to_np(g), r, tols[0], rel, what=what, large_outputs=_large(r))


@pytest.mark.parametrize("case", cases(), ids=lambda c: "-".join(map(str, c)))
def test_random_shape(case):
    import exact_memory_efficient_b200 as m
    i, B, H, Hkv, Nq, Nk, D = case
    G = H // Hkv
    w = custom(B, H, Nq, Nk, D, "bf16", Hkv=Hkv)
    q, k, v, do = make_inputs(w, 1000 + i)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = m.attention_forward(qd, kd, vd, w.scale)
    dq, dk, dv = m.attention_backward(qd, kd, vd, o, lse, dod, w.scale)
    assert m.mea_last_device_error() == m.MEA_OK
    rq, rk, rv, ro, rl = oracle.attention_backward_gqa(to_f64(q), to_f64(k), to_f64(v), to_f64(do), w.scale)
    assert_close(to_np(o), ro, *BF16_O, what="O")
    assert_lse_close(to_np(lse), rl, to_f64(q), np.repeat(to_f64(k), G, axis=1), w.scale)
    for name, g_, r_ in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
        _grad_check(g_, r_, BF16_GRAD, name)
    if D == 128 and i % 3 == 0:
        q8, k8, v8, qs, ks = make_inputs_fp8(w, 1000 + i)
        o8 = torch.empty((B, H, Nq, D), dtype=torch.bfloat16, device="cuda")
        l8 = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
        m.mea_attn_fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), o8, l8, w.scale, qs, ks)
        assert m.mea_last_device_error() == m.MEA_OK
        q8d, k8d = dequant_f64(q8, qs), dequant_f64(k8, ks)
        r8, rl8 = oracle.attention_forward_gqa(q8d, k8d, to_f64(v8), w.scale)
        assert_close(to_np(o8), r8, *BF16_O, what="FP8 O")
        assert_lse_close(to_np(l8), rl8, q8d, np.repeat(k8d, G, axis=1), w.scale, what="FP8 lse")
    if D == 64 and i % 4 == 0:
        w32 = custom(B, H, Nq, Nk, D, "f32", Hkv=Hkv)
        q3, k3, v3, do3 = make_inputs(w32, 1000 + i)
        qd3, kd3, vd3, dod3 = (x.cuda() for x in (q3, k3, v3, do3))
        o3, l3 = m.attention_forward(qd3, kd3, vd3, w32.scale)
        dq3, dk3, dv3 = m.attention_backward(qd3, kd3, vd3, o3, l3, dod3, w32.scale)
        assert m.mea_last_device_error() == m.MEA_OK
        r3 = oracle.attention_backward_gqa(to_f64(q3), to_f64(k3), to_f64(v3), to_f64(do3), w32.scale)
        assert_close(to_np(o3), r3[3], F32_O_MAX_ABS, what="fp32 O")
        assert_lse_close(to_np(l3), r3[4], to_f64(q3), np.repeat(to_f64(k3), G, axis=1), w32.scale,
                         what="fp32 lse")
        for name, g_, r_ in (("dQ", dq3, r3[0]), ("dK", dk3, r3[1]), ("dV", dv3, r3[2])):
            _grad_check(g_, r_, F32_GRAD, f"fp32 {name}")
