"""fp32 SIMT forward against the fp64 oracle, through the C ABI (GPU)."""

import math

import numpy as np
import pytest
import torch

import oracle
from synthetic_inputs import custom, make_inputs, make_workload, to_f64
from tests._parity import F32_O_MAX_ABS, assert_close, assert_lse_close, to_np

pytestmark = pytest.mark.gpu


def run_fwd(q, k, v, scale):
    import exact_memory_efficient_b200 as m
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    o, lse = m.attention_forward(qd, kd, vd, scale)
    assert m.mea_last_device_error() == m.MEA_OK
    return to_np(o), to_np(lse)


def check(w_or_tensors, scale, seed_note=""):
    q, k, v = w_or_tensors
    o, lse = run_fwd(q, k, v, scale)
    q64, k64, v64 = to_f64(q), to_f64(k), to_f64(v)
    o_ref, lse_ref = oracle.attention_forward(q64, k64, v64, scale)
    assert_close(o, o_ref, F32_O_MAX_ABS, what=f"O {seed_note}")
    assert_lse_close(lse, lse_ref, q64, k64, scale, what=f"lse {seed_note}")


@pytest.mark.parametrize("name", ["tiny_f32", "single_query_f32"])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_workloads(name, seed):
    w = make_workload(name)
    q, k, v, _ = make_inputs(w, seed)
    check((q, k, v), w.scale, f"{name} seed {seed}")


@pytest.mark.parametrize("B,H,Nq,Nk,D", [
    (1, 1, 1, 1, 64),        # single key
    (1, 2, 3, 33, 32),       # ragged keys, tiny
    (2, 3, 17, 1000, 96),    # D = 96, ragged
    (1, 4, 5, 4097, 128),    # long ragged key range, split over a cluster
    (1, 1, 300, 77, 64),     # many rows, few keys
    (3, 1, 2, 16384, 64),    # 2-row CTAs with 16-way key split
])
def test_shapes(B, H, Nq, Nk, D):
    w = custom(B, H, Nq, Nk, D, "f32", backward=False)
    q, k, v, _ = make_inputs(w, 5)
    check((q, k, v), w.scale, f"{(B, H, Nq, Nk, D)}")


def test_large_logits_dominant_key():
    """Logits ~1e3: max tracking must hold; the dominant key's value row is returned."""
    Nk, D = 4096, 64
    g = torch.Generator().manual_seed(3)
    k = torch.randn(1, 1, Nk, D, generator=g) * 40
    q = k[:, :, 1234:1235, :].clone() * 1.0  # q = k_1234: its score |k|^2/8 ~ 1.3e4 dominates
    v = torch.randn(1, 1, Nk, D, generator=g)
    o, lse = run_fwd(q, k, v, 1.0 / 8)
    s = (to_f64(q)[0, 0] @ to_f64(k)[0, 0].T)[0] / 8
    srt = np.sort(s)
    assert srt[-1] - srt[-2] > 50
    np.testing.assert_allclose(o[0, 0, 0], to_f64(v)[0, 0, 1234], atol=F32_O_MAX_ABS)
    assert np.isfinite(lse).all()


def test_all_keys_equal_gives_mean_value():
    Nq, Nk, D = 7, 3000, 64
    g = torch.Generator().manual_seed(4)
    q = torch.randn(1, 1, Nq, D, generator=g)
    k = torch.randn(1, 1, 1, D, generator=g).expand(1, 1, Nk, D).contiguous()
    v = torch.randn(1, 1, Nk, D, generator=g)
    o, lse = run_fwd(q, k, v, 0.125)
    np.testing.assert_allclose(o[0, 0], np.tile(to_f64(v)[0, 0].mean(axis=0), (Nq, 1)), atol=F32_O_MAX_ABS)
    expect = 0.125 * (to_f64(q)[0, 0] @ to_f64(k)[0, 0, 0]) + math.log(Nk)
    np.testing.assert_allclose(lse[0, 0], expect, atol=1e-4)


def test_deterministic():
    w = make_workload("single_query_f32")
    q, k, v, _ = make_inputs(w, 0)
    a = run_fwd(q, k, v, w.scale)
    b = run_fwd(q, k, v, w.scale)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("B,H,Nq,Nk,D", [(1, 2, 40, 300, 64), (1, 3, 1, 2000, 128)])
def test_negative_scale(B, H, Nq, Nk, D):
    """scale < 0, forward and backward: the SIMT paths scale each score before the running maximum."""
    import exact_memory_efficient_b200 as m
    w = custom(B, H, Nq, Nk, D, "f32")
    q, k, v, do = make_inputs(w, 15)
    check((q, k, v), -w.scale, "negative scale")
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = m.attention_forward(qd, kd, vd, -w.scale)
    dq, dk, dv = m.attention_backward(qd, kd, vd, o, lse, dod, -w.scale)
    assert m.mea_last_device_error() == m.MEA_OK
    rq, rk, rv, _, _ = oracle.attention_backward(to_f64(q), to_f64(k), to_f64(v), to_f64(do), -w.scale)
    for name, g_, r_ in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
        assert_close(to_np(g_), r_, F32_O_MAX_ABS, what=f"negative scale fp32 {name}")
