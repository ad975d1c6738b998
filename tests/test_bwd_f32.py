"""fp32 SIMT backward against the fp64 oracle, through the C ABI (GPU).

The GPU backward consumes the GPU forward's own o and lse (as a user would);
the oracle computes everything from the inputs in fp64.  Tolerance: the fp32
output bound (max-abs 1e-4) applied to gradients of order one, plus a relative
Frobenius bound of 1e-5 (fp32 arithmetic, u = 6e-8, with dot products of at
most 128 terms and sums over at most a few thousand rows).
"""

import numpy as np
import pytest
import torch

import oracle
from synthetic_inputs import custom, make_inputs, make_workload, to_f64
from tests._parity import F32_O_MAX_ABS, assert_close, to_np

pytestmark = pytest.mark.gpu

F32_GRAD = (F32_O_MAX_ABS, 1e-5)


def gpu_fwd_bwd(q, k, v, do, scale):
    import exact_memory_efficient_b200 as m
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = m.attention_forward(qd, kd, vd, scale)
    dq, dk, dv = m.attention_backward(qd, kd, vd, o, lse, dod, scale)
    assert m.mea_last_device_error() == m.MEA_OK
    return dq, dk, dv


def check(w, seed, what):
    q, k, v, do = make_inputs(w, seed, with_grad_output=True)
    dq, dk, dv = gpu_fwd_bwd(q, k, v, do, w.scale)
    if w.H_kv == w.H:
        rq, rk, rv, _, _ = oracle.attention_backward(to_f64(q), to_f64(k), to_f64(v), to_f64(do), w.scale)
    else:
        rq, rk, rv, _, _ = oracle.attention_backward_gqa(to_f64(q), to_f64(k), to_f64(v), to_f64(do), w.scale)
    for name, g, r in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
        # relative Frobenius is undefined for a gradient that is exactly zero
        # (a single key gives dQ = dK = 0): max-abs alone then
        rel = F32_GRAD[1] if np.linalg.norm(r) > F32_GRAD[0] else None
        assert_close(to_np(g), r, F32_GRAD[0], rel, what=f"{name} {what}")


@pytest.mark.parametrize("B,H,Nq,Nk,D", [
    (1, 1, 32, 32, 32),
    (1, 2, 300, 400, 64),       # ragged groups of 32 on both sides
    (2, 1, 257, 513, 128),
    (1, 3, 100, 77, 96),
    (1, 1, 1, 2000, 64),        # one query row: the dQ row is split over 8 warps
    (1, 1, 2000, 1, 64),        # one key: dK = dQ = 0, dV = sum of dO
    (1, 1, 5000, 3, 32),        # long query loop per key row
])
def test_shapes_full(B, H, Nq, Nk, D):
    check(custom(B, H, Nq, Nk, D, "f32"), 7, f"{(B, H, Nq, Nk, D)}")


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_workload(seed):
    """The tiny fp32 self-attention workload (B1 H1 N256 D64) with a gradient of the output."""
    check(make_workload("tiny_f32"), seed, "tiny_f32")


def test_single_query_shape_unit_logits():
    """Single-query shape (8 heads, one row over 16384 keys, D 64) with N(0,1) logits."""
    w = make_workload("single_query_f32")
    check(custom(w.B, w.H, w.Nq, w.Nk, w.D, "f32"), 3, "single query, unit logits")


def test_gqa_f32():
    check(custom(1, 6, 70, 90, 64, "f32", Hkv=2), 4, "gqa fp32")


def test_single_query_large_logits_dv():
    """The single-query workload itself (logits up to ~8e3).

    The backward recomputes P_ij = exp(scale s_ij - lse_i) from the stored fp32
    lse; rounding lse_i to fp32 moves it by up to half an ulp, 2^-24 |lse_i|,
    and that is a relative error of the same size in every P_ij of the row
    (about 2.4e-4 at |lse| = 7.7e3).  With one query row dV_j = P_j dO, so each
    element of dV carries that relative error (doubled for the score rounding
    and the exponential): |err_j| <= 1e-4 + 2^-22 max|lse| |dV_j|.
    """
    w = make_workload("single_query_f32")
    q, k, v, do = make_inputs(w, 0, with_grad_output=True)
    _, _, dv = gpu_fwd_bwd(q, k, v, do, w.scale)
    rv = np.empty(dv.shape)
    lse_max = 0.0
    for h in range(w.H):
        _, _, rv[0, h], _, lse = oracle.attention_backward_2d(to_f64(q[0, h]), to_f64(k[0, h]), to_f64(v[0, h]),
                                                              to_f64(do[0, h]), w.scale)
        lse_max = max(lse_max, float(np.abs(lse).max()))
    assert lse_max > 1e3  # the case exercises large logits
    err = np.abs(to_np(dv) - rv)
    bound = F32_O_MAX_ABS + 2.0 ** -22 * lse_max * np.abs(rv)
    assert np.isfinite(to_np(dv)).all()
    assert (err <= bound).all(), f"dV large logits: worst excess {(err - bound).max():.3e}"


def test_deterministic():
    import exact_memory_efficient_b200 as m
    w = custom(1, 2, 300, 500, 64, "f32")
    q, k, v, do = (x.cuda() for x in make_inputs(w, 1))
    o, lse = m.attention_forward(q, k, v, w.scale)
    a = m.attention_backward(q, k, v, o, lse, do, w.scale)
    b = m.attention_backward(q, k, v, o, lse, do, w.scale)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_phases_match_single_call():
    import exact_memory_efficient_b200 as m
    w = custom(1, 2, 100, 200, 128, "f32")
    q, k, v, do = (x.cuda() for x in make_inputs(w, 2))
    o, lse = m.attention_forward(q, k, v, w.scale)
    ws = torch.empty(m.mea_attn_bwd_workspace_size(1, 2, 100, 200, 128, torch.float32), dtype=torch.uint8,
                     device="cuda")
    g1 = [torch.empty_like(x) for x in (q, k, v)]
    g2 = [torch.empty_like(x) for x in (q, k, v)]
    m.mea_attn_bwd(q, k, v, o, lse, do, *g1, w.scale, ws)
    for ph in (m.MEA_BWD_PREPROCESS, m.MEA_BWD_MAIN, m.MEA_BWD_FINALIZE):
        m.mea_attn_bwd_phase(ph, q, k, v, o, lse, do, *g2, w.scale, ws)
    torch.cuda.synchronize()
    for x, y in zip(g1, g2):
        assert torch.equal(x, y)


def test_empty_queries_zero_grads():
    import exact_memory_efficient_b200 as m
    k = torch.randn(1, 1, 50, 64).cuda()
    q = torch.empty(1, 1, 0, 64, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty(1, 1, 0, device="cuda")
    dk = torch.full_like(k, 7.0)
    dv = torch.full_like(k, 7.0)
    dq = torch.empty_like(q)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    m.mea_attn_bwd(q, k, k, o, lse, q, dq, dk, dv, 0.125, ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dk) == 0 and torch.count_nonzero(dv) == 0
