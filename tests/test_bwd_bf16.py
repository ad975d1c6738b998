"""bf16 tcgen05 backward against the fp64 oracle, through the C ABI (GPU).

The GPU backward consumes the GPU forward's own o and lse (as a user would);
the oracle computes everything from the inputs in fp64.
"""

import numpy as np
import pytest
import torch

import oracle
from synthetic_inputs import custom, make_inputs, make_workload, to_f64
from tests._parity import BF16_GRAD, assert_close, to_np

pytestmark = pytest.mark.gpu


def gpu_fwd_bwd(q, k, v, do, scale):
    import exact_memory_efficient_b200 as m
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = m.attention_forward(qd, kd, vd, scale)
    dq, dk, dv = m.attention_backward(qd, kd, vd, o, lse, dod, scale)
    assert m.mea_last_device_error() == m.MEA_OK
    return dq, dk, dv


@pytest.mark.parametrize("B,H,Nq,Nk,D", [
    (1, 1, 128, 128, 64),
    (1, 1, 128, 128, 128),
    (1, 2, 300, 400, 64),     # ragged tails on both sides
    (2, 1, 257, 513, 128),
    (1, 1, 1, 200, 128),      # single query row
    (1, 1, 200, 1, 64),       # single key: dK = dQ = 0
    (1, 3, 640, 384, 128),    # several query tiles per key tile
])
def test_shapes_full(B, H, Nq, Nk, D):
    w = custom(B, H, Nq, Nk, D, "bf16")
    q, k, v, do = make_inputs(w, 7)
    dq, dk, dv = gpu_fwd_bwd(q, k, v, do, w.scale)
    rq, rk, rv, _, _ = oracle.attention_backward(to_f64(q), to_f64(k), to_f64(v), to_f64(do), w.scale)
    what = f"{(B, H, Nq, Nk, D)}"
    assert_close(to_np(dq), rq, *BF16_GRAD, what=f"dQ {what}")
    assert_close(to_np(dk), rk, *BF16_GRAD, what=f"dK {what}")
    # a single key makes dV_0 the sum of every dO row (|dV| ~ 33 here): beyond order one
    assert_close(to_np(dv), rv, *BF16_GRAD, what=f"dV {what}", large_outputs=(Nk == 1))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_encoder_512_full(seed):
    w = make_workload("encoder_512_bf16")
    q, k, v, do = make_inputs(w, seed)
    dq, dk, dv = gpu_fwd_bwd(q, k, v, do, w.scale)
    # oracle on 16 of the 256 (batch, head) pairs, all rows and keys
    rng = np.random.default_rng(seed)
    pairs = [(0, 0), (w.B - 1, w.H - 1)] + [(int(rng.integers(w.B)), int(rng.integers(w.H))) for _ in range(14)]
    dq, dk, dv = to_np(dq), to_np(dk), to_np(dv)
    for b, h in pairs:
        rq, rk, rv, _, _ = oracle.attention_backward_2d(to_f64(q[b, h]), to_f64(k[b, h]), to_f64(v[b, h]),
                                                        to_f64(do[b, h]), w.scale)
        assert_close(dq[b, h], rq, *BF16_GRAD, what=f"dQ ({b},{h})")
        assert_close(dk[b, h], rk, *BF16_GRAD, what=f"dK ({b},{h})")
        assert_close(dv[b, h], rv, *BF16_GRAD, what=f"dV ({b},{h})")


@pytest.mark.parametrize("name", ["mha_4k_bf16", "long_256_bf16", "long_1024_bf16", "long_4096_bf16",
                                  "long_16384_bf16"])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_workloads_sampled(name, seed):
    """Full-size launch; oracle on sampled dQ rows and dK/dV key rows of a few heads."""
    w = make_workload(name)
    q, k, v, do = make_inputs(w, seed)
    dq, dk, dv = gpu_fwd_bwd(q, k, v, do, w.scale)
    dq, dk, dv = to_np(dq), to_np(dk), to_np(dv)
    rng = np.random.default_rng(100 + seed)
    heads = sorted({(0, 0), (w.B - 1, w.H - 1), (int(rng.integers(w.B)), int(rng.integers(w.H)))})
    n = min(w.Nq, 32)
    for b, h in heads:
        q2, k2, v2, do2 = to_f64(q[b, h]), to_f64(k[b, h]), to_f64(v[b, h]), to_f64(do[b, h])
        rows = np.unique(np.concatenate([[0, w.Nq - 1], rng.choice(w.Nq, n, replace=False)]))
        keys = np.unique(np.concatenate([[0, w.Nk - 1], rng.choice(w.Nk, n, replace=False)]))
        rq = oracle.attention_backward_rows(q2, k2, v2, do2, w.scale, rows)
        # per-row lse and O of every query row are needed for key-column gradients
        o_all = np.empty_like(q2)
        lse_all = np.empty(w.Nq)
        for r0 in range(0, w.Nq, 2048):
            idx = np.arange(r0, min(w.Nq, r0 + 2048))
            o_all[idx], lse_all[idx] = oracle.attention_forward_rows(q2, k2, v2, w.scale, idx)
        rk, rv = oracle.attention_backward_keys(q2, k2, v2, do2, w.scale, keys, lse_all, o_all)
        assert_close(dq[b, h, rows], rq, *BF16_GRAD, what=f"dQ {name} ({b},{h})")
        assert_close(dk[b, h, keys], rk, *BF16_GRAD, what=f"dK {name} ({b},{h})")
        assert_close(dv[b, h, keys], rv, *BF16_GRAD, what=f"dV {name} ({b},{h})")


def test_gradient_sum_rules():
    """sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i hold at any size."""
    w = custom(1, 2, 1000, 3000, 128, "bf16")
    q, k, v, do = make_inputs(w, 9)
    dq, dk, dv = gpu_fwd_bwd(q, k, v, do, w.scale)
    dk64, dv64 = to_np(dk), to_np(dv)
    np.testing.assert_allclose(dk64.sum(axis=2), 0.0, atol=0.3)
    np.testing.assert_allclose(dv64.sum(axis=2), to_f64(do).sum(axis=2), atol=0.3)


def test_empty_queries_zero_grads():
    import exact_memory_efficient_b200 as m
    k = torch.randn(1, 1, 50, 64).to(torch.bfloat16).cuda()
    q = torch.empty(1, 1, 0, 64, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty(1, 1, 0, device="cuda")
    dk = torch.full_like(k, 7.0)
    dv = torch.full_like(k, 7.0)
    m.mea_attn_bwd(q, k, k, o, lse, q, torch.empty_like(q), dk, dv, 0.125, None)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dk) == 0 and torch.count_nonzero(dv) == 0


def test_dk_dv_deterministic():
    w = custom(1, 2, 700, 500, 64, "bf16")
    q, k, v, do = make_inputs(w, 4)
    a = gpu_fwd_bwd(q, k, v, do, w.scale)
    b = gpu_fwd_bwd(q, k, v, do, w.scale)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    # dQ is accumulated with fp32 atomics: equal up to summation order
    assert torch.allclose(a[0].float(), b[0].float(), atol=1e-2)


@pytest.mark.parametrize("B,H,Nq,Nk,D", [
    (8, 16, 300, 700, 64),    # 768 (head, key tile) items: five or six per persistent CTA, ragged tails
    (16, 16, 128, 77, 64),    # one query tile and one partial key tile per item, 256 items
    (4, 20, 1000, 333, 64),   # eight query tiles per item, the longest loop that runs persistent
    (1, 2, 1100, 260, 64),    # nine query tiles: one CTA per item
])
def test_persistent_items_backward(B, H, Nq, Nk, D):
    """At D = 64 with at most 8 query tiles per key tile the backward runs persistent CTAs: the next
    item's K, V load into the other buffer and its first S^T and P are formed before the current
    item's epilogue has freed the dV, dK accumulators."""
    w = custom(B, H, Nq, Nk, D, "bf16")
    q, k, v, do = make_inputs(w, 19)
    dq, dk, dv = gpu_fwd_bwd(q, k, v, do, w.scale)
    rq, rk, rv, _, _ = oracle.attention_backward(to_f64(q), to_f64(k), to_f64(v), to_f64(do), w.scale)
    what = f"{(B, H, Nq, Nk, D)}"
    assert_close(to_np(dq), rq, *BF16_GRAD, what=f"dQ {what}")
    assert_close(to_np(dk), rk, *BF16_GRAD, what=f"dK {what}")
    assert_close(to_np(dv), rv, *BF16_GRAD, what=f"dV {what}")
