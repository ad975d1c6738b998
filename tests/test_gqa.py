"""Shared key/value heads (grouped- and multi-query attention) through the C ABI (GPU).

The oracle loops over query heads and reads key/value head h // G for each, then
sums the per-head dK, dV over each group; the library instead runs its kernels
over each group's query rows as one contiguous block.  The two routes share
nothing but the seeded inputs.
"""

import numpy as np
import pytest
import torch

import oracle
from synthetic_inputs import custom, make_inputs, make_workload, to_f64
from tests._parity import BF16_GRAD, BF16_O, F32_O_MAX_ABS, assert_close, assert_lse_close, to_np

pytestmark = pytest.mark.gpu


def _gpu(x):
    return None if x is None else x.cuda()


@pytest.mark.parametrize("B,H,Hkv,Nq,Nk,D", [
    (1, 4, 2, 200, 333, 128),    # ragged tails; the group's rows straddle a query tile
    (2, 8, 1, 130, 257, 64),     # multi-query: every head shares one key/value head
    (1, 32, 8, 64, 300, 128),    # the page's example grouping, 32 heads in 8 groups of 4
    (1, 6, 3, 1, 500, 64),       # one query row per head
    (1, 2, 1, 300, 1, 128),      # a single key: dK = 0 and dV sums every dO row of the group
])
def test_gqa_bf16_forward_backward(B, H, Hkv, Nq, Nk, D):
    import exact_memory_efficient_b200 as m
    w = custom(B, H, Nq, Nk, D, "bf16", Hkv=Hkv)
    q, k, v, do = make_inputs(w, 11)
    qd, kd, vd, dod = map(_gpu, (q, k, v, do))
    o, lse = m.attention_forward(qd, kd, vd, w.scale)
    dq, dk, dv = m.attention_backward(qd, kd, vd, o, lse, dod, w.scale)
    assert m.mea_last_device_error() == m.MEA_OK
    rq, rk, rv, ro, rl = oracle.attention_backward_gqa(to_f64(q), to_f64(k), to_f64(v), to_f64(do), w.scale)
    what = f"{(B, H, Hkv, Nq, Nk, D)}"
    assert_close(to_np(o), ro, *BF16_O, what=f"O {what}")
    assert_lse_close(to_np(lse), rl, to_f64(q), np.repeat(to_f64(k), H // Hkv, axis=1), w.scale,
                     what=f"lse {what}")
    assert_close(to_np(dq), rq, *BF16_GRAD, what=f"dQ {what}")
    assert_close(to_np(dk), rk, *BF16_GRAD, what=f"dK {what}")
    # a single key makes dV the sum of every dO row of the group (|dV| ~ 80 here): beyond order one
    assert_close(to_np(dv), rv, *BF16_GRAD, what=f"dV {what}", large_outputs=(Nk == 1))


def test_gqa_equal_heads_is_the_per_head_path():
    """H_kv == H through the _gqa entry points gives bit-identical results to the plain ones."""
    import exact_memory_efficient_b200 as m
    w = custom(2, 3, 257, 129, 128, "bf16")
    q, k, v, do = map(_gpu, make_inputs(w, 3))
    o1 = torch.empty_like(q)
    l1 = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    o2, l2 = torch.empty_like(o1), torch.empty_like(l1)
    m.mea_attn_fwd(q, k, v, o1, l1, w.scale)
    m.mea_attn_fwd_gqa(q, k, v, o2, l2, w.scale)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    ws = torch.empty(m.mea_attn_bwd_gqa_workspace_size(2, 3, 3, 257, 129, 128), dtype=torch.uint8, device=q.device)
    g1 = [torch.empty_like(x) for x in (q, k, v)]
    g2 = [torch.empty_like(x) for x in (q, k, v)]
    m.mea_attn_bwd(q, k, v, o1, l1, do, *g1, w.scale, ws)
    m.mea_attn_bwd_gqa(q, k, v, o1, l1, do, *g2, w.scale, ws)
    torch.cuda.synchronize()
    # dK, dV are deterministic; dQ is summed by reduce-adds in no fixed order
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
    assert_close(to_np(g2[0]), to_np(g1[0]), 1e-2, what="dQ gqa vs per-head")


def test_gqa_dk_dv_deterministic():
    import exact_memory_efficient_b200 as m
    w = custom(1, 8, 300, 700, 64, "bf16", Hkv=2)
    q, k, v, do = map(_gpu, make_inputs(w, 5))
    o, lse = m.attention_forward(q, k, v, w.scale)
    a = m.attention_backward(q, k, v, o, lse, do, w.scale)
    b = m.attention_backward(q, k, v, o, lse, do, w.scale)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


def test_gqa_fp32_forward():
    import exact_memory_efficient_b200 as m
    w = custom(1, 8, 3, 2000, 64, "f32", backward=False, Hkv=2)
    q, k, v, _ = make_inputs(w, 2)
    o, lse = m.attention_forward(q.cuda(), k.cuda(), v.cuda(), w.scale)
    ro, rl = oracle.attention_forward_gqa(to_f64(q), to_f64(k), to_f64(v), w.scale)
    assert_close(to_np(o), ro, F32_O_MAX_ABS, what="fp32 gqa O")
    assert_lse_close(to_np(lse), rl, to_f64(q), np.repeat(to_f64(k), 4, axis=1), w.scale, what="fp32 gqa lse")


@pytest.mark.parametrize("seed", [0, 1])
def test_decode_gqa_full(seed):
    """Decode-shaped grouped-query forward at full size (32 heads over 8 key/value heads, 16384 keys)."""
    import exact_memory_efficient_b200 as m
    w = make_workload("decode_gqa_32x8_16384_bf16")
    q, k, v, _ = make_inputs(w, seed)
    o, lse = m.attention_forward(q.cuda(), k.cuda(), v.cuda(), w.scale)
    assert m.mea_last_device_error() == m.MEA_OK
    ro, rl = oracle.attention_forward_gqa(to_f64(q), to_f64(k), to_f64(v), w.scale)
    assert_close(to_np(o), ro, *BF16_O, what="decode gqa O")
    assert_lse_close(to_np(lse), rl, to_f64(q), np.repeat(to_f64(k), 4, axis=1), w.scale, what="decode gqa lse")


@pytest.mark.parametrize("seed", [0, 1])
def test_gqa_workload_sampled(seed):
    """Full-size grouped-query launch (B1, 32 heads over 8, N 4096, D 128); the oracle checks
    sampled dQ rows and sampled dK/dV key rows of a few key/value heads, summed over the group."""
    import exact_memory_efficient_b200 as m
    w = make_workload("gqa_32x8_4096_bf16")
    G = w.H // w.H_kv
    q, k, v, do = make_inputs(w, seed)
    qd, kd, vd, dod = map(_gpu, (q, k, v, do))
    o, lse = m.attention_forward(qd, kd, vd, w.scale)
    dq, dk, dv = m.attention_backward(qd, kd, vd, o, lse, dod, w.scale)
    assert m.mea_last_device_error() == m.MEA_OK
    o, lse, dq, dk, dv = map(to_np, (o, lse, dq, dk, dv))
    rng = np.random.default_rng(200 + seed)
    for hk in sorted({0, w.H_kv - 1, int(rng.integers(w.H_kv))}):
        k2, v2 = to_f64(k[0, hk]), to_f64(v[0, hk])
        rows = np.unique(np.concatenate([[0, w.Nq - 1], rng.choice(w.Nq, 24, replace=False)]))
        keys = np.unique(np.concatenate([[0, w.Nk - 1], rng.choice(w.Nk, 24, replace=False)]))
        rk = np.zeros((len(keys), w.D))
        rv = np.zeros((len(keys), w.D))
        for g in range(G):
            h = hk * G + g
            q2, do2 = to_f64(q[0, h]), to_f64(do[0, h])
            ro, rl = oracle.attention_forward_rows(q2, k2, v2, w.scale, rows)
            assert_close(o[0, h][rows], ro, *BF16_O, what=f"O head {h}")
            assert_lse_close(lse[0, h][rows], rl, q2[rows], k2, w.scale, what=f"lse head {h}")
            rq = oracle.attention_backward_rows(q2, k2, v2, do2, w.scale, rows)
            assert_close(dq[0, h][rows], rq, *BF16_GRAD, what=f"dQ head {h}")
            o_all, lse_all = oracle.attention_forward_2d(q2, k2, v2, w.scale)
            dk_h, dv_h = oracle.attention_backward_keys(q2, k2, v2, do2, w.scale, keys, lse_all, o_all)
            rk += dk_h
            rv += dv_h
        assert_close(dk[0, hk][keys], rk, *BF16_GRAD, what=f"dK kv head {hk}")
        assert_close(dv[0, hk][keys], rv, *BF16_GRAD, what=f"dV kv head {hk}")
