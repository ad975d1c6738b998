"""Pins for the fp64 oracle, independent of the oracle's own code.

Each check comes from something the pages or the mathematics fix, not from
re-typing the oracle's formula:

* hand-derived closed forms (tests/golden/worked_example.json);
* central finite differences of sum(dO o O) for every gradient;
* an independent library: torch fp64 autograd through torch.softmax;
* shift invariance of a score row, all-equal keys, a dominant key,
  permutations, Nk = 1, gradient sum rules;
* logits of ~1e3, where a max-free exponential overflows;
* the pages' chunked algorithm (any block size) reaching the plain definition,
  and the two-block merge formulas on a hand-computed case;
* planted mistakes in copies of the backward must be caught by the pins.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from synthetic_inputs import make_inputs, make_workload, custom, to_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, mult=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * mult


# ------------------------------------------------------------ closed forms

def test_worked_examples_golden():
    cases = json.load(open(os.path.join(GOLDEN, "worked_example.json")))["cases"]
    assert len(cases) >= 3
    for c in cases:
        q, k, v, do = (np.array(c[x], dtype=np.float64) for x in ("q", "k", "v", "do"))
        o, lse = oracle.attention_forward_2d(q, k, v, c["scale"])
        np.testing.assert_allclose(o, c["o"], rtol=0, atol=1e-13, err_msg=c["name"])
        np.testing.assert_allclose(lse, c["lse"], rtol=0, atol=1e-13, err_msg=c["name"])
        dq, dk, dv, o2, lse2 = oracle.attention_backward_2d(q, k, v, do, c["scale"])
        np.testing.assert_allclose(dq, c["dq"], rtol=0, atol=1e-13, err_msg=c["name"])
        np.testing.assert_allclose(dk, c["dk"], rtol=0, atol=1e-13, err_msg=c["name"])
        np.testing.assert_allclose(dv, c["dv"], rtol=0, atol=1e-13, err_msg=c["name"])
        np.testing.assert_allclose(o2, c["o"], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse2, c["lse"], rtol=0, atol=1e-13)


def test_all_keys_equal():
    """K_j = k for all j: O_i = mean_j V_j, lse_i = scale q_i.k + ln Nk, dQ = 0."""
    Nq, Nk, D, scale = 5, 7, 3, 0.37
    q, v, do = rnd((Nq, D), 1), rnd((Nk, D), 2), rnd((Nq, D), 3)
    kvec = rnd((D,), 4)
    k = np.tile(kvec, (Nk, 1))
    o, lse = oracle.attention_forward_2d(q, k, v, scale)
    np.testing.assert_allclose(o, np.tile(v.mean(axis=0), (Nq, 1)), atol=1e-14)
    np.testing.assert_allclose(lse, scale * (q @ kvec) + math.log(Nk), atol=1e-13)
    dq, dk, dv, _, _ = oracle.attention_backward_2d(q, k, v, do, scale)
    np.testing.assert_allclose(dq, 0.0, atol=1e-14)
    # dV_j = sum_i dO_i / Nk for every key
    np.testing.assert_allclose(dv, np.tile(do.sum(axis=0) / Nk, (Nk, 1)), atol=1e-14)
    # dK_j = scale/Nk * sum_i (dO_i.v_j - dO_i.mean(V)) q_i
    vbar = v.mean(axis=0)
    expect = np.zeros((Nk, D))
    for j in range(Nk):
        for i in range(Nq):
            expect[j] += scale / Nk * (do[i] @ v[j] - do[i] @ vbar) * q[i]
    np.testing.assert_allclose(dk, expect, atol=1e-13)


def test_dominant_key():
    """One-hot keys, Q_i = b e_pi(i): one score exceeds the rest by > 50, O_i = V_pi(i)."""
    D = 8
    Nk = D
    a, b, scale = 10.0, 8.0, 1.0  # scale*a*b = 80 > 50
    perm = np.array([3, 0, 7, 5, 1, 6, 2, 4, 3, 3])
    k = a * np.eye(D)
    q = b * np.eye(D)[perm]
    v = rnd((Nk, D), 5)
    o, lse = oracle.attention_forward_2d(q, k, v, scale)
    np.testing.assert_allclose(o, v[perm], atol=Nk * math.exp(-80) * 10)
    np.testing.assert_allclose(lse, scale * a * b + np.log1p((Nk - 1) * math.exp(-80)), atol=1e-13)


def test_dominant_key_single_query_long():
    """Nq = 1 over 16384 keys, k_star placed so its score is 60 above the runner-up."""
    rng = np.random.default_rng(7)
    D, Nk, scale = 64, 16384, 1.0 / 8
    q = rng.standard_normal((1, D)) * 40
    k = rng.standard_normal((Nk, D)) * 40
    v = rng.standard_normal((Nk, D))
    s = scale * (q @ k.T)[0]
    j_star = 1234
    others = np.delete(s, j_star)
    # move k_star along q so that its score becomes max(others) + 60
    need = others.max() + 60.0 - s[j_star]
    k[j_star] += need / (scale * (q[0] @ q[0])) * q[0]
    o, lse = oracle.attention_forward_2d(q, k, v, scale)
    np.testing.assert_allclose(o[0], v[j_star], atol=Nk * math.exp(-60) * 10)
    assert abs(lse[0] - (others.max() + 60.0)) < 1e-9 * abs(lse[0])


def test_large_logits_closed_form_and_max_free_overflow():
    """Scores 1000 and 1000 - ln 3 give weights 3/4, 1/4; exp without the max overflows."""
    q = np.array([[1.0]])
    k = np.array([[1000.0], [1000.0 - math.log(3.0)]])
    v = np.array([[4.0], [0.0]])
    o, lse = oracle.attention_forward_2d(q, k, v, 1.0)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    np.testing.assert_allclose(o, [[3.0]], atol=1e-12)
    np.testing.assert_allclose(lse, [1000.0 + math.log(4.0 / 3.0)], atol=1e-12)
    # A max-free evaluation of the same definition is not finite here: this is
    # what makes the large-logit workloads a test of the max tracking.
    with np.errstate(over="ignore", invalid="ignore"):
        e = np.exp(1.0 * (q @ k.T))
        o_free = (e @ v) / e.sum(axis=1, keepdims=True)
    assert not np.isfinite(o_free).all()


def test_single_query_workload_logits_overflow_max_free():
    """The single-query fp32 workload really reaches logits beyond exp's fp64 range."""
    w = make_workload("single_query_f32")
    q, k, v, _ = make_inputs(w, 0)
    s = w.scale * (to_f64(q[0, 0]) @ to_f64(k[0, 0]).T)
    assert np.abs(s).max() > 709.8  # exp overflows fp64 beyond ln(DBL_MAX) ~ 709.78
    o, lse = oracle.attention_forward_2d(to_f64(q[0, 0]), to_f64(k[0, 0]), to_f64(v[0, 0]), w.scale)
    assert np.isfinite(o).all() and np.isfinite(lse).all()


# --------------------------------------------------------------- invariants

def test_shift_invariance_of_score_rows():
    """K -> K + 1 u^T shifts row i by scale q_i.u: O and all grads unchanged, lse shifts."""
    Nq, Nk, D, scale = 6, 9, 4, 0.5
    q, k, v, do = rnd((Nq, D), 11), rnd((Nk, D), 12), rnd((Nk, D), 13), rnd((Nq, D), 14)
    u = np.array([1.0, -2.0, 0.0, 3.0])
    o1, lse1 = oracle.attention_forward_2d(q, k, v, scale)
    o2, lse2 = oracle.attention_forward_2d(q, k + u, v, scale)
    np.testing.assert_allclose(o2, o1, atol=1e-13)
    np.testing.assert_allclose(lse2 - lse1, scale * (q @ u), atol=1e-13)
    g1 = oracle.attention_backward_2d(q, k, v, do, scale)
    g2 = oracle.attention_backward_2d(q, k + u, v, do, scale)
    for a, b in zip(g1[:3], g2[:3]):
        np.testing.assert_allclose(a, b, atol=1e-12)


def test_permutations():
    Nq, Nk, D, scale = 7, 10, 5, 0.3
    q, k, v, do = rnd((Nq, D), 21), rnd((Nk, D), 22), rnd((Nk, D), 23), rnd((Nq, D), 24)
    pk = np.random.default_rng(0).permutation(Nk)
    pq = np.random.default_rng(1).permutation(Nq)
    o, lse = oracle.attention_forward_2d(q, k, v, scale)
    o_k, lse_k = oracle.attention_forward_2d(q, k[pk], v[pk], scale)
    np.testing.assert_allclose(o_k, o, atol=1e-13)
    np.testing.assert_allclose(lse_k, lse, atol=1e-13)
    o_q, lse_q = oracle.attention_forward_2d(q[pq], k, v, scale)
    np.testing.assert_allclose(o_q, o[pq], atol=1e-13)
    np.testing.assert_allclose(lse_q, lse[pq], atol=1e-13)
    dq, dk, dv, _, _ = oracle.attention_backward_2d(q, k, v, do, scale)
    dq2, dk2, dv2, _, _ = oracle.attention_backward_2d(q, k[pk], v[pk], do, scale)
    np.testing.assert_allclose(dq2, dq, atol=1e-12)
    np.testing.assert_allclose(dk2, dk[pk], atol=1e-12)
    np.testing.assert_allclose(dv2, dv[pk], atol=1e-12)


def test_gradient_sum_rules():
    """sum_j dK_j = 0 (each dS row sums to 0) and sum_j dV_j = sum_i dO_i (rows of P sum to 1)."""
    Nq, Nk, D, scale = 8, 11, 6, 0.41
    q, k, v, do = rnd((Nq, D), 31), rnd((Nk, D), 32), rnd((Nk, D), 33), rnd((Nq, D), 34)
    dq, dk, dv, _, _ = oracle.attention_backward_2d(q, k, v, do, scale)
    np.testing.assert_allclose(dk.sum(axis=0), 0.0, atol=1e-12)
    np.testing.assert_allclose(dv.sum(axis=0), do.sum(axis=0), atol=1e-12)


def test_single_key():
    """Nk = 1: O = V_0, lse = scale q.k_0, dQ = dK = 0, dV_0 = sum_i dO_i."""
    Nq, D, scale = 5, 3, 0.7
    q, k, v, do = rnd((Nq, D), 41), rnd((1, D), 42), rnd((1, D), 43), rnd((Nq, D), 44)
    o, lse = oracle.attention_forward_2d(q, k, v, scale)
    np.testing.assert_allclose(o, np.tile(v[0], (Nq, 1)), atol=1e-15)
    np.testing.assert_allclose(lse, scale * (q @ k[0]), atol=1e-14)
    dq, dk, dv, _, _ = oracle.attention_backward_2d(q, k, v, do, scale)
    np.testing.assert_allclose(dq, 0.0, atol=1e-15)
    np.testing.assert_allclose(dk, 0.0, atol=1e-15)
    np.testing.assert_allclose(dv[0], do.sum(axis=0), atol=1e-14)


# ---------------------------------------------------- brute force / library

def _loss(q, k, v, do, scale):
    o, _ = oracle.attention_forward_2d(q, k, v, scale)
    return float((do * o).sum())


def _central_diff(f, x, h=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        g[idx] = (f(xp) - f(xm)) / (2 * h)
    return g


@pytest.mark.parametrize("Nq,Nk,D,scale,seed", [(1, 1, 1, 1.0, 0), (3, 5, 2, 0.7, 1),
                                                (8, 8, 4, 0.5, 2), (6, 3, 4, 1.3, 3)])
def test_finite_differences(Nq, Nk, D, scale, seed):
    q, k, v, do = rnd((Nq, D), seed), rnd((Nk, D), seed + 10), rnd((Nk, D), seed + 20), rnd((Nq, D), seed + 30)
    dq, dk, dv, _, _ = oracle.attention_backward_2d(q, k, v, do, scale)
    np.testing.assert_allclose(dq, _central_diff(lambda x: _loss(x, k, v, do, scale), q), atol=1e-8)
    np.testing.assert_allclose(dk, _central_diff(lambda x: _loss(q, x, v, do, scale), k), atol=1e-8)
    np.testing.assert_allclose(dv, _central_diff(lambda x: _loss(q, k, x, do, scale), v), atol=1e-8)


def test_forward_finite_difference_of_lse():
    """d lse_i / d q_i = scale * sum_j P_ij k_j = scale * (softmax-weighted mean key)."""
    Nq, Nk, D, scale = 2, 6, 3, 0.9
    q, k, v = rnd((Nq, D), 51), rnd((Nk, D), 52), rnd((Nk, D), 53)
    _, lse = oracle.attention_forward_2d(q, k, v, scale)
    for i in range(Nq):
        g = _central_diff(lambda x: float(oracle.attention_forward_2d(x[None], k, v, scale)[1][0]), q[i])
        # the same derivative from the forward applied to V := K
        o_k, _ = oracle.attention_forward_2d(q[i:i + 1], k, k, scale)
        np.testing.assert_allclose(g, scale * o_k[0], atol=1e-8)


@pytest.mark.parametrize("B,H,Nq,Nk,D", [(2, 3, 17, 29, 8), (1, 2, 64, 5, 16)])
def test_against_torch_autograd_fp64(B, H, Nq, Nk, D):
    """torch.softmax + autograd in fp64 is an independent library implementation."""
    g = torch.Generator().manual_seed(99)
    q = torch.randn(B, H, Nq, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, H, Nk, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, H, Nk, D, generator=g, dtype=torch.float64)
    do = torch.randn(B, H, Nq, D, generator=g, dtype=torch.float64)
    scale = 1.0 / math.sqrt(D)
    qt, kt, vt = (x.clone().requires_grad_(True) for x in (q, k, v))
    s = torch.matmul(qt, kt.transpose(-1, -2)) * scale
    ot = torch.matmul(torch.softmax(s, dim=-1), vt)
    lse_t = torch.logsumexp(s, dim=-1)
    ot.backward(do)
    o, lse = oracle.attention_forward(q.numpy(), k.numpy(), v.numpy(), scale)
    np.testing.assert_allclose(o, ot.detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(lse, lse_t.detach().numpy(), atol=1e-12)
    dq, dk, dv, o2, lse2 = oracle.attention_backward(q.numpy(), k.numpy(), v.numpy(), do.numpy(), scale)
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-11)


# ------------------------------------------ chunked method and merge rule

def test_two_block_merge_hand_case():
    """Blocks S1 = [0], S2 = [ln 3] with V1 = [0], V2 = [4]: m = ln3, l = 4/3, O = 3."""
    m1, l1, acc1 = np.array([0.0]), np.array([1.0]), np.array([[0.0]])
    m2, l2, acc2 = np.array([math.log(3)]), np.array([1.0]), np.array([[4.0]])
    m, l, acc = oracle.combine_two_blocks(m1, l1, acc1, m2, l2, acc2)
    np.testing.assert_allclose(m, [math.log(3)], atol=1e-15)
    np.testing.assert_allclose(l, [4.0 / 3.0], atol=1e-15)
    np.testing.assert_allclose(acc / l[:, None], [[3.0]], atol=1e-15)
    np.testing.assert_allclose(m + np.log(l), [math.log(4.0)], atol=1e-15)


@pytest.mark.parametrize("Nq,Nk,D", [(5, 100, 8), (3, 256, 64), (1, 1000, 16)])
def test_chunked_method_reaches_definition(Nq, Nk, D):
    q, k, v = rnd((Nq, D), 61, 3.0), rnd((Nk, D), 62, 3.0), rnd((Nk, D), 63)
    scale = 1.0 / math.sqrt(D)
    o, lse = oracle.attention_forward_2d(q, k, v, scale)
    for block in (1, 3, int(math.isqrt(Nk)), Nk):
        oc, lsec = oracle.chunked_forward_2d(q, k, v, scale, block)
        np.testing.assert_allclose(oc, o, atol=1e-12, rtol=0)
        np.testing.assert_allclose(lsec, lse, atol=1e-12, rtol=0)


# -------------------------------------------------- sampled full-size forms

def test_sampled_forms_match_full():
    w = custom(1, 2, 40, 33, 16, "bf16")
    q, k, v, do = make_inputs(w, 3)
    q, k, v, do = (to_f64(x) for x in (q, k, v, do))
    dq, dk, dv, o, lse = oracle.attention_backward(q, k, v, do, w.scale)
    rows = [0, 7, 39]
    keys = [0, 5, 32]
    for h in range(2):
        o_r, lse_r = oracle.attention_forward_rows(q[0, h], k[0, h], v[0, h], w.scale, rows)
        np.testing.assert_allclose(o_r, o[0, h, rows], atol=1e-13)
        np.testing.assert_allclose(lse_r, lse[0, h, rows], atol=1e-13)
        dq_r = oracle.attention_backward_rows(q[0, h], k[0, h], v[0, h], do[0, h], w.scale, rows)
        np.testing.assert_allclose(dq_r, dq[0, h, rows], atol=1e-12)
        dk_c, dv_c = oracle.attention_backward_keys(q[0, h], k[0, h], v[0, h], do[0, h], w.scale, keys,
                                                    lse[0, h], o[0, h])
        np.testing.assert_allclose(dk_c, dk[0, h, keys], atol=1e-12)
        np.testing.assert_allclose(dv_c, dv[0, h, keys], atol=1e-12)


# ------------------------------------------------------ planted mistakes

def _mutant_backward(kind):
    """Copies of the closed-form backward with one plausible mistake planted."""
    def f(q, k, v, do, scale):
        s = scale * (q @ k.T)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        if kind != "unnormalised":
            p /= p.sum(axis=1, keepdims=True)
        o = p @ v
        dv = p.T @ do
        dp = do @ v.T
        d_row = (do * o).sum(axis=1, keepdims=True)
        if kind == "drop_D":
            ds = p * dp
        elif kind == "sign":
            ds = p * (d_row - dp)
        else:
            ds = p * (dp - d_row)
        dq = scale * (ds @ k)
        dk = scale * (ds.T @ q)
        if kind == "no_scale":
            dq = ds @ k
        if kind == "dv_from_ds":
            dv = ds.T @ do
        if kind == "q_for_k":
            dq = scale * (ds @ v)
        return dq, dk, dv
    return f


@pytest.mark.parametrize("kind", ["drop_D", "sign", "no_scale", "dv_from_ds", "q_for_k", "unnormalised"])
def test_pins_catch_planted_backward_mistakes(kind):
    Nq, Nk, D, scale = 4, 6, 3, 0.6
    q, k, v, do = rnd((Nq, D), 71), rnd((Nk, D), 72), rnd((Nk, D), 73), rnd((Nq, D), 74)
    dq, dk, dv = _mutant_backward(kind)(q, k, v, do, scale)
    fd = (_central_diff(lambda x: _loss(x, k, v, do, scale), q),
          _central_diff(lambda x: _loss(q, x, v, do, scale), k),
          _central_diff(lambda x: _loss(q, k, x, do, scale), v))
    errs = [np.abs(a - b).max() for a, b in zip((dq, dk, dv), fd)]
    assert max(errs) > 1e-4, f"planted mistake {kind} not detected"


def test_pins_catch_planted_forward_mistakes():
    """A missing max subtraction, a base-2 lse or a wrong scale fails a closed form."""
    c = json.load(open(os.path.join(GOLDEN, "worked_example.json")))["cases"][1]
    q, k, v = (np.array(c[x]) for x in ("q", "k", "v"))
    s_wrong_scale = (q @ k.T)  # scale dropped
    e = np.exp(s_wrong_scale - s_wrong_scale.max(1, keepdims=True))
    o_bad = (e / e.sum(1, keepdims=True)) @ v
    assert abs(o_bad[0, 0] - c["o"][0][0]) > 1e-3
    s = c["scale"] * (q @ k.T)
    lse_base2 = np.log2(np.exp(s).sum(1))
    assert abs(lse_base2[0] - c["lse"][0]) > 1e-3


# ------------------------------------------------- shared key/value heads

def _loss_gqa(q, k, v, do, scale):
    o, _ = oracle.attention_forward_gqa(q, k, v, scale)
    return float((do * o).sum())


@pytest.mark.parametrize("H,Hkv", [(4, 2), (3, 1), (2, 2)])
def test_gqa_finite_differences(H, Hkv):
    """Brute-force gradients of the shared-head loss, including the sum over each group."""
    rng = np.random.default_rng(H * 10 + Hkv)
    Nq, Nk, D, scale = 3, 4, 2, 0.8
    q = rng.standard_normal((1, H, Nq, D))
    k = rng.standard_normal((1, Hkv, Nk, D))
    v = rng.standard_normal((1, Hkv, Nk, D))
    do = rng.standard_normal((1, H, Nq, D))
    dq, dk, dv, _, _ = oracle.attention_backward_gqa(q, k, v, do, scale)
    np.testing.assert_allclose(dq, _central_diff(lambda x: _loss_gqa(x, k, v, do, scale), q), atol=1e-8)
    np.testing.assert_allclose(dk, _central_diff(lambda x: _loss_gqa(q, x, v, do, scale), k), atol=1e-8)
    np.testing.assert_allclose(dv, _central_diff(lambda x: _loss_gqa(q, k, x, do, scale), v), atol=1e-8)


def test_gqa_matches_torch_autograd_with_shared_heads():
    """torch fp64 autograd with K/V expanded by repeat_interleave (an independent library path)."""
    g = torch.Generator().manual_seed(5)
    B, H, Hkv, Nq, Nk, D = 2, 6, 2, 9, 13, 8
    q = torch.randn(B, H, Nq, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, Hkv, Nk, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, Hkv, Nk, D, generator=g, dtype=torch.float64)
    do = torch.randn(B, H, Nq, D, generator=g, dtype=torch.float64)
    scale = 0.3
    qt, kt, vt = (x.clone().requires_grad_(True) for x in (q, k, v))
    ke = kt.repeat_interleave(H // Hkv, dim=1)
    ve = vt.repeat_interleave(H // Hkv, dim=1)
    ot = torch.matmul(torch.softmax(torch.matmul(qt, ke.transpose(-1, -2)) * scale, dim=-1), ve)
    ot.backward(do)
    o, lse = oracle.attention_forward_gqa(q.numpy(), k.numpy(), v.numpy(), scale)
    np.testing.assert_allclose(o, ot.detach().numpy(), atol=1e-12)
    dq, dk, dv, _, _ = oracle.attention_backward_gqa(q.numpy(), k.numpy(), v.numpy(), do.numpy(), scale)
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-11)


def test_gqa_single_group_is_mha():
    rng = np.random.default_rng(3)
    q, k, v, do = (rng.standard_normal((1, 3, 5, 4)) for _ in range(4))
    a = oracle.attention_backward_gqa(q, k, v, do, 0.5)
    b = oracle.attention_backward(q, k, v, do, 0.5)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, atol=1e-14)


# ------------------------------------------------ merging key-range results

@pytest.mark.parametrize("R", [1, 2, 3, 7])
def test_combine_partials_reaches_the_full_result(R):
    """Attention over R disjoint key ranges, merged, equals attention over all keys (any split)."""
    rng = np.random.default_rng(R)
    q = rng.standard_normal((5, 8))
    k = rng.standard_normal((40, 8)) * 2.0
    v = rng.standard_normal((40, 8))
    cuts = np.sort(rng.choice(np.arange(1, 40), R - 1, replace=False)) if R > 1 else np.array([], dtype=int)
    bounds = np.concatenate([[0], cuts, [40]])
    parts = [oracle.attention_forward_2d(q, k[a:b], v[a:b], 0.7) for a, b in zip(bounds[:-1], bounds[1:])]
    o, lse = oracle.combine_partials(np.stack([p_[0] for p_ in parts]), np.stack([p_[1] for p_ in parts]))
    ro, rl = oracle.attention_forward_2d(q, k, v, 0.7)
    np.testing.assert_allclose(o, ro, atol=1e-13)
    np.testing.assert_allclose(lse, rl, atol=1e-13)


def test_combine_partials_closed_form():
    """Two parts with lse ln 1 and ln 3: weights 1/4 and 3/4, lse ln 4."""
    o, lse = oracle.combine_partials(np.array([[[2.0, 0.0]], [[6.0, 4.0]]]), np.array([[0.0], [np.log(3.0)]]))
    np.testing.assert_allclose(o, [[0.25 * 2 + 0.75 * 6, 0.75 * 4]], atol=1e-15)
    np.testing.assert_allclose(lse, [np.log(4.0)], atol=1e-15)


def test_combine_partials_large_lse_is_finite():
    """Parts whose lse are ~1e3 apart: the merge is taken relative to the largest lse."""
    o, lse = oracle.combine_partials(np.array([[[1.0]], [[3.0]]]), np.array([[1000.0], [-5.0]]))
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    np.testing.assert_allclose(o, [[1.0]], atol=1e-15)
    np.testing.assert_allclose(lse, [1000.0], atol=1e-12)
