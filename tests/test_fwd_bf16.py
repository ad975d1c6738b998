"""bf16 tcgen05 forward against the fp64 oracle, through the C ABI (GPU).

Full element-by-element comparison on shapes the oracle finishes in seconds
(several 128-row tiles and ragged tails), and sampled rows at the full
workload sizes, launched exactly as the bench launches them.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from synthetic_inputs import custom, make_inputs, make_workload, to_f64
from tests._parity import BF16_GRAD, BF16_O, assert_close, assert_lse_close, to_np

pytestmark = pytest.mark.gpu


def gpu_fwd(q, k, v, scale):
    import exact_memory_efficient_b200 as m
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    o, lse = m.attention_forward(qd, kd, vd, scale)
    assert m.mea_last_device_error() == m.MEA_OK
    return o, lse


def full_check(q, k, v, scale, what):
    o, lse = gpu_fwd(q, k, v, scale)
    q64, k64, v64 = to_f64(q), to_f64(k), to_f64(v)
    o_ref, lse_ref = oracle.attention_forward(q64, k64, v64, scale)
    assert_close(to_np(o), o_ref, *BF16_O, what=f"O {what}")
    assert_lse_close(to_np(lse), lse_ref, q64, k64, scale, what=f"lse {what}")


@pytest.mark.parametrize("B,H,Nq,Nk,D", [
    (1, 1, 128, 128, 64),
    (1, 1, 256, 384, 128),
    (2, 3, 300, 700, 64),     # ragged query and key tails, several tiles
    (1, 2, 513, 257, 128),    # odd tile counts
    (1, 1, 1, 1, 64),         # one row, one key
    (1, 1, 1, 1000, 128),     # single query (decode-shaped)
    (2, 2, 77, 5, 128),       # fewer keys than one tile
    (1, 1, 1000, 1, 64),      # one key: O = V_0
])
def test_shapes_full(B, H, Nq, Nk, D):
    w = custom(B, H, Nq, Nk, D, "bf16", backward=False)
    q, k, v, _ = make_inputs(w, 11)
    full_check(q, k, v, w.scale, f"{(B, H, Nq, Nk, D)}")


@pytest.mark.parametrize("B,H,Nq,Nk,D", [
    (1, 8, 1, 16384, 128),    # decode: 16 chunks of 1024 keys over a cluster, merged in distributed smem
    (2, 4, 3, 5000, 64),      # 16 chunks of 384 keys: one of 8 keys, the last two empty
    (1, 2, 200, 2049, 128),   # 8 chunks of 384 keys: one of 129 keys, the last two empty
    (1, 1, 1, 8193, 128),     # 16 chunks of 640 keys: one of 513 keys, the last three empty
    (1, 3, 257, 1024, 64),    # two query tiles per CTA, 4 chunks of 256 keys
])
def test_decode_key_split(B, H, Nq, Nk, D):
    w = custom(B, H, Nq, Nk, D, "bf16", backward=False)
    q, k, v, _ = make_inputs(w, 17)
    full_check(q, k, v, w.scale, f"{(B, H, Nq, Nk, D)}")


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_encoder_512_full(seed):
    w = make_workload("encoder_512_bf16")
    q, k, v, _ = make_inputs(w, seed)
    full_check(q, k, v, w.scale, f"encoder_512 seed {seed}")


@pytest.mark.parametrize("name", ["mha_4k_bf16", "long_256_bf16", "long_1024_bf16", "long_4096_bf16",
                                  "long_16384_bf16"])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_workloads_sampled(name, seed):
    """Full-size launch; oracle on sampled (batch, head, row) triples."""
    w = make_workload(name)
    q, k, v, _ = make_inputs(w, seed)
    o, lse = gpu_fwd(q, k, v, w.scale)
    o, lse = to_np(o), to_np(lse)
    rng = np.random.default_rng(seed)
    heads = {(0, 0), (w.B - 1, w.H - 1), (int(rng.integers(w.B)), int(rng.integers(w.H)))}
    n_rows = min(w.Nq, 48)
    for b, h in sorted(heads):
        rows = np.unique(np.concatenate([[0, w.Nq - 1], rng.choice(w.Nq, n_rows, replace=False)]))
        q64, k64, v64 = to_f64(q[b, h]), to_f64(k[b, h]), to_f64(v[b, h])
        o_ref, lse_ref = oracle.attention_forward_rows(q64, k64, v64, w.scale, rows)
        assert_close(o[b, h, rows], o_ref, *BF16_O, what=f"O {name} s{seed} ({b},{h})")
        assert_lse_close(lse[b, h, rows], lse_ref, q64[rows], k64, w.scale, what=f"lse {name} ({b},{h})")


def _grid(shape, gen, lo=-16, hi=16):
    """Values on the 1/8 grid in [-2, 2]: exactly representable in bf16, also after adding small integers."""
    return (torch.randint(lo, hi + 1, shape, generator=gen).float() / 8).to(torch.bfloat16)


def test_shift_invariance():
    """K -> K + 1 u^T: O unchanged, lse shifts by scale q.u (inputs exact in bf16)."""
    g = torch.Generator().manual_seed(21)
    Nq, Nk, D = 200, 300, 64
    q, k = _grid((1, 2, Nq, D), g), _grid((1, 2, Nk, D), g)
    v = torch.randn(1, 2, Nk, D, generator=g).to(torch.bfloat16)
    u = torch.randint(-2, 3, (D,), generator=g).float()
    k2 = (k.float() + u).to(torch.bfloat16)
    assert torch.equal(k2.float(), k.float() + u)  # exact
    o1, l1 = gpu_fwd(q, k, v, 0.125)
    o2, l2 = gpu_fwd(q, k2, v, 0.125)
    o1, o2, l1, l2 = to_np(o1), to_np(o2), to_np(l1), to_np(l2)
    np.testing.assert_allclose(o2, o1, atol=2e-2)
    shift = 0.125 * (to_f64(q) @ u.double().numpy())
    np.testing.assert_allclose(l2 - l1, shift, atol=2e-3)


def test_all_keys_equal():
    g = torch.Generator().manual_seed(22)
    Nq, Nk, D = 130, 1000, 128
    q = torch.randn(1, 1, Nq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 1, 1, D, generator=g).to(torch.bfloat16).expand(1, 1, Nk, D).contiguous()
    v = torch.randn(1, 1, Nk, D, generator=g).to(torch.bfloat16)
    o, lse = gpu_fwd(q, k, v, 1 / math.sqrt(D))
    vbar = to_f64(v)[0, 0].mean(axis=0)
    np.testing.assert_allclose(to_np(o)[0, 0], np.tile(vbar, (Nq, 1)), atol=2e-2)
    expect = (to_f64(q)[0, 0] @ to_f64(k)[0, 0, 0]) / math.sqrt(D) + math.log(Nk)
    np.testing.assert_allclose(to_np(lse)[0, 0], expect, atol=2e-3)


def test_dominant_key_and_large_logits():
    """One-hot keys scaled so one score beats the rest by > 50 (logits ~1e3)."""
    D, Nk = 64, 64
    a = 64.0
    k = (torch.eye(D) * a).reshape(1, 1, Nk, D).to(torch.bfloat16)
    perm = torch.tensor([5, 0, 63, 17, 17, 40] * 40)
    q = (torch.eye(D)[perm] * 128.0).reshape(1, 1, -1, D).to(torch.bfloat16)  # score 64*128/8 = 1024
    v = torch.randn(1, 1, Nk, D, generator=torch.Generator().manual_seed(23)).to(torch.bfloat16)
    o, lse = gpu_fwd(q, k, v, 0.125)
    np.testing.assert_allclose(to_np(o)[0, 0], to_f64(v)[0, 0][perm.numpy()], atol=1e-6)
    np.testing.assert_allclose(to_np(lse)[0, 0], 1024.0, atol=1e-3)


def test_deterministic():
    w = custom(1, 4, 1000, 1000, 128, "bf16", backward=False)
    q, k, v, _ = make_inputs(w, 3)
    a, la = gpu_fwd(q, k, v, w.scale)
    b, lb = gpu_fwd(q, k, v, w.scale)
    assert torch.equal(a, b) and torch.equal(la, lb)


@pytest.mark.parametrize("shape", [(1, 2, 300, 400, 64), (1, 1, 1, 5000, 128), (1, 2, 129, 700, 128)])
def test_single_tile_split_repeat(shape):
    """CTAs whose rows fit in one query tile split their keys over both TMEM slots and merge the
    two summaries; repeat forward + backward 20 times against the oracle (a race would show as a
    sporadic wrong or non-finite value)."""
    import exact_memory_efficient_b200 as m
    w = custom(*shape, "bf16")
    q, k, v, do = make_inputs(w, 11)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    rq, rk, rv, ro, rl = oracle.attention_backward(to_f64(q), to_f64(k), to_f64(v), to_f64(do), w.scale)
    for _ in range(20):
        o, lse = m.attention_forward(qd, kd, vd, w.scale)
        dq, dk, dv = m.attention_backward(qd, kd, vd, o, lse, dod, w.scale)
        assert m.mea_last_device_error() == m.MEA_OK
        assert_close(to_np(o), ro, *BF16_O, what=f"O {shape}")
        assert_lse_close(to_np(lse), rl, to_f64(q), to_f64(k), w.scale, what=f"lse {shape}")
        assert_close(to_np(dq), rq, *BF16_GRAD, what=f"dQ {shape}")
        assert_close(to_np(dk), rk, *BF16_GRAD, what=f"dK {shape}")
        assert_close(to_np(dv), rv, *BF16_GRAD, what=f"dV {shape}")


@pytest.mark.parametrize("B,H,Nq,Nk,D", [
    (1, 2, 256, 384, 128),    # one CTA per head, three full key tiles
    (2, 2, 512, 700, 128),    # ragged last key tile: keys 64..127 of it partly missing
    (1, 3, 768, 65, 128),     # one key tile, one key past its first half
    (1, 1, 256, 1, 128),      # one key
    (1, 2, 1024, 1000, 128),  # four CTAs per head
])
def test_full_tile_pairs(B, H, Nq, Nk, D):
    """Nq a multiple of 256 at D = 128: every CTA holds two full query tiles."""
    w = custom(B, H, Nq, Nk, D, "bf16", backward=False)
    q, k, v, _ = make_inputs(w, 12)
    full_check(q, k, v, w.scale, f"tile pairs {(B, H, Nq, Nk, D)}")


def test_rising_scores_rescale_often():
    """Scores that grow along the keys make the reference maximum move in most key tiles, so O is
    rescaled in place many times in both query tiles of every CTA."""
    Nq, Nk, D = 512, 2048, 128
    rng = np.random.default_rng(8)
    q = np.ones((1, 2, Nq, D)) * 0.25 + rng.normal(0, 0.01, (1, 2, Nq, D))
    ramp = np.linspace(-1.0, 1.0, Nk)[None, None, :, None]
    k = ramp * 4.0 + rng.normal(0, 0.01, (1, 2, Nk, D))
    v = rng.normal(0, 1, (1, 2, Nk, D))
    qt, kt, vt = (torch.tensor(x, dtype=torch.bfloat16) for x in (q, k, v))
    full_check(qt, kt, vt, 1.0, "rising scores")


@pytest.mark.parametrize("D", [64, 128])
def test_rising_scores_many_items(D):
    """The rising-score construction over 160 heads (320 query-tile pairs, so persistent CTAs walk
    two or three items each): the reference maximum moves in most key tiles of every item, and
    each item starts from a fresh maximum while the previous item's last tile is still in flight."""
    B, H, Nq, Nk = 40, 4, 512, 1000
    rng = np.random.default_rng(9)
    q = np.ones((B, H, Nq, D)) * 0.25 + rng.normal(0, 0.01, (B, H, Nq, D))
    ramp = np.linspace(-1.0, 1.0, Nk)[None, None, :, None] * rng.choice([-1.0, 1.0], (B, H, 1, 1))
    k = ramp * (4.0 * 128 / D) + rng.normal(0, 0.01, (B, H, Nk, D))
    v = rng.normal(0, 1, (B, H, Nk, D))
    qt, kt, vt = (torch.tensor(x, dtype=torch.bfloat16) for x in (q, k, v))
    full_check(qt, kt, vt, 1.0 if D == 128 else 0.5, f"rising scores, many items, D={D}")


@pytest.mark.parametrize("B,H,Nq,Nk,D", [
    (1, 2, 300, 700, 128),    # ragged query tail: the last CTA holds one tile
    (1, 2, 512, 700, 128),    # full tile pairs
    (1, 1, 77, 300, 64),
    (1, 2, 1, 2000, 128),     # decode-shaped: split-KV kernel, scale folded into q
])
def test_negative_scale(B, H, Nq, Nk, D):
    """softmax(scale QK^T) with scale < 0: the block maximum of the scaled scores is the raw minimum."""
    import exact_memory_efficient_b200 as m
    w = custom(B, H, Nq, Nk, D, "bf16", backward=True)
    q, k, v, do = make_inputs(w, 13)
    scale = -w.scale
    full_check(q, k, v, scale, f"negative scale {(B, H, Nq, Nk, D)}")
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = m.attention_forward(qd, kd, vd, scale)
    dq, dk, dv = m.attention_backward(qd, kd, vd, o, lse, dod, scale)
    assert m.mea_last_device_error() == m.MEA_OK
    rq, rk, rv, _, _ = oracle.attention_backward(to_f64(q), to_f64(k), to_f64(v), to_f64(do), scale)
    for name, g_, r_ in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
        assert_close(to_np(g_), r_, *BF16_GRAD, what=f"negative scale {name}")


@pytest.mark.parametrize("B,H,Nq,Nk,D", [
    (16, 16, 512, 77, 128),   # 512 items over at most one CTA per SM: several items per CTA, one key tile each
    (8, 16, 256, 200, 64),    # two key tiles, the second ragged
    (4, 20, 768, 333, 128),   # three query-tile pairs per head, three key tiles
    (2, 3, 256, 4096, 64),    # the longest key range that takes the persistent CTAs at D = 64
    (3, 5, 512, 2048, 128),   # and at D = 128
    # Item lists with single query tiles (the two slots of a CTA split the keys) for the pairs
    # of a partial last round, on a part with 148 SMs:
    (16, 16, 512, 333, 64),   # 512 pairs: three full rounds, the last 68 pairs as 136 single tiles (3 key tiles: 2 + 1)
    (16, 16, 512, 700, 128),  # the same at D = 128 with 6 key tiles (the last ragged)
    (2, 37, 256, 500, 64),    # 74 pairs: all as 148 single tiles, one round
    (1, 16, 1024, 1024, 128), # 64 pairs: 128 single tiles with 8 key tiles each
    (1, 16, 256, 256, 128),   # 16 pairs: 32 single tiles with 2 key tiles each
    # Past the plain key limit (2048 at D = 128, 4096 at D = 64) the persistent CTAs are used
    # only when the item list has single tiles:
    (2, 37, 256, 3000, 128),  # 74 pairs as 148 single tiles, 24 key tiles (the last ragged)
    (2, 37, 256, 6000, 64),   # the same at D = 64 with 47 key tiles
])
def test_persistent_items_full(B, H, Nq, Nk, D):
    """Short key ranges with Nq a multiple of 256: CTAs walk several (head, tile pair) items,
    reusing their barriers, TMEM and K/V ring from one item to the next.  Where the pairs would
    leave most CTAs idle in a last round, those pairs run as single query tiles whose two
    slots take alternate key tiles and merge their summaries with the two-block formulas."""
    w = custom(B, H, Nq, Nk, D, "bf16", backward=False)
    q, k, v, _ = make_inputs(w, 16)
    full_check(q, k, v, w.scale, f"persistent {(B, H, Nq, Nk, D)}")
    full_check(q, k, v, -w.scale, f"persistent negative scale {(B, H, Nq, Nk, D)}")
