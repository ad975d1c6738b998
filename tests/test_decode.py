"""Split-KV decode (mea_attn_decode) against the fp64 oracle (GPU).

The library cuts the keys of each key/value head into chunks, summarises every
chunk (running max, exp-sum, unnormalised accumulator) on its own CTA and
merges the summaries in a second kernel; the oracle forms the full score
matrix per query head and applies the definition.  They share nothing but the
seeded inputs.  Shapes cover every row-count instantiation (1, 2, 4, 8 rows
per key/value head, with padded rows for 3, 5, 6), ragged final tiles and
chunks, a single key, grids where one chunk per head fills the device (no
workspace, also reached through mea_attn_fwd), and both dtypes.
"""

import numpy as np
import pytest
import torch

import oracle
from synthetic_inputs import custom, make_inputs, make_workload, to_f64
from tests._parity import BF16_O, F32_O_MAX_ABS, assert_close, assert_lse_close, to_np

pytestmark = pytest.mark.gpu


def _run(B, H, Hkv, Nq, Nk, D, dtype, seed, qk_mult=1.0):
    import exact_memory_efficient_b200 as m
    w = custom(B, H, Nq, Nk, D, dtype, backward=False, qk_mult=qk_mult, Hkv=Hkv)
    q, k, v, _ = make_inputs(w, seed)
    o, lse = m.attention_decode(q.cuda(), k.cuda(), v.cuda(), w.scale)
    assert m.mea_last_device_error() == m.MEA_OK
    ro, rl = oracle.attention_forward_gqa(to_f64(q), to_f64(k), to_f64(v), w.scale)
    what = f"{(B, H, Hkv, Nq, Nk, D, dtype)}"
    if dtype == "bf16":
        assert_close(to_np(o), ro, *BF16_O, what=f"O {what}")
    else:
        assert_close(to_np(o), ro, F32_O_MAX_ABS, what=f"O {what}")
    assert_lse_close(to_np(lse), rl, to_f64(q), np.repeat(to_f64(k), H // Hkv, axis=1), w.scale,
                     what=f"lse {what}")
    return w, o, lse


@pytest.mark.parametrize("B,H,Hkv,Nq,Nk,D", [
    (1, 8, 8, 1, 16384, 128),    # one row per head, 16K keys: the decode workload's shape
    (1, 32, 8, 1, 16384, 128),   # four rows per key/value head (groups of 4)
    (1, 6, 2, 1, 5000, 64),      # three rows: padded to four; ragged last tile
    (2, 8, 1, 1, 3001, 128),     # eight rows per head (multi-query); ragged
    (1, 8, 2, 2, 4097, 128),     # two queries x four heads = eight rows; one key past a tile
    (1, 5, 1, 1, 777, 64),       # five rows: padded to eight
    (3, 2, 2, 2, 200, 128),      # two rows; chunks of a single tile
    (1, 4, 4, 1, 1, 128),        # a single key
    (1, 2, 2, 1, 63, 64),        # one partial tile
    (1, 2, 2, 1, 65, 64),        # a full tile and one key
    (64, 8, 8, 1, 1000, 128),    # 512 key/value heads: one chunk per head, no workspace
])
def test_decode_bf16(B, H, Hkv, Nq, Nk, D):
    _run(B, H, Hkv, Nq, Nk, D, "bf16", seed=B * 1000 + H * 10 + Nq)


@pytest.mark.parametrize("B,H,Hkv,Nq,Nk,D", [
    (1, 8, 8, 1, 16384, 64),
    (1, 4, 1, 1, 3000, 32),
    (1, 6, 3, 1, 2500, 96),
    (1, 8, 2, 1, 2000, 96),      # four rows per head at D = 96: half-warps, 6 dims per lane
    (2, 8, 2, 2, 1500, 128),
    (1, 8, 4, 1, 3000, 128),     # two rows per head, fp32 rows of 512 bytes
    (1, 3, 3, 1, 1, 64),
])
def test_decode_f32(B, H, Hkv, Nq, Nk, D):
    _run(B, H, Hkv, Nq, Nk, D, "f32", seed=7 + Nk)


def test_decode_rising_scores_rescale_often():
    """Scores that grow along the keys force the running maximum past its
    2^8 slack again and again, so the rescale path runs in most tiles."""
    import exact_memory_efficient_b200 as m
    Nk, D = 4096, 128
    rng = np.random.default_rng(5)
    q = np.ones((1, 2, 1, D)) * 0.25 + rng.normal(0, 0.01, (1, 2, 1, D))
    ramp = np.linspace(-1.0, 1.0, Nk)[None, None, :, None]
    k = ramp * 4.0 + rng.normal(0, 0.01, (1, 2, Nk, D))
    v = rng.normal(0, 1, (1, 2, Nk, D))
    qt, kt, vt = (torch.tensor(x, dtype=torch.bfloat16) for x in (q, k, v))
    scale = 1.0   # scores span about +-128: many times the 2^8 slack in the base-2 domain
    o, lse = m.attention_decode(qt.cuda(), kt.cuda(), vt.cuda(), scale)
    assert m.mea_last_device_error() == m.MEA_OK
    ro, rl = oracle.attention_forward(to_f64(qt), to_f64(kt), to_f64(vt), scale)
    assert_close(to_np(o), ro, *BF16_O, what="rising scores O")
    assert_lse_close(to_np(lse), rl, to_f64(qt), to_f64(kt), scale, what="rising scores lse")


def test_decode_large_logits():
    """qk_mult 40: the softmax is nearly one-hot in every chunk."""
    _run(1, 4, 2, 1, 6000, 128, "bf16", seed=3, qk_mult=40.0)


def test_decode_workload_full_size_matches_oracle():
    """The decode workload (8 heads, one query, 16384 keys, D = 128) at full size: every output."""
    import exact_memory_efficient_b200 as m
    w = make_workload("decode_16384_bf16")
    q, k, v, _ = make_inputs(w, 0)
    o, lse = m.attention_decode(q.cuda(), k.cuda(), v.cuda(), w.scale)
    ro, rl = oracle.attention_forward(to_f64(q), to_f64(k), to_f64(v), w.scale)
    assert_close(to_np(o), ro, *BF16_O, what="decode workload O")
    assert_lse_close(to_np(lse), rl, to_f64(q), to_f64(k), w.scale, what="decode workload lse")


def test_decode_deterministic_and_equal_to_forward_where_unsplit():
    """No atomics: two calls give identical bits.  With one chunk per head the
    decode entry and mea_attn_fwd run the same kernel."""
    import exact_memory_efficient_b200 as m
    w = custom(1, 8, 1, 16384, 128, "bf16", backward=False)
    q, k, v = (x.cuda() for x in make_inputs(w, 9)[:3])
    o1, l1 = m.attention_decode(q, k, v, w.scale)
    o2, l2 = m.attention_decode(q, k, v, w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    w2 = custom(64, 8, 1, 1000, 128, "bf16", backward=False)
    qq, kk, vv, _ = make_inputs(w2, 10)
    qq, kk, vv = qq.cuda(), kk.cuda(), vv.cuda()
    assert m.mea_attn_decode_workspace_size(64, 8, 8, 1, 1000, 128) == 0
    o3, l3 = m.attention_decode(qq, kk, vv, w2.scale)
    o4, l4 = m.attention_forward(qq, kk, vv, w2.scale)
    torch.cuda.synchronize()
    assert torch.equal(o3, o4) and torch.equal(l3, l4)


def test_decode_many_rows_is_the_forward():
    """More than 8 rows per key/value head: the call is mea_attn_fwd_gqa (no workspace)."""
    import exact_memory_efficient_b200 as m
    assert m.mea_attn_decode_workspace_size(1, 16, 1, 1, 4096, 128) == 0
    w = custom(1, 16, 1, 4096, 128, "bf16", backward=False, Hkv=1)
    q, k, v, _ = (x.cuda() if x is not None else None for x in make_inputs(w, 12))
    o1, l1 = m.attention_decode(q, k, v, w.scale)
    o2, l2 = m.attention_forward(q, k, v, w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_workspace_errors():
    import exact_memory_efficient_b200 as m
    w = custom(1, 8, 1, 16384, 128, "bf16", backward=False)
    q, k, v, _ = (x.cuda() if x is not None else None for x in make_inputs(w, 13))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    n = m.mea_attn_decode_workspace_size(1, 8, 8, 1, 16384, 128)
    assert n > 0
    with pytest.raises(m.MeaError) as e:
        m.mea_attn_decode(q, k, v, o, lse, w.scale, None)
    assert e.value.status == m.MEA_ERR_WORKSPACE
    small = torch.empty(n - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(m.MeaError) as e:
        m.mea_attn_decode(q, k, v, o, lse, w.scale, small)
    assert e.value.status == m.MEA_ERR_WORKSPACE
    big = torch.empty(n + 64, dtype=torch.uint8, device="cuda")
    with pytest.raises(m.MeaError) as e:
        m.mea_attn_decode(q, k, v, o, lse, w.scale, big[8:])
    assert e.value.status == m.MEA_ERR_MISALIGNED
    # a workspace holding garbage is fine: it is scratch
    big.fill_(0xFF)
    m.mea_attn_decode(q, k, v, o, lse, w.scale, big)
    ro, rl = oracle.attention_forward(*(to_f64(x.cpu()) for x in (q, k, v)), w.scale)
    assert_close(to_np(o), ro, *BF16_O, what="garbage workspace")


def test_decode_in_cuda_graph():
    """Both decode kernels are launched with programmatic stream serialisation; a CUDA graph
    captures them (and a backward in the same graph) and replays them with new inputs."""
    import exact_memory_efficient_b200 as m
    w = custom(1, 8, 1, 5000, 128, "bf16", backward=False, Hkv=2)
    q, k, v, _ = (x.cuda() if x is not None else None for x in make_inputs(w, 40))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    n = m.mea_attn_decode_workspace_size(1, 8, 2, 1, 5000, 128)
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        m.mea_attn_decode(q, k, v, o, lse, w.scale, ws, stream=s)   # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        m.mea_attn_decode(q, k, v, o, lse, w.scale, ws)
    for seed in (41, 42):
        q2, k2, v2, _ = make_inputs(w, seed)
        q.copy_(q2.cuda())
        k.copy_(k2.cuda())
        v.copy_(v2.cuda())
        g.replay()
        torch.cuda.synchronize()
        ro, rl = oracle.attention_forward_gqa(to_f64(q2), to_f64(k2), to_f64(v2), w.scale)
        assert_close(to_np(o), ro, *BF16_O, what=f"graph replay O seed {seed}")
        assert_lse_close(to_np(lse), rl, to_f64(q2), np.repeat(to_f64(k2), 4, axis=1), w.scale,
                         what=f"graph replay lse seed {seed}")
    assert m.mea_last_device_error() == m.MEA_OK
