"""Key (sequence) split: results over disjoint key ranges merged by mea_attn_combine (GPU).

On one GPU the ranks of a key split are emulated as R key ranges processed one
after another; every launch is an ordinary independent launch (nothing waits
on another rank).  The all-gather of the parts is the list of R local buffers;
the all-reduce of the backward's fp32 dQ accumulators is a sum over the R
workspaces.  The oracle computes attention over all keys at once.
"""

import numpy as np
import pytest
import torch

import oracle
from synthetic_inputs import custom, make_inputs, to_f64
from tests._parity import BF16_GRAD, BF16_O, F32_O_MAX_ABS, assert_close, assert_lse_close, to_np

pytestmark = pytest.mark.gpu


def ranges(Nk, R, seed):
    rng = np.random.default_rng(seed)
    cuts = np.sort(rng.choice(np.arange(1, Nk), R - 1, replace=False)) if R > 1 else np.array([], dtype=int)
    b = np.concatenate([[0], cuts, [Nk]])
    return [(int(x), int(y)) for x, y in zip(b[:-1], b[1:])]


def split_forward(qd, kd, vd, scale, rs):
    import exact_memory_efficient_b200 as m
    parts = [m.attention_forward(qd, kd[:, :, a:b].contiguous(), vd[:, :, a:b].contiguous(), scale) for a, b in rs]
    o = torch.empty_like(qd)
    lse = torch.empty(qd.shape[:3], dtype=torch.float32, device=qd.device)
    m.mea_attn_combine([p[0] for p in parts], [p[1] for p in parts], o, lse)
    return o, lse


@pytest.mark.parametrize("dtype,R", [("bf16", 1), ("bf16", 2), ("bf16", 5), ("bf16", 16), ("f32", 3)])
def test_combine_matches_oracle_merge(dtype, R):
    """The merge alone, on random parts (lse spread over +-30 so the weights span many orders)."""
    import exact_memory_efficient_b200 as m
    g = torch.Generator().manual_seed(R)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    o_parts = [torch.randn(2, 3, 70, 64, generator=g).to(tdt) for _ in range(R)]
    lse_parts = [(torch.rand(2, 3, 70, generator=g) * 60 - 30) for _ in range(R)]
    o = torch.empty(2, 3, 70, 64, dtype=tdt, device="cuda")
    lse = torch.empty(2, 3, 70, device="cuda")
    m.mea_attn_combine([x.cuda() for x in o_parts], [x.cuda() for x in lse_parts], o, lse)
    assert m.mea_last_device_error() == m.MEA_OK
    ro, rl = oracle.combine_partials(np.stack([to_f64(x) for x in o_parts]), np.stack([to_f64(x) for x in lse_parts]))
    tol = BF16_O if dtype == "bf16" else (F32_O_MAX_ABS, None)
    assert_close(to_np(o), ro, *tol, what=f"combine {dtype} R={R}")
    assert float(np.abs(to_np(lse) - rl).max()) <= 1e-5 * max(1.0, float(np.abs(rl).max()))


def test_combine_skips_parts_without_keys():
    """A part with lse = -inf (an empty key range) contributes nothing, even if its o holds NaN."""
    import exact_memory_efficient_b200 as m
    a = torch.randn(1, 1, 9, 64).to(torch.bfloat16).cuda()
    nan = torch.full_like(a, float("nan"))
    la = torch.randn(1, 1, 9).cuda()
    ninf = torch.full_like(la, float("-inf"))
    o = torch.empty_like(a)
    lse = torch.empty_like(la)
    m.mea_attn_combine([a, nan], [la, ninf], o, lse)
    torch.cuda.synchronize()
    assert torch.equal(o, a) and torch.allclose(lse, la)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_combine_row_without_any_keys(dtype):
    """Rows whose parts are all empty (lse = -inf everywhere) have no keys: the empty sum gives
    lse = ln 0 = -inf and o = 0; the other rows merge as usual."""
    import exact_memory_efficient_b200 as m
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    g = torch.Generator().manual_seed(5)
    o_parts = [torch.randn(1, 2, 9, 64, generator=g).to(tdt) for _ in range(3)]
    lse_parts = [torch.randn(1, 2, 9, generator=g) for _ in range(3)]
    empty_rows = [0, 4, 8]
    for lp in lse_parts:
        lp[0, 1, empty_rows] = float("-inf")
    o_parts[2][0, 1, empty_rows] = float("nan")    # an empty part's o is never read into the result
    o = torch.empty(1, 2, 9, 64, dtype=tdt, device="cuda")
    lse = torch.empty(1, 2, 9, device="cuda")
    m.mea_attn_combine([x.cuda() for x in o_parts], [x.cuda() for x in lse_parts], o, lse)
    assert m.mea_last_device_error() == m.MEA_OK
    o, lse = to_np(o), to_np(lse)
    assert np.all(o[0, 1, empty_rows] == 0.0) and np.all(np.isneginf(lse[0, 1, empty_rows]))
    keep = [i for i in range(9) if i not in empty_rows]
    with np.errstate(invalid="ignore"):   # the oracle's merge leaves the keyless rows undefined (compared apart)
        ro, rl = oracle.combine_partials(np.stack([to_f64(x) for x in o_parts]),
                                         np.stack([to_f64(x) for x in lse_parts]))
    tol = BF16_O if dtype == "bf16" else (F32_O_MAX_ABS, None)
    assert_close(o[0, 0], ro[0, 0], *tol, what="rows with keys, head 0")
    assert_close(o[0, 1, keep], ro[0, 1, keep], *tol, what="rows with keys, head 1")
    assert float(np.abs(lse[0, 1, keep] - rl[0, 1, keep]).max()) <= 1e-5 * max(1.0, float(np.abs(rl).max()))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_keysplit_rank_without_keys(dtype):
    """Fewer keys than ranks: an emulated rank whose key range is empty runs no kernel over zero
    keys, contributes o = 0, lse = -inf to the merge and a zero dQ partial to the sum, and (bf16)
    finalises the summed dQ accumulator itself."""
    from exact_memory_efficient_b200.keysplit import CudaOps
    import exact_memory_efficient_b200 as m
    w = custom(1, 2, 7, 3, 64, dtype)            # few rows, so that the gradients stay of order one
    q, k, v, do = make_inputs(w, 25)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    ops = CudaOps()
    rs = [(0, 0), (0, 1), (1, 3), (3, 3)]       # four ranks over three keys: two ranks hold none
    o_parts, lse_parts = [], []
    for a, b in rs:
        if b == a:   # what attention_forward_keysplit contributes for an empty range
            o_parts.append(torch.zeros_like(qd))
            lse_parts.append(torch.full(qd.shape[:3], float("-inf"), device="cuda"))
        else:
            o_r, l_r = ops.forward(qd, kd[:, :, a:b].contiguous(), vd[:, :, a:b].contiguous(), w.scale)
            o_parts.append(o_r)
            lse_parts.append(l_r)
    o, lse = ops.combine(o_parts, lse_parts)
    parts = [ops.backward_partial(qd, kd[:, :, a:b].contiguous(), vd[:, :, a:b].contiguous(), o, lse, dod, w.scale)
             for a, b in rs]
    total = sum(p[0] for p in parts)             # the all-reduce
    for p in parts:
        p[0].copy_(total)
    dqs = [p[3](p[0]) for p in parts]
    assert m.mea_last_device_error() == m.MEA_OK
    rq, rk, rv, ro, rl = oracle.attention_backward(to_f64(q), to_f64(k), to_f64(v), to_f64(do), w.scale)
    if dtype == "bf16":
        assert_close(to_np(o), ro, *BF16_O, what="O")
        for r, dq in enumerate(dqs):         # every rank, the empty ones too, ends with the full dq
            assert_close(to_np(dq), rq, *BF16_GRAD, what=f"dQ rank {r}")
        assert_close(to_np(torch.cat([p[1] for p in parts], dim=2)), rk, *BF16_GRAD, what="dK")
        assert_close(to_np(torch.cat([p[2] for p in parts], dim=2)), rv, *BF16_GRAD, what="dV")
    else:
        assert_close(to_np(o), ro, F32_O_MAX_ABS, what="fp32 O")
        for r, dq in enumerate(dqs):
            assert_close(to_np(dq), rq, F32_O_MAX_ABS, what=f"fp32 dQ rank {r}")
        assert_close(to_np(torch.cat([p[1] for p in parts], dim=2)), rk, F32_O_MAX_ABS, what="fp32 dK")
        assert_close(to_np(torch.cat([p[2] for p in parts], dim=2)), rv, F32_O_MAX_ABS, what="fp32 dV")
    assert_lse_close(to_np(lse), rl, to_f64(q), to_f64(k), w.scale)


@pytest.mark.parametrize("B,H,Nq,Nk,D,R", [
    (1, 2, 300, 1000, 128, 2),
    (2, 3, 129, 777, 64, 3),
    (1, 8, 1, 16384, 128, 8),     # decode: eight ranges of 2048 keys
    (1, 4, 500, 4096, 128, 4),
])
def test_split_forward_bf16(B, H, Nq, Nk, D, R):
    w = custom(B, H, Nq, Nk, D, "bf16", backward=False)
    q, k, v, _ = make_inputs(w, 21)
    o, lse = split_forward(q.cuda(), k.cuda(), v.cuda(), w.scale, ranges(Nk, R, 7))
    ro, rl = oracle.attention_forward(to_f64(q), to_f64(k), to_f64(v), w.scale)
    assert_close(to_np(o), ro, *BF16_O, what=f"split O {(B, H, Nq, Nk, D, R)}")
    assert_lse_close(to_np(lse), rl, to_f64(q), to_f64(k), w.scale, what="split lse")


def test_split_forward_f32():
    w = custom(1, 4, 3, 6000, 64, "f32", backward=False)
    q, k, v, _ = make_inputs(w, 22)
    o, lse = split_forward(q.cuda(), k.cuda(), v.cuda(), w.scale, ranges(6000, 3, 8))
    ro, rl = oracle.attention_forward(to_f64(q), to_f64(k), to_f64(v), w.scale)
    assert_close(to_np(o), ro, F32_O_MAX_ABS, what="split fp32 O")
    assert_lse_close(to_np(lse), rl, to_f64(q), to_f64(k), w.scale, what="split fp32 lse")


@pytest.mark.parametrize("B,H,Nq,Nk,D,R", [(1, 2, 300, 1000, 128, 2), (1, 3, 257, 900, 64, 3)])
def test_split_backward_bf16(B, H, Nq, Nk, D, R):
    """Backward of a key split: each range recomputes P from the merged lse, the fp32 dQ
    accumulators of the ranges are summed before the finalize phase, dk and dv stay local."""
    import exact_memory_efficient_b200 as m
    w = custom(B, H, Nq, Nk, D, "bf16")
    q, k, v, do = make_inputs(w, 23)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    rs = ranges(Nk, R, 9)
    o, lse = split_forward(qd, kd, vd, w.scale, rs)
    wsb = m.mea_attn_bwd_workspace_size(B, H, Nq, Nk, D)
    acc_elems = B * H * Nq * D
    dq = torch.empty_like(qd)
    dks, dvs, wss = [], [], []
    for a, b in rs:
        ks, vs = kd[:, :, a:b].contiguous(), vd[:, :, a:b].contiguous()
        dk, dv = torch.empty_like(ks), torch.empty_like(vs)
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        for ph in (m.MEA_BWD_PREPROCESS, m.MEA_BWD_MAIN):
            m.mea_attn_bwd_phase(ph, qd, ks, vs, o, lse, dod, dq, dk, dv, w.scale, ws)
        dks.append(dk)
        dvs.append(dv)
        wss.append(ws)
    # the all-reduce of the dQ accumulators (fp32, at the start of each workspace)
    acc0 = wss[0][:acc_elems * 4].view(torch.float32)
    for ws in wss[1:]:
        acc0 += ws[:acc_elems * 4].view(torch.float32)
    m.mea_attn_bwd_phase(m.MEA_BWD_FINALIZE, qd, kd[:, :, rs[0][0]:rs[0][1]].contiguous(),
                         vd[:, :, rs[0][0]:rs[0][1]].contiguous(), o, lse, dod, dq, dks[0], dvs[0], w.scale, wss[0])
    assert m.mea_last_device_error() == m.MEA_OK
    rq, rk, rv, _, _ = oracle.attention_backward(to_f64(q), to_f64(k), to_f64(v), to_f64(do), w.scale)
    assert_close(to_np(dq), rq, *BF16_GRAD, what="split dQ")
    assert_close(to_np(torch.cat(dks, dim=2)), rk, *BF16_GRAD, what="split dK")
    assert_close(to_np(torch.cat(dvs, dim=2)), rv, *BF16_GRAD, what="split dV")


@pytest.mark.parametrize("dtype,B,H,Nq,Nk,D,q_cuts,k_cuts", [
    ("bf16", 1, 2, 300, 1000, 128, [0, 128, 300], [0, 333, 700, 1000]),
    ("bf16", 2, 1, 257, 513, 64, [0, 257], [0, 1, 200, 513]),      # a one-key range
    ("f32", 1, 2, 120, 400, 64, [0, 70, 120], [0, 150, 400]),
])
def test_accumulating_backward(dtype, B, H, Nq, Nk, D, q_cuts, k_cuts):
    """mea_attn_bwd_accum over every (query range, key range) pair with the merged o, lse: the fp32
    sums, converted by mea_attn_accum_convert, are the full gradients (contributions of disjoint
    ranges add); the sums start at zero and stay fp32 across the calls."""
    import exact_memory_efficient_b200 as m
    w = custom(B, H, Nq, Nk, D, dtype)
    q, k, v, do = make_inputs(w, 27)
    qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
    o, lse = m.attention_forward(qd, kd, vd, w.scale)
    dq_acc = torch.zeros(qd.shape, dtype=torch.float32, device="cuda")
    dk_acc = torch.zeros(kd.shape, dtype=torch.float32, device="cuda")
    dv_acc = torch.zeros(vd.shape, dtype=torch.float32, device="cuda")
    for qa, qb in zip(q_cuts[:-1], q_cuts[1:]):
        qs = slice(qa, qb)
        q_r, o_r, l_r, do_r = (x[:, :, qs].contiguous() for x in (qd, o, lse, dod))
        dq_r = torch.zeros(q_r.shape, dtype=torch.float32, device="cuda")
        for ka, kb in zip(k_cuts[:-1], k_cuts[1:]):
            ks = slice(ka, kb)
            k_r, v_r = kd[:, :, ks].contiguous(), vd[:, :, ks].contiguous()
            dk_r, dv_r = dk_acc[:, :, ks].contiguous(), dv_acc[:, :, ks].contiguous()
            ws = torch.empty(m.mea_attn_bwd_accum_workspace_size(B, H, qb - qa, kb - ka, D, qd.dtype),
                             dtype=torch.uint8, device="cuda")
            m.mea_attn_bwd_accum(q_r, k_r, v_r, o_r, l_r, do_r, dq_r, dk_r, dv_r, w.scale, ws)
            dk_acc[:, :, ks] = dk_r      # the sums of a key range travel on to the next query range
            dv_acc[:, :, ks] = dv_r
        dq_acc[:, :, qs] = dq_r
    grads = []
    for acc, mul, like in ((dq_acc, w.scale, qd), (dk_acc, w.scale, kd), (dv_acc, 1.0, vd)):
        out = torch.empty_like(like)
        m.mea_attn_accum_convert(acc, out, mul)
        grads.append(out)
    assert m.mea_last_device_error() == m.MEA_OK
    rq, rk, rv, _, _ = oracle.attention_backward(to_f64(q), to_f64(k), to_f64(v), to_f64(do), w.scale)
    tol = BF16_GRAD if dtype == "bf16" else (F32_O_MAX_ABS, 1e-5)
    for name, g_, r_ in (("dQ", grads[0], rq), ("dK", grads[1], rk), ("dV", grads[2], rv)):
        assert_close(to_np(g_), r_, *tol, what=f"accumulated {name}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_keysplit_module_one_rank_nccl(dtype):
    """The library's own key-split path (exact_memory_efficient_b200.keysplit with its CUDA ops)
    in a one-rank NCCL group: the gather and all-reduce are trivial, every kernel and the
    accumulator hand-off are the real ones."""
    import socket
    import torch.distributed as dist
    from exact_memory_efficient_b200.keysplit import attention_backward_keysplit, attention_forward_keysplit
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        w = custom(1, 2, 200, 700, 64, dtype)
        q, k, v, do = make_inputs(w, 24)
        qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
        o, lse = attention_forward_keysplit(qd, kd, vd, w.scale)
        dq, dk, dv = attention_backward_keysplit(qd, kd, vd, o, lse, dod, w.scale)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    rq, rk, rv, ro, rl = oracle.attention_backward(to_f64(q), to_f64(k), to_f64(v), to_f64(do), w.scale)
    if dtype == "bf16":
        assert_close(to_np(o), ro, *BF16_O, what="keysplit O")
        for name, g_, r_ in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
            assert_close(to_np(g_), r_, *BF16_GRAD, what=f"keysplit {name}")
    else:
        assert_close(to_np(o), ro, F32_O_MAX_ABS, what="keysplit fp32 O")
        for name, g_, r_ in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
            assert_close(to_np(g_), r_, F32_O_MAX_ABS, what=f"keysplit fp32 {name}")
