"""The seeded input generator (synthetic_inputs.py), on CPU.

Both the oracle and the CUDA path take their inputs from it, so its recipe is
pinned here: fixed draws per seed, the Q, K, V, dO draw order, the workload
shapes, and the e4m3 values that the FP8 forward's oracle comparison uses.
"""

import numpy as np
import torch

from synthetic_inputs import E4M3_MAX, WORKLOADS, custom, dequant_f64, make_inputs, make_inputs_fp8, to_f64


def test_draws_are_fixed_by_the_seed():
    w = custom(1, 2, 33, 47, 64, "bf16")
    a = make_inputs(w, 7)
    b = make_inputs(w, 7)
    c = make_inputs(w, 8)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert not torch.equal(a[0], c[0])


def test_forward_only_draw_shares_q_k_v():
    fb = custom(1, 2, 33, 47, 64, "bf16", backward=True)
    fo = custom(1, 2, 33, 47, 64, "bf16", backward=False)
    q1, k1, v1, do1 = make_inputs(fb, 3)
    q2, k2, v2, do2 = make_inputs(fo, 3)
    assert do2 is None and do1 is not None
    for x, y in ((q1, q2), (k1, k2), (v1, v2)):
        assert torch.equal(x, y)


def test_shapes_and_dtypes_follow_the_workload():
    for name, w in WORKLOADS.items():
        if w.B * w.H * max(w.Nq, w.Nk) * w.D > (1 << 24):
            continue                          # the large workloads have the same code path
        q, k, v, do = make_inputs(w, 0)
        assert tuple(q.shape) == (w.B, w.H, w.Nq, w.D), name
        assert tuple(k.shape) == tuple(v.shape) == (w.B, w.H_kv, w.Nk, w.D), name
        assert q.dtype == k.dtype == v.dtype == w.torch_dtype, name
        assert q.is_contiguous() and k.is_contiguous() and v.is_contiguous()
        assert (do is not None) == w.backward, name


def test_e4m3_codes_decode_by_the_format_definition():
    """Every byte of e4m3 (the variant without infinities) is
    (-1)^s 2^(e-7) (1 + m/8) for exponent field e >= 1 and (-1)^s 2^-6 m/8 for
    e = 0; S.1111.111 is the only NaN.  The dequantisation that feeds the
    oracle returns exactly these values, and scaling by a descale is exact."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    got = dequant_f64(codes, 1.0)
    for b in range(256):
        s, e, m = b >> 7, (b >> 3) & 15, b & 7
        if e == 15 and m == 7:
            assert np.isnan(got[b]), b
            continue
        mag = 2.0 ** (e - 7) * (1 + m / 8) if e else 2.0 ** -6 * (m / 8)
        assert got[b] == (-mag if s else mag), b
    assert np.nanmax(got) == E4M3_MAX
    assert dequant_f64(codes, 0.375)[0x7E] == 448 * 0.375


def test_e4m3_quantisation_rounds_to_nearest_even():
    # halfway between neighbouring codes: 1.0625 lies between 1 (m = 0) and
    # 1.125 (m = 1); 1.1875 between 1.125 and 1.25 (m = 2)
    x = torch.tensor([1.0625, 1.1875, -1.0625, 0.0], dtype=torch.float32)
    got = x.to(torch.float8_e4m3fn).to(torch.float64).tolist()
    assert got == [1.0, 1.25, -1.0, 0.0]


def test_fp8_inputs_use_the_full_e4m3_range():
    w = custom(1, 2, 40, 50, 128, "bf16", backward=False)
    q8, k8, v, qd, kd = make_inputs_fp8(w, 1)
    q, k, v_ref, _ = make_inputs(custom(1, 2, 40, 50, 128, "f32", backward=False), 1)
    for x8, d, x in ((q8, qd, q), (k8, kd, k)):
        deq = dequant_f64(x8, d)
        assert np.max(np.abs(deq)) == E4M3_MAX * d      # the largest magnitude maps to 448
        assert abs(d - float(x.abs().max()) / E4M3_MAX) <= 1e-7 * d
        # every value is within half an e4m3 step (relative 2^-4) of its fp32 draw
        ref = to_f64(x)
        assert np.all(np.abs(deq - ref) <= 2.0 ** -4 * np.abs(ref) + 2.0 ** -9 * d + 1e-12)
    assert torch.equal(v, v_ref.to(torch.bfloat16))
