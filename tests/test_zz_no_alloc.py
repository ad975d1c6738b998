"""The no-allocation backward entry point, through the C ABI (GPU).

mea_attn_bwd_noalloc serves callers that cannot allocate device memory (a
plugin whose host application owns the memory budget, code with memory fixed
at start-up, code without an allocator handle): its scratch is a static device
array inside the library instead of a caller workspace.  This file is
collected last so that a run stopping at the first failure has already run
every other test; it also passes on its own in a fresh process.
"""

import ctypes

import pytest
import torch

import oracle
from synthetic_inputs import custom, make_inputs, to_f64
from tests._parity import BF16_GRAD, assert_close, to_np

pytestmark = pytest.mark.gpu


def _noalloc_call(lib, q, k, v, o, lse, do, dq, dk, dv, scale):
    B, H, Nq, D = q.shape
    Nk = k.shape[2]
    stream = torch.cuda.current_stream().cuda_stream
    return lib.mea_attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                    do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, Nq, Nk, D,
                                    ctypes.c_float(scale), 1, ctypes.c_void_p(stream))


@pytest.mark.parametrize("B,H,Nq,Nk,D", [(2, 3, 300, 520, 128), (1, 4, 700, 333, 64)])
def test_noalloc_matches_workspace_entry_point(B, H, Nq, Nk, D):
    """Two calls in a row: each is checked element by element against the fp64 oracle and against
    mea_attn_bwd with a caller workspace (same kernels: dK, dV bit-identical; dQ, summed by
    reduce-adds in no fixed order, within the gradient tolerance)."""
    import exact_memory_efficient_b200 as m
    lib = m.load_library()
    w = custom(B, H, Nq, Nk, D, "bf16")
    q_h, k_h, v_h, do_h = make_inputs(w, 13)
    q, k, v, do = (x.cuda() for x in (q_h, k_h, v_h, do_h))
    o, lse = m.attention_forward(q, k, v, w.scale)
    ref_dq, ref_dk, ref_dv = m.attention_backward(q, k, v, o, lse, do, w.scale)  # caller-provided workspace
    torch.cuda.synchronize()
    rq, rk, rv, _, _ = oracle.attention_backward(to_f64(q_h), to_f64(k_h), to_f64(v_h), to_f64(do_h), w.scale)
    for call in range(2):  # the second call reuses the scratch the first one left behind
        dq, dk, dv = torch.full_like(q, 9.0), torch.full_like(k, 9.0), torch.full_like(v, 9.0)
        st = _noalloc_call(lib, q, k, v, o, lse, do, dq, dk, dv, w.scale)
        assert st == m.MEA_OK, m.mea_last_error_message()
        assert m.mea_last_device_error() == m.MEA_OK
        for name, a, r in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
            assert_close(to_np(a), r, *BF16_GRAD, what=f"{name} call {call} vs oracle")
        assert torch.equal(dk, ref_dk) and torch.equal(dv, ref_dv), f"call {call}: dK/dV differ from mea_attn_bwd"
        assert_close(to_np(dq), to_np(ref_dq), *BF16_GRAD, what=f"dQ call {call} vs mea_attn_bwd")


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    import exact_memory_efficient_b200 as m
    lib = m.load_library()
    A = 0x10000
    # B1 H16 N16384 D128 needs ~136 MB of scratch: more than the 64 MiB array
    st = lib.mea_attn_bwd_noalloc(*([A] * 9), 1, 16, 16384, 16384, 128, ctypes.c_float(0.088), 1, None)
    assert st == m.MEA_ERR_WORKSPACE
    assert "static scratch" in m.mea_last_error_message()
