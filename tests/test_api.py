"""Host-side tests of the C ABI (no kernel is launched).

* the shared library builds, loads and exports every function that
  include/mea_attn.h declares;
* every invalid call is rejected with the documented status before any CUDA
  call is made (fake device addresses are never dereferenced on the host);
* the workspace size is O(N*D) and matches its documented layout.
"""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mea_attn.h")


@pytest.fixture(scope="module")
def lib():
    from exact_memory_efficient_b200 import build as b
    b.build()
    import exact_memory_efficient_b200 as m
    return m.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mea_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert {"mea_attn_fwd", "mea_attn_bwd", "mea_attn_bwd_phase", "mea_attn_bwd_workspace_size",
            "mea_last_device_error", "mea_status_string", "mea_last_error_message", "mea_version"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in mea_attn.h but not exported"


def test_status_strings(lib):
    import exact_memory_efficient_b200 as m
    for code in range(0, 7):
        s = m.mea_status_string(code)
        assert s.startswith("MEA_")
    assert m.mea_status_string(99) == "MEA_ERR_UNKNOWN"
    assert m.mea_version() == 100


A = 0x10000  # fake, 16-byte aligned device addresses (never dereferenced on the host)
BF16, F32 = 1, 0


def fwd(lib, q=A, k=A, v=A, o=A, lse=A, B=1, H=1, Nq=16, Nk=16, D=64, scale=0.125, dtype=BF16):
    return lib.mea_attn_fwd(q, k, v, o, lse, B, H, Nq, Nk, D, ctypes.c_float(scale), dtype, None)


def bwd(lib, ptrs=None, B=1, H=1, Nq=16, Nk=16, D=64, scale=0.125, dtype=BF16, ws=A, ws_bytes=1 << 30):
    p = [A] * 9 if ptrs is None else ptrs
    return lib.mea_attn_bwd(*p, B, H, Nq, Nk, D, ctypes.c_float(scale), dtype, ws, ws_bytes, None)


def test_forward_argument_validation(lib):
    assert fwd(lib, q=None) == 1
    assert fwd(lib, lse=None) == 1
    assert fwd(lib, B=-1) == 1
    assert fwd(lib, Nk=0) == 1
    assert fwd(lib, D=0) == 1
    assert fwd(lib, scale=float("nan")) == 1
    assert fwd(lib, scale=float("inf")) == 1
    assert fwd(lib, dtype=7) == 1
    assert fwd(lib, D=96) == 2           # bf16 supports D in {64, 128}
    assert fwd(lib, D=256) == 2
    assert fwd(lib, D=48, dtype=F32) == 2  # fp32 needs D % 32 == 0 and D <= 128
    assert fwd(lib, D=160, dtype=F32) == 2
    assert fwd(lib, q=A + 8) == 3
    assert fwd(lib, o=A + 4) == 3
    assert fwd(lib, lse=A + 2) == 3


def test_forward_empty_is_noop(lib):
    # no rows: nothing is launched, so this succeeds without a GPU
    assert fwd(lib, Nq=0) == 0
    assert fwd(lib, B=0) == 0
    assert fwd(lib, H=0, q=None) == 0


def test_backward_argument_validation(lib):
    assert bwd(lib, dtype=F32, D=48) == 2   # fp32 needs D % 32 == 0 and D <= 128
    assert bwd(lib, dtype=F32, D=160) == 2
    assert bwd(lib, D=96) == 2
    assert bwd(lib, Nk=0) == 1
    assert bwd(lib, Nq=-3) == 1
    ptrs = [A] * 9
    ptrs[5] = None  # dO
    assert bwd(lib, ptrs=ptrs) == 1
    ptrs = [A] * 9
    ptrs[7] = A + 8  # dk misaligned
    assert bwd(lib, ptrs=ptrs) == 3
    assert bwd(lib, ws=None) == 4
    assert bwd(lib, ws_bytes=100) == 4
    assert bwd(lib, ws=A + 16) == 3       # workspace must be 256-byte aligned
    assert bwd(lib, B=0) == 0
    # phased entry point: same validation, unknown phase rejected
    assert lib.mea_attn_bwd_phase(9, *([A] * 9), 1, 1, 16, 16, 64, ctypes.c_float(0.125), BF16, A, 1 << 30,
                                  None) == 1
    assert lib.mea_attn_bwd_phase(2, *([A] * 9), 1, 1, 16, 16, 96, ctypes.c_float(0.125), BF16, A, 1 << 30,
                                  None) == 2


def test_workspace_size(lib):
    out = ctypes.c_size_t(0)
    assert lib.mea_attn_bwd_workspace_size(1, 16, 16384, 16384, 128, BF16, ctypes.byref(out)) == 0
    rows = 16 * 16384
    assert out.value == rows * 128 * 4 + rows * 4  # dQ accumulator + row term, both 256-aligned here
    assert lib.mea_attn_bwd_workspace_size(2, 3, 5, 7, 64, BF16, ctypes.byref(out)) == 0
    r = 2 * 3 * 5
    assert out.value == ((r * 64 * 4 + 255) // 256) * 256 + ((r * 4 + 255) // 256) * 256
    # fp32: the row term only
    assert lib.mea_attn_bwd_workspace_size(1, 1, 4, 4, 64, F32, ctypes.byref(out)) == 0
    assert out.value == 256
    assert lib.mea_attn_bwd_workspace_size(2, 3, 1000, 4, 96, F32, ctypes.byref(out)) == 0
    assert out.value == ((2 * 3 * 1000 * 4 + 255) // 256) * 256
    assert lib.mea_attn_bwd_workspace_size(1, 1, 4, 4, 48, F32, ctypes.byref(out)) == 2
    assert lib.mea_attn_bwd_workspace_size(1, 1, 4, 4, 64, BF16, None) == 1
    # O(N*D) extra memory, never O(N^2): doubling N doubles the workspace
    a, b = ctypes.c_size_t(0), ctypes.c_size_t(0)
    lib.mea_attn_bwd_workspace_size(1, 1, 4096, 4096, 128, BF16, ctypes.byref(a))
    lib.mea_attn_bwd_workspace_size(1, 1, 8192, 8192, 128, BF16, ctypes.byref(b))
    assert b.value == 2 * a.value


def test_python_binding_rejects_bad_tensors(lib):
    import torch
    import exact_memory_efficient_b200 as m
    q = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(m.MeaError):
        m.mea_attn_fwd(q, q, q, q, torch.zeros(1, 1, 4), 0.125)  # CPU tensors are rejected
    with pytest.raises(m.MeaError):
        m.mea_attn_fwd(q[0], q, q, q, torch.zeros(1, 1, 4), 0.125)


@pytest.mark.parametrize("entry", ["mea_attn_bwd", "mea_attn_bwd_noalloc", "mea_attn_bwd_gqa"])
def test_python_backward_rejects_mismatched_operands(lib, entry):
    """The backward wrappers check k, v and lse against q before anything reaches the C side: the
    kernels index every operand by q's sizes, so a smaller k or lse would be read past its end."""
    import torch
    import exact_memory_efficient_b200 as m
    fn = getattr(m, entry)
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    lse = torch.zeros(1, 2, 8)

    def call(k, lse_):
        v, dk, dv = torch.zeros_like(k), torch.zeros_like(k), torch.zeros_like(k)
        args = (q, k, v, q.clone(), lse_, q.clone(), q.clone(), dk, dv, 0.125)
        return fn(*args) if entry == "mea_attn_bwd_noalloc" else fn(*args, None)

    match = "k (must be|shape|dtype)" if entry != "mea_attn_bwd_gqa" else "k must be"
    with pytest.raises(m.MeaError, match=match):
        call(torch.zeros(1, 2, 8, 32, dtype=torch.bfloat16), lse)         # k's D differs from q's
    with pytest.raises(m.MeaError, match=match):
        call(torch.zeros(2, 2, 8, 64, dtype=torch.bfloat16), lse)         # k's B differs from q's
    if entry != "mea_attn_bwd_gqa":                                        # (fewer k heads is GQA there)
        with pytest.raises(m.MeaError, match=match):
            call(torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16), lse)     # k's H differs from q's
    k = torch.zeros(1, 2, 16, 64, dtype=torch.bfloat16)
    with pytest.raises(m.MeaError, match="lse must be"):
        call(k, lse.to(torch.bfloat16))                                    # lse not fp32
    with pytest.raises(m.MeaError, match="lse must be"):
        call(k, torch.zeros(1, 2, 4))                                      # lse shorter than Nq
    with pytest.raises(m.MeaError, match="must be a contiguous CUDA tensor"):
        call(k, lse)                                                       # consistent, but CPU tensors


def test_gqa_argument_validation(lib):
    def fwd_gqa(H=4, Hkv=2, Nq=16, q=A, B=1):
        return lib.mea_attn_fwd_gqa(q, A, A, A, A, B, H, Hkv, Nq, 16, 64, ctypes.c_float(0.125), BF16, None)

    def bwd_gqa(H=4, Hkv=2, Nq=16, ws=A, ws_bytes=1 << 30, D=64):
        return lib.mea_attn_bwd_gqa(*([A] * 9), 1, H, Hkv, Nq, 16, D, ctypes.c_float(0.125), BF16, ws, ws_bytes,
                                    None)

    assert fwd_gqa(Hkv=3) == 1            # H not a multiple of H_kv
    assert fwd_gqa(Hkv=0) == 1
    assert fwd_gqa(Hkv=-2) == 1
    assert fwd_gqa(H=1 << 20, Hkv=1, Nq=1 << 12) == 2   # group rows exceed 2^31-1
    assert fwd_gqa(q=None) == 1
    assert fwd_gqa(q=A + 8) == 3
    assert fwd_gqa(Nq=0) == 0             # no rows: no-op
    assert fwd_gqa(H=0, Hkv=1) == 0
    assert bwd_gqa(Hkv=3) == 1
    assert bwd_gqa(D=96) == 2
    assert bwd_gqa(ws=None) == 4
    out = ctypes.c_size_t(0)
    assert lib.mea_attn_bwd_gqa_workspace_size(1, 4, 3, 16, 16, 64, BF16, ctypes.byref(out)) == 1
    # the workspace follows the query heads: the same bytes as the per-head backward with H heads
    ref = ctypes.c_size_t(0)
    assert lib.mea_attn_bwd_gqa_workspace_size(2, 32, 8, 100, 300, 128, BF16, ctypes.byref(out)) == 0
    assert lib.mea_attn_bwd_workspace_size(2, 32, 100, 300, 128, BF16, ctypes.byref(ref)) == 0
    assert out.value == ref.value


def test_fp8_argument_validation(lib):
    def fwd8(D=128, qd=1.0, kd=1.0, H=4, Hkv=2, q=A, Nq=16):
        return lib.mea_attn_fwd_fp8(q, A, A, A, A, 1, H, Hkv, Nq, 16, D, ctypes.c_float(0.125), ctypes.c_float(qd),
                                    ctypes.c_float(kd), None)

    assert fwd8(D=64) == 2                 # head dim 128 only
    assert fwd8(qd=0.0) == 1
    assert fwd8(kd=-1.0) == 1
    assert fwd8(qd=float("nan")) == 1
    assert fwd8(kd=float("inf")) == 1
    assert fwd8(Hkv=3) == 1                # H not a multiple of H_kv
    assert fwd8(q=None) == 1
    assert fwd8(q=A + 8) == 3
    assert fwd8(Nq=0) == 0                 # no rows: no-op


def test_combine_argument_validation(lib):
    P = ctypes.c_void_p
    def comb(R=2, D=64, dtype=BF16, optr=A, lptr=A, o=A, lse=A, Nq=16):
        op = (P * max(R, 1))(*([optr] * max(R, 1)))
        lp = (P * max(R, 1))(*([lptr] * max(R, 1)))
        return lib.mea_attn_combine(op, lp, R, o, lse, 1, 2, Nq, D, dtype, None)

    assert comb(R=0) == 2
    assert comb(R=17) == 2
    assert comb(D=60) == 2                 # D must be a multiple of 8
    assert comb(D=264) == 2
    assert comb(dtype=7) == 1
    assert comb(optr=None) == 1
    assert comb(optr=A + 8) == 3
    assert comb(lptr=A + 2) == 3
    assert comb(o=A + 4) == 3
    assert comb(Nq=0) == 0                 # nothing to merge


def test_decode_argument_validation(lib):
    def dec(q=A, k=A, v=A, o=A, lse=A, B=1, H=8, Hkv=8, Nq=1, Nk=1024, D=128, scale=0.125, dtype=BF16,
            ws=A, ws_bytes=1 << 20):
        return lib.mea_attn_decode(q, k, v, o, lse, B, H, Hkv, Nq, Nk, D, ctypes.c_float(scale), dtype, ws,
                                   ws_bytes, None)

    assert dec(q=None) == 1
    assert dec(lse=None) == 1
    assert dec(Hkv=3) == 1                 # H not a multiple of H_kv
    assert dec(Hkv=0) == 1
    assert dec(Nk=0) == 1
    assert dec(scale=float("nan")) == 1
    assert dec(dtype=7) == 1
    assert dec(D=96) == 2                  # bf16 head dims are 64 and 128
    assert dec(D=96, dtype=F32, q=A + 8) == 3
    assert dec(k=A + 8) == 3
    assert dec(lse=A + 2) == 3
    assert dec(Nq=0) == 0                  # no rows: no-op
    assert dec(B=0) == 0
    assert dec(Nq=16, q=None) == 1         # 16 rows per head: the mea_attn_fwd_gqa path, same checks
    size = ctypes.c_size_t(99)
    # more than 8 rows per head: no split, no workspace (answered without a device)
    assert lib.mea_attn_decode_workspace_size(1, 8, 8, 16, 1024, 128, BF16, ctypes.byref(size)) == 0
    assert size.value == 0
    assert lib.mea_attn_decode_workspace_size(1, 8, 3, 1, 1024, 128, BF16, ctypes.byref(size)) == 1
    assert lib.mea_attn_decode_workspace_size(1, 8, 8, 1, 1024, 128, BF16, None) == 1
    assert lib.mea_attn_decode_workspace_size(1, 8, 8, 1, 1024, 96, BF16, ctypes.byref(size)) == 2


@pytest.mark.gpu
def test_more_heads_than_the_launch_grid_is_unsupported():
    """B*H above 65535 (the grid dimension that indexes heads) is refused with
    MEA_ERR_UNSUPPORTED before any launch.  The tensors are real and sized to
    the call, so nothing could be read out of bounds even if a kernel ran."""
    import torch
    import exact_memory_efficient_b200 as m
    B, H, N, D = 65536, 1, 16, 64
    for dt in (torch.bfloat16, torch.float32):
        q = torch.zeros(B, H, N, D, dtype=dt, device="cuda")
        o = torch.empty_like(q)
        lse = torch.empty(B, H, N, device="cuda")
        with pytest.raises(m.MeaError) as e:
            m.mea_attn_fwd(q, q, q, o, lse, 0.125)
        assert e.value.status == 2
        del q, o, lse
    q = torch.zeros(B, H, N, D, dtype=torch.bfloat16, device="cuda")
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    lse = torch.zeros(B, H, N, device="cuda")
    ws = torch.empty(m.mea_attn_bwd_workspace_size(B, H, N, N, D), dtype=torch.uint8, device="cuda")
    with pytest.raises(m.MeaError) as e:
        m.mea_attn_bwd(q, q, q, o, lse, q, dq, dk, dv, 0.125, ws)
    assert e.value.status == 2
    torch.cuda.synchronize()
    assert m.mea_last_device_error() == 0


def test_noalloc_scratch_size_matches_header():
    """The binding's MEA_NOALLOC_SCRATCH_BYTES (reported by the bench as resident memory) is the
    header's #define."""
    import exact_memory_efficient_b200 as m
    with open(os.path.join(ROOT, "include", "mea_attn.h")) as f:
        text = f.read()
    a, b, c = re.search(r"#define MEA_NOALLOC_SCRATCH_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", text).groups()
    assert m.MEA_NOALLOC_SCRATCH_BYTES == int(a) * int(b) * int(c)


def test_accumulating_backward_argument_validation(lib):
    """mea_attn_bwd_accum and mea_attn_accum_convert reject bad arguments before any launch."""
    out = ctypes.c_size_t(0)
    assert lib.mea_attn_bwd_accum_workspace_size(2, 3, 100, 50, 64, BF16, ctypes.byref(out)) == 0
    assert out.value == 2 * 3 * 100 * 4 + (256 - (2 * 3 * 100 * 4) % 256) % 256   # the row term, 256-aligned
    assert lib.mea_attn_bwd_accum_workspace_size(1, 1, 16, 16, 96, BF16, ctypes.byref(out)) == 2

    def accum(ptrs=None, Nq=16, Nk=16, D=64, ws=A, ws_bytes=1 << 20, dtype=BF16):
        p = ptrs if ptrs is not None else [A] * 9
        return lib.mea_attn_bwd_accum(*p, 1, 2, Nq, Nk, D, ctypes.c_float(0.125), dtype, ws, ws_bytes, None)

    assert accum(Nq=0) == 0                      # an empty query range adds nothing
    assert accum(Nk=0) == 0                      # an empty key range adds nothing
    assert accum(D=96) == 2                      # bf16 takes D in {64, 128}
    assert accum(ptrs=[A] * 6 + [None, A, A]) == 1
    assert accum(ptrs=[A] * 7 + [A + 4, A]) == 3  # a misaligned fp32 sum
    assert accum(ws=None) == 4
    assert accum(ws_bytes=16) == 4
    assert accum(ws=A + 16) == 3                 # workspace not 256-byte aligned

    def conv(acc=A, o=A, n=1024, mul=1.0, dtype=BF16):
        return lib.mea_attn_accum_convert(acc, o, ctypes.c_longlong(n), ctypes.c_float(mul), dtype, None)

    assert conv(n=0) == 0
    assert conv(n=6) == 2                        # not a multiple of 4
    assert conv(n=-4) == 1
    assert conv(acc=None) == 1
    assert conv(o=A + 8) == 3
    assert conv(mul=float("inf")) == 1
    assert conv(dtype=7) == 2
