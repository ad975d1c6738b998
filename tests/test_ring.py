"""Ring attention with the library's CUDA kernels as the compute steps (GPU).

Two gloo ranks share the one GPU.  Each rank's compute steps are the
library's own (exact_memory_efficient_b200.keysplit.CudaOps: the forward, the
combine, the accumulating backward and the conversion of its fp32 sums) on
device copies of the tensors, while the ring transfers move host copies between the
ranks.  Every launch is an ordinary independent launch: no kernel waits on the
other rank; the ranks meet only on the host, in the transfers.  The oracle
computes full attention over the whole sequence.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from synthetic_inputs import custom, make_inputs, to_f64
from tests._parity import BF16_GRAD, BF16_O, F32_O_MAX_ABS, assert_close, assert_lse_close

pytestmark = pytest.mark.gpu


class HostCudaOps:
    """CudaOps on device copies; tensors in and out stay on the host (gloo transfers them)."""

    def __init__(self):
        from exact_memory_efficient_b200.keysplit import CudaOps
        self.ops = CudaOps()

    def forward(self, q, k, v, scale):
        o, lse = self.ops.forward(q.cuda(), k.cuda(), v.cuda(), scale)
        return o.cpu(), lse.cpu()

    def combine(self, o_parts, lse_parts):
        o, lse = self.ops.combine([x.cuda() for x in o_parts], [x.cuda() for x in lse_parts])
        return o.cpu(), lse.cpu()

    def backward_partial(self, q, k, v, o, lse, do, scale):
        acc, dk, dv, fin = self.ops.backward_partial(q.cuda(), k.cuda(), v.cuda(), o.cuda(), lse.cuda(), do.cuda(),
                                                     scale)

        def finish(summed):
            acc.copy_(summed.cuda())
            return fin(acc).cpu()

        return acc.cpu(), dk.cpu(), dv.cpu(), finish

    def accum_workspace(self, q, k):
        return self.ops.accum_workspace(q.cuda(), k.cuda())

    def backward_accumulate(self, q, k, v, o, lse, do, scale, dq_acc, dk_acc, dv_acc, workspace):
        accs = [a.cuda() for a in (dq_acc, dk_acc, dv_acc)]
        self.ops.backward_accumulate(q.cuda(), k.cuda(), v.cuda(), o.cuda(), lse.cuda(), do.cuda(), scale, *accs,
                                     workspace)
        for host, dev in zip((dq_acc, dk_acc, dv_acc), accs):
            host.copy_(dev.cpu())

    def accum_convert(self, acc, mul, dtype):
        return self.ops.accum_convert(acc.cuda(), mul, dtype).cpu()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, inputs, q_cut, k_cut, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from exact_memory_efficient_b200.ring import ring_attention_backward, ring_attention_forward
        q, k, v, do, scale = inputs
        qs = slice(0, q_cut) if rank == 0 else slice(q_cut, q.shape[2])
        ks = slice(0, k_cut) if rank == 0 else slice(k_cut, k.shape[2])
        q_r, do_r = q[:, :, qs].contiguous(), do[:, :, qs].contiguous()
        k_r, v_r = k[:, :, ks].contiguous(), v[:, :, ks].contiguous()
        ops = HostCudaOps()
        o, lse = ring_attention_forward(q_r, k_r, v_r, scale, ops=ops)
        dq, dk, dv = ring_attention_backward(q_r, k_r, v_r, o, lse, do_r, scale, ops=ops)
        import exact_memory_efficient_b200 as m
        assert m.mea_last_device_error() == m.MEA_OK
        torch.save({"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}, os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("dtype,H,Nq,Nk,D,q_cut,k_cut", [
    ("bf16", 2, 500, 900, 128, 200, 333),
    ("bf16", 3, 300, 640, 64, 150, 500),
    ("f32", 2, 120, 400, 64, 70, 150),
])
def test_ring_two_ranks_cuda_ops(tmp_path, dtype, H, Nq, Nk, D, q_cut, k_cut):
    w = custom(1, H, Nq, Nk, D, dtype)
    q, k, v, do = make_inputs(w, 31)
    mp.start_processes(_worker, args=(2, _free_port(), (q, k, v, do, w.scale), q_cut, k_cut, str(tmp_path)),
                       nprocs=2, join=True, start_method="spawn")
    rq, rk, rv, ro, rl = oracle.attention_backward(to_f64(q), to_f64(k), to_f64(v), to_f64(do), w.scale)
    parts = [torch.load(tmp_path / f"rank{r}.pt") for r in range(2)]
    cat = {n: np.concatenate([p[n].double().numpy() for p in parts], axis=2) for n in ("o", "lse", "dq", "dk", "dv")}
    if dtype == "bf16":
        assert_close(cat["o"], ro, *BF16_O, what="ring O")
        for n, r in (("dq", rq), ("dk", rk), ("dv", rv)):
            assert_close(cat[n], r, *BF16_GRAD, what=f"ring {n}")
    else:
        assert_close(cat["o"], ro, F32_O_MAX_ABS, what="ring fp32 O")
        for n, r in (("dq", rq), ("dk", rk), ("dv", rv)):
            assert_close(cat[n], r, F32_O_MAX_ABS, what=f"ring fp32 {n}")
    assert_lse_close(cat["lse"], rl, to_f64(q), to_f64(k), w.scale, what="ring lse")


def test_ring_module_one_rank_nccl():
    """The default path (CudaOps on CUDA tensors, NCCL) in a one-rank group: no transfer, every
    kernel and the accumulator hand-off are the real ones."""
    from exact_memory_efficient_b200.ring import ring_attention_backward, ring_attention_forward
    port = _free_port()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        w = custom(1, 2, 200, 700, 128, "bf16")
        q, k, v, do = make_inputs(w, 32)
        qd, kd, vd, dod = (x.cuda() for x in (q, k, v, do))
        o, lse = ring_attention_forward(qd, kd, vd, w.scale)
        dq, dk, dv = ring_attention_backward(qd, kd, vd, o, lse, dod, w.scale)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    rq, rk, rv, ro, rl = oracle.attention_backward(to_f64(q), to_f64(k), to_f64(v), to_f64(do), w.scale)
    assert_close(o.double().cpu().numpy(), ro, *BF16_O, what="ring O")
    for n, g_, r_ in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
        assert_close(g_.double().cpu().numpy(), r_, *BF16_GRAD, what=f"ring {n}")
