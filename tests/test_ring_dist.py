"""Ring attention exchange on CPU: world_size 2 and 3 gloo ranks, no GPU.

Every rank holds one shard of the queries and one shard of the keys/values
(unequal lengths, one rank without keys in one case).  The compute steps are
the oracle-based fakes of test_keysplit_dist; what is under test is the
orchestration in exact_memory_efficient_b200.ring: the ring order, the
point-to-point transfers overlapping each step, the running merge of the
per-block results, the accumulators that travel with their block and return
to its owner, and that every rank ends with its share of full attention.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cuts(n, sizes):
    b = np.concatenate([[0], np.cumsum(sizes)])
    assert b[-1] == n
    return [(int(x), int(y)) for x, y in zip(b[:-1], b[1:])]


def _worker(rank, world, port, inputs, q_sizes, k_sizes, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from exact_memory_efficient_b200.ring import ring_attention_backward, ring_attention_forward
        from tests.test_keysplit_dist import OracleOps
        q, k, v, do, scale = inputs
        qa, qb = _cuts(q.shape[2], q_sizes)[rank]
        ka, kb = _cuts(k.shape[2], k_sizes)[rank]
        ops = OracleOps()
        q_r, do_r = q[:, :, qa:qb].contiguous(), do[:, :, qa:qb].contiguous()
        k_r, v_r = k[:, :, ka:kb].contiguous(), v[:, :, ka:kb].contiguous()
        o, lse = ring_attention_forward(q_r, k_r, v_r, scale, ops=ops)
        dq, dk, dv = ring_attention_backward(q_r, k_r, v_r, o, lse, do_r, scale, ops=ops)
        torch.save({"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv},
                   os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,q_sizes,k_sizes", [
    (2, [3, 5], [20, 17]),
    (3, [4, 1, 6], [9, 0, 23]),    # the middle rank holds no keys
    (3, [2, 2, 2], [1, 1, 30]),
])
def test_ring_reaches_full_attention(tmp_path, world, q_sizes, k_sizes):
    g = torch.Generator().manual_seed(world + sum(k_sizes))
    Nq, Nk = sum(q_sizes), sum(k_sizes)
    q = torch.randn(1, 2, Nq, 8, generator=g, dtype=torch.float64)
    k = torch.randn(1, 2, Nk, 8, generator=g, dtype=torch.float64)
    v = torch.randn(1, 2, Nk, 8, generator=g, dtype=torch.float64)
    do = torch.randn(1, 2, Nq, 8, generator=g, dtype=torch.float64)
    scale = 0.4
    mp.start_processes(_worker, args=(world, _free_port(), (q, k, v, do, scale), q_sizes, k_sizes, str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    ro, rl = oracle.attention_forward(q.numpy(), k.numpy(), v.numpy(), scale)
    rq, rk, rv, _, _ = oracle.attention_backward(q.numpy(), k.numpy(), v.numpy(), do.numpy(), scale)
    for r in range(world):
        d = torch.load(tmp_path / f"rank{r}.pt")
        qa, qb = _cuts(Nq, q_sizes)[r]
        ka, kb = _cuts(Nk, k_sizes)[r]
        np.testing.assert_allclose(d["o"].numpy(), ro[:, :, qa:qb], atol=1e-12)
        np.testing.assert_allclose(d["lse"].numpy(), rl[:, :, qa:qb], atol=1e-12)
        np.testing.assert_allclose(d["dq"].numpy(), rq[:, :, qa:qb], atol=1e-12)
        assert d["dk"].shape[2] == kb - ka
        np.testing.assert_allclose(d["dk"].numpy(), rk[:, :, ka:kb], atol=1e-12)
        np.testing.assert_allclose(d["dv"].numpy(), rv[:, :, ka:kb], atol=1e-12)
