"""Exchange logic of the key split on CPU: world_size 2 (and 3) gloo ranks, no GPU.

Each rank holds all queries and one key range.  The compute steps are fakes
built from the fp64 oracle (the library's kernels need a GPU); what is under
test is the orchestration in exact_memory_efficient_b200.keysplit: the key
ranges, the all-gather of the parts, the merge, the all-reduce of the dQ
partials, and that every rank ends with the attention over all keys.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle


class OracleOps:
    def forward(self, q, k, v, scale):
        o, lse = oracle.attention_forward(q.numpy(), k.numpy(), v.numpy(), scale)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def combine(self, o_parts, lse_parts):
        o, lse = oracle.combine_partials(np.stack([x.numpy() for x in o_parts]),
                                         np.stack([x.numpy() for x in lse_parts]))
        return torch.from_numpy(o), torch.from_numpy(lse)

    def backward_partial(self, q, k, v, o, lse, do, scale):
        # this range's contributions, with P recomputed from the merged lse
        qn, kn, vn, on, ln, don = (x.numpy() for x in (q, k, v, o, lse, do))
        p = np.exp(scale * np.einsum("bhid,bhjd->bhij", qn, kn) - ln[..., None])
        dp = np.einsum("bhid,bhjd->bhij", don, vn)
        d_row = (don * on).sum(-1, keepdims=True)
        ds = p * (dp - d_row)
        dq = scale * np.einsum("bhij,bhjd->bhid", ds, kn)
        dk = scale * np.einsum("bhij,bhid->bhjd", ds, qn)
        dv = np.einsum("bhij,bhid->bhjd", p, don)
        return torch.from_numpy(dq), torch.from_numpy(dk), torch.from_numpy(dv), lambda acc: acc

    # accumulating interface (ring attention): unscaled sums, converted at the end
    def accum_workspace(self, q, k):
        return None

    def backward_accumulate(self, q, k, v, o, lse, do, scale, dq_acc, dk_acc, dv_acc, workspace):
        qn, kn, vn, on, ln, don = (x.numpy() for x in (q, k, v, o, lse, do))
        p = np.exp(scale * np.einsum("bhid,bhjd->bhij", qn, kn) - ln[..., None])
        ds = p * (np.einsum("bhid,bhjd->bhij", don, vn) - (don * on).sum(-1, keepdims=True))
        dq_acc += torch.from_numpy(np.einsum("bhij,bhjd->bhid", ds, kn))
        dk_acc += torch.from_numpy(np.einsum("bhij,bhid->bhjd", ds, qn))
        dv_acc += torch.from_numpy(np.einsum("bhij,bhid->bhjd", p, don))

    def accum_convert(self, acc, mul, dtype):
        return (acc * mul).to(dtype)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, inputs, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from exact_memory_efficient_b200.keysplit import (attention_backward_keysplit, attention_forward_keysplit,
                                                          key_range)
        q, k, v, do, scale = inputs
        a, b = key_range(k.shape[2], rank, world)
        ops = OracleOps()
        o, lse = attention_forward_keysplit(q, k[:, :, a:b].contiguous(), v[:, :, a:b].contiguous(), scale, ops=ops)
        dq, dk, dv = attention_backward_keysplit(q, k[:, :, a:b].contiguous(), v[:, :, a:b].contiguous(), o, lse, do,
                                                 scale, ops=ops)
        torch.save({"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv, "range": (a, b)},
                   os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,Nk", [(2, 37), (3, 50), (3, 2), (4, 1)])  # the last two: ranks without keys
def test_keysplit_exchange_reaches_full_attention(tmp_path, world, Nk):
    g = torch.Generator().manual_seed(world)
    q = torch.randn(1, 2, 6, 8, generator=g, dtype=torch.float64)
    k = torch.randn(1, 2, Nk, 8, generator=g, dtype=torch.float64)
    v = torch.randn(1, 2, Nk, 8, generator=g, dtype=torch.float64)
    do = torch.randn(1, 2, 6, 8, generator=g, dtype=torch.float64)
    scale = 0.4
    mp.start_processes(_worker, args=(world, _free_port(), (q, k, v, do, scale), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    ro, rl = oracle.attention_forward(q.numpy(), k.numpy(), v.numpy(), scale)
    rq, rk, rv, _, _ = oracle.attention_backward(q.numpy(), k.numpy(), v.numpy(), do.numpy(), scale)
    covered = []
    for r in range(world):
        d = torch.load(tmp_path / f"rank{r}.pt")
        a, b = d["range"]
        covered.append((a, b))
        np.testing.assert_allclose(d["o"].numpy(), ro, atol=1e-12)
        np.testing.assert_allclose(d["lse"].numpy(), rl, atol=1e-12)
        np.testing.assert_allclose(d["dq"].numpy(), rq, atol=1e-12)
        np.testing.assert_allclose(d["dk"].numpy(), rk[:, :, a:b], atol=1e-12)
        np.testing.assert_allclose(d["dv"].numpy(), rv[:, :, a:b], atol=1e-12)
    assert covered[0][0] == 0 and covered[-1][1] == Nk
    assert (Nk >= world) == all(b > a for a, b in covered)
    assert all(covered[i][1] == covered[i + 1][0] for i in range(world - 1))


def test_key_range_partitions_evenly():
    from exact_memory_efficient_b200.keysplit import key_range
    for Nk in (1, 7, 16, 100):
        for world in (1, 2, 3, 8):
            rs = [key_range(Nk, r, world) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == Nk
            sizes = [b - a for a, b in rs]
            assert max(sizes) - min(sizes) <= 1 and sum(sizes) == Nk
