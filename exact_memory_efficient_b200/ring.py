"""Ring attention: the sequence is split over the ranks of a group for queries and keys alike.

Source: "当注意力成为瓶颈从on困境到线性复杂度的技术突围" (section 分布式：突破单卡限制,
the Ring Attention paragraph): each device keeps one block of the sequence,
the key/value blocks travel around a ring of devices, and every device
attends its query block to each key/value block as it passes, with the
transfer of the next block overlapping the computation on the current one.
The per-block results are merged exactly with the chunk-summary merge of
"Self-attention Does Not Need O(n^2) Memory" (mea_attn_combine), so the
result is the attention of this rank's queries over the keys of every rank.

Rank r holds q_r [B, H, Nq_r, D] and k_r, v_r [B, H_kv, Nk_r, D]; shard lengths
may differ between ranks.  At step s it holds the key/value block of rank
(r - s) mod W.

forward:   per step, the block's (o_b, lse_b) from the forward kernel is merged
           into the running (o, lse); the next block is received from rank
           r - 1 and the current one sent to rank r + 1 while it is computed.
backward:  the key/value blocks travel again, each with fp32 sums of its dk,
           dv.  Per step the library adds this rank's contributions
           (mea_attn_bwd_accum: P recomputed from the merged lse, so every
           contribution is final) to those sums and to the local fp32 dq sum,
           and block and sums pass on; a final send returns every block's sums
           to its owner, and mea_attn_accum_convert turns the three sums into
           gradients.  No step does tensor arithmetic outside the library.

The compute steps come from an ``ops`` object (the CUDA library by default) so
that the exchange can run without a GPU; point-to-point transfers use
torch.distributed (NCCL over NVLink on GPUs, gloo on CPU).
"""

from __future__ import annotations

import math

import torch
import torch.distributed as dist

from .keysplit import CudaOps


def _scale(q, scale):
    return 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)


def _ring_peers(group):
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    to_global = (lambda r: dist.get_global_rank(group, r)) if group is not None else (lambda r: r)
    return world, rank, to_global((rank + 1) % world), to_global((rank - 1) % world)


def _shard_lengths(n_local: int, device, group):
    """Key counts of every rank's shard, in rank order."""
    world = dist.get_world_size(group)
    mine = torch.tensor([n_local], dtype=torch.int64, device=device)
    every = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(every, mine, group=group)
    return [int(x.item()) for x in every]


def _exchange(send, recv_shapes, nxt, prv, group):
    """Start sending the tensors ``send`` to rank ``nxt`` and receiving tensors of
    ``recv_shapes`` (dtypes as ``send``) from rank ``prv``; returns (received, works).
    Empty tensors are not transferred: both ends know every shard's length."""
    recv = [torch.empty(shape, dtype=t.dtype, device=t.device) for t, shape in zip(send, recv_shapes)]
    ops = [dist.P2POp(dist.isend, t.contiguous(), nxt, group) for t in send if t.numel() > 0]
    ops += [dist.P2POp(dist.irecv, t, prv, group) for t in recv if t.numel() > 0]
    return recv, (dist.batch_isend_irecv(ops) if ops else [])


def ring_attention_forward(q, k_local, v_local, scale=None, group=None, ops=None):
    """Attention of this rank's queries over the keys of every rank of ``group``.

    Returns (o, lse) for this rank's query rows.
    """
    ops = CudaOps() if ops is None else ops
    scale = _scale(q, scale)
    world, rank, nxt, prv = _ring_peers(group)
    lengths = _shard_lengths(k_local.shape[2], k_local.device, group)
    k_cur, v_cur = k_local.contiguous(), v_local.contiguous()
    o = lse = None
    for s in range(world):
        works = []
        if s + 1 < world:
            n_next = lengths[(rank - s - 1) % world]
            shape = (k_cur.shape[0], k_cur.shape[1], n_next, k_cur.shape[3])
            (k_nxt, v_nxt), works = _exchange([k_cur, v_cur], [shape, shape], nxt, prv, group)
        if k_cur.shape[2] > 0:
            o_b, lse_b = ops.forward(q, k_cur, v_cur, scale)
            o, lse = (o_b, lse_b) if o is None else ops.combine([o, o_b], [lse, lse_b])
        for w in works:
            w.wait()
        if s + 1 < world:
            k_cur, v_cur = k_nxt, v_nxt
    if o is None:
        raise ValueError("ring_attention_forward: no rank holds any key")
    return o, lse


def ring_attention_backward(q, k_local, v_local, o, lse, do, scale=None, group=None, ops=None):
    """Gradients for this rank's shards: (dq, dk_local, dv_local).

    ``o`` and ``lse`` are this rank's results of ring_attention_forward.  Key and
    value heads equal the query heads.  The library adds every block's
    contributions to fp32 sums (dq's stays here, dk's and dv's travel with their
    block) and converts them to gradients once, at the end.
    """
    ops = CudaOps() if ops is None else ops
    scale = _scale(q, scale)
    world, rank, nxt, prv = _ring_peers(group)
    lengths = _shard_lengths(k_local.shape[2], k_local.device, group)
    k_cur, v_cur = k_local.contiguous(), v_local.contiguous()
    acc_dtype = torch.float64 if q.dtype == torch.float64 else torch.float32
    dq_acc = torch.zeros(q.shape, dtype=acc_dtype, device=q.device)
    dk_cur = torch.zeros(k_cur.shape, dtype=acc_dtype, device=k_cur.device)
    dv_cur = torch.zeros(v_cur.shape, dtype=acc_dtype, device=v_cur.device)
    workspace = ops.accum_workspace(q, k_cur)
    for s in range(world):
        n_next = lengths[(rank - s - 1) % world]
        shape = (k_cur.shape[0], k_cur.shape[1], n_next, k_cur.shape[3])
        works = []
        if s + 1 < world:   # the next block travels while this one is computed
            (k_nxt, v_nxt), works = _exchange([k_cur, v_cur], [shape, shape], nxt, prv, group)
        if k_cur.shape[2] > 0:
            ops.backward_accumulate(q, k_cur, v_cur, o, lse, do, scale, dq_acc, dk_cur, dv_cur, workspace)
        if world > 1:
            # the sums follow their block; after the last step every block's
            # sums are back with their owner
            (dk_nxt, dv_nxt), works_acc = _exchange([dk_cur, dv_cur], [shape, shape], nxt, prv, group)
            works += works_acc
        for w in works:
            w.wait()
        if world > 1:
            dk_cur, dv_cur = dk_nxt, dv_nxt
        if s + 1 < world:
            k_cur, v_cur = k_nxt, v_nxt
    return (ops.accum_convert(dq_acc, scale, q.dtype), ops.accum_convert(dk_cur, scale, k_local.dtype),
            ops.accum_convert(dv_cur, 1.0, v_local.dtype))
