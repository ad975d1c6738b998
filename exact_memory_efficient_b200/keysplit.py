"""Key (sequence) split across ranks: every rank holds all queries and one range of the keys.

Source: "当注意力成为瓶颈从on困境到线性复杂度的技术突围" (section 分布式：突破单卡限制)
splits a long sequence over GPUs; here the keys/values are split and the
per-range results are merged exactly with the chunk-summary merge of
"Self-attention Does Not Need O(n^2) Memory" (mea_attn_combine).

forward:   each rank runs mea_attn_fwd over its key range -> (o_r, lse_r);
           all-gather of the parts (torch.distributed; NCCL over NVLink);
           mea_attn_combine -> the attention over all keys (the same on every rank).
backward:  each rank runs the backward's PREPROCESS and MAIN phases with the
           merged o, lse and its own keys (P is recomputed from the global lse, so
           each range's contributions are final); all-reduce (sum) of the fp32 dQ
           accumulators; FINALIZE -> dq (the same on every rank); dk, dv stay with
           the rank's key range.

The compute steps are taken from an ``ops`` object so that the exchange logic
can be exercised without a GPU; the default is the CUDA library.
"""

from __future__ import annotations

import math

import torch
import torch.distributed as dist


class CudaOps:
    """The library's kernels (C ABI) as the compute steps of a key split."""

    def __init__(self):
        import exact_memory_efficient_b200 as m
        self.m = m

    def forward(self, q, k, v, scale):
        return self.m.attention_forward(q, k, v, scale)

    def combine(self, o_parts, lse_parts):
        o = torch.empty_like(o_parts[0])
        lse = torch.empty_like(lse_parts[0])
        self.m.mea_attn_combine(o_parts, lse_parts, o, lse)
        return o, lse

    def backward_partial(self, q, k, v, o, lse, do, scale):
        """PREPROCESS + MAIN over this rank's keys; returns (fp32 dQ accumulator, dk, dv, finish)."""
        m = self.m
        B, H, Nq, D = q.shape
        dq = torch.empty_like(q)
        dk, dv = torch.empty_like(k), torch.empty_like(v)
        if k.shape[2] == 0:
            return self._backward_no_keys(q, o, lse, do, dq, dk, dv, scale)
        ws = torch.empty(m.mea_attn_bwd_workspace_size(B, H, Nq, k.shape[2], D, q.dtype), dtype=torch.uint8,
                         device=q.device)
        for ph in (m.MEA_BWD_PREPROCESS, m.MEA_BWD_MAIN):
            m.mea_attn_bwd_phase(ph, q, k, v, o, lse, do, dq, dk, dv, scale, ws)
        if q.dtype == torch.float32:
            # the fp32 backward sums dQ per row in registers: its partial dq is final per range
            return dq, dk, dv, lambda acc: acc
        acc = ws[:B * H * Nq * D * 4].view(torch.float32)

        def finish(summed):
            # FINALIZE reads the (now summed) accumulator in place
            m.mea_attn_bwd_phase(m.MEA_BWD_FINALIZE, q, k, v, o, lse, do, dq, dk, dv, scale, ws)
            return dq

        return acc, dk, dv, finish

    def _backward_no_keys(self, q, o, lse, do, dq, dk, dv, scale):
        """A rank whose key range is empty adds nothing to dQ, but still takes part in the
        all-reduce and, for bf16, converts the summed accumulator itself."""
        m = self.m
        if q.dtype == torch.float32:
            return torch.zeros_like(q), dk, dv, lambda acc: acc
        B, H, Nq, D = q.shape
        # the phases take a key count >= 1: a one-key stand-in that PREPROCESS and FINALIZE never read
        k1 = torch.zeros((B, H, 1, D), dtype=q.dtype, device=q.device)
        g1 = torch.empty_like(k1)
        ws = torch.empty(m.mea_attn_bwd_workspace_size(B, H, Nq, 1, D, q.dtype), dtype=torch.uint8, device=q.device)
        m.mea_attn_bwd_phase(m.MEA_BWD_PREPROCESS, q, k1, k1, o, lse, do, dq, g1, g1, scale, ws)  # zeroes the acc
        acc = ws[:B * H * Nq * D * 4].view(torch.float32)

        def finish(summed):
            m.mea_attn_bwd_phase(m.MEA_BWD_FINALIZE, q, k1, k1, o, lse, do, dq, g1, g1, scale, ws)
            return dq

        return acc, dk, dv, finish


    # ---- accumulating backward (ring attention): fp32 sums that travel between calls
    def accum_workspace(self, q, k):
        B, H, Nq, D = q.shape
        n = self.m.mea_attn_bwd_accum_workspace_size(B, H, Nq, k.shape[2], D, q.dtype)
        return torch.empty(n, dtype=torch.uint8, device=q.device)

    def backward_accumulate(self, q, k, v, o, lse, do, scale, dq_acc, dk_acc, dv_acc, workspace):
        """dq_acc += dS K, dk_acc += dS^T Q, dv_acc += P^T dO over this key range (fp32, unscaled)."""
        self.m.mea_attn_bwd_accum(q, k, v, o, lse, do, dq_acc, dk_acc, dv_acc, scale, workspace)

    def accum_convert(self, acc, mul, dtype):
        out = torch.empty(acc.shape, dtype=dtype, device=acc.device)
        self.m.mea_attn_accum_convert(acc, out, mul)
        return out


def _scale(q, scale):
    return 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)


def attention_forward_keysplit(q, k_local, v_local, scale=None, group=None, ops=None):
    """Attention of all queries over the keys of every rank; this rank holds k_local, v_local.

    Returns (o, lse), identical on every rank of ``group``.
    """
    ops = CudaOps() if ops is None else ops
    scale = _scale(q, scale)
    if k_local.shape[2] == 0:
        # a rank without keys (fewer keys than ranks) contributes the empty sum: weight
        # e^{lse} = 0 in the merge, whatever its o; no kernel runs over zero keys
        o_r = torch.zeros(q.shape[:3] + (v_local.shape[3],), dtype=q.dtype, device=q.device)
        lse_dtype = torch.float64 if q.dtype == torch.float64 else torch.float32
        lse_r = torch.full(q.shape[:3], float("-inf"), dtype=lse_dtype, device=q.device)
    else:
        o_r, lse_r = ops.forward(q, k_local, v_local, scale)
    world = dist.get_world_size(group)
    o_all = [torch.empty_like(o_r) for _ in range(world)]
    lse_all = [torch.empty_like(lse_r) for _ in range(world)]
    dist.all_gather(o_all, o_r.contiguous(), group=group)
    dist.all_gather(lse_all, lse_r.contiguous(), group=group)
    return ops.combine(o_all, lse_all)


def attention_backward_keysplit(q, k_local, v_local, o, lse, do, scale=None, group=None, ops=None):
    """Gradients of a key split: (dq, dk_local, dv_local); dq is identical on every rank."""
    ops = CudaOps() if ops is None else ops
    scale = _scale(q, scale)
    acc, dk, dv, finish = ops.backward_partial(q, k_local, v_local, o, lse, do, scale)
    dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)
    return finish(acc), dk, dv


def key_range(Nk: int, rank: int, world: int):
    """The [begin, end) keys of ``rank`` when Nk keys are split as evenly as possible."""
    base, extra = divmod(Nk, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)
