"""Ulysses head-parallel MC-Sparse for sequence-sharded models.

The pages run their video model with Ulysses context parallelism on 7 of 8
GPUs (aimodeling.com article on Tencent's MC-Sparse, section "Numbers,
deployment, and the Hopper ceiling": the 7+1 layout; the aiwillknow analysis
cites the paper's Table 1 and Appendix A for the same setup): each rank holds a
contiguous shard of the sequence. MC-Sparse
is independent per (batch, head), so on P ranks it needs exactly two
exchanges per attention call and none inside the method:

  seq_to_heads  all-to-all of Q, K, V: [B, N/P, H, d] per rank (a sequence
                shard of every head) -> [B, N, H/P, d] (every token of H/P heads)
  (grouping, anchor or reuse on the rank's heads, through the C ABI)
  heads_to_seq  all-to-all of O back: [B, N, H/P, d] -> [B, N/P, H, d]

The per-head metadata (permutation, KV indices, residual) stays on the rank
that owns the head. Rank r holds sequence rows [r*N/P, (r+1)*N/P) and heads
[r*H/P, (r+1)*H/P). The exchanges are torch.distributed all_to_all_single calls
(NCCL over NVLink on GPUs); the attention itself runs only in libmcs.so.
"""
from __future__ import annotations

from . import binding as _mcs


def _world(group):
    import torch.distributed as dist

    return dist.get_world_size(group)


def seq_to_heads(x, group=None):
    """Sequence shard [B, N/P, H, d] -> head shard [B, N, H/P, d] (one all-to-all)."""
    import torch
    import torch.distributed as dist

    P = _world(group)
    B, n, H, d = x.shape
    if H % P:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    # chunk p of the send buffer = this rank's rows of head group p
    send = x.reshape(B, n, P, H // P, d).permute(2, 0, 1, 3, 4).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[r] = rank r's rows (sequence shard r) of this rank's heads
    return recv.permute(1, 0, 2, 3, 4).reshape(B, P * n, H // P, d)


def heads_to_seq(o, group=None):
    """Head shard [B, N, H/P, d] -> sequence shard [B, N/P, H, d] (one all-to-all)."""
    import torch
    import torch.distributed as dist

    P = _world(group)
    B, N, hp, d = o.shape
    if N % P:
        raise ValueError(f"{N} tokens do not split over {P} ranks")
    n = N // P
    # chunk p of the send buffer = sequence shard p of this rank's heads
    send = o.reshape(B, P, n, hp, d).permute(1, 0, 2, 3, 4).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[r] = this rank's sequence shard of rank r's heads
    return recv.permute(1, 2, 0, 3, 4).reshape(B, n, P * hp, d)


class UlyssesMCSparse:
    """MC-Sparse attention of one layer on a sequence-sharded layout.

    anchor(q, k, v) groups the queries and runs the anchor step on this rank's
    heads, keeping their metadata; reuse(q, k, v) runs the reuse step with it.
    Inputs and outputs are this rank's sequence shard, bf16 [B, N/P, H, d] on
    the rank's GPU. krylov_steps > 0 selects the fast grouping (fixed Krylov
    steps per node) instead of the exact one.
    """

    def __init__(self, B: int, H: int, N: int, d: int, topk: int, group=None, krylov_steps: int = 0,
                 device=None):
        import torch

        P = _world(group)
        if H % P or N % P:
            raise ValueError(f"H={H} and N={N} must both split over {P} ranks")
        self.group = group
        self.krylov_steps = krylov_steps
        self.shape = _mcs.Shape(B, H // P, N, d, topk=topk)
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        G = (N + 127) // 128
        hp = H // P
        self.perm = torch.empty(B, hp, N, dtype=torch.int32, device=dev)
        self.kv_idx = torch.empty(B, hp, G, topk, dtype=torch.int32, device=dev)
        self.resid = torch.empty(B, hp, N, d, dtype=torch.bfloat16, device=dev)
        self.ws = {op: _mcs.workspace(self.shape, op, dev)
                   for op in (_mcs.MCS_OP_GROUP, _mcs.MCS_OP_ANCHOR, _mcs.MCS_OP_SPARSE)}
        self.anchored = False

    def anchor(self, q, k, v, stream=None):
        import torch

        qh, kh, vh = (seq_to_heads(t, self.group) for t in (q, k, v))
        if self.krylov_steps > 0:
            _mcs.mcs_group_fast(self.shape, qh, self.perm, self.krylov_steps, self.ws[_mcs.MCS_OP_GROUP], stream)
        else:
            _mcs.mcs_group(self.shape, qh, self.perm, self.ws[_mcs.MCS_OP_GROUP], stream)
        oh = torch.empty_like(qh)
        _mcs.mcs_anchor(self.shape, qh, kh, vh, self.perm, oh, self.kv_idx, self.resid, None,
                        self.ws[_mcs.MCS_OP_ANCHOR], stream)
        self.anchored = True
        return heads_to_seq(oh, self.group)

    def reuse(self, q, k, v, stream=None):
        import torch

        if not self.anchored:
            raise RuntimeError("reuse before the first anchor: no cached metadata")
        qh, kh, vh = (seq_to_heads(t, self.group) for t in (q, k, v))
        oh = torch.empty_like(qh)
        _mcs.mcs_sparse(self.shape, qh, kh, vh, self.perm, self.kv_idx, self.resid, oh,
                        self.ws[_mcs.MCS_OP_SPARSE], stream)
        return heads_to_seq(oh, self.group)

    def status(self, stream=None):
        """Poll every workspace's status block: list of (op, status, info) for the non-OK ones."""
        out = []
        for op, ws in self.ws.items():
            st, info = _mcs.mcs_poll_status(ws, stream)
            if st != 0:
                out.append((op, st, info))
        return out
