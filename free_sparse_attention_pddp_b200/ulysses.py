"""Ulysses head-parallel MC-Sparse for sequence-sharded models.

The pages run their video model with Ulysses context parallelism on 7 of 8
GPUs (aimodeling.com article on Tencent's MC-Sparse, section "Numbers,
deployment, and the Hopper ceiling": the 7+1 layout; the aiwillknow analysis
cites the paper's Table 1 and Appendix A for the same setup): each rank holds a
contiguous shard of the sequence. MC-Sparse is independent per (batch, head),
so on P ranks it needs exactly two exchanges per attention call and none
inside the method:

  seq_to_heads  all-to-all of Q, K, V: [B, n_r, H, d] per rank (a sequence
                shard of every head) -> [B, N, h_r, d] (every token of the
                rank's h_r heads)
  (grouping, anchor or reuse on the rank's heads, through the C ABI)
  heads_to_seq  all-to-all of O back: [B, N, h_r, d] -> [B, n_r, H, d]

Neither count has to divide by P: with H = 24 heads on the 7 denoising ranks
of that layout the ranks hold 4, 4, 4, 3, 3, 3, 3 heads. Both splits are
balanced and contiguous (``split_counts``): rank r holds sequence rows
[s_r, s_r + n_r) and heads [t_r, t_r + h_r), the first (count mod P) ranks
taking one more. The per-head metadata (permutation, KV indices, residual)
stays on the rank that owns the head. The exchanges are
torch.distributed all_to_all_single calls with per-rank split sizes (NCCL over
NVLink on GPUs); the attention itself runs only in libmcs.so.
"""
from __future__ import annotations

from . import binding as _mcs


def _world(group):
    import torch.distributed as dist

    return dist.get_world_size(group)


def _rank(group):
    import torch.distributed as dist

    return dist.get_rank(group)


def split_counts(n: int, P: int):
    """Balanced contiguous split of n items over P ranks: counts, the first n mod P one larger."""
    if n < 0 or P < 1:
        raise ValueError(f"cannot split {n} items over {P} ranks")
    return [n // P + (1 if r < n % P else 0) for r in range(P)]


def _offsets(counts):
    out, acc = [], 0
    for c in counts:
        out.append(acc)
        acc += c
    return out


def seq_to_heads(x, group=None, N=None):
    """Sequence shard [B, n_r, H, d] -> head shard [B, N, h_r, d] (one all-to-all).

    N is the full sequence length (default n_r * P, an even split); every rank
    must hold the shard ``split_counts(N, P)[rank]`` of it."""
    import torch
    import torch.distributed as dist

    P, r = _world(group), _rank(group)
    B, n, H, d = x.shape
    N = n * P if N is None else N
    rows = split_counts(N, P)
    if rows[r] != n:
        raise ValueError(f"rank {r} holds {n} rows; a split of {N} tokens over {P} ranks gives it {rows[r]}")
    heads = split_counts(H, P)
    h0 = _offsets(heads)
    # chunk p of the send buffer: this rank's rows of rank p's heads
    send = torch.cat([x[:, :, h0[p]:h0[p] + heads[p]].reshape(-1) for p in range(P)])
    recv = torch.empty(B * N * heads[r] * d, dtype=x.dtype, device=x.device)
    dist.all_to_all_single(recv, send, output_split_sizes=[B * rows[p] * heads[r] * d for p in range(P)],
                           input_split_sizes=[B * n * heads[p] * d for p in range(P)], group=group)
    # chunk p of recv: rank p's rows (sequence shard p) of this rank's heads
    parts = torch.split(recv, [B * rows[p] * heads[r] * d for p in range(P)])
    return torch.cat([c.view(B, rows[p], heads[r], d) for p, c in enumerate(parts)], dim=1)


def heads_to_seq(o, group=None, H=None):
    """Head shard [B, N, h_r, d] -> sequence shard [B, n_r, H, d] (one all-to-all).

    H is the total head count (default h_r * P, an even split); every rank
    must hold the heads ``split_counts(H, P)[rank]`` of it."""
    import torch
    import torch.distributed as dist

    P, r = _world(group), _rank(group)
    B, N, hr, d = o.shape
    H = hr * P if H is None else H
    heads = split_counts(H, P)
    if heads[r] != hr:
        raise ValueError(f"rank {r} holds {hr} heads; a split of {H} heads over {P} ranks gives it {heads[r]}")
    rows = split_counts(N, P)
    s0 = _offsets(rows)
    # chunk p of the send buffer: sequence shard p of this rank's heads
    send = torch.cat([o[:, s0[p]:s0[p] + rows[p]].reshape(-1) for p in range(P)])
    recv = torch.empty(B * rows[r] * H * d, dtype=o.dtype, device=o.device)
    dist.all_to_all_single(recv, send, output_split_sizes=[B * rows[r] * heads[p] * d for p in range(P)],
                           input_split_sizes=[B * rows[p] * hr * d for p in range(P)], group=group)
    # chunk p of recv: this rank's sequence shard of rank p's heads
    parts = torch.split(recv, [B * rows[r] * heads[p] * d for p in range(P)])
    return torch.cat([c.view(B, rows[r], heads[p], d) for p, c in enumerate(parts)], dim=2)


class UlyssesMCSparse:
    """MC-Sparse attention of one layer on a sequence-sharded layout.

    anchor(q, k, v) groups the queries and runs the anchor step on this rank's
    heads, keeping their metadata; reuse(q, k, v) runs the reuse step with it.
    Inputs and outputs are this rank's sequence shard, bf16 [B, n_r, H, d] on
    the rank's GPU, with n_r = split_counts(N, P)[rank]; the rank computes
    split_counts(H, P)[rank] heads (a rank left with none only takes part in
    the exchanges). krylov_steps > 0 selects the fast grouping (fixed Krylov
    steps per node) instead of the exact one.
    """

    def __init__(self, B: int, H: int, N: int, d: int, topk: int, group=None, krylov_steps: int = 0,
                 device=None):
        import torch

        P, r = _world(group), _rank(group)
        self.group = group
        self.krylov_steps = krylov_steps
        self.H, self.N = H, N
        self.rows = split_counts(N, P)[r]
        hp = split_counts(H, P)[r]
        self.heads = hp
        self.shape = _mcs.Shape(B, max(hp, 1), N, d, topk=topk)
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        G = (N + 127) // 128
        self.perm = torch.empty(B, hp, N, dtype=torch.int32, device=dev)
        self.kv_idx = torch.empty(B, hp, G, topk, dtype=torch.int32, device=dev)
        self.resid = torch.empty(B, hp, N, d, dtype=torch.bfloat16, device=dev)
        self.ws = {} if hp == 0 else {op: _mcs.workspace(self.shape, op, dev)
                                      for op in (_mcs.MCS_OP_GROUP, _mcs.MCS_OP_ANCHOR, _mcs.MCS_OP_SPARSE)}
        self.anchored = False

    def _to_heads(self, q, k, v):
        return tuple(seq_to_heads(t, self.group, N=self.N) for t in (q, k, v))

    def anchor(self, q, k, v, stream=None):
        import torch

        qh, kh, vh = self._to_heads(q, k, v)
        oh = torch.empty_like(qh)
        if self.heads > 0:
            if self.krylov_steps > 0:
                _mcs.mcs_group_fast(self.shape, qh, self.perm, self.krylov_steps, self.ws[_mcs.MCS_OP_GROUP],
                                    stream)
            else:
                _mcs.mcs_group(self.shape, qh, self.perm, self.ws[_mcs.MCS_OP_GROUP], stream)
            _mcs.mcs_anchor(self.shape, qh, kh, vh, self.perm, oh, self.kv_idx, self.resid, None,
                            self.ws[_mcs.MCS_OP_ANCHOR], stream)
        self.anchored = True
        return heads_to_seq(oh, self.group, H=self.H)

    def reuse(self, q, k, v, stream=None):
        import torch

        if not self.anchored:
            raise RuntimeError("reuse before the first anchor: no cached metadata")
        qh, kh, vh = self._to_heads(q, k, v)
        oh = torch.empty_like(qh)
        if self.heads > 0:
            _mcs.mcs_sparse(self.shape, qh, kh, vh, self.perm, self.kv_idx, self.resid, oh,
                            self.ws[_mcs.MCS_OP_SPARSE], stream)
        return heads_to_seq(oh, self.group, H=self.H)

    def status(self, stream=None):
        """Poll every workspace's status block: list of (op, status, info) for the non-OK ones."""
        out = []
        for op, ws in self.ws.items():
            st, info = _mcs.mcs_poll_status(ws, stream)
            if st != 0:
                out.append((op, st, info))
        return out
