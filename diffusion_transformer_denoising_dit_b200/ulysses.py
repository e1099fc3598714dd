"""Sequence-parallel (Ulysses) joint attention and cache gate across ranks.

Source: "FLUX 3 Image Klein / TensorRT-LLM VisualGen", the multi-GPU section:
Ulysses sequence parallelism splits the tokens across GPUs for the per-token
work and exchanges them around attention, which needs every token.

Each rank holds one contiguous token range of Q, K and V, [B, H, n, d] with
n = N / P for P ranks (rank r holds tokens [r n, (r + 1) n)).  One all-to-all
turns the sequence shards into head shards, [B, H / P, N, d]: every token of
H / P heads.  Attention then runs locally and unchanged (this library's
kernels, with the rotary tables of the whole sequence), and a second
all-to-all turns the output back into sequence shards.  The collectives are
torch.distributed's (NCCL between GPUs); no kernel reads another GPU's memory.

The cache gate over a residual that is split the same way needs the sums of
every shard: each rank computes its shard's two totals, an all-reduce adds
them, and every rank takes the same decision from the same totals.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _binding


def seq_to_head(x: torch.Tensor, group=None) -> torch.Tensor:
    """[B, H, n, d] (this rank's tokens, all heads) -> [B, H / P, P n, d]
    (all tokens, this rank's heads: rank r gets heads [r H / P, (r + 1) H / P))."""
    P = dist.get_world_size(group)
    B, H, n, d = x.shape
    if H % P:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    Hp = H // P
    send = x.reshape(B, P, Hp, n, d).permute(1, 0, 2, 3, 4).contiguous()  # block r -> rank r
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)  # block s <- rank s's tokens of our heads
    return recv.permute(1, 2, 0, 3, 4).reshape(B, Hp, P * n, d)


def head_to_seq(y: torch.Tensor, group=None) -> torch.Tensor:
    """[B, H / P, N, d] (all tokens, this rank's heads) -> [B, H, N / P, d]
    (this rank's tokens, all heads); the inverse of seq_to_head."""
    P = dist.get_world_size(group)
    B, Hp, N, d = y.shape
    if N % P:
        raise ValueError(f"{N} tokens do not split over {P} ranks")
    n = N // P
    send = y.reshape(B, Hp, P, n, d).permute(2, 0, 1, 3, 4).contiguous()  # block r: rank r's tokens
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)  # block s <- rank s's heads of our tokens
    return recv.permute(1, 0, 2, 3, 4).reshape(B, P * Hp, n, d)


def attention(q, k, v, cos=None, sin=None, group=None, attend=None, **kwargs):
    """Joint attention of a sequence-sharded Q, K, V ([B, H, N / P, d] per rank).

    cos, sin: rotary tables of the whole sequence ([N, d / 2], as dit_rope_tables
    builds them).  attend: the local attention (default: this library's,
    ``dit.attention``; ``kwargs`` go to it).  Returns this rank's tokens of O.
    """
    attend = _binding.attention if attend is None else attend
    qh, kh, vh = (seq_to_head(t, group) for t in (q, k, v))
    return head_to_seq(attend(qh, kh, vh, cos, sin, **kwargs), group)


def _seq_to_head_chunk(x, c, chunks, group):
    """Start the exchange of head chunk c: every rank sends rank r its tokens of
    rank r's chunk-c heads ([B, H / P / chunks, n, d] per destination).  Returns
    the receive buffer [P, B, H / P / chunks, n, d] and the async work."""
    P = dist.get_world_size(group)
    B, H, n, d = x.shape
    Hp = H // P
    Hc = Hp // chunks
    send = x.reshape(B, P, chunks, Hc, n, d)[:, :, c].permute(1, 0, 2, 3, 4).contiguous()
    recv = torch.empty_like(send)
    work = dist.all_to_all_single(recv, send, group=group, async_op=True)
    return recv, work


def _head_chunk_of(recv):
    """[P, B, Hc, n, d] received blocks -> [B, Hc, P n, d] (all tokens of the chunk's heads)."""
    P, B, Hc, n, d = recv.shape
    return recv.permute(1, 2, 0, 3, 4).reshape(B, Hc, P * n, d)


def attention_overlapped(q, k, v, cos=None, sin=None, group=None, attend=None, chunks=2, **kwargs):
    """ulysses.attention with the exchanges split by head chunk and overlapped
    with the attention of the neighbouring chunks: chunk c + 1's Q, K, V are in
    flight while chunk c's attention runs, and chunk c's output goes back while
    chunk c + 1's runs.  chunks must divide H / P; chunks = 1 is the plain form.
    The result is the same as ulysses.attention's, bit for bit (the same local
    attention on the same heads).  On NCCL the exchanges run on the collective
    stream and each wait orders only the launching stream, never the host."""
    attend = _binding.attention if attend is None else attend
    P = dist.get_world_size(group)
    B, H, n, d = q.shape
    if H % P or (H // P) % chunks:
        raise ValueError(f"{H} heads do not split over {P} ranks x {chunks} chunks")
    Hp, Hc = H // P, H // P // chunks
    inflight = [_seq_to_head_chunk(t, 0, chunks, group) for t in (q, k, v)]
    outs = []
    for c in range(chunks):
        for _, work in inflight:
            work.wait()
        qh, kh, vh = (_head_chunk_of(recv) for recv, _ in inflight)
        if c + 1 < chunks:  # the next chunk's exchange overlaps this chunk's attention
            inflight = [_seq_to_head_chunk(t, c + 1, chunks, group) for t in (q, k, v)]
        o = attend(qh, kh, vh, cos, sin, **kwargs)          # [B, Hc, P n, d]
        send = o.reshape(B, Hc, P, n, d).permute(2, 0, 1, 3, 4).contiguous()  # block r: rank r's tokens
        recv = torch.empty_like(send)
        outs.append((recv, dist.all_to_all_single(recv, send, group=group, async_op=True)))
    res = torch.empty(P, chunks, B, Hc, n, d, dtype=outs[0][0].dtype, device=outs[0][0].device)
    for c, (recv, work) in enumerate(outs):
        work.wait()
        res[:, c] = recv                                      # [P, B, Hc, n, d] from rank s: its heads
    # heads of rank s, chunk c, index i -> global head s Hp + c Hc + i
    return res.permute(2, 0, 1, 3, 4, 5).reshape(B, H, n, d)


def gate(r_cur, r_prev, threshold: float, group=None, sums=None, finalize=None):
    """First-Block-Cache decision over a residual split across ranks: each rank
    passes its shard; all ranks return the same (rel, skip).

    sums(r_cur, r_prev) -> float64 [2] totals and finalize(totals, threshold) ->
    (rel, skip) default to this library's fbcache_gate_sums / _finalize.
    """
    sums = _binding.fbcache_gate_sums if sums is None else sums
    finalize = _binding.fbcache_gate_finalize if finalize is None else finalize
    totals = sums(r_cur, r_prev)
    dist.all_reduce(totals, group=group)  # (sum |a - b|, sum |b|) over every shard
    return finalize(totals, threshold)
