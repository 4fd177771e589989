"""Sequence-parallel ("Ulysses") VSA forward across the ranks of a process
group: each rank holds a sequence shard of every head, the forward runs on
full sequences of a head group per rank.

README "Compiled CUDA extensions" (the fused NVLink Ulysses all-to-all) and
the 4-GPU Wan2.1 sequence-parallel recipe it serves: before attention, an
all-to-all turns sequence shards into head shards; after it, a second one
turns them back.  Here:

  q, k, v, gate on rank r: [B, S_local, H, D] (BSHD), the r-th slice of the
  sequence (the padded block layout split in N equal contiguous parts).

  1. pack   x[:, :, j*H/N:(j+1)*H/N] for every destination j -> [N, B, S_local, H/N, D]
  2. all_to_all_single (NCCL over NVLink)
  3. gather the N received sequence shards -> [B, S, H/N, D]
  4. the whole VSA forward on the head group (BSHD, strided views)
  5. scatter the output into per-source sequence shards -> [N, B, S_local, H/N, D]
  6. all_to_all_single
  7. unpack the N head groups -> [B, S_local, H, D]

Steps 1, 3, 5 and 7 are one library call each (``vsa_permute_rows``, an HBM
copy); step 4 is the library's forward.  The permutations are given as
(extents, source strides) specs so that the same specs can be checked
against a plain reference on the CPU; ``ops`` swaps the three operations
(permute, exchange, forward) for such checks.  With N = 1 every exchange is
the identity and the result equals the single-GPU forward bit for bit.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable

import torch


def pack_heads_spec(B: int, S: int, H: int, N: int):
    """[B, S, H, D] -> [N, B, S, H/N, D]: destination j gets heads j*H/N.. ."""
    Hn = H // N
    return (N, B, S, Hn), (Hn, S * H, H, 1)


def gather_seq_spec(B: int, S: int, Hn: int, N: int):
    """Received [N, B, S, Hn, D] (source i holds sequence shard i) ->
    [B, N*S, Hn, D], shard i at sequence offset i*S."""
    return (B, N, S, Hn), (S * Hn, B * S * Hn, Hn, 1)


def scatter_seq_spec(B: int, S: int, Hn: int, N: int):
    """[B, N*S, Hn, D] -> [N, B, S, Hn, D]: sequence shard i for rank i."""
    return (N, B, S, Hn), (S * Hn, N * S * Hn, Hn, 1)


def unpack_heads_spec(B: int, S: int, Hn: int, N: int):
    """Received [N, B, S, Hn, D] (source j holds head group j) ->
    [B, S, N*Hn, D]."""
    return (B, S, N, Hn), (S * Hn, Hn, B * S * Hn, 1)


@dataclass
class UlyssesOps:
    """The three operations the wrapper needs.  Defaults: the CUDA library's
    row permutation and forward, and torch.distributed's all_to_all_single
    (NCCL on CUDA tensors)."""
    permute: Callable | None = None        # (src, extents, strides) -> tensor (*extents, D)
    all_to_all: Callable | None = None     # (out, inp, group) -> None
    forward: Callable | None = None        # (q, k, v, gate, qbs, kbs, topk, scale, block) -> (out, idx, num)

    def resolved(self) -> "UlyssesOps":
        from . import binding as vsa
        import torch.distributed as dist

        def fwd(q, k, v, gate, qbs, kbs, topk, scale, block):
            return vsa.video_sparse_attn_bshd(q, k, v, gate, qbs, kbs, topk=topk, scale=scale,
                                              block=block)

        return UlyssesOps(
            permute=self.permute or (lambda src, e, st: vsa.permute_rows(src, e, st)),
            all_to_all=self.all_to_all or (lambda out, inp, group: dist.all_to_all_single(out, inp, group=group)),
            forward=self.forward or fwd)


def _exchange(ops, x, group):
    out = torch.empty_like(x)
    ops.all_to_all(out, x.contiguous(), group)
    return out


def vsa_forward_ulysses(q, k, v, gate=None, q_block_sizes=None, kv_block_sizes=None, *,
                        topk: int, scale: float | None = None, block: int = 64, group=None,
                        ops: UlyssesOps | None = None):
    """VSA forward on sequence-sharded BSHD inputs: q, gate [B, Sq_local, H, D],
    k, v [B, Skv_local, H, D] on each of the group's N ranks (rank r holds the
    r-th contiguous slice of the padded sequence).  H must be a multiple of
    N.  Block sizes (if given) describe the whole sequence, as in the
    single-GPU call.  Returns (out [B, Sq_local, H, D], q2k_idx, q2k_num), the
    indices for this rank's head group [B, H/N, n_q_blocks, k]."""
    import torch.distributed as dist
    ops = (ops or UlyssesOps()).resolved()
    N = dist.get_world_size(group)
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    if H % N:
        raise ValueError(f"{H} heads do not split over {N} ranks")
    if k.shape != (B, Skv, H, D) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Skv_local, H, D] matching q")
    if gate is not None and gate.shape != q.shape:
        raise ValueError("gate must be shaped like q")
    if (N * Sq) % block or (N * Skv) % block:
        raise ValueError("the gathered sequences must be multiples of the block size")
    Hn = H // N
    if N == 1:
        # one rank: both exchanges and all four reshards are the identity
        return ops.forward(q, k, v, gate, q_block_sizes, kv_block_sizes, topk, scale, block)

    def to_heads(x, S):
        sent = ops.permute(x.contiguous().view(-1, D), *pack_heads_spec(B, S, H, N))
        got = _exchange(ops, sent, group)
        full = ops.permute(got.view(-1, D), *gather_seq_spec(B, S, Hn, N))   # [B, N, S, Hn, D]
        return full.view(B, N * S, Hn, D)

    qf, kf, vf = to_heads(q, Sq), to_heads(k, Skv), to_heads(v, Skv)
    gf = None if gate is None else to_heads(gate, Sq)
    out_h, idx, num = ops.forward(qf, kf, vf, gf, q_block_sizes, kv_block_sizes, topk, scale, block)
    sent = ops.permute(out_h.contiguous().view(-1, D), *scatter_seq_spec(B, Sq, Hn, N))
    got = _exchange(ops, sent, group)
    out = ops.permute(got.view(-1, D), *unpack_heads_spec(B, Sq, Hn, N))   # [B, Sq, N, Hn, D]
    return out.view(B, Sq, H, D), idx, num
