"""Seeded synthetic inputs for the VSA forward path.

This module holds random-number generation and tensor layout only: it draws
N(0,1) activations, sigmoid gates, sequence-length mixes and uniformly random
block selections (inputs of the entry points that take indices), and places
tokens into the padded 64-slot block layout that every entry point consumes.
It does none of the method's arithmetic (no pooling, no attention, no top-k),
so the CPU oracle and the CUDA library can both be fed from it.

Recipe (used by the tests and by ``bench.py``):

* activations q, k, v: ``torch.randn`` in fp32 from a CPU ``torch.Generator``
  seeded with ``seed * 1_000_003 + stream``, rounded to bf16 (round to nearest
  even, torch's conversion);
* gate: the same normal draw pushed through a sigmoid in fp64, then rounded to
  bf16 -- the gate is the model's ``compress_attn_weight`` activation, which
  the combine page passes as a ``[B, S, H, D]`` tensor;
* padded slots of a block (slots ``>= block size``) hold ``pad_value``
  (0 by default, as the varlen page packs into zero tensors).

Stream ids: q=0, k=1, v=2, gate=3.  Workload seeds are ``1000 + workload#``.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK = 64  # tokens per block slot group (the 64-token VSA tile)

STREAM_Q, STREAM_K, STREAM_V, STREAM_GATE = 0, 1, 2, 3


def _gen(seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 1_000_003 + int(stream))
    return g


def normal_bf16(shape, seed: int, stream: int, scale: float = 1.0) -> torch.Tensor:
    """N(0, scale^2) draw in fp32, rounded to bf16 (CPU tensor)."""
    x = torch.randn(tuple(shape), generator=_gen(seed, stream), dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    return x.to(torch.bfloat16)


def gate_bf16(shape, seed: int, stream: int = STREAM_GATE) -> torch.Tensor:
    """sigmoid(N(0,1)) evaluated in fp64, rounded to bf16 (CPU tensor)."""
    x = torch.randn(tuple(shape), generator=_gen(seed, stream), dtype=torch.float32)
    return torch.sigmoid(x.double()).to(torch.bfloat16)


def full_block_sizes(n_tokens: int) -> list[int]:
    """Block sizes of a contiguous run of ``n_tokens``: 64, ..., 64, remainder."""
    if n_tokens <= 0:
        return []
    nb = (n_tokens + BLOCK - 1) // BLOCK
    return [BLOCK] * (nb - 1) + [n_tokens - BLOCK * (nb - 1)]


def topk_count(frac: float, n_kv_blocks: int) -> int:
    """Workload convention: a top-k fraction becomes floor(frac * n) in [1, n]."""
    return max(1, min(n_kv_blocks, int(math.floor(frac * n_kv_blocks + 1e-9))))


def pad_tokens_bhsd(x_tokens: torch.Tensor, block_sizes: list[int],
                    pad_value: float = 0.0, block: int = BLOCK) -> torch.Tensor:
    """Place contiguous tokens ``[B, H, N, D]`` into the padded layout.

    Block ``j`` takes the next ``block_sizes[j]`` tokens in order and occupies
    slots ``block*j .. block*j + block_sizes[j] - 1``; the rest of its slots
    hold ``pad_value``.  Returns ``[B, H, block*len(block_sizes), D]``.
    """
    B, H, N, D = x_tokens.shape
    assert sum(block_sizes) == N
    out = torch.full((B, H, block * len(block_sizes), D), pad_value, dtype=x_tokens.dtype)
    src = 0
    for j, n in enumerate(block_sizes):
        out[:, :, block * j:block * j + n] = x_tokens[:, :, src:src + n]
        src += n
    return out


def padded_normal_bhsd(B: int, H: int, block_sizes: list[int], D: int, seed: int,
                       stream: int, pad_value: float = 0.0, scale: float = 1.0,
                       block: int = BLOCK) -> torch.Tensor:
    """N(0,1) bf16 activations directly in the padded ``[B, H, block*n, D]`` layout."""
    n_tok = sum(block_sizes)
    x = normal_bf16((B, H, n_tok, D), seed, stream, scale=scale)
    return pad_tokens_bhsd(x, block_sizes, pad_value, block)


@dataclass
class Workload:
    """Sizes of one synthetic workload (no tensors)."""
    name: str
    B: int
    H: int
    D: int
    q_block_sizes: list[int]
    kv_block_sizes: list[int]
    topk: int
    gated: bool = True
    seed: int = 1000
    extra: dict = field(default_factory=dict)
    block: int = BLOCK  # slots per block: 64, or 128 / 256 for VSA-128 / VSA-256 tiles

    @property
    def nq(self) -> int:
        return len(self.q_block_sizes)

    @property
    def nkv(self) -> int:
        return len(self.kv_block_sizes)

    @property
    def selected_tiles(self) -> int:
        return self.B * self.H * self.nq * min(self.topk, self.nkv)

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs of the selected tiles: 4 * block * block * D each
        (QK^T and PV of a block x block tile)."""
        return 4.0 * self.block * self.block * self.D * self.selected_tiles


def workload_tiny() -> Workload:
    """B=1, H=2, D=64, 512 tokens (8 blocks), top-2, gated."""
    return Workload("tiny: B1 H2 D64 S512 top2 gated", 1, 2, 64, [64] * 8, [64] * 8, 2,
                    True, 1001)


def workload_h3() -> Workload:
    """B=1, H=56, D=128, 15488 tokens (242 blocks), top 20% = 48 blocks, gated."""
    nb = 15488 // BLOCK
    return Workload("H3-like: B1 H56 D128 S15488 top48 (20%) gated", 1, 56, 128, [64] * nb,
                    [64] * nb, topk_count(0.20, nb), True, 1003)


def workload_long(frac: float, gated: bool = True) -> Workload:
    """B=1, H=40, D=128, 32768 tokens (512 blocks) at a top-k fraction."""
    nb = 32768 // BLOCK
    k = topk_count(frac, nb)
    return Workload(f"long: B1 H40 D128 S32768 top{k} ({frac:.0%}) {'gated' if gated else 'ungated'}",
                    1, 40, 128, [64] * nb, [64] * nb, k, gated, 1005)


def workload_vsa128() -> Workload:
    """The README's VSA-128 benchmark shape: B=1, H=12, D=128, 39936 tokens
    in 312 blocks of 128 (128-token video tiles), top 40, gated."""
    nb = 39936 // 128
    return Workload("VSA-128: B1 H12 D128 S39936 (312 blocks of 128) top40 gated", 1, 12, 128,
                    [128] * nb, [128] * nb, 40, True, 1006, block=128)


def workload_vsa256() -> Workload:
    """The README's VSA-256 benchmark shape: B=1, H=12, D=128, 39936 tokens
    in 156 blocks of 256 (256-token video tiles), top 20, gated."""
    nb = 39936 // 256
    return Workload("VSA-256: B1 H12 D128 S39936 (156 blocks of 256) top20 gated", 1, 12, 128,
                    [256] * nb, [256] * nb, 20, True, 1007, block=256)


VARLEN_Q_LENS = (3000, 6144, 9216, 15488)
VARLEN_KV_LENS = (3000, 7040, 9216, 12800)


def cu_seqlens(lengths) -> list[int]:
    out = [0]
    for n in lengths:
        out.append(out[-1] + int(n))
    return out


def varlen_random_selection(q_lens, kv_lens, H: int, frac: float, seed: int):
    """Seeded per-sequence block selections for the varlen entry: for every
    sequence i, query block and head (in that order), topk_count(frac, n_kv_i)
    distinct KV blocks of sequence i drawn uniformly, ascending, with -1 after
    them.  Returns (q2k_idx int32 [H, total_q_blocks, max_k], q2k_num int32
    [H, total_q_blocks], per-sequence k)."""
    nq = [-(-int(n) // BLOCK) for n in q_lens]
    nkv = [-(-int(n) // BLOCK) for n in kv_lens]
    ks = [topk_count(frac, n) for n in nkv]
    rng = np.random.default_rng(seed)
    idx = np.full((H, sum(nq), max(ks)), -1, dtype=np.int32)
    num = np.zeros((H, sum(nq)), dtype=np.int32)
    row = 0
    for i in range(len(nq)):
        for _ in range(nq[i]):
            for h in range(H):
                idx[h, row, :ks[i]] = np.sort(rng.choice(nkv[i], size=ks[i], replace=False))
                num[h, row] = ks[i]
            row += 1
    return idx, num, ks
