"""The sequence-parallel ("Ulysses") wrapper's host logic on CPU with two
gloo ranks: the reshard specs, the order of the two all-to-all exchanges and
the head-group bookkeeping.  The row permutation and the forward are plain
CPU stand-ins here (a gather by the same (extents, strides) specs, and the
fp64 oracle on a head group); the library's permutation kernel is checked
against the same gather on the GPU (test_gpu_ulysses.py).  Each rank's
output must equal, exactly, the rows of its sequence shard in the oracle's
forward over the whole sequence and all heads."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_attention_15_b200 import ulysses as U


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def ref_permute(src, extents, strides):
    """out[a0, a1, a2, a3] = src row a0*S0 + a1*S1 + a2*S2 + a3*S3."""
    D = src.shape[-1]
    rows = torch.zeros(extents, dtype=torch.long)
    for ax, (e, s) in enumerate(zip(extents, strides)):
        shape = [1, 1, 1, 1]
        shape[ax] = e
        rows = rows + torch.arange(e).view(shape) * s
    return src.reshape(-1, D)[rows.reshape(-1)].reshape(*extents, D)


def _inputs(B, Sq, Skv, H, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Sq, H, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, Skv, H, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, Skv, H, D, generator=g, dtype=torch.float64)
    gate = torch.sigmoid(torch.randn(B, Sq, H, D, generator=g, dtype=torch.float64))
    return q, k, v, gate


def oracle_forward_bshd(q, k, v, gate, qbs, kbs, topk, scale, block):
    from oracle import vsa_oracle as O
    tr = lambda x: x.permute(0, 2, 1, 3).numpy()
    nq, nkv = q.shape[1] // block, k.shape[1] // block
    res = O.vsa_forward(tr(q), tr(k), tr(v), None if gate is None else gate.numpy(),
                        qbs or [block] * nq, kbs or [block] * nkv, topk, scale, block=block)
    out = torch.from_numpy(res["out"]).permute(0, 2, 1, 3).contiguous()
    return out, torch.from_numpy(res["q2k_idx"]), torch.from_numpy(res["q2k_num"])


def _rank_main(rank, world, port, case, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, Sq, Skv, H, D, topk, block, gated, qbs, kbs = case
        q, k, v, gate = _inputs(B, Sq, Skv, H, D, 77)
        gate = gate if gated else None
        sq, skv = Sq // world, Skv // world
        shard = lambda x, s: x[:, rank * s:(rank + 1) * s].contiguous()
        ops = U.UlyssesOps(permute=ref_permute,
                           all_to_all=lambda out, inp, group: dist.all_to_all_single(out, inp, group=group),
                           forward=oracle_forward_bshd)
        out, idx, num = U.vsa_forward_ulysses(
            shard(q, sq), shard(k, skv), shard(v, skv), None if gate is None else shard(gate, sq),
            qbs, kbs, topk=topk, block=block, ops=ops)
        q_out.put((rank, out.numpy(), idx.numpy(), num.numpy()))
    finally:
        dist.destroy_process_group()


CASES = [
    # B, Sq, Skv, H, D, topk, block, gated, q block sizes, kv block sizes
    (1, 256, 384, 4, 16, 2, 64, True, None, None),
    (2, 256, 256, 6, 8, 3, 64, False, [64, 30, 64, 64], None),
    (1, 512, 256, 2, 16, 1, 128, True, None, [128, 77]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}-H{c[3]}-blk{c[6]}")
def test_ulysses_two_gloo_ranks_equal_the_whole_forward(case):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, q_out)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted([q_out.get(timeout=240) for _ in range(world)], key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, Sq, Skv, H, D, topk, block, gated, qbs, kbs = case
    q, k, v, gate = _inputs(B, Sq, Skv, H, D, 77)
    want, want_idx, want_num = oracle_forward_bshd(q, k, v, gate if gated else None, qbs, kbs,
                                                   topk, None, block)
    sq, Hn = Sq // world, H // world
    for rank, out, idx, num in results:
        assert np.array_equal(out, want[:, rank * sq:(rank + 1) * sq].numpy())
        # rank r ran the forward for head group r
        assert np.array_equal(idx, want_idx[:, rank * Hn:(rank + 1) * Hn].numpy())
        assert np.array_equal(num, want_num[:, rank * Hn:(rank + 1) * Hn].numpy())


def test_specs_invert_each_other():
    """pack then unpack, and gather then scatter, are the identity."""
    B, S, H, N, D = 2, 6, 4, 2, 3
    x = torch.arange(B * S * H * D, dtype=torch.float64).view(B, S, H, D)
    packed = ref_permute(x, *U.pack_heads_spec(B, S, H, N))         # [N, B, S, H/N, D]
    assert torch.equal(packed[1, :, :, 0], x[:, :, 2])
    back = ref_permute(packed, *U.unpack_heads_spec(B, S, H // N, N)).view(B, S, H, D)
    assert torch.equal(back, x)
    y = torch.arange(N * B * S * 2 * D, dtype=torch.float64).view(N, B, S, 2, D)
    full = ref_permute(y, *U.gather_seq_spec(B, S, 2, N)).view(B, N * S, 2, D)
    assert torch.equal(full[:, S:2 * S], y[1])
    again = ref_permute(full, *U.scatter_seq_spec(B, S, 2, N))
    assert torch.equal(again, y)
