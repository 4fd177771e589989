"""The sequence-parallel wrapper's kernels on the GPU: the library's row
permutation (vsa_permute_rows) against the reference gather on the four
reshard specs, bit for bit; and the whole wrapper on a one-rank NCCL group
(where it calls the forward directly) equal to the single-GPU BSHD forward
bit for bit.  (The exchange order across several ranks is covered on the CPU
with two gloo ranks in test_ulysses_multirank.py; this run has one GPU.)"""
import os
import socket

import pytest
import torch
import torch.distributed as dist

from block_sparse_attention_15_b200 import binding as vsa
from block_sparse_attention_15_b200 import inputs as I
from block_sparse_attention_15_b200 import ulysses as U
from tests.test_ulysses_multirank import ref_permute

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("N", [1, 2, 4])
def test_permute_rows_matches_reference_gather(N):
    B, S, H, D = 2, 96, 8, 128
    Hn = H // N
    x = I.normal_bf16((B, S, H, D), 3, 0).to(DEV)
    y = I.normal_bf16((N, B, S, Hn, D), 3, 1).to(DEV)
    big = I.normal_bf16((B, N * S, Hn, D), 3, 2).to(DEV)
    for src, spec in ((x, U.pack_heads_spec(B, S, H, N)), (y, U.gather_seq_spec(B, S, Hn, N)),
                      (big, U.scatter_seq_spec(B, S, Hn, N)), (y, U.unpack_heads_spec(B, S, Hn, N))):
        got = vsa.permute_rows(src, *spec)
        want = ref_permute(src.cpu(), *spec)
        assert torch.equal(got.cpu(), want)


def test_ulysses_one_rank_equals_single_gpu_forward():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device(DEV, 0))
    try:
        B, H, D = 1, 4, 128
        qs, ks = [64] * 6, [64] * 5 + [20]
        q = I.padded_normal_bhsd(B, H, qs, D, 55, 0).transpose(1, 2).contiguous().to(DEV)
        k = I.padded_normal_bhsd(B, H, ks, D, 55, 1).transpose(1, 2).contiguous().to(DEV)
        v = I.padded_normal_bhsd(B, H, ks, D, 55, 2).transpose(1, 2).contiguous().to(DEV)
        gate = I.gate_bf16((B, 64 * len(qs), H, D), 55).to(DEV)
        out, idx, num = U.vsa_forward_ulysses(q, k, v, gate, None, ks, topk=3)
        ref, ridx, rnum = vsa.video_sparse_attn_bshd(q, k, v, gate, None, ks, topk=3)
        vsa.check_device_status()
        assert torch.equal(idx, ridx) and torch.equal(num, rnum)
        assert torch.equal(out, ref)
    finally:
        dist.destroy_process_group()
