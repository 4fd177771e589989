"""vsa_forward_noalloc: the allocation-free variant of vsa_forward.

Some callers cannot allocate device memory while they run (a serving loop
under a fixed memory budget, a plugin whose host owns all device memory), so
this entry point keeps its scratch in a fixed array inside the library
instead of a caller workspace.  These tests call it through the C ABI and
check it against the regular vsa_forward on the same inputs, twice in a row
(the second call with different inputs, so stale scratch from the first call
would show).  Both entry points run the same kernels with the same launch
sequence on the same inputs, only with their scratch in different memory, so
the results must be identical bit for bit.  The file sorts last so that a run stopping at the first failure
has already run every other test.
"""
import ctypes

import pytest
import torch

from block_sparse_attention_15_b200 import binding as vsa
from block_sparse_attention_15_b200 import inputs as I

DEV = "cuda"


def _noalloc(q, k, v, gate, topk, out, idx, num, out_c=None):
    B, H, Sq, D = q.shape
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return vsa.lib().vsa_forward_noalloc(p(q), p(k), p(v), p(gate), None, None, B, H, Sq,
                                         k.shape[2], D, topk, 0.0, p(out), p(idx), p(num),
                                         idx.shape[-1], p(out_c), stream)


def _case(seed, H, nq, nkv, D=128):
    q = I.padded_normal_bhsd(1, H, [64] * nq, D, seed, 0).to(DEV)
    k = I.padded_normal_bhsd(1, H, [64] * nkv, D, seed, 1).to(DEV)
    v = I.padded_normal_bhsd(1, H, [64] * nkv, D, seed, 2).to(DEV)
    gate = I.gate_bf16((1, 64 * nq, H, D), seed).to(DEV)
    return q, k, v, gate


@pytest.mark.gpu
def test_noalloc_matches_vsa_forward_twice():
    cases = [(4100, 4, 20, 24, 6), (4101, 3, 17, 11, 4)]
    for seed, H, nq, nkv, topk in cases:
        q, k, v, gate = _case(seed, H, nq, nkv)
        want_out, want_idx, want_num, want_oc = vsa.vsa_forward(q, k, v, gate, topk=topk,
                                                                return_out_c=True)
        out = torch.empty_like(q)
        idx = torch.empty_like(want_idx)
        num = torch.empty_like(want_num)
        out_c = torch.empty_like(want_oc)
        assert _noalloc(q, k, v, gate, topk, out, idx, num, out_c) == 0
        vsa.check_device_status()
        assert torch.equal(idx, want_idx) and torch.equal(num, want_num)
        assert torch.equal(out, want_out), "noalloc output differs from vsa_forward"
        assert torch.equal(out_c, want_oc), "noalloc out_c differs from vsa_forward"


@pytest.mark.gpu
def test_noalloc_coarse_output_kept_inside():
    q, k, v, gate = _case(4102, 2, 9, 9)
    want_out, want_idx, _ = vsa.vsa_forward(q, k, v, gate, topk=3)
    out = torch.empty_like(q)
    idx = torch.empty_like(want_idx)
    num = torch.empty((1, 2, 9), dtype=torch.int32, device=DEV)
    assert _noalloc(q, k, v, gate, 3, out, idx, num) == 0   # out_c NULL: kept in the array
    vsa.check_device_status()
    assert torch.equal(idx, want_idx)
    assert torch.equal(out, want_out), "noalloc (out_c internal) differs from vsa_forward"


def test_noalloc_rejects_sizes_beyond_the_array():
    """56 heads x 2048 + 2048 blocks of fp32 scratch is far above 32 MiB: the
    call must refuse on the host, before touching any pointer."""
    fake = ctypes.c_void_p(1 << 20)
    rc = vsa.lib().vsa_forward_noalloc(fake, fake, fake, None, None, None, 1, 56, 64 * 2048,
                                       64 * 2048, 128, 48, 0.0, fake, fake, fake, 48, None, None)
    assert rc == 7  # VSA_ERR_WORKSPACE
