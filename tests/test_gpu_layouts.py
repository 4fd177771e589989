"""Layouts and the bool-mask entry on the GPU, through the C ABI:

* the bool block map (block_sparse_attn) gives the oracle's index rows bit
  for bit and the same output as the index entry on those rows;
* the index entry with its logit-bound pass gives the same bits as without
  it (the bound only skips a check whose outcome it proves);
* the BSHD forward and forwards on strided views (slices of a fused QKV
  tensor, a transposed gate, an output inside a wider buffer) give the same
  bits as the contiguous BHSD forward on the same values, and match the
  oracle.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_15_b200 import binding as vsa
from block_sparse_attention_15_b200 import inputs as I
from oracle import vsa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bhsd(B, H, sizes, D, seed, stream, scale=1.0):
    return I.padded_normal_bhsd(B, H, sizes, D, seed, stream, scale=scale)


@pytest.mark.parametrize("D", [64, 128])
def test_bool_mask_matches_index_entry_and_oracle(D):
    B, H = 2, 3
    qs, ks = [64] * 6 + [17], [64] * 9 + [40] + [64]
    nq, nkv = len(qs), len(ks)
    q, k, v = (_bhsd(B, H, s, D, 500 + D, i) for i, s in enumerate((qs, ks, ks)))
    rng = np.random.default_rng(5)
    bm = rng.random((B, H, nq, nkv)) < 0.35
    bm[0, 0, 0] = False          # an empty row
    bm[1, 2, 3] = True           # a full row
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out, idx, num = vsa.block_sparse_attn(qd, kd, vd, torch.from_numpy(bm).to(DEV), qs, ks,
                                          return_indices=True)
    vsa.check_device_status()
    want_idx, want_num = O.block_map_to_indices(bm)
    assert np.array_equal(P.to_np(idx), want_idx) and np.array_equal(P.to_np(num), want_num)
    ref = vsa.block_sparse_attn_from_indices(qd, kd, vd, idx, num, qs, ks)
    assert torch.equal(out, ref)
    want = O.block_sparse_attention(P.to_np(q), P.to_np(k), P.to_np(v), want_idx, want_num, qs, ks,
                                    O.default_scale(D))
    rr = P.real_rows(qs)
    got = P.to_np(out)
    P.assert_outputs_close(got[:, :, rr], want[:, :, rr], "bool mask")
    assert np.all(got[0, 0, :64] == 0.0)


def _within_rounding(a, b):
    """Two bf16 results of the same attention computed with different
    reference maxima: equal up to rounding -- elements differ by a bf16 ulp
    or two (relative 2^-8 each), so the relative RMS difference stays under
    two ulps, inside the oracle tolerance."""
    a, b = a.double(), b.double()
    assert (a - b).abs().max().item() <= 2e-3 + 1e-2 * b.abs().max().item()
    assert ((a - b).norm() / b.norm()).item() <= 8e-3


@pytest.mark.parametrize("scale_q", [1.0, 6.0])
def test_logit_bound_pass_changes_only_rounding(scale_q):
    """N(0,1) inputs: the bound (<= 60 log2 units) becomes the reference max
    and the items skip the running-max work, which changes the probabilities
    only by a common factor per column (so the results only by rounding);
    peaked inputs (q x 6): the bound is too loose and the kernel takes the
    same steps with or without it (the same bits)."""
    B, H, D = 1, 4, 128
    qs, ks = [64] * 20, [64] * 30
    q = _bhsd(B, H, qs, D, 610, 0, scale=scale_q).to(DEV)
    k, v = (_bhsd(B, H, ks, D, 610, i).to(DEV) for i in (1, 2))
    rng = np.random.default_rng(6)
    idx = np.stack([np.sort(rng.choice(30, size=12, replace=False)) for _ in range(B * H * 20)])
    idx = torch.from_numpy(idx.reshape(B, H, 20, 12).astype(np.int32)).to(DEV)
    num = torch.full((B, H, 20), 12, dtype=torch.int32, device=DEV)
    with_bound = vsa.block_sparse_attn_from_indices(q, k, v, idx, num, logit_bound=True)
    without = vsa.block_sparse_attn_from_indices(q, k, v, idx, num, logit_bound=False)
    vsa.check_device_status()
    if scale_q > 1.0:
        assert torch.equal(with_bound, without)
    else:
        _within_rounding(with_bound, without)
    want = O.block_sparse_attention(P.to_np(q), P.to_np(k), P.to_np(v), P.to_np(idx), P.to_np(num),
                                    qs, ks, O.default_scale(D))
    P.assert_outputs_close(P.to_np(with_bound), want, "from indices with the bound")
    P.assert_outputs_close(P.to_np(without), want, "from indices without the bound")


@pytest.mark.parametrize("D,gated", [(128, True), (64, False)])
def test_bshd_forward_equals_bhsd(D, gated):
    B, H = 2, 3
    qs, ks = [64] * 9 + [33], [64] * 7 + [10] + [64] * 4
    q, k, v = (_bhsd(B, H, s, D, 700 + D, i) for i, s in enumerate((qs, ks, ks)))
    gate = I.gate_bf16((B, 64 * len(qs), H, D), 700 + D) if gated else None
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    gd = None if gate is None else gate.to(DEV)
    out, idx, num = vsa.vsa_forward(qd, kd, vd, gd, qs, ks, topk=5)
    # BSHD copies of the same values
    qb, kb, vb = (x.transpose(1, 2).contiguous() for x in (qd, kd, vd))
    out_b, idx_b, num_b = vsa.video_sparse_attn_bshd(qb, kb, vb, gd, qs, ks, topk=5)
    vsa.check_device_status()
    assert out_b.shape == (B, 64 * len(qs), H, D)
    assert torch.equal(idx_b, idx) and torch.equal(num_b, num)
    assert torch.equal(out_b.transpose(1, 2), out)
    # and against the oracle
    qn, kn, vn = P.to_np(q), P.to_np(k), P.to_np(v)
    scale = O.default_scale(D)
    qc, kc, vc = (O.block_pool(x, s) for x, s in ((qn, qs), (kn, ks), (vn, ks)))
    scores, oc = O.coarse_attention(qc, kc, vc, scale)
    P.check_topk(P.to_np(idx), P.to_np(num), scores, 5)
    o_s = O.block_sparse_attention(qn, kn, vn, P.to_np(idx), P.to_np(num), qs, ks, scale)
    want = O.combine(oc, o_s, None if gate is None else P.to_np(gate), qs)
    rr = P.real_rows(qs)
    P.assert_outputs_close(P.to_np(out_b.transpose(1, 2))[:, :, rr], want[:, :, rr], "BSHD")


def test_strided_views_equal_contiguous():
    """q, k, v sliced out of one fused [B, S, 3, H, D] tensor, the gate as
    [B, S, H, D] memory, the output written into every other 128-wide
    column group of a wider buffer."""
    B, H, D = 1, 4, 128
    nb = 12
    S = 64 * nb
    g = torch.Generator().manual_seed(9)
    qkv = torch.randn(B, S, 3, H, D, generator=g).to(torch.bfloat16).to(DEV)
    q, k, v = (qkv[:, :, i].transpose(1, 2) for i in range(3))   # [B, H, S, D] views
    gate = I.gate_bf16((B, S, H, D), 901).to(DEV)
    wide = torch.zeros(B, H, S, 2 * D, dtype=torch.bfloat16, device=DEV)
    out_view = wide[..., D:]
    out, idx, num = vsa.vsa_forward(q, k, v, gate, topk=4, out=out_view)
    vsa.check_device_status()
    assert out.data_ptr() == out_view.data_ptr()
    ref, ridx, rnum = vsa.vsa_forward(q.contiguous(), k.contiguous(), v.contiguous(), gate, topk=4)
    assert torch.equal(idx, ridx) and torch.equal(num, rnum)
    assert torch.equal(out_view, ref)
    assert torch.count_nonzero(wide[..., :D]) == 0
    # the index entry on the same views
    o2 = vsa.block_sparse_attn_from_indices(q, k, v, idx, num)
    r2 = vsa.block_sparse_attn_from_indices(q.contiguous(), k.contiguous(), v.contiguous(), idx, num)
    assert torch.equal(o2, r2)


def test_misaligned_stride_is_refused_on_the_host():
    """A sequence stride of 68 elements (136 bytes) cannot be a TMA stride:
    the binding refuses it before anything is launched."""
    B, H, D = 1, 2, 64
    q = torch.zeros(B, H, 128, D + 4, dtype=torch.bfloat16, device=DEV)[..., :D]
    k = torch.zeros(B, H, 128, D, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError):
        vsa.vsa_forward(q, k, k, topk=1)
