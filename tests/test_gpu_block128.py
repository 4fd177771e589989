"""128-token blocks (VSA-128 tiles) on the GPU, through the C ABI, against
the fp64 oracle at block size 128: the tensor-core operand layouts in
isolation, the sparse kernel on supplied indices (ragged blocks, nq != nkv,
empty rows, duplicates, a one-token tile, peaked logits that move the
reference max), the whole forward stage by stage, the bool-mask and BSHD
entries, and the README's VSA-128 shape (B1 H12 D128, 39936 tokens = 312
blocks, top 40) on every query block."""
import numpy as np
import pytest
import torch

from block_sparse_attention_15_b200 import binding as vsa
from block_sparse_attention_15_b200 import inputs as I
from oracle import vsa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"
BLK = 128


def _padded(B, H, sizes, D, seed, stream, scale=1.0, pad_value=0.0):
    n_tok = sum(sizes)
    x = I.normal_bf16((B, H, n_tok, D), seed, stream, scale=scale)
    out = torch.full((B, H, BLK * len(sizes), D), pad_value, dtype=torch.bfloat16)
    src = 0
    for j, m in enumerate(sizes):
        out[:, :, BLK * j:BLK * j + m] = x[:, :, src:src + m]
        src += m
    return out


def _rows(sizes):
    return np.concatenate([np.arange(BLK * j, BLK * j + m) for j, m in enumerate(sizes)])


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("mode", [2, 3])
def test_umma128_layouts(mode, D):
    g = torch.Generator().manual_seed(40 + mode + D)
    if mode == 2:
        a = torch.randn(128, D, generator=g).to(torch.bfloat16)
        b = torch.randn(128, D, generator=g).to(torch.bfloat16)
        want = a.double() @ b.double().T
    else:
        a = torch.rand(128, 128, generator=g).to(torch.bfloat16)
        b = torch.randn(128, D, generator=g).to(torch.bfloat16)
        want = a.double() @ b.double()
    c = vsa.selftest_umma(mode, a.to(DEV), b.to(DEV))
    torch.cuda.synchronize()
    np.testing.assert_allclose(c.cpu().double().numpy(), want.numpy(), rtol=1e-4, atol=1e-3)


def _selection(rng, B, H, nq, nkv, width, allow_dup=False, empty=()):
    idx = np.full((B, H, nq, width), -1, dtype=np.int32)
    num = np.zeros((B, H, nq), dtype=np.int32)
    for b, h, a in np.ndindex(B, H, nq):
        if (b, h, a) in empty:
            continue
        n = int(rng.integers(1, width + 1))
        sel = rng.integers(0, nkv, size=n) if allow_dup else rng.choice(nkv, size=min(n, nkv), replace=False)
        idx[b, h, a, :len(sel)] = sel
        num[b, h, a] = len(sel)
    return idx, num


CASES = [
    # (D, B, H, q_sizes, kv_sizes, width, dup, seed)
    (128, 1, 2, [128] * 5, [128] * 7, 4, False, 1),
    (64, 2, 3, [128, 128, 90, 128], [128, 40, 128, 128, 1, 128], 5, False, 2),
    (128, 1, 3, [128, 7], [128] * 3 + [100], 6, True, 3),
    (128, 1, 1, [128] * 200, [128] * 9, 3, False, 4),   # more items than SMs
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"D{c[0]}-B{c[1]}H{c[2]}-nq{len(c[3])}-nkv{len(c[4])}")
def test_sparse128_from_indices(case):
    D, B, H, qs, ks, width, dup, seed = case
    rng = np.random.default_rng(seed)
    q = _padded(B, H, qs, D, 800 + seed, 0, pad_value=3.0)
    k = _padded(B, H, ks, D, 800 + seed, 1, pad_value=5.0)
    v = _padded(B, H, ks, D, 800 + seed, 2, pad_value=-5.0)
    idx, num = _selection(rng, B, H, len(qs), len(ks), width, dup, empty={(0, 0, 1)})
    out = vsa.block_sparse_attn_from_indices(q.to(DEV), k.to(DEV), v.to(DEV), torch.from_numpy(idx).to(DEV),
                                             torch.from_numpy(num).to(DEV), qs, ks, block=BLK)
    vsa.check_device_status()
    want = O.block_sparse_attention(P.to_np(q), P.to_np(k), P.to_np(v), idx, num, qs, ks,
                                    O.default_scale(D), block=BLK)
    got = P.to_np(out)
    rr = _rows(qs)
    P.assert_outputs_close(got[:, :, rr], want[:, :, rr], "sparse128")
    pad = np.setdiff1d(np.arange(got.shape[2]), rr)
    assert np.all(got[:, :, pad] == 0.0)
    assert np.all(got[0, 0, BLK:BLK + qs[1]] == 0.0)   # the empty selection


def test_sparse128_peaked_logits_move_the_reference():
    """q x 6 and the keys of later blocks x 4: later tiles exceed the first
    tile's maxima by far more than the refresh threshold, so the reference
    max moves and O is rescaled mid-item."""
    B, H, D = 1, 2, 128
    qs, ks = [128] * 3, [128] * 8
    q = _padded(B, H, qs, D, 901, 0, scale=6.0)
    k = _padded(B, H, ks, D, 901, 1)
    k[:, :, 4 * BLK:] *= 4
    v = _padded(B, H, ks, D, 901, 2)
    idx = np.broadcast_to(np.arange(8, dtype=np.int32), (B, H, 3, 8)).copy()
    num = np.full((B, H, 3), 8, dtype=np.int32)
    out = vsa.block_sparse_attn_from_indices(q.to(DEV), k.to(DEV), v.to(DEV), torch.from_numpy(idx).to(DEV),
                                             torch.from_numpy(num).to(DEV), block=BLK)
    vsa.check_device_status()
    want = O.block_sparse_attention(P.to_np(q), P.to_np(k), P.to_np(v), idx, num, qs, ks,
                                    O.default_scale(D), block=BLK)
    P.assert_outputs_close(P.to_np(out), want, "sparse128 peaked")


FWD_CASES = [
    (128, True, [128] * 6, [128] * 9, 3, 11),
    (128, False, [128, 128, 128, 50], [128, 60, 128, 128, 128], 2, 12),
    (64, True, [128] * 4 + [1], [128] * 5, 5, 13),
]


@pytest.mark.parametrize("case", FWD_CASES, ids=lambda c: f"D{c[0]}-{'gated' if c[1] else 'ungated'}-nq{len(c[2])}")
def test_forward128(case):
    D, gated, qs, ks, topk, seed = case
    B, H = 1, 3
    q, k, v = (_padded(B, H, s, D, 950 + seed, i) for i, s in enumerate((qs, ks, ks)))
    gate = I.gate_bf16((B, BLK * len(qs), H, D), 950 + seed) if gated else None
    out, idx, num, out_c, pooled = vsa.vsa_forward(
        q.to(DEV), k.to(DEV), v.to(DEV), None if gate is None else gate.to(DEV), qs, ks, topk=topk,
        return_out_c=True, return_pooled=True, block=BLK)
    vsa.check_device_status()
    qn, kn, vn = P.to_np(q), P.to_np(k), P.to_np(v)
    scale = O.default_scale(D)
    for got_p, x, sizes in zip(pooled, (qn, kn, vn), (qs, ks, ks)):
        np.testing.assert_allclose(P.to_np(got_p), O.block_pool(x, sizes, block=BLK), rtol=1e-5, atol=1e-6)
    qc, kc, vc = (O.block_pool(x, s, block=BLK) for x, s in ((qn, qs), (kn, ks), (vn, ks)))
    scores, oc = O.coarse_attention(qc, kc, vc, scale)
    np.testing.assert_allclose(P.to_np(out_c), oc, rtol=1e-4, atol=1e-6)
    P.check_topk(P.to_np(idx), P.to_np(num), scores, topk)
    o_s = O.block_sparse_attention(qn, kn, vn, P.to_np(idx), P.to_np(num), qs, ks, scale, block=BLK)
    want = O.combine(oc, o_s, None if gate is None else P.to_np(gate), qs, block=BLK)
    got = P.to_np(out)
    rr = _rows(qs)
    P.assert_outputs_close(got[:, :, rr], want[:, :, rr], "forward128")
    pad = np.setdiff1d(np.arange(got.shape[2]), rr)
    assert np.all(got[:, :, pad] == 0.0)


def test_block128_bool_mask_and_bshd():
    B, H, D = 1, 2, 128
    qs, ks = [128] * 4, [128] * 6
    q, k, v = (_padded(B, H, s, D, 990, i) for i, s in enumerate((qs, ks, ks)))
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    rng = np.random.default_rng(9)
    bm = rng.random((B, H, 4, 6)) < 0.4
    bm[0, 1, 2] = False
    out, idx, num = vsa.block_sparse_attn(qd, kd, vd, torch.from_numpy(bm).to(DEV), block=BLK,
                                          return_indices=True)
    ref = vsa.block_sparse_attn_from_indices(qd, kd, vd, idx, num, block=BLK)
    vsa.check_device_status()
    wi, wn = O.block_map_to_indices(bm)
    assert np.array_equal(P.to_np(idx), wi) and np.array_equal(P.to_np(num), wn)
    assert torch.equal(out, ref)
    gate = I.gate_bf16((B, BLK * 4, H, D), 991).to(DEV)
    o1, i1, n1 = vsa.vsa_forward(qd, kd, vd, gate, topk=2, block=BLK)
    qb, kb, vb = (x.transpose(1, 2).contiguous() for x in (qd, kd, vd))
    o2, i2, n2 = vsa.video_sparse_attn_bshd(qb, kb, vb, gate, topk=2, block=BLK)
    vsa.check_device_status()
    assert torch.equal(i1, i2) and torch.equal(n1, n2)
    assert torch.equal(o2.transpose(1, 2), o1)


def test_vsa128_readme_shape_full():
    """The README's VSA-128 benchmark shape: B1 H12 D128, 39936 tokens
    (312 blocks of 128), top 40, gated; every query block against the
    oracle."""
    B, H, D, nb, topk, seed = 1, 12, 128, 312, 40, 1006
    sizes = [128] * nb
    q, k, v = (_padded(B, H, sizes, D, seed, i) for i in range(3))
    gate = I.gate_bf16((B, BLK * nb, H, D), seed)
    out, idx, num, out_c = vsa.vsa_forward(q.to(DEV), k.to(DEV), v.to(DEV), gate.to(DEV), topk=topk,
                                           return_out_c=True, block=BLK)
    vsa.check_device_status()
    qn, kn, vn = P.to_np(q), P.to_np(k), P.to_np(v)
    scale = O.default_scale(D)
    qc, kc, vc = (O.block_pool(x, sizes, block=BLK) for x in (qn, kn, vn))
    scores, oc = O.coarse_attention(qc, kc, vc, scale)
    np.testing.assert_allclose(P.to_np(out_c), oc, rtol=1e-4, atol=1e-6)
    idx_np, num_np = P.to_np(idx), P.to_np(num)
    P.check_topk(idx_np, num_np, scores, topk)
    o_s = O.block_sparse_attention(qn, kn, vn, idx_np, num_np, sizes, sizes, scale, block=BLK)
    want = O.combine(oc, o_s, P.to_np(gate), sizes, block=BLK)
    P.assert_outputs_close(P.to_np(out), want, "VSA-128 README shape")
