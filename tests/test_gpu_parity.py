"""GPU parity at oracle-sized cases: every entry point through the C ABI
against the fp64 CPU oracle on the same seeded inputs, with several tiles,
ragged tails and the degenerate cases."""
import numpy as np
import pytest
import torch

from block_sparse_attention_15_b200 import binding as vsa
from block_sparse_attention_15_b200 import inputs as I
from oracle import vsa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _bhsd(B, H, sizes, D, seed, stream, pad_value=0.0, scale=1.0):
    return I.padded_normal_bhsd(B, H, sizes, D, seed, stream, pad_value=pad_value, scale=scale)


# ---------------------------------------------------------------------------
# tensor-core operand layouts in isolation
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("mode", [0, 1])
def test_umma_layouts(mode, D):
    g = torch.Generator().manual_seed(7 + mode + D)
    a = torch.randn(128, D, generator=g).to(torch.bfloat16)
    b = torch.randn(64 if mode == 0 else 128, D if mode == 0 else 64, generator=g).to(torch.bfloat16)
    c = vsa.selftest_umma(mode, a.to(DEV), b.to(DEV))
    torch.cuda.synchronize()
    if mode == 0:
        want = a.double() @ b.double().T
    else:
        want = a.double().T @ b.double()
    np.testing.assert_allclose(c.cpu().double().numpy(), want.numpy(), rtol=1e-4, atol=1e-3)


# ---------------------------------------------------------------------------
# a4: block-sparse attention from supplied indices
# ---------------------------------------------------------------------------
def _random_selection(rng, B, H, nq, nkv, width, min_n=1, allow_dup=False):
    idx = np.full((B, H, nq, width), -1, dtype=np.int32)
    num = np.zeros((B, H, nq), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for a in range(nq):
                n = int(rng.integers(min_n, width + 1))
                if allow_dup:
                    sel = rng.integers(0, nkv, size=n)
                else:
                    sel = rng.choice(nkv, size=min(n, nkv), replace=False)
                    n = len(sel)
                idx[b, h, a, :n] = sel
                num[b, h, a] = n
    return idx, num


SPARSE_CASES = [
    # B, H, D, q sizes, kv sizes, width
    (1, 2, 128, [64] * 4, [64] * 6, 3),
    (2, 3, 128, [64, 64, 30, 64, 1], [64, 7, 64, 64, 64, 40, 64], 5),
    (1, 2, 64, [64] * 8, [64] * 8, 2),
    (1, 1, 64, [64, 33], [12, 64, 64], 3),
    (1, 4, 128, [64] * 9, [64] * 20, 20),
]


@pytest.mark.parametrize("case", SPARSE_CASES, ids=lambda c: f"B{c[0]}H{c[1]}D{c[2]}nq{len(c[3])}nkv{len(c[4])}w{c[5]}")
def test_sparse_from_indices(case):
    B, H, D, qs, ks, width = case
    rng = np.random.default_rng(len(qs) * 31 + width)
    q = _bhsd(B, H, qs, D, 11, 0)
    k = _bhsd(B, H, ks, D, 11, 1, pad_value=3.0)   # finite non-zero padding must be masked
    v = _bhsd(B, H, ks, D, 11, 2, pad_value=-3.0)
    idx, num = _random_selection(rng, B, H, len(qs), len(ks), width)
    out = vsa.block_sparse_attn_from_indices(
        q.to(DEV), k.to(DEV), v.to(DEV), torch.from_numpy(idx).to(DEV), torch.from_numpy(num).to(DEV),
        qs, ks)
    vsa.check_device_status()
    want = O.block_sparse_attention(P.to_np(q), P.to_np(k), P.to_np(v), idx, num, qs, ks,
                                    O.default_scale(D))
    got = P.to_np(out)
    rr = P.real_rows(qs)
    P.assert_outputs_close(got[:, :, rr], want[:, :, rr])
    pad = np.setdiff1d(np.arange(got.shape[2]), rr)
    assert np.all(got[:, :, pad] == 0.0), "padded query rows must be written as 0"


@pytest.mark.parametrize("D", [128, 64])
def test_sparse_many_items_mixed_counts(D):
    """More work items than SMs, so each CTA of the persistent grid walks
    several items: selection counts vary per item (0, odd, longer than the
    K/V rings), blocks are ragged, entries repeat."""
    B, H = 1, 8
    qs = [64] * 63 + [17]
    ks = [64] * 10 + [5, 64, 64, 33, 64, 64]
    width = 13
    rng = np.random.default_rng(77 + D)
    q = _bhsd(B, H, qs, D, 16, 0)
    k = _bhsd(B, H, ks, D, 16, 1, pad_value=2.0)
    v = _bhsd(B, H, ks, D, 16, 2, pad_value=-2.0)
    idx = np.full((B, H, len(qs), width), -1, dtype=np.int32)
    num = rng.integers(0, width + 1, size=(B, H, len(qs))).astype(np.int32)
    for b in range(B):
        for h in range(H):
            for a in range(len(qs)):
                idx[b, h, a, :num[b, h, a]] = rng.integers(0, len(ks), size=num[b, h, a])
    out = vsa.block_sparse_attn_from_indices(
        q.to(DEV), k.to(DEV), v.to(DEV), torch.from_numpy(idx).to(DEV), torch.from_numpy(num).to(DEV),
        qs, ks)
    vsa.check_device_status()
    want = O.block_sparse_attention(P.to_np(q), P.to_np(k), P.to_np(v), idx, num, qs, ks,
                                    O.default_scale(D))
    got = P.to_np(out)
    rr = P.real_rows(qs)
    P.assert_outputs_close(got[:, :, rr], want[:, :, rr])
    assert np.all(got[:, :, np.setdiff1d(np.arange(got.shape[2]), rr)] == 0.0)


def test_sparse_edge_cases():
    """q2k_num = 0, a single one-token KV block, repeated entries, odd counts."""
    B, H, D = 1, 2, 128
    qs, ks = [64] * 4, [64, 1, 64, 64, 64]
    q = _bhsd(B, H, qs, D, 12, 0)
    k = _bhsd(B, H, ks, D, 12, 1)
    v = _bhsd(B, H, ks, D, 12, 2)
    idx = np.full((B, H, 4, 4), -1, dtype=np.int32)
    num = np.zeros((B, H, 4), dtype=np.int32)
    idx[:, :, 0, :0] = 0                      # block 0: empty selection
    idx[:, :, 1, :1] = [1]; num[:, :, 1] = 1  # block 1: the one-token block only
    idx[:, :, 2, :3] = [4, 4, 0]; num[:, :, 2] = 3  # repeated entry, odd count
    idx[:, :, 3, :4] = [3, 2, 1, 0]; num[:, :, 3] = 4  # unsorted
    out = vsa.block_sparse_attn_from_indices(
        q.to(DEV), k.to(DEV), v.to(DEV), torch.from_numpy(idx).to(DEV), torch.from_numpy(num).to(DEV),
        qs, ks)
    vsa.check_device_status()
    got = P.to_np(out)
    want = O.block_sparse_attention(P.to_np(q), P.to_np(k), P.to_np(v), idx, num, qs, ks,
                                    O.default_scale(D))
    assert np.all(got[:, :, :64] == 0.0)
    vrow = P.to_np(v)[:, :, 64]
    np.testing.assert_allclose(got[:, :, 64:128], np.broadcast_to(vrow[:, :, None], (B, H, 64, D)),
                               atol=1e-2)
    P.assert_outputs_close(got, want)


def test_sparse_peaked_softmax_rescale():
    """Queries scaled x8 and the keys of blocks 4-11 a further x4 put later
    logits far (tens to hundreds of log2 units) above the first step's max,
    so the running-max refresh and O rescale path must run."""
    B, H, D = 1, 2, 128
    qs, ks = [64] * 3, [64] * 12
    q = _bhsd(B, H, qs, D, 13, 0, scale=8.0)
    k = _bhsd(B, H, ks, D, 13, 1)
    k[:, :, 256:] *= 4
    v = _bhsd(B, H, ks, D, 13, 2)
    idx = np.broadcast_to(np.arange(12, dtype=np.int32), (B, H, 3, 12)).copy()
    num = np.full((B, H, 3), 12, dtype=np.int32)
    out = vsa.block_sparse_attn_from_indices(
        q.to(DEV), k.to(DEV), v.to(DEV), torch.from_numpy(idx).to(DEV), torch.from_numpy(num).to(DEV))
    vsa.check_device_status()
    want = O.block_sparse_attention(P.to_np(q), P.to_np(k), P.to_np(v), idx, num, qs, ks,
                                    O.default_scale(D))
    P.assert_outputs_close(P.to_np(out), want)


def test_sparse_out_of_range_index_sets_status():
    B, H, D = 1, 1, 128
    q = _bhsd(B, H, [64] * 2, D, 14, 0)
    k = _bhsd(B, H, [64] * 3, D, 14, 1)
    idx = torch.tensor([[[[0, 7], [1, 2]]]], dtype=torch.int32)
    num = torch.tensor([[[2, 2]]], dtype=torch.int32)
    vsa.check_device_status()
    vsa.block_sparse_attn_from_indices(q.to(DEV), k.to(DEV), k.to(DEV), idx.to(DEV), num.to(DEV))
    assert vsa.get_device_status() == 6  # VSA_ERR_INDEX_RANGE
    assert vsa.get_device_status() == 0  # read clears it


def test_bad_block_size_sets_status():
    B, H, D = 1, 1, 128
    q = _bhsd(B, H, [64] * 2, D, 15, 0)
    vsa.check_device_status()
    vsa.vsa_forward(q.to(DEV), q.to(DEV), q.to(DEV), None, [64, 0], [64, 65], topk=1)
    assert vsa.get_device_status() == 8  # VSA_ERR_BLOCK_SIZE


# ---------------------------------------------------------------------------
# a1-a5: the whole forward
# ---------------------------------------------------------------------------
FORWARD_CASES = [
    # name, B, H, D, q sizes, kv sizes, topk, gated
    ("tiny", 1, 2, 64, [64] * 8, [64] * 8, 2, True),
    ("tiny-ungated", 1, 2, 64, [64] * 8, [64] * 8, 2, False),
    ("asym-ragged", 2, 3, 128, [64, 64, 64, 20, 64, 64, 64, 64, 64, 9],
     [64] * 5 + [3] + [64] * 6 + [50], 5, True),
    ("single-kv-block", 1, 2, 128, [64] * 3, [64], 4, True),
    ("single-q-block", 1, 2, 128, [37], [64] * 6, 3, False),
    ("dense-topk-all", 1, 2, 128, [64] * 6, [64] * 6, 6, True),
    ("odd-k", 1, 3, 128, [64] * 12, [64] * 16, 7, True),
]


@pytest.mark.parametrize("case", FORWARD_CASES, ids=lambda c: c[0])
def test_vsa_forward(case):
    name, B, H, D, qs, ks, topk, gated = case
    seed = 1001 if name.startswith("tiny") else 2000 + len(qs)
    q = _bhsd(B, H, qs, D, seed, 0)
    k = _bhsd(B, H, ks, D, seed, 1)
    v = _bhsd(B, H, ks, D, seed, 2)
    gate = I.gate_bf16((B, 64 * len(qs), H, D), seed) if gated else None
    out, idx, num, out_c, pooled = vsa.vsa_forward(
        q.to(DEV), k.to(DEV), v.to(DEV), None if gate is None else gate.to(DEV), qs, ks, topk=topk,
        return_out_c=True, return_pooled=True)
    vsa.check_device_status()
    qn, kn, vn = P.to_np(q), P.to_np(k), P.to_np(v)
    scale = O.default_scale(D)
    # a1: pooled q/k/v (fp32 sums vs fp64)
    for got, x, sizes in zip(pooled, (qn, kn, vn), (qs, ks, ks)):
        np.testing.assert_allclose(P.to_np(got), O.block_pool(x, sizes), rtol=1e-5, atol=1e-6)
    qc, kc, vc = (O.block_pool(x, s) for x, s in ((qn, qs), (kn, ks), (vn, ks)))
    scores, oc_want = O.coarse_attention(qc, kc, vc, scale)
    # a2: coarse output
    np.testing.assert_allclose(P.to_np(out_c), oc_want, rtol=1e-4, atol=1e-6)
    # a3: selection (bit-exact up to near-ties)
    P.check_topk(P.to_np(idx), P.to_np(num), scores, topk)
    # a4 + a5 on the GPU's (validated) selection
    o_s = O.block_sparse_attention(qn, kn, vn, P.to_np(idx), P.to_np(num), qs, ks, scale)
    want = O.combine(oc_want, o_s, None if gate is None else P.to_np(gate), qs)
    got = P.to_np(out)
    rr = P.real_rows(qs)
    P.assert_outputs_close(got[:, :, rr], want[:, :, rr])
    pad = np.setdiff1d(np.arange(got.shape[2]), rr)
    assert np.all(got[:, :, pad] == 0.0)


def _forward_vs_oracle(q, k, v, gate, qs, ks, topk):
    out, idx, num, out_c = vsa.vsa_forward(
        q.to(DEV), k.to(DEV), v.to(DEV), None if gate is None else gate.to(DEV), qs, ks, topk=topk,
        return_out_c=True)
    vsa.check_device_status()
    qn, kn, vn = P.to_np(q), P.to_np(k), P.to_np(v)
    scale = O.default_scale(q.shape[-1])
    qc, kc, vc = (O.block_pool(x, s) for x, s in ((qn, qs), (kn, ks), (vn, ks)))
    scores, oc_want = O.coarse_attention(qc, kc, vc, scale)
    P.check_topk(P.to_np(idx), P.to_np(num), scores, topk)
    o_s = O.block_sparse_attention(qn, kn, vn, P.to_np(idx), P.to_np(num), qs, ks, scale)
    want = O.combine(oc_want, o_s, None if gate is None else P.to_np(gate), qs)
    got = P.to_np(out)
    rr = P.real_rows(qs)
    P.assert_outputs_close(got[:, :, rr], want[:, :, rr])
    pad = np.setdiff1d(np.arange(got.shape[2]), rr)
    assert np.all(got[:, :, pad] == 0.0)


def test_forward_large_late_keys_rescale():
    """Keys of the later blocks x16: logits far above the first step's max, so
    the forward's running-max refresh and rescale must run."""
    B, H, D = 1, 2, 128
    qs, ks = [64] * 4, [64] * 10
    q = _bhsd(B, H, qs, D, 2400, 0, scale=2.0)
    k = _bhsd(B, H, ks, D, 2400, 1)
    k[:, :, 256:] *= 16
    v = _bhsd(B, H, ks, D, 2400, 2)
    gate = I.gate_bf16((B, 64 * len(qs), H, D), 2400)
    _forward_vs_oracle(q, k, v, gate, qs, ks, topk=10)


def test_forward_large_padding_rows():
    """Padding rows of a partial query block hold large values: their logits
    are computed in the block's tile but must not reach any real row, and the
    padding rows of the output stay zero."""
    B, H, D = 1, 2, 128
    qs, ks = [64, 17, 64], [64] * 6
    q = _bhsd(B, H, qs, D, 2500, 0, pad_value=30.0)
    k = _bhsd(B, H, ks, D, 2500, 1)
    v = _bhsd(B, H, ks, D, 2500, 2)
    _forward_vs_oracle(q, k, v, None, qs, ks, topk=4)


def test_forward_logit_bound_holds():
    """The workspace's per-query-block bound is at least scale*log2(e)*q.k for
    every query row of the block (padding rows included) and every key row of
    the head, within 1% of the norm product, and the stored block norms equal
    the largest row norms (padding rows count for queries, not for keys)."""
    B, H, D = 1, 3, 128
    qs, ks = [64, 64, 40], [64, 64, 64, 23]
    q = _bhsd(B, H, qs, D, 2600, 0, pad_value=3.0)
    k = _bhsd(B, H, ks, D, 2600, 1)
    k[:, 1] *= 3
    v = _bhsd(B, H, ks, D, 2600, 2)
    nq, nkv = len(qs), len(ks)
    ws = torch.zeros(vsa.lib().vsa_forward_workspace_size(B, H, nq, nkv, D), dtype=torch.uint8, device=DEV)
    vsa.vsa_forward(q.to(DEV), k.to(DEV), v.to(DEV), None, qs, ks, topk=2, workspace=ws)
    vsa.check_device_status()
    a256 = lambda x: (x + 255) // 256 * 256
    g = B * H * D * 4
    off = a256(g * nq) * 2 + a256(g * nkv) * 2
    G = B * H
    norms = ws[off:off + 4 * G * (2 * nq + nkv)].view(torch.float32).cpu().numpy().astype(np.float64)
    qn_got = norms[:G * nq].reshape(B, H, nq)
    kn_got = norms[G * nq:G * (nq + nkv)].reshape(B, H, nkv)
    bound = norms[G * (nq + nkv):].reshape(B, H, nq)
    qq, kk = P.to_np(q), P.to_np(k)
    row_q = np.linalg.norm(qq, axis=-1).reshape(B, H, nq, 64)
    row_k = np.linalg.norm(kk, axis=-1).reshape(B, H, nkv, 64)
    np.testing.assert_allclose(qn_got, row_q.max(-1), rtol=1e-6)
    kmask = np.arange(64)[None, :] < np.array(ks)[:, None]
    np.testing.assert_allclose(kn_got, np.where(kmask, row_k, 0.0).max(-1), rtol=1e-6)
    c = O.default_scale(D) / np.log(2.0)
    kreal = np.concatenate([np.arange(64 * j, 64 * j + n) for j, n in enumerate(ks)])
    for b in range(B):
        for h in range(H):
            logits = c * qq[b, h] @ kk[b, h, kreal].T            # [Sq_pad, real keys]
            worst = logits.reshape(nq, 64, -1).max(axis=(1, 2))
            assert np.all(bound[b, h] >= worst), (bound[b, h], worst)
            assert np.all(bound[b, h] <= 1.01 * c * qn_got[b, h] * kn_got[b, h].max())


def test_forward_ungated_equals_broadcast_plus_sparse():
    """The ungated combine is out_c broadcast per block plus the sparse branch
    computed on the same selection (the combine page's ungated check)."""
    B, H, D = 1, 2, 128
    qs = ks = [64] * 6
    q, k, v = (_bhsd(B, H, qs, D, 2100, s).to(DEV) for s in range(3))
    out, idx, num, out_c = vsa.vsa_forward(q, k, v, None, topk=3, return_out_c=True)
    o_s = vsa.block_sparse_attn_from_indices(q, k, v, idx, num)
    vsa.check_device_status()
    want = (torch.repeat_interleave(out_c, 64, dim=2) + o_s.float()).to(torch.bfloat16)
    # both sides round once from the same fp32 inputs except the sparse branch,
    # which the second call rounds to bf16 first: allow one bf16 ulp
    diff = (out.float() - want.float()).abs()
    assert diff.max().item() <= 2 * torch.finfo(torch.bfloat16).eps * max(1.0, want.float().abs().max().item())


def test_forward_gate_zero_is_sparse_branch():
    B, H, D = 1, 2, 128
    qs = [64] * 5
    q, k, v = (_bhsd(B, H, qs, D, 2200, s).to(DEV) for s in range(3))
    gate = torch.zeros((B, 64 * 5, H, D), dtype=torch.bfloat16, device=DEV)
    out, idx, num = vsa.vsa_forward(q, k, v, gate, topk=2)
    o_s = vsa.block_sparse_attn_from_indices(q, k, v, idx, num)
    vsa.check_device_status()
    assert torch.equal(out, o_s)


def test_forward_topk_ties_take_lowest_index():
    """Identical KV blocks give identical coarse logits: the selection must be
    the lowest indices."""
    B, H, D = 1, 1, 128
    blk = I.normal_bf16((1, 1, 64, D), 2300, 1)
    k = blk.repeat(1, 1, 8, 1)
    q = _bhsd(B, H, [64] * 3, D, 2300, 0)
    out, idx, num = vsa.vsa_forward(q.to(DEV), k.to(DEV), k.to(DEV), None, topk=3)
    vsa.check_device_status()
    assert idx.cpu().tolist() == [[[[0, 1, 2]] * 3]]


# ---------------------------------------------------------------------------
# a6: varlen
# ---------------------------------------------------------------------------
def _varlen_inputs(q_lens, kv_lens, H, D, frac, seed):
    cu_q, cu_kv = I.cu_seqlens(q_lens), I.cu_seqlens(kv_lens)
    q = I.normal_bf16((H, cu_q[-1], D), seed, 0)
    k = I.normal_bf16((H, cu_kv[-1], D), seed, 1)
    v = I.normal_bf16((H, cu_kv[-1], D), seed, 2)
    rng = np.random.default_rng(seed)
    nq = [-(-n // 64) for n in q_lens]
    nkv = [-(-n // 64) for n in kv_lens]
    ks = [max(1, min(n, int(frac * n))) for n in nkv]
    width = max(ks)
    idx = np.full((H, sum(nq), width), -1, dtype=np.int32)
    num = np.zeros((H, sum(nq)), dtype=np.int32)
    row = 0
    for i in range(len(q_lens)):
        for _ in range(nq[i]):
            for h in range(H):
                idx[h, row, :ks[i]] = np.sort(rng.choice(nkv[i], size=ks[i], replace=False))
                num[h, row] = ks[i]
            row += 1
    return cu_q, cu_kv, q, k, v, idx, num


VARLEN_CASES = [
    ("equal", [256, 256], [256, 256], 2, 128, 0.5),
    ("different", [130, 64, 300], [70, 200, 64], 2, 128, 0.5),
    ("single", [200], [150], 2, 64, 0.7),
    ("many-heads", [128, 192], [192, 128], 16, 128, 0.5),
    ("many-seqs", [64 * (i + 1) - 5 for i in range(8)], [64 * (i + 1) for i in range(8)], 2, 128, 0.5),
    ("dense", [100, 64, 7], [90, 128, 200], 2, 128, 1.0),
    ("one-block-each", [64, 10, 33], [5, 64, 1], 2, 128, 1.0),
    ("asymmetric", [3000 // 8, 640], [120, 1400], 3, 128, 0.3),
]


@pytest.mark.parametrize("case", VARLEN_CASES, ids=lambda c: c[0])
def test_varlen(case):
    name, q_lens, kv_lens, H, D, frac = case
    cu_q, cu_kv, q, k, v, idx, num = _varlen_inputs(q_lens, kv_lens, H, D, frac, 3000 + len(q_lens))
    out, pq, pkv, reb = vsa.block_sparse_attn_varlen(
        q.to(DEV), k.to(DEV), v.to(DEV), cu_q, cu_kv, torch.from_numpy(idx).to(DEV),
        torch.from_numpy(num).to(DEV), return_aux=True)
    vsa.check_device_status()
    lay = O.varlen_layout(cu_q, cu_kv)
    assert np.array_equal(P.to_np(pq), lay["pack_index_q"])
    assert np.array_equal(P.to_np(pkv), lay["pack_index_kv"])
    assert np.array_equal(P.to_np(reb), O.rebase_q2k_idx(idx, num, lay))
    want = O.block_sparse_attn_varlen(P.to_np(q), P.to_np(k), P.to_np(v), cu_q, cu_kv, idx, num,
                                      O.default_scale(D))
    P.assert_outputs_close(P.to_np(out), want)


def test_varlen_large_logits_one_sequence_peaked():
    """One sequence's keys scaled x16 and its queries x4: its logit bound is
    far above the refresh limit, so its items keep the running-max check and
    rescale, while the other sequence's items may run the vote-free step."""
    q_lens, kv_lens, H, D = [200, 150], [300, 260], 2, 128
    cu_q, cu_kv, q, k, v, idx, num = _varlen_inputs(q_lens, kv_lens, H, D, 0.8, 3200)
    q[:, cu_q[1]:] *= 4
    k[:, cu_kv[1]:] *= 16
    out = vsa.block_sparse_attn_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu_q, cu_kv,
                                       torch.from_numpy(idx).to(DEV), torch.from_numpy(num).to(DEV))
    vsa.check_device_status()
    want = O.block_sparse_attn_varlen(P.to_np(q), P.to_np(k), P.to_np(v), cu_q, cu_kv, idx, num,
                                      O.default_scale(D))
    P.assert_outputs_close(P.to_np(out), want)


def test_varlen_packed_equals_per_sequence_bitwise():
    """One packed launch gives exactly the per-sequence results (the varlen
    page's error = 0.0), because each query block runs the same arithmetic."""
    q_lens, kv_lens, H, D = [130, 64, 300], [70, 200, 64], 2, 128
    cu_q, cu_kv, q, k, v, idx, num = _varlen_inputs(q_lens, kv_lens, H, D, 0.6, 3100)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    packed = vsa.block_sparse_attn_varlen(qd, kd, vd, cu_q, cu_kv, torch.from_numpy(idx).to(DEV),
                                          torch.from_numpy(num).to(DEV))
    row = 0
    for i in range(len(q_lens)):
        nqi = -(-q_lens[i] // 64)
        one = vsa.block_sparse_attn_varlen(
            qd[:, cu_q[i]:cu_q[i + 1]].contiguous(), kd[:, cu_kv[i]:cu_kv[i + 1]].contiguous(),
            vd[:, cu_kv[i]:cu_kv[i + 1]].contiguous(), [0, q_lens[i]], [0, kv_lens[i]],
            torch.from_numpy(idx[:, row:row + nqi].copy()).to(DEV),
            torch.from_numpy(num[:, row:row + nqi].copy()).to(DEV))
        assert torch.equal(packed[:, cu_q[i]:cu_q[i + 1]], one)
        row += nqi
    vsa.check_device_status()


def test_varlen_variable_block_sizes():
    """Per-sequence block sizes (not only 64 + remainder)."""
    H, D = 2, 128
    q_lens, kv_lens = [150, 64], [100, 70]
    qbl = [[64, 30, 56], [64]]
    kbl = [[40, 60], [7, 63]]
    cu_q, cu_kv = I.cu_seqlens(q_lens), I.cu_seqlens(kv_lens)
    q = I.normal_bf16((H, cu_q[-1], D), 3200, 0)
    k = I.normal_bf16((H, cu_kv[-1], D), 3200, 1)
    v = I.normal_bf16((H, cu_kv[-1], D), 3200, 2)
    idx = np.array([[[0, 1], [1, -1], [0, 1], [0, 1]]] * H, dtype=np.int32)
    num = np.array([[2, 1, 2, 2]] * H, dtype=np.int32)
    out, pq, pkv, reb = vsa.block_sparse_attn_varlen(
        q.to(DEV), k.to(DEV), v.to(DEV), cu_q, cu_kv, torch.from_numpy(idx).to(DEV),
        torch.from_numpy(num).to(DEV), q_block_sizes_list=qbl, kv_block_sizes_list=kbl, return_aux=True)
    vsa.check_device_status()
    lay = O.varlen_layout(cu_q, cu_kv, qbl, kbl)
    assert np.array_equal(P.to_np(pq), lay["pack_index_q"])
    assert np.array_equal(P.to_np(pkv), lay["pack_index_kv"])
    want = O.block_sparse_attn_varlen(P.to_np(q), P.to_np(k), P.to_np(v), cu_q, cu_kv, idx, num,
                                      O.default_scale(D), qbl, kbl)
    P.assert_outputs_close(P.to_np(out), want)


# ---------------------------------------------------------------------------
# a7: tile gather / scatter
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("D", [128, 64, 96, 8])
@pytest.mark.parametrize("shape,tile", [((9, 30, 52), (4, 4, 4)), ((5, 5, 5), (4, 4, 4)),
                                        ((6, 10, 20), (4, 8, 8))])
def test_tile_gather_scatter(shape, tile, D):
    """Rows of 64 and 128 values take the several-slots-per-thread kernel,
    other multiples of 8 the one-slot-per-CTA kernel; both give the tile
    layout exactly (64- and 256-token tiles) and scatter back to the tokens."""
    meta = vsa.build_vsa_metadata(*shape, tile=tile)
    N = int(np.prod(shape))
    x = I.normal_bf16((2, 3, N, D), 3300, 0)
    slot = torch.from_numpy(meta["slot_token"]).to(DEV)
    xp = vsa.gather_tokens(x.reshape(6, N, D).to(DEV), slot)
    want = O.tile_and_pad(P.to_np(x), O.build_vsa_metadata(*shape, tile=tile))
    assert np.array_equal(P.to_np(xp).reshape(want.shape), want)
    back = vsa.scatter_tokens(xp, slot, N)
    assert torch.equal(back.cpu().reshape(x.shape), x)
    vsa.check_device_status()


# ---------------------------------------------------------------------------
# the host-buffer forward: chunked copies around the same forward
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("case", [
    # B, H, D, q sizes, kv sizes, topk, gated, heads per chunk
    (2, 5, 128, [64, 64, 64, 20, 64, 64], [64] * 5 + [3] + [64] * 2, 3, True, 2),
    (1, 9, 64, [64] * 7, [64] * 9, 4, False, 0),
], ids=["B2-H5-gated-chunk2", "B1-H9-default-chunks"])
def test_forward_host_equals_device_forward(case, pinned):
    """vsa_forward_host on host tensors returns exactly what vsa_forward
    returns on the same data on the device (every chunk is one vsa_forward)."""
    B, H, D, qs, ks, topk, gated, hpc = case
    q = _bhsd(B, H, qs, D, 2700, 0)
    k = _bhsd(B, H, ks, D, 2700, 1)
    v = _bhsd(B, H, ks, D, 2700, 2)
    gate = I.gate_bf16((B, 64 * len(qs), H, D), 2700) if gated else None
    host = [t.pin_memory() if pinned else t for t in (q, k, v)]
    gh = None if gate is None else (gate.pin_memory() if pinned else gate)
    out_h, idx_h, num_h, oc_h = vsa.vsa_forward_host(
        host[0], host[1], host[2], gh, qs, ks, topk=topk, return_indices=True, return_out_c=True,
        heads_per_chunk=hpc)
    torch.cuda.current_stream().synchronize()
    vsa.check_device_status()
    out, idx, num, oc = vsa.vsa_forward(q.to(DEV), k.to(DEV), v.to(DEV), None if gate is None else gate.to(DEV),
                                        qs, ks, topk=topk, return_out_c=True)
    vsa.check_device_status()
    assert torch.equal(out_h, out.cpu())
    assert torch.equal(idx_h, idx.cpu())
    assert torch.equal(num_h, num.cpu())
    assert torch.equal(oc_h, oc.cpu())
