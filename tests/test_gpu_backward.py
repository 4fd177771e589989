"""Backward of the block-sparse attention on the GPU, through the C ABI,
against the fp64 oracle: the forward's per-row log-sum-exp, then dq, dk, dv
(ragged blocks, nq != nkv, duplicated and empty selections, more work items
than SMs), the varlen backward against per-sequence calls bit for bit (the
varlen page's "match per-sequence reference exactly") and against the
oracle.  Gradient tolerance: relative RMS error <= 1e-2 and max abs <= 2e-2
of the reference's largest magnitude -- tighter than the varlen page's 5%
relative bound for the backward (measured: ~2.4e-3 relative RMS, from the
bf16 operands dS and P of the gradient products)."""
import numpy as np
import pytest
import torch

from block_sparse_attention_15_b200 import binding as vsa
from block_sparse_attention_15_b200 import inputs as I
from oracle import vsa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"
REL_RMS = 1e-2
MAX_FRAC = 2e-2


def _grad_close(got, want, what):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    st = P.error_stats(got, want)
    scale = np.abs(want).max()
    assert st["rel_rms"] <= REL_RMS, f"{what}: relative RMS {st['rel_rms']:.3e}"
    assert st["max_abs"] <= MAX_FRAC * scale + 1e-6, f"{what}: max abs {st['max_abs']:.3e} vs {scale:.3e}"
    return st


def _selection(rng, B, H, nq, nkv, width, dup, empty=()):
    idx = np.full((B, H, nq, width), -1, dtype=np.int32)
    num = np.zeros((B, H, nq), dtype=np.int32)
    for b, h, a in np.ndindex(B, H, nq):
        if (b, h, a) in empty:
            continue
        n = int(rng.integers(1, width + 1))
        sel = rng.integers(0, nkv, size=n) if dup else rng.choice(nkv, size=min(n, nkv), replace=False)
        idx[b, h, a, :len(sel)] = sel
        num[b, h, a] = len(sel)
    return idx, num


CASES = [
    # D, B, H, q sizes, kv sizes, width, duplicates, seed
    (128, 1, 2, [64] * 4, [64] * 6, 4, True, 1),
    (64, 2, 2, [64, 50, 64], [64, 64, 9, 64, 33], 3, False, 2),
    (128, 1, 8, [64] * 20, [64] * 24, 6, False, 3),   # 160 items: more than the SMs
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"D{c[0]}-B{c[1]}H{c[2]}-nq{len(c[3])}-nkv{len(c[4])}")
def test_backward_matches_oracle(case):
    D, B, H, qs, ks, width, dup, seed = case
    rng = np.random.default_rng(seed)
    q, k, v = (I.padded_normal_bhsd(B, H, s, D, 1200 + seed, i) for i, s in enumerate((qs, ks, ks)))
    do = I.padded_normal_bhsd(B, H, qs, D, 1200 + seed, 7)
    idx, num = _selection(rng, B, H, len(qs), len(ks), width, dup, empty={(0, 0, 1)})
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), do.to(DEV)
    ti, tn = torch.from_numpy(idx).to(DEV), torch.from_numpy(num).to(DEV)
    out, lse = vsa.block_sparse_attn_from_indices(qd, kd, vd, ti, tn, qs, ks, return_lse=True)
    dq, dk, dv = vsa.block_sparse_attn_backward(qd, kd, vd, out, dod, lse, ti, tn, qs, ks)
    vsa.check_device_status()
    qn, kn, vn, don = P.to_np(q), P.to_np(k), P.to_np(v), P.to_np(do)
    scale = O.default_scale(D)
    rr = P.real_rows(qs)
    want_lse = O.block_sparse_lse(qn, kn, idx, num, qs, ks, scale)
    got_lse = P.to_np(lse)
    fin = np.isfinite(want_lse[:, :, rr])
    np.testing.assert_allclose(got_lse[:, :, rr][fin], want_lse[:, :, rr][fin], rtol=1e-4, atol=2e-3)
    assert np.all(np.isneginf(got_lse[:, :, rr][~fin]))
    wq, wk, wv = O.block_sparse_attention_backward(qn, kn, vn, don, idx, num, qs, ks, scale)
    kr = P.real_rows(ks)
    _grad_close(P.to_np(dq)[:, :, rr], wq[:, :, rr], "dq")
    _grad_close(P.to_np(dk)[:, :, kr], wk[:, :, kr], "dk")
    _grad_close(P.to_np(dv)[:, :, kr], wv[:, :, kr], "dv")
    # padded rows are 0
    for g, sizes in ((dq, qs), (dk, ks), (dv, ks)):
        pad = np.setdiff1d(np.arange(g.shape[2]), P.real_rows(sizes))
        assert np.all(P.to_np(g)[:, :, pad] == 0.0)


def test_varlen_backward_packed_equals_per_sequence_and_oracle():
    H, D = 3, 128
    q_lens, kv_lens = [150, 64, 300], [200, 90, 129]
    cu_q, cu_kv = I.cu_seqlens(q_lens), I.cu_seqlens(kv_lens)
    seed = 1300
    q = I.normal_bf16((H, cu_q[-1], D), seed, 0)
    k = I.normal_bf16((H, cu_kv[-1], D), seed, 1)
    v = I.normal_bf16((H, cu_kv[-1], D), seed, 2)
    do = I.normal_bf16((H, cu_q[-1], D), seed, 7)
    idx, num, _ = I.varlen_random_selection(q_lens, kv_lens, H, 0.6, seed)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), do.to(DEV)
    ti, tn = torch.from_numpy(idx).to(DEV), torch.from_numpy(num).to(DEV)
    lse = torch.empty((H, cu_q[-1]), dtype=torch.float32, device=DEV)
    out = vsa.block_sparse_attn_varlen(qd, kd, vd, cu_q, cu_kv, ti, tn, lse=lse)
    dq, dk, dv = vsa.block_sparse_attn_varlen_backward(qd, kd, vd, out, dod, lse, cu_q, cu_kv, ti, tn)
    vsa.check_device_status()
    # per sequence, one call each
    nq = [-(-n // 64) for n in q_lens]
    rows = np.cumsum([0] + nq)
    for i in range(len(q_lens)):
        sq = slice(cu_q[i], cu_q[i + 1])
        skv = slice(cu_kv[i], cu_kv[i + 1])
        qi, ki, vi, doi = (x[:, s].contiguous() for x, s in ((qd, sq), (kd, skv), (vd, skv), (dod, sq)))
        ii = ti[:, rows[i]:rows[i + 1]].contiguous()
        ni = tn[:, rows[i]:rows[i + 1]].contiguous()
        lse_i = torch.empty((H, q_lens[i]), dtype=torch.float32, device=DEV)
        cuq_i, cukv_i = [0, q_lens[i]], [0, kv_lens[i]]
        out_i = vsa.block_sparse_attn_varlen(qi, ki, vi, cuq_i, cukv_i, ii, ni, lse=lse_i)
        gq, gk, gv = vsa.block_sparse_attn_varlen_backward(qi, ki, vi, out_i, doi, lse_i, cuq_i, cukv_i,
                                                           ii, ni)
        assert torch.equal(out_i, out[:, sq])
        assert torch.equal(lse_i, lse[:, sq])
        assert torch.equal(gq, dq[:, sq]) and torch.equal(gk, dk[:, skv]) and torch.equal(gv, dv[:, skv])
    vsa.check_device_status()
    # against the oracle: packed backward = per-sequence backward
    lay = O.varlen_layout(cu_q, cu_kv)
    reb = O.rebase_q2k_idx(idx, num, lay)
    qp, kp, vp, dp = (O.pack_tokens(P.to_np(x), lay["pack_index_" + w])
                      for x, w in ((q, "q"), (k, "kv"), (v, "kv"), (do, "q")))
    wq, wk, wv = O.block_sparse_attention_backward(qp, kp, vp, dp, reb[None], num[None],
                                                   lay["q_block_sizes"], lay["kv_block_sizes"],
                                                   O.default_scale(D))
    pq, pkv = lay["pack_index_q"], lay["pack_index_kv"]
    rq, rk = pq >= 0, pkv >= 0
    _grad_close(P.to_np(dq)[:, pq[rq]], wq[0][:, rq], "varlen dq")
    _grad_close(P.to_np(dk)[:, pkv[rk]], wk[0][:, rk], "varlen dk")
    _grad_close(P.to_np(dv)[:, pkv[rk]], wv[0][:, rk], "varlen dv")


def test_backward_h3_shape_eight_heads():
    """The H3-like shape (242 blocks, top 48) on 8 heads, every row checked."""
    B, H, D, nb, topk = 1, 8, 128, 242, 48
    sizes = [64] * nb
    q, k, v = (I.padded_normal_bhsd(B, H, sizes, D, 1003, i) for i in range(3))
    do = I.padded_normal_bhsd(B, H, sizes, D, 1003, 7)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), do.to(DEV)
    _, idx, num = vsa.vsa_forward(qd, kd, vd, None, topk=topk)
    out, lse = vsa.block_sparse_attn_from_indices(qd, kd, vd, idx, num, return_lse=True)
    dq, dk, dv = vsa.block_sparse_attn_backward(qd, kd, vd, out, dod, lse, idx, num)
    vsa.check_device_status()
    wq, wk, wv = O.block_sparse_attention_backward(P.to_np(q), P.to_np(k), P.to_np(v), P.to_np(do),
                                                   P.to_np(idx), P.to_np(num), sizes, sizes,
                                                   O.default_scale(D))
    _grad_close(P.to_np(dq), wq, "dq H3")
    _grad_close(P.to_np(dk), wk, "dk H3")
    _grad_close(P.to_np(dv), wv, "dv H3")
