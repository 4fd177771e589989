"""Pins that tie the CPU oracle to facts fixed outside itself.

Every ``check_*`` takes the oracle module as ``O`` and raises AssertionError
when the oracle disagrees with a closed form, an invariant, a brute-force
enumeration, a library routine (torch's fp64 scaled-dot-product attention) or
a figure printed on the pages.  ``test_oracle_pins.py`` runs them on the real
oracle; ``test_oracle_mutations.py`` plants plausible mistakes in a copy of
the oracle and requires that some pin catches each one.
"""

from __future__ import annotations

import itertools
import json
import os

import numpy as np
import torch

BLOCK = 64
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16_like(rng, shape, scale=1.0):
    """Random values exactly representable in bf16 (as fp64)."""
    x = torch.from_numpy(rng.standard_normal(shape) * scale).to(torch.bfloat16)
    return x.double().numpy()


def _padded(rng, B, H, sizes, D, pad_value=0.0, scale=1.0):
    x = np.full((B, H, BLOCK * len(sizes), D), pad_value, dtype=np.float64)
    for j, m in enumerate(sizes):
        x[:, :, BLOCK * j:BLOCK * j + m] = _bf16_like(rng, (B, H, m, D), scale)
    return x


def _real_rows(sizes):
    return np.concatenate([np.arange(BLOCK * j, BLOCK * j + m) for j, m in enumerate(sizes)])


def _sdpa(q, k, v, scale, mask=None):
    """torch's fp64 CPU scaled_dot_product_attention (a library routine)."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    m = None if mask is None else torch.from_numpy(mask)
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=m, scale=scale).numpy()


# ---------------------------------------------------------------------------
# pooling
# ---------------------------------------------------------------------------
def check_pool_closed_forms(O):
    sizes = [64, 17, 1, 64, 40]
    B, H, D = 2, 3, 8
    # slot-index ramp: block j of size m averages 64j + (m-1)/2
    S = BLOCK * len(sizes)
    ramp = np.broadcast_to(np.arange(S, dtype=np.float64)[None, None, :, None],
                           (B, H, S, D)).copy()
    got = O.block_pool(ramp, sizes)
    for j, m in enumerate(sizes):
        assert np.allclose(got[:, :, j], BLOCK * j + (m - 1) / 2.0, rtol=0, atol=1e-12), j
    # constant real tokens, poisoned padding -> the constant
    x = np.full((B, H, S, D), 1e6)
    for j, m in enumerate(sizes):
        x[:, :, BLOCK * j:BLOCK * j + m] = 3.25 + j
    got = O.block_pool(x, sizes)
    for j in range(len(sizes)):
        assert np.all(got[:, :, j] == 3.25 + j)
    # a single-token block is that token
    rng = _rng(1)
    x = _padded(rng, B, H, sizes, D, pad_value=7.0)
    got = O.block_pool(x, sizes)
    assert np.array_equal(got[:, :, 2], x[:, :, 2 * BLOCK])
    # linearity
    y = _padded(rng, B, H, sizes, D)
    assert np.allclose(O.block_pool(2.5 * x - y, sizes),
                       2.5 * O.block_pool(x, sizes) - O.block_pool(y, sizes), atol=1e-12)


# ---------------------------------------------------------------------------
# coarse attention
# ---------------------------------------------------------------------------
def check_coarse_special_cases(O):
    rng = _rng(2)
    B, H, D = 1, 2, 16
    qc = rng.standard_normal((B, H, 5, D))
    vc1 = rng.standard_normal((B, H, 1, D))
    # one KV block: the coarse output is that block's pooled value
    _, oc = O.coarse_attention(qc, rng.standard_normal((B, H, 1, D)), vc1, 0.25)
    assert np.allclose(oc, np.broadcast_to(vc1, oc.shape), atol=1e-14)
    # identical keys (or zero scale): uniform weights -> mean of vc
    vc = rng.standard_normal((B, H, 7, D))
    kc_same = np.broadcast_to(rng.standard_normal((B, H, 1, D)), (B, H, 7, D))
    _, oc = O.coarse_attention(qc, kc_same, vc, 0.3)
    assert np.allclose(oc, np.broadcast_to(vc.mean(axis=2, keepdims=True), oc.shape), atol=1e-13)
    _, oc = O.coarse_attention(qc, rng.standard_normal((B, H, 7, D)), vc, 0.0)
    assert np.allclose(oc, np.broadcast_to(vc.mean(axis=2, keepdims=True), oc.shape), atol=1e-13)
    # two KV blocks: weight of block 0 is the logistic of the logit gap
    kc2 = rng.standard_normal((B, H, 2, D))
    vc2 = rng.standard_normal((B, H, 2, D))
    s, oc = O.coarse_attention(qc, kc2, vc2, 0.5)
    gap = 0.5 * (np.einsum("bhqd,bhd->bhq", qc, kc2[:, :, 1]) - np.einsum("bhqd,bhd->bhq", qc, kc2[:, :, 0]))
    w0 = 1.0 / (1.0 + np.exp(gap))
    want = w0[..., None] * vc2[:, :, None, 0] + (1 - w0)[..., None] * vc2[:, :, None, 1]
    assert np.allclose(oc, want, atol=1e-13)
    # scores are the scaled dot products themselves
    assert np.allclose(s[..., 0], 0.5 * np.einsum("bhqd,bhd->bhq", qc, kc2[:, :, 0]), atol=1e-13)
    # one-hot keys with a huge scale pick the matching value (hard attention)
    kc_eye = np.broadcast_to(np.eye(D)[None, None, :6], (B, H, 6, D))
    vc6 = rng.standard_normal((B, H, 6, D))
    q_hot = np.zeros((B, H, 6, D))
    for j in range(6):
        q_hot[:, :, j, j] = 1.0
    _, oc = O.coarse_attention(q_hot, kc_eye, vc6, 200.0)
    assert np.allclose(oc, vc6, atol=1e-12)


def check_coarse_vs_library(O):
    rng = _rng(3)
    qc = rng.standard_normal((2, 3, 9, 32))
    kc = rng.standard_normal((2, 3, 13, 32))
    vc = rng.standard_normal((2, 3, 13, 32))
    _, oc = O.coarse_attention(qc, kc, vc, 0.2)
    assert np.allclose(oc, _sdpa(qc, kc, vc, 0.2), atol=1e-12)


# ---------------------------------------------------------------------------
# top-k
# ---------------------------------------------------------------------------
def _brute_topk_set(row, k):
    """The unique k-subset S with: every i in S beats every j outside S, where
    i beats j iff row[i] > row[j] or (row[i] == row[j] and i < j)."""
    n = len(row)
    found = []
    for S in itertools.combinations(range(n), k):
        inside = set(S)
        ok = all((row[i] > row[j]) or (row[i] == row[j] and i < j)
                 for i in inside for j in range(n) if j not in inside)
        if ok:
            found.append(S)
    assert len(found) == 1
    return list(found[0])


def check_topk_brute_force(O):
    rng = _rng(4)
    for trial in range(40):
        n = int(rng.integers(1, 9))
        k = int(rng.integers(1, n + 1))
        # coarse grid of values so that ties are frequent
        row = rng.integers(-3, 4, size=n).astype(np.float64) * 0.5
        idx, num = O.select_topk(row[None, None, None, :], k)
        assert num[0, 0, 0] == k
        assert list(idx[0, 0, 0]) == _brute_topk_set(row, k), (row, k)


def check_topk_edge_cases(O):
    s = np.linspace(0.0, 1.0, 10)[None, None, None, :]
    idx, num = O.select_topk(s, 10)          # topk = all
    assert list(idx[0, 0, 0]) == list(range(10)) and num[0, 0, 0] == 10
    idx, num = O.select_topk(s, 25)          # clamped to n
    assert list(idx[0, 0, 0]) == list(range(10)) and num[0, 0, 0] == 10
    idx, num = O.select_topk(np.zeros((1, 1, 1, 10)), 3)   # all tied: lowest indices
    assert list(idx[0, 0, 0]) == [0, 1, 2]
    idx, num = O.select_topk(s, 3, width=6)  # ascending, -1 tail
    assert list(idx[0, 0, 0]) == [7, 8, 9, -1, -1, -1] and num[0, 0, 0] == 3
    s2 = np.array([0.5, 2.0, 2.0, -1.0, 2.0])[None, None, None, :]
    idx, _ = O.select_topk(s2, 2)            # planted tie at the boundary
    assert list(idx[0, 0, 0]) == [1, 2]


# ---------------------------------------------------------------------------
# block-sparse attention
# ---------------------------------------------------------------------------
def _mask_from_sel(idx, num, q_sizes, kv_sizes):
    nq, nkv = len(q_sizes), len(kv_sizes)
    B, H = idx.shape[:2]
    mask = np.zeros((B, H, BLOCK * nq, BLOCK * nkv), dtype=bool)
    for b in range(B):
        for h in range(H):
            for a in range(nq):
                for j in range(num[b, h, a]):
                    c = idx[b, h, a, j]
                    mask[b, h, BLOCK * a:BLOCK * (a + 1), BLOCK * c:BLOCK * c + kv_sizes[c]] = True
    return mask


def check_sparse_dense_equivalence(O):
    """topk = all blocks equals dense softmax attention over the real tokens."""
    rng = _rng(5)
    B, H, D = 1, 2, 32
    q_sizes, kv_sizes = [64, 64, 30], [64, 12, 64, 64, 5]   # nq != nkv, partial blocks
    q = _padded(rng, B, H, q_sizes, D, pad_value=0.0)
    k = _padded(rng, B, H, kv_sizes, D, pad_value=9.0)
    v = _padded(rng, B, H, kv_sizes, D, pad_value=-9.0)
    nkv = len(kv_sizes)
    idx = np.broadcast_to(np.arange(nkv, dtype=np.int32), (B, H, len(q_sizes), nkv)).copy()
    num = np.full((B, H, len(q_sizes)), nkv, dtype=np.int32)
    scale = 1 / np.sqrt(D)
    got = O.block_sparse_attention(q, k, v, idx, num, q_sizes, kv_sizes, scale)
    qr, kr = _real_rows(q_sizes), _real_rows(kv_sizes)
    want = _sdpa(q[:, :, qr], k[:, :, kr], v[:, :, kr], scale)
    assert np.allclose(got[:, :, qr], want, atol=1e-12)
    pad_rows = np.setdiff1d(np.arange(q.shape[2]), qr)
    assert np.all(got[:, :, pad_rows] == 0.0)


def check_sparse_vs_masked_library(O):
    """Arbitrary selections equal masked dense attention (torch SDPA, fp64)."""
    rng = _rng(6)
    B, H, D = 2, 2, 16
    q_sizes, kv_sizes = [64, 50, 64, 1], [64, 64, 33, 64, 64, 7]
    q = _padded(rng, B, H, q_sizes, D)
    k = _padded(rng, B, H, kv_sizes, D, pad_value=5.0)
    v = _padded(rng, B, H, kv_sizes, D, pad_value=5.0)
    nq, nkv, width = len(q_sizes), len(kv_sizes), 4
    idx = np.full((B, H, nq, width), -1, dtype=np.int32)
    num = np.zeros((B, H, nq), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for a in range(nq):
                n = int(rng.integers(1, width + 1))
                idx[b, h, a, :n] = rng.choice(nkv, size=n, replace=False)
                num[b, h, a] = n
    scale = 0.3
    got = O.block_sparse_attention(q, k, v, idx, num, q_sizes, kv_sizes, scale)
    mask = _mask_from_sel(idx, num, q_sizes, kv_sizes)
    want = _sdpa(q, k, v, scale, mask)
    qr = _real_rows(q_sizes)
    assert np.allclose(got[:, :, qr], want[:, :, qr], atol=1e-12)


def check_sparse_invariants(O):
    rng = _rng(7)
    B, H, D = 1, 1, 8
    q_sizes, kv_sizes = [64, 64], [64, 1, 64, 64]
    q = _padded(rng, B, H, q_sizes, D)
    k = _padded(rng, B, H, kv_sizes, D)
    v = _padded(rng, B, H, kv_sizes, D)
    # a single selected one-token block: every row returns that v row
    idx = np.array([[[[1, -1], [1, -1]]]], dtype=np.int32)
    num = np.array([[[1, 1]]], dtype=np.int32)
    got = O.block_sparse_attention(q, k, v, idx, num, q_sizes, kv_sizes, 0.7)
    assert np.allclose(got[0, 0], np.broadcast_to(v[0, 0, BLOCK], got[0, 0].shape), atol=1e-14)
    # order of the selection does not matter; a repeated entry changes nothing
    a = O.block_sparse_attention(q, k, v, np.array([[[[0, 2, 3], [3, 0, 2]]]], np.int32),
                                 np.array([[[3, 3]]], np.int32), q_sizes, kv_sizes, 0.7)
    b = O.block_sparse_attention(q, k, v, np.array([[[[3, 2, 0], [2, 3, 0]]]], np.int32),
                                 np.array([[[3, 3]]], np.int32), q_sizes, kv_sizes, 0.7)
    assert np.allclose(a, b, atol=1e-13)
    c = O.block_sparse_attention(q, k, v, np.array([[[[0, 0], [3, 3]]]], np.int32),
                                 np.array([[[2, 2]]], np.int32), q_sizes, kv_sizes, 0.7)
    d = O.block_sparse_attention(q, k, v, np.array([[[[0, -1], [3, -1]]]], np.int32),
                                 np.array([[[1, 1]]], np.int32), q_sizes, kv_sizes, 0.7)
    assert np.allclose(c, d, atol=1e-13)
    # an empty selection gives 0
    e = O.block_sparse_attention(q, k, v, np.array([[[[0, -1], [3, -1]]]], np.int32),
                                 np.array([[[0, 1]]], np.int32), q_sizes, kv_sizes, 0.7)
    assert np.all(e[0, 0, :BLOCK] == 0.0) and np.allclose(e[0, 0, BLOCK:], d[0, 0, BLOCK:])


# ---------------------------------------------------------------------------
# combine
# ---------------------------------------------------------------------------
def check_combine(O):
    rng = _rng(8)
    B, H, D = 2, 3, 8
    sizes = [64, 64, 20]
    S = BLOCK * len(sizes)
    out_c = rng.standard_normal((B, H, len(sizes), D))
    o_s = rng.standard_normal((B, H, S, D))
    real = _real_rows(sizes)
    # the page's earlier form: repeat out_c across each block, then add
    rep = np.repeat(out_c, BLOCK, axis=2)
    ung = O.combine(out_c, o_s, None, sizes)
    assert np.array_equal(ung[:, :, real], (rep + o_s)[:, :, real])
    assert np.all(np.delete(ung, real, axis=2) == 0.0)
    ones = np.ones((B, S, H, D))
    assert np.array_equal(O.combine(out_c, o_s, ones, sizes), ung)
    zeros = np.zeros((B, S, H, D))
    assert np.array_equal(O.combine(out_c, o_s, zeros, sizes)[:, :, real], o_s[:, :, real])
    # gate is [B, S, H, D]: a gate that depends on (s, h) only
    g = np.zeros((B, S, H, D))
    for s in range(S):
        for h in range(H):
            g[:, s, h, :] = 0.01 * s + h
    got = O.combine(out_c, o_s, g, sizes)
    for h in range(H):
        for s in real:
            want = out_c[:, h, s // BLOCK] * (0.01 * s + h) + o_s[:, h, s]
            assert np.allclose(got[:, h, s], want, atol=1e-12)


def check_forward_dense_limit(O):
    """Whole forward with topk = all and gate = 0 is dense attention; with a
    constant gate it adds the gated coarse output per block."""
    rng = _rng(9)
    B, H, D = 1, 2, 16
    sizes = [64, 64, 64, 9]
    q = _padded(rng, B, H, sizes, D)
    k = _padded(rng, B, H, sizes, D)
    v = _padded(rng, B, H, sizes, D)
    S = q.shape[2]
    r = O.vsa_forward(q, k, v, np.zeros((B, S, H, D)), sizes, sizes, topk=len(sizes))
    real = _real_rows(sizes)
    want = _sdpa(q[:, :, real], k[:, :, real], v[:, :, real], 0.25)
    assert np.allclose(r["out"][:, :, real], want, atol=1e-12)
    assert list(r["q2k_idx"][0, 0, 0]) == [0, 1, 2, 3]
    r2 = O.vsa_forward(q, k, v, np.full((B, S, H, D), 0.5), sizes, sizes, topk=len(sizes))
    assert np.allclose(r2["out"][:, :, real] - r["out"][:, :, real],
                       0.5 * np.repeat(r["out_c"], BLOCK, axis=2)[:, :, real], atol=1e-12)


# ---------------------------------------------------------------------------
# varlen
# ---------------------------------------------------------------------------
def _brute_pack_index(cu, sizes_list=None):
    """Enumerate slots directly: sequence i's token t goes to slot
    64 * (first block of i + block of t) + position of t inside its block."""
    slots = {}
    first_block = 0
    for i in range(len(cu) - 1):
        n = cu[i + 1] - cu[i]
        if sizes_list is None:
            sizes = [min(BLOCK, n - BLOCK * j) for j in range(-(-n // BLOCK))]
        else:
            sizes = list(sizes_list[i])
        starts = np.cumsum([0] + sizes)
        for t in range(n):
            blk = int(np.searchsorted(starts, t, side="right") - 1)
            slots[BLOCK * (first_block + blk) + (t - starts[blk])] = cu[i] + t
        first_block += len(sizes)
    out = np.full(BLOCK * first_block, -1, dtype=np.int64)
    for s, tok in slots.items():
        out[s] = tok
    return out


def check_varlen_pack_indices(O):
    cu_q = [0, 100, 164, 165, 400]
    cu_kv = [0, 64, 200, 329, 330]
    lay = O.varlen_layout(cu_q, cu_kv)
    assert np.array_equal(lay["pack_index_q"], _brute_pack_index(cu_q))
    assert np.array_equal(lay["pack_index_kv"], _brute_pack_index(cu_kv))
    assert lay["nq"] == [2, 1, 1, 4] and lay["nkv"] == [1, 3, 3, 1]
    assert lay["qoff"] == [0, 2, 3, 4] and lay["kvoff"] == [0, 1, 4, 7]
    vq = [[30, 64, 6], [64], [1], [64, 64, 64, 43]]
    lay = O.varlen_layout(cu_q, cu_kv, q_block_sizes_list=vq)
    assert np.array_equal(lay["pack_index_q"], _brute_pack_index(cu_q, vq))
    # rebase: local index + the sequence's first packed KV block
    lay = O.varlen_layout(cu_q, cu_kv)
    rows = sum(lay["nq"])
    idx = np.zeros((2, rows, 2), dtype=np.int32)
    num = np.ones((2, rows), dtype=np.int32)
    idx[:, :, 1] = -1
    seq_of_row = np.repeat(np.arange(4), lay["nq"])
    for r in range(rows):
        idx[:, r, 0] = lay["nkv"][seq_of_row[r]] - 1
    reb = O.rebase_q2k_idx(idx, num, lay)
    for r in range(rows):
        s = seq_of_row[r]
        assert reb[0, r, 0] == lay["kvoff"][s] + lay["nkv"][s] - 1 and reb[0, r, 1] == -1


def _varlen_case(rng, q_lens, kv_lens, H, D, frac):
    cu_q = [0] + list(np.cumsum(q_lens))
    cu_kv = [0] + list(np.cumsum(kv_lens))
    q = _bf16_like(rng, (H, cu_q[-1], D))
    k = _bf16_like(rng, (H, cu_kv[-1], D))
    v = _bf16_like(rng, (H, cu_kv[-1], D))
    nq = [-(-n // BLOCK) for n in q_lens]
    nkv = [-(-n // BLOCK) for n in kv_lens]
    width = max(max(1, int(frac * n)) for n in nkv)
    rows = []
    nums = []
    for i in range(len(q_lens)):
        kk = max(1, min(nkv[i], int(frac * nkv[i])))
        for _ in range(nq[i]):
            r = np.full((H, width), -1, dtype=np.int32)
            for h in range(H):
                r[h, :kk] = np.sort(rng.choice(nkv[i], size=kk, replace=False))
            rows.append(r)
            nums.append(np.full(H, kk, dtype=np.int32))
    idx = np.stack(rows, axis=1)
    num = np.stack(nums, axis=1)
    return cu_q, cu_kv, q, k, v, idx, num


def check_varlen_equals_per_sequence(O):
    """Packed result equals running each sequence on its own, exactly
    ([varlen] Test plan: error = 0.0)."""
    rng = _rng(10)
    for q_lens, kv_lens, H, D, frac in (([130, 64, 300], [70, 200, 64], 2, 16, 0.5),
                                         ([64, 64], [64, 64], 1, 8, 1.0),
                                         ([1, 5, 70], [3, 64, 1], 2, 8, 1.0)):
        cu_q, cu_kv, q, k, v, idx, num = _varlen_case(rng, q_lens, kv_lens, H, D, frac)
        got = O.block_sparse_attn_varlen(q, k, v, cu_q, cu_kv, idx, num, 0.3)
        row = 0
        for i in range(len(q_lens)):
            qs = list(O._seq_block_sizes(q_lens[i], None))
            ks = list(O._seq_block_sizes(kv_lens[i], None))
            qi = np.zeros((1, H, BLOCK * len(qs), D))
            ki = np.zeros((1, H, BLOCK * len(ks), D))
            vi = np.zeros((1, H, BLOCK * len(ks), D))
            qi[0, :, :q_lens[i]] = q[:, cu_q[i]:cu_q[i + 1]]
            ki[0, :, :kv_lens[i]] = k[:, cu_kv[i]:cu_kv[i + 1]]
            vi[0, :, :kv_lens[i]] = v[:, cu_kv[i]:cu_kv[i + 1]]
            o = O.block_sparse_attention(qi, ki, vi, idx[None, :, row:row + len(qs)],
                                         num[None, :, row:row + len(qs)], qs, ks, 0.3)
            assert np.array_equal(got[:, cu_q[i]:cu_q[i + 1]], o[0, :, :q_lens[i]])
            row += len(qs)
    # a single sequence is the non-varlen call
    cu_q, cu_kv, q, k, v, idx, num = _varlen_case(rng, [200], [150], 2, 8, 0.7)
    got = O.block_sparse_attn_varlen(q, k, v, cu_q, cu_kv, idx, num, 0.3)
    qs, ks = O._seq_block_sizes(200, None), O._seq_block_sizes(150, None)
    qp = np.zeros((1, 2, 256, 8)); qp[0, :, :200] = q
    kp = np.zeros((1, 2, 192, 8)); kp[0, :, :150] = k
    vp = np.zeros((1, 2, 192, 8)); vp[0, :, :150] = v
    o = O.block_sparse_attention(qp, kp, vp, idx[None], num[None], qs, ks, 0.3)
    assert np.array_equal(got, o[0, :, :200])


def check_varlen_dense_vs_library(O):
    """Varlen with topk = all blocks is per-sequence dense attention."""
    rng = _rng(11)
    cu_q, cu_kv, q, k, v, idx, num = _varlen_case(rng, [100, 64, 7], [90, 128, 200], 2, 16, 1.0)
    got = O.block_sparse_attn_varlen(q, k, v, cu_q, cu_kv, idx, num, 0.25)
    for i in range(3):
        want = _sdpa(q[:, cu_q[i]:cu_q[i + 1]], k[:, cu_kv[i]:cu_kv[i + 1]],
                     v[:, cu_kv[i]:cu_kv[i + 1]], 0.25)
        assert np.allclose(got[:, cu_q[i]:cu_q[i + 1]], want, atol=1e-12)


# ---------------------------------------------------------------------------
# metadata
# ---------------------------------------------------------------------------
def check_metadata(O):
    for (T, Hh, W) in ((5, 5, 5), (9, 30, 52), (8, 4, 12), (1, 3, 7)):
        m = O.build_vsa_metadata(T, Hh, W)
        N = T * Hh * W
        perm, rev = m["tile_partition_indices"], m["reverse_tile_partition_indices"]
        sizes, npi = m["variable_block_sizes"], m["non_pad_index"]
        assert np.array_equal(np.sort(perm), np.arange(N))
        assert np.array_equal(perm[rev], np.arange(N)) and np.array_equal(rev[perm], np.arange(N))
        assert sizes.sum() == N and sizes.max() <= 64 and sizes.min() >= 1
        nT, nH, nW = -(-T // 4), -(-Hh // 4), -(-W // 4)
        assert m["n_tiles"] == nT * nH * nW
        off = 0
        for j, s in enumerate(sizes):
            toks = perm[off:off + s]
            t, h, w = toks // (Hh * W), (toks // W) % Hh, toks % W
            bt, bh, bw = j // (nH * nW), (j // nW) % nH, j % nW
            assert np.all(t // 4 == bt) and np.all(h // 4 == bh) and np.all(w // 4 == bw)
            assert np.all(np.diff(toks) > 0)   # row-major inside a tile
            ext = (min(T, 4 * bt + 4) - 4 * bt) * (min(Hh, 4 * bh + 4) - 4 * bh) * (min(W, 4 * bw + 4) - 4 * bw)
            assert s == ext
            assert np.array_equal(npi[off:off + s], np.arange(64 * j, 64 * j + s))
            off += s
        x = np.arange(N, dtype=np.float64)[None, None, :, None]
        assert np.array_equal(O.untile(O.tile_and_pad(x, m), m), x)
    m = O.build_vsa_metadata(8, 4, 12)
    assert np.all(m["variable_block_sizes"] == 64) and np.array_equal(m["non_pad_index"], np.arange(384))
    # the 9 x 30 x 52 video latent: per-axis tile extents are t (4,4,1),
    # h (4 x7, 2), w (4 x13), so the tile sizes follow by counting products
    m = O.build_vsa_metadata(9, 30, 52)
    counts = {}
    for s in m["variable_block_sizes"]:
        counts[int(s)] = counts.get(int(s), 0) + 1
    want = {}
    for et in (4, 4, 1):
        for eh in [4] * 7 + [2]:
            for ew in [4] * 13:
                want[et * eh * ew] = want.get(et * eh * ew, 0) + 1
    assert m["n_tiles"] == 312 and counts == want == {64: 182, 32: 26, 16: 91, 8: 13}


def check_page_figures(O):
    """Sizes printed on the combine page pin the BHSD bf16 layout arithmetic."""
    with open(os.path.join(GOLDEN, "combine_page_figures.json")) as f:
        g = json.load(f)
    B, H, S, D = g["shape_bhsd"]
    nbytes = B * H * S * D * g["bytes_per_element"]
    assert round(nbytes / 2**20, 1) == g["full_tensor_mib"]
    assert g["peak_gated_before_mib"] - g["peak_gated_after_mib"] == g["saved_gated_mib"]
    assert abs(g["saved_gated_mib"] - 3 * nbytes / 2**20) < 1.0
    assert S % g["block"] == 0 and S // g["block"] == 242
    # one block-resolution coarse output per 64 slots: the combine reads
    # out_c of B*H*(S/64)*D elements, 1/64 of a full-sequence tensor
    sizes = [g["block"]] * (S // g["block"])
    oc = np.arange(len(sizes), dtype=np.float64)[None, None, :, None]
    out = O.combine(oc, np.zeros((1, 1, S, 1)), None, sizes)
    assert np.array_equal(out[0, 0, :, 0], np.repeat(np.arange(len(sizes)), g["block"]))


def check_block_map_to_indices(O):
    """Bool block maps to index rows: against a plain per-entry loop on
    random maps (all-False and all-True rows included), the round trip
    indices -> map -> indices on a top-k selection, and attention from the
    map's indices against masked dense attention (torch SDPA, fp64)."""
    rng = _rng(21)
    bm = rng.random((2, 3, 5, 37)) < 0.3
    bm[0, 0, 0] = False
    bm[1, 2, 4] = True
    idx, num = O.block_map_to_indices(bm)
    for pos in np.ndindex(*bm.shape[:-1]):
        want = [c for c in range(bm.shape[-1]) if bm[pos][c]]
        assert num[pos] == len(want)
        assert list(idx[pos][:len(want)]) == want
        assert np.all(idx[pos][len(want):] == -1)
    # round trip with a top-k selection
    scores = rng.standard_normal((1, 2, 6, 11))
    sel, sn = O.select_topk(scores, 4)
    back = np.zeros((1, 2, 6, 11), dtype=bool)
    for b, h, a in np.ndindex(1, 2, 6):
        back[b, h, a, sel[b, h, a, :sn[b, h, a]]] = True
    idx2, num2 = O.block_map_to_indices(back)
    assert np.array_equal(num2, sn) and np.array_equal(idx2[..., :4], sel)
    # attention through the map equals masked dense attention
    B, H, D = 1, 2, 16
    q_sizes, kv_sizes = [64, 40, 64], [64, 9, 64, 64, 30]
    q = _padded(rng, B, H, q_sizes, D)
    k = _padded(rng, B, H, kv_sizes, D, pad_value=3.0)
    v = _padded(rng, B, H, kv_sizes, D, pad_value=3.0)
    bm = rng.random((B, H, len(q_sizes), len(kv_sizes))) < 0.5
    bm[..., 0] = True
    idx, num = O.block_map_to_indices(bm)
    got = O.block_sparse_attention(q, k, v, idx, num, q_sizes, kv_sizes, 0.25)
    mask = np.zeros((B, H, BLOCK * len(q_sizes), BLOCK * len(kv_sizes)), dtype=bool)
    for b, h, a, c in zip(*np.nonzero(bm)):
        mask[b, h, BLOCK * a:BLOCK * (a + 1), BLOCK * c:BLOCK * c + kv_sizes[c]] = True
    want = _sdpa(q, k, v, 0.25, mask)
    qr = _real_rows(q_sizes)
    assert np.allclose(got[:, :, qr], want[:, :, qr], atol=1e-12)


def _check_large_block(O, blk, seed):
    """Blocks of ``blk`` slots (tile volume 128 or 256): pooling closed forms,
    the dense limit against torch SDPA over the real tokens, arbitrary
    selections against masked SDPA, the ungated combine as broadcast +
    sparse, and the whole forward with topk = all equal to dense attention
    plus out_c."""
    rng = _rng(seed)
    B, H, D = 1, 2, 16

    def padded(sizes, pad_value=0.0):
        x = np.full((B, H, blk * len(sizes), D), pad_value)
        for j, m in enumerate(sizes):
            x[:, :, blk * j:blk * j + m] = _bf16_like(rng, (B, H, m, D))
        return x

    def rows(sizes):
        return np.concatenate([np.arange(blk * j, blk * j + m) for j, m in enumerate(sizes)])

    # pooling: a ramp over the real slots has the mean of its real values
    part = blk // 2 + 6   # a partial block past the half (two sub-tiles at 256)
    sizes = [blk, part, 1]
    x = np.zeros((1, 1, blk * 3, 1))
    for j, m in enumerate(sizes):
        x[0, 0, blk * j:blk * j + m, 0] = np.arange(m)
    x[0, 0, blk * 1 + part:blk * 2, 0] = 1e6   # padding must not count
    got = O.block_pool(x, sizes, block=blk)
    assert np.allclose(got[0, 0, :, 0], [(m - 1) / 2 for m in sizes])
    # dense limit, partial blocks, nq != nkv
    q_sizes, kv_sizes = [blk, blk - 28], [blk, 17, blk]
    q, k, v = padded(q_sizes), padded(kv_sizes, 7.0), padded(kv_sizes, -7.0)
    nkv = len(kv_sizes)
    idx = np.broadcast_to(np.arange(nkv, dtype=np.int32), (B, H, 2, nkv)).copy()
    num = np.full((B, H, 2), nkv, dtype=np.int32)
    scale = 1 / np.sqrt(D)
    got = O.block_sparse_attention(q, k, v, idx, num, q_sizes, kv_sizes, scale, block=blk)
    qr, kr = rows(q_sizes), rows(kv_sizes)
    want = _sdpa(q[:, :, qr], k[:, :, kr], v[:, :, kr], scale)
    assert np.allclose(got[:, :, qr], want, atol=1e-12)
    # arbitrary selections: masked SDPA
    idx = np.array([[[[2, -1], [0, 1]], [[1, 2], [2, -1]]]], dtype=np.int32)
    num = np.array([[[1, 2], [2, 1]]], dtype=np.int32)
    got = O.block_sparse_attention(q, k, v, idx, num, q_sizes, kv_sizes, 0.3, block=blk)
    mask = np.zeros((B, H, blk * 2, blk * 3), dtype=bool)
    for b, h, a in np.ndindex(B, H, 2):
        for j in range(num[b, h, a]):
            c = idx[b, h, a, j]
            mask[b, h, blk * a:blk * (a + 1), blk * c:blk * c + kv_sizes[c]] = True
    want = _sdpa(q, k, v, 0.3, mask)
    assert np.allclose(got[:, :, qr], want[:, :, qr], atol=1e-12)
    # whole forward, topk = all: out = out_c (per block) + dense attention
    res = O.vsa_forward(q, k, v, None, q_sizes, kv_sizes, nkv, block=blk)
    dense = _sdpa(q[:, :, qr], k[:, :, kr], v[:, :, kr], scale)
    oc = res["out_c"]
    bcast = np.concatenate([np.repeat(oc[:, :, a:a + 1], m, axis=2) for a, m in enumerate(q_sizes)],
                           axis=2)
    assert np.allclose(res["out"][:, :, qr], bcast + dense, atol=1e-12)
    pad = np.setdiff1d(np.arange(blk * 2), qr)
    assert np.all(res["out"][:, :, pad] == 0.0)


def check_block128(O):
    """128-slot blocks (VSA-128 tiles)."""
    _check_large_block(O, 128, 31)


def check_block256(O):
    """256-slot blocks (VSA-256 tiles)."""
    _check_large_block(O, 256, 37)


def _torch_sparse_forward(q, k, v, idx, num, q_sizes, kv_sizes, scale, block=BLOCK):
    """Block-sparse attention written in torch ops (row gathers with
    repeats, masked softmax) so that autograd differentiates it: a second,
    independent route to the gradients."""
    B, H, Sq, D = q.shape
    out = torch.zeros_like(q)
    outs = []
    for b in range(B):
        for h in range(H):
            for a in range(len(q_sizes)):
                mq = q_sizes[a]
                n = int(num[b, h, a])
                if n <= 0:
                    continue
                rows = torch.cat([torch.arange(block * int(c), block * int(c) + kv_sizes[int(c)])
                                  for c in idx[b, h, a, :n]])
                qa = q[b, h, block * a:block * a + mq]
                p = torch.softmax(scale * qa @ k[b, h, rows].T, dim=-1)
                outs.append(((b, h, a, mq), p @ v[b, h, rows]))
    for (b, h, a, mq), o in outs:
        out = out.index_put((torch.tensor([b]), torch.tensor([h]),
                             torch.arange(block * a, block * a + mq)), o)
    return out


def check_backward(O):
    """dq, dk, dv against torch autograd (fp64) of an independently written
    forward, with duplicates, partial blocks, an empty selection and
    nq != nkv; against central finite differences on a tiny case; lse
    against torch's logsumexp; and the k2q index against a brute-force
    count."""
    rng = _rng(41)
    B, H, D = 1, 2, 8
    q_sizes, kv_sizes = [64, 37, 64], [64, 64, 20, 64]
    q = _padded(rng, B, H, q_sizes, D)
    k = _padded(rng, B, H, kv_sizes, D, pad_value=2.0)
    v = _padded(rng, B, H, kv_sizes, D, pad_value=-2.0)
    do = _padded(rng, B, H, q_sizes, D)
    idx = np.array([[[[1, 2, 2, -1], [0, 3, -1, -1], [3, 1, 0, 2]],
                     [[0, -1, -1, -1], [0, 0, 0, 0], [2, 3, -1, -1]]]], dtype=np.int32)
    num = np.array([[[3, 2, 4], [0, 4, 2]]], dtype=np.int32)
    scale = 0.37
    dq, dk, dv = O.block_sparse_attention_backward(q, k, v, do, idx, num, q_sizes, kv_sizes, scale)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    out = _torch_sparse_forward(tq, tk, tv, idx, num, q_sizes, kv_sizes, scale)
    out.backward(torch.tensor(do))
    for got, want in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.allclose(got, want.numpy(), atol=1e-12)
    assert np.all(dq[0, 1, 0:64] == 0.0)           # empty selection: no gradient
    # finite differences on a few coordinates of a tiny case
    f = lambda qq, kk, vv: float((O.block_sparse_attention(qq, kk, vv, idx, num, q_sizes, kv_sizes,
                                                            scale) * do).sum())
    eps = 1e-6
    for arr, grad, where in ((q, dq, (0, 0, 70, 3)), (k, dk, (0, 1, 130, 5)), (v, dv, (0, 0, 140, 1)),
                             (k, dk, (0, 0, 200, 0))):
        plus, minus = arr.copy(), arr.copy()
        plus[where] += eps
        minus[where] -= eps
        args_p = [plus if x is arr else x for x in (q, k, v)]
        args_m = [minus if x is arr else x for x in (q, k, v)]
        fd = (f(*args_p) - f(*args_m)) / (2 * eps)
        assert abs(fd - grad[where]) < 1e-6, (where, fd, grad[where])
    # lse against logsumexp over the selected real keys
    lse = O.block_sparse_lse(q, k, idx, num, q_sizes, kv_sizes, scale)
    rows = np.concatenate([np.arange(64 * c, 64 * c + kv_sizes[c]) for c in [3, 1, 0, 2]])
    want = torch.logsumexp(scale * torch.tensor(q[0, 0, 128:192]) @ torch.tensor(k[0, 0, rows]).T, dim=-1)
    assert np.allclose(lse[0, 0, 128:192], want.numpy(), atol=1e-12)
    assert np.all(np.isneginf(lse[0, 1, 0:64]))
    # k2q: brute-force multiplicities
    k2q, cnt, k2n = O.build_k2q(idx, num, len(kv_sizes))
    for h in range(H):
        for c in range(len(kv_sizes)):
            want = [(a, int(np.sum(idx[0, h, a, :num[0, h, a]] == c))) for a in range(len(q_sizes))]
            want = [(a, m) for a, m in want if m]
            assert k2n[0, h, c] == len(want)
            assert [(int(k2q[0, h, c, t]), int(cnt[0, h, c, t])) for t in range(k2n[0, h, c])] == want
            assert np.all(k2q[0, h, c, len(want):] == -1)



def check_backward_large_blocks(O):
    """At 128- and 256-slot blocks: dq, dk, dv against torch autograd (fp64)
    of the independently written forward at that block size, and lse against
    torch's logsumexp, with partial query and key blocks (some holding fewer
    than 64 real rows), duplicates and an empty selection."""
    rng = _rng(43)
    B, H, D = 1, 2, 8
    for blk, q_sizes, kv_sizes in ((128, [128, 50, 100], [128, 30, 70, 128]),
                                   (256, [256, 130], [200, 40, 256])):
        nkv = len(kv_sizes)

        def padded(sizes, pad_value=0.0):
            x = np.full((B, H, blk * len(sizes), D), pad_value, dtype=np.float64)
            for j, m in enumerate(sizes):
                x[:, :, blk * j:blk * j + m] = _bf16_like(rng, (B, H, m, D))
            return x

        q, k, v, do = padded(q_sizes), padded(kv_sizes, 2.0), padded(kv_sizes, -2.0), padded(q_sizes)
        width = 4
        idx = np.full((B, H, len(q_sizes), width), -1, dtype=np.int32)
        num = np.zeros((B, H, len(q_sizes)), dtype=np.int32)
        for h, a in np.ndindex(H, len(q_sizes)):
            if (h, a) == (1, 0):
                continue                                  # empty selection
            n = int(rng.integers(1, width + 1))
            idx[0, h, a, :n] = rng.integers(0, nkv, size=n)   # duplicates allowed
            num[0, h, a] = n
        scale = 0.41
        dq, dk, dv = O.block_sparse_attention_backward(q, k, v, do, idx, num, q_sizes, kv_sizes,
                                                       scale, block=blk)
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        out = _torch_sparse_forward(tq, tk, tv, idx, num, q_sizes, kv_sizes, scale, block=blk)
        out.backward(torch.tensor(do))
        for got, want in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
            assert np.allclose(got, want.numpy(), atol=1e-12), blk
        assert np.all(dq[0, 1, 0:blk] == 0.0)
        lse = O.block_sparse_lse(q, k, idx, num, q_sizes, kv_sizes, scale, block=blk)
        for h, a in np.ndindex(H, len(q_sizes)):
            rows_q = slice(blk * a, blk * a + q_sizes[a])
            if num[0, h, a] == 0:
                assert np.all(np.isneginf(lse[0, h, rows_q]))
                continue
            rows = np.concatenate([np.arange(blk * int(c), blk * int(c) + kv_sizes[int(c)])
                                   for c in idx[0, h, a, :num[0, h, a]]])
            want = torch.logsumexp(scale * torch.tensor(q[0, h, rows_q]) @ torch.tensor(k[0, h, rows]).T,
                                   dim=-1)
            assert np.allclose(lse[0, h, rows_q], want.numpy(), atol=1e-12), (blk, h, a)
            assert np.all(lse[0, h, blk * a + q_sizes[a]:blk * (a + 1)] == 0.0)

ALL_CHECKS = [
    check_pool_closed_forms, check_coarse_special_cases, check_coarse_vs_library,
    check_topk_brute_force, check_topk_edge_cases, check_sparse_dense_equivalence,
    check_sparse_vs_masked_library, check_sparse_invariants, check_combine,
    check_forward_dense_limit, check_varlen_pack_indices, check_varlen_equals_per_sequence,
    check_varlen_dense_vs_library, check_metadata, check_page_figures,
    check_block_map_to_indices, check_block128, check_block256, check_backward,
    check_backward_large_blocks,
]
