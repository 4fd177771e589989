"""Backward at 128- and 256-slot blocks on the GPU, through the C ABI.

* the forward's per-row log-sum-exp from the 128-row kernel, with and
  without the logit-bound pass, against the oracle at that block size;
* dq, dk, dv of ``block_sparse_attn_backward_ex`` against the oracle's
  gradients at that block size (tolerances as for the 64-slot backward);
* the same call equal bit for bit to the 64-slot backward on the selection
  rewritten over 64-slot sub-blocks, written out below from the entry's
  definition (every listed block becomes its sub-blocks holding real keys,
  in order; query sub-blocks without real rows list nothing).

Cases: query blocks whose later sub-blocks hold no real rows, KV blocks with
fewer real keys than one sub-block, duplicated and empty selections, more
work items than SMs."""
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


def _rows(sizes, blk):
    return np.concatenate([np.arange(blk * j, blk * j + m) for j, m in enumerate(sizes)])


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


def _rewrite64(idx, num, qs, ks, blk):
    """The selection over 64-slot sub-blocks: sub-block r*c + i holds slots
    64 i .. 64 i + 63 of block c (r = blk / 64)."""
    r = blk // 64
    B, H, nq, width = idx.shape
    qs64 = [max(0, min(64, m - 64 * i)) for m in qs for i in range(r)]
    ks64 = [max(0, min(64, m - 64 * i)) for m in ks for i in range(r)]
    idx64 = np.full((B, H, nq * r, width * r), -1, dtype=np.int32)
    num64 = np.zeros((B, H, nq * r), dtype=np.int32)
    for b, h, a in np.ndindex(B, H, nq):
        subs = [r * int(c) + i for c in idx[b, h, a, :num[b, h, a]] for i in range(r)
                if ks64[r * int(c) + i] > 0]
        for i in range(r):
            if qs64[r * a + i] > 0:
                idx64[b, h, r * a + i, :len(subs)] = subs
                num64[b, h, r * a + i] = len(subs)
    return idx64, num64, qs64, ks64


CASES = [
    # D, B, H, block, q sizes, kv sizes, width, duplicates, seed
    (128, 1, 2, 128, [128, 100, 50, 128], [128, 70, 128, 30, 128], 3, True, 21),
    (64, 2, 2, 128, [128] * 3, [128, 1, 128, 65], 4, False, 22),
    (128, 1, 2, 256, [256, 130, 60], [256, 200, 40, 256], 3, False, 23),
    (64, 1, 3, 256, [256, 7, 192], [256, 64, 129], 3, True, 24),
    (128, 1, 4, 128, [128] * 40, [128] * 12, 4, False, 25),   # 320 query sub-blocks
]


@pytest.mark.parametrize("case", CASES,
                         ids=lambda c: f"D{c[0]}-B{c[1]}H{c[2]}-blk{c[3]}-nq{len(c[4])}-nkv{len(c[5])}")
def test_backward_blocks_match_oracle_and_64_slot_call(case):
    D, B, H, blk, qs, ks, width, dup, seed = case
    rng = np.random.default_rng(seed)
    q, k, v = (I.padded_normal_bhsd(B, H, s, D, 1400 + seed, i, block=blk)
               for i, s in enumerate((qs, ks, ks)))
    do = I.padded_normal_bhsd(B, H, qs, D, 1400 + seed, 7, block=blk)
    idx, num = _selection(rng, B, H, len(qs), len(ks), width, dup, empty={(0, 0, 1)})
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), do.to(DEV)
    ti, tn = torch.from_numpy(idx).to(DEV), torch.from_numpy(num).to(DEV)
    out, lse = vsa.block_sparse_attn_from_indices(qd, kd, vd, ti, tn, qs, ks, block=blk,
                                                  return_lse=True)
    _, lse_nb = vsa.block_sparse_attn_from_indices(qd, kd, vd, ti, tn, qs, ks, block=blk,
                                                   logit_bound=False, return_lse=True)
    dq, dk, dv = vsa.block_sparse_attn_backward(qd, kd, vd, out, dod, lse, ti, tn, qs, ks, block=blk)
    vsa.check_device_status()
    qn, kn, vn, don = P.to_np(q), P.to_np(k), P.to_np(v), P.to_np(do)
    scale = O.default_scale(D)
    rr, kr = _rows(qs, blk), _rows(ks, blk)
    pad_q = np.setdiff1d(np.arange(q.shape[2]), rr)
    # log-sum-exp: oracle on real rows, -inf where nothing is selected, 0 on padding
    want_lse = O.block_sparse_lse(qn, kn, idx, num, qs, ks, scale, block=blk)
    fin = np.isfinite(want_lse[:, :, rr])
    for got in (P.to_np(lse), P.to_np(lse_nb)):
        np.testing.assert_allclose(got[:, :, rr][fin], want_lse[:, :, rr][fin], rtol=1e-4, atol=2e-3)
        assert np.all(np.isneginf(got[:, :, rr][~fin]))
        assert np.all(got[:, :, pad_q] == 0.0)
    # gradients against the oracle at this block size
    wq, wk, wv = O.block_sparse_attention_backward(qn, kn, vn, don, idx, num, qs, ks, scale, block=blk)
    _grad_close(P.to_np(dq)[:, :, rr], wq[:, :, rr], "dq")
    _grad_close(P.to_np(dk)[:, :, kr], wk[:, :, kr], "dk")
    _grad_close(P.to_np(dv)[:, :, kr], wv[:, :, kr], "dv")
    for g, rows in ((dq, rr), (dk, kr), (dv, kr)):
        pad = np.setdiff1d(np.arange(g.shape[2]), rows)
        assert np.all(P.to_np(g)[:, :, pad] == 0.0)
    # bit for bit the 64-slot backward on the rewritten selection
    i64, n64, qs64, ks64 = _rewrite64(idx, num, qs, ks, blk)
    g64 = vsa.block_sparse_attn_backward(qd, kd, vd, out, dod, lse, torch.from_numpy(i64).to(DEV),
                                         torch.from_numpy(n64).to(DEV), qs64, ks64)
    vsa.check_device_status()
    for a, b, what in zip((dq, dk, dv), g64, ("dq", "dk", "dv")):
        assert torch.equal(a, b), f"{what} differs from the 64-slot call on the rewritten selection"


def test_backward_blocks_out_of_range_entry_reported():
    """An index outside [0, n_kv_blocks) is skipped and reported, as in the
    forward."""
    B, H, D, blk = 1, 1, 64, 128
    qs, ks = [128, 128], [128, 128]
    q, k, v = (I.padded_normal_bhsd(B, H, s, D, 1450, i, block=blk) for i, s in enumerate((qs, ks, ks)))
    idx = np.array([[[[0, 1], [1, 0]]]], dtype=np.int32)
    num = np.array([[[2, 2]]], dtype=np.int32)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    ti, tn = torch.from_numpy(idx).to(DEV), torch.from_numpy(num).to(DEV)
    out, lse = vsa.block_sparse_attn_from_indices(qd, kd, vd, ti, tn, block=blk, return_lse=True)
    vsa.check_device_status()
    bad = ti.clone()
    bad[0, 0, 1, 1] = 5
    vsa.block_sparse_attn_backward(qd, kd, vd, out, qd, lse, bad, tn, block=blk)
    assert vsa.get_device_status() == 6  # VSA_ERR_INDEX_RANGE
    assert vsa.get_device_status() == 0  # read clears it
