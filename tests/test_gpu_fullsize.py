"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times.  Indices are checked in full.  Outputs are checked against
the fp64 oracle on every query block of every head for the H3-like, the
video-tiled and the varlen workloads (the oracle needs about half a minute
for the largest), and on every head x 32 query blocks for the long
(32768-token) workloads, whose dense case alone would take the oracle many
minutes in full."""
import numpy as np
import pytest
import torch

from block_sparse_attention_15_b200 import binding as vsa
from block_sparse_attention_15_b200 import inputs as I
from oracle import vsa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _all_items(B, H, nq):
    return [(b, h, a) for b in range(B) for h in range(H) for a in range(nq)]


def _per_head_items(rng, B, H, nq, per_head):
    """per_head distinct query blocks of every (batch, head), the first and
    last block always among them."""
    items = []
    for b in range(B):
        for h in range(H):
            blocks = {0, nq - 1}
            blocks.update(int(a) for a in rng.choice(nq, size=min(nq, per_head) - 2, replace=False))
            while len(blocks) < min(nq, per_head):
                blocks.add(int(rng.integers(nq)))
            items += [(b, h, a) for a in sorted(blocks)]
    return items


def _rows_of(items, q_sizes):
    return [(b, h, np.arange(64 * a, 64 * a + q_sizes[a])) for b, h, a in items]


def _run_forward_case(wl: I.Workload, q, k, v, gate, seed, per_head=None):
    """Forward on the GPU; stage by stage against the oracle.  Outputs are
    compared on every query block (per_head None) or on per_head blocks of
    every head."""
    out, idx, num, out_c = vsa.vsa_forward(
        q.to(DEV), k.to(DEV), v.to(DEV), None if gate is None else gate.to(DEV),
        None if all(s == 64 for s in wl.q_block_sizes) else wl.q_block_sizes,
        None if all(s == 64 for s in wl.kv_block_sizes) else wl.kv_block_sizes,
        topk=wl.topk, return_out_c=True)
    vsa.check_device_status()
    qn, kn, vn = P.to_np(q), P.to_np(k), P.to_np(v)
    scale = O.default_scale(wl.D)
    qc, kc, vc = (O.block_pool(x, s) for x, s in ((qn, wl.q_block_sizes), (kn, wl.kv_block_sizes),
                                                  (vn, wl.kv_block_sizes)))
    scores, oc = O.coarse_attention(qc, kc, vc, scale)
    np.testing.assert_allclose(P.to_np(out_c), oc, rtol=1e-4, atol=1e-6)
    idx_np, num_np = P.to_np(idx), P.to_np(num)
    P.check_topk(idx_np, num_np, scores, wl.topk)
    rng = np.random.default_rng(seed)
    items = (_all_items(wl.B, wl.H, wl.nq) if per_head is None
             else _per_head_items(rng, wl.B, wl.H, wl.nq, per_head))
    o_s = O.block_sparse_attention(qn, kn, vn, idx_np, num_np, wl.q_block_sizes,
                                   wl.kv_block_sizes, scale, items=items)
    want = O.combine(oc, o_s, None if gate is None else P.to_np(gate), wl.q_block_sizes)
    got = P.to_np(out)
    g_rows, w_rows = [], []
    for b, h, rows in _rows_of(items, wl.q_block_sizes):
        g_rows.append(got[b, h, rows])
        w_rows.append(want[b, h, rows])
    P.assert_outputs_close(np.concatenate(g_rows), np.concatenate(w_rows), wl.name)
    # padded rows are 0 everywhere
    rr = P.real_rows(wl.q_block_sizes)
    if len(rr) < got.shape[2]:
        pad = np.setdiff1d(np.arange(got.shape[2]), rr)
        assert np.all(got[:, :, pad] == 0.0)
    return got, idx_np, num_np


def _inputs(wl: I.Workload):
    q = I.padded_normal_bhsd(wl.B, wl.H, wl.q_block_sizes, wl.D, wl.seed, I.STREAM_Q)
    k = I.padded_normal_bhsd(wl.B, wl.H, wl.kv_block_sizes, wl.D, wl.seed, I.STREAM_K)
    v = I.padded_normal_bhsd(wl.B, wl.H, wl.kv_block_sizes, wl.D, wl.seed, I.STREAM_V)
    gate = I.gate_bf16((wl.B, 64 * wl.nq, wl.H, wl.D), wl.seed) if wl.gated else None
    return q, k, v, gate


def test_h3_like_full():
    """B1 H56 D128 S15488 (242 blocks), top-48, gated: the benchmark's shape."""
    wl = I.workload_h3()
    q, k, v, gate = _inputs(wl)
    _run_forward_case(wl, q, k, v, gate, seed=1)


def test_video_tiled_full():
    """9x30x52 latent in 4x4x4 tiles (312 blocks, edge sizes 32/16/8), H12
    D128, top 25% = 78, gated; tokens placed by the device gather."""
    meta = vsa.build_vsa_metadata(9, 30, 52)
    sizes = [int(s) for s in meta["variable_block_sizes"]]
    wl = I.Workload("video-tiled", 1, 12, 128, sizes, sizes, I.topk_count(0.25, len(sizes)),
                    True, 1002)
    N = sum(sizes)
    slot = torch.from_numpy(meta["slot_token"]).to(DEV)
    toks = [I.normal_bf16((1, wl.H, N, wl.D), wl.seed, s) for s in range(3)]
    q, k, v = (vsa.gather_tokens(t.reshape(wl.H, N, wl.D).to(DEV), slot).reshape(1, wl.H, -1, wl.D).cpu()
               for t in toks)
    gate = I.gate_bf16((1, 64 * wl.nq, wl.H, wl.D), wl.seed)
    got, _, _ = _run_forward_case(wl, q, k, v, gate, seed=2)
    # back to token order
    back = vsa.scatter_tokens(torch.from_numpy(got).to(torch.bfloat16).reshape(wl.H, -1, wl.D).to(DEV),
                              slot, N)
    want = O.untile(got, O.build_vsa_metadata(9, 30, 52))
    assert np.array_equal(P.to_np(back).reshape(want.shape), want)


@pytest.mark.parametrize("frac,gated", [(0.05, True), (0.10, False), (1.0, True)])
def test_long_sequence(frac, gated):
    """B1 H40 D128 S32768 (512 blocks) at top 5% / 10% / 100%."""
    wl = I.workload_long(frac, gated)
    q, k, v, gate = _inputs(wl)
    got, idx, num = _run_forward_case(wl, q, k, v, gate, seed=3, per_head=32)
    if frac == 1.0:
        # dense: every block selected, so the sparse branch is full attention;
        # brute force on sampled rows (fp64, all 32768 keys)
        assert np.all(idx[..., :512] == np.arange(512))
        gate_np = P.to_np(gate)
        qn = P.to_np(q)
        kn, vn = P.to_np(k)[0], P.to_np(v)[0]
        rng = np.random.default_rng(4)
        scale = O.default_scale(wl.D)
        out_c = O.coarse_attention(O.block_pool(qn, wl.q_block_sizes),
                                   O.block_pool(P.to_np(k), wl.kv_block_sizes),
                                   O.block_pool(P.to_np(v), wl.kv_block_sizes), scale)[1]
        g_rows, w_rows = [], []
        for _ in range(16):
            h, s = int(rng.integers(wl.H)), int(rng.integers(32768))
            logits = scale * (kn[h] @ qn[0, h, s])
            w = np.exp(logits - logits.max())
            dense = (w / w.sum()) @ vn[h]
            w_rows.append(out_c[0, h, s // 64] * gate_np[0, s, h] + dense)
            g_rows.append(got[0, h, s])
        P.assert_outputs_close(np.stack(g_rows), np.stack(w_rows), "dense vs brute force")


def test_varlen_full():
    """4 sequences, Q 3000/6144/9216/15488, KV 3000/7040/9216/12800, H24
    D128, top 15% per sequence, one launch."""
    H, D = 24, 128
    q_lens, kv_lens = I.VARLEN_Q_LENS, I.VARLEN_KV_LENS
    cu_q, cu_kv = I.cu_seqlens(q_lens), I.cu_seqlens(kv_lens)
    seed = 1004
    q = I.normal_bf16((H, cu_q[-1], D), seed, 0)
    k = I.normal_bf16((H, cu_kv[-1], D), seed, 1)
    v = I.normal_bf16((H, cu_kv[-1], D), seed, 2)
    nq = [-(-n // 64) for n in q_lens]
    idx, num, ks = I.varlen_random_selection(q_lens, kv_lens, H, 0.15, seed)
    assert ks == [7, 16, 21, 30]
    out, pq, pkv, reb = vsa.block_sparse_attn_varlen(
        q.to(DEV), k.to(DEV), v.to(DEV), cu_q, cu_kv, torch.from_numpy(idx).to(DEV),
        torch.from_numpy(num).to(DEV), return_aux=True)
    vsa.check_device_status()
    lay = O.varlen_layout(cu_q, cu_kv)
    assert sum(lay["nq"]) == 529 and sum(lay["nkv"]) == 501
    assert np.array_equal(P.to_np(pq), lay["pack_index_q"])
    assert np.array_equal(P.to_np(pkv), lay["pack_index_kv"])
    reb_want = O.rebase_q2k_idx(idx, num, lay)
    assert np.array_equal(P.to_np(reb), reb_want)
    # oracle on sampled packed query blocks
    qp = O.pack_tokens(P.to_np(q), lay["pack_index_q"])
    kp = O.pack_tokens(P.to_np(k), lay["pack_index_kv"])
    vp = O.pack_tokens(P.to_np(v), lay["pack_index_kv"])
    items = _all_items(1, H, sum(nq))
    o = O.block_sparse_attention(qp, kp, vp, reb_want[None], num[None], lay["q_block_sizes"],
                                 lay["kv_block_sizes"], O.default_scale(D), items=items)
    got = P.to_np(out)
    g_rows, w_rows = [], []
    for _, h, a in items:
        slots = np.arange(64 * a, 64 * a + lay["q_block_sizes"][a])
        toks = lay["pack_index_q"][slots]
        g_rows.append(got[h, toks])
        w_rows.append(o[0, h, slots])
    P.assert_outputs_close(np.concatenate(g_rows), np.concatenate(w_rows), "varlen full")
