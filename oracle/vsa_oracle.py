"""CPU oracle of the Video Sparse Attention (VSA) forward path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The CUDA library
never calls it, and it shares no code with the library: it imports numpy and
nothing else.

Everything is plain fp64 numpy, written step by step in the order the pages
describe the method; a library primitive (matmul, exp, sort) serves as a step,
and nothing is blocked, fused or reordered.  Inputs are upcast exactly from
bf16 (``tensor.float().numpy()`` is exact), so the oracle sees the same values
the GPU sees.

Sources (FastVideo pages):
  [varlen]   "[kernel] Add varlen support for block-sparse attention" (PR #1319)
  [combine]  "[perf] avoid full-sequence materialization in VSA coarse/sparse
             combine" (PR #1813)
  [release]  "[chore] release fastvideo-kernel 0.3.0" (PR #1478)
  [utils]    "[kernel] Extract VSA utility functions into fastvideo_kernel"
             (PR #1408)
  [readme]   fastvideo-kernel README

Readings where the pages leave a step open:
  R1  the coarse softmax uses the same scale as the fine one, 1/sqrt(D);
  R2  top-k ranks the scaled coarse logits; equal logits go to the lower KV
      block index;
  R3  ``q2k_idx`` rows list the selected KV blocks in ascending order; entries
      past ``q2k_num`` are -1;
  R5  a block's mean divides by its real token count (``variable_block_sizes``);
  R6  padded slots take no part: they are not pooled, not attended to, and the
      padded query rows of the output are 0;
  R7  the coarse stage attends to every KV block (no block masking);
  R8  no block is forced into the selection;
  R9  a query block with ``q2k_num == 0`` gets a sparse output of 0;
  R10 the combine is one fused multiply-add per element, rounded once;
  R11 video tiles are (4,4,4), visited in row-major (t, h, w) tile order, with
      row-major (t, h, w) token order inside a tile and clipped edge tiles;
  R12 varlen inputs are token-packed ``[H, sum(len), D]`` tensors delimited by
      cu_seqlens, and each sequence's ``q2k_idx`` rows hold local KV indices;
  R14 with 128- or 256-token tiles every step is the same with blocks of 128
      or 256 slots (pooling over the block's tokens, selections of block x
      block tiles).
"""

from __future__ import annotations

import numpy as np

BLOCK = 64


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def default_scale(D: int) -> float:
    """Softmax scale 1/sqrt(D) (reading R1)."""
    return 1.0 / np.sqrt(float(D))


# ---------------------------------------------------------------------------
# a1: block mean-pooling
# ---------------------------------------------------------------------------
def block_pool(x, block_sizes, block: int = BLOCK) -> np.ndarray:
    """Mean of each block's real tokens.

    [combine] Problem / Notes: the compression branch works on per-block means
    of q, k and v (the BSHD path takes an fp32 block sum).  Block ``j`` holds
    its ``block_sizes[j]`` real tokens in slots ``block*j ..``; padded slots
    are not pooled (R5, R6).  ``block`` is the tile volume: 64, or 128 / 256 for
    the 128- and 256-token tiles of [readme] / [release] (R14).

    x: [B, H, block*n, D]  ->  [B, H, n, D] fp64
    """
    x = _f64(x)
    B, H, S, D = x.shape
    n = len(block_sizes)
    assert S == block * n, "padded sequence must hold `block` slots per block"
    out = np.zeros((B, H, n, D), dtype=np.float64)
    for j, m in enumerate(block_sizes):
        m = int(m)
        assert 1 <= m <= block
        out[:, :, j, :] = x[:, :, block * j:block * j + m, :].sum(axis=2) / m
    return out


# ---------------------------------------------------------------------------
# a2: coarse block attention
# ---------------------------------------------------------------------------
def softmax_rows(logits: np.ndarray) -> np.ndarray:
    """Two-pass softmax over the last axis: subtract the row max, exponentiate,
    divide by the row sum."""
    m = logits.max(axis=-1, keepdims=True)
    e = np.exp(logits - m)
    return e / e.sum(axis=-1, keepdims=True)


def coarse_attention(qc, kc, vc, scale: float):
    """Attention among pooled blocks.

    [combine] Problem: the compression branch produces a per-block coarse
    output ``out_c`` of shape [B, H, n_blocks, D], later broadcast inside each
    block.  Scores are ``scale * qc . kc`` over every KV block (R1, R7).

    Returns (scores [B,H,nq,nkv], out_c [B,H,nq,D]), both fp64.
    """
    qc, kc, vc = _f64(qc), _f64(kc), _f64(vc)
    scores = scale * np.einsum("bhqd,bhkd->bhqk", qc, kc)
    p = softmax_rows(scores)
    out_c = np.einsum("bhqk,bhkd->bhqd", p, vc)
    return scores, out_c


# ---------------------------------------------------------------------------
# a3: top-k block selection
# ---------------------------------------------------------------------------
def select_topk(scores, topk: int, width: int | None = None):
    """Per query block, the ``topk`` KV blocks with the largest coarse logits.

    [release] "Block-sparse / VSA attention improvements": selections travel
    as compact index tensors ``q2k_idx`` with a count ``q2k_num``; [readme]
    Usage calls ``video_sparse_attn(..., topk=5)`` with an integer count.
    Ranking: logit descending, then KV index ascending (R2); the chosen set is
    written in ascending index order, tail -1 (R3).

    Returns (q2k_idx int32 [B,H,nq,width], q2k_num int32 [B,H,nq]).
    """
    scores = _f64(scores)
    B, H, nq, nkv = scores.shape
    k = max(0, min(int(topk), nkv))
    if width is None:
        width = k
    assert width >= k
    idx = np.full((B, H, nq, width), -1, dtype=np.int32)
    num = np.full((B, H, nq), k, dtype=np.int32)
    cols = np.arange(nkv)
    for b in range(B):
        for h in range(H):
            for a in range(nq):
                order = np.lexsort((cols, -scores[b, h, a]))  # primary: -score
                chosen = np.sort(order[:k])
                idx[b, h, a, :k] = chosen
    return idx, num


# ---------------------------------------------------------------------------
# a4: block-sparse attention over selected tiles
# ---------------------------------------------------------------------------
def block_sparse_attention(q, k, v, q2k_idx, q2k_num, q_block_sizes, kv_block_sizes,
                           scale: float, items=None, block: int = BLOCK) -> np.ndarray:
    """Softmax attention of each query row over the real keys of the KV blocks
    its query block selected.

    [release] ``block_sparse_attn_from_indices(q, k, v, q2k_idx, q2k_num,
    variable_block_sizes)``: attention restricted to the listed 64x64 tiles.
    Each listed entry contributes its block's real keys (a block listed twice
    contributes twice); padded keys are excluded and padded query rows are 0
    (R6); ``q2k_num == 0`` gives 0 (R9).

    q: [B,H,block*nq,D], k/v: [B,H,block*nkv,D] (block = 64, or 128 / 256
    for the larger tiles, R14).  ``items`` optionally restricts the work to an
    iterable of (b, h, query block) triples; other rows stay 0.
    Returns O_s [B,H,block*nq,D] fp64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Sq, D = q.shape
    nq = len(q_block_sizes)
    nkv = len(kv_block_sizes)
    assert Sq == block * nq and k.shape[2] == block * nkv
    out = np.zeros_like(q)
    if items is None:
        items = [(b, h, a) for b in range(B) for h in range(H) for a in range(nq)]
    for b, h, a in items:
        n_sel = int(q2k_num[b, h, a])
        mq = int(q_block_sizes[a])
        if n_sel <= 0:
            continue
        key_rows = []
        for j in range(n_sel):
            c = int(q2k_idx[b, h, a, j])
            if not 0 <= c < nkv:
                raise IndexError(f"q2k_idx entry {c} outside [0, {nkv})")
            key_rows.append(np.arange(block * c, block * c + int(kv_block_sizes[c])))
        rows = np.concatenate(key_rows)
        qa = q[b, h, block * a:block * a + mq, :]
        logits = scale * (qa @ k[b, h, rows, :].T)
        p = softmax_rows(logits)
        out[b, h, block * a:block * a + mq, :] = p @ v[b, h, rows, :]
    return out


def block_map_to_indices(block_map):
    """Selections of a bool block map as index rows.

    [release] "Block-sparse / VSA attention improvements" and "New / changed
    public API": the legacy ``block_sparse_attn(..., block_map, ...)`` bool
    mask is kept as a wrapper over the index-native kernel.  Row
    ``block_map[..., a, :]`` selects KV block ``c`` where it is True; the
    index row lists those blocks in ascending order (R3), ``-1`` after them,
    and the count is the number of True entries.

    block_map: bool [..., nq, nkv]  ->  (q2k_idx int32 [..., nq, nkv],
    q2k_num int32 [..., nq]).
    """
    bm = np.asarray(block_map, dtype=bool)
    idx = np.full(bm.shape, -1, dtype=np.int32)
    num = bm.sum(axis=-1).astype(np.int32)
    for pos in np.ndindex(*bm.shape[:-1]):
        chosen = np.flatnonzero(bm[pos])
        idx[pos][:len(chosen)] = chosen
    return idx, num


def block_sparse_lse(q, k, q2k_idx, q2k_num, q_block_sizes, kv_block_sizes, scale: float,
                     block: int = BLOCK) -> np.ndarray:
    """Natural-log log-sum-exp of each real query row's scaled logits over
    the keys its block selected (the softmax normaliser the backward pass
    reuses); -inf where nothing is selected, 0 on padded rows.

    Returns [B, H, block*nq] fp64.
    """
    q, k = _f64(q), _f64(k)
    B, H, Sq, D = q.shape
    lse = np.zeros((B, H, Sq), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for a in range(len(q_block_sizes)):
                mq = int(q_block_sizes[a])
                n_sel = int(q2k_num[b, h, a])
                if n_sel <= 0:
                    lse[b, h, block * a:block * a + mq] = -np.inf
                    continue
                rows = np.concatenate([np.arange(block * int(c), block * int(c) + int(kv_block_sizes[int(c)]))
                                       for c in q2k_idx[b, h, a, :n_sel]])
                logits = scale * (q[b, h, block * a:block * a + mq] @ k[b, h, rows].T)
                m = logits.max(axis=1)
                lse[b, h, block * a:block * a + mq] = m + np.log(np.exp(logits - m[:, None]).sum(axis=1))
    return lse


def block_sparse_attention_backward(q, k, v, dout, q2k_idx, q2k_num, q_block_sizes,
                                    kv_block_sizes, scale: float, block: int = BLOCK):
    """Gradients of the block-sparse attention output with respect to q, k
    and v, given the output gradient ``dout``.

    "[kernel] Add varlen support for block-sparse attention", Backward
    correctness / Test plan: dQ/dK/dV of the block-sparse attention, the
    varlen backward equal to per-sequence gradients.  Per query block a with
    selected key rows J (a block listed twice contributes its keys twice) and
    P = softmax(scale * q_a k_J^T):
      dV_J += P^T dout_a;  dP = dout_a v_J^T;
      dS = P * (dP - rowsum(dP * P));
      dq_a = scale * dS k_J;  dK_J += scale * dS^T q_a.
    Padded rows (query or key) get 0.

    Returns (dq, dk, dv) fp64, shaped like q, k, v.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, Sq, D = q.shape
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            for a in range(len(q_block_sizes)):
                mq = int(q_block_sizes[a])
                n_sel = int(q2k_num[b, h, a])
                if n_sel <= 0:
                    continue
                rows = np.concatenate([np.arange(block * int(c), block * int(c) + int(kv_block_sizes[int(c)]))
                                       for c in q2k_idx[b, h, a, :n_sel]])
                qa = q[b, h, block * a:block * a + mq]
                da = do[b, h, block * a:block * a + mq]
                p = softmax_rows(scale * (qa @ k[b, h, rows].T))
                np.add.at(dv[b, h], rows, p.T @ da)
                dp = da @ v[b, h, rows].T
                ds = p * (dp - (dp * p).sum(axis=1, keepdims=True))
                dq[b, h, block * a:block * a + mq] = scale * (ds @ k[b, h, rows])
                np.add.at(dk[b, h], rows, scale * (ds.T @ qa))
    return dq, dk, dv


def build_k2q(q2k_idx, q2k_num, n_kv_blocks: int):
    """The transposed selection: for every KV block c, the query blocks that
    selected it, ascending, each with the number of times it lists c.

    "[kernel] Add varlen support for block-sparse attention", Backward: the
    varlen backward runs on a k2q index (KV block -> query blocks).
    Returns (k2q_idx int32 [..., n_kv, nq] with -1 tails, k2q_cnt int32
    [..., n_kv, nq] multiplicities, k2q_num int32 [..., n_kv]).
    """
    idx = np.asarray(q2k_idx)
    num = np.asarray(q2k_num)
    lead = idx.shape[:-2]
    nq = idx.shape[-2]
    k2q = np.full(lead + (n_kv_blocks, nq), -1, dtype=np.int32)
    cnt = np.zeros(lead + (n_kv_blocks, nq), dtype=np.int32)
    k2n = np.zeros(lead + (n_kv_blocks,), dtype=np.int32)
    for pos in np.ndindex(*lead):
        for c in range(n_kv_blocks):
            blocks = []
            for a in range(nq):
                m = int(np.sum(idx[pos][a, :int(num[pos][a])] == c))
                if m:
                    blocks.append((a, m))
            k2n[pos][c] = len(blocks)
            for t, (a, m) in enumerate(blocks):
                k2q[pos][c, t] = a
                cnt[pos][c, t] = m
    return k2q, cnt, k2n


# ---------------------------------------------------------------------------
# a5: coarse/sparse combine
# ---------------------------------------------------------------------------
def combine(out_c, o_s, gate, q_block_sizes, block: int = BLOCK) -> np.ndarray:
    """out = out_c * gate + out_s, with out_c held per block.

    [combine] Problem / Change: the coarse output stays at block resolution
    [B, H, n_blocks, 1, D] and broadcasts over the slots of its block;
    the gate (``compress_attn_weight``) is laid out [B, S, H, D].  Ungated
    (gate None): out_c + out_s.  Padded query rows are 0 (R6).  Returned in
    fp64, i.e. before the single rounding of R10.
    """
    out_c, o_s = _f64(out_c), _f64(o_s)
    B, H, Sq, D = o_s.shape
    nq = len(q_block_sizes)
    out = np.zeros_like(o_s)
    g = None if gate is None else _f64(gate).transpose(0, 2, 1, 3)  # -> [B,H,S,D]
    for a in range(nq):
        m = int(q_block_sizes[a])
        sl = slice(block * a, block * a + m)
        oc = out_c[:, :, a:a + 1, :]
        if g is None:
            out[:, :, sl, :] = oc + o_s[:, :, sl, :]
        else:
            out[:, :, sl, :] = oc * g[:, :, sl, :] + o_s[:, :, sl, :]
    return out


def vsa_forward(q, k, v, gate, q_block_sizes, kv_block_sizes, topk: int,
                scale: float | None = None, width: int | None = None, items=None,
                block: int = BLOCK) -> dict:
    """The whole VSA forward: pool -> coarse attention -> top-k -> block-sparse
    attention -> combine ([readme] Usage ``video_sparse_attn``; [combine]
    Problem for the combine), on blocks of ``block`` slots (R14)."""
    D = np.shape(q)[-1]
    if scale is None:
        scale = default_scale(D)
    qc = block_pool(q, q_block_sizes, block)
    kc = block_pool(k, kv_block_sizes, block)
    vc = block_pool(v, kv_block_sizes, block)
    scores, out_c = coarse_attention(qc, kc, vc, scale)
    q2k_idx, q2k_num = select_topk(scores, topk, width)
    o_s = block_sparse_attention(q, k, v, q2k_idx, q2k_num, q_block_sizes, kv_block_sizes,
                                 scale, items=items, block=block)
    out = combine(out_c, o_s, gate, q_block_sizes, block)
    return dict(qc=qc, kc=kc, vc=vc, scores=scores, out_c=out_c, q2k_idx=q2k_idx,
                q2k_num=q2k_num, o_s=o_s, out=out)


# ---------------------------------------------------------------------------
# a6: varlen packing
# ---------------------------------------------------------------------------
def _seq_block_sizes(length: int, given):
    if given is not None:
        sizes = [int(s) for s in given]
        assert sum(sizes) == length and all(1 <= s <= BLOCK for s in sizes)
        return sizes
    if length == 0:
        return []
    nb = (length + BLOCK - 1) // BLOCK
    return [BLOCK] * (nb - 1) + [length - BLOCK * (nb - 1)]


def varlen_layout(cu_seqlens_q, cu_seqlens_kv, q_block_sizes_list=None,
                  kv_block_sizes_list=None) -> dict:
    """Block-aligned packing of variable-length sequences.

    [varlen] How it works, step 1: sequences are packed into one tensor with
    block-aligned padding, every block occupying 64 slots.  A sequence's
    blocks are consecutive; by default they are full 64-token blocks with a
    partial last block, else the given per-sequence block sizes (the
    ``q_variable_block_sizes_list`` of the test plan).

    Returns per-sequence block counts and block offsets, the flattened block
    sizes, and pack indices: ``pack_index_q[slot]`` is the token row (in the
    token-packed input) stored at that packed slot, or -1 for padding.
    """
    cq = [int(x) for x in cu_seqlens_q]
    ck = [int(x) for x in cu_seqlens_kv]
    n = len(cq) - 1
    assert len(ck) == n + 1
    lay = dict(n_seqs=n, nq=[], nkv=[], qoff=[], kvoff=[], q_block_sizes=[],
               kv_block_sizes=[])
    for which, cu, given in (("q", cq, q_block_sizes_list), ("kv", ck, kv_block_sizes_list)):
        off = 0
        slots = []
        for i in range(n):
            length = cu[i + 1] - cu[i]
            sizes = _seq_block_sizes(length, None if given is None else given[i])
            lay["n" + which].append(len(sizes))
            lay[which + "off"].append(off)
            lay[which + "_block_sizes"].extend(sizes)
            tok = cu[i]
            for s in sizes:
                row = [-1] * BLOCK
                for t in range(s):
                    row[t] = tok
                    tok += 1
                slots.extend(row)
            off += len(sizes)
        lay["pack_index_" + which] = np.asarray(slots, dtype=np.int64)
    return lay


def pack_tokens(x_tokens, pack_index) -> np.ndarray:
    """[H, total, D] token-packed -> [1, H, 64*n_blocks, D] block-aligned, zeros
    in padded slots ([varlen] How it works, step 1)."""
    x = _f64(x_tokens)
    H, _, D = x.shape
    out = np.zeros((1, H, len(pack_index), D), dtype=np.float64)
    real = pack_index >= 0
    out[0, :, real, :] = x[:, pack_index[real], :].transpose(1, 0, 2)
    return out


def rebase_q2k_idx(q2k_idx_local, q2k_num, layout) -> np.ndarray:
    """Per-sequence KV block indices -> indices into the packed KV blocks.

    [varlen] How it works, step 2: each sequence's ``q2k_idx`` rows are offset
    by the first packed block of that sequence's KV.  Entries past
    ``q2k_num`` stay -1.
    """
    out = np.array(q2k_idx_local, dtype=np.int64, copy=True)
    row = 0
    for i in range(layout["n_seqs"]):
        for _ in range(layout["nq"][i]):
            n = q2k_num[:, row]
            for h in range(out.shape[0]):
                nn = int(n[h])
                local = out[h, row, :nn]
                if np.any(local < 0) or np.any(local >= layout["nkv"][i]):
                    raise IndexError("local q2k_idx outside the sequence's KV blocks")
                out[h, row, :nn] = local + layout["kvoff"][i]
                out[h, row, nn:] = -1
            row += 1
    return out.astype(np.int32)


def block_sparse_attn_varlen(q, k, v, cu_seqlens_q, cu_seqlens_kv, q2k_idx, q2k_num,
                             scale: float, q_block_sizes_list=None,
                             kv_block_sizes_list=None) -> np.ndarray:
    """Varlen block-sparse attention: pack, rebase, one block-sparse call,
    unpack ([varlen] How it works, steps 1-4).

    q: [H, total_q, D], k/v: [H, total_kv, D]; q2k_idx: [H, sum(nq_i), width]
    with per-sequence local indices; q2k_num: [H, sum(nq_i)].
    Returns [H, total_q, D] fp64.
    """
    lay = varlen_layout(cu_seqlens_q, cu_seqlens_kv, q_block_sizes_list, kv_block_sizes_list)
    qp = pack_tokens(q, lay["pack_index_q"])
    kp = pack_tokens(k, lay["pack_index_kv"])
    vp = pack_tokens(v, lay["pack_index_kv"])
    idx = rebase_q2k_idx(q2k_idx, q2k_num, lay)[None]
    num = np.asarray(q2k_num)[None]
    o = block_sparse_attention(qp, kp, vp, idx, num, lay["q_block_sizes"],
                               lay["kv_block_sizes"], scale)
    pq = lay["pack_index_q"]
    real = pq >= 0
    H, total_q, D = _f64(q).shape
    out = np.zeros((H, total_q, D), dtype=np.float64)
    out[:, pq[real], :] = o[0][:, real, :]
    return out


# ---------------------------------------------------------------------------
# a7: video tile metadata
# ---------------------------------------------------------------------------
def build_vsa_metadata(T: int, Hh: int, W: int, tile=(4, 4, 4)) -> dict:
    """Tile permutation of a T x Hh x W latent and its block sizes.

    [utils] Summary: one call builds ``tile_partition_indices``,
    ``reverse_tile_partition_indices``, the variable block sizes (tokens per
    tile, at most the tile volume) and the non-pad index
    (``get_non_pad_index(variable_block_sizes, max_block_size)``).  Ordering
    per reading R11.  Tokens are numbered row-major over (t, h, w).

    Returns int64 index arrays of length T*Hh*W, int32 block sizes.
    """
    tt, th, tw = (int(x) for x in tile)
    vol = tt * th * tw
    nT, nH, nW = -(-T // tt), -(-Hh // th), -(-W // tw)
    perm, sizes = [], []
    for bt in range(nT):
        for bh in range(nH):
            for bw in range(nW):
                count = 0
                for t in range(bt * tt, min(T, bt * tt + tt)):
                    for h in range(bh * th, min(Hh, bh * th + th)):
                        for w in range(bw * tw, min(W, bw * tw + tw)):
                            perm.append((t * Hh + h) * W + w)
                            count += 1
                sizes.append(count)
    perm = np.asarray(perm, dtype=np.int64)
    reverse = np.empty_like(perm)
    reverse[perm] = np.arange(len(perm), dtype=np.int64)
    non_pad = []
    for j, s in enumerate(sizes):
        non_pad.extend(range(vol * j, vol * j + s))
    return dict(tile_partition_indices=perm, reverse_tile_partition_indices=reverse,
                variable_block_sizes=np.asarray(sizes, dtype=np.int32),
                non_pad_index=np.asarray(non_pad, dtype=np.int64), n_tiles=len(sizes),
                max_block_size=vol)


def tile_and_pad(x_tokens, meta) -> np.ndarray:
    """[B, H, N, D] tokens in row-major (t,h,w) order -> [B, H, 64*n_tiles, D]
    tiled and padded with zeros (the tile-partition gather followed by the
    non-pad scatter)."""
    x = _f64(x_tokens)
    B, H, N, D = x.shape
    out = np.zeros((B, H, meta["max_block_size"] * meta["n_tiles"], D), dtype=np.float64)
    out[:, :, meta["non_pad_index"], :] = x[:, :, meta["tile_partition_indices"], :]
    return out


def untile(x_padded, meta) -> np.ndarray:
    """Inverse of :func:`tile_and_pad` on the real tokens."""
    x = _f64(x_padded)
    return x[:, :, meta["non_pad_index"][meta["reverse_tile_partition_indices"]], :]
