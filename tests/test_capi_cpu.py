"""C-ABI checks that need no GPU: the library loads, exports every function
include/vsa.h declares, rejects bad arguments on the host before launching
anything, and its host metadata routine matches the oracle bit for bit."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vsa.h")


def _lib():
    from block_sparse_attention_15_b200 import binding
    if not os.path.exists(binding.LIB_PATH):
        from block_sparse_attention_15_b200 import build
        build.build()
    return binding.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+char\s*\*|int|size_t)\s+([a-z_0-9]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("vsa_forward", "block_sparse_attn_from_indices", "block_sparse_attn_varlen",
                     "build_vsa_metadata", "vsa_forward_workspace_size", "vsa_get_device_status"):
        assert required in names


@pytest.mark.parametrize("name", declared_functions())
def test_symbol_exported(name):
    lib = _lib()
    assert hasattr(lib, name), f"{name} declared in vsa.h but not exported"


def test_exports_are_c_symbols():
    _lib()
    from block_sparse_attention_15_b200 import binding
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in declared_functions():
        assert name in exported, f"{name} is not an unmangled exported symbol"


def test_binding_signatures_cover_header():
    from block_sparse_attention_15_b200 import binding
    assert set(declared_functions()) == set(binding.SIGNATURES)


def test_status_strings():
    lib = _lib()
    assert lib.vsa_status_string(0) == b"ok"
    assert b"range" in lib.vsa_status_string(6)
    assert lib.vsa_abi_version() >> 16 == 2


def _fwd(lib, **kw):
    args = dict(q=1, k=1, v=1, gate=None, qbs=None, kbs=None, B=1, H=1, Sq=64, Skv=64, D=128,
                topk=1, scale=0.0, out=1, idx=1, num=1, stride=1, out_c=None, ws=None, wsb=0,
                stream=None)
    args.update(kw)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.vsa_forward(v(args["q"]), v(args["k"]), v(args["v"]), v(args["gate"]), v(args["qbs"]),
                           v(args["kbs"]), args["B"], args["H"], args["Sq"], args["Skv"], args["D"],
                           args["topk"], args["scale"], v(args["out"]), v(args["idx"]),
                           v(args["num"]), args["stride"], v(args["out_c"]), v(args["ws"]),
                           args["wsb"], None)


def test_forward_host_argument_checks():
    """Bad arguments come back as status codes before any CUDA call."""
    lib = _lib()
    fake = 1 << 20  # never dereferenced: every case fails on the host
    base = dict(q=fake, k=fake, v=fake, out=fake, idx=fake, num=fake)
    assert _fwd(lib, **{**base, "q": None}) == 1                       # null input
    assert _fwd(lib, **base, D=96) == 3                                 # unsupported head dim
    assert _fwd(lib, **base, Sq=100) == 2                               # not 64 * n
    assert _fwd(lib, **base, topk=0) == 1                               # topk >= 1
    assert _fwd(lib, **base, Sq=64 * 4, Skv=64 * 4, topk=3, stride=2) == 2  # stride < k
    assert _fwd(lib, **base, B=0) == 1                                  # empty batch
    assert _fwd(lib, **base, Sq=64 * 4096) == 3                         # above VSA_MAX_BLOCKS
    assert _fwd(lib, **{**base, "q": fake + 2}) == 1                    # misaligned
    assert _fwd(lib, **base) == 7                                       # no workspace
    assert _fwd(lib, **base, ws=fake + 64, wsb=1 << 30) == 7            # misaligned workspace


def _fwd_host(lib, **kw):
    args = dict(q=1, k=1, v=1, gate=None, qbs=None, kbs=None, B=1, H=1, Sq=64, Skv=64, D=128,
                topk=1, scale=0.0, out=1, idx=None, num=None, stride=1, out_c=None, hpc=0, ws=None,
                wsb=0)
    args.update(kw)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.vsa_forward_host(v(args["q"]), v(args["k"]), v(args["v"]), v(args["gate"]),
                                v(args["qbs"]), v(args["kbs"]), args["B"], args["H"], args["Sq"],
                                args["Skv"], args["D"], args["topk"], args["scale"], v(args["out"]),
                                v(args["idx"]), v(args["num"]), args["stride"], v(args["out_c"]),
                                args["hpc"], v(args["ws"]), args["wsb"], None)


def test_forward_host_entry_argument_checks():
    """The host-buffer forward rejects bad arguments before it enqueues anything."""
    lib = _lib()
    fake = 1 << 20
    base = dict(q=fake, k=fake, v=fake, out=fake)
    assert _fwd_host(lib, **{**base, "out": None}) == 1                 # null output
    assert _fwd_host(lib, **base, D=96) == 3                            # unsupported head dim
    assert _fwd_host(lib, **base, Skv=100) == 2                         # not 64 * n
    assert _fwd_host(lib, **base, hpc=-1) == 1                          # negative chunk
    assert _fwd_host(lib, **base, Sq=64 * 4, Skv=64 * 4, topk=3, stride=2) == 2
    assert _fwd_host(lib, **base) == 7                                  # no workspace
    need = lib.vsa_forward_host_workspace_size(1, 1, 1, 1, 128, 1, 0, 0)
    assert _fwd_host(lib, **base, ws=fake, wsb=need - 1) == 7           # too small
    assert _fwd_host(lib, **base, ws=fake + 64, wsb=need) == 7          # misaligned


def test_forward_host_workspace_size():
    """Two slots of one chunk each: inputs, outputs and a forward workspace."""
    lib = _lib()
    a = lambda x: (x + 255) // 256 * 256
    B, H, nq, nkv, D, stride = 1, 56, 242, 242, 128, 48
    hc = 7  # about eight chunks of 56 heads
    fwd = lib.vsa_forward_workspace_size(1, hc, nq, nkv, D)
    slot = (a(hc * 64 * nq * D * 2) + 2 * a(hc * 64 * nkv * D * 2) + a(64 * nq * hc * D * 2) +
            a(hc * 64 * nq * D * 2) + a(hc * nq * stride * 4) + a(hc * nq * 4) + a(hc * nq * D * 4) + a(fwd))
    assert lib.vsa_forward_host_workspace_size(B, H, nq, nkv, D, stride, 1, 0) == a(4 * (nq + nkv)) + 2 * slot
    # an explicit chunk of all heads needs more; ungated needs less; bad sizes give 0
    assert lib.vsa_forward_host_workspace_size(B, H, nq, nkv, D, stride, 1, H) > 2 * slot
    assert lib.vsa_forward_host_workspace_size(B, H, nq, nkv, D, stride, 0, 0) < a(4 * (nq + nkv)) + 2 * slot
    assert lib.vsa_forward_host_workspace_size(B, H, 0, nkv, D, stride, 1, 0) == 0


def test_varlen_workspace_size():
    """Block tables (4 ints per query block, 2 per KV block), then fp32 norms
    and bounds for H heads, each region 256-aligned."""
    lib = _lib()
    a = lambda x: (x + 255) // 256 * 256
    assert lib.block_sparse_attn_varlen_workspace_size(2, 5, 3, 4) == a(4 * (20 + 6)) + a(4 * 4 * (10 + 3))
    assert lib.block_sparse_attn_varlen_workspace_size(2, 529, 501, 24) == a(4 * (4 * 529 + 2 * 501)) + a(4 * 24 * (2 * 529 + 501))
    assert lib.block_sparse_attn_varlen_workspace_size(2, 5, 3, 0) == 0


def test_varlen_host_argument_checks():
    lib = _lib()
    from block_sparse_attention_15_b200.binding import _P32
    fake = ctypes.c_void_p(1 << 20)

    def call(cu_q, cu_kv, n, qs=None, qcb=None):
        a = np.asarray(cu_q, np.int32)
        b = np.asarray(cu_kv, np.int32)
        qs_a = None if qs is None else np.asarray(qs, np.int32)
        qcb_a = None if qcb is None else np.asarray(qcb, np.int32)
        p = lambda x: None if x is None else x.ctypes.data_as(_P32)
        return lib.block_sparse_attn_varlen(fake, fake, fake, p(a), p(b), p(qs_a), p(qcb_a), None,
                                            None, n, 2, 128, fake, fake, 4, 0.0, fake, None, None,
                                            None, None, None, 0, None)

    assert call([0], [0], 0) == 2                                 # empty batch
    assert call([0, 64, 64], [0, 64, 128], 2) == 2                # zero-token sequence
    assert call([1, 64], [0, 64], 1) == 2                         # cu_seqlens must start at 0
    assert call([0, 100], [0, 64], 1, qs=[64, 30], qcb=[0, 2]) == 2   # sizes must sum to length
    assert call([0, 100], [0, 64], 1, qs=[64, 36, 0], qcb=[0, 3]) == 8  # size 0 not allowed
    assert call([0, 100], [0, 64], 1, qs=[64, 36]) == 1           # sizes need per-seq counts
    assert call([0, 100], [0, 64], 1) == 7                        # valid, but no workspace


@pytest.mark.parametrize("shape,tile", [((9, 30, 52), (4, 4, 4)), ((5, 5, 5), (4, 4, 4)),
                                        ((8, 4, 12), (4, 4, 4)), ((3, 7, 10), (2, 4, 8)),
                                        ((1, 1, 1), (4, 4, 4))])
def test_metadata_matches_oracle(shape, tile):
    from block_sparse_attention_15_b200 import build_vsa_metadata
    from oracle import vsa_oracle as O
    got = build_vsa_metadata(*shape, tile=tile)
    want = O.build_vsa_metadata(*shape, tile=tile)
    for key in ("tile_partition_indices", "reverse_tile_partition_indices",
                "variable_block_sizes", "non_pad_index"):
        assert np.array_equal(got[key], want[key]), key
    assert got["n_tiles"] == want["n_tiles"]
    # the slot map is the non-pad scatter of the partition
    slot = np.full(want["n_tiles"] * want["max_block_size"], -1, dtype=np.int64)
    slot[want["non_pad_index"]] = want["tile_partition_indices"]
    assert np.array_equal(got["slot_token"], slot)


def test_metadata_rejects_bad_tiles():
    lib = _lib()
    n = ctypes.c_int32(0)
    assert lib.build_vsa_metadata(8, 8, 8, 8, 8, 8, None, None, None, None, None,
                                  ctypes.byref(n)) == 1          # tile volume 512 > 256
    assert lib.build_vsa_metadata(8, 4, 4, 8, 4, 4, None, None, None, None, None,
                                  ctypes.byref(n)) == 0          # 128-token tiles (VSA-128)
    assert n.value == 1
    assert lib.build_vsa_metadata(4, 8, 8, 4, 8, 8, None, None, None, None, None,
                                  ctypes.byref(n)) == 0          # 256-token tiles (VSA-256)
    assert n.value == 1
    assert lib.build_vsa_metadata(0, 4, 4, 4, 4, 4, None, None, None, None, None,
                                  ctypes.byref(n)) == 1


def test_layouts_and_strided_argument_checks():
    """vsa_make_layout fills the documented strides; a view stride that is not
    a multiple of 8 elements and a missing layout come back as status codes
    before any CUDA call."""
    from block_sparse_attention_15_b200.binding import VsaLayout
    lib = _lib()
    L = VsaLayout()
    B, H, Sq, Skv, D = 2, 3, 128, 192, 64
    assert lib.vsa_make_layout(1, B, H, Sq, Skv, D, ctypes.byref(L)) == 0
    assert (L.q.batch, L.q.head, L.q.seq) == (Sq * H * D, D, H * D)
    assert (L.k.batch, L.k.head, L.k.seq) == (Skv * H * D, D, H * D)
    assert (L.gate.batch, L.gate.head, L.gate.seq) == (Sq * H * D, D, H * D)
    assert lib.vsa_make_layout(0, B, H, Sq, Skv, D, ctypes.byref(L)) == 0
    assert (L.out.batch, L.out.head, L.out.seq) == (H * Sq * D, Sq * D, D)
    assert lib.vsa_make_layout(7, B, H, Sq, Skv, D, ctypes.byref(L)) == 1
    fake = ctypes.c_void_p(1 << 20)

    def fwd(layout):
        return lib.vsa_forward_strided(fake, fake, fake, None, layout, None, None, B, H, Sq, Skv, D,
                                       block, 1, 0.0, fake, fake, fake, 1, None, None, 0, None)
    block = 64
    assert fwd(None) == 1
    L.q.seq = 68   # 136 bytes: not a TMA stride
    assert fwd(ctypes.byref(L)) == 3
    lib.vsa_make_layout(0, B, H, Sq, Skv, D, ctypes.byref(L))
    assert fwd(ctypes.byref(L)) == 7   # valid layout: next check is the missing workspace
    block = 96
    assert fwd(ctypes.byref(L)) == 3   # block size neither 64 nor 128
    block = 128
    assert fwd(ctypes.byref(L)) == 2   # Skv = 192 is not a multiple of 128



def test_bool_mask_entry_argument_checks():
    lib = _lib()
    fake = ctypes.c_void_p(1 << 20)

    def call(bm=fake, idx=fake, num=fake, Sq=128, Skv=128, D=128, block=64):
        return lib.block_sparse_attn(fake, fake, fake, bm, None, None, 1, 1, Sq, Skv, D, block, 0.0,
                                     fake, idx, num, None, None, 0, None)
    assert call(bm=None) == 1
    assert call(idx=None) == 1
    assert call(Sq=100) == 2
    assert call(Skv=64 * 4096) == 3
    assert call(block=96) == 3
    assert call(Sq=192, block=128) == 2


def test_backward_ex_workspace_size():
    """Block 64 needs the plain backward's bytes; 128 / 256 add the selection
    rewritten over 64-slot sub-blocks (rows r times as many, r times as
    wide, plus counts and sub-block sizes); bad sizes give 0."""
    lib = _lib()
    a = lambda x: (x + 255) // 256 * 256
    B, H, Sq, Skv, stride = 1, 4, 128 * 10, 128 * 12, 5
    base = lib.block_sparse_attn_backward_workspace_size(B, H, Sq, Skv // 64)
    assert base > 0
    assert lib.block_sparse_attn_backward_ex_workspace_size(B, H, Sq, Skv, 64, stride) == base
    for blk in (128, 256):
        Sq_b, Skv_b = blk * 5, blk * 6
        r = blk // 64
        nq, nkv = Sq_b // blk, Skv_b // blk
        want = (lib.block_sparse_attn_backward_workspace_size(B, H, Sq_b, Skv_b // 64) +
                a(4 * B * H * nq * r * stride * r) + a(4 * B * H * nq * r) + a(4 * nq * r) +
                a(4 * nkv * r))
        assert lib.block_sparse_attn_backward_ex_workspace_size(B, H, Sq_b, Skv_b, blk, stride) == want
    assert lib.block_sparse_attn_backward_ex_workspace_size(B, H, 128 * 3 + 64, Skv, 128, 1) == 0
    assert lib.block_sparse_attn_backward_ex_workspace_size(B, H, Sq, Skv, 96, 1) == 0
    assert lib.block_sparse_attn_backward_ex_workspace_size(B, H, Sq, Skv, 128, 0) == 0


def test_backward_ex_host_argument_checks():
    """The block-size backward rejects bad arguments before any CUDA call."""
    lib = _lib()
    fake = 1 << 20
    v = ctypes.c_void_p

    def call(B=1, H=1, Sq=256, Skv=256, D=128, blk=128, stride=2, q=fake, ws=None, wsb=0):
        return lib.block_sparse_attn_backward_ex(
            v(q), v(fake), v(fake), v(fake), v(fake), v(fake), v(fake), v(fake), None, None, B, H,
            Sq, Skv, D, blk, stride, 0.0, v(fake), v(fake), v(fake), None if ws is None else v(ws),
            wsb, None)

    assert call(q=None) == 1                                  # null input
    assert call(D=96) == 3                                    # unsupported head dim
    assert call(blk=96) == 3                                  # unsupported block size
    assert call(Sq=128 + 64) == 2                             # not a multiple of the block
    assert call(Sq=256 * 3, Skv=256 * 2, blk=256, stride=600) == 3   # 4 x 600 > VSA_MAX_BLOCKS
    assert call(Skv=64 * 2050, Sq=128) == 3                   # Skv / 64 above VSA_MAX_BLOCKS
    assert call(q=fake + 2) == 1                              # misaligned
    assert call() == 7                                        # no workspace
    need = lib.block_sparse_attn_backward_ex_workspace_size(1, 1, 256, 256, 128, 2)
    assert call(ws=fake, wsb=need - 1) == 7                   # too small
    assert call(ws=fake + 64, wsb=need) == 7                  # misaligned
