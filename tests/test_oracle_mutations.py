"""Plant plausible mistakes in a copy of the oracle (on the CPU) and require
that the pins catch every one.  A pin set that lets a dropped term, a wrong
index or a transposed operand through would not be pinning anything."""
import importlib.util
import os

import pytest

from tests import oracle_pins

ORACLE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "oracle", "vsa_oracle.py")

# (name, exact source fragment, replacement)
MUTATIONS = [
    ("backward drops the softmax's rowsum term",
     "ds = p * (dp - (dp * p).sum(axis=1, keepdims=True))", "ds = p * dp"),
    ("backward dk without the scale", "np.add.at(dk[b, h], rows, scale * (ds.T @ qa))",
     "np.add.at(dk[b, h], rows, ds.T @ qa)"),
    ("backward dv ignores duplicates", "np.add.at(dv[b, h], rows, p.T @ da)",
     "dv[b, h][rows] += p.T @ da"),
    ("backward query rows at 64-slot offsets", "qa = q[b, h, block * a:block * a + mq]\n",
     "qa = q[b, h, BLOCK * a:BLOCK * a + mq]\n"),
    ("backward dq written at 64-slot offsets",
     "dq[b, h, block * a:block * a + mq] = scale * (ds @ k[b, h, rows])",
     "dq[b, h, BLOCK * a:BLOCK * a + mq] = scale * (ds @ k[b, h, rows])"),
    ("lse written at 64-slot offsets", "lse[b, h, block * a:block * a + mq] = m + np.log(",
     "lse[b, h, BLOCK * a:BLOCK * a + mq] = m + np.log("),
    ("k2q drops multiplicities", "m = int(np.sum(idx[pos][a, :int(num[pos][a])] == c))",
     "m = int(np.any(idx[pos][a, :int(num[pos][a])] == c))"),
    ("block map rows not ascending", "idx[pos][:len(chosen)] = chosen",
     "idx[pos][:len(chosen)] = chosen[::-1]"),
    ("block map counts all entries", "num = bm.sum(axis=-1).astype(np.int32)",
     "num = np.full(bm.shape[:-1], bm.shape[-1], dtype=np.int32)"),
    ("pool divides by the block", "sum(axis=2) / m", "sum(axis=2) / block"),
    ("pool includes padding", "x[:, :, block * j:block * j + m, :].sum(axis=2)",
     "x[:, :, block * j:block * j + block, :].sum(axis=2)"),
    ("coarse drops scale", 'scores = scale * np.einsum("bhqd,bhkd->bhqk", qc, kc)',
     'scores = np.einsum("bhqd,bhkd->bhqk", qc, kc)'),
    ("coarse softmax over q", "    p = softmax_rows(scores)\n",
     "    p = softmax_rows(scores.swapaxes(-1, -2)).swapaxes(-1, -2)\n"),
    ("coarse output uses kc", 'out_c = np.einsum("bhqk,bhkd->bhqd", p, vc)',
     'out_c = np.einsum("bhqk,bhkd->bhqd", p, kc)'),
    ("topk ties to higher index", "order = np.lexsort((cols, -scores[b, h, a]))",
     "order = np.lexsort((-cols, -scores[b, h, a]))"),
    ("topk keeps rank order", "chosen = np.sort(order[:k])", "chosen = order[:k]"),
    ("topk picks smallest", "order = np.lexsort((cols, -scores[b, h, a]))",
     "order = np.lexsort((cols, scores[b, h, a]))"),
    ("sparse attends padded keys",
     "key_rows.append(np.arange(block * c, block * c + int(kv_block_sizes[c])))",
     "key_rows.append(np.arange(block * c, block * c + block))"),
    ("sparse drops scale", "logits = scale * (qa @ k[b, h, rows, :].T)",
     "logits = (qa @ k[b, h, rows, :].T)"),
    ("sparse uses k as values", "p @ v[b, h, rows, :]", "p @ k[b, h, rows, :]"),
    ("sparse ignores q block size",
     "        n_sel = int(q2k_num[b, h, a])\n        mq = int(q_block_sizes[a])\n",
     "        n_sel = int(q2k_num[b, h, a])\n        mq = block\n"),
    ("sparse keys at 64-slot offsets", "key_rows.append(np.arange(block * c,",
     "key_rows.append(np.arange(BLOCK * c,"),
    ("combine gate not transposed", "g = None if gate is None else _f64(gate).transpose(0, 2, 1, 3)",
     "g = None if gate is None else _f64(gate).reshape(o_s.shape)"),
    ("combine gates the sparse branch", "out[:, :, sl, :] = oc * g[:, :, sl, :] + o_s[:, :, sl, :]",
     "out[:, :, sl, :] = oc + g[:, :, sl, :] * o_s[:, :, sl, :]"),
    ("combine shifts coarse block", "oc = out_c[:, :, a:a + 1, :]",
     "oc = out_c[:, :, max(a - 1, 0):max(a - 1, 0) + 1, :]"),
    ("varlen rebase drops offset", 'out[h, row, :nn] = local + layout["kvoff"][i]',
     "out[h, row, :nn] = local"),
    ("varlen pack not block aligned", "                row = [-1] * BLOCK\n",
     "                row = [-1] * s\n"),
    ("metadata column-major in tile",
     "                for t in range(bt * tt, min(T, bt * tt + tt)):\n"
     "                    for h in range(bh * th, min(Hh, bh * th + th)):\n"
     "                        for w in range(bw * tw, min(W, bw * tw + tw)):\n",
     "                for w in range(bw * tw, min(W, bw * tw + tw)):\n"
     "                    for h in range(bh * th, min(Hh, bh * th + th)):\n"
     "                        for t in range(bt * tt, min(T, bt * tt + tt)):\n"),
    ("metadata reverse is forward", "reverse[perm] = np.arange(len(perm), dtype=np.int64)",
     "reverse[:] = perm"),
    ("metadata pads every tile to the end", "non_pad.extend(range(vol * j, vol * j + s))",
     "non_pad.extend(range(vol * j + vol - s, vol * j + vol))"),
]


def _mutant(old, new):
    src = open(ORACLE).read()
    assert src.count(old) == 1, f"mutation anchor not unique/present: {old!r}"
    spec = importlib.util.spec_from_loader("oracle_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(src.replace(old, new), ORACLE + " (mutant)", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_mutation(name, old, new):
    mod = _mutant(old, new)
    caught = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(mod)
        except Exception as e:  # noqa: BLE001 - any failure counts as caught
            caught.append((check.__name__, type(e).__name__))
    assert caught, f"no pin caught the planted mistake '{name}'"
