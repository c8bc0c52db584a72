"""The read split over ranks, on the CPU.

fl_shard_blocks (host code of libfl): contiguous ranges that cover every block, balanced by
the bytes each block's depth reads to within one block. Two gloo ranks (one process each, as
torchrun launches them) run the exchange the multi-GPU read uses: each rank computes its block
rows of a layer (the oracle stands in for the GPU read here), the rows are padded and
all-gathered in rank order, and the assembled output equals the whole layer's; each rank's
gate partial over its piece of the logits is all-gathered and merged in rank order, and the
merged gate equals the gate of the whole row.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fl():
    from variable_precision_weight_b200 import build
    build.build()
    from variable_precision_weight_b200 import fl
    return fl


def block_bytes(levels, inn):
    G = inn // 128
    d = np.minimum(levels.astype(np.int64), 4)
    return np.where(d > 0, 256 * G + 2048 * G * d, 0)


@pytest.mark.parametrize("nranks", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_shard_ranges_cover_and_balance(fl, nranks, seed):
    from variable_precision_weight_b200 import synth
    nblocks, inn = 37 + 11 * seed, 1024 * (seed + 1)
    lv = synth.seeded_levels(nblocks, 60, seed)
    first = fl.fl_shard_blocks(lv, inn, nranks)
    assert len(first) == nranks + 1 and first[0] == 0 and first[-1] == nblocks
    assert all(a <= b for a, b in zip(first, first[1:]))                  # contiguous, in order
    w = block_bytes(lv, inn)
    total = w.sum()
    per = [w[first[r]:first[r + 1]].sum() for r in range(nranks)]
    assert sum(per) == total
    assert max(abs(p - total / nranks) for p in per) <= w.max()             # within one block's bytes
    # a block belongs to the range holding the midpoint of its bytes
    cum = np.concatenate([[0], np.cumsum(w)])
    for r in range(nranks):
        for b in range(first[r], first[r + 1]):
            mid = cum[b] + 0.5 * w[b]
            if w[b] > 0:
                assert total * r / nranks <= mid <= total * (r + 1) / nranks + 1e-9


def test_shard_edge_cases(fl):
    assert fl.fl_shard_blocks(np.array([2, 2], np.uint8), 1024, 5)[-1] == 2           # more ranks than blocks
    assert fl.fl_shard_blocks(np.array([0, 0, 0, 0], np.uint8), 1024, 2) == [0, 2, 4]  # nothing read: by count
    assert fl.fl_shard_blocks(np.array([], np.uint8), 1024, 3) == [0, 0, 0, 0]
    assert fl.fl_shard_blocks(np.array([0, 0, 4, 4], np.uint8), 1024, 2) == [0, 3, 4]  # ZERO blocks weigh nothing
    with pytest.raises(fl.FlError):
        fl.fl_shard_blocks(np.array([1], np.uint8), 100, 2)                              # in % 128
    with pytest.raises(fl.FlError):
        fl.fl_shard_blocks(np.array([1], np.uint8), 128, 0)


WORKER = r"""
import json, os, sys
sys.path.insert(0, os.environ["REPO"])
import numpy as np, torch, torch.distributed as dist
import oracle
from variable_precision_weight_b200 import fl, shard, synth
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo")
out, inn, batch = 1216, 512, 2
q, s = synth.int8_layer(out, inn, 61)
lv = synth.seeded_levels(out // 64, 62)
x = synth.bf16_normal((batch, inn), 63)
plans = shard.plan([lv], [inn], world)
rows, total = shard.rank_rows(plans, rank)
(_, r0, n), = rows
y_local = np.zeros((batch, n), np.float32)
if n:
    y_local[:] = oracle.gemv_depth(q[r0:r0 + n], s[r0:r0 + n], lv[r0 // 64:(r0 + n) // 64], x)
counts = [batch * 64 * (plans[0][r + 1] - plans[0][r]) for r in range(world)]
parts = shard.gather_rows(torch.from_numpy(y_local.reshape(-1)), counts)
y = np.concatenate([p.numpy().reshape(batch, -1) for p in parts], axis=1)
yref = oracle.gemv_depth(q, s, lv, x)
ok_rows = bool(np.array_equal(y, yref.astype(np.float32)))
# the gate over a vocabulary split with the blocks: partial of this rank's logits, global indices
V = 4096
z = synth.rng(64).standard_normal((batch, V)).astype(np.float32)
cut = [V * r // world // 4 * 4 for r in range(world)] + [V]
piece = z[:, cut[rank]:cut[rank + 1]]
rec = np.zeros((batch, 8), np.float32)
for b in range(batch):
    zz = piece[b].astype(np.float64)
    m = zz.max(); e = np.exp(zz - m)
    order = np.lexsort((np.arange(zz.size), -zz))
    rec[b, 0], rec[b, 1], rec[b, 2], rec[b, 3] = m, e.sum(), ((zz - m) * e).sum(), zz[order[1]]
    rec[b, 4:6] = np.array([order[0] + cut[rank], order[1] + cut[rank]], np.int32).view(np.float32)
gathered = shard.gather_partials(torch.from_numpy(rec.view(np.uint8).reshape(-1)), world).numpy()
recs = gathered.view(np.float32).reshape(world, batch, 8)
res = []
for b in range(batch):
    M = recs[:, b, 0].astype(np.float64).max()
    S = sum(recs[r, b, 1] * np.exp(recs[r, b, 0] - M) for r in range(world))
    T = sum((recs[r, b, 2] + (recs[r, b, 0] - M) * recs[r, b, 1]) * np.exp(recs[r, b, 0] - M) for r in range(world))
    cand = [(float(recs[r, b, 0]), int(recs[r, b, 4:5].view(np.int32)[0])) for r in range(world)]
    cand += [(float(recs[r, b, 3]), int(recs[r, b, 5:6].view(np.int32)[0])) for r in range(world)]
    cand.sort(key=lambda t: (-t[0], t[1]))
    res.append((float(np.log(S) - T / S), cand[0][1], cand[1][1]))
H, _, top2, _ = oracle.logit_gate(z, 1e30, -1.0)
ok_gate = all(abs(res[b][0] - H[b]) <= 1e-5 * abs(H[b]) and [res[b][1], res[b][2]] == list(top2[b]) for b in range(batch))
print(json.dumps({"rank": rank, "rows": ok_rows, "gate": ok_gate, "counts": counts}), flush=True)
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_ranks_exchange_rows_and_gate_partials(fl, orc, world):
    port = _free_port()
    procs = []
    for rank in range(world):
        env = dict(os.environ, REPO=ROOT, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", WORKER], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=300)
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["rows"] and o["gate"], o
        assert sum(o["counts"]) == 2 * 1216   # every row once; ranges balance bytes, not block counts
