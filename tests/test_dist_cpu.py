"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (127.0.0.1), the
timing taken as the max over ranks, the whole-job throughput summed over the
replicas, and the reference arm leaving non-zero ranks without work."""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r'''
import os, sys, json
sys.path.insert(0, {root!r})
import torch, torch.distributed as dist
import bench
rank = int(os.environ["RANK"]); world = int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", init_method="tcp://127.0.0.1:{port}", rank=rank,
                        world_size=world)
ms = 10.0 + 5.0 * rank
got = bench.max_over_ranks(ms, torch.device("cpu"), world)
val = bench.aggregate_gbs(1e9, 10, got, world)
dist.barrier()
print(json.dumps({{"rank": rank, "max_ms": got, "gbs": val}}), flush=True)
dist.destroy_process_group()
'''


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_max_over_ranks_and_aggregate():
    port = _free_port()
    code = WORKER.format(root=ROOT, port=port)
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1")
        procs.append(subprocess.Popen([sys.executable, "-c", code], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=120) for p in procs]
    for p, (o, e) in zip(procs, outs):
        assert p.returncode == 0, e
    import json
    lines = [json.loads(o.strip().splitlines()[-1]) for o, _ in outs]
    for d in lines:
        assert d["max_ms"] == 15.0                      # the slowest rank
        assert abs(d["gbs"] - 2 * 1e9 * 10 / 15e-3 / 1e9) < 1e-6  # both replicas' bytes


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line():
    """The reference arm times the CPU oracle on bounded row samples."""
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "1"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


TP_WORKER = r'''
import os, sys, json
sys.path.insert(0, {root!r})
sys.path.insert(0, os.path.join({root!r}, "tests"))
import numpy as np
import torch, torch.distributed as dist
from sparse_weight_b200 import hyb, inputs, tp
import oracle
rank = int(os.environ["RANK"]); world = int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", init_method="tcp://127.0.0.1:{port}", rank=rank,
                        world_size=world)
orc = oracle.Oracle()
n, k, b1, b2, batch = 640, 512, 64, 64, 3
T = (n // b1) * (k // b2)
tmap = inputs.tile_map_bernoulli(T, 0.5, inputs.seed_of("tp_cpu", "map"))
W = inputs.weight(n, k, 0.02, inputs.seed_of("tp_cpu", "W"))
X = inputs.activations(batch, k, inputs.seed_of("tp_cpu", "X"))
ref = orc.pack(inputs.bits(W), b1, b2, tmap)
# the packed matrix as host tensors (the shard views are plain slices)
P = hyb.Packed(n, k, b1, b2, torch.from_numpy(tmap.copy()),
               torch.from_numpy(ref["vals"].view(np.int16).copy()),
               torch.from_numpy(np.concatenate([ref["meta"], np.zeros(16, np.uint8)])),
               torch.from_numpy(ref["val_off"].copy()), torch.from_numpy(ref["meta_off"].copy()),
               int(ref["val_off"][-1]), int(ref["meta_off"][-1]))
sh = tp.RowShard(P, rank, world, plan=False)
lo, hi = sh.rows[rank]
ok_views = True
if sh.local is not None:
    # the shard's slices equal the pack of its own rows
    sub = orc.pack(inputs.bits(W[lo:hi]), b1, b2, tmap[(lo // b1) * (k // b2):(hi // b1) * (k // b2)])
    L = sh.local
    ok_views = (np.array_equal(L.vals.numpy().view(np.uint16), sub["vals"])
                and np.array_equal(L.val_off.numpy(), sub["val_off"])
                and np.array_equal(L.meta_off.numpy(), sub["meta_off"])
                and np.array_equal(L.meta.numpy()[:L.n_meta], sub["meta"][:L.n_meta]))
def product(S, x, out):
    pk = dict(vals=S.vals.numpy().view(np.uint16), meta=S.meta.numpy(),
              val_off=S.val_off.numpy(), meta_off=S.meta_off.numpy())
    y, _ = orc.spmv(S.n, S.k, S.b1, S.b2, S.tile_map.numpy(), pk, inputs.bits(x))
    y32 = torch.from_numpy(y.astype(np.float32))
    if out is not None:
        out.copy_(y32)
    return y32
Y = sh.apply(X, product=product)
y_full, _ = orc.spmv(n, k, b1, b2, tmap, ref, inputs.bits(X))
same = bool(np.array_equal(Y.numpy(), y_full.astype(np.float32)))
dist.barrier()
print(json.dumps({{"rank": rank, "rows": [lo, hi], "views": bool(ok_views), "same": same}}),
      flush=True)
dist.destroy_process_group()
'''


@pytest.mark.parametrize("world", [2, 3])
def test_row_sharded_product_gathers_the_full_output(world):
    """Row-sharded decode (tensor-parallel): each gloo rank holds its bands
    (hyb_shard_bands), its slices equal the pack of its own rows, its rows
    are computed by the oracle, and one all-gather reassembles exactly the
    full product."""
    port = _free_port()
    code = TP_WORKER.format(root=ROOT, port=port)
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1")
        procs.append(subprocess.Popen([sys.executable, "-c", code], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=300) for p in procs]
    for p, (o, e) in zip(procs, outs):
        assert p.returncode == 0, e
    import json
    lines = sorted((json.loads(o.strip().splitlines()[-1]) for o, _ in outs),
                   key=lambda d: d["rank"])
    assert [d["rows"][0] for d in lines][0] == 0 and lines[-1]["rows"][1] == 640
    for a, b in zip(lines, lines[1:]):
        assert a["rows"][1] == b["rows"][0]        # contiguous, every row once
    assert all(d["views"] and d["same"] for d in lines)


def test_shard_bands_rule():
    """The shard plan against its definition: rank i holds the bands whose
    first packed byte b satisfies i * total <= b * world < (i + 1) * total."""
    import numpy as np
    sys.path.insert(0, ROOT)
    from sparse_weight_b200 import hyb
    rng = np.random.default_rng(3)
    for trial in range(20):
        b1, b2 = 64, 64
        R, tpr = int(rng.integers(1, 12)), int(rng.integers(1, 6))
        tm = (rng.random(R * tpr) < 0.5).astype(np.uint8)
        sizes = np.where(tm == 1, b1 * b2 + b1 * b2 // 8, 2 * b1 * b2).reshape(R, tpr).sum(1)
        first = np.concatenate([[0], np.cumsum(sizes)[:-1]])
        total = int(sizes.sum())
        for world in (1, 2, 3, 5, 8):
            got = [hyb.shard_bands(R * b1, tpr * b2, b1, b2, tm, world, r) for r in range(world)]
            for r, (lo, hi) in enumerate(got):
                want = [band for band in range(R)
                        if r * total <= first[band] * world < (r + 1) * total]
                assert list(range(lo, hi)) == want, (trial, world, r)
