"""The exchange protocol of the context-parallel decode (hs2_decode_cp_*), on
the CPU with two gloo ranks: each rank holds its slice of every sequence's
FP8 cache (context_parallel.slice_bounds) and exchanges, through the same
all-gather helper the GPU path uses (context_parallel.dist_all_gather), the
three record sets the steps produce: a softmax state (base-2 max, sum,
unnormalised output) per query head, its exact top k as (score, position)
records, and a softmax state per sparse layer.  The per-rank steps are
written out here in numpy (fp64) from those record definitions; merging the
gathered records must give the oracle's decode over the whole cache on every
rank.  The GPU kernels of the same steps are tested on a device in
test_gpu_context_parallel.py."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import json, math, os, sys
sys.path.insert(0, {root!r}); sys.path.insert(0, os.path.join({root!r}, "tests"))
import numpy as np, torch
import torch.distributed as dist
import oracle, synth
from long_context_bridge_b200 import context_parallel as cp
from helpers import check_index_lists
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo")
gather = cp.dist_all_gather()
lens, Hq, Hkv, k, w, L = [700, 333, 130], 8, 2, 64, 16, 2
G, B, sc = Hq // Hkv, 3, 1 / math.sqrt(128)
cfg = synth.BlockConfig("cp protocol", 7, max(lens), Hq, Hkv, n_needles=8, q_mix=True,
                        batch=B, fp8_cache=True)
cache = synth.decode_cache_np(cfg, max(lens), batch=B)
q = synth.decode_queries_np(cfg, synth.TID_Q, batch=B)
qs = [synth.decode_queries_np(cfg, synth.TID_QS0 + l, batch=B) for l in range(L)]
tab = oracle.e4m3_table()
deq = lambda codes, s: tab[codes] * s[..., None].astype(np.float64)
bf = lambda bits: synth.bf16_bits_to_f32(bits).astype(np.float64)
lo, hi = cp.slice_bounds(lens, world, rank)
K = [deq(cache.Kc[b, lo[b]:hi[b]], cache.scale[b, lo[b]:hi[b]]) for b in range(B)]  # this rank's slice
V = [deq(cache.Vc[b, lo[b]:hi[b]], cache.scale[b, lo[b]:hi[b]]) for b in range(B)]
L2E = 1 / math.log(2)

def state(x, v):  # softmax-state record over base-2 logits x [n] and values v [n, 128]
    if len(x) == 0:
        return np.concatenate([[-np.inf, 0.0], np.zeros(128)])
    m = x.max(); p = np.exp2(x - m)
    return np.concatenate([[m, p.sum()], p @ v])

def merge(recs):  # records [R, ..., 130] -> (o, base-2 lse)
    m = recs[..., 0].max(0)
    f = np.where(recs[..., 0] == -np.inf, 0.0, np.exp2(recs[..., 0] - m))
    l = (recs[..., 1] * f).sum(0)
    o = (recs[..., 2:] * f[..., None]).sum(0) / l[..., None]
    return o, m + np.log2(l)

# 1. attention over the slice
rec = np.stack([np.stack([state(K[b][:, h // G] @ bf(q[b, h]) * sc * L2E, V[b][:, h // G])
                          for h in range(Hq)]) for b in range(B)])
recs = gather(torch.from_numpy(rec)).numpy()
o_full, lse2 = merge(recs)
# 2. local top k of the slice's candidates (ties to the smaller position)
sel = np.zeros((B, Hkv, k, 2), np.float64); sel[..., 0] = -1.0; sel[..., 1] = -1
for b in range(B):
    i = lens[b] - 1
    for g in range(Hkv):
        js = np.arange(lo[b], min(hi[b], i - w + 1))
        if len(js):
            x = np.stack([K[b][js - lo[b], g] @ bf(q[b, g * G + h]) * sc * L2E - lse2[b, g * G + h]
                          for h in range(G)])
            s = np.exp2(x).sum(0)
            order = np.lexsort((js, -s))[:k]
            sel[b, g, :len(order), 0] = s[order]; sel[b, g, :len(order), 1] = js[order]
sels = gather(torch.from_numpy(sel)).numpy()
# 3. merge of the ranks' top k -> index lists; sparse layers over the slice
idx = np.full((B, Hkv, k + w), -1, np.int32)
for b in range(B):
    i = lens[b] - 1
    ncand = max(0, i - w + 1)
    for g in range(Hkv):
        if ncand <= k:
            top = np.arange(ncand)
        else:
            cand = sels[:, b, g].reshape(-1, 2); cand = cand[cand[:, 1] >= 0]
            top = np.sort(cand[np.lexsort((cand[:, 1], -cand[:, 0]))][:k, 1].astype(np.int64))
        idx[b, g, :len(top)] = top
        win = np.arange(i - w + 1, i + 1); idx[b, g, k:] = np.where(win >= 0, win, -1)
srec = np.zeros((L, B, Hq, 130))
for l in range(L):
    for b in range(B):
        for h in range(Hq):
            js = idx[b, h // G]; js = js[(js >= lo[b]) & (js < hi[b])]
            srec[l, b, h] = state(K[b][js - lo[b], h // G] @ bf(qs[l][b, h]) * sc * L2E,
                                  V[b][js - lo[b], h // G])
srecs = gather(torch.from_numpy(srec)).numpy()
o_sparse = [merge(srecs[:, l])[0] for l in range(L)]
# the oracle on the whole cache
kvs = [oracle.KV(cache.Kc[b, :lens[b]], cache.Vc[b, :lens[b]], cache.scale[b, :lens[b]],
                 cache.scale[b, :lens[b]]) for b in range(B)]
ref = oracle.decode(kvs, q, qs, sc, k, w)
err_o = max(np.abs(o_full[b] - ref[b]["O"][0]).max() for b in range(B))
err_lse = max(np.abs(lse2[b] / L2E - ref[b]["lse"][0]).max() for b in range(B))
n_diff = 0
for b in range(B):
    n_diff += check_index_lists(idx[b:b + 1], ref[b]["idx"], ref[b]["kth"], [lens[b] - 1], k, w,
                                lambda r, g, js: oracle.scores(kvs[b], q[b], g, sc,
                                                               ref[b]["lse"][0], js))
err_s = max(np.abs(o_sparse[l][b] - oracle.sparse_attn(kvs[b], qs[l][b:b + 1], idx[b:b + 1], sc)[0][0]).max()
            for l in range(L) for b in range(B))
print(json.dumps({{"rank": rank, "lo": lo, "hi": hi, "err_o": float(err_o), "err_lse": float(err_lse),
                   "n_diff": int(n_diff), "err_sparse": float(err_s),
                   "checksum": float(o_full.sum() + sum(o.sum() for o in o_sparse)),
                   "idx_sum": int(idx.astype(np.int64).sum())}}), flush=True)
dist.barrier()
dist.destroy_process_group()
"""


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_context_parallel_decode_protocol_on_two_gloo_ranks():
    port, world = _free_port(), 2
    code = WORKER.format(root=ROOT)
    procs = []
    for r in range(world):
        env = dict(os.environ)
        env.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(r),
                   WORLD_SIZE=str(world), LOCAL_RANK=str(r))
        procs.append(subprocess.Popen([sys.executable, "-c", code], env=env, cwd=ROOT,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=300)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            raise
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    outs.sort(key=lambda o: o["rank"])
    # the slices tile every sequence in rank order
    assert outs[0]["lo"] == [0, 0, 0] and outs[0]["hi"] == outs[1]["lo"]
    assert outs[1]["hi"] == [700, 333, 130]
    for o in outs:
        assert o["err_o"] < 1e-9 and o["err_lse"] < 1e-9 and o["err_sparse"] < 1e-9
        assert o["n_diff"] == 0
    # every rank ends with the same outputs
    assert outs[0]["checksum"] == outs[1]["checksum"] and outs[0]["idx_sum"] == outs[1]["idx_sum"]


PREFILL_WORKER = r"""
import json, os, sys
sys.path.insert(0, {root!r})
import numpy as np, torch
import torch.distributed as dist
from long_context_bridge_b200 import Shape
from long_context_bridge_b200 import context_parallel as cp
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo")
T = 4 * world * 128
K = torch.from_numpy(np.random.default_rng(3).standard_normal((T, 2, 128)).astype(np.float32))
x = cp.PrefillRows(Shape.make(T, 8, 2), world, rank, "cpu")
rows = x.rows()
got = x.assemble(cp.dist_all_gather()(K[rows].contiguous()))  # this rank's rows only, exchanged
print(json.dumps({{"rank": rank, "chunks": x.chunks, "same": bool(torch.equal(got, K)),
                   "work": int((rows + 1).sum())}}), flush=True)
dist.barrier()
dist.destroy_process_group()
"""


def test_prefill_rows_exchange_on_gloo_ranks():
    """Row-sharded prefill: with R ranks owning zig-zag chunks r and 2R-1-r,
    exchanging each rank's own rows of K/V and reassembling them gives the
    whole prompt's K/V on every rank, and every rank's causal work (the sum
    over its rows of the keys each row attends to) is the same."""
    for world in (2, 3):
        port = _free_port()
        code = PREFILL_WORKER.format(root=ROOT)
        procs = []
        for r in range(world):
            env = dict(os.environ)
            env.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(r),
                       WORLD_SIZE=str(world), LOCAL_RANK=str(r))
            procs.append(subprocess.Popen([sys.executable, "-c", code], env=env, cwd=ROOT,
                                          stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                          text=True))
        outs = []
        for p in procs:
            try:
                out, err = p.communicate(timeout=300)
            except subprocess.TimeoutExpired:
                for q in procs:
                    q.kill()
                raise
            assert p.returncode == 0, err
            outs.append(json.loads(out.strip().splitlines()[-1]))
        assert all(o["same"] for o in outs)
        assert len({o["work"] for o in outs}) == 1
        spans = sorted(tuple(c) for o in outs for c in o["chunks"])
        assert spans[0][0] == 0 and all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
