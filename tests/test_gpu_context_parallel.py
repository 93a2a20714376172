"""Decode with each sequence's context split over ranks (hs2_decode_cp_*), on
one GPU: R virtual ranks, each holding only its slice of every sequence's
FP8 cache, run the four steps in lockstep; their records are stacked in rank
order as an all-gather would.  Outputs are checked against the oracle on the
whole cache and against the single-device hs2_block_decode; every virtual
rank must end with the same outputs."""
import math

import numpy as np
import pytest

import synth
from helpers import LSE_ABS, assert_close_bf16, check_index_lists, dev, dev_bf16, host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hs2():
    import torch
    assert torch.cuda.is_available()
    import long_context_bridge_b200 as m
    return m


@pytest.mark.parametrize("R,lens", [(2, [20000, 9001, 3000]), (3, [16384, 12000, 1200]),
                                    (1, [5000, 4097])])
def test_decode_context_parallel_virtual_ranks(hs2, orc, R, lens):
    import torch
    from long_context_bridge_b200 import context_parallel as cp
    B, Hq, Hkv, k, w, L = len(lens), 32, 4, 1024, 128, 3
    cap = max(lens)
    cfg = synth.BlockConfig("context-parallel decode", 5, cap, Hq, Hkv, n_needles=256,
                            q_mix=True, batch=B, fp8_cache=True)
    cache = synth.decode_cache_np(cfg, cap, batch=B)
    q = synth.decode_queries_np(cfg, synth.TID_Q, batch=B)
    qs = [synth.decode_queries_np(cfg, synth.TID_QS0 + l, batch=B) for l in range(L)]
    qd, qsd = dev_bf16(q), [dev_bf16(x) for x in qs]
    sc = 1 / math.sqrt(128)

    # each virtual rank's cache holds its slice of every sequence only
    cap_r = cp.local_capacity(lens, R)
    shape_r = hs2.Shape.make(cap_r, Hq, Hkv, k_global=k, window=w)
    ranks = []
    for r in range(R):
        lo, hi = cp.slice_bounds(lens, R, r)
        Kc = np.zeros((B, cap_r, Hkv, 128), np.uint8)
        Vc = np.zeros_like(Kc)
        S = np.ones((B, cap_r, Hkv), np.float32)
        for b in range(B):
            Kc[b, :hi[b] - lo[b]] = cache.Kc[b, lo[b]:hi[b]]
            Vc[b, :hi[b] - lo[b]] = cache.Vc[b, lo[b]:hi[b]]
            S[b, :hi[b] - lo[b]] = cache.scale[b, lo[b]:hi[b]]
        ranks.append(dict(lo=lo, hi=hi, Kc=dev(Kc), Vc=dev(Vc), S=dev(S),
                          cp=cp.DecodeCP(B, shape_r, R, L, "cuda"),
                          o=torch.empty(B, Hq, 128, dtype=torch.bfloat16, device="cuda"),
                          lse=torch.empty(B, Hq, dtype=torch.float32, device="cuda"),
                          idx=torch.full((B, Hkv, k + w), -7, dtype=torch.int32, device="cuda"),
                          os=[torch.empty(B, Hq, 128, dtype=torch.bfloat16, device="cuda")
                              for _ in range(L)]))
    stack = lambda ts: torch.stack([t.clone() for t in ts])  # an all-gather, rank order
    recs = stack([x["cp"].attn(lens, x["lo"], x["hi"], qd, x["Kc"], x["Vc"], x["S"], x["S"])
                  for x in ranks])
    recs = stack([x["cp"].select(lens, x["lo"], x["hi"], recs, x["o"], x["lse"]) for x in ranks])
    recs = stack([x["cp"].sparse(lens, x["lo"], x["hi"], recs, x["idx"], x["Kc"], x["Vc"], x["S"],
                                 x["S"], qsd) for x in ranks])
    for x in ranks:
        x["cp"].finish(recs, x["os"])
    assert hs2.hs2_get_device_status() == hs2.OK
    # every rank ends with the same outputs
    for x in ranks[1:]:
        assert torch.equal(x["o"], ranks[0]["o"]) and torch.equal(x["lse"], ranks[0]["lse"])
        assert torch.equal(x["idx"], ranks[0]["idx"])
        for l in range(L):
            assert torch.equal(x["os"][l], ranks[0]["os"][l])
    got = ranks[0]

    # the single-device block decode on the whole cache
    shape = hs2.Shape.make(cap, Hq, Hkv, k_global=k, window=w)
    o1 = torch.empty(B, Hq, 128, dtype=torch.bfloat16, device="cuda")
    lse1 = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    idx1 = torch.empty(B, Hkv, k + w, dtype=torch.int32, device="cuda")
    os1 = [torch.empty_like(o1) for _ in range(L)]
    ws = torch.empty(hs2.workspace_size(hs2.OP_BLOCK_DECODE, shape, B), dtype=torch.uint8,
                     device="cuda")
    Sd = dev(cache.scale)
    hs2.hs2_block_decode(lens, qd, dev(cache.Kc), dev(cache.Vc), Sd, Sd, o1, lse1, idx1, qsd, os1,
                         shape, ws)
    assert hs2.hs2_get_device_status() == hs2.OK
    assert_close_bf16(host_f64(got["o"]), host_f64(o1), "o_full vs one device")
    assert np.max(np.abs(got["lse"].cpu().numpy() - lse1.cpu().numpy())) <= 1e-5

    # the oracle on the whole cache
    kvs = [orc.KV(cache.Kc[b, :lens[b]], cache.Vc[b, :lens[b]], cache.scale[b, :lens[b]],
                  cache.scale[b, :lens[b]]) for b in range(B)]
    ref = orc.decode(kvs, q, qs, sc, k, w)
    go, gl, gi = host_f64(got["o"]), got["lse"].cpu().numpy(), got["idx"].cpu().numpy()
    n_diff = 0
    for b in range(B):
        r = ref[b]
        assert_close_bf16(go[b], r["O"][0], f"o_full[{b}]")
        assert np.max(np.abs(gl[b] - r["lse"][0])) <= LSE_ABS
        n_diff += check_index_lists(gi[b:b + 1], r["idx"], r["kth"], [lens[b] - 1], k, w,
                                    lambda rr, g, js: orc.scores(kvs[b], q[b], g, sc,
                                                                 r["lse"][0], js))
        same = np.array_equal(gi[b], r["idx"][0])
        for l in range(L):
            want = r["O_sparse"][l][0] if same else orc.sparse_attn(
                kvs[b], qs[l][b:b + 1], gi[b:b + 1], sc)[0][0]
            assert_close_bf16(host_f64(got["os"][l])[b], want, f"o_sparse[{l}][{b}]")
    assert n_diff <= 1


@pytest.mark.parametrize("R,T,Hq,Hkv", [(2, 8192, 16, 2), (4, 8192, 8, 1), (2, 4096, 32, 4)])
def test_prefill_rows_split_over_virtual_ranks(hs2, R, T, Hq, Hkv):
    """Row-sharded prefill on one GPU: R virtual ranks each bridge their
    zig-zag chunks' rows, their K/V are stacked as an all-gather would and
    reassembled, and each rank runs hs2_block_prefill_rows on its chunks.
    Every row must equal, bit for bit, what the single-device
    hs2_block_prefill (bridge inside) computes for the whole prompt: the rows
    of a chunk see the same K/V tiles in the same order."""
    import torch
    from long_context_bridge_b200 import context_parallel as cp
    cfg = synth.BlockConfig("row-sharded prefill", 8, T, Hq, Hkv, d_model=2048, q_mix=True)
    H, Wk, Wv = synth.bridge_inputs_torch(cfg)
    Q = synth.q_rows_torch(cfg, synth.TID_Q)
    Qs = [synth.q_rows_torch(cfg, synth.TID_QS0 + l) for l in range(2)]
    shape = hs2.Shape.make(T, Hq, Hkv)
    # one device, the whole prompt
    K1 = torch.empty(T, Hkv, 128, dtype=torch.bfloat16, device="cuda")
    V1 = torch.empty_like(K1)
    O1, Os1 = torch.empty_like(Q), [torch.empty_like(Q) for _ in Qs]
    lse1 = torch.empty(T, Hq, dtype=torch.float32, device="cuda")
    idx1 = torch.empty(T, Hkv, 1152, dtype=torch.int32, device="cuda")
    ws = torch.empty(hs2.workspace_size(hs2.OP_BLOCK_PREFILL, shape), dtype=torch.uint8,
                     device="cuda")
    hs2.hs2_block_prefill(H, Wk, Wv, K1, V1, Q, O1, lse1, idx1, Qs, Os1, shape, ws)
    # R virtual ranks
    ranks = [cp.PrefillRows(shape, R, r, "cuda") for r in range(R)]
    own = [x.bridge(H[x.rows().cuda()].contiguous(), Wk, Wv) for x in ranks]
    Kg = torch.stack([k for k, _ in own])
    Vg = torch.stack([v for _, v in own])
    for x in ranks:
        K, V = x.assemble(Kg), x.assemble(Vg)
        assert torch.equal(K, K1) and torch.equal(V, V1)
        rows = x.rows().cuda()
        n = rows.numel()
        O, Os = torch.empty(n, Hq, 128, dtype=torch.bfloat16, device="cuda"), None
        Os = [torch.empty_like(O) for _ in Qs]
        lse = torch.empty(n, Hq, dtype=torch.float32, device="cuda")
        idx = torch.empty(n, Hkv, 1152, dtype=torch.int32, device="cuda")
        x.block(K, V, Q[rows].contiguous(), O, lse, idx, [q[rows].contiguous() for q in Qs], Os)
        assert hs2.hs2_get_device_status() == hs2.OK
        assert torch.equal(O, O1[rows]), f"rank {x.rank}: O_full"
        assert torch.equal(lse, lse1[rows]), f"rank {x.rank}: lse"
        assert torch.equal(idx, idx1[rows]), f"rank {x.rank}: idx"
        for l in range(len(Qs)):
            assert torch.equal(Os[l], Os1[l][rows]), f"rank {x.rank}: O_sparse[{l}]"
