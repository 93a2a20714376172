"""Parity at the workloads' full sizes, in the launch configuration bench.py
times, on sampled rows the oracle computes one by one: the 128K block with
the bridge (C3), the 1M-token block (C4), and the 8 x 1M FP8 decode (C5).
Inputs come from the seeded generator on the device (pinned bit for bit to
the numpy definition); the oracle reads the same bits on the host."""
import numpy as np
import pytest

import synth
from helpers import bits, compare_rows, edge_rows, check_index_lists, assert_close_bf16, host_f64, dev_bf16, LSE_ABS

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def hs2():
    import torch
    assert torch.cuda.is_available()
    import long_context_bridge_b200 as m
    return m


def run_prefill(hs2, cfg, K, V):
    import torch
    T = cfg.T
    Q = synth.q_rows_torch(cfg, synth.TID_Q)
    Qs = [synth.q_rows_torch(cfg, synth.TID_QS0 + l) for l in range(cfg.n_sparse)]
    shape = hs2.Shape.make(T, cfg.n_q_heads, cfg.n_kv_heads)
    O = torch.empty_like(Q)
    Os = [torch.empty_like(Q) for _ in Qs]
    lse = torch.empty(T, cfg.n_q_heads, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, cfg.n_kv_heads, 1152, dtype=torch.int32, device="cuda")
    ws = torch.empty(hs2.workspace_size(hs2.OP_BLOCK_PREFILL, shape), dtype=torch.uint8,
                     device="cuda")
    hs2.hs2_block_prefill(None, None, None, K, V, Q, O, lse, idx, Qs, Os, shape, ws)
    assert hs2.hs2_get_device_status() == hs2.OK
    del Q, Qs
    return {"O": O, "lse": lse, "idx": idx, "O_sparse": Os}


def test_c3_block_128k_sampled_rows(hs2, orc):
    import torch
    cfg = synth.CONFIGS["C3"]
    T, Hkv = cfg.T, cfg.n_kv_heads
    H, Wk, Wv = synth.bridge_inputs_torch(cfg)
    # oracle bridge of every row (the attention of a sampled row reads all
    # earlier K/V), then the GPU bridge against it
    Hb, Wkb, Wvb = bits(H), bits(Wk), bits(Wv)
    Ko = orc.bridge(Hb, Wkb).reshape(T, Hkv, 128)
    Vo = orc.bridge(Hb, Wvb).reshape(T, Hkv, 128)
    Kg = torch.empty(T, Hkv, 128, dtype=torch.bfloat16, device="cuda")
    Vg = torch.empty_like(Kg)
    hs2.hs2_bridge_kv(H, Wk, Wv, Kg, Vg, hs2.Shape.make(T, cfg.n_q_heads, Hkv))
    for g_, o_ in ((Kg, Ko), (Vg, Vo)):
        gb = bits(g_)
        assert np.mean(gb == o_) > 0.99
        d = np.abs(synth.bf16_bits_to_f32(gb).astype(np.float64) - synth.bf16_bits_to_f32(o_))
        assert d.max() <= 2 ** -5
    del H, Kg, Vg
    synth.plant_needles_np(cfg, Ko, synth.prefill_needles(cfg))
    got = run_prefill(hs2, cfg, dev_bf16(Ko), dev_bf16(Vo))
    rows = edge_rows(T, n_random=116, seed=3)
    Qr = synth.q_rows_np(cfg, synth.TID_Q, rows)
    Qsr = [synth.q_rows_np(cfg, synth.TID_QS0 + l, rows) for l in range(cfg.n_sparse)]
    n_diff = compare_rows(orc, cfg, orc.KV(Ko, Vo), Qr, Qsr, rows, got)
    assert n_diff <= 0.05 * len(rows) * Hkv


def test_c4_block_1m_sampled_rows(hs2, orc):
    cfg = synth.CONFIGS["C4"]
    K = synth.kv_torch(cfg, synth.TID_K)
    V = synth.kv_torch(cfg, synth.TID_V)
    nr, nh, nv = synth.needle_scatter_torch(cfg)
    K[nr, nh] = nv
    got = run_prefill(hs2, cfg, K, V)
    Kb, Vb = bits(K), bits(V)
    del K, V
    rows = edge_rows(cfg.T, n_random=500, seed=4)
    Qr = synth.q_rows_np(cfg, synth.TID_Q, rows)
    Qsr = [synth.q_rows_np(cfg, synth.TID_QS0 + l, rows) for l in range(cfg.n_sparse)]
    n_diff = compare_rows(orc, cfg, orc.KV(Kb, Vb), Qr, Qsr, rows, got)
    assert n_diff <= 0.05 * len(rows) * cfg.n_kv_heads


def test_c5_decode_1m_all_sequences(hs2, orc):
    import torch
    cfg = synth.CONFIGS["C5"]
    B, N, Hq, Hkv, k, w = cfg.batch, cfg.T, cfg.n_q_heads, cfg.n_kv_heads, cfg.k_global, cfg.window
    Kc, Vc, S = synth.decode_cache_torch(cfg, N)
    q = synth.decode_queries_np(cfg, synth.TID_Q)
    qs = [synth.decode_queries_np(cfg, synth.TID_QS0 + l) for l in range(cfg.n_sparse)]
    shape = hs2.Shape.make(N, Hq, Hkv, k_global=k, window=w)
    o = torch.empty(B, Hq, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    idx = torch.empty(B, Hkv, k + w, dtype=torch.int32, device="cuda")
    os_ = [torch.empty_like(o) for _ in qs]
    ws = torch.empty(hs2.workspace_size(hs2.OP_BLOCK_DECODE, shape, B), dtype=torch.uint8,
                     device="cuda")
    lens = [N] * B
    hs2.hs2_block_decode(lens, dev_bf16(q), Kc, Vc, S, S, o, lse, idx, [dev_bf16(x) for x in qs],
                         os_, shape, ws)
    assert hs2.hs2_get_device_status() == hs2.OK
    Kh, Vh, Sh = Kc.cpu().numpy(), Vc.cpu().numpy(), S.cpu().numpy()
    del Kc, Vc
    kvs = [orc.KV(Kh[b], Vh[b], Sh[b], Sh[b]) for b in range(B)]
    ref = orc.decode(kvs, q, qs, cfg.scale, k, w)
    go, gl, gi = host_f64(o), lse.cpu().numpy(), idx.cpu().numpy()
    n_diff = 0
    for b in range(B):
        r = ref[b]
        assert_close_bf16(go[b], r["O"][0], f"o_full[{b}]")
        assert np.max(np.abs(gl[b] - r["lse"][0])) <= LSE_ABS
        n_diff += check_index_lists(gi[b:b + 1], r["idx"], r["kth"], [N - 1], k, w,
                                    lambda rr, g, js: orc.scores(kvs[b], q[b], g, cfg.scale,
                                                                 r["lse"][0], js))
        same = np.array_equal(gi[b], r["idx"][0])
        for l in range(cfg.n_sparse):
            want = r["O_sparse"][l][0] if same else orc.sparse_attn(
                kvs[b], qs[l][b:b + 1], gi[b:b + 1], cfg.scale)[0][0]
            assert_close_bf16(host_f64(os_[l])[b], want, f"o_sparse[{l}][{b}]")
    assert n_diff <= 2
