"""Block-level GPU parity: hs2_block_prefill (bridge, full attention,
selection, sparse layers sharing K/V and the index list) against the oracle on
the configured workloads' shapes and value recipes."""
import math

import numpy as np
import pytest

import synth
from helpers import assert_close_bf16, check_index_lists, dev, dev_bf16, host_f64, LSE_ABS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hs2():
    import torch
    assert torch.cuda.is_available()
    import long_context_bridge_b200 as m
    return m


def edge_rows(T, k=1024, w=128, n_random=0, seed=0):
    base = [0, 1, w - 1, w, w + 1, k + w - 2, k + w - 1, k + w, k + w + 1, T // 2, T - 2, T - 1]
    rows = set(r for r in base if 0 <= r < T)
    if n_random:
        rng = np.random.default_rng(seed)
        rows |= set(rng.integers(0, T, n_random).tolist())
    return np.array(sorted(rows), np.int64)


def run_block(hs2, cfg, K, V, Q, Qs, H=None, Wk=None, Wv=None, T=None):
    import torch
    T = cfg.T if T is None else T
    shape = hs2.Shape.make(T, cfg.n_q_heads, cfg.n_kv_heads)
    Kd, Vd = (dev_bf16(K), dev_bf16(V)) if H is None else (
        torch.empty(T, cfg.n_kv_heads, 128, dtype=torch.bfloat16, device="cuda"),
        torch.empty(T, cfg.n_kv_heads, 128, dtype=torch.bfloat16, device="cuda"))
    Qd = dev_bf16(Q)
    Qsd = [dev_bf16(q) for q in Qs]
    O = torch.empty_like(Qd)
    Os = [torch.empty_like(Qd) for _ in Qs]
    lse = torch.empty(T, cfg.n_q_heads, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, cfg.n_kv_heads, 1152, dtype=torch.int32, device="cuda")
    ws = torch.empty(hs2.workspace_size(hs2.OP_BLOCK_PREFILL, shape), dtype=torch.uint8,
                     device="cuda")
    hs2.hs2_block_prefill(None if H is None else dev_bf16(H), None if H is None else dev_bf16(Wk),
                          None if H is None else dev_bf16(Wv), Kd, Vd, Qd, O, lse, idx, Qsd, Os,
                          shape, ws)
    assert hs2.hs2_get_device_status() == hs2.OK
    return {"K": Kd, "V": Vd, "O": O, "lse": lse, "idx": idx, "O_sparse": Os}


def compare_block(orc, cfg, kv, Q, Qs, rows, got):
    """Compare GPU block outputs on `rows` with the oracle.  Sparse outputs:
    against the oracle on its own lists where the GPU list is identical, and
    on the GPU's list (validated by check_index_lists) where it differs."""
    sc = cfg.scale
    Qr = Q[rows]
    ref = orc.block_rows(kv, Qr, [q[rows] for q in Qs], rows, sc)
    assert_close_bf16(host_f64(got["O"][rows]), ref["O"], "O_full")
    assert np.max(np.abs(got["lse"][rows].cpu().numpy() - ref["lse"])) <= LSE_ABS
    gi = got["idx"][rows].cpu().numpy()
    n_diff = check_index_lists(gi, ref["idx"], ref["kth"], rows, cfg.k_global, cfg.window,
                               lambda r, g, js: orc.scores(kv, Qr[r], g, sc, ref["lse"][r], js))
    same = np.all(gi == ref["idx"], axis=(1, 2))
    for l, q in enumerate(Qs):
        gs = host_f64(got["O_sparse"][l][rows])
        if same.any():
            assert_close_bf16(gs[same], ref["O_sparse"][l][same], f"O_sparse[{l}]")
        if (~same).any():
            o_on_gpu_list, _ = orc.sparse_attn(kv, q[rows][~same], gi[~same], sc)
            assert_close_bf16(gs[~same], o_on_gpu_list, f"O_sparse[{l}] on GPU lists")
    return n_diff


def test_block_c1_all_rows(hs2, orc):
    cfg = synth.CONFIGS["C1"]
    K, V = synth.kv_np(cfg, synth.TID_K), synth.kv_np(cfg, synth.TID_V)
    rows = np.arange(cfg.T)
    Q = synth.q_rows_np(cfg, synth.TID_Q, rows)
    Qs = [synth.q_rows_np(cfg, synth.TID_QS0 + l, rows) for l in range(cfg.n_sparse)]
    got = run_block(hs2, cfg, K, V, Q, Qs)
    n_diff = compare_block(orc, cfg, orc.KV(K, V), Q, Qs, rows, got)
    assert n_diff <= 0.01 * cfg.T


@pytest.mark.slow
def test_block_c2_sampled_rows_with_bridge(hs2, orc):
    """C2: bridge from H, needles planted after the bridge.  The block runs on
    the oracle's bridged K/V (so selection compares like with like); the GPU
    bridge is checked against the same K/V separately."""
    import torch
    cfg = synth.CONFIGS["C2"]
    T = cfg.T
    H, Wk, Wv = synth.bridge_inputs_np(cfg)
    Ko = orc.bridge(H, Wk).reshape(T, cfg.n_kv_heads, 128)
    Vo = orc.bridge(H, Wv).reshape(T, cfg.n_kv_heads, 128)
    # GPU bridge vs oracle bridge (before needles): at most a bf16 ulp apart
    Kg = torch.empty(T, cfg.n_kv_heads, 128, dtype=torch.bfloat16, device="cuda")
    Vg = torch.empty_like(Kg)
    hs2.hs2_bridge_kv(dev_bf16(H), dev_bf16(Wk), dev_bf16(Wv), Kg, Vg,
                      hs2.Shape.make(T, cfg.n_q_heads, cfg.n_kv_heads))
    for g_, o_ in ((Kg, Ko), (Vg, Vo)):
        gb = g_.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.mean(gb == o_) > 0.99
        d = np.abs(synth.bf16_bits_to_f32(gb).astype(np.float64) - synth.bf16_bits_to_f32(o_))
        assert d.max() <= 2 ** -6
    synth.plant_needles_np(cfg, Ko, synth.prefill_needles(cfg))
    rows = edge_rows(T, n_random=120, seed=2)
    allrows = np.arange(T)
    Q = synth.q_rows_np(cfg, synth.TID_Q, allrows)
    Qs = [synth.q_rows_np(cfg, synth.TID_QS0 + l, allrows) for l in range(cfg.n_sparse)]
    got = run_block(hs2, cfg, Ko, Vo, Q, Qs)
    n_diff = compare_block(orc, cfg, orc.KV(Ko, Vo), Q, Qs, rows, got)
    assert n_diff <= 0.02 * len(rows) * cfg.n_kv_heads
