"""GPU parity on paths the other block tests do not reach: the bridge inside
hs2_block_prefill, the selection's buffer-overflow fall-backs, exact ties
everywhere (prefill selection and decode), and a decode cache whose K and V
rows carry different scales.  Every case goes through the C ABI and is
compared with the oracle on the same inputs."""
import math

import numpy as np
import pytest

import synth
from helpers import (LSE_ABS, assert_close_bf16, bits, check_index_lists, compare_rows, dev,
                     dev_bf16, edge_rows, host_f64)

pytestmark = pytest.mark.gpu
RNG = np.random.default_rng(20261203)


@pytest.fixture(scope="module")
def hs2():
    import torch
    assert torch.cuda.is_available()
    import long_context_bridge_b200 as m
    return m


def rand_bf16(shape, sd=1.0):
    return synth.f64_to_bf16_bits(RNG.standard_normal(shape) * sd)


# ---------------------------------------------------------------------------
# the bridge inside the block call
# ---------------------------------------------------------------------------
@pytest.mark.slow
@pytest.mark.parametrize("name,n_random", [("C2", 120), ("C3", 116)])
def test_block_prefill_with_bridge_inside(hs2, orc, name, n_random):
    """hs2_block_prefill with H: the call bridges K/V itself, then runs full
    attention, selection and the sparse layers on them.  H and W follow the
    workload's recipe on a dyadic grid (synth.bridge_inputs_dyadic_*), where
    every partial sum of the projection is exact in fp32, so the K/V the call
    writes must equal the oracle's bridge bit for bit.  The block's outputs on
    sampled rows are then compared with the oracle run on the oracle's own
    K/V.  Needles are not planted: the call runs the bridge and the attention
    back to back."""
    import torch
    cfg = synth.CONFIGS[name]
    T, Hq, Hkv = cfg.T, cfg.n_q_heads, cfg.n_kv_heads
    H, Wk, Wv = synth.bridge_inputs_dyadic_torch(cfg)
    Q = synth.q_rows_torch(cfg, synth.TID_Q)
    Qs = [synth.q_rows_torch(cfg, synth.TID_QS0 + l) for l in range(cfg.n_sparse)]
    shape = hs2.Shape.make(T, Hq, Hkv)
    K = torch.empty(T, Hkv, 128, dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    O = torch.empty_like(Q)
    Os = [torch.empty_like(Q) for _ in Qs]
    lse = torch.empty(T, Hq, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, Hkv, cfg.k_global + cfg.window, dtype=torch.int32, device="cuda")
    ws = torch.empty(hs2.workspace_size(hs2.OP_BLOCK_PREFILL, shape), dtype=torch.uint8,
                     device="cuda")
    hs2.hs2_block_prefill(H, Wk, Wv, K, V, Q, O, lse, idx, Qs, Os, shape, ws)
    assert hs2.hs2_get_device_status() == hs2.OK
    del Q, Qs
    Hb, Wkb, Wvb = bits(H), bits(Wk), bits(Wv)
    del H
    Ko = orc.bridge(Hb, Wkb).reshape(T, Hkv, 128)
    Vo = orc.bridge(Hb, Wvb).reshape(T, Hkv, 128)
    del Hb
    assert np.array_equal(bits(K), Ko), "K written by the block call differs from the oracle"
    assert np.array_equal(bits(V), Vo), "V written by the block call differs from the oracle"
    rows = edge_rows(T, n_random=n_random, seed=11)
    Qr = synth.q_rows_np(cfg, synth.TID_Q, rows)
    Qsr = [synth.q_rows_np(cfg, synth.TID_QS0 + l, rows) for l in range(cfg.n_sparse)]
    got = {"O": O, "lse": lse, "idx": idx, "O_sparse": Os}
    n_diff = compare_rows(orc, cfg, orc.KV(Ko, Vo), Qr, Qsr, rows, got)
    assert n_diff <= 0.05 * len(rows) * Hkv


# ---------------------------------------------------------------------------
# selection: exact ties and buffer overflow
# ---------------------------------------------------------------------------
def _select_on_device(hs2, Q, K, lse, shape, T, Hkv, k, w):
    import torch
    ws = torch.empty(max(16, hs2.workspace_size(hs2.OP_SELECT, shape)), dtype=torch.uint8,
                     device="cuda")
    idx = torch.full((T, Hkv, k + w), -7, dtype=torch.int32, device="cuda")
    kth = torch.full((T, Hkv), -7.0, dtype=torch.float32, device="cuda")
    hs2.hs2_select_topk(dev_bf16(Q), dev_bf16(K), dev(lse.astype(np.float32)), idx, kth, shape, ws)
    assert hs2.hs2_get_device_status() == hs2.OK
    return idx.cpu().numpy(), kth.cpu().numpy()


def _expected_all_ties(T, Hkv, k, w):
    idx = np.full((T, Hkv, k + w), -1, np.int32)
    for i in range(T):
        c = max(0, i - w + 1)
        idx[i, :, :min(c, k)] = np.arange(min(c, k))
        win = np.arange(i - w + 1, i + 1)
        idx[i, :, k:] = np.where(win >= 0, win, -1)
    return idx


@pytest.mark.parametrize("T,Hq,Hkv,k,w", [(4000, 8, 1, 64, 16), (3000, 16, 2, 64, 32),
                                          (2600, 4, 1, 1024, 128), (1500, 2, 1, 100, 8)])
def test_select_all_ties_takes_smallest_positions(hs2, orc, T, Hq, Hkv, k, w):
    """Every key row of a KV head is the same row, so every candidate of a
    query has exactly the same score and the k selected must be positions
    0 .. k-1 (equal scores go to the smaller position).  The 1e-4 tolerance
    of the other selection tests would accept any k of them, so the lists
    are asserted exactly, on the GPU and on the oracle.

    Buffer arithmetic: a tie leaves every candidate at or above any score
    floor, so no candidate is ever filtered out while streaming.  A query at
    position i has c = i - w + 1 candidates, spread evenly over the four
    32-key sub-buffers that hold its candidates (one per key quarter of a
    128-key tile), about c / 4 per sub-buffer, each of capacity
    max(2k, 256) = 256 for k <= 128.  A sub-buffer makes room once it holds
    more than 224 entries, i.e. for every query with c > 4 * 224 = 896
    (T = 4000: rows 912 .. 3999); dropping the entries below the floor frees
    nothing (all are at the floor), so it then keeps its own exact k best by
    the in-buffer radix select (n > capacity / 2 + k / 2 - 32 and n > k)."""
    Q = rand_bf16((T, Hq, 128))
    K = np.repeat(rand_bf16((1, Hkv, 128)), T, axis=0)
    V = rand_bf16((T, Hkv, 128))
    kv, sc = orc.KV(K, V), 1 / math.sqrt(128)
    rows = np.arange(T)
    _, lse = orc.full_attn(kv, Q, rows, sc)
    want = _expected_all_ties(T, Hkv, k, w)
    idx_o, kth_o = orc.select(kv, Q, rows, sc, lse, k, w)
    assert np.array_equal(idx_o, want), "oracle: ties must go to the smaller position"
    shape = hs2.Shape.make(T, Hq, Hkv, k_global=k, window=w)
    gi, gk = _select_on_device(hs2, Q, K, lse, shape, T, Hkv, k, w)
    bad = np.argwhere(np.any(gi != want, axis=2))
    assert len(bad) == 0, f"GPU lists differ from 0..k-1 at (row, head) {bad[:5].tolist()}"
    sel = ~np.isnan(kth_o)
    assert np.all(gk[~sel] == -1.0)
    np.testing.assert_allclose(gk[sel], kth_o[sel], rtol=1e-4)


@pytest.mark.parametrize("T,Hq,Hkv,k,w", [(4000, 8, 1, 64, 16), (5000, 8, 2, 1024, 128)])
def test_select_rising_scores(hs2, orc, T, Hq, Hkv, k, w):
    """Scores that rise with position: K_j = (1 + 2 j / T) * 4 u_g and every
    query head of KV head g points along u_g (plus a little noise), so a new
    key beats the earlier ones and the streaming filter keeps admitting keys
    to the end of each query's range; the k best are the most recent
    candidates up to the bf16 rounding of K.  Compared with the oracle at the
    block's tolerance."""
    u = RNG.standard_normal((Hkv, 128))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    ramp = 1.0 + 2.0 * np.arange(T) / T
    K = synth.f64_to_bf16_bits(4.0 * ramp[:, None, None] * u[None])
    G = Hq // Hkv
    Q = synth.f64_to_bf16_bits(np.repeat(u, G, axis=0)[None] * math.sqrt(128) +
                               0.05 * RNG.standard_normal((T, Hq, 128)))
    V = rand_bf16((T, Hkv, 128))
    kv, sc = orc.KV(K, V), 1 / math.sqrt(128)
    rows = np.arange(T)
    _, lse = orc.full_attn(kv, Q, rows, sc)
    idx_o, kth_o = orc.select(kv, Q, rows, sc, lse, k, w)
    shape = hs2.Shape.make(T, Hq, Hkv, k_global=k, window=w)
    gi, gk = _select_on_device(hs2, Q, K, lse, shape, T, Hkv, k, w)
    n_diff = check_index_lists(gi, idx_o, kth_o, rows, k, w,
                               lambda r, g, js: orc.scores(kv, Q[r], g, sc, lse[r], js))
    assert n_diff <= 0.05 * T * Hkv
    sel = ~np.isnan(kth_o)
    np.testing.assert_allclose(gk[sel], kth_o[sel], rtol=1e-4)


# ---------------------------------------------------------------------------
# decode: exact ties over the whole cache; separate K and V scales
# ---------------------------------------------------------------------------
def _decode(hs2, orc, Kc, Vc, KS, VS, lens, Hq, Hkv, k, w, n_sparse=3, seed=0):
    import torch
    B, cap = Kc.shape[0], Kc.shape[1]
    rng = np.random.default_rng(seed)
    q = synth.f64_to_bf16_bits(rng.standard_normal((B, Hq, 128)))
    qs = [synth.f64_to_bf16_bits(rng.standard_normal((B, Hq, 128))) for _ in range(n_sparse)]
    shape = hs2.Shape.make(cap, Hq, Hkv, k_global=k, window=w)
    o = torch.empty(B, Hq, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    idx = torch.full((B, Hkv, k + w), -7, dtype=torch.int32, device="cuda")
    os_ = [torch.empty_like(o) for _ in range(n_sparse)]
    ws = torch.empty(hs2.workspace_size(hs2.OP_BLOCK_DECODE, shape, B), dtype=torch.uint8,
                     device="cuda")
    hs2.hs2_block_decode(lens, dev_bf16(q), dev(Kc), dev(Vc), dev(KS), dev(VS), o, lse, idx,
                         [dev_bf16(x) for x in qs], os_, shape, ws)
    assert hs2.hs2_get_device_status() == hs2.OK
    kvs = [orc.KV(Kc[b, :lens[b]], Vc[b, :lens[b]], KS[b, :lens[b]], VS[b, :lens[b]])
           for b in range(B)]
    ref = orc.decode(kvs, q, qs, 1 / math.sqrt(128), k, w)
    got = {"o": host_f64(o), "lse": lse.cpu().numpy(), "idx": idx.cpu().numpy(),
           "os": [host_f64(x) for x in os_]}
    return got, ref, kvs, q, qs


def test_decode_all_ties_overflows_candidate_list(hs2, orc):
    """Every cache row of a sequence holds the same K codes and scale, so all
    of its candidates tie and the k selected must be positions 0 .. k-1.  All
    candidates then fall in the one score bucket that holds the k-th best, so
    the per-(sequence, KV head) candidate list (capacity 8192) overflows for
    both sequences (19873 and 8874 candidates) and the final step takes the
    exact radix select over every candidate's score."""
    B, cap, Hq, Hkv, k, w = 2, 20000, 32, 4, 1024, 128
    lens = [20000, 9001]
    rng = np.random.default_rng(7)
    Kc = np.repeat(rng.integers(0, 0x7E, (B, 1, Hkv, 128)).astype(np.uint8), cap, axis=1)
    Kc |= (rng.integers(0, 2, (B, 1, Hkv, 128)).astype(np.uint8) << 7)
    Vc = rng.integers(0, 0x7E, (B, cap, Hkv, 128)).astype(np.uint8)
    KS = np.full((B, cap, Hkv), 1.0 / 64, np.float32)
    VS = (rng.random((B, cap, Hkv)) * 0.01 + 0.001).astype(np.float32)
    got, ref, _, _, _ = _decode(hs2, orc, Kc, Vc, KS, VS, lens, Hq, Hkv, k, w, seed=8)
    for b in range(B):
        i = lens[b] - 1
        want = np.concatenate([np.arange(k), np.arange(i - w + 1, i + 1)]).astype(np.int32)
        assert np.array_equal(ref[b]["idx"][0], np.broadcast_to(want, (Hkv, k + w)))
        assert np.array_equal(got["idx"][b], np.broadcast_to(want, (Hkv, k + w))), \
            f"sequence {b}: GPU list is not 0..k-1 plus the window"
        assert_close_bf16(got["o"][b], ref[b]["O"][0], f"o_full[{b}]")
        assert np.max(np.abs(got["lse"][b] - ref[b]["lse"][0])) <= LSE_ABS
        for l in range(3):
            assert_close_bf16(got["os"][l][b], ref[b]["O_sparse"][l][0], f"o_sparse[{l}][{b}]")


def test_decode_separate_k_and_v_scales(hs2, orc):
    """K and V rows quantised with their own per-(token, KV head) scales, V
    eight times larger than K, passed as two separate scale tensors.  The
    outputs must match the oracle on the same cache, and must NOT match the
    oracle with the two scale tensors swapped (so a mix-up of k_scale and
    v_scale anywhere in the decode path fails this test)."""
    cfg = synth.BlockConfig("decode split scales", 5, 9000, 32, 4, n_needles=64, q_mix=True,
                            batch=3, fp8_cache=True)
    lens = [9000, 4097, 1100]
    Kc, Vc, KS, VS = synth.decode_cache_split_scales_np(cfg, 9000, batch=3)
    got, ref, kvs, q, qs = _decode(hs2, orc, Kc, Vc, KS, VS, lens, 32, 4, 1024, 128, seed=9)
    n_diff = 0
    for b in range(3):
        r = ref[b]
        assert_close_bf16(got["o"][b], r["O"][0], f"o_full[{b}]")
        assert np.max(np.abs(got["lse"][b] - r["lse"][0])) <= LSE_ABS
        n_diff += check_index_lists(got["idx"][b:b + 1], r["idx"], r["kth"], [lens[b] - 1], 1024,
                                    128, lambda rr, g, js: orc.scores(kvs[b], q[b], g,
                                                                      1 / math.sqrt(128),
                                                                      r["lse"][0], js))
        same = np.array_equal(got["idx"][b], r["idx"][0])
        for l in range(3):
            want = r["O_sparse"][l][0] if same else orc.sparse_attn(
                kvs[b], qs[l][b:b + 1], got["idx"][b:b + 1], 1 / math.sqrt(128))[0][0]
            assert_close_bf16(got["os"][l][b], want, f"o_sparse[{l}][{b}]")
        swapped = orc.KV(Kc[b, :lens[b]], Vc[b, :lens[b]], VS[b, :lens[b]], KS[b, :lens[b]])
        o_sw, _ = orc.full_attn(swapped, q[b:b + 1], np.array([lens[b] - 1]), 1 / math.sqrt(128))
        rel = np.linalg.norm(got["o"][b] - o_sw[0]) / np.linalg.norm(o_sw[0])
        assert rel > 0.1, "swapped scales give the same output"
    assert n_diff <= 1


@pytest.mark.parametrize("T,Hq,Hkv,k,w", [(6000, 8, 2, 1024, 128), (9000, 32, 4, 256, 64),
                                          (5000, 4, 1, 64, 16)])
def test_select_speculative_floor_never_changes_results(hs2, orc, T, Hq, Hkv, k, w):
    """The selection starts each work item's floor at a fraction of the
    smallest k-th best score its CTA found in its previous item of the same KV
    head.  A floor above an item's true k-th best is detected and that item is
    recomputed without it, so the lists and k-th scores must be bit for bit
    the same with the default fraction, with speculation off, and with a
    fraction so large that every speculative item fails and is recomputed;
    and they must match the oracle.  T is large enough that CTAs take several
    items of one head."""
    import torch
    Q, K, V = rand_bf16((T, Hq, 128)), rand_bf16((T, Hkv, 128)), rand_bf16((T, Hkv, 128))
    kv, sc = orc.KV(K, V), 1 / math.sqrt(128)
    rows = np.arange(T)
    _, lse = orc.full_attn(kv, Q, rows, sc)
    shape = hs2.Shape.make(T, Hq, Hkv, k_global=k, window=w)
    got = {}
    try:
        for name, f in (("default", 0.9), ("off", 0.0), ("forced", 1e30)):
            hs2.hs2_debug_set_select_speculation(f)
            got[name] = _select_on_device(hs2, Q, K, lse, shape, T, Hkv, k, w)
    finally:
        hs2.hs2_debug_set_select_speculation(0.9)
    for name in ("off", "forced"):
        assert np.array_equal(got[name][0], got["default"][0]), f"{name}: index lists differ"
        assert np.array_equal(got[name][1], got["default"][1]), f"{name}: k-th scores differ"
    idx_o, kth_o = orc.select(kv, Q, rows, sc, lse, k, w)
    n_diff = check_index_lists(got["default"][0], idx_o, kth_o, rows, k, w,
                               lambda r, g, js: orc.scores(kv, Q[r], g, sc, lse[r], js))
    assert n_diff <= 0.01 * T * Hkv
