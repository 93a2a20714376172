"""GPU parity of each kernel of the block against the CPU oracle, through the
C ABI, at sizes the oracle finishes in seconds that span several tiles and a
ragged tail."""
import math

import numpy as np
import pytest

import synth
from helpers import assert_close_bf16, dev, dev_bf16, host_f64, LSE_ABS

pytestmark = pytest.mark.gpu
RNG = np.random.default_rng(20260925)


def rand_bf16(shape, sd=1.0):
    return synth.f64_to_bf16_bits(RNG.standard_normal(shape) * sd)


@pytest.fixture(scope="module")
def hs2():
    import torch
    assert torch.cuda.is_available()
    import long_context_bridge_b200 as m
    return m


@pytest.mark.parametrize("T,dm,Hkv", [(300, 256, 2), (1024, 2048, 4), (130, 128, 1)])
def test_bridge_matches_oracle(hs2, orc, T, dm, Hkv):
    import torch
    H = rand_bf16((T, dm))
    Wk, Wv = rand_bf16((dm, Hkv * 128), dm ** -0.5), rand_bf16((dm, Hkv * 128), dm ** -0.5)
    K = torch.empty(T, Hkv, 128, dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    shape = hs2.Shape.make(T, Hkv, Hkv)
    hs2.hs2_bridge_kv(dev_bf16(H), dev_bf16(Wk), dev_bf16(Wv), K, V, shape)
    assert hs2.hs2_get_device_status() == hs2.OK
    for got, W in ((K, Wk), (V, Wv)):
        want = orc.bridge(H, W)
        g = got.view(torch.int16).cpu().numpy().view(np.uint16).reshape(T, -1)
        # fp32 accumulation then one bf16 rounding, against the exact product:
        # within half a bf16 ulp plus the recursive-summation bound
        # dm * 2^-24 * sum |H||W| (the oracle itself is within half an ulp)
        a = synth.bf16_bits_to_f32(g).astype(np.float64)
        hf = synth.bf16_bits_to_f32(H).astype(np.float64)
        wf = synth.bf16_bits_to_f32(W).astype(np.float64)
        exact = hf @ wf
        half_ulp = np.spacing(np.abs(exact).astype(np.float32)).astype(np.float64) * 2.0 ** 15
        bound = half_ulp * 2 + dm * 2.0 ** -24 * (np.abs(hf) @ np.abs(wf))
        assert np.all(np.abs(a - exact) <= bound)
        assert np.mean(g == want) > 0.99


@pytest.mark.parametrize("T,dm,Hkv", [(300, 256, 2), (1000, 2048, 4), (130, 128, 1)])
def test_bridge_fp8_matches_oracle(hs2, orc, T, dm, Hkv):
    """Bridge-only prefill into the FP8 cache against the oracle.  An element
    is ambiguous when its exact product lies within the fp32 summation bound
    dm * 2^-24 * sum|h||w| of a bf16 rounding boundary: there the GPU's bf16
    K/V may differ from the oracle's by one ulp.  Scales are bit-exact wherever
    the row pair's largest element is unambiguous; codes are bit-exact (a zero
    code with either sign) except at ambiguous elements, which stay within one
    e4m3 step, as do all decoded values."""
    import torch
    H = rand_bf16((T, dm))
    Wk, Wv = rand_bf16((dm, Hkv * 128), dm ** -0.5), rand_bf16((dm, Hkv * 128), dm ** -0.5)
    H[min(5, T - 1)] = 0                                   # an all-zero row: scale 1
    Kc = torch.empty(T, Hkv, 128, dtype=torch.uint8, device="cuda")
    Vc = torch.empty_like(Kc)
    S = torch.empty(T, Hkv, dtype=torch.float32, device="cuda")
    shape = hs2.Shape.make(T, Hkv, Hkv)
    hs2.hs2_bridge_kv_fp8(dev_bf16(H), dev_bf16(Wk), dev_bf16(Wv), Kc, Vc, S, shape)
    assert hs2.hs2_get_device_status() == hs2.OK
    Kc_o, Vc_o, S_o, K_o, V_o = orc.bridge_fp8(H, Wk, Wv, Hkv)
    hf = synth.bf16_bits_to_f32(H).astype(np.float64)
    amb, mag = [], []
    for W, Xo in ((Wk, K_o), (Wv, V_o)):
        wf = synth.bf16_bits_to_f32(W).astype(np.float64)
        exact = (hf @ wf).reshape(T, Hkv, 128)
        bound = (dm * 2.0 ** -24 * (np.abs(hf) @ np.abs(wf))).reshape(T, Hkv, 128)
        xo = synth.bf16_bits_to_f32(Xo).astype(np.float64)
        half_ulp = np.spacing(np.abs(xo).astype(np.float32)).astype(np.float64) * 2.0 ** 15
        amb.append(half_ulp - np.abs(exact - xo) <= bound)
        mag.append(np.abs(xo))
    amax = np.maximum(mag[0].max(axis=2), mag[1].max(axis=2))
    top_amb = ((mag[0] == amax[..., None]) & amb[0]).any(axis=2) | \
              ((mag[1] == amax[..., None]) & amb[1]).any(axis=2)
    Sg, Kg, Vg = S.cpu().numpy(), Kc.cpu().numpy(), Vc.cpu().numpy()
    assert np.array_equal(Sg[~top_amb], S_o[~top_amb])
    same_s = Sg == S_o
    assert same_s.mean() > 0.99
    tab = orc.e4m3_table()
    for g_codes, o_codes, a in ((Kg, Kc_o, amb[0]), (Vg, Vc_o, amb[1])):
        same = (g_codes == o_codes) | (((g_codes | o_codes) & 0x7F) == 0)
        assert same[same_s & ~a.any(axis=2)].all()            # rows with no ambiguity
        assert not (~same & ~a & same_s[..., None]).any()     # elsewhere only ambiguous ones
        assert same.mean() > 0.99                             # and those seldom differ
        dg = tab[g_codes] * Sg[..., None]
        do = tab[o_codes] * S_o[..., None]
        step = np.maximum(np.abs(do), np.abs(dg)) * 2.0 ** -3 + S_o[..., None] * 2.0 ** -9
        assert np.all(np.abs(dg - do) <= step)
    assert np.all(Sg[min(5, T - 1)] == 1.0)


@pytest.mark.parametrize("T,Hq,Hkv", [(2048, 4, 1), (1000, 16, 2), (333, 2, 1), (700, 16, 1),
                                      (130, 4, 4)])
def test_full_attn_matches_oracle(hs2, orc, T, Hq, Hkv):
    import torch
    Q, K, V = rand_bf16((T, Hq, 128)), rand_bf16((T, Hkv, 128)), rand_bf16((T, Hkv, 128))
    O = torch.empty(T, Hq, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(T, Hq, dtype=torch.float32, device="cuda")
    shape = hs2.Shape.make(T, Hq, Hkv)
    hs2.hs2_full_attn_lse(dev_bf16(Q), dev_bf16(K), dev_bf16(V), O, lse, shape)
    assert hs2.hs2_get_device_status() == hs2.OK
    rows = np.arange(T)
    Oo, lo = orc.full_attn(orc.KV(K, V), Q, rows, 1 / math.sqrt(128))
    assert_close_bf16(host_f64(O), Oo, "O")
    assert np.max(np.abs(lse.cpu().numpy() - lo)) <= LSE_ABS


@pytest.mark.parametrize("T,Hq,Hkv,k,w", [(2048, 4, 1, 1024, 128), (500, 16, 2, 64, 16),
                                          (300, 8, 1, 0, 128), (2600, 8, 1, 2048, 256)])
def test_sparse_attn_on_oracle_lists(hs2, orc, T, Hq, Hkv, k, w):
    import torch
    Q, K, V = rand_bf16((T, Hq, 128)), rand_bf16((T, Hkv, 128)), rand_bf16((T, Hkv, 128))
    Qs = rand_bf16((T, Hq, 128))
    kv, sc = orc.KV(K, V), 1 / math.sqrt(128)
    rows = np.arange(T)
    _, lse = orc.full_attn(kv, Q, rows, sc)
    idx, _ = orc.select(kv, Q, rows, sc, lse, k, w)
    O = torch.empty(T, Hq, 128, dtype=torch.bfloat16, device="cuda")
    lse_s = torch.empty(T, Hq, dtype=torch.float32, device="cuda")
    shape = hs2.Shape.make(T, Hq, Hkv, k_global=k, window=w)
    hs2.hs2_sparse_attn(dev_bf16(Qs), dev_bf16(K), dev_bf16(V), dev(idx), O, lse_s, shape)
    assert hs2.hs2_get_device_status() == hs2.OK
    Oo, lo = orc.sparse_attn(kv, Qs, idx, sc)
    assert_close_bf16(host_f64(O), Oo, "O_sparse")
    assert np.max(np.abs(lse_s.cpu().numpy() - lo)) <= LSE_ABS


@pytest.mark.parametrize("T,Hq,Hkv,k,w,L", [(1500, 16, 2, 1024, 128, 3), (700, 4, 1, 64, 16, 2),
                                            (900, 32, 4, 100, 32, 4), (500, 32, 2, 64, 64, 3)])
def test_sparse_layers_fused_on_oracle_lists(hs2, orc, T, Hq, Hkv, k, w, L):
    """Several sparse layers in one pass over the gathered rows: each layer's
    output against the oracle's sparse attention with that layer's queries
    (G <= 8 fuses up to three layers per pass, G = 16 none; four layers mix
    a fused pass with a single one)."""
    import torch
    Q, K, V = rand_bf16((T, Hq, 128)), rand_bf16((T, Hkv, 128)), rand_bf16((T, Hkv, 128))
    Qs = [rand_bf16((T, Hq, 128)) for _ in range(L)]
    kv, sc = orc.KV(K, V), 1 / math.sqrt(128)
    rows = np.arange(T)
    _, lse = orc.full_attn(kv, Q, rows, sc)
    idx, _ = orc.select(kv, Q, rows, sc, lse, k, w)
    Os = [torch.empty(T, Hq, 128, dtype=torch.bfloat16, device="cuda") for _ in range(L)]
    lses = [torch.empty(T, Hq, dtype=torch.float32, device="cuda") for _ in range(L)]
    lses[-1] = None                                        # lse is optional per layer
    shape = hs2.Shape.make(T, Hq, Hkv, k_global=k, window=w)
    hs2.hs2_sparse_attn_layers([dev_bf16(q) for q in Qs], dev_bf16(K), dev_bf16(V), dev(idx), Os,
                               lses, shape)
    assert hs2.hs2_get_device_status() == hs2.OK
    for l in range(L):
        Oo, lo = orc.sparse_attn(kv, Qs[l], idx, sc)
        assert_close_bf16(host_f64(Os[l]), Oo, f"O_sparse[{l}]")
        if lses[l] is not None:
            assert np.max(np.abs(lses[l].cpu().numpy() - lo)) <= LSE_ABS


@pytest.mark.parametrize("T,Hq,Hkv,k,w", [(2048, 4, 1, 1024, 128), (1500, 16, 2, 64, 16),
                                          (900, 2, 1, 100, 32), (700, 16, 1, 32, 128),
                                          (333, 8, 1, 1024, 128), (1200, 4, 2, 0, 128),
                                          (3000, 8, 1, 2048, 256)])
def test_select_matches_oracle(hs2, orc, T, Hq, Hkv, k, w):
    import torch
    from helpers import check_index_lists
    Q, K, V = rand_bf16((T, Hq, 128)), rand_bf16((T, Hkv, 128)), rand_bf16((T, Hkv, 128))
    # planted identical key rows: exact score ties, resolved by smaller position
    K[[p for p in (5, 77, 300, 301, 640) if p < T], 0] = K[3, 0]
    kv, sc = orc.KV(K, V), 1 / math.sqrt(128)
    rows = np.arange(T)
    _, lse = orc.full_attn(kv, Q, rows, sc)
    idx_o, kth_o = orc.select(kv, Q, rows, sc, lse, k, w)
    shape = hs2.Shape.make(T, Hq, Hkv, k_global=k, window=w)
    ws = torch.empty(max(16, hs2.workspace_size(hs2.OP_SELECT, shape)), dtype=torch.uint8,
                     device="cuda")
    idx = torch.full((T, Hkv, k + w), -7, dtype=torch.int32, device="cuda")
    kth = torch.empty(T, Hkv, dtype=torch.float32, device="cuda")
    hs2.hs2_select_topk(dev_bf16(Q), dev_bf16(K), dev(lse.astype(np.float32)), idx, kth, shape, ws)
    assert hs2.hs2_get_device_status() == hs2.OK
    gi, gk = idx.cpu().numpy(), kth.cpu().numpy()
    n_diff = check_index_lists(gi, idx_o, kth_o, rows, k, w,
                               lambda r, g, js: orc.scores(kv, Q[r], g, sc, lse[r], js))
    assert n_diff <= 0.01 * T * Hkv
    sel = ~np.isnan(kth_o)
    assert np.all(gk[~sel] == -1.0)
    if sel.any():
        np.testing.assert_allclose(gk[sel], kth_o[sel], rtol=1e-4)
