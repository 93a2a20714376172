"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle function to a library routine (torch / numpy in
fp64), a closed form, an invariant the pages fix, or brute force on tiny
inputs.  A dropped term, wrong sign, wrong index or transposed operand in the
oracle fails at least one of them.  CPU only.
"""
import math

import numpy as np
import pytest
import torch

import synth

RNG = np.random.default_rng(1234)


def rand_bf16(shape, sd=1.0):
    return synth.f64_to_bf16_bits(RNG.standard_normal(shape) * sd)


def f(b):
    return synth.bf16_bits_to_f32(b).astype(np.float64)


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------
def test_bf16_round_matches_torch(orc):
    x = RNG.standard_normal(20000).astype(np.float32).astype(np.float64) * 37.0
    ties = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0, -0.0])
    x = np.concatenate([x, ties])
    ours = orc.bf16_round(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(ours.view(np.int16), ref)
    # ties to even: 1 + 2^-8 is halfway between 1 and 1 + 2^-7 -> 1.0
    assert ours[-5] == 0x3F80 and ours[-4] == 0x3F82


def test_e4m3_table_matches_format_and_torch(orc):
    tab = orc.e4m3_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(tab), nan)
    assert np.array_equal(tab[~nan], ref[~nan])
    assert tab[0x7E] == 448.0 and tab[0x01] == 2.0 ** -9 and tab[0x38] == 1.0
    assert math.isnan(tab[0x7F]) and math.isnan(tab[0xFF]) and tab[0xFE] == -448.0
    assert np.nanmax(tab) == 448.0


def test_synth_numpy_equals_torch_generator():
    # integer draws and uniforms agree bit for bit; fp64 log/cos may differ by
    # an ulp between libraries, which the bf16 rounding of stored values removes
    for start in (0, 12345, (1 << 33) + 7):
        a = synth.normals_np(77, 4, start, 1 << 18)
        b = synth.normals_torch(77, 4, start, 1 << 18, device="cpu").numpy()
        assert np.max(np.abs(a - b)) < 1e-14
        assert np.array_equal(synth.f64_to_bf16_bits(a), synth.f64_to_bf16_bits(b))
        bt = synth.normal_bf16_torch(77, 4, start, 1 << 18, device="cpu")
        assert np.array_equal(bt.view(torch.int16).numpy().view(np.uint16),
                              synth.normal_bf16_np(77, 4, start, 1 << 18))


def test_synth_e4m3_quantiser_matches_torch_cast():
    x = np.concatenate([np.linspace(-460, 460, 200001), RNG.standard_normal(100000) * 3,
                        RNG.standard_normal(100000) * 1e-2]).astype(np.float32)
    x = np.clip(x, -448, 448)
    ours = synth.e4m3_quantize_np(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # +-0: torch keeps the sign of zero results, the quantiser writes +0
    zero = (ref & 0x7F) == 0
    assert np.array_equal(ours[~zero], ref[~zero])
    assert np.all((ours[zero] & 0x7F) == 0)


def test_oracle_e4m3_encoder_matches_torch_cast(orc):
    # f1's rounding rule (nearest, ties to the even code, saturation, sign of
    # zero kept) against torch's float8_e4m3fn cast of values clamped to 448
    tab = orc.e4m3_table()
    pos = tab[:0x7F]
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)       # exact ties
    x = np.concatenate([np.linspace(-460, 460, 20001), RNG.standard_normal(20000) * 3,
                        RNG.standard_normal(20000) * 1e-2, pos, -pos, mids, -mids,
                        [0.0, -0.0, 1e-30, -1e-30, 449.0, -1e9]]).astype(np.float32)
    ours = orc.e4m3_encode(x)
    ref = torch.from_numpy(np.clip(x, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_bridge_fp8_is_nearest_code_of_scaled_row(orc):
    # brute force on a small case: the scale is the row pair's amax / 448 in
    # fp32 and each code is the nearest e4m3 value of x / scale (fp32 quotient)
    T, dm, Hkv = 48, 128, 2
    H = rand_bf16((T, dm))
    Wk, Wv = rand_bf16((dm, Hkv * 128), 1 / 16), rand_bf16((dm, Hkv * 128), 1 / 16)
    H[3] = 0                                               # an all-zero row: scale 1
    Kc, Vc, S, K, V = orc.bridge_fp8(H, Wk, Wv, Hkv)
    assert np.array_equal(K.reshape(T, -1), orc.bridge(H, Wk))
    kf = synth.bf16_bits_to_f32(K)
    vf = synth.bf16_bits_to_f32(V)
    amax = np.maximum(np.abs(kf).max(axis=2), np.abs(vf).max(axis=2)).astype(np.float32)
    want_s = np.where(amax > 0, amax / np.float32(448), np.float32(1)).astype(np.float32)
    assert np.array_equal(S, want_s) and np.all(S[3] == 1)
    tab = orc.e4m3_table()
    vals = tab[:0x7F]
    for codes, x in ((Kc, kf), (Vc, vf)):
        q = (x / S[:, :, None]).astype(np.float32).astype(np.float64)
        dist = np.abs(np.abs(q)[..., None] - vals)            # [T, Hkv, d, 127]
        best = dist.min(axis=-1)
        mag = codes & 0x7F
        assert np.all(np.abs(np.abs(q) - vals[mag]) == best)  # a nearest value
        tie = (dist == best[..., None]).sum(axis=-1) > 1
        assert np.all(mag[tie] % 2 == 0)                      # ties to the even code
        assert np.array_equal(codes >> 7, np.signbit(q).astype(np.uint8))
    # the largest magnitude of each row pair maps to 448
    top = np.maximum((Kc & 0x7F).max(axis=2), (Vc & 0x7F).max(axis=2))
    assert np.all(top[amax > 0] == 0x7E)


def test_bridge_fp8_rule_equals_decode_cache_recipe(orc):
    # the cache f1 writes follows the same rule as the decode workload's input
    # recipe: on the same bf16 rows, equal scales and codes (zero codes with
    # either sign: the recipe's numpy quantiser writes +0)
    T, Hkv = 64, 2
    K = rand_bf16((T * Hkv, 128))
    V = rand_bf16((T * Hkv, 128))
    Kc = np.empty((T * Hkv, 128), np.uint8)
    Vc = np.empty_like(Kc)
    S = np.empty(T * Hkv, np.float32)
    orc.lib().orc_quantize_rows(orc._p(K), orc._p(V), T * Hkv, 128, orc._p(Kc), orc._p(Vc),
                                orc._p(S))
    kf, vf = synth.bf16_bits_to_f32(K), synth.bf16_bits_to_f32(V)
    amax = np.maximum(np.abs(kf).max(axis=1), np.abs(vf).max(axis=1)).astype(np.float32)
    s_rec = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    assert np.array_equal(S, s_rec)
    for codes, x in ((Kc, kf), (Vc, vf)):
        rec = synth.e4m3_quantize_np((x / s_rec[:, None]).astype(np.float32))
        same = (codes == rec) | (((codes | rec) & 0x7F) == 0)
        assert same.all()


# --------------------------------------------------------------------------
# S1 bridge
# --------------------------------------------------------------------------
def test_bridge_within_half_ulp_of_exact(orc):
    H, W = rand_bf16((64, 256)), rand_bf16((256, 96), 1 / 16)
    out = orc.bridge(H, W)
    exact = f(H) @ f(W)
    got = f(out)
    ulp = np.spacing(np.abs(exact).astype(np.float32)).astype(np.float64) * 2.0 ** 16
    assert np.all(np.abs(got - exact) <= 0.5 * ulp * (1 + 1e-9))


def test_bridge_identity_weights(orc):
    H = rand_bf16((40, 128))
    W = np.zeros((128, 64), np.uint16)
    W[np.arange(64), np.arange(64)] = 0x3F80          # [I; 0]
    assert np.array_equal(orc.bridge(H, W), H[:, :64])


# --------------------------------------------------------------------------
# S2 full attention
# --------------------------------------------------------------------------
def _sdpa_ref(Q, K, V, scale, mask_fn):
    """torch fp64 attention of all rows; Q [T,Hq,d], K/V [T,Hkv,d] values."""
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    q = torch.from_numpy(Q).permute(1, 0, 2)
    k = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(G, 0)
    v = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(G, 0)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    allowed = mask_fn(i, j)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=allowed, scale=scale)
    logits = (q @ k.transpose(1, 2)) * scale
    lse = torch.logsumexp(logits.masked_fill(~allowed, -math.inf), dim=-1)
    return o.permute(1, 0, 2).numpy(), lse.T.numpy()


@pytest.mark.parametrize("T,Hq,Hkv", [(150, 4, 1), (97, 6, 2)])
def test_full_attn_matches_sdpa(orc, T, Hq, Hkv):
    d = 128
    Q, K, V = rand_bf16((T, Hq, d)), rand_bf16((T, Hkv, d)), rand_bf16((T, Hkv, d))
    rows = np.array([0, 1, 5, T // 2, T - 1])
    O, lse = orc.full_attn(orc.KV(K, V), Q[rows], rows, 1 / math.sqrt(d))
    Oref, lref = _sdpa_ref(f(Q), f(K), f(V), 1 / math.sqrt(d), lambda i, j: j <= i)
    np.testing.assert_allclose(O, Oref[rows], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, lref[rows], rtol=1e-12, atol=1e-12)


def test_full_attn_closed_forms(orc):
    d, Hq, T = 128, 4, 64
    Q, K, V = rand_bf16((T, Hq, d)), rand_bf16((T, 1, d)), rand_bf16((T, 1, d))
    sc = 1 / math.sqrt(d)
    # row 0 sees only key 0: o = v_0, lse = s_00
    O, lse = orc.full_attn(orc.KV(K, V), Q[:1], np.array([0]), sc)
    assert np.array_equal(O[0], np.broadcast_to(f(V[0, 0]), (Hq, d)))
    np.testing.assert_allclose(lse[0], sc * f(Q[0]) @ f(K[0, 0]), rtol=1e-14)
    # identical keys: o = mean of V[0..i], lse = s + ln(i+1)
    Kc = np.broadcast_to(K[:1], K.shape).copy()
    rows = np.array([10, 63])
    O, lse = orc.full_attn(orc.KV(Kc, V), Q[rows], rows, sc)
    for r, i in enumerate(rows):
        np.testing.assert_allclose(O[r], np.broadcast_to(f(V[:i + 1, 0]).mean(0), (Hq, d)),
                                   rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[r], sc * f(Q[i]) @ f(K[0, 0]) + math.log(i + 1), rtol=1e-13)
        assert np.all(lse[r] >= sc * f(Q[i]) @ f(K[0, 0]))


# --------------------------------------------------------------------------
# S3 scores and selection
# --------------------------------------------------------------------------
def _softmax_scores(Q, K, sc, i, g, G):
    """Brute force: torch softmax over j <= i, summed over the group's heads."""
    q = torch.from_numpy(f(Q[i, g * G:(g + 1) * G]))
    k = torch.from_numpy(f(K[:i + 1, g]))
    return torch.softmax((q @ k.T) * sc, dim=-1).sum(0).numpy()


def test_score_mass_equals_group_size(orc):
    T, Hq, Hkv, d = 300, 8, 2, 128
    Q, K, V = rand_bf16((T, Hq, d)), rand_bf16((T, Hkv, d)), rand_bf16((T, Hkv, d))
    kv, sc = orc.KV(K, V), 1 / math.sqrt(d)
    for i in (0, 127, 299):
        _, lse = orc.full_attn(kv, Q[i:i + 1], np.array([i]), sc)
        for g in range(Hkv):
            s = orc.scores(kv, Q[i], g, sc, lse[0], np.arange(i + 1))
            assert abs(s.sum() - Hq // Hkv) < 1e-12 * Hq
            np.testing.assert_allclose(s, _softmax_scores(Q, K, sc, i, g, Hq // Hkv),
                                       rtol=1e-11, atol=1e-15)


def _check_invariants(idx, rows, k, w):
    for r, i in enumerate(rows):
        for lst in idx[r]:
            glob, win = lst[:k], lst[k:]
            assert np.array_equal(win, np.where(np.arange(i - w + 1, i + 1) >= 0,
                                                np.arange(i - w + 1, i + 1), -1))
            gv = glob[glob >= 0]
            assert np.all(glob[len(gv):] == -1)           # padding at the tail
            assert np.all(np.diff(gv) > 0)                # ascending, no duplicates
            assert np.all(gv <= i - w)                    # no window or future positions
            assert len(gv) == min(k, max(0, i - w + 1))
            allv = lst[lst >= 0]
            assert len(set(allv.tolist())) == len(allv) == min(i + 1, w + min(k, max(0, i - w + 1)))


@pytest.mark.parametrize("k,w", [(16, 8), (1024, 128)])
def test_select_brute_force(orc, k, w):
    T, Hq, Hkv, d = 1400 if k == 1024 else 200, 8, 2, 128
    Q, K, V = rand_bf16((T, Hq, d)), rand_bf16((T, Hkv, d)), rand_bf16((T, Hkv, d))
    # planted identical key rows force exact score ties: the smaller position wins
    K[[3, 40, 41, 90, 150], 0] = K[7, 0]
    kv, sc, G = orc.KV(K, V), 1 / math.sqrt(d), Hq // Hkv
    rows = np.array([0, 5, w - 1, w, w + 1, k + w - 1, k + w, T - 1])
    rows = np.unique(rows[rows < T])
    _, lse = orc.full_attn(kv, Q[rows], rows, sc)
    idx, kth = orc.select(kv, Q[rows], rows, sc, lse, k, w)
    _check_invariants(idx, rows, k, w)
    for r, i in enumerate(rows):
        for g in range(Hkv):
            nc = max(0, i - w + 1)
            if nc == 0:
                continue
            s = _softmax_scores(Q, K, sc, i, g, G)[:nc]
            order = sorted(range(nc), key=lambda j: (-s[j], j))
            want = np.sort(order[:k])
            got = idx[r, g, :k][idx[r, g, :k] >= 0]
            if nc <= k:
                assert np.array_equal(got, np.arange(nc)) and math.isnan(kth[r, g])
                continue
            tau = s[order[k - 1]]
            np.testing.assert_allclose(kth[r, g], tau, rtol=1e-12)
            diff = set(got.tolist()) ^ set(want.tolist())
            assert all(abs(s[j] - tau) <= 1e-12 * tau for j in diff)


def test_select_tie_break_prefers_smaller_position(orc):
    # all keys identical: every candidate ties, so the k smallest positions win
    T, Hq, d, k, w = 100, 4, 128, 10, 8
    Q = rand_bf16((T, Hq, d))
    K = np.broadcast_to(rand_bf16((1, 1, d)), (T, 1, d)).copy()
    kv, sc = orc.KV(K, K), 1 / math.sqrt(d)
    rows = np.array([50, 99])
    _, lse = orc.full_attn(kv, Q[rows], rows, sc)
    idx, _ = orc.select(kv, Q[rows], rows, sc, lse, k, w)
    for r in range(2):
        assert np.array_equal(idx[r, 0, :k], np.arange(k))


# --------------------------------------------------------------------------
# S4 sparse attention
# --------------------------------------------------------------------------
def test_sparse_with_everything_selected_equals_full(orc):
    T, Hq, Hkv, d, k, w = 160, 8, 2, 128, 1024, 128
    Q, K, V = rand_bf16((T, Hq, d)), rand_bf16((T, Hkv, d)), rand_bf16((T, Hkv, d))
    kv, sc = orc.KV(K, V), 1 / math.sqrt(d)
    rows = np.arange(T)
    O, lse = orc.full_attn(kv, Q, rows, sc)
    idx, _ = orc.select(kv, Q, rows, sc, lse, k, w)
    Os, ls = orc.sparse_attn(kv, Q, idx, sc)
    np.testing.assert_allclose(Os, O, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(ls, lse, rtol=1e-13)


def test_sparse_with_k0_equals_sliding_window(orc):
    T, Hq, Hkv, d, w = 300, 4, 2, 128, 128
    Q, K, V = rand_bf16((T, Hq, d)), rand_bf16((T, Hkv, d)), rand_bf16((T, Hkv, d))
    kv, sc = orc.KV(K, V), 1 / math.sqrt(d)
    rows = np.arange(T)
    _, lse = orc.full_attn(kv, Q, rows, sc)
    idx, kth = orc.select(kv, Q, rows, sc, lse, 0, w)
    assert np.all(np.isnan(kth)) and np.all(idx[:, :, :0] == 0)
    Os, ls = orc.sparse_attn(kv, Q, idx, sc)
    Oref, lref = _sdpa_ref(f(Q), f(K), f(V), sc, lambda i, j: (j <= i) & (j > i - w))
    np.testing.assert_allclose(Os, Oref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(ls, lref, rtol=1e-12)


# --------------------------------------------------------------------------
# S5 FP8 decode source
# --------------------------------------------------------------------------
def test_e4m3_source_matches_dequantised_reference(orc):
    cfg = synth.CONFIGS["C5"]
    N, Hq, Hkv, d = 700, 8, 2, 128
    cache = synth.decode_cache_np(synth.BlockConfig("t", 5, N, Hq, Hkv, n_needles=16,
                                                    q_mix=True, batch=1, fp8_cache=True), N)
    tab = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    Kd = tab[cache.Kc[0]] * cache.scale[0][:, :, None].astype(np.float64)
    Vd = tab[cache.Vc[0]] * cache.scale[0][:, :, None].astype(np.float64)
    kv = orc.KV(cache.Kc[0], cache.Vc[0], cache.scale[0], cache.scale[0])
    q = rand_bf16((1, Hq, d))
    O, lse = orc.full_attn(kv, q, np.array([N - 1]), cfg.scale)
    Qf = np.zeros((N, Hq, d))
    Qf[N - 1] = f(q[0])
    Oref, lref = _sdpa_ref(Qf, Kd, Vd, cfg.scale, lambda i, j: j <= i)
    np.testing.assert_allclose(O[0], Oref[N - 1], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse[0], lref[N - 1], rtol=1e-12)
    # the round trip of the stored values is exact: codes decode to x/s rounded
    assert np.all(np.abs(Kd / cache.scale[0][:, :, None] ) <= 448)


def test_decode_equals_prefill_last_row(orc):
    T, Hq, Hkv, d = 400, 8, 2, 128
    Q, K, V = rand_bf16((T, Hq, d)), rand_bf16((T, Hkv, d)), rand_bf16((T, Hkv, d))
    Qs = rand_bf16((T, Hq, d))
    kv, sc = orc.KV(K, V), 1 / math.sqrt(d)
    full = orc.block_rows(kv, Q[[T - 1]], [Qs[[T - 1]]], np.array([T - 1]), sc, 64, 16)
    dec = orc.decode([kv], Q[[T - 1]], [Qs[[T - 1]]], sc, 64, 16)[0]
    for key in ("O", "lse", "idx"):
        assert np.array_equal(full[key], dec[key])
    assert np.array_equal(full["O_sparse"][0], dec["O_sparse"][0])


def test_synth_decode_cache_torch_matches_numpy():
    cfg = synth.BlockConfig("t", 5, 3000, 8, 2, n_needles=16, q_mix=True, batch=2, fp8_cache=True)
    a = synth.decode_cache_np(cfg, 3000)
    Kc, Vc, S = synth.decode_cache_torch(cfg, 3000, device="cpu")
    assert np.array_equal(S.numpy(), a.scale)
    # +-0 codes may differ in sign between the two quantisers
    for got, want in ((Kc.numpy(), a.Kc), (Vc.numpy(), a.Vc)):
        nz = (want & 0x7F) != 0
        assert np.array_equal(got[nz], want[nz]) and np.all((got[~nz] & 0x7F) == 0)


def test_synth_device_recipes_match_numpy():
    cfg = synth.BlockConfig("t", 3, 600, 8, 2, d_model=128, n_needles=8, q_mix=True)
    q = synth.q_rows_torch(cfg, synth.TID_Q, device="cpu", rows=128)
    assert np.array_equal(q.view(torch.int16).numpy().view(np.uint16),
                          synth.q_rows_np(cfg, synth.TID_Q, np.arange(600)))
    H, Wk, Wv = synth.bridge_inputs_torch(cfg, device="cpu")
    h2, wk2, wv2 = synth.bridge_inputs_np(cfg)
    for a, b in ((H, h2), (Wk, wk2), (Wv, wv2)):
        assert np.array_equal(a.view(torch.int16).numpy().view(np.uint16), b)
    K = synth.kv_torch(cfg, synth.TID_K, device="cpu")
    assert np.array_equal(K.view(torch.int16).numpy().view(np.uint16), synth.kv_np(cfg, synth.TID_K))
    rows, heads, vals = synth.needle_scatter_torch(cfg, device="cpu")
    Kn = synth.kv_np(cfg, synth.TID_K)
    synth.plant_needles_np(cfg, Kn, synth.prefill_needles(cfg))
    K[rows, heads] = vals
    assert np.array_equal(K.view(torch.int16).numpy().view(np.uint16), Kn)
