"""Device-side guards of the library on a real GPU: index-list entries
outside [-1, T) are skipped and reported instead of read.  The buffers are
allocated with spare rows on both sides of the T rows the shape names, so
that even a broken guard would read memory this test owns."""
import math

import numpy as np
import pytest

import synth
from helpers import assert_close_bf16, check_index_lists, dev, dev_bf16, host_f64

pytestmark = pytest.mark.gpu
RNG = np.random.default_rng(31)


@pytest.fixture(scope="module")
def hs2():
    import torch
    assert torch.cuda.is_available()
    import long_context_bridge_b200 as m
    return m


def rand_bf16(shape):
    return synth.f64_to_bf16_bits(RNG.standard_normal(shape))


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (16, 1)])
def test_sparse_attn_skips_out_of_range_entries(hs2, orc, Hq, Hkv):
    import torch
    T, k, w, pad = 600, 64, 16, 64
    Kfull, Vfull = rand_bf16((T + 2 * pad, Hkv, 128)), rand_bf16((T + 2 * pad, Hkv, 128))
    Q, Qs = rand_bf16((T, Hq, 128)), rand_bf16((T, Hq, 128))
    K, V = Kfull[pad:pad + T], Vfull[pad:pad + T]
    kv, sc = orc.KV(K, V), 1 / math.sqrt(128)
    rows = np.arange(T)
    _, lse = orc.full_attn(kv, Q, rows, sc)
    idx, _ = orc.select(kv, Q, rows, sc, lse, k, w)
    bad = idx.copy()
    # out-of-range entries in place of selected positions: past the end (still
    # inside the spare rows after K/V) and negative other than -1 (inside the
    # spare rows before them)
    planted = [(300, 0, 3, T), (300, 0, 10, T + 5), (450, Hkv - 1, 0, -3), (599, 0, k - 1, -pad),
               (599, Hkv - 1, k + 2, T + pad - 1)]
    for r, g, e, j in planted:
        bad[r, g, e] = j
    clean = bad.copy()
    for r, g, e, _ in planted:
        clean[r, g, e] = -1
    Kd_full, Vd_full = dev_bf16(Kfull), dev_bf16(Vfull)
    Kd, Vd = Kd_full[pad:pad + T], Vd_full[pad:pad + T]
    assert Kd.is_contiguous() and Vd.is_contiguous()
    shape = hs2.Shape.make(T, Hq, Hkv, k_global=k, window=w)
    O_bad = torch.empty(T, Hq, 128, dtype=torch.bfloat16, device="cuda")
    O_clean = torch.empty_like(O_bad)
    Qd = dev_bf16(Qs)
    hs2.hs2_sparse_attn(Qd, Kd, Vd, dev(bad), O_bad, None, shape)
    assert hs2.hs2_get_device_status() == hs2.ERR_BAD_INDEX
    assert hs2.hs2_get_device_status() == hs2.OK          # reading the status clears it
    hs2.hs2_sparse_attn(Qd, Kd, Vd, dev(clean), O_clean, None, shape)
    assert hs2.hs2_get_device_status() == hs2.OK
    # a skipped entry is exactly a -1 entry
    assert torch.equal(O_bad, O_clean)
    Oo, _ = orc.sparse_attn(kv, Qs, clean, sc)
    assert_close_bf16(host_f64(O_clean), Oo, "O_sparse on the cleaned lists")
    # the fused-layers entry point shares the guard
    Os = [torch.empty_like(O_bad) for _ in range(2)]
    hs2.hs2_sparse_attn_layers([Qd, Qd], Kd, Vd, dev(bad), Os, None, shape)
    assert hs2.hs2_get_device_status() == hs2.ERR_BAD_INDEX
    for x in Os:
        assert_close_bf16(host_f64(x), Oo, "fused layers on lists with bad entries")


def test_waits_that_run_out_unwind_and_report(hs2, orc):
    """With the spin budget of every bounded wait cut to one cycle, the waits
    of the TMA/tensor-core kernels run out.  Each kernel then waits (with its
    own fixed budget) for the copies and MMAs it already issued, releases its
    tensor memory and exits, and the next status read is HS2_ERR_TIMEOUT.
    With the default budget restored, the same calls in the same process
    return the oracle's results: the context is still usable."""
    import torch
    T, Hq, Hkv, k, w, dm = 1500, 8, 2, 256, 64, 256
    # the dyadic grid makes the bridge exact in fp32, so the block's K/V equal
    # the oracle's bit for bit and the oracle runs on its own K/V
    H, Wk, Wv = synth.bridge_inputs_dyadic_np(
        synth.BlockConfig("timeouts", 6, T, Hq, Hkv, d_model=dm))
    Q, Qs = rand_bf16((T, Hq, 128)), rand_bf16((T, Hq, 128))
    shape = hs2.Shape.make(T, Hq, Hkv, k_global=k, window=w)
    ws = torch.empty(hs2.workspace_size(hs2.OP_BLOCK_PREFILL, shape), dtype=torch.uint8,
                     device="cuda")
    Hd, Wkd, Wvd, Qd, Qsd = dev_bf16(H), dev_bf16(Wk), dev_bf16(Wv), dev_bf16(Q), dev_bf16(Qs)

    def block():
        K = torch.empty(T, Hkv, 128, dtype=torch.bfloat16, device="cuda")
        V = torch.empty_like(K)
        O, Os = torch.empty_like(Qd), torch.empty_like(Qd)
        lse = torch.empty(T, Hq, dtype=torch.float32, device="cuda")
        idx = torch.empty(T, Hkv, k + w, dtype=torch.int32, device="cuda")
        hs2.hs2_block_prefill(Hd, Wkd, Wvd, K, V, Qd, O, lse, idx, [Qsd], [Os], shape, ws)
        return K, V, O, lse, idx, Os

    def decode():
        cap, lens = 3000, [3000, 1700]
        Kc = torch.randint(0, 0x7E, (2, cap, Hkv, 128), dtype=torch.uint8, device="cuda")
        Vc = torch.randint(0, 0x7E, (2, cap, Hkv, 128), dtype=torch.uint8, device="cuda")
        S = torch.full((2, cap, Hkv), 1.0 / 256, dtype=torch.float32, device="cuda")
        sh = hs2.Shape.make(cap, Hq, Hkv, k_global=k, window=w)
        wsd = torch.empty(hs2.workspace_size(hs2.OP_BLOCK_DECODE, sh, 2), dtype=torch.uint8,
                          device="cuda")
        q = torch.randn(2, Hq, 128, device="cuda").bfloat16()
        o = torch.empty_like(q)
        hs2.hs2_block_decode(lens, q, Kc, Vc, S, S, o,
                             torch.empty(2, Hq, dtype=torch.float32, device="cuda"),
                             torch.empty(2, Hkv, k + w, dtype=torch.int32, device="cuda"), [q],
                             [torch.empty_like(q)], sh, wsd)

    assert hs2.hs2_get_device_status() == hs2.OK
    hs2.hs2_debug_set_wait_budget(1)
    try:
        block()
        st_block = hs2.hs2_get_device_status()
        decode()
        st_decode = hs2.hs2_get_device_status()
        K8 = torch.empty(T, Hkv, 128, dtype=torch.uint8, device="cuda")
        hs2.hs2_bridge_kv_fp8(Hd, Wkd, Wvd, K8, torch.empty_like(K8),
                              torch.empty(T, Hkv, dtype=torch.float32, device="cuda"),
                              hs2.Shape.make(T, Hkv, Hkv))
        st_f8 = hs2.hs2_get_device_status()
    finally:
        hs2.hs2_debug_set_wait_budget(0)
    assert st_block == hs2.ERR_TIMEOUT
    assert st_decode == hs2.ERR_TIMEOUT
    assert st_f8 == hs2.ERR_TIMEOUT
    assert hs2.hs2_get_device_status() == hs2.OK
    # default budget again: the same block, checked against the oracle
    K, V, O, lse, idx, Os = block()
    assert hs2.hs2_get_device_status() == hs2.OK
    Ko, Vo = orc.bridge(H, Wk).reshape(T, Hkv, 128), orc.bridge(H, Wv).reshape(T, Hkv, 128)
    assert np.array_equal(K.view(torch.int16).cpu().numpy().view(np.uint16), Ko)
    assert np.array_equal(V.view(torch.int16).cpu().numpy().view(np.uint16), Vo)
    kv = orc.KV(Ko, Vo)
    rows = np.array([0, 63, 64, 319, 320, 777, 1200, T - 1])
    ref = orc.block_rows(kv, Q[rows], [Qs[rows]], rows, 1 / math.sqrt(128), k, w)
    assert_close_bf16(host_f64(O[rows]), ref["O"], "O_full after the timeouts")
    assert np.max(np.abs(lse[rows].cpu().numpy() - ref["lse"])) <= 2e-4
    gi = idx[rows].cpu().numpy()
    check_index_lists(gi, ref["idx"], ref["kth"], rows, k, w,
                      lambda r, g, js: orc.scores(kv, Q[rows][r], g, 1 / math.sqrt(128),
                                                  ref["lse"][r], js))
    same = np.all(gi == ref["idx"], axis=(1, 2))
    assert_close_bf16(host_f64(Os[rows])[same], ref["O_sparse"][0][same], "O_sparse")
    decode()
    assert hs2.hs2_get_device_status() == hs2.OK
