"""Device-side guards of the library on a real GPU: index-list entries
outside [-1, T) are skipped and reported instead of read.  The buffers are
allocated with spare rows on both sides of the T rows the shape names, so
that even a broken guard would read memory this test owns."""
import math

import numpy as np
import pytest

import synth
from helpers import assert_close_bf16, dev, dev_bf16, host_f64

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
