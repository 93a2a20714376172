"""Sparse attention over the union plan (hs2_sparse_plan, then
hs2_sparse_attn_planned) against the oracle's sparse attention on the same
lists.  Item = P = 256/G consecutive query rows of one KV head: the cases
cover G = 8 and 16, ragged T (a partial last item), unions of one to several
128-row chunks, lists in scrambled order, rows whose list is empty, and
entries that are out of range or repeated (reported as bad and used at most
once)."""
import math

import numpy as np
import pytest

import synth
from helpers import LSE_ABS, assert_close_bf16, dev, dev_bf16, host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hs2():
    import torch
    assert torch.cuda.is_available()
    import long_context_bridge_b200 as m
    return m


def rand_bf16(shape, seed):
    return synth.f64_to_bf16_bits(np.random.default_rng(seed).standard_normal(shape))


def run_planned(hs2, Qs, K, V, idx, T, Hq, Hkv, k, w, spare_rows=0):
    """K/V carry spare_rows rows past T, so that an entry the guard should drop
    still points into owned memory."""
    import torch
    shape = hs2.Shape.make(T, Hq, Hkv, k_global=k, window=w)
    plan = torch.empty(hs2.workspace_size(hs2.OP_SPARSE_PLAN, shape), dtype=torch.uint8,
                       device="cuda")
    Kd, Vd = dev_bf16(K), dev_bf16(V)
    if spare_rows:
        pad = torch.zeros(spare_rows, Hkv, 128, dtype=torch.bfloat16, device="cuda")
        Kd, Vd = torch.cat([Kd, pad]), torch.cat([Vd, pad])
    hs2.hs2_sparse_plan(dev(idx), shape, plan)
    O = torch.empty(T, Hq, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(T, Hq, dtype=torch.float32, device="cuda")
    hs2.hs2_sparse_attn_planned(dev_bf16(Qs), Kd, Vd, plan, O, lse, shape)
    st = hs2.hs2_get_device_status()
    return O, lse, st


@pytest.mark.parametrize("T,Hq,Hkv,k,w", [(2000, 8, 1, 1024, 128), (1337, 16, 2, 256, 64),
                                          (700, 32, 2, 64, 16), (2600, 16, 1, 2048, 256)])
def test_planned_sparse_on_oracle_lists(hs2, orc, T, Hq, Hkv, k, w):
    Q, K, V = rand_bf16((T, Hq, 128), 1), rand_bf16((T, Hkv, 128), 2), rand_bf16((T, Hkv, 128), 3)
    Qs = rand_bf16((T, Hq, 128), 4)
    kv, sc = orc.KV(K, V), 1 / math.sqrt(128)
    rows = np.arange(T)
    _, lse_f = orc.full_attn(kv, Q, rows, sc)
    idx, _ = orc.select(kv, Q, rows, sc, lse_f, k, w)
    O, lse, st = run_planned(hs2, Qs, K, V, idx, T, Hq, Hkv, k, w)
    assert st == hs2.OK
    Oo, lo = orc.sparse_attn(kv, Qs, idx, sc)
    assert_close_bf16(host_f64(O), Oo, "O_sparse (planned)")
    assert np.max(np.abs(lse.cpu().numpy() - lo)) <= LSE_ABS


def test_planned_sparse_scrambled_lists_and_empty_rows(hs2, orc):
    """The union and the masks do not depend on the order inside a list; a
    row whose list is all -1 gets O = 0 and lse = -inf exactly (as the
    per-list kernel and the oracle); an item whose every list is empty still
    writes its rows."""
    T, Hq, Hkv, k, w = 1500, 16, 2, 192, 32
    Q, K, V = rand_bf16((T, Hq, 128), 11), rand_bf16((T, Hkv, 128), 12), rand_bf16((T, Hkv, 128), 13)
    Qs = rand_bf16((T, Hq, 128), 14)
    kv, sc = orc.KV(K, V), 1 / math.sqrt(128)
    rows = np.arange(T)
    _, lse_f = orc.full_attn(kv, Q, rows, sc)
    idx, _ = orc.select(kv, Q, rows, sc, lse_f, k, w)
    rng = np.random.default_rng(5)
    for r in range(T):
        for g in range(Hkv):
            idx[r, g] = idx[r, g, rng.permutation(k + w)]
    empty = [3, 700, 701, 1499]
    idx[empty, 1] = -1
    idx[1024:1056, 0] = -1   # every list of one item (P = 32 rows) of KV head 0
    idx[1200:1216, 0] = -1   # the first of the two tiles of another item
    O, lse, st = run_planned(hs2, Qs, K, V, idx, T, Hq, Hkv, k, w)
    assert st == hs2.OK
    Oo, lo = orc.sparse_attn(kv, Qs, idx, sc)
    assert_close_bf16(host_f64(O), Oo, "O_sparse (scrambled)")
    got_l = lse.cpu().numpy()
    fin = np.isfinite(lo)
    assert np.array_equal(np.isfinite(got_l), fin)
    assert np.max(np.abs(got_l[fin] - lo[fin])) <= LSE_ABS
    G = Hq // Hkv
    Oh = host_f64(O)
    for r in empty:
        assert np.all(Oh[r, G:2 * G] == 0.0) and np.all(got_l[r, G:2 * G] == -np.inf)
    for a, b in [(1024, 1056), (1200, 1216)]:
        assert np.all(Oh[a:b, :G] == 0.0) and np.all(got_l[a:b, :G] == -np.inf)


def test_planned_sparse_bad_entries_reported_and_used_once(hs2, orc):
    """Entries at or past T and entries listed twice: the plan reports
    HS2_ERR_BAD_INDEX, drops the former and takes the latter once, so the
    output is the oracle's on the cleaned lists.  K/V carry spare rows past T,
    so no access can leave owned memory even if the guard failed."""
    T, Hq, Hkv, k, w = 900, 8, 1, 128, 32
    Q, K, V = rand_bf16((T, Hq, 128), 21), rand_bf16((T, Hkv, 128), 22), rand_bf16((T, Hkv, 128), 23)
    Qs = rand_bf16((T, Hq, 128), 24)
    kv, sc = orc.KV(K, V), 1 / math.sqrt(128)
    rows = np.arange(T)
    _, lse_f = orc.full_attn(kv, Q, rows, sc)
    idx, _ = orc.select(kv, Q, rows, sc, lse_f, k, w)
    clean = idx.copy()
    bad = idx.copy()
    bad[500, 0, 0] = T          # out of range: dropped
    bad[501, 0, 3] = T + 40     # out of range: dropped
    clean[500, 0, 0] = -1
    clean[501, 0, 3] = -1
    bad[600, 0, 5] = bad[600, 0, 6]   # listed twice: taken once
    clean[600, 0, 5] = -1
    O, lse, st = run_planned(hs2, Qs, K, V, bad, T, Hq, Hkv, k, w, spare_rows=64)
    assert st == hs2.ERR_BAD_INDEX
    Oo, lo = orc.sparse_attn(kv, Qs, clean, sc)
    assert_close_bf16(host_f64(O), Oo, "O_sparse (cleaned lists)")
    assert np.max(np.abs(lse.cpu().numpy() - lo)) <= LSE_ABS


def test_plan_path_refuses_unsupported_shapes(hs2):
    """G outside {8, 16}, or P * (k + w) above the plan's limit: no plan path
    (the block calls then use the per-list kernel)."""
    import torch
    for Hq, Hkv, k, w in [(4, 1, 64, 16), (8, 1, 2048, 256), (32, 8, 64, 16)]:
        shape = hs2.Shape.make(1024, Hq, Hkv, k_global=k, window=w)
        with pytest.raises(hs2.HS2Error):
            hs2.workspace_size(hs2.OP_SPARSE_PLAN, shape)
        idx = torch.zeros(1024, Hkv, k + w, dtype=torch.int32, device="cuda")
        plan = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
        with pytest.raises(hs2.HS2Error) as e:
            hs2.hs2_sparse_plan(idx, shape, plan)
        assert e.value.status == hs2.ERR_UNSUPPORTED
