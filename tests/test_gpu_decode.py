"""GPU parity of hs2_block_decode (full attention, selection and sparse layers
over an e4m3 KV cache with per-(token, KV head) scales) against the oracle on
the dequantised cache, with ragged sequence lengths."""
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


def run_decode(hs2, orc, cfg, cap, lens, n_sparse=3):
    import torch
    B = len(lens)
    cache = synth.decode_cache_np(cfg, cap, batch=B)
    q = synth.decode_queries_np(cfg, synth.TID_Q, batch=B)
    qs = [synth.decode_queries_np(cfg, synth.TID_QS0 + l, batch=B) for l in range(n_sparse)]
    Hq, Hkv, k, w = cfg.n_q_heads, cfg.n_kv_heads, cfg.k_global, cfg.window
    shape = hs2.Shape.make(cap, Hq, Hkv, k_global=k, window=w)
    o = torch.empty(B, Hq, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    idx = torch.full((B, Hkv, k + w), -7, dtype=torch.int32, device="cuda")
    os_ = [torch.empty_like(o) for _ in range(n_sparse)]
    ws = torch.empty(hs2.workspace_size(hs2.OP_BLOCK_DECODE, shape, B), dtype=torch.uint8,
                     device="cuda")
    sc = dev(cache.scale)
    hs2.hs2_block_decode(lens, dev_bf16(q), dev(cache.Kc), dev(cache.Vc), sc, sc, o, lse, idx,
                         [dev_bf16(x) for x in qs], os_, shape, ws)
    assert hs2.hs2_get_device_status() == hs2.OK
    kvs = [orc.KV(cache.Kc[b, :lens[b]], cache.Vc[b, :lens[b]], cache.scale[b, :lens[b]],
                  cache.scale[b, :lens[b]]) for b in range(B)]
    ref = orc.decode(kvs, q, qs, cfg.scale, k, w)
    go, gl, gi = host_f64(o), lse.cpu().numpy(), idx.cpu().numpy()
    gs = [host_f64(x) for x in os_]
    n_diff = 0
    for b in range(B):
        r = ref[b]
        assert_close_bf16(go[b], r["O"][0], f"o_full[{b}]")
        assert np.max(np.abs(gl[b] - r["lse"][0])) <= LSE_ABS
        n_diff += check_index_lists(gi[b:b + 1], r["idx"], r["kth"], [lens[b] - 1], k, w,
                                    lambda rr, g, js: orc.scores(kvs[b], q[b], g, cfg.scale,
                                                                 r["lse"][0], js))
        same = np.array_equal(gi[b], r["idx"][0])
        for l in range(n_sparse):
            want = r["O_sparse"][l][0] if same else orc.sparse_attn(kvs[b], qs[l][b:b + 1],
                                                                   gi[b:b + 1], cfg.scale)[0][0]
            assert_close_bf16(gs[l][b], want, f"o_sparse[{l}][{b}]")
    return n_diff


@pytest.mark.parametrize("Hq,Hkv", [(32, 4), (16, 4), (16, 1)])
def test_decode_small_ragged(hs2, orc, Hq, Hkv):
    cfg = synth.BlockConfig("decode test", 5, 9000, Hq, Hkv, n_needles=64, q_mix=True, batch=4,
                            fp8_cache=True)
    lens = [9000, 4097, 1200, 1100]   # over a chunk, just past k + w, below k + w
    assert run_decode(hs2, orc, cfg, 9000, lens) <= 1


def test_decode_c5_shape_64k(hs2, orc):
    cfg = synth.CONFIGS["C5"]
    n = 65536
    lens = [n - 17 * b for b in range(cfg.batch)]
    assert run_decode(hs2, orc, cfg, n, lens) <= 2
