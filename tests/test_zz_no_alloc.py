"""hs2_select_topk_noalloc: the selection for callers that cannot allocate
device memory (their device memory belongs to another runtime's allocator, or
they must not call cudaMalloc on a latency-critical path).  It must return
exactly what hs2_select_topk returns with a caller-provided workspace, on two
calls in a row (its scratch keeps the previous call's contents).

This file is collected last on purpose, so a run stopping at the first failure
has run every other test before it."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,Hq,Hkv,k,w", [(3000, 32, 4, 1024, 128), (2500, 8, 2, 64, 16)])
def test_noalloc_selection_matches_workspace_selection(T, Hq, Hkv, k, w):
    import torch
    import long_context_bridge_b200 as hs2
    g = torch.Generator(device="cuda").manual_seed(T + k)
    Q = torch.randn(T, Hq, 128, device="cuda", generator=g).bfloat16()
    K = torch.randn(T, Hkv, 128, device="cuda", generator=g).bfloat16()
    V = torch.randn(T, Hkv, 128, device="cuda", generator=g).bfloat16()
    K[[7, 99, 500, 1500]] = K[3].clone()  # exact score ties
    shape = hs2.Shape.make(T, Hq, Hkv, k_global=k, window=w)
    O = torch.empty_like(Q)
    lse = torch.empty(T, Hq, dtype=torch.float32, device="cuda")
    hs2.hs2_full_attn_lse(Q, K, V, O, lse, shape)
    ws = torch.empty(hs2.workspace_size(hs2.OP_SELECT, shape), dtype=torch.uint8, device="cuda")
    idx_ref = torch.empty(T, Hkv, k + w, dtype=torch.int32, device="cuda")
    kth_ref = torch.empty(T, Hkv, dtype=torch.float32, device="cuda")
    hs2.hs2_select_topk(Q, K, lse, idx_ref, kth_ref, shape, ws)
    for call in range(2):
        idx = torch.full((T, Hkv, k + w), -9, dtype=torch.int32, device="cuda")
        kth = torch.full((T, Hkv), -9.0, dtype=torch.float32, device="cuda")
        hs2.hs2_select_topk_noalloc(Q, K, lse, idx, kth, shape)
        assert hs2.hs2_get_device_status() == hs2.OK
        # integer work: identical lists; the k-th scores are the same floats
        assert torch.equal(idx, idx_ref), f"call {call}: index lists differ"
        assert torch.equal(kth, kth_ref), f"call {call}: k-th scores differ"
