"""Shared helpers of the GPU parity tests: moving seeded inputs to the device,
and the tolerances of the block (bf16 outputs: max-abs <= 2e-2 and relative
L2 <= 5e-3; index sets identical except tokens whose oracle score lies within
1e-4 relative of the oracle's k-th score)."""
import math

import numpy as np

MAX_ABS = 2e-2
REL_L2 = 5e-3
LSE_ABS = 2e-4
SEL_REL = 1e-4


def dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def assert_close_bf16(got, want, what=""):
    """got: GPU result as fp64 array; want: oracle fp64."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - want)
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3e} > {MAX_ABS}"
    assert rel <= REL_L2, f"{what}: rel L2 err {rel:.3e} > {REL_L2}"
    return err.max(), rel


def check_index_lists(gpu_idx, orc_idx, kth, rows, k, w, score_fn):
    """Compare GPU and oracle index lists row by row.

    gpu_idx, orc_idx: [n, Hkv, k+w]; kth: oracle k-th score [n, Hkv] (NaN when
    all candidates are selected); score_fn(r, g, js) -> oracle scores.
    Windows must be identical; global parts identical except positions whose
    oracle score is within SEL_REL of the oracle's k-th score.  Returns the
    number of (row, head) lists that differ (all within tolerance)."""
    n_diff = 0
    for r, i in enumerate(rows):
        for g in range(gpu_idx.shape[1]):
            a, b = gpu_idx[r, g], orc_idx[r, g]
            assert np.array_equal(a[k:], b[k:]), f"window differs at row {i} head {g}"
            ga = a[:k][a[:k] >= 0]
            gb = b[:k][b[:k] >= 0]
            assert np.all(a[:k][len(ga):] == -1), f"padding not at the tail, row {i}"
            assert np.all(np.diff(ga) > 0), f"globals not ascending/unique at row {i} head {g}"
            assert len(ga) == len(gb), f"selected count differs at row {i} head {g}"
            if np.array_equal(ga, gb):
                continue
            n_diff += 1
            tau = kth[r, g]
            assert not math.isnan(tau), f"row {i} head {g}: sets differ with nothing to rank"
            sym = np.array(sorted(set(ga.tolist()) ^ set(gb.tolist())), np.int64)
            s = score_fn(r, g, sym)
            bad = np.abs(s - tau) > SEL_REL * tau
            assert not bad.any(), (f"row {i} head {g}: positions {sym[bad][:8]} differ with "
                                   f"scores {s[bad][:8]} vs k-th {tau}")
    return n_diff


def compare_rows(orc, cfg, kv, Qr, Qsr, rows, got, k=None, w=None):
    """Compare the GPU block's outputs on `rows` with the oracle.

    Qr [n, Hq, d] and Qsr (list of [n, Hq, d]) are the rows' query bits;
    got holds the GPU tensors (O, lse, idx, O_sparse) for all rows.  Sparse
    outputs are compared with the oracle on its own lists where the GPU list is
    identical, and on the GPU's list (validated by check_index_lists) where it
    differs.  Returns the number of (row, KV head) lists that differ."""
    import torch
    k = cfg.k_global if k is None else k
    w = cfg.window if w is None else w
    sc = cfg.scale
    ridx = torch.from_numpy(np.asarray(rows)).to(got["O"].device)
    ref = orc.block_rows(kv, Qr, Qsr, rows, sc, k, w)
    assert_close_bf16(host_f64(got["O"][ridx]), ref["O"], "O_full")
    assert np.max(np.abs(got["lse"][ridx].cpu().numpy() - ref["lse"])) <= LSE_ABS
    gi = got["idx"][ridx].cpu().numpy()
    n_diff = check_index_lists(gi, ref["idx"], ref["kth"], rows, k, w,
                               lambda r, g, js: orc.scores(kv, Qr[r], g, sc, ref["lse"][r], js))
    same = np.all(gi == ref["idx"], axis=(1, 2))
    for l, q in enumerate(Qsr):
        gs = host_f64(got["O_sparse"][l][ridx])
        if same.any():
            assert_close_bf16(gs[same], ref["O_sparse"][l][same], f"O_sparse[{l}]")
        if (~same).any():
            o_gpu_list, _ = orc.sparse_attn(kv, q[~same], gi[~same], sc)
            assert_close_bf16(gs[~same], o_gpu_list, f"O_sparse[{l}] on GPU lists")
    return n_diff


def edge_rows(T, k=1024, w=128, n_random=0, seed=0):
    base = [0, 1, w - 1, w, w + 1, k + w - 2, k + w - 1, k + w, k + w + 1, T // 2, T - 2, T - 1]
    rows = set(r for r in base if 0 <= r < T)
    if n_random:
        rng = np.random.default_rng(seed)
        rows |= set(rng.integers(0, T, n_random).tolist())
    return np.array(sorted(rows), np.int64)


def bits(t):
    """bf16 tensor -> uint16 numpy bits (host)."""
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)
