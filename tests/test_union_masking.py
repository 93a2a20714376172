"""The masking argument of the planned sparse path, checked in fp32 numpy on
the CPU (no kernel involved): attending the union of several queries' lists
in 128-row chunks, with a row's logits of rows it does not list lowered by
2^e (2^e * scale * log2 e in [2^13, 2^14)) and the online base-2 softmax with
a lazily raised max (rescale only when the max grows by more than 2^3), gives
each query exactly the softmax over its own list: unlisted rows get
probability 0 even when they lead a chunk or come before the query's first
listed row.  Compared with the oracle's sparse attention on the same lists."""
import math

import numpy as np
import pytest

import synth

F32 = np.float32


def mask_bias(scale):
    # the power of two 2^e with 2^e * scale * log2(e) in [2^13, 2^14)
    c = scale / math.log(2)
    e = 0
    while math.ldexp(c, e) < 8192.0:
        e += 1
    while math.ldexp(c, e) >= 16384.0:
        e -= 1
    return math.ldexp(1.0, e)


def union_attention(q, K, V, lists, scale):
    """q [P, d] (one head per query here), K/V [T, d] fp32; lists: P lists of
    positions.  Returns O [P, d] in fp32 by the chunked masked online softmax."""
    union = sorted(set(j for l in lists for j in l))
    member = np.array([[j in set(l) for l in lists] for j in union])  # [U, P]
    B = F32(mask_bias(scale))
    c = F32(scale / math.log(2))
    P, d = q.shape
    m = np.full(P, -np.inf, F32)
    lsum = np.zeros(P, F32)
    acc = np.zeros((P, d), F32)
    for c0 in range(0, max(1, len(union)), 128):
        rows = union[c0:c0 + 128]
        mem = member[c0:c0 + 128]
        s = (K[rows] @ q.T).astype(F32)                       # [n, P] logits
        s = (s - np.where(mem, F32(0), B)).astype(F32)        # the mask step of the MMA
        x = (s * c).astype(F32)
        m_new = x.max(0)
        raise_ = m_new > m + F32(8)
        with np.errstate(over="ignore"):  # the branch not taken may overflow
            alpha = np.where(raise_, np.exp2((m - m_new).astype(F32)), F32(1)).astype(F32)
        m = np.where(raise_, m_new, m).astype(F32)
        p = np.exp2((x - m).astype(F32)).astype(F32)
        lsum = (lsum * alpha + p.sum(0)).astype(F32)
        acc = (acc * alpha[:, None] + p.T @ V[rows]).astype(F32)
    nonempty = np.array([len(l) > 0 for l in lists])
    out = np.where(nonempty[:, None], acc / np.where(lsum > 0, lsum, 1)[:, None], 0)
    return out.astype(F32)


@pytest.mark.parametrize("scale", [1 / math.sqrt(128), 1.0, 0.01])
def test_masked_union_softmax_equals_per_list_softmax(orc, scale):
    rng = np.random.default_rng(7)
    T, d, P = 700, 128, 16
    K = synth.f64_to_bf16_bits(rng.standard_normal((T, 1, d)))
    V = synth.f64_to_bf16_bits(rng.standard_normal((T, 1, d)))
    Q = synth.f64_to_bf16_bits(rng.standard_normal((P, 1, d)))
    # a key whose logit for query 1 is very large, listed by query 0 only: for
    # query 1 it leads its chunk and must still get probability 0
    K[10, 0] = synth.f64_to_bf16_bits(8.0 * synth.bf16_bits_to_f32(Q[1, 0]).astype(np.float64))
    Kf = synth.bf16_bits_to_f32(K)[:, 0]
    Vf = synth.bf16_bits_to_f32(V)[:, 0]
    Qf = synth.bf16_bits_to_f32(Q)[:, 0]
    # lists: overlapping random sets without row 10 except query 0's; query 3
    # lists only late rows (its first chunks are all masked); query 5 nothing
    lists = []
    for qq in range(P):
        n = int(rng.integers(40, 200))
        lists.append(sorted(j for j in rng.choice(T, n, replace=False).tolist() if j != 10))
    lists[0] = sorted(set(lists[0]) | {10})
    lists[3] = list(range(650, 700))
    lists[5] = []
    got = union_attention(Qf, Kf, Vf, lists, scale)
    kw = max(len(l) for l in lists)
    idx = np.full((P, 1, kw), -1, np.int32)
    for qq, l in enumerate(lists):
        idx[qq, 0, :len(l)] = l
    want, _ = orc.sparse_attn(orc.KV(K, V), Q, idx, scale)
    want = want[:, 0]
    assert np.all(np.isfinite(got))
    assert np.all(got[5] == 0.0)
    err = np.abs(got - want).max()
    assert err < 2e-5, f"max abs err {err:.2e}"
