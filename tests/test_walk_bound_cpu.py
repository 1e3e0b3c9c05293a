"""The bound the pruned Markov walk rests on, checked on the CPU.

For every vocabulary entry v and previous token p, |w2[v] . w1[p]| <=
|w2[v]| * max_p |w1[p]| (Cauchy-Schwarz), so at a draft position with logits U
the entry argmax_v (U[v] + w2[v] . w1[p]) satisfies
U[v] + B |w2[v]| >= max_u (U[u] - B |w2[u]|) for every p. The kernels keep the
entries that pass this test (with a slack of 1e-3 + 1e-3 |T| and norms inflated
by 1e-4): this checks, over many previous tokens and logit scales, that the
winner under fp32 arithmetic always passes, and that the list is short when the
bias is small next to the spread of U.
"""
import numpy as np
import pytest


def _bf16(x):
    b = np.asarray(x, dtype=np.float32).view(np.uint32)
    r = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16          # round to nearest even
    return r.astype(np.uint32).view(np.float32)


def _candidates(U, w1, w2):
    n2 = (np.sqrt((w2 * w2).sum(1, dtype=np.float32)) * np.float32(1 + 1e-4)).astype(np.float32)
    B = np.float32(np.sqrt((w1 * w1).sum(1, dtype=np.float32)).max() * np.float32(1 + 1e-4))
    T = np.max(U - B * n2)
    thr = T - (np.float32(1e-3) + np.float32(1e-3) * abs(T))
    return set(np.nonzero(U + B * n2 >= thr)[0].tolist())


@pytest.mark.parametrize("u_scale,bias_scale,seed", [(1.0, 0.02, 0), (1.0, 1.0, 1), (0.05, 1.0, 2), (3.0, 5.0, 3)])
def test_winner_always_in_candidates(u_scale, bias_scale, seed):
    rng = np.random.default_rng(seed)
    V, r = 2048, 64
    w1 = _bf16(rng.normal(0, 0.02 * bias_scale ** 0.5 * 10, (V, r)))
    w2 = _bf16(rng.normal(0, 0.02 * bias_scale ** 0.5 * 10, (V, r)))
    for trial in range(4):
        U = (rng.normal(0, u_scale, V)).astype(np.float32)
        U[rng.integers(V)] = U.max()                       # an exact tie in U
        cand = _candidates(U, w1, w2)
        for p in rng.integers(0, V, 64):
            val = U + (w2 @ w1[p]).astype(np.float32)      # fp32 values of the full walk
            best = np.flatnonzero(val == val.max()).min()  # lowest index on ties
            assert best in cand, (trial, int(p))
            exact = np.argmax(U.astype(np.float64) + w2.astype(np.float64) @ w1[p].astype(np.float64))
            assert exact in cand


def test_short_lists_when_the_bias_is_small():
    rng = np.random.default_rng(7)
    V, r = 8192, 64
    w1 = _bf16(rng.normal(0, 0.02, (V, r)))
    w2 = _bf16(rng.normal(0, 0.02, (V, r)))
    U = rng.normal(0, 1.0, V).astype(np.float32)
    assert len(_candidates(U, w1, w2)) <= 8


def test_winner_at_the_edge_of_the_bound():
    """The winner's logit is far below the top one and its bias is exactly the
    bound B |w2[v*]| (w2[v*] parallel to the longest w1 row): it passes only
    because the bound charges every entry its own |w2[v]| times max_p |w1[p]|."""
    V, r = 512, 64
    w1 = np.zeros((V, r), np.float32)
    w2 = np.zeros((V, r), np.float32)
    w1[:, 1] = 0.5                                   # every previous token: norm 0.5 ...
    w1[7] = 0.0
    w1[7, 0] = 1.0                                   # ... but token 7, norm 1 (= B)
    vstar = 300
    w2[vstar, 0] = 0.75                              # bias(v*, 7) = 0.75 = B |w2[v*]|
    U = np.zeros(V, np.float32)
    U[0] = 1.0
    U[vstar] = np.float32(0.25 + 1e-4)
    val = U + (w2 @ w1[7]).astype(np.float32)
    assert int(np.argmax(val)) == vstar              # 1.0001 beats 1.0
    assert vstar in _candidates(U, w1, w2)
