"""The mask kernel's threshold search, restated on the host: a bitwise search
for the need-th largest order-preserving key that stops as soon as exactly
`need` keys lie at or above the candidate, followed by "keep keys above T and
the lowest-index keys equal to T".  Checked against a plain sort-based top-k
(score descending, index ascending) on random keys with many ties, and
against the full 32-step search, so that the early exit cannot change a
selection."""
import numpy as np


def order_keys(x):
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return np.where(u & 0x80000000, (~u) & 0xFFFFFFFF, u | 0x80000000).astype(np.uint64)


def search(keys, need, early_exit):
    T, steps = 0, 0
    for bit in range(31, -1, -1):
        cand = T | (1 << bit)
        steps += 1
        tot = int((keys >= cand).sum())
        if tot >= need:
            T = cand
            if early_exit and tot == need:
                break
    take_eq = need - int((keys > T).sum())
    kept = np.flatnonzero(keys > T).tolist()
    eq = np.flatnonzero(keys == T)[:take_eq].tolist()
    return sorted(kept + eq), steps


def reference(scores, need):
    order = sorted(range(len(scores)), key=lambda j: (-scores[j], j))
    return sorted(order[:need])


def test_early_exit_search_selects_the_top_k_with_lowest_index_ties():
    r = np.random.default_rng(7)
    total_steps = 0
    for trial in range(400):
        n = int(r.integers(2, 700))
        levels = r.choice([3, 17, 1000, 10 ** 6])
        scores = (r.integers(-levels, levels, n) / levels * r.choice([0.01, 1.0, 300.0])).astype(np.float32)
        need = int(r.integers(1, n + 1))
        keys = order_keys(scores)
        got, steps = search(keys, need, True)
        full, _ = search(keys, need, False)
        assert got == full == reference(scores.tolist(), need), (trial, n, need)
        total_steps += steps
    assert total_steps < 400 * 32                      # it does stop early on typical rows
