"""Pins for the fp64 oracle: each test checks the oracle against something other
than itself -- hand-derived fixtures, closed forms, brute force on tiny inputs,
invariants of softmax attention and the rolling-window recurrence of
FlashDecoder's Algorithm 1.  None of these needs a GPU."""
import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import (RollingWindow, block_mask, block_ranges, block_scores, block_sparse_attention,
                    from_tile_order, pool_blocks, rope, select_blocks, tile_order, to_tile_order,
                    window_blocks, window_rope)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _window(chunks_k, chunks_v=None, W=None):
    w = RollingWindow(W or len(chunks_k))
    for n, kc in enumerate(chunks_k):
        vc = kc if chunks_v is None else chunks_v[n]
        w.append(kc, vc)
    return w


# ---------------------------------------------------------------- blocks ----
@pytest.mark.parametrize("Lc,blk,nb,last", [
    (256, 64, 4, 64),        # tiny: 16x16 frame
    (4680, 128, 37, 72),     # 480P chunk: 3 x 30 x 52
    (18720, 128, 147, 32),   # 1K chunk: 3 x 60 x 104
    (42120, 128, 330, 8),    # 2K chunk: 3 x 90 x 156
    (3600, 128, 29, 16),     # GQA decoder frame: 45 x 80
])
def test_block_counts(Lc, blk, nb, last):
    r = block_ranges(Lc, blk)
    assert len(r) == nb
    assert r[-1][1] - r[-1][0] == last
    assert r[0] == (0, blk)
    # contiguous, non-overlapping, covering
    assert all(a[1] == b[0] for a, b in zip(r, r[1:])) and r[-1][1] == Lc


def test_window_blocks_logical_order():
    wb = window_blocks(3, 10, 4)   # 3 blocks per chunk: 4,4,2
    assert len(wb) == 9
    assert wb[0] == (0, 0, 4) and wb[2] == (0, 8, 10) and wb[3] == (1, 0, 4) and wb[8] == (2, 8, 10)


# --------------------------------------------------------------- pooling ----
def test_pool_arithmetic_sequence_closed_form():
    # token t holds value t in every channel -> block mean = (start + stop - 1) / 2,
    # including the partial last block (divides by its true token count)
    Lc, blk = 37, 8
    x = np.broadcast_to(np.arange(Lc, dtype=np.float64)[None, :, None, None], (2, Lc, 3, 5)).copy()
    p = pool_blocks(x, blk)
    for n, (s, e) in enumerate(block_ranges(Lc, blk)):
        assert np.all(p[:, :, n, :] == (s + e - 1) / 2.0)
    assert p[0, 0, -1, 0] == (32 + 36) / 2.0   # last block holds 5 tokens, not 8


def test_pool_constant_blocks():
    x = rng.standard_normal((1, 3, 2, 4))
    x = np.repeat(x, 7, axis=1)  # 21 tokens, each original token repeated 7x
    p = pool_blocks(x, 7)
    assert np.allclose(p[0, :, :, :], np.transpose(x[0, ::7], (1, 0, 2)))


# ----------------------------------------------------------- golden mask ----
def test_golden_mask_small():
    g = json.load(open(os.path.join(GOLDEN, "mask_small.json")))
    q = np.array(g["q"], dtype=np.float64)[None, :, None, :]
    ks = [np.array(c, dtype=np.float64)[None, :, None, :] for c in g["k_chunks"]]
    w = _window(ks)
    for k_str, want in g["idx"].items():
        r = block_mask(q, w, g["blk"], int(k_str))
        assert np.array_equal(r["qpool"][0, 0], np.array(g["qpool"]))
        assert np.array_equal(r["kpool"][0, 0], np.array(g["kpool"]))
        assert np.allclose(r["scores"][0, 0], np.array(g["scores"]), rtol=0, atol=1e-15)
        assert r["idx"][0, 0].tolist() == want, k_str


# ---------------------------------------------------------- top-k pins ------
def _bruteforce_select(row, k, d):
    """Among all k-subsets containing d, the one with the largest score sum,
    ties broken by the smallest index sum (that is the (score desc, index asc)
    rule: a max-sum subset holds every block above the boundary value plus the
    lowest-index blocks at it)."""
    others = [j for j in range(len(row)) if j != d]
    best, best_key = None, None
    for sub in itertools.combinations(others, k - 1):
        key = (math.fsum(row[j] for j in sub), -sum(sub))
        if best_key is None or key > best_key:
            best, best_key = sub, key
    return sorted(list(best) + [d])


@pytest.mark.parametrize("seed", range(6))
def test_topk_bruteforce_distinct(seed):
    r = np.random.default_rng(seed)
    B, H, NQ, NKV, k = 1, 2, 4, 8, 4
    scores = r.standard_normal((B, H, NQ, NKV))
    diag = [4 + i for i in range(NQ)]
    idx, cnt, _ = select_blocks(scores, k, diag)
    assert np.all(cnt == k)
    for h in range(H):
        for i in range(NQ):
            assert idx[0, h, i].tolist() == _bruteforce_select(scores[0, h, i], k, diag[i])


@pytest.mark.parametrize("seed", range(6))
def test_topk_bruteforce_ties(seed):
    # integer-valued scores -> many exact ties; brute force fixes the tie rule
    r = np.random.default_rng(100 + seed)
    scores = r.integers(-2, 3, size=(1, 1, 3, 9)).astype(np.float64)
    diag = [6, 7, 8]
    for k in (1, 2, 3, 5, 9):
        idx, _, _ = select_blocks(scores, k, diag)
        for i in range(3):
            assert idx[0, 0, i].tolist() == _bruteforce_select(scores[0, 0, i], k, diag[i])


def test_topk_diagonal_forced_even_when_worst():
    scores = np.zeros((1, 1, 2, 6))
    scores[0, 0, :, :] = [5, 4, 3, 2, 1, 0]
    scores[0, 0, 0, 3] = -100.0      # diagonal of row 0 is the worst block
    scores[0, 0, 1, 4] = -100.0
    idx, _, _ = select_blocks(scores, 3, [3, 4])
    assert idx[0, 0, 0].tolist() == [0, 1, 3]
    assert idx[0, 0, 1].tolist() == [0, 1, 4]


def test_topk_boundary_scores():
    scores = np.array([[[[0.9, 0.1, 0.5, 0.7, 0.3]]]])
    idx, _, bnd = select_blocks(scores, 3, [4])
    assert idx[0, 0, 0].tolist() == [0, 3, 4]
    assert bnd[0, 0, 0, 0] == 0.7 and bnd[0, 0, 0, 1] == 0.5


def test_density_one_keeps_all_blocks():
    r = np.random.default_rng(7)
    scores = r.standard_normal((1, 3, 5, 10))
    idx, cnt, bnd = select_blocks(scores, 10, [5, 6, 7, 8, 9])
    assert np.all(idx == np.arange(10)) and np.all(cnt == 10)
    assert np.all(np.isnan(bnd[..., 1]))
    idx2, cnt2, _ = select_blocks(scores, 50, [5, 6, 7, 8, 9])   # k clamped to NKV
    assert np.array_equal(idx, idx2) and np.all(cnt2 == 10)


# ------------------------------------------------ local-band pins ----------
def _bruteforce_select_forced(row, k, forced):
    """Among all k-subsets containing every forced block, the one with the
    largest score sum, ties broken by the smallest index sum."""
    others = [j for j in range(len(row)) if j not in forced]
    best, best_key = (), None
    for sub in itertools.combinations(others, k - len(forced)):
        key = (math.fsum(row[j] for j in sub), -sum(sub))
        if best_key is None or key > best_key:
            best, best_key = sub, key
    return sorted(list(best) + list(forced))


@pytest.mark.parametrize("seed", range(4))
def test_local_band_bruteforce(seed):
    # band [d - local, d + local] clipped to the window, then the best others
    r = np.random.default_rng(200 + seed)
    NQ, NKV = 4, 10
    scores = r.standard_normal((1, 2, NQ, NKV))
    diag = [6 + i for i in range(NQ)]
    for local in (1, 2):
        for k in (2 * local + 1, 2 * local + 2, 2 * local + 3, 8):
            idx, cnt, _ = select_blocks(scores, k, diag, local=local)
            assert np.all(cnt == k)
            for h in range(2):
                for i in range(NQ):
                    band = [j for j in range(NKV) if abs(j - diag[i]) <= local]
                    want = _bruteforce_select_forced(scores[0, h, i], k, band)
                    assert idx[0, h, i].tolist() == want, (local, k, i)


def test_local_only_is_the_clipped_band():
    scores = np.random.default_rng(5).standard_normal((1, 1, 4, 10))
    idx, cnt, bnd = select_blocks(scores, 7, [6, 7, 8, 9], local=2, local_only=True)
    assert cnt[0, 0].tolist() == [5, 5, 4, 3]            # the last rows run past the window
    assert idx[0, 0, 0].tolist() == [4, 5, 6, 7, 8, -1, -1]
    assert idx[0, 0, 3].tolist() == [7, 8, 9, -1, -1, -1, -1]
    assert np.all(np.isnan(bnd))                          # no scored block, no boundary


def test_local_band_wider_than_window_keeps_everything():
    scores = np.random.default_rng(6).standard_normal((1, 1, 2, 6))
    idx, cnt, _ = select_blocks(scores, 11, [4, 5], local=5)
    assert np.all(cnt == 6) and np.all(idx == np.arange(6))


def test_local_band_must_fit_in_k():
    scores = np.zeros((1, 1, 1, 8))
    with pytest.raises(ValueError):
        select_blocks(scores, 4, [7], local=2)


def test_local_band_with_ties_prefers_low_index():
    # all scores equal: after the band, the lowest-index blocks are taken
    scores = np.zeros((1, 1, 1, 12))
    idx, _, _ = select_blocks(scores, 5, [9], local=1)
    assert idx[0, 0, 0].tolist() == [0, 1, 8, 9, 10]


def test_mask_known_argmax_one_hot_offsets():
    # every key block of the older chunk points along its own axis e_j, the query
    # block i points along e_{(3*i) % 8}; the best non-diagonal block is therefore
    # the one whose axis matches, far above the noise
    Lc, blk, D = 32, 4, 16
    nb = Lc // blk
    q = np.zeros((1, Lc, 1, D))
    k_old = np.zeros((1, Lc, 1, D))
    k_new = 1e-3 * np.random.default_rng(3).standard_normal((1, Lc, 1, D))
    for j in range(nb):
        k_old[0, j * blk:(j + 1) * blk, 0, j] = 10.0
    for i in range(nb):
        q[0, i * blk:(i + 1) * blk, 0, (3 * i) % 8] = 1.0
    w = _window([k_old, k_new])
    r = block_mask(q, w, blk, k=2)
    for i in range(nb):
        assert r["idx"][0, 0, i].tolist() == sorted([(3 * i) % 8, nb + i])


def test_block_scores_gqa_head_mapping():
    # KV head g holds constant (g+1) * e_0; query head h must see group h // (H/G)
    B, H, G, D = 1, 6, 3, 4
    qpool = np.zeros((B, H, 1, D)); qpool[..., 0] = 1.0
    kpool = np.zeros((B, G, 2, D))
    for g in range(G):
        kpool[0, g, :, 0] = g + 1
    s = block_scores(qpool, kpool, 0.5)
    for h in range(H):
        assert np.all(s[0, h] == 0.5 * (h // 2 + 1))


# ------------------------------------------------------- attention pins -----
def test_golden_attention_small():
    g = json.load(open(os.path.join(GOLDEN, "attention_small.json")))
    q = np.array(g["q"], dtype=np.float64)[None, :, None, :]
    k = np.array(g["k"], dtype=np.float64)[None, :, None, :]
    v = np.array(g["v"], dtype=np.float64)[None, :, None, :]
    w = RollingWindow(1)
    w.append(k, v)
    O, LSE = block_sparse_attention(q, w, g["blk"])
    assert np.allclose(O[0, :, 0, :], np.array(g["O"]), rtol=0, atol=1e-14)
    assert np.allclose(LSE[0, 0], np.array(g["LSE"]), rtol=0, atol=1e-14)


def _explicit_mask_attention(q, kchunks, vchunks, blk, idx, scale):
    """Brute force in pure Python: an explicit Lq x Lkv token mask built token by
    token from the kept block set, then a dense masked softmax with math.exp."""
    B, Lc, H, D = q.shape
    G = kchunks[0].shape[2]
    nb = -(-Lc // blk)
    n = len(kchunks)
    O = np.zeros((B, Lc, H, D))
    LSE = np.zeros((B, H, Lc))
    for b in range(B):
        for h in range(H):
            g = h // (H // G)
            for t in range(Lc):
                i = t // blk
                allowed = set(int(j) for j in idx[b, h, i])
                logits, vals = [], []
                for c in range(n):
                    for u in range(Lc):
                        if c * nb + u // blk not in allowed:
                            continue
                        kk = kchunks[c][b, u, g]
                        logits.append(scale * math.fsum(float(q[b, t, h, d]) * float(kk[d]) for d in range(D)))
                        vals.append(vchunks[c][b, u, g])
                m = max(logits)
                ws = [math.exp(x - m) for x in logits]
                l = math.fsum(ws)
                for d in range(D):
                    O[b, t, h, d] = math.fsum(w_ * v_[d] for w_, v_ in zip(ws, vals)) / l
                LSE[b, h, t] = m + math.log(l)
    return O, LSE


@pytest.mark.parametrize("seed", range(3))
def test_attention_vs_explicit_token_mask(seed):
    r = np.random.default_rng(50 + seed)
    B, H, G, D, Lc, blk, W, k = 1, 4, 2, 8, 22, 8, 2, 3   # 3 blocks per chunk, last of 6 tokens
    q = r.standard_normal((B, Lc, H, D))
    ks = [r.standard_normal((B, Lc, G, D)) for _ in range(W)]
    vs = [r.standard_normal((B, Lc, G, D)) for _ in range(W)]
    w = _window(ks, vs)
    m = block_mask(q, w, blk, k)
    O, LSE = block_sparse_attention(q, w, blk, m["idx"], m["cnt"])
    O2, LSE2 = _explicit_mask_attention(q, ks, vs, blk, m["idx"], 1.0 / math.sqrt(D))
    assert np.allclose(O, O2, rtol=0, atol=1e-12)
    assert np.allclose(LSE, LSE2, rtol=0, atol=1e-12)


def test_attention_weights_are_a_masked_distribution():
    # V = identity over window tokens -> O row = attention weights: rows sum to 1,
    # weights are >= 0 and exactly zero on tokens of dropped blocks
    Lc, blk, D = 12, 4, 24          # D = window tokens
    r = np.random.default_rng(9)
    q = r.standard_normal((1, Lc, 1, D))
    ks = [r.standard_normal((1, Lc, 1, D)) for _ in range(2)]
    eye = np.eye(2 * Lc)
    vs = [eye[c * Lc:(c + 1) * Lc][None, :, None, :] for c in range(2)]
    w = _window(ks, vs)
    m = block_mask(q, w, blk, 2)
    O, _ = block_sparse_attention(q, w, blk, m["idx"], m["cnt"])
    assert np.allclose(O[0, :, 0, :].sum(axis=1), 1.0, atol=1e-14)
    assert np.all(O >= 0)
    for t in range(Lc):
        kept = set(int(j) for j in m["idx"][0, 0, t // blk])
        for u in range(2 * Lc):
            j = (u // Lc) * 3 + (u % Lc) // blk
            if j not in kept:
                assert O[0, t, 0, u] == 0.0


def test_lse_independent_recompute():
    r = np.random.default_rng(11)
    Lc, blk, D = 16, 8, 8
    q = r.standard_normal((1, Lc, 2, D))
    ks = [r.standard_normal((1, Lc, 1, D)) for _ in range(2)]
    w = _window(ks)
    m = block_mask(q, w, blk, 2)
    _, LSE = block_sparse_attention(q, w, blk, m["idx"], m["cnt"])
    kall = np.concatenate(ks, axis=1)
    for h in range(2):
        for t in range(Lc):
            toks = [u for u in range(2 * Lc) if (u // Lc) * 2 + (u % Lc) // blk in set(m["idx"][0, h, t // blk].tolist())]
            ref = math.log(math.fsum(math.exp(float(q[0, t, h] @ kall[0, u, 0]) / math.sqrt(D)) for u in toks))
            assert abs(LSE[0, h, t] - ref) < 1e-12


def test_constant_keys_closed_form():
    # identical keys -> uniform weights: O = mean of V over kept tokens and
    # LSE = scale * q.k + ln(#kept tokens)
    r = np.random.default_rng(12)
    Lc, blk, D = 10, 4, 8            # blocks 4,4,2 per chunk
    kvec = r.standard_normal(D)
    ks = [np.broadcast_to(kvec, (1, Lc, 1, D)).copy() for _ in range(2)]
    vs = [r.standard_normal((1, Lc, 1, D)) for _ in range(2)]
    q = r.standard_normal((1, Lc, 1, D))
    w = _window(ks, vs)
    idx = np.array([[[[0, 2, 3], [1, 4, 5], [0, 5, 2]]]], dtype=np.int32)
    O, LSE = block_sparse_attention(q, w, blk, idx)
    vall = np.concatenate(vs, axis=1)[0, :, 0, :]
    sizes = [4, 4, 2, 4, 4, 2]
    starts = [0, 4, 8, 10, 14, 18]
    for i in range(3):
        toks = np.concatenate([np.arange(starts[j], starts[j] + sizes[j]) for j in idx[0, 0, i]])
        for t in range(i * blk, min((i + 1) * blk, Lc)):
            assert np.allclose(O[0, t, 0], vall[toks].mean(axis=0), atol=1e-13)
            want = float(q[0, t, 0] @ kvec) / math.sqrt(D) + math.log(len(toks))
            assert abs(LSE[0, 0, t] - want) < 1e-12


def test_single_kept_token_returns_its_value():
    # window of one chunk with one 1-token block kept -> O = that token's v, LSE = s
    r = np.random.default_rng(13)
    Lc, blk, D = 3, 1, 4
    q = r.standard_normal((1, Lc, 1, D)); k = r.standard_normal((1, Lc, 1, D)); v = r.standard_normal((1, Lc, 1, D))
    w = RollingWindow(1); w.append(k, v)
    idx = np.array([[[[2], [0], [1]]]], dtype=np.int32)
    O, LSE = block_sparse_attention(q, w, blk, idx)
    for t, j in enumerate([2, 0, 1]):
        assert np.allclose(O[0, t, 0], v[0, j, 0], atol=1e-15)
        assert abs(LSE[0, 0, t] - float(q[0, t, 0] @ k[0, j, 0]) / 2.0) < 1e-14


def test_order_of_kept_blocks_is_irrelevant():
    r = np.random.default_rng(14)
    Lc, blk, D = 16, 4, 8
    q = r.standard_normal((1, Lc, 2, D))
    ks = [r.standard_normal((1, Lc, 2, D)) for _ in range(2)]
    vs = [r.standard_normal((1, Lc, 2, D)) for _ in range(2)]
    w = _window(ks, vs)
    m = block_mask(q, w, blk, 3)
    O1, L1 = block_sparse_attention(q, w, blk, m["idx"], m["cnt"])
    shuffled = m["idx"][..., ::-1].copy()
    O2, L2 = block_sparse_attention(q, w, blk, shuffled, m["cnt"])
    assert np.allclose(O1, O2, atol=1e-13) and np.allclose(L1, L2, atol=1e-13)


def test_dense_equals_textbook_window_attention():
    # density 1.0 -> plain softmax(q K^T / sqrt(D)) V over all window tokens
    r = np.random.default_rng(15)
    B, H, G, D, Lc, blk = 2, 4, 2, 16, 19, 8
    q = r.standard_normal((B, Lc, H, D))
    ks = [r.standard_normal((B, Lc, G, D)) for _ in range(3)]
    vs = [r.standard_normal((B, Lc, G, D)) for _ in range(3)]
    w = _window(ks, vs)
    O, LSE = block_sparse_attention(q, w, blk)
    K = np.concatenate(ks, axis=1); V = np.concatenate(vs, axis=1)
    for b in range(B):
        for h in range(H):
            s = q[b, :, h, :] @ K[b, :, h * G // H, :].T / math.sqrt(D)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            ref = (p / p.sum(axis=1, keepdims=True)) @ V[b, :, h * G // H, :]
            assert np.allclose(O[b, :, h, :], ref, atol=1e-12)
            lse = np.log(np.exp(s).sum(axis=1))
            assert np.allclose(LSE[b, h], lse, atol=1e-12)


def test_dense_mask_and_dense_attention_agree():
    r = np.random.default_rng(16)
    Lc, blk, D = 20, 8, 8
    q = r.standard_normal((1, Lc, 2, D))
    ks = [r.standard_normal((1, Lc, 2, D)) for _ in range(2)]
    w = _window(ks)
    m = block_mask(q, w, blk, 6)           # 6 = all blocks of the window
    O1, L1 = block_sparse_attention(q, w, blk, m["idx"], m["cnt"])
    O2, L2 = block_sparse_attention(q, w, blk)
    assert np.allclose(O1, O2, atol=1e-14) and np.allclose(L1, L2, atol=1e-14)


def test_items_subset_matches_full():
    r = np.random.default_rng(17)
    Lc, blk, D = 24, 8, 8
    q = r.standard_normal((1, Lc, 2, D))
    ks = [r.standard_normal((1, Lc, 2, D)) for _ in range(2)]
    w = _window(ks)
    m = block_mask(q, w, blk, 2)
    O, L = block_sparse_attention(q, w, blk, m["idx"], m["cnt"])
    O2, L2 = block_sparse_attention(q, w, blk, m["idx"], m["cnt"], items=[(0, 1, 2), (0, 0, 0)])
    assert np.array_equal(O2[0, 16:24, 1], O[0, 16:24, 1]) and np.array_equal(O2[0, 0:8, 0], O[0, 0:8, 0])
    assert np.isnan(O2[0, 8:16]).all()


# ---------------------------------------------------------- rolling window --
def test_window_matches_algorithm1_tail_concat():
    # FlashDecoder Algorithm 1: per frame t the backbone sees the tail (W-1)*L
    # tokens of the stored cache followed by frame t's own K; the stored cache
    # becomes concat(tail_{(W-1)L}(cache), K_t).  Replayed token by token.
    W, L, D = 2, 5, 3
    r = np.random.default_rng(20)
    frames = [r.standard_normal((1, L, 1, D)) for _ in range(16)]
    w = RollingWindow(W)
    cache = np.zeros((1, 0, 1, D))
    sizes = []
    for t, f in enumerate(frames):
        seen = np.concatenate([cache[:, max(0, cache.shape[1] - (W - 1) * L):], f], axis=1)
        cache = np.concatenate([cache[:, max(0, cache.shape[1] - (W - 1) * L):], f], axis=1)
        w.append(f, f)
        assert np.array_equal(np.concatenate(w.k, axis=1), seen), t
        sizes.append(sum(x.shape[1] for x in w.k))
    assert sizes[W - 1:] == [W * L] * (16 - W + 1)   # constant footprint once full


def test_window_replace_newest_and_crop():
    a, b, c, d = (np.full((1, 2, 1, 1), float(x)) for x in range(4))
    w = RollingWindow(3)
    w.append(a, a); w.append(b, b)
    w.append(c, c, replace_newest=True)          # recompute of the newest chunk
    assert [x[0, 0, 0, 0] for x in w.k] == [0.0, 2.0]
    w.append(d, d)
    assert [x[0, 0, 0, 0] for x in w.k] == [0.0, 2.0, 3.0]
    w.append(a, a, keep_chunks=2)                  # crop the window to 2 chunks
    assert [x[0, 0, 0, 0] for x in w.k] == [3.0, 0.0]
    w.append(b, b, keep_chunks=1)
    assert [x[0, 0, 0, 0] for x in w.k] == [1.0]
    with pytest.raises(ValueError):
        RollingWindow(2).append(a, a, replace_newest=True)
    with pytest.raises(ValueError):
        w.append(a, a, keep_chunks=4)


def test_first_chunk_window_is_own_chunk_only():
    # before the window fills, attention covers only the chunks seen so far and
    # the diagonal is the newest chunk's block
    r = np.random.default_rng(21)
    Lc, blk, D = 8, 4, 4
    q = r.standard_normal((1, Lc, 1, D))
    k0 = r.standard_normal((1, Lc, 1, D))
    w = RollingWindow(3)
    w.append(k0, k0)
    m = block_mask(q, w, blk, 5)
    assert m["idx"].shape[-1] == 2 and np.all(m["cnt"] == 2)
    assert m["scores"].shape[-1] == 2


# ------------------------------------------------------------ RoPE pins ------

def test_rope_position_zero_is_identity():
    x = np.random.default_rng(1).standard_normal((2, 3, 4, 16))
    assert np.array_equal(rope(x, np.zeros(3, dtype=np.int64)), x)


def test_rope_is_complex_multiplication_per_pair():
    # RoFormer's complex form: (x_2i + i x_2i+1) * exp(i * pos * theta_i)
    r = np.random.default_rng(2)
    D, L = 8, 6
    x = r.standard_normal((1, L, 1, D))
    pos = np.array([0, 1, 7, 100, 12345, 987654])
    y = rope(x, pos, base=500.0)
    z = x[..., 0::2] + 1j * x[..., 1::2]
    ang = np.outer(pos, [math.pow(500.0, -2.0 * i / D) for i in range(D // 2)])
    w = z * np.exp(1j * ang)[None, :, None, :]
    assert np.allclose(y[..., 0::2], w.real, atol=1e-9) and np.allclose(y[..., 1::2], w.imag, atol=1e-9)


def test_rope_frequencies_form_the_roformer_ladder():
    # rotate unit vectors by position 1 and read each pair's angle back
    D, base = 16, 10000.0
    x = np.zeros((1, 1, D // 2, D))
    for i in range(D // 2):
        x[0, 0, i, 2 * i] = 1.0
    y = rope(x, np.array([1]), base)
    ang = np.array([math.atan2(y[0, 0, i, 2 * i + 1], y[0, 0, i, 2 * i]) for i in range(D // 2)])
    assert abs(ang[0] - 1.0) < 1e-15                                  # theta_0 = 1 rad per position
    ratio = ang[1:] / ang[:-1]
    assert np.allclose(ratio, base ** (-2.0 / D), rtol=1e-12)         # geometric in the pair index
    assert abs(ang[-1] - base ** (-(D - 2) / D)) < 1e-15


def test_rope_scores_depend_on_position_difference_only():
    r = np.random.default_rng(3)
    q, k = r.standard_normal((1, 1, 1, 32)), r.standard_normal((1, 1, 1, 32))
    for m, n, c in [(5, 2, 100), (0, 17, 4096), (300, 300, 7)]:
        a = float(np.sum(rope(q, [m]) * rope(k, [n])))
        b = float(np.sum(rope(q, [m + c]) * rope(k, [n + c])))
        d = float(np.sum(q * rope(k, [n - m])))                       # only the difference rotates
        assert abs(a - b) < 1e-9 and abs(a - d) < 1e-9


def _shifted_window(q, w, Lc, shift, base=10000.0):
    out = RollingWindow(w.W)
    for c in range(w.n_valid):
        out.append(rope(w.k[c], shift + c * Lc + np.arange(Lc), base), w.v[c])
    return rope(q, shift + (w.n_valid - 1) * Lc + np.arange(Lc), base), out


def test_window_relative_rope_equals_any_common_shift():
    # window-relative positions give the same pooled scores, masks and attention
    # as positions shifted by any constant (e.g. absolute stream positions)
    r = np.random.default_rng(4)
    Lc, blk, D = 40, 8, 16
    w = RollingWindow(3)
    for _ in range(3):
        w.append(r.standard_normal((1, Lc, 1, D)), r.standard_normal((1, Lc, 1, D)))
    q = r.standard_normal((1, Lc, 2, D))
    qa, wa = window_rope(q, w)
    qb, wb = _shifted_window(q, w, Lc, shift=3 * 10 ** 6 + 17)
    ma, mb = block_mask(qa, wa, blk, 4), block_mask(qb, wb, blk, 4)
    assert np.allclose(ma["scores"], mb["scores"], atol=1e-9)
    assert np.array_equal(ma["idx"], mb["idx"])
    Oa, La = block_sparse_attention(qa, wa, blk, ma["idx"], ma["cnt"])
    Ob, Lb = block_sparse_attention(qb, wb, blk, ma["idx"], ma["cnt"])
    assert np.allclose(Oa, Ob, atol=1e-9) and np.allclose(La, Lb, atol=1e-9)


def test_window_rope_positions_follow_the_window():
    # after the window slides, chunk c of the window is rotated by c * Lc + r
    r = np.random.default_rng(5)
    Lc, D = 6, 4
    w = RollingWindow(2)
    chunks = [r.standard_normal((1, Lc, 1, D)) for _ in range(3)]
    for ch in chunks:
        w.append(ch, ch)
    q = r.standard_normal((1, Lc, 1, D))
    qr, wr = window_rope(q, w)
    assert np.allclose(wr.k[0], rope(chunks[1], np.arange(Lc)))
    assert np.allclose(wr.k[1], rope(chunks[2], Lc + np.arange(Lc)))
    assert np.allclose(qr, rope(q, Lc + np.arange(Lc)))
    assert np.array_equal(wr.v[1], chunks[2])


def test_round_bf16_matches_torch_on_float32_values():
    # from float32 values, torch's bf16 conversion (nearest even) is a single
    # rounding, so it must agree exactly with the direct fp64 -> bf16 rounding
    import torch
    from oracle import round_bf16
    r = np.random.default_rng(8)
    x = (r.standard_normal(20000) * np.exp2(r.integers(-20, 20, 20000))).astype(np.float32)
    ties = np.array([1.00390625, 1.01171875, -3.0078125, 257.0, 259.0], dtype=np.float32)   # exact halfway cases
    x = np.concatenate([x, ties])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(round_bf16(x.astype(np.float64)), want)
    assert round_bf16(np.array([1.00390625]))[0] == 1.0 and round_bf16(np.array([1.01171875]))[0] == 1.015625


def test_window_rope_shift_and_rounding():
    from oracle import round_bf16
    r = np.random.default_rng(9)
    Lc, D = 8, 16
    w = RollingWindow(2)
    for _ in range(2):
        w.append(r.standard_normal((1, Lc, 1, D)), r.standard_normal((1, Lc, 1, D)))
    q = r.standard_normal((1, Lc, 1, D))
    qs, ws = window_rope(q, w, shift=5 * Lc, to_bf16=True)
    assert np.array_equal(ws.k[1], round_bf16(rope(w.k[1], 6 * Lc + np.arange(Lc))))
    assert np.array_equal(qs, round_bf16(rope(q, 6 * Lc + np.arange(Lc))))


# ---------------------------------------------------------- anchor pins ------
def _chunks(n, Lc=4, D=2):
    return [np.full((1, Lc, 1, D), float(t)) for t in range(n)]


def test_anchor_window_keeps_the_anchor_and_the_newest():
    # HiStream's anchor-guided window: the anchor plus the W - 1 newest chunks
    w = RollingWindow(3)
    ch = _chunks(6)
    w.append(ch[0], ch[0], anchor=True)
    for t in range(1, 6):
        w.append(ch[t], ch[t])
    assert [c[0, 0, 0, 0] for c in w.k] == [0.0, 4.0, 5.0]
    w.append(ch[1], ch[1], keep_chunks=2)                        # crop: the anchor stays
    assert [c[0, 0, 0, 0] for c in w.k] == [0.0, 1.0]
    w.append(ch[3], ch[3], keep_chunks=2, replace_newest=True)    # replace the newest, not the anchor
    assert [c[0, 0, 0, 0] for c in w.k] == [0.0, 3.0]


def test_anchor_alone_is_the_newest_chunk():
    w = RollingWindow(2)
    a, b = _chunks(2)
    w.append(a, a, anchor=True)
    w.append(b, b, replace_newest=True)                           # only the anchor: it is replaced
    assert w.n_valid == 1 and w.k[0][0, 0, 0, 0] == 1.0 and w.anchored


@pytest.mark.parametrize("bad", [dict(W=1), dict(nonempty=True), dict(replace=True)])
def test_anchor_rejections(bad):
    w = RollingWindow(bad.get("W", 3))
    a = _chunks(1)[0]
    if bad.get("nonempty"):
        w.append(a, a)
    with pytest.raises(ValueError):
        w.append(a, a, anchor=True, replace_newest=bad.get("replace", False))


def test_anchor_keep_must_leave_room():
    w = RollingWindow(3)
    a = _chunks(1)[0]
    w.append(a, a, anchor=True)
    with pytest.raises(ValueError):
        w.append(a, a, keep_chunks=1)


def test_dense_attention_over_anchored_window_is_plain_softmax():
    # dense attention over the anchored window equals a softmax over the
    # explicit concatenation anchor | recent chunks
    r = np.random.default_rng(12)
    Lc, blk, D = 12, 4, 8
    w = RollingWindow(3)
    ks = [r.standard_normal((1, Lc, 1, D)) for _ in range(5)]
    vs = [r.standard_normal((1, Lc, 1, D)) for _ in range(5)]
    w.append(ks[0], vs[0], anchor=True)
    for t in range(1, 5):
        w.append(ks[t], vs[t])
    q = r.standard_normal((1, Lc, 1, D))
    O, L = block_sparse_attention(q, w, blk)
    K = np.concatenate([ks[0], ks[3], ks[4]], axis=1)[0, :, 0]
    V = np.concatenate([vs[0], vs[3], vs[4]], axis=1)[0, :, 0]
    s = q[0, :, 0] @ K.T / math.sqrt(D)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    assert np.allclose(O[0, :, 0], (p @ V) / p.sum(axis=1, keepdims=True), atol=1e-12)
    assert np.allclose(L[0, 0], np.log(np.exp(s).sum(axis=1)), atol=1e-12)


# ---------------------------------------------------------- tile order pins --

def test_tile_order_worked_example():
    # a 2 x 2 x 4 grid with (1, 2, 2) tiles, written out by hand:
    # frame 0: rows [0 1 2 3], [4 5 6 7]; frame 1: rows [8 9 10 11], [12 13 14 15]
    want = [0, 1, 4, 5, 2, 3, 6, 7, 8, 9, 12, 13, 10, 11, 14, 15]
    assert tile_order(2, 2, 4, (1, 2, 2)).tolist() == want


def test_tile_order_clipped_edges_worked_example():
    # 1 x 3 x 3 grid, (1, 2, 2) tiles: tiles (0,0) {0,1,3,4}, (0,1) {2,5}, (1,0) {6,7}, (1,1) {8}
    assert tile_order(1, 3, 3, (1, 2, 2)).tolist() == [0, 1, 3, 4, 2, 5, 6, 7, 8]


@pytest.mark.parametrize("grid", [(3, 60, 104), (3, 30, 52), (1, 45, 80), (4, 16, 16), (3, 90, 156)])
def test_tile_order_is_a_permutation_with_full_interior_tiles(grid):
    T, Hg, Wg = grid
    o = tile_order(T, Hg, Wg)
    assert np.array_equal(np.sort(o), np.arange(T * Hg * Wg))
    t, rem = np.divmod(o, Hg * Wg)
    y, x = np.divmod(rem, Wg)
    tile_id = (t // 2) * (-(-Hg // 8)) * (-(-Wg // 8)) + (y // 8) * (-(-Wg // 8)) + x // 8
    assert np.all(np.diff(tile_id) >= 0)                   # tiles are contiguous runs, in tile order
    # every full (2, 8, 8) tile is one run of 128 tokens spanning exactly 2 x 8 x 8
    ids, starts, counts = np.unique(tile_id, return_index=True, return_counts=True)
    full = counts == 128
    for s0 in starts[full][:50]:
        seg = slice(s0, s0 + 128)
        assert np.ptp(t[seg]) == 1 and np.ptp(y[seg]) == 7 and np.ptp(x[seg]) == 7
    if T % 2 == 0 and Hg % 8 == 0 and Wg % 8 == 0:
        assert np.all(full)


def test_tile_order_round_trip():
    r = np.random.default_rng(13)
    o = tile_order(3, 10, 12, (2, 4, 4))
    x = r.standard_normal((2, 360, 3, 4))
    y = to_tile_order(x, o)
    assert np.array_equal(from_tile_order(y, o), x)
    assert np.array_equal(y[:, 5], x[:, o[5]])


# ------------------------------------------------------------- FP8 pins ------
def test_quantize_e4m3_matches_torch_float8():
    import torch
    from oracle import quantize_e4m3
    r = np.random.default_rng(14)
    x = (r.standard_normal(50000) * np.exp2(r.integers(-12, 8, 50000))).astype(np.float32)
    x = x[np.abs(x) <= 448]
    halfway = np.array([1.0625, 1.1875, -3.125, 2.0 ** -9 * 1.5, 2.0 ** -9 * 0.5, 240.0, 416.0], dtype=np.float32)
    x = np.concatenate([x, halfway])
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(quantize_e4m3(x.astype(np.float64), 1.0), want)
    assert quantize_e4m3(np.array([1.0625, 1.1875]), 1.0).tolist() == [1.0, 1.25]    # ties to even


def test_quantize_e4m3_scaled_quotient_is_exact():
    # power-of-two scales make x / scale exact in fp32 as well, so torch's
    # float8 cast of the fp32 quotient is the reference there
    import torch
    from oracle import quantize_e4m3
    r = np.random.default_rng(16)
    x = (r.standard_normal(50000) * 3.0).astype(np.float32)
    for scale in (2.0 ** -7, 2.0 ** -3, 0.5, 4.0):
        want = (torch.from_numpy(x) / scale).clamp(-448, 448).to(torch.float8_e4m3fn).to(torch.float64).numpy()
        assert np.array_equal(quantize_e4m3(x, scale), want)


def test_quantize_e4m3_rounds_the_exact_quotient_not_an_fp32_product():
    # x = 175/512 and scale = 7/64 (both exact in bf16): x / scale = 25/8 =
    # 3.125 exactly, the midpoint between the e4m3 values 3.0 (mantissa 100)
    # and 3.25 (mantissa 101); ties to even give 3.0.  The fp32 reciprocal of
    # 7/64 rounds up (64/7 = 9.142857142..., fp32 9.1428575516), so the fp32
    # product x * fp32(1 / scale) = 3.1250002384 lies above the midpoint and
    # would round to 3.25: an oracle that formed the quotient that way fails.
    from oracle import quantize_e4m3
    x, scale = 175.0 / 512.0, 7.0 / 64.0
    assert quantize_e4m3(np.array([x, -x]), scale).tolist() == [3.0, -3.0]
    inv32 = np.float32(1.0) / np.float32(scale)
    assert float(np.float32(x) * inv32) > 3.125        # the fp32 product passes the midpoint
    # just off the midpoint either way the nearest value wins
    assert quantize_e4m3(np.array([3.125 * (1 + 2 ** -20), 3.125 * (1 - 2 ** -20)]), 1.0).tolist() == [3.25, 3.0]


def test_e4m3_near_boundary_rule_of_the_gpu_comparison():
    # the code comparison of the FP8 parity tests accepts a different code only
    # next to an e4m3 rounding boundary, and only a neighbouring code
    from uf_testlib import e4m3_codes_agree
    x = np.array([175.0 / 512.0, 175.0 / 512.0, 175.0 / 512.0, 0.3, 0.3])
    got = np.array([3.0, 3.25, 3.5, 2.75, 2.5])       # 0.3 / (7/64) = 2.742857 -> 2.75
    near, bad = e4m3_codes_agree(got, x, 7.0 / 64.0)
    assert near == 1 and bad.tolist() == [False, False, True, False, True]


def test_quantize_e4m3_saturates_and_scales():
    from oracle import quantize_e4m3
    assert quantize_e4m3(np.array([1000.0, -1e9, 449.0]), 1.0).tolist() == [448.0, -448.0, 448.0]
    assert quantize_e4m3(np.array([3.0]), 0.5)[0] == 6.0                              # in units of the scale


def test_fp8_scores_attention_is_exact_on_the_e4m3_grid():
    # queries and keys already on the scaled e4m3 grid: nothing to round, so the
    # FP8-score attention is the plain one
    from oracle import fp8_scores_attention, quantize_e4m3
    r = np.random.default_rng(15)
    Lc, blk, D, qs, ks = 16, 8, 16, 0.01, 0.02
    w = RollingWindow(2)
    for _ in range(2):
        w.append(quantize_e4m3(r.standard_normal((1, Lc, 1, D)), ks) * ks, r.standard_normal((1, Lc, 1, D)))
    q = quantize_e4m3(r.standard_normal((1, Lc, 2, D)), qs) * qs
    O1, L1 = block_sparse_attention(q, w, blk)
    O2, L2 = fp8_scores_attention(q, w, blk, qs, ks)
    assert np.allclose(O1, O2, atol=1e-12) and np.allclose(L1, L2, atol=1e-12)
