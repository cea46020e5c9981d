"""Pins for the float64 oracle: facts fixed by the FOCUS pages and by mathematics,
checked without a second implementation of the oracle's own formula.

Sources: "FOCUS: DLLMs Know How to Tame Their Compute Bound" (pith.science
review page) -- "What carries the argument" (I_j as the column sum of the
block queries' softmax weights; Delta I = I(layer 1) - I(layer 0), Eq. 3;
MaxPool1D smoothing; top-K under a budget), Referee Report minor comment on
Eq. (2) (row-wise softmax), Free-Parameter Ledger (MaxPool1D k = 3, Eq. 15).

Each pin is a plain function of an ``oracle.Oracle``; ``tests/test_oracle_pins.py``
runs them on the committed oracle and ``tests/test_oracle_mutations.py`` runs them
on deliberately broken copies to show that each plausible mistake fails one.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def bf16(x) -> torch.Tensor:
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def rand_bf16(gen, shape, std=1.0):
    return (torch.randn(*shape, generator=gen) * std).to(torch.bfloat16)


def small_problem(seed, R=3, B=6, Hq=4, Hkv=2, d=8, L=(0, 5, 9), std=0.7):
    gen = torch.Generator().manual_seed(seed)
    L = np.asarray(L, np.int64)
    cu = torch.from_numpy(np.concatenate([[0], np.cumsum(L)]).astype(np.int32))
    T = int(L.sum())
    q = rand_bf16(gen, (R, B, Hq, d), std)
    kp = rand_bf16(gen, (T, Hkv, d), std)
    kb = rand_bf16(gen, (R, B, Hkv, d), std)
    return q, kp, cu, kb


def _expr(s: str) -> float:
    return float(eval(s, {"__builtins__": {}}, {"exp": math.exp, "inf": math.inf}))


# --------------------------------------------------------------------------- importance

def pin_hand_two_tokens(orc):
    """Closed-form two-token cases worked by hand (tests/golden/hand_two_tokens.json)."""
    fx = json.load(open(os.path.join(GOLDEN, "hand_two_tokens.json")))
    for c in fx["cases"]:
        q = bf16(np.array(c["q"]).reshape(1, 2, 1, 1))
        k = bf16(np.array(c["k"]).reshape(1, 2, 1, 1))
        kp = bf16(np.zeros((0, 1, 1)))
        cu = torch.tensor([0, 0], dtype=torch.int32)
        got = orc.importance(q, kp, cu, k, Hq=1, Hkv=1, scale=c["scale"])[0]
        want = [_expr(e) for e in c["expected"]]
        np.testing.assert_allclose(got, want, rtol=1e-13, atol=0)


def pin_rows_sum_to_one_without_prefix(orc):
    """No prefix: every query row's weights sum to 1, so sum_j I_j = B * Hq."""
    q, _, _, kb = small_problem(1, L=(0, 0, 0))
    R, B, Hq = q.shape[0], q.shape[1], q.shape[2]
    kp = bf16(np.zeros((0, 2, 8)))
    cu = torch.zeros(R + 1, dtype=torch.int32)
    I = orc.importance(q, kp, cu, kb, Hq=Hq, Hkv=2, scale=0.9)
    np.testing.assert_allclose(I.sum(axis=1), B * Hq, rtol=1e-13)
    assert (I > 0).all()


def pin_prefix_takes_share(orc):
    """With a prefix the block columns receive strictly less than B * Hq in total, and
    the prefix share grows with the prefix length (keys all equal -> exact shares)."""
    q, kp, cu, kb = small_problem(2)
    I = orc.importance(q, kp, cu, kb, Hq=4, Hkv=2, scale=0.9)
    tot = I.sum(axis=1)
    assert abs(tot[0] - 6 * 4) < 1e-12          # request 0 has no prefix
    assert (tot[1:] < 6 * 4).all() and (tot[1:] > 0).all()
    # identical keys everywhere: each row is uniform over N keys -> block share B/N exactly
    kp1 = bf16(np.ones((int(cu[-1]), 2, 8)))
    kb1 = bf16(np.ones((3, 6, 2, 8)))
    I1 = orc.importance(q, kp1, cu, kb1, Hq=4, Hkv=2, scale=0.9)
    for r, L in enumerate((0, 5, 9)):
        np.testing.assert_allclose(I1[r], 6 * 4 / (L + 6), rtol=1e-13)


def pin_zero_queries_uniform(orc):
    """Q = 0 (or scale = 0): every row is uniform, I_j = B * Hq / N_r."""
    q, kp, cu, kb = small_problem(3)
    z = torch.zeros_like(q)
    Iz = orc.importance(z, kp, cu, kb, Hq=4, Hkv=2, scale=1.3)
    Is = orc.importance(q, kp, cu, kb, Hq=4, Hkv=2, scale=0.0)
    for r, L in enumerate((0, 5, 9)):
        np.testing.assert_allclose(Iz[r], 6 * 4 / (L + 6), rtol=1e-13)
        np.testing.assert_allclose(Is[r], 6 * 4 / (L + 6), rtol=1e-13)


def pin_single_key_block(orc):
    """B = 1, no prefix: the single weight of every row is 1, so I_0 = Hq."""
    gen = torch.Generator().manual_seed(4)
    q = rand_bf16(gen, (2, 1, 6, 4))
    kb = rand_bf16(gen, (2, 1, 3, 4))
    I = orc.importance(q, bf16(np.zeros((0, 3, 4))), torch.zeros(3, dtype=torch.int32), kb,
                       Hq=6, Hkv=3, scale=2.0)
    np.testing.assert_allclose(I, 6.0, rtol=1e-14)


def pin_prefix_permutation_invariance(orc):
    """The softmax denominator is a sum over keys: permuting a request's prefix keys
    changes nothing."""
    q, kp, cu, kb = small_problem(5, L=(7, 11, 4))
    I = orc.importance(q, kp, cu, kb, Hq=4, Hkv=2, scale=0.8)
    rng = np.random.default_rng(5)
    perm = np.concatenate([rng.permutation(np.arange(a, b)) for a, b in
                           zip(cu[:-1].tolist(), cu[1:].tolist())])
    Ip = orc.importance(q, kp[torch.from_numpy(perm)], cu, kb, Hq=4, Hkv=2, scale=0.8)
    np.testing.assert_allclose(Ip, I, rtol=1e-12, atol=1e-15)


def pin_block_permutation_equivariance(orc):
    """Permuting the block keys permutes the block columns of I the same way
    (queries held fixed)."""
    q, kp, cu, kb = small_problem(6, L=(3, 0, 8))
    I = orc.importance(q, kp, cu, kb, Hq=4, Hkv=2, scale=0.8)
    perm = torch.tensor([3, 0, 5, 1, 4, 2])
    Ip = orc.importance(q, kp, cu, kb[:, perm], Hq=4, Hkv=2, scale=0.8)
    np.testing.assert_allclose(Ip, I[:, perm.numpy()], rtol=1e-12, atol=1e-15)


def pin_key_shift_invariance(orc):
    """Adding one vector v to every key of a kv head adds q.v to every logit of each
    row that reads it, a per-row constant the softmax removes.  Integer-valued keys
    keep the shifted keys exact in bf16."""
    gen = torch.Generator().manual_seed(7)
    R, B, Hq, Hkv, d = 2, 5, 4, 2, 6
    L = np.array([4, 7])
    cu = torch.from_numpy(np.concatenate([[0], np.cumsum(L)]).astype(np.int32))
    q = (torch.randint(-2, 3, (R, B, Hq, d), generator=gen).float() * 0.25).to(torch.bfloat16)
    kp = torch.randint(-3, 4, (int(L.sum()), Hkv, d), generator=gen).float()
    kb = torch.randint(-3, 4, (R, B, Hkv, d), generator=gen).float()
    v = torch.randint(-2, 3, (Hkv, d), generator=gen).float()
    I = orc.importance(q, kp.to(torch.bfloat16), cu, kb.to(torch.bfloat16), Hq=Hq, Hkv=Hkv, scale=0.5)
    Is = orc.importance(q, (kp + v).to(torch.bfloat16), cu, (kb + v).to(torch.bfloat16),
                        Hq=Hq, Hkv=Hkv, scale=0.5)
    np.testing.assert_allclose(Is, I, rtol=1e-11, atol=1e-14)


def pin_gqa_expansion(orc):
    """Grouped-query heads: query head h reads kv head h // (Hq/Hkv).  Expanding the
    kv heads so each query head has its own copy (Hkv = Hq) gives the same I."""
    q, kp, cu, kb = small_problem(8, R=2, B=5, Hq=6, Hkv=2, d=4, L=(3, 6))
    I = orc.importance(q, kp, cu, kb, Hq=6, Hkv=2, scale=0.9)
    idx = torch.arange(6) // 3
    Ie = orc.importance(q, kp[:, idx].contiguous(), cu, kb[:, :, idx].contiguous(),
                        Hq=6, Hkv=6, scale=0.9)
    np.testing.assert_allclose(Ie, I, rtol=1e-13, atol=1e-15)


def pin_heads_sum(orc):
    """I sums over query heads: computing each head alone (Hq = Hkv = 1) and adding
    the results gives the multi-head I."""
    q, kp, cu, kb = small_problem(9, R=2, B=4, Hq=4, Hkv=4, d=5, L=(2, 5))
    I = orc.importance(q, kp, cu, kb, Hq=4, Hkv=4, scale=0.7)
    acc = np.zeros_like(I)
    for h in range(4):
        acc += orc.importance(q[:, :, h:h + 1].contiguous(), kp[:, h:h + 1].contiguous(), cu,
                              kb[:, :, h:h + 1].contiguous(), Hq=1, Hkv=1, scale=0.7)
    np.testing.assert_allclose(acc, I, rtol=1e-13, atol=1e-15)


def pin_requests_independent(orc):
    """Each request is computed alone: a batch equals its requests run one by one."""
    q, kp, cu, kb = small_problem(10, L=(4, 0, 6))
    I = orc.importance(q, kp, cu, kb, Hq=4, Hkv=2, scale=0.9)
    for r in range(3):
        a, b = int(cu[r]), int(cu[r + 1])
        Ir = orc.importance(q[r:r + 1], kp[a:b], torch.tensor([0, b - a], dtype=torch.int32),
                            kb[r:r + 1], Hq=4, Hkv=2, scale=0.9)
        np.testing.assert_allclose(Ir[0], I[r], rtol=1e-14)


def pin_library_softmax_columns(orc):
    """Tiny shapes against torch float64 softmax along the key axis (a library routine)."""
    q, kp, cu, kb = small_problem(11, R=2, B=5, Hq=4, Hkv=2, d=6, L=(3, 7), std=1.0)
    scale = 0.6
    I = orc.importance(q, kp, cu, kb, Hq=4, Hkv=2, scale=scale)
    want = np.zeros_like(I)
    for r in range(2):
        keys = torch.cat([kp[int(cu[r]):int(cu[r + 1])], kb[r]], 0).double()   # [N, Hkv, d]
        L = int(cu[r + 1] - cu[r])
        for h in range(4):
            w = torch.softmax(scale * q[r, :, h].double() @ keys[:, h // 2].T, dim=-1)
            want[r] += w[:, L:].sum(0).numpy()
    np.testing.assert_allclose(I, want, rtol=1e-12, atol=1e-15)


def _true_lse(q, kp, cu, kb, Hkv, scale):
    """Row log-sum-exps over prefix + block keys with torch float64 logsumexp."""
    R, B, Hq, _ = q.shape
    G = Hq // Hkv
    out = np.zeros((R, B, Hq))
    for r in range(R):
        keys = torch.cat([kp[int(cu[r]):int(cu[r + 1])], kb[r]], 0).double()
        for h in range(Hq):
            s = scale * q[r, :, h].double() @ keys[:, h // G].T
            out[r, :, h] = torch.logsumexp(s, dim=-1).numpy()
    return out


def pin_paged_prefix_matches_packed(orc):
    """The same prefix keys read through a page table (shuffled pages, junk in the
    unused tail of each last page) give the same importance as the packed layout,
    for pages shorter and longer than the prefixes."""
    import synth
    for page_size in (1, 3, 4, 16):
        p = synth.make_problem(0, overrides=dict(R=4, B=5, Hq=4, Hkv=2, d=8, H=8,
                                                 prefix=("uniform", 0, 11), decoded=("exact", 1),
                                                 lift=("count", 1), budget=("fixed", 2)),
                               seed=page_size)
        pg = synth.to_paged(p, page_size, seed=page_size)
        packed = orc.importance(p.q0, p.k0_prefix, p.cu_prefix, p.k0_block, Hq=4, Hkv=2,
                                scale=p.scale)
        paged = orc.importance_paged(p.q0, pg.k0_pages, pg.page_table, pg.prefix_len, p.k0_block,
                                     Hq=4, Hkv=2, scale=p.scale)
        np.testing.assert_allclose(paged, packed, rtol=1e-13, atol=1e-16)


def pin_hand_dynamic_budget(orc):
    """Dynamic budgets worked by hand (tests/golden/hand_dynamic_budget.json)."""
    fx = json.load(open(os.path.join(GOLDEN, "hand_dynamic_budget.json")))
    for c in fx["cases"]:
        pooled = np.array([[_num(x) for x in c["pooled"]]])
        dec = np.array([c["decoded"]], np.uint8)
        got = orc.dynamic_budget(pooled, dec, np.array([c["decode_avg"]]), c["alpha"])
        assert got.tolist() == [c["budget"]], (c["derivation"], got)


def pin_dynamic_budget_bounds(orc):
    """On random blocks: 1 <= K_r <= masked_r (0 when nothing is masked); K_r grows with
    the historical yield; a large yield saturates at masked_r."""
    rng = np.random.default_rng(22)
    R, B = 40, 16
    pooled = rng.normal(size=(R, B))
    dec = (rng.random((R, B)) < 0.4).astype(np.uint8)
    pooled[dec != 0] = -np.inf
    masked = (dec == 0).sum(1)
    k_lo = orc.dynamic_budget(pooled, dec, np.zeros(R))
    k_hi = orc.dynamic_budget(pooled, dec, np.full(R, 3.0))
    k_sat = orc.dynamic_budget(pooled, dec, np.full(R, 1e6))
    assert ((k_lo >= np.minimum(1, masked)) & (k_lo <= masked)).all()
    assert (k_hi >= k_lo).all() and (k_hi >= np.minimum(5, masked)).all()  # ceil(1.5 * 3) = 5
    np.testing.assert_array_equal(k_sat, masked)


def pin_importance_lse_matches_full(orc):
    """Given the true row log-sum-exps (torch logsumexp over prefix and block keys),
    the block-keys-only importance equals the full one."""
    q, kp, cu, kb = small_problem(17, R=3, B=5, Hq=4, Hkv=2, d=6, L=(0, 4, 9), std=1.0)
    lse = _true_lse(q, kp, cu, kb, 2, 0.7)
    full = orc.importance(q, kp, cu, kb, Hq=4, Hkv=2, scale=0.7)
    via = orc.importance_lse(q, kb, lse, Hq=4, Hkv=2, scale=0.7)
    np.testing.assert_allclose(via, full, rtol=1e-12, atol=1e-15)


def pin_importance_lse_closed_form(orc):
    """One head, one query, lse = c: I_j = exp(s_j - c), and a shift of c scales I by e^-shift."""
    q = bf16(np.array([1.0, 2.0]).reshape(1, 2, 1, 1))
    k = bf16(np.array([0.5, -1.0]).reshape(1, 2, 1, 1))
    lse = np.zeros((1, 2, 1))
    got = orc.importance_lse(q, k, lse, Hq=1, Hkv=1, scale=1.0)
    # column j sums over the two queries i: exp(q_i * k_j)
    want = [math.exp(0.5) + math.exp(1.0), math.exp(-1.0) + math.exp(-2.0)]
    np.testing.assert_allclose(got[0], want, rtol=1e-14)
    got2 = orc.importance_lse(q, k, lse + 0.75, Hq=1, Hkv=1, scale=1.0)
    np.testing.assert_allclose(got2, got * math.exp(-0.75), rtol=1e-14)


# --------------------------------------------------------------------------- delta / pool / mask

def pin_delta_sign_and_pool(orc):
    """Delta = I1 - I0 (Eq. 3); MaxPool1D k=3 stride 1 same padding against
    torch.nn.functional.max_pool1d (padding cells ignored); decoded -> -inf."""
    rng = np.random.default_rng(12)
    for B, w in ((1, 3), (2, 3), (7, 3), (32, 3), (9, 5), (6, 1)):
        i0 = rng.normal(size=(4, B))
        i1 = rng.normal(size=(4, B))
        dec = (rng.random((4, B)) < 0.3).astype(np.uint8)
        raw, pooled = orc.delta_pool_mask(i0, i1, dec, window=w)
        np.testing.assert_array_equal(raw, i1 - i0)
        ref = torch.nn.functional.max_pool1d(torch.from_numpy(i1 - i0)[:, None], w, 1,
                                             w // 2)[:, 0].numpy()
        ref = np.where(dec != 0, -np.inf, ref)
        np.testing.assert_array_equal(pooled, ref)


def pin_pool_spreads_decoded_neighbour(orc):
    """Pooling runs before the mask, so a decoded token's delta reaches its masked
    neighbours while the decoded token itself becomes -inf."""
    i0 = np.zeros((1, 5))
    i1 = np.array([[0.0, 0.0, 5.0, 0.0, 1.0]])
    dec = np.array([[0, 0, 1, 0, 0]], np.uint8)
    _, pooled = orc.delta_pool_mask(i0, i1, dec, window=3)
    np.testing.assert_array_equal(pooled, [[0.0, 5.0, -np.inf, 5.0, 1.0]])


# --------------------------------------------------------------------------- select

def pin_topk_lexsort(orc):
    """Top-k by (value desc, position asc) against numpy.lexsort, with many exact ties
    (values on a coarse grid) and -inf at decoded positions."""
    rng = np.random.default_rng(13)
    R, B = 40, 16
    pooled = rng.integers(-3, 4, size=(R, B)).astype(np.float64) * 0.5
    dec = (rng.random((R, B)) < 0.35).astype(np.uint8)
    pooled[dec != 0] = -np.inf
    budget = rng.integers(-2, B + 3, size=R).astype(np.int32)
    kept, cu, st = orc.select(pooled, dec, budget)
    assert st == 0 and cu[0] == 0
    for r in range(R):
        m = int((dec[r] == 0).sum())
        k = min(max(int(budget[r]), 0), m)
        assert cu[r + 1] - cu[r] == k
        order = np.lexsort((np.arange(B), -pooled[r]))
        want = np.sort(order[:k])
        np.testing.assert_array_equal(kept[cu[r]:cu[r + 1]], want)


def pin_topk_bruteforce(orc):
    """For B <= 8, the kept set maximises the sum of values over all k-subsets of
    masked positions and is the lexicographically smallest such set (lower positions
    win ties).  Small integer values make every sum exact."""
    rng = np.random.default_rng(14)
    for trial in range(150):
        B = int(rng.integers(1, 9))
        vals = rng.integers(-2, 3, size=B).astype(np.float64)
        dec = (rng.random(B) < 0.3).astype(np.uint8)
        vals[dec != 0] = -np.inf
        K = int(rng.integers(0, B + 2))
        masked = np.flatnonzero(dec == 0)
        k = min(K, masked.size)
        best = None
        for sub in itertools.combinations(masked.tolist(), k):
            s = float(sum(vals[list(sub)])) if sub else 0.0
            if best is None or s > best[0] or (s == best[0] and list(sub) < best[1]):
                best = (s, list(sub))
        kept, cu, _ = orc.select(vals[None], dec[None], np.array([K], np.int32))
        assert kept.tolist() == best[1], (vals, dec, K, kept, best)


def pin_topk_signed_zeros(orc):
    """-0.0 and +0.0 are the same value: they tie, and the lower position wins whatever
    the sign (an order on the bit patterns would put every +0.0 first)."""
    pooled = np.array([[-0.0, 0.0, -0.0, 0.0, 1.0, -1.0],
                       [0.0, -0.0, 0.0, -0.0, -0.0, 0.0]], np.float64)
    dec = np.zeros((2, 6), np.uint8)
    kept, cu, st = orc.select(pooled, dec, np.array([3, 4], np.int32))
    assert st == 0 and cu.tolist() == [0, 3, 7]
    assert kept.tolist() == [0, 1, 4] + [0, 1, 2, 3]


def pin_capacity_status(orc):
    """Selecting more rows than the packed buffer holds is reported, cu_seqlens is
    still complete, and only the rows that fit are written."""
    pooled = np.arange(12, dtype=np.float64).reshape(2, 6)
    dec = np.zeros((2, 6), np.uint8)
    kept, cu, st = orc.select(pooled, dec, np.array([4, 4], np.int32), capacity=5)
    assert st == 3 and cu.tolist() == [0, 4, 8]
    assert kept.tolist() == [2, 3, 4, 5, 2]


# --------------------------------------------------------------------------- compact

def pin_compact_fancy_indexing(orc):
    """Compaction is a bit copy: numpy fancy indexing on the raw bf16 bits."""
    rng = np.random.default_rng(15)
    R, B, H = 5, 7, 24
    bits = rng.integers(0, 1 << 16, size=(R, B, H), dtype=np.uint16)
    bits[(bits & 0x7F80) == 0x7F80] = 0x3F80   # keep the patterns finite
    counts = rng.integers(0, B + 1, size=R)
    cu = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    kept = np.concatenate([np.sort(rng.choice(B, size=c, replace=False)) for c in counts]).astype(np.int32)
    packed = orc.compact(bits, kept, cu)
    rows = np.repeat(np.arange(R), counts)
    np.testing.assert_array_equal(packed, bits[rows, kept])


# --------------------------------------------------------------------------- end to end

def pin_hand_evict(orc):
    """The four-token step worked by hand (tests/golden/hand_evict_b4.json)."""
    fx = json.load(open(os.path.join(GOLDEN, "hand_evict_b4.json")))
    B, H, a = fx["B"], fx["H"], fx["a"]
    q0 = bf16(np.zeros((1, B, 1, 1)))
    q1 = bf16(np.ones((1, B, 1, 1)))
    k = bf16(np.array([0.0, 0.0, a, 0.0]).reshape(1, B, 1, 1))
    kp = bf16(np.zeros((0, 1, 1)))
    cu = torch.tensor([0, 0], dtype=torch.int32)
    i0 = orc.importance(q0, kp, cu, k, Hq=1, Hkv=1, scale=1.0)
    i1 = orc.importance(q1, kp, cu, k, Hq=1, Hkv=1, scale=1.0)
    np.testing.assert_allclose(i0[0], [_expr(e) for e in fx["i0"]], rtol=1e-14)
    np.testing.assert_allclose(i1[0], [_expr(e) for e in fx["i1"]], rtol=1e-13)
    dec = np.array([fx["decoded"]], np.uint8)
    _, pooled = orc.delta_pool_mask(i0, i1, dec, window=3)
    np.testing.assert_allclose(pooled[0], [_expr(e) for e in fx["pooled"]], rtol=1e-13)
    hidden = bf16(np.arange(B * H, dtype=np.float32).reshape(1, B, H))
    for K, want in fx["budgets"].items():
        kept, cu_s, _ = orc.select(pooled, dec, np.array([int(K)], np.int32))
        assert kept.tolist() == want, (K, kept)
        assert cu_s.tolist() == [0, len(want)]
        packed = orc.compact(hidden, kept, cu_s)
        np.testing.assert_array_equal(
            packed, hidden[0, want].view(torch.int16).numpy().view(np.uint16).reshape(len(want), H))


# --------------------------------------------------------------------------- structural constraints

def _num(x):
    return -np.inf if x == "-inf" else float(x)


def pin_hand_structural(orc):
    """Hand-worked retained sets for every constraint combination
    (tests/golden/hand_structural_b8.json)."""
    fx = json.load(open(os.path.join(GOLDEN, "hand_structural_b8.json")))
    for case in fx["cases"]:
        dec = np.array([case["decoded"]], np.uint8)
        pooled = np.array([[_num(x) for x in case["pooled"]]])
        bud = np.array([case["budget"]], np.int32)
        for c, want in case["retained"].items():
            kept, cu, st = orc.select_structured(pooled, dec, bud, int(c))
            assert st == 0 and kept.tolist() == want, (case["derivation"], c, kept, want)
            assert cu.tolist() == [0, len(want)]


def pin_structural_properties(orc):
    """On random blocks: constraints 0 equal the plain top-k; the retained set
    contains the candidates, every candidate's predecessor (bit 1) and every masked
    position left of the rightmost candidate (bit 2), and nothing else; it is
    ascending and unique."""
    rng = np.random.default_rng(16)
    R, B = 30, 12
    pooled = rng.integers(-3, 4, size=(R, B)).astype(np.float64)
    dec = (rng.random((R, B)) < 0.3).astype(np.uint8)
    pooled[dec != 0] = -np.inf
    budget = rng.integers(0, 6, size=R).astype(np.int32)
    cand, ccu, _ = orc.select(pooled, dec, budget)
    k0, cu0, _ = orc.select_structured(pooled, dec, budget, 0)
    np.testing.assert_array_equal(k0, cand)
    np.testing.assert_array_equal(cu0, ccu)
    for c in (1, 2, 3):
        kept, cu, _ = orc.select_structured(pooled, dec, budget, c)
        for r in range(R):
            got = kept[cu[r]:cu[r + 1]].tolist()
            S = set(cand[ccu[r]:ccu[r + 1]].tolist())
            assert got == sorted(set(got))
            want = set(S)
            if c & 1:
                want |= {j - 1 for j in S if j >= 1}
            if c & 2 and S:
                want |= {j for j in range(max(S)) if dec[r, j] == 0}
            assert set(got) == want, (r, c, got, sorted(want))


PINS = [
    pin_hand_two_tokens, pin_rows_sum_to_one_without_prefix, pin_prefix_takes_share,
    pin_zero_queries_uniform, pin_single_key_block, pin_prefix_permutation_invariance,
    pin_block_permutation_equivariance, pin_key_shift_invariance, pin_gqa_expansion,
    pin_heads_sum, pin_requests_independent, pin_library_softmax_columns,
    pin_delta_sign_and_pool, pin_pool_spreads_decoded_neighbour, pin_topk_lexsort,
    pin_topk_bruteforce, pin_topk_signed_zeros, pin_capacity_status, pin_compact_fancy_indexing,
    pin_hand_evict,
    pin_hand_structural, pin_structural_properties, pin_importance_lse_matches_full,
    pin_importance_lse_closed_form, pin_paged_prefix_matches_packed, pin_hand_dynamic_budget,
    pin_dynamic_budget_bounds,
]
