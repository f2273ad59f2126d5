"""Pins of the oracle's router (R1-R3) and align (R4) steps (CPU)."""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy.special import softmax as scipy_softmax

from oracle import align_ref, bf16_bits_to_f64, route_ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_array(a):
    t = torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return bf16_bits_to_f64(t.view(torch.int16).numpy().view(np.uint16))


def brute_force_topk(x, wr, bias, k):
    """Top-k by exhaustive subset search on exact rational logits.

    A k-subset S is the answer iff every member beats every non-member under
    (value desc, index asc); the members are then ordered by that relation.
    """
    T, E = x.shape[0], wr.shape[0]
    out = []
    for t in range(T):
        lg = [sum((Fraction(float(a)) * Fraction(float(b)) for a, b in zip(x[t], wr[e])), Fraction(0))
              + (Fraction(float(np.float32(bias[e]))) if bias is not None else 0) for e in range(E)]

        def beats(a, b):
            return lg[a] > lg[b] or (lg[a] == lg[b] and a < b)

        found = None
        for S in itertools.combinations(range(E), k):
            rest = [e for e in range(E) if e not in S]
            if all(beats(a, b) for a in S for b in rest):
                assert found is None
                found = S
        ordered = sorted(found, key=lambda e: sum(beats(o, e) for o in found))
        out.append(ordered)
    return np.array(out, dtype=np.int32)


@pytest.mark.parametrize("seed,E,k,use_bias", [(0, 6, 1, False), (1, 6, 2, False), (2, 6, 3, True),
                                               (3, 5, 5, False), (4, 7, 4, True)])
def test_route_matches_brute_force(seed, E, k, use_bias):
    rng = np.random.default_rng(seed)
    T, H = 6, 16
    x = bf16_array(rng.standard_normal((T, H)))
    wr = bf16_array(rng.standard_normal((E, H)) * 0.1)
    wr[1] = wr[0]                       # an exact tie in every token
    bias = (rng.standard_normal(E) * 0.3).astype(np.float32) if use_bias else None
    if use_bias:
        bias[1] = bias[0]
    ids, w, _, _ = route_ref(x, wr, bias, k)
    assert np.array_equal(ids, brute_force_topk(x, wr, bias, k))
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-12, rtol=0)


def test_exact_tie_lower_index_first():
    rng = np.random.default_rng(5)
    x = bf16_array(rng.standard_normal((16, 32)))
    row = bf16_array(rng.standard_normal(32) * 0.1)
    wr = np.stack([row * 0.0] + [row] * 4 + [-row] * 3)   # experts 1..4 identical
    ids, _, _, n_exact = route_ref(x, wr, None, 2)
    for t in range(16):
        if x[t] @ row > 0:
            assert list(ids[t]) == [1, 2]
        elif x[t] @ row < 0:
            assert list(ids[t]) == [5, 6]
    assert n_exact > 0


def test_all_equal_logits_pick_first_experts():
    x = np.zeros((3, 8))
    wr = bf16_array(np.ones((6, 8)))
    ids, w, _, _ = route_ref(x, wr, None, 4)
    assert np.array_equal(ids, np.tile(np.arange(4, dtype=np.int32), (3, 1)))
    assert np.allclose(w, 0.25, rtol=0, atol=1e-15)


def test_near_tie_needs_exact_arithmetic():
    # l0 = 2^60 + 1 and l1 = 2^60 round to the same fp64 number; exact order is 0 > 1
    # only through the tiny term; with expert 2 exactly equal to expert 1.
    H = 4
    x = np.array([[2.0 ** 30, 1.0, 0.0, 0.0]])
    wr = np.array([[2.0 ** 30, 1.0, 0, 0], [2.0 ** 30, 0.0, 0, 0], [2.0 ** 30, 0.0, 0, 0],
                   [1.0, 0, 0, 0]])
    assert np.all(bf16_array(wr) == wr) and np.all(bf16_array(x) == x)
    ids, _, L, n_exact = route_ref(x, wr, None, 2)
    assert L[0, 0] == L[0, 1]            # fp64 cannot tell them apart
    assert n_exact == 1
    assert list(ids[0]) == [0, 1]
    ids, _, _, _ = route_ref(-x * 0 + np.array([[2.0 ** 30, -1.0, 0, 0]]), wr, None, 2)
    assert list(ids[0]) == [1, 2]        # now expert 0 is the smaller one; 1 and 2 tie


def test_weights_full_softmax_when_k_equals_E():
    rng = np.random.default_rng(6)
    x = bf16_array(rng.standard_normal((5, 24)))
    wr = bf16_array(rng.standard_normal((7, 24)) * 0.1)
    bias = (rng.standard_normal(7)).astype(np.float32)
    ids, w, L, _ = route_ref(x, wr, bias, 7)
    p = scipy_softmax(x @ wr.T + bias.astype(np.float64), axis=1)
    assert np.allclose(np.take_along_axis(p, ids.astype(np.int64), 1), w, rtol=1e-12, atol=0)
    ids1, w1, _, _ = route_ref(x, wr, bias, 1)
    assert np.all(w1 == 1.0)
    assert np.array_equal(ids1[:, 0], np.argmax(p, axis=1))


def _golden_cases():
    with open(os.path.join(GOLDEN, "router_closed_form.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            lg, k, ids, ws = [s.strip() for s in line.split(";")]
            yield ([float(v) for v in lg.split()], int(k), [int(v) for v in ids.split()],
                   [eval(s, {"__builtins__": {}}, {"exp": math.exp}) for s in ws.split(",")])


@pytest.mark.parametrize("case", list(_golden_cases()))
def test_router_closed_forms(case):
    logits, k, want_ids, want_w = case
    E = len(logits)
    x = np.zeros((1, 8))
    x[0, 0] = 1.0
    wr = np.zeros((E, 8))
    wr[:, 0] = logits
    assert np.all(bf16_array(wr) == wr)
    ids, w, _, _ = route_ref(x, wr, None, k)
    assert list(ids[0]) == want_ids
    assert np.allclose(w[0], want_w, rtol=1e-14, atol=1e-15)


def test_zipf_bias_only_routing_closed_form():
    E, k = 16, 8
    bias = np.array([-1.1 * math.log(e + 1) for e in range(E)], dtype=np.float32)
    x = np.zeros((2, 8))
    wr = np.zeros((E, 8))
    ids, w, _, _ = route_ref(x, wr, bias, k)
    assert np.array_equal(ids[0], np.arange(k))
    zk = np.array([(j + 1) ** -1.1 for j in range(k)])
    assert np.allclose(w[0], zk / zk.sum(), rtol=1e-6, atol=0)


# ---------------------------------------------------------------- align -----
def naive_align(ids, E):
    T, k = ids.shape
    buckets = [[] for _ in range(E)]
    for t in range(T):
        for j in range(k):
            buckets[ids[t, j]].append(t * k + j)
    counts = [len(b) for b in buckets]
    offsets = [0]
    for c in counts:
        offsets.append(offsets[-1] + c)
    perm = [f for b in buckets for f in b]
    return counts, offsets, perm


@pytest.mark.parametrize("seed,T,E,k", [(0, 1, 4, 1), (1, 7, 8, 2), (2, 33, 64, 8), (3, 100, 5, 5),
                                        (4, 64, 256, 8)])
def test_align_invariants_and_brute_force(seed, T, E, k):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv_perm = align_ref(ids, E)
    A = T * k
    assert counts.sum() == A
    assert offsets[0] == 0 and offsets[-1] == A and np.all(np.diff(offsets) == counts)
    assert np.array_equal(np.sort(perm), np.arange(A))            # bijection
    assert np.array_equal(inv_perm[perm], np.arange(A))
    assert np.array_equal(perm[inv_perm], np.arange(A))
    flat = ids.reshape(-1)
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)
    c2, o2, p2 = naive_align(ids, E)
    assert list(counts) == c2 and list(offsets) == o2 and list(perm) == p2
