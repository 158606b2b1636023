"""Pins for the CPU oracle: each oracle function is checked against something
other than itself -- hand-worked tiny cases, brute force, closed forms,
invariants and independent numpy / Python re-statements -- chosen so that a
plausible mistake (transposed W_H, wrong bit order, '>=' for '>', a dropped
tie rule, a wrong softmax) fails at least one of them.

Definitions pinned (HATA review page, arXiv 2506.02572):
  * "Assumptions & free parameters": h(x) = sign(x W_H), rbit = 128;
  * "What carries the argument": XOR + popcount Hamming score, top-k by it,
    attention over the selected keys only;
  * Figure 2 caption (Algorithm 1): rbit/32 32-bit words per cached code;
  * major comment 1 (Algorithm 3): 129 possible scores, boundary ties.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def pack_bits_le(bits: np.ndarray) -> np.ndarray:
    """[..., r] 0/1 -> [..., r/32] uint32, bit j in word j//32 at position j%32."""
    b = np.packbits(bits.astype(np.uint8), axis=-1, bitorder="little")
    return b.view("<u4")


def popcount_u32(x: np.ndarray) -> np.ndarray:
    return np.unpackbits(np.ascontiguousarray(x).view(np.uint8), axis=-1).sum(-1)


def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (no NaNs here)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def widen(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------- hash ---

def test_hash_worked_by_hand():
    """Tiny case worked by hand from h(x) = sign(x W_H) (golden fixture)."""
    with open(os.path.join(GOLDEN, "hash_by_hand.json")) as f:
        case = json.load(f)
    x = np.array(case["x"], np.float32)
    W = np.array(case["W"], np.float32)
    code = oracle.hash_vec(x, W)
    assert [int(c) for c in code] == case["code_words"]


def test_hash_agrees_with_fp64_projection_sign():
    """Bit j = [x . W[:, j] > 0] with W stored [d][r], packed LSB-first.  An
    independent fp64 numpy product decides every bit whose projection is not
    within rounding distance of zero."""
    d = r = 128
    flagged = 0
    for _ in range(40):
        W = (RNG.standard_normal((d, r)) / math.sqrt(d)).astype(np.float32)
        x = RNG.standard_normal(d).astype(np.float32)
        proj = x.astype(np.float64) @ W.astype(np.float64)
        bound = 1e-5 * np.linalg.norm(x) * np.linalg.norm(W.astype(np.float64), axis=0)
        safe = np.abs(proj) > bound
        flagged += int((~safe).sum())
        expect = pack_bits_le(proj > 0)
        got = oracle.hash_vec(x, W)
        mask = pack_bits_le(safe)
        assert np.array_equal(got & mask, expect & mask)
    assert flagged <= 2


def test_hash_negation_gives_complement():
    """hash(-x) == ~hash(x) whenever no projection is exactly zero (the fp32
    fma chain is sign-symmetric under round-to-nearest)."""
    d = r = 128
    for _ in range(20):
        W = (RNG.standard_normal((d, r)) / math.sqrt(d)).astype(np.float32)
        x = RNG.standard_normal(d).astype(np.float32)
        assert np.all(np.abs(x.astype(np.float64) @ W) > 1e-6)
        a = oracle.hash_vec(x, W)
        b = oracle.hash_vec(-x, W)
        assert np.array_equal(b, ~a)


def test_hash_zero_projection_is_zero_bit():
    """sign(0) is read as bit 0: the zero vector hashes to all-zero, and so
    does a zero column of W_H for any x."""
    d = r = 128
    W = (RNG.standard_normal((d, r)) / math.sqrt(d)).astype(np.float32)
    assert np.all(oracle.hash_vec(np.zeros(d, np.float32), W) == 0)
    W[:, 37] = 0.0
    for _ in range(10):
        x = RNG.standard_normal(d).astype(np.float32)
        c = oracle.hash_vec(x, W)
        assert (int(c[1]) >> 5) & 1 == 0


def test_hash_projection_is_fp32_fma_chain_in_index_order():
    """The projection is the fp32 chain acc = fma(x_i, W[i][j], acc) over
    i ascending.  x = (1, 1e8, -1e8) on a ones column: the chain rounds
    1 + 1e8 to 1e8 and ends at exactly 0 (bit 0), although the exact sum is 1
    (and the descending chain would end at 1)."""
    W = np.zeros((3, 32), np.float32)
    W[:, 0] = 1.0
    x = np.array([1.0, 1e8, -1e8], np.float32)
    assert int(oracle.hash_vec(x, W)[0]) & 1 == 0
    x_rev = x[::-1].copy()  # (-1e8, 1e8, 1): chain ends at exactly 1 -> bit 1
    assert int(oracle.hash_vec(x_rev, W)[0]) & 1 == 1


def test_hash_bf16_input_is_exact_widening():
    d = r = 128
    W = (RNG.standard_normal((d, r)) / math.sqrt(d)).astype(np.float32)
    for _ in range(10):
        bits = bf16_round_bits(RNG.standard_normal(d).astype(np.float32))
        assert np.array_equal(oracle.hash_vec(bits, W), oracle.hash_vec(widen(bits), W))


@pytest.mark.parametrize("kv", ["f32", "bf16"])
def test_hash_keys_layout(kv):
    """Algorithm 1: codes[b][h][t] is the hash of K[b][h][t] with head h's W_H,
    for t in [pos0, pos0+n) only.  A bf16 cache is read as 2-byte rows whose
    values widen exactly to fp32, so its codes are the fp64 projection signs
    of the widened values (a wrong row stride or widening reads other keys)."""
    B, H, n_cap, d, r = 2, 3, 9, 128, 128
    K = RNG.standard_normal((B, H, n_cap, d)).astype(np.float32)
    if kv == "bf16":
        K = bf16_round_bits(K)
        Kf = widen(K)
    else:
        Kf = K
    W = (RNG.standard_normal((H, d, r)) / math.sqrt(d)).astype(np.float32)
    codes = oracle.hash_keys(K, W, pos0=2, n=5)
    for b, h, t in itertools.product(range(B), range(H), range(n_cap)):
        if 2 <= t < 7:
            proj = Kf[b, h, t].astype(np.float64) @ W[h]
            assert np.array_equal(codes[b, h, t], pack_bits_le(proj > 0))
        else:
            assert np.all(codes[b, h, t] == 0)


def test_random_hyperplane_collision_closed_form():
    """Random-hyperplane hashing (Gaussian W_H): a bit differs with
    probability theta/pi, so E[Hamming] = 128 * theta / pi for vectors at
    angle theta.  Checked within 5 standard errors."""
    d = r = 128
    W = RNG.standard_normal((d, r)).astype(np.float32) / np.float32(math.sqrt(d))
    for theta in (math.pi / 6, math.pi / 3, math.pi / 2, 2 * math.pi / 3):
        dists = []
        for _ in range(600):
            a = RNG.standard_normal(d)
            a /= np.linalg.norm(a)
            z = RNG.standard_normal(d)
            z -= (z @ a) * a
            z /= np.linalg.norm(z)
            bvec = math.cos(theta) * a + math.sin(theta) * z
            ca = oracle.hash_vec(a.astype(np.float32), W)
            cb = oracle.hash_vec(bvec.astype(np.float32), W)
            dists.append(oracle.hamming(ca, cb))
        p = theta / math.pi
        mean = np.mean(dists)
        se = math.sqrt(r * p * (1 - p) / len(dists)) * 3.0  # columns share W: widen
        assert abs(mean - r * p) < 5 * se, (theta, mean, r * p)


# -------------------------------------------------------------- hamming ---

def test_hamming_brute_force_bits():
    for _ in range(200):
        a = RNG.integers(0, 2**32, 4, dtype=np.uint64).astype(np.uint32)
        b = RNG.integers(0, 2**32, 4, dtype=np.uint64).astype(np.uint32)
        ua = np.unpackbits(a.view(np.uint8))
        ub = np.unpackbits(b.view(np.uint8))
        assert oracle.hamming(a, b) == int((ua != ub).sum())


def test_hamming_identities():
    for _ in range(100):
        a, b, c = (RNG.integers(0, 2**32, 4, dtype=np.uint64).astype(np.uint32)
                   for _ in range(3))
        assert oracle.hamming(a, a) == 0
        assert oracle.hamming(a, ~a) == 128
        assert oracle.hamming(a, b) == oracle.hamming(b, a)
        assert oracle.hamming(a, c) <= oracle.hamming(a, b) + oracle.hamming(b, c)
    one = np.array([1, 0, 0, 0], np.uint32)
    top = np.array([0, 0, 0, 1 << 31], np.uint32)
    zero = np.zeros(4, np.uint32)
    assert oracle.hamming(one, zero) == 1 and oracle.hamming(top, zero) == 1


def test_hamming_all_matches_popcount():
    codes = RNG.integers(0, 2**32, (300, 4), dtype=np.uint64).astype(np.uint32)
    q = RNG.integers(0, 2**32, 4, dtype=np.uint64).astype(np.uint32)
    expect = popcount_u32(codes ^ q[None, :])
    assert np.array_equal(oracle.hamming_all(q, codes), expect)


# ----------------------------------------------------------------- top-k ---

def brute_topk(dist, k):
    order = sorted(range(len(dist)), key=lambda i: (dist[i], i))
    sel = sorted(order[:min(k, len(dist))])
    return sel + [-1] * (k - len(sel))


def bucket_topk(dist, k):
    """A second, different selection: walk the 129 distance buckets upwards,
    taking each bucket's keys in index order until k are taken."""
    sel = []
    for t in range(129):
        for i, dv in enumerate(dist):
            if dv == t and len(sel) < k:
                sel.append(i)
    sel.sort()
    return sel + [-1] * (k - len(sel))


def test_topk_brute_force_tiny():
    for n in list(range(1, 20)) + [31, 32, 33, 64]:
        for spread in (1, 3, 129):
            dist = RNG.integers(0, spread, n).astype(np.int32) + (60 if spread < 129 else 0)
            for k in range(1, n + 3):
                got = oracle.topk(dist, k).tolist()
                assert got == brute_topk(dist.tolist(), k)
                assert got == bucket_topk(dist.tolist(), k)


def test_topk_invariants():
    for _ in range(30):
        n = int(RNG.integers(50, 500))
        dist = RNG.binomial(128, 0.5, n).astype(np.int32)
        k = int(RNG.integers(1, n))
        idx = oracle.topk(dist, k)
        assert (idx >= 0).sum() == min(k, n)
        sel = idx[idx >= 0]
        assert np.all(np.diff(sel) > 0)
        rest = np.setdiff1d(np.arange(n), sel)
        T = dist[sel].max()
        assert T <= dist[rest].min()
        tied_in = sel[dist[sel] == T]
        tied_out = rest[dist[rest] == T]
        if tied_out.size and tied_in.size:
            assert tied_in.max() < tied_out.min()


def test_topk_all_equal_and_oversized_k():
    dist = np.full(100, 64, np.int32)
    assert oracle.topk(dist, 10).tolist() == list(range(10))
    got = oracle.topk(dist[:5], 8).tolist()
    assert got == [0, 1, 2, 3, 4, -1, -1, -1]


# ------------------------------------------------------------- attention ---

def np_softmax_attend(q, K, V, idx, scale):
    s = scale * (K[idx].astype(np.float64) @ q.astype(np.float64))
    p = np.exp(s - s.max())
    p /= p.sum()
    return p @ V[idx].astype(np.float64)


@pytest.mark.parametrize("kv", ["f32", "bf16"])
def test_attend_full_set_equals_dense_softmax(kv):
    n, d = 200, 128
    q = RNG.standard_normal(d).astype(np.float32)
    Kf = RNG.standard_normal((n, d)).astype(np.float32)
    Vf = RNG.standard_normal((n, d)).astype(np.float32)
    if kv == "bf16":
        K, V = bf16_round_bits(Kf), bf16_round_bits(Vf)
        Kv, Vv = widen(K), widen(V)
    else:
        K, V, Kv, Vv = Kf, Vf, Kf, Vf
    scale = 1 / math.sqrt(d)
    expect = np_softmax_attend(q, Kv, Vv, np.arange(n), scale)
    got = oracle.attend(q, K, V, np.arange(n, dtype=np.int32), scale)
    np.testing.assert_allclose(got, expect, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.dense(q, K, V, n, scale), expect, rtol=1e-12, atol=1e-12)


def test_attend_single_key_returns_that_row():
    n, d = 50, 128
    q = RNG.standard_normal(d).astype(np.float32)
    K = RNG.standard_normal((n, d)).astype(np.float32)
    V = RNG.standard_normal((n, d)).astype(np.float32)
    for i in (0, 17, 49):
        got = oracle.attend(q, K, V, np.array([i], np.int32), 0.3)
        assert np.array_equal(got, V[i].astype(np.float64))


def test_attend_zero_scale_is_mean_and_two_key_sigmoid():
    n, d = 40, 128
    q = RNG.standard_normal(d).astype(np.float32)
    K = RNG.standard_normal((n, d)).astype(np.float32)
    V = RNG.standard_normal((n, d)).astype(np.float32)
    idx = np.array([3, 9, 20, 33], np.int32)
    np.testing.assert_allclose(oracle.attend(q, K, V, idx, 0.0),
                               V[idx].astype(np.float64).mean(0), rtol=1e-12, atol=1e-14)
    scale = 0.125
    s1 = scale * float(K[5].astype(np.float64) @ q)
    s2 = scale * float(K[7].astype(np.float64) @ q)
    w1 = 1.0 / (1.0 + math.exp(s2 - s1))
    expect = w1 * V[5].astype(np.float64) + (1 - w1) * V[7].astype(np.float64)
    got = oracle.attend(q, K, V, np.array([5, 7], np.int32), scale)
    np.testing.assert_allclose(got, expect, rtol=1e-12, atol=1e-13)


def test_attend_empty_set_is_zero():
    d = 128
    q = np.ones(d, np.float32)
    K = np.ones((3, d), np.float32)
    got = oracle.attend(q, K, K, np.zeros(0, np.int32), 1.0)
    assert np.all(got == 0)


# ---------------------------------------------------------- decode step ---

@pytest.mark.parametrize("r", [128, 64, 32, 256])
def test_decode_head_matches_independent_restatement(r):
    """The composed step against an independent numpy/Python restatement
    (fp64 projection sign, unpackbits popcount, sorted() top-k, numpy
    softmax) on cases with no projection near zero; also at the narrower
    code widths, where far more keys tie."""
    d = 128
    for trial in range(6):
        n = int(RNG.integers(100, 700))
        k = int(RNG.integers(1, n + 5))
        W = (RNG.standard_normal((d, r)) / math.sqrt(d)).astype(np.float32)
        q = RNG.standard_normal(d).astype(np.float32)
        K = bf16_round_bits(RNG.standard_normal((n, d)).astype(np.float32))
        V = bf16_round_bits(RNG.standard_normal((n, d)).astype(np.float32))
        Kw = widen(K).astype(np.float64)
        qproj = q.astype(np.float64) @ W
        kproj = Kw @ W
        if min(np.abs(qproj).min(), np.abs(kproj).min()) < 1e-4:
            continue
        qc = pack_bits_le(qproj > 0)
        kc = pack_bits_le(kproj > 0)
        dist = popcount_u32(kc ^ qc[None, :])
        idx = brute_topk(dist.tolist(), k)
        sel = np.array([i for i in idx if i >= 0])
        out = np_softmax_attend(q, Kw, widen(V), sel, 1 / math.sqrt(d))
        oqc, odist, oidx, oout, m = oracle.decode_head(q, W, kc, K, V, n, k, 1 / math.sqrt(d))
        assert np.array_equal(oqc, qc)
        assert np.array_equal(odist, dist)
        assert oidx.tolist() == idx
        assert m == min(k, n)
        np.testing.assert_allclose(oout, out, rtol=1e-10, atol=1e-12)


def test_needles_are_selected_on_synthetic_workload():
    """Property of the method on the planted-needle input: keys at
    0.8 * (query direction) + 0.2 * noise sit at small Hamming distance, so the
    1.56% budget keeps every needle."""
    import torch
    from hash_aware_top_hata_b200 import workloads as wl
    cfg = wl.scaled(wl.CONFIGS["needle_gqa_1m"], N=8192, topk=128, B=1)
    cfg = wl.dataclasses.replace(cfg, H_q=4, H_kv=1, needles=16)
    w = wl.make_workload(cfg, seed=7, steps=1)
    K = wl.to_numpy_kv(w.K[0, 0, :cfg.N])
    V = wl.to_numpy_kv(w.V[0, 0, :cfg.N])
    W = w.W_H[0].numpy()
    codes = oracle.hash_rows(K, W)
    q = w.q[0, 0, 0].numpy()
    _, _, idx, _, _ = oracle.decode_head(q, W, codes, K, V, cfg.N, cfg.topk, 1 / math.sqrt(128))
    needles = set(w.planted[0, 0].tolist())
    assert needles <= set(idx.tolist())
    del torch


# --------------------------------------------------- narrower codes (r) ---
# The page's ablation also runs r = 32 and 64 bits: code bit j depends on
# column j of W_H alone, so a narrower code is the leading words of the wide
# one, and the Hamming range is 0..r.

@pytest.mark.parametrize("r", [32, 64])
def test_narrow_code_is_prefix_of_wide_code(r):
    W = RNG.standard_normal((128, 128)).astype(np.float32) / math.sqrt(128)
    for _ in range(20):
        x = RNG.standard_normal(128).astype(np.float32)
        wide = oracle.hash_vec(x, W)
        narrow = oracle.hash_vec(x, np.ascontiguousarray(W[:, :r]))
        assert narrow.shape == (r // 32,)
        assert np.array_equal(narrow, wide[: r // 32])
        # and each bit is the sign of its own projection (fp64 reference,
        # well away from zero)
        proj = x.astype(np.float64) @ W[:, :r].astype(np.float64)
        bits = np.unpackbits(narrow.view(np.uint8), bitorder="little")
        sure = np.abs(proj) > 1e-4
        assert np.array_equal(bits[sure], (proj[sure] > 0).astype(np.uint8))


@pytest.mark.parametrize("r", [32, 64, 256])
def test_narrow_hamming_range_and_brute_force(r):
    w = r // 32
    codes = RNG.integers(0, 2**32, (200, w), dtype=np.uint64).astype(np.uint32)
    q = RNG.integers(0, 2**32, w, dtype=np.uint64).astype(np.uint32)
    d = oracle.hamming_all(q, codes)
    ub = np.unpackbits(codes.view(np.uint8), axis=-1)
    uq = np.unpackbits(q.view(np.uint8))
    assert np.array_equal(d, (ub != uq[None, :]).sum(-1))
    assert oracle.hamming(q, ~q) == r and oracle.hamming(q, q) == 0
    assert d.min() >= 0 and d.max() <= r


# ------------------------------------------------------ 256-bit codes (r) ---
# The ablation's widest code: bit j still depends on column j of W_H alone,
# so the 128-bit code is the first four words of the 256-bit one, and the
# Hamming range is 0..256 (257 values, one more than a byte holds).

def test_wide_code_extends_the_128_bit_code():
    W = RNG.standard_normal((128, 256)).astype(np.float32) / math.sqrt(128)
    for _ in range(20):
        x = RNG.standard_normal(128).astype(np.float32)
        wide = oracle.hash_vec(x, W)
        assert wide.shape == (8,)
        assert np.array_equal(wide[:4], oracle.hash_vec(x, np.ascontiguousarray(W[:, :128])))
        proj = x.astype(np.float64) @ W.astype(np.float64)
        bits = np.unpackbits(wide.view(np.uint8), bitorder="little")
        sure = np.abs(proj) > 1e-4
        assert np.array_equal(bits[sure], (proj[sure] > 0).astype(np.uint8))


def test_topk_at_the_top_of_the_wide_range():
    """Boundaries at 255 and 256 (the values a byte-wide row cannot tell
    apart) against brute force."""
    for trial in range(30):
        n = int(RNG.integers(1, 300))
        d = RNG.choice([250, 254, 255, 256], size=n).astype(np.int32)
        k = int(RNG.integers(1, n + 3))
        assert oracle.topk(d, k).tolist() == brute_topk(d.tolist(), k)


def test_wide_decode_head_complement_codes():
    """Keys coded as the complement of the query code sit at distance 256,
    one flipped bit back at 255: the oracle's selection over them is the
    brute-force one (lower distance first, then lower index)."""
    d = 128
    W = (RNG.standard_normal((d, 256)) / math.sqrt(d)).astype(np.float32)
    q = RNG.standard_normal(d).astype(np.float32)
    qc = oracle.hash_vec(q, W)
    n = 97
    codes = np.tile(~qc, (n, 1))
    flip = RNG.choice(n, 20, replace=False)
    for i in flip:  # distance 255
        w, b = divmod(int(RNG.integers(0, 256)), 32)
        codes[i, w] ^= np.uint32(1 << b)
    K = bf16_round_bits(RNG.standard_normal((n, d)).astype(np.float32))
    V = bf16_round_bits(RNG.standard_normal((n, d)).astype(np.float32))
    for k in (5, 20, 21, 60, n, n + 4):
        oqc, odist, oidx, oout, m = oracle.decode_head(q, W, codes, K, V, n, k, 0.1)
        assert np.array_equal(oqc, qc)
        want = np.full(n, 256, np.int32)
        want[flip] = 255
        assert np.array_equal(odist, want)
        assert oidx.tolist() == brute_topk(want.tolist(), k)
        assert m == min(k, n)
