"""Pins for the float64 oracle: checks that do not re-run the oracle's own code.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError on
a mismatch.  ``test_oracle_pins.py`` runs them against the committed oracle
(all must pass) and ``test_oracle_mutants.py`` runs them against copies of the
oracle with a planted mistake (each mistake must fail at least one pin).

The independent formulations used here:
  * the attended set written as a dense mask over the interleaved sequence
    [chunk 0 raw tokens, gist 0, chunk 1 raw tokens, gist 1, ..., own tokens]
    and a numpy softmax over it (no gather, no per-token list);
  * selection by brute-force enumeration of every k-subset, keeping the one
    with the largest score sum, earliest in lexicographic order on ties;
  * closed forms: all chunks selected = dense attention; k = 0 = compression
    only; a zero query = uniform weights = the mean of the attended values,
    with lse = log(set size);
  * hand-derived examples in ``tests/golden/``.
Sources: gist.science explainers of "Forget, Then Recall ... Gist Sparse
Attention" -- Dutch page "Het Proces" (Compressie, Scoring, Selectie,
Selectieve Ontvouwing, Hierarchische Uitbreiding), Japanese page sections 2.1
and 2.2.
"""
from __future__ import annotations

import itertools
import json
import math
from pathlib import Path

import numpy as np

GOLDEN = Path(__file__).resolve().parent / "golden"


# ----------------------------------------------------------------- helpers
def softmax_attend(q, K, V, mask, scale):
    """Dense masked softmax attention in float64: returns (out, lse, w)."""
    z = scale * (K @ q)
    z = np.where(mask, z, -np.inf)
    Z = z.max()
    e = np.exp(z - Z)
    w = e / e.sum()
    return w @ V, Z + math.log(e.sum()), w


def brute_topk(scores, k):
    """Best k-subset by score sum; first in lexicographic order on ties."""
    n = len(scores)
    k = min(k, n)
    best, best_sum = (), -np.inf
    for sub in itertools.combinations(range(n), k):
        s = float(sum(scores[i] for i in sub))
        if s > best_sum:
            best, best_sum = sub, s
    return set(best)


def interleaved(raw_k, raw_v, gk, gv, N, c, own):
    """Keys/values of the interleaved sequence of one (b, kv head), plus labels."""
    K, V, lab = [], [], []
    for m in range(N):
        for j in range(c):
            K.append(raw_k[m * c + j]); V.append(raw_v[m * c + j]); lab.append(("raw", m))
        K.append(gk[m]); V.append(gv[m]); lab.append(("gist", m))
    for j in range(own):
        K.append(raw_k[N * c + j]); V.append(raw_v[N * c + j]); lab.append(("own", j))
    return np.array(K, dtype=np.float64), np.array(V, dtype=np.float64), lab


def decode_mask(lab, S, exclude):
    return np.array([(kind == "raw" and m in S) or (kind == "gist" and (m in S or not exclude)) or kind == "own"
                     for kind, m in lab])


def rand_decode(rng, B, Hq, Hkv, d, c, N, own, extra_gists=1, dtype="f32"):
    n_max = N + extra_gists
    t_max = n_max * c + c
    arr = {
        "q": rng.standard_normal((B, Hq, d)),
        "gist_k": rng.standard_normal((B, Hkv, n_max, d)),
        "gist_v": rng.standard_normal((B, Hkv, n_max, d)),
        "raw_k": rng.standard_normal((B, Hkv, t_max, d)),
        "raw_v": rng.standard_normal((B, Hkv, t_max, d)),
    }
    arr = {k: v.astype(np.float32) for k, v in arr.items()}
    if dtype == "bf16":
        from oracle import bf16_bits
        arr = {k: bf16_bits(v) for k, v in arr.items()}
    arr["n_gists"] = np.full(B, N, np.int32)
    arr["own_len"] = np.full(B, own, np.int32)
    return arr


def as_f64(a):
    if a.dtype == np.uint16:
        from oracle import bf16_to_f32
        return bf16_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def run_decode(orc, arr, c, k, exclude, **kw):
    return orc.decode(arr["q"], arr["gist_k"], arr["gist_v"], arr["raw_k"], arr["raw_v"], arr["n_gists"],
                      arr["own_len"], chunk=c, topk=k, exclude=exclude, **kw)


def dense_decode_reference(arr, b, h, Hq, Hkv, c, k, exclude, scale=None, S=None):
    """Brute-force selection + dense masked attention for one decode row."""
    d = arr["q"].shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    kvh = h // (Hq // Hkv)
    N, own = int(arr["n_gists"][b]), int(arr["own_len"][b])
    q = as_f64(arr["q"])[b, h]
    gk, gv = as_f64(arr["gist_k"])[b, kvh], as_f64(arr["gist_v"])[b, kvh]
    rk, rv = as_f64(arr["raw_k"])[b, kvh], as_f64(arr["raw_v"])[b, kvh]
    scores = scale * (gk[:N] @ q)
    if S is None:
        S = brute_topk(list(scores), k)
    K, V, lab = interleaved(rk, rv, gk, gv, N, c, own)
    out, lse, _ = softmax_attend(q, K, V, decode_mask(lab, S, exclude), scale)
    return out, lse, S


# ------------------------------------------------------------ decode pins
def pin_decode_bruteforce(orc):
    """Tiny problems: selection = best subset, output = dense masked softmax."""
    rng = np.random.default_rng(11)
    for trial in range(24):
        c = int(rng.integers(1, 4))
        N = int(rng.integers(0, 7))
        k = int(rng.integers(0, 5))
        own = int(rng.integers(1, c + 1))
        Hkv = int(rng.integers(1, 3))
        G = int(rng.integers(1, 3))
        d = int(rng.choice([2, 3, 5]))
        dtype = "bf16" if trial % 3 == 2 else "f32"
        arr = rand_decode(rng, 2, Hkv * G, Hkv, d, c, N, own, dtype=dtype)
        arr["n_gists"][1] = max(0, N - 1)  # ragged batch
        arr["own_len"][1] = 1
        for exclude in (False, True):
            res = run_decode(orc, arr, c, k, exclude)
            for r in range(2 * Hkv * G):
                b, h = divmod(r, Hkv * G)
                out, lse, S = dense_decode_reference(arr, b, h, Hkv * G, Hkv, c, k, exclude)
                got = {int(x) for x in res["sel"][r] if x >= 0}
                assert got == S, (trial, r, got, S)
                np.testing.assert_allclose(res["out"][r], out, rtol=1e-12, atol=1e-12)
                assert abs(res["lse"][r] - lse) < 1e-12


def pin_decode_dense_limit(orc):
    """k >= N: every chunk unfolded, the output is dense attention over the whole sequence."""
    rng = np.random.default_rng(12)
    B, Hq, Hkv, d, c, N, own = 2, 4, 2, 8, 4, 9, 3
    arr = rand_decode(rng, B, Hq, Hkv, d, c, N, own)
    for exclude in (False, True):
        res = run_decode(orc, arr, c, N + 2, exclude)
        for r in range(B * Hq):
            b, h = divmod(r, Hq)
            kvh = h // (Hq // Hkv)
            q = arr["q"][b, h].astype(np.float64)
            K = np.concatenate([arr["raw_k"][b, kvh, : N * c + own], arr["gist_k"][b, kvh, :N]]).astype(np.float64)
            V = np.concatenate([arr["raw_v"][b, kvh, : N * c + own], arr["gist_v"][b, kvh, :N]]).astype(np.float64)
            z = (K @ q) / math.sqrt(d)
            w = np.exp(z - z.max())
            w /= w.sum()
            np.testing.assert_allclose(res["out"][r], w @ V, rtol=1e-12, atol=1e-12)
            assert sorted(res["sel"][r][:N]) == list(range(N)) and (res["sel"][r][N:] == -1).all()


def pin_decode_k0_compression_only(orc):
    """k = 0: all gists + own tokens (default); own tokens only (exclude)."""
    rng = np.random.default_rng(13)
    B, Hq, Hkv, d, c, N, own = 1, 2, 1, 6, 3, 5, 2
    arr = rand_decode(rng, B, Hq, Hkv, d, c, N, own)
    for exclude in (False, True):
        res = run_decode(orc, arr, c, 0, exclude)
        for h in range(Hq):
            q = arr["q"][0, h].astype(np.float64)
            own_k = arr["raw_k"][0, 0, N * c: N * c + own]
            own_v = arr["raw_v"][0, 0, N * c: N * c + own]
            K = own_k if exclude else np.concatenate([arr["gist_k"][0, 0, :N], own_k])
            V = own_v if exclude else np.concatenate([arr["gist_v"][0, 0, :N], own_v])
            z = (K.astype(np.float64) @ q) / math.sqrt(d)
            w = np.exp(z - z.max())
            w /= w.sum()
            np.testing.assert_allclose(res["out"][h], w @ V.astype(np.float64), rtol=1e-12, atol=1e-12)


def pin_decode_zero_query(orc):
    """q = 0: all scores tie, so chunks 0..k-1 are chosen; weights are uniform,
    the output is the plain mean of the attended values and lse = log(set size)."""
    rng = np.random.default_rng(14)
    d, c, N, own, k = 4, 3, 7, 2, 3
    arr = rand_decode(rng, 1, 1, 1, d, c, N, own)
    arr["q"][:] = 0
    for exclude in (False, True):
        res = run_decode(orc, arr, c, k, exclude, set_cap=64)
        assert list(res["sel"][0]) == [0, 1, 2]
        rows = [arr["raw_v"][0, 0, m * c + j] for m in range(k) for j in range(c)]
        gists = list(range(N)) if not exclude else list(range(k))
        rows += [arr["gist_v"][0, 0, m] for m in gists]
        rows += [arr["raw_v"][0, 0, N * c + j] for j in range(own)]
        expect = np.mean(np.array(rows, dtype=np.float64), axis=0)
        np.testing.assert_allclose(res["out"][0], expect, rtol=1e-12, atol=1e-13)
        size = k * (c + 1) + (0 if exclude else N - k) + own
        assert abs(res["lse"][0] - math.log(size)) < 1e-12
        assert res["set_n"][0] == size


def pin_decode_invariants(orc):
    """Weights >= 0 sum to 1; output in the coordinate-wise hull of the attended
    values; consistent chunk permutation leaves the output unchanged; a positive
    score scale leaves the selection unchanged."""
    rng = np.random.default_rng(15)
    B, Hq, Hkv, d, c, N, own, k = 1, 2, 1, 8, 4, 12, 2, 4
    arr = rand_decode(rng, B, Hq, Hkv, d, c, N, own)
    cap = 256
    res = run_decode(orc, arr, c, k, False, set_cap=cap)
    for r in range(Hq):
        n = res["set_n"][r]
        w = res["set_w"][r, :n]
        assert (w >= 0).all() and abs(w.sum() - 1) < 1e-12
        vals = []
        for kind, idx in zip(res["set_kind"][r, :n], res["set_idx"][r, :n]):
            src = arr["raw_v"] if kind == 0 else arr["gist_v"]
            vals.append(src[0, 0, idx])
        vals = np.array(vals, dtype=np.float64)
        assert (res["out"][r] >= vals.min(0) - 1e-12).all() and (res["out"][r] <= vals.max(0) + 1e-12).all()
    # permute whole chunks (raw rows + gist together)
    perm = rng.permutation(N)
    arr2 = {kk: v.copy() for kk, v in arr.items()}
    for new, old in enumerate(perm):
        arr2["gist_k"][:, :, new] = arr["gist_k"][:, :, old]
        arr2["gist_v"][:, :, new] = arr["gist_v"][:, :, old]
        arr2["raw_k"][:, :, new * c:(new + 1) * c] = arr["raw_k"][:, :, old * c:(old + 1) * c]
        arr2["raw_v"][:, :, new * c:(new + 1) * c] = arr["raw_v"][:, :, old * c:(old + 1) * c]
    res2 = run_decode(orc, arr2, c, k, False)
    np.testing.assert_allclose(res2["out"], res["out"], rtol=1e-12, atol=1e-12)
    for r in range(Hq):
        assert {int(perm[x]) for x in res2["sel"][r]} == {int(x) for x in res["sel"][r]}
    res3 = run_decode(orc, arr, c, k, False, scale=0.37)
    assert (res3["sel"] == res["sel"]).all()


def pin_decode_exact_ties(orc):
    """Duplicate gist keys give exactly equal scores; the lower chunk index wins."""
    rng = np.random.default_rng(16)
    d, c, N, own = 4, 2, 6, 1
    arr = rand_decode(rng, 1, 1, 1, d, c, N, own)
    q = arr["q"][0, 0]
    base = q / np.linalg.norm(q)
    for m in (1, 3, 4):
        arr["gist_k"][0, 0, m] = (3 * base).astype(np.float32)  # highest, tied
    for m in (0, 2, 5):
        arr["gist_k"][0, 0, m] = (-3 * base).astype(np.float32)
    res = run_decode(orc, arr, c, 2, False)
    assert list(res["sel"][0]) == [1, 3]
    res = run_decode(orc, arr, c, 4, False)
    assert list(res["sel"][0][:3]) == [1, 3, 4] and res["sel"][0][3] == 0


def pin_decode_gqa_mapping(orc):
    """Query head h reads kv head h // (Hq/Hkv): each head equals a one-head problem."""
    rng = np.random.default_rng(17)
    B, Hq, Hkv, d, c, N, own, k = 1, 6, 2, 4, 2, 5, 1, 2
    arr = rand_decode(rng, B, Hq, Hkv, d, c, N, own)
    res = run_decode(orc, arr, c, k, False)
    for h in range(Hq):
        kvh = h // (Hq // Hkv)
        one = {"q": arr["q"][:, h:h + 1], "n_gists": arr["n_gists"], "own_len": arr["own_len"]}
        for name in ("gist_k", "gist_v", "raw_k", "raw_v"):
            one[name] = arr[name][:, kvh:kvh + 1]
        r1 = run_decode(orc, one, c, k, False)
        np.testing.assert_allclose(res["out"][h], r1["out"][0], rtol=0, atol=0)


def pin_decode_golden(orc):
    """Hand-derived example (tests/golden/decode_hand.json)."""
    _check_golden(orc, json.loads((GOLDEN / "decode_hand.json").read_text()))


# --------------------------------------------------------------- H-GSA pins
def rand_hgsa(rng, B, Hq, Hkv, d, c, N, g, own):
    arr = rand_decode(rng, B, Hq, Hkv, d, c, N, own)
    M = max(1, N // g)
    arr["meta_k"] = rng.standard_normal((B, Hkv, M + 1, d)).astype(np.float32)
    arr["meta_v"] = rng.standard_normal((B, Hkv, M + 1, d)).astype(np.float32)
    return arr


def run_hgsa(orc, arr, c, g, km, k, exclude, **kw):
    return orc.hgsa(arr["q"], arr["meta_k"], arr["meta_v"], arr["gist_k"], arr["gist_v"], arr["raw_k"],
                    arr["raw_v"], arr["n_gists"], arr["own_len"], chunk=c, group=g, topk_meta=km, topk=k,
                    exclude=exclude, **kw)


def pin_hgsa_bruteforce(orc):
    """Meta subsets then child subsets by enumeration; dense mask over raw, gist and meta tokens."""
    rng = np.random.default_rng(21)
    for trial in range(20):
        c = int(rng.integers(1, 3))
        g = int(rng.integers(1, 4))
        N = int(rng.integers(0, 11))
        km = int(rng.integers(0, 4))
        k = int(rng.integers(0, 4))
        own = int(rng.integers(1, c + 1))
        d = 3
        arr = rand_hgsa(rng, 1, 2, 1, d, c, N, g, own)
        M = N // g
        for exclude in (False, True):
            res = run_hgsa(orc, arr, c, g, km, k, exclude)
            for h in range(2):
                q = arr["q"][0, h].astype(np.float64)
                sc = 1 / math.sqrt(d)
                mk, mv = arr["meta_k"][0, 0].astype(np.float64), arr["meta_v"][0, 0].astype(np.float64)
                gk, gv = arr["gist_k"][0, 0].astype(np.float64), arr["gist_v"][0, 0].astype(np.float64)
                rk, rv = arr["raw_k"][0, 0].astype(np.float64), arr["raw_v"][0, 0].astype(np.float64)
                Sm = brute_topk(list(sc * (mk[:M] @ q)), km)
                cand = [m for m in range(N) if m // g >= M or m // g in Sm]
                cs = sc * (gk[cand] @ q) if cand else np.zeros(0)
                S = {cand[i] for i in brute_topk(list(cs), k)}
                K, V, lab = interleaved(rk, rv, gk, gv, N, c, own)
                K = np.concatenate([K, mk[:M]]) if M else K
                V = np.concatenate([V, mv[:M]]) if M else V
                lab = lab + [("meta", j) for j in range(M)]
                mask = np.array([(kind == "raw" and m in S)
                                 or (kind == "gist" and m in cand and (m in S or not exclude))
                                 or kind == "own"
                                 or (kind == "meta" and m not in Sm and not exclude) for kind, m in lab])
                out, lse, _ = softmax_attend(q, K, V, mask, sc)
                assert {int(x) for x in res["meta_sel"][h] if x >= 0} == Sm
                assert {int(x) for x in res["sel"][h] if x >= 0} == S
                np.testing.assert_allclose(res["out"][h], out, rtol=1e-12, atol=1e-12)
                assert abs(res["lse"][h] - lse) < 1e-12


def pin_hgsa_reduces_to_flat(orc):
    """All meta groups chosen -> flat GSA; g = 1 with meta = gist -> flat GSA."""
    rng = np.random.default_rng(22)
    B, Hq, Hkv, d, c, N, g, own, k = 1, 4, 2, 6, 2, 12, 3, 2, 3
    arr = rand_hgsa(rng, B, Hq, Hkv, d, c, N, g, own)
    for exclude in (False, True):
        flat = run_decode(orc, arr, c, k, exclude)
        res = run_hgsa(orc, arr, c, g, N // g, k, exclude)
        np.testing.assert_allclose(res["out"], flat["out"], rtol=1e-12, atol=1e-12)
        assert (res["sel"] == flat["sel"]).all()
        arr1 = dict(arr)
        arr1["meta_k"], arr1["meta_v"] = arr["gist_k"], arr["gist_v"]
        res1 = run_hgsa(orc, arr1, c, 1, k + 2, k, exclude)
        np.testing.assert_allclose(res1["out"], flat["out"], rtol=1e-12, atol=1e-12)


def rand_hgsa2(rng, B, Hq, Hkv, d, c, N, g1, g2, own):
    arr = rand_hgsa(rng, B, Hq, Hkv, d, c, N, g1, own)
    M2 = max(1, (N // g1) // g2)
    arr["meta2_k"] = rng.standard_normal((B, Hkv, M2 + 1, d)).astype(np.float32)
    arr["meta2_v"] = rng.standard_normal((B, Hkv, M2 + 1, d)).astype(np.float32)
    return arr


def run_hgsa2(orc, arr, c, g1, g2, k2, k1, k, exclude, **kw):
    return orc.hgsa2(arr["q"], arr["meta2_k"], arr["meta2_v"], arr["meta_k"], arr["meta_v"], arr["gist_k"],
                     arr["gist_v"], arr["raw_k"], arr["raw_v"], arr["n_gists"], arr["own_len"], chunk=c, group1=g1,
                     group2=g2, topk2=k2, topk1=k1, topk=k, exclude=exclude, **kw)


def pin_hgsa2_bruteforce(orc):
    """Two meta levels: subsets by enumeration at each level (level-2 groups,
    then level-1 children, then gist children); dense mask over raw, gist,
    level-1 and level-2 tokens."""
    rng = np.random.default_rng(23)
    for trial in range(24):
        c = int(rng.integers(1, 3))
        g1, g2 = int(rng.integers(1, 4)), int(rng.integers(1, 4))
        N = int(rng.integers(0, 16))
        k2, k1, k = int(rng.integers(0, 3)), int(rng.integers(0, 4)), int(rng.integers(0, 4))
        own = int(rng.integers(1, c + 1))
        d = 3
        arr = rand_hgsa2(rng, 1, 2, 1, d, c, N, g1, g2, own)
        M1 = N // g1
        M2 = M1 // g2
        for exclude in (False, True):
            res = run_hgsa2(orc, arr, c, g1, g2, k2, k1, k, exclude)
            for h in range(2):
                q = arr["q"][0, h].astype(np.float64)
                sc = 1 / math.sqrt(d)
                m2k, m2v = arr["meta2_k"][0, 0].astype(np.float64), arr["meta2_v"][0, 0].astype(np.float64)
                mk, mv = arr["meta_k"][0, 0].astype(np.float64), arr["meta_v"][0, 0].astype(np.float64)
                gk, gv = arr["gist_k"][0, 0].astype(np.float64), arr["gist_v"][0, 0].astype(np.float64)
                rk, rv = arr["raw_k"][0, 0].astype(np.float64), arr["raw_v"][0, 0].astype(np.float64)
                S2 = brute_topk(list(sc * (m2k[:M2] @ q)), k2)
                cand1 = [j for j in range(M1) if j // g2 >= M2 or j // g2 in S2]
                s1 = sc * (mk[cand1] @ q) if cand1 else np.zeros(0)
                S1 = {cand1[i] for i in brute_topk(list(s1), k1)}
                cand0 = [m for m in range(N) if m // g1 >= M1 or m // g1 in S1]
                s0 = sc * (gk[cand0] @ q) if cand0 else np.zeros(0)
                S0 = {cand0[i] for i in brute_topk(list(s0), k)}
                K, V, lab = interleaved(rk, rv, gk, gv, N, c, own)
                if M1:
                    K, V = np.concatenate([K, mk[:M1]]), np.concatenate([V, mv[:M1]])
                    lab = lab + [("meta", j) for j in range(M1)]
                if M2:
                    K, V = np.concatenate([K, m2k[:M2]]), np.concatenate([V, m2v[:M2]])
                    lab = lab + [("meta2", i) for i in range(M2)]
                mask = np.array([(kind == "raw" and m in S0)
                                 or (kind == "gist" and m in cand0 and (m in S0 or not exclude))
                                 or kind == "own"
                                 or (kind == "meta" and m in cand1 and m not in S1 and not exclude)
                                 or (kind == "meta2" and m not in S2 and not exclude) for kind, m in lab])
                out, lse, _ = softmax_attend(q, K, V, mask, sc)
                assert {int(x) for x in res["meta2_sel"][h] if x >= 0} == S2
                assert {int(x) for x in res["meta_sel"][h] if x >= 0} == S1
                assert {int(x) for x in res["sel"][h] if x >= 0} == S0
                np.testing.assert_allclose(res["out"][h], out, rtol=1e-12, atol=1e-12)
                assert abs(res["lse"][h] - lse) < 1e-12


def pin_hgsa2_reduces_to_one_level(orc):
    """Every level-2 group chosen -> the one-level H-GSA (a separate routine)
    with the same level-1 budget; one level-1 meta per level-2 meta with the
    same keys and values behaves like one level with the budget of level 2."""
    rng = np.random.default_rng(24)
    B, Hq, Hkv, d, c, N, g1, g2, own, k1, k = 1, 4, 2, 6, 2, 24, 3, 2, 2, 3, 4
    arr = rand_hgsa2(rng, B, Hq, Hkv, d, c, N, g1, g2, own)
    M2 = (N // g1) // g2
    for exclude in (False, True):
        one = run_hgsa(orc, arr, c, g1, k1, k, exclude)
        two = run_hgsa2(orc, arr, c, g1, g2, M2, k1, k, exclude)
        np.testing.assert_allclose(two["out"], one["out"], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(two["lse"], one["lse"], rtol=1e-12, atol=1e-12)
        assert (two["sel"] == one["sel"]).all() and (two["meta_sel"] == one["meta_sel"]).all()
        # g2 = 1 and level-2 rows equal to the level-1 rows: level 2 picks the
        # same groups the one-level H-GSA picks, and every level-1 candidate
        # is chosen (k1 = its budget), so the sets coincide
        arr1 = dict(arr)
        arr1["meta2_k"], arr1["meta2_v"] = arr["meta_k"], arr["meta_v"]
        two1 = run_hgsa2(orc, arr1, c, g1, 1, k1, k1, k, exclude)
        np.testing.assert_allclose(two1["out"], one["out"], rtol=1e-12, atol=1e-12)
        assert (two1["sel"] == one["sel"]).all()


def pin_hgsa_golden(orc):
    """Hand-derived example (tests/golden/hgsa_hand.json)."""
    _check_golden(orc, json.loads((GOLDEN / "hgsa_hand.json").read_text()))


# ------------------------------------------------------------- prefill pins
def rand_prefill(rng, B, Hq, Hkv, d, c, N):
    L = N * c
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    return {"q_raw": f(B, Hq, L, d), "k_raw": f(B, Hkv, L, d), "v_raw": f(B, Hkv, L, d),
            "q_gist": f(B, Hq, N, d), "k_gist": f(B, Hkv, N, d), "v_gist": f(B, Hkv, N, d)}


def run_prefill(orc, arr, c, k, exclude, **kw):
    return orc.prefill(arr["q_raw"], arr["k_raw"], arr["v_raw"], arr["q_gist"], arr["k_gist"], arr["v_gist"],
                       chunk=c, topk=k, exclude=exclude, **kw)


def pin_prefill_dense_and_gist_rows(orc):
    """Rows with m <= k completed chunks = dense causal attention over the interleaved
    prefix; gist rows = their own chunk's raw tokens + gists 0..m."""
    rng = np.random.default_rng(31)
    B, Hq, Hkv, d, c, N, k = 1, 2, 1, 4, 3, 6, 2
    arr = rand_prefill(rng, B, Hq, Hkv, d, c, N)
    L = N * c
    sc = 1 / math.sqrt(d)
    for exclude in (False, True):
        res = run_prefill(orc, arr, c, k, exclude)
        for h in range(Hq):
            base = h * (L + N)
            for pos in range(L + N):
                r = base + pos
                if pos < L:
                    m, j = divmod(pos, c)
                    if m > k:
                        continue
                    K = np.concatenate([arr["k_raw"][0, 0, : pos + 1], arr["k_gist"][0, 0, :m]])
                    V = np.concatenate([arr["v_raw"][0, 0, : pos + 1], arr["v_gist"][0, 0, :m]])
                    q = arr["q_raw"][0, h, pos]
                else:
                    m = pos - L
                    K = np.concatenate([arr["k_raw"][0, 0, m * c:(m + 1) * c], arr["k_gist"][0, 0, : m + 1]])
                    V = np.concatenate([arr["v_raw"][0, 0, m * c:(m + 1) * c], arr["v_gist"][0, 0, : m + 1]])
                    q = arr["q_gist"][0, h, m]
                z = sc * (K.astype(np.float64) @ q.astype(np.float64))
                w = np.exp(z - z.max())
                w /= w.sum()
                np.testing.assert_allclose(res["out"][r], w @ V.astype(np.float64), rtol=1e-12, atol=1e-12)


def pin_prefill_bruteforce(orc):
    """Raw rows with m > k: brute-force selection and a dense mask over the prefix."""
    rng = np.random.default_rng(32)
    B, Hq, Hkv, d, c, N, k = 1, 4, 2, 3, 2, 6, 2
    arr = rand_prefill(rng, B, Hq, Hkv, d, c, N)
    L = N * c
    sc = 1 / math.sqrt(d)
    for exclude in (False, True):
        res = run_prefill(orc, arr, c, k, exclude)
        for h in range(Hq):
            kvh = h // (Hq // Hkv)
            for pos in range(L):
                m, j = divmod(pos, c)
                q = arr["q_raw"][0, h, pos].astype(np.float64)
                gk = arr["k_gist"][0, kvh].astype(np.float64)
                S = brute_topk(list(sc * (gk[:m] @ q)), k)
                K, V, lab = interleaved(arr["k_raw"][0, kvh].astype(np.float64), arr["v_raw"][0, kvh].astype(np.float64),
                                        gk, arr["v_gist"][0, kvh].astype(np.float64), m, c, j + 1)
                out, lse, _ = softmax_attend(q, K, V, decode_mask(lab, S, exclude), sc)
                r = h * (L + N) + pos
                assert {int(x) for x in res["sel"][r] if x >= 0} == S
                np.testing.assert_allclose(res["out"][r], out, rtol=1e-12, atol=1e-12)


def pin_prefill_large_k(orc):
    """k above 16 (the GPU's wide scorer): rows with m > k against brute-force
    selection and the dense mask, with k close to the number of chunks."""
    rng = np.random.default_rng(33)
    B, Hq, Hkv, d, c, N, k = 1, 2, 1, 3, 2, 26, 21
    arr = rand_prefill(rng, B, Hq, Hkv, d, c, N)
    L = N * c
    sc = 1 / math.sqrt(d)
    rows = [h * (L + N) + pos for h in range(Hq) for pos in range((k + 1) * c, L)]
    for exclude in (False, True):
        res = run_prefill(orc, arr, c, k, exclude, rows=rows)
        for i, r in enumerate(rows):
            h, pos = divmod(r, L + N)
            m, j = divmod(pos, c)
            q = arr["q_raw"][0, h, pos].astype(np.float64)
            gk = arr["k_gist"][0, 0].astype(np.float64)
            S = brute_topk(list(sc * (gk[:m] @ q)), k)
            K, V, lab = interleaved(arr["k_raw"][0, 0].astype(np.float64), arr["v_raw"][0, 0].astype(np.float64),
                                    gk, arr["v_gist"][0, 0].astype(np.float64), m, c, j + 1)
            out, lse, _ = softmax_attend(q, K, V, decode_mask(lab, S, exclude), sc)
            assert {int(x) for x in res["sel"][i] if x >= 0} == S
            np.testing.assert_allclose(res["out"][i], out, rtol=1e-12, atol=1e-12)


def pin_prefill_golden(orc):
    """Hand-derived example (tests/golden/prefill_hand.json)."""
    _check_golden(orc, json.loads((GOLDEN / "prefill_hand.json").read_text()))


# ------------------------------------------------------------- golden files
def _arr(x, dtype=np.float32):
    return np.array(x, dtype=dtype)


def _expected_from_logits(tokens):
    """out = sum e^z v / sum e^z and lse = log sum e^z over the listed tokens."""
    z = np.array([t["logit"] for t in tokens], dtype=np.float64)
    v = np.array([t["value"] for t in tokens], dtype=np.float64)
    e = np.exp(z)
    return (e @ v) / e.sum(), math.log(e.sum())


def _check_golden(orc, G):
    kind = G["kind"]
    for case in G["cases"]:
        inp = {k: _arr(v) for k, v in G["inputs"].items()}
        p = dict(G["params"], **case.get("params", {}))
        if kind == "decode":
            inp["n_gists"] = _arr(G["n_gists"], np.int32)
            inp["own_len"] = _arr(G["own_len"], np.int32)
            res = run_decode(orc, inp, p["chunk"], p["topk"], p["exclude"], scale=p["scale"])
            row = 0
        elif kind == "hgsa":
            inp["n_gists"] = _arr(G["n_gists"], np.int32)
            inp["own_len"] = _arr(G["own_len"], np.int32)
            res = run_hgsa(orc, inp, p["chunk"], p["group"], p["topk_meta"], p["topk"], p["exclude"], scale=p["scale"])
            row = 0
            assert [int(x) for x in res["meta_sel"][0]] == case["meta_selection"]
        else:
            res = run_prefill(orc, inp, p["chunk"], p["topk"], p["exclude"], scale=p["scale"], rows=[case["row"]])
            row = 0
        assert [int(x) for x in res["sel"][row]] == case["selection"], (case["name"], res["sel"][row])
        out, lse = _expected_from_logits(case["tokens"])
        np.testing.assert_allclose(res["out"][row], out, rtol=1e-13, atol=1e-14, err_msg=case["name"])
        assert abs(res["lse"][row] - lse) < 1e-13, case["name"]


# ------------------------------------------------------------ selection alone
def pin_topk_selection(orc):
    """Selection on given scores: the chosen set is the brute-force best
    subset on tiny rows; on larger tie-heavy rows every chosen entry
    outranks every other by (score desc, index asc); output in ascending
    index order, -1 / -inf padded; k >= n keeps all, k = 0 keeps none."""
    rng = np.random.default_rng(5)
    for trial in range(40):
        n = int(rng.integers(0, 8))
        k = int(rng.integers(0, 6))
        sc = rng.integers(0, 4, size=(1, 8)).astype(np.float64) * 0.5  # many exact ties
        sel, ssc = orc.topk(sc, [n], k)
        want = brute_topk(list(sc[0, :n]), k)
        got = [int(x) for x in sel[0] if x >= 0]
        assert set(got) == want, (trial, got, want)
        assert got == sorted(got) and len(got) == min(k, n)
        assert all(int(x) == -1 for x in sel[0][len(got):])
        assert all(ssc[0, i] == sc[0, got[i]] for i in range(len(got)))
        assert all(ssc[0, i] == -np.inf for i in range(len(got), k))
    for n, k, levels in ((300, 17, 5), (1000, 64, 1000), (50, 50, 3), (64, 80, 2)):
        sc = rng.integers(0, levels, size=(3, n)).astype(np.float64)
        nv = [n, n // 2, 0]
        sel, _ = orc.topk(sc, nv, k)
        for r in range(3):
            got = [int(x) for x in sel[r] if x >= 0]
            assert got == sorted(got) and len(got) == min(k, nv[r])
            chosen = set(got)
            rest = [m for m in range(nv[r]) if m not in chosen]
            if got and rest:
                worst = min(got, key=lambda m: (sc[r, m], -m))     # lowest-ranked chosen
                best = max(rest, key=lambda m: (sc[r, m], -m))     # highest-ranked other
                assert (sc[r, worst], -worst) > (sc[r, best], -best)
    sel, _ = orc.topk(np.zeros((1, 10)), [10], 4)
    assert [int(x) for x in sel[0]] == [0, 1, 2, 3]  # all equal: the lowest indices


def pin_topp_selection(orc):
    """Top-p against closed forms: uniform scores need ceil(p*n) chunks (the
    lowest indices); scores -i*ln2 give masses 2^-i, so the count has a closed
    form; p >= 1 keeps min(k, n); a dominant chunk alone covers p below its
    mass; a constant shift of the scores changes nothing; the set is always
    the rank-order prefix of that length (the top-k set of the same size)."""
    rng = np.random.default_rng(9)
    # uniform: p = 0.5 of n = 4 is exactly two chunks (masses 1/4 are exact)
    r = orc.topp(np.zeros((1, 4)), [4], 4, 0.5)
    assert r["count"][0] == 2 and [int(x) for x in r["sel"][0][:2]] == [0, 1]
    for n, pp in ((10, 0.35), (64, 0.26), (7, 0.99)):
        r = orc.topp(np.zeros((1, n)), [n], n, pp)
        want = math.ceil(pp * n)
        assert r["count"][0] == want and [int(x) for x in r["sel"][0][:want]] == list(range(want)), (n, pp, r["count"])
    # geometric: mass of the first m chunks = (1 - 2^-m) / (1 - 2^-n)
    n = 20
    sc = -np.arange(n) * math.log(2.0)
    perm = rng.permutation(n)
    for pp in (0.3, 0.6, 0.9, 0.999):
        want = next(m for m in range(1, n + 1) if (1 - 2.0 ** -m) / (1 - 2.0 ** -n) >= pp)
        r = orc.topp(sc[perm][None, :], [n], n, pp)
        assert r["count"][0] == want, (pp, r["count"][0], want)
        assert sorted(int(x) for x in r["sel"][0][:want]) == sorted(int(np.where(perm == i)[0][0]) for i in range(want))
        assert r["mass_lo"][0] < pp <= r["mass_hi"][0]
    # p >= 1, the cap k, and a dominant chunk
    r = orc.topp(rng.standard_normal((2, 30)), [30, 12], 16, 1.0)
    assert list(r["count"]) == [16, 12]
    sc = rng.standard_normal((1, 50))
    sc[0, 17] = 40.0
    r = orc.topp(sc, [50], 8, 0.9)
    assert r["count"][0] == 1 and r["sel"][0][0] == 17
    # shift invariance (also keeps large scores finite) and the prefix property
    sc = rng.standard_normal((3, 200)) * 3
    a = orc.topp(sc, [200, 150, 1], 64, 0.7)
    b = orc.topp(sc + 1000.0, [200, 150, 1], 64, 0.7)
    assert np.array_equal(a["sel"], b["sel"]) and np.array_equal(a["count"], b["count"])
    assert a["count"][2] == 1
    for r_ in range(2):
        c = int(a["count"][r_])
        t, _ = orc.topk(sc[r_:r_ + 1], [[200, 150][r_]], c)
        assert [int(x) for x in a["sel"][r_][:c]] == [int(x) for x in t[0]]


def pin_decode_backward(orc):
    """Gradients of L = sum(g * out) for a fixed selection: central finite
    differences of the forward oracle in every input; a single attended
    token gives d_q = 0, d_v = g, d_k = 0; the value gradients sum to g."""
    rng = np.random.default_rng(31)
    B, Hq, Hkv, d, c, N, own, k = 1, 2, 1, 4, 2, 6, 2, 2
    for exclude in (False, True):
        arr = rand_decode(rng, B, Hq, Hkv, d, c, N, own)
        sel = np.array([[1, 4], [3, -1]], np.int32)
        g = rng.standard_normal((B, Hq, d))
        grads = orc.decode_backward(arr["q"], arr["gist_k"], arr["gist_v"], arr["raw_k"], arr["raw_v"],
                                    arr["n_gists"], arr["own_len"], sel, g, chunk=c, topk=k, exclude=exclude)

        def loss(a2):
            r = run_decode(orc, a2, c, k, exclude, sel_in=sel)
            return float((r["out"] * g.reshape(B * Hq, d)).sum())

        eps = 1e-2
        for key, gkey in (("q", "d_q"), ("gist_k", "d_gist_k"), ("gist_v", "d_gist_v"), ("raw_k", "d_raw_k"),
                          ("raw_v", "d_raw_v")):
            flat = arr[key].reshape(-1)
            for _ in range(6):
                i = int(rng.integers(0, flat.size))
                a_p, a_m = dict(arr), dict(arr)
                a_p[key] = flat.copy()
                a_p[key][i] += eps
                a_p[key] = a_p[key].reshape(arr[key].shape)
                a_m[key] = flat.copy()
                a_m[key][i] -= eps
                a_m[key] = a_m[key].reshape(arr[key].shape)
                # the inputs are float32: use the perturbation actually stored
                h = float(a_p[key].reshape(-1)[i]) - float(a_m[key].reshape(-1)[i])
                fd = (loss(a_p) - loss(a_m)) / h
                an = grads[gkey].reshape(-1)[i]
                assert abs(fd - an) <= 1e-4 + 2e-3 * abs(an), (exclude, key, i, fd, an)
        # the value gradients of a row sum to its g (softmax weights sum to 1); one kv head here
        total_v = grads["d_gist_v"].sum(axis=(0, 1, 2)) + grads["d_raw_v"].sum(axis=(0, 1, 2))
        np.testing.assert_allclose(total_v, g.sum(axis=(0, 1)), rtol=1e-12, atol=1e-12)
    # a single attended token: the own row alone
    arr = rand_decode(rng, 1, 1, 1, 3, 2, 0, 1)
    g = rng.standard_normal((1, 1, 3))
    gr = orc.decode_backward(arr["q"], arr["gist_k"], arr["gist_v"], arr["raw_k"], arr["raw_v"], arr["n_gists"],
                             arr["own_len"], np.zeros((1, 0), np.int32), g, chunk=2, topk=0)
    assert np.abs(gr["d_q"]).max() < 1e-15 and np.abs(gr["d_raw_k"]).max() < 1e-15
    np.testing.assert_allclose(gr["d_raw_v"][0, 0, 0], g[0, 0], rtol=0, atol=1e-15)


def pin_gist_step_is_prefill_gist_row(orc):
    """The gist-position step at chunk completion equals the prefill oracle's
    gist row N of the same sequence: chunk N's raw tokens plus gists 0..N,
    the new gist (k_new, v_new) being gist N ([nl] Compressie)."""
    rng = np.random.default_rng(41)
    Hq, Hkv, d, c = 4, 2, 5, 3
    for N in (0, 1, 4):
        arr = rand_decode(rng, 1, Hq, Hkv, d, c, N, c)
        k_new = rng.standard_normal((1, Hkv, d)).astype(np.float32)
        v_new = rng.standard_normal((1, Hkv, d)).astype(np.float32)
        res = orc.gist_step(arr["q"], k_new, v_new, arr["gist_k"], arr["gist_v"], arr["raw_k"], arr["raw_v"],
                            arr["n_gists"], arr["own_len"], chunk=c)
        Np, L = N + 1, (N + 1) * c
        q_raw = rng.standard_normal((1, Hq, L, d)).astype(np.float32)
        q_gist = rng.standard_normal((1, Hq, Np, d)).astype(np.float32)
        q_gist[:, :, N] = arr["q"]
        k_gist = np.concatenate([arr["gist_k"][:, :, :N], k_new[:, :, None]], axis=2)
        v_gist = np.concatenate([arr["gist_v"][:, :, :N], v_new[:, :, None]], axis=2)
        rows = [h * (L + Np) + L + N for h in range(Hq)]
        pf = orc.prefill(q_raw, arr["raw_k"][:, :, :L].copy(), arr["raw_v"][:, :, :L].copy(), q_gist, k_gist, v_gist,
                         chunk=c, topk=1, rows=rows)
        np.testing.assert_allclose(res["out"], pf["out"], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(res["lse"], pf["lse"], rtol=1e-12, atol=1e-12)


def pin_gist_step_closed_form(orc):
    """Dense softmax over the written-out set, including a partial own chunk
    and GQA heads sharing a kv head; the weights of the set sum to one, so a
    constant value row is returned unchanged."""
    rng = np.random.default_rng(42)
    Hq, Hkv, d, c = 4, 2, 3, 4
    for N, own in ((0, 4), (2, 1), (3, 4)):
        arr = rand_decode(rng, 2, Hq, Hkv, d, c, N, own)
        k_new = rng.standard_normal((2, Hkv, d)).astype(np.float32)
        v_new = rng.standard_normal((2, Hkv, d)).astype(np.float32)
        res = orc.gist_step(arr["q"], k_new, v_new, arr["gist_k"], arr["gist_v"], arr["raw_k"], arr["raw_v"],
                            arr["n_gists"], arr["own_len"], chunk=c)
        for b in range(2):
            for h in range(Hq):
                kv = h // (Hq // Hkv)
                K = np.concatenate([arr["gist_k"][b, kv, :N], arr["raw_k"][b, kv, N * c:N * c + own],
                                    k_new[b, kv][None]]).astype(np.float64)
                V = np.concatenate([arr["gist_v"][b, kv, :N], arr["raw_v"][b, kv, N * c:N * c + own],
                                    v_new[b, kv][None]]).astype(np.float64)
                z = (K @ arr["q"][b, h].astype(np.float64)) / math.sqrt(d)
                w = np.exp(z - z.max())
                np.testing.assert_allclose(res["out"][b * Hq + h], (w / w.sum()) @ V, rtol=1e-12, atol=1e-12)
                assert abs(res["lse"][b * Hq + h] - (z.max() + math.log(w.sum()))) < 1e-12
        const = {k: np.full_like(v, 0.75) for k, v in arr.items() if k in ("gist_v", "raw_v")}
        r2 = orc.gist_step(arr["q"], k_new, np.full_like(v_new, 0.75), arr["gist_k"], const["gist_v"], arr["raw_k"],
                           const["raw_v"], arr["n_gists"], arr["own_len"], chunk=c)
        np.testing.assert_allclose(r2["out"], 0.75, rtol=0, atol=1e-14)


def pin_multiquery_bruteforce(orc):
    """Multi-query selection against a shared cache: per query, the k
    highest scale*q.k over all N gists by (score desc, index asc), found by
    sorting in numpy; GQA heads read their group's kv head; exact ties go
    to the lower index."""
    rng = np.random.default_rng(43)
    B, Hq, Hkv, Q, N, d, k = 2, 4, 2, 3, 9, 4, 3
    q = rng.standard_normal((B, Hq, Q, d)).astype(np.float32)
    gk = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    gk[1, 0, 2] = 10.0 * gk[1, 0, 2] / np.linalg.norm(gk[1, 0, 2])
    gk[1, 0, 5] = gk[1, 0, 2]  # an exact tie between two gists of one kv head
    res = orc.multiquery_select(q, gk, topk=k)
    for b in range(B):
        for h in range(Hq):
            kv = h // (Hq // Hkv)
            for i in range(Q):
                s = (gk[b, kv].astype(np.float64) @ q[b, h, i].astype(np.float64)) / math.sqrt(d)
                order = np.lexsort((np.arange(N), -s))[:k]
                r = (b * Hq + h) * Q + i
                assert list(res["sel"][r]) == order.tolist(), (b, h, i)  # rank order
                np.testing.assert_allclose(res["scores"][r], s, rtol=1e-12, atol=1e-12)
    # the tie (the top score of a query along the tied key): the lower index wins when only one fits
    q1 = np.zeros((1, 1, 1, d), np.float32)
    q1[0, 0, 0] = gk[1, 0, 2]
    r1 = orc.multiquery_select(q1, gk[1:2, :1], topk=1)
    assert list(r1["sel"][0]) == [2]


DECODE_PINS = [pin_decode_bruteforce, pin_decode_dense_limit, pin_decode_k0_compression_only,
               pin_decode_zero_query, pin_decode_invariants, pin_decode_exact_ties, pin_decode_gqa_mapping,
               pin_decode_golden, pin_decode_backward, pin_gist_step_is_prefill_gist_row,
               pin_gist_step_closed_form, pin_multiquery_bruteforce]
HGSA_PINS = [pin_hgsa_bruteforce, pin_hgsa_reduces_to_flat, pin_hgsa_golden, pin_hgsa2_bruteforce,
             pin_hgsa2_reduces_to_one_level]
PREFILL_PINS = [pin_prefill_dense_and_gist_rows, pin_prefill_bruteforce, pin_prefill_large_k, pin_prefill_golden]
ALL_PINS = [pin_topk_selection, pin_topp_selection] + DECODE_PINS + HGSA_PINS + PREFILL_PINS
