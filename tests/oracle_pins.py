"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError on a
mismatch.  They are run against the committed oracle (test_oracle_pins.py) and
against copies with planted mistakes (test_oracle_mutants.py), which must fail
at least one of them.

What pins what:
  * topk: a hand-worked example (tests/golden), closed forms (equal logits ->
    1/k or 1/E; two experts -> the logistic function, evaluated through tanh),
    brute force over every k-subset for E <= 8 on tie-heavy inputs, the
    logits-not-probabilities selection rule, overflow safety, invariants.
  * align: hand-worked examples, the page-pinned all-duplicate tile ownership,
    the all-remote rank, the decode route patterns, equality with a stable
    library sort, padding invariants.
  * gather: the hand-worked example, row identity invariants, zero-pad rule.
  * combine: the hand-worked example, the identity (unit total weight) cases,
    the error bound against exact rational accumulation, remote dropping.
"""
from __future__ import annotations

import itertools
import json
import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------- helpers --
def f32_to_bf16_bits(x) -> np.ndarray:
    """Round float32 values to bf16 (nearest-even), returned as uint16 bits (test-side input maker)."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    return r


def bf16_bits_to_f32(b) -> np.ndarray:
    b = np.ascontiguousarray(np.asarray(b, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32)


def ordered_int32(x: np.ndarray) -> np.ndarray:
    """Map float32 to integers whose order and differences count ulps (+0 and -0 both map to 0)."""
    i = np.asarray(x, np.float32).view(np.int32).astype(np.int64)
    return np.where(i < 0, -(i & 0x7FFFFFFF), i)


def ordered_bf16(bits: np.ndarray) -> np.ndarray:
    i = np.asarray(bits, np.uint16).astype(np.int64)
    return np.where(i >= 0x8000, -(i & 0x7FFF), i)


def rank1_of_4_map(E_global: int = 160, E_local: int = 40, rank: int = 1) -> np.ndarray:
    m = np.full(E_global, -1, np.int32)
    m[rank * E_local:(rank + 1) * E_local] = np.arange(E_local, dtype=np.int32)
    return m


def load_golden(name: str) -> dict:
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _better(xa, ia, xb, ib) -> bool:
    """Total order of the selection: larger logit first, lower index first among equals."""
    return xa > xb or (xa == xb and ia < ib)


def brute_force_topk(row: np.ndarray, k: int):
    """The unique k-subset whose every member beats every non-member, in selection order."""
    E = len(row)
    found = None
    for S in itertools.combinations(range(E), k):
        rest = [e for e in range(E) if e not in S]
        if all(_better(row[a], a, row[b], b) for a in S for b in rest):
            assert found is None, "two dominating subsets"
            found = S
    assert found is not None
    # order inside the subset by the same total order (bubble by pairwise comparisons)
    order = list(found)
    for i in range(len(order)):
        for j in range(len(order) - 1 - i):
            a, b = order[j], order[j + 1]
            if _better(row[b], b, row[a], a):
                order[j], order[j + 1] = b, a
    return order


# -------------------------------------------------------------------- topk --
def pin_topk_hand_example(orc) -> None:
    g = load_golden("topk_softmax_hand_example.json")
    logits = np.array(g["logits"], np.float32)
    for bits in (False, True):
        x = f32_to_bf16_bits(logits) if bits else logits
        w, ids = orc.topk_softmax(x, g["k"], renormalize=False)
        assert ids.tolist() == g["ids"], ids
        getcontext().prec = 40
        want = np.array([[np.float32(float(Decimal(v))) for v in row] for row in g["weights_no_renorm_decimal"]],
                        np.float32)
        assert np.array_equal(w, want), (w, want)
        w, ids = orc.topk_softmax(x, g["k"], renormalize=True)
        assert ids.tolist() == g["ids"]
        assert np.array_equal(w, np.array(g["weights_renorm"], np.float32)), w


def pin_topk_equal_logits(orc) -> None:
    for E in (1, 3, 8, 60, 128):
        for k in sorted(v for v in {1, 2, 4, E} if v <= E):
            for c in (0.0, -3.5, 2.25):
                x = np.full((3, E), c, np.float32)
                w, ids = orc.topk_softmax(x, k, renormalize=False)
                assert (ids == np.arange(k)).all(), ids
                assert (w == np.float32(1.0 / E)).all(), (w, 1.0 / E)
                w, ids = orc.topk_softmax(f32_to_bf16_bits(x), k, renormalize=True)
                assert (ids == np.arange(k)).all()
                assert (w == np.float32(1.0 / k)).all(), (w, 1.0 / k)


def pin_topk_two_expert_logistic(orc) -> None:
    """E=2 softmax is the logistic function: p(top) = (1 + tanh(d/2)) / 2 for a logit gap d."""
    rng = np.random.default_rng(11)
    gaps = np.concatenate([[0.5, 1.0, 3.0, 10.0, 0.0078125], rng.uniform(0.01, 12, 40)]).astype(np.float32)
    for d in gaps:
        for order in (0, 1):
            row = np.array([0.0, d] if order == 0 else [d, 0.0], np.float32)
            w, ids = orc.topk_softmax(row[None, :], 2, renormalize=False)
            top = 1 if order == 0 else 0
            assert ids[0].tolist() == [top, 1 - top], (row, ids)
            hi = (1.0 + math.tanh(float(d) / 2.0)) / 2.0
            lo = (1.0 - math.tanh(float(d) / 2.0)) / 2.0
            for got, want in ((w[0, 0], hi), (w[0, 1], lo)):
                err = abs(int(ordered_int32(np.float32(got))) - int(ordered_int32(np.float32(want))))
                assert err <= 1, (d, got, want)


def pin_topk_brute_force(orc) -> None:
    rng = np.random.default_rng(7)
    for E in range(1, 9):
        for k in range(1, E + 1):
            # tie-heavy rows (values in {0,1,2,3}) and continuous rows
            rows = np.concatenate([rng.integers(0, 4, size=(12, E)).astype(np.float32),
                                   rng.standard_normal((4, E)).astype(np.float32)])
            bits = f32_to_bf16_bits(rows)
            vals = bf16_bits_to_f32(bits)
            _, ids = orc.topk_softmax(bits, k, renormalize=True)
            for t in range(rows.shape[0]):
                assert ids[t].tolist() == brute_force_topk(vals[t], k), (vals[t], k, ids[t])


def pin_topk_selects_on_logits(orc) -> None:
    """Two logits that differ by less than the fp32 resolution of their probabilities: the larger logit wins."""
    tiny = np.float32(2.0 ** -30)
    x = np.array([[0.0, tiny], [tiny, 0.0]], np.float32)
    w, ids = orc.topk_softmax(x, 1, renormalize=False)
    assert ids[:, 0].tolist() == [1, 0], ids
    w2, _ = orc.topk_softmax(x, 2, renormalize=False)
    assert w2[0, 0] == w2[0, 1]  # the rounded probabilities do tie


def pin_topk_overflow_and_shift(orc) -> None:
    # the maximum is not the first entry, so a missing max-subtraction overflows exp
    base = np.array([[-998.0, 0.0, 1.0, 2.0], [0.0, -1.0, 1.0, 2.0]], np.float32)
    for renorm in (False, True):
        w0, i0 = orc.topk_softmax(base, 3, renorm)
        w1, i1 = orc.topk_softmax(base + np.float32(998.0), 3, renorm)  # shift is exact for these integers
        assert np.isfinite(w1).all()
        assert np.array_equal(i0, i1) and np.array_equal(w0, w1), (w0, w1)


def pin_topk_invariants(orc) -> None:
    rng = np.random.default_rng(3)
    for E, k in ((8, 2), (60, 4), (128, 8), (160, 6), (256, 8), (33, 33)):
        x = (rng.standard_normal((50, E)) * 2).astype(np.float32)
        wr, ir = orc.topk_softmax(x, k, True)
        wn, inn = orc.topk_softmax(x, k, False)
        assert np.array_equal(ir, inn)
        assert (np.diff(wr, axis=1) <= 0).all() and (np.diff(wn, axis=1) <= 0).all()
        assert (np.abs(wr.astype(np.float64).sum(1) - 1.0) <= k * 2.0 ** -24).all()
        if k < E:
            assert (wn <= wr).all()
        for t in range(x.shape[0]):
            assert len(set(ir[t].tolist())) == k
        if k == E:  # renormalising over every expert changes nothing (up to one rounding)
            assert (np.abs(ordered_int32(wr) - ordered_int32(wn)) <= 1).all()


TOPK_PINS = [pin_topk_hand_example, pin_topk_equal_logits, pin_topk_two_expert_logistic, pin_topk_brute_force,
             pin_topk_selects_on_logits, pin_topk_overflow_and_shift, pin_topk_invariants]


# ------------------------------------------------------------ sigmoid topk --
def _sigmoid_tanh(x: float) -> float:
    """The logistic function through tanh: (1 + tanh(x/2)) / 2 (an independent evaluation)."""
    return (1.0 + math.tanh(x / 2.0)) / 2.0


def pin_sigmoid_closed_forms(orc) -> None:
    # sigmoid(0) = 1/2 and sigmoid(ln 3) = 3/4; an expert alone with renormalisation weighs 1
    x = np.array([[0.0, -2.0, -3.0], [math.log(3.0), 0.0, -1.0]], np.float32)
    w, ids = orc.topk_sigmoid(x, 1, renormalize=False)
    assert ids[:, 0].tolist() == [0, 0]
    assert w[0, 0] == np.float32(0.5)
    assert abs(int(ordered_int32(w[1:2, 0])[0]) - int(ordered_int32(np.float32(_sigmoid_tanh(float(x[1, 0]))))))<= 1
    w, _ = orc.topk_sigmoid(x, 1, renormalize=True)
    assert (w == np.float32(1.0)).all(), w
    # far tails: no NaN, 0 and 1
    x = np.array([[-1000.0, 1000.0, 0.0]], np.float32)
    w, ids = orc.topk_sigmoid(x, 3, renormalize=False)
    assert ids[0].tolist() == [1, 2, 0] and w[0].tolist() == [1.0, 0.5, 0.0], w


def pin_sigmoid_tanh_identity(orc) -> None:
    rng = np.random.default_rng(21)
    x = (rng.standard_normal((40, 24)) * 4).astype(np.float32)
    for bits in (False, True):
        xin = f32_to_bf16_bits(x) if bits else x
        vals = bf16_bits_to_f32(xin) if bits else x
        w, ids = orc.topk_sigmoid(xin, 5, renormalize=False)
        for t in range(x.shape[0]):
            for j in range(5):
                want = np.float32(_sigmoid_tanh(float(vals[t, ids[t, j]])))
                assert abs(int(ordered_int32(w[t:t + 1, j])[0]) - int(ordered_int32(want))) <= 1, (t, j)
        wr, idr = orc.topk_sigmoid(xin, 5, renormalize=True)
        assert np.array_equal(ids, idr)
        # renormalised: the ratio of two weights is the ratio of their scores
        for t in range(x.shape[0]):
            s = np.array([_sigmoid_tanh(float(vals[t, e])) for e in ids[t]])
            want = (s / s.sum()).astype(np.float32)
            assert (np.abs(ordered_int32(wr[t]) - ordered_int32(want)) <= 2).all(), (wr[t], want)


def pin_sigmoid_symmetry_and_equal_logits(orc) -> None:
    # sigmoid(d) + sigmoid(-d) = 1: with k = 2 over [d, -d] the raw and renormalised weights agree
    for d in (0.25, 1.0, 3.5, 7.0):
        x = np.array([[d, -d], [-d, d]], np.float32)
        wn, idn = orc.topk_sigmoid(x, 2, renormalize=False)
        wr, idr = orc.topk_sigmoid(x, 2, renormalize=True)
        assert idn.tolist() == [[0, 1], [1, 0]] and np.array_equal(idn, idr)
        assert (np.abs(ordered_int32(wn) - ordered_int32(wr)) <= 1).all(), (wn, wr)
        assert abs(float(wn[0].astype(np.float64).sum()) - 1.0) <= 2.0 ** -23
    for E, k in ((8, 2), (60, 4), (160, 6)):
        x = np.full((2, E), -1.25, np.float32)
        w, ids = orc.topk_sigmoid(x, k, renormalize=True)
        assert (ids == np.arange(k)).all() and (w == np.float32(1.0 / k)).all(), w


def pin_sigmoid_selection_is_the_softmax_selection(orc) -> None:
    rng = np.random.default_rng(23)
    for E in range(1, 9):
        for k in range(1, E + 1):
            rows = np.concatenate([rng.integers(0, 4, size=(8, E)).astype(np.float32),
                                   rng.standard_normal((4, E)).astype(np.float32)])
            bits = f32_to_bf16_bits(rows)
            vals = bf16_bits_to_f32(bits)
            _, ids = orc.topk_sigmoid(bits, k, renormalize=False)
            for t in range(rows.shape[0]):
                assert ids[t].tolist() == brute_force_topk(vals[t], k), (vals[t], k, ids[t])


SIGMOID_PINS = [pin_sigmoid_closed_forms, pin_sigmoid_tanh_identity, pin_sigmoid_symmetry_and_equal_logits,
                pin_sigmoid_selection_is_the_softmax_selection]


# ------------------------------------------------------------------- align --
def _resolve_map(spec, E_global, E_local):
    if spec is None:
        return None
    if spec == "rank1_of_4":
        return rank1_of_4_map(E_global, E_local, 1)
    return np.array(spec, np.int32)


def check_align_invariants(res: dict, topk_ids: np.ndarray, E_global: int, block_size: int,
                           expert_map=None, E_local=None) -> None:
    """Everything the align outputs must satisfy, checked without re-deriving them."""
    ids = np.asarray(topk_ids, np.int64).reshape(-1)
    T, k = np.asarray(topk_ids).shape
    P = T * k
    E_local = E_global if E_local is None else E_local
    bs = block_size
    le = np.full(P, -1, np.int64)
    ok = (ids >= 0) & (ids < E_global)
    if expert_map is None:
        le[ok] = ids[ok]
    else:
        le[ok] = np.asarray(expert_map, np.int64)[ids[ok]]
    le[le >= E_local] = -1
    local = np.nonzero(le >= 0)[0]

    counts, offsets = res["counts"], res["offsets"]
    sti, eids, inv = res["sorted_token_ids"], res["expert_ids"], res["inv_perm"]
    npad = int(res["num_tokens_post_pad"][0])
    C = P + E_local * (bs - 1)
    assert len(sti) == C and len(eids) == -(-C // bs) and len(inv) == P
    assert counts.sum() == len(local)
    assert np.array_equal(counts, np.bincount(le[local], minlength=E_local)[:E_local])
    assert offsets[0] == 0 and offsets[-1] == npad and npad % bs == 0 and npad <= C
    width = np.diff(offsets.astype(np.int64))
    assert (width % bs == 0).all()
    assert (width >= counts).all() and (width < counts + bs).all()
    assert ((width == 0) == (counts == 0)).all()
    # every local slot sits once, in its expert's range, and inv_perm points back at it
    rows = inv[local]
    assert (rows >= 0).all() and len(set(rows.tolist())) == len(local)
    assert np.array_equal(sti[rows], local)
    assert (inv[le < 0] == -1).all()
    assert ((rows >= offsets[le[local]]) & (rows < offsets[le[local]] + counts[le[local]])).all()
    # everything else is the pad value
    pad = np.ones(C, bool)
    pad[rows] = False
    assert (sti[pad] == P).all()
    # stability: ascending s within every expert
    for e in range(E_local):
        seg = sti[offsets[e]:offsets[e] + counts[e]]
        assert (np.diff(seg) > 0).all()
    # one expert per block, -1 past N_pad
    nvalid = npad // bs
    assert (eids[nvalid:] == -1).all()
    for b in range(nvalid):
        e = eids[b]
        assert offsets[e] <= b * bs < offsets[e + 1]


def pin_align_hand_examples(orc) -> None:
    g = load_golden("align_hand_examples.json")
    for ex in g["examples"]:
        emap = _resolve_map(ex["expert_map"], ex["E_global"], ex["E_local"])
        ids = np.array(ex["topk_ids"], np.int32)
        r = orc.align_permute(ids, ex["E_global"], ex["block_size"], emap, ex["E_local"])
        assert int(r["num_tokens_post_pad"][0]) == ex["num_tokens_post_pad"], ex["name"]
        assert r["inv_perm"].tolist() == ex["inv_perm"], (ex["name"], r["inv_perm"])
        if "counts" in ex:
            assert r["counts"].tolist() == ex["counts"], ex["name"]
            assert r["offsets"].tolist() == ex["offsets"], ex["name"]
            assert r["sorted_token_ids"].tolist() == ex["sorted_token_ids"], (ex["name"], r["sorted_token_ids"])
            assert r["expert_ids"].tolist() == ex["expert_ids"], ex["name"]
        else:
            want = np.zeros(ex["E_local"], np.int32)
            for e, c in ex["counts_nonzero"].items():
                want[int(e)] = c
            assert np.array_equal(r["counts"], want), ex["name"]
            n = len(ex["sorted_token_ids_prefix"])
            assert r["sorted_token_ids"][:n].tolist() == ex["sorted_token_ids_prefix"], ex["name"]
            assert (r["sorted_token_ids"][n:] == ex["sorted_token_ids_tail_value"]).all(), ex["name"]
            n = len(ex["expert_ids_prefix"])
            assert r["expert_ids"][:n].tolist() == ex["expert_ids_prefix"], ex["name"]
            assert (r["expert_ids"][n:] == ex["expert_ids_tail_value"]).all(), ex["name"]
        check_align_invariants(r, ids, ex["E_global"], ex["block_size"], emap, ex["E_local"])


def pin_align_decode_patterns(orc) -> None:
    g = load_golden("decode_route_patterns.json")
    emap = rank1_of_4_map(g["E_global"], g["E_local"], 1)
    for name, pat in g["patterns"].items():
        ids = np.array(pat["ids"], np.int32)
        r = orc.align_permute(ids, g["E_global"], g["block_size"], emap, g["E_local"])
        want = np.zeros(g["E_local"], np.int32)
        for e, c in pat["counts_nonzero"].items():
            want[int(e)] = c
        assert np.array_equal(r["counts"], want), name
        assert int(r["num_tokens_post_pad"][0]) == pat["num_tokens_post_pad"], name
        n = len(pat["expert_ids_prefix"])
        assert r["expert_ids"][:n].tolist() == pat["expert_ids_prefix"], (name, r["expert_ids"][:n])
        check_align_invariants(r, ids, g["E_global"], g["block_size"], emap, g["E_local"])


def pin_align_matches_stable_sort(orc) -> None:
    """The non-pad rows, read in order, are the local slots stably sorted by local expert (Python's sort)."""
    rng = np.random.default_rng(5)
    cases = [(1, 1, 1, None, 1, 1), (5, 3, 8, None, 8, 4), (37, 4, 60, None, 60, 16), (64, 8, 128, None, 128, 64),
             (200, 6, 160, "strided", 40, 8), (100, 8, 256, None, 256, 128), (0, 4, 16, None, 16, 8),
             (50, 2, 10, "rank", 3, 3)]
    for T, k, E, mapkind, E_local, bs in cases:
        ids = rng.integers(-2, E + 2, size=(T, k)).astype(np.int32) if mapkind else \
            rng.integers(0, E, size=(T, k)).astype(np.int32)
        if mapkind == "strided":
            emap = np.array([g // 4 if g % 4 == 1 else -1 for g in range(E)], np.int32)
        elif mapkind == "rank":
            emap = np.full(E, -1, np.int32)
            emap[4:7] = np.arange(3)
        else:
            emap = None
        r = orc.align_permute(ids, E, bs, emap, E_local)
        flat = ids.reshape(-1).astype(np.int64)

        def local_of(s):
            g = flat[s]
            if g < 0 or g >= E:
                return -1
            le = int(emap[g]) if emap is not None else int(g)
            return le if le < E_local else -1

        slots = [s for s in range(T * k) if local_of(s) >= 0]
        want = sorted(slots, key=local_of)
        sti = r["sorted_token_ids"]
        got = [int(v) for v in sti[:int(r["num_tokens_post_pad"][0])] if v != T * k]
        assert got == want, (T, k, E)
        check_align_invariants(r, ids, E, bs, emap, E_local)


ALIGN_PINS = [pin_align_hand_examples, pin_align_decode_patterns, pin_align_matches_stable_sort]


# ---------------------------------------------------------- gather/combine --
def _example_b(orc):
    g = load_golden("gather_combine_hand_example.json")
    ids = np.array(g["topk_ids"], np.int32)
    r = orc.align_permute(ids, g["E_global"], g["block_size"], np.array(g["expert_map"], np.int32), g["E_local"])
    return g, ids, r


def pin_gather_hand_example(orc) -> None:
    g, ids, r = _example_b(orc)
    hidden = f32_to_bf16_bits(np.array(g["hidden"], np.float32))
    npad = int(r["num_tokens_post_pad"][0])
    perm = orc.gather(hidden, ids.shape[1], r["sorted_token_ids"], npad, r["capacity"], fill=0x7777)
    want = f32_to_bf16_bits(np.array(g["permuted_rows_0_to_3"], np.float32))
    assert np.array_equal(perm[:4], want), perm
    assert (perm[4:] == 0x7777).all()


def pin_gather_rows_and_pads(orc) -> None:
    rng = np.random.default_rng(9)
    T, k, E, bs, H = 33, 4, 12, 8, 24
    ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
    r = orc.align_permute(ids, E, bs)
    hidden = rng.integers(0, 0x10000, size=(T, H)).astype(np.uint16)
    npad = int(r["num_tokens_post_pad"][0])
    for zero in (False, True):
        perm = orc.gather(hidden, k, r["sorted_token_ids"], npad, r["capacity"], zero_pad=zero, fill=0x1234)
        for p in range(r["capacity"]):
            s = int(r["sorted_token_ids"][p])
            if p < npad and s < T * k:
                assert np.array_equal(perm[p], hidden[s // k])
            elif p < npad and zero:
                assert (perm[p] == 0).all()
            else:
                assert (perm[p] == 0x1234).all()


def pin_combine_hand_example(orc) -> None:
    g, ids, r = _example_b(orc)
    hidden = f32_to_bf16_bits(np.array(g["hidden"], np.float32))
    npad = int(r["num_tokens_post_pad"][0])
    y = orc.gather(hidden, ids.shape[1], r["sorted_token_ids"], npad, r["capacity"], zero_pad=True)
    out = orc.combine(y, np.array(g["topk_weights"], np.float32), r["inv_perm"])
    assert np.array_equal(out, f32_to_bf16_bits(np.array(g["out"], np.float32))), bf16_bits_to_f32(out)


def pin_combine_identity(orc) -> None:
    """Permute then combine with unit total weight returns the input rows."""
    rng = np.random.default_rng(13)
    T, E, H, bs = 40, 16, 40, 4
    hidden = f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32) * 3)
    for k in (1, 2, 4, 8):
        ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        r = orc.align_permute(ids, E, bs)
        y = orc.gather(hidden, k, r["sorted_token_ids"], int(r["num_tokens_post_pad"][0]), r["capacity"], True)
        w = np.full((T, k), np.float32(1.0 / k))  # exact: every partial sum fits in fp32
        out = orc.combine(y, w, r["inv_perm"])
        assert np.array_equal(out, hidden), k
    # softmax weights (sum to 1 within rounding) leave every bf16 value within one ulp
    k = 6
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    r = orc.align_permute(ids, E, bs)
    y = orc.gather(hidden, k, r["sorted_token_ids"], int(r["num_tokens_post_pad"][0]), r["capacity"], True)
    w, _ = orc.topk_softmax(rng.standard_normal((T, E)).astype(np.float32), k, True)
    out = orc.combine(y, w, r["inv_perm"])
    assert (np.abs(ordered_bf16(out) - ordered_bf16(hidden)) <= 1).all()


def pin_combine_error_bound(orc) -> None:
    """|oracle - exact| <= k * 2^-24 * sum|w*y| + half a bf16 ulp of the exact value (exact = rational sum)."""
    rng = np.random.default_rng(17)
    T, k, H, R = 24, 5, 16, 64
    y = f32_to_bf16_bits(rng.standard_normal((R, H)).astype(np.float32))
    yv = bf16_bits_to_f32(y)
    w = rng.uniform(-1, 1, size=(T, k)).astype(np.float32)
    inv = rng.integers(-1, R, size=T * k).astype(np.int32)
    out = bf16_bits_to_f32(orc.combine(y, w, inv))
    for t in range(T):
        for h in range(H):
            exact = Fraction(0)
            mag = Fraction(0)
            for j in range(k):
                r = int(inv[t * k + j])
                if r < 0:
                    continue
                term = Fraction(float(w[t, j])) * Fraction(float(yv[r, h]))
                exact += term
                mag += abs(term)
            err32 = k * Fraction(1, 2 ** 24) * mag
            big = abs(exact) + err32
            ulp = Fraction(2) ** (math.frexp(float(big))[1] - 8) if big != 0 else Fraction(0)
            bound = err32 + ulp / 2
            assert abs(Fraction(float(out[t, h])) - exact) <= bound, (t, h, float(out[t, h]), float(exact))


def pin_combine_remote_dropped(orc) -> None:
    y = f32_to_bf16_bits(np.array([[1.0, 2.0], [3.0, -4.0]], np.float32))
    w = np.array([[0.5, 0.5], [1.0, 1.0]], np.float32)
    inv = np.array([-1, 1, -1, -1], np.int32)
    out = orc.combine(y, w, inv)
    assert np.array_equal(bf16_bits_to_f32(out), np.array([[1.5, -2.0], [0.0, 0.0]], np.float32))
    assert (out[1] == 0).all()  # +0, not -0


def round_to_f32(q: Fraction) -> Fraction:
    """Exact round-to-nearest-even of a rational to binary32 (no double rounding)."""
    if q == 0:
        return Fraction(0)
    f = np.float32(float(q))
    cands = [f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))]
    best = None
    for c in cands:
        d = abs(Fraction(float(c)) - q)
        even = int(np.asarray(c, np.float32).view(np.uint32)) & 1 == 0
        key = (d, not even)
        if best is None or key < best[0]:
            best = (key, c)
    return Fraction(float(best[1]))


def pin_combine_fma_sequence(orc) -> None:
    """The combine is a chain of correctly rounded fp32 fused multiply-adds in ascending j from +0,
    then one bf16 round-to-nearest-even; emulated here with exact rationals."""
    rng = np.random.default_rng(19)
    T, k, H, R = 16, 8, 12, 40
    y = f32_to_bf16_bits(rng.standard_normal((R, H)).astype(np.float32) * np.float32(7.0))
    yv = bf16_bits_to_f32(y)
    w = rng.uniform(-1, 1, size=(T, k)).astype(np.float32) * np.float32(1.0 + 2.0 ** -12)
    inv = rng.integers(-1, R, size=T * k).astype(np.int32)
    _check_fma_chain(orc, y, yv, w, inv)
    # near-cancelling rows (H = 1): the last weight cancels the running sum, so the result is of the
    # order of the fp32 rounding errors and any change of order or rounding shows up in bf16
    T, k, R = 64, 8, 64
    y = f32_to_bf16_bits(rng.standard_normal((R, 1)).astype(np.float32) * np.float32(3.0))
    y[y == 0] = 0x3F80
    yv = bf16_bits_to_f32(y)
    inv = np.stack([rng.permutation(R)[:k] for _ in range(T)]).astype(np.int32).reshape(-1)
    w = rng.uniform(-1, 1, size=(T, k)).astype(np.float32)
    for t in range(T):
        part = sum(float(w[t, j]) * float(yv[inv[t * k + j], 0]) for j in range(k - 1))
        w[t, k - 1] = np.float32(-part / float(yv[inv[t * k + k - 1], 0]))
    _check_fma_chain(orc, y, yv, w, inv)


def _check_fma_chain(orc, y, yv, w, inv) -> None:
    T, k = w.shape
    H = y.shape[1]
    out = orc.combine(y, w, inv)
    want = np.empty((T, H), np.float32)
    for t in range(T):
        for h in range(H):
            acc = Fraction(0)
            for j in range(k):
                r = int(inv[t * k + j])
                if r >= 0:
                    acc = round_to_f32(Fraction(float(w[t, j])) * Fraction(float(yv[r, h])) + acc)
            want[t, h] = np.float32(float(acc))
    assert np.array_equal(out, f32_to_bf16_bits(want)), np.nonzero(out != f32_to_bf16_bits(want))


GATHER_COMBINE_PINS = [pin_gather_hand_example, pin_gather_rows_and_pads, pin_combine_hand_example,
                       pin_combine_identity, pin_combine_error_bound, pin_combine_remote_dropped,
                       pin_combine_fma_sequence]


# ----------------------------------------------------------------------------------------------
# The expert-parallel exchange: the sum of the ranks' bf16 partial combines, widened to fp32 and
# added in ascending rank order from +0, rounded once to bf16 (the reading the oracle takes where
# the closure note leaves the collective out).
# ----------------------------------------------------------------------------------------------
def _partials(values) -> np.ndarray:
    """[n] values -> [n, 1, 1] bf16 bits (each value must be a bf16 number)."""
    b = f32_to_bf16_bits(np.array(values, np.float32).reshape(-1, 1, 1))
    assert np.array_equal(bf16_bits_to_f32(b).reshape(-1), np.array(values, np.float32))
    return b


def pin_reduce_hand_examples(orc) -> None:
    # fp32 accumulation: 1 + 2^-8 + 2^-8 = 1 + 2^-7, a bf16 number; bf16 accumulation would give 1
    assert float(bf16_bits_to_f32(orc.reduce_partials(_partials([1.0, 2.0 ** -8, 2.0 ** -8])))[0, 0]) == 1.0 + 2.0 ** -7
    # ascending rank order: 2^24 + 1 rounds to 2^24 in fp32, so (2^24, 1, -2^24) gives 0 and
    # (2^24, -2^24, 1) gives 1
    assert float(bf16_bits_to_f32(orc.reduce_partials(_partials([2.0 ** 24, 1.0, -2.0 ** 24])))[0, 0]) == 0.0
    assert float(bf16_bits_to_f32(orc.reduce_partials(_partials([2.0 ** 24, -2.0 ** 24, 1.0])))[0, 0]) == 1.0
    # x + (-x) is +0 (bits 0), as is a lone -0 (0 + -0 = +0)
    assert int(orc.reduce_partials(_partials([3.5, -3.5]))[0, 0]) == 0
    assert int(orc.reduce_partials(np.full((1, 1, 1), 0x8000, np.uint16))[0, 0]) == 0
    # one rank: its partial, bit for bit (no -0 among them)
    rng = np.random.default_rng(23)
    one = f32_to_bf16_bits(rng.standard_normal((1, 7, 24)).astype(np.float32))
    one[one == 0x8000] = 0
    assert np.array_equal(orc.reduce_partials(one), one[0])
    # a sum that needs rounding: 1 + 2^-8 + 2^-9 = 1.005859375 lies between the bf16 numbers 1 and
    # 1.0078125, nearer the second (truncation would give 1)
    assert float(bf16_bits_to_f32(orc.reduce_partials(_partials([1.0, 2.0 ** -8, 2.0 ** -9])))[0, 0]) == 1.0078125


def pin_reduce_fp32_chain(orc) -> None:
    """Each element is a chain of correctly rounded fp32 additions in ascending rank order from +0,
    then one bf16 round-to-nearest-even; emulated here with exact rationals."""
    rng = np.random.default_rng(29)
    for n in (2, 3, 5, 8):
        mags = np.float32(2.0) ** rng.integers(-12, 13, size=(n, 9, 8)).astype(np.float32)
        p = f32_to_bf16_bits(rng.standard_normal((n, 9, 8)).astype(np.float32) * mags)
        pv = bf16_bits_to_f32(p)
        want = np.empty((9, 8), np.float32)
        for i in range(9):
            for h in range(8):
                acc = Fraction(0)
                for r in range(n):
                    acc = round_to_f32(acc + Fraction(float(pv[r, i, h])))
                want[i, h] = np.float32(float(acc))
        got = orc.reduce_partials(p)
        assert np.array_equal(got, f32_to_bf16_bits(want)), n


def pin_reduce_of_rank_partials(orc) -> None:
    """Expert-parallel decomposition: each of 4 ranks combines over its own block of experts; the
    reduce of the 4 partials agrees with the single-rank combine within the rounding of the
    partials (each is rounded to bf16 once) and of the sums."""
    rng = np.random.default_rng(31)
    T, E, k, H, bs, n = 20, 16, 4, 24, 4, 4
    logits = rng.standard_normal((T, E)).astype(np.float32)
    w, ids = orc.topk_softmax(logits, k, True)
    full = orc.align_permute(ids, E, bs)
    y_full = f32_to_bf16_bits(rng.standard_normal((full["capacity"], H)).astype(np.float32))
    ref = bf16_bits_to_f32(orc.combine(y_full, w, full["inv_perm"]))
    # the rank-local expert-output rows are the same rows of the full layout, relaid per rank
    parts, bound = [], np.zeros((T, H))
    for r in range(n):
        m = np.full(E, -1, np.int32)
        m[r * 4:(r + 1) * 4] = np.arange(4)
        loc = orc.align_permute(ids, E, bs, m, 4)
        y = np.zeros((loc["capacity"], H), np.uint16)
        for s in range(T * k):
            if loc["inv_perm"][s] >= 0:
                y[loc["inv_perm"][s]] = y_full[full["inv_perm"][s]]
        part = orc.combine(y, w, loc["inv_perm"])
        parts.append(part)
        pv = np.abs(bf16_bits_to_f32(part).astype(np.float64))
        bound += 2.0 ** (np.floor(np.log2(np.maximum(pv, 2.0 ** -126))) - 8)
    got = bf16_bits_to_f32(orc.reduce_partials(np.stack(parts))).astype(np.float64)
    mag = np.abs(ref.astype(np.float64))
    bound += 2.0 ** (np.floor(np.log2(np.maximum(mag + bound, 2.0 ** -126))) - 7) + 1e-6
    assert (np.abs(got - ref) <= bound).all(), float(np.max(np.abs(got - ref) - bound))


REDUCE_PINS = [pin_reduce_hand_examples, pin_reduce_fp32_chain, pin_reduce_of_rank_partials]

ALL_PINS = TOPK_PINS + SIGMOID_PINS + ALIGN_PINS + GATHER_COMBINE_PINS + REDUCE_PINS
