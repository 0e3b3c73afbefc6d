"""Pins of the CPU oracle against what the routing pages and mathematics fix.

Nothing here compares the oracle with itself: every check is either a
hand-worked fixture (tests/golden/), a brute-force restatement written
differently (numpy, whole-array), an invariant the pages state, a closed form,
or a library routine for a special case (torch's bf16 and float8_e4m3fn casts).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import CONFIGS, Workload, bf16_bits_from_f32, make

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def f2b(a):
    return bf16_bits_from_f32(np.asarray(a, np.float32))


def b2f(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# hand-worked fixtures
# ---------------------------------------------------------------------------

def test_golden_tiny_normal_path():
    g = gold("routing_tiny.json")
    idx = np.array(g["topk_idx"], np.int64)
    w = np.array(g["topk_weights"], np.float32)
    x = f2b(g["x"])
    E = g["E"]
    res = oracle.normal_path(x, idx, w, E)
    np.testing.assert_array_equal(res["num_tokens_per_rank"], g["num_tokens_per_rank"])
    np.testing.assert_array_equal(res["num_tokens_per_expert"], g["num_tokens_per_expert"])
    np.testing.assert_array_equal(res["is_token_in_rank"], g["is_token_in_rank"])
    np.testing.assert_array_equal(res["rank_prefix_matrix"], g["rank_prefix_matrix"])
    np.testing.assert_array_equal(res["recv_count"], g["recv_count"])
    np.testing.assert_array_equal(res["send_pos"], g["send_pos"])
    np.testing.assert_array_equal(res["num_recv_tokens_per_expert"],
                                  g["num_recv_tokens_per_expert_align1"])
    lay = oracle.layout(idx, E, g["R"])
    np.testing.assert_array_equal(
        oracle.expert_recv_counts(lay["num_tokens_per_expert"], g["R"], 4),
        g["num_recv_tokens_per_expert_align4"])
    for d, n in enumerate(g["recv_count"]):
        np.testing.assert_array_equal(res["recv_src_idx"][d, :n], g["recv_src_idx"][d])
        np.testing.assert_array_equal(res["recv_topk_idx"][d, :n], g["recv_topk_idx"][d])
        np.testing.assert_array_equal(res["recv_topk_weights"][d, :n], g["recv_topk_weights"][d])
        np.testing.assert_array_equal(b2f(res["recv_x"][d, :n]),
                                      np.array(g["x"], np.float32)[
                                          [s for s in range(g["R"]) for t in range(g["T"])
                                           if g["is_token_in_rank"][s][t][d]],
                                          [t for s in range(g["R"]) for t in range(g["T"])
                                           if g["is_token_in_rank"][s][t][d]]])
    np.testing.assert_array_equal(b2f(res["combined_x"]), np.array(g["combined_x"], np.float32))
    np.testing.assert_array_equal(res["combined_topk_weights"], g["combined_topk_weights"])


def test_golden_tiny_low_latency():
    g = gold("routing_tiny.json")
    idx = np.array(g["topk_idx"], np.int64)
    ll = oracle.ll_layout(idx, g["E"])
    np.testing.assert_array_equal(ll["recv_count"], g["ll_recv_count"])
    np.testing.assert_array_equal(ll["layout_range"], g["ll_layout_range"])
    np.testing.assert_array_equal(ll["ll_pos"], g["ll_pos"])
    for d in range(g["R"]):
        for j in range(g["E"] // g["R"]):
            n = g["ll_recv_count"][d][j]
            np.testing.assert_array_equal(ll["recv_src_info"][d, j, :n], g["ll_recv_src_info"][d][j])
    # identity experts: the bf16 slab rows go back unchanged
    slab, _ = oracle.ll_dispatch_rows(f2b(g["x"]), idx, ll["ll_pos"], g["E"], use_fp8=False)
    out = oracle.ll_combine(slab, idx, np.array(g["topk_weights"], np.float32), ll["ll_pos"])
    np.testing.assert_array_equal(b2f(out), np.array(g["ll_combined_x"], np.float32))


def test_golden_fp8_and_bf16_codes():
    g = gold("fp8_codes.json")
    for c in g["e4m3_decode"]:
        assert oracle.e4m3_to_f32(c["code"]) == c["value"], c
    for c in g["e4m3_encode"]:
        assert oracle.f32_to_e4m3(c["value"]) == c["code"], c
    for c in g["bf16_round"]:
        assert oracle.f32_to_bf16(c["f32"]) == c["bits"], c


def test_golden_quant_block():
    g = gold("fp8_codes.json")["quant_block"]
    x = np.zeros(128, np.float32)
    x[:4] = g["x_head"]
    q, s = oracle.quantize_row(f2b(x))
    np.testing.assert_array_equal(q[:4], g["q_head"])
    assert (q[4:] == g["q_rest"]).all()
    assert s[0] == np.float32(1.0 / 224.0)


def test_quant_zero_and_tiny_blocks():
    # an all-zero block must quantise to zero codes with a finite positive
    # scale (the amax floor keeps 448/amax finite); a block far below the
    # floor keeps its signs and stays finite, and the round trip stays within
    # the floor's quantum
    x = np.zeros(256, np.float32)
    x[128:] = np.where(np.arange(128) % 2 == 0, 1e-6, -1e-6)
    for rs in (False, True):
        q, s, _ = oracle.quantize_row_ex(f2b(x), round_scale=rs)
        assert (q[:128] == 0).all()
        assert np.isfinite(s).all() and (s > 0).all()
        codes = oracle.e4m3_to_f32_array(q[128:])
        assert np.isfinite(codes).all()
        assert (np.sign(codes) == np.sign(x[128:])).all()
        deq = codes.astype(np.float64) * s[1]
        xv = b2f(f2b(x[128:])).astype(np.float64)
        v = np.abs(xv) / s[1]
        ulp = np.where(v < 2 ** -6, 2.0 ** -9,
                       2.0 ** (np.floor(np.log2(np.maximum(v, 2 ** -6))) - 3))
        assert (np.abs(deq - xv) <= 0.5 * ulp * s[1] * (1 + 1e-6)).all()


def test_golden_quant_block_round_scale():
    g = gold("fp8_codes.json")["quant_block_round_scale"]
    x = np.zeros(128, np.float32)
    x[:4] = g["x_head"]
    q, s, u = oracle.quantize_row_ex(f2b(x), round_scale=True)
    np.testing.assert_array_equal(q[:4], g["q_head"])
    assert (q[4:] == g["q_rest"]).all()
    assert s[0] == g["scale"] and u[0] == g["ue8m0"]


def test_round_scale_properties():
    # scale is the smallest power of two >= amax'/448; UE8M0 byte is its
    # biased exponent; round trip within half an e4m3 step
    rng = np.random.default_rng(12)
    H = 2048
    x = f2b(rng.standard_normal(H).astype(np.float32) * np.repeat(
        np.exp(rng.uniform(-10, 10, H // 128)), 128).astype(np.float32))
    q, s, u = oracle.quantize_row_ex(x, round_scale=True)
    xf = b2f(x).astype(np.float64)
    for b in range(H // 128):
        amax = max(np.abs(xf[b * 128:(b + 1) * 128]).max(), float(np.float32(1e-4)))
        target = float(np.float32(np.float32(amax) / np.float32(448.0)))
        e = int(u[b]) - 127
        assert s[b] == 2.0 ** e and 2.0 ** e >= target and 2.0 ** (e - 1) < target
        v = xf[b * 128:(b + 1) * 128] / s[b]
        assert np.abs(v).max() <= 448.0
        deq = oracle.e4m3_to_f32_array(q[b * 128:(b + 1) * 128]).astype(np.float64) * s[b]
        ulp = np.where(np.abs(v) < 2 ** -6, 2.0 ** -9,
                       2.0 ** (np.floor(np.log2(np.maximum(np.abs(v), 2 ** -6))) - 3))
        assert (np.abs(deq - xf[b * 128:(b + 1) * 128]) <= 0.5 * ulp * s[b] + 1e-30).all()


def test_ll_mask_drops_failed_ranks():
    # shrink mode: counts equal (topk_idx == e).sum() over unmasked source
    # ranks (legacy-test analysis page, the masked count check); experts on a
    # masked rank receive nothing
    w = Workload("msk", R=6, T=40, H=128, E=24, K=4)
    idx = make(w, with_x=False)["topk_idx"]
    mask = np.array([0, 1, 0, 1, 0, 0], np.int32)
    ll = oracle.ll_layout(idx, w.E, mask=mask)
    El = w.E // w.R
    for e in range(w.E):
        d, j = divmod(e, El)
        want = 0 if mask[d] else int((idx[mask == 0] == e).sum())
        assert ll["recv_count"][d, j] == want
    for s in range(w.R):
        if mask[s]:
            assert (ll["ll_pos"][s] == -1).all()
    owner = np.where(idx >= 0, idx // El, 0)
    assert (ll["ll_pos"][mask[owner] == 1] == -1).all()


# ---------------------------------------------------------------------------
# A1 layout: brute force written whole-array, plus the pages' invariants
# ---------------------------------------------------------------------------

def brute_layout(idx, E, R):
    S, T, K = idx.shape
    El = E // R
    valid = (idx >= 0) & (idx < E)
    owner = np.where(valid, idx // El, -1)
    in_rank = np.stack([(owner == d).any(axis=2) for d in range(R)], axis=2).astype(np.uint8)
    ntpe = np.zeros((S, E), np.int32)
    for e in range(E):               # full E x T x K scan
        ntpe[:, e] = (idx == e).sum(axis=(1, 2))
    ntpr = in_rank.sum(axis=1).astype(np.int32)
    return ntpr, ntpe, in_rank


def random_tiny_idx(rng, S, T, K, E, p_mask=0.2, p_dup=0.2, p_bad=0.0):
    idx = rng.integers(0, E, size=(S, T, K))
    m = rng.random((S, T, K))
    idx[m < p_mask] = -1
    if K > 1:
        d = rng.random((S, T)) < p_dup
        idx[..., 1][d] = idx[..., 0][d]
    if p_bad > 0:
        b = rng.random((S, T, K)) < p_bad
        idx[b] = rng.choice([E, E + 3, -2, -5], size=int(b.sum()))
    return idx.astype(np.int64)


@pytest.mark.parametrize("seed", range(12))
def test_layout_brute_force_tiny(seed):
    rng = np.random.default_rng(seed)
    R = int(rng.choice([1, 2, 3, 4]))
    El = int(rng.integers(1, 5))
    E = R * El
    S = int(rng.choice([1, R]))
    T = int(rng.integers(1, 17))
    K = int(rng.integers(1, min(E, 6) + 1))
    idx = random_tiny_idx(rng, S, T, K, E, p_bad=0.05 if seed % 3 == 0 else 0.0)
    lay = oracle.layout(idx, E, R)
    ntpr, ntpe, in_rank = brute_layout(idx, E, R)
    np.testing.assert_array_equal(lay["is_token_in_rank"], in_rank)
    np.testing.assert_array_equal(lay["num_tokens_per_expert"], ntpe)
    np.testing.assert_array_equal(lay["num_tokens_per_rank"], ntpr)
    assert lay["bad_slots"] == int(((idx < -1) | (idx >= E)).sum())


@pytest.mark.parametrize("name", ["pr1", "layout", "normal", "skewed", "ll"])
def test_layout_invariants_on_configs(name):
    w = CONFIGS[name]
    inp = make(w, with_x=False)
    idx = inp["topk_idx"]
    lay = oracle.layout(idx, w.E, w.R)
    valid = int(((idx >= 0) & (idx < w.E)).sum())
    # sum(num_tokens_per_expert) == number of valid top-k slots
    assert int(lay["num_tokens_per_expert"].sum()) == valid
    # num_tokens_per_rank == is_token_in_rank summed over the token rows
    np.testing.assert_array_equal(lay["num_tokens_per_rank"],
                                  lay["is_token_in_rank"].sum(axis=1))
    if name == "skewed":
        assert int((idx == -1).sum()) == w.S * round(0.1 * w.T * w.K)


# ---------------------------------------------------------------------------
# A2/A3: positions by sorting (d, s, t) triples; check_data block structure
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(10))
def test_prefix_matches_sorted_triples(seed):
    rng = np.random.default_rng(100 + seed)
    R = int(rng.integers(1, 6))
    T = int(rng.integers(1, 20))
    in_rank = (rng.random((R, T, R)) < rng.random()).astype(np.uint8)
    cap = R * T if seed % 4 else max(0, int(in_rank.sum(axis=(0, 1)).max()) - 2)
    pre = oracle.prefix(in_rank, cap)
    ntpr = in_rank.sum(axis=1).astype(np.int64)
    for d in range(R):
        triples = sorted((s, t) for s in range(R) for t in range(T) if in_rank[s, t, d])
        for row, (s, t) in enumerate(triples):
            assert pre["send_pos"][s, t, d] == row
            if row < cap:
                assert pre["recv_src_idx"][d, row] == t
        assert pre["recv_count"][d] == len(triples)
        for s in range(R):
            assert pre["rank_prefix_matrix"][s, d] == ntpr[: s + 1, d].sum()
    assert (pre["send_pos"][in_rank == 0] == -1).all()
    np.testing.assert_array_equal(pre["rank_prefix_matrix"][-1], ntpr.sum(axis=0))
    assert pre["overflow"] == int(np.maximum(ntpr.sum(axis=0) - cap, 0).sum())


def test_check_data_rank_encoded_payload():
    # x = ones * rank; rows [P[s-1][d], P[s][d]) of receiver d all hold s.
    w = Workload("enc", R=6, T=50, H=16, E=24, K=3)
    inp = make(w)
    x = f2b(np.broadcast_to(np.arange(w.R, dtype=np.float32)[:, None, None], (w.R, w.T, w.H)))
    res = oracle.normal_path(x, inp["topk_idx"], inp["topk_weights"], w.E)
    P = res["rank_prefix_matrix"]
    for d in range(w.R):
        rows = b2f(res["recv_x"][d, : res["recv_count"][d]])
        assert (rows.min(axis=1) == rows.max(axis=1)).all()
        start = 0
        for s in range(w.R):
            end = P[s, d]
            assert (rows[start:end, 0] == s).all()
            start = end


def test_dispatch_meta_remap():
    rng = np.random.default_rng(7)
    R, El, T, K = 3, 4, 9, 3
    E = R * El
    idx = random_tiny_idx(rng, R, T, K, E)
    w = rng.random((R, T, K)).astype(np.float32)
    lay = oracle.layout(idx, E, R)
    pre = oracle.prefix(lay["is_token_in_rank"])
    ri, rw = oracle.dispatch_meta(idx, w, pre["send_pos"], E)
    for s in range(R):
        for t in range(T):
            for d in range(R):
                p = pre["send_pos"][s, t, d]
                if p < 0:
                    continue
                for k in range(K):
                    e = idx[s, t, k]
                    if e >= 0 and e // El == d:
                        assert ri[d, p, k] == e - d * El and rw[d, p, k] == w[s, t, k]
                    else:
                        assert ri[d, p, k] == -1 and rw[d, p, k] == 0.0


# ---------------------------------------------------------------------------
# A4 combine: closed form with identity experts; bound for random y
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["pr1", "skewed_small", "uniform_mid"])
def test_combine_identity_closed_form(name):
    if name == "pr1":
        w = CONFIGS["pr1"]
    elif name == "skewed_small":
        w = Workload("sk", R=16, T=256, H=128, E=128, K=6, routing="zipf", masked_frac=0.1)
    else:
        w = Workload("um", R=8, T=200, H=136, E=64, K=8)
    inp = make(w)
    idx, wts, x = inp["topk_idx"], inp["topk_weights"], inp["x"]
    res = oracle.normal_path(x, idx, wts, w.E)
    n_dest = res["is_token_in_rank"].sum(axis=2).astype(np.float64)
    # n * x is exact in fp32; the sum starts from +0.0, so -0.0 inputs give +0.0
    expect = f2b((n_dest[..., None] * b2f(x).astype(np.float64) + 0.0).astype(np.float32))
    np.testing.assert_array_equal(res["combined_x"], expect)
    masked = np.where((idx >= 0) & (idx < w.E), wts, np.float32(0.0))
    np.testing.assert_array_equal(res["combined_topk_weights"], masked)


def test_combine_signed_zero():
    # one token to two ranks, payload -0.0 everywhere: the fp32 sum from +0.0
    # gives +0.0 (IEEE: +0 + -0 = +0 under round to nearest)
    idx = np.array([[[0, 1]]], np.int64)          # R=1 would keep one copy; use R=2
    idx = np.array([[[0, 2]], [[-1, -1]]], np.int64)
    x = np.full((2, 1, 8), 0x8000, np.uint16)    # -0.0
    w = np.ones((2, 1, 2), np.float32)
    res = oracle.normal_path(x, idx, w, 4)
    assert res["recv_count"].tolist() == [1, 1]
    assert (res["combined_x"][0, 0] == 0x0000).all()
    assert (res["combined_x"][1, 0] == 0x0000).all()


def test_combine_bias_matches_the_pages_check():
    # (combined - bias_0 - bias_1) / n_dest == x, to within two fp32 roundings of
    # the bias adds and one bf16 rounding of the result (fp64 reference)
    w = Workload("cb", R=4, T=60, H=64, E=16, K=3)
    inp = make(w)
    b0 = make(Workload("cb0", R=4, T=60, H=64, E=16, K=3, seed=1))["x"]
    b1 = make(Workload("cb1", R=4, T=60, H=64, E=16, K=3, seed=2))["x"]
    res = oracle.normal_path(inp["x"], inp["topk_idx"], inp["topk_weights"], w.E)
    out, _ = oracle.combine(res["recv_x"], res["send_pos"], bias=(b0, b1))
    n = res["is_token_in_rank"].sum(axis=2).astype(np.float64)[..., None]
    xf, f0, f1 = (b2f(a).astype(np.float64) for a in (inp["x"], b0, b1))
    exact = n * xf + f0 + f1
    mag = np.abs(n * xf) + np.abs(f0) + np.abs(f1)
    got = b2f(out).astype(np.float64)
    assert (np.abs(got - exact) <= 2.0 ** -8 * np.abs(exact) + 3 * 2.0 ** -24 * mag + 1e-30).all()
    # and without the second bias it differs by exactly that bias, up to rounding
    out0, _ = oracle.combine(res["recv_x"], res["send_pos"], bias=(b0, None))
    got0 = b2f(out0).astype(np.float64)
    assert (np.abs(got0 - (n * xf + f0)) <= 2.0 ** -8 * np.abs(n * xf + f0) + 2 * 2.0 ** -24 * mag + 1e-30).all()


def test_fp8_input_rows_are_copied_by_send_pos():
    rng = np.random.default_rng(9)
    R, T, H = 3, 7, 256
    q = rng.integers(0, 256, size=(R, T, H), dtype=np.uint8)
    sc = rng.random((R, T, H // 128)).astype(np.float32)
    in_rank = (rng.random((R, T, R)) < 0.5).astype(np.uint8)
    pre = oracle.prefix(in_rank)
    rq, rs = oracle.dispatch_rows_fp8(q, sc, pre["send_pos"])
    rq2, rs2 = oracle.dispatch_rows_fp8(q, np.ascontiguousarray(sc.transpose(0, 2, 1)),
                                        pre["send_pos"], col_major=True)
    for d in range(R):
        triples = sorted((s, t) for s in range(R) for t in range(T) if in_rank[s, t, d])
        for row, (s, t) in enumerate(triples):
            np.testing.assert_array_equal(rq[d, row], q[s, t])
            np.testing.assert_array_equal(rs[d, row], sc[s, t])
            np.testing.assert_array_equal(rs2[d, row], sc[s, t])
    np.testing.assert_array_equal(rq, rq2)


def test_combine_random_y_error_bound():
    rng = np.random.default_rng(3)
    R, T, H, E, K = 5, 40, 64, 20, 4
    idx = random_tiny_idx(rng, R, T, K, E, p_mask=0.1, p_dup=0.0)
    lay = oracle.layout(idx, E, R)
    pre = oracle.prefix(lay["is_token_in_rank"])
    cap = R * T
    y = f2b(rng.standard_normal((R, cap, H)).astype(np.float32) * 3)
    out, _ = oracle.combine(y, pre["send_pos"])
    yf = b2f(y).astype(np.float64)
    sp = pre["send_pos"]
    exact = np.zeros((R, T, H))
    absum = np.zeros((R, T, H))
    nd = np.zeros((R, T))
    for s in range(R):
        for t in range(T):
            for d in range(R):
                if sp[s, t, d] >= 0:
                    exact[s, t] += yf[d, sp[s, t, d]]
                    absum[s, t] += np.abs(yf[d, sp[s, t, d]])
                    nd[s, t] += 1
    got = b2f(out).astype(np.float64)
    u32, ubf = 2.0 ** -24, 2.0 ** -8
    bound = ubf * np.abs(exact) + (nd[..., None] * u32 * absum) * (1 + ubf) + 1e-30
    assert (np.abs(got - exact) <= bound).all()


# ---------------------------------------------------------------------------
# A5: e4m3 encoder pinned exhaustively; quantiser round trip; LL positions
# ---------------------------------------------------------------------------

def e4m3_table():
    """Decode the 256 codes from the bit layout (float64)."""
    vals = np.empty(256)
    for c in range(256):
        s = -1.0 if c & 0x80 else 1.0
        e = (c >> 3) & 15
        m = c & 7
        if e == 15 and m == 7:
            vals[c] = np.nan
        elif e == 0:
            vals[c] = s * (m / 8.0) * 2.0 ** -6
        else:
            vals[c] = s * (1 + m / 8.0) * 2.0 ** (e - 7)
    return vals


def nearest_e4m3(v):
    """Brute force: nearest finite code, ties to the even mantissa, |v|>448 -> 448."""
    tab = e4m3_table()
    codes = np.array([c for c in range(256) if not np.isnan(tab[c])])
    cv = tab[codes]
    out = np.empty(v.shape, np.uint8)
    vv = np.clip(v.astype(np.float64), -448.0, 448.0)
    for i0 in range(0, v.size, 8192):
        chunk = vv[i0:i0 + 8192]
        dist = np.abs(chunk[:, None] - cv[None, :])
        best = dist.min(axis=1, keepdims=True)
        cand = dist == best
        # among ties prefer the even mantissa; keep the sign of v for zero
        even = (codes & 1) == 0
        sgn_ok = ((codes & 0x80) != 0)[None, :] == np.signbit(chunk)[:, None]
        score = cand * 4 + (cand & even[None, :]) * 2 + (cand & sgn_ok) * 1
        out[i0:i0 + 8192] = codes[score.argmax(axis=1)]
    return out


@pytest.mark.parametrize("scale", [1.0, 448.0 / 3.7, 0.125, 32.0, 3.3, 1e-3])
def test_e4m3_encoder_exhaustive_over_bf16(scale):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = b2f(bits)
    f = f[np.isfinite(f)]
    with np.errstate(over="ignore"):
        v = (f * np.float32(scale)).astype(np.float32)
    v = v[np.isfinite(v)]
    got = oracle.f32_to_e4m3_array(v)
    np.testing.assert_array_equal(got, nearest_e4m3(v))
    # library special case: torch's float8_e4m3fn cast is round-to-nearest-even
    # inside the finite range
    inr = np.abs(v) < 448.0
    tt = torch.from_numpy(v[inr]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(got[inr], tt)


def test_e4m3_decoder_all_codes_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_to_f32_array(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    nan = np.isnan(ref)
    assert (np.isnan(got) == nan).all()
    np.testing.assert_array_equal(got[~nan], ref[~nan])


def test_bf16_rounding_vs_torch():
    rng = np.random.default_rng(11)
    v = (rng.standard_normal(200000) * np.exp(rng.uniform(-30, 30, 200000))).astype(np.float32)
    # exact ties: low 16 bits == 0x8000
    ties = (rng.integers(0, 2 ** 32, 20000, dtype=np.uint64).astype(np.uint32) & 0xFFFF0000) | 0x8000
    ties = ties.view(np.float32)
    v = np.concatenate([v, ties[np.isfinite(ties)]])
    np.testing.assert_array_equal(oracle.f32_to_bf16_array(v), f2b(v))


def test_quantizer_round_trip_bound():
    rng = np.random.default_rng(5)
    H = 1024
    x = f2b(rng.standard_normal(H).astype(np.float32) * np.repeat(
        np.exp(rng.uniform(-8, 8, H // 128)), 128).astype(np.float32))
    q, sc = oracle.quantize_row(x)
    xf = b2f(x).astype(np.float64)
    deq = oracle.e4m3_to_f32_array(q).astype(np.float64) * np.repeat(sc, 128)
    for b in range(H // 128):
        blk = slice(b * 128, (b + 1) * 128)
        amax = np.abs(xf[blk]).max()
        assert abs(sc[b] - max(amax, np.float32(1e-4)) / 448.0) <= 2 ** -23 * sc[b]
        # every scaled value v = x / scale lies in [-448, 448] (up to fp32 error);
        # e4m3 spacing there is at most 32, and 2^-9 below 2^-6.
        v = np.abs(xf[blk]) / sc[b]
        ulp = np.where(v < 2 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(v, 2 ** -6))) - 3))
        err = np.abs(deq[blk] - xf[blk])
        assert (err <= (0.5 * ulp + 1e-5 * v) * sc[b] * (1 + 1e-6)).all()
    # the block maximum maps to 448 exactly
    assert (q.reshape(-1, 128).view(np.uint8) & 0x7F).max(axis=1).tolist() == [0x7E] * (H // 128)


def brute_ll_positions(idx, E):
    R, T, K = idx.shape
    pos = np.full((R, T, K), -1, np.int64)
    for s in range(R):
        for t in range(T):
            for k in range(K):
                e = idx[s, t, k]
                if e < 0 or e >= E:
                    continue
                # number of (s', t') before (s, t) whose slot set contains e
                before = 0
                for s2 in range(R):
                    for t2 in range(T):
                        if (s2, t2) >= (s, t):
                            break
                        before += int(e in set(idx[s2, t2].tolist()))
                pos[s, t, k] = before
    return pos


@pytest.mark.parametrize("seed", range(6))
def test_ll_layout_brute_force(seed):
    rng = np.random.default_rng(200 + seed)
    R = int(rng.integers(1, 4))
    El = int(rng.integers(1, 4))
    E = R * El
    T = int(rng.integers(1, 9))
    K = int(rng.integers(1, min(E, 4) + 1))
    idx = random_tiny_idx(rng, R, T, K, E, p_bad=0.05 if seed == 0 else 0.0)
    ll = oracle.ll_layout(idx, E)
    np.testing.assert_array_equal(ll["ll_pos"], brute_ll_positions(idx, E))
    cnt = ll["recv_count"].reshape(-1)
    lr = ll["layout_range"].reshape(E, R, 2)
    for e in range(E):
        has = np.array([[e in set(idx[s, t].tolist()) for t in range(T)] for s in range(R)])
        assert cnt[e] == has.sum()
        np.testing.assert_array_equal(lr[e, :, 1], has.sum(axis=1))
        np.testing.assert_array_equal(lr[e, :, 0], np.concatenate([[0], np.cumsum(has.sum(axis=1))[:-1]]))


def test_ll_count_and_token_encoding():
    # legacy LL test data: x = rank - 128 everywhere except the last 128
    # channels, which hold the token id; counts == (topk_idx == expert).sum().
    w = Workload("llenc", R=4, T=24, H=256, E=16, K=4)
    inp = make(w, with_x=False)
    idx = inp["topk_idx"]
    R, T, H, E = w.R, w.T, w.H, w.E
    El = E // R
    xf = np.zeros((R, T, H), np.float32)
    xf[:, :, : H - 128] = (np.arange(R, dtype=np.float32) - 128)[:, None, None]
    xf[:, :, H - 128:] = np.arange(T, dtype=np.float32)[None, :, None]
    x = f2b(xf)
    ll = oracle.ll_layout(idx, E)
    slab, _ = oracle.ll_dispatch_rows(x, idx, ll["ll_pos"], E, use_fp8=False)
    for e in range(E):
        d, j = divmod(e, El)
        n = ll["recv_count"][d, j]
        assert n == int((idx == e).sum())
        rows = b2f(slab[d, j, :n])
        assert (rows[:, : H - 128].min(axis=1) == rows[:, : H - 128].max(axis=1)).all()
        for s in range(R):
            b, c = ll["layout_range"][d, j, s]
            assert (rows[b:b + c, 0] == s - 128).all()
            assert c == int((idx[s] == e).sum())
            np.testing.assert_array_equal(rows[b:b + c, H - 1], ll["recv_src_info"][d, j, b:b + c])
            np.testing.assert_array_equal(ll["recv_src_info"][d, j, b:b + c],
                                          np.nonzero((idx[s] == e).any(axis=1))[0])


# ---------------------------------------------------------------------------
# A6 LL combine: identity experts give x * sum of the valid weights
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fp8", [False, True])
def test_ll_combine_identity_bound(fp8):
    w = Workload("llc", R=4, T=32, H=256, E=16, K=4, masked_frac=0.1)
    inp = make(w)
    idx, wts, x = inp["topk_idx"], inp["topk_weights"], inp["x"]
    ll = oracle.ll_layout(idx, w.E)
    q, sc = oracle.ll_dispatch_rows(x, idx, ll["ll_pos"], w.E, use_fp8=fp8)
    y = oracle.dequant_rows(q, sc) if fp8 else q
    out = oracle.ll_combine(y, idx, wts, ll["ll_pos"])
    xf = b2f(x).astype(np.float64)
    valid = (idx >= 0) & (idx < w.E)
    wsum = np.where(valid, wts, 0).astype(np.float64).sum(axis=2)
    wabs = np.where(valid, np.abs(wts), 0).astype(np.float64).sum(axis=2)
    exact = xf * wsum[..., None]
    got = b2f(out).astype(np.float64)
    K = w.K
    if fp8:
        # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 per element, plus
        # the subnormal floor of the block scale, plus bf16 rounding of y.
        amax = np.abs(xf).reshape(w.R, w.T, -1, 128).max(axis=3)
        floor = np.repeat(amax / 448.0 * 2.0 ** -10, 128, axis=2)
        tol = (2.0 ** -4 + 2.0 ** -8) * np.abs(xf) * wabs[..., None] + floor * wabs[..., None]
        tol = tol + 2.0 ** -8 * np.abs(exact) + K * 2.0 ** -24 * np.abs(xf) * wabs[..., None]
    else:
        tol = 2.0 ** -8 * np.abs(exact) + (K + 1) * 2.0 ** -24 * np.abs(xf) * wabs[..., None]
    assert (np.abs(got - exact) <= tol + 1e-30).all()
    assert not np.isnan(got).any()
