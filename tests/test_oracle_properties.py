"""Property-based pins of the oracle (hypothesis, CPU): random small shapes,
masked and repeated slots and out-of-range ids, each checked against the
brute-force restatements in test_oracle_pins and against identities the
definitions imply -- the LL slab rows of an expert are the normal receive
order restricted to the tokens that select it, and the combine of identity
experts is n_dest(s, t) times the row."""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from tests.test_oracle_pins import brute_layout, brute_ll_positions, random_tiny_idx

SETTINGS = settings(max_examples=60, deadline=None,
                    suppress_health_check=[HealthCheck.too_slow])


@st.composite
def routing(draw, max_t=12):
    R = draw(st.integers(1, 5))
    El = draw(st.integers(1, 4))
    E = R * El
    T = draw(st.integers(0, max_t))
    K = draw(st.integers(1, min(E, 6)))
    seed = draw(st.integers(0, 2**31 - 1))
    p_bad = draw(st.sampled_from([0.0, 0.0, 0.05]))
    rng = np.random.default_rng(seed)
    idx = random_tiny_idx(rng, R, T, K, E, p_mask=draw(st.sampled_from([0.0, 0.2, 0.6])),
                          p_dup=0.2, p_bad=p_bad)
    return idx, E, R, rng


@SETTINGS
@given(routing())
def test_layout_equals_brute_force(case):
    idx, E, R, _ = case
    lay = oracle.layout(idx, E, R)
    ntpr, ntpe, in_rank = brute_layout(idx, E, R)
    np.testing.assert_array_equal(lay["is_token_in_rank"], in_rank)
    np.testing.assert_array_equal(lay["num_tokens_per_expert"], ntpe)
    np.testing.assert_array_equal(lay["num_tokens_per_rank"], ntpr)


@SETTINGS
@given(routing())
def test_positions_are_the_stable_receive_order(case):
    idx, E, R, _ = case
    T = idx.shape[1]
    lay = oracle.layout(idx, E, R)
    pre = oracle.prefix(lay["is_token_in_rank"])
    for d in range(R):
        order = [(s, t) for s in range(R) for t in range(T) if lay["is_token_in_rank"][s, t, d]]
        for row, (s, t) in enumerate(order):
            assert pre["send_pos"][s, t, d] == row
            assert pre["recv_src_idx"][d, row] == t
        assert pre["recv_count"][d] == len(order)


@SETTINGS
@given(routing(max_t=8))
def test_ll_rows_equal_brute_force_and_restricted_receive_order(case):
    idx, E, R, _ = case
    T, K = idx.shape[1], idx.shape[2]
    ll = oracle.ll_layout(idx, E)
    np.testing.assert_array_equal(ll["ll_pos"], brute_ll_positions(idx, E))
    # expert e's rows list, in (source, token) order, exactly the tokens that
    # select e -- the normal receive order of rank e / E_l restricted to them
    El = E // R
    for e in range(E):
        tokens = [(s, t) for s in range(R) for t in range(T) if e in set(idx[s, t].tolist())]
        d, j = divmod(e, El)
        assert ll["recv_count"][d, j] == len(tokens)
        for row, (s, t) in enumerate(tokens):
            assert ll["recv_src_info"][d, j, row] == t
            ks = [k for k in range(K) if idx[s, t, k] == e]
            assert all(ll["ll_pos"][s, t, k] == row for k in ks)


@SETTINGS
@given(routing(max_t=10), st.integers(1, 3))
def test_identity_combine_is_n_dest_times_the_row(case, h8):
    idx, E, R, rng = case
    T, K = idx.shape[1], idx.shape[2]
    H = 8 * h8
    # bf16 rows of small integers times powers of two: every partial sum exact
    vals = rng.integers(-8, 9, size=(R, T, H)).astype(np.float32) * np.float32(0.25)
    x = (vals.view(np.uint32) >> 16).astype(np.uint16)
    w = rng.random((R, T, K)).astype(np.float32)
    ref = oracle.normal_path(x, idx, w, E)
    n_dest = ref["is_token_in_rank"].sum(axis=2).astype(np.float32)
    expect = vals * n_dest[..., None] + np.float32(0.0)
    got = (ref["combined_x"].astype(np.uint32) << 16).view(np.float32)
    np.testing.assert_array_equal(got, expect)
    # combined weights restore the valid slots' weights and zero the others
    valid = (idx >= 0) & (idx < E)
    np.testing.assert_array_equal(ref["combined_topk_weights"], np.where(valid, w, 0.0))
