"""Property test of bsgemm_make_plan (host only, no GPU): for random sizes,
granularities, layouts, SM counts and tunings, a plan either satisfies the
invariants the kernels rely on or is refused for a documented reason.

The invariants are those the launch code and the kernels' work walk assume:
tiles cover the output, the K splits cover every K-block with none empty (and,
at g = 64, start on a 128-deep stage), the stream-K fields describe full waves
of whole tiles followed by an even share of the rest, the grid never exceeds
the SMs, and a tuning the caller gives is honoured."""
from hypothesis import HealthCheck, given, settings, strategies as st

import fp8_block_scaled_bsgemm_b200 as bsg


def cdiv(a, b):
    return -(-a // b)


def expected_refusal(M, t, num_sms):
    """True when the tuning is one the library documents as invalid."""
    if not t:
        return False
    v, bnq, splits, sk = t["variant"], t["bnq"], t["splits"], t["stream_k"]
    if v == "cta_pair":
        return (bnq not in (0, 256)) or splits > 1 or sk > 0 or num_sms < 2
    if v == "auto":
        v = "swap_ab" if M <= 64 else "data_parallel"   # a tuned plan never pairs automatically
    if v == "swap_ab":
        return bnq not in (0, 16, 32, 64, 128)
    return bnq not in (0, 128, 256)


tunings = st.one_of(
    st.none(),
    st.fixed_dictionaries({
        "variant": st.sampled_from(["auto", "data_parallel", "swap_ab", "cta_pair"]),
        "bnq": st.sampled_from([0, 0, 16, 32, 64, 128, 256, 96]),
        "splits": st.sampled_from([0, 0, 1, 2, 3, 7]),
        "stream_k": st.sampled_from([0, 0, 1, -1]),
    }))


@settings(max_examples=600, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(M=st.integers(1, 20000), N=st.integers(1, 20000), K=st.integers(1, 70000),
       gran=st.sampled_from([64, 128, 256]), layout=st.sampled_from(["nt", "tn", "nn", "tt"]),
       num_sms=st.integers(1, 200), t=tunings)
def test_plans_keep_their_invariants(M, N, K, gran, layout, num_sms, t):
    try:
        pl = bsg.make_plan(M, N, K, gran, layout, num_sms, t)
    except bsg.BsgemmError as e:
        assert e.status == 1 and expected_refusal(M, t, num_sms), (M, N, K, gran, num_sms, t)
        return
    assert not expected_refusal(M, t, num_sms), (M, N, K, gran, num_sms, t, pl)
    assert pl["layout"] == bsg.LAYOUTS[layout] and pl["gran"] == gran and pl["kernels"] == 1
    assert 1 <= pl["grid"] <= num_sms
    Kb = cdiv(K, gran)
    if t and t["variant"] != "auto":
        assert pl["cta_pair"] == (t["variant"] == "cta_pair")
        if t["variant"] != "cta_pair":
            assert pl["swap_ab"] == (t["variant"] == "swap_ab")
    if pl["cta_pair"]:
        assert pl["bnq"] == 256 and pl["splits"] == 1 and pl["sk_ctas"] == 0 and pl["grid"] % 2 == 0
        assert pl["tiles_p"] == cdiv(M, 256) and pl["tiles_q"] == cdiv(N, 256)
        assert pl["grid"] == 2 * min(pl["tiles_p"] * pl["tiles_q"], num_sms // 2)
        return
    P, Q = (N, M) if pl["swap_ab"] else (M, N)
    assert pl["bnq"] in ((16, 32, 64, 128) if pl["swap_ab"] else (128, 256))
    if t and t["bnq"]:
        assert pl["bnq"] == t["bnq"]
    assert pl["tiles_p"] == cdiv(P, 128) and pl["tiles_q"] == cdiv(Q, pl["bnq"])
    tiles = pl["tiles_p"] * pl["tiles_q"]
    s, per = pl["splits"], pl["kb_per_split"]
    assert s >= 1 and s * per >= Kb > (s - 1) * per
    if gran == 64:
        assert per % 2 == 0 or s == 1
    if t and t["splits"] > 0:
        assert pl["sk_ctas"] == 0 and s <= t["splits"]
    if t and t["stream_k"] == -1:
        assert pl["sk_ctas"] == 0
    U = cdiv(Kb, 2 if gran == 64 else 1)
    assert pl["sk_units_per_tile"] == U
    if pl["sk_ctas"] > 0:
        assert s == 1 and pl["sk_first_tile"] % num_sms == 0 and pl["sk_first_tile"] < tiles
        assert pl["sk_units"] == (tiles - pl["sk_first_tile"]) * U
        assert 1 <= pl["sk_ctas"] <= min(num_sms, pl["sk_units"])
        assert pl["grid"] == min(num_sms, max(pl["sk_first_tile"], pl["sk_ctas"]))
    else:
        assert pl["grid"] == min(num_sms, tiles * s)
