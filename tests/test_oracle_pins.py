"""Pins for the fp64 oracle: each test ties a part of the oracle to something
other than itself -- values the pages print, closed forms, special cases that
reduce to a textbook or library result, invariants, or brute force on tiny
inputs. Chosen so a dropped term, a wrong sign or index, or a transposed
operand in the oracle fails at least one of them.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def rng(seed=0):
    return np.random.default_rng(seed)


def rand_expert(r, H, I, scale=0.3):
    return (r.normal(0, scale, (I, H)), r.normal(0, scale, (I, H)), r.normal(0, scale, (I, H)))


# ---------------------------------------------------------------- bf16 / int4


def test_bf16_round_matches_library_for_fp32_inputs():
    # For values exactly representable in fp32, nearest-even rounding to bf16
    # must equal torch's fp32 -> bf16 conversion (a library routine).
    torch = pytest.importorskip("torch")
    r = rng(1)
    x = np.concatenate([r.normal(0, 1, 4000), r.normal(0, 1e-3, 1000), r.normal(0, 300, 1000)])
    x = x.astype(np.float32)
    # include exact halfway cases: 1 + 2^-8 (ties to 1), 1 + 3*2^-8 (ties up to 1 + 2^-6)
    x = np.concatenate([x, np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2.0 ** -126 * 1.5],
                                    dtype=np.float32)])
    ours = O.f64_to_bf16_bits_rne(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(ours, ref)
    assert O.bf16_round(np.array([1 + 2 ** -8]))[0] == 1.0
    assert O.bf16_round(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6


def test_bf16_decode_known_patterns():
    bits = np.array([0x3F80, 0xBF80, 0x4000, 0x0000, 0x3F81, 0x4300], dtype=np.uint16)
    vals = O.bf16_bits_to_f64(bits)
    assert vals.tolist() == [1.0, -1.0, 2.0, 0.0, 1.0 + 2 ** -7, 128.0]


def test_int4_unpack_known_bytes():
    # element 2i = low nibble, 2i+1 = high nibble, two's complement
    packed = np.array([[0x80, 0x7F, 0x12, 0xF0]], dtype=np.uint8)
    assert O.int4_unpack(packed).tolist() == [[0, -8, -1, 7, 2, 1, 0, -1]]


def test_int4_dequant_group_boundaries():
    I, H = 128, 128
    codes = np.full((I, H // 2), 0x11, dtype=np.uint8)  # every element q = 1
    s_rows = np.arange(1, I * (H // 64) + 1, dtype=np.float64).reshape(I, H // 64)
    W = O.dequant_rows_int4(codes, s_rows)
    assert W[5, 63] == s_rows[5, 0] and W[5, 64] == s_rows[5, 1]
    s_down = np.arange(1, (I // 64) * H + 1, dtype=np.float64).reshape(I // 64, H)
    Dt = O.dequant_down_t_int4(codes, s_down)
    assert Dt[63, 7] == s_down[0, 7] and Dt[64, 7] == s_down[1, 7]
    codes2 = np.full((I, H // 2), 0x9F, dtype=np.uint8)  # low -1, high -7
    W2 = O.dequant_rows_int4(codes2, np.ones((I, H // 64)))
    assert W2[0, 0] == -1 and W2[0, 1] == -7


# ---------------------------------------------------------------- SiLU


def test_silu_identities():
    z = np.linspace(-20, 20, 401)
    s = O.silu(z)
    assert O.silu(np.array([0.0]))[0] == 0.0
    # z*sigmoid(z) - (-z)*sigmoid(-z) = z (sigmoid(z) + sigmoid(-z) = 1)
    assert np.allclose(s - O.silu(-z), z, atol=1e-12)
    assert abs(O.silu(np.array([40.0]))[0] - 40.0) < 1e-12
    h = 1e-6
    assert abs((O.silu(np.array([h]))[0] - O.silu(np.array([-h]))[0]) / (2 * h) - 0.5) < 1e-9
    assert abs(O.silu(np.array([1.0]))[0] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15


# ---------------------------------------------------------------- router / top-k


def test_topk_set_is_best_subset_bruteforce():
    r = rng(2)
    for E in range(2, 9):
        for k in range(1, E + 1):
            x = r.normal(0, 1, 6)
            R = r.normal(0, 1, (E, 6))
            ids, w, logits, _ = O.route_topk(x, R, k)
            best = max(itertools.combinations(range(E), k), key=lambda S: sum(logits[list(S)]))
            assert set(ids.tolist()) == set(best)
            assert all(logits[ids[i]] >= logits[ids[i + 1]] for i in range(k - 1))


def test_topk_ties_go_to_lowest_index():
    R = np.zeros((7, 4))
    ids, w, logits, margin = O.route_topk(np.ones(4), R, 3)
    assert ids.tolist() == [0, 1, 2]
    assert np.allclose(w, 1 / 3)
    assert margin == 0.0
    R2 = np.zeros((6, 2))
    R2[:, 0] = [1, 3, 3, 2, 3, 0]
    ids2, _, _, _ = O.route_topk(np.array([1.0, 0.0]), R2, 4)
    assert ids2.tolist() == [1, 2, 4, 3]


def test_topk_decision_taken_in_fp32():
    # two logits that differ only below fp32 resolution tie in fp32 -> lower index
    R = np.array([[1.0, 0.0], [1.0 + 1e-12, 0.0]])
    ids, _, logits, _ = O.route_topk(np.array([1.0, 0.0]), R, 1)
    assert logits[1] > logits[0] and ids.tolist() == [0]


def test_two_expert_weights_are_logistic():
    # softmax restricted to two experts: w_1 = sigmoid(l_1 - l_2) (textbook identity)
    r = rng(3)
    for _ in range(20):
        x = r.normal(0, 1, 5)
        R = r.normal(0, 1, (9, 5))
        ids, w, logits, _ = O.route_topk(x, R, 2)
        d = logits[ids[0]] - logits[ids[1]]
        assert abs(w[0] - 1 / (1 + math.exp(-d))) < 1e-14
        assert abs(w.sum() - 1) < 1e-15


def test_router_onehot_rows_closed_form():
    H, E = 16, 5
    cols = [3, 0, 11, 7, 3]
    c = [2.0, -1.0, 0.5, 3.0, -4.0]
    R = np.zeros((E, H))
    for e in range(E):
        R[e, cols[e]] = c[e]
    x = np.arange(1, H + 1, dtype=np.float64)
    logits = O.router_logits(x, R)
    assert logits.tolist() == [c[e] * x[cols[e]] for e in range(E)]


def test_margin_is_gap_at_boundary():
    R = np.array([[5.0], [1.0], [4.0], [2.0]])
    ids, _, _, margin = O.route_topk(np.array([1.0]), R, 2)
    assert ids.tolist() == [0, 2] and margin == 2.0
    _, _, _, m_all = O.route_topk(np.array([1.0]), R, 4)
    assert m_all == math.inf


def test_tie_positions_flags_only_near_ties():
    logits = np.array([1.0, 0.5, 0.5 + 5e-6, -1.0])
    ids = O.topk_order(logits, 2)
    assert ids.tolist() == [0, 2]
    assert O.tie_positions(logits, ids) == {1}


# ---------------------------------------------------------------- experts


def perm_expert(H, I, a, b, p1, p2, p3):
    G = np.zeros((I, H)); V = np.zeros((I, H)); Dt = np.zeros((I, H))
    for i in range(I):
        G[i, p1[i]] = a
        V[i, p2[i]] = b
        Dt[i, p3[i]] = 1.0
    return G, V, Dt


def test_swiglu_expert_permutation_closed_form():
    # G = a P1, V = b P2, D^T rows one-hot at p3: y[p3(j)] = silu(a x[p1 j]) * b x[p2 j]
    r = rng(4)
    for H, I in [(8, 8), (12, 5)]:
        p1 = r.permutation(H)[:I]; p2 = r.permutation(H)[:I]; p3 = r.permutation(H)[:I]
        a, b = 0.7, -1.3
        x = r.normal(0, 1, H)
        y = O.swiglu_expert(x, *perm_expert(H, I, a, b, p1, p2, p3))
        want = np.zeros(H)
        for j in range(I):
            z = a * x[p1[j]]
            want[p3[j]] = z / (1 + math.exp(-z)) * (b * x[p2[j]])
        assert np.allclose(y, want, rtol=0, atol=1e-14)


def test_expert_is_linear_in_down_and_gate_up_roles_differ():
    r = rng(5)
    H, I = 16, 8
    G, V, Dt = rand_expert(r, H, I)
    x = r.normal(0, 1, H)
    y = O.swiglu_expert(x, G, V, Dt)
    assert np.allclose(O.swiglu_expert(x, G, V, 3 * Dt), 3 * y, atol=1e-13)
    assert np.all(O.swiglu_expert(x, G, V, 0 * Dt) == 0)
    # gate passes through phi, up does not: swapping them changes the result
    assert not np.allclose(O.swiglu_expert(x, V, G, Dt), y)
    # V = 0 kills the output (a_j = phi(g) * 0)
    assert np.all(O.swiglu_expert(x, G, 0 * V, Dt) == 0)


def make_layer(r, H, E, I, scale=0.3):
    experts = [rand_expert(r, H, I, scale) for _ in range(E)]
    R = r.normal(0, 1, (E, H))
    return R, experts


def test_k_equals_E_is_dense_softmax_mixture():
    r = rng(6)
    for H, E, I in [(16, 4, 8), (24, 7, 5)]:
        R, ex = make_layer(r, H, E, I)
        x = r.normal(0, 1, H)
        y, ids, w, logits, _ = O.moe_layer(x, R, lambda e: ex[e], E)
        dense = O.dense_mixture(x, R, lambda e: ex[e], E)
        assert np.allclose(y, dense, rtol=1e-12, atol=1e-14)
        assert np.allclose(w, O.softmax(logits)[ids], rtol=1e-14)


def test_k1_selects_argmax_expert_with_weight_one():
    r = rng(7)
    R, ex = make_layer(r, 16, 6, 8)
    x = r.normal(0, 1, 16)
    y, ids, w, logits, _ = O.moe_layer(x, R, lambda e: ex[e], 1)
    e = int(np.argmax(logits))
    assert ids.tolist() == [e] and w.tolist() == [1.0]
    assert np.array_equal(y, O.swiglu_expert(x, *ex[e]))


def test_expert_relabelling_invariance():
    # Relabel experts by a permutation pi (router rows and weights together):
    # y is unchanged and ids are relabelled. Catches slot/id mix-ups.
    r = rng(8)
    H, E, I, k = 16, 8, 4, 3
    R, ex = make_layer(r, H, E, I)
    x = r.normal(0, 1, H)
    y, ids, w, _, _ = O.moe_layer(x, R, lambda e: ex[e], k)
    pi = r.permutation(E)  # new expert e' holds old expert pi[e']
    y2, ids2, w2, _, _ = O.moe_layer(x, R[pi], lambda e: ex[pi[e]], k)
    assert np.allclose(y, y2, atol=1e-13)
    assert [int(pi[e]) for e in ids2] == ids.tolist()
    assert np.allclose(w, w2)


def test_shared_expert_is_added_with_unit_weight():
    r = rng(9)
    H, E, I = 16, 5, 4
    R, ex = make_layer(r, H, E, I)
    sh = rand_expert(r, H, 6)
    x = r.normal(0, 1, H)
    y0, *_ = O.moe_layer(x, R, lambda e: ex[e], 2)
    y1, *_ = O.moe_layer(x, R, lambda e: ex[e], 2, shared=sh)
    assert np.allclose(y1 - y0, O.swiglu_expert(x, *sh), atol=1e-13)


def test_residual_keeps_bf16_input_when_y_zero():
    x = O.bf16_round(rng(10).normal(0, 1, 64))
    assert np.array_equal(O.residual_bf16(x, np.zeros(64)), x)
    # 1 + 2^-9 is below half an ulp of bf16 at 1: rounds back to 1
    assert O.residual_bf16(np.array([1.0]), np.array([2 ** -9]))[0] == 1.0


def test_linear_experts_closed_forms():
    r = rng(11)
    H = 10
    x = r.normal(0, 1, H)
    c = [0.5, -2.0, 3.0, 1.5]
    y = O.linear_experts(x, lambda e: c[e] * np.eye(H), [2, 0, 3], [1.0, 1.0, 0.25])
    assert np.allclose(y, (3.0 + 0.5 + 0.25 * 1.5) * x, atol=1e-14)
    P = np.zeros((H, H)); perm = r.permutation(H)
    P[np.arange(H), perm] = 1.0  # (P x)[i] = x[perm[i]]
    y2 = O.linear_experts(x, lambda e: P, [0], [1.0])
    assert np.array_equal(y2, x[perm])


# ---------------------------------------------------------------- touched experts


def test_touched_formula_matches_printed_theory_column():
    g = golden("touched_batch_sweep.json")
    for B, printed in zip(g["batch"], g["theory_printed"]):
        assert round(O.expected_touched(g["E"], g["k"], B), 1) == printed


def test_touched_worked_example_printed_values():
    g = golden("touched_batch_sweep.json")
    we = g["worked_example"]
    q = 1 - g["k"] / g["E"]
    assert round(q, 3) == we["p_not_chosen_by_one_token"]
    assert round(q ** we["B"], 2) == we["p_not_chosen_by_16_tokens"]
    assert round(1 - q ** we["B"], 2) == we["p_touched"]


def test_half_touch_batch_printed_is_small_p_approximation():
    g = golden("touched_batch_sweep.json")
    approx = O.half_touch_batch_small_p(g["E"], g["k"])
    exact = O.half_touch_batch_exact(g["E"], g["k"])
    assert round(approx, 1) == g["half_touch_batch_printed"]
    assert abs(exact - 14.44) < 0.01
    assert abs((1 - g["k"] / g["E"]) ** exact - 0.5) < 1e-12


def test_touched_monte_carlo_within_sampling_error():
    g = golden("touched_batch_sweep.json")
    E, k = g["E"], g["k"]
    r = rng(12)
    draws = 2000
    for B in g["batch"]:
        counts = np.empty(draws)
        for t in range(draws):
            ids = np.stack([r.permutation(E)[:k] for _ in range(B)])
            counts[t] = O.touched_experts(ids, E)[0]
        theory = O.expected_touched(E, k, B)
        # standard error: the sample's, floored by the independent-indicator
        # bound sqrt(E p (1-p) / draws) with p = P(an expert is missed)
        p_miss = (1 - k / E) ** B
        se = max(counts.std(ddof=1), math.sqrt(E * p_miss * (1 - p_miss))) / math.sqrt(draws)
        assert abs(counts.mean() - theory) <= 4 * se + 1e-12, (B, counts.mean(), theory)
        if B == 1:
            assert np.all(counts == k)


def test_touched_counting_sort_bruteforce():
    r = rng(13)
    for B, k, E in [(1, 2, 16), (5, 3, 8), (8, 8, 256), (16, 3, 64)]:
        ids = np.stack([r.permutation(E)[:k] for _ in range(B)])
        count, bitmap, offsets, pairs = O.touched_experts(ids, E)
        flat = ids.reshape(-1)
        assert count == len(set(flat.tolist()))
        assert offsets[0] == 0 and offsets[-1] == B * k
        assert np.all(np.diff(offsets) >= 0)
        assert sorted(pairs.tolist()) == list(range(B * k))
        for e in range(E):
            seg = pairs[offsets[e]:offsets[e + 1]]
            assert np.all(np.diff(seg) > 0)
            assert all(flat[p] == e for p in seg)
            bit = (int(bitmap[e // 32]) >> (e % 32)) & 1
            assert bit == (1 if len(seg) else 0)


# ---------------------------------------------------------------- channel-sparse


def test_sector_example_from_fig2c():
    g = golden("sector_example.json")
    # 80 needed bytes as four 20-byte pieces, each in its own 32-byte sector
    ranges = [(0, 20), (70, 90), (128, 148), (300, 320)]
    assert sum(hi - lo for lo, hi in ranges) == g["bytes_needed"]
    n = O.sectors_touched(ranges)
    assert n == g["sectors_touched"]
    assert n * g["sector_bytes"] == g["bytes_charged"]
    # the same 80 bytes packed at a sector boundary need 3 sectors
    assert O.sectors_touched([(0, 80)]) == 3
    assert O.sectors_touched([(31, 33)]) == 2
    assert O.sectors_touched([(0, 10), (5, 20)]) == 1


def test_sectors_of_aligned_channel_major_rows():
    H, I = 2048, 768
    kept = [0, 1, 5, 767, 768, 6143]
    ranges = O.channel_major_ranges(kept, H)
    assert O.sectors_touched(ranges) == 384 * len(kept)
    # an unaligned base straddles one extra sector per non-adjacent run
    assert O.sectors_touched(O.channel_major_ranges([0, 1], H, base=16)) == 2 * 384 + 1


def test_channel_select_bruteforce_and_ties():
    r = rng(14)
    E, I = 5, 3
    for keep in range(0, 7):
        S = r.normal(0, 1, (E, I))
        ids = [4, 1]
        kept = O.channel_topk_select(S, ids, keep)
        cand = [e * I + c for e in ids for c in range(I)]
        best = max(itertools.combinations(cand, keep),
                   key=lambda T: sum(S[j // I, j % I] for j in T)) if keep else ()
        assert set(kept.tolist()) == set(best)
    T = np.zeros((4, 2))
    assert O.channel_topk_select(T, [3, 1], 3).tolist() == [2, 3, 6]


def channel_view(ex, I):
    return lambda e, c: np.stack([ex[e][0][c], ex[e][1][c], ex[e][2][c]])


def test_channel_keep_all_equals_planar_experts():
    r = rng(15)
    H, E, I, k = 16, 6, 5, 3
    R, ex = make_layer(r, H, E, I)
    x = r.normal(0, 1, H)
    ids, w, _, _ = O.route_topk(x, R, k)
    S = np.abs(r.normal(0, 1, (E, I)))
    kept = O.channel_topk_select(S, ids, k * I)
    y_sparse = O.channel_sparse_forward(x, channel_view(ex, I), ids, w, kept, I)
    y_planar = O.moe_experts_given(x, lambda e: ex[e], ids, w)
    assert np.allclose(y_sparse, y_planar, rtol=1e-12, atol=1e-14)
    y0 = O.channel_sparse_forward(x, channel_view(ex, I), ids, w, [], I)
    assert np.all(y0 == 0)


def test_channel_partial_keep_equals_masked_planar():
    # keeping a subset equals the planar expert with the dropped channels'
    # down rows zeroed
    r = rng(16)
    H, E, I, k = 12, 4, 6, 2
    R, ex = make_layer(r, H, E, I)
    x = r.normal(0, 1, H)
    ids, w, _, _ = O.route_topk(x, R, k)
    S = np.abs(r.normal(0, 1, (E, I)))
    kept = O.channel_topk_select(S, ids, 5)
    keep_set = set(kept.tolist())

    def masked(e):
        G, V, Dt = ex[e]
        Dm = Dt.copy()
        for c in range(I):
            if e * I + c not in keep_set:
                Dm[c] = 0
        return G, V, Dm
    y = O.channel_sparse_forward(x, channel_view(ex, I), ids, w, kept, I)
    assert np.allclose(y, O.moe_experts_given(x, masked, ids, w), atol=1e-13)


# ---------------------------------------------------------------- bytes / ceilings


def test_decode_ceilings_match_moe_promise():
    g = golden("decode_ceilings.json")
    gb = g["gb_per_token"]["Qwen3.5-35B-A3B-4bit"]
    fr = []
    for m, bw in g["achieved_gbs"].items():
        c = O.decode_ceiling(bw, gb)
        assert round(c) == g["moe_ceiling_printed"][m]
        fr.append(100 * g["moe_measured_printed"][m] / c)
    lo, hi = g["moe_fraction_range_printed_pct"]
    assert round(min(fr)) == lo and round(max(fr)) == hi
    big = g["large_moe_example"]
    assert round(O.decode_ceiling(big["achieved_gbs"], big["gb_per_token"])) == big["tok_s_printed"]


def test_beam_memory_table():
    g = golden("beam_memory.json")
    assert round(O.param_bytes(g["total_params"], 16) / 1e9) == g["bf16"]["resident_gb_printed"]
    assert round(O.param_bytes(g["active_params"], 16) / 1e9) == g["bf16"]["per_token_gb_printed"]
    assert abs(O.param_bytes(g["total_params"], 4) / 1e9 - g["int4"]["resident_gb_printed"]) <= 0.5
    assert O.param_bytes(g["active_params"], 4) / 1e9 == g["int4"]["per_token_gb_printed"]
    assert round(100 * g["active_params"] / g["total_params"], 1) == g["active_ratio_pct_printed"]


def test_reader_layer_bytes_vs_table7():
    g = golden("reader_shapes.json")
    q = g["table3"]["Qwen3-Thinking"]
    assert q["k"] * q["I"] == g["candidates_per_layer_printed"]
    routed = q["k"] * O.swiglu_expert_bytes(q["H"], q["I"])
    assert routed == 75_497_472
    # the profiler's cold-cache figure (router excluded) is within 0.2% of the count
    assert abs(routed / 1e6 - g["table7_full_model_mb"]["1"]) / g["table7_full_model_mb"]["1"] < 2e-3
    # real routing touches no more experts than the uniform-routing bound
    for B in (4, 8):
        bound = O.expected_touched(q["E"], q["k"], B) * O.swiglu_expert_bytes(q["H"], q["I"]) / 1e6
        assert g["table7_full_model_mb"][str(B)] <= bound


def test_layer_bytes_closed_forms():
    # A3B-like layer: 8 routed + shared (I=512) + 256x2048 router, bf16
    assert O.layer_bytes_b1(2048, 256, 512, 8, I_shared=512) == 57_671_680
    assert O.swiglu_expert_bytes(2048, 512, "int4") == 1_671_168
    assert O.layer_bytes_b1(2048, 256, 512, 8, I_shared=512, wtype="int4") == 20_709_376
    assert O.layer_bytes_b1(512, 16, 256, 2) == 1_589_248


# ---------------------------------------------------------------- stack pre-norm


def test_rmsnorm_closed_forms():
    # constant vector c: mean(x^2) = c^2, so u = c / sqrt(c^2 + eps) ~ sign(c)
    x = np.full(64, 3.0)
    u = O.rmsnorm_bf16(x)
    assert np.all(u == O.bf16_round(np.array([3.0 / math.sqrt(9.0 + O.RMS_EPS)]))[0])
    # scale invariance (up to eps): rms(a x) normalises to the same u
    r = rng(17)
    x = r.normal(0, 1, 256)
    assert np.array_equal(O.rmsnorm_bf16(x), O.rmsnorm_bf16(1024.0 * x))
    # unit rms output (before bf16 rounding: within bf16 precision)
    assert abs(np.sqrt(np.mean(O.rmsnorm_bf16(x) ** 2)) - 1.0) < 1e-2


def test_stack_layer_residual_uses_unnormalised_x():
    r = rng(18)
    H, E, I, k = 32, 4, 8, 2
    R, ex = make_layer(r, H, E, I)
    x = O.bf16_round(r.normal(0, 5, H))
    xn, y, ids, w, _, _ = O.stack_layer(x, R, lambda e: ex[e], k)
    u = O.rmsnorm_bf16(x)
    y2, ids2, *_ = O.moe_layer(u, R, lambda e: ex[e], k)
    assert np.allclose(y, y2) and ids.tolist() == ids2.tolist()
    assert np.array_equal(xn, O.residual_bf16(x, y))
    xn0, y0, *_ = O.stack_layer(x, R, lambda e: ex[e], k, pre_norm=False)
    assert np.allclose(y0, O.moe_layer(x, R, lambda e: ex[e], k)[0])


# ---------------------------------------------------------------- reader screen
# [Reader] "가중치만으로 만든 reader", step 1 (rotated ternary sketch) and
# step 2 (eq. 1 scores).


def test_hadamard_matches_popcount_definition_and_is_orthogonal():
    # Sylvester's recursion against the closed form H[i][j] = (-1)^popcount(i & j),
    # and H H^T = n I (so R = H diag(s) / sqrt(n) is orthogonal).
    for n in (1, 2, 8, 128):
        h = O.sylvester_hadamard(n)
        i = np.arange(n)
        closed = np.array([[(-1.0) ** bin(a & b).count("1") for b in i] for a in i])
        assert np.array_equal(h, closed)
        assert np.array_equal(h @ h.T, n * np.eye(n))


def test_rotation_preserves_dot_products():
    # The page's reason for the rotation: g^T x = (R g)^T (R x). With the
    # unnormalised u = H (s * v) that is u_g . u_x / 128.
    r = rng(41)
    H = 512
    s = r.choice([-1.0, 1.0], H)
    g, x = O.bf16_round(r.normal(0, 0.02, H)), O.bf16_round(r.normal(0, 1, H))
    lhs = float(O.reader_rotate(g, s) @ O.reader_rotate(x, s)) / 128
    assert abs(lhs - float(g @ x)) <= 1e-12 * float(np.abs(g) @ np.abs(x)) * 128
    # a basis vector e_h maps to s_h times column h % 128 of H_128 in its block
    e = np.zeros(H)
    e[300] = 1.0
    u = O.reader_rotate(e, s).reshape(-1, 128)
    col = O.sylvester_hadamard(128)[:, 300 % 128] * s[300]
    assert np.array_equal(u[300 // 128], col)
    assert not np.any(np.delete(u, 300 // 128, axis=0))


def test_ternary_block_hand_example():
    # mean|u| = 21/128, delta = 0.7 * 21/128 ~ 0.115: codes (+1, -1, +1), the
    # scale the mean |u| of those three = 7, rho = (3^2 + 3^2 + 6^2) / 128 / 128.
    u = np.zeros(128)
    u[:3] = (10.0, -10.0, 1.0)
    codes, scale, rho = O.ternary_block(u)
    assert codes[:3].tolist() == [1, -1, 1] and not np.any(codes[3:])
    assert scale == 7.0
    assert abs(rho - (9 + 9 + 36) / 128 / 128) <= 1e-15  # 1/sqrt(128) is not exact in fp64
    # every |u| equal to the mean: delta = 0.7 * mean < |u| keeps them all;
    # a single value carrying the whole mass is the only code kept
    c2, s2, _ = O.ternary_block(np.full(128, -2.0))
    assert np.all(c2 == -1) and s2 == 2.0
    u3 = np.zeros(128)
    u3[5] = 100.0
    c3, s3, _ = O.ternary_block(u3)
    assert c3[5] == 1 and s3 == 100.0 and np.count_nonzero(c3) == 1


def test_ternary_block_exact_for_ternary_input_and_zero_block():
    # u = a * c with c ternary: delta = 0.7 a nnz/128 < a, so the codes are c,
    # the scale a (exact in fp16 for a = 0.375), rho = 0. All-zero block: no codes.
    r = rng(42)
    c = r.choice([-1, 0, 1], 128).astype(np.int8)
    codes, scale, rho = O.ternary_block(0.375 * c)
    assert np.array_equal(codes, c) and scale == 0.375 and rho == 0.0
    codes, scale, rho = O.ternary_block(np.zeros(128))
    assert not np.any(codes) and scale == 0.0 and rho == 0.0


def test_fp16_scale_rounding_matches_library():
    # fp64 -> fp32 -> fp16 round-to-nearest-even against torch's conversions.
    torch = pytest.importorskip("torch")
    r = rng(43)
    for a in r.uniform(1e-4, 30.0, 200):
        want = torch.tensor(a, dtype=torch.float64).to(torch.float32).to(torch.float16).item()
        assert O.fp16_through_fp32(a) == want


def test_estimate_is_exact_when_the_row_is_its_own_sketch():
    # A row built from ternary codes and fp16 scales by the inverse rotation
    # (H^-1 = H / 128, diag(s)^-1 = diag(s)) has that sketch exactly, and the
    # estimate then equals the true dot product.
    r = rng(44)
    H = 256
    s = r.choice([-1.0, 1.0], H)
    c = r.choice([-1, 0, 1], H).astype(np.int8)
    scales = np.array([0.5, 0.25])
    u = (c.reshape(-1, 128) * scales[:, None]).reshape(-1)
    hm = O.sylvester_hadamard(128)
    row = s * ((u.reshape(-1, 128) @ hm) / 128).reshape(-1)
    codes, sc, rho = O.reader_sketch_row(row, s)
    assert np.array_equal(codes, c) and np.array_equal(sc, scales) and np.all(rho == 0)
    x = O.bf16_round(r.normal(0, 1, H))
    assert abs(O.reader_estimate(x, codes, sc, s) - float(row @ x)) <= 1e-12 * float(np.abs(row) @ np.abs(x)) * 64


def test_estimate_error_bounded_by_rho():
    # Cauchy-Schwarz per block: |g^T x - g_hat| <= sum_b sqrt(128 rho_b) ||R x_b||
    # (the error vector of block b has squared norm 128 rho_b in the
    # orthonormal rotation's units).
    r = rng(45)
    H = 512
    s = r.choice([-1.0, 1.0], H)
    g = O.bf16_round(r.normal(0, 0.02, H))
    x = O.bf16_round(r.normal(0, 1, H))
    codes, sc, rho = O.reader_sketch_row(g, s)
    ux = O.reader_rotate(x, s).reshape(-1, 128) / math.sqrt(128)
    bound = float(np.sum(np.sqrt(128 * rho) * np.linalg.norm(ux, axis=1)))
    err = abs(float(g @ x) - O.reader_estimate(x, codes, sc, s))
    assert err <= bound * (1 + 1e-9)
    assert 0 < err  # a real approximation


def test_eq1_score_hand_values():
    # s = w ||d|| |phi(g) v| with phi = SiLU: 0.5 * 2 * |silu(1) * (-3)| = 3 / (1 + e^-1)
    assert abs(O.reader_score(0.5, 2.0, 1.0, -3.0) - 3.0 / (1.0 + math.exp(-1.0))) < 1e-15
    # the sign of v_hat and of phi(g_hat) do not matter; a zero estimate scores 0
    assert O.reader_score(0.5, 2.0, -1.0, 3.0) == O.reader_score(0.5, 2.0, -1.0, -3.0)
    assert O.reader_score(0.5, 2.0, 0.0, 5.0) == 0.0


def test_partial_mask_bruteforce_and_ties():
    # The mask against a direct count per coordinate: i is kept iff fewer than
    # m coordinates of its block beat it (larger |u|, or equal and lower index).
    r = rng(46)
    H = 256
    s = r.choice([-1.0, 1.0], H)
    x = O.bf16_round(r.normal(0, 1, H))
    for m in (0, 1, 80, 127, 128):
        mask = O.reader_partial_mask(x, s, m).reshape(-1, 128)
        ua = np.abs(O.reader_rotate(x, s)).reshape(-1, 128)
        for b in range(ua.shape[0]):
            for i in range(128):
                beat = np.sum(ua[b] > ua[b, i]) + np.sum((ua[b] == ua[b, i]) & (np.arange(128) < i))
                assert mask[b, i] == (beat < m)
    # ties: x = e_0 rotates to +-1 everywhere in block 0; the first 80 indices win
    e0 = np.zeros(H)
    e0[0] = 1.0
    mk = O.reader_partial_mask(e0, s, 80).reshape(-1, 128)
    assert mk[0, :80].all() and not mk[0, 80:].any()


def test_partial_estimate_special_cases():
    # m = 128 reads every code (the full estimate); m = 0 reads none.
    r = rng(47)
    H = 256
    s = r.choice([-1.0, 1.0], H)
    g = O.bf16_round(r.normal(0, 0.02, H))
    x = O.bf16_round(r.normal(0, 1, H))
    codes, sc, _ = O.reader_sketch_row(g, s)
    assert O.reader_estimate_partial(x, codes, sc, s, 128) == O.reader_estimate(x, codes, sc, s)
    assert O.reader_estimate_partial(x, codes, sc, s, 0) == 0.0
    # the dropped coordinates are those of smallest |Rx|: with codes all +1
    # and unit scales, the partial estimate is the sum of the kept u_x / 128
    ones = np.ones(H, dtype=np.int8)
    ux = O.reader_rotate(x, s)
    keep = O.reader_partial_mask(x, s, 80)
    got = O.reader_estimate_partial(x, ones, np.ones(2), s, 80)
    assert abs(got - ux[keep].sum() / 128) <= 1e-12 * np.abs(ux).sum()


def test_recovery_full_rank_is_exact():
    # Eq. 2 with rank = H (U square, orthogonal): U b_j = U U^T d_j = d_j, so the
    # recovered part is sum_S w_j p_j d_j exactly; with p_j = a_j the output is
    # the all-kept (dense) channel output.
    r = rng(48)
    H, n = 16, 40
    D = r.normal(0, 1, (n, H))
    U = O.recovery_basis(D, rank=H)
    assert np.allclose(U.T @ U, np.eye(H), atol=1e-12)
    w = r.uniform(0.1, 1.0, n)
    a = r.normal(0, 1, n)
    kept = [0, 3, 7]
    dropped = [j for j in range(n) if j not in kept]
    y = O.reader_output([(w[j], a[j], D[j]) for j in kept],
                        [(w[j], a[j], O.recovery_coeffs(U, D[j])) for j in dropped], U)
    dense = sum(w[j] * a[j] * D[j] for j in range(n))
    assert np.allclose(y, dense, atol=1e-10)


def test_recovery_exact_on_low_rank_columns_and_eckart_young():
    # Down columns inside a 3-dim subspace: a rank-3 basis spans them, so the
    # recovery of every dropped channel is exact. And the residual of the
    # rank-r projection of D is the sum of the squared trailing singular values.
    r = rng(49)
    H, n, k = 24, 60, 3
    A = r.normal(0, 1, (H, k))
    D = (A @ r.normal(0, 1, (k, n))).T
    U = O.recovery_basis(D, rank=k)
    for j in range(n):
        assert np.allclose(U @ O.recovery_coeffs(U, D[j]), D[j], atol=1e-10)
    D2 = r.normal(0, 1, (n, H))
    s = np.linalg.svd(D2.T, compute_uv=False)
    for rank in (1, 5, 12):
        U2 = O.recovery_basis(D2, rank=rank)
        resid = D2.T - U2 @ (U2.T @ D2.T)
        assert abs(np.sum(resid ** 2) - np.sum(s[rank:] ** 2)) <= 1e-9 * np.sum(s ** 2)


def test_recovery_map_is_half_a_percent_of_a_channel():
    # [Reader] step 3: the map adds about 0.5% of resident memory. With 32 fp16
    # coefficients per channel against its 3 bf16 rows of H = 2048 (Qwen3-Thinking):
    frac = 32 * 2 / (3 * 2048 * 2)
    assert abs(frac - 0.005) < 0.0005


def test_channel_union_of_a_batch():
    # brute force against a set; one token gives its own kept list; tokens
    # with the same kept list read it once; disjoint lists add up
    r = rng(50)
    lists = [sorted(r.choice(600, 37, replace=False).tolist()) for _ in range(5)]
    u = O.channel_union(lists)
    assert u.tolist() == sorted(set().union(*map(set, lists)))
    assert O.channel_union(lists[:1]).tolist() == lists[0]
    assert O.channel_union([lists[0]] * 4).tolist() == lists[0]
    a, b = list(range(0, 10)), list(range(10, 25))
    assert O.channel_union([a, b]).size == 25
    assert O.channel_union([[], []]).size == 0
    # read bytes of the union: 384 sectors per aligned channel-major channel
    H = 2048
    assert O.sectors_touched(O.channel_major_ranges(u, H)) == 384 * u.size


def test_reader_screen_pairs_each_slot_with_its_own_weight_and_expert():
    # Two routed experts in slots (1, 0) with distinct slot weights, two
    # channels each. With x = e_0 and s_0 = +1 the rotated token is all ones in
    # block 0 (column 0 of H_128), so an estimate is scale * (sum of codes) / 128;
    # the sketch below gives every (expert, channel) its own (g_hat, v_hat), so
    # the eq. 1 scores follow in closed form. Pairing slot t with w[e] instead
    # of w[t], reading expert t instead of ids[t], or swapping the gate and up
    # sketches gives other numbers.
    H, I = 128, 2
    s = np.ones(H)
    x = np.zeros(H)
    x[0] = 1.0
    ids, w = [1, 0], [0.25, 0.75]
    half = np.zeros(H, dtype=np.int8)
    half[:64] = 1                                   # sum of codes = 64: estimate = scale / 2
    g_hat = {(0, 0): 1.0, (0, 1): -0.5, (1, 0): 2.0, (1, 1): 0.25}
    v_hat = {(0, 0): 3.0, (0, 1): 1.5, (1, 0): -1.0, (1, 1): 4.0}
    dn = {(0, 0): 1.0, (0, 1): 2.0, (1, 0): 0.5, (1, 1): 3.0}

    def sketch(e, c):
        return half, np.array([2 * g_hat[e, c]]), half, np.array([2 * v_hat[e, c]]), dn[e, c]

    scores, est = O.reader_screen(x, ids, w, sketch, I, s)
    sil = lambda z: z / (1.0 + math.exp(-z))
    for t, e in enumerate(ids):
        for c in range(I):
            assert est[t, c].tolist() == [g_hat[e, c], v_hat[e, c]]
            want = w[t] * dn[e, c] * abs(sil(g_hat[e, c]) * v_hat[e, c])
            assert abs(scores[t, c] - want) <= 1e-15 * want
    # the closed forms above are not symmetric in the plausible slips
    assert abs(scores[0, 0] - 0.25 * 0.5 * abs(sil(2.0) * -1.0)) < 1e-15
    assert scores[0, 0] != 0.75 * 0.5 * abs(sil(2.0) * -1.0)   # w[e] for e = 1 would be 0.75
    assert scores[0, 0] != 0.25 * 0.5 * abs(sil(-1.0) * 2.0)   # gate and up swapped
    assert scores[1, 0] != 0.75 * 1.0 * abs(sil(2.0) * -1.0)   # slot 1 read as expert 1


def test_channel_stack_layer_routes_and_computes_on_u_and_adds_y_to_x():
    # H = 4, E = 3, k = 2, I = 2 with one-hot router rows (logit of expert e =
    # u[h_e]), one-hot gate rows, scaled one-hot up rows and one-hot down
    # columns, so every a_j and y are closed forms of u = rmsnorm_bf16(x).
    # x has rms sqrt(10) != 1: routing on x (weights from 4, 2 instead of u's
    # 1.27, 0.63), experts fed x, or the residual added to u all change the result.
    H, E, I, k, keep = 4, 3, 2, 2, 3
    x = np.array([4.0, -4.0, 2.0, -2.0])
    u = O.rmsnorm_bf16(x)
    onehot = np.eye(H)
    R = onehot[[0, 2, 1]]                             # logits = (u0, u2, u1)
    scores = np.array([[5.0, 1.0], [4.0, 3.0], [9.0, 9.0]])  # expert 2 is not routed

    def channel(e, c):
        return np.stack([onehot[c], (e + 1) * onehot[c + 2], onehot[(e + c) % H]])

    xn, y, ids, w, logits, kept = O.channel_stack_layer(x, R, channel, scores, k, keep, I)
    assert np.array_equal(logits, u[[0, 2, 1]])
    assert ids.tolist() == [0, 1]
    w0 = 1.0 / (1.0 + math.exp(u[2] - u[0]))
    assert np.allclose(w, [w0, 1.0 - w0], rtol=0, atol=1e-15)
    assert kept.tolist() == [0, 2, 3]                 # scores 5, 4, 3 of the routed rows
    sil = lambda z: z / (1.0 + math.exp(-z))
    want = np.zeros(H)
    for e, c in ((0, 0), (1, 0), (1, 1)):
        a = sil(u[c]) * (e + 1) * u[c + 2]
        want[(e + c) % H] += w[list(ids).index(e)] * a
    assert np.allclose(y, want, rtol=0, atol=1e-14)
    assert np.array_equal(xn, O.residual_bf16(x, want))
    assert not np.array_equal(xn, O.residual_bf16(u, want))
    wx = 1.0 / (1.0 + math.exp(x[2] - x[0]))
    assert abs(w[0] - wx) > 0.1                       # routing on x is told apart
    # without the pre-norm the layer works on x itself
    _, y0, _, w_raw, l0, _ = O.channel_stack_layer(x, R, channel, scores, k, keep, I, pre_norm=False)
    assert np.array_equal(l0, x[[0, 2, 1]]) and abs(w_raw[0] - wx) < 1e-15
