"""GPU parity of the weight-only channel screen ([Reader] "가중치만으로 만든
reader", step 1: rotated ternary sketch; step 2, eq. 1: output-unit scores)
through the C ABI against the fp64 oracle.

Sketch: ternary codes and fp16 scales are compared bit-exactly. For these
bf16 rows every sum the rule needs is exact in fp64, so the oracle's matrix
product and the kernel's fp64 butterfly reach the same values and the same
decisions. rho (a sum of squares, order-dependent in fp64) within 1e-9
relative; dnorm within 2 fp32 ulps.

Screen: the estimates g_hat, v_hat within 1e-5 x B, where B =
sum_b scale_b n_b sum_{i in b}|x_i| / 128 (n_b nonzero codes) bounds every
partial sum of the estimate, rotation included. The kernel rounds in fp32 at
most ~32 times along any path (7 butterfly stages, 3 in a subset-sum table
entry, 8 combining a code word's table lookups, 4 accumulations per lane, 5
shuffle steps: 27): 32 x 2^-24 = 1.9e-6 x B, so 1e-5 leaves a factor 5.
Scores within the propagated bound w ||d|| (1.1 |v| dg + |SiLU(g)| dv + dg dv)
+ 1e-5 s (|SiLU'| <= 1.1; the last term covers fp32 dnorm and SiLU).
"""

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from tests.parity_util import REL_TOL, f64, rel_err

pytestmark = pytest.mark.gpu

DEV = "cuda"
EST_TOL = 1e-5


@pytest.fixture(scope="module")
def M():
    from mixture_experts_decode_moe_b200 import build
    build.build()
    from mixture_experts_decode_moe_b200 import moedec
    return moedec


@pytest.fixture(scope="module")
def S():
    from mixture_experts_decode_moe_b200 import synth
    return synth


def unpack_codes(words: np.ndarray, H: int) -> np.ndarray:
    """[..., H/16] uint32 words -> int8 codes [..., H] (documented 2-bit layout:
    bit 2i nonzero, bit 2i+1 negative; the pattern 0b10 never occurs)."""
    w = words.astype(np.uint64)[..., None]
    f = (w >> (2 * np.arange(16, dtype=np.uint64))) & np.uint64(3)
    assert not np.any(f == 2)
    c = np.where(f == 1, 1, np.where(f == 3, -1, 0)).astype(np.int8)
    return c.reshape(*words.shape[:-1], H)


def build_sketch(M, desc, signs):
    shp = M.reader_sketch_shapes(desc)
    codes = torch.empty(shp["codes"], dtype=torch.int32, device=DEV)
    scales = torch.empty(shp["scales"], dtype=torch.int16, device=DEV)
    rho = torch.empty(shp["rho"], dtype=torch.float32, device=DEV)
    dnorm = torch.empty(shp["dnorm"], dtype=torch.float32, device=DEV)
    M.moe_reader_build(desc, signs, codes, scales, rho, dnorm)
    torch.cuda.synchronize()
    return codes, scales, rho, dnorm


def host_sketch(codes, scales, rho, dnorm, H):
    c = unpack_codes(codes.cpu().numpy().view(np.uint32), H)
    s = scales.cpu().numpy().view(np.float16).astype(np.float64)
    return c, s, f64(rho), f64(dnorm)


def check_channel_sketch(cm_host, signs_np, c, s, r, dn, j, H):
    """Channel j: GPU sketch (codes c[j], scales s[j], rho r[j], dnorm dn[j])
    against the oracle's, built from the bf16 rows."""
    rows = cm_host(j)
    for row in range(2):
        oc, osc, orho = O.reader_sketch_row(rows[row], signs_np)
        assert np.array_equal(c[j, row], oc), (j, row)
        assert np.array_equal(s[j, row], osc), (j, row)
        assert np.allclose(r[j, row], orho, rtol=1e-6, atol=1e-30), (j, row)  # stored as fp32
    want = float(np.float32(np.sqrt(np.sum(rows[2] ** 2))))
    assert abs(dn[j] - want) <= 2 * np.spacing(np.float32(want)), j


@pytest.mark.parametrize("H,E,I", [(512, 4, 48), (2048, 2, 24), (128, 3, 8)])
def test_sketch_matches_oracle(M, S, H, E, I):
    Ld = S.channel_major_layer(H, E, I, seed=700 + H, device=DEV)
    cm = Ld["cm"]
    desc = M.make_desc(H, E, I, 2, layout=M.MOE_LAYOUT_CHANNEL_MAJOR, gate=cm)
    signs = S.reader_signs(H, seed=701, device=DEV)
    c, s, r, dn = host_sketch(*build_sketch(M, desc, signs), H)
    host = f64(cm).reshape(E * I, 3, H)
    sg = f64(signs)
    for j in range(E * I):
        check_channel_sketch(lambda q: host[q], sg, c, s, r, dn, j, H)


def est_and_score_tolerances(x, cg, sg, cv, sv, w_e, dn, gh, vh):
    tg = EST_TOL * O.reader_estimate_bound(x, cg, sg)
    tv = EST_TOL * O.reader_estimate_bound(x, cv, sv)
    silu = float(O.silu(np.float64(gh)))
    ts = w_e * dn * (1.1 * abs(vh) * tg + abs(silu) * tv + tg * tv) + 1e-5 * O.reader_score(w_e, dn, gh, vh)
    return tg, tv, ts


@pytest.mark.parametrize("H,E,I,k,B", [(512, 8, 64, 3, 2), (2048, 6, 40, 4, 3), (128, 4, 16, 2, 1)])
def test_screen_matches_oracle(M, S, H, E, I, k, B):
    Ld = S.channel_major_layer(H, E, I, seed=710 + H, device=DEV)
    cm = Ld["cm"]
    desc = M.make_desc(H, E, I, k, layout=M.MOE_LAYOUT_CHANNEL_MAJOR, gate=cm)
    signs = S.reader_signs(H, seed=711, device=DEV)
    codes, scales, rho, dnorm = build_sketch(M, desc, signs)
    x = S.tokens(B, H, seed=712, device=DEV)
    ids = S.uniform_ids(B, E, k, seed=713, device=DEV)
    wt = S.router_weights(B, k, seed=714, device=DEV)
    scores = torch.full((B, E, I), -1.0, dtype=torch.float32, device=DEV)
    est = torch.zeros((B, k, I, 2), dtype=torch.float32, device=DEV)
    M.moe_reader_screen(desc, x, ids, wt, signs, codes, scales, dnorm, scores, est)
    torch.cuda.synchronize()
    # the oracle builds its own sketch from the weights
    host = f64(cm)
    sg = f64(signs)
    sk = {}

    def sketch(e, c):
        if (e, c) not in sk:
            g, v, d = host[e, c]
            cg, scg, _ = O.reader_sketch_row(g, sg)
            cv, scv, _ = O.reader_sketch_row(v, sg)
            sk[(e, c)] = (cg, scg, cv, scv, float(np.sqrt(np.sum(d ** 2))))
        return sk[(e, c)]

    sc_gpu, est_gpu = f64(scores), f64(est)
    for b in range(B):
        xb = f64(x[b])
        idl = ids[b].tolist()
        wl = f64(wt[b])
        o_sc, o_est = O.reader_screen(xb, idl, wl, sketch, I, sg)
        for t, e in enumerate(idl):
            for c in range(I):
                cg, scg, cv, scv, dn = sketch(e, c)
                gh, vh = o_est[t, c]
                tg, tv, ts = est_and_score_tolerances(xb, cg, scg, cv, scv, wl[t], dn, gh, vh)
                assert abs(est_gpu[b, t, c, 0] - gh) <= tg, (b, e, c)
                assert abs(est_gpu[b, t, c, 1] - vh) <= tv, (b, e, c)
                assert abs(sc_gpu[b, e, c] - o_sc[t, c]) <= ts, (b, e, c)
        # rows of experts this token did not route to are untouched
        others = [e for e in range(E) if e not in idl]
        assert np.all(sc_gpu[b, others] == -1.0)


def test_screen_then_channel_topk_end_to_end(M, S):
    """Screen -> keep the top `keep` -> exact compute of the kept channels
    ([Reader] step 2): the kept set matches the oracle's (any difference only
    between channels whose oracle scores tie within the score tolerance at the
    cut), and y matches the oracle's channel-sparse output on its kept set."""
    H, E, I, k, keep = 512, 8, 64, 3, 50
    Ld = S.channel_major_layer(H, E, I, seed=720, device=DEV)
    cm = Ld["cm"]
    desc = M.make_desc(H, E, I, k, layout=M.MOE_LAYOUT_CHANNEL_MAJOR, gate=cm)
    signs = S.reader_signs(H, seed=721, device=DEV)
    codes, scales, rho, dnorm = build_sketch(M, desc, signs)
    x = S.tokens(1, H, seed=722, device=DEV)
    ids = S.uniform_ids(1, E, k, seed=723, device=DEV)
    wt = S.router_weights(1, k, seed=724, device=DEV)
    scores = torch.zeros((1, E, I), dtype=torch.float32, device=DEV)
    M.moe_reader_screen(desc, x, ids, wt, signs, codes, scales, dnorm, scores)
    ws = M.alloc_workspace(desc, 1)
    y = torch.empty((1, H), dtype=torch.float32, device=DEV)
    kept = torch.empty((1, keep), dtype=torch.int32, device=DEV)
    sec = torch.empty((1,), dtype=torch.int64, device=DEV)
    M.moe_channel_topk_forward(desc, x, ids, wt, scores, keep, y, sec, ws, kept=kept)
    torch.cuda.synchronize()
    assert M.moe_get_status(ws) == M.MOE_OK
    host = f64(cm)
    sg = f64(signs)
    xb = f64(x[0])
    idl = ids[0].tolist()
    wl = f64(wt[0])

    def sketch(e, c):
        g, v, d = host[e, c]
        cg, scg, _ = O.reader_sketch_row(g, sg)
        cv, scv, _ = O.reader_sketch_row(v, sg)
        return cg, scg, cv, scv, float(np.sqrt(np.sum(d ** 2)))

    o_sc, _ = O.reader_screen(xb, idl, wl, sketch, I, sg)
    full = np.full((E, I), -np.inf)
    for t, e in enumerate(idl):
        full[e] = o_sc[t]
    want = O.channel_topk_select(full, idl, keep)
    got = np.array(sorted(kept[0].tolist()))
    # the GPU's kept set is a valid keep: `keep` distinct channels of the routed experts
    assert got.size == keep and np.unique(got).size == keep
    assert set((got // I).tolist()) <= set(idl)
    cut = np.sort(o_sc.ravel())[::-1][keep - 1]
    diff = set(got.tolist()) ^ set(want.tolist())
    assert len(diff) <= 4, len(diff)  # at most a couple of swaps at the cut
    for j in diff:
        e, c = divmod(int(j), I)
        assert abs(full[e, c] - cut) <= 1e-4 * cut, j  # only near-ties at the cut may differ
    # the output always matches the oracle's channel-sparse sum over the
    # GPU's own kept set (and over the oracle's when the sets agree)
    y_ref = O.channel_sparse_forward(xb, lambda e, c: host[e, c], idl, wl, got, I)
    assert rel_err(f64(y[0]), y_ref) <= REL_TOL


def test_sketch_and_screen_at_thinking_shape_sampled(M, S):
    """The Qwen3-Thinking channel layer (H 2048, E 128, I 768, k 8): the whole
    layer's sketch is built; 64 sampled channels of the routed experts are
    checked against the oracle (sketch and estimates)."""
    w = S.WORKLOADS["channel_topk"]
    H, E, I, k = w["H"], w["E"], w["I"], w["k"]
    Ld = S.channel_major_layer(H, E, I, seed=S.weight_seed(5, 0), device=DEV)
    cm = Ld["cm"]
    desc = M.make_desc(H, E, I, k, layout=M.MOE_LAYOUT_CHANNEL_MAJOR, gate=cm)
    signs = S.reader_signs(H, seed=730, device=DEV)
    codes, scales, rho, dnorm = build_sketch(M, desc, signs)
    x = S.tokens(1, H, seed=731, device=DEV)
    ids = S.uniform_ids(1, E, k, seed=732, device=DEV)
    wt = S.router_weights(1, k, seed=733, device=DEV)
    scores = torch.zeros((1, E, I), dtype=torch.float32, device=DEV)
    est = torch.zeros((1, k, I, 2), dtype=torch.float32, device=DEV)
    M.moe_reader_screen(desc, x, ids, wt, signs, codes, scales, dnorm, scores, est)
    torch.cuda.synchronize()
    sg = f64(signs)
    xb = f64(x[0])
    idl = ids[0].tolist()
    wl = f64(wt[0])
    rng = np.random.default_rng(734)
    picks = [(int(t), int(c)) for t, c in zip(rng.integers(0, k, 64), rng.integers(0, I, 64))]
    est_gpu, sc_gpu = f64(est), f64(scores)
    for t, c in picks:
        e = idl[t]
        j = e * I + c
        rows = f64(cm[e, c])
        cj = unpack_codes(codes[j].cpu().numpy().view(np.uint32), H)
        sj = scales[j].cpu().numpy().view(np.float16).astype(np.float64)
        oc = [O.reader_sketch_row(rows[r], sg) for r in range(2)]
        for r in range(2):
            assert np.array_equal(cj[r], oc[r][0]) and np.array_equal(sj[r], oc[r][1]), (e, c, r)
        gh = O.reader_estimate(xb, oc[0][0], oc[0][1], sg)
        vh = O.reader_estimate(xb, oc[1][0], oc[1][1], sg)
        dn = float(np.sqrt(np.sum(rows[2] ** 2)))
        tg, tv, ts = est_and_score_tolerances(xb, oc[0][0], oc[0][1], oc[1][0], oc[1][1], wl[t], dn, gh, vh)
        assert abs(est_gpu[0, t, c, 0] - gh) <= tg and abs(est_gpu[0, t, c, 1] - vh) <= tv, (e, c)
        assert abs(sc_gpu[0, e, c] - O.reader_score(wl[t], dn, gh, vh)) <= ts, (e, c)


@pytest.mark.parametrize("H,E,I,k,pre_norm", [(512, 16, 64, 4, True), (2048, 12, 64, 3, True), (512, 8, 48, 2, False)])
def test_screened_channel_stack_teacher_forced(M, S, H, E, I, k, pre_norm):
    """The channel stack computing its own scores in the kernel ([Reader]
    steps 1-2 per layer: the screen of u_l with the layer's routing weights,
    then the top-keep selection and the exact compute of the kept channels),
    teacher-forced layer by layer against reader_screen -> channel_topk_select
    -> channel_sparse_forward in the oracle (the oracle builds its own sketch
    from the weights). Kept sets may differ only between channels whose
    oracle scores tie at the cut within the score tolerance; y is checked on
    the GPU's own kept set, which must be a valid keep."""
    from tests.parity_util import check_ids
    Lc, keep = 3, max(1, (k * I) // 7)
    from oracle import moe_oracle as O2
    layers = [S.channel_major_layer(H, E, I, seed=1100 + 10 * H + l, device=DEV, router_scale=0.5) for l in range(Lc)]
    descs = [M.make_desc(H, E, I, k, layout=M.MOE_LAYOUT_CHANNEL_MAJOR, router=Ld["router"], gate=Ld["cm"])
             for Ld in layers]
    signs = S.reader_signs(H, seed=1150, device=DEV)
    sk = [build_sketch(M, d, signs) for d in descs]
    sketches = [M.make_sketch(c, s_, dn) for (c, s_, _r, dn) in sk]
    x = S.tokens(1, H, seed=1160, device=DEV)
    ws = M.alloc_workspace(descs[0], 1)
    xo = torch.empty((1, H), dtype=torch.bfloat16, device=DEV)
    xh = torch.empty((Lc + 1, H), dtype=torch.bfloat16, device=DEV)
    yh = torch.empty((Lc, H), dtype=torch.float32, device=DEV)
    ih = torch.empty((Lc, k), dtype=torch.int32, device=DEV)
    wh = torch.empty((Lc, k), dtype=torch.float32, device=DEV)
    kh = torch.empty((Lc, keep), dtype=torch.int32, device=DEV)
    sec = torch.empty((Lc,), dtype=torch.int64, device=DEV)
    M.moe_channel_stack_forward(descs, x, None, keep, xo, sec, ws, x_hist=xh, y_hist=yh, ids_hist=ih, w_hist=wh,
                                kept_hist=kh, flags=M.MOE_STACK_PRE_RMSNORM if pre_norm else 0,
                                sketches=sketches, signs=signs)
    torch.cuda.synchronize()
    assert M.moe_get_status(ws) == M.MOE_OK
    sg = f64(signs)
    log = []
    for l in range(Lc):
        host = f64(layers[l]["cm"])
        xl = f64(xh[l])
        u = O2.rmsnorm_bf16(xl) if pre_norm else xl
        io, wo, lo, _ = O2.route_topk(u, f64(layers[l]["router"]), k)
        if check_ids(ih[l].tolist(), io, lo, log, f"l{l}"):
            continue
        idl = io.tolist()

        def sketch(e, c):
            g, v, d = host[e, c]
            cg, scg, _ = O2.reader_sketch_row(g, sg)
            cv, scv, _ = O2.reader_sketch_row(v, sg)
            return cg, scg, cv, scv, float(np.sqrt(np.sum(d ** 2)))
        o_sc, _ = O2.reader_screen(u, idl, wo, sketch, I, sg)
        full = np.full((E, I), -np.inf)
        for t, e in enumerate(idl):
            full[e] = o_sc[t]
        want = O2.channel_topk_select(full, idl, keep)
        got = np.array(sorted(kh[l].tolist()))
        assert got.size == keep and np.unique(got).size == keep and set((got // I).tolist()) <= set(idl)
        cut = np.sort(o_sc.ravel())[::-1][keep - 1]
        diff = set(got.tolist()) ^ set(want.tolist())
        assert len(diff) <= 4, (l, len(diff))
        for j in diff:
            e, c = divmod(int(j), I)
            assert abs(full[e, c] - cut) <= 1e-4 * cut, (l, j)
        yo = O2.channel_sparse_forward(u, lambda e, c: host[e][c], idl, wo, got, I)
        assert rel_err(f64(yh[l]), yo) <= REL_TOL, l
        assert rel_err(f64(xh[l + 1]), O2.residual_bf16(xl, f64(yh[l]))) <= REL_TOL, l
