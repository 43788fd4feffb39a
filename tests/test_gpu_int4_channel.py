"""GPU parity for the int4 group-64 experts (A3B shapes, batch 1 and 8) and the
channel-sparse top-k reader (Qwen3-Thinking shapes, 13% and 18% budgets), both
through the C ABI against the fp64 oracle.

Channel-sparse checks: the kept set and the 32-byte sector count are compared
bit-exactly (scores are fp32 inputs, so the selection is exact on both sides);
the output within the layer tolerance.
"""

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from tests.parity_util import REL_TOL, check_ids, f64, rel_err

pytestmark = pytest.mark.gpu

DEV = "cuda"


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


# --------------------------------------------------------------------- int4


class HostInt4:
    def __init__(self, L):
        self.L = L
        self.R = f64(L["router"])
        self.shared = (f64(L["sh_gate"]), f64(L["sh_up"]), f64(L["sh_down_t"])) if "sh_gate" in L else None
        self._c = {}

    def expert(self, e):
        if e not in self._c:
            L = self.L
            G = O.dequant_rows_int4(L["gate"][e].cpu().numpy(), f64(L["gate_s"][e]))
            V = O.dequant_rows_int4(L["up"][e].cpu().numpy(), f64(L["up_s"][e]))
            D = O.dequant_down_t_int4(L["down_t"][e].cpu().numpy(), f64(L["down_s"][e]))
            self._c[e] = (G, V, D)
        return self._c[e]


def int4_desc(M, L, H, E, I, k, router=True):
    return M.make_desc(H, E, I, k, wtype=M.MOE_W_INT4_G64, router=L["router"] if router else None,
                       gate=L["gate"], up=L["up"], down_t=L["down_t"], gate_s=L["gate_s"], up_s=L["up_s"],
                       down_s=L["down_s"], sh_gate=L.get("sh_gate"), sh_up=L.get("sh_up"),
                       sh_down_t=L.get("sh_down_t"))


@pytest.fixture(scope="module")
def a3b_int4(S):
    w = S.WORKLOADS["a3b_int4"]
    layers = [S.swiglu_layer_int4(w["H"], w["E"], w["I"], w["I_shared"], seed=S.weight_seed(4, l), device=DEV,
                                  router_scale=w["router_scale"]) for l in range(2)]
    return w, layers


@pytest.mark.parametrize("B", [1, 3, 8])
def test_int4_layer_a3b_shapes(M, S, a3b_int4, B):
    w, layers = a3b_int4
    H, E, I, k = w["H"], w["E"], w["I"], w["k"]
    L = layers[0]
    desc = int4_desc(M, L, H, E, I, k)
    x = S.tokens(B, H, seed=S.act_seed(4), device=DEV)
    ws = M.alloc_workspace(desc, B)
    y = torch.empty((B, H), dtype=torch.float32, device=DEV)
    ids = torch.empty((B, k), dtype=torch.int32, device=DEV)
    wt = torch.empty((B, k), dtype=torch.float32, device=DEV)
    M.moe_layer_forward(desc, x, y, ws, ids_out=ids, w_out=wt)
    torch.cuda.synchronize()
    assert M.moe_get_status(ws) == M.MOE_OK
    HL = HostInt4(L)
    log = []
    for b in range(B):
        yo, io, wo, lo, _ = O.moe_layer(f64(x[b]), HL.R, HL.expert, k, shared=HL.shared)
        if check_ids(ids[b].tolist(), io, lo, log, f"tok{b}"):
            continue
        assert rel_err(f64(y[b]), yo) <= REL_TOL, b
        assert np.allclose(f64(wt[b]), wo, rtol=1e-5)


@pytest.mark.parametrize("B", [1, 8])
def test_int4_stack_teacher_forced(M, S, a3b_int4, B):
    w, layers = a3b_int4
    H, E, I, k = w["H"], w["E"], w["I"], w["k"]
    descs = [int4_desc(M, L, H, E, I, k) for L in layers]
    Lc = len(layers)
    x = S.tokens(B, H, seed=S.act_seed(4) + 1, device=DEV)
    ws = M.alloc_workspace(descs[0], B)
    xo = torch.empty((B, H), dtype=torch.bfloat16, device=DEV)
    xh = torch.empty((Lc + 1, B, H), dtype=torch.bfloat16, device=DEV)
    yh = torch.empty((Lc, B, H), dtype=torch.float32, device=DEV)
    ih = torch.empty((Lc, B, k), dtype=torch.int32, device=DEV)
    wh = torch.empty((Lc, B, k), dtype=torch.float32, device=DEV)
    M.moe_stack_forward(descs, x, xo, ws, x_hist=xh, y_hist=yh, ids_hist=ih, w_hist=wh,
                        flags=M.MOE_STACK_PRE_RMSNORM)
    torch.cuda.synchronize()
    log = []
    for l in range(Lc):
        HL = HostInt4(layers[l])
        for b in range(B):
            xl = f64(xh[l, b])
            xn, yo, io, wo, lo, _ = O.stack_layer(xl, HL.R, HL.expert, k, shared=HL.shared)
            if check_ids(ih[l, b].tolist(), io, lo, log, f"l{l}b{b}"):
                continue
            assert rel_err(f64(yh[l, b]), yo) <= REL_TOL
            assert rel_err(f64(xh[l + 1, b]), xn) <= REL_TOL


def test_int4_expert_forward_ragged(M, S):
    # a small int4 layer with routing given: I = 128 (two scale groups), B = 3
    H, E, I, k = 512, 12, 128, 3
    L = S.swiglu_layer_int4(H, E, I, 0, seed=77, device=DEV)
    desc = int4_desc(M, L, H, E, I, k, router=False)
    B = 3
    ids = S.uniform_ids(B, E, k, seed=78, device=DEV)
    wt = torch.rand((B, k), device=DEV)
    x = S.tokens(B, H, seed=79, device=DEV)
    ws = M.alloc_workspace(desc, B)
    y = torch.empty((B, H), dtype=torch.float32, device=DEV)
    M.moe_expert_forward(desc, x, ids, wt, y, ws)
    torch.cuda.synchronize()
    HL = HostInt4(L)
    for b in range(B):
        yo = O.moe_experts_given(f64(x[b]), HL.expert, ids[b].tolist(), f64(wt[b]))
        assert rel_err(f64(y[b]), yo) <= REL_TOL


def test_int4_layer_batched_tied_router_rows(M, S, a3b_int4):
    # router rows in identical pairs at A3B shapes (the tensor-core router rows
    # and the per-warp batch routing): the ids match the oracle exactly
    w, layers = a3b_int4
    H, E, I, k = w["H"], w["E"], w["I"], w["k"]
    R = layers[0]["router"].clone()
    R[1::2] = R[0::2]
    L = dict(layers[0], router=R)
    desc = int4_desc(M, L, H, E, I, k)
    B = 5
    x = S.tokens(B, H, seed=S.act_seed(4) + 9, device=DEV)
    ws = M.alloc_workspace(desc, B)
    y = torch.empty((B, H), dtype=torch.float32, device=DEV)
    ids = torch.empty((B, k), dtype=torch.int32, device=DEV)
    wt = torch.empty((B, k), dtype=torch.float32, device=DEV)
    M.moe_layer_forward(desc, x, y, ws, ids_out=ids, w_out=wt)
    torch.cuda.synchronize()
    assert M.moe_get_status(ws) == M.MOE_OK
    HL = HostInt4(L)
    for b in range(B):
        yo, io, wo, lo, _ = O.moe_layer(f64(x[b]), HL.R, HL.expert, k, shared=HL.shared)
        got = ids[b].tolist()
        assert got == [int(v) for v in io], b
        assert all(got[2 * i] % 2 == 0 and got[2 * i + 1] == got[2 * i] + 1 for i in range(k // 2)), got
        assert rel_err(f64(y[b]), yo) <= REL_TOL, b


@pytest.mark.parametrize("B", [2, 5, 8])
def test_int4_expert_forward_a3b_batches(M, S, a3b_int4, B):
    # routing given at A3B shapes (H = 2048, I = 768): the tensor-core dots of
    # the batch path, with fewer than 8 tokens (unused token rows) and tokens
    # that share experts (ids drawn from 12 of the 128 experts)
    w, layers = a3b_int4
    H, E, I, k = w["H"], w["E"], w["I"], w["k"]
    L = layers[1]
    desc = int4_desc(M, L, H, E, I, k, router=False)
    g = torch.Generator().manual_seed(90 + B)
    pool = torch.randperm(E, generator=g)[:12]
    ids = torch.stack([pool[torch.randperm(12, generator=g)[:k]] for _ in range(B)]).to(torch.int32).to(DEV)
    wt = torch.rand((B, k), generator=g).to(DEV)
    x = S.tokens(B, H, seed=91 + B, device=DEV)
    ws = M.alloc_workspace(desc, B)
    y = torch.empty((B, H), dtype=torch.float32, device=DEV)
    M.moe_expert_forward(desc, x, ids, wt, y, ws)
    torch.cuda.synchronize()
    assert M.moe_get_status(ws) == M.MOE_OK
    HL = HostInt4(L)
    for b in range(B):
        yo = O.moe_experts_given(f64(x[b]), HL.expert, ids[b].tolist(), f64(wt[b]))
        assert rel_err(f64(y[b]), yo) <= REL_TOL, b


# ------------------------------------------------------------ channel-sparse


def cm_desc(M, cm, H, E, I, k):
    return M.make_desc(H, E, I, k, layout=M.MOE_LAYOUT_CHANNEL_MAJOR, gate=cm)


def run_channel(M, desc, x, ids, wt, scores, keep, H):
    B = x.shape[0]
    ws = M.alloc_workspace(desc, B)
    y = torch.empty((B, H), dtype=torch.float32, device=DEV)
    kept = torch.empty((B, max(keep, 1)), dtype=torch.int32, device=DEV)
    sec = torch.empty((B,), dtype=torch.int64, device=DEV)
    M.moe_channel_topk_forward(desc, x, ids, wt, scores, keep, y, sec, ws, kept=kept)
    torch.cuda.synchronize()
    assert M.moe_get_status(ws) == M.MOE_OK
    return y, kept, sec


def check_channel(desc_gate, cm_host, x, ids, wt, scores, keep, y, kept, sec, I, H):
    for b in range(x.shape[0]):
        want = O.channel_topk_select(scores[b].cpu().numpy(), ids[b].tolist(), keep)
        assert kept[b, :keep].cpu().numpy().tolist() == want.tolist(), b
        ranges = O.channel_major_ranges(want, H, base=desc_gate.data_ptr())
        assert int(sec[b]) == O.sectors_touched(ranges), b
        yo = O.channel_sparse_forward(f64(x[b]), cm_host, ids[b].tolist(), f64(wt[b]), want, I)
        if keep > 0:
            assert rel_err(f64(y[b]), yo) <= REL_TOL, b
        else:
            assert np.all(f64(y[b]) == 0)


@pytest.fixture(scope="module")
def thinking(S):
    w = S.WORKLOADS["channel_topk"]
    H, E, I = w["H"], w["E"], w["I"]
    Ld = S.channel_major_layer(H, E, I, seed=S.weight_seed(5, 0), device=DEV)
    scale = S.channel_scale(E, I, seed=S.weight_seed(5, 0) + 7, device=DEV)
    return w, Ld, scale


@pytest.mark.parametrize("frac", [0.13, 0.18])
def test_channel_topk_thinking_shapes(M, S, thinking, frac):
    w, Ld, scale = thinking
    H, E, I, k = w["H"], w["E"], w["I"], w["k"]
    keep = S.keep_count(frac, k, I)
    cm = Ld["cm"]
    desc = cm_desc(M, cm, H, E, I, k)
    x = S.tokens(1, H, seed=S.act_seed(5), device=DEV)
    ids = S.uniform_ids(1, E, k, seed=S.act_seed(5) + 1, device=DEV)
    wt = torch.softmax(torch.randn((1, k), device=DEV), dim=1)
    scores = S.channel_scores(1, E, I, scale, seed=S.act_seed(5) + 2, device=DEV)
    y, kept, sec = run_channel(M, desc, x, ids, wt, scores, keep, H)
    cache = {}

    def cm_host(e, c):
        if e not in cache:
            cache[e] = f64(cm[e])
        return cache[e][c]
    check_channel(cm, cm_host, x, ids, wt, scores, keep, y, kept, sec, I, H)
    # the pages' accounting: kept channels x 12,288 bytes, aligned -> 384 sectors each
    assert int(sec[0]) == 384 * keep


@pytest.mark.parametrize("keep_mode", ["zero", "all", "ties", "one"])
def test_channel_topk_edge_cases(M, S, keep_mode):
    H, E, I, k = 512, 10, 40, 3
    Ld = S.channel_major_layer(H, E, I, seed=55, device=DEV)
    cm = Ld["cm"]
    desc = cm_desc(M, cm, H, E, I, k)
    B = 2
    x = S.tokens(B, H, seed=56, device=DEV)
    ids = S.uniform_ids(B, E, k, seed=57, device=DEV)
    wt = torch.rand((B, k), device=DEV)
    scores = torch.rand((B, E, I), device=DEV)
    keep = {"zero": 0, "all": k * I, "ties": 17, "one": 1}[keep_mode]
    if keep_mode == "ties":
        scores = torch.floor(scores * 4) / 4  # many equal scores: ties go to the lowest index
    y, kept, sec = run_channel(M, desc, x, ids, wt, scores, keep, H)
    host = f64(cm)
    check_channel(cm, lambda e, c: host[e][c], x, ids, wt, scores, keep, y, kept, sec, I, H)
    if keep_mode == "all":
        # keeping every channel equals the planar expert output
        for b in range(B):
            planar = O.moe_experts_given(f64(x[b]), lambda e: (host[e][:, 0], host[e][:, 1], host[e][:, 2]),
                                         ids[b].tolist(), f64(wt[b]))
            assert rel_err(f64(y[b]), planar) <= REL_TOL


@pytest.mark.parametrize("pre_norm", [True, False])
def test_channel_stack_small_teacher_forced(M, S, pre_norm):
    H, E, I, k, Lc, keep = 512, 16, 64, 4, 3, 37
    layers = [S.channel_major_layer(H, E, I, seed=600 + l, device=DEV, router_scale=0.5) for l in range(Lc)]
    descs = [M.make_desc(H, E, I, k, layout=M.MOE_LAYOUT_CHANNEL_MAJOR, router=Ld["router"], gate=Ld["cm"])
             for Ld in layers]
    scale = S.channel_scale(E, I, seed=610, device=DEV)
    scores = torch.cat([S.channel_scores(1, E, I, scale, seed=620 + l, device=DEV) for l in range(Lc)])
    x = S.tokens(1, H, seed=630, device=DEV)
    ws = M.alloc_workspace(descs[0], 1)
    xo = torch.empty((1, H), dtype=torch.bfloat16, device=DEV)
    xh = torch.empty((Lc + 1, H), dtype=torch.bfloat16, device=DEV)
    yh = torch.empty((Lc, H), dtype=torch.float32, device=DEV)
    ih = torch.empty((Lc, k), dtype=torch.int32, device=DEV)
    wh = torch.empty((Lc, k), dtype=torch.float32, device=DEV)
    kh = torch.empty((Lc, keep), dtype=torch.int32, device=DEV)
    sec = torch.empty((Lc,), dtype=torch.int64, device=DEV)
    M.moe_channel_stack_forward(descs, x, scores, keep, xo, sec, ws, x_hist=xh, y_hist=yh, ids_hist=ih,
                                w_hist=wh, kept_hist=kh, flags=M.MOE_STACK_PRE_RMSNORM if pre_norm else 0)
    torch.cuda.synchronize()
    assert M.moe_get_status(ws) == M.MOE_OK
    log = []
    for l in range(Lc):
        host = f64(layers[l]["cm"])
        xl = f64(xh[l])
        xn, yo, io, wo, lo, kept = O.channel_stack_layer(xl, f64(layers[l]["router"]), lambda e, c: host[e][c],
                                                         scores[l].cpu().numpy(), k, keep, I, pre_norm=pre_norm)
        if check_ids(ih[l].tolist(), io, lo, log, f"l{l}"):
            continue
        assert kh[l].cpu().numpy().tolist() == kept.tolist()
        assert int(sec[l]) == O.sectors_touched(O.channel_major_ranges(kept, H, base=layers[l]["cm"].data_ptr()))
        assert rel_err(f64(yh[l]), yo) <= REL_TOL
        assert rel_err(f64(xh[l + 1]), xn) <= REL_TOL
