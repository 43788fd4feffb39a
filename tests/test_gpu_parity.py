"""GPU parity: every entry point of libmoedec, called through the C ABI, against
the fp64 oracle on the same seeded inputs.

Sizes: the tiny workload in full (64 tokens), small multi-tile shapes with
ragged tails, and the A3B-shaped bf16 stack at full size (40 layers, 64 GB)
in the launch configuration bench.py times, checked per layer with teacher
forcing (the oracle recomputes layer l from the GPU's x_l).
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


def planar_desc(M, L, H, E, I, k, with_router=True):
    return M.make_desc(H, E, I, k, router=L["router"] if with_router else None, gate=L["gate"], up=L["up"],
                       down_t=L["down_t"], sh_gate=L.get("sh_gate"), sh_up=L.get("sh_up"),
                       sh_down_t=L.get("sh_down_t"))


class HostLayer:
    """fp64 views of one planar bf16 layer, fetched expert by expert."""

    def __init__(self, L):
        self.L = L
        self.R = f64(L["router"])
        self._cache = {}
        self.shared = None
        if "sh_gate" in L:
            self.shared = (f64(L["sh_gate"]), f64(L["sh_up"]), f64(L["sh_down_t"]))

    def expert(self, e):
        if e not in self._cache:
            self._cache[e] = (f64(self.L["gate"][e]), f64(self.L["up"][e]), f64(self.L["down_t"][e]))
        return self._cache[e]


# --------------------------------------------------------------------- tiny


@pytest.fixture(scope="module")
def tiny(S):
    w = S.WORKLOADS["tiny"]
    L = S.swiglu_layer_bf16(w["H"], w["E"], w["I"], 0, seed=0, device=DEV)
    x = S.tokens(w["tokens"], w["H"], seed=S.act_seed(1), device=DEV)
    return w, L, x


def test_route_topk_tiny_all_tokens(M, tiny):
    w, L, x = tiny
    B, H, E, k = x.shape[0], w["H"], w["E"], w["k"]
    ws = M.alloc_workspace(M.make_desc(H, E, w["I"], k, gate=L["gate"]), B)
    ids = torch.empty((B, k), dtype=torch.int32, device=DEV)
    wt = torch.empty((B, k), dtype=torch.float32, device=DEV)
    mg = torch.empty((B,), dtype=torch.float32, device=DEV)
    M.moe_route_topk(x, L["router"], k, ids, wt, mg, ws)
    torch.cuda.synchronize()
    R, X = f64(L["router"]), f64(x)
    log = []
    for b in range(B):
        io, wo, lo, mo = O.route_topk(X[b], R, k)
        if check_ids(ids[b].tolist(), io, lo, log, f"tok{b}") == 0:
            assert np.allclose(wt[b].cpu().numpy(), wo, rtol=1e-5, atol=1e-6)
            assert abs(float(mg[b]) - mo) <= 1e-5 + 1e-4 * abs(mo)


def test_route_topk_k_equals_E_and_ties(M, S):
    H, E = 64, 16
    router = torch.zeros((E, H), dtype=torch.bfloat16, device=DEV)
    x = S.tokens(3, H, seed=7, device=DEV)
    ws = M.alloc_workspace(M.make_desc(H, E, 64, E, gate=router), 3)
    for k in (1, 5, E):
        ids = torch.empty((3, k), dtype=torch.int32, device=DEV)
        wt = torch.empty((3, k), dtype=torch.float32, device=DEV)
        mg = torch.empty((3,), dtype=torch.float32, device=DEV)
        M.moe_route_topk(x, router, k, ids, wt, mg, ws)
        torch.cuda.synchronize()
        # all logits equal: ids 0..k-1 (lowest index first), w = 1/k
        assert ids.cpu().tolist() == [list(range(k))] * 3
        assert torch.allclose(wt.cpu(), torch.full((3, k), 1.0 / k))
        assert (mg.cpu() == (float("inf") if k == E else 0.0)).all()


def test_layer_forward_tiny_all_tokens_b1(M, tiny):
    w, L, x = tiny
    H, E, I, k = w["H"], w["E"], w["I"], w["k"]
    desc = planar_desc(M, L, H, E, I, k)
    ws = M.alloc_workspace(desc, 1)
    HL = HostLayer(L)
    log = []
    for b in range(x.shape[0]):
        y = torch.empty((1, H), dtype=torch.float32, device=DEV)
        xn = torch.empty((1, H), dtype=torch.bfloat16, device=DEV)
        ids = torch.empty((1, k), dtype=torch.int32, device=DEV)
        wt = torch.empty((1, k), dtype=torch.float32, device=DEV)
        M.moe_layer_forward(desc, x[b:b + 1], y, ws, x_next=xn, ids_out=ids, w_out=wt)
        torch.cuda.synchronize()
        xb = f64(x[b])
        yo, io, wo, lo, _ = O.moe_layer(xb, HL.R, HL.expert, k)
        if check_ids(ids[0].tolist(), io, lo, log, f"tok{b}"):
            continue
        assert rel_err(f64(y[0]), yo) <= REL_TOL
        assert rel_err(f64(xn[0]), O.residual_bf16(xb, yo)) <= REL_TOL
        assert np.allclose(f64(wt[0]), wo, rtol=1e-5)
    assert M.moe_get_status(ws) == M.MOE_OK


@pytest.mark.parametrize("B", [2, 3, 8])
def test_layer_forward_tiny_batched(M, tiny, B):
    w, L, x = tiny
    H, E, I, k = w["H"], w["E"], w["I"], w["k"]
    desc = planar_desc(M, L, H, E, I, k)
    ws = M.alloc_workspace(desc, B)
    HL = HostLayer(L)
    log = []
    for b0 in range(0, 16, B):
        xb = x[b0:b0 + B].contiguous()
        y = torch.empty((B, H), dtype=torch.float32, device=DEV)
        ids = torch.empty((B, k), dtype=torch.int32, device=DEV)
        wt = torch.empty((B, k), dtype=torch.float32, device=DEV)
        M.moe_layer_forward(desc, xb, y, ws, ids_out=ids, w_out=wt)
        torch.cuda.synchronize()
        for b in range(B):
            yo, io, wo, lo, _ = O.moe_layer(f64(xb[b]), HL.R, HL.expert, k)
            if check_ids(ids[b].tolist(), io, lo, log, f"tok{b0 + b}"):
                continue
            assert rel_err(f64(y[b]), yo) <= REL_TOL, (b0, b)


def test_layer_forward_batched_tied_router_rows(M, S, tiny):
    # router rows in identical pairs (2i, 2i + 1): every logit appears twice,
    # bit-identical on both sides, so each chosen pair must come out lower
    # index first, and the batch routing must match the oracle exactly
    w, L, x = tiny
    H, E, I, k = w["H"], w["E"], w["I"], w["k"]
    R = L["router"].clone()
    R[1::2] = R[0::2]
    Lt = dict(L, router=R)
    desc = planar_desc(M, Lt, H, E, I, k)
    B = 3
    ws = M.alloc_workspace(desc, B)
    HL = HostLayer(Lt)
    xb = x[:B].contiguous()
    y = torch.empty((B, H), dtype=torch.float32, device=DEV)
    ids = torch.empty((B, k), dtype=torch.int32, device=DEV)
    wt = torch.empty((B, k), dtype=torch.float32, device=DEV)
    M.moe_layer_forward(desc, xb, y, ws, ids_out=ids, w_out=wt)
    torch.cuda.synchronize()
    assert M.moe_get_status(ws) == M.MOE_OK
    for b in range(B):
        yo, io, wo, lo, _ = O.moe_layer(f64(xb[b]), HL.R, HL.expert, k)
        assert ids[b].tolist() == [int(v) for v in io], b
        assert ids[b, 0] % 2 == 0 and ids[b, 1] == ids[b, 0] + 1, b
        assert np.allclose(f64(wt[b]), wo, rtol=1e-5)
        assert rel_err(f64(y[b]), yo) <= REL_TOL, b


def test_expert_forward_given_ids(M, S, tiny):
    w, L, x = tiny
    H, E, I, k = w["H"], w["E"], w["I"], w["k"]
    desc = planar_desc(M, L, H, E, I, k, with_router=False)
    HL = HostLayer(L)
    for B in (1, 5, 8):
        ids = S.uniform_ids(B, E, k, seed=11 + B, device=DEV)
        wt = torch.rand((B, k), device=DEV)
        ws = M.alloc_workspace(desc, B)
        y = torch.empty((B, H), dtype=torch.float32, device=DEV)
        M.moe_expert_forward(desc, x[:B].contiguous(), ids, wt, y, ws)
        torch.cuda.synchronize()
        for b in range(B):
            yo = O.moe_experts_given(f64(x[b]), HL.expert, ids[b].tolist(), f64(wt[b]))
            assert rel_err(f64(y[b]), yo) <= REL_TOL
        assert M.moe_get_status(ws) == M.MOE_OK


def test_expert_forward_bad_ids_sets_status(M, S, tiny):
    w, L, x = tiny
    H, E, I, k = w["H"], w["E"], w["I"], w["k"]
    desc = planar_desc(M, L, H, E, I, k, with_router=False)
    ws = M.alloc_workspace(desc, 1)
    y = torch.empty((1, H), dtype=torch.float32, device=DEV)
    wt = torch.ones((1, k), device=DEV)
    for bad in ([3, 3], [0, E], [-1, 2]):
        M.moe_workspace_init(ws)
        ids = torch.tensor([bad], dtype=torch.int32, device=DEV)
        M.moe_expert_forward(desc, x[:1].contiguous(), ids, wt, y, ws)
        assert M.moe_get_status(ws) == M.MOE_ERR_INVALID


# ------------------------------------------------- small multi-tile / ragged


@pytest.mark.parametrize("H,E,I,k,I_sh,B", [
    (64, 5, 7, 2, 0, 1),        # smallest hidden, ragged channel count
    (1024, 37, 200, 3, 96, 3),  # E not a multiple of 32, ragged I, shared expert
    (2048, 64, 128, 8, 64, 8),  # a3b hidden, max batch
    (512, 16, 256, 16, 0, 2),   # k = E: dense softmax mixture
    (2048, 8, 64, 8, 0, 1),     # batch-1 fast path, one expert per warp's keys, k = E
    (2048, 24, 128, 12, 64, 1), # batch-1 fast path with k > 8 (router barrier, two-level top-k)
])
def test_layer_forward_shapes(M, S, H, E, I, k, I_sh, B):
    L = S.swiglu_layer_bf16(H, E, I, I_sh, seed=123, device=DEV)
    x = S.tokens(B, H, seed=321, device=DEV)
    desc = planar_desc(M, L, H, E, I, k)
    ws = M.alloc_workspace(desc, B)
    y = torch.empty((B, H), dtype=torch.float32, device=DEV)
    ids = torch.empty((B, k), dtype=torch.int32, device=DEV)
    wt = torch.empty((B, k), dtype=torch.float32, device=DEV)
    M.moe_layer_forward(desc, x, y, ws, ids_out=ids, w_out=wt)
    torch.cuda.synchronize()
    HL = HostLayer(L)
    log = []
    for b in range(B):
        xb = f64(x[b])
        yo, io, wo, lo, _ = O.moe_layer(xb, HL.R, HL.expert, k, shared=HL.shared)
        if check_ids(ids[b].tolist(), io, lo, log, f"tok{b}"):
            continue
        assert rel_err(f64(y[b]), yo) <= REL_TOL
        if k == E:
            dense = O.dense_mixture(xb, HL.R, HL.expert, E)
            assert rel_err(f64(y[b]), dense) <= REL_TOL


@pytest.mark.parametrize("pre_norm", [True, False])
def test_stack_small_teacher_forced(M, S, pre_norm):
    H, E, I, k, I_sh, Lc, B = 512, 32, 192, 4, 128, 5, 2
    layers = [S.swiglu_layer_bf16(H, E, I, I_sh, seed=900 + l, device=DEV, router_scale=0.5) for l in range(Lc)]
    descs = [planar_desc(M, Ld, H, E, I, k) for Ld in layers]
    x = S.tokens(B, H, seed=901, device=DEV)
    ws = M.alloc_workspace(descs[0], B)
    xo = torch.empty((B, H), dtype=torch.bfloat16, device=DEV)
    xh = torch.empty((Lc + 1, B, H), dtype=torch.bfloat16, device=DEV)
    yh = torch.empty((Lc, B, H), dtype=torch.float32, device=DEV)
    ih = torch.empty((Lc, B, k), dtype=torch.int32, device=DEV)
    wh = torch.empty((Lc, B, k), dtype=torch.float32, device=DEV)
    M.moe_stack_forward(descs, x, xo, ws, x_hist=xh, y_hist=yh, ids_hist=ih, w_hist=wh,
                        flags=M.MOE_STACK_PRE_RMSNORM if pre_norm else 0)
    torch.cuda.synchronize()
    assert torch.equal(xh[0], x) and torch.equal(xh[Lc], xo)
    log = []
    for l in range(Lc):
        HL = HostLayer(layers[l])
        for b in range(B):
            xl = f64(xh[l, b])
            xn, yo, io, wo, lo, _ = O.stack_layer(xl, HL.R, HL.expert, k, shared=HL.shared, pre_norm=pre_norm)
            if check_ids(ih[l, b].tolist(), io, lo, log, f"l{l}b{b}"):
                continue
            assert rel_err(f64(yh[l, b]), yo) <= REL_TOL
            assert rel_err(f64(xh[l + 1, b]), xn) <= REL_TOL
            assert np.allclose(f64(wh[l, b]), wo, rtol=1e-5)


def test_repeat_calls_same_ids(M, tiny):
    # the workspace barrier counter and accumulator survive repeated launches
    w, L, x = tiny
    H, E, I, k = w["H"], w["E"], w["I"], w["k"]
    desc = planar_desc(M, L, H, E, I, k)
    ws = M.alloc_workspace(desc, 4)
    outs = []
    for _ in range(3):
        y = torch.empty((4, H), dtype=torch.float32, device=DEV)
        ids = torch.empty((4, k), dtype=torch.int32, device=DEV)
        wt = torch.empty((4, k), dtype=torch.float32, device=DEV)
        M.moe_layer_forward(desc, x[:4].contiguous(), y, ws, ids_out=ids, w_out=wt)
        outs.append((y, ids))
    torch.cuda.synchronize()
    for y, ids in outs[1:]:
        assert torch.equal(ids, outs[0][1])
        assert rel_err(f64(y), f64(outs[0][0])) <= 1e-5


# --------------------------------------------------------------------- touched


@pytest.mark.parametrize("B,k,E", [(1, 2, 16), (4, 3, 64), (16, 3, 64), (64, 3, 64), (256, 3, 64),
                                   (8, 8, 256), (256, 32, 1024), (7, 5, 37)])
def test_touched_experts_bit_exact(M, S, B, k, E):
    ids = S.uniform_ids(B, E, k, seed=B * 1000 + k, device=DEV)
    cnt = torch.empty((1,), dtype=torch.int32, device=DEV)
    bm = torch.empty(((E + 31) // 32,), dtype=torch.int32, device=DEV)
    off = torch.empty((E + 1,), dtype=torch.int32, device=DEV)
    pairs = torch.empty((B * k,), dtype=torch.int32, device=DEV)
    M.moe_touched_experts(ids, E, cnt, bm, off, pairs)
    torch.cuda.synchronize()
    c, bitmap, offsets, pr = O.touched_experts(ids.cpu().numpy(), E)
    assert int(cnt) == c
    assert (bm.cpu().numpy().astype(np.uint32) == bitmap).all()
    assert (off.cpu().numpy() == offsets).all()
    assert (pairs.cpu().numpy() == pr).all()


def test_touched_experts_invalid(M):
    cnt = torch.empty((1,), dtype=torch.int32, device=DEV)
    for bad in ([[1, 1]], [[0, 9]]):
        ids = torch.tensor(bad, dtype=torch.int32, device=DEV)
        M.moe_touched_experts(ids, 9 if bad[0][1] != 9 else 9, cnt)
        torch.cuda.synchronize()
        assert int(cnt) == -1
