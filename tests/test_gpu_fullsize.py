"""Full-size parity. The launch configuration bench.py times: the A3B-shaped
bf16 stack (40 layers, hidden 2048, 256 experts top-8, intermediate 512, one
shared expert, 64.7 GB of weights), batch 1, pre-norm on, one token per launch;
and the channel-sparse stack at the Qwen3-Thinking shape (48 layers, 58 GB).

Every layer of two tokens is checked with teacher forcing: the oracle
recomputes layer l from the GPU's x_l (ids bit-exact except logged near-ties,
y and x_{l+1} within the layer tolerance).
"""

import pytest
import torch

from oracle import moe_oracle as O
from tests.parity_util import REL_TOL, check_ids, f64, rel_err

pytestmark = pytest.mark.gpu

DEV = "cuda"


class HostLayer:
    def __init__(self, L):
        self.L = L
        self.R = f64(L["router"])
        self.shared = (f64(L["sh_gate"]), f64(L["sh_up"]), f64(L["sh_down_t"]))

    def expert(self, e):
        L = self.L
        return f64(L["gate"][e]), f64(L["up"][e]), f64(L["down_t"][e])


def test_a3b_stack_full_size_teacher_forced():
    from mixture_experts_decode_moe_b200 import build
    build.build()
    from mixture_experts_decode_moe_b200 import moedec as M
    from mixture_experts_decode_moe_b200 import synth as S

    w = S.WORKLOADS["a3b_bf16"]
    H, E, I, k, I_sh, nl = w["H"], w["E"], w["I"], w["k"], w["I_shared"], w["layers"]
    layers = [S.swiglu_layer_bf16(H, E, I, I_sh, seed=S.weight_seed(w["cfg"], l), device=DEV,
                                  router_scale=w["router_scale"]) for l in range(nl)]
    descs = [M.make_desc(H, E, I, k, router=L["router"], gate=L["gate"], up=L["up"], down_t=L["down_t"],
                         sh_gate=L["sh_gate"], sh_up=L["sh_up"], sh_down_t=L["sh_down_t"]) for L in layers]
    xs = S.tokens(w["tokens"], H, seed=S.act_seed(w["cfg"]), device=DEV)
    ws = M.alloc_workspace(descs[0], 1)
    log = []
    for tok in (0, 137):
        xo = torch.empty((1, H), dtype=torch.bfloat16, device=DEV)
        xh = torch.empty((nl + 1, 1, H), dtype=torch.bfloat16, device=DEV)
        yh = torch.empty((nl, 1, H), dtype=torch.float32, device=DEV)
        ih = torch.empty((nl, 1, k), dtype=torch.int32, device=DEV)
        wh = torch.empty((nl, 1, k), dtype=torch.float32, device=DEV)
        M.moe_stack_forward(descs, xs[tok:tok + 1], xo, ws, x_hist=xh, y_hist=yh, ids_hist=ih, w_hist=wh,
                            flags=M.MOE_STACK_PRE_RMSNORM)
        torch.cuda.synchronize()
        assert M.moe_get_status(ws) == M.MOE_OK
        assert torch.equal(xh[nl], xo)
        for l in range(nl):
            HL = HostLayer(layers[l])
            xl = f64(xh[l, 0])
            xn, yo, io, wo, lo, _ = O.stack_layer(xl, HL.R, HL.expert, k, shared=HL.shared)
            if check_ids(ih[l, 0].tolist(), io, lo, log, f"tok{tok}l{l}"):
                continue
            assert rel_err(f64(yh[l, 0]), yo) <= REL_TOL, (tok, l)
            assert rel_err(f64(xh[l + 1, 0]), xn) <= REL_TOL, (tok, l)
    print("near-tie id differences logged:", log)


def test_channel_stack_full_size_teacher_forced():
    """The Qwen3-Thinking-shaped channel-sparse stack: 48 layers, hidden 2048,
    128 experts top-8, 768 channels (58 GB channel-major), 13% of the 6144
    candidates kept, every layer of one token checked."""
    from mixture_experts_decode_moe_b200 import build
    build.build()
    from mixture_experts_decode_moe_b200 import moedec as M
    from mixture_experts_decode_moe_b200 import synth as S

    w = S.WORKLOADS["channel_topk"]
    H, E, I, k, nl = w["H"], w["E"], w["I"], w["k"], w["layers"]
    keep = S.keep_count(w["keep_frac"][0], k, I)
    layers = [S.channel_major_layer(H, E, I, seed=S.weight_seed(5, l), device=DEV) for l in range(nl)]
    descs = [M.make_desc(H, E, I, k, layout=M.MOE_LAYOUT_CHANNEL_MAJOR, router=Ld["router"], gate=Ld["cm"])
             for Ld in layers]
    scale = [S.channel_scale(E, I, seed=S.weight_seed(5, l) + 7, device=DEV) for l in range(nl)]
    scores = torch.cat([S.channel_scores(1, E, I, scale[l], seed=S.act_seed(5, l), device=DEV) for l in range(nl)])
    x = S.tokens(1, H, seed=S.act_seed(5) + 99, device=DEV)
    ws = M.alloc_workspace(descs[0], 1)
    xo = torch.empty((1, H), dtype=torch.bfloat16, device=DEV)
    xh = torch.empty((nl + 1, H), dtype=torch.bfloat16, device=DEV)
    yh = torch.empty((nl, H), dtype=torch.float32, device=DEV)
    ih = torch.empty((nl, k), dtype=torch.int32, device=DEV)
    wh = torch.empty((nl, k), dtype=torch.float32, device=DEV)
    kh = torch.empty((nl, keep), dtype=torch.int32, device=DEV)
    sec = torch.empty((nl,), dtype=torch.int64, device=DEV)
    M.moe_channel_stack_forward(descs, x, scores, keep, xo, sec, ws, x_hist=xh, y_hist=yh, ids_hist=ih, w_hist=wh,
                                kept_hist=kh, flags=M.MOE_STACK_PRE_RMSNORM)
    torch.cuda.synchronize()
    assert M.moe_get_status(ws) == M.MOE_OK
    log = []
    for l in range(nl):
        cm = layers[l]["cm"]
        xl = f64(xh[l])
        u = O.rmsnorm_bf16(xl)
        io, _, lo, _ = O.route_topk(u, f64(layers[l]["router"]), k)
        cache = {int(e): f64(cm[int(e)]) for e in io}
        xn, yo, io, wo, lo, kept = O.channel_stack_layer(xl, f64(layers[l]["router"]), lambda e, c: cache[e][c],
                                                         scores[l].cpu().numpy(), k, keep, I)
        if check_ids(ih[l].tolist(), io, lo, log, f"l{l}"):
            continue
        assert kh[l].cpu().numpy().tolist() == kept.tolist(), l
        assert int(sec[l]) == 384 * keep
        assert rel_err(f64(yh[l]), yo) <= REL_TOL, l
        assert rel_err(f64(xh[l + 1]), xn) <= REL_TOL, l
    print("near-tie id differences logged:", log)
