"""The timeout path of the persistent decode kernel, driven from the host.

Every device-side wait in libmoedec is bounded. These tests make one wait run
out without any GPU fault: the workspace gets a short wait budget and the
injection bit that makes every grid-wide barrier wait for one arrival more
than the grid makes (an arrival nothing ever makes). The call must come back
on its own, with MOE_ERR_TIMEOUT in the workspace status word, and after
moe_workspace_init() the same workspace must run a normal call that matches
the fp64 oracle. The budget alone, without the injection, leaves a normal
call untouched.
"""

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from tests.parity_util import REL_TOL, f64, rel_err

pytestmark = pytest.mark.gpu

DEV = "cuda"
SHORT_BUDGET = 1_000_000  # cycles: about 0.5 ms at 2 GHz, far above any wait of a normal call


@pytest.fixture(scope="module")
def M():
    from mixture_experts_decode_moe_b200 import build
    build.build()
    from mixture_experts_decode_moe_b200 import moedec
    return moedec


def oracle_check(L, x, y, k):
    R, G, V, D = (f64(L[n]) for n in ("router", "gate", "up", "down_t"))
    shared = tuple(f64(L[n]) for n in ("sh_gate", "sh_up", "sh_down_t"))
    for b in range(x.shape[0]):
        want, *_ = O.moe_layer(f64(x[b]), R, lambda e: (G[e], V[e], D[e]), k, shared)
        assert rel_err(f64(y[b]), want) <= REL_TOL, b


@pytest.mark.parametrize("B", [1, 4])
def test_injected_barrier_wait_times_out_and_workspace_recovers(M, B):
    from mixture_experts_decode_moe_b200 import synth as S
    H, E, I, k, I_sh = 2048, 64, 128, 8, 128
    L = S.swiglu_layer_bf16(H, E, I, I_sh, seed=4300 + B, device=DEV, router_scale=0.1)
    desc = M.make_desc(H, E, I, k, router=L["router"], gate=L["gate"], up=L["up"], down_t=L["down_t"],
                       sh_gate=L["sh_gate"], sh_up=L["sh_up"], sh_down_t=L["sh_down_t"])
    x = S.tokens(B, H, seed=4310 + B, device=DEV)
    y = torch.zeros((B, H), dtype=torch.float32, device=DEV)
    ws = M.alloc_workspace(desc, B)

    # the budget alone changes nothing for a normal call
    M.moe_workspace_set_wait_budget(ws, SHORT_BUDGET)
    M.moe_layer_forward(desc, x, y, ws)
    assert M.moe_get_status(ws) == M.MOE_OK
    oracle_check(L, x, y, k)

    # an arrival that never comes: the barrier's wait runs out, the call returns
    M.moe_workspace_set_inject(ws, M.MOE_INJECT_BARRIER_EXTRA_ARRIVAL)
    M.moe_layer_forward(desc, x, y, ws)
    torch.cuda.synchronize()
    assert M.moe_get_status(ws) == M.MOE_ERR_TIMEOUT

    # a cleared workspace (default budget, no injection) runs normally again
    M.moe_workspace_init(ws)
    y.zero_()
    M.moe_layer_forward(desc, x, y, ws)
    assert M.moe_get_status(ws) == M.MOE_OK
    oracle_check(L, x, y, k)

