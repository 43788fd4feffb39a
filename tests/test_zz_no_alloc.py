"""The no-allocation entry point, moe_layer_forward_static.

Callers that cannot allocate device memory (for example code recording into a
stream while allocation calls are forbidden, or a host process whose device
memory is all owned by its own pool) run a layer through this entry point; its
scratch space is a fixed array inside the library instead of a caller
workspace. These checks call it through the C ABI and compare it with the
workspace entry point, moe_layer_forward, on the same inputs, twice in a row
(the second call runs on the scratch the first one left behind). This file is
collected last so that a run stopping at the first failure has already run
every other test; it also passes on its own in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

from tests.parity_util import REL_TOL, f64, rel_err

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def M():
    from mixture_experts_decode_moe_b200 import build
    build.build()
    from mixture_experts_decode_moe_b200 import moedec
    return moedec


def layer(M, S, wtype):
    H, E, I, k, I_sh = 2048, 64, 256, 8, 128
    if wtype == "int4":
        L = S.swiglu_layer_int4(H, E, I, I_sh, seed=4244, device=DEV, router_scale=0.1)
        extra = {"wtype": M.MOE_W_INT4_G64, "gate_s": L["gate_s"], "up_s": L["up_s"], "down_s": L["down_s"]}
    else:
        L = S.swiglu_layer_bf16(H, E, I, I_sh, seed=4242, device=DEV, router_scale=0.1)
        extra = {}
    desc = M.make_desc(H, E, I, k, router=L["router"], gate=L["gate"], up=L["up"], down_t=L["down_t"],
                       sh_gate=L["sh_gate"], sh_up=L["sh_up"], sh_down_t=L["sh_down_t"], **extra)
    return L, desc, H, k


@pytest.mark.parametrize("wtype,B", [("bf16", 1), ("bf16", 4), ("int4", 1), ("int4", 8)])
def test_static_scratch_matches_workspace_entry_point(M, wtype, B):
    from mixture_experts_decode_moe_b200 import synth as S
    L, desc, H, k = layer(M, S, wtype)
    x = S.tokens(B, H, seed=4243, device=DEV)

    def outputs():
        return (torch.empty((B, H), dtype=torch.float32, device=DEV),
                torch.empty((B, H), dtype=torch.bfloat16, device=DEV),
                torch.empty((B, k), dtype=torch.int32, device=DEV),
                torch.empty((B, k), dtype=torch.float32, device=DEV))

    ws = M.alloc_workspace(desc, B)
    y0, xn0, ids0, w0 = outputs()
    M.moe_layer_forward(desc, x, y0, ws, x_next=xn0, ids_out=ids0, w_out=w0)
    for call in range(2):
        y, xn, ids, w = outputs()
        status = torch.full((1,), -1, dtype=torch.int32, device=DEV)
        torch.cuda.synchronize()
        free0, used0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        allocs0 = torch.cuda.memory_stats().get("allocation.all.allocated", 0)
        M.moe_layer_forward_static(desc, x, y, x_next=xn, ids_out=ids, w_out=w, status_out=status)
        torch.cuda.synchronize()
        # nothing was allocated: not through torch, and not from the device
        # (the second call runs with the library already loaded in this context)
        assert torch.cuda.memory_allocated() == used0, call
        assert torch.cuda.memory_stats().get("allocation.all.allocated", 0) == allocs0, call
        if call == 1:
            assert torch.cuda.mem_get_info()[0] == free0
        assert int(status) == M.MOE_OK, (call, int(status))
        assert torch.equal(ids, ids0), call
        assert np.allclose(f64(w), f64(w0), rtol=1e-6), call
        assert rel_err(f64(y), f64(y0)) <= REL_TOL, call
        assert rel_err(f64(xn), f64(xn0)) <= REL_TOL, call
    assert M.moe_get_status(ws) == M.MOE_OK


def test_static_scratch_rejected_call_leaves_scratch_alone(M):
    """A call with a bad argument returns an error before anything is
    launched; the next valid call still matches the workspace entry point."""
    from mixture_experts_decode_moe_b200 import synth as S
    L, desc, H, k = layer(M, S, "bf16")
    x = S.tokens(1, H, seed=4245, device=DEV)
    y0 = torch.empty((1, H), dtype=torch.float32, device=DEV)
    ws = M.alloc_workspace(desc, 1)
    M.moe_layer_forward(desc, x, y0, ws)
    # ids without weights: rejected on the host
    ids = torch.empty((1, k), dtype=torch.int32, device=DEV)
    st = M._lib.moe_layer_forward_static(ctypes.byref(desc), M._ptr(x), 1, M._ptr(y0), None, M._ptr(ids), None,
                                         None, M._stream(None))
    assert st == M.MOE_ERR_INVALID
    y = torch.empty((1, H), dtype=torch.float32, device=DEV)
    M.moe_layer_forward_static(desc, x, y)
    torch.cuda.synchronize()
    assert rel_err(f64(y), f64(y0)) <= REL_TOL


def test_static_scratch_rejects_shapes_beyond_its_size(M):
    # E = 1024 experts at batch 8 needs more scratch than the fixed array holds:
    # rejected on the host before anything is launched (pointers are never read)
    d = M.LayerDesc(2048, 1024, 512, 8, 0, 0, 0, 0)
    need = M.moe_workspace_bytes(d, 8)
    assert need > M.MOE_STATIC_SCRATCH_BYTES
    dummy = ctypes.c_void_p(4096)
    st = M._lib.moe_layer_forward_static(ctypes.byref(d), dummy, 8, dummy, None, None, None, None, None)
    assert st == M.MOE_ERR_UNSUPPORTED
    assert M.moe_workspace_bytes(M.LayerDesc(2048, 256, 512, 8, 0, 0, 0, 512), 8) <= M.MOE_STATIC_SCRATCH_BYTES
