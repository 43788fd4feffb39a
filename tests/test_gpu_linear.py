"""GPU parity for experts that are one matrix (y[b] = sum_s w W_ids x[b]): the
batch-sweep workload at full size (64 experts of 8192 x 8192 bf16, top-3,
B in {1, 4, 16, 64, 256}), checked on every output row of up to 16 tokens
(all tokens for B <= 16) against fp64, and small shapes that drive each engine (token groups below
and above the tensor-core threshold, groups wider than 32, the widest 256)
checked in full. Touched-expert counts are compared with the oracle's.
"""

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from tests.parity_util import REL_TOL, f64, rel_err

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


def linear_desc(M, W, H, E, k):
    return M.make_desc(H, E, H, k, kind=M.MOE_EXPERT_LINEAR, gate=W)


def run(M, desc, x, ids, w):
    B, H = x.shape
    ws = M.alloc_workspace(desc, B)
    y = torch.empty((B, H), dtype=torch.float32, device=DEV)
    M.moe_expert_forward(desc, x, ids, w, y, ws)
    torch.cuda.synchronize()
    assert M.moe_get_status(ws) == M.MOE_OK
    return y


@pytest.mark.parametrize("H,E,k,B", [
    (1024, 16, 3, 5),     # all groups below the tensor-core threshold
    (1024, 8, 3, 64),     # groups of ~24 tokens: tensor cores, N = 32
    (512, 4, 3, 64),      # groups of 48: N = 64
    (256, 3, 3, 256),     # every token picks every expert: N = 256
    (768, 24, 5, 48),     # a mix of both engines
])
def test_linear_small_shapes_full_check(M, S, H, E, k, B):
    W = S.linear_experts(E, H, seed=700 + E, device=DEV)
    x = S.tokens(B, H, seed=701, device=DEV)
    ids = S.uniform_ids(B, E, k, seed=702 + B, device=DEV)
    w = torch.rand((B, k), device=DEV) + 0.5
    y = run(M, linear_desc(M, W, H, E, k), x, ids, w)
    Wh = f64(W)
    X = f64(x)
    for b in range(B):
        want = O.linear_experts(X[b], lambda e: Wh[e], ids[b].tolist(), f64(w[b]))
        assert rel_err(f64(y[b]), want) <= REL_TOL, b


@pytest.fixture(scope="module")
def sweep(S):
    wl = S.WORKLOADS["batch_sweep"]
    W = S.linear_experts(wl["E"], wl["H"], seed=S.weight_seed(3, 0), device=DEV)
    return wl, W


@pytest.mark.parametrize("B", [1, 4, 16, 64, 256])
def test_batch_sweep_full_size_sampled(M, S, sweep, B):
    wl, W = sweep
    H, E, k = wl["H"], wl["E"], wl["k"]
    x = S.tokens(B, H, seed=S.act_seed(3) + B, device=DEV)
    ids = S.uniform_ids(B, E, k, seed=S.act_seed(3) + 1000 + B, device=DEV)
    w = torch.ones((B, k), device=DEV)  # the sweep sums the k experts' outputs
    y = run(M, linear_desc(M, W, H, E, k), x, ids, w)
    # touched experts: the device counting sort against the oracle's
    cnt = torch.empty((1,), dtype=torch.int32, device=DEV)
    M.moe_touched_experts(ids, E, cnt)
    torch.cuda.synchronize()
    assert int(cnt) == O.touched_experts(ids.cpu().numpy(), E)[0]
    # every output row of up to 16 tokens (all tokens for B <= 16) against the
    # oracle; one expert matrix is converted to fp64 at a time and applied to
    # all chosen tokens that route to it
    r = np.random.default_rng(B)
    toks = sorted(r.choice(B, min(B, 16), replace=False).tolist())
    X = f64(x)
    idh = ids.cpu().numpy()
    wh = f64(w)
    want = {b: np.zeros(H) for b in toks}
    for e in sorted({int(idh[b, s]) for b in toks for s in range(k)}):
        We = f64(W[e])
        users = [(b, s) for b in toks for s in range(k) if idh[b, s] == e]
        Ye = O.linear_experts(X[[b for b, _ in users]].T, lambda _e: We, [e], [1.0])
        for col, (b, s) in enumerate(users):
            want[b] += wh[b, s] * Ye[:, col]
    yh = f64(y)
    for b in toks:
        assert rel_err(yh[b], want[b]) <= REL_TOL, (B, b)
