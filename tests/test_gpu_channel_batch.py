"""GPU parity of the batched channel-sparse path (2..8 tokens in one launch
that reads the union of the tokens' kept channels once; review of
arXiv:2610.37386, keep-rule table, "2단계", Table 7 rows B = 4 and 8, "속도")
against the fp64 oracle.

Per token: the kept list against channel_topk_select (bit-exact: the scores
are fp32 inputs, so both sides rank the same values), its sector count
against the brute-force sector function, and y within the layer tolerance
of the oracle's channel-sparse sum. Per batch: the union count and the union's
sector count against channel_union and sectors_touched (bit-exact).
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


def run_batch(M, desc, x, ids, wt, scores, keep):
    B, H = x.shape
    ws = M.alloc_workspace(desc, B)
    y = torch.full((B, H), float("nan"), dtype=torch.float32, device=DEV)
    kept = torch.full((B, max(keep, 1)), -1, dtype=torch.int32, device=DEV)
    sec = torch.empty((B,), dtype=torch.int64, device=DEV)
    ucount = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    usec = torch.full((1,), -1, dtype=torch.int64, device=DEV)
    M.moe_channel_topk_forward(desc, x, ids, wt, scores, keep, y, sec, ws, kept=kept, union_count=ucount,
                               union_sectors=usec)
    torch.cuda.synchronize()
    assert M.moe_get_status(ws) == M.MOE_OK
    return y, kept, sec, int(ucount), int(usec)


def check_batch(cm, cm_host, x, ids, wt, scores, keep, out, I, H):
    y, kept, sec, ucount, usec = out
    lists = []
    for b in range(x.shape[0]):
        want = O.channel_topk_select(scores[b].cpu().numpy(), ids[b].tolist(), keep)
        assert kept[b, :keep].cpu().numpy().tolist() == want.tolist(), b
        assert int(sec[b]) == O.sectors_touched(O.channel_major_ranges(want, H, base=cm.data_ptr())), b
        yo = O.channel_sparse_forward(f64(x[b]), cm_host, ids[b].tolist(), f64(wt[b]), want, I)
        if keep > 0:
            assert rel_err(f64(y[b]), yo) <= REL_TOL, b
        else:
            assert np.all(f64(y[b]) == 0)
        lists.append(want)
    u = O.channel_union(lists)
    assert ucount == u.size
    assert usec == O.sectors_touched(O.channel_major_ranges(u, H, base=cm.data_ptr()))
    return u


@pytest.mark.parametrize("B,keep", [(2, 40), (4, 33), (8, 1), (3, 0), (5, 4 * 64)])
def test_channel_batch_small(M, S, B, keep):
    H, E, I, k = 512, 16, 64, 4
    Ld = S.channel_major_layer(H, E, I, seed=900 + B, device=DEV)
    cm = Ld["cm"]
    desc = M.make_desc(H, E, I, k, layout=M.MOE_LAYOUT_CHANNEL_MAJOR, gate=cm)
    x = S.tokens(B, H, seed=901 + B, device=DEV)
    ids = S.uniform_ids(B, E, k, seed=902 + B, device=DEV)
    wt = S.router_weights(B, k, seed=903 + B, device=DEV)
    scale = S.channel_scale(E, I, seed=904 + B, device=DEV)
    scores = S.channel_scores(B, E, I, scale, seed=905 + B, device=DEV)
    out = run_batch(M, desc, x, ids, wt, scores, keep)
    host = f64(cm)
    check_batch(cm, lambda e, c: host[e][c], x, ids, wt, scores, keep, out, I, H)


def test_channel_batch_shared_channels_read_once(M, S):
    # every token routes to the same experts with the same scores: the union
    # is one token's kept set, read once, and each token's y is its own
    H, E, I, k, B, keep = 512, 8, 48, 3, 6, 50
    Ld = S.channel_major_layer(H, E, I, seed=910, device=DEV)
    cm = Ld["cm"]
    desc = M.make_desc(H, E, I, k, layout=M.MOE_LAYOUT_CHANNEL_MAJOR, gate=cm)
    x = S.tokens(B, H, seed=911, device=DEV)
    ids = S.uniform_ids(1, E, k, seed=912, device=DEV).repeat(B, 1).contiguous()
    wt = S.router_weights(B, k, seed=913, device=DEV)
    scores = torch.rand((1, E, I), device=DEV).repeat(B, 1, 1).contiguous()
    out = run_batch(M, desc, x, ids, wt, scores, keep)
    host = f64(cm)
    u = check_batch(cm, lambda e, c: host[e][c], x, ids, wt, scores, keep, out, I, H)
    assert u.size == keep


@pytest.mark.parametrize("B,frac", [(4, 0.13), (8, 0.18)])
def test_channel_batch_thinking_shape(M, S, B, frac):
    """One Qwen3-Thinking layer (H 2048, E 128, I 768, k 8) at batch 4 and 8:
    the union the batch reads is smaller than the sum of the tokens' kept
    sets, and every kept list, sector count and output matches the oracle."""
    w = S.WORKLOADS["channel_topk"]
    H, E, I, k = w["H"], w["E"], w["I"], w["k"]
    keep = S.keep_count(frac, k, I)
    Ld = S.channel_major_layer(H, E, I, seed=S.weight_seed(5, 1), device=DEV)
    cm = Ld["cm"]
    desc = M.make_desc(H, E, I, k, layout=M.MOE_LAYOUT_CHANNEL_MAJOR, gate=cm)
    x = S.tokens(B, H, seed=S.act_seed(5, 1), device=DEV)
    ids = S.uniform_ids(B, E, k, seed=S.act_seed(5, 1) + 1, device=DEV)
    wt = torch.softmax(torch.randn((B, k), device=DEV), dim=1)
    scale = S.channel_scale(E, I, seed=S.weight_seed(5, 1) + 7, device=DEV)
    scores = S.channel_scores(B, E, I, scale, seed=S.act_seed(5, 1) + 2, device=DEV)
    out = run_batch(M, desc, x, ids, wt, scores, keep)
    cache = {}

    def cm_host(e, c):
        if e not in cache:
            cache[e] = f64(cm[e])
        return cache[e][c]
    u = check_batch(cm, cm_host, x, ids, wt, scores, keep, out, I, H)
    assert u.size < B * keep
    assert out[4] == 384 * u.size  # aligned channel-major channels: 384 sectors each
