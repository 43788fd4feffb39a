"""GPU parity of the partial screen ([Reader] "가중치만으로 만든 reader", step 1,
partial scan: in each block of 128 rotated coordinates only the codes of the
m coordinates with the largest |R x| are read) against the fp64 oracle.

  * layout: the coordinate-major codes are the channel-major codes
    transposed, bit for bit;
  * estimates: g_hat, v_hat within 1e-5 x the oracle's bound on the partial
    sums (reader_estimate_bound over the masked codes), against
    reader_estimate_partial. The kernel rotates the token in fp64, so its
    choice of the m coordinates is exact and is the oracle's;
  * scores: within the propagated bound (as for the full screen);
  * m = 128 reads every code (the full screen's estimates), m = 0 none.
"""

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from tests.parity_util import f64
from tests.test_gpu_reader import EST_TOL, build_sketch, unpack_codes

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


def setup(M, S, H, E, I, k, B, seed):
    Ld = S.channel_major_layer(H, E, I, seed=seed, device=DEV)
    cm = Ld["cm"]
    desc = M.make_desc(H, E, I, k, layout=M.MOE_LAYOUT_CHANNEL_MAJOR, gate=cm)
    signs = S.reader_signs(H, seed=seed + 1, device=DEV)
    codes, scales, rho, dnorm = build_sketch(M, desc, signs)
    cmaj = torch.empty(M.reader_cmaj_shape(desc), dtype=torch.int32, device=DEV)
    M.moe_reader_codes_coordinate_major(desc, codes, cmaj)
    x = S.tokens(B, H, seed=seed + 2, device=DEV)
    ids = S.uniform_ids(B, E, k, seed=seed + 3, device=DEV)
    wt = S.router_weights(B, k, seed=seed + 4, device=DEV)
    torch.cuda.synchronize()
    return cm, desc, signs, codes, scales, dnorm, cmaj, x, ids, wt


@pytest.mark.parametrize("H,E,I,k,B", [(512, 8, 64, 3, 2), (2048, 6, 48, 4, 2)])
def test_coordinate_major_codes_are_a_transpose(M, S, H, E, I, k, B):
    _, _, _, codes, _, _, cmaj, *_ = setup(M, S, H, E, I, k, B, seed=960 + H)
    c = unpack_codes(codes.cpu().numpy().view(np.uint32), H).reshape(E, I, 2, H)  # [e, c, r, h]
    t = unpack_codes(cmaj.cpu().numpy().view(np.uint32), I)                        # [e, r, h, c]
    assert np.array_equal(t, c.transpose(0, 2, 3, 1))


@pytest.mark.parametrize("m", [80, 1, 128, 0])
@pytest.mark.parametrize("H,E,I,k,B", [(512, 8, 64, 3, 2), (2048, 6, 48, 4, 2)])
def test_partial_screen_matches_oracle(M, S, H, E, I, k, B, m):
    cm, desc, signs, codes, scales, dnorm, cmaj, x, ids, wt = setup(M, S, H, E, I, k, B, seed=970 + H)
    scores = torch.full((B, E, I), -1.0, dtype=torch.float32, device=DEV)
    est = torch.zeros((B, k, I, 2), dtype=torch.float32, device=DEV)
    M.moe_reader_screen_partial(desc, x, ids, wt, signs, cmaj, scales, dnorm, m, scores, est)
    full_sc = torch.zeros((B, E, I), dtype=torch.float32, device=DEV)
    full_est = torch.zeros((B, k, I, 2), dtype=torch.float32, device=DEV)
    M.moe_reader_screen(desc, x, ids, wt, signs, codes, scales, dnorm, full_sc, full_est)
    torch.cuda.synchronize()
    host = f64(cm)
    sg = f64(signs)
    sc_gpu, est_gpu = f64(scores), f64(est)
    for b in range(B):
        xb = f64(x[b])
        mask = O.reader_partial_mask(xb, sg, m)
        for t, e in enumerate(ids[b].tolist()):
            for c in range(I):
                g, v, d = host[e, c]
                cg, scg, _ = O.reader_sketch_row(g, sg)
                cv, scv, _ = O.reader_sketch_row(v, sg)
                gh = O.reader_estimate_partial(xb, cg, scg, sg, m)
                vh = O.reader_estimate_partial(xb, cv, scv, sg, m)
                tg = EST_TOL * O.reader_estimate_bound(xb, np.where(mask, cg, 0), scg)
                tv = EST_TOL * O.reader_estimate_bound(xb, np.where(mask, cv, 0), scv)
                assert abs(est_gpu[b, t, c, 0] - gh) <= tg, (b, e, c)
                assert abs(est_gpu[b, t, c, 1] - vh) <= tv, (b, e, c)
                dn = float(np.sqrt(np.sum(d ** 2)))
                sil = float(O.silu(np.float64(gh)))
                ts = wt[b, t].item() * dn * (1.1 * abs(vh) * tg + abs(sil) * tv + tg * tv) + \
                    1e-5 * O.reader_score(wt[b, t].item(), dn, gh, vh)
                assert abs(sc_gpu[b, e, c] - O.reader_score(wt[b, t].item(), dn, gh, vh)) <= ts, (b, e, c)
    if m == 128:
        assert np.allclose(est_gpu, f64(full_est), rtol=1e-4, atol=1e-6)
    if m == 0:
        assert not np.any(est_gpu) and not np.any(sc_gpu[sc_gpu != -1.0])
