"""GPU parity of the rank-32 recovery of dropped channels (review of
arXiv:2610.37386, "가중치만으로 만든 reader", step 3, eq. 2) against the fp64
oracle, on channel-major layers whose down columns share a planted rank-32
subspace (channel_major_layer_lowrank), so that the top-32 subspace is well
separated and both sides must find the same one.

  * basis: the largest principal angle between the GPU's U and the oracle's
    SVD basis (recovery_basis) is below 1e-2;
  * coefficients: U b_j (the projection of d_j, independent of the basis
    chosen inside the subspace) within 2e-3 of the oracle's U U^T d_j
    (b_j is stored as fp16: 2^-11 relative per coefficient);
  * output: kept channels exact (moe_channel_topk_forward) plus the recovered
    part from the GPU screen's estimates (moe_reader_screen) against eq. 2 in
    the oracle (reader_output with the oracle's own sketch estimates, basis
    and coefficients), within the layer tolerance.
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


def build_map(M, desc, H, n):
    U = torch.empty((H, M.MOE_RECOVERY_RANK), dtype=torch.float32, device=DEV)
    coeffs = torch.empty((n, M.MOE_RECOVERY_RANK), dtype=torch.int16, device=DEV)
    M.moe_recovery_build(desc, U, coeffs)
    torch.cuda.synchronize()
    return U, coeffs


def fp16_host(t):
    return t.cpu().numpy().view(np.float16).astype(np.float64)


@pytest.fixture(scope="module")
def layer(M, S):
    H, E, I = 512, 16, 256
    Ld = S.channel_major_layer_lowrank(H, E, I, seed=940, device=DEV)
    cm = Ld["cm"]
    desc = M.make_desc(H, E, I, 4, layout=M.MOE_LAYOUT_CHANNEL_MAJOR, gate=cm)
    U, coeffs = build_map(M, desc, H, E * I)
    host = f64(cm)                              # [E, I, 3, H]
    D = host[:, :, 2, :].reshape(E * I, H)      # every down column, one per row
    Uo = O.recovery_basis(D)
    return dict(H=H, E=E, I=I, cm=cm, desc=desc, U=U, coeffs=coeffs, host=host, D=D, Uo=Uo)


def test_basis_spans_the_oracle_subspace(layer):
    Ug = f64(layer["U"])
    assert np.allclose(Ug.T @ Ug, np.eye(Ug.shape[1]), atol=1e-5)
    cos = np.linalg.svd(Ug.T @ layer["Uo"], compute_uv=False)
    assert np.sqrt(max(0.0, 1.0 - cos.min() ** 2)) < 1e-2


def test_coefficients_project_onto_the_subspace(layer):
    Ug = f64(layer["U"])
    b = fp16_host(layer["coeffs"])
    Uo, D = layer["Uo"], layer["D"]
    rng = np.random.default_rng(941)
    for j in rng.choice(D.shape[0], 64, replace=False):
        want = Uo @ O.recovery_coeffs(Uo, D[j])
        got = Ug @ b[j]
        assert np.linalg.norm(got - want) <= 2e-3 * np.linalg.norm(want), j


@pytest.mark.parametrize("keep", [0, 133, 4 * 256])
def test_recovered_output_matches_eq2(M, S, layer, keep):
    H, E, I, k, B = layer["H"], layer["E"], layer["I"], 4, 2
    desc, cm, host = layer["desc"], layer["cm"], layer["host"]
    signs = S.reader_signs(H, seed=942, device=DEV)
    shp = M.reader_sketch_shapes(desc)
    codes = torch.empty(shp["codes"], dtype=torch.int32, device=DEV)
    scales = torch.empty(shp["scales"], dtype=torch.int16, device=DEV)
    rho = torch.empty(shp["rho"], dtype=torch.float32, device=DEV)
    dnorm = torch.empty(shp["dnorm"], dtype=torch.float32, device=DEV)
    M.moe_reader_build(desc, signs, codes, scales, rho, dnorm)
    x = S.tokens(B, H, seed=943, device=DEV)
    ids = S.uniform_ids(B, E, k, seed=944, device=DEV)
    wt = S.router_weights(B, k, seed=945, device=DEV)
    scores = S.channel_scores(B, E, I, S.channel_scale(E, I, seed=946, device=DEV), seed=947, device=DEV)
    sc_unused = torch.zeros((B, E, I), dtype=torch.float32, device=DEV)
    est = torch.zeros((B, k, I, 2), dtype=torch.float32, device=DEV)
    M.moe_reader_screen(desc, x, ids, wt, signs, codes, scales, dnorm, sc_unused, est)
    ws = M.alloc_workspace(desc, B)
    y = torch.empty((B, H), dtype=torch.float32, device=DEV)
    kept = torch.zeros((B, max(keep, 1)), dtype=torch.int32, device=DEV)
    sec = torch.empty((B,), dtype=torch.int64, device=DEV)
    M.moe_channel_topk_forward(desc, x, ids, wt, scores, keep, y, sec, ws, kept=kept)
    M.moe_channel_recover(desc, ids, wt, est, kept, keep, layer["U"], layer["coeffs"], y)
    torch.cuda.synchronize()
    assert M.moe_get_status(ws) == M.MOE_OK
    sg = f64(signs)
    Uo = layer["Uo"]
    for b in range(B):
        xb = f64(x[b])
        idl = ids[b].tolist()
        wl = f64(wt[b])
        kept_o = O.channel_topk_select(scores[b].cpu().numpy(), idl, keep)
        assert kept[b, :keep].cpu().numpy().tolist() == kept_o.tolist()
        kset = set(kept_o.tolist())

        def sketch(e, c):
            g, v, d = host[e, c]
            cg, scg, _ = O.reader_sketch_row(g, sg)
            cv, scv, _ = O.reader_sketch_row(v, sg)
            return cg, scg, cv, scv, float(np.sqrt(np.sum(d ** 2)))
        _, o_est = O.reader_screen(xb, idl, wl, sketch, I, sg)
        kept_terms, dropped_terms = [], []
        for t, e in enumerate(idl):
            for c in range(I):
                g, v, d = host[e, c]
                if e * I + c in kset:
                    kept_terms.append((wl[t], float(O.silu(g @ xb) * (v @ xb)), d))
                else:
                    gh, vh = o_est[t, c]
                    dropped_terms.append((wl[t], float(O.silu(np.float64(gh)) * vh), O.recovery_coeffs(Uo, d)))
        want = O.reader_output(kept_terms, dropped_terms, Uo)
        assert rel_err(f64(y[b]), want) <= REL_TOL, (b, keep)
