"""The seeded input generators: determinism, shapes, value ranges, and that
int4 codes are laid out as the format defines (decoded by the oracle)."""

import numpy as np
import torch

from mixture_experts_decode_moe_b200 import synth as S
from oracle import moe_oracle as O


def test_deterministic_and_shaped():
    a = S.swiglu_layer_bf16(64, 4, 8, 16, seed=5)
    b = S.swiglu_layer_bf16(64, 4, 8, 16, seed=5)
    for n in a:
        assert torch.equal(a[n], b[n])
    assert a["gate"].shape == (4, 8, 64) and a["sh_up"].shape == (16, 64)
    assert a["gate"].dtype == torch.bfloat16
    c = S.swiglu_layer_bf16(64, 4, 8, 16, seed=6)
    assert not torch.equal(a["gate"], c["gate"])
    x = S.tokens(3, 64, seed=1)
    assert x.shape == (3, 64) and abs(float(x.float().std()) - 1) < 0.2


def test_uniform_ids_distinct_in_range():
    ids = S.uniform_ids(256, 64, 3, seed=2)
    assert ids.dtype == torch.int32 and ids.shape == (256, 3)
    assert int(ids.min()) >= 0 and int(ids.max()) < 64
    for row in ids.tolist():
        assert len(set(row)) == 3


def test_int4_codes_decode_to_quantised_weights():
    L = S.swiglu_layer_int4(512, 2, 64, 0, seed=3)
    assert L["gate"].dtype == torch.uint8 and L["gate"].shape == (2, 64, 256)
    assert L["gate_s"].shape == (2, 64, 8) and L["down_s"].shape == (2, 1, 512)
    q = O.int4_unpack(L["gate"][1].numpy())
    assert q.min() >= -8 and q.max() <= 7
    s = L["gate_s"][1].float().numpy()
    w = O.dequant_rows_int4(L["gate"][1].numpy(), s)
    assert np.allclose(w, q * np.repeat(s, 64, axis=1))
    assert (s >= 0.005 - 1e-4).all() and (s <= 0.03 + 1e-4).all()
    # codes are the rounded w0/s: |q*s| stays within the N(0, 0.02) range
    assert np.abs(w).max() < 8 * 0.03 + 1e-6


def test_channel_scores_and_keep():
    sc = S.channel_scale(128, 768, seed=4)
    assert (sc >= 1.0).all()
    scores = S.channel_scores(1, 128, 768, sc, seed=5)
    assert scores.shape == (1, 128, 768) and (scores >= 0).all()
    assert S.keep_count(0.13, 8, 768) == 799 and S.keep_count(0.18, 8, 768) == 1106
    cm = S.channel_major_layer(64, 2, 3, seed=6)
    assert cm["cm"].shape == (2, 3, 3, 64)


def test_lowrank_down_columns_concentrate_in_the_planted_subspace():
    # the oracle's rank-32 basis of the generated down columns spans the
    # planted subspace (principal angles near 0), and captures about
    # 1 - noise^2 of the columns' energy
    import numpy as np
    from oracle import moe_oracle as O
    from mixture_experts_decode_moe_b200 import synth as S
    H, E, I, r, nu = 256, 4, 96, 8, 0.3
    L = S.channel_major_layer_lowrank(H, E, I, seed=5, rank=r, noise=nu)
    cm = L["cm"].float().double().numpy()
    assert cm.shape == (E, I, 3, H)
    D = cm[:, :, 2, :].reshape(E * I, H)
    assert abs(D.std() / S.W_STD - 1.0) < 0.05
    U = O.recovery_basis(D, rank=r)
    B = np.linalg.qr(L["basis"].double().numpy())[0]
    cosines = np.linalg.svd(U.T @ B, compute_uv=False)
    assert cosines.min() > 0.97
    captured = np.sum((D @ U) ** 2) / np.sum(D ** 2)
    assert abs(captured - (1 - nu ** 2 + nu ** 2 * r / H)) < 0.03
