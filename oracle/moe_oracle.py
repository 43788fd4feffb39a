"""fp64 CPU oracle for the routed mixture-of-experts decode layer.

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import this module. The
product path (``libmoedec`` and its Python binding) never imports, calls or
links it, and this module imports nothing from the product path.

Everything here is a plain, slow, fp64 restatement of what the pages define.
Inputs are exact in fp64 (bf16 -> fp64 and int4 code x bf16 scale are exact),
so the only rounding is fp64 summation order. Library primitives used as
steps: numpy ``@`` (a matrix-vector product), ``np.exp``, ``np.unique``.

Pages cited (titles as printed):
  [MoE-arith]  "Mixture of Experts Changes the Arithmetic"
               (creativeworksofknowledge, llm-physics/experts; English and
               Korean editions), sections "Two Numbers Instead of One",
               "What the Runtime Does With the Promise", "Code: moe_promise.py".
  [Reader]     jaehun.me review of arXiv:2610.37386, the channel "reader" for
               routed experts: "배경: 채널과 유지 규칙" (channels and keep
               rules, Fig. 2), "가중치만으로 만든 reader" (steps 1-3, eq. 1,
               eq. 2), Table 3 (model shapes), Table 7 (DRAM MB per layer).
  [MoE-intro]  "MoE 입문: 36B 모델이 27B보다 6배 빨랐던 이유" (duolabs),
               sections "MoE는 일부만 부릅니다", "누가 8명을 고르나요".
  [Beam]       "5,010억 개 중 230억 개만 켠다 — 4.6% 의 산수" (mna-game
               blog), §2 "핵심 개념" (active ratio, touched-expert formula,
               memory table, "둘째 식 — 배치의 함정"), §3 [A] and [B].

Readings where the pages are silent:
  * phi is SiLU (the layer is a SwiGLU MLP; [Reader] only writes phi).
  * routing = softmax over all E logits, top-k by logit (descending, ties to
    the lowest expert index), weights renormalised over the chosen k.
  * the top-k decision is taken on the logits rounded to fp32, the
    precision the GPU path decides in; weights use the fp64 logits.
  * the shared expert is added with weight 1 (no gate is described).
  * the stack residual is x_next = bf16_rne(x + y), no attention; with the
    pre-norm option each layer's MoE input is u = bf16_rne(x / rms(x)),
    rms(x) = sqrt(mean(x^2) + 1e-6), unit norm weight (without it a stack of
    N(0, 0.02) SwiGLU layers grows without bound: see rmsnorm_bf16).
  * int4: two's-complement nibbles, element 2i in the low nibble, symmetric
    (zero point 0), value = q * s with one bf16 scale per 64 consecutive
    input elements.
"""

from __future__ import annotations

import math
from typing import Callable, Iterable, Sequence

import numpy as np

# ----------------------------------------------------------------------------
# bf16 encoding (definition: the upper 16 bits of an IEEE-754 binary32).
# ----------------------------------------------------------------------------


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode raw bf16 bit patterns (uint16 or int16 views) exactly to fp64."""
    u = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def f64_to_bf16_bits_rne(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (8 significant bits), nearest-even, return bits.

    For x = m * 2**e with m in [0.5, 1) the bf16 quantum is 2**(e-8) (for
    normal bf16 numbers; below the smallest normal exponent the quantum stays
    at 2**-133). ``np.rint`` rounds halves to even. The rounded value is
    exactly representable in binary32, whose upper half is the bf16 pattern.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros(x.shape, dtype=np.float64)
    nz = x != 0
    _, e = np.frexp(x[nz])
    quantum = np.ldexp(1.0, np.maximum(e, -125) - 8)
    out[nz] = np.rint(x[nz] / quantum) * quantum
    f32 = out.astype(np.float32)  # exact: out has <= 8 significant bits
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp64 -> nearest-even bf16 value, returned as fp64."""
    return bf16_bits_to_f64(f64_to_bf16_bits_rne(x))


# ----------------------------------------------------------------------------
# int4 group-64 symmetric codes.
# ----------------------------------------------------------------------------

INT4_GROUP = 64


def int4_unpack(packed: np.ndarray) -> np.ndarray:
    """Unpack two's-complement nibbles: byte i holds element 2i (low nibble)
    and element 2i+1 (high nibble). Returns int64 codes in [-8, 7] with the
    last axis doubled."""
    p = np.asarray(packed).astype(np.uint8)
    lo = (p & 0x0F).astype(np.int64)
    hi = ((p >> 4) & 0x0F).astype(np.int64)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.int64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def dequant_rows_int4(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Gate/up rows: codes [I, H/2] bytes, scales [I, H/64] -> fp64 [I, H].

    Group of 64 along the input dimension H: w[i, h] = q[i, h] * s[i, h // 64].
    """
    q = int4_unpack(packed).astype(np.float64)
    s = np.repeat(np.asarray(scales, dtype=np.float64), INT4_GROUP, axis=1)
    return q * s


def dequant_down_t_int4(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Transposed down projection: codes [I, H/2], scales [I/64, H] -> [I, H].

    Row j of D^T is column j of D (input channel j of the down projection), so
    the group of 64 runs along I: w[j, h] = q[j, h] * s[j // 64, h].
    """
    q = int4_unpack(packed).astype(np.float64)
    s = np.repeat(np.asarray(scales, dtype=np.float64), INT4_GROUP, axis=0)
    return q * s


# ----------------------------------------------------------------------------
# Router: GEMV, softmax, top-k, renormalise.
# [MoE-intro] "누가 8명을 고르나요" (a learned router picks the experts per
# layer); [Beam] §2 (each token turns on k of E experts); [MoE-arith] "Two
# Numbers Instead of One" (8 of 256 in the A3B model).
# ----------------------------------------------------------------------------


def silu(z: np.ndarray) -> np.ndarray:
    """phi(z) = z * sigmoid(z) = z / (1 + exp(-z)) (SwiGLU gate reading)."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def router_logits(x: np.ndarray, router: np.ndarray) -> np.ndarray:
    """logits[e] = sum_h W_r[e, h] x[h]; x [H], router [E, H]."""
    return np.asarray(router, dtype=np.float64) @ np.asarray(x, dtype=np.float64)


def softmax(logits: np.ndarray) -> np.ndarray:
    """Softmax over all entries, with max-subtraction."""
    l = np.asarray(logits, dtype=np.float64)
    z = np.exp(l - l.max())
    return z / z.sum()


def topk_order(keys: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest keys, descending; equal keys -> lower index first."""
    keys = np.asarray(keys)
    order = sorted(range(len(keys)), key=lambda i: (-keys[i], i))
    return np.array(order[:k], dtype=np.int64)


def route_topk(x: np.ndarray, router: np.ndarray, k: int):
    """One token's routing. Returns (ids [k], w [k], logits fp64 [E], margin).

    ids: top-k experts by logit, the decision taken on fp32(logit) with ties to
    the lowest index. w_i = p[ids_i] / sum_{j in ids} p[j] with p the softmax
    over all E fp64 logits. margin = l_(k) - l_(k+1) of the fp64 logits in the
    chosen order (+inf when k == E).
    """
    logits = router_logits(x, router)
    E = logits.shape[0]
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    dec = logits.astype(np.float32).astype(np.float64)
    ids = topk_order(dec, k)
    p = softmax(logits)
    w = p[ids] / p[ids].sum()
    if k < E:
        rest = np.array([i for i in range(E) if i not in set(ids.tolist())])
        margin = float(logits[ids[-1]] - logits[rest].max())
    else:
        margin = math.inf
    return ids, w, logits, margin


def tie_positions(logits: np.ndarray, ids: np.ndarray, tol: float = 1e-5) -> set:
    """Positions i of the chosen list that a near-tie may legitimately change.

    Position i is flagged if the fp64 logit of ids[i] lies within ``tol`` of
    another expert's logit that ranks next to it (its neighbour in the sorted
    order, including the first unchosen expert at the k/(k+1) boundary).
    """
    l = np.asarray(logits, dtype=np.float64)
    full = topk_order(l, len(l))
    rank = {int(e): r for r, e in enumerate(full)}
    flagged = set()
    for i, e in enumerate(np.asarray(ids).tolist()):
        r = rank[int(e)]
        for rr in (r - 1, r + 1):
            if 0 <= rr < len(full) and abs(l[full[rr]] - l[e]) < tol:
                flagged.add(i)
    return flagged


# ----------------------------------------------------------------------------
# Experts.
# [Reader] "배경: 채널과 유지 규칙": channel j owns row j of the gate G_e, row
# j of the up V_e and column j of the down D_e; a_j = phi(g_j.x) (v_j.x); the
# routed output is the router-weighted sum of a_j d_j.
# ----------------------------------------------------------------------------


def swiglu_expert(x: np.ndarray, G: np.ndarray, V: np.ndarray, Dt: np.ndarray) -> np.ndarray:
    """E(x) = D (phi(G x) * (V x)); G, V [I, H]; Dt = D^T stored [I, H].

    D h = sum_j h_j D[:, j] = sum_j h_j Dt[j, :] = Dt^T h.
    """
    a = silu(G @ x) * (V @ x)
    return Dt.T @ a


def channel_activations(x, G, V) -> np.ndarray:
    """a_j = phi(g_j^T x) (v_j^T x) for every channel j (vector [I])."""
    return silu(G @ x) * (V @ x)


ExpertFn = Callable[[int], tuple]


def moe_layer(x: np.ndarray, router: np.ndarray, experts: ExpertFn, k: int,
              shared: tuple | None = None):
    """One token through one routed MoE layer.

    experts(e) -> (G_e, V_e, Dt_e) as fp64 [I, H]. shared = (G, V, Dt) or None.
    y = sum_i w_i E_{ids_i}(x) + E_shared(x). Returns (y, ids, w, logits, margin).
    """
    ids, w, logits, margin = route_topk(x, router, k)
    y = np.zeros_like(np.asarray(x, dtype=np.float64))
    for wi, e in zip(w, ids):
        y += wi * swiglu_expert(x, *experts(int(e)))
    if shared is not None:
        y += swiglu_expert(x, *shared)
    return y, ids, w, logits, margin


def moe_experts_given(x: np.ndarray, experts: ExpertFn, ids: Sequence[int],
                      w: Sequence[float]) -> np.ndarray:
    """y = sum_i w_i E_{ids_i}(x) with the routing supplied (no router/shared)."""
    y = np.zeros_like(np.asarray(x, dtype=np.float64))
    for wi, e in zip(w, ids):
        y += float(wi) * swiglu_expert(x, *experts(int(e)))
    return y


def dense_mixture(x, router, experts: ExpertFn, E: int) -> np.ndarray:
    """Softmax-weighted sum over all E experts (no selection)."""
    p = softmax(router_logits(x, router))
    y = np.zeros_like(np.asarray(x, dtype=np.float64))
    for e in range(E):
        y += p[e] * swiglu_expert(x, *experts(e))
    return y


RMS_EPS = 1e-6


def rmsnorm_bf16(x: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    """Pre-norm MoE input u = bf16_rne(x / sqrt(mean(x^2) + eps)), unit weight.

    The pages give only the depth of the decode stack ([MoE-intro], 40
    blocks), not the block internals. Transformer blocks normalise the hidden
    state before the feed-forward layer; without it, a residual stack of
    random N(0, 0.02) SwiGLU experts at hidden 2048 grows roughly
    quadratically per layer and overflows fp32 after about 25 layers.
    """
    x = np.asarray(x, dtype=np.float64)
    return bf16_round(x / np.sqrt(np.mean(x * x) + eps))


def stack_layer(x: np.ndarray, router: np.ndarray, experts: ExpertFn, k: int,
                shared: tuple | None = None, pre_norm: bool = True):
    """One layer of the attention-free decode stack.

    u = rmsnorm_bf16(x) (or x without the pre-norm); y = MoE(u);
    x_next = bf16_rne(x + y). Returns (x_next, y, ids, w, logits, margin).
    """
    u = rmsnorm_bf16(x) if pre_norm else np.asarray(x, dtype=np.float64)
    y, ids, w, logits, margin = moe_layer(u, router, experts, k, shared)
    return residual_bf16(x, y), y, ids, w, logits, margin


def residual_bf16(x: np.ndarray, y: np.ndarray) -> np.ndarray:
    """x_next = bf16_rne(x + y) (attention-free residual stack reading)."""
    return bf16_round(np.asarray(x, dtype=np.float64) + np.asarray(y, dtype=np.float64))


def linear_experts(x: np.ndarray, weight: Callable[[int], np.ndarray],
                   ids: Sequence[int], w: Sequence[float]) -> np.ndarray:
    """Experts that are one square bf16 matrix each ([Beam] §3 [A]/[B]).

    y = sum_i w_i W_{ids_i} x with W_e [H_out, H_in].
    """
    y = None
    for wi, e in zip(w, ids):
        t = float(wi) * (weight(int(e)) @ x)
        y = t if y is None else y + t
    return y


# ----------------------------------------------------------------------------
# Touched experts at batch B.
# [Beam] §2: active ratio k/E; touched experts ~ E[1 - (1 - k/E)^B];
# "둘째 식 — 배치의 함정" worked example; §3 [B] measured vs theory.
# ----------------------------------------------------------------------------


def expected_touched(E: int, k: int, B: int) -> float:
    """E[|union of B tokens' expert sets|] when each token's k distinct ids are
    uniform: an expert is missed by one token with prob 1 - k/E, by all B
    independent tokens with prob (1 - k/E)^B."""
    return E * (1.0 - (1.0 - k / E) ** B)


def half_touch_batch_exact(E: int, k: int) -> float:
    """B at which P(an expert is touched) = 1/2: (1-k/E)^B = 1/2."""
    return math.log(0.5) / math.log(1.0 - k / E)


def half_touch_batch_small_p(E: int, k: int) -> float:
    """The small-k/E approximation ln 2 / (k/E) that [Beam] §3 [B] prints."""
    return math.log(2.0) / (k / E)


def touched_experts(ids: np.ndarray, E: int):
    """Stable counting sort of (token, slot) pairs by expert.

    ids [B, k]. Returns (count, bitmap [ceil(E/32)] uint32, offsets [E+1],
    pairs [B*k]) where pairs[offsets[e]:offsets[e+1]] lists the pair indices
    b*k + s with ids[b, s] == e in ascending order.
    """
    ids = np.asarray(ids, dtype=np.int64)
    B, k = ids.shape
    buckets = [[] for _ in range(E)]
    for b in range(B):
        for s in range(k):
            buckets[int(ids[b, s])].append(b * k + s)
    offsets = [0]
    pairs = []
    for e in range(E):
        pairs.extend(buckets[e])
        offsets.append(len(pairs))
    touched = [e for e in range(E) if buckets[e]]
    bitmap = np.zeros((E + 31) // 32, dtype=np.uint32)
    for e in touched:
        bitmap[e // 32] |= np.uint32(1 << (e % 32))
    return (len(touched), bitmap, np.array(offsets, dtype=np.int64),
            np.array(pairs, dtype=np.int64))


# ----------------------------------------------------------------------------
# Channel-sparse (top-k keep rule) and 32-byte sector accounting.
# [Reader] keep-rule table (top-k keeps exactly k channels per token); step 2
# (one top-k across all of the token's routed experts); Fig. 2(c) and its
# small table (bytes are charged per touched 32-byte sector); the down
# projection is transposed at load so a channel's down column is contiguous.
# ----------------------------------------------------------------------------

SECTOR_BYTES = 32


def channel_topk_select(scores: np.ndarray, ids: Sequence[int], keep: int) -> np.ndarray:
    """Kept candidates for one token.

    scores [E, I]; candidates are (e, c) for e in ids, with index e*I + c.
    Keep the ``keep`` largest scores, ties to the lowest index. Returned in
    ascending index order (the set is what the rule defines).
    """
    scores = np.asarray(scores)
    E, I = scores.shape
    cand = [(float(scores[e, c]), int(e) * I + c) for e in ids for c in range(I)]
    if not 0 <= keep <= len(cand):
        raise ValueError("keep out of range")
    cand.sort(key=lambda t: (-t[0], t[1]))
    return np.array(sorted(idx for _, idx in cand[:keep]), dtype=np.int64)


def channel_sparse_forward(x: np.ndarray, channel: Callable[[int, int], np.ndarray],
                           ids: Sequence[int], w: Sequence[float], kept: Iterable[int],
                           I: int) -> np.ndarray:
    """y = sum over kept j = (e, c) of w_e a_{e,c} d_{e,c}; dropped channels add 0.

    channel(e, c) -> [3, H] fp64 rows (gate row, up row, down column).
    """
    wmap = {int(e): float(wi) for e, wi in zip(ids, w)}
    y = None
    for j in kept:
        e, c = divmod(int(j), I)
        g, v, d = channel(e, c)
        a = silu(np.dot(g, x)) * np.dot(v, x)
        t = wmap[e] * a * d
        y = t if y is None else y + t
    if y is None:
        y = np.zeros_like(np.asarray(x, dtype=np.float64))
    return y


def channel_stack_layer(x: np.ndarray, router: np.ndarray, channel: Callable[[int, int], np.ndarray],
                        scores: np.ndarray, k: int, keep: int, I: int, pre_norm: bool = True):
    """One layer of the channel-sparse decode stack: u = rmsnorm_bf16(x) (or
    x), routing of u, the `keep` best channels of the routed experts by the
    given scores [E, I], y from the kept channels only, x_next = bf16(x + y).
    Returns (x_next, y, ids, w, logits, kept)."""
    u = rmsnorm_bf16(x) if pre_norm else np.asarray(x, dtype=np.float64)
    ids, w, logits, _ = route_topk(u, router, k)
    kept = channel_topk_select(scores, ids, keep)
    y = channel_sparse_forward(u, channel, ids, w, kept, I)
    return residual_bf16(x, y), y, ids, w, logits, kept


def channel_union(kept_lists: Iterable[Iterable[int]]) -> np.ndarray:
    """Channels a batch reads once: the union of every token's kept channel
    indices e*I + c, ascending ([Reader] "속도": at batch > 1 the tokens' kept
    channels are read as their union, which grows with the batch)."""
    parts = [np.asarray(list(k), dtype=np.int64) for k in kept_lists]
    parts = [q for q in parts if q.size]
    if not parts:
        return np.zeros(0, dtype=np.int64)
    return np.unique(np.concatenate(parts))


def sectors_touched(ranges: Iterable[tuple]) -> int:
    """Distinct 32-byte sectors covering the half-open byte ranges [lo, hi).

    Brute force: the union of every range's sector indices byte//32.
    """
    parts = [np.arange(lo // SECTOR_BYTES, (hi - 1) // SECTOR_BYTES + 1, dtype=np.int64)
             for lo, hi in ranges if hi > lo]
    if not parts:
        return 0
    return int(np.unique(np.concatenate(parts)).size)


def channel_major_ranges(kept: Iterable[int], H: int, base: int = 0, elem_bytes: int = 2):
    """Byte ranges read for kept channels of channel-major storage [E][I][3][H].

    Channel index j = e*I + c occupies [base + j*3*H*b, base + (j+1)*3*H*b).
    """
    step = 3 * H * elem_bytes
    return [(base + int(j) * step, base + (int(j) + 1) * step) for j in kept]


# ----------------------------------------------------------------------------
# Weight-only channel screen. [Reader] "가중치만으로 만든 reader":
#   step 1 ("삼원 스케치로 선별한다"): the gate row g_j and up row v_j are
#   rotated in blocks of 128 coordinates by a random Hadamard transform R
#   (orthogonal, so g^T x = (R g)^T (R x)); each rotated block is stored as
#   ternary codes in {-1, 0, 1}, one fp16 scale and rho_b, the block's mean
#   squared quantisation error. At decode time x is rotated once and the
#   sketch gives g_hat ~ g^T x and v_hat ~ v^T x.
#   step 2 ("출력 단위 점수로 상위 k개를 정확히 계산한다", eq. 1): the score
#   of channel j is s_j = w_j ||d_j|| |phi(g_hat_j) v_hat_j|, with w_j the
#   router weight of its expert and ||d_j|| the norm of its down column,
#   computed once at load; one top-k runs across all routed experts.
# Readings where the page is silent:
#   * R = H_128 diag(s) / sqrt(128) per block: H_128 the Sylvester Hadamard
#     matrix, s a given vector of H random signs (an input). Both sides work
#     with the unnormalised u = H_128 (s * v); (R g)^T (R x) = u_g^T u_x / 128.
#   * the ternary code of a block is the ternary-weight-network rule (Li and
#     Liu, 2016): threshold delta = 0.7 * mean|u|, code = sign(u) where
#     |u| > delta, else 0; scale = mean of |u| over the nonzero codes, stored
#     as fp16 (rounded through fp32, both round-to-nearest-even).
#   * rho_b = mean over the block of ((u - scale * code) / sqrt(128))^2, the
#     error in the orthonormal rotation's units, with the stored scale.
# For bf16 rows whose block values span less than 2^38 in magnitude, u, the
# sum of |u| and the code decisions are exact in fp64, so any exact
# implementation (matrix product or butterfly) gives the same codes.
# ----------------------------------------------------------------------------

READER_BLOCK = 128
TWN_THRESHOLD = 0.7


def sylvester_hadamard(n: int) -> np.ndarray:
    """H_1 = [1]; H_2m = [[H_m, H_m], [H_m, -H_m]] (entries +-1, unnormalised)."""
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    if h.shape[0] != n:
        raise ValueError("n must be a power of two")
    return h


def reader_rotate(v: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """u = H_128 (s * v) on each block of 128 coordinates (unnormalised)."""
    v = np.asarray(v, dtype=np.float64)
    hm = sylvester_hadamard(READER_BLOCK)
    blocks = (np.asarray(signs, dtype=np.float64) * v).reshape(-1, READER_BLOCK)
    return (blocks @ hm.T).reshape(-1)


def fp16_through_fp32(a: float) -> float:
    """fp64 -> fp32 -> fp16, each round-to-nearest-even; returned as fp64."""
    return float(np.float16(np.float32(a)))


def ternary_block(u: np.ndarray):
    """One rotated block -> (codes int8 [128], fp16 scale, rho)."""
    u = np.asarray(u, dtype=np.float64)
    a = np.abs(u)
    delta = TWN_THRESHOLD * (a.sum() / READER_BLOCK)
    nz = a > delta
    codes = np.where(nz, np.sign(u), 0.0).astype(np.int8)
    n = int(nz.sum())
    scale = fp16_through_fp32(a[nz].sum() / n) if n else 0.0
    rho = float(np.mean(((u - scale * codes) / math.sqrt(READER_BLOCK)) ** 2))
    return codes, scale, rho


def reader_sketch_row(v: np.ndarray, signs: np.ndarray):
    """Sketch of one row: codes int8 [H], scales [H/128], rho [H/128]."""
    u = reader_rotate(v, signs)
    parts = [ternary_block(b) for b in u.reshape(-1, READER_BLOCK)]
    codes = np.concatenate([p[0] for p in parts])
    return codes, np.array([p[1] for p in parts]), np.array([p[2] for p in parts])


def reader_estimate(x: np.ndarray, codes: np.ndarray, scales: np.ndarray, signs: np.ndarray) -> float:
    """Sketch estimate of v^T x: sum over blocks of scale_b codes_b . u_x,b / 128."""
    ux = reader_rotate(x, signs).reshape(-1, READER_BLOCK)
    c = np.asarray(codes, dtype=np.float64).reshape(-1, READER_BLOCK)
    return float(np.sum(np.asarray(scales, dtype=np.float64) * np.sum(c * ux, axis=1)) / READER_BLOCK)


def reader_estimate_bound(x: np.ndarray, codes: np.ndarray, scales: np.ndarray) -> float:
    """sum_b scale_b * (number of nonzero codes in b) * sum_{i in b} |x_i| / 128:
    a bound on every |partial sum| of the estimate (each |u_x,i| <= sum_b |x|)."""
    xa = np.abs(np.asarray(x, dtype=np.float64)).reshape(-1, READER_BLOCK).sum(axis=1)
    nzc = (np.asarray(codes).reshape(-1, READER_BLOCK) != 0).sum(axis=1)
    return float(np.sum(np.abs(np.asarray(scales, dtype=np.float64)) * nzc * xa) / READER_BLOCK)


def reader_score(w_e: float, dnorm: float, g_hat: float, v_hat: float) -> float:
    """Eq. 1: s = w_e ||d|| |phi(g_hat) v_hat|, phi = SiLU."""
    return float(w_e * dnorm * abs(silu(np.float64(g_hat)) * v_hat))


def reader_screen(x: np.ndarray, ids: Sequence[int], w: Sequence[float], sketch, I: int, signs: np.ndarray):
    """Scores [len(ids), I] and estimates [len(ids), I, 2] of the routed
    experts' channels. sketch(e, c) -> (codes_g, scales_g, codes_v, scales_v,
    dnorm)."""
    k = len(ids)
    scores = np.zeros((k, I))
    est = np.zeros((k, I, 2))
    for t, e in enumerate(ids):
        for c in range(I):
            cg, sg, cv, sv, dn = sketch(int(e), c)
            gh = reader_estimate(x, cg, sg, signs)
            vh = reader_estimate(x, cv, sv, signs)
            est[t, c] = (gh, vh)
            scores[t, c] = reader_score(float(w[t]), dn, gh, vh)
    return scores, est


# ----------------------------------------------------------------------------
# Partial screen and recovery of dropped channels. [Reader] "가중치만으로 만든
# reader": step 1's partial scan (at low budgets only the ternary codes of
# the 80 coordinates with the largest |Rx| in each block are read) and step 3
# ("버린 채널을 rank-32 맵으로 복구한다", eq. 2): U = the top 32 left singular
# vectors of the layer's stacked down columns, b_j = U^T d_j per channel, and
#   y_hat = sum_{j in K} w_j d_j a_j + U sum_{j in S} w_j b_j p_j,
# K the kept channels (exact a_j), S the dropped ones with the screen's
# estimate p_j = phi(g_hat_j) v_hat_j.
# Readings: ties in |Rx| go to the lower coordinate; "all down columns of the
# layer" are the E*I columns d_{e,c} of every expert.
# ----------------------------------------------------------------------------

PARTIAL_COORDS = 80
RECOVERY_RANK = 32


def reader_partial_mask(x: np.ndarray, signs: np.ndarray, m: int = PARTIAL_COORDS) -> np.ndarray:
    """Boolean [H]: in each block, the m coordinates with the largest |u_x|
    (u_x = H_128 (s * x), the same order as |R x|), ties to the lower index."""
    ux = np.abs(reader_rotate(x, signs)).reshape(-1, READER_BLOCK)
    mask = np.zeros_like(ux, dtype=bool)
    for b in range(ux.shape[0]):
        order = sorted(range(READER_BLOCK), key=lambda i: (-ux[b, i], i))
        mask[b, order[:m]] = True
    return mask.reshape(-1)


def reader_estimate_partial(x: np.ndarray, codes: np.ndarray, scales: np.ndarray, signs: np.ndarray,
                            m: int = PARTIAL_COORDS) -> float:
    """The estimate of reader_estimate over the masked coordinates only."""
    keep = reader_partial_mask(x, signs, m)
    c = np.where(keep, np.asarray(codes, dtype=np.float64), 0.0)
    return reader_estimate(x, c, scales, signs)


def recovery_basis(down_cols: np.ndarray, rank: int = RECOVERY_RANK) -> np.ndarray:
    """U [H, rank]: the top `rank` left singular vectors of D = [d_1 ... d_n]
    (down_cols [n, H], one down column per row), by the library SVD."""
    u, _, _ = np.linalg.svd(np.asarray(down_cols, dtype=np.float64).T, full_matrices=False)
    return u[:, :rank]


def recovery_coeffs(U: np.ndarray, d: np.ndarray) -> np.ndarray:
    """b_j = U^T d_j."""
    return np.asarray(U).T @ np.asarray(d, dtype=np.float64)


def reader_output(kept_terms: Iterable[tuple], dropped_terms: Iterable[tuple], U: np.ndarray) -> np.ndarray:
    """Eq. 2. kept_terms: (w_j, a_j, d_j) of the kept channels; dropped_terms:
    (w_j, p_j, b_j) of the dropped ones."""
    H = U.shape[0]
    y = np.zeros(H)
    for wj, aj, dj in kept_terms:
        y = y + wj * aj * np.asarray(dj, dtype=np.float64)
    r = np.zeros(U.shape[1])
    for wj, pj, bj in dropped_terms:
        r = r + wj * pj * np.asarray(bj, dtype=np.float64)
    return y + U @ r


# ----------------------------------------------------------------------------
# Bytes-per-token accounting and decode ceiling.
# [MoE-arith] "Two Numbers Instead of One" / moe_promise.py: ceiling =
# achieved bandwidth / bytes per token. [Beam] §2 memory table: resident =
# total params x bytes/param; per token = active params x bytes/param.
# ----------------------------------------------------------------------------


def decode_ceiling(bandwidth_gbs: float, gb_per_token: float) -> float:
    return bandwidth_gbs / gb_per_token


def param_bytes(n_params: float, bits: float) -> float:
    return n_params * bits / 8.0


def swiglu_expert_bytes(H: int, I: int, wtype: str = "bf16") -> int:
    """Bytes of one SwiGLU expert (G, V and D), bf16 or int4-group-64."""
    if wtype == "bf16":
        return 3 * I * H * 2
    if wtype == "int4":
        codes = 3 * I * H // 2
        scales = (I * (H // INT4_GROUP) * 2) * 2 + (I // INT4_GROUP) * H * 2
        return codes + scales
    raise ValueError(wtype)


def layer_bytes_b1(H: int, E: int, I: int, k: int, I_shared: int = 0,
                   wtype: str = "bf16", router: bool = True) -> int:
    """Algorithmic bytes one batch-1 token must read in one layer: router +
    k routed experts + the shared expert (bf16)."""
    b = k * swiglu_expert_bytes(H, I, wtype)
    if I_shared:
        b += swiglu_expert_bytes(H, I_shared, "bf16")
    if router:
        b += E * H * 2
    return b
