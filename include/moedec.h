/*
 * libmoedec -- routed mixture-of-experts feed-forward layer at decode time,
 * for NVIDIA B200 (sm_100a). Plain C ABI: device pointers, sizes, a CUDA
 * stream; no C++ or framework types cross this boundary.
 *
 * The operation (pages cited by title and section):
 *  - Router: logits = W_r x over E experts, softmax, top-k; a learned router
 *    picks k experts per token and layer ("MoE 입문: 36B 모델이 27B보다 6배
 *    빨랐던 이유", section "누가 8명을 고르나요"; "Mixture of Experts Changes
 *    the Arithmetic", "Two Numbers Instead of One": 8 of 256).
 *  - Expert = gated MLP. Channel j owns row j of the gate G_e, row j of the
 *    up V_e and column j of the down D_e; a_j = phi(g_j.x)(v_j.x); the routed
 *    output is the router-weighted sum of a_j d_j (review of arXiv:2610.37386,
 *    "배경: 채널과 유지 규칙"). phi = SiLU (SwiGLU).
 *  - Optional always-on shared expert ("Mixture of Experts Changes the
 *    Arithmetic", checkpoint table: "256, 8 (+1 shared)").
 *  - Channel-sparse top-k keep rule with 32-byte sector charging (same review,
 *    keep-rule table, Fig. 2(c), and "2단계": one top-k across all of the
 *    token's routed experts; down projection stored transposed).
 *  - Touched experts at batch B ~ E[1-(1-k/E)^B] ("5,010억 개 중 230억 개만
 *    켠다 — 4.6% 의 산수", §2 핵심 개념 and "둘째 식 — 배치의 함정").
 *
 * Conventions for every call:
 *  - Pointers named x, y, ids, w, ... and every weight pointer are CUDA DEVICE
 *    pointers owned by the caller; the library never allocates or frees
 *    device memory. Descriptor structs (moe_layer_desc) live in HOST memory
 *    and are read during the call only.
 *  - Every device pointer must be 16-byte aligned.
 *  - Calls are asynchronous on `stream` (NULL = the legacy default stream).
 *    Outputs are valid after the stream is synchronised.
 *  - Host-side argument errors return MOE_ERR_INVALID / MOE_ERR_UNSUPPORTED
 *    before anything is launched. CUDA launch errors return MOE_ERR_CUDA.
 *    Errors found on the device (a wait that ran out of its time budget,
 *    expert ids out of range or repeated) are written to the workspace
 *    status word and read with moe_get_status(); kernels never trap.
 *  - A workspace is owned by one stream at a time: calls that share a
 *    workspace must not run concurrently.
 *  - bf16 is IEEE binary32's upper half; int32/float are 4 bytes.
 *
 * Layouts (row-major, innermost dimension last):
 *  - x: [B, H] bf16.  y: [B, H] fp32 (overwritten).
 *  - router: [E, H] bf16.
 *  - PLANAR bf16 experts: gate, up, down_t each [E, I, H]; down_t[e, j, :] is
 *    column j of D_e (the down projection stored transposed).
 *  - PLANAR int4 (MOE_W_INT4_G64) experts: codes packed two per byte, element
 *    2i in the low nibble, two's complement in [-8, 7], value = q * s with one
 *    bf16 scale per 64 consecutive INPUT elements:
 *      gate/up codes [E, I, H/2] u8, gate_s/up_s [E, I, H/64] bf16;
 *      down_t codes [E, I, H/2] u8, down_s [E, I/64, H] bf16 (the down
 *      projection's input is the channel index j, so its groups run along I).
 *  - CHANNEL_MAJOR bf16 experts: gate = [E, I, 3, H]: for channel (e, c) the
 *    gate row, up row and down column are contiguous (3*H*2 bytes); up and
 *    down_t are NULL.
 *  - LINEAR experts: gate = [E, H, H] (one H x H matrix per expert, output
 *    row-major); E_e(x) = W_e x.
 *  - Shared expert (SwiGLU, bf16, PLANAR): sh_gate, sh_up, sh_down_t each
 *    [I_shared, H]; all NULL / I_shared = 0 for none.
 */
#ifndef MOEDEC_H
#define MOEDEC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOEDEC_ABI_VERSION 2

typedef struct CUstream_st* moe_stream_t; /* a cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID = 1,     /* bad argument, or invalid expert ids found on the device */
  MOE_ERR_UNSUPPORTED = 2, /* valid but outside what this build implements */
  MOE_ERR_CUDA = 3,        /* a CUDA runtime call failed */
  MOE_ERR_TIMEOUT = 4      /* a device-side wait ran out of its time budget */
} moe_status;

typedef enum { MOE_W_BF16 = 0, MOE_W_INT4_G64 = 1 } moe_wtype;
typedef enum { MOE_EXPERT_SWIGLU = 0, MOE_EXPERT_LINEAR = 1 } moe_ekind;
typedef enum { MOE_LAYOUT_PLANAR = 0, MOE_LAYOUT_CHANNEL_MAJOR = 1 } moe_layout;

/* One MoE layer's shape and weights (host struct, device pointers). */
typedef struct {
  int32_t H;      /* hidden size; multiple of 64 (of 512 for int4)           */
  int32_t E;      /* routed experts, 1..1024                                   */
  int32_t I;      /* expert intermediate size (channels), 1..65536; multiple of 64 for int4 */
  int32_t k;      /* experts per token, 1..min(E, 32)                          */
  int32_t kind;   /* moe_ekind                                                 */
  int32_t wtype;  /* moe_wtype                                                 */
  int32_t layout; /* moe_layout                                                */
  int32_t I_shared; /* shared-expert intermediate size, 0..65536, 0 = none   */
  const void* router;          /* [E, H] bf16; may be NULL when ids are given */
  const void* gate;            /* see Layouts above                           */
  const void* up;
  const void* down_t;
  const void* gate_s;          /* int4 scales, else NULL                      */
  const void* up_s;
  const void* down_s;
  const void* sh_gate;         /* shared expert, bf16 [I_shared, H] each      */
  const void* sh_up;
  const void* sh_down_t;
} moe_layer_desc;

/* ABI version compiled into the library (MOEDEC_ABI_VERSION). */
int moe_abi_version(void);

/* Text for a status code (static storage, never NULL). */
const char* moe_status_string(moe_status s);

/* Bytes of device workspace needed by any call below on layers of this shape
 * at batch B (B tokens decoded together). 0 if the descriptor or B is
 * invalid. The caller allocates it (16-byte aligned) and must clear it once
 * with moe_workspace_init() before the first call. */
size_t moe_workspace_bytes(const moe_layer_desc* desc, int32_t B);

/* Clear a workspace (status word, barrier counters): once after allocation,
 * and again after any call reported MOE_ERR_TIMEOUT. Asynchronous on stream. */
moe_status moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream);

/* Read (and keep) the device status word of a workspace. Synchronises
 * `stream`. Returns MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_INVALID (bad ids). */
moe_status moe_get_status(const void* ws, moe_stream_t stream);

/* Time budget of every device-side wait of later calls on this workspace, in
 * SM clock cycles (a wait that runs out ends the call with MOE_ERR_TIMEOUT in
 * the status word; the kernels then drain their copies in flight and return).
 * 0 restores the default of 2e9 cycles (about 1 s). moe_workspace_init()
 * also restores it. Asynchronous on stream; returns MOE_ERR_INVALID for a
 * NULL or misaligned workspace. */
moe_status moe_workspace_set_wait_budget(void* ws, unsigned long long cycles, moe_stream_t stream);

/* Fault injection for tests of the timeout path. With
 * MOE_INJECT_BARRIER_EXTRA_ARRIVAL set, every grid-wide barrier of later
 * calls on this workspace waits for one arrival more than the grid makes, so
 * the wait runs out after the workspace's budget and the call reports
 * MOE_ERR_TIMEOUT (no GPU fault is involved). 0 clears it, and so does
 * moe_workspace_init(). Asynchronous on stream; unknown bits are rejected
 * with MOE_ERR_INVALID. */
#define MOE_INJECT_BARRIER_EXTRA_ARRIVAL 1u
moe_status moe_workspace_set_inject(void* ws, uint32_t flags, moe_stream_t stream);

/* Router only: for each token b, logits = router @ x[b] (fp32 accumulate),
 * ids[b, :] = the k experts with the largest logits in descending order,
 * ties to the lowest index; w[b, i] = softmax over all E logits restricted to
 * the chosen k and renormalised (= exp(l_i) / sum_{j chosen} exp(l_j)).
 * margin_opt[b] = (k-th largest logit) - ((k+1)-th largest), +inf if k == E.
 *   x [B, H] bf16; router [E, H] bf16; ids [B, k] int32; w [B, k] fp32;
 *   margin_opt [B] fp32 or NULL. 1 <= B <= 256, H % 64 == 0, E <= 1024. */
moe_status moe_route_topk(const void* x, const void* router, int32_t B, int32_t H,
                          int32_t E, int32_t k, int32_t* ids, float* w, float* margin_opt,
                          void* ws, size_t ws_bytes, moe_stream_t stream);

/* Routed experts only (no router, no shared expert, no residual):
 *   y[b] = sum_i w[b, i] * E_{ids[b, i]}(x[b]).
 * SWIGLU: E_e(x) = D_e (silu(G_e x) * (V_e x)); LINEAR: E_e(x) = W_e x.
 * ids [B, k] int32 (distinct per token, < E; checked on the device),
 * w [B, k] fp32, y [B, H] fp32 overwritten.
 * SWIGLU PLANAR (bf16 or int4): 1 <= B <= 8. LINEAR bf16: 1 <= B <= 256. */
moe_status moe_expert_forward(const moe_layer_desc* desc, const void* x, int32_t B,
                              const int32_t* ids, const float* w, float* y,
                              void* ws, size_t ws_bytes, moe_stream_t stream);

/* One full layer: router, top-k, routed SwiGLU experts, shared expert:
 *   y[b] = sum_i w[b,i] E_{ids[b,i]}(x[b]) + E_shared(x[b]);
 * x_next_opt [B, H] bf16 = bf16_rne(x + y) (attention-free residual) or NULL;
 * ids_out_opt [B, k], w_out_opt [B, k] or NULL. SWIGLU PLANAR, 1 <= B <= 8.
 * One persistent launch; no per-expert dispatch. */
moe_status moe_layer_forward(const moe_layer_desc* desc, const void* x, int32_t B, float* y,
                             void* x_next_opt, int32_t* ids_out_opt, float* w_out_opt,
                             void* ws, size_t ws_bytes, moe_stream_t stream);

/* Stack option: normalise each layer's MoE input, u_l = bf16_rne(x_l /
 * sqrt(mean(x_l^2) + 1e-6)) (unit weight); the residual stays x_l + y_l. */
#define MOE_STACK_PRE_RMSNORM 1u

/* L layers in one persistent launch: x_{l+1} = bf16_rne(x_l + y_l) with y_l
 * the full layer output above, computed on u_l = x_l, or on the RMS-normalised
 * x_l when flags has MOE_STACK_PRE_RMSNORM (transformer blocks normalise the
 * feed-forward input; the pages give the depth of the stack only, and without
 * a norm a stack of random N(0, 0.02) SwiGLU layers overflows fp32 within
 * ~25 layers). layers[L] share H, E, I, k, kind, wtype, layout and I_shared
 * (weights differ). x_out [B, H] bf16 = x_L.
 * Optional histories for per-layer checking (NULL to skip):
 *   x_hist [L+1, B, H] bf16 (x_0 .. x_L), y_hist [L, B, H] fp32,
 *   ids_hist [L, B, k] int32, w_hist [L, B, k] fp32.
 * 1 <= L <= 64, 1 <= B <= 8. */
moe_status moe_stack_forward(const moe_layer_desc* layers, int32_t L, const void* x, int32_t B,
                             uint32_t flags, void* x_out, void* x_hist_opt, float* y_hist_opt,
                             int32_t* ids_hist_opt, float* w_hist_opt,
                             void* ws, size_t ws_bytes, moe_stream_t stream);

/* Channel-sparse routed experts (CHANNEL_MAJOR bf16 SWIGLU): for token b the
 * candidates are the k*I channels (e, c) of its routed experts e = ids[b, :],
 * indexed e*I + c. Keep the `keep` largest scores[b, e, c] (ties to the lowest
 * index); dropped channels are not read and contribute 0:
 *   y[b] = sum_{kept (e,c)} w[b, e] a_{b,e,c} d_{e,c}
 * (review of arXiv:2610.37386, keep-rule table and "2단계"). A batch (B >= 2)
 * reads the UNION of its tokens' kept channels once, in one launch, and
 * applies each union channel to every token that kept it (same review,
 * Table 7 rows B = 4 and 8, "속도").
 *   scores [B, E, I] fp32 (only the routed rows are read);
 *   kept_opt [B, keep] int32 = each token's kept indices, ascending, or NULL;
 *   sectors [B] uint64 = distinct 32-byte sectors of routed-expert weights
 *     covered by that token's kept channels;
 *   union_count_opt [1] int32 = channels in the union (what the batch read);
 *   union_sectors_opt [1] uint64 = distinct 32-byte sectors the batch read.
 * ids distinct per token and < E (else MOE_ERR_INVALID in the status word and
 * y undefined). 0 <= keep <= k*I <= 8192, 1 <= B <= 8, H <= 2048; for B >= 2
 * also min(E, B*k) * I <= 65536 (else MOE_ERR_UNSUPPORTED). */
moe_status moe_channel_topk_forward(const moe_layer_desc* desc, const void* x, int32_t B,
                                    const int32_t* ids, const float* w, const float* scores,
                                    int32_t keep, float* y, int32_t* kept_opt,
                                    unsigned long long* sectors, int32_t* union_count_opt,
                                    unsigned long long* union_sectors_opt,
                                    void* ws, size_t ws_bytes, moe_stream_t stream);

/* One layer's channel-screen sketch (the buffers moe_reader_build writes);
 * codes 16-byte, scales and dnorm 4-byte aligned, else MOE_ERR_INVALID. */
typedef struct {
  const uint32_t* codes;   /* [E*I][2][H/16] 2-bit codes */
  const uint16_t* scales;  /* [E*I][2][H/128] fp16 bit patterns */
  const float* dnorm;      /* [E*I] down-column norms */
} moe_sketch_desc;

/* Channel-sparse decode stack (one token): per layer l, u_l = x_l (or its RMS
 * normalisation with MOE_STACK_PRE_RMSNORM), the router picks k experts of u_l
 * as in moe_route_topk, then only the `keep` best channels of those experts by
 * their scores are read and applied as in moe_channel_topk_forward;
 * x_{l+1} = bf16_rne(x_l + y_l). layers[L]: CHANNEL_MAJOR bf16 SWIGLU with a
 * router, same shape. The scores come from exactly one of:
 *   scores [L, E, I] fp32, given; or
 *   sketches [L] + signs [H]: computed in the kernel for each layer by the
 *   weight-only screen of moe_reader_screen on u_l (eq. 1 with the layer's
 *   routing weights); needs H % 128 == 0 (else MOE_ERR_UNSUPPORTED).
 * x [1, H] bf16; x_out [1, H]; optional x_hist [L+1, H], y_hist [L, H],
 * ids_hist / w_hist [L, k], kept_hist [L, keep] (ascending); sectors [L] =
 * 32-byte sectors of routed weights read per layer. 1 <= L <= 64,
 * 0 <= keep <= k*I. */
moe_status moe_channel_stack_forward(const moe_layer_desc* layers, int32_t L, const void* x, uint32_t flags,
                                     const float* scores, const moe_sketch_desc* sketches, const int8_t* signs,
                                     int32_t keep, void* x_out, void* x_hist_opt,
                                     float* y_hist_opt, int32_t* ids_hist_opt, float* w_hist_opt,
                                     int32_t* kept_hist_opt, unsigned long long* sectors,
                                     void* ws, size_t ws_bytes, moe_stream_t stream);

/* Touched experts of a batch: the union of the B tokens' expert sets.
 *   ids [B, k] int32 (distinct per token, < E); count [1] int32 = |union|;
 *   bitmap_opt [ceil(E/32)] uint32, bit e set iff expert e is touched;
 *   offsets_opt [E+1] int32 exclusive prefix sum of per-expert pair counts;
 *   pairs_opt [B*k] int32: pairs[offsets[e] .. offsets[e+1]) are the pair
 *   indices b*k + s with ids[b, s] == e, ascending (a stable counting sort).
 * 1 <= B <= 256, 1 <= k <= 32, E <= 1024. Invalid ids set count = -1. */
moe_status moe_touched_experts(const int32_t* ids, int32_t B, int32_t k, int32_t E,
                               int32_t* count, uint32_t* bitmap_opt, int32_t* offsets_opt,
                               int32_t* pairs_opt, moe_stream_t stream);

/* ---- No-allocation variant (the pages have no counterpart; it is a service
 * for callers that cannot allocate device memory) ----------------------------
 *
 * Some callers cannot call cudaMalloc (or any allocating routine) at the
 * point where they run a layer: code that records into a stream while the
 * runtime forbids allocation calls, plug-in hosts whose device memory is all
 * owned by the host's own pool, or real-time loops that must never block on
 * the allocator. moe_layer_forward_static() computes exactly what
 * moe_layer_forward() computes, but its scratch space is a fixed array inside
 * the library (MOE_STATIC_SCRATCH_BYTES per device, held by every GPU that
 * loads the library until the process exits) instead of a workspace the
 * caller passes. The caller still passes inputs and outputs.
 *
 *  - The scratch needed is moe_workspace_bytes(desc, B); a shape that needs
 *    more than MOE_STATIC_SCRATCH_BYTES is rejected with MOE_ERR_UNSUPPORTED
 *    before anything is launched.
 *  - Every call looks up the array's device address in the context current on
 *    the calling thread (a host-side lookup). The first call in a context,
 *    the first after a device reset included, may load the library's device
 *    code there: make that call outside any stream capture.
 *  - Every argument is checked before the array is touched: a call that
 *    returns an error launches nothing and leaves the array as it was.
 *  - All calls on a device share the one array and it keeps the previous
 *    call's contents; each call first clears the part that must start at zero
 *    (the status word and barrier counter). Calls whose executions overlap on
 *    the GPU (concurrent streams, or host threads on one device) race on the
 *    array: serialise them.
 *  - status_out_opt (device int32, or NULL) receives the call's device status
 *    (the value moe_get_status() would report) after the kernel, stream-ordered.
 *  - Nothing is allocated or freed: no cudaMalloc/cudaFree, no library routine
 *    that allocates. */
#define MOE_STATIC_SCRATCH_BYTES (256u * 1024u)
moe_status moe_layer_forward_static(const moe_layer_desc* desc, const void* x, int32_t B, float* y,
                                    void* x_next_opt, int32_t* ids_out_opt, float* w_out_opt,
                                    int32_t* status_out_opt, moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Weight-only channel screen ([Reader] "가중치만으로 만든 reader", step 1:
 * the gate and up rows of every channel are rotated in blocks of 128
 * coordinates by a random Hadamard transform and stored as ternary codes with
 * one fp16 scale and one squared error rho per block; step 2, eq. 1: a
 * channel's score is w_e ||d_j|| |SiLU(g_hat_j) v_hat_j| from the sketch
 * estimates g_hat ~ g_j.x and v_hat ~ v_j.x). The scores feed
 * moe_channel_topk_forward's `scores` input.
 *
 * Rotation: R = H_128 diag(s) / sqrt(128) per block, H_128 the Sylvester
 * Hadamard matrix, s = signs[H] (+1 or -1 as int8, chosen by the caller at
 * random once per model and shared by the builder and the screen).
 * Ternary rule per rotated block u (unnormalised, u = H_128 (s * v)):
 * delta = 0.7 * mean|u|, code = sign(u) where |u| > delta else 0, scale =
 * mean |u| over the coded coordinates rounded to fp16 (through fp32),
 * rho = mean((u - scale * code)^2) / 128. Decisions are taken in fp64.
 *
 * Layout (j = e*I + c, row r = 0 gate / 1 up):
 *   codes  [E*I][2][H/16] uint32: coordinate h of a row in word h/16, bit
 *          2(h%16) = nonzero, bit 2(h%16)+1 = negative (2 bits per code);
 *   scales [E*I][2][H/128] uint16 (fp16 bit patterns);
 *   rho    [E*I][2][H/128] fp32;
 *   dnorm  [E*I] fp32 = ||down column of channel j||.
 * All device pointers, owned by the caller; codes/scales/dnorm 4-byte
 * aligned. desc: CHANNEL_MAJOR bf16 SWIGLU with gate = [E][I][3][H];
 * H % 128 == 0 and H <= 2048, else MOE_ERR_UNSUPPORTED. */

/* Builds the sketch of every channel of one layer (once per model load). */
moe_status moe_reader_build(const moe_layer_desc* desc, const int8_t* signs, uint32_t* codes,
                            uint16_t* scales, float* rho, float* dnorm, moe_stream_t stream);

/* Screen of B tokens (1 <= B <= 256): for each token b and each of its
 * routed experts e = ids[b, slot] (w[b, slot] its router weight), writes
 * scores[b, e, c] for c < I; rows of experts token b did not route to, and
 * of ids outside [0, E), are not written. est_opt [B, k, I, 2] fp32 receives {g_hat, v_hat} (or NULL).
 * x [B, H] bf16 is the expert input (the normalised x under pre-norm).
 * Here codes must be 16-byte and scales 4-byte aligned (the screen copies
 * them with 16- and 4-byte pieces), else MOE_ERR_INVALID. */
moe_status moe_reader_screen(const moe_layer_desc* desc, const void* x, int32_t B, const int32_t* ids,
                             const float* w, const int8_t* signs, const uint32_t* codes,
                             const uint16_t* scales, const float* dnorm, float* scores, float* est_opt,
                             moe_stream_t stream);

/* Partial screen ([Reader] "가중치만으로 만든 reader", step 1, partial scan):
 * in each block of 128 rotated coordinates only the codes of the m coordinates
 * with the largest |R x_b| (ties to the lower coordinate; the page uses m =
 * 80) are read; otherwise as moe_reader_screen. It reads the codes in the
 * coordinate-major layout, where skipping a coordinate skips its bytes:
 *   codes_cmaj [E][2][H][I/16] uint32: coordinate h of row r (0 gate, 1 up) of
 *   expert e, channel c at bits 2(c%16) (nonzero) and 2(c%16)+1 (negative)
 *   of word c/16 (moe_reader_codes_coordinate_major builds it from codes).
 * Codes read per token and routed expert: 2 * (H/128) * m * (I/16) words.
 * 0 <= m <= 128, I % 16 == 0, I <= 1024, (I/16) * (H/128) <= 1024, else
 * MOE_ERR_UNSUPPORTED. est_opt [B, k, I, 2] or NULL. */
moe_status moe_reader_codes_coordinate_major(const moe_layer_desc* desc, const uint32_t* codes,
                                             uint32_t* codes_cmaj, moe_stream_t stream);
moe_status moe_reader_screen_partial(const moe_layer_desc* desc, const void* x, int32_t B, const int32_t* ids,
                                     const float* w, const int8_t* signs, const uint32_t* codes_cmaj,
                                     const uint16_t* scales, const float* dnorm, int32_t m, float* scores,
                                     float* est_opt, moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Rank-32 recovery of dropped channels ([Reader] "가중치만으로 만든 reader",
 * step 3, eq. 2): y_hat = sum_{kept j} w_j a_j d_j + U sum_{dropped j} w_j p_j
 * b_j, with U [H, 32] an orthonormal basis of the top-32 left singular
 * subspace of the layer's stacked down columns D = [d_1 .. d_n] (n = E*I, all
 * experts' channels), b_j = U^T d_j, and p_j = SiLU(g_hat_j) v_hat_j the
 * channel screen's estimate. desc: CHANNEL_MAJOR bf16 SWIGLU, H <= 2048. */
#define MOE_RECOVERY_RANK 32

/* Device scratch (bytes) moe_recovery_build needs for this layer shape
 * (H*H fp32 plus two H x 32 fp64 blocks); 0 for an unsupported descriptor. */
size_t moe_recovery_scratch_bytes(const moe_layer_desc* desc);

/* Load time, once per layer: U [H, 32] fp32 row-major (U[h * 32 + i]) from
 * the Gram matrix D D^T by 12 rounds of subspace iteration (fp64 CholeskyQR2
 * orthonormalisation); coeffs [E*I, 32] fp16 bit patterns, coeffs[j] =
 * U^T d_j rounded to nearest. Eq. 2 depends on U only through U U^T: any
 * orthonormal basis of the subspace gives the same output. scratch is
 * caller-owned (moe_recovery_scratch_bytes), 16-byte aligned; U 16-byte
 * aligned, coeffs 16-byte aligned. Asynchronous on stream. */
moe_status moe_recovery_build(const moe_layer_desc* desc, float* U, uint16_t* coeffs, void* scratch,
                              size_t scratch_bytes, moe_stream_t stream);

/* Decode time: for each token b (1 <= B <= 256), with ids [B, k] and w
 * [B, k] its routing, est [B, k, I, 2] the screen's {g_hat, v_hat} of its
 * routed experts' channels (moe_reader_screen's est_opt, same slot order),
 * kept [B, keep] the channels the sparse forward kept (indices e*I + c, as
 * moe_channel_topk_forward writes them): y[b] += U r_b with
 * r_b = sum over the routed candidates (e, c) not kept of
 * w[b, slot(e)] SiLU(g_hat) v_hat coeffs[e*I + c]. y [B, H] fp32 (added to).
 * 0 <= keep <= k*I <= 8192; est 8-byte and coeffs 16-byte aligned. */
moe_status moe_channel_recover(const moe_layer_desc* desc, int32_t B, const int32_t* ids, const float* w,
                               const float* est, const int32_t* kept, int32_t keep, const float* U,
                               const uint16_t* coeffs, float* y, moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOEDEC_H */
