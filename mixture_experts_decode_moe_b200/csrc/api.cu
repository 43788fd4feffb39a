// libmoedec C ABI: argument validation, launch planning and launches.
//
// The definitions of each operation (and the passages of the pages they
// follow) are documented in include/moedec.h.

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "small_kernels.cuh"
#include "linear.cuh"
#include "reader.cuh"
#include "channel_batch.cuh"
#include "recovery.cuh"

using namespace moedec;

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v, size_t a = kAlign) { return (v + a - 1) / a * a; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Workspace parts (byte offsets).
struct WsLayout {
  size_t logits, yacc, total;
};

inline WsLayout ws_layout(int B, int H, int E) {
  WsLayout w;
  size_t off = sizeof(WsControl);
  // 8 bytes per logit: {value, tag} on the batch-1 path (plain floats
  // [B, E] at batch > 1), then two buffers of E words for the next layer's
  // predicted logits (batch-1 stacks, alternating by layer)
  w.logits = off;
  off = align_up(off + (size_t)(B + 2) * E * sizeof(unsigned long long));
  w.yacc = off;     // three layer accumulators in rotation
  off = align_up(off + 3 * (size_t)B * H * sizeof(float));
  w.total = off;
  return w;
}

// Channel-major batches (2..8 tokens): the tokens' kept lists follow the
// common workspace parts ([B, min(k*I, 8192)] int32).
inline size_t chan_kept_offset(int B, const moe_layer_desc* d) { return ws_layout(B, d->H, d->E).total; }
inline size_t chan_kept_bytes(int B, const moe_layer_desc* d) {
  return align_up((size_t)B * std::min((size_t)d->k * d->I, (size_t)kMaxCand) * sizeof(int32_t));
}
// ... then the screened scores of a channel-major stack layer ([E*I] fp32).
inline size_t chan_scr_offset(int B, const moe_layer_desc* d) { return chan_kept_offset(B, d) + chan_kept_bytes(B, d); }
inline size_t chan_scr_bytes(const moe_layer_desc* d) { return align_up((size_t)d->E * d->I * sizeof(float)); }

// LINEAR experts: control block, the plan, and the packed token rows of the
// tensor-core units (at most B*k + 32*min(E, B*k) rows of H bf16).
struct LinWsLayout {
  size_t plan, xp, total;
  int xp_rows_max;
};
inline LinWsLayout lin_ws_layout(int B, int H, int E, int k) {
  LinWsLayout w;
  size_t off = sizeof(WsControl);
  w.plan = off;
  off = align_up(off + sizeof(LinPlan));
  w.xp = off;
  w.xp_rows_max = B * k + kTcRowsPerLoad * std::min(E, B * k);
  off = align_up(off + (size_t)w.xp_rows_max * H * 2);
  w.total = off;
  return w;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

int max_dyn_smem() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return 0;
  return n;
}

bool valid_shape(const moe_layer_desc* d) {
  if (d == nullptr) return false;
  if (d->H <= 0 || d->E <= 0 || d->I <= 0 || d->k <= 0) return false;
  if (d->E > kMaxE || d->k > kMaxK || d->k > d->E) return false;
  if (d->H % 64 != 0) return false;
  if (d->kind != MOE_EXPERT_SWIGLU && d->kind != MOE_EXPERT_LINEAR) return false;
  if (d->wtype != MOE_W_BF16 && d->wtype != MOE_W_INT4_G64) return false;
  if (d->layout != MOE_LAYOUT_PLANAR && d->layout != MOE_LAYOUT_CHANNEL_MAJOR) return false;
  if (d->wtype == MOE_W_INT4_G64 && (d->H % 512 != 0 || d->I % 64 != 0)) return false;
  if (d->I_shared < 0) return false;
  if (d->I > 65536 || d->I_shared > 65536) return false;  // keeps per-CTA range products in 32 bits
  return true;
}

// Weights present and aligned for a SwiGLU layer of this descriptor.
moe_status check_weights(const moe_layer_desc* d, bool need_router) {
  if (need_router && (d->router == nullptr || !aligned16(d->router))) return MOE_ERR_INVALID;
  if (d->gate == nullptr || !aligned16(d->gate)) return MOE_ERR_INVALID;
  if (d->kind == MOE_EXPERT_SWIGLU && d->layout == MOE_LAYOUT_PLANAR) {
    if (d->up == nullptr || d->down_t == nullptr || !aligned16(d->up) || !aligned16(d->down_t))
      return MOE_ERR_INVALID;
    if (d->wtype == MOE_W_INT4_G64) {
      if (!d->gate_s || !d->up_s || !d->down_s || !aligned16(d->gate_s) || !aligned16(d->up_s) ||
          !aligned16(d->down_s))
        return MOE_ERR_INVALID;
    }
  }
  if (d->I_shared > 0) {
    if (!d->sh_gate || !d->sh_up || !d->sh_down_t || !aligned16(d->sh_gate) || !aligned16(d->sh_up) ||
        !aligned16(d->sh_down_t))
      return MOE_ERR_INVALID;
  }
  return MOE_OK;
}

// Batch-1 bf16 rows of 2048: the kernel's warp-owned-channel path.
inline bool fast_path(const moe_layer_desc* d, int B) {
  return B == 1 && d->H == 2048 && (d->wtype == MOE_W_BF16 || d->layout == MOE_LAYOUT_PLANAR);
}

// Channels per job (template NCH). The warp-owned-channel path takes jobs of
// 4 channels (48 KB stages for bf16: four stages in flight, two warp groups
// of four warps, one channel per warp); other bf16 planar batch-1 shapes
// take 8, the rest 4.
inline int pick_nch(const moe_layer_desc* d, int B) {
  if (fast_path(d, B)) return 4;
  return (B == 1 && d->wtype == MOE_W_BF16 && d->layout == MOE_LAYOUT_PLANAR) ? 8 : 4;
}

// Shared-memory carve-up of the persistent decode kernel: as many ring stages
// as fit next to the fixed tiles, given the kernel's static shared memory.
bool plan_smem(DecodeParams* p, int static_bytes, bool fast, bool tc_batch) {
  const int H = p->H, rowb = 2 * H, B = p->B, NCH = p->nch;
  const int budget = max_dyn_smem() - static_bytes - 1024;
  if (budget <= 0) return false;
  const bool cm = p->layout == MOE_LAYOUT_CHANNEL_MAJOR;
  const int x_bytes = (int)align_up((size_t)B * H * 2, 128);
  // u (pre-normed x); the int4 batch path keeps it as 8 token rows of A fragments
  const int u_bytes = tc_batch ? (int)align_up((size_t)kMaxB * H * 2, 128) : (p->pre_norm ? x_bytes : 0);
  const int lg_bytes = (p->mode == MODE_LAYERS) ? (int)align_up((size_t)B * p->E * 4, 128) : 0;
  // keys: router top-k keys [B*E] and channel-sparse candidates [k*I]
  size_t nkeys = (p->mode == MODE_LAYERS) ? (size_t)B * p->E : 0;
  if (cm) nkeys = std::max(nkeys, (size_t)p->k * p->I);
  if (cm && p->screen) nkeys = std::max(nkeys, (size_t)kLutFloats);  // the screen's subset-sum table
  const int keys_bytes = (int)align_up(std::max<size_t>(nkeys, 1) * 4, 128);
  const int kept_bytes = cm ? (int)align_up((size_t)std::max(p->keep, 1) * 4, 128) : 0;
  const int hist_bytes = cm ? (int)align_up((size_t)(2 * kSelBins + kSelScratch) * 4, 128) : 0;  // the channel select's bins and scratch
  // output sums in shared memory: [H] (batch-1 fast path), [B][H] (int4 batch path)
  const int ysum_bytes = fast ? (int)align_up((size_t)H * 4, 128) : (tc_batch ? (int)align_up((size_t)B * H * 4, 128) : 0);
  const int xf_bytes = fast ? H * 2 : 0;  // x fragments, [segment][lane] x 16 B
  int stage;
  if (cm || p->wtype == MOE_W_BF16) stage = NCH * 3 * rowb;
  else stage = NCH * (3 * (H / 2) + 2 * (H / 32)) + rowb;
  if (tc_batch) {
    // stages sized for the int4 jobs: router jobs take as many rows, shared
    // jobs one channel (three bf16 rows)
    p->rows_per_job = std::max(1, std::min(p->rows_per_job, stage / rowb));
    if (p->I_sh > 0) stage = std::max(stage, 3 * rowb);
  } else {
    stage = std::max(stage, p->rows_per_job * rowb);
    if (p->I_sh > 0) stage = std::max(stage, NCH * 3 * rowb);
  }
  stage = (int)align_up(stage, 128);
  const int fixed = x_bytes + u_bytes + lg_bytes + keys_bytes + kept_bytes + hist_bytes + ysum_bytes + xf_bytes;
  const int nst = std::min(8, (budget - fixed - 256) / stage);
  if (nst < 2) return false;
  p->stage_bytes = stage;
  p->nstages = nst;
  int off = nst * stage;
  p->off_x = off; off += x_bytes;
  p->off_u = off; off += u_bytes;
  p->off_lg = off; off += lg_bytes;
  p->off_keys = off; off += keys_bytes;
  p->off_kept = off; off += kept_bytes;
  p->off_hist = off; off += hist_bytes;
  p->off_ysum = off; off += ysum_bytes;
  p->off_xf = off; off += xf_bytes;
  p->off_bar = off; off += (int)align_up((size_t)3 * nst * 8, 128);  // full, empty, dots-ready
  p->smem_bytes = off;
  return true;
}

template <int MODE, int BMAX, int WT, int LAYOUT, int NCH, int HV, bool SCREEN>
cudaError_t launch_decode_h(const DecodeParams& p0, int grid, cudaStream_t s) {
  auto kern = decode_kernel<MODE, BMAX, WT, LAYOUT, NCH, HV, SCREEN>;
  cudaFuncAttributes fa;
  cudaError_t err = cudaFuncGetAttributes(&fa, kern);
  if (err != cudaSuccess) return err;
  DecodeParams p = p0;
  constexpr bool kFast = (BMAX == 1 && HV == 8 && (WT == MOE_W_BF16 || LAYOUT == MOE_LAYOUT_PLANAR));
  constexpr bool kTcB = WT == MOE_W_INT4_G64 && BMAX == 8 && HV == 8 && NCH == 4 && LAYOUT == MOE_LAYOUT_PLANAR;
  if (!plan_smem(&p, (int)fa.sharedSizeBytes, kFast, kTcB)) return cudaErrorInvalidConfiguration;
  if (p.screen) {
    // the in-stack screen stages each CTA's candidates (code rows, scale
    // rows, down-column norm) in the ring
    const long long per_cand = (long long)p.H / 2 + p.H / 32 + 4;
    const long long nmax = ((long long)p.k * p.I + grid - 1) / grid;
    if (nmax * per_cand > (long long)p.nstages * p.stage_bytes) return cudaErrorInvalidConfiguration;
  }
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem_bytes);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kCtaThreads);
  cfg.dynamicSmemBytes = p.smem_bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

// Full-row dot loops are specialised for H = 2048 (HV = H/256 = 8 vectors per
// lane); other hidden sizes use the guarded generic loop.
template <int MODE, int BMAX, int WT, int LAYOUT, int NCH, bool SCREEN>
cudaError_t launch_decode_n(const DecodeParams& p, int grid, cudaStream_t s) {
  if (p.H == 2048) {
    // batch-1 H = 2048 kernels are the pipelined fast path: 4 channels per job
    if constexpr (BMAX == 1 && NCH != 4) return cudaErrorInvalidValue;
    else return launch_decode_h<MODE, BMAX, WT, LAYOUT, NCH, 8, SCREEN>(p, grid, s);
  }
  return launch_decode_h<MODE, BMAX, WT, LAYOUT, NCH, 0, SCREEN>(p, grid, s);
}

template <int MODE, int BMAX, int WT, int LAYOUT, bool SCREEN>
cudaError_t launch_decode_m(const DecodeParams& p, int grid, cudaStream_t s) {
  if constexpr (BMAX == 1 && WT == MOE_W_BF16) {
    if (p.nch == 8) return launch_decode_n<MODE, BMAX, WT, LAYOUT, 8, SCREEN>(p, grid, s);
  }
  if (p.nch != 4) return cudaErrorInvalidValue;
  return launch_decode_n<MODE, BMAX, WT, LAYOUT, 4, SCREEN>(p, grid, s);
}

template <int BMAX, int WT, int LAYOUT, bool SCREEN = false>
cudaError_t launch_decode_t(const DecodeParams& p, int grid, cudaStream_t s) {
  if constexpr (SCREEN) {  // the screened channel stack (layers mode only)
    if (p.mode != MODE_LAYERS) return cudaErrorInvalidValue;
    return launch_decode_m<MODE_LAYERS, BMAX, WT, LAYOUT, true>(p, grid, s);
  } else {
    if (p.mode == MODE_LAYERS) return launch_decode_m<MODE_LAYERS, BMAX, WT, LAYOUT, false>(p, grid, s);
    return launch_decode_m<MODE_EXPERTS, BMAX, WT, LAYOUT, false>(p, grid, s);
  }
}

moe_status launch_decode(const DecodeParams& p, int bmax, cudaStream_t s) {
  const int grid = sm_count();
  if (grid <= 0) return MOE_ERR_CUDA;
  cudaError_t err;
  if (p.layout == MOE_LAYOUT_CHANNEL_MAJOR) {
    if (bmax != 1) return MOE_ERR_UNSUPPORTED;
    err = p.screen ? launch_decode_t<1, MOE_W_BF16, MOE_LAYOUT_CHANNEL_MAJOR, true>(p, grid, s)
                   : launch_decode_t<1, MOE_W_BF16, MOE_LAYOUT_CHANNEL_MAJOR, false>(p, grid, s);
  } else if (p.wtype == MOE_W_BF16) {
    err = (bmax == 1) ? launch_decode_t<1, MOE_W_BF16, MOE_LAYOUT_PLANAR>(p, grid, s)
                      : launch_decode_t<kMaxB, MOE_W_BF16, MOE_LAYOUT_PLANAR>(p, grid, s);
  } else {
    err = (bmax == 1) ? launch_decode_t<1, MOE_W_INT4_G64, MOE_LAYOUT_PLANAR>(p, grid, s)
                      : launch_decode_t<kMaxB, MOE_W_INT4_G64, MOE_LAYOUT_PLANAR>(p, grid, s);
  }
  if (err == cudaErrorInvalidConfiguration) return MOE_ERR_UNSUPPORTED;
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

void fill_layer(LayerW* lw, const moe_layer_desc* d) {
  lw->router = static_cast<const uint8_t*>(d->router);
  lw->gate = static_cast<const uint8_t*>(d->gate);
  lw->up = static_cast<const uint8_t*>(d->up);
  lw->down = static_cast<const uint8_t*>(d->down_t);
  lw->gate_s = static_cast<const uint8_t*>(d->gate_s);
  lw->up_s = static_cast<const uint8_t*>(d->up_s);
  lw->down_s = static_cast<const uint8_t*>(d->down_s);
  lw->sh_gate = static_cast<const uint8_t*>(d->sh_gate);
  lw->sh_up = static_cast<const uint8_t*>(d->sh_up);
  lw->sh_down = static_cast<const uint8_t*>(d->sh_down_t);
  lw->scores = nullptr;
}

void fill_common(DecodeParams* p, const moe_layer_desc* d, int B, void* ws) {
  std::memset(p, 0, sizeof(*p));
  p->B = B;
  p->H = d->H;
  p->E = d->E;
  p->I = d->I;
  p->k = d->k;
  p->I_sh = d->I_shared;
  p->wtype = d->wtype;
  p->layout = d->layout;
  p->nch = pick_nch(d, B);
  p->nch_sh = p->nch;
  p->rows_per_job = 2 * p->nch;
  const WsLayout w = ws_layout(B, d->H, d->E);
  uint8_t* base = static_cast<uint8_t*>(ws);
  p->ctl = reinterpret_cast<WsControl*>(base);
  p->logits = reinterpret_cast<float*>(base + w.logits);
  p->plogits = reinterpret_cast<unsigned long long*>(base + w.logits) + (size_t)B * d->E;
  p->yacc = reinterpret_cast<float*>(base + w.yacc);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows][cols] array: box 64 x box_rows,
// 128-byte swizzle (the K-major tcgen05 operand layout).
bool encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kTcBlockK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

moe_status linear_forward(const moe_layer_desc* d, const void* x, int B, const int32_t* ids, const float* w, float* y,
                          void* ws, cudaStream_t s) {
  const int H = d->H;
  const int sms = sm_count();
  if (sms <= 0) return MOE_ERR_CUDA;
  const LinWsLayout wl = lin_ws_layout(B, H, d->E, d->k);
  uint8_t* base = static_cast<uint8_t*>(ws);
  LinTcParams tp;
  std::memset(&tp, 0, sizeof(tp));
  LinParams& lp = tp.lp;
  lp.B = B;
  lp.H = H;
  lp.E = d->E;
  lp.k = d->k;
  lp.x = static_cast<const uint16_t*>(x);
  lp.W = static_cast<const uint16_t*>(d->gate);
  lp.ids = ids;
  lp.w = w;
  lp.y = y;
  lp.plan = reinterpret_cast<LinPlan*>(base + wl.plan);
  lp.xp = reinterpret_cast<uint16_t*>(base + wl.xp);
  lp.xp_rows_max = wl.xp_rows_max;
  lp.num_sms = sms;
  lp.ctl = reinterpret_cast<WsControl*>(base);
  if (!encode_bf16_2d(&tp.tmap_w, d->gate, (uint64_t)H, (uint64_t)d->E * H, kTcBlockM)) return MOE_ERR_CUDA;
  if (!encode_bf16_2d(&tp.tmap_x, lp.xp, (uint64_t)H, (uint64_t)wl.xp_rows_max, kTcRowsPerLoad)) return MOE_ERR_CUDA;
  if (cudaMemsetAsync(y, 0, (size_t)B * H * sizeof(float), s) != cudaSuccess) return MOE_ERR_CUDA;
  linear_plan_kernel<<<1, kThreads, 0, s>>>(lp);
  linear_gather_kernel<<<sms * 4, kThreads, 0, s>>>(lp);
  const int gemv_smem = (kTcMin - 1) * H * 2;
  if (cudaFuncSetAttribute(linear_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, gemv_smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  linear_gemv_kernel<<<sms * 2, kThreads, gemv_smem, s>>>(lp);
  if (cudaFuncSetAttribute(linear_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem) != cudaSuccess)
    return MOE_ERR_CUDA;
  linear_tc_kernel<<<sms, kThreads, kTcSmem, s>>>(tp);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Argument checks of moe_layer_forward that do not involve the workspace.
moe_status layer_forward_args(const moe_layer_desc* d, const void* x, int B, const float* y, const void* x_next_opt,
                              const int32_t* ids_out_opt, const float* w_out_opt) {
  if (!y || !aligned16(y)) return MOE_ERR_INVALID;
  if (!valid_shape(d) || B < 1 || B > 256) return MOE_ERR_INVALID;
  if (d->kind != MOE_EXPERT_SWIGLU || d->layout != MOE_LAYOUT_PLANAR) return MOE_ERR_UNSUPPORTED;
  if (B > kMaxB || d->H > 2048) return MOE_ERR_UNSUPPORTED;
  if ((ids_out_opt == nullptr) != (w_out_opt == nullptr)) return MOE_ERR_INVALID;
  if (!x || !aligned16(x) || (x_next_opt && !aligned16(x_next_opt))) return MOE_ERR_INVALID;
  return check_weights(d, true);
}

// Experts of layer l+1 that a batch-1 stack predicts in layer l and
// prefetches into L2 (the tagged-word routing path: planar, k <= 8, E <= 256,
// H = 2048). 0 (off) by default; the environment variable
// MOEDEC_PREFETCH_EXPERTS (0..32) sets it for tuning.
int prefetch_experts(const moe_layer_desc* d, int B, int L) {
  if (B != 1 || L < 2 || !fast_path(d, B) || d->layout != MOE_LAYOUT_PLANAR || d->k > kWarps || d->E > 256)
    return 0;
  // off by default: measured on the A3B stack, the prefetch flood delays the
  // grid barrier and the next layer's serial chain by more than it saves
  int n = 0;
  if (const char* env = std::getenv("MOEDEC_PREFETCH_EXPERTS")) n = std::atoi(env);
  return std::max(0, std::min(std::min(n, kMaxPred), d->E));
}

bool same_shape(const moe_layer_desc* a, const moe_layer_desc* b) {
  return a->H == b->H && a->E == b->E && a->I == b->I && a->k == b->k && a->kind == b->kind &&
         a->wtype == b->wtype && a->layout == b->layout && a->I_shared == b->I_shared;
}

__global__ void set_i32_kernel(int32_t* dst, int32_t v) { *dst = v; }

// Sets one field of a workspace's control block, stream-ordered with the
// calls around it (what = 1: the wait budget, 2: the injection bits).
__global__ void ctl_set_kernel(WsControl* ctl, int what, unsigned long long budget, uint32_t inject) {
  if (what == 1) ctl->wait_budget = budget;
  else ctl->inject = inject;
}

}  // namespace

extern "C" {

int moe_abi_version(void) { return MOEDEC_ABI_VERSION; }

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID: return "invalid argument or expert ids";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or mode";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

size_t moe_workspace_bytes(const moe_layer_desc* d, int32_t B) {
  if (!valid_shape(d) || B < 1 || B > 256) return 0;
  if (d->kind == MOE_EXPERT_LINEAR) return std::max(ws_layout(B, d->H, d->E).total, lin_ws_layout(B, d->H, d->E, d->k).total);
  if (d->layout == MOE_LAYOUT_CHANNEL_MAJOR) return chan_scr_offset(B, d) + chan_scr_bytes(d);
  return ws_layout(B, d->H, d->E).total;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (ws == nullptr || !aligned16(ws) || ws_bytes < sizeof(WsControl)) return MOE_ERR_INVALID;
  return cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_get_status(const void* ws, moe_stream_t stream) {
  if (ws == nullptr) return MOE_ERR_INVALID;
  uint32_t st = 0;
  if (cudaMemcpyAsync(&st, ws, sizeof(st), cudaMemcpyDeviceToHost, (cudaStream_t)stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
  return (moe_status)st;
}

moe_status moe_workspace_set_wait_budget(void* ws, unsigned long long cycles, moe_stream_t stream) {
  if (ws == nullptr || !aligned16(ws)) return MOE_ERR_INVALID;
  WsControl* ctl = static_cast<WsControl*>(ws);
  ctl_set_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(ctl, 1, cycles, 0u);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_workspace_set_inject(void* ws, uint32_t flags, moe_stream_t stream) {
  if (ws == nullptr || !aligned16(ws) || (flags & ~(uint32_t)MOE_INJECT_BARRIER_EXTRA_ARRIVAL)) return MOE_ERR_INVALID;
  WsControl* ctl = static_cast<WsControl*>(ws);
  ctl_set_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(ctl, 2, 0ull, flags);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_route_topk(const void* x, const void* router, int32_t B, int32_t H, int32_t E, int32_t k,
                          int32_t* ids, float* w, float* margin_opt, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
  if (!x || !router || !ids || !w || !ws) return MOE_ERR_INVALID;
  if (B < 1 || B > 256 || H < 64 || H % 64 || E < 1 || E > kMaxE || k < 1 || k > kMaxK || k > E)
    return MOE_ERR_INVALID;
  if (!aligned16(x) || !aligned16(router) || !aligned16(ws)) return MOE_ERR_INVALID;
  if (H > 8192) return MOE_ERR_UNSUPPORTED;
  const WsLayout wl = ws_layout(B, H, E);
  if (ws_bytes < wl.total) return MOE_ERR_INVALID;
  float* logits = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + wl.logits);
  cudaStream_t s = (cudaStream_t)stream;
  const size_t sm1 = (size_t)kMaxB * H * 2;
  if (sm1 > 48 * 1024 &&
      cudaFuncSetAttribute(router_logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1) !=
          cudaSuccess)
    return MOE_ERR_CUDA;
  router_logits_kernel<<<dim3((E + kWarps - 1) / kWarps, (B + kMaxB - 1) / kMaxB), kThreads, sm1, s>>>(
      static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(router), B, H, E, logits);
  const size_t sm2 = (size_t)kWarps * E * 4;
  topk_kernel<<<(B + kWarps - 1) / kWarps, kThreads, sm2, s>>>(logits, B, E, k, ids, w, margin_opt);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_touched_experts(const int32_t* ids, int32_t B, int32_t k, int32_t E, int32_t* count,
                               uint32_t* bitmap_opt, int32_t* offsets_opt, int32_t* pairs_opt,
                               moe_stream_t stream) {
  if (!ids || !count) return MOE_ERR_INVALID;
  if (B < 1 || B > 256 || k < 1 || k > kMaxK || E < 1 || E > kMaxE || k > E) return MOE_ERR_INVALID;
  touched_kernel<<<1, kThreads, 0, (cudaStream_t)stream>>>(ids, B, k, E, count, bitmap_opt, offsets_opt,
                                                           pairs_opt);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

static bool reader_shape_ok(const moe_layer_desc* d) {
  return d->kind == MOE_EXPERT_SWIGLU && d->layout == MOE_LAYOUT_CHANNEL_MAJOR && d->wtype == MOE_W_BF16;
}

moe_status moe_reader_build(const moe_layer_desc* d, const int8_t* signs, uint32_t* codes, uint16_t* scales,
                            float* rho, float* dnorm, moe_stream_t stream) {
  if (!valid_shape(d) || !reader_shape_ok(d) || !d->gate || !signs || !codes || !scales || !rho || !dnorm)
    return MOE_ERR_INVALID;
  if (d->H % kRdBlock != 0 || d->H > 2048) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(d->gate) || ((uintptr_t)codes & 3u) || ((uintptr_t)rho & 3u) || ((uintptr_t)dnorm & 3u) ||
      ((uintptr_t)scales & 1u))
    return MOE_ERR_INVALID;
  const long long nch = (long long)d->E * d->I;
  if (nch > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  reader_build_kernel<<<(unsigned)nch, kRdBlock, 0, (cudaStream_t)stream>>>(
      static_cast<const uint16_t*>(d->gate), signs, d->H, codes, scales, rho, dnorm);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_reader_screen(const moe_layer_desc* d, const void* x, int32_t B, const int32_t* ids,
                             const float* w, const int8_t* signs, const uint32_t* codes, const uint16_t* scales,
                             const float* dnorm, float* scores, float* est_opt, moe_stream_t stream) {
  if (!valid_shape(d) || !reader_shape_ok(d) || !x || !ids || !w || !signs || !codes || !scales || !dnorm ||
      !scores)
    return MOE_ERR_INVALID;
  if (B < 1 || B > 256) return MOE_ERR_INVALID;
  if (d->H % kRdBlock != 0 || d->H > 2048) return MOE_ERR_UNSUPPORTED;
  if (((uintptr_t)x & 1u) || ((uintptr_t)codes & 15u) || ((uintptr_t)dnorm & 3u) || ((uintptr_t)scales & 3u) ||
      ((uintptr_t)scores & 3u) || ((uintptr_t)est_opt & 3u))
    return MOE_ERR_INVALID;
  const int sms = sm_count();
  if (sms <= 0) return MOE_ERR_CUDA;
  // about two CTAs per SM over the batch, each CTA at least 8 channels; a
  // CTA stages its candidates' code and scale rows in shared memory
  const int nq = d->k * d->I, wpc = kRdScreenThreads / 32;
  int gx = std::max(1, std::min((nq + wpc - 1) / wpc, (2 * sms + B - 1) / B));
  const size_t per_cand = (size_t)d->H / 2 + (size_t)d->H / 32;  // bytes of one candidate's codes and scales
  const size_t lut_bytes = sizeof(float) * kLutFloats + sizeof(int) * kMaxK;
  const size_t room = (size_t)max_dyn_smem() - lut_bytes - 1024;
  while ((size_t)((nq + gx - 1) / gx) * per_cand > room) ++gx;  // more CTAs, fewer candidates each
  const size_t dyn = (size_t)((nq + gx - 1) / gx) * per_cand + 16;
  if (cudaFuncSetAttribute(reader_screen_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn) != cudaSuccess)
    return MOE_ERR_CUDA;
  reader_screen_kernel<<<dim3((unsigned)gx, (unsigned)B), kRdScreenThreads, dyn, (cudaStream_t)stream>>>(
      static_cast<const uint16_t*>(x), d->H, d->E, d->I, d->k, ids, w, signs, codes, scales, dnorm, scores,
      est_opt);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_expert_forward(const moe_layer_desc* d, const void* x, int32_t B, const int32_t* ids,
                              const float* w, float* y, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!valid_shape(d) || !x || !ids || !w || !y || !ws) return MOE_ERR_INVALID;
  if (!aligned16(x) || !aligned16(y) || !aligned16(ws) || B < 1 || B > 256) return MOE_ERR_INVALID;
  if (ws_bytes < moe_workspace_bytes(d, B)) return MOE_ERR_INVALID;
  if (d->kind == MOE_EXPERT_LINEAR) {
    if (d->wtype != MOE_W_BF16 || d->layout != MOE_LAYOUT_PLANAR) return MOE_ERR_UNSUPPORTED;
    if (d->H % 256 != 0 || d->gate == nullptr || !aligned16(d->gate) || !aligned16(w) || !aligned16(ids))
      return MOE_ERR_INVALID;
    return linear_forward(d, x, B, ids, w, y, ws, (cudaStream_t)stream);
  }
  if (d->kind != MOE_EXPERT_SWIGLU || d->layout != MOE_LAYOUT_PLANAR) return MOE_ERR_UNSUPPORTED;
  if (B > kMaxB || d->H > 2048) return MOE_ERR_UNSUPPORTED;
  moe_status st = check_weights(d, false);
  if (st != MOE_OK) return st;
  DecodeParams p;
  fill_common(&p, d, B, ws);
  p.L = 1;
  p.mode = MODE_EXPERTS;
  p.I_sh = 0;
  p.x_in = static_cast<const uint16_t*>(x);
  p.y_out = y;
  p.ids_in = ids;
  p.w_in = w;
  fill_layer(&p.layer[0], d);
  return launch_decode(p, B <= 1 ? 1 : kMaxB, (cudaStream_t)stream);
}

moe_status moe_stack_forward(const moe_layer_desc* layers, int32_t L, const void* x, int32_t B, uint32_t flags,
                             void* x_out, void* x_hist_opt, float* y_hist_opt, int32_t* ids_hist_opt,
                             float* w_hist_opt, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (flags & ~(uint32_t)MOE_STACK_PRE_RMSNORM) return MOE_ERR_INVALID;
  if (layers == nullptr || L < 1 || L > kMaxLayers || !x || !ws) return MOE_ERR_INVALID;
  const moe_layer_desc* d = &layers[0];
  if (!valid_shape(d) || B < 1 || B > 256) return MOE_ERR_INVALID;
  if (!aligned16(x) || !aligned16(ws) || (x_out && !aligned16(x_out)) || (x_hist_opt && !aligned16(x_hist_opt)) ||
      (y_hist_opt && !aligned16(y_hist_opt)))
    return MOE_ERR_INVALID;
  if ((ids_hist_opt == nullptr) != (w_hist_opt == nullptr)) return MOE_ERR_INVALID;
  if (ws_bytes < moe_workspace_bytes(d, B)) return MOE_ERR_INVALID;
  if (d->kind != MOE_EXPERT_SWIGLU || d->layout != MOE_LAYOUT_PLANAR) return MOE_ERR_UNSUPPORTED;
  if (B > kMaxB || d->H > 2048) return MOE_ERR_UNSUPPORTED;
  for (int l = 0; l < L; ++l) {
    if (!same_shape(&layers[l], d)) return MOE_ERR_INVALID;
    moe_status st = check_weights(&layers[l], true);
    if (st != MOE_OK) return st;
  }
  const bool pre_norm = (flags & MOE_STACK_PRE_RMSNORM) != 0;
  DecodeParams p;
  fill_common(&p, d, B, ws);
  p.L = L;
  p.mode = MODE_LAYERS;
  p.npred = prefetch_experts(d, B, L);
  p.pre_norm = pre_norm ? 1 : 0;
  p.x_in = static_cast<const uint16_t*>(x);
  p.x_out = static_cast<uint16_t*>(x_out);
  p.x_hist = static_cast<uint16_t*>(x_hist_opt);
  p.y_hist = y_hist_opt;
  p.ids_out = ids_hist_opt;
  p.w_out = w_hist_opt;
  for (int l = 0; l < L; ++l) fill_layer(&p.layer[l], &layers[l]);
  return launch_decode(p, B <= 1 ? 1 : kMaxB, (cudaStream_t)stream);
}

moe_status moe_channel_stack_forward(const moe_layer_desc* layers, int32_t L, const void* x, uint32_t flags,
                                     const float* scores, const moe_sketch_desc* sketches, const int8_t* signs,
                                     int32_t keep, void* x_out, void* x_hist_opt,
                                     float* y_hist_opt, int32_t* ids_hist_opt, float* w_hist_opt,
                                     int32_t* kept_hist_opt, unsigned long long* sectors, void* ws,
                                     size_t ws_bytes, moe_stream_t stream) {
  if (layers == nullptr || L < 1 || L > kMaxLayers || !x || !sectors || !ws) return MOE_ERR_INVALID;
  if ((scores == nullptr) == (sketches == nullptr) || (sketches != nullptr && signs == nullptr)) return MOE_ERR_INVALID;
  if (flags & ~(uint32_t)MOE_STACK_PRE_RMSNORM) return MOE_ERR_INVALID;
  const moe_layer_desc* d = &layers[0];
  if (!valid_shape(d)) return MOE_ERR_INVALID;
  if (d->kind != MOE_EXPERT_SWIGLU || d->layout != MOE_LAYOUT_CHANNEL_MAJOR || d->wtype != MOE_W_BF16)
    return MOE_ERR_INVALID;
  if (keep < 0 || keep > d->k * d->I) return MOE_ERR_INVALID;
  if ((long long)d->k * d->I > kMaxCand || d->H > 2048) return MOE_ERR_UNSUPPORTED;
  if (sketches != nullptr && d->H % kRdBlock != 0) return MOE_ERR_UNSUPPORTED;
  if ((ids_hist_opt == nullptr) != (w_hist_opt == nullptr)) return MOE_ERR_INVALID;
  if (!aligned16(x) || !aligned16(ws) || (scores && !aligned16(scores)) || (x_out && !aligned16(x_out)) ||
      (x_hist_opt && !aligned16(x_hist_opt)) || (y_hist_opt && !aligned16(y_hist_opt)))
    return MOE_ERR_INVALID;
  if (ws_bytes < moe_workspace_bytes(d, 1)) return MOE_ERR_INVALID;
  for (int l = 0; l < L; ++l) {
    if (!same_shape(&layers[l], d)) return MOE_ERR_INVALID;
    moe_status st = check_weights(&layers[l], true);
    if (st != MOE_OK) return st;
  }
  DecodeParams p;
  fill_common(&p, d, 1, ws);
  p.L = L;
  p.mode = MODE_LAYERS;
  p.pre_norm = (flags & MOE_STACK_PRE_RMSNORM) ? 1 : 0;
  p.keep = keep;
  p.x_in = static_cast<const uint16_t*>(x);
  p.x_out = static_cast<uint16_t*>(x_out);
  p.x_hist = static_cast<uint16_t*>(x_hist_opt);
  p.y_hist = y_hist_opt;
  p.ids_out = ids_hist_opt;
  p.w_out = w_hist_opt;
  p.kept_out = kept_hist_opt;
  p.sectors_out = sectors;
  for (int l = 0; l < L; ++l) {
    fill_layer(&p.layer[l], &layers[l]);
    if (scores != nullptr) {
      p.layer[l].scores = scores + (size_t)l * d->E * d->I;
    } else {
      const moe_sketch_desc& sk = sketches[l];
      if (!sk.codes || !sk.scales || !sk.dnorm || ((uintptr_t)sk.codes & 15u) || ((uintptr_t)sk.scales & 3u) ||
          ((uintptr_t)sk.dnorm & 3u))
        return MOE_ERR_INVALID;
      p.layer[l].sk_codes = sk.codes;
      p.layer[l].sk_scales = sk.scales;
      p.layer[l].sk_dnorm = sk.dnorm;
    }
  }
  if (sketches != nullptr) {
    p.screen = 1;
    p.signs = signs;
    p.scr = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + chan_scr_offset(1, d));
  }
  return launch_decode(p, 1, (cudaStream_t)stream);
}

moe_status moe_layer_forward(const moe_layer_desc* d, const void* x, int32_t B, float* y, void* x_next_opt,
                             int32_t* ids_out_opt, float* w_out_opt, void* ws, size_t ws_bytes,
                             moe_stream_t stream) {
  moe_status st = layer_forward_args(d, x, B, y, x_next_opt, ids_out_opt, w_out_opt);
  if (st != MOE_OK) return st;
  if (!ws || !aligned16(ws)) return MOE_ERR_INVALID;
  if (ws_bytes < moe_workspace_bytes(d, B)) return MOE_ERR_INVALID;
  DecodeParams p;
  fill_common(&p, d, B, ws);
  p.L = 1;
  p.mode = MODE_LAYERS;
  p.x_in = static_cast<const uint16_t*>(x);
  p.x_out = static_cast<uint16_t*>(x_next_opt);
  p.y_out = y;
  p.ids_out = ids_out_opt;
  p.w_out = w_out_opt;
  fill_layer(&p.layer[0], d);
  return launch_decode(p, B <= 1 ? 1 : kMaxB, (cudaStream_t)stream);
}

moe_status moe_channel_topk_forward(const moe_layer_desc* d, const void* x, int32_t B, const int32_t* ids,
                                    const float* w, const float* scores, int32_t keep, float* y,
                                    int32_t* kept_opt, unsigned long long* sectors, int32_t* union_count_opt,
                                    unsigned long long* union_sectors_opt, void* ws, size_t ws_bytes,
                                    moe_stream_t stream) {
  if (!valid_shape(d) || !x || !ids || !w || !scores || !y || !sectors || !ws) return MOE_ERR_INVALID;
  if (B < 1 || B > kMaxB) return MOE_ERR_INVALID;
  if (d->kind != MOE_EXPERT_SWIGLU || d->layout != MOE_LAYOUT_CHANNEL_MAJOR || d->wtype != MOE_W_BF16)
    return MOE_ERR_INVALID;
  if (keep < 0 || keep > d->k * d->I) return MOE_ERR_INVALID;
  if ((long long)d->k * d->I > kMaxCand || d->H > 2048) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(y) || !aligned16(ws) || !aligned16(d->gate)) return MOE_ERR_INVALID;
  if (ws_bytes < moe_workspace_bytes(d, B)) return MOE_ERR_INVALID;
  cudaStream_t s = (cudaStream_t)stream;
  const int nk = std::min(keep, d->k * d->I);
  if (B == 1) {
    // one token: the persistent decode kernel's channel-major path; its
    // union is its own kept set
    DecodeParams p;
    fill_common(&p, d, 1, ws);
    p.L = 1;
    p.mode = MODE_EXPERTS;
    p.I_sh = 0;
    p.keep = keep;
    p.x_in = static_cast<const uint16_t*>(x);
    p.y_out = y;
    p.ids_in = ids;
    p.w_in = w;
    p.kept_out = kept_opt;
    p.sectors_out = sectors;
    fill_layer(&p.layer[0], d);
    p.layer[0].scores = scores;
    moe_status st = launch_decode(p, 1, s);
    if (st != MOE_OK) return st;
    if (union_count_opt) set_i32_kernel<<<1, 1, 0, s>>>(union_count_opt, nk);
    if (union_sectors_opt &&
        cudaMemcpyAsync(union_sectors_opt, sectors, sizeof(unsigned long long), cudaMemcpyDeviceToDevice, s) !=
            cudaSuccess)
      return MOE_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  // 2..8 tokens: one cooperative launch that reads the union once
  const int G = sm_count();
  if (G <= 0) return MOE_ERR_CUDA;
  const long long units = std::min<long long>(d->E, (long long)B * d->k);
  if (units > kCbMaxUnits || (long long)d->E * d->I > kCbMaxChanBits) return MOE_ERR_UNSUPPORTED;
  if (((long long)B * nk + G - 1) / G > kCbMaxSlice) return MOE_ERR_UNSUPPORTED;
  ChanBatchParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = B; p.H = d->H; p.E = d->E; p.I = d->I; p.k = d->k; p.keep = keep;
  p.x = static_cast<const uint16_t*>(x);
  p.ids = ids;
  p.w = w;
  p.scores = scores;
  p.cm = static_cast<const uint8_t*>(d->gate);
  p.y = y;
  p.kept_out = kept_opt;
  p.sectors = sectors;
  p.union_count = union_count_opt;
  p.union_sectors = union_sectors_opt;
  uint8_t* base = static_cast<uint8_t*>(ws);
  p.ctl = reinterpret_cast<WsControl*>(base);
  p.kept_ws = reinterpret_cast<int32_t*>(base + chan_kept_offset(B, d));
  // the tokens' kept-channel bitmaps (B x jstride words) use the scores area
  // of the channel workspace: B * E*I / 8 bytes <= E*I * 4 bytes
  const long long jstride = (((long long)d->E * d->I + 31) / 32 + 3) / 4 * 4;
  p.jstride = (int)jstride;
  p.bits_ws = reinterpret_cast<uint32_t*>(base + chan_scr_offset(B, d));
  if ((size_t)B * jstride * 4 > chan_scr_bytes(d)) return MOE_ERR_UNSUPPORTED;
  size_t ring = (size_t)kCbStages * kCbNch * 3 * d->H * 2;
  // phase A: keys, the select's bins and scratch, the token's bitmap
  ring = std::max(ring, align_up((size_t)d->k * d->I * 4, 128) + (size_t)(2 * kSelBins + kSelScratch) * 4 +
                            (size_t)jstride * 4);
  ring = std::max(ring, (size_t)(B + 2) * (size_t)jstride * 4);  // phase B: the bitmaps, the union, its prefix
  ring = std::max(ring, (size_t)(d->E + 31) / 32 * 4);
  ring = align_up(ring, (size_t)128);
  p.ring_bytes = (int)ring;
  p.smem_bytes = (int)(ring + (size_t)B * d->H * 2);
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, channel_batch_kernel) != cudaSuccess) return MOE_ERR_CUDA;
  if (p.smem_bytes + (int)fa.sharedSizeBytes + 1024 > max_dyn_smem()) return MOE_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(channel_batch_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem_bytes) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(kCbThreads);
  cfg.dynamicSmemBytes = p.smem_bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, channel_batch_kernel, p) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

static bool partial_shape_ok(const moe_layer_desc* d) {
  // one thread per (code word, block) in one CTA; per-channel sums in shared memory (I <= 1024)
  return d->H % kRdBlock == 0 && d->H <= 2048 && d->I % 16 == 0 && d->I <= 1024 &&
         (d->I / 16) * (d->H / kRdBlock) <= 1024;
}

moe_status moe_reader_codes_coordinate_major(const moe_layer_desc* d, const uint32_t* codes, uint32_t* codes_cmaj,
                                             moe_stream_t stream) {
  if (!valid_shape(d) || !reader_shape_ok(d) || !codes || !codes_cmaj) return MOE_ERR_INVALID;
  if (!partial_shape_ok(d)) return MOE_ERR_UNSUPPORTED;
  if (((uintptr_t)codes & 3u) || ((uintptr_t)codes_cmaj & 3u)) return MOE_ERR_INVALID;
  const int sms = sm_count();
  if (sms <= 0) return MOE_ERR_CUDA;
  reader_cmaj_kernel<<<sms * 8, 256, 0, (cudaStream_t)stream>>>(codes, d->E, d->I, d->H, codes_cmaj);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_reader_screen_partial(const moe_layer_desc* d, const void* x, int32_t B, const int32_t* ids,
                                     const float* w, const int8_t* signs, const uint32_t* codes_cmaj,
                                     const uint16_t* scales, const float* dnorm, int32_t m, float* scores,
                                     float* est_opt, moe_stream_t stream) {
  if (!valid_shape(d) || !reader_shape_ok(d) || !x || !ids || !w || !signs || !codes_cmaj || !scales || !dnorm ||
      !scores)
    return MOE_ERR_INVALID;
  if (B < 1 || B > 256 || m < 0 || m > kRdBlock) return MOE_ERR_INVALID;
  if (!partial_shape_ok(d)) return MOE_ERR_UNSUPPORTED;
  if (((uintptr_t)x & 1u) || ((uintptr_t)codes_cmaj & 3u) || ((uintptr_t)dnorm & 3u) || ((uintptr_t)scales & 1u) ||
      ((uintptr_t)scores & 3u) || ((uintptr_t)est_opt & 3u))
    return MOE_ERR_INVALID;
  const int nt = (d->I / 16) * (d->H / kRdBlock);
  reader_screen_partial_kernel<<<dim3((unsigned)d->k, (unsigned)B), std::max(nt, d->H / kRdBlock), 0,
                                 (cudaStream_t)stream>>>(static_cast<const uint16_t*>(x), d->H, d->E, d->I, d->k,
                                                         ids, w, signs, codes_cmaj, scales, dnorm, m, scores,
                                                         est_opt);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

static bool recovery_shape_ok(const moe_layer_desc* d) {
  return valid_shape(d) && reader_shape_ok(d) && d->H <= 2048 && (long long)d->E * d->I < 0x7fffffffLL;
}

size_t moe_recovery_scratch_bytes(const moe_layer_desc* d) {
  if (!recovery_shape_ok(d)) return 0;
  return align_up((size_t)d->H * d->H * sizeof(float)) + 2 * align_up((size_t)d->H * kRecRank * sizeof(double));
}

moe_status moe_recovery_build(const moe_layer_desc* d, float* U, uint16_t* coeffs, void* scratch, size_t scratch_bytes,
                              moe_stream_t stream) {
  if (!recovery_shape_ok(d)) return valid_shape(d) && reader_shape_ok(d) ? MOE_ERR_UNSUPPORTED : MOE_ERR_INVALID;
  if (!d->gate || !U || !coeffs || !scratch || !aligned16(d->gate) || !aligned16(U) || !aligned16(coeffs) ||
      !aligned16(scratch))
    return MOE_ERR_INVALID;
  if (scratch_bytes < moe_recovery_scratch_bytes(d)) return MOE_ERR_INVALID;
  const int H = d->H, n = d->E * d->I;
  const int sms = sm_count();
  if (sms <= 0) return MOE_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  float* C = reinterpret_cast<float*>(base);
  double* Q = reinterpret_cast<double*>(base + align_up((size_t)H * H * sizeof(float)));
  double* Y = Q + align_up((size_t)H * kRecRank * sizeof(double)) / sizeof(double);
  const uint16_t* cm = static_cast<const uint16_t*>(d->gate);
  const int nt = H / kGramTile;
  gram_kernel<<<nt * (nt + 1) / 2, 256, 0, s>>>(cm, H, n, C);
  subspace_init_kernel<<<(H * kRecRank + 255) / 256, 256, 0, s>>>(H, Q);
  for (int r = 0; r < kRecRounds; ++r) {
    subspace_mul_kernel<<<(H + 7) / 8, 256, 0, s>>>(C, H, Q, Y);
    subspace_qr_kernel<<<1, 256, 0, s>>>(H, Y);
    std::swap(Q, Y);
  }
  subspace_store_kernel<<<(H * kRecRank + 255) / 256, 256, 0, s>>>(H, Q, U);
  coeff_kernel<<<sms * 4, 256, 0, s>>>(cm, H, n, U, coeffs);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_channel_recover(const moe_layer_desc* d, int32_t B, const int32_t* ids, const float* w,
                               const float* est, const int32_t* kept, int32_t keep, const float* U,
                               const uint16_t* coeffs, float* y, moe_stream_t stream) {
  if (!valid_shape(d) || !reader_shape_ok(d) || !ids || !w || !est || !U || !coeffs || !y) return MOE_ERR_INVALID;
  if (B < 1 || B > 256 || keep < 0 || keep > d->k * d->I || (keep > 0 && !kept)) return MOE_ERR_INVALID;
  if ((long long)d->k * d->I > kMaxCand) return MOE_ERR_UNSUPPORTED;
  if (((uintptr_t)est & 7u) || !aligned16(coeffs) || ((uintptr_t)U & 3u) || ((uintptr_t)y & 3u))
    return MOE_ERR_INVALID;
  recover_kernel<<<B, 256, 0, (cudaStream_t)stream>>>(d->H, d->E, d->I, d->k, ids, w, est, kept, keep, U, coeffs,
                                                      y);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------- no-allocation variant
//
// A library-owned scratch array stands in for the caller's workspace. In host
// code the symbol below is only a handle: its device address is looked up with
// cudaGetSymbolAddress, with the caller's device current, and that address is
// what the kernel receives. The lookup runs on every call (it is a host-side
// table lookup once the library's device code is loaded in the current
// context), so the address always belongs to the context that is current now,
// also after a device reset has replaced the context.
namespace {

static __device__ __align__(256) unsigned char g_static_scratch[MOE_STATIC_SCRATCH_BYTES];

moe_status static_scratch_address(void** out) {
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_static_scratch) != cudaSuccess || addr == nullptr) return MOE_ERR_CUDA;
  *out = addr;
  return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_layer_forward_static(const moe_layer_desc* desc, const void* x, int32_t B, float* y,
                                                void* x_next_opt, int32_t* ids_out_opt, float* w_out_opt,
                                                int32_t* status_out_opt, moe_stream_t stream) {
  const size_t need = moe_workspace_bytes(desc, B);
  if (need == 0) return MOE_ERR_INVALID;
  if (need > MOE_STATIC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED;  // beyond the fixed scratch size
  // every argument check runs before the shared scratch is touched: a
  // rejected call launches nothing and leaves the previous contents alone
  moe_status st = layer_forward_args(desc, x, B, y, x_next_opt, ids_out_opt, w_out_opt);
  if (st != MOE_OK) return st;
  void* scratch = nullptr;
  st = static_scratch_address(&scratch);
  if (st != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  // the previous call's status word and barrier counter must not leak into
  // this one; the counter restarts, so the tagged logit words of the previous
  // call (which carry the same tags) are cleared as well
  const WsLayout wl = ws_layout(B, desc->H, desc->E);
  if (cudaMemsetAsync(scratch, 0, wl.yacc, s) != cudaSuccess) return MOE_ERR_CUDA;
  st = moe_layer_forward(desc, x, B, y, x_next_opt, ids_out_opt, w_out_opt, scratch, MOE_STATIC_SCRATCH_BYTES,
                         stream);
  if (st != MOE_OK) return st;
  if (status_out_opt != nullptr &&
      cudaMemcpyAsync(status_out_opt, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
