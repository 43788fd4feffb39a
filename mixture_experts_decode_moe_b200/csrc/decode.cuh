// Persistent decode kernel: router -> top-k -> routed SwiGLU experts (+ shared
// expert) -> router-weighted sum -> residual, for L layers in ONE cooperative
// launch with one CTA per SM.
//
// What it computes (pages cited by title and section):
//  * router GEMV, softmax, top-k ("MoE 입문: 36B 모델이 27B보다 6배 빨랐던
//    이유", "누가 8명을 고르나요"); ties go to the lowest expert index;
//  * channel j of expert e: a_j = phi(g_j.x)(v_j.x), phi = SiLU, output
//    += w_e a_j d_j (review of arXiv:2610.37386, "배경: 채널과 유지 규칙");
//  * the shared expert every token touches, weight 1 ("Mixture of Experts
//    Changes the Arithmetic", "Two Numbers Instead of One");
//  * channel-sparse: one top-k over all routed experts' channels by a
//    given score, only kept channels are read (same review, keep-rule table,
//    "2단계", Fig. 2(c) for the 32-byte sector charge).
//
// How (B200 design):
//  * the work unit is a run of up to `nch` consecutive channels of one
//    expert: its gate rows, up rows and transposed-down rows are three
//    contiguous byte ranges, fetched by 1-D bulk copies (TMA) into a ring of
//    shared-memory stages with an L2 evict-first hint; one thread issues,
//    all 256 compute; the ring keeps several stages in flight per SM;
//  * each CTA owns a contiguous slice of (router rows, shared channels,
//    routed channels); its partial y stays in registers and is added to an
//    fp32 accumulator in L2 with vector reductions;
//  * two grid-wide barriers per layer: after the router logits, and after
//    the partial sums. Shared-expert work runs between the router's arrival
//    and the top-k, and the next layer's router/shared weights are fetched
//    into the ring while the current layer drains.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace moedec {

constexpr int kMaxLayers = 64;
constexpr int kMaxB = 8;
constexpr int kMaxK = 32;
constexpr int kMaxE = 1024;
constexpr int kMaxCand = 8192;  // channel-sparse candidates per token (k*I)
constexpr int kMaxPred = 32;    // experts of the next layer prefetched into L2

enum DecodeMode : int { MODE_EXPERTS = 0, MODE_LAYERS = 1 };

struct LayerW {
  const uint8_t* router;  // [E, H] bf16
  const uint8_t* gate;    // planar [E, I, H] bf16 | int4 codes [E, I, H/2] | channel-major [E, I, 3, H]
  const uint8_t* up;
  const uint8_t* down;    // transposed down, same shape as gate (planar)
  const uint8_t* gate_s;  // int4 scales [E, I, H/64] bf16
  const uint8_t* up_s;
  const uint8_t* down_s;  // int4 [E, I/64, H] bf16
  const uint8_t* sh_gate; // shared expert bf16 [I_sh, H]
  const uint8_t* sh_up;
  const uint8_t* sh_down;
  const float* scores;    // channel-sparse scores [B, E, I] fp32
  // channel screen sketch of the layer (channel-major stacks that compute
  // their scores): codes [E*I][2][H/16], fp16 scales [E*I][2][H/128], dnorm [E*I]
  const uint32_t* sk_codes;
  const uint16_t* sk_scales;
  const float* sk_dnorm;
};

struct DecodeParams {
  int L, B, H, E, I, k, I_sh;
  int mode;     // DecodeMode
  int wtype;    // MOE_W_BF16 / MOE_W_INT4_G64
  int layout;   // MOE_LAYOUT_PLANAR / MOE_LAYOUT_CHANNEL_MAJOR
  int keep;     // channel-sparse keep count
  int pre_norm; // stack: RMS-normalise each layer's input (unit weight, eps 1e-6)
  int nch;      // channels per job (routed); shared jobs use nch_sh
  int nch_sh;
  int rows_per_job;  // router rows per job
  int nstages;
  int stage_bytes;
  // batch-1 stack: experts of layer l+1 predicted in layer l from
  // R_{l+1} u_l and prefetched into L2 (0 = off), at most kMaxPred
  int npred;
  // channel-major stack: scores from the weight-only screen, computed in the
  // kernel per layer into scr [E*I] (0 = scores are an input)
  int screen;
  const int8_t* signs;    // [H] rotation signs of the screen
  float* scr;             // ws [E*I]
  // shared-memory carve-up (byte offsets from the dynamic smem base)
  int off_x, off_u, off_lg, off_keys, off_kept, off_hist, off_ysum, off_xf, off_bar, smem_bytes;
  // io
  const uint16_t* x_in;   // [B, H]
  uint16_t* x_out;        // [B, H] final x (or null)
  uint16_t* x_hist;       // [L+1, B, H] (or null)
  float* y_out;           // [B, H] last layer's y (or null)
  float* y_hist;          // [L, B, H] (or null)
  const int32_t* ids_in;  // MODE_EXPERTS: [B, k]
  const float* w_in;
  int32_t* ids_out;       // [L, B, k] (or null)
  float* w_out;
  int32_t* kept_out;      // channel-sparse [B, keep] (or null)
  unsigned long long* sectors_out;  // channel-sparse [B] (or null)
  WsControl* ctl;
  float* logits;          // ws [B, E]
  unsigned long long* plogits;  // ws [E]: predicted logits of the next layer, {value, tag} words
  float* yacc;            // ws [2, B, H]
  LayerW layer[kMaxLayers];
};

// Per-CTA routing state in shared memory, sized for at most BMAX tokens.
template <int BMAX>
struct RouteSmem {
  int U;                     // routed units (touched experts, ascending)
  int ncand;                 // channel-sparse: number of kept channels
  int unit_e[BMAX * kMaxK];
  uint32_t unit_mask[BMAX * kMaxK];
  float unit_w[BMAX * kMaxK][BMAX];
  int cpre[BMAX * kMaxK + 1];  // batch > 1: cost offset of each unit's first channel (cpre[U] = total)
  uint32_t bitmap[kMaxE / 32];
  int rank_base[kMaxE / 32];
  int ids[BMAX][kMaxK];
  float w[BMAX][kMaxK];
  uint32_t hist[256];
  int scan[kThreads];
  int sel_prefix, sel_rank;
  unsigned long long sectors;
};

enum JobType : int { JOB_ROUTER = 0, JOB_SHARED = 1, JOB_ROUTED = 2, JOB_END = 3 };

struct Job {
  int type;
  int layer;
  int u;    // routed: unit index; channel-sparse: position in the kept list
  int c0;   // first row / channel
  int n;    // rows / channels
};

// Walks one CTA's job sequence: for each layer, its router rows, then its
// shared channels, then its routed channels (known only after top-k). All
// counters are 32-bit; the only divisions happen once per layer.
struct JobCursor {
  int layer;
  int type;
  int t;    // cursor inside the current type's range
  int t1;   // end of the range (-1: routed range not known yet)
  int u, c; // routed planar: t = u * I + c

  __device__ void begin_layer(const DecodeParams& p, int l) {
    layer = l;
    type = JOB_ROUTER;
    set_range(p);
  }
  __device__ void set_range(const DecodeParams& p) {
    // 32-bit products: E <= 1024 and I_sh, routed channels < 2^21, grid < 2^11
    const unsigned G = gridDim.x, cb = blockIdx.x;
    if (type == JOB_ROUTER) {
      if (p.mode == MODE_LAYERS && layer < p.L && p.layer[layer].router != nullptr) {
        t = (int)(cb * (unsigned)p.E / G); t1 = (int)((cb + 1) * (unsigned)p.E / G);
        if (t < t1) return;
      }
      type = JOB_SHARED;
    }
    if (type == JOB_SHARED) {
      if (p.mode == MODE_LAYERS && p.I_sh > 0) {
        t = (int)(cb * (unsigned)p.I_sh / G); t1 = (int)((cb + 1) * (unsigned)p.I_sh / G);
        if (t < t1) return;
      }
      type = JOB_ROUTED;
    }
    t = -1; t1 = -1;  // routed: set once the routing is known
  }
  // Routed range given directly (batch 1: the same every layer).
  __device__ void set_routed_fixed(const int4& r) {
    t = r.x; t1 = r.y; u = r.z; c = r.w;
  }
  // Routed range of this CTA once the number of routed channels R is known.
  __device__ void set_routed(int R, int I) {
    const unsigned G = gridDim.x, cb = blockIdx.x;
    t = (int)(cb * (unsigned)R / G); t1 = (int)((cb + 1) * (unsigned)R / G);
    u = t / I; c = t - u * I;
  }
};

__device__ __forceinline__ long long llmin(long long a, long long b) { return a < b ? a : b; }

// SiLU with the fast exponential and division intrinsics (relative error a
// few ulp; __fdividef returns 0 when 1 + e^-z overflows past 2^126, the limit).
__device__ __forceinline__ float silu_f(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// dot of 8 bf16 weights with 8 bf16 activations
__device__ __forceinline__ float dot8_bf16(const uint4& wv, const uint4& xv) {
  float a = bf16_lo(wv.x) * bf16_lo(xv.x);
  a = fmaf(bf16_hi(wv.x), bf16_hi(xv.x), a);
  a = fmaf(bf16_lo(wv.y), bf16_lo(xv.y), a);
  a = fmaf(bf16_hi(wv.y), bf16_hi(xv.y), a);
  a = fmaf(bf16_lo(wv.z), bf16_lo(xv.z), a);
  a = fmaf(bf16_hi(wv.z), bf16_hi(xv.z), a);
  a = fmaf(bf16_lo(wv.w), bf16_lo(xv.w), a);
  a = fmaf(bf16_hi(wv.w), bf16_hi(xv.w), a);
  return a;
}

// ---- tensor-core dot products of bf16 rows with one token (batch 1) ----
//
// A row segment of 256 bf16 weights w[0..256) is one 16x16 A tile of
// mma.m16n8k16 with A[i][k] = w[8i + k] (k < 8) and w[128 + 8i + k - 8]
// (k >= 8): one ldmatrix.x4 reads it as a contiguous 512-byte block (lane L
// points at byte 16L), so the read is free of bank conflicts. B holds x in the
// matching positions: B0[k][j] pairs with A row j (j < 8) and B1[k][j] with A
// row 8 + j. The dot product of the segment is the sum of the diagonal
// D0[i][i] + D1[8+j][j]; summed over segments the diagonals accumulate the
// full row. Products of bf16 are exact in fp32; accumulation is fp32.
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& a0, uint32_t& a1, uint32_t& a2,
                                            uint32_t& a3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// B fragments of x for one 256-element segment (4 words per lane):
// lane (g = lane/4, t = lane%4) needs bf16 pairs at 8g + 2t + {0, 128}
// (B0) and 64 + 8g + 2t + {0, 128} (B1).
__device__ __forceinline__ void x_frag(const uint16_t* xseg, int lane, uint32_t (&b)[4]) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(xseg);
  const int o = (8 * (lane >> 2) + 2 * (lane & 3)) >> 1;
  b[0] = w[o];
  b[1] = w[o + 64];
  b[2] = w[o + 32];
  b[3] = w[o + 96];
}

// Sum the diagonals of D0 and D1 held by this lane (lanes 4g + g/2).
__device__ __forceinline__ float diag_part(const float (&d0)[4], const float (&d1)[4], int lane) {
  const int g = lane >> 2, t = lane & 3;
  if (t != (g >> 1)) return 0.f;
  return (g & 1) ? (d0[1] + d1[3]) : (d0[0] + d1[2]);
}

// int4: two's-complement nibble j of word w (elements 8m..8m+7 of a row live
// in one 32-bit word, element 2i in the low nibble of byte i) -> float q.
// (w ^ 0x88888888) turns q into q + 8 in [0, 15]; OR-ing that into the
// mantissa of 2^23 gives 2^23 + q + 8 exactly; subtracting 2^23 + 8 leaves q.
// a - b on packed bf16 pairs (round to nearest)
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Codes i and i + 4 of an int4 word (two's complement nibbles, element 8 v + i
// in bits 4 i .. 4 i + 3) as a bf16 pair {lo: code i, hi: code i + 4}, exact:
// the nibble flipped to c + 8 fills the low mantissa bits of 128.0, and
// 136 is taken off.
__device__ __forceinline__ uint32_t int4_pair_bf16(uint32_t w, int i) {
  const uint32_t t = ((w ^ 0x88888888u) >> (4 * i)) & 0x000F000Fu;
  return bf16x2_sub(t | 0x43004300u, 0x43084308u);
}

__device__ __forceinline__ void int4x8_to_f(uint32_t w, float* q) {
  const uint32_t t = w ^ 0x88888888u;
#pragma unroll
  for (int j = 0; j < 8; ++j) q[j] = __uint_as_float(0x4B000000u | ((t >> (4 * j)) & 0xFu)) - 8388616.0f;
}

}  // namespace moedec
