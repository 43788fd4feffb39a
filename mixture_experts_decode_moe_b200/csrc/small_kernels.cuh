// Small, non-persistent kernels: the standalone router (GEMV + top-k for up to
// 256 tokens) and the touched-expert counting sort.
#pragma once

#include "decode_kernel.cuh"

namespace moedec {

// logits[b, e] = router[e, :] . x[b, :] for a tile of 8 router rows (one per
// warp) and up to 8 tokens (blockIdx.y). fp32 accumulation.
__global__ void __launch_bounds__(kThreads) router_logits_kernel(const uint16_t* __restrict__ x,
                                                                 const uint16_t* __restrict__ router, int B,
                                                                 int H, int E, float* __restrict__ logits) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint4* xs4 = reinterpret_cast<uint4*>(sm);
  const int H8 = H >> 3, b0 = blockIdx.y * kMaxB, nb = min(kMaxB, B - b0);
  for (int i = threadIdx.x; i < nb * H8; i += kThreads)
    xs4[i] = reinterpret_cast<const uint4*>(x + (size_t)b0 * H)[i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * kWarps + warp;
  if (e >= E) return;
  const uint4* row = reinterpret_cast<const uint4*>(router + (size_t)e * H);
  float part[kMaxB];
#pragma unroll
  for (int b = 0; b < kMaxB; ++b) part[b] = 0.f;
  for (int v = lane; v < H8; v += 32) {
    const uint4 wv = __ldg(row + v);
#pragma unroll
    for (int b = 0; b < kMaxB; ++b)
      if (b < nb) part[b] += dot8_bf16(wv, xs4[b * H8 + v]);
  }
#pragma unroll
  for (int b = 0; b < kMaxB; ++b)
    if (b < nb) {
      const float s = warp_sum(part[b]);
      if (lane == 0) logits[(size_t)(b0 + b) * E + e] = s;
    }
}

// One warp per token: top-k (ties -> lowest index), renormalised weights, margin.
__global__ void __launch_bounds__(kThreads) topk_kernel(const float* __restrict__ logits, int B, int E, int k,
                                                        int32_t* ids, float* w, float* margin) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(sm);
  __shared__ int pos_s[kWarps][kMaxK + 1];
  __shared__ float l_s[kWarps][kMaxK + 1];
  __shared__ float w_s[kWarps][kMaxK];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x * kWarps + warp;
  if (b >= B) return;
  uint32_t* kw = keys + warp * E;
  const float* lb = logits + (size_t)b * E;
  for (int i = lane; i < E; i += 32) kw[i] = float_key(lb[i]);
  __syncwarp();
  const int kk = (k < E) ? k + 1 : k;
  warp_select(kw, E, kk, pos_s[warp]);
  __syncwarp();
  for (int i = lane; i < kk; i += 32) l_s[warp][i] = key_float(kw[pos_s[warp][i]]);
  __syncwarp();
  warp_weights(l_s[warp], k, w_s[warp]);
  __syncwarp();
  for (int i = lane; i < k; i += 32) {
    ids[(size_t)b * k + i] = pos_s[warp][i];
    w[(size_t)b * k + i] = w_s[warp][i];
  }
  if (lane == 0 && margin != nullptr) margin[b] = (k < E) ? l_s[warp][k - 1] - l_s[warp][k] : INFINITY;
}

// Stable counting sort of the (token, slot) pairs by expert, one CTA.
// Invalid ids (out of range or repeated in a token) set count = -1.
__global__ void __launch_bounds__(kThreads) touched_kernel(const int32_t* __restrict__ ids, int B, int k, int E,
                                                           int32_t* count, uint32_t* bitmap, int32_t* offsets,
                                                           int32_t* pairs) {
  __shared__ int cnt[kMaxE];
  __shared__ int cursor[kMaxE];
  __shared__ int scratch[kWarps + 1];
  __shared__ int bad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int P = B * k;
  for (int e = tid; e < E; e += kThreads) cnt[e] = 0;
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int p = tid; p < P; p += kThreads) {
    const int e = ids[p];
    if (e < 0 || e >= E) { bad = 1; continue; }
    atomicAdd(&cnt[e], 1);
    // a repeat inside one token: another slot of the same token with the same id
    for (int s = 0; s < k; ++s) {
      const int q = (p / k) * k + s;
      if (q != p && ids[q] == e) bad = 1;
    }
  }
  __syncthreads();
  // exclusive scan of cnt over E (E <= 1024: 4 per thread)
  const int per = (E + kThreads - 1) / kThreads;
  const int lo = min(E, tid * per), hi = min(E, lo + per);
  int loc = 0, touched = 0;
  for (int e = lo; e < hi; ++e) { loc += cnt[e]; touched += cnt[e] > 0; }
  int tot;
  int base = block_excl_scan(loc, scratch, &tot);
  int tcount;
  block_excl_scan(touched, scratch, &tcount);
  for (int e = lo; e < hi; ++e) {
    cursor[e] = base;
    if (offsets != nullptr) offsets[e] = base;
    base += cnt[e];
  }
  if (tid == 0 && offsets != nullptr) offsets[E] = tot;
  if (bitmap != nullptr)
    for (int w = tid; w < (E + 31) / 32; w += kThreads) {
      uint32_t m = 0;
      for (int i = 0; i < 32 && w * 32 + i < E; ++i) m |= (cnt[w * 32 + i] > 0 ? 1u : 0u) << i;
      bitmap[w] = m;
    }
  __syncthreads();
  if (tid == 0) *count = bad ? -1 : tcount;
  if (pairs == nullptr || bad) return;
  // placement in pair order: chunks of 256 pairs, warp by warp
  for (int c0 = 0; c0 < P; c0 += kThreads) {
    const int p = c0 + tid;
    const int e = p < P ? ids[p] : -1;
    const uint32_t same = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(same & ((1u << lane) - 1u));
    for (int w = 0; w < kWarps; ++w) {
      if (warp == w && p < P) {
        pairs[cursor[e] + rank] = p;
        __syncwarp(same);
        if (rank == 0) cursor[e] += __popc(same);
      }
      __syncthreads();
    }
  }
}

}  // namespace moedec
