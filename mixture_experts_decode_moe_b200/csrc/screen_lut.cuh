// The channel screen's rotation of the token and its subset-sum table, shared
// by the per-token screen kernel and the screen inside the channel stack
// ([Reader] "가중치만으로 만든 reader", steps 1-2, eq. 1).
//
// A code word holds the 2-bit ternary codes of 16 rotated coordinates
// (coordinate h at bits 2(h % 16): nonzero and 2(h % 16) + 1: negative of
// word h / 16). Its contribution to an estimate is the sum of +ux over the
// positive and -ux over the negative coordinates. Instead of decoding the 16
// codes one by one (7 integer-heavy instructions each, and the screen is
// bound by instruction issue), the word is split into a positive and a
// negative 4-bit mask per group of 4 coordinates, and a table of the 16
// subset sums of every group's ux turns each mask into one lookup: 8 lookups
// per word, laid out so that a warp's lookups never share a bank.
#pragma once

#include "common.cuh"

namespace moedec {

constexpr int kLutFloats = 4 * 2048;  // 16 entries per 4 coordinates, H <= 2048

// Table slot of entry m of group g = h / 4. The lane that decodes code word
// wd = g / 4 is wd % 32 (words wd % 32 + 32 t), so every entry of the word's
// groups sits in that lane's bank: slot = 32 (16 (4 t + g % 4) + m) + wd % 32,
// t = wd / 32. The 32 lanes of a lookup then always hit 32 different banks.
__device__ __forceinline__ int lut_slot(int g, int m) {
  const int wd = g >> 2;
  return 32 * (16 * (4 * (wd >> 5) + (g & 3)) + m) + (wd & 31);
}

// ux = H_128 (s * x) per block of 128 coordinates (unnormalised Sylvester
// transform), fp32, over the 256 threads of a CTA or of its consumer warps:
// thread t holds coordinates 8t .. 8t + 7 (a block is a half-warp), the
// stages of distance 1, 2 and 4 in registers, those of 8 .. 64 by shuffles
// with lanes t ^ 1 .. t ^ 8. Then lut[lut_slot(g, m)] = sum of ux_{4g + i}
// over the set bits i of m (at most 2 + 1 roundings). v holds s_h x_h of the
// thread's 8 coordinates (0 beyond H); H <= 2048, H % 128 == 0. The caller
// synchronises before reading lut.
__device__ __forceinline__ void screen_rotate_lut(int H, float (&v)[8], float* lut) {
  const int tid = threadIdx.x & 255, lane = tid & 31;
#pragma unroll
  for (int m = 1; m < 8; m <<= 1)
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (!(i & m)) {
        const float a = v[i], b = v[i + m];
        v[i] = a + b;
        v[i + m] = a - b;
      }
#pragma unroll
  for (int d = 1; d < 16; d <<= 1)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], d);
      v[i] = (lane & d) ? o - v[i] : v[i] + o;
    }
  if (8 * tid < H) {
#pragma unroll
    for (int hg = 0; hg < 2; ++hg) {
      const int g = 2 * tid + hg;
      const float s01[4] = {0.f, v[4 * hg], v[4 * hg + 1], v[4 * hg] + v[4 * hg + 1]};
      const float s23[4] = {0.f, v[4 * hg + 2], v[4 * hg + 3], v[4 * hg + 2] + v[4 * hg + 3]};
#pragma unroll
      for (int m = 0; m < 16; ++m) lut[lut_slot(g, m)] = s01[m & 3] + s23[m >> 2];
    }
  }
}
// The same, loading thread t's s_h x_h, h = 8t .. 8t + 7, through sx(h).
template <class SX>
__device__ __forceinline__ void screen_build_lut(int H, SX sx, float* lut) {
  const int tid = threadIdx.x & 255;
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = 8 * tid < H ? sx(8 * tid + i) : 0.f;
  screen_rotate_lut(H, v, lut);
}

// Sum of the code word wd's 16 signed coordinates of ux, from the table
// (called by lane wd % 32).
__device__ __forceinline__ float screen_word(const float* lut, int wd, uint32_t w) {
  const uint32_t nz = w & 0x55555555u, ng = (w >> 1) & 0x55555555u;
  uint32_t P = nz & ~ng, N = nz & ng;
  P = (P | (P >> 1)) & 0x33333333u;
  P = (P | (P >> 2)) & 0x0F0F0F0Fu;  // byte k: the positive coordinates 4k .. 4k + 3
  N = (N | (N >> 1)) & 0x33333333u;
  N = (N | (N >> 2)) & 0x0F0F0F0Fu;
  const float* t = lut + 32 * 16 * 4 * (wd >> 5) + (wd & 31);
  float pt = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    pt += t[32 * (16 * k + ((P >> (8 * k)) & 15u))] - t[32 * (16 * k + ((N >> (8 * k)) & 15u))];
  return pt;
}

}  // namespace moedec
