// Weight-only channel screen of the channel-sparse reader: the rotated
// ternary sketch of every channel's gate and up rows, built once per layer
// from the weights, and the per-token screen that turns it into output-unit
// scores for the top-keep selection ([Reader] "가중치만으로 만든 reader",
// step 1 and step 2, eq. 1).
#pragma once

#include <cuda_fp16.h>

#include "screen_lut.cuh"
#include "small_kernels.cuh"

namespace moedec {

constexpr int kRdBlock = 128;        // coordinates per rotation block
constexpr int kRdMaxWords = 4;       // 2-bit code words per lane and row (H <= 2048)
constexpr int kRdScreenThreads = 256;

// Sketch builder: one CTA of 128 threads per channel j = e*I + c of a
// channel-major layer [E][I][3][H] bf16 (gate row, up row, down column).
// For the gate and the up row, block by block (thread t = coordinate t):
//   u = H_128 (s * v) in fp64 by the Sylvester butterfly (unnormalised, so
//       R v = u / sqrt(128) for the orthogonal R = H_128 diag(s) / sqrt(128));
//       every sum is exact while the block's bf16 values span < 2^38;
//   delta = 0.7 * (sum |u| / 128); code = sign(u) where |u| > delta, else 0;
//   scale = fp16(fp32(sum of |u| over the coded coordinates / their count));
//   rho = sum((u - scale * code)^2) / 128 / 128 (mean squared error of the
//       block in the orthogonal rotation's units).
// Codes of row r of channel j: words (2j + r) * H/16 .., coordinate h at
// bits 2(h % 16) (nonzero) and 2(h % 16) + 1 (negative) of word h / 16.
// dnorm[j] = fp32(sqrt(sum of the squared down column)), summed in fp64.
__global__ void __launch_bounds__(kRdBlock) reader_build_kernel(const uint16_t* __restrict__ cm,
                                                                const int8_t* __restrict__ signs, int H,
                                                                uint32_t* __restrict__ codes,
                                                                uint16_t* __restrict__ scales,
                                                                float* __restrict__ rho,
                                                                float* __restrict__ dnorm) {
  __shared__ double u[kRdBlock];
  __shared__ double red[3][kRdBlock / 32];
  __shared__ int rcnt[kRdBlock / 32];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const size_t j = blockIdx.x;
  const uint16_t* rows = cm + j * 3 * (size_t)H;
  const int nb = H / kRdBlock, words = H / 16;
  auto block_sum = [&](double v, int slot) -> double {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[slot][warp] = v;
    __syncthreads();
    return (red[slot][0] + red[slot][1]) + (red[slot][2] + red[slot][3]);
  };
  for (int r = 0; r < 2; ++r) {
    const uint16_t* v = rows + (size_t)r * H;
    const size_t row = 2 * j + r;
    for (int b = 0; b < nb; ++b) {
      const int h = b * kRdBlock + t;
      u[t] = (double)bf16_to_f(v[h]) * (double)signs[h];
      __syncthreads();
      // stage m: (x_i, x_{i+m}) <- (x_i + x_{i+m}, x_i - x_{i+m}) for i & m == 0
      for (int m = 1; m < kRdBlock; m <<= 1) {
        const double a = u[t], p = u[t ^ m];
        const double nv = (t & m) ? (p - a) : (a + p);
        __syncthreads();
        u[t] = nv;
        __syncthreads();
      }
      const double ut = u[t], au = fabs(ut);
      const double delta = 0.7 * (block_sum(au, 0) / 128.0);
      const bool nz = au > delta, neg = ut < 0.0;
      const double ssum = block_sum(nz ? au : 0.0, 1);
      int c = nz ? 1 : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
      if (lane == 0) rcnt[warp] = c;
      __syncthreads();
      const int cnt = rcnt[0] + rcnt[1] + rcnt[2] + rcnt[3];
      const double scale64 = cnt ? ssum / (double)cnt : 0.0;
      const __half s16 = __float2half_rn(__double2float_rn(scale64));
      const double sc = (double)__half2float(s16);
      const double err = ut - (nz ? (neg ? -sc : sc) : 0.0);
      const double esum = block_sum(err * err, 2);
      // 2-bit fields of 16 coordinates OR-ed into one word
      uint32_t bits = (nz ? (neg ? 3u : 1u) : 0u) << (2 * (t & 15));
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) bits |= __shfl_xor_sync(0xffffffffu, bits, o);
      if ((t & 15) == 0) codes[row * words + b * (kRdBlock / 16) + (t >> 4)] = bits;
      if (t == 0) {
        scales[row * nb + b] = __half_as_ushort(s16);
        rho[row * nb + b] = (float)(esum / 128.0 / 128.0);
      }
      __syncthreads();  // u and red are rewritten by the next block
    }
  }
  const uint16_t* d = rows + 2 * (size_t)H;
  double q = 0.0;
  for (int h = t; h < H; h += kRdBlock) {
    const double dv = (double)bf16_to_f(d[h]);
    q += dv * dv;
  }
  const double tot = block_sum(q, 0);
  if (t == 0) dnorm[j] = (float)sqrt(tot);
}

// Screen: token b = blockIdx.y; CTA x takes the contiguous candidates
// q in [x * k*I / G, (x + 1) * k*I / G) (slot q / I, channel q % I of expert
// ids[b, slot]):
//   g_hat = sum_blocks scale_b * (codes_b . ux_b) / 128, v_hat likewise,
//   scores[b, e, c] = w[b, slot] * dnorm[e*I + c] * |SiLU(g_hat) * v_hat|.
// The CTA first copies its candidates' code rows and scales into shared
// memory (cp.async through L2: one round trip for all of them, no registers
// held) and, while they land, rotates x_b, ux = H_128 (s * x_b) per block in
// fp32, into the table of subset sums of every 4 coordinates
// (screen_build_lut). Then warp w decodes candidates w, w + 8, ...: lane l
// takes code words l + 32 t of each row, 8 table lookups per word
// (screen_word). est_opt[b, slot, c] = {g_hat, v_hat} when given. Rows of
// unrouted experts, and of ids outside [0, E), are not written.
// Dynamic shared memory: ceil(k*I / G) * (H / 2 + H / 32) bytes.
__global__ void __launch_bounds__(kRdScreenThreads) reader_screen_kernel(
    const uint16_t* __restrict__ x, int H, int E, int I, int k, const int32_t* __restrict__ ids,
    const float* __restrict__ w, const int8_t* __restrict__ signs, const uint32_t* __restrict__ codes,
    const uint16_t* __restrict__ scales, const float* __restrict__ dnorm, float* __restrict__ scores,
    float* __restrict__ est) {
  __shared__ float lut[kLutFloats];
  __shared__ int ids_s[kMaxK];
  extern __shared__ __align__(16) uint32_t staged[];
  const int b = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int words = H / 16, nb = H / kRdBlock, cw = 2 * words;
  const int nq = k * I, G = gridDim.x;
  const int q0 = (int)((long long)blockIdx.x * nq / G), q1 = (int)((long long)(blockIdx.x + 1) * nq / G);
  const int n = q1 - q0;
  uint32_t* st_codes = staged;                                               // [n][2][words]
  uint16_t* st_scales = reinterpret_cast<uint16_t*>(staged + (size_t)n * cw);  // [n][2][nb]
  // x_b (s * x) into registers while the ids arrive
  float xv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int h = 8 * tid + i;
    xv[i] = h < H ? bf16_to_f(x[(size_t)b * H + h]) * (float)signs[h] : 0.f;
  }
  if (tid < k) ids_s[tid] = __ldg(ids + b * k + tid);
  __syncthreads();
  auto chan = [&](int q) -> int {  // channel e*I + c of candidate q, or -1
    const int slot = q / I, e = ids_s[slot];
    return (unsigned)e < (unsigned)E ? e * I + (q - slot * I) : -1;
  };
  // warp w copies candidates w, w + 8, ...: their two code rows (16-byte
  // pieces, lane l taking pieces l + 32 i) and two scale rows (4-byte pieces)
  for (int i = warp; i < n; i += kRdScreenThreads / 32) {
    const int j = chan(q0 + i);
    if (j < 0) continue;  // warp-uniform
    for (int o = lane; o < cw / 4; o += 32)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(st_codes + (size_t)i * cw + 4 * o)),
                   "l"(codes + (size_t)j * cw + 4 * o)
                   : "memory");
    for (int o = lane; o < nb; o += 32)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(st_scales + (size_t)i * 2 * nb + 2 * o)),
                   "l"(scales + (size_t)j * 2 * nb + 2 * o)
                   : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  screen_rotate_lut(H, xv, lut);
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  for (int i = warp; i < n; i += kRdScreenThreads / 32) {
    const int q = q0 + i, j = chan(q);
    if (j < 0) continue;  // warp-uniform
    const uint32_t* cr = st_codes + (size_t)i * cw;
    const uint16_t* sr = st_scales + (size_t)i * 2 * nb;
    float acc[2] = {0.f, 0.f};
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int t = 0; t < kRdMaxWords; ++t) {
        const int wd = lane + 32 * t;
        if (wd < words)
          acc[r] = fmaf(__half2float(__ushort_as_half(sr[r * nb + (wd >> 3)])), screen_word(lut, wd, cr[r * words + wd]),
                        acc[r]);
      }
    const float g = warp_sum(acc[0]) * (1.0f / 128.0f), v = warp_sum(acc[1]) * (1.0f / 128.0f);
    if (lane == 0) {
      const int slot = q / I, c = q - slot * I;
      scores[((size_t)b * E + ids_s[slot]) * I + c] = __ldg(w + b * k + slot) * __ldg(dnorm + j) * fabsf(silu_f(g) * v);
      if (est != nullptr) {
        float* o = est + (((size_t)b * k + slot) * I + c) * 2;
        o[0] = g;
        o[1] = v;
      }
    }
  }
}

// ---------------------------------------------------------------- partial screen
//
// [Reader] "가중치만으로 만든 reader", step 1, partial scan: at low budgets the
// screen reads, in each block of 128 rotated coordinates, only the codes of
// the m (80 on the page) coordinates with the largest |R x|. In the
// channel-major code layout a block's 128 codes of one row are a single
// 32-byte sector, so skipping coordinates saves nothing; in the
// coordinate-major layout below the codes of one coordinate of all of an
// expert's channels are contiguous, so a skipped coordinate is bytes not read.

// Coordinate-major codes: [E][2][H][I/16] uint32, coordinate h of row r of
// expert e, channel c at bits 2(c % 16) (nonzero) and 2(c % 16) + 1
// (negative) of word c / 16 -- the same 2-bit code as the channel-major
// sketch, transposed. One thread per output word (load time).
__global__ void reader_cmaj_kernel(const uint32_t* __restrict__ codes, int E, int I, int H,
                                   uint32_t* __restrict__ codes_cmaj) {
  const int wpr = I / 16, wpc = H / 16;
  const size_t total = (size_t)E * 2 * H * wpr;
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += (size_t)gridDim.x * blockDim.x) {
    const int w = (int)(idx % wpr);
    const size_t t = idx / wpr;
    const int h = (int)(t % H);
    const size_t er = t / H;
    const int r = (int)(er % 2), e = (int)(er / 2);
    uint32_t bits = 0u;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const size_t j = (size_t)e * I + 16 * w + i;
      const uint32_t word = __ldg(codes + (j * 2 + r) * wpc + (h >> 4));
      bits |= ((word >> (2 * (h & 15))) & 3u) << (2 * i);
    }
    codes_cmaj[idx] = bits;
  }
}

// Partial screen: CTA (slot t, token b), (I/16) x (H/128) threads: thread
// (w = tid % (I/16), block bl = tid / (I/16)) handles code word w (channels
// 16w .. 16w + 15) in block bl. The token is rotated in fp64 (every sum of
// the bf16 inputs is exact there), so the m largest |u_x| of each block --
// ties to the lower coordinate -- are exactly the oracle's choice; the kept
// coordinates' codes are then read (one coalesced word per lane and
// coordinate) and accumulated in fp32 against u_x, scaled per block by the
// channel's fp16 scale, and summed over blocks:
//   g_hat = sum_bl scale_bl * sum_{h kept in bl} code_h u_x,h / 128,
// likewise v_hat; scores[b, e, c] = w[b, t] dnorm[e*I + c] |SiLU(g_hat) v_hat|
// and est_opt[b, t, c] = {g_hat, v_hat}. Rows of unrouted experts and ids
// outside [0, E) are not written.
__global__ void __launch_bounds__(1024) reader_screen_partial_kernel(
    const uint16_t* __restrict__ x, int H, int E, int I, int k, const int32_t* __restrict__ ids,
    const float* __restrict__ w, const int8_t* __restrict__ signs, const uint32_t* __restrict__ codes_cmaj,
    const uint16_t* __restrict__ scales, const float* __restrict__ dnorm, int m, float* __restrict__ scores,
    float* __restrict__ est) {
  __shared__ double u64[2048];
  __shared__ float uf[2048];
  __shared__ short kc[16][128];
  __shared__ int nkc[16];
  __shared__ float gsum[1024], vsum[1024];
  const int t = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, nt = blockDim.x;
  const int e = __ldg(ids + b * k + t);
  if (e < 0 || e >= E) return;  // uniform over the CTA
  const int wpr = I / 16, nb = H / kRdBlock;
  for (int i = tid; i < H; i += nt) u64[i] = (double)bf16_to_f(x[(size_t)b * H + i]) * (double)signs[i];
  for (int i = tid; i < I; i += nt) { gsum[i] = 0.f; vsum[i] = 0.f; }
  __syncthreads();
  for (int lg = 0; lg < 7; ++lg) {
    const int mm = 1 << lg;
    for (int p = tid; p < H / 2; p += nt) {
      const int i = ((p >> lg) << (lg + 1)) | (p & (mm - 1));
      const double a0 = u64[i], a1 = u64[i + mm];
      u64[i] = a0 + a1;
      u64[i + mm] = a0 - a1;
    }
    __syncthreads();
  }
  // keep flag of each coordinate: fewer than m of its block beat it
  for (int i = tid; i < H; i += nt) {
    const int blk = i / kRdBlock, o = i - blk * kRdBlock;
    const double ai = fabs(u64[i]);
    int beat = 0;
    for (int j = 0; j < kRdBlock; ++j) {
      const double aj = fabs(u64[blk * kRdBlock + j]);
      beat += (aj > ai) || (aj == ai && j < o);
    }
    uf[i] = (float)u64[i];
    kc[blk][o] = (short)(beat < m ? 1 : 0);
  }
  __syncthreads();
  if (tid < nb) {  // each block's kept coordinates, ascending
    int n = 0;
    for (int o = 0; o < kRdBlock; ++o)
      if (kc[tid][o]) kc[tid][n++] = (short)(tid * kRdBlock + o);
    nkc[tid] = n;
  }
  __syncthreads();
  const int wd = tid % wpr, bl = tid / wpr;
  if (bl < nb) {
    const int n = nkc[bl];
    for (int r = 0; r < 2; ++r) {
      const uint32_t* cw = codes_cmaj + ((size_t)e * 2 + r) * H * wpr + wd;
      float acc[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = 0.f;
      for (int q = 0; q < n; ++q) {
        const int h = kc[bl][q];
        const uint32_t word = __ldg(cw + (size_t)h * wpr);
        const float xv = uf[h];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t sgn = (word << (30 - 2 * i)) & 0x80000000u;
          const float v = __uint_as_float(__float_as_uint(xv) ^ sgn);
          acc[i] += ((word >> (2 * i)) & 1u) ? v : 0.f;
        }
      }
      float* dst = r ? vsum : gsum;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int c = 16 * wd + i;
        const float sc = __half2float(__ushort_as_half(__ldg(scales + (((size_t)e * I + c) * 2 + r) * nb + bl)));
        atomicAdd(&dst[c], sc * acc[i]);
      }
    }
  }
  __syncthreads();
  const float wt = __ldg(w + b * k + t);
  for (int c = tid; c < I; c += nt) {
    const float gh = gsum[c] * (1.0f / 128.0f), vh = vsum[c] * (1.0f / 128.0f);
    scores[((size_t)b * E + e) * I + c] = wt * __ldg(dnorm + (size_t)e * I + c) * fabsf(silu_f(gh) * vh);
    if (est != nullptr) {
      float* o = est + (((size_t)b * k + t) * I + c) * 2;
      o[0] = gh;
      o[1] = vh;
    }
  }
}

}  // namespace moedec
