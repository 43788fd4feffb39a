// Rank-32 recovery of the dropped channels of the channel-sparse reader
// (review of arXiv:2610.37386, "가중치만으로 만든 reader", step 3, eq. 2):
//   y_hat = sum_{kept j} w_j a_j d_j + U sum_{dropped j} w_j p_j b_j,
// U = the top 32 left singular vectors of the layer's stacked down columns
// D = [d_1 ... d_n] (n = E * I), b_j = U^T d_j (32 coefficients per channel,
// stored as fp16: 64 bytes against the channel's 12 KB, the page's ~0.5% of
// resident memory), p_j = SiLU(g_hat_j) v_hat_j the screen's estimate.
//
// Load time (once per layer):
//   gram_kernel       C = D D^T (H x H, fp32 sums of exact bf16 products),
//                     one 64 x 64 tile of the upper triangle per CTA;
//   subspace_mul_kernel + subspace_qr_kernel
//                     subspace iteration Q <- orth(C Q), 32 columns, a fixed
//                     number of rounds; the orthonormalisation is CholeskyQR2
//                     in fp64 in one CTA. span(Q) -> the top-32 eigenspace of
//                     C = the top-32 left singular subspace of D at the rate
//                     (lambda_33 / lambda_32)^rounds. Eq. 2 depends on U only
//                     through U U^T, so any orthonormal basis of the subspace
//                     gives the same output.
//   coeff_kernel      b_j = U^T d_j for every channel, fp16.
// Decode time, per token: recover_kernel adds U r to y with
//   r = sum over the routed candidates (e, c) not in the kept list of
//       w_e SiLU(g_hat) v_hat b_{e*I+c}.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace moedec {

constexpr int kRecRank = MOE_RECOVERY_RANK;  // 32
constexpr int kGramTile = 64;
constexpr int kGramChunk = 32;                // channels per shared-memory chunk
constexpr int kRecRounds = 12;                // subspace iterations

// C[h1, h2] = sum_j d_j[h1] d_j[h2]; d_j = row 2 of channel j of cm [n][3][H].
// CTA (ti, tj), ti <= tj, over blockIdx.x in the upper triangle; 256 threads,
// thread t computes the 4 x 4 outputs (4 (t / 16) + a, 4 (t % 16) + b).
__global__ void __launch_bounds__(256) gram_kernel(const uint16_t* __restrict__ cm, int H, int n,
                                                   float* __restrict__ C) {
  __shared__ float As[kGramChunk][kGramTile + 4];
  __shared__ float Bs[kGramChunk][kGramTile + 4];
  const int nt = H / kGramTile;
  // blockIdx.x -> (ti, tj) of the upper triangle, row by row
  int t = blockIdx.x, ti = 0;
  while (t >= nt - ti) { t -= nt - ti; ++ti; }
  const int tj = ti + t;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
  const size_t cstride = 3 * (size_t)H;
  for (int j0 = 0; j0 < n; j0 += kGramChunk) {
    // 32 channels x 64 columns of each tile: 2048 bf16 per tile, 8 per thread
    for (int i = tid; i < kGramChunk * kGramTile / 8; i += 256) {
      const int jj = i / (kGramTile / 8), c8 = (i % (kGramTile / 8)) * 8;
      float fa[8], fb[8];
      if (j0 + jj < n) {
        const uint16_t* d = cm + (size_t)(j0 + jj) * cstride + 2 * (size_t)H;
        unpack8(*reinterpret_cast<const uint4*>(d + ti * kGramTile + c8), fa);
        unpack8(*reinterpret_cast<const uint4*>(d + tj * kGramTile + c8), fb);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) { fa[e] = 0.f; fb[e] = 0.f; }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) { As[jj][c8 + e] = fa[e]; Bs[jj][c8 + e] = fb[e]; }
    }
    __syncthreads();
#pragma unroll 8
    for (int jj = 0; jj < kGramChunk; ++jj) {
      float a4[4], b4[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) { a4[a] = As[jj][4 * ty + a]; b4[a] = Bs[jj][4 * tx + a]; }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(a4[a], b4[b], acc[a][b]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int r = ti * kGramTile + 4 * ty + a, c = tj * kGramTile + 4 * tx + b;
      C[(size_t)r * H + c] = acc[a][b];
      C[(size_t)c * H + r] = acc[a][b];
    }
}

// Deterministic start of the subspace iteration: Q0[h, i] in [-1, 1) from a
// counter hash (splitmix64 of h * 32 + i); any start not orthogonal to the
// target subspace converges.
__global__ void subspace_init_kernel(int H, double* __restrict__ Q) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= H * kRecRank) return;
  unsigned long long z = (unsigned long long)i + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z ^= z >> 31;
  Q[i] = (double)(z >> 11) * (1.0 / 4503599627370496.0) - 1.0;  // 2^52
}

// Y = C Q: one warp per row h of C, lane i < 32 owns column i; C rows are
// read coalesced and broadcast through shared memory, Q (fp64, H x 32) is
// read by lane i along its column.
__global__ void __launch_bounds__(256) subspace_mul_kernel(const float* __restrict__ C, int H,
                                                           const double* __restrict__ Q, double* __restrict__ Y) {
  __shared__ float crow[8][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x * 8 + warp;
  if (h >= H) return;
  double acc = 0.0;
  for (int k0 = 0; k0 < H; k0 += 256) {
    for (int t = lane; t < 256; t += 32) crow[warp][t] = (k0 + t < H) ? C[(size_t)h * H + k0 + t] : 0.f;
    __syncwarp();
    const int kn = min(256, H - k0);
    for (int t = 0; t < kn; ++t) acc = fma((double)crow[warp][t], Q[(size_t)(k0 + t) * kRecRank + lane], acc);
    __syncwarp();
  }
  Y[(size_t)h * kRecRank + lane] = acc;
}

// Q = orth(Y) by CholeskyQR2 in fp64, one CTA of 256 threads: G = Y^T Y,
// G = L L^T, Y <- Y L^-T, twice. Y is overwritten with Q (H x 32).
__global__ void __launch_bounds__(256) subspace_qr_kernel(int H, double* __restrict__ Y) {
  __shared__ double G[kRecRank][kRecRank + 1];
  __shared__ double L[kRecRank][kRecRank + 1];
  const int tid = threadIdx.x;
  for (int pass = 0; pass < 2; ++pass) {
    for (int idx = tid; idx < kRecRank * kRecRank; idx += 256) {
      const int a = idx >> 5, b = idx & 31;
      double s = 0.0;
      for (int h = 0; h < H; ++h) s = fma(Y[(size_t)h * kRecRank + a], Y[(size_t)h * kRecRank + b], s);
      G[a][b] = s;
    }
    __syncthreads();
    if (tid < 32) {
      // Cholesky G = L L^T, one warp, column by column (lane = row)
      const int r = tid;
      for (int c = 0; c < kRecRank; ++c) {
        double v = G[r][c];
        for (int m = 0; m < c; ++m) v -= L[r][m] * L[c][m];
        __syncwarp();
        if (r == c) L[c][c] = sqrt(fmax(v, 1e-300));
        __syncwarp();
        if (r > c) L[r][c] = v / L[c][c];
        if (r < c) L[r][c] = 0.0;
        __syncwarp();
      }
    }
    __syncthreads();
    // row h of Y: solve q L^T = y (forward substitution over the 32 columns)
    for (int h = tid; h < H; h += 256) {
      double q[kRecRank];
#pragma unroll
      for (int c = 0; c < kRecRank; ++c) {
        double v = Y[(size_t)h * kRecRank + c];
#pragma unroll
        for (int m = 0; m < c; ++m) v -= q[m] * L[c][m];
        q[c] = v / L[c][c];
      }
#pragma unroll
      for (int c = 0; c < kRecRank; ++c) Y[(size_t)h * kRecRank + c] = q[c];
    }
    __syncthreads();
  }
}

__global__ void subspace_store_kernel(int H, const double* __restrict__ Q, float* __restrict__ U) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < H * kRecRank) U[i] = (float)Q[i];
}

// b_j = U^T d_j for every channel j: one warp per channel, d_j staged in
// shared memory, lane i accumulates coefficient i over h (U read along its
// column, L1/L2 resident), written as fp16 (round to nearest).
__global__ void __launch_bounds__(256) coeff_kernel(const uint16_t* __restrict__ cm, int H, int n,
                                                    const float* __restrict__ U, uint16_t* __restrict__ coeffs) {
  __shared__ __align__(16) uint16_t ds[8][2048];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int j = blockIdx.x * 8 + warp; j < n; j += gridDim.x * 8) {
    const uint16_t* d = cm + (size_t)j * 3 * H + 2 * (size_t)H;
    for (int v = lane; v < H / 8; v += 32)
      reinterpret_cast<uint4*>(ds[warp])[v] = *reinterpret_cast<const uint4*>(d + 8 * v);
    __syncwarp();
    float acc = 0.f;
    for (int h = 0; h < H; ++h) acc = fmaf(U[(size_t)h * kRecRank + lane], bf16_to_f(ds[warp][h]), acc);
    coeffs[(size_t)j * kRecRank + lane] = __half_as_ushort(__float2half_rn(acc));
    __syncwarp();
  }
}

// Decode time, token b = blockIdx.x (256 threads): candidates q = t * I + c
// (slot t of ids[b], channel c); the kept list (indices e * I + c) marks the
// kept ones in a shared bitmap; every other candidate adds
// w[b, t] SiLU(g_hat) v_hat b_{e*I+c} to r (est [B, k, I, 2] from the
// screen); then y[b] += U r. ids distinct and < E (checked on the host side
// of the layer call that produced the kept list).
__global__ void __launch_bounds__(256) recover_kernel(int H, int E, int I, int k, const int32_t* __restrict__ ids,
                                                      const float* __restrict__ w, const float* __restrict__ est,
                                                      const int32_t* __restrict__ kept, int keep,
                                                      const float* __restrict__ U, const uint16_t* __restrict__ coeffs,
                                                      float* __restrict__ y) {
  __shared__ uint32_t keptbits[kMaxCand / 32];
  __shared__ int ids_s[kMaxK];
  __shared__ float w_s[kMaxK];
  __shared__ float rpart[8][kRecRank];
  __shared__ float r_s[kRecRank];
  const int b = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = k * I;
  for (int i = tid; i < (N + 31) / 32; i += 256) keptbits[i] = 0u;
  if (tid < k) { ids_s[tid] = ids[b * k + tid]; w_s[tid] = w[b * k + tid]; }
  __syncthreads();
  for (int i = tid; i < keep; i += 256) {
    const int j = kept[(size_t)b * keep + i];
    const int e = j / I, c = j - e * I;
    for (int t = 0; t < k; ++t)
      if (ids_s[t] == e) { atomicOr(&keptbits[(t * I + c) >> 5], 1u << ((t * I + c) & 31)); break; }
  }
  __syncthreads();
  float r[kRecRank];
#pragma unroll
  for (int i = 0; i < kRecRank; ++i) r[i] = 0.f;
  for (int q = tid; q < N; q += 256) {
    if ((keptbits[q >> 5] >> (q & 31)) & 1u) continue;
    const int t = q / I, c = q - t * I;
    const int e = ids_s[t];
    if (e < 0 || e >= E) continue;
    const float2 gv = *reinterpret_cast<const float2*>(est + (((size_t)b * k + t) * I + c) * 2);
    const float s = w_s[t] * silu_f(gv.x) * gv.y;
    const uint4* cf = reinterpret_cast<const uint4*>(coeffs + ((size_t)e * I + c) * kRecRank);
#pragma unroll
    for (int v = 0; v < kRecRank / 8; ++v) {
      const uint4 u = cf[v];
      const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wd[m]));
        r[8 * v + 2 * m] = fmaf(s, f.x, r[8 * v + 2 * m]);
        r[8 * v + 2 * m + 1] = fmaf(s, f.y, r[8 * v + 2 * m + 1]);
      }
    }
  }
  // r summed over the CTA: within each warp, then over the 8 warps
#pragma unroll
  for (int i = 0; i < kRecRank; ++i) {
    const float v = warp_sum(r[i]);
    if (lane == 0) rpart[warp][i] = v;
  }
  __syncthreads();
  if (tid < kRecRank) {
    float v = 0.f;
    for (int wi = 0; wi < 8; ++wi) v += rpart[wi][tid];
    r_s[tid] = v;
  }
  __syncthreads();
  for (int h = tid; h < H; h += 256) {
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < kRecRank; ++i) acc = fmaf(U[(size_t)h * kRecRank + i], r_s[i], acc);
    y[(size_t)b * H + h] += acc;
  }
}

}  // namespace moedec
