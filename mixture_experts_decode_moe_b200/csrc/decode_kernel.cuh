// Body of the persistent decode kernel (see decode.cuh for the design).
#pragma once

#include "decode.cuh"

namespace moedec {

// ---------------------------------------------------------------- block helpers

// Exclusive prefix sum over the CTA; `total` receives the sum. All threads call.
__device__ __forceinline__ int block_excl_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int t = lane < kWarps ? scratch[lane] : 0;
    int ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int u = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += u;
    }
    if (lane < kWarps) scratch[lane] = ti - t;
    if (lane == kWarps - 1) scratch[kWarps] = ti;
  }
  __syncthreads();
  int r = inc - v + scratch[warp];
  *total = scratch[kWarps];
  __syncthreads();
  return r;
}

// ---------------------------------------------------------------- top-k

// One warp selects the k largest of lg[0, E) (ties -> lowest index) in
// descending order, the renormalised softmax weights over them, and the gap
// between the k-th and (k+1)-th logit. E <= 1024, k <= 32.
__device__ __forceinline__ void warp_topk(const float* lg, int E, int k, int* ids, float* w,
                                          float* margin_out) {
  const int lane = threadIdx.x & 31;
  const int per = (E + 31) >> 5;
  const int lo = lane * per, hi = min(E, lo + per);
  uint32_t taken = 0, bk = 0;
  int bi = -1;
  auto rescan = [&]() {
    bk = 0;
    bi = -1;
    for (int i = lo; i < hi; ++i) {
      if ((taken >> (i - lo)) & 1u) continue;
      const uint32_t kk = float_key(lg[i]);
      if (bi < 0 || kk > bk) { bk = kk; bi = i; }
    }
  };
  rescan();
  float l0 = 0.f, lk = 0.f, mine = 0.f, margin = INFINITY;
  const int rounds = (k < E) ? k + 1 : k;
  for (int r = 0; r < rounds; ++r) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, bi >= 0 ? bk : 0u);
    const uint32_t ball = __ballot_sync(0xffffffffu, bi >= 0 && bk == m);
    const int win = __ffs(ball) - 1;
    const int idx = __shfl_sync(0xffffffffu, bi, win);
    const float val = key_float(m);
    if (r < k) {
      if (lane == 0) ids[r] = idx;
      if (lane == r) mine = val;
      if (r == 0) l0 = val;
      if (r == k - 1) lk = val;
    } else {
      margin = lk - val;
    }
    if (lane == win) {
      taken |= 1u << (idx - lo);
      rescan();
    }
  }
  const float e = (lane < k) ? expf(mine - l0) : 0.f;
  const float s = warp_sum(e);
  if (lane < k) w[lane] = e / s;
  if (lane == 0 && margin_out != nullptr) *margin_out = margin;
}

// ---------------------------------------------------------------- job compute

// Gate/up dot products of `n` channels of bf16 rows for the tokens in `mask`.
// Row (ch, mat) starts at stage + ch*ch_stride + mat*mat_stride (mat 0 = gate,
// 1 = up). dots[(2*ch + mat)*BMAX + b].
template <int BMAX>
__device__ __forceinline__ void dots_bf16(const uint8_t* stage, int n, int ch_stride, int mat_stride,
                                          const uint4* xs4, int H8, uint32_t mask, float* dots) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int pidx = warp; pidx < 2 * n; pidx += kWarps) {
    const int ch = pidx >> 1, mat = pidx & 1;
    const uint4* row = reinterpret_cast<const uint4*>(stage + ch * ch_stride + mat * mat_stride);
    float part[BMAX];
#pragma unroll
    for (int b = 0; b < BMAX; ++b) part[b] = 0.f;
    for (int v = lane; v < H8; v += 32) {
      const uint4 wv = row[v];
#pragma unroll
      for (int b = 0; b < BMAX; ++b)
        if ((mask >> b) & 1u) part[b] += dot8_bf16(wv, xs4[b * H8 + v]);
    }
#pragma unroll
    for (int b = 0; b < BMAX; ++b)
      if ((mask >> b) & 1u) {
        const float s = warp_sum(part[b]);
        if (lane == 0) dots[pidx * BMAX + b] = s;
      }
  }
}

// int4 gate/up rows: codes [n][H/2] at gc / uc, scales [n][H/64] bf16 at gs / us.
template <int BMAX>
__device__ __forceinline__ void dots_int4(const uint8_t* stage, int n, int H, int nch, const uint4* xs4,
                                          uint32_t mask, float* dots) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H8 = H >> 3, rowc = H >> 1, rows = H >> 5;  // code bytes / scale bytes per row
  const int gc = 0, uc = nch * rowc, gs = 3 * nch * rowc, us = gs + nch * rows;
  for (int pidx = warp; pidx < 2 * n; pidx += kWarps) {
    const int ch = pidx >> 1, mat = pidx & 1;
    const uint4* codes = reinterpret_cast<const uint4*>(stage + (mat ? uc : gc) + ch * rowc);
    const uint16_t* sc = reinterpret_cast<const uint16_t*>(stage + (mat ? us : gs) + ch * rows);
    float part[BMAX];
#pragma unroll
    for (int b = 0; b < BMAX; ++b) part[b] = 0.f;
    for (int v = lane; v < (H >> 5); v += 32) {  // 16-byte code vector = 32 elements
      const uint4 cv = codes[v];
      const float s = bf16_to_f(sc[v >> 1]);
      float q[4][8];
      int4x8_to_f(cv.x, q[0]);
      int4x8_to_f(cv.y, q[1]);
      int4x8_to_f(cv.z, q[2]);
      int4x8_to_f(cv.w, q[3]);
#pragma unroll
      for (int b = 0; b < BMAX; ++b)
        if ((mask >> b) & 1u) {
          float a = 0.f;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            float xf[8];
            unpack8(xs4[b * H8 + 4 * v + m], xf);
#pragma unroll
            for (int j = 0; j < 8; ++j) a = fmaf(q[m][j], xf[j], a);
          }
          part[b] = fmaf(s, a, part[b]);
        }
    }
#pragma unroll
    for (int b = 0; b < BMAX; ++b)
      if ((mask >> b) & 1u) {
        const float s = warp_sum(part[b]);
        if (lane == 0) dots[pidx * BMAX + b] = s;
      }
  }
}

// h[ch][b] = w_b * silu(g) * u for tokens in mask, 0 otherwise.
template <int BMAX>
__device__ __forceinline__ void swiglu_h(int n, uint32_t mask, const float* wts, const float* dots, float* hs) {
  for (int t = threadIdx.x; t < n * BMAX; t += kThreads) {
    const int ch = t / BMAX, b = t % BMAX;
    float h = 0.f;
    if ((mask >> b) & 1u) {
      const float g = dots[(2 * ch) * BMAX + b], u = dots[(2 * ch + 1) * BMAX + b];
      h = wts[b] * silu_f(g) * u;
    }
    hs[ch * BMAX + b] = h;
  }
}

// acc[b][0..8) += sum_ch h[ch][b] * D^T[ch][8v .. 8v+8) for bf16 down rows.
template <int BMAX>
__device__ __forceinline__ void down_bf16(const uint8_t* stage, int n, int ch_stride, int down_off, int H8,
                                          uint32_t mask, const float* hs, float (&acc)[BMAX][8]) {
  const int v = threadIdx.x;
  if (v >= H8) return;
  for (int ch = 0; ch < n; ++ch) {
    const uint4 dv = reinterpret_cast<const uint4*>(stage + down_off + ch * ch_stride)[v];
    float d[8];
    unpack8(dv, d);
#pragma unroll
    for (int b = 0; b < BMAX; ++b)
      if ((mask >> b) & 1u) {
        const float h = hs[ch * BMAX + b];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[b][i] = fmaf(h, d[i], acc[b][i]);
      }
  }
}

// int4 down rows: codes [n][H/2] at dc, one scale row [H] bf16 at ds (the job
// lies inside one 64-channel group, so the scale factors out of the job).
template <int BMAX>
__device__ __forceinline__ void down_int4(const uint8_t* stage, int n, int H, int nch, uint32_t mask,
                                          const float* hs, float (&acc)[BMAX][8]) {
  const int v = threadIdx.x, H8 = H >> 3, rowc = H >> 1;
  if (v >= H8) return;
  const int dc = 2 * nch * rowc, ds = 3 * nch * rowc + 2 * nch * (H >> 5);
  float s[8];
  unpack8(reinterpret_cast<const uint4*>(stage + ds)[v], s);
  float inner[BMAX][8];
#pragma unroll
  for (int b = 0; b < BMAX; ++b)
#pragma unroll
    for (int i = 0; i < 8; ++i) inner[b][i] = 0.f;
  for (int ch = 0; ch < n; ++ch) {
    const uint32_t wv = reinterpret_cast<const uint32_t*>(stage + dc + ch * rowc)[v];
    float q[8];
    int4x8_to_f(wv, q);
#pragma unroll
    for (int b = 0; b < BMAX; ++b)
      if ((mask >> b) & 1u) {
        const float h = hs[ch * BMAX + b];
#pragma unroll
        for (int i = 0; i < 8; ++i) inner[b][i] = fmaf(h, q[i], inner[b][i]);
      }
  }
#pragma unroll
  for (int b = 0; b < BMAX; ++b)
    if ((mask >> b) & 1u)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[b][i] = fmaf(s[i], inner[b][i], acc[b][i]);
}

// ---------------------------------------------------------------- the kernel

template <int BMAX, int WT, int LAYOUT>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ RouteSmem rs;
  __shared__ int route_ready_layer_s;
  __shared__ int bad_s, okw_s;
  __shared__ unsigned long long target_s;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int G = gridDim.x, cta = blockIdx.x;
  const int B = p.B, H = p.H, H8 = H >> 3, E = p.E, I = p.I, k = p.k;
  const int rowb = 2 * H;  // bf16 row bytes
  uint8_t* ring = smem;
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + p.off_x);
  const uint4* xs4 = reinterpret_cast<const uint4*>(xs);
  float* lg = reinterpret_cast<float*>(smem + p.off_lg);
  float* dots = reinterpret_cast<float*>(smem + p.off_dots);
  float* hs = reinterpret_cast<float*>(smem + p.off_hs);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + p.off_keys);
  int* kept = reinterpret_cast<int*>(smem + p.off_kept);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  WsControl* ctl = p.ctl;

  if (tid == 0) {
    for (int s = 0; s < p.nstages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
    route_ready_layer_s = -1;
  }
  // x_0 -> shared memory (and x_hist[0])
  for (int i = tid; i < B * H8; i += kThreads) {
    const uint4 v = reinterpret_cast<const uint4*>(p.x_in)[i];
    reinterpret_cast<uint4*>(xs)[i] = v;
  }
  if (p.x_hist != nullptr) {
    const long long n = (long long)B * H8;
    for (long long i = cta * n / G + tid; i < (cta + 1) * n / G; i += kThreads)
      reinterpret_cast<uint4*>(p.x_hist)[i] = reinterpret_cast<const uint4*>(p.x_in)[i];
  }
  __syncthreads();

  // ------------------------------------------------------------ producer (thread 0)
  JobCursor pcur;
  long long jp = 0;  // jobs issued
  long long jc = 0;  // jobs consumed
  uint64_t pol = 0;
  if (tid == 0) {
    pol = policy_evict_first();
    pcur.begin_layer(p, 0);
  }

  auto next_job = [&](JobCursor& cur, Job& j, int ready_layer) -> bool {
    for (;;) {
      if (cur.layer >= p.L) { j.type = JOB_END; return true; }
      if (cur.type == JOB_ROUTER) {
        const int n = (int)llmin(p.rows_per_job, cur.t1 - cur.t);
        j = Job{JOB_ROUTER, cur.layer, 0, (int)cur.t, n};
        cur.t += n;
        if (cur.t >= cur.t1) { cur.type = JOB_SHARED; cur.set_range(p); }
        return true;
      }
      if (cur.type == JOB_SHARED) {
        const int c = (int)cur.t;
        const int n = (int)llmin(p.nch_sh - c % p.nch_sh, cur.t1 - cur.t);
        j = Job{JOB_SHARED, cur.layer, 0, c, n};
        cur.t += n;
        if (cur.t >= cur.t1) { cur.type = JOB_ROUTED; cur.t = -1; cur.t1 = -1; }
        return true;
      }
      // routed
      if (cur.t1 < 0) {
        if (ready_layer != cur.layer) return false;
        cur.set_routed(LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR ? (long long)rs.ncand : (long long)rs.U * I);
      }
      if (cur.t >= cur.t1) { cur.begin_layer(p, cur.layer + 1); continue; }
      if (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR) {
        const int pos = (int)cur.t;
        const int j0 = kept[pos];
        int n = 1;
        while (n < p.nch && cur.t + n < cur.t1 && kept[pos + n] == j0 + n && (j0 + n) % I != 0) ++n;
        j = Job{JOB_ROUTED, cur.layer, pos, j0, n};
        cur.t += n;
      } else {
        const int u = (int)(cur.t / I), c = (int)(cur.t % I);
        const int n = (int)llmin(min(p.nch - c % p.nch, I - c), cur.t1 - cur.t);
        j = Job{JOB_ROUTED, cur.layer, u, c, n};
        cur.t += n;
      }
      return true;
    }
  };

  auto issue = [&](const Job& j, int slot) {
    uint64_t* bar = &full[slot];
    uint8_t* dst = ring + (size_t)slot * p.stage_bytes;
    const LayerW& Lw = p.layer[j.layer];
    if (j.type == JOB_ROUTER) {
      const uint32_t bytes = (uint32_t)j.n * rowb;
      mbar_expect_tx(bar, bytes);
      bulk_g2s(dst, Lw.router + (size_t)j.c0 * rowb, bytes, bar, pol);
    } else if (j.type == JOB_SHARED) {
      const uint32_t bytes = (uint32_t)j.n * rowb;
      mbar_expect_tx(bar, 3 * bytes);
      const size_t off = (size_t)j.c0 * rowb;
      bulk_g2s(dst, Lw.sh_gate + off, bytes, bar, pol);
      bulk_g2s(dst + p.nch_sh * rowb, Lw.sh_up + off, bytes, bar, pol);
      bulk_g2s(dst + 2 * p.nch_sh * rowb, Lw.sh_down + off, bytes, bar, pol);
    } else if (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR) {
      const uint32_t bytes = (uint32_t)j.n * 3 * rowb;
      mbar_expect_tx(bar, bytes);
      bulk_g2s(dst, Lw.gate + (size_t)j.c0 * 3 * rowb, bytes, bar, pol);
    } else if (WT == MOE_W_BF16) {
      const int e = rs.unit_e[j.u];
      const uint32_t bytes = (uint32_t)j.n * rowb;
      const size_t off = ((size_t)e * I + j.c0) * rowb;
      mbar_expect_tx(bar, 3 * bytes);
      bulk_g2s(dst, Lw.gate + off, bytes, bar, pol);
      bulk_g2s(dst + p.nch * rowb, Lw.up + off, bytes, bar, pol);
      bulk_g2s(dst + 2 * p.nch * rowb, Lw.down + off, bytes, bar, pol);
    } else {  // int4 planar
      const int e = rs.unit_e[j.u];
      const int rowc = H >> 1, rows = H >> 5;
      const uint32_t cb = (uint32_t)j.n * rowc, sb = (uint32_t)j.n * rows;
      const size_t offc = ((size_t)e * I + j.c0) * rowc, offs = ((size_t)e * I + j.c0) * rows;
      const size_t offd = ((size_t)e * (I >> 6) + (j.c0 >> 6)) * rowb;
      mbar_expect_tx(bar, 3 * cb + 2 * sb + rowb);
      bulk_g2s(dst, Lw.gate + offc, cb, bar, pol);
      bulk_g2s(dst + p.nch * rowc, Lw.up + offc, cb, bar, pol);
      bulk_g2s(dst + 2 * p.nch * rowc, Lw.down + offc, cb, bar, pol);
      bulk_g2s(dst + 3 * p.nch * rowc, Lw.gate_s + offs, sb, bar, pol);
      bulk_g2s(dst + 3 * p.nch * rowc + p.nch * rows, Lw.up_s + offs, sb, bar, pol);
      bulk_g2s(dst + 3 * p.nch * rowc + 2 * p.nch * rows, Lw.down_s + offd, rowb, bar, pol);
    }
  };

  // Thread 0: issue every job that is known and has a free stage.
  auto produce = [&]() {
    if (tid != 0) return;
    const int ready = route_ready_layer_s;
    while (jp < jc + p.nstages) {
      JobCursor save = pcur;
      Job j;
      if (!next_job(pcur, j, ready)) { pcur = save; break; }
      if (j.type == JOB_END) { pcur = save; break; }
      issue(j, (int)(jp % p.nstages));
      ++jp;
    }
  };

  // ------------------------------------------------------------ consumer
  JobCursor ccur;
  ccur.begin_layer(p, 0);
  float acc[BMAX][8];
#pragma unroll
  for (int b = 0; b < BMAX; ++b)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[b][i] = 0.f;

  const float ones[kMaxB] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
  const uint32_t all_tokens = (B >= 32) ? 0xffffffffu : ((1u << B) - 1u);

  // Error path: before leaving, wait (bounded) for every copy this CTA has in
  // flight so no bulk copy lands in shared memory after the CTA exits.
  auto drain = [&]() {
    if (tid == 0)
      for (long long q = jc; q < jp; ++q) mbar_wait(&full[q % p.nstages], (uint32_t)((q / p.nstages) & 1));
    __syncthreads();
  };

  // Consume one job: wait for its stage, compute, release the stage.
  // Returns false on a timeout (status already recorded).
  auto consume = [&](const Job& j) -> bool {
    const int slot = (int)(jc % p.nstages);
    const uint32_t parity = (uint32_t)((jc / p.nstages) & 1);
    const uint8_t* st = ring + (size_t)slot * p.stage_bytes;
    const bool ok = mbar_wait(&full[slot], parity);
    if (j.type == JOB_ROUTER) {
      if (ok) {
        for (int r = warp; r < j.n; r += kWarps) {
          const uint4* row = reinterpret_cast<const uint4*>(st + r * rowb);
          float part[BMAX];
#pragma unroll
          for (int b = 0; b < BMAX; ++b) part[b] = 0.f;
          for (int v = (tid & 31); v < H8; v += 32) {
            const uint4 wv = row[v];
#pragma unroll
            for (int b = 0; b < BMAX; ++b)
              if (b < B) part[b] += dot8_bf16(wv, xs4[b * H8 + v]);
          }
#pragma unroll
          for (int b = 0; b < BMAX; ++b)
            if (b < B) {
              const float s = warp_sum(part[b]);
              if ((tid & 31) == 0) p.logits[b * E + j.c0 + r] = s;
            }
        }
      }
      if (__syncthreads_or(!ok)) { set_status(ctl, kStatusTimeout); return false; }
    } else {
      uint32_t mask;
      const float* wts;
      int nstride;
      if (j.type == JOB_SHARED) {
        mask = all_tokens;
        wts = ones;
        nstride = p.nch_sh;
      } else if (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR) {
        mask = 1u;
        const int e = j.c0 / I;
        int u = 0;
        while (u < rs.U - 1 && rs.unit_e[u] != e) ++u;
        wts = &rs.wmap_unit[u];
        nstride = 0;
      } else {
        mask = rs.unit_mask[j.u];
        wts = rs.unit_w[j.u];
        nstride = p.nch;
      }
      const bool shared_or_bf16 = (j.type == JOB_SHARED) || (WT == MOE_W_BF16);
      if (ok) {
        if (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR && j.type != JOB_SHARED)
          dots_bf16<BMAX>(st, j.n, 3 * rowb, rowb, xs4, H8, mask, dots);
        else if (shared_or_bf16)
          dots_bf16<BMAX>(st, j.n, rowb, nstride * rowb, xs4, H8, mask, dots);
        else
          dots_int4<BMAX>(st, j.n, H, p.nch, xs4, mask, dots);
      }
      if (__syncthreads_or(!ok)) { set_status(ctl, kStatusTimeout); return false; }
      swiglu_h<BMAX>(j.n, mask, wts, dots, hs);
      __syncthreads();
      if (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR && j.type != JOB_SHARED)
        down_bf16<BMAX>(st, j.n, 3 * rowb, 2 * rowb, H8, mask, hs, acc);
      else if (shared_or_bf16)
        down_bf16<BMAX>(st, j.n, rowb, 2 * nstride * rowb, H8, mask, hs, acc);
      else
        down_int4<BMAX>(st, j.n, H, p.nch, mask, hs, acc);
      __syncthreads();
    }
    ++jc;
    produce();
    return true;
  };

  // Build the routed units (touched experts, ascending) from rs.ids / rs.w.
  // Returns false if ids were out of range or repeated within a token.
  auto build_units = [&]() -> bool {
    const int nw = (E + 31) >> 5;
    if (tid == 0) bad_s = 0;
    for (int i = tid; i < nw; i += kThreads) rs.bitmap[i] = 0u;
    __syncthreads();
    for (int t = tid; t < B * k; t += kThreads) {
      const int e = rs.ids[t / k][t % k];
      if (e < 0 || e >= E) bad_s = 1;
      else atomicOr(&rs.bitmap[e >> 5], 1u << (e & 31));
    }
    __syncthreads();
    if (warp == 0) {
      const int lane = tid & 31;
      const int c = lane < nw ? __popc(rs.bitmap[lane]) : 0;
      int inc = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
      }
      if (lane < nw) rs.rank_base[lane] = inc - c;
      if (lane == 31) rs.U = inc;
    }
    __syncthreads();
    for (int u = tid; u < rs.U; u += kThreads) {
      rs.unit_mask[u] = 0u;
#pragma unroll
      for (int b = 0; b < kMaxB; ++b) rs.unit_w[u][b] = 0.f;
    }
    for (int e = tid; e < E; e += kThreads)
      if ((rs.bitmap[e >> 5] >> (e & 31)) & 1u)
        rs.unit_e[rs.rank_base[e >> 5] + __popc(rs.bitmap[e >> 5] & ((1u << (e & 31)) - 1u))] = e;
    __syncthreads();
    for (int t = tid; t < B * k; t += kThreads) {
      const int b = t / k, e = rs.ids[b][t % k];
      if (e < 0 || e >= E) continue;
      const int u = rs.rank_base[e >> 5] + __popc(rs.bitmap[e >> 5] & ((1u << (e & 31)) - 1u));
      const uint32_t old = atomicOr(&rs.unit_mask[u], 1u << b);
      if (old & (1u << b)) bad_s = 1;
      else rs.unit_w[u][b] = rs.w[b][t % k];
    }
    __syncthreads();
    return bad_s == 0;
  };

  // Channel-sparse (B = 1): keep the p.keep best candidates of the routed
  // units' channels by score; fills kept[] ascending and rs.ncand.
  auto select_channels = [&](int l) {
    const int N = rs.U * I;
    const float* sc = p.layer[l].scores;  // token 0's [E, I] block
    for (int q = tid; q < N; q += kThreads) {
      const int u = q / I, c = q - u * I;
      keys[q] = float_key(__ldg(sc + (size_t)rs.unit_e[u] * I + c));
    }
    if (tid < rs.U) {
      // weight of each unit for token 0
      rs.wmap_unit[tid] = rs.unit_w[tid][0];
    }
    __syncthreads();
    const int keep = p.keep;
    uint32_t T = 0;
    int rank = 0;
    if (keep > 0 && keep < N) {
      uint32_t prefix = 0, pmask = 0;
      rank = keep;
      for (int shift = 24; shift >= 0; shift -= 8) {
        rs.hist[tid] = 0u;
        __syncthreads();
        for (int q = tid; q < N; q += kThreads) {
          const uint32_t kk = keys[q];
          if ((kk & pmask) == prefix) atomicAdd(&rs.hist[(kk >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (warp == 0) {
          const int lane = tid & 31;
          uint32_t c8[8], loc = 0;
#pragma unroll
          for (int i = 0; i < 8; ++i) { c8[i] = rs.hist[255 - 8 * lane - i]; loc += c8[i]; }
          uint32_t inc = loc;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += t;
          }
          const uint32_t exc = inc - loc;
          const bool hit = exc < (uint32_t)rank && (uint32_t)rank <= inc;
          if (hit) {
            uint32_t cum = exc;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              if (cum + c8[i] >= (uint32_t)rank) {
                rs.sel_rank = rank - (int)cum;
                rs.sel_prefix = (int)(prefix | ((uint32_t)(255 - 8 * lane - i) << shift));
                break;
              }
              cum += c8[i];
            }
          }
        }
        __syncthreads();
        prefix = (uint32_t)rs.sel_prefix;
        rank = rs.sel_rank;
        pmask |= 255u << shift;
      }
      T = prefix;
    }
    // ordered compaction: kept iff key > T, or key == T among the first `rank`
    const int chunk = (N + kThreads - 1) / kThreads;
    const int lo = min(N, tid * chunk), hi = min(N, lo + chunk);
    auto is_kept_all = [&](int) { return keep >= N; };
    int eq = 0;
    if (keep > 0 && keep < N)
      for (int q = lo; q < hi; ++q) eq += (keys[q] == T);
    int tot;
    const int eq_before = block_excl_scan(eq, rs.scan, &tot);
    int cnt = 0;
    {
      int e_seen = eq_before;
      for (int q = lo; q < hi; ++q) {
        bool kp;
        if (keep <= 0) kp = false;
        else if (is_kept_all(q)) kp = true;
        else {
          const uint32_t kk = keys[q];
          kp = kk > T || (kk == T && e_seen < rank);
          e_seen += (kk == T);
        }
        cnt += kp;
      }
    }
    const int pos0 = block_excl_scan(cnt, rs.scan, &tot);
    {
      int e_seen = eq_before, pos = pos0;
      for (int q = lo; q < hi; ++q) {
        bool kp;
        if (keep <= 0) kp = false;
        else if (is_kept_all(q)) kp = true;
        else {
          const uint32_t kk = keys[q];
          kp = kk > T || (kk == T && e_seen < rank);
          e_seen += (kk == T);
        }
        if (kp && pos < keep) {
          const int u = q / I;
          kept[pos++] = rs.unit_e[u] * I + (q - u * I);
        }
      }
    }
    if (tid == 0) { rs.ncand = min(tot, keep); rs.sectors = 0ull; }
    __syncthreads();
    // sectors the kernel reads: union of the kept channels' 32-byte sectors
    const unsigned long long base = (unsigned long long)(uintptr_t)p.layer[l].gate;
    const unsigned long long cb = 3ull * rowb;
    unsigned long long sec = 0;
    for (int i = tid; i < rs.ncand; i += kThreads) {
      const unsigned long long s0 = (base + (unsigned long long)kept[i] * cb) >> 5;
      const unsigned long long s1 = (base + (unsigned long long)(kept[i] + 1) * cb - 1) >> 5;
      sec += s1 - s0 + 1;
      if (i > 0 && ((base + (unsigned long long)(kept[i - 1] + 1) * cb - 1) >> 5) == s0) sec -= 1;
    }
    if (sec) atomicAdd(&rs.sectors, sec);
    __syncthreads();
  };

  // ------------------------------------------------------------ main loop
  produce();  // prefetch layer 0's router rows and shared channels

  for (int l = 0; l < p.L; ++l) {
    float* yacc = p.yacc + (size_t)(l & 1) * B * H;
    // 1. zero this CTA's slice of the accumulator used by this layer
    {
      const long long n4 = (long long)B * H / 4;
      for (long long i = cta * n4 / G + tid; i < (cta + 1) * n4 / G; i += kThreads)
        reinterpret_cast<float4*>(yacc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    Job j;
    if (p.mode == MODE_LAYERS) {
      // 2. router rows of this CTA -> logits in the workspace
      while (ccur.layer == l && ccur.type == JOB_ROUTER) {
        next_job(ccur, j, -1);
        if (!consume(j)) { drain(); return; }
      }
      // 3. split grid barrier: arrive now, run the shared expert, then wait
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        const unsigned long long n = (unsigned long long)G;
        const unsigned long long ticket = atom_add_release_gpu(&ctl->bar, 1ull);
        target_s = (ticket / n + 1ull) * n;
      }
      while (ccur.layer == l && ccur.type == JOB_SHARED) {
        next_job(ccur, j, -1);
        if (!consume(j)) { drain(); return; }
      }
      {
        __syncthreads();
        if (tid == 0) {
          int ok = 1;
          if (ld_acquire_gpu(&ctl->bar) < target_s) {
            const long long t0 = clock64();
            while (ld_acquire_gpu(&ctl->bar) < target_s)
              if (clock64() - t0 > kWaitBudgetCycles) { ok = 0; set_status(ctl, kStatusTimeout); break; }
          }
          __threadfence();
          okw_s = ok;
        }
        __syncthreads();
        if (!okw_s) { drain(); return; }
      }
      // 4. logits -> shared memory, top-k per token (one warp per token)
      for (int i = tid; i < B * E; i += kThreads) lg[i] = __ldcg(p.logits + i);
      __syncthreads();
      if (warp < B) warp_topk(lg + warp * E, E, k, rs.ids[warp], rs.w[warp], nullptr);
      __syncthreads();
      if (cta == 0 && p.ids_out != nullptr)
        for (int t = tid; t < B * k; t += kThreads) {
          p.ids_out[(size_t)l * B * k + t] = rs.ids[t / k][t % k];
          p.w_out[(size_t)l * B * k + t] = rs.w[t / k][t % k];
        }
    } else {
      // experts only: routing supplied by the caller
      for (int t = tid; t < B * k; t += kThreads) {
        rs.ids[t / k][t % k] = p.ids_in[t];
        rs.w[t / k][t % k] = p.w_in[t];
      }
      if (!grid_barrier(ctl)) { drain(); return; }  // accumulator zeroed everywhere
    }
    // 5. routed units (+ channel selection), then stream the routed channels
    if (!build_units() && cta == 0 && tid == 0) set_status(ctl, kStatusBadIds);
    if (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR) {
      select_channels(l);
      if (cta == 0) {
        if (p.kept_out != nullptr)
          for (int i = tid; i < rs.ncand; i += kThreads) p.kept_out[(size_t)l * p.keep + i] = kept[i];
        if (tid == 0 && p.sectors_out != nullptr) p.sectors_out[l] = rs.sectors;
      }
    }
    if (tid == 0) route_ready_layer_s = l;
    __syncthreads();
    produce();
    for (;;) {
      const JobCursor save = ccur;
      if (!next_job(ccur, j, l) || j.type == JOB_END || j.layer != l) { ccur = save; break; }
      if (!consume(j)) { drain(); return; }
    }
    ccur.begin_layer(p, l + 1);
    // 6. partial sums -> L2 accumulator; grid barrier
    if (tid < H8) {
#pragma unroll
      for (int b = 0; b < BMAX; ++b)
        if (b < B) {
          float* dst = yacc + (size_t)b * H + 8 * tid;
          red_add_v4(dst, acc[b][0], acc[b][1], acc[b][2], acc[b][3]);
          red_add_v4(dst + 4, acc[b][4], acc[b][5], acc[b][6], acc[b][7]);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[b][i] = 0.f;
        }
    }
    if (!grid_barrier(ctl)) { drain(); return; }
    // 7. epilogue: y, residual, outputs (each CTA writes its slice)
    {
      const long long n4 = (long long)B * H / 4;
      const long long s0 = cta * n4 / G, s1 = (cta + 1) * n4 / G;
      float* yh = p.y_hist ? p.y_hist + (size_t)l * B * H : nullptr;
      float* yo = (l == p.L - 1) ? p.y_out : nullptr;
      if (p.mode == MODE_LAYERS) {
        // every CTA needs the whole next x
        for (long long i = tid; i < n4; i += kThreads) {
          const float4 y4 = __ldcg(reinterpret_cast<const float4*>(yacc) + i);
          uint2 xv = reinterpret_cast<uint2*>(xs)[i];
          const float x0 = bf16_lo(xv.x) + y4.x, x1 = bf16_hi(xv.x) + y4.y;
          const float x2 = bf16_lo(xv.y) + y4.z, x3 = bf16_hi(xv.y) + y4.w;
          xv.x = uint32_t(f_to_bf16(x0)) | (uint32_t(f_to_bf16(x1)) << 16);
          xv.y = uint32_t(f_to_bf16(x2)) | (uint32_t(f_to_bf16(x3)) << 16);
          reinterpret_cast<uint2*>(xs)[i] = xv;
          if (i >= s0 && i < s1) {
            if (yh) reinterpret_cast<float4*>(yh)[i] = y4;
            if (yo) reinterpret_cast<float4*>(yo)[i] = y4;
            if (p.x_hist) reinterpret_cast<uint2*>(p.x_hist + (size_t)(l + 1) * B * H)[i] = xv;
            if (l == p.L - 1 && p.x_out) reinterpret_cast<uint2*>(p.x_out)[i] = xv;
          }
        }
      } else {
        for (long long i = s0 + tid; i < s1; i += kThreads) {
          const float4 y4 = __ldcg(reinterpret_cast<const float4*>(yacc) + i);
          if (yo) reinterpret_cast<float4*>(yo)[i] = y4;
          if (yh) reinterpret_cast<float4*>(yh)[i] = y4;
        }
      }
      __syncthreads();
    }
  }
}

}  // namespace moedec
