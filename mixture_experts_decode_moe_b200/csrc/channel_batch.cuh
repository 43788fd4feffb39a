// Channel-sparse routed experts for a batch of 2..8 tokens in ONE cooperative
// launch that reads the union of the tokens' kept channels once.
//
// What it computes (pages cited by title and section): for every token b the
// candidates are the channels (e, c) of its k routed experts; the `keep`
// largest scores are kept (one top-k across all of the token's routed
// experts, ties to the lowest index e*I + c; review of arXiv:2610.37386,
// "배경: 채널과 유지 규칙" keep-rule table and "2단계"); a kept channel adds
// w_{b,e} a_{b,j} d_j with a_{b,j} = SiLU(g_j.x_b)(v_j.x_b), a dropped one
// adds nothing. At batch > 1 the channels the batch reads are the union of
// the tokens' kept sets, which grows with the batch (same review, Table 7
// rows B = 4 and B = 8, and "속도"): each union channel is fetched once and
// applied to every token that kept it.
//
// How (B200 design), one CTA per SM, 8 consumer warps + 1 producer warp:
//  A. CTA b < B selects token b's kept channels (the keep-th largest key
//     by histogram passes over the keys' own range, ordered compaction),
//     writes them ascending to the workspace (and the caller's kept list)
//     and as a bitmap over the channel ids, with the token's sector count;
//     every CTA zeroes its slice of y. One grid-wide barrier.
//  B. Every CTA builds the batch's touched experts (ascending), ORs the
//     tokens' kept-channel bitmaps (over channel ids j = e*I + c, written by
//     phase A) into the union and its prefix counts, and takes a contiguous
//     slice of the union list with each channel's token mask; it adds its
//     slice's sectors to the union's sector count.
//  C. The producer warp streams the slice's channels (12 KB each at H =
//     2048, one bulk copy per run of consecutive channels) through a ring of
//     shared-memory stages; per job of 4 channels, warp w computes half of
//     channel w % 4's gate and up dots with every token that kept it, then
//     warp w applies the job's down columns to its 1/8 of the output for all
//     tokens, accumulating in registers. One vector reduction per element at
//     the end.
#pragma once

#include "decode_kernel.cuh"

namespace moedec {

constexpr int kCbConsumers = 256;                // 8 consumer warps
constexpr int kCbThreads = kCbConsumers + 32;    // + 1 producer warp
constexpr int kCbNch = 4;                        // channels per job
constexpr int kCbStages = 3;
constexpr int kCbMaxUnits = kMaxB * kMaxK;       // touched experts of a batch (<= B * k <= 256)
constexpr int kCbMaxChanBits = 1 << 20;          // E * I (the union is kept over channel ids)
constexpr int kCbMaxSlice = 1024;                // union channels per CTA
static_assert(kCbNch * kMaxB == 32, "a job's activations: one lane per (channel, token)");
static_assert(kCbMaxUnits <= 256, "slice units are stored as bytes");

struct ChanBatchParams {
  int B, H, E, I, k, keep;
  const uint16_t* x;       // [B, H] bf16
  const int32_t* ids;      // [B, k]
  const float* w;          // [B, k]
  const float* scores;     // [B, E, I] fp32
  const uint8_t* cm;       // [E, I, 3, H] bf16 (gate row, up row, down column)
  float* y;                // [B, H] fp32, overwritten
  int32_t* kept_out;       // [B, keep] or null
  unsigned long long* sectors;        // [B]
  int32_t* union_count;               // [1] or null
  unsigned long long* union_sectors;  // [1] or null
  WsControl* ctl;
  int32_t* kept_ws;        // [B, keep] workspace
  uint32_t* bits_ws;       // [B, jstride] workspace: each token's kept channels as bits of j = e*I + c
  int jstride;             // words per token bitmap: ceil(E*I / 32) rounded up to a multiple of 4
  int ring_bytes;          // shared-memory ring (also the selection keys and the union bitmaps)
  int smem_bytes;          // ring + x
};

__global__ void __launch_bounds__(kCbThreads, 1) channel_batch_kernel(const __grid_constant__ ChanBatchParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint64_t full[kCbStages], empty[kCbStages];
  __shared__ short unit_of_e[kMaxE];
  __shared__ float wt[kCbMaxUnits][kMaxB];
  __shared__ int tu_e[kMaxK];               // phase A: token's experts, ascending
  __shared__ int sl_j[kCbMaxSlice];         // phase C: this CTA's union channels,
  __shared__ uint8_t sl_m[kCbMaxSlice];     //          their token masks
  __shared__ uint8_t sl_u[kCbMaxSlice];     //          and their units (touched experts)
  __shared__ float hw[kWarps][kCbNch * kMaxB];  // per warp: a job's activations w * SiLU(g) * u
  __shared__ float part[2][kCbNch][2][kMaxB][2];
  __shared__ int scan_s[2 * kWarps + 2];
  __shared__ uint32_t red_s[2 * kWarps];
  __shared__ int U_s, bad_s, ok_s, abort_s;
  __shared__ long long budget_s;
  __shared__ long long issued_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int B = p.B, H = p.H, H8 = H >> 3, E = p.E, I = p.I, k = p.k, keep = p.keep;
  const int rowb = 2 * H, cb = 3 * rowb;
  const int stage_bytes = kCbNch * cb;
  uint8_t* ring = smem;
  uint4* xs4 = reinterpret_cast<uint4*>(smem + p.ring_bytes);
  WsControl* ctl = p.ctl;

  if (tid == 0) {
    for (int s = 0; s < kCbStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kWarps);
    }
    fence_mbar_init();
    bad_s = 0;
    abort_s = 0;
    issued_s = 0;
    budget_s = ctl_wait_budget(ctl);
  }
  for (int i = tid; i < B * H8; i += kCbThreads) xs4[i] = reinterpret_cast<const uint4*>(p.x)[i];
  // this CTA's slice of y is zeroed before the barrier; every add comes after it
  {
    const int n4 = B * H / 4;
    const int y0 = (int)((long long)cta * n4 / G), y1 = (int)((long long)(cta + 1) * n4 / G);
    for (int i = y0 + tid; i < y1; i += kCbThreads) reinterpret_cast<float4*>(p.y)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (cta == 0 && tid == 0) {
    if (p.union_sectors) *p.union_sectors = 0ull;
  }
  __syncthreads();
  const long long budget = budget_s;
  bool failed = false;

  // ---------------------------------------------------------------- A: selection of token cta
  if (cta < B && warp < kWarps) {
    const int b = cta;
    if (warp == 0) {
      const int e = lane < k ? __ldg(p.ids + b * k + lane) : 0x7fffffff;
      int rank = 0, dup = 0;
      for (int i = 0; i < k; ++i) {
        const int o = __shfl_sync(0xffffffffu, e, i);
        rank += (o < e) || (o == e && i < lane);
        dup |= (o == e && i != lane);
      }
      if (lane < k) {
        if (e < 0 || e >= E || dup) bad_s = 1;
        tu_e[rank] = (e >= 0 && e < E) ? e : 0;
      }
    }
    cbar();
    const int N = k * I;
    // keys, then the select's bins and scratch, in the ring (unused until
    // phase C)
    uint32_t* keys = reinterpret_cast<uint32_t*>(ring);
    int* hist = reinterpret_cast<int*>(ring + ((size_t)N * 4 + 127) / 128 * 128);
    int* sel_sc = hist + 2 * kSelBins;
    // the token's kept channels as bits of j = e*I + c, after the scratch
    uint32_t* bm = reinterpret_cast<uint32_t*>(sel_sc + kSelScratch);
    for (int i = tid; i < p.jstride; i += kCbConsumers) bm[i] = 0u;
    const float* srow = p.scores + (size_t)b * E * I;
    const bool vec = (I & 3) == 0 && ((uintptr_t)p.scores & 15u) == 0;
    sel_load_keys(keys, N, I, vec, [&](int u) { return srow + (size_t)tu_e[u] * I; }, hist, sel_sc);
    cbar();
    int* kws = p.kept_ws + (size_t)b * keep;
    if (keep > 0)
      // the kept list, ascending
      sel_kept(keys, N, keep, hist, sel_sc, [&](int pos, int q) {
        const int u = q / I;
        const int j = tu_e[u] * I + (q - u * I);
        kws[pos] = j;
        atomicOr(&bm[j >> 5], 1u << (j & 31));
        if (p.kept_out) p.kept_out[(size_t)b * keep + pos] = j;
      });
    cbar();  // the kept list is complete (global writes of this CTA, ordered by the barrier)
    for (int i = tid; i < p.jstride; i += kCbConsumers) p.bits_ws[(size_t)b * p.jstride + i] = bm[i];
    // sectors of the token's kept channels (channel-major ranges, a sector
    // shared with the previous kept channel counted once; channels that
    // start and end on 32-byte boundaries share none)
    const unsigned long long base = (unsigned long long)(uintptr_t)p.cm;
    const int nk = keep < N ? keep : N;
    if (((base | (unsigned long long)cb) & 31ull) == 0) {
      if (tid == 0) p.sectors[b] = (unsigned long long)nk * ((unsigned long long)cb >> 5);
    } else {
      uint32_t sec = 0;
      for (int i = tid; i < nk; i += kCbConsumers) {
        const unsigned long long s0 = (base + (unsigned long long)kws[i] * cb) >> 5;
        const unsigned long long s1 = (base + (unsigned long long)(kws[i] + 1) * cb - 1) >> 5;
        sec += (uint32_t)(s1 - s0 + 1);
        if (i > 0 && ((base + (unsigned long long)(kws[i - 1] + 1) * cb - 1) >> 5) == s0) sec -= 1;
      }
      sec = __reduce_add_sync(0xffffffffu, sec);
      if (lane == 0) red_s[warp] = sec;
      cbar();
      if (tid == 0) {
        unsigned long long t = 0;
        for (int w = 0; w < kWarps; ++w) t += red_s[w];
        p.sectors[b] = t;
      }
    }
    if (tid == 0) {
      if (bad_s) set_status(ctl, kStatusBadIds);
    }
  }

  // ---------------------------------------------------------------- grid barrier
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned long long Gu = (unsigned long long)G;
    const unsigned long long ticket = atom_add_release_gpu(&ctl->bar, 1ull);
    unsigned long long target = (ticket / Gu + 1ull) * Gu;
    if (ctl->inject & kInjectBarrierExtraArrival) target += 1;  // an injected fault: never reached
    int ok = 1;
    if (ld_acquire_gpu(&ctl->bar) < target) {
      const long long t0 = clock64();
      while (ld_acquire_gpu(&ctl->bar) < target)
        if (clock64() - t0 > budget) { ok = 0; break; }
    }
    if (!ok) set_status(ctl, kStatusTimeout);
    __threadfence();
    ok_s = ok;
  }
  __syncthreads();
  failed = ok_s == 0;

  // ---------------------------------------------------------------- B: union and this CTA's slice
  // every CTA checks the ids itself (in range, distinct per token): with a
  // bad id nothing is computed (CTA b recorded the status in phase A)
  __shared__ int ids_s[kCbMaxUnits];
  if (!failed) {
    if (tid == 0) bad_s = 0;
    for (int t = tid; t < B * k; t += kCbThreads) ids_s[t] = __ldg(p.ids + t);
    __syncthreads();
    for (int t = tid; t < B * k; t += kCbThreads) {
      const int e = ids_s[t], b = t / k;
      bool bad = e < 0 || e >= E;
      for (int s2 = 0; s2 < k; ++s2)
        if (b * k + s2 != t && ids_s[b * k + s2] == e) bad = true;
      if (bad) bad_s = 1;
    }
    __syncthreads();
    failed = bad_s != 0;
  }
  int ns = 0;
  if (!failed) {
    // touched experts of the batch, ascending, and their weights per token
    uint32_t* ebits = reinterpret_cast<uint32_t*>(ring);  // [E / 32]
    const int ne32 = (E + 31) >> 5;
    for (int i = tid; i < ne32; i += kCbThreads) ebits[i] = 0u;
    __syncthreads();
    for (int t = tid; t < B * k; t += kCbThreads) {
      const int e = ids_s[t];
      if (e >= 0 && e < E) atomicOr(&ebits[e >> 5], 1u << (e & 31));
    }
    __syncthreads();
    if (warp == 0) {
      int base = 0;
      for (int w0 = 0; w0 < ne32; w0 += 32) {
        const int wi = w0 + lane;
        const uint32_t bits = wi < ne32 ? ebits[wi] : 0u;
        int inc = __popc(bits);
        const int cnt = inc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += t;
        }
        int rk = base + inc - cnt;
        for (uint32_t m = bits; m; m &= m - 1) {
          const int e = wi * 32 + __ffs(m) - 1;
          unit_of_e[e] = (short)rk;
          ++rk;
        }
        base += __shfl_sync(0xffffffffu, inc, 31);
      }
      if (lane == 0) U_s = base;
    }
    __syncthreads();
    const int U = U_s;
    for (int i = tid; i < U * kMaxB; i += kCbThreads) wt[i / kMaxB][i % kMaxB] = 0.f;
    __syncthreads();
    for (int t = tid; t < B * k; t += kCbThreads) {
      const int e = ids_s[t];
      if (e >= 0 && e < E) wt[unit_of_e[e]][t / k] = __ldg(p.w + t);
    }
    // the union of the tokens' kept channels over j = e*I + c: thread t takes
    // the contiguous words [w0, w1) (a multiple of 4: 16-byte loads of every
    // token's bitmap, written by phase A), keeps them in the (still unused)
    // ring for the slice below and ORs them
    const int JS = p.jstride;
    uint32_t* tb = reinterpret_cast<uint32_t*>(ring);          // [B][JS]
    uint32_t* uw = tb + (size_t)B * JS;                          // [JS] union
    int* upre = reinterpret_cast<int*>(uw + JS);                 // [JS] exclusive prefix of popc
    const int per = ((JS + 4 * kCbThreads - 1) / (4 * kCbThreads)) * 4;
    const int w0 = min(JS, tid * per), w1 = min(JS, w0 + per);
    int cnt = 0;
    for (int i = w0; i < w1; i += 4) {
      uint4 m = make_uint4(0u, 0u, 0u, 0u);
      for (int b = 0; b < B; ++b) {
        const uint4 v = __ldcg(reinterpret_cast<const uint4*>(p.bits_ws + (size_t)b * JS + i));
        *reinterpret_cast<uint4*>(tb + (size_t)b * JS + i) = v;
        m.x |= v.x; m.y |= v.y; m.z |= v.z; m.w |= v.w;
      }
      *reinterpret_cast<uint4*>(uw + i) = m;
      cnt += __popc(m.x) + __popc(m.y) + __popc(m.z) + __popc(m.w);
    }
    // block-wide exclusive scan over all 288 threads (9 warps)
    {
      int inc = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += t;
      }
      if (lane == 31) scan_s[warp] = inc;
      __syncthreads();
      if (tid == 0) {
        int s = 0;
        for (int w = 0; w < kCbThreads / 32; ++w) { const int v = scan_s[w]; scan_s[w] = s; s += v; }
        scan_s[kCbThreads / 32] = s;
      }
      __syncthreads();
      int run = scan_s[warp] + inc - cnt;
      for (int i = w0; i < w1; ++i) { upre[i] = run; run += __popc(uw[i]); }
    }
    const int NU = scan_s[kCbThreads / 32];
    const int s0 = (int)((long long)cta * NU / G), s1 = (int)((long long)(cta + 1) * NU / G);
    ns = s1 - s0;
    __syncthreads();
    // this CTA's slice of the union (ascending j) with token masks, and the
    // union channel just before it (for the shared-sector rule)
    __shared__ int prev_j_s;
    if (tid == 0) prev_j_s = -1;
    __syncthreads();
    // thread t finds union channel s0 - 1 + t (its word: the last with
    // prefix <= rank, by binary search; its bit: the rank's set bit of the
    // word), so the slice is extracted in parallel
    for (int t = tid; t <= ns; t += kCbThreads) {
      const int rk = s0 - 1 + t;
      if (rk < 0) continue;
      int lo = 0, hi = JS - 1;  // upre[lo] <= rk < upre[hi + 1]
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (upre[mid] <= rk) lo = mid; else hi = mid - 1;
      }
      const uint32_t mw = uw[lo];
      int nth = rk - upre[lo], bit = 0;
      uint32_t m = mw;
#pragma unroll
      for (int wdt = 16; wdt >= 1; wdt >>= 1) {
        const int c = __popc(m & ((1u << wdt) - 1u));
        if (nth >= c) { nth -= c; m >>= wdt; bit += wdt; }
      }
      const int j = lo * 32 + bit;
      if (t == 0) {
        prev_j_s = j;
      } else {
        uint32_t tm = 0u;
        for (int b = 0; b < B; ++b) tm |= ((tb[(size_t)b * JS + lo] >> bit) & 1u) << b;
        sl_j[t - 1] = j;
        sl_m[t - 1] = (uint8_t)tm;
        sl_u[t - 1] = (uint8_t)unit_of_e[j / I];
      }
    }
    __syncthreads();
    if (cta == 0 && tid == 0 && p.union_count) *p.union_count = NU;
    if (p.union_sectors != nullptr && warp < kWarps) {
      const unsigned long long base = (unsigned long long)(uintptr_t)p.cm;
      uint32_t sec = 0;
      for (int i = tid; i < ns; i += kCbConsumers) {
        const unsigned long long a0 = (base + (unsigned long long)sl_j[i] * cb) >> 5;
        const unsigned long long a1 = (base + (unsigned long long)(sl_j[i] + 1) * cb - 1) >> 5;
        sec += (uint32_t)(a1 - a0 + 1);
        const int pj = i > 0 ? sl_j[i - 1] : prev_j_s;
        if (pj >= 0 && ((base + (unsigned long long)(pj + 1) * cb - 1) >> 5) == a0) sec -= 1;
      }
      sec = __reduce_add_sync(0xffffffffu, sec);
      if (lane == 0 && sec) atomicAdd(p.union_sectors, (unsigned long long)sec);
    }
    __syncthreads();  // the ring's bitmaps are dead from here on
  }

  // ---------------------------------------------------------------- C: the slice's channels
  const int nj = (ns + kCbNch - 1) / kCbNch;
  if (!failed) {
    if (warp == kWarps) {
      // producer: one bulk copy per run of consecutive channels of a job
      if (lane == 0) {
        const uint64_t pol = policy_evict_first();
        long long issued = 0;
        for (int q = 0; q < nj; ++q) {
          const int s = q % kCbStages;
          if (q >= kCbStages) {
            const long long t0 = clock64();
            bool ok = true;
            while (!mbar_try_wait_sleep(&empty[s], (uint32_t)(((q / kCbStages) - 1) & 1), 20000)) {
              if (*(volatile int*)&abort_s || clock64() - t0 > budget) { ok = false; break; }
            }
            if (!ok) break;
          }
          const int i0 = q * kCbNch, n = min(kCbNch, ns - i0);
          uint8_t* dst = ring + (size_t)s * stage_bytes;
          mbar_expect_tx(&full[s], (uint32_t)(n * cb));
          for (int i = 0; i < n;) {
            const int j0 = sl_j[i0 + i];
            int r = 1;
            while (i + r < n && sl_j[i0 + i + r] == j0 + r) ++r;
            bulk_g2s(dst + (size_t)i * cb, p.cm + (size_t)j0 * cb, (uint32_t)(r * cb), &full[s], pol);
            i += r;
          }
          ++issued;
        }
        issued_s = issued;
      }
    } else {
      // consumers
      float acc[kMaxB][8];
#pragma unroll
      for (int b = 0; b < kMaxB; ++b)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[b][e] = 0.f;
      const int ch = warp & (kCbNch - 1), half = warp / kCbNch;
      const int hv = H8 >> 1;                     // vectors per half row
      const int dv = H8 / kWarps;                 // down vectors per warp (<= 32 for H <= 2048)
      const int vd = warp * dv + lane;            // this lane's down vector
      bool ok = true;
      for (int q = 0; q < nj && ok; ++q) {
        const int s = q % kCbStages;
        const uint32_t ph = (uint32_t)((q / kCbStages) & 1);
        bool landed = mbar_try_wait_sleep(&full[s], ph, 20000);
        if (!landed) {
          const long long t0 = clock64();
          while (!(landed = mbar_try_wait_sleep(&full[s], ph, 20000)))
            if (*(volatile int*)&abort_s || clock64() - t0 > budget) break;
        }
        // all consumer warps agree before any of them meets a barrier
        if (cbar_or(!landed)) {
          ok = false;
          if (tid == 0) { *(volatile int*)&abort_s = 1; set_status(ctl, kStatusTimeout); }
          break;
        }
        const uint8_t* st = ring + (size_t)s * stage_bytes;
        const int i0 = q * kCbNch, n = min(kCbNch, ns - i0);
        // 1. half of channel ch's gate and up dots with every token that kept it
        float dg[kMaxB], du[kMaxB];
#pragma unroll
        for (int b = 0; b < kMaxB; ++b) { dg[b] = 0.f; du[b] = 0.f; }
        const uint32_t tm = ch < n ? sl_m[i0 + ch] : 0u;
        if (tm) {
          const uint4* g4 = reinterpret_cast<const uint4*>(st + (size_t)ch * cb);
          const uint4* u4 = reinterpret_cast<const uint4*>(st + (size_t)ch * cb + rowb);
          for (int v = half * hv + lane; v < (half + 1) * hv; v += 32) {
            float gf[8], uf[8];
            unpack8(g4[v], gf);
            unpack8(u4[v], uf);
#pragma unroll
            for (int b = 0; b < kMaxB; ++b)
              if ((tm >> b) & 1u) {
                float xf[8];
                unpack8(xs4[b * H8 + v], xf);
                float g0 = gf[0] * xf[0], g1 = gf[1] * xf[1], u0 = uf[0] * xf[0], u1 = uf[1] * xf[1];
#pragma unroll
                for (int e = 2; e < 8; e += 2) {
                  g0 = fmaf(gf[e], xf[e], g0);
                  g1 = fmaf(gf[e + 1], xf[e + 1], g1);
                  u0 = fmaf(uf[e], xf[e], u0);
                  u1 = fmaf(uf[e + 1], xf[e + 1], u1);
                }
                dg[b] += g0 + g1;
                du[b] += u0 + u1;
              }
          }
        }
        {
          float v16[2 * kMaxB];
#pragma unroll
          for (int b = 0; b < kMaxB; ++b) { v16[2 * b] = dg[b]; v16[2 * b + 1] = du[b]; }
          warp_reduce_multi<2 * kMaxB>(v16, &part[q & 1][ch][half][0][0]);
        }
        cbar();
        // 2. the job's activations h = w * SiLU(g) * u, lane c * 8 + b of
        // every warp taking channel c and token b (all in parallel), then the
        // job's down columns on this warp's 1/8 of the outputs
        {
          const int c = lane >> 3, b = lane & 7;
          float h = 0.f;
          if (c < n && b < B && ((sl_m[i0 + c] >> b) & 1u)) {
            const float g = part[q & 1][c][0][b][0] + part[q & 1][c][1][b][0];
            const float uu = part[q & 1][c][0][b][1] + part[q & 1][c][1][b][1];
            h = wt[sl_u[i0 + c]][b] * silu_f(g) * uu;
          }
          hw[warp][lane] = h;
          __syncwarp();
        }
        if (lane < dv) {
#pragma unroll
          for (int c = 0; c < kCbNch; ++c)
            if (c < n) {
              const uint32_t m = sl_m[i0 + c];
              float d[8];
              unpack8(reinterpret_cast<const uint4*>(st + (size_t)c * cb + 2 * rowb)[vd], d);
#pragma unroll
              for (int b = 0; b < kMaxB; ++b)
                if ((m >> b) & 1u) {
                  const float h = hw[warp][c * kMaxB + b];
#pragma unroll
                  for (int e = 0; e < 8; ++e) acc[b][e] = fmaf(h, d[e], acc[b][e]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      if (ok && lane < dv) {
#pragma unroll
        for (int b = 0; b < kMaxB; ++b)
          if (b < B) {
            float* dst = p.y + (size_t)b * H + 8 * vd;
            red_add_v4(dst, acc[b][0], acc[b][1], acc[b][2], acc[b][3]);
            red_add_v4(dst + 4, acc[b][4], acc[b][5], acc[b][6], acc[b][7]);
          }
      }
    }
  }
  __syncthreads();
  // after an abort, copies may still be landing in stages no consumer read:
  // wait (bounded) for the last kCbStages issued before the CTA exits
  if (tid == 0 && abort_s) {
    const long long n = issued_s < kCbStages ? issued_s : kCbStages;
    for (long long q = issued_s - n; q < issued_s; ++q)
      (void)mbar_wait(&full[q % kCbStages], (uint32_t)((q / kCbStages) & 1), budget);
  }
}

}  // namespace moedec
