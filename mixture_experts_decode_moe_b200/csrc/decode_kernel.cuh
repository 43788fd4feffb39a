// Body of the persistent decode kernel (see decode.cuh for the design).
//
// Roles inside a CTA (288 threads):
//   warps 0-7  consumers: dot products, SwiGLU, down projection, top-k,
//              grid barriers, epilogue; synchronise with named barrier 1;
//   warp 8     producer: walks the same job sequence and issues the bulk
//              copies of each job into a free stage of the ring (full/empty
//              mbarriers per stage), running ahead of the consumers.
#pragma once

#include "decode.cuh"
#include "screen_lut.cuh"

namespace moedec {

constexpr int kConsumers = kThreads;          // 256 consumer threads
constexpr int kProducers = 2;                // producer warps (alternate jobs)
constexpr int kCtaThreads = kThreads + 32 * kProducers;

__device__ __forceinline__ void cbar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ int cbar_or(int pred) {
  int r;
  asm volatile(
      "{ .reg .pred p, q; setp.ne.s32 p, %1, 0; bar.red.or.pred q, 1, 256, p; selp.s32 %0, 1, 0, q; }"
      : "=r"(r)
      : "r"(pred)
      : "memory");
  return r;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void red_release_gpu(unsigned long long* p, unsigned long long v) {
  asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_gpu(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
// two 8-byte words with one 16-byte load (each word read whole)
__device__ __forceinline__ void ld_relaxed_gpu_v2(const unsigned long long* p, unsigned long long& a,
                                                  unsigned long long& b) {
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}
__device__ __forceinline__ void st_relaxed_gpu_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_cta(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared::cta.s32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_cta(int* p, int v) {
  asm volatile("st.release.cta.shared::cta.s32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

// ---------------------------------------------------------------- block helpers

// Exclusive prefix sum over the 256 consumer threads; `total` gets the sum.
__device__ __forceinline__ int block_excl_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) scratch[warp] = inc;
  cbar();
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
  cbar();
  int r = inc - v + scratch[warp];
  *total = scratch[kWarps];
  cbar();
  return r;
}

// Transpose-style reduction of NV per-lane values across a warp. Afterwards
// the warp's sums are written to out[0..NV) (smem).
template <int NV>
__device__ __forceinline__ void warp_reduce_multi(float (&v)[NV], float* out) {
  static_assert((NV & (NV - 1)) == 0, "NV must be a power of two");
  const int lane = threadIdx.x & 31;
  int base = 0;
  // halving steps (offsets 16, 8, ...) while more than one value remains
  constexpr int S = (NV >= 32) ? 5 : (NV >= 16 ? 4 : (NV >= 8 ? 3 : (NV >= 4 ? 2 : (NV >= 2 ? 1 : 0))));
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int off = 16 >> s;
    const int C = NV >> s;
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < C / 2; ++i) {
      const float send = up ? v[i] : v[i + C / 2];
      const float keep = up ? v[i + C / 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
    if (up) base += C / 2;
  }
  // remaining offsets: plain butterfly sums of the values each lane keeps
  constexpr int CF = NV >> S;
#pragma unroll
  for (int s = S; s < 5; ++s) {
    const int off = 16 >> s;
#pragma unroll
    for (int i = 0; i < CF; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], off);
  }
  if ((lane & ((1 << (5 - S)) - 1)) == 0) {
#pragma unroll
    for (int i = 0; i < CF; ++i) out[base + i] = v[i];
  }
}

// ---------------------------------------------------------------- key selection

constexpr int kSelBins = 2048;                    // histogram bins of one select pass
constexpr int kSelGather = 64;                    // class size ranked directly
constexpr int kSelScratch = 160 + kConsumers;     // ints of scratch the select needs

// The channel select runs once per layer on 256 threads; its costs here are
// shared-memory wavefronts, shared atomics (about three per cycle per SM),
// warp collectives (30-60 cycles of latency, about 19 cycles apart when
// independent) and divergent branches. So: few passes over the keys, branch-
// free per-key code, ballots only where they do not chain.
//
// The loader places key q at keys[q], warp w loading candidates
// [w * kw, (w + 1) * kw), kw = ceil(n / 8) rounded up to a multiple of 128.
__device__ __forceinline__ int sel_kw(int n) { return (((n + kWarps - 1) / kWarps) + 127) & ~127; }

// The select's own walk: thread t owns the contiguous chunk q in
// [t * c, min(n, t * c + c)), c = ceil(n / 256) rounded up to a multiple of
// 4 (at most 32), read as 16-byte words.
__device__ __forceinline__ int sel_chunk(int n) { return ((n + kConsumers - 1) / kConsumers + 3) & ~3; }

// Exclusive prefix over the warp's lanes of v < 2^NB, and the warp total,
// from NB ballots that do not depend on one another (a shuffle scan would
// chain five 50-cycle steps).
template <int NB>
__device__ __forceinline__ int warp_scan_bits(uint32_t v, int* total) {
  const uint32_t lt = (1u << (threadIdx.x & 31)) - 1u;
  uint32_t m[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) m[b] = __ballot_sync(0xffffffffu, (v >> b) & 1u);
  int pre = 0, tot = 0;
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    pre += __popc(m[b] & lt) << b;
    tot += __popc(m[b]) << b;
  }
  *total = tot;
  return pre;
}

// A predicated shared-memory add of 1 (no branch around it).
__device__ __forceinline__ void red_shared_add_if(bool p, int* addr) {
  asm volatile("{ .reg .pred q; setp.ne.u32 q, %0, 0; @q red.shared.add.u32 [%1], 1; }" ::"r"((int)p), "r"(smem_u32(addr))
               : "memory");
}
#ifndef CLK
#define CLK(i)
#endif
// keys[q] = float_key(score of candidate q), candidate q = u * I + c being
// channel c of unit u, row(u) its unit's I scores. With vec (I % 4 == 0 and
// every row 16-byte aligned) each lane copies up to eight 16-byte groups of
// its warp's range straight into shared memory (cp.async through L2, no
// registers held), then turns its own groups into keys in place; otherwise a
// rolled loop of four loads per lane. It also starts the select: sc[w] /
// sc[8 + w] = min / max key of warp w's share, hist[0, kSelBins) and the
// class-bit words zeroed. The caller synchronises before sel_kept.
template <class Row>
__device__ __forceinline__ void sel_load_keys(uint32_t* keys, int n, int I, bool vec, Row row, int* hist, int* sc) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kw = sel_kw(n);
  const int q1 = min(n, (warp + 1) * kw);
  const float invI = 1.0f / (float)I;
  uint32_t mn = 0xffffffffu, mx = 0u;
  if (vec) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int q = warp * kw + 4 * (lane + 32 * j);
      if (q < q1) {
        const int u = __float2int_rz(((float)q + 0.5f) * invI);
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(keys + q)), "l"(row(u) + (q - u * I))
                     : "memory");
      }
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int q = warp * kw + 4 * (lane + 32 * j);
      if (q < q1) {
        uint4 w = *reinterpret_cast<const uint4*>(keys + q);
        w.x = float_key(__uint_as_float(w.x));
        w.y = float_key(__uint_as_float(w.y));
        w.z = float_key(__uint_as_float(w.z));
        w.w = float_key(__uint_as_float(w.w));
        mn = min(min(mn, min(w.x, w.y)), min(w.z, w.w));
        mx = max(max(mx, max(w.x, w.y)), max(w.z, w.w));
        *reinterpret_cast<uint4*>(keys + q) = w;
      }
    }
  } else {
#pragma unroll 1
    for (int q0 = warp * kw + lane; q0 < q1; q0 += 128) {
      float v[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int q = q0 + 32 * t;
        v[t] = 0.f;
        if (q < q1) {
          const int u = __float2int_rz(((float)q + 0.5f) * invI);
          v[t] = __ldcg(row(u) + (q - u * I));
        }
      }
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (q0 + 32 * t < q1) {
          const uint32_t k = float_key(v[t]);
          keys[q0 + 32 * t] = k;
          mn = min(mn, k);
          mx = max(mx, k);
        }
    }
  }
  mn = __reduce_min_sync(0xffffffffu, mn);
  mx = __reduce_max_sync(0xffffffffu, mx);
  for (int b = tid; b < kSelBins; b += kConsumers) hist[b] = 0;
  sc[160 + tid] = 0;
  if (lane == 0) {
    sc[warp] = (int)mn;
    sc[kWarps + warp] = (int)mx;
  }
  if (tid == 0) sc[27] = 0;
}

// The kept channels of one token, exact: every key > T plus the first
// keep - #{> T} keys == T in index order, T the keep-th largest key, listed
// ascending through emit(pos, q). 0 < keep; n <= kMaxCand; keys and sc as
// sel_load_keys left them, after a barrier.
//  1. The class of keys that can still hold T starts as [min, max]. A pass
//     counts the class's keys in up to 2048 equal power-of-two-wide bins over
//     its range (predicated shared adds; the bins follow the data's own
//     range, so keys spread over them); warp totals of the bins (thread t
//     owns bins [8t, 8t + 8)) locate the warp, and a ballot scan the thread,
//     whose bins hold the rank still needed: that bin becomes the class. At
//     most three passes, typically one; they stop once the class holds at
//     most 64 keys or one value.
//  2. One branch-free pass marks each thread's keys above the class (a
//     32-bit mask per thread) and its class keys.
//  3. A class of one value: its first `need` keys in index order are kept
//     (ballot scan of the per-thread counts). Otherwise the class keys are
//     gathered (a shared counter) and thread t < cnt ranks class key t
//     against the class: T and, among keys == T, the index order; kept class
//     keys set their bit in their owner's word.
//  4. Positions: a ballot scan of the per-thread kept counts, one barrier for
//     the warp totals, then each thread emits its set bits in order.
template <class Emit>
__device__ __forceinline__ void sel_kept(const uint32_t* keys, int n, int keep, int* hist, int* sc, Emit emit) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = sel_chunk(n);
  const int q0 = tid * c, q1 = min(n, q0 + c);
  const int nq = max(0, q1 - q0);
  const uint4* kp = reinterpret_cast<const uint4*>(keys + q0);
  int* xm = sc + 160;  // [256] kept bits of class keys, per owning thread
  uint32_t mask = 0u;  // bit i: candidate q0 + i kept
  if (keep >= n) {
    mask = nq >= 32 ? 0xffffffffu : ((1u << nq) - 1u);
  } else {
    uint32_t lo = (uint32_t)sc[0], hi = (uint32_t)sc[kWarps];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
      lo = min(lo, (uint32_t)sc[w]);
      hi = max(hi, (uint32_t)sc[kWarps + w]);
    }
    int need = keep;  // rank of T inside the class [lo, hi]
    int cnt = n;      // keys in the class
    // 2. histogram passes until the class is small or one value
#pragma unroll 1
    for (int pass = 0; pass < 3 && lo != hi && cnt > kSelGather; ++pass) {
      int* h = hist + (pass & 1) * kSelBins;
      int* hn = hist + ((pass + 1) & 1) * kSelBins;
      const int sh = max(0, 32 - __clz(hi - lo) - 11);
#pragma unroll 2
      for (int j = 0; 4 * j < nq; ++j) {
        const uint4 w = kp[j];
        const uint32_t e[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const bool ok = 4 * j + t < nq && e[t] >= lo && e[t] <= hi;
          red_shared_add_if(ok, &h[ok ? (e[t] - lo) >> sh : 0]);
        }
      }
      for (int b = tid; b < kSelBins; b += kConsumers) hn[b] = 0;
      cbar();
      const int4 c0 = reinterpret_cast<const int4*>(h)[2 * tid];
      const int4 c1 = reinterpret_cast<const int4*>(h)[2 * tid + 1];
      const int mine = c0.x + c0.y + c0.z + c0.w + c1.x + c1.y + c1.z + c1.w;
      const int wsum = __reduce_add_sync(0xffffffffu, mine);
      if (lane == 0) sc[16 + warp] = wsum;
      cbar();
      int W = -1, wabove = 0;
      {
        int acc = 0;
#pragma unroll
        for (int w = kWarps - 1; w >= 0; --w) {
          const int t = sc[16 + w];
          if (W < 0 && acc + t >= need) {
            W = w;
            wabove = acc;
          }
          acc += t;
        }
      }
      if (warp == W) {
        const uint32_t gtm = ~((2u << lane) - 1u);
        uint32_t m[14];
#pragma unroll
        for (int b = 0; b < 14; ++b) m[b] = __ballot_sync(0xffffffffu, ((uint32_t)mine >> b) & 1u);
        int above = wabove;
#pragma unroll
        for (int b = 0; b < 14; ++b) above += __popc(m[b] & gtm) << b;
        if (above < need && above + mine >= need) {
          const int cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
          int acc = above, dj = 0, aj = 0, cj = 0;
          bool found = false;
#pragma unroll
          for (int j = 7; j >= 0; --j)
            if (!found) {
              if (acc + cv[j] >= need) {
                found = true;
                dj = 8 * tid + j;
                aj = acc;
                cj = cv[j];
              } else {
                acc += cv[j];
              }
            }
          sc[24] = dj;
          sc[25] = aj;
          sc[26] = cj;
        }
      }
      cbar();
      const uint32_t d = (uint32_t)sc[24];
      need -= sc[25];
      cnt = sc[26];
      lo += d << sh;
      hi = min(hi, lo + ((1u << sh) - 1u));
    }
    // 3. classify: keys above the class are kept; the class's keys are
    // gathered (at most kSelGather of them unless the class is one value)
    uint32_t cm = 0u;  // this thread's class keys
#pragma unroll 2
    for (int j = 0; 4 * j < nq; ++j) {
      const uint4 w = kp[j];
      const uint32_t e[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int i = 4 * j + t;
        const bool ok = i < nq;
        mask |= (ok && e[t] > hi) ? (1u << i) : 0u;
        cm |= (ok && e[t] >= lo && e[t] <= hi) ? (1u << i) : 0u;
      }
    }
    if (lo == hi) {
      // one value T = lo: its first `need` keys in index order are kept
      int tot;
      int pre = warp_scan_bits<6>((uint32_t)__popc(cm), &tot);
      if (lane == 0) sc[16 + warp] = tot;
      cbar();
#pragma unroll
      for (int w = 0; w < kWarps; ++w)
        if (w < warp) pre += sc[16 + w];
      for (int take = need - pre; cm != 0u && take > 0; --take) {
        mask |= cm & (0u - cm);  // lowest remaining class key
        cm &= cm - 1u;
      }
    } else {
      // gather the class (at most kSelGather keys)
      while (cm != 0u) {
        const int i = __ffs(cm) - 1;
        cm &= cm - 1u;
        const int sl = atomicAdd(&sc[27], 1);
        if (sl < kSelGather) {
          sc[32 + sl] = (int)keys[q0 + i];
          sc[96 + sl] = q0 + i;
        }
      }
      cbar();
      // threads t < cnt rank class key t against the whole class: T is the
      // key with fewer than need larger and at least need larger-or-equal
      // class keys (any such thread writes the same T); of the keys == T
      // the first need - #{> T} in index order are kept
      const bool ac = tid < cnt;
      const uint32_t v = ac ? (uint32_t)sc[32 + tid] : 0u;
      const int iv = ac ? sc[96 + tid] : 0;
      int g = 0, e = 0;
      if (ac) {
#pragma unroll 1
        for (int m = 0; m < cnt; m += 4) {
          const int4 o4 = *reinterpret_cast<const int4*>(sc + 32 + m);
          const uint32_t o[4] = {(uint32_t)o4.x, (uint32_t)o4.y, (uint32_t)o4.z, (uint32_t)o4.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            g += (m + t < cnt && o[t] > v) ? 1 : 0;
            e += (m + t < cnt && o[t] >= v) ? 1 : 0;
          }
        }
        if (g < need && e >= need) {
          sc[28] = (int)v;
          sc[29] = g;
        }
      }
      cbar();
      if (ac) {
        const uint32_t T = (uint32_t)sc[28];
        const int r = need - sc[29];  // keys == T to keep
        bool kept = v > T;
        if (v == T) {
          int t0 = 0;
#pragma unroll 1
          for (int m = 0; m < cnt; m += 4) {
            const int4 o4 = *reinterpret_cast<const int4*>(sc + 32 + m);
            const int4 p4 = *reinterpret_cast<const int4*>(sc + 96 + m);
            const uint32_t o[4] = {(uint32_t)o4.x, (uint32_t)o4.y, (uint32_t)o4.z, (uint32_t)o4.w};
            const int oq[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) t0 += (m + t < cnt && o[t] == T && oq[t] < iv) ? 1 : 0;
          }
          kept = t0 < r;
        }
        if (kept) atomicOr(&xm[iv / c], 1 << (iv % c));
      }
      cbar();
      mask |= (uint32_t)xm[tid];
    }
  }
  // 4. positions: exclusive prefix of the per-thread kept counts
  int tot;
  int pos = warp_scan_bits<6>((uint32_t)__popc(mask), &tot);
  if (lane == 0) sc[16 + warp] = tot;
  cbar();
#pragma unroll
  for (int w = 0; w < kWarps; ++w)
    if (w < warp) pos += sc[16 + w];
  while (mask) {
    const int b = __ffs(mask) - 1;
    emit(pos++, q0 + b);
    mask &= mask - 1u;
  }
}

// ---------------------------------------------------------------- top-k

// One warp: the kk largest keys among keys[0, n) (n <= 1024), ties to the
// lowest position; positions in descending key order -> out_pos[0, kk).
__device__ __forceinline__ void warp_select(const uint32_t* keys, int n, int kk, int* out_pos) {
  const int lane = threadIdx.x & 31;
  const int per = (n + 31) >> 5;
  const int lo = min(n, lane * per), hi = min(n, lo + per);
  uint32_t taken = 0, bk = 0;
  int bi = -1;
  auto rescan = [&]() {
    bk = 0;
    bi = -1;
    for (int i = lo; i < hi; ++i) {
      if ((taken >> (i - lo)) & 1u) continue;
      const uint32_t kv = keys[i];
      if (bi < 0 || kv > bk) { bk = kv; bi = i; }
    }
  };
  rescan();
  for (int r = 0; r < kk; ++r) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, bi >= 0 ? bk : 0u);
    const uint32_t ball = __ballot_sync(0xffffffffu, bi >= 0 && bk == m);
    const int win = __ffs(ball) - 1;
    const int pos = __shfl_sync(0xffffffffu, bi, win);
    if (lane == 0) out_pos[r] = pos;
    if (lane == win) {
      taken |= 1u << (pos - lo);
      rescan();
    }
  }
}

// Renormalised softmax weights over the chosen logits l[0..k) (l[0] largest).
__device__ __forceinline__ void warp_weights(const float* l, int k, float* w) {
  const int lane = threadIdx.x & 31;
  const float e = (lane < k) ? expf(l[lane] - l[0]) : 0.f;
  const float s = warp_sum(e);
  if (lane < k) w[lane] = e / s;
}

// Cross-warp sum of per-warp output accumulators (64 per lane, element
// 256 c + 8 lane + e in acc[8 c + e]) into ysum (element 256 c + 8 lane + e
// at 256 c + 32 e + lane): at step st warp w adds its chunk (w + st) % 8, so
// no two warps touch a chunk at once; one barrier per step. Every warp runs
// the same code (a switch picks the chunk, so that every register index is a
// constant): it runs once per layer, and one shared copy is fetched once
// instead of eight. (The accumulators are zeroed by the caller just before
// the next layer's first job that adds to them, so that they are not live
// through routing and selection.)
template <int C>
__device__ __forceinline__ void ysum_chunk(const float (&acc)[64], float* ysum, int lane, bool first) {
  float* yc = ysum + 256 * C + lane;
#pragma unroll
  for (int e = 0; e < 8; ++e) yc[32 * e] = first ? acc[8 * C + e] : yc[32 * e] + acc[8 * C + e];
}
__device__ __forceinline__ void ysum_all(const float (&acc)[64], float* ysum, int lane, int warp) {
#pragma unroll 1
  for (int st = 0; st < 8; ++st) {
    const bool first = st == 0;
    switch ((warp + st) & 7) {
      case 0: ysum_chunk<0>(acc, ysum, lane, first); break;
      case 1: ysum_chunk<1>(acc, ysum, lane, first); break;
      case 2: ysum_chunk<2>(acc, ysum, lane, first); break;
      case 3: ysum_chunk<3>(acc, ysum, lane, first); break;
      case 4: ysum_chunk<4>(acc, ysum, lane, first); break;
      case 5: ysum_chunk<5>(acc, ysum, lane, first); break;
      case 6: ysum_chunk<6>(acc, ysum, lane, first); break;
      default: ysum_chunk<7>(acc, ysum, lane, first); break;
    }
    cbar();
  }
}

// ---------------------------------------------------------------- the kernel

// One CTA of kCtaThreads (320) threads per SM. Ten warps put three on some of
// the SM's four sub-partitions of 16K registers each, so a thread gets at
// most 168 registers; spills would go to local memory, i.e. to L2, since
// shared memory takes nearly all of L1 (live ranges are kept short instead).
// SCREEN (channel-major stacks only): the scores are screened in the kernel
// from per-layer sketches (a separate instance: the screen's registers would
// make the plain channel-major instance spill).
template <int MODE, int BMAX, int WT, int LAYOUT, int NCH, int HV, bool SCREEN = false>
__global__ void __launch_bounds__(kCtaThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int NR = 2 * NCH;        // dot rows per job (gate+up rows; router rows)
  constexpr int NV = NR * BMAX;      // values reduced per job
  // Batch-1 bf16 rows of 2048 elements: every warp owns whole channels (see
  // consume_fast); job q goes to warp group q % kGroups of NCH warps.
  // (int4 experts too, planar: their router and shared rows are bf16)
  constexpr bool kFast = (BMAX == 1 && HV == 8 && (WT == MOE_W_BF16 || LAYOUT == MOE_LAYOUT_PLANAR));
  constexpr bool kFastI4 = kFast && WT == MOE_W_INT4_G64;
  // int4 experts at batch > 1 with H = 2048: a routed job's gate and up dots
  // for all tokens on tensor cores (each code decoded once per job); the
  // output sums live in shared memory (registers hold one token's at a time)
  constexpr bool kTcB = WT == MOE_W_INT4_G64 && BMAX == 8 && HV == 8 && NCH == 4 && LAYOUT == MOE_LAYOUT_PLANAR;
  static_assert(!kTcB || NCH * BMAX == 32, "one lane per (channel, token) activation");
  // batch > 1: cost of a routed channel in units of one token's work is
  // kJobW + (tokens routed to its expert): its fetch (and, on the int4 batch
  // path, its tensor-core dots for all tokens at once) plus the per-token work
  constexpr int kJobW = kTcB ? 4 : 1;
  // channels per shared-expert job (bf16 rows): one on the int4 batch path,
  // whose ring stages are sized for int4 jobs
  constexpr int kShN = kTcB ? 1 : NCH;
  static_assert(!kFast || (NCH == 2 || NCH == 4 || NCH == 8), "warp groups of 2, 4 or 8 warps");
  constexpr int kGroups = kFast ? kWarps / NCH : 1;
  // fast path: warp group g and producer g form pipeline g with the ring
  // stages s, s % kPipes == g, and count their jobs independently
  constexpr int kPipes = kFast ? kGroups : 1;
  static_assert(!kFast || kPipes == kProducers, "one producer per warp group on the fast path");
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ RouteSmem<BMAX> rs;
  __shared__ int route_ready_s, prod_layer_s[kProducers], abort_s, bad_s, okw_s;
  __shared__ int units_s;  // planar batch 1: layer * 64 + units of its routing published so far
  __shared__ int bar_l_s;  // last layer whose closing grid barrier the consumers passed
  __shared__ uint32_t ltag_s;  // logit tag of layer 0 in this launch (fast path)
  __shared__ unsigned long long bar_base_s;  // grid-barrier count at launch (a multiple of G)
  __shared__ long long budget_s;  // cycles per bounded wait (the workspace's budget)
  __shared__ uint32_t inject_s;   // fault-injection bits of the workspace
  __shared__ long long jp_s[kProducers], jc_s, jcg_s[kProducers];
  __shared__ Job jdesc[8];     // fast path: the job held by each stage
  __shared__ int rcnt_s[2 * kProducers];  // fast path: router-partial counters
  __shared__ int pred_s[kProducers][kMaxPred];  // fast path: predicted experts of the next layer
  __shared__ float dotbuf[16][NV];
  __shared__ float hbuf[kWarps][NCH * BMAX];
  __shared__ float2 tcpart[kTcB ? 2 : 1][kWarps][32];  // per warp: (gate, up) partial dots [channel][token]
  __shared__ float2 hb2[kTcB ? kWarps : 1][32];        // per warp: activations as pairs {h, h}
  __shared__ uint32_t cand_key[kWarps * kMaxK];
  __shared__ int cand_idx[kWarps * kMaxK];
  __shared__ int sel_pos[kWarps][kMaxK];
  __shared__ float sel_l[kWarps][kMaxK];

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int B = p.B, H = p.H, H8 = H >> 3, E = p.E, I = p.I, k = p.k;
  const int rowb = 2 * H;
  uint8_t* ring = smem;
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + p.off_x);  // residual stream x
  const uint4* xs4 = reinterpret_cast<const uint4*>(xs);
  // MoE input u: RMS-normalised x with the pre-norm, else x itself
  // u: the pre-normed x (or x itself); on the int4 batch path always its own
  // buffer, holding u as a table of tensor-core A fragments (build_xfrags)
  uint16_t* us = (kTcB || (MODE == MODE_LAYERS && p.pre_norm)) ? reinterpret_cast<uint16_t*>(smem + p.off_u) : xs;
  const uint4* us4 = reinterpret_cast<const uint4*>(us);
  float* lg = reinterpret_cast<float*>(smem + p.off_lg);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + p.off_keys);
  int* kept = reinterpret_cast<int*>(smem + p.off_kept);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* empty = full + p.nstages;
  uint64_t* hready = empty + p.nstages;
  WsControl* ctl = p.ctl;

  if (tid == 0) {
    for (int s = 0; s < p.nstages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kFast ? NCH : kWarps);
      mbar_init(&hready[s], kWarps);
    }
    fence_mbar_init();
    route_ready_s = -1;  // last layer whose routing the consumers published
    units_s = -1;
    bar_l_s = -1;
    for (int q = 0; q < kProducers; ++q) {
      prod_layer_s[q] = -1;  // last layer whose routed jobs producer q issued
      jp_s[q] = 0;           // jobs producer q has passed (its own ones issued)
    }
    abort_s = 0;
    // every launch passes at least one grid barrier, so bar_base / G differs
    // between launches on a workspace and the tags (launch * 64 + layer, top
    // bit set so that a cleared word never matches) do not repeat; a slot is
    // rewritten only after the grid barrier that follows every reader's
    // routing, so a reader never meets a later layer's tag. (Other CTAs may
    // already have arrived at this launch's first barrier: fewer than G
    // arrivals do not change the quotient.)
    bar_base_s = (ld_relaxed_gpu(&ctl->bar) / (unsigned long long)G) * (unsigned long long)G;
    ltag_s = 0x80000000u | ((uint32_t)(bar_base_s / (unsigned long long)G) * (uint32_t)kMaxLayers);
    budget_s = ctl_wait_budget(ctl);
    inject_s = ctl->inject;
    jc_s = 0;
    for (int q = 0; q < kProducers; ++q) jcg_s[q] = 0;
    for (int q = 0; q < 2 * kProducers; ++q) rcnt_s[q] = 0;
  }
  for (int i = tid; i < B * H8; i += kCtaThreads)
    reinterpret_cast<uint4*>(xs)[i] = reinterpret_cast<const uint4*>(p.x_in)[i];
  if constexpr (kFast)
    for (int i = tid; i < H; i += kCtaThreads) reinterpret_cast<float*>(smem + p.off_ysum)[i] = 0.f;
  if constexpr (kTcB)  // the batch path's output sums [B][H] (thread t owns 8 t .. 8 t + 7 of each token)
    for (int i = tid; i < B * H; i += kCtaThreads) reinterpret_cast<float*>(smem + p.off_ysum)[i] = 0.f;
  if (p.x_hist != nullptr) {
    const long long n = (long long)B * H8;
    for (long long i = (unsigned)cta * (unsigned)n / (unsigned)G + tid; i < (unsigned)(cta + 1) * (unsigned)n / (unsigned)G;
         i += kCtaThreads)
      reinterpret_cast<uint4*>(p.x_hist)[i] = reinterpret_cast<const uint4*>(p.x_in)[i];
  }
  __syncthreads();
  const long long budget = budget_s;

  // Batch-1 planar stacks are routed by consumer warp 0 alone (route_warp
  // below) while the other warps go on with their shared-expert jobs.
  // (Measured: routing in a producer warp, and writing the tagged logits to
  // several copies polled by different CTAs, were both slower.)
  const bool warp_routes = kFast && LAYOUT == MOE_LAYOUT_PLANAR && MODE == MODE_LAYERS && k <= kWarps && E <= 256;

  // ---- B = 1, k <= 8, E <= 256, tagged logit words of layer `lay`: one
  // warp routes alone, with no CTA barrier, while the other warps go on
  // with their jobs. Lane l polls words 64q + 2l and 64q + 2l + 1 (q < 4;
  // the warp's four 16-byte loads cover the 2 KB once) until all carry the
  // layer's tag, then the k largest are taken by k rounds over per-lane
  // sorted lists (ties: the lower expert index), followed by the softmax over
  // the k and the units in ascending expert id. Returns false on a poll
  // timeout. Warp-wide steps cost 30-60 cycles each here, so each round has
  // two on its dependent path and the rest stays in registers.
  auto route_warp = [&](int lay) -> bool {
    const unsigned long long* wb = reinterpret_cast<const unsigned long long*>(p.logits);
    const uint32_t want = 0x80000000u | (ltag_s + (uint32_t)lay);
    uint32_t key[8];
    bool done[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      done[q] = 64 * q + 2 * lane >= E;
      key[2 * q] = 0u;
      key[2 * q + 1] = 0u;
    }
    const long long t0 = clock64();
    for (;;) {
      unsigned long long a[4], b[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (!done[q]) ld_relaxed_gpu_v2(wb + 64 * q + 2 * lane, a[q], b[q]);
      bool all = true;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (!done[q]) {
          const int i = 64 * q + 2 * lane;
          const bool has_b = i + 1 < E;
          if ((uint32_t)(a[q] >> 32) == want && (!has_b || (uint32_t)(b[q] >> 32) == want)) {
            done[q] = true;
            key[2 * q] = float_key(__uint_as_float((uint32_t)a[q]));
            key[2 * q + 1] = has_b ? float_key(__uint_as_float((uint32_t)b[q])) : 0u;
          } else {
            all = false;
          }
        }
      if (__all_sync(0xffffffffu, all)) break;
      if (__any_sync(0xffffffffu, clock64() - t0 > budget)) return false;  // warp-uniform
    }
    // Slot s of lane l holds expert 64 (s / 2) + 2 l + s % 2. Each lane
    // sorts its 8 slots best first as 64-bit values key << 32 | ~expert
    // (larger key, then lower index; empty slots 0) with a 19-comparator
    // network; then each of the k rounds takes the best head over the warp
    // (one max reduction over the head keys and one ballot; a second
    // reduction, on the index, only when several heads tie) and the winner
    // drops its head. Every lane follows the chosen keys, so the softmax
    // needs no exchange.
    unsigned long long v[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const int e = 64 * (s >> 1) + 2 * lane + (s & 1);
      v[s] = e < E ? (((unsigned long long)key[s] << 32) | (unsigned long long)(~(uint32_t)e)) : 0ull;
    }
    auto cas = [&](int i, int j) {
      const unsigned long long a = v[i], b = v[j];
      v[i] = a < b ? b : a;
      v[j] = a < b ? a : b;
    };
    cas(0, 1); cas(2, 3); cas(4, 5); cas(6, 7);
    cas(0, 2); cas(1, 3); cas(4, 6); cas(5, 7);
    cas(1, 2); cas(5, 6);
    cas(0, 4); cas(1, 5); cas(2, 6); cas(3, 7);
    cas(2, 4); cas(3, 5);
    cas(1, 2); cas(3, 4); cas(5, 6);
    float m0 = 0.f, esum = 0.f, my_e = 0.f;
    for (int r = 0; r < k; ++r) {
      const uint32_t hk = (uint32_t)(v[0] >> 32);
      const uint32_t M = __reduce_max_sync(0xffffffffu, hk);
      uint32_t tie = __ballot_sync(0xffffffffu, hk == M);
      if (tie & (tie - 1)) {
        // several heads hold the key M: the lowest expert index wins
        const uint32_t lo = __reduce_max_sync(0xffffffffu, hk == M ? (uint32_t)v[0] : 0u);
        tie = __ballot_sync(0xffffffffu, hk == M && (uint32_t)v[0] == lo);
      }
      const bool win = lane == __ffs(tie) - 1;
      if (win) {
        const int ew = (int)~(uint32_t)v[0];
        cand_key[kWarps + r] = M;
        cand_idx[r] = ew;
        if (warp_routes) {
          // planar: unit r is the r-th chosen expert, published at once so
          // that the producers can start its copies during the next rounds
          rs.unit_e[r] = ew;
          rs.unit_mask[r] = 1u;
          st_release_cta(&units_s, lay * 64 + r + 1);
        }
      }
#pragma unroll
      for (int s = 0; s < 7; ++s) v[s] = win ? v[s + 1] : v[s];
      v[7] = win ? 0ull : v[7];
      const float lm = key_float(M);
      if (r == 0) m0 = lm;
      const float er = __expf(lm - m0);
      esum += er;
      if (lane == r) my_e = er;
    }
    __syncwarp();
    const bool sel = lane < k;
    const int ic = sel ? cand_idx[lane] : 0x7fffffff;
    const float wl = my_e / esum;
    // units: the chosen order (planar, published above) or ascending expert
    // id (channel-major, whose candidate order must follow the channel ids)
    int urank = lane;
    if (!warp_routes) {
      urank = 0;
#pragma unroll
      for (int m = 0; m < 8; ++m) urank += (m < k && cand_idx[m] < ic) ? 1 : 0;
    }
    if (sel) {
      rs.ids[0][lane] = ic;
      rs.w[0][lane] = wl;
      rs.unit_e[urank] = ic;
      rs.unit_mask[urank] = 1u;
      rs.unit_w[urank][0] = wl;
      if (cta == 0 && p.ids_out != nullptr) {
        p.ids_out[(size_t)lay * k + lane] = ic;
        p.w_out[(size_t)lay * k + lane] = wl;
      }
    }
    if (lane == 0) rs.U = k;
    __syncwarp();
    return true;
  };

  // At batch 1 the routed channel count is the same every layer (k * I, or
  // the kept count), so this CTA's routed range {t0, t1, unit, channel} is
  // computed once here instead of on the critical path after each routing.
  int4 rfix = make_int4(0, 0, 0, 0);
  if constexpr (BMAX == 1) {
    const int N1 = k * I;
    const int R1 = (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR) ? (p.keep > 0 ? min(N1, p.keep) : 0) : N1;
    const int t0 = (int)((unsigned)cta * (unsigned)R1 / (unsigned)G);
    const int t1 = (int)((unsigned)(cta + 1) * (unsigned)R1 / (unsigned)G);
    rfix = make_int4(t0, t1, t0 / I, t0 - (t0 / I) * I);
  }
  // Job sequence, shared by producer and consumers.
  auto next_job = [&](JobCursor& cur, Job& j, int ready_layer) -> bool {
    for (;;) {
      if (cur.layer >= p.L) { j.type = JOB_END; return true; }
      if (cur.type == JOB_ROUTER) {
        const int n = min(p.rows_per_job, cur.t1 - cur.t);
        j = Job{JOB_ROUTER, cur.layer, 0, cur.t, n};
        cur.t += n;
        if (cur.t >= cur.t1) { cur.type = JOB_SHARED; cur.set_range(p); }
        return true;
      }
      if (cur.type == JOB_SHARED) {
        const int n = min(kShN, cur.t1 - cur.t);
        j = Job{JOB_SHARED, cur.layer, 0, cur.t, n};
        cur.t += n;
        if (cur.t >= cur.t1) { cur.type = JOB_ROUTED; cur.t = -1; cur.t1 = -1; }
        return true;
      }
      if (cur.t1 < 0) {
        if (ready_layer < cur.layer) return false;
        if constexpr (BMAX == 1) {
          cur.set_routed_fixed(rfix);
        } else if constexpr (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR) {
          cur.set_routed(rs.ncand, I);
        } else {
          // batch > 1: a routed channel of unit u costs kJobW + (tokens
          // routed to u), so CTA c takes the channels whose cost offset falls
          // in [c C / G, (c + 1) C / G); the units' cost offsets rs.cpre were
          // summed when the units were built
          const int U = rs.U;
          const long long C = rs.cpre[U];
          auto first_from = [&](long long x) -> int {  // first channel whose cost offset is >= x
            if (x >= C) return U * I;
            int lo = 0, hi = U - 1;  // the last unit whose offset is <= x
            while (lo < hi) {
              const int mid = (lo + hi + 1) >> 1;
              if (rs.cpre[mid] <= x) lo = mid;
              else hi = mid - 1;
            }
            const long long wu = kJobW + __popc(rs.unit_mask[lo]);
            return lo * I + (int)((x - rs.cpre[lo] + wu - 1) / wu);
          };
          const unsigned long long Gu = (unsigned long long)G;
          cur.t = first_from((long long)((unsigned long long)cta * (unsigned long long)C / Gu));
          cur.t1 = first_from((long long)((unsigned long long)(cta + 1) * (unsigned long long)C / Gu));
          cur.u = cur.t / I;
          cur.c = cur.t - cur.u * I;
        }
      }
      if (cur.t >= cur.t1) { cur.begin_layer(p, cur.layer + 1); continue; }
      if (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR) {
        const int pos = cur.t;
        const int j0 = kept[pos];
        int n = 1;
        if (kFast) n = min(NCH, cur.t1 - cur.t);  // any kept channels, one per warp
        else
          while (n < NCH && cur.t + n < cur.t1 && kept[pos + n] == j0 + n && (j0 + n) % I != 0) ++n;
        j = Job{JOB_ROUTED, cur.layer, pos, j0, n};
        cur.t += n;
      } else {
        int n;
        if (WT == MOE_W_INT4_G64) {
          // int4 jobs stay inside one 64-channel scale group: cut at multiples of NCH
          n = min(min(NCH - (cur.c & (NCH - 1)), I - cur.c), cur.t1 - cur.t);
        } else {
          // bf16 jobs may run on into the next expert (two segments at most)
          n = min(min(NCH, cur.t1 - cur.t), 2 * I - cur.c);
        }
        j = Job{JOB_ROUTED, cur.layer, cur.u, cur.c, n};
        cur.t += n;
        cur.c += n;
        while (cur.c >= I) { cur.c -= I; ++cur.u; }
      }
      return true;
    }
  };

  // ================================================================ producer
  // The whole warp walks the job sequence (uniform control flow: every lane
  // computes the same job); lane 0 arms the stage's barrier with the job's
  // byte count and issues its copies. Routed jobs of layer l wait until the
  // consumers publish routing for layer l.
  if (warp >= kWarps) {
    if constexpr (kFast) {
    // ---- pipeline producer pi: per layer, its share of the static jobs
    // (router rows, shared channels: static job s belongs to pipe s % 2),
    // then routed jobs taken from the layer's pool (an atomic counter, the
    // next one grabbed while the current one is issued), then an end marker.
    const int pi = warp - kWarps;
    const uint64_t pol = policy_evict_first();
    const uint64_t pol_n = policy_evict_normal();
    const int nps = (p.nstages - pi + kPipes - 1) / kPipes;
    int pm = 0;
    uint32_t pph = 0;
    long long lq = 0;
    const unsigned Gu = (unsigned)G, cu = (unsigned)cta;
    const int rr0 = (MODE == MODE_LAYERS) ? (int)(cu * (unsigned)E / Gu) : 0;
    const int rr1 = (MODE == MODE_LAYERS) ? (int)((cu + 1) * (unsigned)E / Gu) : 0;
    const int sr0 = (MODE == MODE_LAYERS) ? (int)(cu * (unsigned)p.I_sh / Gu) : 0;
    const int sr1 = (MODE == MODE_LAYERS) ? (int)((cu + 1) * (unsigned)p.I_sh / Gu) : 0;
    const int R1 = (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR) ? (p.keep > 0 ? min(k * I, p.keep) : 0) : k * I;
    const int nj = (R1 + NCH - 1) / NCH;
    int held = -1;  // a pool index grabbed ahead for the coming layer
    // wait for this pipe's next stage to be free, then describe the job
    auto take_stage = [&](const Job& jb) -> int {
      const int slot = pi + kPipes * pm;
      if (lq >= nps) {
        const long long t0 = clock64();
        while (!mbar_try_wait_sleep(&empty[slot], pph ^ 1u, 20000)) {
          if (*(volatile int*)&abort_s || clock64() - t0 > budget) return -1;
        }
      }
      if (lane == 0) jdesc[slot] = jb;
      return slot;
    };
    // planar batch 1: until units_s (layer * 64 + units published) reaches
    // want; lane 0 polls, the warp learns the outcome; false on an abort or
    // when the wait runs out
    auto wait_units = [&](int want) -> bool {
      int ok = 1;
      if (lane == 0) {
        const long long tw = clock64();
        while (*(volatile int*)&units_s < want)
          if (*(volatile int*)&abort_s || clock64() - tw > budget) {
            ok = 0;
            break;
          }
        (void)ld_acquire_cta(&units_s);
      }
      return __shfl_sync(0xffffffffu, ok, 0) != 0;
    };
    auto next_stage = [&]() {
      ++lq;
      if (++pm == nps) { pm = 0; pph ^= 1u; }
      if (lane == 0) *(volatile long long*)&jp_s[pi] = lq;
    };
    // Prediction of layer ln's experts: the tagged words R_ln u_{ln-1} (E <=
    // 256, written by every CTA's prediction jobs in layer ln - 1) are polled
    // like the routing words, and the npred largest taken by rounds of a
    // warp-wide argmax (ties to the lower index). Then the chunks of those
    // experts' weights (gate, up, down, and int4 scales; 16 KB chunks) are
    // spread over the CTAs, and this producer's lanes prefetch every other
    // chunk of this CTA's share into L2. Returns false on a poll timeout or
    // an abort. The prefetch only warms L2: results do not depend on it.
    auto predict_prefetch = [&](int ln) -> bool {
      // the words of layer ln sit in buffer ln % 2: the next writes of that
      // buffer (layer ln + 2's prediction, made in layer ln + 1) come after
      // the grid barrier that ends layer ln, which this CTA reaches only
      // after this producer has issued layer ln's routed jobs
      const unsigned long long* wb = p.plogits + (size_t)(ln & 1) * E;
      const uint32_t want = 0x80000000u | (ltag_s + (uint32_t)ln);
      uint32_t key[8];
      bool done[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        done[q] = 64 * q + 2 * lane >= E;
        key[2 * q] = 0u;
        key[2 * q + 1] = 0u;
      }
      const long long t0 = clock64();
      for (;;) {
        unsigned long long a[4], b[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (!done[q]) ld_relaxed_gpu_v2(wb + 64 * q + 2 * lane, a[q], b[q]);
        bool all = true;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (!done[q]) {
            const bool has_b = 64 * q + 2 * lane + 1 < E;
            if ((uint32_t)(a[q] >> 32) == want && (!has_b || (uint32_t)(b[q] >> 32) == want)) {
              done[q] = true;
              key[2 * q] = float_key(__uint_as_float((uint32_t)a[q]));
              key[2 * q + 1] = has_b ? float_key(__uint_as_float((uint32_t)b[q])) : 0u;
            } else {
              all = false;
            }
          }
        if (__all_sync(0xffffffffu, all)) break;
        if (__any_sync(0xffffffffu, *(volatile int*)&abort_s != 0 || clock64() - t0 > budget)) {
          if (lane == 0 && !*(volatile int*)&abort_s) set_status(ctl, kStatusTimeout);
          return false;
        }
        __nanosleep(32);
      }
      auto slot_idx = [&](int s) { return 64 * (s >> 1) + 2 * lane + (s & 1); };
      const int np = min(p.npred, E);
      uint32_t bk = key[0];
      int bs = 0;
#pragma unroll
      for (int s = 1; s < 8; ++s)
        if (key[s] > bk) { bk = key[s]; bs = s; }
      for (int r = 0; r < np; ++r) {
        const uint32_t M = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t tie = __ballot_sync(0xffffffffu, bk == M);
        int wl = __ffs(tie) - 1;
        if (tie & (tie - 1)) {
          const uint32_t mi = __reduce_min_sync(0xffffffffu, bk == M ? (uint32_t)slot_idx(bs) : 0xffffffffu);
          wl = __ffs(__ballot_sync(0xffffffffu, bk == M && (uint32_t)slot_idx(bs) == mi)) - 1;
        }
        if (lane == wl) {
          pred_s[pi][r] = slot_idx(bs);
#pragma unroll
          for (int s = 0; s < 8; ++s)
            if (s == bs) key[s] = 0u;
          bk = key[0];
          bs = 0;
#pragma unroll
          for (int s = 1; s < 8; ++s)
            if (key[s] > bk) { bk = key[s]; bs = s; }
        }
      }
      __syncwarp();
      // byte ranges of one expert: gate, up, down (+ int4 gate, up, down scales)
      constexpr int NRNG = (WT == MOE_W_BF16) ? 3 : 6;
      constexpr uint32_t kChunk = 16384;
      const LayerW& Ln = p.layer[ln];
      auto range_of = [&](int e, int r, const uint8_t*& ptr, uint32_t& bytes) {
        if constexpr (WT == MOE_W_BF16) {
          const uint8_t* base = r == 0 ? Ln.gate : (r == 1 ? Ln.up : Ln.down);
          bytes = (uint32_t)I * (uint32_t)rowb;
          ptr = base + (size_t)e * bytes;
        } else {
          if (r < 3) {
            const uint8_t* base = r == 0 ? Ln.gate : (r == 1 ? Ln.up : Ln.down);
            bytes = (uint32_t)I * (uint32_t)(H >> 1);
            ptr = base + (size_t)e * bytes;
          } else if (r < 5) {
            bytes = (uint32_t)I * (uint32_t)(H >> 5);
            ptr = (r == 3 ? Ln.gate_s : Ln.up_s) + (size_t)e * bytes;
          } else {
            bytes = (uint32_t)(I >> 6) * (uint32_t)rowb;
            ptr = Ln.down_s + (size_t)e * bytes;
          }
        }
      };
      int cpe = 0;  // chunks per expert
#pragma unroll
      for (int r = 0; r < NRNG; ++r) {
        const uint8_t* ptr;
        uint32_t bytes;
        range_of(0, r, ptr, bytes);
        cpe += (int)((bytes + kChunk - 1) / kChunk);
      }
      const long long Q = (long long)np * cpe;
      const long long q0 = (long long)cta * Q / G, q1 = (long long)(cta + 1) * Q / G;
      for (long long q = q0 + pi + kProducers * lane; q < q1; q += kProducers * 32) {
        const int e = pred_s[pi][(int)(q / cpe)];
        int w = (int)(q % cpe);
#pragma unroll
        for (int r = 0; r < NRNG; ++r) {
          const uint8_t* ptr;
          uint32_t bytes;
          range_of(e, r, ptr, bytes);
          const int nc = (int)((bytes + kChunk - 1) / kChunk);
          if (w < nc) {
            const uint32_t off = (uint32_t)w * kChunk;
            prefetch_l2(ptr + off, min(kChunk, bytes - off));
            break;
          }
          w -= nc;
        }
      }
      __syncwarp();
      return true;
    };
    for (int l = 0; l < p.L; ++l) {
      const LayerW& Lw = p.layer[l];
      int sidx = 0;
      for (int r = rr0; r < rr1; r += p.rows_per_job, ++sidx) {
        if (sidx % kPipes != pi) continue;
        const Job jb{JOB_ROUTER, l, 0, r, min(p.rows_per_job, rr1 - r)};
        const int slot = take_stage(jb);
        if (slot < 0) goto producer_done;
        if (lane == 0) {
          const uint32_t bytes = (uint32_t)jb.n * rowb;
          mbar_expect_tx(&full[slot], bytes);
          bulk_g2s(ring + (size_t)slot * p.stage_bytes, Lw.router + (size_t)r * rowb, bytes, &full[slot], pol);
        }
        __syncwarp();
        next_stage();
      }
      for (int c = sr0; c < sr1; c += NCH, ++sidx) {
        if (sidx % kPipes != pi) continue;
        const Job jb{JOB_SHARED, l, 0, c, min(NCH, sr1 - c)};
        const int slot = take_stage(jb);
        if (slot < 0) goto producer_done;
        if (lane == 0) {
          uint8_t* dst = ring + (size_t)slot * p.stage_bytes;
          const uint32_t bytes = (uint32_t)jb.n * rowb;
          const size_t off = (size_t)c * rowb;
          mbar_expect_tx(&full[slot], 3 * bytes);
          bulk_g2s(dst, Lw.sh_gate + off, bytes, &full[slot], pol);
          bulk_g2s(dst + NCH * rowb, Lw.sh_up + off, bytes, &full[slot], pol);
          bulk_g2s(dst + 2 * NCH * rowb, Lw.sh_down + off, bytes, &full[slot], pol);
        }
        __syncwarp();
        next_stage();
      }
      if (p.npred > 0 && l + 1 < p.L) {
        // the next layer's router rows, applied to this layer's input by the
        // consumers: a prediction of the next layer's experts (job u = 1).
        // Read with normal L2 priority, so that the next layer's own router
        // job finds them in L2.
        const LayerW& Ln = p.layer[l + 1];
        for (int r = rr0; r < rr1; r += p.rows_per_job, ++sidx) {
          if (sidx % kPipes != pi) continue;
          const Job jb{JOB_ROUTER, l, 1, r, min(p.rows_per_job, rr1 - r)};
          const int slot = take_stage(jb);
          if (slot < 0) goto producer_done;
          if (lane == 0) {
            const uint32_t bytes = (uint32_t)jb.n * rowb;
            mbar_expect_tx(&full[slot], bytes);
            bulk_g2s(ring + (size_t)slot * p.stage_bytes, Ln.router + (size_t)r * rowb, bytes, &full[slot], pol_n);
          }
          __syncwarp();
          next_stage();
        }
      }
      // the experts predicted for layer l (made in layer l - 1) into L2, once
      // layer l - 1's closing grid barrier has passed: from then until layer
      // l's routed copies start, HBM has nothing else to stream
      if (p.npred > 0 && l > 0) {
        int okb = 1;
        if (lane == 0) {
          const long long tb0 = clock64();
          while (*(volatile int*)&bar_l_s < l - 1) {
            if (*(volatile int*)&abort_s || clock64() - tb0 > budget) {
              okb = 0;
              break;
            }
            __nanosleep(32);
          }
        }
        if (!__shfl_sync(0xffffffffu, okb, 0)) goto producer_done;
        if (!predict_prefetch(l)) goto producer_done;
      }
      if (!warp_routes) {
        // routing of layer l (plain polls with short sleeps, then one acquire)
        const long long t0 = clock64();
        while (*(volatile int*)&route_ready_s < l) {
          if (*(volatile int*)&abort_s || clock64() - t0 > budget) goto producer_done;
          __nanosleep(20);
        }
        (void)ld_acquire_cta(&route_ready_s);
      }
      // pool grabs: lane 0 alone touches the counter, the warp shares the
      // value (every lane must walk the same jobs); at most nj + 8 grabs
      for (int it = 0;; ++it) {
        if (it > nj + 8) goto producer_done;
        int idx = held;
        held = -1;
        if (idx < 0) {
          // a grab without one held from the previous layer (layer 0): on
          // the planar batch-1 path nothing else orders it after the launch's
          // reset of the pools, so wait for the layer's first unit, which is
          // published after that reset's grid barrier
          if (warp_routes && !wait_units(l * 64 + 1)) goto producer_done;
          unsigned v = 0;
          if (lane == 0) v = atomicAdd(&ctl->pool[l % 3], 1u);
          idx = (int)__shfl_sync(0xffffffffu, v, 0);
        }
        if (idx >= nj) {
          const Job jb{JOB_END, l, 0, 0, 0};
          const int slot = take_stage(jb);
          if (slot < 0) goto producer_done;
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[slot]);
          next_stage();
          break;
        }
        unsigned nxt = 0;
        if (lane == 0) nxt = atomicAdd(&ctl->pool[l % 3], 1u);  // in flight while the copies issue
        const int ch0 = idx * NCH, n = min(NCH, R1 - ch0);
        Job jb;
        if constexpr (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR) {
          jb = Job{JOB_ROUTED, l, ch0, 0, n};
        } else {
          const int u = ch0 / I;
          jb = Job{JOB_ROUTED, l, u, ch0 - u * I, n};
        }
        const int slot = take_stage(jb);
        if (slot < 0) goto producer_done;
        // planar batch 1: wait only for this job's units (published one by
        // one during the top-k), not for the whole routing
        if (warp_routes && !wait_units(l * 64 + (ch0 + n - 1) / I + 1)) goto producer_done;
        if (lane == 0) {
          uint64_t* bar = &full[slot];
          uint8_t* dst = ring + (size_t)slot * p.stage_bytes;
          if constexpr (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR) {
            const uint32_t cb = 3u * (uint32_t)rowb;
            mbar_expect_tx(bar, (uint32_t)n * cb);
            for (int i = 0; i < n;) {
              const int c0 = kept[ch0 + i];
              int r = 1;
              while (i + r < n && kept[ch0 + i + r] == c0 + r) ++r;
              bulk_g2s(dst + (size_t)i * cb, Lw.gate + (size_t)c0 * cb, (uint32_t)r * cb, bar, pol);
              i += r;
            }
          } else if constexpr (WT == MOE_W_BF16) {
            const int n1 = min(n, I - jb.c0);
            mbar_expect_tx(bar, 3u * (uint32_t)n * rowb);
            for (int sg = 0; sg < 2; ++sg) {
              const int ns = sg ? n - n1 : n1;
              if (ns <= 0) break;
              const int e = rs.unit_e[jb.u + sg];
              const uint32_t bytes = (uint32_t)ns * rowb;
              const size_t off = ((size_t)e * I + (sg ? 0 : jb.c0)) * rowb;
              uint8_t* d0 = dst + (sg ? n1 : 0) * rowb;
              bulk_g2s(d0, Lw.gate + off, bytes, bar, pol);
              bulk_g2s(d0 + NCH * rowb, Lw.up + off, bytes, bar, pol);
              bulk_g2s(d0 + 2 * NCH * rowb, Lw.down + off, bytes, bar, pol);
            }
          } else {
            const int e = rs.unit_e[jb.u];
            const int rowc = H >> 1, rws = H >> 5;
            const uint32_t cbt = (uint32_t)n * rowc, sb = (uint32_t)n * rws;
            const size_t offc = ((size_t)e * I + jb.c0) * rowc, offs = ((size_t)e * I + jb.c0) * rws;
            const size_t offd = ((size_t)e * (I >> 6) + (jb.c0 >> 6)) * rowb;
            mbar_expect_tx(bar, 3 * cbt + 2 * sb + rowb);
            bulk_g2s(dst, Lw.gate + offc, cbt, bar, pol);
            bulk_g2s(dst + NCH * rowc, Lw.up + offc, cbt, bar, pol);
            bulk_g2s(dst + 2 * NCH * rowc, Lw.down + offc, cbt, bar, pol);
            bulk_g2s(dst + 3 * NCH * rowc, Lw.gate_s + offs, sb, bar, pol);
            bulk_g2s(dst + 3 * NCH * rowc + NCH * rws, Lw.up_s + offs, sb, bar, pol);
            bulk_g2s(dst + 3 * NCH * rowc + 2 * NCH * rws, Lw.down_s + offd, rowb, bar, pol);
          }
        }
        __syncwarp();
        next_stage();
        held = (int)__shfl_sync(0xffffffffu, nxt, 0);
      }
      // done with layer l's routing: the consumers may overwrite it; grab
      // ahead for the next layer (its counter was cleared two layers ago)
      if (lane == 0) st_release_cta(&prod_layer_s[pi], l);
      {
        unsigned v = 0;
        if (lane == 0 && l + 1 < p.L) v = atomicAdd(&ctl->pool[(l + 1) % 3], 1u);
        v = __shfl_sync(0xffffffffu, v, 0);
        held = (l + 1 < p.L) ? (int)v : -1;
      }
      // channel-major stacks with given scores: this CTA's 1/G of the next
      // layer's score tensor [E, I] into L2 (every CTA's selection reads the
      // routed rows of it right after routing)
      if (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR && !SCREEN && l + 1 < p.L && pi == 0 && lane == 0) {
        const size_t bytes = (size_t)E * I * 4;
        const size_t b0 = ((size_t)cta * bytes / G) & ~(size_t)15, b1 = ((size_t)(cta + 1) * bytes / G) & ~(size_t)15;
        const uint8_t* sc1 = reinterpret_cast<const uint8_t*>(p.layer[l + 1].scores);
        if (b1 > b0 && ((uintptr_t)sc1 & 15u) == 0) prefetch_l2(sc1 + b0, (uint32_t)(b1 - b0));
      }
    }
    } else {
    // producer pi issues the jobs q with q % kProducers == pi; both walk the
    // whole sequence so that slots and phases stay in step
    const int pi = warp - kWarps;
    const uint64_t pol = policy_evict_first();
    JobCursor pc;
    pc.begin_layer(p, 0);
    long long jp = 0;
    int pslot = 0;
    uint32_t pph = 0;
    int ready = -1;  // routing of layers <= ready is known
    int pub = -1;    // last value published to prod_layer_s
    for (;;) {
      Job j;
      const bool got = next_job(pc, j, ready);
      {
        // once the cursor reaches layer cl, the routing of cl - 1 is no
        // longer read here: let the consumers overwrite it
        const int cl = !got ? pc.layer : (j.type == JOB_END ? p.L : j.layer);
        if (cl - 1 > pub) {
          pub = cl - 1;
          if (lane == 0) st_release_cta(&prod_layer_s[pi], pub);
        }
      }
      if (!got) {
        // the cursor stopped at the routed jobs of pc.layer: poll (plain
        // loads and short sleeps, which leave the shared-memory pipe to the
        // consumers routing meanwhile) until the consumers publish a routed
        // layer >= pc.layer, then one acquire load orders the reads of the
        // routing after it. The published value only grows.
        const long long t0 = clock64();
        while (*(volatile int*)&route_ready_s < pc.layer) {
          if (*(volatile int*)&abort_s || clock64() - t0 > budget) goto producer_done;
          __nanosleep(20);
        }
        (void)ld_acquire_cta(&route_ready_s);
        ready = pc.layer;
        continue;
      }
      if (j.type == JOB_END) break;
      const int slot = pslot;
      if ((int)(jp % kProducers) != pi) {
        ++jp;
        if (++pslot == p.nstages) { pslot = 0; pph ^= 1u; }
        continue;
      }
      if (jp >= p.nstages) {
        const uint32_t par = pph ^ 1u;
        const long long t0 = clock64();
        while (!mbar_try_wait_sleep(&empty[slot], par, 20000)) {
          if (*(volatile int*)&abort_s || clock64() - t0 > budget) goto producer_done;
        }
      }
      {
        uint64_t* bar = &full[slot];
        uint8_t* dst = ring + (size_t)slot * p.stage_bytes;
        const LayerW& Lw = p.layer[j.layer];
        // lane 0 issues the job's copies one after another (one thread
        // issuing is faster than several issuing at once)
        if (lane == 0) {
          if (j.type == JOB_ROUTER) {
            const uint32_t bytes = (uint32_t)j.n * rowb;
            mbar_expect_tx(bar, bytes);
            bulk_g2s(dst, Lw.router + (size_t)j.c0 * rowb, bytes, bar, pol);
          } else if (j.type == JOB_SHARED) {
            const uint32_t bytes = (uint32_t)j.n * rowb;
            const size_t off = (size_t)j.c0 * rowb;
            mbar_expect_tx(bar, 3 * bytes);
            bulk_g2s(dst, Lw.sh_gate + off, bytes, bar, pol);
            bulk_g2s(dst + kShN * rowb, Lw.sh_up + off, bytes, bar, pol);
            bulk_g2s(dst + 2 * kShN * rowb, Lw.sh_down + off, bytes, bar, pol);
          } else if (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR) {
            // one copy per run of consecutive kept channels (12 KB each)
            const uint32_t cb = 3u * (uint32_t)rowb;
            mbar_expect_tx(bar, (uint32_t)j.n * cb);
            for (int i = 0; i < j.n;) {
              const int c0 = kept[j.u + i];
              int r = 1;
              while (i + r < j.n && kept[j.u + i + r] == c0 + r) ++r;
              bulk_g2s(dst + (size_t)i * cb, Lw.gate + (size_t)c0 * cb, (uint32_t)r * cb, bar, pol);
              i += r;
            }
          } else if (WT == MOE_W_BF16) {
            // a job may run on into the next expert: two segments at most
            const int n1 = min(j.n, I - j.c0);
            mbar_expect_tx(bar, 3u * (uint32_t)j.n * rowb);
            for (int sg = 0; sg < 2; ++sg) {
              const int ns = sg ? j.n - n1 : n1;
              if (ns <= 0) break;
              const int e = rs.unit_e[j.u + sg];
              const uint32_t bytes = (uint32_t)ns * rowb;
              const size_t off = ((size_t)e * I + (sg ? 0 : j.c0)) * rowb;
              uint8_t* d0 = dst + (sg ? n1 : 0) * rowb;
              bulk_g2s(d0, Lw.gate + off, bytes, bar, pol);
              bulk_g2s(d0 + NCH * rowb, Lw.up + off, bytes, bar, pol);
              bulk_g2s(d0 + 2 * NCH * rowb, Lw.down + off, bytes, bar, pol);
            }
          } else {
            const int e = rs.unit_e[j.u];
            const int rowc = H >> 1, rows = H >> 5;
            const uint32_t cb = (uint32_t)j.n * rowc, sb = (uint32_t)j.n * rows;
            const size_t offc = ((size_t)e * I + j.c0) * rowc, offs = ((size_t)e * I + j.c0) * rows;
            const size_t offd = ((size_t)e * (I >> 6) + (j.c0 >> 6)) * rowb;
            mbar_expect_tx(bar, 3 * cb + 2 * sb + rowb);
            bulk_g2s(dst, Lw.gate + offc, cb, bar, pol);
            bulk_g2s(dst + NCH * rowc, Lw.up + offc, cb, bar, pol);
            bulk_g2s(dst + 2 * NCH * rowc, Lw.down + offc, cb, bar, pol);
            bulk_g2s(dst + 3 * NCH * rowc, Lw.gate_s + offs, sb, bar, pol);
            bulk_g2s(dst + 3 * NCH * rowc + NCH * rows, Lw.up_s + offs, sb, bar, pol);
            bulk_g2s(dst + 3 * NCH * rowc + 2 * NCH * rows, Lw.down_s + offd, rowb, bar, pol);
          }
        }
        __syncwarp();
      }
      ++jp;
      if (++pslot == p.nstages) { pslot = 0; pph ^= 1u; }
      if (lane == 0) *(volatile long long*)&jp_s[pi] = jp;
    }
    }  // producer model
  producer_done:;
    __syncwarp();
  } else {
    // ============================================================== consumers
    JobCursor ccur;
    ccur.begin_layer(p, 0);
    int cslot = 0;          // stage of the next job
    uint32_t cph = 0;       // its phase parity
    long long jc = 0;       // jobs consumed
    const unsigned long long bar_base = bar_base_s;
    unsigned long long nbar = 0;

    // token b's partial output, elements 8 tid + 2 i and 8 tid + 2 i + 1 in
    // acc[b][i] (fp32 pairs: one packed FMA updates both)
    float2 acc[BMAX][4];
#pragma unroll
    for (int b = 0; b < BMAX; ++b)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[b][i] = make_float2(0.f, 0.f);
    const int H8c = H8;
    const bool has_v = tid < H8;
    int tcn = 0;  // int4 batch path: routed jobs consumed (tcpart buffer tcn % 2)
    const uint32_t all_tokens = (1u << B) - 1u;
    // tensor-core dots (B = 1, H = 2048): x fragments for the 8 segments
    constexpr bool kMmaDots = (BMAX == 1 && HV == 8);
    // fast path: the fragments live in shared memory, [segment][lane] x 16 B
    uint32_t xf_frag[(kMmaDots && !kFast) ? 8 : 1][4];
    uint4* xfs = reinterpret_cast<uint4*>(smem + p.off_xf);
    // fast path: thread t owns elements 8t..8t+7 of x (4 bf16 words). With
    // the pre-norm their u = bf16(x * rsqrt(mean(x^2) + eps)), else u = x;
    // word m of thread t (segment s = t / 32) is word o + 32 k' of that
    // segment's fragment table with o = 4 (t % 8) + m and k' = (t / 8) % 4,
    // i.e. component {0, 2, 1, 3}[k'] of lane 4 (t % 8) + m: each thread
    // writes its own words, no pass through a u buffer.
    auto fast_frags = [&](const float* xv, bool norm) {
      float sc = 1.f;
      if (norm) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(xv[i], xv[i], ss);
        ss = warp_sum(ss);
        if (lane == 0) hbuf[warp][0] = ss;
        cbar();
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) t += hbuf[w][0];
        sc = rsqrtf(t / (float)H + 1e-6f);
      }
      uint32_t* xw = reinterpret_cast<uint32_t*>(xfs);
      const int seg = tid >> 5, kk = (tid >> 3) & 3;
      const int comp = (kk == 1) ? 2 : (kk == 2 ? 1 : kk);
      uint4 uw;
      uint32_t* uwp = reinterpret_cast<uint32_t*>(&uw);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const uint32_t w = uint32_t(f_to_bf16(xv[2 * m] * sc)) | (uint32_t(f_to_bf16(xv[2 * m + 1] * sc)) << 16);
        xw[(seg * 32 + 4 * (tid & 7) + m) * 4 + comp] = w;
        uwp[m] = w;
      }
      // u as plain bf16 for the int4 rows' FMA dots and for the channel screen
      if (kFastI4 || (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR && SCREEN)) reinterpret_cast<uint4*>(us)[tid] = uw;
      cbar();
    };
    auto load_xfrag = [&]() {
      if constexpr (kFast) {
        float xv[8];
        unpack8(xs4[tid], xv);
        fast_frags(xv, MODE == MODE_LAYERS && p.pre_norm);
      } else if constexpr (kMmaDots) {
#pragma unroll
        for (int t = 0; t < 8; ++t) x_frag(us + 256 * t, lane, xf_frag[t]);
      }
    };

    auto arrive_grid = [&]() -> unsigned long long {  // thread 0 only
      red_release_gpu(&ctl->bar, 1ull);
      ++nbar;
      return bar_base + nbar * (unsigned long long)G;
    };
    auto wait_grid = [&](unsigned long long target) -> bool {  // thread 0 only
      // (an injected fault asks for one arrival that never comes)
      if (inject_s & kInjectBarrierExtraArrival) target += 1;
      if (ld_acquire_gpu(&ctl->bar) >= target) return true;
      const long long t0 = clock64();
      while (ld_acquire_gpu(&ctl->bar) < target)
        if (clock64() - t0 > budget) return false;
      return true;
    };
    auto grid_sync = [&]() -> bool {
      cbar();
      if (tid == 0) okw_s = wait_grid(arrive_grid()) ? 1 : 0;
      cbar();
      return okw_s != 0;
    };
    // bounded mbarrier wait that gives up at once after an abort
    auto wait_mb = [&](uint64_t* bar, uint32_t parity) -> bool {
      if (mbar_try_wait_sleep(bar, parity, 20000)) return true;
      const long long t0 = clock64();
      while (!mbar_try_wait_sleep(bar, parity, 20000)) {
        if (*(volatile int*)&abort_s || clock64() - t0 > budget) return false;
      }
      return true;
    };

    // Dot products of RPW rows (one warp's share of a job) with token b's x,
    // summed over the warp. Lane takes vectors v = i*32 + lane of H; HV =
    // H/256 vectors per lane when H is a multiple of 256 (no guards, x loaded
    // once for all rows), else a guarded generic loop. int4 rows carry one
    // bf16 scale per 64 elements (sc[r][v >> 3]).
    auto rows_dot = [&](const uint8_t* const* rowp, const uint16_t* const* scp, int nrows, int b, bool int4row,
                        float* out) {
      constexpr int RPW = NCH * 2 / kWarps > 0 ? NCH * 2 / kWarps : 1;
      float s8[RPW][8];
#pragma unroll
      for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int e = 0; e < 8; ++e) s8[r][e] = 0.f;
      const uint4* xb = us4 + b * H8c;
      if constexpr (kMmaDots) {
        if (!int4row) {
          float d0[RPW][4], d1[RPW][4];
#pragma unroll
          for (int r = 0; r < RPW; ++r)
#pragma unroll
            for (int i = 0; i < 4; ++i) { d0[r][i] = 0.f; d1[r][i] = 0.f; }
#pragma unroll
          for (int t = 0; t < 8; ++t)
#pragma unroll
            for (int r = 0; r < RPW; ++r)
              if (r < nrows) {
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4(smem_u32(rowp[r]) + 512 * t + 16 * lane, a0, a1, a2, a3);
                mma_bf16_16816(d0[r], a0, a1, a2, a3, xf_frag[t][0], xf_frag[t][1]);
                mma_bf16_16816(d1[r], a0, a1, a2, a3, xf_frag[t][2], xf_frag[t][3]);
              }
#pragma unroll
          for (int r = 0; r < RPW; ++r) out[r] = warp_sum(diag_part(d0[r], d1[r], lane));
          return;
        }
      }
      if (HV > 0) {
#pragma unroll
        for (int i = 0; i < (HV > 0 ? HV : 1); ++i) {
          const int v = i * 32 + lane;
          float xf[8];
          unpack8(xb[v], xf);
#pragma unroll
          for (int r = 0; r < RPW; ++r)
            if (r < nrows) {
              float wf[8];
              if (!int4row) {
                unpack8(reinterpret_cast<const uint4*>(rowp[r])[v], wf);
              } else {
                int4x8_to_f(reinterpret_cast<const uint32_t*>(rowp[r])[v], wf);
                const float sv = bf16_to_f(scp[r][v >> 3]);
#pragma unroll
                for (int e = 0; e < 8; ++e) wf[e] *= sv;
              }
#pragma unroll
              for (int e = 0; e < 8; ++e) s8[r][e] = fmaf(wf[e], xf[e], s8[r][e]);
            }
        }
      } else {
        for (int v = lane; v < H8c; v += 32) {
          float xf[8];
          unpack8(xb[v], xf);
#pragma unroll
          for (int r = 0; r < RPW; ++r)
            if (r < nrows) {
              float wf[8];
              if (!int4row) unpack8(reinterpret_cast<const uint4*>(rowp[r])[v], wf);
              else {
                int4x8_to_f(reinterpret_cast<const uint32_t*>(rowp[r])[v], wf);
                const float sv = bf16_to_f(scp[r][v >> 3]);
#pragma unroll
                for (int e = 0; e < 8; ++e) wf[e] *= sv;
              }
#pragma unroll
              for (int e = 0; e < 8; ++e) s8[r][e] = fmaf(wf[e], xf[e], s8[r][e]);
            }
        }
      }
#pragma unroll
      for (int r = 0; r < RPW; ++r) {
        const float t = ((s8[r][0] + s8[r][1]) + (s8[r][2] + s8[r][3])) + ((s8[r][4] + s8[r][5]) + (s8[r][6] + s8[r][7]));
        out[r] = warp_sum(t);
      }
    };

    // ---- one job, per warp: its dot rows, then (after all warps' dots) the
    // SwiGLU activations and this thread's H-slice of the down projection
    auto consume = [&](const Job& j) -> bool {
      constexpr int RPW = NCH * 2 / kWarps > 0 ? NCH * 2 / kWarps : 1;
      const int slot = cslot;
      const uint32_t ph = cph;
      const uint8_t* st = ring + (size_t)slot * p.stage_bytes;
      bool ok = wait_mb(&full[slot], ph);
      // token masks and router weights of the (at most two) segments
      uint32_t mask0, mask1 = 0u;
      const float* wts0 = nullptr;
      const float* wts1 = nullptr;
      int n1 = j.n;
      if (j.type == JOB_ROUTER || j.type == JOB_SHARED) mask0 = all_tokens;
      else if (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR) {
        mask0 = 1u;
        const int e = j.c0 / I;
        int u = 0;
        while (u < rs.U - 1 && rs.unit_e[u] != e) ++u;
        wts0 = &rs.unit_w[u][0];
      } else {
        mask0 = rs.unit_mask[j.u];
        wts0 = rs.unit_w[j.u];
        if (WT == MOE_W_BF16) {
          n1 = min(j.n, I - j.c0);
          if (n1 < j.n) { mask1 = rs.unit_mask[j.u + 1]; wts1 = rs.unit_w[j.u + 1]; }
        }
      }
      const uint32_t mask_any = mask0 | mask1;
      if constexpr (kTcB) {
        if (j.type == JOB_SHARED || j.type == JOB_ROUTER) {
          // bf16 rows n at st + n rowb with all tokens: one shared channel
          // (gate n = 0, up n = 1) or the job's router rows; the same
          // tensor-core split of H over the warps (no scales: the pairs
          // {8 w + i, 8 w + i + 4} of the rows themselves)
          const int tb = tcn & 1;
          ++tcn;
          const int nrows = j.type == JOB_SHARED ? 2 : j.n;
          if (ok) {
            const int n = lane >> 2, q = lane & 3;
            const uint4* wr = reinterpret_cast<const uint4*>(st + (size_t)(n < nrows ? n : 0) * rowb) + 2 * q;
            const uint4* xfr = us4 + 256 * warp + lane;  // this warp's A fragments
            const bool wact = n < nrows;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int g = 0; g < 4; ++g)
#pragma unroll
              for (int s2 = 0; s2 < 2; ++s2) {
                const int w8 = 8 * (4 * warp + g) + s2;
                const uint4 v = xfr[64 * g + 32 * s2];
                const uint4 wv = wact ? wr[w8] : make_uint4(0u, 0u, 0u, 0u);
                mma_bf16_16816(d, v.x, 0u, v.y, 0u, __byte_perm(wv.x, wv.z, 0x5410), __byte_perm(wv.x, wv.z, 0x7632));
                mma_bf16_16816(d, v.z, 0u, v.w, 0u, __byte_perm(wv.y, wv.w, 0x5410), __byte_perm(wv.y, wv.w, 0x7632));
              }
            tcpart[tb][warp][q * 8 + (lane >> 2)] = make_float2(d[0], d[1]);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&hready[slot]);
          ok = ok && wait_mb(&hready[slot], ph);
          if (ok && j.type == JOB_ROUTER) {
            // warp 0: lane (q = lane / 8, token m = lane % 8) sums rows 2 q
            // and 2 q + 1 over the warps into the logits
            if (warp == 0) {
              float2 v2 = tcpart[tb][0][lane];
#pragma unroll
              for (int w = 1; w < kWarps; ++w) {
                const float2 v = tcpart[tb][w][lane];
                v2.x += v.x;
                v2.y += v.y;
              }
              const int q = lane >> 3, m = lane & 7;
              if (m < B) {
                if (2 * q < j.n) p.logits[(size_t)m * E + j.c0 + 2 * q] = v2.x;
                if (2 * q + 1 < j.n) p.logits[(size_t)m * E + j.c0 + 2 * q + 1] = v2.y;
              }
            }
          } else if (ok) {
            if (lane < 8) {
              float2 gu = tcpart[tb][0][lane];
#pragma unroll
              for (int w = 1; w < kWarps; ++w) {
                const float2 v = tcpart[tb][w][lane];
                gu.x += v.x;
                gu.y += v.y;
              }
              const float h = lane < B ? silu_f(gu.x) * gu.y : 0.f;
              hb2[warp][lane] = make_float2(h, h);
            }
            __syncwarp();
            float dv[8];
            unpack8(reinterpret_cast<const uint4*>(st + 2 * kShN * rowb)[tid], dv);
            float4* ysb = reinterpret_cast<float4*>(smem + p.off_ysum);
            for (int b2 = 0; b2 < B; ++b2) {
              float4* ya = ysb + b2 * (H >> 2) + tid;
              const float4 y0 = ya[0], y1 = ya[H >> 3];
              const float2 hh = hb2[warp][b2];
              const float2 a0 = __ffma2_rn(make_float2(dv[0], dv[1]), hh, make_float2(y0.x, y0.y));
              const float2 a1 = __ffma2_rn(make_float2(dv[2], dv[3]), hh, make_float2(y0.z, y0.w));
              const float2 a2 = __ffma2_rn(make_float2(dv[4], dv[5]), hh, make_float2(y1.x, y1.y));
              const float2 a3 = __ffma2_rn(make_float2(dv[6], dv[7]), hh, make_float2(y1.z, y1.w));
              ya[0] = make_float4(a0.x, a0.y, a1.x, a1.y);
              ya[H >> 3] = make_float4(a2.x, a2.y, a3.x, a3.y);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[slot]);
          if (++cslot == p.nstages) { cslot = 0; cph ^= 1u; }
          ++jc;
          if (!ok) *(volatile int*)&abort_s = 1;
          return ok;
        }
        if (j.type == JOB_ROUTED) {
          // 1. warp w: elements 256 w .. 256 w + 255 of the job's 8 rows (row
          // n = 2 ch + mat) for all 8 tokens. mma D[m][n] (m: token, n: row)
          // per 64-element group, scaled by the group's scale of row n: lane
          // (m, q) ends with token m's gate and up partials of channel q.
          const int tb = tcn & 1;
          ++tcn;
          if (ok) {
            const int n = lane >> 2, q = lane & 3;
            const uint8_t* wrow = st + (n >> 1) * (H >> 1) + (n & 1) * (NCH * (H >> 1));
            const uint16_t* sgp = reinterpret_cast<const uint16_t*>(st + 3 * NCH * (H >> 1)) + q * (H >> 6);
            const uint16_t* sup = sgp + NCH * (H >> 6);
            // A fragments (build_xfrags): token m's elements 8 w + i and
            // 8 w + i + 4 of its words w = 8 G + 2 q + s, the pairs
            // int4_pair_bf16 makes of the codes (rows m >= B are zero)
            const uint4* xfr = us4 + 256 * warp + lane;
            // one accumulator per group: four independent mma chains
            float d[4][4];
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const int G = 4 * warp + g;
              const uint2 wv = *reinterpret_cast<const uint2*>(wrow + 4 * (8 * G + 2 * q));
#pragma unroll
              for (int i = 0; i < 4; ++i) d[g][i] = 0.f;
#pragma unroll
              for (int s2 = 0; s2 < 2; ++s2) {
                const uint32_t w = s2 ? wv.y : wv.x;
                const uint4 v = xfr[64 * g + 32 * s2];
                mma_bf16_16816(d[g], v.x, 0u, v.y, 0u, int4_pair_bf16(w, 0), int4_pair_bf16(w, 1));
                mma_bf16_16816(d[g], v.z, 0u, v.w, 0u, int4_pair_bf16(w, 2), int4_pair_bf16(w, 3));
              }
            }
            float pg = 0.f, pu = 0.f;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              pg = fmaf(bf16_to_f(sgp[4 * warp + g]), d[g][0], pg);
              pu = fmaf(bf16_to_f(sup[4 * warp + g]), d[g][1], pu);
            }
            tcpart[tb][warp][q * 8 + n] = make_float2(pg, pu);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&hready[slot]);
          // 2. the job's down rows, scaled, while the other warps finish their
          // dots (codes of channels c >= j.n are stale but finite, and their
          // h is 0); then every warp: the 32 activations (lane = 8 ch + b)
          // from the 8 warps' partials, and thread tid's 8 outputs of each
          // routed token: elements 8 tid .. 8 tid + 3 at float4 slot tid of
          // the token's first half, 8 tid + 4 .. 8 tid + 7 in its second
          float2 q2[NCH][4];
          if (ok) {
            float sv[8];
            unpack8(reinterpret_cast<const uint4*>(st + 3 * NCH * (H >> 1) + 2 * NCH * (H >> 5))[tid], sv);
#pragma unroll
            for (int c2 = 0; c2 < NCH; ++c2) {
              float qv[8];
              int4x8_to_f(reinterpret_cast<const uint32_t*>(st + 2 * NCH * (H >> 1) + c2 * (H >> 1))[tid], qv);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                q2[c2][i] = __fmul2_rn(make_float2(qv[2 * i], qv[2 * i + 1]), make_float2(sv[2 * i], sv[2 * i + 1]));
            }
          }
          ok = ok && wait_mb(&hready[slot], ph);
          if (ok) {
            float2 gu = tcpart[tb][0][lane];
#pragma unroll
            for (int w = 1; w < kWarps; ++w) {
              const float2 v = tcpart[tb][w][lane];
              gu.x += v.x;
              gu.y += v.y;
            }
            const int ch = lane >> 3, b = lane & 7;
            float h = 0.f;
            if (ch < j.n && ((mask0 >> b) & 1u)) h = wts0[b] * silu_f(gu.x) * gu.y;
            hb2[warp][lane] = make_float2(h, h);
            __syncwarp();
            float4* ysb = reinterpret_cast<float4*>(smem + p.off_ysum);
            for (uint32_t mm = mask0; mm != 0u; mm &= mm - 1u) {
              const int b2 = __ffs(mm) - 1;
              float4* ya = ysb + b2 * (H >> 2) + tid;
              const float4 y0 = ya[0], y1 = ya[H >> 3];
              float2 a[4] = {make_float2(y0.x, y0.y), make_float2(y0.z, y0.w), make_float2(y1.x, y1.y),
                             make_float2(y1.z, y1.w)};
#pragma unroll
              for (int c2 = 0; c2 < NCH; ++c2) {
                const float2 hh = hb2[warp][8 * c2 + b2];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = __ffma2_rn(q2[c2][i], hh, a[i]);
              }
              ya[0] = make_float4(a[0].x, a[0].y, a[1].x, a[1].y);
              ya[H >> 3] = make_float4(a[2].x, a[2].y, a[3].x, a[3].y);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[slot]);
          if (++cslot == p.nstages) { cslot = 0; cph ^= 1u; }
          ++jc;
          if (!ok) *(volatile int*)&abort_s = 1;
          return ok;
        }
      }
      int ch_stride, mat_stride, down_off;
      if (j.type == JOB_ROUTER) { ch_stride = rowb; mat_stride = 0; down_off = 0; }
      else if (j.type == JOB_SHARED) { ch_stride = rowb; mat_stride = kShN * rowb; down_off = 2 * kShN * rowb; }
      else if (LAYOUT == MOE_LAYOUT_PLANAR && WT == MOE_W_BF16) {
        ch_stride = rowb; mat_stride = NCH * rowb; down_off = 2 * NCH * rowb;
      } else if (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR) {
        ch_stride = 3 * rowb; mat_stride = rowb; down_off = 2 * rowb;
      } else {
        ch_stride = H >> 1; mat_stride = NCH * (H >> 1); down_off = 2 * NCH * (H >> 1);
      }
      const bool int4_rows = (WT == MOE_W_INT4_G64) && (j.type == JOB_ROUTED);
      const int ndot = (j.type == JOB_ROUTER) ? j.n : 2 * j.n;
      float* db = dotbuf[slot];
      // 1. this warp's dot rows: rows warp + 8*i
      if (ok) {
        const uint8_t* rowp[RPW];
        const uint16_t* scp[RPW];
        int nr = 0;
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
          const int r = warp + kWarps * i;
          const int ch = (j.type == JOB_ROUTER) ? r : (r >> 1);
          const int mat = (j.type == JOB_ROUTER) ? 0 : (r & 1);
          rowp[i] = st + ch * ch_stride + mat * mat_stride;
          scp[i] = int4_rows ? reinterpret_cast<const uint16_t*>(st + 3 * NCH * (H >> 1) + (mat * NCH + ch) * (H >> 5))
                             : nullptr;
          if (r < ndot) nr = i + 1;
        }
        if (nr > 0) {
#pragma unroll
          for (int b = 0; b < BMAX; ++b)
            if ((mask_any >> b) & 1u) {
              float t[RPW];
              rows_dot(rowp, scp, nr, b, int4_rows, t);
              if (lane == 0)
#pragma unroll
                for (int i = 0; i < RPW; ++i)
                  if (i < nr) {
                    const int r = warp + kWarps * i;
                    if (j.type == JOB_ROUTER) p.logits[b * E + j.c0 + r] = t[i];
                    else db[r * BMAX + b] = t[i];
                  }
            }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&hready[slot]);
      // 2. SwiGLU activations and the down projection, once every warp's dots are in
      if (j.type != JOB_ROUTER) {
        ok = ok && wait_mb(&hready[slot], ph);
        if (ok) {
          for (int idx = lane; idx < NCH * BMAX; idx += 32) {
            const int ch = idx / BMAX, b = idx % BMAX;
            const uint32_t m = ch < n1 ? mask0 : mask1;
            const float* wt = ch < n1 ? wts0 : wts1;
            float h = 0.f;
            if (ch < j.n && ((m >> b) & 1u)) {
              const float g = db[(2 * ch) * BMAX + b], u = db[(2 * ch + 1) * BMAX + b];
              h = (wt ? wt[b] : 1.f) * silu_f(g) * u;
            }
            hbuf[warp][idx] = h;
          }
          __syncwarp();
          // (the int4 batch path handles its shared and routed jobs above)
          if (!kTcB && has_v) {
            if (!int4_rows) {
#pragma unroll
              for (int ch = 0; ch < NCH; ++ch)
                if (ch < j.n) {
                  float d[8];
                  unpack8(reinterpret_cast<const uint4*>(st + down_off + ch * ch_stride)[tid], d);
                  const uint32_t m = ch < n1 ? mask0 : mask1;
#pragma unroll
                  for (int b = 0; b < BMAX; ++b)
                    if ((m >> b) & 1u) {
                      const float h = hbuf[warp][ch * BMAX + b];
                      const float2 hh = make_float2(h, h);
#pragma unroll
                      for (int i = 0; i < 4; ++i) acc[b][i] = __ffma2_rn(make_float2(d[2 * i], d[2 * i + 1]), hh, acc[b][i]);
                    }
                }
            } else {
              const int rows = H >> 5;
              float s[8];
              unpack8(reinterpret_cast<const uint4*>(st + 3 * NCH * (H >> 1) + 2 * NCH * rows)[tid], s);
              // the output's scale (one per 64-channel group, the job's group)
              // folded into each product, so no second accumulator set is live
#pragma unroll
              for (int ch = 0; ch < NCH; ++ch)
                if (ch < j.n) {
                  float q[8];
                  int4x8_to_f(reinterpret_cast<const uint32_t*>(st + down_off + ch * ch_stride)[tid], q);
#pragma unroll
                  for (int i = 0; i < 8; ++i) q[i] *= s[i];
#pragma unroll
                  for (int b = 0; b < BMAX; ++b)
                    if ((mask0 >> b) & 1u) {
                      const float h = hbuf[warp][ch * BMAX + b];
                      const float2 hh = make_float2(h, h);
#pragma unroll
                      for (int i = 0; i < 4; ++i) acc[b][i] = __ffma2_rn(make_float2(q[2 * i], q[2 * i + 1]), hh, acc[b][i]);
                    }
                }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      if (++cslot == p.nstages) { cslot = 0; cph ^= 1u; }
      ++jc;
      if (!ok) *(volatile int*)&abort_s = 1;
      return ok;
    };

    // ---- batch-1 bf16 fast path: a warp owns whole channels. Each job of the
    // sequence goes to one warp group (NCH warps; job q to group q % kGroups);
    // warp wi of the group takes channel wi of the job: its gate and up dots,
    // h = w_e SiLU(g) u, and its down row, accumulated in 64 registers per
    // lane (elements 256 i + 8 lane + e). Warps never wait for one another
    // inside a job; the stage is released once the group's NCH warps arrive.
    // Router jobs give warp wi the rows wi and wi + NCH.
    float accf[kFast ? 64 : 1];
#pragma unroll
    for (int i = 0; i < (kFast ? 64 : 1); ++i) accf[i] = 0.f;
    const int my_group = kFast ? warp / NCH : 0;
    const int wi = kFast ? warp % NCH : 0;
    // dots of one or two bf16 rows of 2048 elements with us (tensor-core
    // diagonals, 8 segments of 256); every lane receives both sums
    auto dot2 = [&](const uint8_t* r0, const uint8_t* r1, bool two, float& o0, float& o1) {
      float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
      float b0[4] = {0.f, 0.f, 0.f, 0.f}, b1[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (kFast) {
        const uint32_t s0 = smem_u32(r0) + 16 * lane, s1 = smem_u32(r1) + 16 * lane;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const uint4 xf = xfs[32 * t + lane];
          uint32_t q0, q1, q2, q3;
          ldmatrix_x4(s0 + 512 * t, q0, q1, q2, q3);
          mma_bf16_16816(a0, q0, q1, q2, q3, xf.x, xf.y);
          mma_bf16_16816(a1, q0, q1, q2, q3, xf.z, xf.w);
          if (two) {
            ldmatrix_x4(s1 + 512 * t, q0, q1, q2, q3);
            mma_bf16_16816(b0, q0, q1, q2, q3, xf.x, xf.y);
            mma_bf16_16816(b1, q0, q1, q2, q3, xf.z, xf.w);
          }
        }
      }
      o0 = warp_sum(diag_part(a0, a1, lane));
      o1 = two ? warp_sum(diag_part(b0, b1, lane)) : 0.f;
    };
    // named barrier of this warp's group (ids 2.., NCH warps)
    auto group_bar = [&]() {
      asm volatile("bar.sync %0, %1;" ::"r"(2 + my_group), "r"(NCH * 32) : "memory");
    };
    // run one job that has landed in `slot` (fast path)
    auto run_job = [&](const Job& j, int slot, int buf) {
      {
        if (j.type == JOB_ROUTER) {
          // rows split over K: warp wi of the group takes segments
          // [wi * SPW, (wi + 1) * SPW) of every row; the last warp of the
          // group to finish (a shared counter, double-buffered by job) sums
          // the partials and writes the logits, so no warp waits for another
          constexpr int SPW = 8 / NCH;
          float* part = dotbuf[warp + kWarps * buf];
          const uint8_t* st = ring + (size_t)slot * p.stage_bytes;
          const uint32_t sbase = smem_u32(st) + 16 * lane;
          for (int r = 0; r < j.n; ++r) {
            float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int q = 0; q < SPW; ++q) {
              const int t = wi * SPW + q;
              const uint4 xf = xfs[32 * t + lane];
              uint32_t q0, q1, q2, q3;
              ldmatrix_x4(sbase + r * rowb + 512 * t, q0, q1, q2, q3);
              mma_bf16_16816(a0, q0, q1, q2, q3, xf.x, xf.y);
              mma_bf16_16816(a1, q0, q1, q2, q3, xf.z, xf.w);
            }
            const float pv = warp_sum(diag_part(a0, a1, lane));
            if (lane == 0) part[r] = pv;
          }
          if (lane == 0) {
            __threadfence_block();
            int* cnt = &rcnt_s[2 * my_group + buf];
            if (atomicAdd(cnt, 1) == NCH - 1) {
              __threadfence_block();
              for (int r = 0; r < j.n; ++r) {
                float t = 0.f;
                for (int w = 0; w < NCH; ++w) t += dotbuf[my_group * NCH + w + kWarps * buf][r];
                if (k <= kWarps) {
                  // {value, tag}: readers poll the word itself, no router barrier.
                  // A prediction job (u = 1) holds the next layer's router
                  // rows: its words carry the next layer's tag.
                  const bool pred = j.u != 0;
                  const unsigned long long tag =
                      (unsigned long long)(0x80000000u | (ltag_s + (uint32_t)(j.layer + (pred ? 1 : 0))));
                  const unsigned long long word = (tag << 32) | __float_as_uint(t);
                  if (pred) {
                    st_relaxed_gpu_u64(p.plogits + (size_t)((j.layer + 1) & 1) * E + j.c0 + r, word);
                  } else {
                    st_relaxed_gpu_u64(reinterpret_cast<unsigned long long*>(p.logits) + j.c0 + r, word);
                  }
                } else {
                  p.logits[j.c0 + r] = t;  // read after the router barrier
                }
              }
              *cnt = 0;
            }
          }
        } else {
          const uint8_t* st = ring + (size_t)slot * p.stage_bytes;
          if (kFastI4 && j.type == JOB_ROUTED) {
            if (wi < j.n) {
              // int4 channel: codes of its gate/up rows (H/2 bytes each) and
              // their bf16 scales (one per 64 inputs); lane v-vectors of 8
              // inputs, v = 32 i + lane, scale index v / 8. The down row's
              // codes are scaled per output by the job's scale row.
              const int rowc = H >> 1, rws = H >> 5;
              const uint32_t* gc = reinterpret_cast<const uint32_t*>(st + wi * rowc);
              const uint32_t* uc = reinterpret_cast<const uint32_t*>(st + NCH * rowc + wi * rowc);
              const uint32_t* dc = reinterpret_cast<const uint32_t*>(st + 2 * NCH * rowc + wi * rowc);
              const uint16_t* gs = reinterpret_cast<const uint16_t*>(st + 3 * NCH * rowc + wi * rws);
              const uint16_t* ust = reinterpret_cast<const uint16_t*>(st + 3 * NCH * rowc + NCH * rws + wi * rws);
              const uint4* ds = reinterpret_cast<const uint4*>(st + 3 * NCH * rowc + 2 * NCH * rws);
              float ga = 0.f, ua = 0.f;
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int v = 32 * i + lane;
                float xf[8], qg[8], qu[8];
                unpack8(us4[v], xf);
                int4x8_to_f(gc[v], qg);
                int4x8_to_f(uc[v], qu);
                float pg = 0.f, pu = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  pg = fmaf(qg[e], xf[e], pg);
                  pu = fmaf(qu[e], xf[e], pu);
                }
                ga = fmaf(bf16_to_f(gs[v >> 3]), pg, ga);
                ua = fmaf(bf16_to_f(ust[v >> 3]), pu, ua);
              }
              const float gv = warp_sum(ga), uv = warp_sum(ua);
              const float h = rs.unit_w[j.u][0] * silu_f(gv) * uv;
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int v = 32 * i + lane;
                float q[8], sv[8];
                int4x8_to_f(dc[v], q);
                unpack8(ds[v], sv);
#pragma unroll
                for (int e = 0; e < 8; ++e) accf[8 * i + e] = fmaf(h * sv[e], q[e], accf[8 * i + e]);
              }
            }
          } else if (wi < j.n) {
            const uint8_t *g, *u, *d;
            float wt;
            if (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR && j.type == JOB_ROUTED) {
              g = st + (size_t)wi * 3 * rowb;
              u = g + rowb;
              d = g + 2 * rowb;
              const int e = kept[j.u + wi] / I;
              int q = 0;
              while (q < rs.U - 1 && rs.unit_e[q] != e) ++q;
              wt = rs.unit_w[q][0];
            } else {
              g = st + wi * rowb;
              u = g + NCH * rowb;
              d = g + 2 * NCH * rowb;
              if (j.type == JOB_SHARED) wt = 1.f;
              else wt = rs.unit_w[j.u + (wi < I - j.c0 ? 0 : 1)][0];
            }
            float gv, uv;
            dot2(g, u, true, gv, uv);
            const float h = wt * silu_f(gv) * uv;
            const uint4* d4 = reinterpret_cast<const uint4*>(d);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float dv[8];
              unpack8(d4[32 * i + lane], dv);
#pragma unroll
              for (int e = 0; e < 8; ++e) accf[8 * i + e] = fmaf(h, dv[e], accf[8 * i + e]);
            }
          }
        }
      }
    };
    // fast path: take this group's next job from its pipeline, run it and
    // release the stage; returns the job type (JOB_END closes the routed
    // phase) or -1 when the wait failed
    const int cnps = kFast ? (p.nstages - my_group + kPipes - 1) / kPipes : 1;
    int cpm = 0;
    uint32_t cpph = 0;
    long long lc = 0;
    auto consume_pipe = [&]() -> int {
      const int slot = my_group + kPipes * cpm;
      const bool ok = wait_mb(&full[slot], cpph);
      int ty = -1;
      if (ok) {
        const Job j = jdesc[slot];
        ty = j.type;
        if (ty != JOB_END) run_job(j, slot, (int)(lc & 1));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      ++lc;
      if (++cpm == cnps) { cpm = 0; cpph ^= 1u; }
      if (lane == 0 && wi == 0) *(volatile long long*)&jcg_s[my_group] = lc;
      if (!ok) *(volatile int*)&abort_s = 1;
      return ty;
    };

    // ---- pre-norm: us[b] = bf16(x[b] / sqrt(mean(x[b]^2) + eps)), unit weight
    // (x is read twice from shared memory, once for the sums of squares and
    // once to scale, so that no token's values stay live in registers)
    auto normalize_x = [&]() {
      float ss[BMAX];
#pragma unroll
      for (int b = 0; b < BMAX; ++b) {
        ss[b] = 0.f;
        if (b < B && has_v) {
          float xv[8];
          unpack8(xs4[b * H8c + tid], xv);
#pragma unroll
          for (int i = 0; i < 8; ++i) ss[b] = fmaf(xv[i], xv[i], ss[b]);
        }
      }
#pragma unroll
      for (int b = 0; b < BMAX; ++b) {
        const float t = warp_sum(ss[b]);
        if (lane == 0) hbuf[warp][b] = t;
      }
      cbar();
#pragma unroll
      for (int b = 0; b < BMAX; ++b)
        if (b < B && has_v) {
          float t = 0.f;
#pragma unroll
          for (int w = 0; w < kWarps; ++w) t += hbuf[w][b];
          const float sc = rsqrtf(t / (float)H + 1e-6f);
          float xv[8];
          unpack8(xs4[b * H8c + tid], xv);
          uint4 o;
          o.x = uint32_t(f_to_bf16(xv[0] * sc)) | (uint32_t(f_to_bf16(xv[1] * sc)) << 16);
          o.y = uint32_t(f_to_bf16(xv[2] * sc)) | (uint32_t(f_to_bf16(xv[3] * sc)) << 16);
          o.z = uint32_t(f_to_bf16(xv[4] * sc)) | (uint32_t(f_to_bf16(xv[5] * sc)) << 16);
          o.w = uint32_t(f_to_bf16(xv[6] * sc)) | (uint32_t(f_to_bf16(xv[7] * sc)) << 16);
          reinterpret_cast<uint4*>(us)[b * H8c + tid] = o;
        }
      cbar();
    };
    // int4 batch path: u as the tensor-core A fragments, one uint4 per
    // (warp w, group g, half s, lane) at entry 256 w + 64 g + 32 s + lane: for
    // lane (m = lane / 4, q = lane % 4) the bf16 pairs {u[m][8 W + i],
    // u[m][8 W + i + 4]}, i = 0..3, of word W = 8 (4 w + g) + 2 q + s, zero for
    // m >= B; u = bf16(x * rsqrt(mean(x^2) + eps)) with the pre-norm, else x
    __shared__ float xsc_s[kMaxB];
    auto build_xfrags = [&](bool norm) {
      if constexpr (kTcB) {
        if (norm) {
          float ss[BMAX];
#pragma unroll
          for (int b = 0; b < BMAX; ++b) {
            ss[b] = 0.f;
            if (b < B) {
              float xv[8];
              unpack8(xs4[b * H8c + tid], xv);
#pragma unroll
              for (int i = 0; i < 8; ++i) ss[b] = fmaf(xv[i], xv[i], ss[b]);
            }
          }
#pragma unroll
          for (int b = 0; b < BMAX; ++b) {
            const float t = warp_sum(ss[b]);
            if (lane == 0) hbuf[warp][b] = t;
          }
          cbar();
          if (tid < B) {
            float t = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) t += hbuf[w][tid];
            xsc_s[tid] = rsqrtf(t / (float)H + 1e-6f);
          }
          cbar();
        }
        uint4* xf4 = reinterpret_cast<uint4*>(us);
        for (int e = tid; e < 8 * H8c; e += kConsumers) {
          const int le = e & 31, m = le >> 2;
          uint4 o = make_uint4(0u, 0u, 0u, 0u);
          if (m < B) {
            float xv[8];
            unpack8(xs4[m * H8c + 8 * (e >> 6) + 2 * (le & 3) + ((e >> 5) & 1)], xv);
            const float c = norm ? xsc_s[m] : 1.f;
            uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              ow[i] = uint32_t(f_to_bf16(xv[i] * c)) | (uint32_t(f_to_bf16(xv[i + 4] * c)) << 16);
          }
          xf4[e] = o;
        }
        cbar();
      }
    };
    if constexpr (kTcB) build_xfrags(MODE == MODE_LAYERS && p.pre_norm);
    else if constexpr (MODE == MODE_LAYERS && !kFast)
      if (p.pre_norm) normalize_x();
    load_xfrag();

    // ---- routed units from rs.ids / rs.w (ascending expert ids)
    auto build_units = [&]() -> bool {
      if (tid == 0) bad_s = 0;
      if constexpr (BMAX == 1) {
        cbar();
        if (warp == 0) {
          const int e = lane < k ? rs.ids[0][lane] : 0x7fffffff;
          const float wl = lane < k ? rs.w[0][lane] : 0.f;
          int rank = 0, dup = 0;
          for (int i = 0; i < k; ++i) {
            const int o = __shfl_sync(0xffffffffu, e, i);
            rank += (o < e) || (o == e && i < lane);
            dup |= (o == e && i != lane);
          }
          if (lane < k) {
            const bool valid = e >= 0 && e < E && !dup;
            rs.unit_e[rank] = valid ? e : 0;
            rs.unit_mask[rank] = valid ? 1u : 0u;
            rs.unit_w[rank][0] = valid ? wl : 0.f;
            if (!valid) bad_s = 1;
          }
          if (lane == 0) rs.U = k;
        }
        cbar();
        return bad_s == 0;
      } else {
      const int nw = (E + 31) >> 5;
      for (int i = tid; i < nw; i += kConsumers) rs.bitmap[i] = 0u;
      cbar();
      for (int t = tid; t < B * k; t += kConsumers) {
        const int e = rs.ids[t / k][t % k];
        if (e < 0 || e >= E) bad_s = 1;
        else atomicOr(&rs.bitmap[e >> 5], 1u << (e & 31));
      }
      cbar();
      if (warp == 0) {
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
      cbar();
      for (int u = tid; u < rs.U; u += kConsumers) {
        rs.unit_mask[u] = 0u;
#pragma unroll
        for (int b = 0; b < BMAX; ++b) rs.unit_w[u][b] = 0.f;
      }
      for (int e = tid; e < E; e += kConsumers)
        if ((rs.bitmap[e >> 5] >> (e & 31)) & 1u)
          rs.unit_e[rs.rank_base[e >> 5] + __popc(rs.bitmap[e >> 5] & ((1u << (e & 31)) - 1u))] = e;
      cbar();
      for (int t = tid; t < B * k; t += kConsumers) {
        const int b = t / k, e = rs.ids[b][t % k];
        if (e < 0 || e >= E) continue;
        const int u = rs.rank_base[e >> 5] + __popc(rs.bitmap[e >> 5] & ((1u << (e & 31)) - 1u));
        const uint32_t old = atomicOr(&rs.unit_mask[u], 1u << b);
        if (old & (1u << b)) bad_s = 1;
        else rs.unit_w[u][b] = rs.w[b][t % k];
      }
      cbar();
      // cost offsets of the units (lane l: units 8 l .. 8 l + 7), for the
      // split of the routed channels over the CTAs
      if (warp == 0) {
        const int U = rs.U;
        int c[8], tot = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int u = 8 * lane + i;
          c[i] = u < U ? I * (kJobW + __popc(rs.unit_mask[u])) : 0;
          tot += c[i];
        }
        int inc = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += t;
        }
        int base = inc - tot;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int u = 8 * lane + i;
          if (u <= U) rs.cpre[u] = base;
          base += c[i];
        }
        if (lane == 31) rs.cpre[U] = inc;
      }
      cbar();
      return bad_s == 0;
      }
    };

    // ---- top-k of every token from lg[B][E]
    // B = 1, k <= 8: every warp's largest key is >= T = the smallest of the
    // warp maxima, so at least 8 keys reach T and the k-th largest key is >= T.
    // Only keys >= T are ranked: with at most 32 candidates every thread
    // compares 4 candidate pairs and adds to a shared rank counter; ties go
    // to the lower index. The routed units (ascending expert id) are built in
    // the same pass. Logits come from lg[] or straight from the workspace.
    // src: 0 = lg[] (shared), 1 = workspace floats (after the router
    // barrier), 2 = workspace {value, tag} words of layer `lay`, polled until
    // the tag matches (bounded; a timeout clears okw_s, which the caller set)
    auto route_b1_small_k = [&](int src, int lay) -> bool {
      uint32_t kq[4];
      uint32_t kmax = 0u;
      bool has = false;
      // expert i sits in warp i % 8 (lane (i / 8) % 32, slot i / 256): every
      // warp holds keys as soon as E >= 8
      auto key_idx = [&](int q) { return kConsumers * q + kWarps * lane + warp; };
      if (src == 2) {
        // tagged words polled in order (a warp's 32 words are 256 contiguous
        // bytes, two L2 lines per poll), values to lg[]
        const unsigned long long* wb = reinterpret_cast<const unsigned long long*>(p.logits);
        const uint32_t want = 0x80000000u | (ltag_s + (uint32_t)lay);
        unsigned long long t[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (kConsumers * q + tid < E) t[q] = ld_relaxed_gpu(wb + kConsumers * q + tid);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = kConsumers * q + tid;
          if (i < E) {
            if ((uint32_t)(t[q] >> 32) != want) {
              const long long t0 = clock64();
              do {
                t[q] = ld_relaxed_gpu(wb + i);
              } while ((uint32_t)(t[q] >> 32) != want && clock64() - t0 < budget);
              if ((uint32_t)(t[q] >> 32) != want) okw_s = 0;
            }
            lg[i] = __uint_as_float((uint32_t)t[q]);
          }
        }
        cbar();
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int idx = key_idx(q);
        kq[q] = 0u;
        if (idx < E) {
          const float v = src == 1 ? __ldcg(p.logits + idx) : lg[idx];
          kq[q] = float_key(v);
          kmax = max(kmax, kq[q]);
          has = true;
        }
      }
      const uint32_t wm = __reduce_max_sync(0xffffffffu, kmax);
      const bool whas = __any_sync(0xffffffffu, has);
      if (lane == 0) { sel_pos[0][warp] = whas ? 1 : 0; cand_key[warp] = wm; }
      if (warp == 0) sel_pos[1][lane] = 0;  // rank counters
      cbar();
      if (!okw_s) return false;
      uint32_t T = 0xffffffffu;
      int nw = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w)
        if (sel_pos[0][w]) { T = min(T, cand_key[w]); ++nw; }
      if (nw < k) T = 0u;  // too few warps hold keys: rank them all
      // candidates: count per warp, then place
      int mine = 0;
      uint32_t ball[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int idx = key_idx(q);
        ball[q] = __ballot_sync(0xffffffffu, idx < E && kq[q] >= T);
        mine += __popc(ball[q]);
      }
      if (lane == 0) sel_pos[2][warp] = mine;
      cbar();
      int base = 0, C = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const int c = sel_pos[2][w];
        if (w < warp) base += c;
        C += c;
      }
      int* cidx = reinterpret_cast<int*>(lg);
      {
        int off = base;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if ((ball[q] >> lane) & 1u) {
            const int pos = off + __popc(ball[q] & ((1u << lane) - 1u));
            keys[pos] = kq[q];
            cidx[pos] = key_idx(q);
          }
          off += __popc(ball[q]);
        }
      }
      cbar();
      if (C <= 32) {
        {
          const int i = tid & 31, j0 = (tid >> 5) * 4;
          int cnt = 0;
          if (i < C) {
            const uint32_t ki = keys[i];
            const int ii = cidx[i];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const int jx = j0 + jj;
              if (jx < C) {
                const uint32_t kj = keys[jx];
                cnt += (kj > ki) || (kj == ki && cidx[jx] < ii);
              }
            }
          }
          if (cnt) atomicAdd(&sel_pos[1][i], cnt);
        }
        cbar();
        if (warp == 0) {
          if (lane < C) {
            const int r = sel_pos[1][lane];
            if (r < k) { cand_key[kWarps + r] = keys[lane]; cand_idx[r] = cidx[lane]; }
          }
          __syncwarp();
          const bool sel = lane < k;
          const uint32_t kc = sel ? cand_key[kWarps + lane] : 0u;
          const int ic = sel ? cand_idx[lane] : 0x7fffffff;
          const float e = sel ? __expf(key_float(kc) - key_float(cand_key[kWarps])) : 0.f;
          const float wl = e / warp_sum(e);
          int urank = 0;
          for (int m = 0; m < k; ++m) urank += cand_idx[m] < ic;
          if (sel) {
            rs.ids[0][lane] = ic;
            rs.w[0][lane] = wl;
            rs.unit_e[urank] = ic;
            rs.unit_mask[urank] = 1u;
            rs.unit_w[urank][0] = wl;
          }
          if (lane == 0) rs.U = k;
        }
        cbar();
        return true;
      }
      for (int c = tid; c < C; c += kConsumers) {
        const uint32_t kc = keys[c];
        const int ic = cidx[c];
        int rank = 0;
        for (int o = 0; o < C; ++o) {
          const uint32_t ko = keys[o];
          rank += (ko > kc) || (ko == kc && cidx[o] < ic);
        }
        if (rank < k) { sel_pos[2][rank] = ic; cand_key[kWarps + rank] = kc; }
      }
      cbar();
      if (warp == 0) {
        const int e = lane < k ? sel_pos[2][lane] : 0x7fffffff;
        if (lane < k) sel_l[0][lane] = key_float(cand_key[kWarps + lane]);
        __syncwarp();
        warp_weights(sel_l[0], k, rs.w[0]);
        __syncwarp();
        if (lane < k) rs.ids[0][lane] = e;
        // units: ascending expert id
        int urank = 0;
        for (int i = 0; i < k; ++i) urank += __shfl_sync(0xffffffffu, e, i) < e;
        if (lane < k) {
          rs.unit_e[urank] = e;
          rs.unit_mask[urank] = 1u;
          rs.unit_w[urank][0] = rs.w[0][lane];
        }
        if (lane == 0) rs.U = k;
      }
      cbar();
      return true;
    };

    // Batch > 1 with E <= 256: warp b ranks token b straight from the
    // workspace logits. Slot s of lane l holds expert 64 (s / 2) + 2 l + s % 2;
    // each lane sorts its 8 slots best first as key << 32 | ~expert (larger
    // logit, then lower index) and each of the k rounds takes the best head
    // over the warp (as in route_warp).
    auto route_tokens_warp = [&]() {
      if (warp < B) {
        const float* lt = p.logits + (size_t)warp * E;
        unsigned long long v[8];
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2) {
          const int e = 64 * (s2 >> 1) + 2 * lane + (s2 & 1);
          v[s2] = e < E ? (((unsigned long long)float_key(__ldcg(lt + e)) << 32) | (unsigned long long)(~(uint32_t)e))
                        : 0ull;
        }
        auto cas = [&](int i, int j2) {
          const unsigned long long a = v[i], b = v[j2];
          v[i] = a < b ? b : a;
          v[j2] = a < b ? a : b;
        };
        cas(0, 1); cas(2, 3); cas(4, 5); cas(6, 7);
        cas(0, 2); cas(1, 3); cas(4, 6); cas(5, 7);
        cas(1, 2); cas(5, 6);
        cas(0, 4); cas(1, 5); cas(2, 6); cas(3, 7);
        cas(2, 4); cas(3, 5);
        cas(1, 2); cas(3, 4); cas(5, 6);
        for (int r = 0; r < k; ++r) {
          const uint32_t hk = (uint32_t)(v[0] >> 32);
          const uint32_t M = __reduce_max_sync(0xffffffffu, hk);
          uint32_t tie = __ballot_sync(0xffffffffu, hk == M);
          if (tie & (tie - 1)) {
            const uint32_t lo = __reduce_max_sync(0xffffffffu, hk == M ? (uint32_t)v[0] : 0u);
            tie = __ballot_sync(0xffffffffu, hk == M && (uint32_t)v[0] == lo);
          }
          const bool win = lane == __ffs(tie) - 1;
          if (win) {
            rs.ids[warp][r] = (int)~(uint32_t)v[0];
            sel_l[warp][r] = key_float(M);
          }
#pragma unroll
          for (int s2 = 0; s2 < 7; ++s2) v[s2] = win ? v[s2 + 1] : v[s2];
          v[7] = win ? 0ull : v[7];
        }
        __syncwarp();
        warp_weights(sel_l[warp], k, rs.w[warp]);
      }
      cbar();
    };
    auto route = [&]() {
      if constexpr (BMAX == 1) {
        // two levels: each warp takes the best k of its 1/8 of the experts,
        // warp 0 picks the best k of those candidates
        const int per8 = (E + kWarps - 1) / kWarps;
        const int lo = min(E, warp * per8), n = min(E, lo + per8) - lo;
        const int kk = min(k, n);
        for (int i = tid; i < E; i += kConsumers) keys[i] = float_key(lg[i]);
        cbar();
        if (kk > 0) warp_select(keys + lo, n, kk, sel_pos[warp]);
        __syncwarp();
        for (int i = lane; i < k; i += 32) {
          cand_key[warp * k + i] = (i < kk) ? keys[lo + sel_pos[warp][i]] : 0u;
          cand_idx[warp * k + i] = (i < kk) ? lo + sel_pos[warp][i] : -1;
        }
        cbar();
        if (warp == 0) {
          warp_select(cand_key, kWarps * k, k, sel_pos[0]);
          __syncwarp();
          if (lane < k) {
            const int q = sel_pos[0][lane];
            rs.ids[0][lane] = cand_idx[q];
            sel_l[0][lane] = key_float(cand_key[q]);
          }
          __syncwarp();
          warp_weights(sel_l[0], k, rs.w[0]);
        }
        cbar();
      } else {
        // one warp per token
        for (int i = tid; i < B * E; i += kConsumers) keys[i] = float_key(lg[i]);
        cbar();
        if (warp < B) {
          warp_select(keys + warp * E, E, k, sel_pos[warp]);
          __syncwarp();
          if (lane < k) {
            rs.ids[warp][lane] = sel_pos[warp][lane];
            sel_l[warp][lane] = lg[warp * E + sel_pos[warp][lane]];
          }
          __syncwarp();
          warp_weights(sel_l[warp], k, rs.w[warp]);
        }
        cbar();
      }
    };

    // ---- channel-sparse selection (B = 1): kept[] ascending, rs.ncand
    // Candidate q = u * I + c (routed unit u in ascending expert order,
    // channel c). The keys are loaded into shared memory (sel_load_keys);
    // sel_kept finds the keep-th largest key T by histogram passes over the
    // keys' own range and lists the kept set (every key > T plus the first
    // keep - #{> T} keys == T in index order) ascending.
    // ---- weight-only channel screen of layer l inside the stack ([Reader]
    // "가중치만으로 만든 reader", steps 1-2, eq. 1): every CTA rotates u (fp32,
    // u_x = H_128 (s * u) per block of 128, in registers and shuffles) into
    // the subset-sum table of every 4 coordinates (in the keys buffer), then
    // scores its share of the k*I candidates (candidate q = unit * I + c):
    // warp per channel, lane l taking code words l + 32t of each row, the next
    // channel's words fetched before the current one is decoded;
    //   s_j = w_e ||d_j|| |SiLU(g_hat) v_hat|, g_hat = sum_b scale_b codes_b . u_x,b / 128
    // written to scr[e*I + c]. A grid barrier then makes every CTA's scores
    // visible to the selection. Returns false when the barrier ran out.
    auto screen_layer = [&](int l) -> bool {
      if constexpr (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR && SCREEN) {
        const LayerW& Lw = p.layer[l];
        // This CTA's candidates q in [q0, q1): their code rows, scale rows and
        // down-column norms are copied into the ring (idle between the
        // routing and the routed copies; cp.async through L2, one round trip
        // for all of them) while every thread rotates u into the subset-sum
        // table (in the keys buffer, free until the selection). Then a warp
        // per candidate, 8 table lookups per code word.
        float* lut = reinterpret_cast<float*>(keys);
        const int words = H >> 4, nb = H >> 7, cw = 2 * words;
        const int N = k * I;
        const int q0 = (int)((long long)cta * N / G), q1 = (int)((long long)(cta + 1) * N / G);
        const int n = q1 - q0;
        uint32_t* st_codes = reinterpret_cast<uint32_t*>(ring);                       // [n][2][words]
        uint16_t* st_scales = reinterpret_cast<uint16_t*>(ring + (size_t)n * cw * 4);  // [n][2][nb]
        float* st_dn = reinterpret_cast<float*>(ring + (size_t)n * (cw * 4 + nb * 4));  // [n]
        auto chan = [&](int q) {
          const int u = q / I;
          return rs.unit_e[u] * I + (q - u * I);
        };
        // warp w copies candidates w, w + 8, ...: lane l the 16-byte pieces
        // l + 32 i of the two code rows and the 4-byte pieces of the scale
        // rows, lane 0 the norm
        for (int i = warp; i < n; i += kWarps) {
          const int j = chan(q0 + i);
          for (int o = lane; o < cw / 4; o += 32)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(st_codes + (size_t)i * cw + 4 * o)),
                         "l"(Lw.sk_codes + (size_t)j * cw + 4 * o)
                         : "memory");
          for (int o = lane; o < nb; o += 32)
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(st_scales + (size_t)i * 2 * nb + 2 * o)),
                         "l"(Lw.sk_scales + (size_t)j * 2 * nb + 2 * o)
                         : "memory");
          if (lane == 0)
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(st_dn + i)), "l"(Lw.sk_dnorm + j)
                         : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        screen_build_lut(H, [&](int h) { return bf16_to_f(us[h]) * (float)p.signs[h]; }, lut);
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        cbar();
        for (int i = warp; i < n; i += kWarps) {
          const uint32_t* cr = st_codes + (size_t)i * cw;
          const uint16_t* sr = st_scales + (size_t)i * 2 * nb;
          float acc[2] = {0.f, 0.f};
#pragma unroll
          for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const int wd = lane + 32 * t;
              if (wd < words)
                acc[r] = fmaf(__half2float(__ushort_as_half(sr[r * nb + (wd >> 3)])), screen_word(lut, wd, cr[r * words + wd]),
                              acc[r]);
            }
          const float gv0 = warp_sum(acc[0]) * (1.0f / 128.0f), gv1 = warp_sum(acc[1]) * (1.0f / 128.0f);
          if (lane == 0) {
            const int q = q0 + i, u = q / I;
            p.scr[chan(q)] = rs.unit_w[u][0] * st_dn[i] * fabsf(silu_f(gv0) * gv1);
          }
        }
        return grid_sync();
      } else {
        return true;
      }
    };

    auto select_channels = [&](int l) {
      const int N = rs.U * I;
      const float* sc = SCREEN ? p.scr : p.layer[l].scores;
      int* hist = reinterpret_cast<int*>(smem + p.off_hist);
      int* ssc = hist + 2 * kSelBins;
      // 1. the candidates' keys (written in this launch when screened: read
      // through L2)
      const bool vec = (I & 3) == 0 && ((uintptr_t)sc & 15u) == 0;
      sel_load_keys(keys, N, I, vec, [&](int u) { return sc + (size_t)rs.unit_e[u] * I; }, hist, ssc);
      const int keep = p.keep;
      cbar();
      // 2. the kept list, ascending
      if (keep > 0) {
        const float invI = 1.0f / (float)I;
        sel_kept(keys, N, keep, hist, ssc, [&](int pos, int q) {
          const int u = __float2int_rz(((float)q + 0.5f) * invI);
          kept[pos] = rs.unit_e[u] * I + (q - u * I);
        });
      }
      if (tid == 0) rs.ncand = keep > 0 ? min(N, keep) : 0;
      cbar();
      // sectors (reported by CTA 0 only): each kept channel's byte range,
      // less a sector shared with the previous kept channel; channels that
      // start and end on 32-byte boundaries share none
      if (cta == 0 && p.sectors_out != nullptr) {
        const unsigned long long base = (unsigned long long)(uintptr_t)p.layer[l].gate;
        const unsigned long long cb = 3ull * rowb;
        if (((base | cb) & 31ull) == 0) {
          if (tid == 0) rs.sectors = (unsigned long long)rs.ncand * (cb >> 5);
        } else {
          uint32_t sec = 0;
          for (int i = tid; i < rs.ncand; i += kConsumers) {
            const unsigned long long s0 = (base + (unsigned long long)kept[i] * cb) >> 5;
            const unsigned long long s1 = (base + (unsigned long long)(kept[i] + 1) * cb - 1) >> 5;
            sec += (uint32_t)(s1 - s0 + 1);
            if (i > 0 && ((base + (unsigned long long)(kept[i - 1] + 1) * cb - 1) >> 5) == s0) sec -= 1;
          }
          sec = __reduce_add_sync(0xffffffffu, sec);
          if (lane == 0) rs.scan[warp] = (int)sec;
          cbar();
          if (tid == 0) {
            unsigned long long t = 0;
            for (int w = 0; w < kWarps; ++w) t += (uint32_t)rs.scan[w];
            rs.sectors = t;
          }
          cbar();
        }
      }
    };

    bool failed = false;
    Job j;
    // fast path: this group's static jobs per layer (router rows in jobs of
    // rows_per_job, shared channels in jobs of NCH; static job s belongs to
    // pipe s % kPipes)
    int own_router = 0, own_shared = 0, own_pred = 0;
    const int nj_pool = ((LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR) ? (p.keep > 0 ? min(k * I, p.keep) : 0) : k * I) / NCH + 1;
    if constexpr (kFast && MODE == MODE_LAYERS) {
      const unsigned Gu = (unsigned)G, cu = (unsigned)cta;
      const int nr = (int)((cu + 1) * (unsigned)E / Gu) - (int)(cu * (unsigned)E / Gu);
      const int ns = (int)((cu + 1) * (unsigned)p.I_sh / Gu) - (int)(cu * (unsigned)p.I_sh / Gu);
      const int nrj = (nr + p.rows_per_job - 1) / p.rows_per_job, nsj = (ns + NCH - 1) / NCH;
      const int npj = p.npred > 0 ? nrj : 0;  // prediction jobs (all layers but the last)
      for (int sx = 0; sx < nrj + nsj + npj; ++sx)
        if (sx % kPipes == my_group) {
          if (sx < nrj) ++own_router;
          else if (sx < nrj + nsj) ++own_shared;
          else ++own_pred;
        }
    }
    // this CTA's slice [ys0, ys1) of the B*H/4 float4 slots of an accumulator
    // (outputs, zeroing); B*H/4 <= 2^14, so 32-bit products suffice
    const int n4s = B * H / 4;
    const int ys0 = (int)((unsigned)cta * (unsigned)n4s / (unsigned)G);
    const int ys1 = (int)((unsigned)(cta + 1) * (unsigned)n4s / (unsigned)G);
    // layer 0's accumulator: zeroed here, ordered before any CTA adds into it
    // by the router barrier, by the ids barrier (given ids), or on the fast
    // path (no router barrier) by one grid barrier now
    {
      for (int i = ys0 + tid; i < ys1; i += kConsumers)
        reinterpret_cast<float4*>(p.yacc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      // routed-job pools of layers 0 and 1 (layer l clears the pool of l + 2)
      if (kFast && cta == 0 && tid == 0) { ctl->pool[0] = 0u; ctl->pool[1] = 0u; }
      if constexpr (kFast && MODE == MODE_LAYERS)
        if (k <= kWarps && !grid_sync()) { failed = true; if (tid == 0) set_status(ctl, kStatusTimeout); }
    }
    for (int l = 0; l < p.L && !failed; ++l) {
      // accumulators rotate over three buffers: layer l adds into l % 3 and
      // zeroes its slice of (l + 1) % 3, last read in layer l - 2's epilogue
      // (finished everywhere before the barrier that ended layer l - 1) and
      // next written after the barrier that ends layer l
      float* yacc = p.yacc + (size_t)(l % 3) * B * H;
      {
        float* ynext = p.yacc + (size_t)((l + 1) % 3) * B * H;
        for (int i = ys0 + tid; i < ys1; i += kConsumers)
          reinterpret_cast<float4*>(ynext)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        // the pool of layer l + 2: its last users (layer l - 1's producers)
        // finished before the barrier that ended layer l - 1, its next users
        // start after the barrier that ends layer l
        if (kFast && cta == 0 && tid == 0) ctl->pool[(l + 2) % 3] = 0u;
      }
      // phase 0: router rows, 1: shared expert, 2: routed experts
      int phase = (MODE == MODE_LAYERS) ? 0 : 1;
      int ready = l - 1;
      unsigned long long target = 0;
      const bool route_early = kFast && MODE == MODE_LAYERS;
      // routing of layer l: logits (after the router barrier) or the given
      // ids -> routed units (and kept channels), published to the producer
      auto do_route = [&]() -> bool {
        constexpr bool kWarpRoute = MODE == MODE_LAYERS && BMAX == 1;
        if (warp_routes) {
          // warp 0 routes; the other warps need nothing from it and go on.
          // The producers must be done with layer l - 1's units first.
          ready = l;
          if (warp != 0) return true;
          if (lane == 0 && l > 0) {
            const long long t0 = clock64();
            while (min(*(volatile int*)&prod_layer_s[0], *(volatile int*)&prod_layer_s[1]) < l - 1) {
              if (clock64() - t0 > budget) { set_status(ctl, kStatusTimeout); break; }
              __nanosleep(20);
            }
            (void)ld_acquire_cta(&prod_layer_s[0]);
            (void)ld_acquire_cta(&prod_layer_s[1]);
          }
          __syncwarp();
          if (!route_warp(l)) {
            // the others learn of it through the abort flag
            if (lane == 0) { set_status(ctl, kStatusTimeout); st_release_cta(&abort_s, 1); }
            return false;
          }
          if (lane == 0) st_release_cta(&route_ready_s, l);
          return true;
        }
        bool units_done = false;
        // the producer must be done with the previous layer's routing
        // before it is overwritten (it always is, unless this CTA had no
        // work at all in some layers)
        if (tid == 0 && l > 0) {
          const long long t0 = clock64();
          while (min(*(volatile int*)&prod_layer_s[0], *(volatile int*)&prod_layer_s[1]) < l - 1) {
            if (clock64() - t0 > budget) { set_status(ctl, kStatusTimeout); break; }
            __nanosleep(20);
          }
          (void)ld_acquire_cta(&prod_layer_s[0]);
          (void)ld_acquire_cta(&prod_layer_s[1]);
        }
        if constexpr (MODE == MODE_LAYERS) {
          // (planar batch-1 stacks with k <= 8, E <= 256 are routed by
          // warp 0 above and never get here)
          if (kFast && k <= kWarps && E <= 256) {
            // channel-major: warp 0 routes from the tagged words, the others
            // wait; every warp learns the outcome from one barrier reduction
            const int bad = (warp == 0) ? (route_warp(l) ? 0 : 1) : 0;
            if (cbar_or(bad)) { if (tid == 0) set_status(ctl, kStatusTimeout); return false; }
            units_done = true;
          } else if (kFast && k <= kWarps) {
            // logits straight from their tagged words (okw_s = 1 was set
            // before the phase barrier)
            if (!route_b1_small_k(2, l)) { if (tid == 0) set_status(ctl, kStatusTimeout); return false; }
            units_done = true;
          } else if (kWarpRoute && k <= kWarps) {
            if (tid == 0) okw_s = wait_grid(target) ? 1 : 0;
            cbar();
            if (!okw_s) { if (tid == 0) set_status(ctl, kStatusTimeout); return false; }
            route_b1_small_k(1, l);
            units_done = true;
          } else {
            if (tid == 0) okw_s = wait_grid(target) ? 1 : 0;
            cbar();
            if (!okw_s) { if (tid == 0) set_status(ctl, kStatusTimeout); return false; }
            if (BMAX > 1 && E <= 256 && k <= 32) {
              route_tokens_warp();
            } else {
              for (int i = tid; i < B * E; i += kConsumers) lg[i] = __ldcg(p.logits + i);
              cbar();
              if (BMAX == 1 && k <= kWarps) { route_b1_small_k(0, l); units_done = true; }
              else route();
            }
          }
          if (cta == 0 && p.ids_out != nullptr)
            for (int t = tid; t < B * k; t += kConsumers) {
              p.ids_out[(size_t)l * B * k + t] = rs.ids[t / k][t % k];
              p.w_out[(size_t)l * B * k + t] = rs.w[t / k][t % k];
            }
        } else {
          for (int t = tid; t < B * k; t += kConsumers) {
            rs.ids[t / k][t % k] = p.ids_in[t];
            rs.w[t / k][t % k] = p.w_in[t];
          }
          if (!grid_sync()) { if (tid == 0) set_status(ctl, kStatusTimeout); return false; }
        }
        if (!units_done && !build_units() && cta == 0 && tid == 0) set_status(ctl, kStatusBadIds);
        if constexpr (LAYOUT == MOE_LAYOUT_CHANNEL_MAJOR) {
          if (SCREEN && !screen_layer(l)) { if (tid == 0) set_status(ctl, kStatusTimeout); return false; }
          select_channels(l);
          if (cta == 0) {
            if (p.kept_out != nullptr)
              for (int i = tid; i < rs.ncand; i += kConsumers) p.kept_out[(size_t)l * p.keep + i] = kept[i];
            if (tid == 0 && p.sectors_out != nullptr) p.sectors_out[l] = rs.sectors;
          }
        }
        if (tid == 0) st_release_cta(&route_ready_s, l);
        ready = l;
        return true;
      };
      if constexpr (kFast) {
        // pipeline g: this group's router jobs, routing (whole CTA), its
        // shared jobs, then routed jobs until the end marker
        bool fl = false;
        for (int i = 0; i < own_router; ++i) fl = fl || consume_pipe() != JOB_ROUTER;
        if (tid == 0) okw_s = 1;
        if (cbar_or(fl)) { failed = true; break; }
        if (!(MODE == MODE_LAYERS && k <= kWarps) && MODE == MODE_LAYERS && tid == 0) target = arrive_grid();
        // planar: a failed routing (warp 0 alone) skips this warp's jobs and
        // every warp meets the others at the barrier after the routed phase;
        // channel-major: all threads agree on it
        if constexpr (LAYOUT == MOE_LAYOUT_PLANAR) {
          fl = !do_route();
        } else {
          if (!do_route()) { failed = true; break; }
        }
        // the output accumulators start from zero here: not live before
#pragma unroll
        for (int i = 0; i < (kFast ? 64 : 1); ++i) accf[i] = 0.f;
        for (int i = 0; i < own_shared && !fl; ++i) fl = consume_pipe() != JOB_SHARED;
        if (l + 1 < p.L)
          for (int i = 0; i < own_pred && !fl; ++i) fl = consume_pipe() != JOB_ROUTER;
        if (warp_routes && !fl) {
          // the routed copies may start before the routing is complete (its
          // units are published one by one); their weights come last
          int ok = 1;
          if (lane == 0) {
            const long long tw = clock64();
            while (*(volatile int*)&route_ready_s < l)
              if (*(volatile int*)&abort_s || clock64() - tw > budget) {
                ok = 0;
                break;
              }
            (void)ld_acquire_cta(&route_ready_s);
          }
          __syncwarp();
          fl = !__shfl_sync(0xffffffffu, ok, 0);
          if (fl && lane == 0 && !*(volatile int*)&abort_s) set_status(ctl, kStatusTimeout);
        }
        for (int it = 0; !fl; ++it) {
          const int ty = consume_pipe();
          if (ty == JOB_END) break;
          fl = ty != JOB_ROUTED || it > nj_pool + 8;  // a pipe gets at most all jobs
        }
        failed = fl;
      } else {
      // (int4 batch path: once next_job has set this layer's routed range, the
      // rest of its jobs come straight from the cursor, in next_job's order)
      int ft = 0, ft1 = 0, fc = 0, fu = 0;
      for (;;) {
        bool take;
        JobCursor save;
        if (kTcB && ft < ft1) {
          const int n = min(min(NCH - (fc & (NCH - 1)), I - fc), ft1 - ft);
          j = Job{JOB_ROUTED, l, fu, fc, n};
          ft += n;
          fc += n;
          if (fc >= I) { fc -= I; ++fu; }
          take = true;
        } else {
          save = ccur;
          const bool got = next_job(ccur, j, ready);
          take = got && j.type != JOB_END && j.layer == l && j.type == phase;
          if (kTcB && take && j.type == JOB_ROUTED) {
            ft = ccur.t; ft1 = ccur.t1; fc = ccur.c; fu = ccur.u;
            ccur.t = ccur.t1;  // the cursor moves on to the end of the layer
          }
        }
        if (take) {
          if (!consume(j)) { failed = true; break; }
          continue;
        }
        ccur = save;
        if (phase == 0) {
          // router logits written: arrive at the grid barrier; on the fast
          // path route at once (the shared expert's compute then overlaps the
          // routed copies' latency), else do the shared expert first
          if (tid == 0) okw_s = 1;
          cbar();
          if (!(kFast && MODE == MODE_LAYERS && k <= kWarps) && tid == 0) target = arrive_grid();
          if (route_early && !do_route()) { failed = true; break; }
          phase = 1;
          continue;
        }
        if (phase == 1) {
          if (!(route_early || do_route())) { failed = true; break; }
          phase = 2;
          continue;
        }

        break;
      }
      }
      if (cbar_or(failed)) { failed = true; break; }
      ccur.begin_layer(p, l + 1);
      // partial sums -> L2 accumulator
      if constexpr (kFast) {
        // warps -> shared sum in 8 steps: at step s warp w adds its chunk
        // (w + s) % 8 (elements 256 c + 8 lane + e, stored at 256 c + 32 e +
        // lane), so no two warps touch a chunk at once; then thread t adds
        // elements 8t..8t+7 to the L2 accumulator
        float* ysum = reinterpret_cast<float*>(smem + p.off_ysum);
        ysum_all(accf, ysum, lane, warp);
        float v[8];
        {
          const float* yt = ysum + 256 * (tid >> 5) + (tid & 31);
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = yt[32 * e];
        }
        float* dst = yacc + 8 * tid;
        red_add_v4(dst, v[0], v[1], v[2], v[3]);
        red_add_v4(dst + 4, v[4], v[5], v[6], v[7]);
      } else if constexpr (kTcB) {
        float4* ysb = reinterpret_cast<float4*>(smem + p.off_ysum);
        for (int b = 0; b < B; ++b) {
          float4* ya = ysb + b * (H >> 2) + tid;
          const float4 y0 = ya[0], y1 = ya[H >> 3];
          float* dst = yacc + (size_t)b * H + 8 * tid;
          red_add_v4(dst, y0.x, y0.y, y0.z, y0.w);
          red_add_v4(dst + 4, y1.x, y1.y, y1.z, y1.w);
          ya[0] = make_float4(0.f, 0.f, 0.f, 0.f);
          ya[H >> 3] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      } else if (has_v) {
#pragma unroll
        for (int b = 0; b < BMAX; ++b)
          if (b < B) {
            float* dst = yacc + (size_t)b * H + 8 * tid;
            red_add_v4(dst, acc[b][0].x, acc[b][0].y, acc[b][1].x, acc[b][1].y);
            red_add_v4(dst + 4, acc[b][2].x, acc[b][2].y, acc[b][3].x, acc[b][3].y);
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[b][i] = make_float2(0.f, 0.f);
          }
      }
      if (!grid_sync()) { failed = true; if (tid == 0) set_status(ctl, kStatusTimeout); break; }
      if (kFast && p.npred > 0 && tid == 0) *(volatile int*)&bar_l_s = l;  // (for the expert prefetch)
      // epilogue: y, residual, outputs (each CTA writes its slice)
      const long long n4 = n4s;
      const long long s0 = ys0, s1 = ys1;
      float* yh = p.y_hist ? p.y_hist + (size_t)l * B * H : nullptr;
      float* yo = (l == p.L - 1) ? p.y_out : nullptr;
      if constexpr (MODE == MODE_LAYERS && kFast) {
        // thread t: elements 8t..8t+7 (float4 slots 2t, 2t+1)
        const float4 ya = __ldcg(reinterpret_cast<const float4*>(yacc) + 2 * tid);
        const float4 yb = __ldcg(reinterpret_cast<const float4*>(yacc) + 2 * tid + 1);
        float xv[8];
        unpack8(xs4[tid], xv);
        const float yv[8] = {ya.x, ya.y, ya.z, ya.w, yb.x, yb.y, yb.z, yb.w};
        uint4 xn;
        uint32_t* xnw = reinterpret_cast<uint32_t*>(&xn);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint16_t lo = f_to_bf16(xv[2 * m] + yv[2 * m]), hi = f_to_bf16(xv[2 * m + 1] + yv[2 * m + 1]);
          xnw[m] = uint32_t(lo) | (uint32_t(hi) << 16);
          xv[2 * m] = bf16_to_f(lo);
          xv[2 * m + 1] = bf16_to_f(hi);
        }
        reinterpret_cast<uint4*>(xs)[tid] = xn;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const long long i = 2 * tid + h;
          if (i >= s0 && i < s1) {
            const float4 y4 = h ? yb : ya;
            const uint2 x2 = make_uint2(xnw[2 * h], xnw[2 * h + 1]);
            if (yh) reinterpret_cast<float4*>(yh)[i] = y4;
            if (yo) reinterpret_cast<float4*>(yo)[i] = y4;
            if (p.x_hist) reinterpret_cast<uint2*>(p.x_hist + (size_t)(l + 1) * B * H)[i] = x2;
            if (l == p.L - 1 && p.x_out) reinterpret_cast<uint2*>(p.x_out)[i] = x2;
          }
        }
        fast_frags(xv, p.pre_norm != 0);
      } else if constexpr (MODE == MODE_LAYERS) {
        // accumulator loads in flight per thread, then their updates (8 on
        // the int4 batch path, whose sums left the registers free)
        constexpr int kEpU = kTcB ? 8 : 1;
        for (long long i0 = tid; i0 < n4; i0 += kEpU * kConsumers) {
          float4 yv4[kEpU];
#pragma unroll
          for (int u = 0; u < kEpU; ++u) {
            const long long i = i0 + (long long)u * kConsumers;
            if (i < n4) yv4[u] = __ldcg(reinterpret_cast<const float4*>(yacc) + i);
          }
#pragma unroll
          for (int u = 0; u < kEpU; ++u) {
          const long long i = i0 + (long long)u * kConsumers;
          if (i >= n4) break;
          const float4 y4 = yv4[u];
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
        }
        cbar();
        if constexpr (kTcB) build_xfrags(p.pre_norm != 0);
        else if (p.pre_norm) normalize_x();
        load_xfrag();
      } else {
        for (long long i = s0 + tid; i < s1; i += kConsumers) {
          const float4 y4 = __ldcg(reinterpret_cast<const float4*>(yacc) + i);
          if (yo) reinterpret_cast<float4*>(yo)[i] = y4;
          if (yh) reinterpret_cast<float4*>(yh)[i] = y4;
        }
      }
    }
    if (failed && tid == 0) {
      // every failure is a wait that ran out (bad ids do not stop the
      // kernel); the first status recorded stays
      set_status(ctl, kStatusTimeout);
      jc_s = jc;
      st_release_cta(&abort_s, 1);
    }
  }
  __syncthreads();
  // on an error path, wait (bounded) for the copies still in flight so that
  // none lands in shared memory after the CTA has exited
  if (tid == 0 && abort_s) {
    if constexpr (kFast) {
      // pipeline g: jobs [consumed, issued) of its stages
      for (int g = 0; g < kPipes; ++g) {
        const int n = (p.nstages - g + kPipes - 1) / kPipes;
        for (long long q = jcg_s[g]; q < jp_s[g]; ++q)
          mbar_wait(&full[g + kPipes * (int)(q % n)], (uint32_t)((q / n) & 1), budget);
      }
    } else {
      // job q was issued iff producer q % kProducers got past it
      const long long issued = max(jp_s[0], jp_s[1]);
      for (long long q = jc_s; q < issued; ++q)
        if (q < jp_s[q % kProducers]) mbar_wait(&full[q % p.nstages], (uint32_t)((q / p.nstages) & 1), budget);
    }
  }
}

}  // namespace moedec
