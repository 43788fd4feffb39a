// Experts that are a single matrix (E_e(x) = W_e x, W_e [H, H] bf16) at batch B:
// the batch-sweep workload ("5,010억 개 중 230억 개만 켠다 — 4.6% 의 산수",
// §3 [A] and [B]: each expert one 8192 x 8192 bf16 matrix, k of E experts per
// token, touched experts grow with B as E[1 - (1 - k/E)^B]).
//
//   y[b] = sum_s w[b, s] * W_{ids[b, s]} x[b]
//
// Each touched expert's weights are read from HBM once per step, for all the
// tokens routed to it (a stable counting sort groups the (token, slot) pairs
// by expert). Two engines, chosen per expert by its token count n_e:
//  * n_e < kTcMin: a streaming GEMV (128-bit loads, fp32 FMA), rows handed out
//    in chunks through a global counter;
//  * n_e >= kTcMin: a dense contraction on the 5th-generation tensor cores.
//    The expert's tokens are packed into rows of a bf16 buffer, then a
//    warp-specialised kernel streams [128 x 64] weight tiles and [N x 64] token
//    tiles with 2-D TMA (128-byte swizzle) into a stage ring; one thread issues
//    tcgen05.mma (bf16 in, fp32 accumulate in TMEM, M = 128, N = n_e rounded up
//    to 32); a warpgroup reads the accumulator with tcgen05.ld and adds the
//    router-weighted columns into y.
// Both engines are bound by HBM (a [128 x 64] tile carries 16 KB for at most
// 128 x 64 x 256 MACs); the tensor cores take the arithmetic once n_e grows
// beyond what the FP32 pipes can sustain at full bandwidth.
#pragma once

#include <cuda.h>

#include "decode_kernel.cuh"

namespace moedec {

constexpr int kTcMin = 4;        // tokens per expert from which the tensor-core engine runs
constexpr int kTcBlockM = 128;   // weight rows per tile (M)
constexpr int kTcBlockK = 64;    // K per stage (128 bytes of bf16: one swizzle row)
constexpr int kTcStages = 4;
constexpr int kTcMaxN = 256;     // N per unit (tokens, padded to 32)
constexpr int kTcRowsPerLoad = 32;
constexpr int kGemvRows = 16;    // rows per GEMV chunk

// Plan written by linear_plan_kernel into the workspace.
struct LinPlan {
  int ntouched, ngemv, ntc, bad;
  int xp_rows;     // packed token rows for the tensor-core units
  int ks;          // K splits of a tensor-core unit
  int gemv_next;   // GEMV chunk counter (grabbed with atomicAdd)
  int pad[9];
  int uexp[kMaxE];     // expert of touched unit u (ascending)
  int ucnt[kMaxE];     // tokens of unit u
  int uoff[kMaxE + 1]; // offset of unit u in pairs
  int uxrow[kMaxE];    // first packed row of unit u (tensor-core units)
  int upad[kMaxE];     // packed rows of unit u (n_u rounded up to 32)
  int gemv_u[kMaxE];   // GEMV units
  int tc_u[kMaxE];     // tensor-core units
  int pairs[kMaxB * 32 * kMaxK];  // b*k + s, grouped by unit, ascending (B <= 256)
};

struct LinParams {
  int B, H, E, k;
  const uint16_t* x;   // [B, H]
  const uint16_t* W;   // [E, H, H]
  const int32_t* ids;  // [B, k]
  const float* w;      // [B, k]
  float* y;            // [B, H] (zeroed before the engines run)
  LinPlan* plan;
  uint16_t* xp;        // [xp_rows_max, H] packed token rows
  int xp_rows_max;
  int num_sms;
  WsControl* ctl;
};

// ---------------------------------------------------------------- plan (1 CTA)
__global__ void __launch_bounds__(kThreads) linear_plan_kernel(const __grid_constant__ LinParams p) {
  __shared__ int cnt[kMaxE];
  __shared__ int cursor[kMaxE];
  __shared__ int scratch[kWarps + 1];
  __shared__ int bad;
  LinPlan* pl = p.plan;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = p.E, k = p.k, P = p.B * p.k;
  for (int e = tid; e < E; e += kThreads) cnt[e] = 0;
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int q = tid; q < P; q += kThreads) {
    const int e = p.ids[q];
    if (e < 0 || e >= E) { bad = 1; continue; }
    bool dup = false;
    for (int s = 0; s < k; ++s) {
      const int o = (q / k) * k + s;
      if (o != q && p.ids[o] == e) dup = true;
    }
    if (dup) { bad = 1; continue; }  // repeated expert in a token: not routed
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  // prefix over experts: pair offsets, touched ranks, tensor-core rows
  const int per = (E + kThreads - 1) / kThreads;
  const int lo = min(E, tid * per), hi = min(E, lo + per);
  int loc = 0, tl = 0, tcl = 0, rows = 0;
  for (int e = lo; e < hi; ++e) {
    loc += cnt[e];
    tl += cnt[e] > 0;
    if (cnt[e] >= kTcMin) { ++tcl; rows += (cnt[e] + kTcRowsPerLoad - 1) / kTcRowsPerLoad * kTcRowsPerLoad; }
  }
  int tot, ttot, tctot, rtot;
  int base = block_excl_scan(loc, scratch, &tot);
  int tbase = block_excl_scan(tl, scratch, &ttot);
  int tcbase = block_excl_scan(tcl, scratch, &tctot);
  int rbase = block_excl_scan(rows, scratch, &rtot);
  int gbase = tbase - tcbase;  // gemv units before this thread's experts
  for (int e = lo; e < hi; ++e) {
    cursor[e] = base;
    if (cnt[e] > 0) {
      const int u = tbase++;
      pl->uexp[u] = e;
      pl->ucnt[u] = cnt[e];
      pl->uoff[u] = base;
      if (cnt[e] >= kTcMin) {
        const int pad = (cnt[e] + kTcRowsPerLoad - 1) / kTcRowsPerLoad * kTcRowsPerLoad;
        pl->uxrow[u] = rbase;
        pl->upad[u] = pad;
        rbase += pad;
        pl->tc_u[tcbase++] = u;
      } else {
        pl->uxrow[u] = -1;
        pl->upad[u] = 0;
        pl->gemv_u[gbase++] = u;
      }
    }
    base += cnt[e];
  }
  __syncthreads();
  // stable placement of the pairs, warp by warp
  for (int c0 = 0; c0 < P; c0 += kThreads) {
    const int q = c0 + tid;
    int e = q < P ? p.ids[q] : -1;
    if (e >= 0 && (e >= E)) e = -1;
    if (e >= 0) {
      for (int s = 0; s < k; ++s) {
        const int o = (q / k) * k + s;
        if (o != q && p.ids[o] == e) e = -1;
      }
    }
    const uint32_t same = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(same & ((1u << lane) - 1u));
    for (int w = 0; w < kWarps; ++w) {
      if (warp == w && e >= 0) {
        pl->pairs[cursor[e] + rank] = q;
        __syncwarp(same);
        if (rank == 0) cursor[e] += __popc(same);
      }
      __syncthreads();
    }
  }
  if (tid == 0) {
    pl->ntouched = ttot;
    pl->ntc = tctot;
    pl->ngemv = ttot - tctot;
    pl->bad = bad;
    pl->xp_rows = rtot;
    pl->uoff[ttot] = tot;
    // split K so that there are at least ~4 tensor-core units per SM
    const int mt = p.H / kTcBlockM;
    int ks = 1;
    while (ks < 8 && tctot > 0 && tctot * mt * ks < 4 * p.num_sms && (p.H / (2 * ks)) % kTcBlockK == 0) ks *= 2;
    pl->ks = ks;
    pl->gemv_next = 0;
    if (bad) set_status(p.ctl, kStatusBadIds);
  }
}

// ---------------------------------------------------------------- gather
// xp row r of tensor-core unit u: x[b] of its n-th pair (b = pair / k), or
// zeros past n_u. Grid-stride over packed rows, 16 bytes per thread.
__global__ void __launch_bounds__(kThreads) linear_gather_kernel(const __grid_constant__ LinParams p) {
  const LinPlan* pl = p.plan;
  const int ntc = pl->ntc, rows = pl->xp_rows, H8 = p.H >> 3;
  for (int r = blockIdx.x; r < rows; r += gridDim.x) {
    // unit of row r: the last tensor-core unit whose first row is <= r
    int lo = 0, hi = ntc - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pl->uxrow[pl->tc_u[mid]] <= r) lo = mid; else hi = mid - 1;
    }
    const int u = pl->tc_u[lo];
    const int n = r - pl->uxrow[u];
    uint4* dst = reinterpret_cast<uint4*>(p.xp + (size_t)r * p.H);
    if (n < pl->ucnt[u]) {
      const int b = pl->pairs[pl->uoff[u] + n] / p.k;
      const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)b * p.H);
      for (int v = threadIdx.x; v < H8; v += kThreads) dst[v] = src[v];
    } else {
      for (int v = threadIdx.x; v < H8; v += kThreads) dst[v] = make_uint4(0, 0, 0, 0);
    }
  }
}

// ---------------------------------------------------------------- GEMV engine
// Chunks of kGemvRows rows of one small-group unit; each warp streams whole
// rows (16-byte loads, 8 in flight per lane) against the unit's n_u < kTcMin
// token vectors held in shared memory, and adds w * dot into y.
__global__ void __launch_bounds__(kThreads, 2) linear_gemv_kernel(const __grid_constant__ LinParams p) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint4* xs = reinterpret_cast<uint4*>(sm);  // [kTcMin - 1][H8]
  __shared__ int chunk_s;
  LinPlan* pl = p.plan;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H, H8 = H >> 3;
  const int cpu = H / kGemvRows;  // chunks per unit
  const int total = pl->ngemv * cpu;
  int cur_unit = -1;
  if (tid == 0) chunk_s = atomicAdd(&pl->gemv_next, 1);
  __syncthreads();
  int c = chunk_s;
  while (c < total) {
    __syncthreads();
    if (tid == 0) chunk_s = atomicAdd(&pl->gemv_next, 1);  // next chunk, fetched early
    const int u = pl->gemv_u[c / cpu];
    const int row0 = (c % cpu) * kGemvRows;
    const int n_u = pl->ucnt[u];
    if (u != cur_unit) {
      for (int t = 0; t < n_u; ++t) {
        const int b = pl->pairs[pl->uoff[u] + t] / p.k;
        const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)b * H);
        for (int v = tid; v < H8; v += kThreads) xs[t * H8 + v] = src[v];
      }
      cur_unit = u;
    }
    __syncthreads();
    const int e = pl->uexp[u];
    for (int rr = warp; rr < kGemvRows; rr += kWarps) {
      const int row = row0 + rr;
      const uint4* wr = reinterpret_cast<const uint4*>(p.W + ((size_t)e * H + row) * H);
      float acc[kTcMin - 1];
#pragma unroll
      for (int t = 0; t < kTcMin - 1; ++t) acc[t] = 0.f;
      for (int v0 = 0; v0 < H8; v0 += 32 * 8) {
        uint4 wv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int v = v0 + i * 32 + lane;
          wv[i] = v < H8 ? __ldcs(wr + v) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int v = v0 + i * 32 + lane;
          if (v < H8) {
            float wf[8];
            unpack8(wv[i], wf);
#pragma unroll
            for (int t = 0; t < kTcMin - 1; ++t)
              if (t < n_u) {
                float xf[8];
                unpack8(xs[t * H8 + v], xf);
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[t] = fmaf(wf[q], xf[q], acc[t]);
              }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kTcMin - 1; ++t)
        if (t < n_u) {
          const float s = warp_sum(acc[t]);
          if (lane == 0) {
            const int pr = pl->pairs[pl->uoff[u] + t];
            atomicAdd(p.y + (size_t)(pr / p.k) * H + row, p.w[pr] * s);
          }
        }
    }
    c = chunk_s;
  }
}

// ---------------------------------------------------------------- tensor-core engine

// Shared-memory matrix descriptor (tcgen05): K-major operand stored as rows of
// 128 bytes with the 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
         (2ull << 61);
}
// Instruction descriptor, kind::f16: bf16 A and B (K-major), fp32 D, M x N.
__device__ __forceinline__ uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t dtmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile("{ .reg .pred q; setp.ne.b32 q, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, q; }" ::"r"(
                   dtmem),
               "l"(a), "l"(b), "r"(idesc), "r"(acc)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

struct __align__(64) LinTcParams {
  CUtensorMap tmap_w;  // W as [E*H rows][H]: box 64 x 128, 128-byte swizzle
  CUtensorMap tmap_x;  // xp as [rows][H]: box 64 x 32, 128-byte swizzle
  LinParams lp;
};

constexpr int kTcAStage = kTcBlockM * kTcBlockK * 2;  // 16 KB
constexpr int kTcBStage = kTcMaxN * kTcBlockK * 2;    // 32 KB
constexpr int kTcStageBytes = kTcAStage + kTcBStage;
constexpr int kTcSmem = kTcStages * kTcStageBytes + 1024;
constexpr uint32_t kTmemCols = 2 * kTcMaxN;  // two accumulators of 256 fp32 columns

// Warp roles: 0 = TMA producer, 1 = MMA issuer (and TMEM owner), 4..7 =
// epilogue warpgroup (warp w reads TMEM lanes 32*(w%4) .. +31). Units are
// (tensor-core expert, 128-row tile, K split), handed out round-robin.
__global__ void __launch_bounds__(kThreads, 1) linear_tc_kernel(const __grid_constant__ LinTcParams tp) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full[kTcStages], empty[kTcStages], tfull[2], tempty[2], done_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ long long issued_s;  // loads the producer issued
  __shared__ long long budget_s;  // cycles per bounded wait (the workspace's budget)
  const LinParams& p = tp.lp;
  const LinPlan* pl = p.plan;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H;
  const int mt = H / kTcBlockM;
  const int ks = pl->ks;
  const int per_unit = mt * ks;
  const int total = pl->ntc * per_unit;
  const int nk = (H / ks) / kTcBlockK;  // K stages per unit

  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], 4); }
    mbar_init(&done_bar, 1);
    fence_mbar_init();
    abort_s = 0;
    issued_s = 0;
    budget_s = ctl_wait_budget(p.ctl);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const long long budget = budget_s;

  auto unit_info = [&](int unit, int& e, int& xrow, int& npad, int& n_u, int& uoff, int& m0, int& k0) {
    const int i = unit / per_unit, rem = unit - i * per_unit;
    const int u = pl->tc_u[i];
    e = pl->uexp[u];
    xrow = pl->uxrow[u];
    npad = pl->upad[u];
    n_u = pl->ucnt[u];
    uoff = pl->uoff[u];
    m0 = (rem / ks) * kTcBlockM;
    k0 = (rem % ks) * (H / ks);
  };
  auto bounded_wait = [&](uint64_t* bar, uint32_t par) -> bool {
    const long long t0 = clock64();
    while (!mbar_try_wait_sleep(bar, par, 20000)) {
      if (*(volatile int*)&abort_s || clock64() - t0 > budget) {
        *(volatile int*)&abort_s = 1;
        return false;
      }
    }
    return true;
  };

  if (warp == 0) {
    // ---------------- producer
    if (lane == 0) {
      int slot = 0;
      uint32_t ph = 0;
      long long issued = 0;
      for (int unit = blockIdx.x; unit < total && !*(volatile int*)&abort_s; unit += gridDim.x) {
        int e, xrow, npad, n_u, uoff, m0, k0;
        unit_info(unit, e, xrow, npad, n_u, uoff, m0, k0);
        for (int kb = 0; kb < nk; ++kb) {
          if (issued >= kTcStages && !bounded_wait(&empty[slot], ph ^ 1u)) break;
          uint8_t* a = sm + slot * kTcStageBytes;
          uint8_t* bsm = a + kTcAStage;
          mbar_expect_tx(&full[slot], kTcAStage + npad * kTcBlockK * 2);
          const int kx = k0 + kb * kTcBlockK;
          tma_load_2d(a, &tp.tmap_w, kx, e * H + m0, &full[slot]);
          for (int c = 0; c < npad; c += kTcRowsPerLoad)
            tma_load_2d(bsm + c * kTcBlockK * 2, &tp.tmap_x, kx, xrow + c, &full[slot]);
          ++issued;
          if (++slot == kTcStages) { slot = 0; ph ^= 1u; }
        }
      }
      issued_s = issued;
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int slot = 0, buf = 0, ucount = 0;
      uint32_t ph = 0, tph = 0;
      for (int unit = blockIdx.x; unit < total && !*(volatile int*)&abort_s; unit += gridDim.x) {
        int e, xrow, npad, n_u, uoff, m0, k0;
        unit_info(unit, e, xrow, npad, n_u, uoff, m0, k0);
        if (ucount >= 2 && !bounded_wait(&tempty[buf], tph ^ 1u)) break;
        const uint32_t dt = tmem + (uint32_t)(buf * kTcMaxN);
        const uint32_t idesc = idesc_bf16(kTcBlockM, npad);
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!bounded_wait(&full[slot], ph)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a = smem_u32(sm + slot * kTcStageBytes);
          const uint64_t ad = sw128_desc(a), bd = sw128_desc(a + kTcAStage);
#pragma unroll
          for (int j = 0; j < kTcBlockK / 16; ++j)
            tc_mma(dt, ad + (uint64_t)(2 * j), bd + (uint64_t)(2 * j), idesc, (kb > 0 || j > 0) ? 1u : 0u);
          tc_commit(&empty[slot]);  // the stage is free once these MMAs have read it
          if (++slot == kTcStages) { slot = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&tfull[buf]);  // accumulator complete
        ++ucount;
        if (++buf == 2) { buf = 0; tph ^= 1u; }
      }
      // all issued MMAs done before the teardown (waited for even after an
      // abort: the accumulator is deallocated below)
      tc_commit(&done_bar);
      if (!mbar_wait(&done_bar, 0, budget)) *(volatile int*)&abort_s = 1;
    }
  } else if (warp >= 4) {
    // ---------------- epilogue warpgroup
    const int q = warp & 3;
    int buf = 0;
    uint32_t tph = 0;
    for (int unit = blockIdx.x; unit < total; unit += gridDim.x) {
      int e, xrow, npad, n_u, uoff, m0, k0;
      unit_info(unit, e, xrow, npad, n_u, uoff, m0, k0);
      if (!bounded_wait(&tfull[buf], tph)) break;
      tc_fence_after();
      const int row = m0 + 32 * q + lane;
      for (int c0 = 0; c0 < n_u; c0 += 16) {
        float v[16];
        tc_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * kTcMaxN + c0), v);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = c0 + j;
          if (n < n_u) {
            const int pr = pl->pairs[uoff + n];
            atomicAdd(p.y + (size_t)(pr / p.k) * H + row, p.w[pr] * v[j]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      if (++buf == 2) { buf = 0; tph ^= 1u; }
    }
  }
  tc_fence_before();
  __syncthreads();
  // after an abort, loads may still be landing in stages that no MMA read:
  // the producer waits (bounded) for the last kTcStages it issued, the only
  // ones whose phase can still be open, before the shared memory is released
  if (tid == 0 && abort_s) {
    const long long n = issued_s < kTcStages ? issued_s : kTcStages;
    for (long long q = issued_s - n; q < issued_s; ++q)
      (void)mbar_wait(&full[q % kTcStages], (uint32_t)((q / kTcStages) & 1), budget);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
  if (tid == 0 && abort_s) set_status(p.ctl, kStatusTimeout);
}

}  // namespace moedec
