// Persistent log-domain Sinkhorn over the dustbin-augmented score matrix, with
// the mutual-nearest-neighbour extraction fused into its tail.
//
// The method (realcat notes "笔记：SuperGlue:Learning Feature Matching with Graph
// Neural Networks论文阅读", sections 遮挡以及可见性 and Sinkhorn Algorithm):
//   Z = [[S, z 1], [z 1^T, z]],  log mu = [norm]*M ++ [log N + norm],
//   log nu = [norm]*N ++ [log M + norm],  norm = -log(M + N),
//   u = v = 0;  T times:  u = log mu - LSE_j(Z + v);  v = log nu - LSE_i(Z + u);
//   log P = Z + u + v - norm.
// Extraction (Jazihars notes "SuperGlue_Code_Learning / SuperGlue_model_forward_learning",
// forward()): row/column argmax over the real block, mutual check, score
// exp(max), strict threshold, -1 for unmatched.
//
// Work decomposition.  A group of `cpp` co-resident CTAs (cooperative launch)
// owns one pair at a time; its CTAs split the M+1 rows into contiguous bands
// and keep as many band rows as fit in shared memory, pre-scaled by log2(e)
// and padded with -inf to LDW = 128*NQ columns, for all T iterations (the rest
// are re-read from L2).  Inside a CTA a team of SPLIT warps owns whole rows
// (8 teams): warp h of a team holds the float4 column groups q*32 + l,
// h*NQ/SPLIT <= q < (h+1)*NQ/SPLIT, of a row in lane l, and lane 0 of warp 0
// the dustbin column; a row's reductions are warp shuffles plus, with
// SPLIT > 1, one exchange of the warps' partials through shared memory under
// a named barrier of the team.  Splitting rows keeps the per-thread state
// small enough for 256*SPLIT threads, whose latency hiding the MUFU-bound row
// pass needs.  The column potentials live in shared memory (one copy per CTA).
//
// One iteration:
//   row pass (team-local): each row's LSE with the shift m_r = log mu_r - u_r
//     (the row's previous LSE; the exact max on the first iteration), one MUFU
//     ex2 per element; the same exponentials scaled by mu_r / rowsum_r are the
//     plan mass P_rj = exp(Z + u + v) that the column update needs, summed per
//     column in registers and then across the CTA's teams by a tree through
//     shared memory;
//   column pass: with cpp == 1 the CTA's column sums are final; otherwise
//     every CTA adds its whole column vector to a global accumulator with ONE
//     bulk asynchronous reduction (cp.reduce.async.bulk ... add.f32), the group
//     meets at a counter barrier, and every CTA reads the totals back;
//     v_j(new) = v_j + log nu_j - log(sum_r P_rj)   (sum_r P_rj <= 1).
// Where a sum comes out tiny (below 2^-40 for rows, 2^-50 for columns:
// precision could have been lost to underflow) that LSE is recomputed exactly
// with its true max.  Every decision that steers control flow is taken on
// values that are identical in all the threads that have to agree on it (rows:
// the team; columns: the whole group).
//
// Waits: the group barrier spins with a time limit and, on expiry, latches a
// timeout in the status word, raises an abort flag that ends every other
// wait, and the kernel returns.
#include "sg_internal.cuh"

#include <math.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>

namespace sg {
namespace {

constexpr int NTEAM = 8;                 // row teams per CTA
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRowTiny = 9.094947017729282e-13f;   // 2^-40
constexpr float kColTiny = 8.881784197001252e-16f;   // 2^-50
constexpr size_t kMaxSmem = 220 * 1024;

// float4 column groups per lane for N real columns (LDW = 128 * NQ >= N)
__host__ __device__ inline int nq_for(int N) {
  const int q = (N + 127) / 128;
  return q <= 1 ? 1 : q <= 2 ? 2 : q <= 4 ? 4 : q <= 8 ? 8 : q <= 16 ? 16 : q <= 24 ? 24 : -1;
}
// column vector: LDW real slots + the dustbin column at LDW (16-byte multiple)
__host__ __device__ inline int acc_pitch(int N) { return nq_for(N) * 128 + 4; }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_relaxed(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Monotone map float -> uint32 (larger float, larger key).
__device__ __forceinline__ unsigned f2key(float f) {
  const unsigned u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key2f(unsigned k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, o);
    x = y > x ? y : x;
  }
  return x;
}

// Counter barrier with a time limit, executed by ONE thread.  Returns true if
// it failed (its own limit ran out, or another participant gave up).
__device__ bool counter_wait(unsigned* counter, unsigned target, unsigned* abort_flag, unsigned* status,
                             unsigned long long timeout_ns) {
  __threadfence();
  atomicAdd(counter, 1u);
  if (ld_acquire(counter) >= target) return false;
  const unsigned long long t0 = globaltimer();
  for (unsigned polls = 1;; ++polls) {
    if (ld_acquire(counter) >= target) return false;
    if ((polls & 255u) == 0u) {               // rare checks keep the spin tight
      if (ld_relaxed(abort_flag)) return true;
      if (globaltimer() - t0 > timeout_ns) {
        atomicOr(status, kStatusTimeout);
        atomicExch(abort_flag, 1u);
        return true;
      }
    }
  }
}

// Barrier over the CTAs of a group.  Returns true if it failed.
__device__ bool group_barrier(unsigned* counter, unsigned target, unsigned* abort_flag,
                              unsigned* status, unsigned long long timeout_ns) {
  __shared__ int s_fail;
  __syncthreads();
  if (threadIdx.x == 0) s_fail = counter_wait(counter, target, abort_flag, status, timeout_ns) ? 1 : 0;
  __syncthreads();
  return s_fail != 0;
}

// Adds `bytes` of shared memory (16-byte multiple, 16-byte aligned both sides)
// into global memory with one bulk asynchronous reduction and waits for its
// completion.  Executed by one thread.
__device__ __forceinline__ void bulk_add_f32(float* gdst, const float* ssrc, unsigned bytes) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(ssrc));
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;"
               ::"l"(gdst), "r"(s), "r"(bytes) : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ kernel
// Named barrier of the SPLIT warps of team t (ids 1..8; 0 is __syncthreads).
template <int SPLIT>
__device__ __forceinline__ void team_sync(int t) {
  if (SPLIT > 1) asm volatile("bar.sync %0, %1;" ::"r"(1 + t), "n"(32 * SPLIT) : "memory");
}

template <int NQ, int SPLIT>
__global__ void __launch_bounds__(256 * SPLIT, 1) sinkhorn_kernel(SinkhornArgs a) {
  constexpr int NT = 256 * SPLIT;
  constexpr int NWARP = NT / 32;
  constexpr int NQW = NQ / SPLIT;                 // float4 groups per lane (one warp's share of a row)
  constexpr int CPW = 4 * NQW;                    // columns per lane
  static_assert(NQ % SPLIT == 0 && NWARP == NTEAM * SPLIT, "row split");
  constexpr int LDW = 128 * NQ;                   // padded row length
  constexpr int CV = LDW + 4;                     // column vector (+ dustbin at LDW)
  extern __shared__ __align__(16) unsigned char smraw[];

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int team = warp % NTEAM, part = warp / NTEAM;   // row team, share of the row
  const int cpp = a.cpp;
  const int group = blockIdx.x / cpp;
  const int rank = blockIdx.x % cpp;
  const int ngroups = gridDim.x / cpp;
  if (group >= ngroups) return;                   // CTAs beyond the last full group stay idle
  const int M = a.M, N = a.N, R = M + 1, C = N + 1;
  const int Cp = acc_pitch(N);
  const int band = (R + cpp - 1) / cpp;
  const int r0 = min(R, rank * band), r1 = min(R, r0 + band);
  const int cached = min(r1 - r0, a.cached_rows);

  // shared memory: [cache rows x LDW | v (CV) | column totals (CV) |
  //                 team partials (NTEAM/2 x CV) | u (band)]
  float* cache = reinterpret_cast<float*>(smraw);
  float* vbuf = cache + (size_t)a.cached_rows * LDW;
  float* ctot = vbuf + CV;
  unsigned* ckey = reinterpret_cast<unsigned*>(ctot);
  float* xbuf = ctot + CV;                        // NTEAM/2 partial column vectors
  float* u2s = xbuf + (size_t)(NTEAM / 2) * CV;
  // per team and row parity: the parts' partial maxima and sums of a row
  __shared__ float xr_max[2][NTEAM][SPLIT], xr_sum[2][NTEAM][SPLIT];
  // extraction only: per-column best (value, row) keys over the row cache
  unsigned long long* cbest = reinterpret_cast<unsigned long long*>(smraw);

  // log2-domain constants: log mu, log nu and the dustbin score, times log2(e)
  const float norm = -logf((float)(M + N));
  const float lmu_r2 = norm * kLog2e, lmu_b2 = (logf((float)N) + norm) * kLog2e;
  const float lnu_r2 = norm * kLog2e, lnu_b2 = (logf((float)M) + norm) * kLog2e;
  const float alpha2 = a.alpha * kLog2e;

  unsigned* counter = a.barrier + group;
  unsigned gen = 0;
  bool failed = false;
  auto barrier = [&]() -> bool {
    if (cpp == 1) {
      __syncthreads();
      return false;
    }
    ++gen;
    return group_barrier(counter, gen * cpp, a.abort_flag, a.status, a.timeout_ns);
  };

  for (int pair = group; pair < a.B && !failed; pair += ngroups) {
    const float* S = a.S + (long long)pair * a.strideS;
    float* u2 = u2s - r0;                         // row potentials of the band (log2 domain)
    float* acc = a.acc + (long long)pair * 3 * Cp;
    float* fbm = a.fb + (long long)pair * 2 * Cp;  // exact column fallback: max keys
    float* fbs = fbm + Cp;                         // exact column fallback: sums
    unsigned* fbk = reinterpret_cast<unsigned*>(fbm);

    // z2 (log2 domain) of row r, from the source matrix, for this lane's float4
    // groups g0 .. g0 + NQW - 1
    auto load_src = [&](int r, int g0, float (&z)[CPW]) {
      if (r == M) {
#pragma unroll
        for (int qq = 0; qq < NQW; ++qq)
#pragma unroll
          for (int i = 0; i < 4; ++i) z[4 * qq + i] = ((g0 + qq) * 128 + lane * 4 + i) < N ? alpha2 : -INFINITY;
        return;
      }
      const float* src = S + (long long)r * a.lds;
#pragma unroll
      for (int qq = 0; qq < NQW; ++qq) {
        const int o = (g0 + qq) * 128 + lane * 4;
        float4 t = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        if (a.lds_vec && o + 3 < N) {
          t = __ldg(reinterpret_cast<const float4*>(src + o));
          t.x *= kLog2e; t.y *= kLog2e; t.z *= kLog2e; t.w *= kLog2e;
        } else {
          if (o < N) t.x = __ldg(src + o) * kLog2e;
          if (o + 1 < N) t.y = __ldg(src + o + 1) * kLog2e;
          if (o + 2 < N) t.z = __ldg(src + o + 2) * kLog2e;
          if (o + 3 < N) t.w = __ldg(src + o + 3) * kLog2e;
        }
        z[4 * qq] = t.x; z[4 * qq + 1] = t.y; z[4 * qq + 2] = t.z; z[4 * qq + 3] = t.w;
      }
    };
    // z2 of row r: from the shared-memory cache when the row is cached
    auto load_row = [&](int r, int g0, float (&z)[CPW]) {
      if (r - r0 < cached) {
        const float4* row = reinterpret_cast<const float4*>(cache + (size_t)(r - r0) * LDW);
#pragma unroll
        for (int qq = 0; qq < NQW; ++qq) {
          const float4 t = row[(g0 + qq) * 32 + lane];
          z[4 * qq] = t.x; z[4 * qq + 1] = t.y; z[4 * qq + 2] = t.z; z[4 * qq + 3] = t.w;
        }
      } else {
        load_src(r, g0, z);
      }
    };
    // ---- stage the band in shared memory (pre-scaled, padded with -inf)
    __syncthreads();
    for (int r = r0; r < r0 + cached; ++r) {
      const float* src = S + (long long)r * a.lds;
      float* dst = cache + (size_t)(r - r0) * LDW;
      for (int j = tid; j < LDW; j += NT)
        dst[j] = j < N ? (r < M ? __ldg(src + j) : a.alpha) * kLog2e : -INFINITY;
    }
    for (int r = r0 + tid; r < r1; r += NT) u2[r] = 0.f;
    for (int j = tid; j < CV; j += NT) { vbuf[j] = 0.f; ctot[j] = 0.f; }
    __syncthreads();

    for (int it = 0; it < a.iters; ++it) {
      // ------------------------------------------------ row pass (team per row)
      float colacc[CPW];
#pragma unroll
      for (int c = 0; c < CPW; ++c) colacc[c] = 0.f;
      float colbin = 0.f;
      const float4* v4 = reinterpret_cast<const float4*>(vbuf);
      const float vb = vbuf[LDW];
      const int g0 = part * NQW;                  // this warp's first float4 group
      // this lane's column potentials, re-read from shared memory per row (held
      // in registers next to the row and its column sums they cost more in
      // lost latency hiding than the shared-memory reads)
      auto vq_at = [&](int qq) -> float4 { return v4[(g0 + qq) * 32 + lane]; };
      const bool bin_lane = part == 0 && lane == 0;
      int k = 0;                                  // rows taken by the team (slot parity)
      for (int r = r0 + team; r < r1; r += NTEAM, ++k) {
        const float lmu2 = r < M ? lmu_r2 : lmu_b2;
        float e[CPW];
        load_row(r, g0, e);
        bool exact = (it == 0);
        float m = exact ? 0.f : lmu2 - u2[r];
        float s, eb;
        while (true) {
          if (exact) {
            float mx = bin_lane ? alpha2 + vb : -INFINITY;
#pragma unroll
            for (int qq = 0; qq < NQW; ++qq) {
              const float4 vq = vq_at(qq);
              mx = fmaxf(mx, fmaxf(fmaxf(e[4 * qq] + vq.x, e[4 * qq + 1] + vq.y),
                                   fmaxf(e[4 * qq + 2] + vq.z, e[4 * qq + 3] + vq.w)));
            }
            m = warp_max(mx);
            if (SPLIT > 1) {
              if (lane == 0) xr_max[k & 1][team][part] = m;
              team_sync<SPLIT>(team);
              m = xr_max[k & 1][team][0];
#pragma unroll
              for (int h = 1; h < SPLIT; ++h) m = fmaxf(m, xr_max[k & 1][team][h]);
            }
          }
          float part_s = 0.f;
#pragma unroll
          for (int qq = 0; qq < NQW; ++qq) {
            const float4 vq = vq_at(qq);
            const float x0 = ex2((e[4 * qq] + vq.x) - m);
            const float x1 = ex2((e[4 * qq + 1] + vq.y) - m);
            const float x2 = ex2((e[4 * qq + 2] + vq.z) - m);
            const float x3 = ex2((e[4 * qq + 3] + vq.w) - m);
            e[4 * qq] = x0; e[4 * qq + 1] = x1; e[4 * qq + 2] = x2; e[4 * qq + 3] = x3;
            part_s += (x0 + x1) + (x2 + x3);
          }
          eb = bin_lane ? ex2((alpha2 + vb) - m) : 0.f;
          s = warp_sum(part_s + eb);
          if (SPLIT > 1) {
            // every part adds the same partials in the same order: s is
            // identical in the whole team
            if (lane == 0) xr_sum[k & 1][team][part] = s;
            team_sync<SPLIT>(team);
            s = xr_sum[k & 1][team][0];
#pragma unroll
            for (int h = 1; h < SPLIT; ++h) s += xr_sum[k & 1][team][h];
          }
          if (exact || (s >= kRowTiny && s < INFINITY)) break;   // team-uniform
          exact = true;                           // reload the raw row and redo it exactly
          load_row(r, g0, e);
          ++k;                                    // fresh exchange slots for the redo
        }
        const float ls = lg2(s);
        const float ratio = ex2(lmu2 - ls);       // mu_r / rowsum_r
        if (bin_lane) u2[r] = lmu2 - m - ls;
#pragma unroll
        for (int c = 0; c < CPW; ++c) colacc[c] = fmaf(e[c], ratio, colacc[c]);
        colbin = fmaf(eb, ratio, colbin);
      }
      // CTA column sums: a 3-round tree over the teams through shared memory
      // (8 -> 4 -> 2 -> 1 partial vectors; the parts of a team own disjoint
      // columns of the same vectors; shared fp32 atomics from 8 warps on the
      // same addresses are an order of magnitude slower).  Each round writes
      // into slots that only the writing team itself read in the round before,
      // so one barrier per round suffices:
      //   round 1: teams 4-7 -> slots 0-3, read by teams 0-3;
      //   round 2: teams 2-3 -> slots 2-3, read by teams 0-1;
      //   round 3: team 1    -> slot 1,    read by team 0, which writes the total.
      auto put = [&](int slot) {
        float4* dst = reinterpret_cast<float4*>(xbuf + (size_t)slot * CV);
#pragma unroll
        for (int qq = 0; qq < NQW; ++qq)
          dst[(g0 + qq) * 32 + lane] =
              make_float4(colacc[4 * qq], colacc[4 * qq + 1], colacc[4 * qq + 2], colacc[4 * qq + 3]);
        if (bin_lane) xbuf[(size_t)slot * CV + LDW] = colbin;
      };
      auto take = [&](int slot) {
        const float4* src = reinterpret_cast<const float4*>(xbuf + (size_t)slot * CV);
#pragma unroll
        for (int qq = 0; qq < NQW; ++qq) {
          const float4 t = src[(g0 + qq) * 32 + lane];
          colacc[4 * qq] += t.x; colacc[4 * qq + 1] += t.y; colacc[4 * qq + 2] += t.z; colacc[4 * qq + 3] += t.w;
        }
        if (bin_lane) colbin += xbuf[(size_t)slot * CV + LDW];
      };
      static_assert(NTEAM == 8, "tree shape");
      if (team >= 4) put(team - 4);
      __syncthreads();
      if (team < 4) take(team);
      if (team == 2 || team == 3) put(team);
      __syncthreads();
      if (team < 2) take(team + 2);
      if (team == 1) put(1);
      __syncthreads();
      if (team == 0) {
        take(1);
        float4* dst = reinterpret_cast<float4*>(ctot);
#pragma unroll
        for (int qq = 0; qq < NQW; ++qq)
          dst[(g0 + qq) * 32 + lane] =
              make_float4(colacc[4 * qq], colacc[4 * qq + 1], colacc[4 * qq + 2], colacc[4 * qq + 3]);
        if (bin_lane) ctot[LDW] = colbin;
        if (cpp > 1) fence_proxy_async_smem();    // ctot is the source of a bulk copy
      }
      __syncthreads();
      // ------------------------------------------------ column pass (group)
      // column totals: ctot (one CTA per pair) or the group's accumulator
      const float* tot = ctot;
      if (cpp > 1) {
        float* acc_now = acc + (size_t)(it % 3) * Cp;
        float* acc_zero = acc + (size_t)((it + 1) % 3) * Cp;   // last read two barriers ago
        if (tid == 0) bulk_add_f32(acc_now, ctot, (unsigned)(CV * sizeof(float)));
        for (int j = rank * NT + tid; j < Cp; j += cpp * NT) acc_zero[j] = 0.f;
        if (barrier()) { failed = true; break; }
        tot = acc_now;
      }
      // column update straight from the totals (each thread its columns of the
      // shared v), with the guard; a tiny total anywhere sends the whole group
      // to the exact recomputation below, which rebuilds v from scratch
      bool bad = false;
      for (int j4 = tid; j4 < CV / 4; j4 += NT) {   // one float4 per thread: one round of latency
        const float4 c4 = cpp > 1 ? __ldcg(reinterpret_cast<const float4*>(tot) + j4)
                                  : reinterpret_cast<const float4*>(tot)[j4];
        float4 v = reinterpret_cast<float4*>(vbuf)[j4];
        const float cm[4] = {c4.x, c4.y, c4.z, c4.w};
        float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = 4 * j4 + i;
          if (j < N || j == LDW) {
            if (!(cm[i] >= kColTiny && cm[i] < INFINITY)) bad = true;
            else vv[i] += (j < N ? lnu_r2 : lnu_b2) - lg2(cm[i]);
          }
        }
        reinterpret_cast<float4*>(vbuf)[j4] = make_float4(vv[0], vv[1], vv[2], vv[3]);
      }
      if (!__syncthreads_or(bad)) {
        // nothing more: the next row pass reads the new v
      } else {
        // exact column LSE: the true column max, then the shifted sum, each
        // combined over the CTA with shared atomics and over the group with
        // global atomics
        for (int j = tid; j < CV; j += NT) ckey[j] = 0u;
        __syncthreads();
        for (int r = r0 + warp; r < r1; r += NWARP) {
          const float ur = u2[r];
          for (int h = 0; h < SPLIT; ++h) {
            float z[CPW];
            load_row(r, h * NQW, z);
#pragma unroll
            for (int qq = 0; qq < NQW; ++qq)
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int j = (h * NQW + qq) * 128 + lane * 4 + i;
                if (j < N) atomicMax(ckey + j, f2key(z[4 * qq + i] + ur));
              }
          }
          if (lane == 0) atomicMax(ckey + LDW, f2key(alpha2 + ur));
        }
        __syncthreads();
        for (int j = tid; j < CV; j += NT)
          if ((j < N || j == LDW) && r1 > r0) atomicMax(fbk + j, ckey[j]);
        if (barrier()) { failed = true; break; }
        // the new v does not depend on the old one: vbuf holds the column max now
        for (int j = tid; j < CV; j += NT) { vbuf[j] = key2f(__ldcg(fbk + j)); ctot[j] = 0.f; }
        __syncthreads();
        for (int r = r0 + warp; r < r1; r += NWARP) {
          const float ur = u2[r];
          const float4* mx4 = reinterpret_cast<const float4*>(vbuf);
          for (int h = 0; h < SPLIT; ++h) {
            float z[CPW];
            load_row(r, h * NQW, z);
#pragma unroll
            for (int qq = 0; qq < NQW; ++qq) {
              const float4 mq = mx4[(h * NQW + qq) * 32 + lane];
              const float mm[4] = {mq.x, mq.y, mq.z, mq.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int j = (h * NQW + qq) * 128 + lane * 4 + i;
                if (j < N) atomicAdd(ctot + j, ex2((z[4 * qq + i] + ur) - mm[i]));
              }
            }
          }
          if (lane == 0) atomicAdd(ctot + LDW, ex2((alpha2 + ur) - vbuf[LDW]));
        }
        __syncthreads();
        for (int j = tid; j < CV; j += NT)
          if ((j < N || j == LDW) && r1 > r0) atomicAdd(fbs + j, ctot[j]);
        if (barrier()) { failed = true; break; }
        for (int j = tid; j < CV; j += NT) {
          if (j < N) vbuf[j] = lnu_r2 - vbuf[j] - lg2(__ldcg(fbs + j));
          else if (j == LDW) vbuf[j] = lnu_b2 - vbuf[j] - lg2(__ldcg(fbs + j));
          ctot[j] = 0.f;
        }
        // clear the fallback buffers for a later use
        if (barrier()) { failed = true; break; }
        for (int j = rank * NT + tid; j < 2 * Cp; j += cpp * NT) fbm[j] = 0.f;
        if (barrier()) { failed = true; break; }
      }
      __syncthreads();
    }
    if (failed) break;

    // ------------------------------------------------ output + extraction
    bool nonfinite = false;
    for (int j = tid; j < CV; j += NT)
      if ((j < N || j == LDW) && !isfinite(vbuf[j])) nonfinite = true;
    const float vb = vbuf[LDW];
    const float4* v4 = reinterpret_cast<const float4*>(vbuf);
    // per-column best keys in shared memory over the row cache (when it has
    // room for them; otherwise straight to global memory)
    const bool smem_best = a.cached_rows >= 2;
    __syncthreads();
    if (smem_best) for (int j = tid; j < LDW; j += NT) cbest[j] = 0ull;
    __syncthreads();
    unsigned long long* cb = a.colbest + (long long)pair * N;
    float* lp = a.logP ? a.logP + (long long)pair * R * C : nullptr;
    for (int r = r0 + warp; r < r1; r += NWARP) {
      const float ur = u2[r];
      if (!isfinite(ur)) nonfinite = true;
      unsigned long long best = 0ull;
      for (int h = 0; h < SPLIT; ++h) {
      float z[CPW];
      load_src(r, h * NQW, z);
#pragma unroll
      for (int qq = 0; qq < NQW; ++qq) {
        const int q = h * NQW + qq;
        const float4 vq = v4[q * 32 + lane];
        const float vv[4] = {vq.x, vq.y, vq.z, vq.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = q * 128 + lane * 4 + i;
          if (j >= N) continue;
          const float val = ((z[4 * qq + i] + ur) + vv[i]) * kLn2 - norm;
          if (lp) lp[(long long)r * C + j] = val;
          if (r < M) {
            const unsigned long long kr = ((unsigned long long)f2key(val) << 32) | (0xffffffffu - (unsigned)j);
            best = kr > best ? kr : best;
            const unsigned long long kc = ((unsigned long long)f2key(val) << 32) | (0xffffffffu - (unsigned)r);
            if (smem_best) atomicMax(cbest + j, kc);
            else atomicMax(cb + j, kc);
          }
        }
      }
      }
      if (lane == 0 && lp) lp[(long long)r * C + N] = ((alpha2 + ur) + vb) * kLn2 - norm;
      if (r < M) {
        best = warp_max_u64(best);
        if (lane == 0) {
          a.idx0[(long long)pair * M + r] = (int)(0xffffffffu - (unsigned)(best & 0xffffffffu));
          a.max0[(long long)pair * M + r] = key2f((unsigned)(best >> 32));
        }
      }
    }
    __syncthreads();
    if (smem_best && r1 > r0 && r0 < M)
      for (int j = tid; j < N; j += NT) atomicMax(cb + j, cbest[j]);
    if (__syncthreads_or(nonfinite) && tid == 0 && rank == 0) atomicOr(a.status, kStatusNumeric);
    if (tid == 0) __threadfence();
    if (barrier()) { failed = true; break; }
    const int32_t* idx0 = a.idx0 + (long long)pair * M;
    const float* max0 = a.max0 + (long long)pair * M;
    for (int r = r0 + tid; r < min(r1, M); r += NT) {
      const int j = __ldcg(idx0 + r);
      const bool jok = j >= 0 && j < N;
      const unsigned long long k = jok ? __ldcg(cb + j) : 0ull;
      const int i = (int)(0xffffffffu - (unsigned)(k & 0xffffffffu));
      const bool mutual = jok && (i == r);
      const float ms = mutual ? expf(__ldcg(max0 + r)) : 0.f;
      const bool valid = mutual && ms > a.threshold;
      a.matches0[(long long)pair * M + r] = valid ? j : -1;
      a.mscores0[(long long)pair * M + r] = ms;
    }
    for (int j = rank * NT + tid; j < N; j += cpp * NT) {
      const unsigned long long k = __ldcg(cb + j);
      const int i = (int)(0xffffffffu - (unsigned)(k & 0xffffffffu));
      const bool iok = k != 0ull && i >= 0 && i < M;
      const bool mutual = iok && __ldcg(idx0 + i) == j;
      const float ms = mutual ? expf(__ldcg(max0 + i)) : 0.f;
      const bool valid = mutual && ms > a.threshold;
      a.matches1[(long long)pair * N + j] = valid ? i : -1;
      a.mscores1[(long long)pair * N + j] = ms;
    }
    // the group's next pair re-stages shared memory; its first barrier orders
    // these reads before any reuse of the scratch
    __syncthreads();
  }
}

// A group of two CTAs of which only one is launched: its barrier can never
// complete, so it must end by its time limit, latch the timeout and return.
__global__ void barrier_selftest_kernel(unsigned* counter, unsigned* abort_flag, unsigned* status,
                                        unsigned long long timeout_ns, int* returned) {
  const bool failed = group_barrier(counter, 2u, abort_flag, status, timeout_ns);
  if (threadIdx.x == 0) *returned = failed ? 1 : 2;
}

// ------------------------------------------------------------------ host side
// Warps per row: one for short rows; for long rows two (three for the longest),
// so that the per-thread row state stays small enough for 512 (768) threads.
template <int NQ> struct SplitOf { static constexpr int value = NQ >= 24 ? 3 : NQ >= 8 ? 2 : 1; };

template <int NQ>
cudaError_t prepare() {
  static bool done = false;
  if (done) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(sinkhorn_kernel<NQ, SplitOf<NQ>::value>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxSmem);
  if (e == cudaSuccess) done = true;
  return e;
}

template <int NQ>
cudaError_t launch_t(SinkhornArgs a, int num_sms, cudaStream_t s, int* launches) {
  constexpr int SPLIT = SplitOf<NQ>::value;
  constexpr int NT = 256 * SPLIT;
  auto kern = sinkhorn_kernel<NQ, SPLIT>;
  constexpr int LDW = 128 * NQ;
  constexpr int CV = LDW + 4;
  cudaError_t e = prepare<NQ>();
  if (e != cudaSuccess) return e;
  const int R = a.M + 1;
  const size_t fixed = (2 + NTEAM / 2) * (size_t)CV * 4;
  const double clk = 1.9e9;
  const double pair_bytes = (double)R * a.N * 4;
  // CTAs per pair, from a cost model of one iteration: MUFU ex2 and issue
  // throughput, re-reads of rows that do not fit on chip (from L2 while the
  // concurrently processed pairs fit there, else from HBM), and the group
  // synchronisation (none for a single CTA).  Groups process pairs
  // concurrently, one CTA per SM.
  const int G = num_sms;
  double best_t = 1e300;
  int best_cpp = 0, best_cached = 0, best_band = 0;
  for (int cpp = 1; cpp <= G && cpp <= R; ++cpp) {
    const int band = (R + cpp - 1) / cpp;
    const size_t ubytes = (size_t)((band + 3) & ~3) * 4;
    if (fixed + ubytes > kMaxSmem) continue;
    const int fit = (int)((kMaxSmem - fixed - ubytes) / ((size_t)LDW * 4));
    const int cached = band < fit ? band : fit;
    const int groups = G / cpp;
    const int conc = a.B < groups ? a.B : groups;
    const double rounds = std::ceil((double)a.B / groups);
    // rows are taken by NTEAM teams in rounds: the busiest team sets the pace
    const double rows = std::ceil((double)band / NTEAM) * NTEAM;
    // per row: one MUFU ex2 per element (16 per clock and SM) and the row plus
    // the column potentials out of shared memory (8 bytes per element at 128
    // bytes per clock), which overlap poorly
    const double mufu = rows * LDW * (1.0 / 16.0 + 8.0 / 128.0) / clk;
    const double issue = rows * (LDW / 32.0 * 6.0 + 60.0) / (4.0 * clk);
    // rows that are not cached are re-read every iteration by latency-bound
    // loads: measured about 40 GB/s per SM from L2 and 17 GB/s per SM when the
    // concurrently processed pairs overflow L2; that time adds to the compute
    const double stream_bw = (double)conc * pair_bytes < 100e6 ? 40e9 : 17e9;
    const double stream = (double)(band - cached) * LDW * 4 / stream_bw;
    const double sync = cpp == 1 ? 0.2e-6 : 2.5e-6 + cpp * 1.0e-8;
    const double work = (mufu > issue ? mufu : issue) + stream;
    const double t = rounds * (work + sync);
    if (t < best_t) { best_t = t; best_cpp = cpp; best_cached = cached; best_band = band; }
  }
  if (const char* f = std::getenv("SG_SINKHORN_CPP")) {
    // tuning override of the CTAs per pair (ignored when it does not fit)
    const int cpp = std::atoi(f);
    if (cpp >= 1 && cpp <= G && cpp <= R) {
      const int band = (R + cpp - 1) / cpp;
      const size_t ubytes = (size_t)((band + 3) & ~3) * 4;
      if (fixed + ubytes <= kMaxSmem) {
        const int fit = (int)((kMaxSmem - fixed - ubytes) / ((size_t)LDW * 4));
        best_cpp = cpp;
        best_band = band;
        best_cached = band < fit ? band : fit;
      }
    }
  }
  if (best_cpp == 0) return cudaErrorInvalidConfiguration;
  a.cpp = best_cpp;
  a.cached_rows = best_cached;
  a.band_alloc = best_band;
  const size_t smem = (size_t)best_cached * LDW * 4 + fixed + (size_t)((best_band + 3) & ~3) * 4;
  if (std::getenv("SG_DEBUG_PLAN"))
    std::fprintf(stderr, "sinkhorn plan: B=%d M=%d N=%d LDW=%d cpp=%d groups=%d band=%d cached=%d smem=%zu\n",
                 a.B, a.M, a.N, LDW, best_cpp, G / best_cpp, best_band, best_cached, smem);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((G / best_cpp) * best_cpp);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (launches) ++*launches;
  return e;
}

}  // namespace

cudaError_t launch_barrier_selftest(unsigned* scratch, unsigned* status, unsigned long long timeout_ns,
                                    int* returned, cudaStream_t s) {
  barrier_selftest_kernel<<<1, 32, 0, s>>>(scratch, scratch + 1, status, timeout_ns, returned);
  return cudaGetLastError();
}

// Scratch layout (floats unless noted), zero-initialised part first:
//   barrier[B] + abort (uint), acc[B][3][pitch], fb[B][2][pitch], colbest[B][N] (u64),
//   then u[B][M+1] (unused), idx0[B][M], max0[B][M].
size_t sinkhorn_acc_floats_per_buffer(int N) { return (size_t)acc_pitch(N); }

size_t sinkhorn_scratch_bytes(int B, int M, int N) {
  size_t z = (B + 1) * sizeof(unsigned);
  z = (z + 255) & ~(size_t)255;
  z += (size_t)B * 5 * acc_pitch(N) * 4;
  z = (z + 255) & ~(size_t)255;
  z += (size_t)B * N * 8;
  z = (z + 255) & ~(size_t)255;
  const size_t nz = (size_t)B * (M + 1) * 4 + (size_t)B * M * 4 * 2 + 3 * 256;
  return z + nz;
}

cudaError_t sinkhorn_prepare(int num_sms) {
  (void)num_sms;
  cudaError_t e = prepare<1>();
  if (e == cudaSuccess) e = prepare<2>();
  if (e == cudaSuccess) e = prepare<4>();
  if (e == cudaSuccess) e = prepare<8>();
  if (e == cudaSuccess) e = prepare<16>();
  if (e == cudaSuccess) e = prepare<24>();
  return e;
}

int sinkhorn_max_columns() { return 24 * 128; }

cudaError_t launch_sinkhorn(SinkhornArgs a, int num_sms, cudaStream_t s, int* launches) {
  switch (nq_for(a.N)) {
    case 1: return launch_t<1>(a, num_sms, s, launches);
    case 2: return launch_t<2>(a, num_sms, s, launches);
    case 4: return launch_t<4>(a, num_sms, s, launches);
    case 8: return launch_t<8>(a, num_sms, s, launches);
    case 16: return launch_t<16>(a, num_sms, s, launches);
    case 24: return launch_t<24>(a, num_sms, s, launches);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sg
