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
// Work decomposition.  A team of TC thread-block clusters of CS CTAs owns one
// pair at a time; the team's CTAs split the M+1 rows into contiguous bands and
// keep as many band rows as fit in shared memory (pre-scaled by log2(e),
// padded with -inf to LD = NT*CPT columns) for all T iterations; the rest are
// re-read from L2 each iteration.  Thread t of every CTA owns the real columns
// j = (q*NT + t)*VW + i (q < NV, i < VW) and warp 0 the dustbin column, so the
// column potentials a thread needs live in its registers and are identical in
// every CTA of the team.
//
// One iteration:
//   row pass (CTA-local): each row's LSE with the shift m_r = log mu_r - u_r
//     (the row's previous LSE; the exact max on the first iteration), one block
//     reduction per RB rows, one MUFU ex2 per element; the same exponentials,
//     scaled by mu_r / rowsum_r, are the plan mass P_rj = exp(Z + u + v) that
//     the column update needs, accumulated per column in registers;
//   column pass: the CTAs of a cluster reduce-scatter their column partials
//     through distributed shared memory (DSMEM); with TC == 1 the slice totals
//     are all-gathered the same way and no global memory is involved; with
//     TC > 1 each cluster adds its slice totals to a global accumulator (one
//     fp32 red per column and cluster), rank 0 of every cluster meets the other
//     clusters at a global counter, and every CTA reads the totals back;
//     v_j(new) = v_j + log nu_j - log(sum_r P_rj)   (sum_r P_rj <= 1).
// Where a sum comes out tiny (below 2^-40 for rows, 2^-50 for columns: precision
// could have been lost to underflow) that LSE is recomputed exactly with its
// true max.  Every decision that steers control flow is taken on values that
// are identical in all CTAs of the team, so they all take the same path through
// the barriers.
//
// Waits: cluster barriers are hardware barriers that every CTA of a cluster
// reaches the same number of times; the global meeting spins with a time limit
// and, on expiry, latches a timeout in the status word, raises an abort flag
// that ends every other wait, and the team returns.
#include "sg_internal.cuh"

#include <cooperative_groups.h>
#include <math.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>

namespace cg = cooperative_groups;

namespace sg {
namespace {

constexpr int NT = 512;
constexpr int NW = NT / 32;
constexpr int kMaxCS = 16;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRowTiny = 9.094947017729282e-13f;   // 2^-40
constexpr float kColTiny = 8.881784197001252e-16f;   // 2^-50

__host__ __device__ inline int acc_pitch(int N) { return ((N + 1) + 31) & ~31; }

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

// Grid barrier over a group of CTAs (used by the self-test).
__device__ bool group_barrier(unsigned* counter, unsigned target, unsigned* abort_flag,
                              unsigned* status, unsigned long long timeout_ns) {
  __shared__ int s_fail;
  __syncthreads();
  if (threadIdx.x == 0) s_fail = counter_wait(counter, target, abort_flag, status, timeout_ns) ? 1 : 0;
  __syncthreads();
  return s_fail != 0;
}

// ------------------------------------------------------------------ reductions
template <int RB> struct Log2;
template <> struct Log2<2> { static constexpr int v = 1; };
template <> struct Log2<4> { static constexpr int v = 2; };
template <> struct Log2<8> { static constexpr int v = 3; };
template <> struct Log2<16> { static constexpr int v = 4; };

struct OpSum { __device__ float operator()(float a, float b) const { return a + b; } };
struct OpMax { __device__ float operator()(float a, float b) const { return fmaxf(a, b); } };

// Block reduction of RB values per thread (RB in {2,4,8,16}).  Warp stage: a
// reduce-scatter by shuffles, after which lane l holds the warp total of value
// l / (32/RB); block stage: the RB x NW warp totals are combined from shared
// memory.  Returns, in every lane l of every warp, the block total of value
// l / (32/RB).
template <int RB, typename Op>
__device__ __forceinline__ float block_reduce_lane(const float (&v)[RB], float* red, Op op) {
  constexpr int LG = Log2<RB>::v;
  constexpr int L = 32 / RB;
  constexpr int P = RB * NW / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float x[RB];
#pragma unroll
  for (int i = 0; i < RB; ++i) x[i] = v[i];
#pragma unroll
  for (int st = 0; st < LG; ++st) {
    const int mask = 16 >> st;
    const int n = RB >> st;
    const bool hi = (lane & mask) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float send = hi ? x[i] : x[i + n / 2];
      const float keep = hi ? x[i + n / 2] : x[i];
      x[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, mask));
    }
  }
  float t = x[0];
#pragma unroll
  for (int mask = L / 2; mask > 0; mask >>= 1) t = op(t, __shfl_xor_sync(0xffffffffu, t, mask));
  if ((lane & (L - 1)) == 0) red[(lane / L) * NW + w] = t;
  __syncthreads();
  const float* src = red + (lane / L) * NW + (lane % L) * P;
  float tot = src[0];
#pragma unroll
  for (int i = 1; i < P; ++i) tot = op(tot, src[i]);
#pragma unroll
  for (int mask = L / 2; mask > 0; mask >>= 1) tot = op(tot, __shfl_xor_sync(0xffffffffu, tot, mask));
  return tot;
}

template <int RB, typename Op>
__device__ __forceinline__ void block_reduce(float (&v)[RB], float* red, Op op) {
  const float tot = block_reduce_lane<RB>(v, red, op);
#pragma unroll
  for (int i = 0; i < RB; ++i) v[i] = __shfl_sync(0xffffffffu, tot, i * (32 / RB));
}

template <int RB>
__device__ __forceinline__ float select_k(const float (&v)[RB], int k) {
  float r = v[0];
#pragma unroll
  for (int i = 1; i < RB; ++i) r = (k == i) ? v[i] : r;
  return r;
}

__device__ __forceinline__ unsigned long long block_max_u64(unsigned long long x, unsigned long long* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, o);
    x = y > x ? y : x;
  }
  if (lane == 0) red[w] = x;
  __syncthreads();
  unsigned long long r = 0;
#pragma unroll
  for (int i = 0; i < NW; ++i) r = red[i] > r ? red[i] : r;
  return r;
}

// ------------------------------------------------------------------ kernel
template <int VW, int NV, int RB>
__global__ void __launch_bounds__(NT, 1) sinkhorn_kernel(SinkhornArgs a) {
  constexpr int CPT = VW * NV;
  constexpr int LD = NT * CPT;                    // padded row length in shared memory
  extern __shared__ __align__(16) unsigned char smraw[];
  __shared__ float s_binpart[kMaxCS];             // dustbin-column partials (rank 0 receives)
  __shared__ float s_binmass;                     // dustbin-column total
  __shared__ int s_fail;

  cg::cluster_group cluster = cg::this_cluster();
  const int CS = (int)cluster.num_blocks();
  const int crank = (int)cluster.block_rank();
  const int TC = a.team_clusters;
  const int cpp = CS * TC;                        // CTAs per team
  const int cluster_id = blockIdx.x / CS;
  const int nteams = (gridDim.x / CS) / TC;
  const int team = cluster_id / TC;
  const int rank = (cluster_id % TC) * CS + crank;  // rank within the team
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  constexpr int LR = 32 / RB;                     // lanes per row in the row bookkeeping
  const int SL = LD / CS;                         // column slice owned by each cluster rank

  const int M = a.M, N = a.N, R = M + 1, C = N + 1;
  const int Cp = acc_pitch(N);
  const int band = (R + cpp - 1) / cpp;
  const int r0 = min(R, rank * band), r1 = min(R, r0 + band);
  const int cached = min(r1 - r0, a.cached_rows);

  // shared memory: [cache | reduction x2 | u (band) | xbuf (CS x SL) | mass (LD)]
  float* cache = reinterpret_cast<float*>(smraw);
  unsigned char* redbase = smraw + (size_t)a.cached_rows * LD * sizeof(float);
  float* u2s = reinterpret_cast<float*>(redbase + 2 * RB * NW * 8);
  float* xbuf = u2s + ((a.band_alloc + 3) & ~3);
  float* mass = xbuf + LD;
  unsigned nred = 0;
  auto redf = [&]() { return reinterpret_cast<float*>(redbase + (size_t)((nred++) & 1u) * RB * NW * 8); };
  auto red64 = [&]() {
    return reinterpret_cast<unsigned long long*>(redbase + (size_t)((nred++) & 1u) * RB * NW * 8);
  };

  // log2-domain constants: log mu, log nu and the dustbin score, times log2(e)
  const float norm = -logf((float)(M + N));
  const float lmu_r2 = norm * kLog2e, lmu_b2 = (logf((float)N) + norm) * kLog2e;
  const float lnu_r2 = norm * kLog2e, lnu_b2 = (logf((float)M) + norm) * kLog2e;
  const float alpha2 = a.alpha * kLog2e;

  int col[CPT];                                   // real column of each register slot
#pragma unroll
  for (int q = 0; q < NV; ++q)
#pragma unroll
    for (int i = 0; i < VW; ++i) col[q * VW + i] = (q * NT + tid) * VW + i;

  // every CTA of the cluster must be running before any DSMEM access
  cluster.sync();

  unsigned gen = 0;
  unsigned* counter = a.barrier + team;
  const bool active_team = team < nteams;
  bool failed = false;

  // Team barrier: a cluster barrier, and with TC > 1 a global meeting of the
  // team's clusters by their rank-0 CTAs.  Returns true if it failed; the
  // result is the same in every CTA of a cluster.
  auto team_barrier = [&]() -> bool {
    if (TC == 1) {
      cluster.sync();
      return false;
    }
    __syncthreads();
    if (tid == 0) __threadfence();
    cluster.sync();
    if (crank == 0 && tid == 0) {
      ++gen;
      const bool f = counter_wait(counter, gen * TC, a.abort_flag, a.status, a.timeout_ns);
      for (int r = 0; r < CS; ++r) *cluster.map_shared_rank(&s_fail, r) = f ? 1 : 0;
    }
    cluster.sync();
    return s_fail != 0;
  };

  // Column reduction over the team: vals[c] are this thread's partials of its
  // columns, bin is the dustbin-column partial held by thread 0.  On return
  // vals[c] and bin hold the team totals (in every thread).  Sum, or max when
  // ismax.  gacc: zeroed global accumulator (TC > 1); gzero: buffer to clear.
  auto team_columns = [&](float (&vals)[CPT], float& bin, bool ismax, float* gacc, float* gzero,
                          int gzero_len) -> bool {
    // reduce-scatter through DSMEM: rank k receives slice k from every rank
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const int jv = (q * NT + tid) * VW;
      const int dst = jv / SL, off = jv % SL;
      float* p = cluster.map_shared_rank(xbuf, dst) + crank * SL + off;
      if (VW == 4) {
        *reinterpret_cast<float4*>(p) =
            make_float4(vals[q * 4], vals[q * 4 + 1], vals[q * 4 + 2], vals[q * 4 + 3]);
      } else if (VW == 2) {
        *reinterpret_cast<float2*>(p) = make_float2(vals[q * 2], vals[q * 2 + 1]);
      } else {
        *p = vals[q];
      }
    }
    if (tid == 0) *cluster.map_shared_rank(&s_binpart[crank], 0) = bin;
    if (TC > 1 && gzero)
      for (int j = rank * NT + tid; j < gzero_len; j += cpp * NT) gzero[j] = 0.f;
    cluster.sync();
    float tot = ismax ? -INFINITY : 0.f;
    const bool mine = tid < SL;
    if (mine) {
      for (int r = 0; r < CS; ++r) {
        const float x = xbuf[r * SL + tid];
        tot = ismax ? fmaxf(tot, x) : tot + x;
      }
    }
    float btot = ismax ? -INFINITY : 0.f;
    if (crank == 0 && tid == 0)
      for (int r = 0; r < CS; ++r) btot = ismax ? fmaxf(btot, s_binpart[r]) : btot + s_binpart[r];
    const int jslice = crank * SL + tid;
    if (TC == 1) {
      // all-gather the slice totals into every CTA's mass buffer
      if (mine)
        for (int r = 0; r < CS; ++r) cluster.map_shared_rank(mass, r)[jslice] = tot;
      if (crank == 0 && tid == 0)
        for (int r = 0; r < CS; ++r) *cluster.map_shared_rank(&s_binmass, r) = btot;
      cluster.sync();
#pragma unroll
      for (int c = 0; c < CPT; ++c) vals[c] = mass[col[c]];
      bin = s_binmass;
      return false;
    }
    // TC > 1: the clusters' slice totals meet in global memory
    if (mine && jslice < N) {
      if (ismax) atomicMax(reinterpret_cast<unsigned*>(gacc) + jslice, f2key(tot));
      else atomicAdd(gacc + jslice, tot);
    }
    if (crank == 0 && tid == 0) {
      if (ismax) atomicMax(reinterpret_cast<unsigned*>(gacc) + N, f2key(btot));
      else atomicAdd(gacc + N, btot);
    }
    if (team_barrier()) return true;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      if (col[c] < N) {
        const float g = __ldcg(gacc + col[c]);
        vals[c] = ismax ? key2f(__float_as_uint(g)) : g;
      }
    }
    const float gb = __ldcg(gacc + N);
    bin = ismax ? key2f(__float_as_uint(gb)) : gb;
    return false;
  };

  for (int pair = team; active_team && pair < a.B && !failed; pair += nteams) {
    const float* S = a.S + (long long)pair * a.strideS;
    float* u2 = u2s - r0;                         // row potentials of the band (log2 domain)
    float* acc = a.acc + (long long)pair * 3 * Cp;
    float* fbm = a.fb + (long long)pair * 2 * Cp;  // exact column fallback: max keys
    float* fbs = fbm + Cp;                         // exact column fallback: sums

    // z2 of row r (log2 domain) for this thread's column slots
    auto load_row = [&](int r, float (&z)[CPT]) {
      if (r - r0 < cached) {
        const float* row = cache + (size_t)(r - r0) * LD;
#pragma unroll
        for (int q = 0; q < NV; ++q) {
          const int o = (q * NT + tid) * VW;
          if (VW == 4) {
            const float4 t = *reinterpret_cast<const float4*>(row + o);
            z[q * 4 + 0] = t.x; z[q * 4 + 1] = t.y; z[q * 4 + 2] = t.z; z[q * 4 + 3] = t.w;
          } else if (VW == 2) {
            const float2 t = *reinterpret_cast<const float2*>(row + o);
            z[q * 2 + 0] = t.x; z[q * 2 + 1] = t.y;
          } else {
            z[q] = row[o];
          }
        }
      } else if (VW == 4 && a.lds_vec && r < M) {
        const float* src = S + (long long)r * a.lds;
#pragma unroll
        for (int q = 0; q < NV; ++q) {
          const int o = (q * NT + tid) * VW;
          float4 t = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
          if (o + 3 < N) {
            t = __ldg(reinterpret_cast<const float4*>(src + o));
            t.x *= kLog2e; t.y *= kLog2e; t.z *= kLog2e; t.w *= kLog2e;
          } else {
            if (o < N) t.x = __ldg(src + o) * kLog2e;
            if (o + 1 < N) t.y = __ldg(src + o + 1) * kLog2e;
            if (o + 2 < N) t.z = __ldg(src + o + 2) * kLog2e;
          }
          z[q * 4 + 0] = t.x; z[q * 4 + 1] = t.y; z[q * 4 + 2] = t.z; z[q * 4 + 3] = t.w;
        }
      } else {
        const float* src = S + (long long)r * a.lds;
#pragma unroll
        for (int c = 0; c < CPT; ++c)
          z[c] = col[c] < N ? (r < M ? __ldg(src + col[c]) : a.alpha) * kLog2e : -INFINITY;
      }
    };

    // ---- stage the band in shared memory (pre-scaled, padded with -inf)
    __syncthreads();
    for (int r = r0; r < r0 + cached; ++r) {
      const float* src = S + (long long)r * a.lds;
      float* dst = cache + (size_t)(r - r0) * LD;
      for (int j = tid; j < LD; j += NT)
        dst[j] = j < N ? (r < M ? __ldg(src + j) : a.alpha) * kLog2e : -INFINITY;
    }
    for (int r = r0 + tid; r < r1; r += NT) u2[r] = 0.f;
    __syncthreads();

    float v2[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) v2[c] = 0.f;
    float vb2 = 0.f;                              // dustbin column (warp 0)

    for (int it = 0; it < a.iters; ++it) {
      // ------------------------------------------------ row pass (CTA-local)
      float colacc[CPT];
#pragma unroll
      for (int c = 0; c < CPT; ++c) colacc[c] = 0.f;
      float colbin = 0.f;
      for (int rc = r0; rc < r1; rc += RB) {
        float e[RB][CPT];
        float m2[RB];
#pragma unroll
        for (int k = 0; k < RB; ++k) {
          const int r = rc + k;
          if (r < r1) load_row(r, e[k]);
          else {
#pragma unroll
            for (int c = 0; c < CPT; ++c) e[k][c] = -INFINITY;
          }
          m2[k] = (r < r1 && it > 0) ? (r < M ? lmu_r2 : lmu_b2) - u2[r] : 0.f;
        }
        // lane-parallel row bookkeeping: lane l of every warp handles row rc + l / LR
        const int kk = lane / LR;
        const int rr = rc + kk;
        const bool row_ok = rr < r1;
        const float lmu2_l = rr < M ? lmu_r2 : lmu_b2;
        const bool bin_lane = (warp == 0) && (lane < RB) && (rc + lane < r1);   // dustbin column
        float tot, ebin = 0.f;
        bool exact = (it == 0);
        while (true) {
          if (exact) {
#pragma unroll
            for (int k = 0; k < RB; ++k) {
              float mx = (bin_lane && lane == k) ? alpha2 + vb2 : -INFINITY;
#pragma unroll
              for (int c = 0; c < CPT; ++c) mx = fmaxf(mx, e[k][c] + v2[c]);
              m2[k] = mx;
            }
            block_reduce<RB>(m2, redf(), OpMax());
#pragma unroll
            for (int k = 0; k < RB; ++k) if (rc + k >= r1) m2[k] = 0.f;
          }
          float part[RB];
#pragma unroll
          for (int k = 0; k < RB; ++k) {
            float acc_k = 0.f;
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
              const float x = ex2((e[k][c] + v2[c]) - m2[k]);
              e[k][c] = x;
              acc_k += x;
            }
            part[k] = acc_k;
          }
          ebin = bin_lane ? ex2((alpha2 + vb2) - select_k<RB>(m2, lane)) : 0.f;
#pragma unroll
          for (int k = 0; k < RB; ++k) if (lane == k) part[k] += ebin;
          tot = block_reduce_lane<RB>(part, redf(), OpSum());
          if (exact) break;
          // identical in every warp (same totals), hence block-uniform
          const bool bad = __any_sync(0xffffffffu, row_ok && !(tot >= kRowTiny && tot < INFINITY));
          if (!bad) break;
          exact = true;                           // reload the raw rows and redo them exactly
#pragma unroll
          for (int k = 0; k < RB; ++k)
            if (rc + k < r1) load_row(rc + k, e[k]);
        }
        const float ls = lg2(tot);
        const float ratio_l = row_ok ? ex2(lmu2_l - ls) : 0.f;   // mu_r / rowsum_r
        if (warp == 0 && row_ok && (lane % LR) == 0) u2[rr] = lmu2_l - select_k<RB>(m2, kk) - ls;
#pragma unroll
        for (int k = 0; k < RB; ++k) {
          const float ratio = __shfl_sync(0xffffffffu, ratio_l, k * LR);
#pragma unroll
          for (int c = 0; c < CPT; ++c) colacc[c] = fmaf(e[k][c], ratio, colacc[c]);
          if (bin_lane && lane == k) colbin = fmaf(ebin, ratio, colbin);
        }
      }
      // ------------------------------------------------ column pass (team)
      if (warp == 0) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) colbin += __shfl_xor_sync(0xffffffffu, colbin, o);
      }
      float* acc_now = acc + (size_t)(it % 3) * Cp;
      float* acc_zero = acc + (size_t)((it + 1) % 3) * Cp;   // last read two barriers ago
      if (team_columns(colacc, colbin, false, acc_now, acc_zero, Cp)) { failed = true; break; }
      bool bad = false;
#pragma unroll
      for (int c = 0; c < CPT; ++c)
        if (col[c] < N && !(colacc[c] >= kColTiny && colacc[c] < INFINITY)) bad = true;
      if (!(colbin >= kColTiny && colbin < INFINITY)) bad = true;
      if (!__syncthreads_or(bad)) {
#pragma unroll
        for (int c = 0; c < CPT; ++c) if (col[c] < N) v2[c] += lnu_r2 - lg2(colacc[c]);
        if (warp == 0) vb2 += lnu_b2 - lg2(colbin);
      } else {
        // exact column LSE: the true column max, then the shifted sum
        float mx[CPT];
        float mxb = -INFINITY;
#pragma unroll
        for (int c = 0; c < CPT; ++c) mx[c] = -INFINITY;
        for (int r = r0; r < r1; ++r) {
          float z[CPT];
          load_row(r, z);
          const float ur = u2[r];
#pragma unroll
          for (int c = 0; c < CPT; ++c) mx[c] = fmaxf(mx[c], z[c] + ur);
          mxb = fmaxf(mxb, alpha2 + ur);
        }
        if (team_columns(mx, mxb, true, fbm, nullptr, 0)) { failed = true; break; }
        float sm[CPT];
        float smb = 0.f;
#pragma unroll
        for (int c = 0; c < CPT; ++c) sm[c] = 0.f;
        for (int r = r0; r < r1; ++r) {
          float z[CPT];
          load_row(r, z);
          const float ur = u2[r];
#pragma unroll
          for (int c = 0; c < CPT; ++c) sm[c] += ex2((z[c] + ur) - mx[c]);
          smb += ex2((alpha2 + ur) - mxb);
        }
        if (team_columns(sm, smb, false, fbs, nullptr, 0)) { failed = true; break; }
#pragma unroll
        for (int c = 0; c < CPT; ++c) if (col[c] < N) v2[c] = lnu_r2 - mx[c] - lg2(sm[c]);
        if (warp == 0) vb2 = lnu_b2 - mxb - lg2(smb);
        if (TC > 1) {                             // clear the fallback buffers for a later use
          if (team_barrier()) { failed = true; break; }
          for (int j = rank * NT + tid; j < 2 * Cp; j += cpp * NT) fbm[j] = 0.f;
          if (team_barrier()) { failed = true; break; }
        }
      }
    }
    if (failed) break;

    // ------------------------------------------------ output + extraction
    bool nonfinite = !isfinite(vb2);
#pragma unroll
    for (int c = 0; c < CPT; ++c) if (col[c] < N && !isfinite(v2[c])) nonfinite = true;
    float* lp = a.logP ? a.logP + (long long)pair * R * C : nullptr;
    unsigned long long colb[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) colb[c] = 0ull;
    for (int r = r0; r < r1; ++r) {
      float z[CPT];
      load_row(r, z);
      const float ur = u2[r];
      if (!isfinite(ur)) nonfinite = true;
      unsigned long long best = 0ull;
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        const int j = col[c];
        if (j >= N) continue;
        const float val = ((z[c] + ur) + v2[c]) * kLn2 - norm;
        if (lp) lp[(long long)r * C + j] = val;
        if (r < M) {
          const unsigned long long kr = ((unsigned long long)f2key(val) << 32) | (0xffffffffu - (unsigned)j);
          best = kr > best ? kr : best;
          const unsigned long long kc = ((unsigned long long)f2key(val) << 32) | (0xffffffffu - (unsigned)r);
          colb[c] = kc > colb[c] ? kc : colb[c];
        }
      }
      if (tid == 0 && lp) lp[(long long)r * C + N] = ((alpha2 + ur) + vb2) * kLn2 - norm;
      if (r < M) {
        best = block_max_u64(best, red64());
        if (tid == 0) {
          a.idx0[(long long)pair * M + r] = (int)(0xffffffffu - (unsigned)(best & 0xffffffffu));
          a.max0[(long long)pair * M + r] = key2f((unsigned)(best >> 32));
        }
      }
    }
    unsigned long long* cb = a.colbest + (long long)pair * N;
#pragma unroll
    for (int c = 0; c < CPT; ++c)
      if (col[c] < N && colb[c]) atomicMax(cb + col[c], colb[c]);
    if (__syncthreads_or(nonfinite) && tid == 0 && rank == 0) atomicOr(a.status, kStatusNumeric);
    if (tid == 0) __threadfence();
    if (team_barrier()) { failed = true; break; }
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
    // the team's next pair re-stages shared memory only after this point
    __syncthreads();
  }
  // no CTA may leave while a peer could still write into its shared memory
  cluster.sync();
}

// A group of two CTAs of which only one is launched: its barrier can never
// complete, so it must end by its time limit, latch the timeout and return.
__global__ void barrier_selftest_kernel(unsigned* counter, unsigned* abort_flag, unsigned* status,
                                        unsigned long long timeout_ns, int* returned) {
  const bool failed = group_barrier(counter, 2u, abort_flag, status, timeout_ns);
  if (threadIdx.x == 0) *returned = failed ? 1 : 2;
}

// ------------------------------------------------------------------ host side
constexpr size_t kMaxSmem = 220 * 1024;

// Kernel attributes and, per cluster size, how many clusters can be resident
// at once (queried once, outside any stream capture).
template <int VW, int NV, int RB>
cudaError_t prepare(int num_sms, int (*&out)[5]) {
  static int max_clusters[5] = {-1, -1, -1, -1, -1};
  static bool done = false;
  out = &max_clusters;
  if (done) return cudaSuccess;
  auto kern = sinkhorn_kernel<VW, NV, RB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  const int cs_list[5] = {1, 2, 4, 8, 16};
  for (int ci = 0; ci < 5; ++ci) {
    const int CS = cs_list[ci];
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(CS);
    q.blockDim = dim3(NT);
    q.dynamicSmemBytes = kMaxSmem;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = CS;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.attrs = qa;
    q.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &q) != cudaSuccess) { cudaGetLastError(); n = 0; }
    if (n * CS > num_sms) n = num_sms / CS;
    max_clusters[ci] = n;
  }
  done = true;
  return cudaSuccess;
}

template <int VW, int NV, int RB>
cudaError_t launch_t(SinkhornArgs a, int num_sms, cudaStream_t s, int* launches) {
  auto kern = sinkhorn_kernel<VW, NV, RB>;
  constexpr int LD = NT * VW * NV;
  const int R = a.M + 1;
  const size_t max_smem = kMaxSmem;
  int (*mc)[5] = nullptr;
  cudaError_t pe = prepare<VW, NV, RB>(num_sms, mc);
  if (pe != cudaSuccess) return pe;
  const int* max_clusters = *mc;
  // shared memory besides the row cache: reductions, two LD-wide exchange
  // buffers, and the band's row potentials
  const size_t fixed = 2 * RB * NW * 8 + 2 * (size_t)LD * 4;
  // Candidate decompositions: cluster size CS, clusters per team TC.  Cost
  // model per iteration: the team's MUFU ex2 throughput, re-reads of the rows
  // that do not fit on chip (from L2 while the concurrently processed pairs fit
  // there, else from HBM), and synchronisation (intra-cluster for TC == 1, a
  // global meeting otherwise).  Teams process pairs concurrently.
  const double clk = 1.9e9;
  const double pair_bytes = (double)R * LD * 4;
  double best_t = 1e300;
  int bCS = 0, bTC = 0, bcached = 0, bband = 0, bgrid = 0;
  const int cs_list[5] = {1, 2, 4, 8, 16};
  for (int ci = 0; ci < 5; ++ci) {
    const int CS = cs_list[ci];
    if (LD % CS != 0 || LD / CS > NT) continue;
    const int nclusters = max_clusters[ci];
    for (int TC = 1; TC <= nclusters; ++TC) {
      const int cpp = CS * TC;
      if (cpp > R) break;
      const int band = (R + cpp - 1) / cpp;
      const size_t ubytes = (size_t)((band + 3) & ~3) * 4;
      if (fixed + ubytes > max_smem) continue;
      const int fit = (int)((max_smem - fixed - ubytes) / ((size_t)LD * 4));
      const int cached = band < fit ? band : fit;
      const int teams = nclusters / TC;
      const int conc = a.B < teams ? a.B : teams;
      const double rounds = std::ceil((double)a.B / teams);
      const double mufu = (double)band * LD / 16.0 / clk;
      const double stream_bw = (double)conc * pair_bytes < 100e6 ? 100e9 : 6.5e12 / num_sms;
      const double stream = (double)(band - cached) * LD * 4 / stream_bw;
      // one global fp32 red per column and cluster (measured ~27 ps each when
      // many CTAs add into the same few KB)
      const double sync = TC == 1 ? (CS == 1 ? 0.3e-6 : 1.0e-6) : 3.5e-6 + 2.7e-11 * TC * a.N;
      const double t = rounds * ((mufu > stream ? mufu : stream) + sync);
      if (t < best_t) {
        best_t = t;
        bCS = CS; bTC = TC; bcached = cached; bband = band; bgrid = teams * TC * CS;
      }
    }
  }
  if (bCS == 0) return cudaErrorInvalidConfiguration;
  a.team_clusters = bTC;
  a.cached_rows = bcached;
  a.band_alloc = bband;
  if (std::getenv("SG_DEBUG_PLAN"))
    std::fprintf(stderr, "sinkhorn plan: B=%d M=%d N=%d LD=%d CS=%d TC=%d teams=%d band=%d cached=%d grid=%d\n",
                 a.B, a.M, a.N, LD, bCS, bTC, bgrid / (bCS * bTC), bband, bcached, bgrid);
  const size_t smem = (size_t)bcached * LD * 4 + fixed + (size_t)((bband + 3) & ~3) * 4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(bgrid);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute la[1];
  la[0].id = cudaLaunchAttributeClusterDimension;
  la[0].val.clusterDim.x = bCS;
  la[0].val.clusterDim.y = 1;
  la[0].val.clusterDim.z = 1;
  cfg.attrs = la;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a);
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
  int (*mc)[5] = nullptr;
  cudaError_t e = prepare<1, 1, 16>(num_sms, mc);
  if (e == cudaSuccess) e = prepare<2, 1, 16>(num_sms, mc);
  if (e == cudaSuccess) e = prepare<4, 1, 8>(num_sms, mc);
  if (e == cudaSuccess) e = prepare<4, 2, 4>(num_sms, mc);
  if (e == cudaSuccess) e = prepare<4, 4, 2>(num_sms, mc);
  return e;
}

cudaError_t launch_sinkhorn(SinkhornArgs a, int num_sms, cudaStream_t s, int* launches) {
  const int N = a.N;
  if (N <= NT) return launch_t<1, 1, 16>(a, num_sms, s, launches);
  if (N <= 2 * NT) return launch_t<2, 1, 16>(a, num_sms, s, launches);
  if (N <= 4 * NT) return launch_t<4, 1, 8>(a, num_sms, s, launches);
  if (N <= 8 * NT) return launch_t<4, 2, 4>(a, num_sms, s, launches);
  if (N <= 16 * NT) return launch_t<4, 4, 2>(a, num_sms, s, launches);
  return cudaErrorInvalidValue;
}

}  // namespace sg
