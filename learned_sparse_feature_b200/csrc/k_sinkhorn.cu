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
// Layout: a group of `cpp` co-resident CTAs owns one pair at a time; CTA k of
// the group owns a contiguous band of rows (the dustbin row included) and keeps
// as many of them as fit in shared memory for all T iterations (the rest are
// re-read from L2).  Thread t of every CTA owns the columns j = t + c*512, so
// the potentials v_j of its columns live in registers and are identical in all
// CTAs of the group.
//
// Each log-sum-exp is evaluated with a shift that is known before the pass:
//   rows:    m_r = log mu_r - u_r(prev)   (the previous LSE of the row)
//   columns: the column pass accumulates the plan mass P_rj = exp(Z + u + v)
//            after the row update, which is at most 1 per column; then
//            v_j(new) = v_j + log nu_j - log(sum_r P_rj).
// So a row pass needs one block reduction and a column pass one fp32 atomic per
// column and CTA plus ONE grid barrier per iteration, and every element costs a
// single exp: P_rj = exp(Z_rj + v_j - m_r) * (mu_r / rowsum_r).  Where a sum
// comes out tiny (below 2^-40 for rows, 2^-50 for columns: precision could have
// been lost to underflow), that LSE is recomputed exactly with its true max;
// the first row pass always uses the true max.  All decisions that steer
// control flow are taken on block-uniform values, so every CTA of a group takes
// the same path through the barriers.
//
// Grid barriers spin with a time limit: on expiry they latch a timeout in the
// status word, raise an abort flag that ends every other wait at once, and the
// kernel returns.
#include "sg_internal.cuh"

#include <math.h>

namespace sg {
namespace {

constexpr int NT = 512;
constexpr int NW = NT / 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRowTiny = 9.094947017729282e-13f;   // 2^-40
constexpr float kColTiny = 8.881784197001252e-16f;   // 2^-50

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

// Grid barrier over the cpp CTAs of a group.  Returns true if it failed.
__device__ bool group_barrier(unsigned* counter, unsigned target, unsigned* abort_flag,
                              unsigned* status, unsigned long long timeout_ns) {
  __shared__ int s_fail;
  __syncthreads();
  if (threadIdx.x == 0) {
    int fail = 0;
    __threadfence();
    atomicAdd(counter, 1u);
    const unsigned long long t0 = globaltimer();
    while (true) {
      if (ld_acquire(counter) >= target) break;
      if (ld_relaxed(abort_flag)) { fail = 1; break; }
      if (globaltimer() - t0 > timeout_ns) {
        atomicOr(status, kStatusTimeout);
        atomicExch(abort_flag, 1u);
        fail = 1;
        break;
      }
      __nanosleep(32);
    }
    __threadfence();
    s_fail = fail;
  }
  __syncthreads();
  return s_fail != 0;
}

template <int RB>
__device__ __forceinline__ void block_sum(float (&v)[RB], float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int k = 0; k < RB; ++k) {
    float x = v[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (lane == 0) red[k * NW + w] = x;
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < RB; ++k) {
    float x = 0.f;
#pragma unroll
    for (int i = 0; i < NW; ++i) x += red[k * NW + i];
    v[k] = x;
  }
}

template <int RB>
__device__ __forceinline__ void block_max(float (&v)[RB], float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int k = 0; k < RB; ++k) {
    float x = v[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    if (lane == 0) red[k * NW + w] = x;
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < RB; ++k) {
    float x = -INFINITY;
#pragma unroll
    for (int i = 0; i < NW; ++i) x = fmaxf(x, red[k * NW + i]);
    v[k] = x;
  }
}

template <int RB>
__device__ __forceinline__ void block_max_u64(unsigned long long (&v)[RB], unsigned long long* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int k = 0; k < RB; ++k) {
    unsigned long long x = v[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, o);
      x = y > x ? y : x;
    }
    if (lane == 0) red[k * NW + w] = x;
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < RB; ++k) {
    unsigned long long x = 0;
#pragma unroll
    for (int i = 0; i < NW; ++i) x = red[k * NW + i] > x ? red[k * NW + i] : x;
    v[k] = x;
  }
}

struct PairView {
  const float* S;    // real block, row stride lds
  long long lds;
  float* cache;      // shared memory rows [r0, r0 + cached) x C
  int r0, cached, M, N, C;
  float alpha;
  __device__ __forceinline__ float z(int r, int j) const {
    if (r - r0 < cached) return cache[(r - r0) * C + j];
    return (r < M && j < N) ? __ldg(S + (long long)r * lds + j) : alpha;
  }
};

template <int CPT, int RB>
__global__ void __launch_bounds__(NT, 1) sinkhorn_kernel(SinkhornArgs a) {
  extern __shared__ __align__(16) unsigned char smraw[];
  const int tid = threadIdx.x;
  const int cpp = a.cpp;
  const int group = blockIdx.x / cpp;
  const int rank = blockIdx.x % cpp;
  const int ngroups = gridDim.x / cpp;
  if (group >= ngroups) return;      // CTAs beyond the last full group stay idle
  const int M = a.M, N = a.N, R = M + 1, C = N + 1;
  const int band = (R + cpp - 1) / cpp;
  const int r0 = min(R, rank * band), r1 = min(R, r0 + band);
  const int cached = min(r1 - r0, a.cached_rows);

  float* cache = reinterpret_cast<float*>(smraw);
  const size_t off = ((size_t)a.cached_rows * C * sizeof(float) + 15) & ~(size_t)15;
  // Two reduction buffers of RB x NW 8-byte slots, used alternately (nred) so
  // that one __syncthreads per block reduction suffices.
  unsigned char* redbase = smraw + off;
  unsigned nred = 0;
#define SG_REDF() reinterpret_cast<float*>(redbase + (size_t)((nred++) & 1u) * RB * NW * 8)
#define SG_RED64() reinterpret_cast<unsigned long long*>(redbase + (size_t)((nred++) & 1u) * RB * NW * 8)

  unsigned* counter = a.barrier + group;
  unsigned gen = 0;
  const float norm = -logf((float)(M + N));
  const float lmu_real = norm, lmu_bin = logf((float)N) + norm;
  const float lnu_real = norm, lnu_bin = logf((float)M) + norm;

  for (int pair = group; pair < a.B; pair += ngroups) {
    PairView pv{a.S + (long long)pair * a.strideS, a.lds, cache, r0, cached, M, N, C, a.alpha};
    float* u = a.u + (long long)pair * R;
    float* acc = a.acc + (long long)pair * 3 * C;
    float* fbm = a.fb + (long long)pair * 2 * C;     // exact fallback: max keys
    float* fbs = fbm + C;                            // exact fallback: sums
    unsigned* fbk = reinterpret_cast<unsigned*>(fbm);

    // ---- stage the band (with the dustbin border) in shared memory
    __syncthreads();
    for (int r = r0; r < r0 + cached; ++r) {
      const float* src = pv.S + (long long)r * pv.lds;
      for (int j = tid; j < C; j += NT)
        cache[(r - r0) * C + j] = (r < M && j < N) ? __ldg(src + j) : a.alpha;
    }
    for (int r = r0 + tid; r < r1; r += NT) u[r] = 0.f;
    __syncthreads();

    float v[CPT], lnu[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int j = tid + c * NT;
      v[c] = 0.f;
      lnu[c] = j < N ? lnu_real : lnu_bin;
    }

    bool failed = false;
    for (int it = 0; it < a.iters && !failed; ++it) {
      // ------------------------------------------------ row pass (local)
      float colacc[CPT];
#pragma unroll
      for (int c = 0; c < CPT; ++c) colacc[c] = 0.f;
      for (int rc = r0; rc < r1; rc += RB) {
        float e[RB][CPT];
        float m[RB], s[RB];
        bool exact = (it == 0);
#pragma unroll
        for (int k = 0; k < RB; ++k) {
          const int r = rc + k;
          const float lmu = r < M ? lmu_real : lmu_bin;
          m[k] = (r < r1 && !exact) ? lmu - u[r] : 0.f;
        }
        while (true) {
          if (exact) {
#pragma unroll
            for (int k = 0; k < RB; ++k) {
              float mx = -INFINITY;
              const int r = rc + k;
#pragma unroll
              for (int c = 0; c < CPT; ++c) {
                const int j = tid + c * NT;
                if (r < r1 && j < C) mx = fmaxf(mx, pv.z(r, j) + v[c]);
              }
              m[k] = mx;
            }
            block_max<RB>(m, SG_REDF());
          }
#pragma unroll
          for (int k = 0; k < RB; ++k) {
            const int r = rc + k;
            float part = 0.f;
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
              const int j = tid + c * NT;
              float x = 0.f;
              if (r < r1 && j < C) x = ex2((pv.z(r, j) + v[c] - m[k]) * kLog2e);
              e[k][c] = x;
              part += x;
            }
            s[k] = part;
          }
          block_sum<RB>(s, SG_REDF());
          if (exact) break;
          bool bad = false;       // block-uniform: s[] is the same in every thread
#pragma unroll
          for (int k = 0; k < RB; ++k)
            if (rc + k < r1 && !(s[k] >= kRowTiny && s[k] < INFINITY)) bad = true;
          if (!bad) break;
          exact = true;
        }
#pragma unroll
        for (int k = 0; k < RB; ++k) {
          const int r = rc + k;
          if (r >= r1) break;
          const float lmu = r < M ? lmu_real : lmu_bin;
          const float lsum = lg2(s[k]) * kLn2;
          const float ratio = ex2((lmu - lsum) * kLog2e);   // mu_r / rowsum_r
          if (tid == k) u[r] = lmu - m[k] - lsum;
#pragma unroll
          for (int c = 0; c < CPT; ++c) colacc[c] = fmaf(e[k][c], ratio, colacc[c]);
        }
      }
      // ------------------------------------------------ column pass (group)
      float* acc_now = acc + (it % 3) * C;
      float* acc_zero = acc + ((it + 1) % 3) * C;   // last read two barriers ago
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        const int j = tid + c * NT;
        if (j < C) atomicAdd(acc_now + j, colacc[c]);
      }
      for (int j = rank * NT + tid; j < C; j += cpp * NT) acc_zero[j] = 0.f;
      ++gen;
      if (group_barrier(counter, gen * cpp, a.abort_flag, a.status, a.timeout_ns)) { failed = true; break; }
      float cm[CPT];
      bool bad = false;
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        const int j = tid + c * NT;
        cm[c] = 1.f;
        if (j < C) {
          cm[c] = __ldcg(acc_now + j);
          if (!(cm[c] >= kColTiny && cm[c] < INFINITY)) bad = true;
        }
      }
      if (!__syncthreads_or(bad)) {
#pragma unroll
        for (int c = 0; c < CPT; ++c) v[c] += lnu[c] - lg2(cm[c]) * kLn2;
      } else {
        // exact column LSE: true column max, then the shifted sum
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
          const int j = tid + c * NT;
          if (j >= C) continue;
          float mx = -INFINITY;
          for (int r = r0; r < r1; ++r) mx = fmaxf(mx, pv.z(r, j) + u[r]);
          if (r1 > r0) atomicMax(fbk + j, f2key(mx));
        }
        ++gen;
        if (group_barrier(counter, gen * cpp, a.abort_flag, a.status, a.timeout_ns)) { failed = true; break; }
        float mxc[CPT];
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
          const int j = tid + c * NT;
          mxc[c] = 0.f;
          if (j >= C) continue;
          mxc[c] = key2f(__ldcg(fbk + j));
          float sum = 0.f;
          for (int r = r0; r < r1; ++r) sum += ex2((pv.z(r, j) + u[r] - mxc[c]) * kLog2e);
          atomicAdd(fbs + j, sum);
        }
        ++gen;
        if (group_barrier(counter, gen * cpp, a.abort_flag, a.status, a.timeout_ns)) { failed = true; break; }
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
          const int j = tid + c * NT;
          if (j < C) v[c] = lnu[c] - mxc[c] - lg2(__ldcg(fbs + j)) * kLn2;
        }
        ++gen;
        if (group_barrier(counter, gen * cpp, a.abort_flag, a.status, a.timeout_ns)) { failed = true; break; }
        for (int j = rank * NT + tid; j < C; j += cpp * NT) { fbk[j] = 0u; fbs[j] = 0.f; }
        ++gen;
        if (group_barrier(counter, gen * cpp, a.abort_flag, a.status, a.timeout_ns)) { failed = true; break; }
      }
    }
    if (failed) return;

    // ------------------------------------------------ output + extraction
    bool nonfinite = false;
#pragma unroll
    for (int c = 0; c < CPT; ++c) if (!isfinite(v[c])) nonfinite = true;
    float* lp = a.logP ? a.logP + (long long)pair * R * C : nullptr;
    unsigned long long colb[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) colb[c] = 0ull;
    for (int rc = r0; rc < r1; rc += RB) {
      unsigned long long best[RB];
#pragma unroll
      for (int k = 0; k < RB; ++k) {
        const int r = rc + k;
        best[k] = 0ull;
        if (r >= r1) continue;
        const float ur = u[r];
        if (!isfinite(ur)) nonfinite = true;
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
          const int j = tid + c * NT;
          if (j >= C) continue;
          const float val = ((pv.z(r, j) + ur) + v[c]) - norm;
          if (lp) lp[(long long)r * C + j] = val;
          if (r < M && j < N) {
            const unsigned long long kr =
                ((unsigned long long)f2key(val) << 32) | (0xffffffffu - (unsigned)j);
            best[k] = kr > best[k] ? kr : best[k];
            const unsigned long long kc =
                ((unsigned long long)f2key(val) << 32) | (0xffffffffu - (unsigned)r);
            colb[c] = kc > colb[c] ? kc : colb[c];
          }
        }
      }
      block_max_u64<RB>(best, SG_RED64());
      if (tid < RB && rc + tid < r1 && rc + tid < M) {
        const int r = rc + tid;
        unsigned long long b = 0ull;
#pragma unroll
        for (int k = 0; k < RB; ++k) if (k == tid) b = best[k];
        a.idx0[(long long)pair * M + r] = (int)(0xffffffffu - (unsigned)(b & 0xffffffffu));
        a.max0[(long long)pair * M + r] = key2f((unsigned)(b >> 32));
      }
    }
    unsigned long long* cb = a.colbest + (long long)pair * N;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int j = tid + c * NT;
      if (j < N && colb[c]) atomicMax(cb + j, colb[c]);
    }
    if (__syncthreads_or(nonfinite) && tid == 0 && rank == 0) atomicOr(a.status, kStatusNumeric);
    ++gen;
    if (group_barrier(counter, gen * cpp, a.abort_flag, a.status, a.timeout_ns)) return;
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
    // the next pair of this group re-stages shared memory and reuses nothing else
  }
#undef SG_REDF
#undef SG_RED64
}

template <int CPT, int RB>
cudaError_t launch_t(SinkhornArgs a, int num_sms, cudaStream_t s, int* launches) {
  auto kern = sinkhorn_kernel<CPT, RB>;
  const int C = a.N + 1, R = a.M + 1;
  const size_t red_bytes = 2 * RB * NW * sizeof(unsigned long long);
  const size_t max_smem = 220 * 1024;
  // Grid: one CTA per SM (co-residency is checked by the cooperative launch).
  int occ = 0;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)max_smem);
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, NT, max_smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  const int G = num_sms;
  // CTAs per pair: enough to keep a pair's Z on chip if possible, and all of
  // them when the whole batch fits at once.
  const size_t row_bytes = (size_t)C * sizeof(float);
  const size_t rows_per_cta_fit = (max_smem - red_bytes - 16) / row_bytes;
  int cpp;
  if (rows_per_cta_fit == 0) {
    cpp = G;
  } else {
    const long long need = (R + (long long)rows_per_cta_fit - 1) / (long long)rows_per_cta_fit;
    if ((long long)a.B * need <= G) cpp = G / a.B;
    else if (need <= G) cpp = (int)need;
    else cpp = G;
  }
  if (cpp < 1) cpp = 1;
  if (cpp > R) cpp = R;
  const int band = (R + cpp - 1) / cpp;
  a.cpp = cpp;
  a.cached_rows = (int)((size_t)band < rows_per_cta_fit ? (size_t)band : rows_per_cta_fit);
  const size_t smem = (((size_t)a.cached_rows * row_bytes + 15) & ~(size_t)15) + red_bytes;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
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

// A group of two CTAs of which only one is launched: its barrier can never
// complete, so it must end by its time limit, latch the timeout and return.
__global__ void barrier_selftest_kernel(unsigned* counter, unsigned* abort_flag, unsigned* status,
                                        unsigned long long timeout_ns, int* returned) {
  const bool failed = group_barrier(counter, 2u, abort_flag, status, timeout_ns);
  if (threadIdx.x == 0) *returned = failed ? 1 : 2;
}

}  // namespace

cudaError_t launch_barrier_selftest(unsigned* scratch, unsigned* status, unsigned long long timeout_ns,
                                    int* returned, cudaStream_t s) {
  barrier_selftest_kernel<<<1, 32, 0, s>>>(scratch, scratch + 1, status, timeout_ns, returned);
  return cudaGetLastError();
}

// Scratch layout (floats unless noted), zero-initialised part first:
//   barrier[B] + abort (uint), acc[B][3][C], fb[B][2][C], colbest[B][N] (u64),
//   then u[B][R], idx0[B][M], max0[B][M].
size_t sinkhorn_scratch_bytes(int B, int M, int N) {
  const size_t C = N + 1, R = M + 1;
  size_t z = (B + 1) * sizeof(unsigned);
  z = (z + 255) & ~(size_t)255;
  z += (size_t)B * 3 * C * 4 + (size_t)B * 2 * C * 4;
  z = (z + 255) & ~(size_t)255;
  z += (size_t)B * N * 8;
  z = (z + 255) & ~(size_t)255;
  size_t nz = (size_t)B * R * 4 + (size_t)B * M * 4 * 2 + 3 * 256;
  return z + nz;
}

cudaError_t launch_sinkhorn(SinkhornArgs a, int num_sms, cudaStream_t s, int* launches) {
  const int C = a.N + 1;
  if (C <= NT) return launch_t<1, 16>(a, num_sms, s, launches);
  if (C <= 2 * NT) return launch_t<2, 16>(a, num_sms, s, launches);
  if (C <= 4 * NT) return launch_t<4, 8>(a, num_sms, s, launches);
  if (C <= 8 * NT) return launch_t<8, 4>(a, num_sms, s, launches);
  if (C <= 16 * NT) return launch_t<16, 2>(a, num_sms, s, launches);
  if (C <= 32 * NT) return launch_t<32, 1>(a, num_sms, s, launches);
  return cudaErrorInvalidValue;
}

}  // namespace sg
