// Double-softmax matching head: the closed-form assignment that replaces the
// dustbin and the Sinkhorn iterations ("论文解读:LightGlue,让稀疏特征匹配随难度自适应地快",
// section 2.4 匹配头:把「相似」和「可匹配」拆开):
//
//   log P_ij = log_softmax_j(sim_i.)_j + log_softmax_i(sim_.j)_i
//              + log sigmoid(z0_i) + log sigmoid(z1_j)            (real block)
//   log P_iN = log sigmoid(-z0_i),  log P_Mj = log sigmoid(-z1_j),  log P_MN = 0,
//
// with z = matchability(x) = x . wz + bz on the final GNN states, followed by the
// same mutual-argmax extraction as the Sinkhorn head.
//
// Everything here streams the similarity matrix from L2 (it was just written by
// the score GEMM and fits there at these sizes), on the CUDA cores:
//   dsm_matchability   z0, z1 from the fp32 residual stream (warp per row);
//   dsm_row_lse        log sum_j exp(sim_ij) (warp per row, online max/sum);
//   dsm_col_partial    per 128-row chunk and column: online (max, sum) partials;
//   dsm_col_final      the column log-sum-exp from the partials;
//   dsm_rows           log P rows, the last column, and the row argmax;
//   dsm_col_argmax     per chunk and column: the best (value, row) key, merged
//                      into the column's key with one 64-bit atomicMax;
//   dsm_extract        mutual check, exp(max) scores, strict threshold.
// The value of an entry is formed by one device function in the row pass and
// the column pass alike, so both argmaxes see bit-identical values.
#include "sg_internal.cuh"

#include <cmath>

namespace sg {
namespace {

constexpr int kChunk = 128;      // rows per column-partial block

__device__ __forceinline__ float log_sigmoid(float x) {
  return fminf(x, 0.f) - log1pf(expf(-fabsf(x)));
}

// One entry of the real block, from its parts (the same expression everywhere).
__device__ __forceinline__ float dsm_value(float s, float row_lse, float col_lse, float ls0, float ls1) {
  return ((s - row_lse) + (s - col_lse)) + (ls0 + ls1);
}

__device__ __forceinline__ unsigned f2key(float f) {
  const unsigned u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key2f(unsigned k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// (m, s) online log-sum-exp state: s = sum exp(x - m); m = -inf means empty.
__device__ __forceinline__ void lse_push(float& m, float& s, float x) {
  if (x > m) {
    s = s * expf(m - x) + 1.f;   // expf(-inf) = 0 when the state was empty
    m = x;
  } else {
    s += expf(x - m);
  }
}
__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) { m = m2; s = s2; return; }
  if (m2 > m) {
    s = s * expf(m - m2) + s2;
    m = m2;
  } else {
    s += s2 * expf(m2 - m);
  }
}

__global__ void dsm_matchability(const float* x32, int B, int M, int N, const float* wz, float bz, float* z0,
                                 float* z1) {
  const int P = M + N;
  const long long r = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (r >= (long long)B * P) return;
  const float* row = x32 + r * kD;
  float acc = 0.f;
  for (int c = lane; c < kD; c += 32) acc = fmaf(row[c], wz[c], acc);
#pragma unroll
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    const int b = (int)(r / P), i = (int)(r % P);
    if (i < M) z0[(long long)b * M + i] = acc + bz;
    else z1[(long long)b * N + (i - M)] = acc + bz;
  }
}

__global__ void dsm_row_lse(const float* S, long long lds, long long strideS, int B, int M, int N, float* row_lse) {
  const long long w = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (w >= (long long)B * M) return;
  const int b = (int)(w / M), i = (int)(w % M);
  const float* row = S + b * strideS + (long long)i * lds;
  float m = -INFINITY, s = 0.f;
  for (int j = lane; j < N; j += 32) lse_push(m, s, row[j]);
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    lse_merge(m, s, m2, s2);
  }
  if (lane == 0) row_lse[w] = m + logf(s);
}

// grid (ceil(N / 128), ceil(M / kChunk), B), block 128: thread = column
__global__ void dsm_col_partial(const float* S, long long lds, long long strideS, int M, int N, float2* part) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  const int c = blockIdx.y, b = blockIdx.z;
  if (j >= N) return;
  const int i0 = c * kChunk, i1 = min(M, i0 + kChunk);
  const float* col = S + b * strideS + j;
  float m = -INFINITY, s = 0.f;
  for (int i = i0; i < i1; ++i) lse_push(m, s, col[(long long)i * lds]);
  part[((long long)b * gridDim.y + c) * N + j] = make_float2(m, s);
}

__global__ void dsm_col_final(const float2* part, int nchunk, int B, int N, float* col_lse) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)B * N) return;
  const int b = (int)(t / N), j = (int)(t % N);
  float m = -INFINITY, s = 0.f;
  for (int c = 0; c < nchunk; ++c) {
    const float2 p = part[((long long)b * nchunk + c) * N + j];
    lse_merge(m, s, p.x, p.y);
  }
  col_lse[t] = m + logf(s);
}

// warp per row: log P of the row (if requested), its last column, row argmax
__global__ void dsm_rows(const float* S, long long lds, long long strideS, int B, int M, int N,
                         const float* row_lse, const float* col_lse, const float* z0, const float* z1,
                         float* logP, int32_t* idx0, float* max0) {
  const long long w = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (w >= (long long)B * M) return;
  const int b = (int)(w / M), i = (int)(w % M);
  const float* row = S + b * strideS + (long long)i * lds;
  const float rl = row_lse[w];
  const float ls0 = log_sigmoid(z0[w]);
  const float* cl = col_lse + (long long)b * N;
  const float* zz1 = z1 + (long long)b * N;
  float* out = logP ? logP + (long long)b * (M + 1) * (N + 1) + (long long)i * (N + 1) : nullptr;
  unsigned long long best = 0ull;
  for (int j = lane; j < N; j += 32) {
    const float v = dsm_value(row[j], rl, cl[j], ls0, log_sigmoid(zz1[j]));
    if (out) out[j] = v;
    const unsigned long long k = ((unsigned long long)f2key(v) << 32) | (0xffffffffu - (unsigned)j);
    best = k > best ? k : best;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const unsigned long long y = __shfl_xor_sync(0xffffffffu, best, o);
    best = y > best ? y : best;
  }
  if (lane == 0) {
    if (out) out[N] = log_sigmoid(-z0[w]);
    idx0[w] = (int)(0xffffffffu - (unsigned)(best & 0xffffffffu));
    max0[w] = key2f((unsigned)(best >> 32));
  }
}

// grid (ceil(N / 128), ceil(M / kChunk), B), block 128: thread = column; the
// chunk's best (value, row) key of the column goes into colbest[b][j]; chunk 0
// also writes the last row of log P (and the corner)
__global__ void dsm_col_argmax(const float* S, long long lds, long long strideS, int M, int N,
                               const float* row_lse, const float* col_lse, const float* z0, const float* z1,
                               unsigned long long* colbest, float* logP) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  const int c = blockIdx.y, b = blockIdx.z;
  if (j >= N) return;
  const int i0 = c * kChunk, i1 = min(M, i0 + kChunk);
  const float* col = S + b * strideS + j;
  const float cl = col_lse[(long long)b * N + j];
  const float ls1 = log_sigmoid(z1[(long long)b * N + j]);
  const float* rl = row_lse + (long long)b * M;
  const float* zz0 = z0 + (long long)b * M;
  unsigned long long best = 0ull;
  for (int i = i0; i < i1; ++i) {
    const float v = dsm_value(col[(long long)i * lds], rl[i], cl, log_sigmoid(zz0[i]), ls1);
    const unsigned long long k = ((unsigned long long)f2key(v) << 32) | (0xffffffffu - (unsigned)i);
    best = k > best ? k : best;
  }
  atomicMax(colbest + (long long)b * N + j, best);
  if (c == 0 && logP) {
    float* last = logP + (long long)b * (M + 1) * (N + 1) + (long long)M * (N + 1);
    last[j] = log_sigmoid(-z1[(long long)b * N + j]);
    if (j == 0) last[N] = 0.f;
  }
}

// thread per row (first B*M threads) and per column (next B*N threads)
__global__ void dsm_extract(int B, int M, int N, const int32_t* idx0, const float* max0,
                            const unsigned long long* colbest, float threshold, int32_t* matches0,
                            int32_t* matches1, float* mscores0, float* mscores1) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nr = (long long)B * M;
  if (t < nr) {
    const int b = (int)(t / M), i = (int)(t % M);
    const int j = idx0[t];
    const unsigned long long k = colbest[(long long)b * N + j];
    const bool mutual = (int)(0xffffffffu - (unsigned)(k & 0xffffffffu)) == i;
    const float ms = mutual ? expf(max0[t]) : 0.f;
    matches0[t] = (mutual && ms > threshold) ? j : -1;
    mscores0[t] = ms;
  } else if (t < nr + (long long)B * N) {
    const long long u = t - nr;
    const int b = (int)(u / N), j = (int)(u % N);
    const unsigned long long k = colbest[u];
    const int i = (int)(0xffffffffu - (unsigned)(k & 0xffffffffu));
    const bool iok = k != 0ull && i >= 0 && i < M;
    const long long ri = (long long)b * M + i;
    const bool mutual = iok && idx0[ri] == j;
    const float ms = mutual ? expf(max0[ri]) : 0.f;
    matches1[u] = (mutual && ms > threshold) ? i : -1;
    mscores1[u] = ms;
  }
}

}  // namespace

size_t dsm_scratch_bytes(int B, int M, int N) {
  const size_t nchunk = (size_t)(M + kChunk - 1) / kChunk;
  size_t z = 0;
  auto take = [&](size_t bytes) { z = (z + 255) & ~(size_t)255; z += bytes; };
  take((size_t)B * N * 8);                 // colbest (zeroed per call)
  take((size_t)B * M * 4);                 // row log-sum-exp
  take((size_t)B * N * 4);                 // column log-sum-exp
  take((size_t)B * nchunk * N * 8);        // column partials
  take((size_t)B * M * 4);                 // idx0
  take((size_t)B * M * 4);                 // max0
  return (z + 255) & ~(size_t)255;
}

cudaError_t launch_dsm_matchability(const float* x32, int B, int M, int N, const float* wz, float bz, float* z0,
                                    float* z1, cudaStream_t s) {
  const long long rows = (long long)B * (M + N);
  if (rows == 0) return cudaSuccess;
  dsm_matchability<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(x32, B, M, N, wz, bz, z0, z1);
  return cudaGetLastError();
}

cudaError_t launch_dsm_assign(const float* S, long long lds, long long strideS, int B, int M, int N,
                              const float* z0, const float* z1, float threshold, float* logP, int32_t* matches0,
                              int32_t* matches1, float* mscores0, float* mscores1, void* scratch, cudaStream_t s,
                              int* launches) {
  if (B == 0 || M == 0 || N == 0) return cudaSuccess;
  const int nchunk = (M + kChunk - 1) / kChunk;
  unsigned char* p = static_cast<unsigned char*>(scratch);
  size_t off = 0;
  auto take = [&](size_t bytes) -> unsigned char* {
    off = (off + 255) & ~(size_t)255;
    unsigned char* q = p + off;
    off += bytes;
    return q;
  };
  auto* colbest = reinterpret_cast<unsigned long long*>(take((size_t)B * N * 8));
  auto* row_lse = reinterpret_cast<float*>(take((size_t)B * M * 4));
  auto* col_lse = reinterpret_cast<float*>(take((size_t)B * N * 4));
  auto* part = reinterpret_cast<float2*>(take((size_t)B * nchunk * N * 8));
  auto* idx0 = reinterpret_cast<int32_t*>(take((size_t)B * M * 4));
  auto* max0 = reinterpret_cast<float*>(take((size_t)B * M * 4));
  cudaError_t e = cudaMemsetAsync(colbest, 0, (size_t)B * N * 8, s);
  if (e != cudaSuccess) return e;
  const long long rows = (long long)B * M;
  const dim3 cgrid((N + 127) / 128, nchunk, B);
  dsm_row_lse<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(S, lds, strideS, B, M, N, row_lse);
  dsm_col_partial<<<cgrid, 128, 0, s>>>(S, lds, strideS, M, N, part);
  dsm_col_final<<<(unsigned)(((long long)B * N + 255) / 256), 256, 0, s>>>(part, nchunk, B, N, col_lse);
  dsm_rows<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(S, lds, strideS, B, M, N, row_lse, col_lse, z0, z1, logP,
                                                     idx0, max0);
  dsm_col_argmax<<<cgrid, 128, 0, s>>>(S, lds, strideS, M, N, row_lse, col_lse, z0, z1, colbest, logP);
  const long long all = (long long)B * (M + N);
  dsm_extract<<<(unsigned)((all + 255) / 256), 256, 0, s>>>(B, M, N, idx0, max0, colbest, threshold, matches0,
                                                            matches1, mscores0, mscores1);
  if (launches) *launches += 6;
  return cudaGetLastError();
}

}  // namespace sg
