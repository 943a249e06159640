// CUDA-core GEMM with fused epilogues: the float32 path of every linear layer
// (kernel-size-1 Conv1d) of the matcher and its score matrix.
//
// C[r, c] = sum_k A[r, k] W[c, k]: the 64 x 64 output tile of a CTA is staged
// through shared memory in K-steps of 16; each of the 256 threads owns a 4 x 4
// block of outputs.  A may be split along K into two sources (the update MLP
// reads [x || message] without materialising the concatenation, realcat notes
// "笔记：SuperGlue:Learning Feature Matching with Graph Neural Networks论文阅读",
// section 多层GNN).
#include "sg_internal.cuh"

namespace sg {
namespace {

constexpr int BM = 64, BN = 64, BK = 16, TH = 256;

template <typename T> __device__ __forceinline__ void load4(const T* p, float* o);
template <> __device__ __forceinline__ void load4<float>(const float* p, float* o) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
template <> __device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, float* o) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&v.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&v.y);
  const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  o[0] = fa.x; o[1] = fa.y; o[2] = fb.x; o[3] = fb.y;
}

template <typename T> __device__ __forceinline__ void store1(T* p, float v);
template <> __device__ __forceinline__ void store1<float>(float* p, float v) { *p = v; }
template <> __device__ __forceinline__ void store1<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

template <typename TI, typename TO, int EPI>
__global__ void __launch_bounds__(TH) gemm_simt_kernel(GemmArgs g) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Ws[BK][BN + 4];
  // adaptive depth: the exit flag of an earlier kernel of the pass ends the work
  if (g.skip != nullptr && *reinterpret_cast<const volatile unsigned*>(g.skip) != 0u) return;
  const int bz = blockIdx.z;
  const TI* A0 = reinterpret_cast<const TI*>(g.A0) + bz * g.strideA;
  const TI* A1 = g.A1 ? reinterpret_cast<const TI*>(g.A1) + bz * g.strideA : nullptr;
  const TI* W = reinterpret_cast<const TI*>(g.W) + bz * g.strideW;
  const int row0 = blockIdx.y * BM;
  const int col0 = blockIdx.x * BN;
  const int tid = threadIdx.x;
  const int tr = tid / 16, tc = tid % 16;        // 16 x 16 threads, 4 x 4 outputs each
  // loader mapping: 64 rows x 16 k = 256 x 4 elements
  const int lr = tid / 4, lk = (tid % 4) * 4;

  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.K; k0 += BK) {
    float a4[4] = {0.f, 0.f, 0.f, 0.f}, w4[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int r = row0 + lr;
      const int k = k0 + lk;
      if (r < g.rows) {
        if (k < g.k_split) load4<TI>(A0 + (long long)r * g.lda + k, a4);
        else load4<TI>(A1 + (long long)r * g.lda + (k - g.k_split), a4);
      }
      const int c = col0 + lr;
      if (c < g.cols) load4<TI>(W + (long long)c * g.K + k, w4);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      As[lk + j][lr] = a4[j];
      Ws[lk + j][lr] = w4[j];
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      const float4 av = *reinterpret_cast<const float4*>(&As[kk][tr * 4]);
      const float4 wv = *reinterpret_cast<const float4*>(&Ws[kk][tc * 4]);
      const float ar[4] = {av.x, av.y, av.z, av.w};
      const float wr[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ar[i], wr[j], acc[i][j]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = row0 + tr * 4 + i;
    if (r >= g.rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = col0 + tc * 4 + j;
      if (c >= g.cols) continue;
      const long long o = bz * g.strideO + (long long)r * g.ldo + c;
      float v = acc[i][j];
      if (EPI == EPI_BIAS || EPI == EPI_BIAS_RELU) {
        v += g.bias[c];
        if (EPI == EPI_BIAS_RELU) v = fmaxf(v, 0.f);
        store1<TO>(reinterpret_cast<TO*>(g.out) + o, v);
      } else if (EPI == EPI_RESIDUAL) {
        float* x32 = reinterpret_cast<float*>(g.out);
        const float x = x32[o] + v;
        x32[o] = x;
        if (g.out2) store1<__nv_bfloat16>(reinterpret_cast<__nv_bfloat16*>(g.out2) + o, x);
      } else {
        store1<TO>(reinterpret_cast<TO*>(g.out) + o, v * g.scale);
      }
    }
  }
}

template <typename TI, typename TO>
cudaError_t dispatch(const GemmArgs& g, int epi, int batch, cudaStream_t s) {
  dim3 grid((g.cols + BN - 1) / BN, (g.rows + BM - 1) / BM, batch);
  switch (epi) {
    case EPI_BIAS: gemm_simt_kernel<TI, TO, EPI_BIAS><<<grid, TH, 0, s>>>(g); break;
    case EPI_BIAS_RELU: gemm_simt_kernel<TI, TO, EPI_BIAS_RELU><<<grid, TH, 0, s>>>(g); break;
    case EPI_RESIDUAL: gemm_simt_kernel<TI, TO, EPI_RESIDUAL><<<grid, TH, 0, s>>>(g); break;
    default: gemm_simt_kernel<TI, TO, EPI_SCALE><<<grid, TH, 0, s>>>(g); break;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_simt(const GemmArgs& g, int epi, bool in_bf16, bool out_bf16, int batch,
                             cudaStream_t s) {
  if (g.rows <= 0 || g.cols <= 0 || batch <= 0) return cudaSuccess;
  if (in_bf16) {
    return out_bf16 ? dispatch<__nv_bfloat16, __nv_bfloat16>(g, epi, batch, s)
                    : dispatch<__nv_bfloat16, float>(g, epi, batch, s);
  }
  return out_bf16 ? dispatch<float, __nv_bfloat16>(g, epi, batch, s)
                  : dispatch<float, float>(g, epi, batch, s);
}

}  // namespace sg
