// CUDA-core multi-head attention (the float32 path), flash-style.
//
// Per head: alpha_ij = softmax_j(q_i . k_j / sqrt(d_head)), m_i = sum_j alpha_ij v_j
// ("SuperGlue 的注意力图神经网络怎样传递信息", section Attention 让节点自己选择消息来源;
// realcat notes, section Attentional Aggregation).  Self stages read keys/values
// of the query's own image, cross stages those of the other image; one launch
// serves all four directions of a stage (A<-A and B<-B, or A<-B and B<-A).
//
// One thread owns one query row (q and the running output in registers); a CTA
// of 128 queries walks the source image in key tiles of 32 staged in shared
// memory.  The softmax is online: per tile, the running max is raised once and
// the accumulated output rescaled once.
#include "sg_internal.cuh"

namespace sg {
namespace {

constexpr int QT = 128;   // queries per CTA
constexpr int KT = 32;    // keys per tile

template <typename T> __device__ __forceinline__ float ld1(const T* p);
template <> __device__ __forceinline__ float ld1<float>(const float* p) { return *p; }
template <> __device__ __forceinline__ float ld1<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ void st1(T* p, float v);
template <> __device__ __forceinline__ void st1<float>(float* p, float v) { *p = v; }
template <> __device__ __forceinline__ void st1<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <typename T>
__global__ void __launch_bounds__(QT) attn_simt_kernel(AttnArgs a) {
  __shared__ float Ks[KT][kDh];
  __shared__ float Vs[KT][kDh];
  // adaptive depth: the exit flag of an earlier kernel of the pass ends the work
  if (a.skip != nullptr && *reinterpret_cast<const volatile unsigned*>(a.skip) != 0u) return;
  const int P = a.M + a.N;
  const int pair = blockIdx.z >> 1;
  const int img = blockIdx.z & 1;
  const int h = blockIdx.y;
  const int nq = img ? a.N : a.M;
  const int src = a.cross ? 1 - img : img;
  const int nk = src ? a.N : a.M;
  const int q0 = blockIdx.x * QT;
  if (q0 >= nq) return;
  const T* qkv = reinterpret_cast<const T*>(a.qkv);
  const long long qbase = (long long)pair * P + (img ? a.M : 0);
  const long long kbase = (long long)pair * P + (src ? a.M : 0);
  const int qi = q0 + threadIdx.x;
  const bool active = qi < nq;

  float q[kDh], o[kDh];
  if (active) {
    const T* qp = qkv + (qbase + qi) * kQKV + h * kDh;
#pragma unroll
    for (int d = 0; d < kDh; ++d) q[d] = ld1<T>(qp + d) * a.scale_log2;
  } else {
#pragma unroll
    for (int d = 0; d < kDh; ++d) q[d] = 0.f;
  }
#pragma unroll
  for (int d = 0; d < kDh; ++d) o[d] = 0.f;
  float m = -INFINITY, l = 0.f;

  for (int k0 = 0; k0 < nk; k0 += KT) {
    const int nt = min(KT, nk - k0);
    __syncthreads();
    for (int e = threadIdx.x; e < KT * kDh; e += QT) {
      const int j = e / kDh, d = e % kDh;
      float kv = 0.f, vv = 0.f;
      if (j < nt) {
        const T* kp = qkv + (kbase + k0 + j) * kQKV;
        kv = ld1<T>(kp + kD + h * kDh + d);
        vv = ld1<T>(kp + 2 * kD + h * kDh + d);
      }
      Ks[j][d] = kv;
      Vs[j][d] = vv;
    }
    __syncthreads();
    float s[KT];
    float tmax = -INFINITY;
#pragma unroll
    for (int j = 0; j < KT; ++j) {
      float acc = 0.f;
#pragma unroll
      for (int d = 0; d < kDh; ++d) acc = fmaf(q[d], Ks[j][d], acc);
      s[j] = j < nt ? acc : -INFINITY;
      tmax = fmaxf(tmax, s[j]);
    }
    const float mnew = fmaxf(m, tmax);
    const float corr = fast_exp2(m - mnew);    // m = -inf on the first tile -> 0
    l *= corr;
#pragma unroll
    for (int d = 0; d < kDh; ++d) o[d] *= corr;
#pragma unroll
    for (int j = 0; j < KT; ++j) {
      const float p = fast_exp2(s[j] - mnew);
      l += p;
#pragma unroll
      for (int d = 0; d < kDh; ++d) o[d] = fmaf(p, Vs[j][d], o[d]);
    }
    m = mnew;
  }
  if (active) {
    const float inv = 1.f / l;
    T* mp = reinterpret_cast<T*>(a.msg) + (qbase + qi) * kD + h * kDh;
#pragma unroll
    for (int d = 0; d < kDh; ++d) st1<T>(mp + d, o[d] * inv);
  }
}

}  // namespace

cudaError_t launch_attention_simt(const AttnArgs& a, bool bf16, cudaStream_t s) {
  const int nmax = a.M > a.N ? a.M : a.N;
  if (a.B == 0 || nmax == 0) return cudaSuccess;
  dim3 grid((nmax + QT - 1) / QT, kH, 2 * a.B);
  if (bf16) attn_simt_kernel<__nv_bfloat16><<<grid, QT, 0, s>>>(a);
  else attn_simt_kernel<float><<<grid, QT, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sg
