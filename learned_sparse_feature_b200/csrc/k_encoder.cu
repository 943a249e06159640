// Keypoint encoder, fused: normalisation + MLP 3-32-64-128-256-256 (BatchNorm
// folded into the weights on the host) + descriptor add.
//
// x0_i = d_i + MLP_enc((x_i, y_i, c_i)) with the keypoint normalised as
// (p - (W/2, H/2)) / scale ("笔记：SuperGlue:Learning Feature Matching with
// Graph Neural Networks论文阅读", section 特征点Encode; "SuperGlue_Code_Learning /
// SuperGlue_model_forward_learning", normalize_keypoints).
//
// One CTA encodes kPts points of the stacked [A; B] rows of the batch.  The
// activations live in shared memory channel-major (act[c][p]) so that every
// weight read from L2 is reused kPts times and every activation read is a
// warp-wide broadcast.
#include "sg_internal.cuh"

namespace sg {
namespace {

constexpr int kPts = 32;
constexpr int kThreads = 256;

template <int IN, int OUT, bool RELU>
__device__ __forceinline__ void enc_layer(const float* Wt, const float* b,
                                          const float* act_in, float* act_out) {
  constexpr int groups = kThreads / OUT;       // thread groups sharing one output channel
  constexpr int ppt = kPts / groups;           // points per thread
  const int o = threadIdx.x % OUT;
  const int g = threadIdx.x / OUT;
  float acc[ppt];
  const float bo = b[o];
#pragma unroll
  for (int k = 0; k < ppt; ++k) acc[k] = bo;
#pragma unroll 4
  for (int i = 0; i < IN; ++i) {
    const float w = Wt[i * OUT + o];             // global (fused kernel) or shared (head kernel)
    const float* a = act_in + i * kPts + g;
#pragma unroll
    for (int k = 0; k < ppt; ++k) acc[k] = fmaf(w, a[k * groups], acc[k]);
  }
#pragma unroll
  for (int k = 0; k < ppt; ++k) {
    float v = acc[k];
    if (RELU) v = fmaxf(v, 0.f);
    act_out[o * kPts + g + k * groups] = v;
  }
}

__global__ void __launch_bounds__(kThreads) encoder_kernel(EncArgs a, int write_bf16) {
  extern __shared__ float sm[];
  float* bufA = sm;                  // up to 256 x kPts
  float* bufB = sm + kD * kPts;
  const int P = a.M + a.N;
  const long long total = (long long)a.B * P;
  const long long row0 = (long long)blockIdx.x * kPts;

  // normalised (x, y, c) for the tile, channel-major
  if (threadIdx.x < kPts) {
    const int p = threadIdx.x;
    const long long r = row0 + p;
    float x = 0.f, y = 0.f, c = 0.f;
    if (r < total) {
      const int b = (int)(r / P);
      const int i = (int)(r % P);
      const int img = i < a.M ? 0 : 1;
      const int n = img ? a.N : a.M;
      const int li = img ? i - a.M : i;
      const long long pi = (long long)b * n + li;
      x = (a.kpts[img][2 * pi] - a.cx) * a.inv_scale;
      y = (a.kpts[img][2 * pi + 1] - a.cy) * a.inv_scale;
      c = a.conf[img][pi];
    }
    bufA[0 * kPts + p] = x;
    bufA[1 * kPts + p] = y;
    bufA[2 * kPts + p] = c;
  }
  __syncthreads();
  enc_layer<3, 32, true>(a.W[0], a.b[0], bufA, bufB);
  __syncthreads();
  enc_layer<32, 64, true>(a.W[1], a.b[1], bufB, bufA);
  __syncthreads();
  enc_layer<64, 128, true>(a.W[2], a.b[2], bufA, bufB);
  __syncthreads();
  enc_layer<128, 256, true>(a.W[3], a.b[3], bufB, bufA);
  __syncthreads();
  enc_layer<256, 256, false>(a.W[4], a.b[4], bufA, bufB);
  __syncthreads();

  // x = d + enc(p); thread o writes channel o of every point (coalesced rows)
  const int o = threadIdx.x;
  for (int p = 0; p < kPts; ++p) {
    const long long r = row0 + p;
    if (r >= total) break;
    const int b = (int)(r / P);
    const int i = (int)(r % P);
    const int img = i < a.M ? 0 : 1;
    const int n = img ? a.N : a.M;
    const int li = img ? i - a.M : i;
    const float d = a.desc[img][((long long)b * n + li) * kD + o];
    const float x = d + bufB[o * kPts + p];
    a.x32[r * kD + o] = x;
    if (write_bf16) a.x16[r * kD + o] = __float2bfloat16_rn(x);
  }
}

// Encoder head for the bf16 path: layers 3-32-64-128 (folded BN + ReLU) from
// weights staged in shared memory, h2 written as bf16 (points x 128) for the
// tensor-core GEMMs of layers 128-256 and 256-256, and x = d written into the
// stacked residual stream (the last GEMM adds MLP_enc(p) to it).
__global__ void __launch_bounds__(kThreads) encoder_head_kernel(EncArgs a, __nv_bfloat16* h2) {
  extern __shared__ float sm[];
  float* bufA = sm;                    // up to 128 x kPts activations
  float* bufB = sm + 128 * kPts;
  float* w0 = bufB + 128 * kPts;       // 3 x 32, 32 x 64, 64 x 128 (in x out) and biases
  float* w1 = w0 + 3 * 32;
  float* w2 = w1 + 32 * 64;
  float* bb = w2 + 64 * 128;           // 32 + 64 + 128 biases
  for (int i = threadIdx.x; i < 3 * 32; i += kThreads) w0[i] = a.W[0][i];
  for (int i = threadIdx.x; i < 32 * 64; i += kThreads) w1[i] = a.W[1][i];
  for (int i = threadIdx.x; i < 64 * 128; i += kThreads) w2[i] = a.W[2][i];
  for (int i = threadIdx.x; i < 32; i += kThreads) bb[i] = a.b[0][i];
  for (int i = threadIdx.x; i < 64; i += kThreads) bb[32 + i] = a.b[1][i];
  for (int i = threadIdx.x; i < 128; i += kThreads) bb[96 + i] = a.b[2][i];
  const int P = a.M + a.N;
  const long long total = (long long)a.B * P;
  const long long row0 = (long long)blockIdx.x * kPts;
  if (threadIdx.x < kPts) {
    const int p = threadIdx.x;
    const long long r = row0 + p;
    float x = 0.f, y = 0.f, c = 0.f;
    if (r < total) {
      const int b = (int)(r / P);
      const int i = (int)(r % P);
      const int img = i < a.M ? 0 : 1;
      const int n = img ? a.N : a.M;
      const int li = img ? i - a.M : i;
      const long long pi = (long long)b * n + li;
      x = (a.kpts[img][2 * pi] - a.cx) * a.inv_scale;
      y = (a.kpts[img][2 * pi + 1] - a.cy) * a.inv_scale;
      c = a.conf[img][pi];
    }
    bufA[0 * kPts + p] = x;
    bufA[1 * kPts + p] = y;
    bufA[2 * kPts + p] = c;
  }
  __syncthreads();
  enc_layer<3, 32, true>(w0, bb, bufA, bufB);
  __syncthreads();
  enc_layer<32, 64, true>(w1, bb + 32, bufB, bufA);
  __syncthreads();
  enc_layer<64, 128, true>(w2, bb + 96, bufA, bufB);
  __syncthreads();
  // h2 rows (bf16) and the descriptor copy, both coalesced along channels
  for (int e = threadIdx.x; e < kPts * 128; e += kThreads) {
    const int p = e / 128, o = e % 128;
    const long long r = row0 + p;
    if (r < total) h2[r * 128 + o] = __float2bfloat16_rn(bufB[o * kPts + p]);
  }
  for (int p = 0; p < kPts; ++p) {
    const long long r = row0 + p;
    if (r >= total) break;
    const int b = (int)(r / P);
    const int i = (int)(r % P);
    const int img = i < a.M ? 0 : 1;
    const int n = img ? a.N : a.M;
    const int li = img ? i - a.M : i;
    const float* d = a.desc[img] + ((long long)b * n + li) * kD;
    a.x32[r * kD + threadIdx.x] = d[threadIdx.x];
  }
}

}  // namespace

cudaError_t launch_encoder_head(const EncArgs& a, __nv_bfloat16* h2, cudaStream_t s) {
  const long long total = (long long)a.B * (a.M + a.N);
  if (total == 0) return cudaSuccess;
  const int grid = (int)((total + kPts - 1) / kPts);
  const size_t smem = (2 * 128 * kPts + 3 * 32 + 32 * 64 + 64 * 128 + 32 + 64 + 128) * sizeof(float);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(encoder_head_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  encoder_head_kernel<<<grid, kThreads, smem, s>>>(a, h2);
  return cudaGetLastError();
}

cudaError_t launch_encoder(const EncArgs& a, bool write_bf16, cudaStream_t s) {
  const long long total = (long long)a.B * (a.M + a.N);
  if (total == 0) return cudaSuccess;
  const int grid = (int)((total + kPts - 1) / kPts);
  const size_t smem = 2 * kD * kPts * sizeof(float);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(encoder_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  encoder_kernel<<<grid, kThreads, smem, s>>>(a, write_bf16 ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace sg
