// Adaptive depth: the exit decision after a (self, cross) layer of the GNN.
//
// After layer l (all but the last), every point i of every pair gets a
// confidence c_i = sigmoid(w_l . x_i + b_l) from the fp32 residual stream; the
// pass stops when the share of points whose confidence is not below
// lambda_l = clip(0.8 + 0.1 exp(-4 l / L), 0, 1) exceeds depth_confidence
// ("论文解读:LightGlue,让稀疏特征匹配随难度自适应地快", section 2.6 自适应深度,
// confidence_threshold / check_if_stop).  One decision covers the whole batch:
// the share is taken over all B (M + N) points.
//
// One launch per checked layer: warps take rows (one 256-wide dot product per
// row, eight values per lane), blocks add their count of low-confidence points
// to the layer's counter, and the last block to finish (a finished-block
// counter) takes the decision and sets the stop word that every later GNN
// kernel of the pass reads.  Nothing waits on another block.  Launched with
// programmatic dependent launch; griddepcontrol.wait gates the read of x.
#include "sg_internal.cuh"

#include <cmath>

namespace sg {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads) depth_check_kernel(const float* __restrict__ x32, int rows,
                                                               const float* __restrict__ w, float b,
                                                               float lambda, float depth_conf, int layer,
                                                               unsigned* words) {
  pdl_wait();
  volatile unsigned* stop = words;
  if (*stop != 0u) return;                        // an earlier layer already stopped the pass
  unsigned* low = words + 2 + layer;
  unsigned* done = words + 2 + 16 + layer;
  __shared__ unsigned s_low[kWarps];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // this lane's eight weights: columns 4 lane .. 4 lane + 3 and 128 + the same
  const float4 w0 = reinterpret_cast<const float4*>(w)[lane];
  const float4 w1 = reinterpret_cast<const float4*>(w)[32 + lane];
  unsigned cnt = 0;
  for (int r = blockIdx.x * kWarps + warp; r < rows; r += gridDim.x * kWarps) {
    const float4* xr = reinterpret_cast<const float4*>(x32 + (long long)r * 256);
    const float4 a0 = xr[lane], a1 = xr[32 + lane];
    float z = a0.x * w0.x + a0.y * w0.y + a0.z * w0.z + a0.w * w0.w +
              a1.x * w1.x + a1.y * w1.y + a1.z * w1.z + a1.w * w1.w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    z += b;
    // sigmoid without overflow for large |z|
    const float e = expf(-fabsf(z));
    const float c = z >= 0.f ? 1.f / (1.f + e) : e / (1.f + e);
    cnt += (c < lambda) ? 1u : 0u;                 // the same value in every lane
  }
  if (lane == 0) s_low[warp] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned blk = 0;
    for (int i = 0; i < kWarps; ++i) blk += s_low[i];
    if (blk) atomicAdd(low, blk);
    __threadfence();                               // the count is visible before this block is
    const unsigned prev = atomicAdd(done, 1u);     // counted as finished
    if (prev == gridDim.x - 1) {
      __threadfence();
      const unsigned lowv = *reinterpret_cast<volatile unsigned*>(low);
      const double ratio = 1.0 - (double)lowv / (double)rows;
      if (ratio > (double)depth_conf) {
        words[1] = (unsigned)(layer + 1);
        __threadfence();
        *stop = 1u;
      }
    }
  }
}

}  // namespace

cudaError_t launch_depth_check(const float* x32, int rows, const float* w, float b, float lambda,
                               float depth_conf, int layer, unsigned* words, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (layer < 0 || layer >= 16) return cudaErrorInvalidValue;
  int blocks = (rows + kWarps - 1) / kWarps;
  if (blocks > 148 * 4) blocks = 148 * 4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = s;
  cudaLaunchAttribute la[1];
  la[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap with the previous kernel
  la[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = la;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, depth_check_kernel, x32, rows, w, b, lambda, depth_conf, layer, words);
}

}  // namespace sg
