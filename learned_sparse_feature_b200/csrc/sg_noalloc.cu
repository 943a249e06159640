// sg_optimal_transport_static: the transport + extraction step for callers that
// cannot allocate device memory (an allocator-less runtime, a plugin whose host
// owns every allocation, or code that runs after memory has been reserved up
// front).  It needs no handle and calls no cudaMalloc/cudaFree: its scratch
// lives in the file-scope device array below, which every GPU that loads the
// library holds until the process exits.
#include "sg_internal.cuh"

#include <cmath>

namespace {

// Scratch of every call: barrier counters, column accumulators, fallback
// buffers, per-column argmax keys and per-row argmax.  4 MiB covers, e.g.,
// B = 8 pairs of 4096 x 3072 or B = 32 pairs of 1024 x 1024.
constexpr size_t kStaticScratchBytes = 4u << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};   // device address of g_static_scratch, per device

}  // namespace

extern "C" sg_status_t sg_optimal_transport_static(int B, int M, int N, const float* scores,
                                                   float bin_score, int sinkhorn_iters,
                                                   float match_threshold, float* out_logP,
                                                   int32_t* matches0, int32_t* matches1,
                                                   float* mscores0, float* mscores1,
                                                   unsigned* status, void* stream) {
  if (B < 0 || M < 0 || N < 0 || sinkhorn_iters < 0) return SG_ERR_INVALID_ARG;
  if (B == 0) return SG_OK;
  if (M == 0 || N == 0) return SG_ERR_SHAPE;
  if (!scores || !matches0 || !matches1 || !mscores0 || !mscores1 || !status) return SG_ERR_INVALID_ARG;
  if (N > sg::sinkhorn_max_columns()) return SG_ERR_SHAPE;
  const size_t need = sg::sinkhorn_scratch_bytes(B, M, N);
  if (need > kStaticScratchBytes) return SG_ERR_SHAPE;   // more scratch than the static array holds

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SG_ERR_UNSUPPORTED;
  if (!g_scratch_addr[dev]) {
    // one-time set-up on this device (not capturable: make this first call
    // before any stream capture)
    if (sg::sinkhorn_prepare(0) != cudaSuccess) return SG_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return SG_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  int num_sms = 0;
  if (cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return SG_ERR_CUDA;

  // the same layout as the handle's scratch (see run_transport in sg_api.cu)
  cudaStream_t s = (cudaStream_t)stream;
  unsigned char* p = static_cast<unsigned char*>(g_scratch_addr[dev]);
  const size_t C = (size_t)N + 1, R = (size_t)M + 1;
  sg::SinkhornArgs a{};
  a.barrier = reinterpret_cast<unsigned*>(p);
  a.abort_flag = a.barrier + B;
  size_t off = ((size_t)(B + 1) * sizeof(unsigned) + 255) & ~(size_t)255;
  a.acc = reinterpret_cast<float*>(p + off);
  a.fb = a.acc + (size_t)B * 3 * sg::sinkhorn_acc_floats_per_buffer(N);
  off += (size_t)B * 5 * sg::sinkhorn_acc_floats_per_buffer(N) * 4;
  off = (off + 255) & ~(size_t)255;
  a.colbest = reinterpret_cast<unsigned long long*>(p + off);
  off += (size_t)B * N * 8;
  off = (off + 255) & ~(size_t)255;
  const size_t zero_bytes = off;   // what must start at zero: counters, accumulators, argmax keys
  a.u = reinterpret_cast<float*>(p + off);
  off += (size_t)B * R * 4;
  off = (off + 255) & ~(size_t)255;
  a.idx0 = reinterpret_cast<int32_t*>(p + off);
  off += (size_t)B * M * 4;
  off = (off + 255) & ~(size_t)255;
  a.max0 = reinterpret_cast<float*>(p + off);
  (void)C;
  if (cudaMemsetAsync(p, 0, zero_bytes, s) != cudaSuccess) return SG_ERR_CUDA;
  a.S = scores;
  a.lds = N;
  a.strideS = (long long)M * N;
  a.lds_vec = (N % 4 == 0) && ((reinterpret_cast<uintptr_t>(scores) & 15) == 0);
  a.alpha = bin_score;
  a.B = B; a.M = M; a.N = N; a.iters = sinkhorn_iters;
  a.threshold = match_threshold;
  a.logP = out_logP;
  a.matches0 = matches0; a.matches1 = matches1; a.mscores0 = mscores0; a.mscores1 = mscores1;
  a.status = status;
  a.timeout_ns = 1000000000ull;
  if (sg::launch_sinkhorn(a, num_sms, s, nullptr) != cudaSuccess) return SG_ERR_CUDA;
  return SG_OK;
}
