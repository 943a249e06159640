// Internal declarations shared by the libsg translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/sg.h"

namespace sg {

constexpr int kD = 256;        // state width
constexpr int kH = 4;          // heads
constexpr int kDh = 64;        // head width
constexpr int kQKV = 3 * kD;   // fused q|k|v row width

// Device status word bits (latched by kernels, read by sg_status).
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusNumeric = 2u;
constexpr unsigned kStatusPipeline = 4u;   // a tcgen05 pipeline wait ran out

// ------------------------------------------------------------------ GEMM epilogues
enum Epilogue : int {
  EPI_BIAS = 0,        // out = acc + bias
  EPI_BIAS_RELU = 1,   // out = max(acc + bias, 0)
  EPI_RESIDUAL = 2,    // x32 += acc; x16 = bf16(x32)   (out = x32, out2 = x16)
  EPI_SCALE = 3,       // out = acc * scale               (score matrix)
};

// C[r, c] = sum_k A[r, k] * W[c, k], A row-major (lda), W row-major (ldw = K).
// The A operand may be split along K: columns [0, k_split) come from A0 and
// [k_split, K) from A1 (both row-major with lda).  Batched over blockIdx.z with
// element strides for A0/A1, W and out.
struct GemmArgs {
  const void* A0;
  const void* A1;
  long long lda;
  int k_split;
  const void* W;
  const float* bias;
  void* out;
  void* out2;
  long long ldo;
  int rows, cols, K;
  long long strideA, strideW, strideO;
  float scale;
  int w_dynamic;   // W is written by an earlier kernel of the pass (the score GEMM's f_B), not a weight
  const unsigned* skip;   // adaptive depth: when *skip != 0 (set by an earlier kernel) the launch does nothing
};

// Attention over the stacked state of B pairs: rows [b*P, b*P+M) are image A of
// pair b, [b*P+M, (b+1)*P) image B.  qkv row = q|k|v (each D wide, head h at
// [h*64, h*64+64)).  Self: A<-A, B<-B; cross: A<-B, B<-A.  msg row: D wide.
struct AttnArgs {
  const void* qkv;
  void* msg;
  int B, M, N;
  int cross;
  float scale_log2;   // log2(e) / sqrt(d_head)
  int exp_emu;        // tensor-core path: of every 8 exp2 pairs, how many use the FMA pipe (0, 2, 3 or 4)
  float blind_limit;  // tensor-core path: bound on a key tile's sum of 2^(s - m) before the row's max is renewed
  const unsigned* skip;   // adaptive depth: when *skip != 0 (set by an earlier kernel) the launch does nothing
};

struct EncArgs {
  const float* kpts[2];
  const float* conf[2];
  const float* desc[2];
  const float* W[5];   // transposed (in x out), BN folded
  const float* b[5];
  float* x32;
  __nv_bfloat16* x16;  // may be null
  int B, M, N;
  float cx, cy, inv_scale;
};

struct SinkhornArgs {
  const float* S;       // B x M x lds (real block only)
  long long lds;
  long long strideS;    // elements between pairs
  float alpha;
  int B, M, N, iters;
  float threshold;
  float* logP;          // B x (M+1) x (N+1) or null
  int32_t* matches0;
  int32_t* matches1;
  float* mscores0;
  float* mscores1;
  // scratch (zeroed before the launch)
  float* u;             // B x (M+1)
  float* v;             // B x (N+1)
  float* acc;           // B x 3 x (N+1)
  float* fb;            // B x 2 x (N+1): exact-fallback max (as ordered uint) and sum
  unsigned long long* colbest;   // B x N
  int32_t* idx0;        // B x M
  float* max0;          // B x M
  unsigned* barrier;    // one counter per group
  unsigned* abort_flag;
  unsigned* status;
  int cpp;              // CTAs per pair group (set by the launcher)
  int band_alloc;       // rows per CTA band (set by the launcher)
  int lds_vec;          // S rows are 16-byte aligned (vector loads allowed)
  int cached_rows;      // rows of the band kept in shared memory
  unsigned long long timeout_ns;   // limit of every grid-barrier wait
};

// ------------------------------------------------------------------ launchers
cudaError_t launch_encoder(const EncArgs& a, bool write_bf16, cudaStream_t s);
// bf16 path: layers 0-2 -> h2 (points x 128, bf16) and x32 = descriptors
cudaError_t launch_encoder_head(const EncArgs& a, __nv_bfloat16* h2, cudaStream_t s);
cudaError_t launch_gemm_simt(const GemmArgs& g, int epi, bool in_bf16, bool out_bf16,
                             int batch, cudaStream_t s);
cudaError_t launch_attention_simt(const AttnArgs& a, bool bf16, cudaStream_t s);
cudaError_t launch_sinkhorn(SinkhornArgs a, int num_sms, cudaStream_t s, int* launches);
cudaError_t sinkhorn_prepare(int num_sms);   // kernel attributes (called once, outside capture)
int sinkhorn_max_columns();                  // largest N the transport kernel supports
size_t sinkhorn_scratch_bytes(int B, int M, int N);
size_t sinkhorn_acc_floats_per_buffer(int N);   // column accumulator floats per (pair, rotation)
// Adaptive depth (k_depth.cu): after layer `layer`, count the points of the
// rows x 256 fp32 states x32 whose confidence sigmoid(w . x + b) is below
// lambda; the last block to finish sets words[0] = 1 (stop) and words[1] =
// layer + 1 when 1 - low / rows > depth_conf.  words: [stop, layers run,
// low count per layer (16), finished blocks per layer (16)], zeroed per pass.
// Does nothing when words[0] is already set.
constexpr int kDepthWords = 2 + 2 * 16;
cudaError_t launch_depth_check(const float* x32, int rows, const float* w, float b, float lambda,
                               float depth_conf, int layer, unsigned* words, cudaStream_t s);

// Double-softmax matching head (k_dsm.cu).
size_t dsm_scratch_bytes(int B, int M, int N);
cudaError_t launch_dsm_matchability(const float* x32, int B, int M, int N, const float* wz, float bz, float* z0,
                                    float* z1, cudaStream_t s);
cudaError_t launch_dsm_assign(const float* S, long long lds, long long strideS, int B, int M, int N,
                              const float* z0, const float* z1, float threshold, float* logP, int32_t* matches0,
                              int32_t* matches1, float* mscores0, float* mscores1, void* scratch, cudaStream_t s,
                              int* launches);
cudaError_t launch_exp2_poly_selftest(const float* x, float* y, int n, cudaStream_t s);
cudaError_t launch_barrier_selftest(unsigned* scratch, unsigned* status, unsigned long long timeout_ns,
                                    int* returned, cudaStream_t s);

// tcgen05 paths (sm_100a)
// status: device status word; a pipeline wait that runs out sets a bit in it.
cudaError_t launch_gemm_tc(const GemmArgs& g, int epi, int batch, cudaStream_t s, unsigned* status);
cudaError_t launch_attention_tc(const AttnArgs& a, cudaStream_t s, unsigned* status);
bool tc_available();

}  // namespace sg
