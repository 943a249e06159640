// tcgen05 GEMM with fused epilogues: every linear layer of the bf16 path (q|k|v
// projection, the two update-MLP layers with folded BatchNorm + ReLU and the
// residual add, the final projection) and the batched score matrix
// S = <f_A, f_B> / sqrt(D) ("笔记：SuperGlue:Learning Feature Matching with Graph
// Neural Networks论文阅读", sections 多层GNN and 匹配得分预测).
//
// C[128 x BN tile] = A[rows x K] * W[cols x K]^T, both operands K-major bf16.
// A persistent CTA of 6 warps loops over output tiles:
//   warp 0 (one lane)  TMA producer: 128x64 A and BNx64 W tiles per K-block,
//                      128-byte swizzle, STAGES-deep ring of shared buffers;
//   warp 1 (one lane)  MMA issuer: 4 x tcgen05.mma (K = 16 each) per K-block into
//                      one of two 128 x BN fp32 accumulators in TMEM;
//                      tcgen05.commit frees the stage / publishes the tile;
//   warps 2-5          epilogue: tcgen05.ld of the thread's accumulator row (TMEM
//                      lane = tile row), bias / ReLU / residual / scale, store,
//                      while the MMA warp already fills the other accumulator.
// Launched with programmatic dependent launch: the prologue (barriers, TMEM,
// descriptor prefetch) overlaps the previous kernel; griddepcontrol.wait gates
// the first read of its outputs.
// The A operand may come from two tensors split along K (the update MLP reads
// [x || message] without materialising the concatenation).
#include "sg_internal.cuh"
#include "tc_common.cuh"

#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

namespace sg {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;                   // one 128-byte swizzle atom of bf16
constexpr int kThreads = 192;                // producer, MMA, 4 epilogue warps
constexpr unsigned kErrGemmWait = 4u;    // status bit: a GEMM pipeline wait ran out

struct TcArgs {
  int rows, cols, K, k_split, batch;
  int a_batch_rows;      // row offset between batches in the A tensor
  int b_batch_rows;      // row offset between batches in the W tensor
  int b_row0;            // first W row of batch 0
  const float* bias;
  void* out;
  void* out2;
  long long ldo;
  long long strideO;
  float scale;
  unsigned* status;
};

template <int BN, int STAGES>
struct Smem {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BYTES = STAGES * STAGE_BYTES + 1024;   // + alignment slack
};

template <int BN> __host__ __device__ constexpr uint32_t tmem_cols() {
  return BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
}

// Barrier of the 128 epilogue threads (named barrier 1) that also returns the
// AND of their predicates.
__device__ __forceinline__ bool epi_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Persistent: CTA c computes output tiles c, c + gridDim.x, ...; tiles are
// ordered (batch, row tile, column tile) with the column tile fastest so
// consecutive CTAs share the A tile in L2.  The accumulator is double-buffered
// in TMEM: the epilogue warps drain tile i while the MMA warp accumulates tile
// i + 1.
template <int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
               const __grid_constant__ CUtensorMap tmB, TcArgs g) {
  using SM = Smem<BN, STAGES>;
  constexpr uint32_t BNA = tmem_cols<BN>();      // TMEM columns of one accumulator buffer
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(16) float s_bias[2][BN];   // bias of the tile, by accumulator buffer
  __shared__ uint32_t tmem_slot;
  __shared__ int s_abort;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t base = (tc::smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - tc::smem_u32(smem_raw));

  const int ntn = (g.cols + BN - 1) / BN;
  const int ntm = (g.rows + BM - 1) / BM;
  const int ntiles = ntn * ntm * g.batch;
  const int nkb = g.K / BK;
  const int nkb0 = g.k_split / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&full_bar[s], 1);
      tc::mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&tfull_bar[b], 1);
      tc::mbar_init(&tempty_bar[b], 4);          // one arrival per epilogue warp
    }
    tc::fence_barrier_init();
    s_abort = 0;
  }
  if (warp == 1) tc::tmem_alloc(&tmem_slot, 2 * BNA);
  if (threadIdx.x == 64) {
    tc::prefetch_tmap(&tmA0);
    tc::prefetch_tmap(&tmA1);
    tc::prefetch_tmap(&tmB);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  pdl_wait();                                    // the previous kernel's outputs are complete

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int it = 0;
      for (int t = blockIdx.x; t < ntiles && !s_abort; t += gridDim.x) {
        const int tn = t % ntn, tm = (t / ntn) % ntm, bz = t / (ntn * ntm);
        const int a_row = bz * g.a_batch_rows + tm * BM;
        const int b_row = g.b_row0 + bz * g.b_batch_rows + tn * BN;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % STAGES;
          const int round = it / STAGES;
          if (round > 0 && !tc::mbar_wait(&empty_bar[s], (round - 1) & 1, g.status, kErrGemmWait)) {
            s_abort = 1;
            break;
          }
          uint8_t* sa = sbase + s * SM::STAGE_BYTES;
          uint8_t* sb = sa + SM::A_BYTES;
          tc::mbar_arrive_expect_tx(&full_bar[s], SM::STAGE_BYTES);
          if (kb < nkb0) tc::tma_load_2d(&tmA0, &full_bar[s], sa, kb * BK, a_row);
          else tc::tma_load_2d(&tmA1, &full_bar[s], sa, (kb - nkb0) * BK, a_row);
          tc::tma_load_2d(&tmB, &full_bar[s], sb, kb * BK, b_row);
        }
      }
      // drain: copies in flight must land before the CTA may exit
      for (int k = (it > STAGES ? it - STAGES : 0); k < it; ++k)
        tc::mbar_wait(&full_bar[k % STAGES], (k / STAGES) & 1, g.status, kErrGemmWait);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc = tc::idesc_bf16_f32(BM, BN);
      int it = 0, i = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++i) {
        const int b = i & 1;
        if (i >= 2 && !tc::mbar_wait(&tempty_bar[b], ((i >> 1) - 1) & 1, g.status, kErrGemmWait)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t acc = tmem + b * BNA;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % STAGES;
          if (!tc::mbar_wait(&full_bar[s], (it / STAGES) & 1, g.status, kErrGemmWait)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t sa = base + s * SM::STAGE_BYTES;
          const uint32_t sb = sa + SM::A_BYTES;
          const uint64_t da = tc::sdesc_k_sw128(sa);
          const uint64_t db = tc::sdesc_k_sw128(sb);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)     // +32 B along K inside the swizzle atom
            tc::umma_bf16(acc, da + 2 * kk, db + 2 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          tc::umma_commit(&empty_bar[s]);
        }
        if (!ok) break;
        tc::umma_commit(&tfull_bar[b]);
      }
      pdl_trigger();                             // no more tensor work: the next kernel may start
      if (!ok) {
        s_abort = 1;
        // release epilogue warps that wait for accumulators that will not come
        tc::mbar_arrive(&tfull_bar[0]);
        tc::mbar_arrive(&tfull_bar[1]);
      }
    }
  } else {
    // ---------------- epilogue warps 2..5: TMEM lane quarter = warp % 4
    // While the MMA warp accumulates a tile, these warps stage its bias in
    // shared memory and start the loads of its first residual chunk, so that no
    // global-memory latency sits between the accumulator and the stores.
    const int q = warp & 3;
    const int et = threadIdx.x - 64;             // 0..127
    int i = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
      const int b = i & 1;
      const int tn = t % ntn, tm = (t / ntn) % ntm, bz = t / (ntn * ntm);
      const int n0 = tn * BN;
      const int row = tm * BM + q * 32 + lane;
      const bool row_ok = row < g.rows;
      const long long rbase = (long long)bz * g.strideO + (long long)row * g.ldo + n0;
      if (EPI == EPI_BIAS || EPI == EPI_BIAS_RELU) {
        for (int c = et; c < BN; c += 128) s_bias[b][c] = (n0 + c < g.cols) ? __ldg(g.bias + n0 + c) : 0.f;
      }
      float4 rnext[8];
      const bool vec_res = EPI == EPI_RESIDUAL && n0 + BN <= g.cols;   // full-width tile: float4 path
      if (EPI == EPI_RESIDUAL && vec_res && row_ok) {
        const float4* x4 = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(g.out) + rbase);
#pragma unroll
        for (int k = 0; k < 8; ++k) rnext[k] = __ldcg(x4 + k);
      }
      const bool got = tc::mbar_wait(&tfull_bar[b], (i >> 1) & 1, g.status, kErrGemmWait);
      // one barrier of the 128 epilogue threads per tile: publishes the staged
      // bias and makes the go / stop decision the same for all of them
      if (!epi_all(got && !s_abort)) break;
      tc::tc_fence_after();
      const uint32_t trow = tmem + b * BNA + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        float v[32];
        tc::tmem_ld32(trow + c0, v);             // warp-collective: every lane takes part
        float4 rcur[8];
        if (EPI == EPI_RESIDUAL && vec_res) {
#pragma unroll
          for (int k = 0; k < 8; ++k) rcur[k] = rnext[k];
          if (c0 + 32 < BN && row_ok) {
            const float4* x4 = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(g.out) + rbase + c0 + 32);
#pragma unroll
            for (int k = 0; k < 8; ++k) rnext[k] = __ldcg(x4 + k);
          }
        }
        if (!row_ok || n0 + c0 >= g.cols) continue;
        const long long obase = rbase + c0;
        const int ncol = min(32, g.cols - (n0 + c0));
        if (EPI == EPI_BIAS || EPI == EPI_BIAS_RELU) {
          __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(g.out) + obase;
          const float* sbv = s_bias[b] + c0;
          if (ncol == 32) {
            uint4 pk[4];
            uint32_t* p = reinterpret_cast<uint32_t*>(pk);
            const float4* b4 = reinterpret_cast<const float4*>(sbv);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float4 bb = b4[k];
              float x0 = v[4 * k] + bb.x, x1 = v[4 * k + 1] + bb.y, x2 = v[4 * k + 2] + bb.z, x3 = v[4 * k + 3] + bb.w;
              if (EPI == EPI_BIAS_RELU) {
                x0 = fmaxf(x0, 0.f); x1 = fmaxf(x1, 0.f); x2 = fmaxf(x2, 0.f); x3 = fmaxf(x3, 0.f);
              }
              p[2 * k] = tc::pack_bf16x2(x0, x1);
              p[2 * k + 1] = tc::pack_bf16x2(x2, x3);
            }
            uint4* o4 = reinterpret_cast<uint4*>(o);
#pragma unroll
            for (int k = 0; k < 4; ++k) o4[k] = pk[k];
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) {           // static indices keep v in registers
              if (k < ncol) {
                float x = v[k] + sbv[k];
                if (EPI == EPI_BIAS_RELU) x = fmaxf(x, 0.f);
                o[k] = __float2bfloat16_rn(x);
              }
            }
          }
        } else if (EPI == EPI_RESIDUAL) {
          float* x = reinterpret_cast<float*>(g.out) + obase;
          __nv_bfloat16* xb = reinterpret_cast<__nv_bfloat16*>(g.out2) + obase;
          if (vec_res) {
            float4* x4 = reinterpret_cast<float4*>(x);
            uint4 pk[4];
            uint32_t* p = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              float4 r = rcur[k];
              r.x += v[4 * k]; r.y += v[4 * k + 1]; r.z += v[4 * k + 2]; r.w += v[4 * k + 3];
              x4[k] = r;
              p[2 * k] = tc::pack_bf16x2(r.x, r.y);
              p[2 * k + 1] = tc::pack_bf16x2(r.z, r.w);
            }
            uint4* o4 = reinterpret_cast<uint4*>(xb);
#pragma unroll
            for (int k = 0; k < 4; ++k) o4[k] = pk[k];
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              if (k < ncol) {
                const float r = x[k] + v[k];
                x[k] = r;
                xb[k] = __float2bfloat16_rn(r);
              }
            }
          }
        } else {
          float* o = reinterpret_cast<float*>(g.out) + obase;
          if (ncol == 32 && (g.ldo % 4) == 0 && (g.strideO % 4) == 0) {
            float4* o4 = reinterpret_cast<float4*>(o);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              o4[k] = make_float4(v[4 * k] * g.scale, v[4 * k + 1] * g.scale, v[4 * k + 2] * g.scale,
                                  v[4 * k + 3] * g.scale);
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (k < ncol) o[k] = v[k] * g.scale;
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&tempty_bar[b]);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, 2 * BNA);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

// Row-major bf16 matrix [rows x cols] (row stride ld elements), boxes of
// box_rows x 64 with the 128-byte swizzle.
bool make_bf16_map(CUtensorMap* m, const void* ptr, long long rows, long long cols, long long ld, int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

int num_sms_cached() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

template <int BN, int STAGES, int EPI>
cudaError_t launch_t(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b, const TcArgs& t,
                     int grid, cudaStream_t s) {
  auto kern = gemm_tc_kernel<BN, STAGES, EPI>;
  constexpr int smem = Smem<BN, STAGES>::BYTES;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute la[1];
  la[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap with the previous kernel
  la[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = la;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a0, a1, b, t);
}

template <int BN, int STAGES>
cudaError_t launch_epi(int epi, const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                       const TcArgs& t, int grid, cudaStream_t s) {
  switch (epi) {
    case EPI_BIAS: return launch_t<BN, STAGES, EPI_BIAS>(a0, a1, b, t, grid, s);
    case EPI_BIAS_RELU: return launch_t<BN, STAGES, EPI_BIAS_RELU>(a0, a1, b, t, grid, s);
    case EPI_RESIDUAL: return launch_t<BN, STAGES, EPI_RESIDUAL>(a0, a1, b, t, grid, s);
    default: return launch_t<BN, STAGES, EPI_SCALE>(a0, a1, b, t, grid, s);
  }
}

}  // namespace

bool tc_available() { return get_encode() != nullptr; }

// GemmArgs (shared with the CUDA-core path) -> tensor maps + tcgen05 launch.
// Requirements: K and k_split multiples of 64, lda/ldo multiples of 8 elements.
cudaError_t launch_gemm_tc(const GemmArgs& g, int epi, int batch, cudaStream_t s, unsigned* status) {
  if (g.rows <= 0 || g.cols <= 0 || batch <= 0) return cudaSuccess;
  if (g.K % BK || g.k_split % BK || g.lda % 8) return cudaErrorInvalidValue;
  // Column tile: fewest waves of (tile work + a fixed per-tile latency) over the
  // SMs; among ties the wider tile (A is read fewer times).
  const int nsm = num_sms_cached();
  const long long row_tiles = (long long)((g.rows + BM - 1) / BM) * batch;
  int BN = 64;
  double best = 1e300;
  const int cands[4] = {256, 192, 128, 64};
  for (int ci = 0; ci < 4; ++ci) {
    const int bn = cands[ci];
    if (bn != 64 && g.cols % bn != 0) continue;
    const long long tiles = row_tiles * ((g.cols + bn - 1) / bn);
    const double waves = std::ceil((double)tiles / nsm);
    const double cost = waves * (bn + 64.0);
    if (cost < best - 1e-9) { best = cost; BN = bn; }
  }
  // A rows: rows of one batch item live at strideA / lda rows apart
  const long long a_batch_rows = batch > 1 ? g.strideA / g.lda : 0;
  const long long b_batch_rows = batch > 1 ? g.strideW / g.K : 0;
  const long long a_total_rows = batch > 1 ? a_batch_rows * (batch - 1) + g.rows : g.rows;
  CUtensorMap a0, a1, b;
  if (!make_bf16_map(&a0, g.A0, a_total_rows, g.k_split, g.lda, BM)) return cudaErrorInvalidValue;
  if (g.A1) {
    if (!make_bf16_map(&a1, g.A1, a_total_rows, g.K - g.k_split, g.lda, BM)) return cudaErrorInvalidValue;
  } else {
    a1 = a0;
  }
  // For the batched score GEMM W is a row window of a taller matrix (f_B rows);
  // map the whole window of all batches.
  const long long b_total_rows = batch > 1 ? b_batch_rows * (batch - 1) + g.cols : g.cols;
  if (!make_bf16_map(&b, g.W, b_total_rows, g.K, g.K, BN)) return cudaErrorInvalidValue;
  TcArgs t{};
  t.rows = g.rows; t.cols = g.cols; t.K = g.K; t.k_split = g.k_split; t.batch = batch;
  t.a_batch_rows = (int)a_batch_rows;
  t.b_batch_rows = (int)b_batch_rows;
  t.b_row0 = 0;
  t.bias = g.bias; t.out = g.out; t.out2 = g.out2; t.ldo = g.ldo; t.strideO = g.strideO;
  t.scale = g.scale; t.status = status;
  const long long tiles = row_tiles * ((g.cols + BN - 1) / BN);
  const int grid = (int)(tiles < nsm ? tiles : nsm);
  switch (BN) {
    case 256: return launch_epi<256, 3>(epi, a0, a1, b, t, grid, s);
    case 192: return launch_epi<192, 4>(epi, a0, a1, b, t, grid, s);
    case 128: return launch_epi<128, 4>(epi, a0, a1, b, t, grid, s);
    default: return launch_epi<64, 6>(epi, a0, a1, b, t, grid, s);
  }
}


}  // namespace sg
