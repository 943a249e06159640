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
//                      lane = tile row), bias / ReLU / residual / scale, written as
//                      a 32 x 32 chunk into swizzled shared memory and stored by
//                      one TMA tensor store per chunk (double-buffered; the
//                      residual comes in by TMA tensor loads two chunks ahead),
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
constexpr int kEpiWarps = 8;                 // two per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps;    // producer, MMA, epilogue warps
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
  int b_const;           // W is constant (weights), not an output of an earlier kernel
  const unsigned* skip;  // adaptive depth: nothing to compute once *skip is set
};

// Epilogue staging of one epilogue warp: one buffer set, a 32-row chunk of the
// output (fp32 rows of 128 B or bf16 rows of 64 B) and, for the residual
// epilogue, its bf16 copy and the fp32 residual input.  The two warps of a lane
// quarter alternate chunks, so a quarter's chunks are double-buffered.  Offsets
// are multiples of 1024 B (the swizzle atoms of the TMA boxes).
template <int EPI>
struct EpiStage {
  static constexpr bool F32 = EPI == EPI_SCALE || EPI == EPI_RESIDUAL;
  static constexpr int OUT = F32 ? 4096 : 2048;
  static constexpr int OUT2 = EPI == EPI_RESIDUAL ? 2048 : 0;
  static constexpr int RES = EPI == EPI_RESIDUAL ? 4096 : 0;
  static constexpr int OUT2_OFF = OUT;
  static constexpr int RES_OFF = OUT + OUT2;
  static constexpr int BUF = OUT + OUT2 + RES;
  static constexpr int BYTES = kEpiWarps * BUF;
};

constexpr int kMaxDynSmem = 224 * 1024;

template <int BN, int EPI>
struct Smem {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // as many ring stages as fit next to the epilogue staging (at most 8)
  static constexpr int FIT = (kMaxDynSmem - EpiStage<EPI>::BYTES - 1024) / STAGE_BYTES;
  static constexpr int STAGES = FIT > 8 ? 8 : FIT;
  static constexpr int EPI_OFF = STAGES * STAGE_BYTES;
  static constexpr int BYTES = EPI_OFF + EpiStage<EPI>::BYTES + 1024;   // + alignment slack
  static_assert(STAGES >= 2, "shared memory");
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
      "bar.red.and.pred q, 1, 256, p;\n\t"
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
// i + 1.  SKIP: the launch reads the adaptive-depth exit flag (a separate
// instantiation, so the launches of a pass without adaptive depth run the
// kernel without any of it).
template <int BN, int EPI, bool SKIP>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
               const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmO,
               const __grid_constant__ CUtensorMap tmO2, TcArgs g) {
  using SM = Smem<BN, EPI>;
  using ES = EpiStage<EPI>;
  constexpr int STAGES = SM::STAGES;
  constexpr uint32_t BNA = tmem_cols<BN>();      // TMEM columns of one accumulator buffer
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t res_bar[kEpiWarps];   // residual chunk loads, per epilogue warp
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
      tc::mbar_init(&tempty_bar[b], kEpiWarps);  // one arrival per epilogue warp
    }
    for (int w = 0; w < kEpiWarps; ++w) tc::mbar_init(&res_bar[w], 1);
    tc::fence_barrier_init();
    s_abort = 0;
  }
  if (warp == 1) tc::tmem_alloc(&tmem_slot, 2 * BNA);
  if (threadIdx.x == 64) {
    tc::prefetch_tmap(&tmA0);
    tc::prefetch_tmap(&tmA1);
    tc::prefetch_tmap(&tmB);
    tc::prefetch_tmap(&tmO);
    if (EPI == EPI_RESIDUAL) tc::prefetch_tmap(&tmO2);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // tiles this launch computes: none once the adaptive-depth exit flag, written
  // by an earlier kernel of the pass, is set (every role reads it after its
  // griddepcontrol.wait, so all see the same value)
  int nt = ntiles;
  auto exit_set = [&]() { return *reinterpret_cast<const volatile unsigned*>(g.skip) != 0u; };
  // the previous kernel's outputs must be complete before they are read and
  // before this kernel's outputs overwrite anything it still reads; the
  // producer first fetches constant weight tiles, which need neither
  if (!(warp == 0 && lane == 0)) {
    pdl_wait();
    if constexpr (SKIP) {
      if (exit_set()) nt = 0;
    }
  }

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int pre = 0;                               // ring stages whose W tile is already in flight
      if (g.b_const && !SKIP && (int)blockIdx.x < ntiles) {
        const int t = blockIdx.x;
        const int tn = t % ntn, bz = t / (ntn * ntm);
        const int b_row = g.b_row0 + bz * g.b_batch_rows + tn * BN;
        pre = nkb < STAGES ? nkb : STAGES;
        for (int kb = 0; kb < pre; ++kb) {
          tc::mbar_arrive_expect_tx(&full_bar[kb], SM::STAGE_BYTES);
          tc::tma_load_2d(&tmB, &full_bar[kb], sbase + kb * SM::STAGE_BYTES + SM::A_BYTES, kb * BK, b_row);
        }
      }
      pdl_wait();
      if constexpr (SKIP) {
        if (exit_set()) nt = 0;
      }
      int it = 0;
      for (int t = blockIdx.x; t < nt && !s_abort; t += gridDim.x) {
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
          if (it >= pre) tc::mbar_arrive_expect_tx(&full_bar[s], SM::STAGE_BYTES);
          if (kb < nkb0) tc::tma_load_2d(&tmA0, &full_bar[s], sa, kb * BK, a_row);
          else tc::tma_load_2d(&tmA1, &full_bar[s], sa, (kb - nkb0) * BK, a_row);
          if (it >= pre) tc::tma_load_2d(&tmB, &full_bar[s], sb, kb * BK, b_row);
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
      for (int t = blockIdx.x; t < nt && ok; t += gridDim.x, ++i) {
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
    // ---------------- epilogue warps 2..9: TMEM lane quarter q = warp % 4;
    // the two warps of a quarter (hf = 0, 1) take alternate 32-column chunks.
    // While the MMA warp accumulates a tile, these warps stage its bias in
    // shared memory and (residual) start the TMA load of their first residual
    // chunk.  Thread = tile row 32q + lane.
    const int q = warp & 3;
    const int ew = warp - 2;                     // 0..7: staging slot
    const int hf = ew >> 2;                      // which chunks of the quarter
    const int et = threadIdx.x - 64;             // 0..255
    uint8_t* sbuf = sbase + SM::EPI_OFF + ew * ES::BUF;
    constexpr int NCH = BN / 32;                 // 32-column chunks per tile (even)
    constexpr int MYCH = NCH / 2;                // chunks of one warp per tile
    uint32_t res_par = 0;                        // residual barrier parity
    bool res_pend = false;                       // a residual load issued and not yet waited for
    int i = 0;
    for (int t = blockIdx.x; t < nt; t += gridDim.x, ++i) {
      const int b = i & 1;
      const int tn = t % ntn, tm = (t / ntn) % ntm, bz = t / (ntn * ntm);
      const int n0 = tn * BN;
      const int row0 = tm * BM + q * 32;         // first row of this warp's chunks
      if (EPI == EPI_BIAS || EPI == EPI_BIAS_RELU) {
        for (int c = et; c < BN; c += 32 * kEpiWarps)
          s_bias[b][c] = (n0 + c < g.cols) ? __ldg(g.bias + n0 + c) : 0.f;
      }
      if (EPI == EPI_RESIDUAL && lane == 0) {
        tc::mbar_arrive_expect_tx(&res_bar[ew], 4096);
        tc::tma_load_3d(&tmO, &res_bar[ew], sbuf + ES::RES_OFF, n0 + 32 * hf, row0, bz);
        res_pend = true;
      }
      const bool got = tc::mbar_wait(&tfull_bar[b], (i >> 1) & 1, g.status, kErrGemmWait);
      // one barrier of the epilogue threads per tile: publishes the staged bias
      // and makes the go / stop decision the same for all of them
      if (!epi_all(got && !s_abort)) break;
      tc::tc_fence_after();
      const uint32_t trow = tmem + b * BNA + ((uint32_t)(q * 32) << 16);
      bool ok = true;
      // the next chunk's accumulator columns arrive while a chunk is processed
      float va[32], vb[32];
      tc::tmem_ld32_async(trow + hf * 32, va);  // warp-collective: every lane takes part
#pragma unroll
      for (int k = 0; k < MYCH; ++k) {
        const int ci = hf + 2 * k;
        float (&v)[32] = (k & 1) ? vb : va;
        tc::tmem_wait_ld(v);
        if (k + 1 < MYCH) tc::tmem_ld32_async(trow + (ci + 2) * 32, (k & 1) ? va : vb);
        // the store issued from this buffer (this warp's previous chunk) must have read it
        if (lane == 0) tc::bulk_wait_read<0>();
        __syncwarp();
        if (EPI == EPI_BIAS || EPI == EPI_BIAS_RELU) {
          // bf16 row of 64 B, 64-byte swizzle: 16-byte chunk k at k ^ ((row >> 1) & 3)
          const float4* b4 = reinterpret_cast<const float4*>(s_bias[b] + ci * 32);
          uint8_t* rowp = sbuf + lane * 64;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            uint32_t pk[4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float4 bb4 = b4[2 * kk + h];
              float x0 = v[8 * kk + 4 * h] + bb4.x, x1 = v[8 * kk + 4 * h + 1] + bb4.y;
              float x2 = v[8 * kk + 4 * h + 2] + bb4.z, x3 = v[8 * kk + 4 * h + 3] + bb4.w;
              if (EPI == EPI_BIAS_RELU) {
                x0 = fmaxf(x0, 0.f); x1 = fmaxf(x1, 0.f); x2 = fmaxf(x2, 0.f); x3 = fmaxf(x3, 0.f);
              }
              pk[2 * h] = tc::pack_bf16x2(x0, x1);
              pk[2 * h + 1] = tc::pack_bf16x2(x2, x3);
            }
            *reinterpret_cast<uint4*>(rowp + ((kk ^ ((lane >> 1) & 3)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        } else if (EPI == EPI_SCALE) {
          // fp32 row of 128 B, 128-byte swizzle: 16-byte chunk k at k ^ (row & 7)
          uint8_t* rowp = sbuf + lane * 128;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            *reinterpret_cast<float4*>(rowp + ((kk ^ (lane & 7)) << 4)) =
                make_float4(v[4 * kk] * g.scale, v[4 * kk + 1] * g.scale, v[4 * kk + 2] * g.scale,
                            v[4 * kk + 3] * g.scale);
        } else {
          // residual: x (fp32) += acc, and its bf16 copy
          ok = tc::mbar_wait(&res_bar[ew], res_par, g.status, kErrGemmWait);
          res_par ^= 1u;
          res_pend = false;
          const uint8_t* rin = sbuf + ES::RES_OFF + lane * 128;
          uint8_t* rout = sbuf + lane * 128;
          uint8_t* rout2 = sbuf + ES::OUT2_OFF + lane * 64;
          uint32_t pk[16];
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int off = (kk ^ (lane & 7)) << 4;
            float4 r = *reinterpret_cast<const float4*>(rin + off);
            r.x += v[4 * kk]; r.y += v[4 * kk + 1]; r.z += v[4 * kk + 2]; r.w += v[4 * kk + 3];
            *reinterpret_cast<float4*>(rout + off) = r;
            pk[2 * kk] = tc::pack_bf16x2(r.x, r.y);
            pk[2 * kk + 1] = tc::pack_bf16x2(r.z, r.w);
          }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            *reinterpret_cast<uint4*>(rout2 + ((kk ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(pk[4 * kk], pk[4 * kk + 1], pk[4 * kk + 2], pk[4 * kk + 3]);
        }
        tc::fence_proxy_async_smem();           // generic writes -> async-proxy reads
        __syncwarp();
        if (lane == 0) {
          // (a box wholly past the last row or column stores nothing: skip it)
          if (row0 < g.rows && n0 + ci * 32 < g.cols) {
            tc::tma_store_3d(&tmO, sbuf, n0 + ci * 32, row0, bz);
            if (EPI == EPI_RESIDUAL) tc::tma_store_3d(&tmO2, sbuf + ES::OUT2_OFF, n0 + ci * 32, row0, bz);
          }
          tc::bulk_commit();
          if (EPI == EPI_RESIDUAL && k + 1 < MYCH) {
            // this warp's residual input is consumed: fetch its next chunk
            tc::mbar_arrive_expect_tx(&res_bar[ew], 4096);
            tc::tma_load_3d(&tmO, &res_bar[ew], sbuf + ES::RES_OFF, n0 + 32 * (ci + 2), row0, bz);
            res_pend = true;
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&tempty_bar[b]);
      if (!ok) s_abort = 1;
    }
    // stores must be complete and residual loads landed before the CTA exits
    // (a break above can leave a prefetched residual chunk in flight)
    if (lane == 0) {
      tc::bulk_wait_all();
      if (res_pend) tc::mbar_wait(&res_bar[ew], res_par, g.status, kErrGemmWait);
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

// Output tensor [batch][rows][cols] (row stride ld, batch stride sb elements)
// as 32 x 32 x 1 boxes: fp32 rows of 128 B with the 128-byte swizzle, bf16 rows
// of 64 B with the 64-byte swizzle (the layouts the epilogue writes).
bool make_out_map(CUtensorMap* m, void* ptr, bool f32, long long rows, long long cols, long long ld,
                  long long batch, long long sb) {
  auto enc = get_encode();
  if (!enc) return false;
  const long long es = f32 ? 4 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)batch};
  cuuint64_t strides[2] = {(cuuint64_t)(ld * es), (cuuint64_t)((batch > 1 ? sb : rows * ld) * es)};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ptr, dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, int EPI, bool SKIP>
cudaError_t launch_t(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b, const CUtensorMap& o,
                     const CUtensorMap& o2, const TcArgs& t, int grid, cudaStream_t s) {
  auto kern = gemm_tc_kernel<BN, EPI, SKIP>;
  constexpr int smem = Smem<BN, EPI>::BYTES;
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
  return cudaLaunchKernelEx(&cfg, kern, a0, a1, b, o, o2, t);
}

template <int BN, bool SKIP>
cudaError_t launch_epi(int epi, const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                       const CUtensorMap& o, const CUtensorMap& o2, const TcArgs& t, int grid, cudaStream_t s) {
  switch (epi) {
    case EPI_BIAS: return launch_t<BN, EPI_BIAS, SKIP>(a0, a1, b, o, o2, t, grid, s);
    case EPI_BIAS_RELU: return launch_t<BN, EPI_BIAS_RELU, SKIP>(a0, a1, b, o, o2, t, grid, s);
    case EPI_RESIDUAL: return launch_t<BN, EPI_RESIDUAL, SKIP>(a0, a1, b, o, o2, t, grid, s);
    default: return launch_t<BN, EPI_SCALE, SKIP>(a0, a1, b, o, o2, t, grid, s);
  }
}

template <int BN>
cudaError_t launch_bn(int epi, const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                      const CUtensorMap& o, const CUtensorMap& o2, const TcArgs& t, int grid, cudaStream_t s) {
  // the exit-flag instantiations only for launches that carry the flag
  return t.skip ? launch_epi<BN, true>(epi, a0, a1, b, o, o2, t, grid, s)
                : launch_epi<BN, false>(epi, a0, a1, b, o, o2, t, grid, s);
}

}  // namespace

bool tc_available() { return get_encode() != nullptr; }

// GemmArgs (shared with the CUDA-core path) -> tensor maps + tcgen05 launch.
// Requirements: K and k_split multiples of 64, lda/ldo multiples of 8 elements.
cudaError_t launch_gemm_tc(const GemmArgs& g, int epi, int batch, cudaStream_t s, unsigned* status) {
  if (g.rows <= 0 || g.cols <= 0 || batch <= 0) return cudaSuccess;
  if (g.K % BK || g.k_split % BK || g.lda % 8) return cudaErrorInvalidValue;
  // the output tensor maps need 16-byte row (and batch) strides
  const int align_elems = (epi == EPI_BIAS || epi == EPI_BIAS_RELU) ? 8 : 4;
  if (g.ldo % align_elems || (epi == EPI_RESIDUAL && g.ldo % 8)) return cudaErrorInvalidValue;
  if (batch > 1 && g.strideO % align_elems) return cudaErrorInvalidValue;
  // Column tile: fewest waves of (tile work + a fixed per-tile latency) over the
  // SMs; among ties the wider tile (A is read fewer times).  The residual
  // epilogue needs more staging, which leaves a 256-wide tile too few ring stages.
  const int nsm = num_sms_cached();
  const long long row_tiles = (long long)((g.rows + BM - 1) / BM) * batch;
  int BN = 64;
  double best = 1e300;
  const int cands[4] = {256, 192, 128, 64};
  for (int ci = 0; ci < 4; ++ci) {
    const int bn = cands[ci];
    if (bn != 64 && g.cols % bn != 0) continue;
    if (epi == EPI_RESIDUAL && bn > 128) continue;
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
  t.b_const = g.w_dynamic ? 0 : 1;
  t.skip = g.skip;
  // outputs: bf16 (bias epilogues), fp32 scores, fp32 residual stream + its bf16 copy
  CUtensorMap o, o2;
  const bool f32 = epi == EPI_SCALE || epi == EPI_RESIDUAL;
  if (!make_out_map(&o, g.out, f32, g.rows, g.cols, g.ldo, batch, g.strideO)) return cudaErrorInvalidValue;
  if (epi == EPI_RESIDUAL) {
    if (!make_out_map(&o2, g.out2, false, g.rows, g.cols, g.ldo, batch, g.strideO)) return cudaErrorInvalidValue;
  } else {
    o2 = o;
  }
  const long long tiles = row_tiles * ((g.cols + BN - 1) / BN);
  const int grid = (int)(tiles < nsm ? tiles : nsm);
  switch (BN) {
    case 256: return launch_bn<256>(epi, a0, a1, b, o, o2, t, grid, s);
    case 192: return launch_bn<192>(epi, a0, a1, b, o, o2, t, grid, s);
    case 128: return launch_bn<128>(epi, a0, a1, b, o, o2, t, grid, s);
    default: return launch_bn<64>(epi, a0, a1, b, o, o2, t, grid, s);
  }
}


}  // namespace sg
