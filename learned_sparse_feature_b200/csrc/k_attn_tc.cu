// tcgen05 flash attention for the bf16 path: one launch per stage serves all
// four directions of the stage (self: A<-A, B<-B; cross: A<-B, B<-A).
//
// Per head h and query i: alpha_ij = softmax_j(q_i . k_j / sqrt(64)),
// m_i = sum_j alpha_ij v_j ("SuperGlue 的注意力图神经网络怎样传递信息", section
// Attention 让节点自己选择消息来源; realcat notes "笔记：SuperGlue:Learning Feature
// Matching with Graph Neural Networks论文阅读", section Attentional Aggregation).
//
// One CTA = one 128-query tile of one (pair, image, head); it walks the source
// image in 128-key tiles:
//   warp 4 (one lane)  TMA: Q once, then K and V tiles into a 3-deep ring;
//   warp 5 (one lane)  MMA: S_j = Q K_j^T (M=128, N=128, K=64) into one of two
//                      TMEM score buffers, then O_j = P_j V_j (M=128, N=64, K=128,
//                      V read MN-major) into one of two TMEM output buffers;
//   warps 0-3          softmax, thread t = query row t = TMEM lane t: loads its
//                      128 scores, online max/sum in fp32 (exp2 on the MUFU), writes
//                      P_j as bf16 into shared memory in the 128-byte-swizzled
//                      K-major layout the MMA reads, and folds O_j into a running
//                      fp32 output kept in registers (rescaled when the max grows).
// The S MMA of tile j+1 overlaps the softmax of tile j.  Every wait is bounded.
// Launched with programmatic dependent launch (prologue overlaps the previous
// kernel; griddepcontrol.wait gates the first read of q|k|v).
#include "sg_internal.cuh"
#include "tc_common.cuh"

#include <cudaTypedefs.h>

namespace sg {

bool make_bf16_map(CUtensorMap* m, const void* ptr, long long rows, long long cols, long long ld,
                   int box_rows);

namespace {

constexpr int QT = 128;      // queries per CTA
constexpr int KT = 128;      // keys per tile
constexpr int ST = 3;        // K/V ring depth
constexpr int kThreads = 192;
constexpr unsigned kErr = 4u;

constexpr int Q_BYTES = QT * kDh * 2;           // 16 KB
constexpr int KV_TILE = KT * kDh * 2;           // 16 KB
constexpr int STAGE_BYTES = 2 * KV_TILE;        // K + V
constexpr int P_BYTES = QT * KT * 2;            // 32 KB (two 64-key swizzled sub-tiles)
constexpr int OFF_KV = Q_BYTES;
constexpr int OFF_P = OFF_KV + ST * STAGE_BYTES;
constexpr int SMEM_BYTES = OFF_P + 2 * P_BYTES + 1024;

// TMEM columns: S buffers [0,128) and [128,256); O buffers [256,320), [320,384)
constexpr uint32_t TM_S0 = 0, TM_O0 = 256, TMEM_COLS = 512;

struct AttnTcArgs {
  __nv_bfloat16* msg;
  int B, M, N, cross;
  float scale_log2;
  unsigned* status;
};

__device__ __forceinline__ float fast_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm, AttnTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full;
  __shared__ __align__(8) uint64_t kv_full[ST], kv_empty[ST];
  __shared__ __align__(8) uint64_t s_full[2], s_empty[2], p_full[2], o_full[2], o_empty[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int s_abort;

  const int P = a.M + a.N;
  const int pair = blockIdx.z >> 1;
  const int img = blockIdx.z & 1;
  const int h = blockIdx.y;
  const int nq = img ? a.N : a.M;
  const int src = a.cross ? 1 - img : img;
  const int nk = src ? a.N : a.M;
  const int q0 = blockIdx.x * QT;
  if (q0 >= nq) return;
  const int qrow0 = pair * P + (img ? a.M : 0) + q0;
  const int krow0 = pair * P + (src ? a.M : 0);
  const int ntiles = (nk + KT - 1) / KT;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t base = (tc::smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sb = smem_raw + (base - tc::smem_u32(smem_raw));

  if (threadIdx.x == 0) {
    tc::mbar_init(&q_full, 1);
    for (int s = 0; s < ST; ++s) { tc::mbar_init(&kv_full[s], 1); tc::mbar_init(&kv_empty[s], 1); }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&s_full[b], 1);
      tc::mbar_init(&s_empty[b], 4);
      tc::mbar_init(&p_full[b], 4);
      tc::mbar_init(&o_full[b], 1);
      tc::mbar_init(&o_empty[b], 4);
    }
    tc::fence_barrier_init();
    s_abort = 0;
  }
  if (warp == 5) tc::tmem_alloc(&tmem_slot, TMEM_COLS);
  if (threadIdx.x == 128) tc::prefetch_tmap(&tm);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  pdl_wait();                                    // q|k|v of the previous kernel are complete

  if (warp == 4) {
    if (lane == 0) {
      // ---------------- TMA producer
      tc::mbar_arrive_expect_tx(&q_full, Q_BYTES);
      tc::tma_load_2d(&tm, &q_full, sb, h * kDh, qrow0);
      int issued = 0;
      for (int j = 0; j < ntiles; ++j) {
        const int st = j % ST, u = j / ST;
        if (u > 0 && !tc::mbar_wait(&kv_empty[st], (u - 1) & 1, a.status, kErr)) { s_abort = 1; break; }
        uint8_t* kd = sb + OFF_KV + st * STAGE_BYTES;
        tc::mbar_arrive_expect_tx(&kv_full[st], STAGE_BYTES);
        tc::tma_load_2d(&tm, &kv_full[st], kd, kD + h * kDh, krow0 + j * KT);
        tc::tma_load_2d(&tm, &kv_full[st], kd + KV_TILE, 2 * kD + h * kDh, krow0 + j * KT);
        ++issued;
      }
      tc::mbar_wait(&q_full, 0, a.status, kErr);
      for (int j = (issued > ST ? issued - ST : 0); j < issued; ++j)
        tc::mbar_wait(&kv_full[j % ST], (j / ST) & 1, a.status, kErr);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(QT, KT);
      constexpr uint32_t idesc_o = tc::idesc_bf16_f32(QT, kDh, false, true);
      const uint64_t dq = tc::sdesc_k_sw128(base);
      bool ok = tc::mbar_wait(&q_full, 0, a.status, kErr);
      auto issue_pv = [&](int jp) -> bool {
        const int b = jp & 1;
        if (!tc::mbar_wait(&p_full[b], (jp >> 1) & 1, a.status, kErr)) return false;
        if (jp >= 2 && !tc::mbar_wait(&o_empty[b], ((jp >> 1) - 1) & 1, a.status, kErr)) return false;
        tc::tc_fence_after();
        const uint32_t pbase = base + OFF_P + b * P_BYTES;
        const uint32_t vbase = base + OFF_KV + (jp % ST) * STAGE_BYTES + KV_TILE;
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk) {
          const uint64_t da = tc::sdesc_k_sw128(pbase + (kk >> 2) * (QT * 128)) + 2 * (kk & 3);
          const uint64_t dv = tc::sdesc_mn_sw128(vbase + kk * 2048, 8192, 1024);
          tc::umma_bf16(tmem + TM_O0 + b * kDh, da, dv, idesc_o, kk > 0 ? 1u : 0u);
        }
        tc::umma_commit(&o_full[b]);
        tc::umma_commit(&kv_empty[jp % ST]);
        return true;
      };
      for (int j = 0; ok && j < ntiles; ++j) {
        const int st = j % ST, b = j & 1;
        if (!tc::mbar_wait(&kv_full[st], (j / ST) & 1, a.status, kErr)) { ok = false; break; }
        if (j >= 2 && !tc::mbar_wait(&s_empty[b], ((j >> 1) - 1) & 1, a.status, kErr)) { ok = false; break; }
        tc::tc_fence_after();
        const uint64_t dk = tc::sdesc_k_sw128(base + OFF_KV + st * STAGE_BYTES);
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk)
          tc::umma_bf16(tmem + TM_S0 + b * KT, dq + 2 * kk, dk + 2 * kk, idesc_s, kk > 0 ? 1u : 0u);
        tc::umma_commit(&s_full[b]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_pv(ntiles - 1);
      pdl_trigger();                             // no more tensor work: the next kernel may start
      if (!ok) s_abort = 1;
    }
  } else {
    // ---------------- softmax warps 0-3: thread = query row
    const int r = threadIdx.x;                       // 0..127
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    float o[kDh];
#pragma unroll
    for (int d = 0; d < kDh; ++d) o[d] = 0.f;
    float m = -INFINITY, l = 0.f, frame = -INFINITY;
    float mprev = -INFINITY;                         // max of the tile whose O is pending
    bool ok = true;
    auto take_o = [&](int jp) -> bool {
      const int b = jp & 1;
      if (!tc::mbar_wait(&o_full[b], (jp >> 1) & 1, a.status, kErr)) return false;
      tc::tc_fence_after();
      float pv[64];
      float t0[32], t1[32];
      tc::tmem_ld32(tl + TM_O0 + b * kDh, t0);
      tc::tmem_ld32(tl + TM_O0 + b * kDh + 32, t1);
#pragma unroll
      for (int i = 0; i < 32; ++i) { pv[i] = t0[i]; pv[32 + i] = t1[i]; }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&o_empty[b]);
      const float c = fast_ex2(frame - mprev);
#pragma unroll
      for (int d = 0; d < kDh; ++d) o[d] = fmaf(o[d], c, pv[d]);
      frame = mprev;
      return true;
    };
    for (int j = 0; j < ntiles; ++j) {
      const int b = j & 1;
      if (!tc::mbar_wait(&s_full[b], (j >> 1) & 1, a.status, kErr)) { ok = false; break; }
      tc::tc_fence_after();
      float s[KT];
#pragma unroll
      for (int c = 0; c < KT / 32; ++c) {
        float t[32];
        tc::tmem_ld32(tl + TM_S0 + b * KT + c * 32, t);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c * 32 + i] = t[i];
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s_empty[b]);
      const int valid = nk - j * KT;                 // keys of this tile that exist
      float tmax = -INFINITY;
#pragma unroll
      for (int i = 0; i < KT; ++i) {
        s[i] = (i < valid) ? s[i] * a.scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, s[i]);
      }
      const float mnew = fmaxf(m, tmax);
      float sum = 0.f;
      uint8_t* prow = sb + OFF_P + b * P_BYTES + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = fast_ex2(s[half * 64 + c * 8 + 2 * e] - mnew);
            const float p1 = fast_ex2(s[half * 64 + c * 8 + 2 * e + 1] - mnew);
            sum += p0 + p1;
            pk[e] = tc::pack_bf16x2(p0, p1);
          }
          *reinterpret_cast<uint4*>(prow + half * (QT * 128) + ((c ^ (r & 7)) << 4)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      l = l * fast_ex2(m - mnew) + sum;
      m = mnew;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&p_full[b]);
      if (j >= 1 && !take_o(j - 1)) { ok = false; break; }
      mprev = mnew;
    }
    if (ok) ok = take_o(ntiles - 1);
    if (!ok) s_abort = 1;
    const int q = q0 + r;
    if (ok && q < nq) {
      const float inv = 1.f / l;
      uint4* out = reinterpret_cast<uint4*>(a.msg + (long long)(qrow0 + r) * kD + h * kDh);
#pragma unroll
      for (int c = 0; c < kDh / 8; ++c) {
        out[c] = make_uint4(tc::pack_bf16x2(o[8 * c] * inv, o[8 * c + 1] * inv),
                            tc::pack_bf16x2(o[8 * c + 2] * inv, o[8 * c + 3] * inv),
                            tc::pack_bf16x2(o[8 * c + 4] * inv, o[8 * c + 5] * inv),
                            tc::pack_bf16x2(o[8 * c + 6] * inv, o[8 * c + 7] * inv));
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 5) tc::tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace

cudaError_t launch_attention_tc(const AttnArgs& a, cudaStream_t s, unsigned* status) {
  const int nmax = a.M > a.N ? a.M : a.N;
  if (a.B == 0 || nmax == 0) return cudaSuccess;
  const long long R = (long long)a.B * (a.M + a.N);
  CUtensorMap tm;
  if (!make_bf16_map(&tm, a.qkv, R, kQKV, kQKV, 128)) return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  AttnTcArgs t{reinterpret_cast<__nv_bfloat16*>(a.msg), a.B, a.M, a.N, a.cross, a.scale_log2, status};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((nmax + QT - 1) / QT, kH, 2 * a.B);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute la[1];
  la[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap with the previous kernel
  la[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = la;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attn_tc_kernel, tm, t);
}

}  // namespace sg
