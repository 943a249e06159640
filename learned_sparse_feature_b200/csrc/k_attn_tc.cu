// tcgen05 flash attention for the bf16 path: one launch per stage serves all
// four directions of the stage (self: A<-A, B<-B; cross: A<-B, B<-A).
//
// Per head h and query i: alpha_ij = softmax_j(q_i . k_j / sqrt(64)),
// m_i = sum_j alpha_ij v_j ("SuperGlue 的注意力图神经网络怎样传递信息", section
// Attention 让节点自己选择消息来源; realcat notes "笔记：SuperGlue:Learning Feature
// Matching with Graph Neural Networks论文阅读", section Attentional Aggregation).
//
// One CTA = one 128-query tile of one (pair, image, head); it walks the source
// image in 128-key tiles j = 0, 1, ...:
//   warp 8 (one lane)  TMA: Q once, then K and V tiles into a 4-deep ring;
//   warp 9 (one lane)  MMA: S_j = Q K_j^T (M=128, N=128, K=64) into TMEM score
//                      buffer j%2, then O_{j%2} += P_j V_j (M=128, N=64, K=128, V read
//                      MN-major) into TMEM output buffer j%2;
//   warps 0-3, 4-7     two softmax warpgroups; group g takes the tiles j = g mod 2,
//                      thread t = query row t = TMEM lane t.  Each group keeps its own
//                      running max and sum for its half of the keys and its own
//                      output accumulator in TMEM; the two halves are merged at the
//                      end (the softmax normaliser is a sum over keys, so it splits).
// Softmax of a tile: the 128 scores come out of TMEM, exp2 on the MUFU, P_j goes to
// shared memory as bf16 in the 128-byte-swizzled K-major layout the MMA reads.  The
// reference max of a row only moves when a tile's max exceeds it by more than 2^8
// (P stays <= 256, exact in fp32 and bf16 range); then that group's TMEM output
// row is rescaled in place before the next P V accumulates into it.
// S_{j+2} is issued before P_j V_j, so a group finds its next scores ready when it
// finishes a tile.  Every wait is bounded.  Launched with programmatic dependent
// launch (prologue overlaps the previous kernel; griddepcontrol.wait gates the
// first read of q|k|v).
#include "sg_internal.cuh"
#include "tc_common.cuh"

#include <cudaTypedefs.h>

namespace sg {

bool make_bf16_map(CUtensorMap* m, const void* ptr, long long rows, long long cols, long long ld,
                   int box_rows);

namespace {

constexpr int QT = 128;      // queries per CTA
constexpr int KT = 128;      // keys per tile
constexpr int ST = 4;        // K/V ring depth
constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = kSoftmaxThreads + 64;
constexpr unsigned kErr = 4u;
constexpr float kRescaleLog2 = 8.f;   // lazy rescale threshold (P <= 2^8)

constexpr int Q_BYTES = QT * kDh * 2;           // 16 KB
constexpr int KV_TILE = KT * kDh * 2;           // 16 KB
constexpr int STAGE_BYTES = 2 * KV_TILE;        // K + V
constexpr int P_BYTES = QT * KT * 2;            // 32 KB (two 64-key swizzled sub-tiles)
constexpr int OFF_KV = Q_BYTES;
constexpr int OFF_P = OFF_KV + ST * STAGE_BYTES;
constexpr int SMEM_BYTES = OFF_P + 2 * P_BYTES + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");

// TMEM columns: S buffers [0,128) and [128,256); O accumulators [256,320), [320,384)
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

__device__ __forceinline__ void softmax_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kSoftmaxThreads) : "memory");
}

// A bounded wait whose outcome is the same for every lane of the warp (the
// warp-collective TMEM loads that follow need all 32 lanes).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, unsigned* status) {
  const bool ok = tc::mbar_wait(bar, parity, status, kErr);
  return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm, AttnTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full;
  __shared__ __align__(8) uint64_t kv_full[ST], kv_empty[ST];
  __shared__ __align__(8) uint64_t s_full[2], s_empty[2], p_full[2], o_full[2];
  __shared__ float2 part_ml[2][QT];      // per group and row: (reference max, sum)
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
    }
    tc::fence_barrier_init();
    s_abort = 0;
  }
  if (warp == 9) tc::tmem_alloc(&tmem_slot, TMEM_COLS);
  if (threadIdx.x == 256) tc::prefetch_tmap(&tm);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  pdl_wait();                                    // q|k|v of the previous kernel are complete

  if (warp == 8) {
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
      // the CTA must not exit with copies in flight
      tc::mbar_wait(&q_full, 0, a.status, kErr);
      for (int j = (issued > ST ? issued - ST : 0); j < issued; ++j)
        tc::mbar_wait(&kv_full[j % ST], (j / ST) & 1, a.status, kErr);
    }
  } else if (warp == 9) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(QT, KT);
      constexpr uint32_t idesc_o = tc::idesc_bf16_f32(QT, kDh, false, true);
      const uint64_t dq = tc::sdesc_k_sw128(base);
      bool ok = tc::mbar_wait(&q_full, 0, a.status, kErr);
      auto issue_s = [&](int j) -> bool {
        const int st = j % ST, b = j & 1;
        if (!tc::mbar_wait(&kv_full[st], (j / ST) & 1, a.status, kErr)) return false;
        if (j >= 2 && !tc::mbar_wait(&s_empty[b], ((j >> 1) - 1) & 1, a.status, kErr)) return false;
        tc::tc_fence_after();
        const uint64_t dk = tc::sdesc_k_sw128(base + OFF_KV + st * STAGE_BYTES);
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk)
          tc::umma_bf16(tmem + TM_S0 + b * KT, dq + 2 * kk, dk + 2 * kk, idesc_s, kk > 0 ? 1u : 0u);
        tc::umma_commit(&s_full[b]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int b = j & 1;
        if (!tc::mbar_wait(&p_full[b], (j >> 1) & 1, a.status, kErr)) return false;
        tc::tc_fence_after();
        const uint32_t pbase = base + OFF_P + b * P_BYTES;
        const uint32_t vbase = base + OFF_KV + (j % ST) * STAGE_BYTES + KV_TILE;
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk) {
          const uint64_t da = tc::sdesc_k_sw128(pbase + (kk >> 2) * (QT * 128)) + 2 * (kk & 3);
          const uint64_t dv = tc::sdesc_mn_sw128(vbase + kk * 2048, 8192, 1024);
          tc::umma_bf16(tmem + TM_O0 + b * kDh, da, dv, idesc_o, (j >= 2 || kk > 0) ? 1u : 0u);
        }
        tc::umma_commit(&o_full[b]);
        tc::umma_commit(&kv_empty[j % ST]);
        return true;
      };
      for (int j = 0; ok && j < 2 && j < ntiles; ++j) ok = issue_s(j);
      for (int j = 0; ok && j < ntiles; ++j) {
        if (j + 2 < ntiles) ok = issue_s(j + 2);
        if (ok) ok = issue_pv(j);
      }
      pdl_trigger();                             // no more tensor work: the next kernel may start
      if (!ok) s_abort = 1;
    }
  } else {
    // ---------------- softmax groups: g = 0 (warps 0-3) and 1 (warps 4-7)
    const int g = warp >> 2;
    const int r = threadIdx.x & (QT - 1);            // query row = TMEM lane
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t t_s = tl + TM_S0 + g * KT;
    const uint32_t t_o = tl + TM_O0 + g * kDh;
    uint8_t* prow = sb + OFF_P + g * P_BYTES + (r >> 3) * 1024 + (r & 7) * 128;
    float m = -INFINITY, l = 0.f;                    // log2-domain reference max, running sum
    int k = 0;                                       // tiles this group has taken
    bool ok = true;
    for (int j = g; j < ntiles; j += 2, ++k) {
      if (!warp_wait(&s_full[g], k & 1, a.status)) { ok = false; break; }
      tc::tc_fence_after();
      float s[KT];
      {
        float (&s0)[32] = *reinterpret_cast<float(*)[32]>(&s[0]);
        float (&s1)[32] = *reinterpret_cast<float(*)[32]>(&s[32]);
        float (&s2)[32] = *reinterpret_cast<float(*)[32]>(&s[64]);
        float (&s3)[32] = *reinterpret_cast<float(*)[32]>(&s[96]);
        tc::tmem_ld32_async(t_s, s0);
        tc::tmem_ld32_async(t_s + 32, s1);
        tc::tmem_ld32_async(t_s + 64, s2);
        tc::tmem_ld32_async(t_s + 96, s3);
        tc::tmem_wait_ld();
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s_empty[g]);
      const int valid = nk - j * KT;                 // keys of this tile that exist
      if (valid < KT) {
#pragma unroll
        for (int i = 0; i < KT; ++i)
          if (i >= valid) s[i] = -INFINITY;
      }
      float t0 = s[0], t1 = s[1];
#pragma unroll
      for (int i = 2; i < KT; i += 4) {
        t0 = tc::max3(t0, s[i], s[i + 1]);
        t1 = tc::max3(t1, s[i + 2], s[i + 3]);
      }
      const float tmax = fmaxf(t0, t1) * a.scale_log2;
      const bool need = tmax > m + kRescaleLog2;
      // the previous P_{j-2} V_{j-2} must be done: it reads the P buffer about to
      // be overwritten and accumulates into the output row that may be rescaled
      if (k >= 1 && !warp_wait(&o_full[g], (k - 1) & 1, a.status)) { ok = false; break; }
      float c = 1.f;
      if (need) {
        c = fast_ex2(m - tmax);                      // 0 on the first tile (m = -inf)
        l *= c;
        m = tmax;
      }
      const uint64_t sc2 = tc::f2(a.scale_log2, a.scale_log2);
      const uint64_t nm2 = tc::f2(-m, -m);
      uint64_t sum2 = tc::f2(0.f, 0.f);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = half * 64 + cc * 8 + 2 * e;
            float x0, x1;
            tc::f2_split(tc::f2_fma(tc::f2(s[i], s[i + 1]), sc2, nm2), x0, x1);
            const float p0 = fast_ex2(x0), p1 = fast_ex2(x1);
            const uint64_t p2 = tc::f2(p0, p1);
            sum2 = tc::f2_add(sum2, p2);
            pk[e] = tc::pack_bf16x2(p0, p1);
          }
          *reinterpret_cast<uint4*>(prow + half * (QT * 128) + ((cc ^ (r & 7)) << 4)) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      float sa, sb2;
      tc::f2_split(sum2, sa, sb2);
      l += sa + sb2;
      // (after the P writes: the 128 scores are dead and their registers free)
      const bool rescale_o = k >= 1 && __any_sync(0xffffffffu, need);
      if (rescale_o) {
        tc::tc_fence_after();
        float o[32];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          tc::tmem_ld32(t_o + hh * 32, o);
#pragma unroll
          for (int d = 0; d < 32; ++d) o[d] *= c;
          tc::tmem_st32(t_o + hh * 32, o);
        }
        tc::tmem_wait_st();
      }
      fence_proxy_async_smem();
      if (rescale_o) tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&p_full[g]);
    }
    // the last P V of this group must be done before its accumulator is read
    if (ok && k >= 1 && !warp_wait(&o_full[g], (k - 1) & 1, a.status)) ok = false;
    if (!ok) s_abort = 1;
    part_ml[g][r] = make_float2(m, l);
    tc::tc_fence_before();
    softmax_bar();
    tc::tc_fence_after();
    // merge the two groups: group g writes output channels [32 g, 32 g + 32)
    if (!s_abort) {
      const float2 ml0 = part_ml[0][r], ml1 = part_ml[1][r];
      const bool two = ntiles >= 2;                  // uniform: group 1 took a tile
      const float mm = two ? fmaxf(ml0.x, ml1.x) : ml0.x;
      const float c0 = fast_ex2(ml0.x - mm);
      const float c1 = two ? fast_ex2(ml1.x - mm) : 0.f;
      const float inv = 1.f / (ml0.y * c0 + ml1.y * c1);
      float o0[32];
      tc::tmem_ld32(tl + TM_O0 + g * 32, o0);
      if (two) {
        float o1[32];
        tc::tmem_ld32(tl + TM_O0 + kDh + g * 32, o1);
#pragma unroll
        for (int d = 0; d < 32; ++d) o0[d] = (o0[d] * c0 + o1[d] * c1) * inv;
      } else {
#pragma unroll
        for (int d = 0; d < 32; ++d) o0[d] *= c0 * inv;
      }
      const int q = q0 + r;
      if (q < nq) {
        uint4* out = reinterpret_cast<uint4*>(a.msg + (long long)(qrow0 + r) * kD + h * kDh + g * 32);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          out[cc] = make_uint4(tc::pack_bf16x2(o0[8 * cc], o0[8 * cc + 1]),
                               tc::pack_bf16x2(o0[8 * cc + 2], o0[8 * cc + 3]),
                               tc::pack_bf16x2(o0[8 * cc + 4], o0[8 * cc + 5]),
                               tc::pack_bf16x2(o0[8 * cc + 6], o0[8 * cc + 7]));
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 9) tc::tmem_dealloc(tmem, TMEM_COLS);
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
