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
//   warp 8 (one lane)  TMA: Q once, then K and V tiles into a 6-deep ring;
//   warp 9 (one lane)  MMA: S_j = Q K_j^T (M=128, N=128, K=64) into TMEM buffer
//                      j%3, then O_{j%2} += P_j V_j (M=128, N=64, K=128) with P_j
//                      read from TMEM (it overwrites S_j in its buffer) and V_j
//                      from shared memory (MN-major); S_{j+3} is issued right
//                      after P_j V_j, which the in-order tensor pipe finishes first;
//   warps 0-3, 4-7     two softmax warpgroups; group g takes the tiles j = g mod 2,
//                      thread t = query row t = TMEM lane t.  Each group keeps its own
//                      reference max and sum for its half of the keys and its own
//                      output accumulator in TMEM; the two halves are merged at the
//                      end (the softmax normaliser is a sum over keys, so it splits).
// Softmax of a tile: the 128 scores come out of TMEM, p = 2^(s log2e/8 - m) in
// fp32 is packed to bf16 pairs and stored back into the first 64 columns of the
// same TMEM buffer for the P V product.  The reference max m of a row is its first
// tile's max; later tiles reuse it as long as their sum of p stays below 2^64
// (then p <= 2^64: no overflow in fp32, bf16 or the fp32 accumulators); a tile
// that exceeds that renews m, recomputes its p and rescales the group's TMEM
// output row.  With three score buffers a group never waits for its own previous
// P V before writing the next P.  Every wait is bounded.  Launched with
// programmatic dependent launch (prologue overlaps the previous kernel;
// griddepcontrol.wait gates the first read of q|k|v).
#include "sg_internal.cuh"
#include "tc_common.cuh"

#include <cudaTypedefs.h>

namespace sg {

bool make_bf16_map(CUtensorMap* m, const void* ptr, long long rows, long long cols, long long ld,
                   int box_rows);

namespace {

constexpr int QT = 128;      // queries per CTA
constexpr int KT = 128;      // keys per tile
constexpr int ST = 6;        // K/V ring depth
constexpr int NSB = 3;       // TMEM score / P buffers
constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = kSoftmaxThreads + 64;
constexpr unsigned kErr = 4u;

constexpr int Q_BYTES = QT * kDh * 2;           // 16 KB
constexpr int KV_TILE = KT * kDh * 2;           // 16 KB
constexpr int STAGE_BYTES = 2 * KV_TILE;        // K + V
constexpr int OFF_KV = Q_BYTES;
constexpr int SMEM_BYTES = OFF_KV + ST * STAGE_BYTES + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");

// TMEM columns: score / P buffers [0,128), [128,256), [256,384); O accumulators
// [384,448) and [448,512)
constexpr uint32_t TM_S0 = 0, TM_O0 = NSB * KT, TMEM_COLS = 512;
static_assert(TM_O0 + 2 * kDh <= TMEM_COLS, "tensor memory");

struct AttnTcArgs {
  __nv_bfloat16* msg;
  int B, M, N, cross;
  float scale_log2;
  float blind_limit;
  unsigned* status;
  const unsigned* skip;   // adaptive depth: nothing to compute once *skip is set
};

__device__ __forceinline__ float fast_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }


__device__ __forceinline__ void softmax_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kSoftmaxThreads) : "memory");
}

// A bounded wait whose outcome is the same for every lane of the warp (the
// warp-collective TMEM loads that follow need all 32 lanes).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, unsigned* status) {
  const bool ok = tc::mbar_wait(bar, parity, status, kErr);
  return __all_sync(0xffffffffu, ok);
}

// Largest of a row's 128 raw scores (four independent chains).
__device__ __forceinline__ float row_max(const float (&s)[KT]) {
  float t0 = -INFINITY, t1 = -INFINITY, t2 = -INFINITY, t3 = -INFINITY;
#pragma unroll
  for (int i = 0; i < KT; i += 8) {
    t0 = tc::max3(t0, s[i], s[i + 1]);
    t1 = tc::max3(t1, s[i + 2], s[i + 3]);
    t2 = tc::max3(t2, s[i + 4], s[i + 5]);
    t3 = tc::max3(t3, s[i + 6], s[i + 7]);
  }
  return fmaxf(fmaxf(t0, t1), fmaxf(t2, t3));
}

// p = 2^(s * scale - m) for the row's 128 scores, packed to bf16 pairs and stored
// into TMEM columns [tp, tp + 64) of this thread's lane; returns the fp32 sum.
// EMU of every 8 pairs take the FMA-pipe exponential, the rest the MUFU.
template <int EMU>
__device__ __forceinline__ float exp_row(const float (&s)[KT], float scale, float m, uint32_t tp) {
  if (EMU == 0) {
    // all on the MUFU: one FFMA, one ex2 and one FADD per score, four
    // independent sums (no register-pair packing in the dependency chain)
    const float nm = -m;
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
    for (int cc = 0; cc < KT / 16; ++cc) {
      uint32_t pk[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int i = cc * 16 + 2 * e;
        const float p0 = fast_ex2(fmaf(s[i], scale, nm));
        const float p1 = fast_ex2(fmaf(s[i + 1], scale, nm));
        if (e & 1) { s2 += p0; s3 += p1; } else { s0 += p0; s1 += p1; }
        pk[e] = tc::pack_bf16x2(p0, p1);
      }
      tc::tmem_st8(tp + cc * 8, pk);
    }
    return (s0 + s1) + (s2 + s3);
  }
  const uint64_t sc2 = tc::f2(scale, scale);
  const uint64_t nm2 = tc::f2(-m, -m);
  uint64_t sa = tc::f2(0.f, 0.f), sb = sa;
#pragma unroll
  for (int cc = 0; cc < KT / 16; ++cc) {
    uint32_t pk[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = cc * 16 + 2 * e;
      const uint64_t x2 = tc::f2_fma(tc::f2(s[i], s[i + 1]), sc2, nm2);
      uint64_t p2;
      if (((cc * 8 + e) & 7) < EMU) {
        p2 = tc::f2_exp2_poly(x2);
      } else {
        float x0, x1;
        tc::f2_split(x2, x0, x1);
        p2 = tc::f2(fast_ex2(x0), fast_ex2(x1));
      }
      if (e & 1) sb = tc::f2_add(sb, p2); else sa = tc::f2_add(sa, p2);
      float p0, p1;
      tc::f2_split(p2, p0, p1);
      pk[e] = tc::pack_bf16x2(p0, p1);
    }
    tc::tmem_st8(tp + cc * 8, pk);
  }
  float a0, a1, b0, b1;
  tc::f2_split(sa, a0, a1);
  tc::f2_split(sb, b0, b1);
  return (a0 + a1) + (b0 + b1);
}

// SKIP: the launch reads the adaptive-depth exit flag (a separate instantiation,
// so the launches of a pass without adaptive depth run the kernel without it).
template <int EMU, bool SKIP>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm, AttnTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full;
  __shared__ __align__(8) uint64_t kv_full[ST], kv_empty[ST];
  __shared__ __align__(8) uint64_t s_full[NSB], p_full[NSB];
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
    for (int b = 0; b < NSB; ++b) {
      tc::mbar_init(&s_full[b], 1);
      tc::mbar_init(&p_full[b], 4);
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
  // the adaptive-depth exit flag (written by an earlier kernel of the pass):
  // once it is set no role does anything; all threads read it here
  bool skipped = false;
  if constexpr (SKIP) skipped = *reinterpret_cast<const volatile unsigned*>(a.skip) != 0u;

  if (skipped) {
    if (warp == 9 && lane == 0) pdl_trigger();
  } else if (warp == 8) {
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
      // A barrier probe by this thread between two batches of MMAs costs the
      // tensor pipe about 80 cycles (measured), so each key tile's two waits
      // (P_j ready, K/V of tile j+3 landed) are taken together before its batch.
      auto wait_kv = [&](int j) -> bool {
        return tc::mbar_wait(&kv_full[j % ST], (j / ST) & 1, a.status, kErr);
      };
      auto wait_p = [&](int j) -> bool {
        return tc::mbar_wait(&p_full[j % NSB], (j / NSB) & 1, a.status, kErr);
      };
      auto issue_s = [&](int j) {
        const int st = j % ST, b = j % NSB;
        // buffer b last held P_{j-3}; P_{j-3} V_{j-3} was issued before this and
        // the tensor pipe runs this thread's MMAs in order
        const uint64_t dk = tc::sdesc_k_sw128(base + OFF_KV + st * STAGE_BYTES);
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk)
          tc::umma_bf16(tmem + TM_S0 + b * KT, dq + 2 * kk, dk + 2 * kk, idesc_s, kk > 0 ? 1u : 0u);
        tc::umma_commit(&s_full[b]);
      };
      auto issue_pv = [&](int j) {
        const int b = j % NSB;
        const uint32_t vbase = base + OFF_KV + (j % ST) * STAGE_BYTES + KV_TILE;
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk) {
          const uint64_t dv = tc::sdesc_mn_sw128(vbase + kk * 2048, 8192, 1024);
          // 16 keys of P = 8 TMEM columns of bf16 pairs
          tc::umma_bf16_ts(tmem + TM_O0 + (j & 1) * kDh, tmem + TM_S0 + b * KT + kk * 8, dv, idesc_o,
                           (j >= 2 || kk > 0) ? 1u : 0u);
        }
        // one commit: it frees the K/V ring slot and tells the softmax group
        // that P_j V_j has landed in its accumulator
        tc::umma_commit(&kv_empty[j % ST]);
      };
      for (int j = 0; ok && j < NSB && j < ntiles; ++j) {
        ok = wait_kv(j);
        tc::tc_fence_after();
        if (ok) issue_s(j);
      }
      for (int j = 0; ok && j < ntiles; ++j) {
        const bool more = j + NSB < ntiles;
        ok = wait_p(j) && (!more || wait_kv(j + NSB));
        tc::tc_fence_after();
        if (!ok) break;
        issue_pv(j);
        if (more) issue_s(j + NSB);
      }
      pdl_trigger();                             // no more tensor work: the next kernel may start
      if (!ok) s_abort = 1;
    }
  } else {
    // ---------------- softmax groups: g = 0 (warps 0-3) and 1 (warps 4-7)
    const int g = warp >> 2;
    const int r = threadIdx.x & (QT - 1);            // query row = TMEM lane
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t t_o = tl + TM_O0 + g * kDh;
    float m = -INFINITY, l = 0.f;                    // log2-domain reference max, running sum
    int k = 0;                                       // tiles this group has taken
    int pv_seen = 0;                                 // this group's P V products waited for
    bool ok = true;
    // wait, in order, for this group's P V products up to count `upto`.  Its
    // product number i (tile t = g + 2 i) completes on the ring slot's
    // kv_empty[t % ST]; the next completion of that slot is this group's
    // product i + 3, and a group waits for number i only before it has written
    // P number i + 2, so the barrier is never a phase ahead of the parity asked for
    auto wait_pv = [&](int upto) -> bool {
      for (; pv_seen < upto; ++pv_seen)
        if (!warp_wait(&kv_empty[(g + 2 * pv_seen) % ST], ((g + 2 * pv_seen) / ST) & 1, a.status)) return false;
      return true;
    };
    for (int j = g; j < ntiles; j += 2, ++k) {
      const int b = j % NSB;
      const uint32_t t_s = tl + TM_S0 + b * KT;
      if (!warp_wait(&s_full[b], (j / NSB) & 1, a.status)) { ok = false; break; }
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
        tc::tmem_wait_ld(s0);                       // (one wait covers all four loads; the
        tc::tmem_wait_ld(s1);                       //  others only pin their registers)
        tc::tmem_wait_ld(s2);
        tc::tmem_wait_ld(s3);
      }
      const int valid = nk - j * KT;                 // keys of this tile that exist
      if (valid < KT) {
#pragma unroll
        for (int i = 0; i < KT; ++i)
          if (i >= valid) s[i] = -INFINITY;
      }
      // reference max of the row: the first tile's max; later tiles reuse it
      // unless their exponentials overflow the budget checked below
      if (k == 0) m = row_max(s) * a.scale_log2;
      // consume the completion of this group's P V two tiles back (long done)
      if (!wait_pv(k - 1)) { ok = false; break; }
      float sum = exp_row<EMU>(s, a.scale_log2, m, t_s);
      const bool redo = !(sum <= a.blind_limit);     // a score far above m (or a NaN)
      float c = 1.f;
      const bool any_redo = __any_sync(0xffffffffu, redo);
      if (any_redo) {                                // warp-uniform: the TMEM stores need all lanes
        if (redo) {
          const float tmax = fmaxf(m, row_max(s) * a.scale_log2);
          c = fast_ex2(m - tmax);
          l *= c;
          m = tmax;
        }
        sum = exp_row<0>(s, a.scale_log2, m, t_s);   // (other lanes rewrite their row unchanged)
      }
      l += sum;
      // (the 128 scores are dead here and their registers free)
      if (k >= 1 && any_redo) {
        // every earlier P V of this group must have landed before its rows scale
        if (!wait_pv(k)) { ok = false; break; }
        tc::tc_fence_after();
        float o[32];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          tc::tmem_ld32(t_o + hh * 32, o);
#pragma unroll
          for (int d = 0; d < 32; ++d) o[d] *= c;
          tc::tmem_st32(t_o + hh * 32, o);
        }
      }
      tc::tmem_wait_st();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&p_full[b]);
    }
    // every P V of this group must be done before its accumulator is read
    if (ok && !wait_pv(k)) ok = false;
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

__global__ void exp2_poly_selftest_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : 0.f;
  float y0, y1;
  tc::f2_split(tc::f2_exp2_poly(tc::f2(x0, x1)), y0, y1);
  y[i] = y0;
  if (i + 1 < n) y[i + 1] = y1;
}

}  // namespace

cudaError_t launch_attention_tc(const AttnArgs& a, cudaStream_t s, unsigned* status) {
  const int nmax = a.M > a.N ? a.M : a.N;
  if (a.B == 0 || nmax == 0) return cudaSuccess;
  const long long R = (long long)a.B * (a.M + a.N);
  CUtensorMap tm;
  if (!make_bf16_map(&tm, a.qkv, R, kQKV, kQKV, 128)) return cudaErrorInvalidValue;
  // share of the exponentials taken on the FMA pipe: exp_emu of every 8 pairs
  const int emu = (a.exp_emu == 2 || a.exp_emu == 3 || a.exp_emu == 4) ? a.exp_emu : 0;
  using Kern = void (*)(const CUtensorMap, AttnTcArgs);
  const bool sk = a.skip != nullptr;
  Kern kern = sk ? (emu == 0 ? attn_tc_kernel<0, true> : emu == 2 ? attn_tc_kernel<2, true>
                    : emu == 4 ? attn_tc_kernel<4, true> : attn_tc_kernel<3, true>)
                 : (emu == 0 ? attn_tc_kernel<0, false> : emu == 2 ? attn_tc_kernel<2, false>
                    : emu == 4 ? attn_tc_kernel<4, false> : attn_tc_kernel<3, false>);
  static bool attr[2][5] = {};
  if (!attr[sk][emu]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr[sk][emu] = true;
  }
  AttnTcArgs t{reinterpret_cast<__nv_bfloat16*>(a.msg), a.B, a.M, a.N, a.cross, a.scale_log2,
               a.blind_limit > 0.f ? a.blind_limit : 18446744073709551616.f, status, a.skip};
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
  return cudaLaunchKernelEx(&cfg, kern, tm, t);
}

cudaError_t launch_exp2_poly_selftest(const float* x, float* y, int n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int pairs = (n + 1) / 2;
  exp2_poly_selftest_kernel<<<(pairs + 255) / 256, 256, 0, s>>>(x, y, n);
  return cudaGetLastError();
}

}  // namespace sg
