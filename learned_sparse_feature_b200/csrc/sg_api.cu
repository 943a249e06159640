// Host side of libsg: the C ABI, weight folding/packing, workspace planning and
// the launch sequence of one forward pass (optionally replayed as a CUDA graph).
//
// Launch sequence of sg_match for B pairs (P = M + N stacked rows per pair):
//   encoder (1) -> n_stages x [QKV GEMM, attention, update-MLP layer 1 GEMM,
//   update-MLP layer 2 GEMM + residual] -> final projection GEMM -> score GEMM
//   -> persistent Sinkhorn with fused extraction.
// The merge layer of the attention and the eval-mode BatchNorm are folded into
// the first update-MLP layer at create time (all in float64 on the host):
//   W1 [x || Wm m + bm] + b1, then BN  ==  W1' [x || m] + b1'
//   with W1' = diag(s) [W1x | W1m Wm],  b1' = s (b1 + W1m bm - mean) + beta,
//   s = gamma / sqrt(var + eps)
// (update MLP of the realcat notes, "笔记：SuperGlue:Learning Feature Matching with
// Graph Neural Networks论文阅读", section 多层GNN).
#include "sg_internal.cuh"

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <vector>

using namespace sg;

namespace {

template <typename T> T* dmalloc(size_t n, bool* ok) {
  void* p = nullptr;
  if (n == 0) n = 1;
  if (cudaMalloc(&p, n * sizeof(T)) != cudaSuccess) { *ok = false; return nullptr; }
  return reinterpret_cast<T*>(p);
}

struct StageW {
  void* Wqkv;        // 768 x 256 (bf16 or fp32)
  float* bqkv;       // 768
  void* W1;          // 512 x 512 folded
  float* b1;         // 512 folded
  void* W2;          // 256 x 512
};

struct GraphKey {
  int B, M, N, kind;
  const void* p[12];
  bool operator==(const GraphKey& o) const { return std::memcmp(this, &o, sizeof(*this)) == 0; }
};

}  // namespace

struct sg_handle {
  sg_config cfg;
  int device;
  int num_sms;
  bool bf16;
  bool use_tc;        // tcgen05 GEMMs
  bool use_tc_attn;   // tcgen05 attention
  int attn_exp_emu;   // softmax exponentials on the FMA pipe, of every 8 pairs
  float attn_blind_limit;   // bound on a key tile's sum of P under a stale row max
  // weights
  float* encW[SG_ENC_LAYERS];
  float* encb[SG_ENC_LAYERS];
  void* encW3;         // bf16 256 x 128 (folded BN), tensor-core encoder layer 3
  void* encW4;         // bf16 256 x 256, encoder layer 4
  std::vector<StageW> stages;
  void* Wf;
  float* bf;
  float alpha;
  float score_scale;   // 1/sqrt(D) for the Sinkhorn head; 1 when folded into Wf (double softmax)
  float* lg_wz;        // double-softmax head: matchability weights (fp32) and bias
  float lg_bz;
  // adaptive depth (cfg.depth_confidence > 0): per-layer token-confidence
  // classifiers and the pass's stop / count words
  bool adaptive;
  bool last_empty;     // the last sg_match had no points on one side: no layer ran
  float* tc_w[SG_MAX_STAGES / 2];
  float tc_b[SG_MAX_STAGES / 2];
  unsigned* depth_words;
  // workspace
  float* x32;
  __nv_bfloat16* x16;
  void* qkv;
  void* msg;
  void* hid;
  void* f;
  float* Z;
  unsigned char* sk_scratch;
  size_t sk_scratch_bytes;
  unsigned char* dsm_scratch;   // double-softmax head
  float* z0;                    // matchability logits (B x M), (B x N)
  float* z1;
  unsigned* status;
  // host-buffer staging
  float *s_k0, *s_c0, *s_d0, *s_k1, *s_c1, *s_d1, *s_logP, *s_ms0, *s_ms1;
  int32_t *s_m0, *s_m1;
  // graph cache
  bool use_graph;
  cudaStream_t cap_stream;
  bool graph_valid;
  GraphKey gkey;
  cudaGraphExec_t gexec;
  std::vector<void*> allocs;
  sg_status_t sticky;
  // per-kernel timing (events between launches, also captured into graphs);
  // profiling 1 = an event before every kernel, 2 = at segment boundaries only
  int profiling;
  int prof_seg;
  std::vector<cudaEvent_t> prof_ev;
  std::vector<int> prof_cls;
  int prof_n;
};

namespace {

sg_status_t cuda_err(sg_handle* h, cudaError_t e) {
  if (e == cudaSuccess) return SG_OK;
  if (h) h->sticky = SG_ERR_CUDA;
  return SG_ERR_CUDA;
}

// Kernel classes of the per-kernel timing (sg_profile_read).
// K_GNN is the q|k|v-to-score segment timed as one interval (segment mode).
enum KClass { K_ENCODER = 0, K_QKV, K_ATTN, K_MLP1, K_MLP2, K_PROJ, K_SCORE, K_SINKHORN, K_GNN, K_END };

void mark(sg_handle* h, cudaStream_t s, int cls) {
  if (!h->profiling) return;
  if (h->profiling == 2) {
    // one event where the pass moves from the encoder to the GNN, from the GNN
    // to the assignment step, and at the end: the GNN's launches stay chained
    // (programmatic dependent launch) as they are without profiling
    if (cls >= K_QKV && cls <= K_SCORE) cls = K_GNN;
    if (h->prof_n > 0 && cls == h->prof_seg) return;
    h->prof_seg = cls;
  }
  if (h->prof_n >= (int)h->prof_ev.size()) return;
  cudaEventRecordWithFlags(h->prof_ev[h->prof_n], s, cudaEventRecordExternal);
  h->prof_cls[h->prof_n] = cls;
  ++h->prof_n;
}

// ---------------------------------------------------------------- weight folding
struct HostW {
  std::vector<double> W;   // out x in
  std::vector<double> b;
  int out, in;
};

HostW load_linear(const float* W, const float* b, int out, int in) {
  HostW r;
  r.out = out; r.in = in;
  r.W.assign(W, W + (size_t)out * in);
  r.b.assign(out, 0.0);
  if (b) for (int i = 0; i < out; ++i) r.b[i] = b[i];
  return r;
}

void fold_bn(HostW& l, const float* const bn[4], double eps) {
  for (int o = 0; o < l.out; ++o) {
    const double s = (double)bn[0][o] / std::sqrt((double)bn[3][o] + eps);
    for (int i = 0; i < l.in; ++i) l.W[(size_t)o * l.in + i] *= s;
    l.b[o] = s * (l.b[o] - (double)bn[2][o]) + (double)bn[1][o];
  }
}

template <typename T> T cvt(double v);
template <> float cvt<float>(double v) { return (float)v; }
template <> __nv_bfloat16 cvt<__nv_bfloat16>(double v) { return __float2bfloat16_rn((float)v); }

template <typename T>
void* upload_matrix(sg_handle* h, const std::vector<double>& W, size_t n, bool* ok) {
  std::vector<T> tmp(n);
  for (size_t i = 0; i < n; ++i) tmp[i] = cvt<T>(W[i]);
  T* d = dmalloc<T>(n, ok);
  if (!*ok) return nullptr;
  h->allocs.push_back(d);
  if (cudaMemcpy(d, tmp.data(), n * sizeof(T), cudaMemcpyHostToDevice) != cudaSuccess) *ok = false;
  return d;
}

float* upload_f32(sg_handle* h, const std::vector<double>& v, bool* ok) {
  return reinterpret_cast<float*>(upload_matrix<float>(h, v, v.size(), ok));
}

void* upload_w(sg_handle* h, const std::vector<double>& W, bool* ok) {
  return h->bf16 ? upload_matrix<__nv_bfloat16>(h, W, W.size(), ok)
                 : upload_matrix<float>(h, W, W.size(), ok);
}

sg_status_t pack_weights(sg_handle* h, const sg_weights* w) {
  const sg_config& c = h->cfg;
  const double eps = c.bn_eps;
  bool ok = true;
  static const int ch[6] = {3, 32, 64, 128, 256, 256};
  for (int l = 0; l < SG_ENC_LAYERS; ++l) {
    if (!w->enc_W[l]) return SG_ERR_INVALID_ARG;
    if (l < SG_ENC_LAYERS - 1) {
      if (!w->enc_b[l]) return SG_ERR_INVALID_ARG;
      for (int k = 0; k < 4; ++k) if (!w->enc_bn[l][k]) return SG_ERR_INVALID_ARG;
    }
    HostW L = load_linear(w->enc_W[l], l < SG_ENC_LAYERS - 1 ? w->enc_b[l] : nullptr, ch[l + 1], ch[l]);
    if (l < SG_ENC_LAYERS - 1) fold_bn(L, w->enc_bn[l], eps);
    // transpose to in x out for the encoder kernel
    std::vector<double> Wt((size_t)L.in * L.out);
    for (int o = 0; o < L.out; ++o)
      for (int i = 0; i < L.in; ++i) Wt[(size_t)i * L.out + o] = L.W[(size_t)o * L.in + i];
    h->encW[l] = upload_f32(h, Wt, &ok);
    h->encb[l] = upload_f32(h, L.b, &ok);
    if (h->bf16 && l == 3) h->encW3 = upload_matrix<__nv_bfloat16>(h, L.W, L.W.size(), &ok);
    if (h->bf16 && l == 4) h->encW4 = upload_matrix<__nv_bfloat16>(h, L.W, L.W.size(), &ok);
  }
  const int D = kD;
  h->stages.resize(c.n_stages);
  for (int s = 0; s < c.n_stages; ++s) {
    if (!w->Wq[s] || !w->bq[s] || !w->Wk[s] || !w->bk[s] || !w->Wv[s] || !w->bv[s] ||
        !w->Wm[s] || !w->bm[s] || !w->W1[s] || !w->b1[s] || !w->W2[s])
      return SG_ERR_INVALID_ARG;
    for (int k = 0; k < 4; ++k) if (!w->bn1[s][k]) return SG_ERR_INVALID_ARG;
    std::vector<double> Wqkv((size_t)3 * D * D), bqkv(3 * D);
    const float* Ws[3] = {w->Wq[s], w->Wk[s], w->Wv[s]};
    const float* bs[3] = {w->bq[s], w->bk[s], w->bv[s]};
    for (int t = 0; t < 3; ++t) {
      for (size_t i = 0; i < (size_t)D * D; ++i) Wqkv[(size_t)t * D * D + i] = Ws[t][i];
      for (int i = 0; i < D; ++i) bqkv[t * D + i] = bs[t][i];
    }
    // W1' = diag(s) [W1x | W1m Wm],  b1' = s (b1 + W1m bm - mean) + beta
    const int D2 = 2 * D;
    std::vector<double> W1f((size_t)D2 * D2), b1f(D2);
    const float* W1 = w->W1[s];
    const float* Wm = w->Wm[s];
    const float* bm = w->bm[s];
    std::vector<double> Wmd((size_t)D * D);
    for (size_t i = 0; i < (size_t)D * D; ++i) Wmd[i] = Wm[i];
    for (int o = 0; o < D2; ++o) {
      const float* row = W1 + (size_t)o * D2;
      for (int i = 0; i < D; ++i) W1f[(size_t)o * D2 + i] = row[i];
      std::vector<double> acc(D, 0.0);
      double bacc = w->b1[s][o];
      for (int k = 0; k < D; ++k) {
        const double wk = row[D + k];
        const double* wm = &Wmd[(size_t)k * D];
        for (int i = 0; i < D; ++i) acc[i] += wk * wm[i];
        bacc += wk * bm[k];
      }
      for (int i = 0; i < D; ++i) W1f[(size_t)o * D2 + D + i] = acc[i];
      b1f[o] = bacc;
    }
    HostW L1{W1f, b1f, D2, D2};
    fold_bn(L1, w->bn1[s], eps);
    std::vector<double> W2((size_t)D * D2);
    for (size_t i = 0; i < (size_t)D * D2; ++i) W2[i] = w->W2[s][i];
    StageW& st = h->stages[s];
    st.Wqkv = upload_w(h, Wqkv, &ok);
    st.bqkv = upload_f32(h, bqkv, &ok);
    st.W1 = upload_w(h, L1.W, &ok);
    st.b1 = upload_f32(h, L1.b, &ok);
    st.W2 = upload_w(h, W2, &ok);
  }
  if (c.head == SG_HEAD_DOUBLE_SOFTMAX) {
    // m = (Wp x + bp) / D^(1/4) on both sides: the 1/D^(1/4) goes into the
    // projection and the score GEMM runs unscaled
    if (!w->lg_Wp || !w->lg_bp || !w->lg_wz) return SG_ERR_INVALID_ARG;
    const double sc = 1.0 / std::pow((double)D, 0.25);
    std::vector<double> Wp((size_t)D * D), bp(D), wz(D);
    for (size_t i = 0; i < (size_t)D * D; ++i) Wp[i] = w->lg_Wp[i] * sc;
    for (int i = 0; i < D; ++i) { bp[i] = w->lg_bp[i] * sc; wz[i] = w->lg_wz[i]; }
    h->Wf = upload_w(h, Wp, &ok);
    h->bf = upload_f32(h, bp, &ok);
    h->lg_wz = upload_f32(h, wz, &ok);
    h->lg_bz = w->lg_bz;
    h->score_scale = 1.f;
    h->alpha = 0.f;
  } else {
    if (!w->Wf || !w->bf) return SG_ERR_INVALID_ARG;
    std::vector<double> Wf(w->Wf, w->Wf + (size_t)D * D), bf(w->bf, w->bf + D);
    h->Wf = upload_w(h, Wf, &ok);
    h->bf = upload_f32(h, bf, &ok);
    h->alpha = w->bin_score;
    h->score_scale = (float)(1.0 / std::sqrt((double)D));
  }
  if (h->adaptive) {
    // one token-confidence classifier after every layer but the last
    for (int l = 0; l + 1 < c.n_stages / 2; ++l) {
      if (!w->tc_w[l]) return SG_ERR_INVALID_ARG;
      std::vector<double> tw(w->tc_w[l], w->tc_w[l] + D);
      h->tc_w[l] = upload_f32(h, tw, &ok);
      h->tc_b[l] = w->tc_b[l];
    }
  }
  return ok ? SG_OK : SG_ERR_OOM;
}

// ---------------------------------------------------------------- launch sequence
struct Inputs {
  const float *k0, *c0, *d0, *k1, *c1, *d1;
};

cudaError_t gemm(sg_handle* h, const GemmArgs& g, int epi, bool out_bf16, int batch, cudaStream_t s,
                 int* launches, int cls) {
  mark(h, s, cls);
  ++*launches;
  if (h->use_tc) return launch_gemm_tc(g, epi, batch, s, h->status);
  return launch_gemm_simt(g, epi, h->bf16, out_bf16, batch, s);
}

// Steps 1-3: encoder, GNN, projection, scores -> S (B x M x lds, pair stride strideS)
cudaError_t run_network(sg_handle* h, int B, int M, int N, const Inputs& in, float* S, long long lds,
                        long long strideS, cudaStream_t s, int* launches) {
  const sg_config& c = h->cfg;
  const int P = M + N;
  const int R = B * P;
  const size_t esz = h->bf16 ? 2 : 4;
  EncArgs ea{};
  ea.kpts[0] = in.k0; ea.kpts[1] = in.k1;
  ea.conf[0] = in.c0; ea.conf[1] = in.c1;
  ea.desc[0] = in.d0; ea.desc[1] = in.d1;
  for (int l = 0; l < SG_ENC_LAYERS; ++l) { ea.W[l] = h->encW[l]; ea.b[l] = h->encb[l]; }
  ea.x32 = h->x32;
  ea.x16 = h->x16;
  ea.B = B; ea.M = M; ea.N = N;
  ea.cx = c.img_w * 0.5f;
  ea.cy = c.img_h * 0.5f;
  const float mx = c.img_w > c.img_h ? c.img_w : c.img_h;
  ea.inv_scale = (float)(1.0 / (c.norm_mode == 0 ? 0.7 * (double)mx : 0.5 * (double)mx));
  mark(h, s, K_ENCODER);
  cudaError_t e;
  // adaptive depth: clear the stop word and the per-layer counters of the pass
  const unsigned* skip = nullptr;
  if (h->adaptive) {
    if ((e = cudaMemsetAsync(h->depth_words, 0, kDepthWords * sizeof(unsigned), s)) != cudaSuccess) return e;
    skip = h->depth_words;
  }
  if (h->use_tc) {
    // layers 0-2 on CUDA cores, layers 3-4 on the tensor cores
    __nv_bfloat16* h2 = reinterpret_cast<__nv_bfloat16*>(h->msg);   // R x 128, free until attention
    e = launch_encoder_head(ea, h2, s);
    ++*launches;
    if (e != cudaSuccess) return e;
    GemmArgs g{};
    g.A0 = h2; g.A1 = nullptr; g.lda = 128; g.k_split = 128;
    g.W = h->encW3; g.bias = h->encb[3]; g.out = h->hid; g.ldo = kD;
    g.rows = R; g.cols = kD; g.K = 128; g.scale = 1.f;
    ++*launches;
    if ((e = launch_gemm_tc(g, EPI_BIAS_RELU, 1, s, h->status)) != cudaSuccess) return e;
    g = GemmArgs{};
    g.A0 = h->hid; g.A1 = nullptr; g.lda = kD; g.k_split = kD;
    g.W = h->encW4; g.bias = nullptr; g.out = h->x32; g.out2 = h->x16; g.ldo = kD;
    g.rows = R; g.cols = kD; g.K = kD; g.scale = 1.f;
    ++*launches;
    if ((e = launch_gemm_tc(g, EPI_RESIDUAL, 1, s, h->status)) != cudaSuccess) return e;
  } else {
    e = launch_encoder(ea, h->bf16, s);
    ++*launches;
    if (e != cudaSuccess) return e;
  }
  const void* xin = h->bf16 ? (const void*)h->x16 : (const void*)h->x32;
  for (int st = 0; st < c.n_stages; ++st) {
    const StageW& w = h->stages[st];
    GemmArgs g{};
    // q|k|v = x Wqkv^T + b
    g.A0 = xin; g.A1 = nullptr; g.lda = kD; g.k_split = kD;
    g.W = w.Wqkv; g.bias = w.bqkv; g.out = h->qkv; g.ldo = kQKV;
    g.rows = R; g.cols = kQKV; g.K = kD; g.scale = 1.f;
    g.skip = skip;
    if ((e = gemm(h, g, EPI_BIAS, h->bf16, 1, s, launches, K_QKV)) != cudaSuccess) return e;
    AttnArgs aa{};
    aa.qkv = h->qkv; aa.msg = h->msg; aa.B = B; aa.M = M; aa.N = N;
    aa.cross = (st % 2 == 1);
    aa.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)kDh));
    aa.exp_emu = h->attn_exp_emu;
    aa.blind_limit = h->attn_blind_limit;
    aa.skip = skip;
    mark(h, s, K_ATTN);
    ++*launches;
    e = h->use_tc_attn ? launch_attention_tc(aa, s, h->status) : launch_attention_simt(aa, h->bf16, s);
    if (e != cudaSuccess) return e;
    // h = relu(W1' [x || m] + b1')
    g = GemmArgs{};
    g.A0 = xin; g.A1 = h->msg; g.lda = kD; g.k_split = kD;
    g.W = w.W1; g.bias = w.b1; g.out = h->hid; g.ldo = 2 * kD;
    g.rows = R; g.cols = 2 * kD; g.K = 2 * kD; g.scale = 1.f;
    g.skip = skip;
    if ((e = gemm(h, g, EPI_BIAS_RELU, h->bf16, 1, s, launches, K_MLP1)) != cudaSuccess) return e;
    // x += W2 h   (bias 0), refresh the bf16 shadow
    g = GemmArgs{};
    g.A0 = h->hid; g.A1 = nullptr; g.lda = 2 * kD; g.k_split = 2 * kD;
    g.W = w.W2; g.bias = nullptr; g.out = h->x32; g.out2 = h->x16; g.ldo = kD;
    g.rows = R; g.cols = kD; g.K = 2 * kD; g.scale = 1.f;
    g.skip = skip;
    if ((e = gemm(h, g, EPI_RESIDUAL, h->bf16, 1, s, launches, K_MLP2)) != cudaSuccess) return e;
    // adaptive depth: exit check after every (self, cross) layer but the last
    // (LightGlue review, section 2.6); later GNN launches see its stop word
    const int L = c.n_stages / 2, layer = st / 2;
    if (h->adaptive && st % 2 == 1 && layer + 1 < L) {
      const double lam = std::min(1.0, std::max(0.0, 0.8 + 0.1 * std::exp(-4.0 * layer / L)));
      ++*launches;
      if ((e = launch_depth_check(h->x32, R, h->tc_w[layer], h->tc_b[layer], (float)lam, c.depth_confidence,
                                  layer, h->depth_words, s)) != cudaSuccess)
        return e;
    }
  }
  // f = Wf x + bf
  GemmArgs g{};
  g.A0 = xin; g.A1 = nullptr; g.lda = kD; g.k_split = kD;
  g.W = h->Wf; g.bias = h->bf; g.out = h->f; g.ldo = kD;
  g.rows = R; g.cols = kD; g.K = kD; g.scale = 1.f;
  if ((e = gemm(h, g, EPI_BIAS, h->bf16, 1, s, launches, K_PROJ)) != cudaSuccess) return e;
  // S_b = f_A f_B^T / sqrt(D), batched over pairs
  g = GemmArgs{};
  g.A0 = h->f; g.A1 = nullptr; g.lda = kD; g.k_split = kD;
  g.W = (const unsigned char*)h->f + (size_t)M * kD * esz;
  g.out = S; g.ldo = lds;
  g.rows = M; g.cols = N; g.K = kD;
  g.strideA = (long long)P * kD; g.strideW = (long long)P * kD; g.strideO = strideS;
  g.scale = h->score_scale;
  g.w_dynamic = 1;   // W = f_B, the projection just computed
  return gemm(h, g, EPI_SCALE, false, B, s, launches, K_SCORE);
}

// Steps 4-5 from S.
cudaError_t run_transport(sg_handle* h, int B, int M, int N, const float* S, long long lds,
                          long long strideS, float* logP, int32_t* m0, int32_t* m1, float* s0,
                          float* s1, cudaStream_t st, int* launches) {
  const size_t R = M + 1;
  unsigned char* p = h->sk_scratch;
  SinkhornArgs a{};
  a.barrier = reinterpret_cast<unsigned*>(p);
  a.abort_flag = a.barrier + B;
  size_t off = ((B + 1) * sizeof(unsigned) + 255) & ~(size_t)255;
  a.acc = reinterpret_cast<float*>(p + off);
  a.fb = a.acc + (size_t)B * 3 * sinkhorn_acc_floats_per_buffer(N);
  off += (size_t)B * 5 * sinkhorn_acc_floats_per_buffer(N) * 4;
  off = (off + 255) & ~(size_t)255;
  a.colbest = reinterpret_cast<unsigned long long*>(p + off);
  off += (size_t)B * N * 8;
  off = (off + 255) & ~(size_t)255;
  const size_t zero_bytes = off;
  a.u = reinterpret_cast<float*>(p + off);
  off += (size_t)B * R * 4;
  off = (off + 255) & ~(size_t)255;
  a.idx0 = reinterpret_cast<int32_t*>(p + off);
  off += (size_t)B * M * 4;
  off = (off + 255) & ~(size_t)255;
  a.max0 = reinterpret_cast<float*>(p + off);
  mark(h, st, K_SINKHORN);
  cudaError_t e = cudaMemsetAsync(p, 0, zero_bytes, st);
  if (e != cudaSuccess) return e;
  a.S = S; a.lds = lds; a.strideS = strideS; a.alpha = h->alpha;
  a.lds_vec = (lds % 4 == 0) && (strideS % 4 == 0) && ((reinterpret_cast<uintptr_t>(S) & 15) == 0);
  a.B = B; a.M = M; a.N = N; a.iters = h->cfg.sinkhorn_iters;
  a.threshold = h->cfg.match_threshold;
  a.logP = logP; a.matches0 = m0; a.matches1 = m1; a.mscores0 = s0; a.mscores1 = s1;
  a.status = h->status;
  a.timeout_ns = 1000000000ull;   // 1 s per barrier wait
  e = launch_sinkhorn(a, h->num_sms, st, launches);
  mark(h, st, K_END);
  return e;
}

sg_status_t check_shape(sg_handle* h, int B, int M, int N) {
  if (!h) return SG_ERR_INVALID_ARG;
  if (B < 0 || M < 0 || N < 0) return SG_ERR_SHAPE;
  if (B > h->cfg.max_B || M > h->cfg.max_M || N > h->cfg.max_N) return SG_ERR_SHAPE;
  return SG_OK;
}

sg_status_t empty_outputs(sg_handle* h, int B, int M, int N, int32_t* m0, int32_t* m1, float* s0,
                          float* s1, cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  if (B * M > 0) {
    if (!m0 || !s0) return SG_ERR_INVALID_ARG;
    e = cudaMemsetAsync(m0, 0xff, (size_t)B * M * sizeof(int32_t), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(s0, 0, (size_t)B * M * sizeof(float), s);
  }
  if (e == cudaSuccess && B * N > 0) {
    if (!m1 || !s1) return SG_ERR_INVALID_ARG;
    e = cudaMemsetAsync(m1, 0xff, (size_t)B * N * sizeof(int32_t), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(s1, 0, (size_t)B * N * sizeof(float), s);
  }
  return cuda_err(h, e);
}

// Run `fn` (which enqueues work on a stream) either directly or through a
// cached CUDA graph keyed by the call's sizes and pointers.
template <typename F>
sg_status_t run_maybe_graph(sg_handle* h, const GraphKey& key, cudaStream_t s, F&& fn) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (s) cudaStreamIsCapturing(s, &cs);
  if (!h->use_graph || cs != cudaStreamCaptureStatusNone) {
    int launches = 0;
    return cuda_err(h, fn(s, &launches));
  }
  if (!(h->graph_valid && h->gkey == key)) {
    cudaGraph_t g = nullptr;
    cudaError_t e = cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal);
    if (e != cudaSuccess) return cuda_err(h, e);
    int launches = 0;
    cudaError_t fe = fn(h->cap_stream, &launches);
    e = cudaStreamEndCapture(h->cap_stream, &g);
    if (fe != cudaSuccess || e != cudaSuccess) {
      if (g) cudaGraphDestroy(g);
      cudaGetLastError();
      return cuda_err(h, fe != cudaSuccess ? fe : e);
    }
    bool updated = false;
    if (h->graph_valid) {
      cudaGraphExecUpdateResultInfo info;
      if (cudaGraphExecUpdate(h->gexec, g, &info) == cudaSuccess) updated = true;
      else cudaGetLastError();
    }
    if (!updated) {
      if (h->graph_valid) cudaGraphExecDestroy(h->gexec);
      h->graph_valid = false;
      e = cudaGraphInstantiate(&h->gexec, g, 0);
      if (e != cudaSuccess) { cudaGraphDestroy(g); return cuda_err(h, e); }
    }
    cudaGraphDestroy(g);
    h->graph_valid = true;
    h->gkey = key;
  }
  return cuda_err(h, cudaGraphLaunch(h->gexec, s));
}

}  // namespace

extern "C" {

const char* sg_strerror(sg_status_t s) {
  switch (s) {
    case SG_OK: return "ok";
    case SG_ERR_INVALID_ARG: return "invalid argument";
    case SG_ERR_SHAPE: return "size outside the handle's configured maxima";
    case SG_ERR_OOM: return "device allocation failed";
    case SG_ERR_CUDA: return "CUDA runtime error";
    case SG_ERR_TIMEOUT: return "a bounded device-side wait ran out";
    case SG_ERR_NUMERIC: return "non-finite value in the transport solver";
    case SG_ERR_UNSUPPORTED: return "unsupported device or configuration";
  }
  return "unknown status";
}

int sg_launches_per_match(const sg_handle* h, int B, int M, int N) {
  if (!h || B == 0 || M == 0 || N == 0) return 0;
  const int net = (h->use_tc ? 5 : 3) + 4 * h->cfg.n_stages;   // encoder .. score GEMM
  const int depth = h->adaptive ? h->cfg.n_stages / 2 - 1 : 0;  // exit checks
  return net + depth + (h->cfg.head == SG_HEAD_DOUBLE_SOFTMAX ? 7 : 1);  // matchability + 6 head kernels, or Sinkhorn
}

sg_status_t sg_create(const sg_weights* w, const sg_config* cfg, sg_handle** out) {
  if (!out) return SG_ERR_INVALID_ARG;
  *out = nullptr;
  if (!w || !cfg) return SG_ERR_INVALID_ARG;
  if (cfg->D != kD || cfg->H != kH) return SG_ERR_UNSUPPORTED;
  if (cfg->n_stages < 1 || cfg->n_stages > SG_MAX_STAGES || cfg->sinkhorn_iters < 0 ||
      cfg->max_B < 0 || cfg->max_M < 0 || cfg->max_N < 0 || !(cfg->bn_eps >= 0.f) ||
      !(cfg->img_w > 0.f) || !(cfg->img_h > 0.f) || (cfg->norm_mode != 0 && cfg->norm_mode != 1) ||
      (cfg->precision != SG_PRECISION_FP32 && cfg->precision != SG_PRECISION_BF16) ||
      (cfg->head != SG_HEAD_SINKHORN && cfg->head != SG_HEAD_DOUBLE_SOFTMAX))
    return SG_ERR_INVALID_ARG;
  if (cfg->max_N > sinkhorn_max_columns()) return SG_ERR_UNSUPPORTED;   // transport kernel columns
  if (std::isnan(cfg->depth_confidence)) return SG_ERR_INVALID_ARG;
  // adaptive depth works on whole (self, cross) layers
  if (cfg->depth_confidence > 0.f && (cfg->n_stages % 2 != 0 || cfg->n_stages / 2 > 16))
    return SG_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return SG_ERR_UNSUPPORTED; }
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return SG_ERR_CUDA;
  if (prop.major != 10) return SG_ERR_UNSUPPORTED;

  sg_handle* h = new sg_handle();
  h->cfg = *cfg;
  h->device = dev;
  h->num_sms = prop.multiProcessorCount;
  h->bf16 = cfg->precision == SG_PRECISION_BF16;
  h->adaptive = cfg->depth_confidence > 0.f;
  h->use_tc = h->bf16 && tc_available() && std::getenv("SG_FORCE_SIMT") == nullptr;
  h->use_tc_attn = h->use_tc && std::getenv("SG_SIMT_ATTENTION") == nullptr;
  {
    // SG_ATTN_EXP_EMU=2|3|4 moves that many of every 8 exp2 pairs of the
    // attention softmax to the FMA pipe (default 0: all on the MUFU, measured
    // fastest at these shapes); for tests and tuning
    const char* e = std::getenv("SG_ATTN_EXP_EMU");
    const int v = e ? std::atoi(e) : 0;
    h->attn_exp_emu = (v == 2 || v == 3 || v == 4) ? v : 0;
    // SG_ATTN_BLIND_LIMIT_LOG2=x (0 <= x <= 64) lowers the 2^64 bound so that
    // the max-renewal path runs on ordinary inputs; for tests
    const char* b = std::getenv("SG_ATTN_BLIND_LIMIT_LOG2");
    const double lb = b ? std::atof(b) : 64.0;
    h->attn_blind_limit = (float)std::exp2(lb >= 0.0 && lb <= 64.0 ? lb : 64.0);
  }
  h->use_graph = std::getenv("SG_NO_GRAPH") == nullptr;
  h->sticky = SG_OK;
  sg_status_t st = pack_weights(h, w);
  if (st != SG_OK) { sg_destroy(h); return st; }
  bool ok = true;
  const size_t Bm = cfg->max_B, Mm = cfg->max_M, Nm = cfg->max_N;
  const size_t R = Bm * (Mm + Nm);
  const size_t esz = h->bf16 ? 2 : 4;
  auto al = [&](size_t bytes) -> void* {
    void* p = dmalloc<unsigned char>(bytes + 256, &ok);
    if (p) h->allocs.push_back(p);
    return p;
  };
  h->x32 = (float*)al(R * kD * 4);
  h->x16 = h->bf16 ? (__nv_bfloat16*)al(R * kD * 2) : nullptr;
  h->qkv = al(R * kQKV * esz);
  h->msg = al(R * kD * esz);
  h->hid = al(R * 2 * kD * esz);
  h->f = al(R * kD * esz);
  h->Z = (float*)al(Bm * Mm * ((Nm + 3) & ~(size_t)3) * 4);
  h->sk_scratch_bytes = sinkhorn_scratch_bytes((int)Bm, (int)Mm, (int)Nm);
  h->sk_scratch = (unsigned char*)al(h->sk_scratch_bytes);
  h->dsm_scratch = (unsigned char*)al(dsm_scratch_bytes((int)Bm, (int)Mm, (int)Nm));
  h->z0 = (float*)al(Bm * Mm * 4);
  h->z1 = (float*)al(Bm * Nm * 4);
  h->status = (unsigned*)al(sizeof(unsigned));
  h->depth_words = (unsigned*)al(kDepthWords * sizeof(unsigned));
  h->s_k0 = (float*)al(Bm * Mm * 2 * 4);
  h->s_c0 = (float*)al(Bm * Mm * 4);
  h->s_d0 = (float*)al(Bm * Mm * kD * 4);
  h->s_k1 = (float*)al(Bm * Nm * 2 * 4);
  h->s_c1 = (float*)al(Bm * Nm * 4);
  h->s_d1 = (float*)al(Bm * Nm * kD * 4);
  h->s_logP = (float*)al(Bm * (Mm + 1) * (Nm + 1) * 4);
  h->s_m0 = (int32_t*)al(Bm * Mm * 4);
  h->s_m1 = (int32_t*)al(Bm * Nm * 4);
  h->s_ms0 = (float*)al(Bm * Mm * 4);
  h->s_ms1 = (float*)al(Bm * Nm * 4);
  if (!ok) { cudaGetLastError(); sg_destroy(h); return SG_ERR_OOM; }
  if (sinkhorn_prepare(h->num_sms) != cudaSuccess) { cudaGetLastError(); sg_destroy(h); return SG_ERR_CUDA; }
  if (cudaMemset(h->status, 0, sizeof(unsigned)) != cudaSuccess ||
      cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking) != cudaSuccess) {
    sg_destroy(h);
    return SG_ERR_CUDA;
  }
  *out = h;
  return SG_OK;
}

void sg_destroy(sg_handle* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  if (h->graph_valid) cudaGraphExecDestroy(h->gexec);
  if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
  for (cudaEvent_t ev : h->prof_ev) cudaEventDestroy(ev);
  for (void* p : h->allocs) cudaFree(p);
  delete h;
}

sg_status_t sg_scores(sg_handle* h, int B, int M, int N, const float* kpts0, const float* conf0,
                      const float* desc0, const float* kpts1, const float* conf1, const float* desc1,
                      float* out_scores, void* stream) {
  sg_status_t st = check_shape(h, B, M, N);
  if (st != SG_OK) return st;
  if (B == 0) return SG_OK;
  if (M == 0 || N == 0) return SG_ERR_SHAPE;
  if (!kpts0 || !conf0 || !desc0 || !kpts1 || !conf1 || !desc1 || !out_scores)
    return SG_ERR_INVALID_ARG;
  h->last_empty = false;
  cudaStream_t s = (cudaStream_t)stream;
  Inputs in{kpts0, conf0, desc0, kpts1, conf1, desc1};
  int launches = 0;
  // The tensor-core score GEMM stores 16-byte-aligned rows: a caller layout
  // that is not (N % 4 != 0 or a misaligned buffer) goes through the handle's
  // score buffer and one strided copy.
  const bool direct = !h->use_tc || (N % 4 == 0 && (reinterpret_cast<uintptr_t>(out_scores) & 15) == 0);
  if (direct) return cuda_err(h, run_network(h, B, M, N, in, out_scores, N, (long long)M * N, s, &launches));
  const long long lds = (N + 3) & ~3;
  cudaError_t e = run_network(h, B, M, N, in, h->Z, lds, (long long)M * lds, s, &launches);
  if (e == cudaSuccess)
    e = cudaMemcpy2DAsync(out_scores, (size_t)N * sizeof(float), h->Z, (size_t)lds * sizeof(float),
                          (size_t)N * sizeof(float), (size_t)B * M, cudaMemcpyDeviceToDevice, s);
  return cuda_err(h, e);
}

sg_status_t sg_optimal_transport(sg_handle* h, int B, int M, int N, const float* scores,
                                 float* out_logP, int32_t* matches0, int32_t* matches1,
                                 float* mscores0, float* mscores1, void* stream) {
  sg_status_t st = check_shape(h, B, M, N);
  if (st != SG_OK) return st;
  if (B == 0) return SG_OK;
  if (M == 0 || N == 0) return SG_ERR_SHAPE;
  if (!scores || !matches0 || !matches1 || !mscores0 || !mscores1) return SG_ERR_INVALID_ARG;
  int launches = 0;
  return cuda_err(h, run_transport(h, B, M, N, scores, N, (long long)M * N, out_logP, matches0,
                                   matches1, mscores0, mscores1, (cudaStream_t)stream, &launches));
}

sg_status_t sg_assign_double_softmax(sg_handle* h, int B, int M, int N, const float* sim, const float* z0,
                                     const float* z1, float* out_logP, int32_t* matches0, int32_t* matches1,
                                     float* mscores0, float* mscores1, void* stream) {
  sg_status_t st = check_shape(h, B, M, N);
  if (st != SG_OK) return st;
  if (B == 0) return SG_OK;
  if (M == 0 || N == 0) return SG_ERR_SHAPE;
  if (!sim || !z0 || !z1 || !matches0 || !matches1 || !mscores0 || !mscores1) return SG_ERR_INVALID_ARG;
  int launches = 0;
  return cuda_err(h, launch_dsm_assign(sim, N, (long long)M * N, B, M, N, z0, z1, h->cfg.match_threshold,
                                       out_logP, matches0, matches1, mscores0, mscores1, h->dsm_scratch,
                                       (cudaStream_t)stream, &launches));
}

sg_status_t sg_match(sg_handle* h, int B, int M, int N, const float* kpts0, const float* conf0,
                     const float* desc0, const float* kpts1, const float* conf1, const float* desc1,
                     float* out_logP, int32_t* matches0, int32_t* matches1, float* mscores0,
                     float* mscores1, void* stream) {
  sg_status_t st = check_shape(h, B, M, N);
  if (st != SG_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (B == 0) return SG_OK;
  h->last_empty = (M == 0 || N == 0);
  if (M == 0 || N == 0) return empty_outputs(h, B, M, N, matches0, matches1, mscores0, mscores1, s);
  if (!kpts0 || !conf0 || !desc0 || !kpts1 || !conf1 || !desc1 || !matches0 || !matches1 ||
      !mscores0 || !mscores1)
    return SG_ERR_INVALID_ARG;
  const long long lds = (N + 3) & ~3;
  const long long strideS = (long long)M * lds;
  Inputs in{kpts0, conf0, desc0, kpts1, conf1, desc1};
  GraphKey key{};
  key.B = B; key.M = M; key.N = N; key.kind = 1 + h->profiling;
  const void* ps[12] = {kpts0, conf0, desc0, kpts1, conf1, desc1, out_logP, matches0, matches1,
                        mscores0, mscores1, nullptr};
  std::memcpy(key.p, ps, sizeof(ps));
  return run_maybe_graph(h, key, s, [&](cudaStream_t cs, int* launches) -> cudaError_t {
    h->prof_n = 0;
    cudaError_t e = run_network(h, B, M, N, in, h->Z, lds, strideS, cs, launches);
    if (e != cudaSuccess) return e;
    if (h->cfg.head == SG_HEAD_DOUBLE_SOFTMAX) {
      // matchability from the final GNN states, then the closed-form assignment
      mark(h, cs, K_SINKHORN);
      e = launch_dsm_matchability(h->x32, B, M, N, h->lg_wz, h->lg_bz, h->z0, h->z1, cs);
      ++*launches;
      if (e != cudaSuccess) return e;
      e = launch_dsm_assign(h->Z, lds, strideS, B, M, N, h->z0, h->z1, h->cfg.match_threshold, out_logP,
                            matches0, matches1, mscores0, mscores1, h->dsm_scratch, cs, launches);
      mark(h, cs, K_END);
      return e;
    }
    return run_transport(h, B, M, N, h->Z, lds, strideS, out_logP, matches0, matches1, mscores0,
                         mscores1, cs, launches);
  });
}

sg_status_t sg_match_host(sg_handle* h, int B, int M, int N, const float* kpts0, const float* conf0,
                          const float* desc0, const float* kpts1, const float* conf1,
                          const float* desc1, float* out_logP, int32_t* matches0, int32_t* matches1,
                          float* mscores0, float* mscores1, void* stream) {
  sg_status_t st = check_shape(h, B, M, N);
  if (st != SG_OK) return st;
  if (B == 0) return SG_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t nM = (size_t)B * M, nN = (size_t)B * N;
  auto h2d = [&](void* d, const void* src, size_t bytes) -> cudaError_t {
    if (bytes == 0) return cudaSuccess;
    return cudaMemcpyAsync(d, src, bytes, cudaMemcpyHostToDevice, s);
  };
  auto d2h = [&](void* dst, const void* d, size_t bytes) -> cudaError_t {
    if (bytes == 0) return cudaSuccess;
    return cudaMemcpyAsync(dst, d, bytes, cudaMemcpyDeviceToHost, s);
  };
  if ((nM && (!matches0 || !mscores0)) || (nN && (!matches1 || !mscores1))) return SG_ERR_INVALID_ARG;
  if (M > 0 && N > 0) {
    if (!kpts0 || !conf0 || !desc0 || !kpts1 || !conf1 || !desc1) return SG_ERR_INVALID_ARG;
    cudaError_t e = h2d(h->s_k0, kpts0, nM * 8);
    if (e == cudaSuccess) e = h2d(h->s_c0, conf0, nM * 4);
    if (e == cudaSuccess) e = h2d(h->s_d0, desc0, nM * kD * 4);
    if (e == cudaSuccess) e = h2d(h->s_k1, kpts1, nN * 8);
    if (e == cudaSuccess) e = h2d(h->s_c1, conf1, nN * 4);
    if (e == cudaSuccess) e = h2d(h->s_d1, desc1, nN * kD * 4);
    if (e != cudaSuccess) return cuda_err(h, e);
  }
  st = sg_match(h, B, M, N, h->s_k0, h->s_c0, h->s_d0, h->s_k1, h->s_c1, h->s_d1,
                out_logP ? h->s_logP : nullptr, h->s_m0, h->s_m1, h->s_ms0, h->s_ms1, stream);
  if (st != SG_OK) return st;
  cudaError_t e = d2h(matches0, h->s_m0, nM * 4);
  if (e == cudaSuccess) e = d2h(matches1, h->s_m1, nN * 4);
  if (e == cudaSuccess) e = d2h(mscores0, h->s_ms0, nM * 4);
  if (e == cudaSuccess) e = d2h(mscores1, h->s_ms1, nN * 4);
  if (e == cudaSuccess && out_logP && M > 0 && N > 0)
    e = d2h(out_logP, h->s_logP, (size_t)B * (M + 1) * (N + 1) * 4);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return cuda_err(h, e);
}

sg_status_t sg_selftest_exp2_poly(const float* x, float* y, int n, void* stream) {
  if (n < 0) return SG_ERR_INVALID_ARG;
  if (n == 0) return SG_OK;
  if (!x || !y) return SG_ERR_INVALID_ARG;
  return launch_exp2_poly_selftest(x, y, n, (cudaStream_t)stream) == cudaSuccess ? SG_OK : SG_ERR_CUDA;
}

sg_status_t sg_selftest_barrier_timeout(sg_handle* h, unsigned timeout_us, void* stream) {
  if (!h) return SG_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  unsigned* scratch = reinterpret_cast<unsigned*>(h->sk_scratch);
  int* returned = reinterpret_cast<int*>(h->sk_scratch + 16);
  cudaError_t e = cudaMemsetAsync(h->sk_scratch, 0, 32, s);
  if (e == cudaSuccess)
    e = launch_barrier_selftest(scratch, h->status, (unsigned long long)timeout_us * 1000ull, returned, s);
  int ret = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&ret, returned, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_err(h, e);
  if (ret != 1) return SG_ERR_INVALID_ARG;   // the wait did not report its expiry
  return sg_status(h, stream);
}

sg_status_t sg_profile(sg_handle* h, int enable) {
  if (!h) return SG_ERR_INVALID_ARG;
  if (enable && h->prof_ev.empty()) {
    const int n = 8 + 4 * h->cfg.n_stages + 4;
    h->prof_ev.resize(n);
    h->prof_cls.assign(n, -1);
    for (int i = 0; i < n; ++i)
      if (cudaEventCreate(&h->prof_ev[i]) != cudaSuccess) return cuda_err(h, cudaGetLastError());
  }
  if (enable < 0 || enable > 2) return SG_ERR_INVALID_ARG;
  h->profiling = enable;
  h->prof_n = 0;
  return SG_OK;
}

int sg_profile_read(sg_handle* h, float* ms_by_class, int* launches_by_class, int n_classes) {
  if (!h || !ms_by_class || !launches_by_class || n_classes < K_GNN) return -1;
  if (n_classes > K_END) n_classes = K_END;
  for (int c = 0; c < n_classes; ++c) { ms_by_class[c] = 0.f; launches_by_class[c] = 0; }
  for (int i = 0; i + 1 < h->prof_n; ++i) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, h->prof_ev[i], h->prof_ev[i + 1]) != cudaSuccess) {
      cudaGetLastError();
      return -1;
    }
    const int c = h->prof_cls[i];
    if (c >= 0 && c < n_classes) { ms_by_class[c] += ms; launches_by_class[c] += 1; }
  }
  return n_classes;
}

sg_status_t sg_layers_run(sg_handle* h, int* layers, void* stream) {
  if (!h || !layers) return SG_ERR_INVALID_ARG;
  const int all = (h->cfg.n_stages + 1) / 2;
  if (h->last_empty) {                 // M == 0 or N == 0: the early return ran no layer
    *layers = 0;
    return SG_OK;
  }
  if (!h->adaptive) {
    *layers = all;
    return SG_OK;
  }
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  unsigned w[2] = {0u, 0u};
  if (e == cudaSuccess) e = cudaMemcpy(w, h->depth_words, sizeof(w), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_err(h, e);
  *layers = w[0] ? (int)w[1] : all;
  return SG_OK;
}

sg_status_t sg_status(sg_handle* h, void* stream) {
  if (!h) return SG_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_err(h, e);
  unsigned word = 0;
  e = cudaMemcpy(&word, h->status, sizeof(unsigned), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_err(h, e);
  if (word) cudaMemset(h->status, 0, sizeof(unsigned));
  sg_status_t sticky = h->sticky;
  h->sticky = SG_OK;
  if (sticky != SG_OK) return sticky;
  if (word & (kStatusTimeout | kStatusPipeline)) return SG_ERR_TIMEOUT;
  if (word & kStatusNumeric) return SG_ERR_NUMERIC;
  return SG_OK;
}

}  // extern "C"
