/*
 * sg.h -- C ABI of libsg, a B200 (sm_100a) implementation of the SuperGlue
 * matcher forward pass.
 *
 * The pass, in the order the library runs it:
 *   1. keypoint normalisation and the keypoint encoder x = d + MLP_enc(x, y, c)
 *      ("笔记：SuperGlue:Learning Feature Matching with Graph Neural Networks论文阅读",
 *      realcat notes, section 特征点Encode; "SuperGlue_Code_Learning /
 *      SuperGlue_model_forward_learning", Jazihars notes, normalize_keypoints);
 *   2. n_stages attentional propagation stages alternating self and cross edges,
 *      x <- x + MLP([x || m]) with multi-head softmax(q.k/sqrt(d_head)) v messages
 *      (realcat notes, sections 多层GNN and Attentional Aggregation;
 *      "SuperGlue 的注意力图神经网络怎样传递信息", huluoboge blog);
 *   3. final projection f = W x + b and scores S = <f_A, f_B> / sqrt(D), augmented
 *      with a dustbin row and column holding the scalar bin score
 *      (realcat notes, sections 匹配得分预测 and 遮挡以及可见性; Jazihars notes,
 *      forward(), score scaling);
 *   4. log-domain Sinkhorn with marginals a = [1_M; N], b = [1_N; M]
 *      (realcat notes, section Sinkhorn Algorithm);
 *   5. mutual-nearest-neighbour extraction with a strict score threshold
 *      (Jazihars notes, forward(), matches / matching scores).
 *
 * Conventions for every entry point:
 *   - Device pointers are CUDA global-memory pointers of the current device,
 *     owned by the caller; the library never frees them.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls only enqueue work and never synchronise, except sg_status,
 *     sg_match_host and sg_create/sg_destroy.
 *   - Layouts are row-major, point-major float32:
 *       kpts  B x n x 2   (pixel x, y)
 *       conf  B x n       (detection confidence)
 *       desc  B x n x D   (descriptor of point i contiguous; the pages store
 *                          descriptors channels-first, the caller transposes)
 *       out_logP  B x (M+1) x (N+1)  log of the dustbin-augmented assignment
 *       matches0 B x M, matches1 B x N int32 (-1 = unmatched)
 *       mscores0 B x M, mscores1 B x N float32
 *   - Argument errors are reported synchronously by the return value.  Errors
 *     raised on the device (a bounded wait that ran out, a non-finite value)
 *     are latched in a per-handle status word that sg_status reads.
 *   - A handle is not thread-safe; separate handles are independent.
 */
#ifndef SG_H
#define SG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SG_MAX_STAGES 32
#define SG_ENC_LAYERS 5

typedef struct sg_handle sg_handle;

typedef enum {
    SG_OK = 0,
    SG_ERR_INVALID_ARG = 1,   /* null pointer, bad config value */
    SG_ERR_SHAPE = 2,         /* B, M or N outside [0, max] of the handle */
    SG_ERR_OOM = 3,           /* device allocation failed in sg_create */
    SG_ERR_CUDA = 4,          /* a CUDA runtime call failed */
    SG_ERR_TIMEOUT = 5,       /* a bounded device-side wait ran out */
    SG_ERR_NUMERIC = 6,       /* a non-finite value reached the transport solver */
    SG_ERR_UNSUPPORTED = 7    /* no sm_100 device, or an unsupported config */
} sg_status_t;

/* Precision of the network part (encoder, attention, projections, scores).
 * Sinkhorn and extraction always run in float32. */
typedef enum {
    SG_PRECISION_FP32 = 0,    /* float32 operands and accumulation everywhere */
    SG_PRECISION_BF16 = 1     /* bf16 GEMM/attention operands, fp32 accumulation,
                                 fp32 softmax, fp32 residual stream */
} sg_precision_t;

/* Matching head after the attentional GNN. */
typedef enum {
    SG_HEAD_SINKHORN = 0,        /* score matrix + dustbin + log-domain Sinkhorn (SuperGlue) */
    SG_HEAD_DOUBLE_SOFTMAX = 1   /* double softmax + matchability (the LightGlue review's
                                    section 2.4): no dustbin score, no iterations */
} sg_head_t;

/*
 * Weights, all HOST float32 arrays, read once by sg_create (which copies,
 * folds and packs them; the caller may free them afterwards).  Every linear
 * layer is (out_channels x in_channels), row-major: the weight of a
 * kernel-size-1 Conv1d without its trailing 1.
 *   enc_W[l], enc_b[l]: encoder layers 3->32->64->128->256->256 (channels as
 *       in the realcat notes, section 特征点Encode); enc_b[4] must be zeros
 *       or NULL (the last bias is fixed at 0 by the method).
 *   enc_bn[l][0..3]: gamma, beta, running_mean, running_var of the eval-mode
 *       BatchNorm after encoder layer l (l < 4).
 *   per stage s < n_stages:
 *       Wq, bq, Wk, bk, Wv, bv: D x D projections (head h = channels
 *           [h*D/H, (h+1)*D/H));
 *       Wm, bm: D x D merge of the concatenated heads;
 *       W1 (2D x 2D), b1, bn1[4]: first update-MLP layer on [x || m'] and its
 *           BatchNorm; W2 (D x 2D): second layer, bias fixed at 0.
 *   Wf, bf: final projection D x D.
 *   bin_score: the dustbin score z (alpha).
 *   lg_Wp, lg_bp, lg_wz, lg_bz: the double-softmax head (only read when
 *       cfg.head == SG_HEAD_DOUBLE_SOFTMAX): final projection D x D and bias
 *       (the similarity is <m0, m1> with m = (lg_Wp x + lg_bp) / D^(1/4)),
 *       matchability weights (D) and bias of z = lg_wz . x + lg_bz on the GNN
 *       states.  Wf, bf and bin_score are then not used.
 *   tc_w[l], tc_b[l]: adaptive depth (only read when cfg.depth_confidence > 0):
 *       the token-confidence classifier after layer l (stages 2l and 2l+1),
 *       c = sigmoid(tc_w[l] . x + tc_b[l]) on each point's state, D weights;
 *       needed for l < n_stages/2 - 1 (the LightGlue review, section 2.6).
 */
typedef struct {
    const float* enc_W[SG_ENC_LAYERS];
    const float* enc_b[SG_ENC_LAYERS];
    const float* enc_bn[SG_ENC_LAYERS - 1][4];
    const float* Wq[SG_MAX_STAGES];
    const float* bq[SG_MAX_STAGES];
    const float* Wk[SG_MAX_STAGES];
    const float* bk[SG_MAX_STAGES];
    const float* Wv[SG_MAX_STAGES];
    const float* bv[SG_MAX_STAGES];
    const float* Wm[SG_MAX_STAGES];
    const float* bm[SG_MAX_STAGES];
    const float* W1[SG_MAX_STAGES];
    const float* b1[SG_MAX_STAGES];
    const float* bn1[SG_MAX_STAGES][4];
    const float* W2[SG_MAX_STAGES];
    const float* Wf;
    const float* bf;
    float bin_score;
    const float* lg_Wp;
    const float* lg_bp;
    const float* lg_wz;
    float lg_bz;
    const float* tc_w[SG_MAX_STAGES / 2];
    float tc_b[SG_MAX_STAGES / 2];
} sg_weights;

/*
 * Configuration.  The library supports D = 256 and H = 4 (d_head = 64), and
 * max_N <= 3072; other values return SG_ERR_UNSUPPORTED.  max_B/max_M/max_N size the workspace that
 * the handle owns.  norm_mode 0 = (p - (W/2, H/2)) / (0.7 max(W, H)) as in the
 * Jazihars notes' normalize_keypoints; 1 = divide by max(W, H)/2 instead.
 */
typedef struct {
    int D;
    int H;
    int n_stages;            /* 1 .. SG_MAX_STAGES; stage s is self if s even */
    int sinkhorn_iters;      /* T >= 0 */
    float match_threshold;   /* strict: a match needs exp(max) > threshold */
    float bn_eps;
    int precision;           /* sg_precision_t */
    float img_w, img_h;      /* image size used by the keypoint normalisation */
    int norm_mode;
    int max_B, max_M, max_N;
    int head;                /* sg_head_t; the pages' LightGlue default threshold is 0.1 */
    float depth_confidence;  /* adaptive depth: > 0 enables the exit after a (self, cross)
                                layer l < L-1 when the share of points with confidence not
                                below clip(0.8 + 0.1 exp(-4 l / L), 0, 1) exceeds it (one
                                decision for the whole batch, over all B (M+N) points);
                                <= 0 runs every stage.  Needs an even n_stages <= 32. */
} sg_config;

/* Create a handle on the current device: validates cfg, copies and packs the
 * weights, allocates the workspace.  Synchronous.  On error *out is NULL. */
sg_status_t sg_create(const sg_weights* w, const sg_config* cfg, sg_handle** out);

/* Release the handle and everything it allocated (synchronises the device). */
void sg_destroy(sg_handle* h);

/*
 * The whole forward pass for B pairs of M and N keypoints, enqueued on
 * `stream`.  All pointers are device pointers (layouts above).  out_logP may
 * be NULL (then log P is not written, the matches still are).  M == 0 or
 * N == 0 is the pages' "no keypoints" case: matches are set to -1 and scores
 * to 0, out_logP is not touched.  Returns SG_ERR_SHAPE if B > max_B,
 * M > max_M or N > max_N.
 */
sg_status_t sg_match(sg_handle* h, int B, int M, int N,
                     const float* kpts0, const float* conf0, const float* desc0,
                     const float* kpts1, const float* conf1, const float* desc1,
                     float* out_logP,
                     int32_t* matches0, int32_t* matches1,
                     float* mscores0, float* mscores1,
                     void* stream);

/*
 * sg_match on HOST buffers: copies the inputs to handle-owned device staging
 * buffers, runs the pass, copies the outputs back and synchronises `stream`.
 * Host buffers should be pinned for the copies to be asynchronous; pageable
 * memory works but is slower.  out_logP may be NULL.
 */
sg_status_t sg_match_host(sg_handle* h, int B, int M, int N,
                          const float* kpts0, const float* conf0, const float* desc0,
                          const float* kpts1, const float* conf1, const float* desc1,
                          float* out_logP,
                          int32_t* matches0, int32_t* matches1,
                          float* mscores0, float* mscores1,
                          void* stream);

/*
 * Steps 1-3 only: writes the raw score matrix S = <f_A, f_B>/sqrt(D) (without
 * the dustbin) to out_scores, device B x M x N float32.  M, N >= 1.
 */
sg_status_t sg_scores(sg_handle* h, int B, int M, int N,
                      const float* kpts0, const float* conf0, const float* desc0,
                      const float* kpts1, const float* conf1, const float* desc1,
                      float* out_scores, void* stream);

/*
 * Steps 4-5 only, from a caller-given score matrix (device B x M x N float32):
 * dustbin augmentation with the handle's bin score, T Sinkhorn iterations and
 * extraction.  out_logP may be NULL.  M, N >= 1.
 */
sg_status_t sg_optimal_transport(sg_handle* h, int B, int M, int N,
                                 const float* scores, float* out_logP,
                                 int32_t* matches0, int32_t* matches1,
                                 float* mscores0, float* mscores1,
                                 void* stream);

/*
 * Synchronise `stream`, then return and clear the handle's device status word
 * (SG_OK, SG_ERR_TIMEOUT or SG_ERR_NUMERIC), or SG_ERR_CUDA if a CUDA call
 * reported an error.
 */
sg_status_t sg_status(sg_handle* h, void* stream);

/*
 * Adaptive depth: synchronises `stream` and writes to *layers how many
 * (self, cross) layers the last sg_match / sg_scores on this handle ran
 * (ceil(n_stages / 2) when adaptive depth is off or no exit was taken; 0 after
 * a call with M == 0 or N == 0).
 * The skipped layers' kernels still launch and return at once; the final
 * projection and the matching head run on the states at the exit.
 * Returns SG_ERR_INVALID_ARG for a null pointer, SG_ERR_CUDA if the stream
 * failed.
 */
sg_status_t sg_layers_run(sg_handle* h, int* layers, void* stream);

/*
 * Step 5 of the double-softmax head on given inputs (the counterpart of
 * sg_optimal_transport for cfg.head == SG_HEAD_DOUBLE_SOFTMAX; the handle may
 * have either head): from the similarity sim (B x M x N, float32, row-major,
 * device) and the matchability logits z0 (B x M) and z1 (B x N), writes the
 * (M+1) x (N+1) log assignment per pair into out_logP (NULL to skip):
 *   real block  log_softmax over j + log_softmax over i + log sigmoid(z0_i)
 *               + log sigmoid(z1_j);  last column log sigmoid(-z0_i);
 *   last row    log sigmoid(-z1_j);   corner 0
 * ("论文解读:LightGlue,让稀疏特征匹配随难度自适应地快", section 2.4), and the mutual
 * argmax matches with the strict threshold cfg.match_threshold, as sg_match
 * does.  Uses the handle's scratch; asynchronous on `stream`.  Errors as
 * sg_optimal_transport (SG_ERR_SHAPE for B, M or N outside the handle's
 * maxima or M == 0 or N == 0 with B > 0).
 */
sg_status_t sg_assign_double_softmax(sg_handle* h, int B, int M, int N, const float* sim,
                                     const float* z0, const float* z1, float* out_logP,
                                     int32_t* matches0, int32_t* matches1,
                                     float* mscores0, float* mscores1, void* stream);

/*
 * Self-test of the device-side failure detection: launches one CTA of a
 * two-CTA grid barrier (the same barrier the Sinkhorn kernel uses), which can
 * never complete.  The wait must end by its limit (timeout_us microseconds),
 * latch SG_ERR_TIMEOUT in the status word and return, leaving the context
 * usable.  Synchronises `stream`; returns what sg_status then reports
 * (SG_ERR_TIMEOUT when detection works).  Uses the handle's scratch memory, so
 * it must not overlap a running sg_match on the same handle.
 */
sg_status_t sg_selftest_barrier_timeout(sg_handle* h, unsigned timeout_us, void* stream);

/*
 * Self-test of the FMA-pipe exponential that the attention softmax uses for part
 * of its exp2 evaluations (Cody-Waite reduction + cubic; not in the pages, which
 * only specify the softmax).  Computes y[i] = 2^x[i] for n device floats with
 * x clamped to [-125, 126], on `stream` (asynchronous).  x and y are device
 * pointers owned by the caller, n >= 0 (n odd is fine).  Returns
 * SG_ERR_INVALID_ARG on a null pointer with n > 0, SG_ERR_CUDA if the launch
 * fails.  Expected accuracy: relative error below 1e-4 against 2^x.
 */
sg_status_t sg_selftest_exp2_poly(const float* x, float* y, int n, void* stream);

/*
 * Per-kernel timing.  enable = 1: sg_match records a CUDA event before every
 * kernel (and the Sinkhorn scratch clear) and one after the last; the events
 * are part of the captured graph.  An event between two kernels also ends the
 * programmatic dependent launch overlap between them, so the per-class times
 * add up to more than the pass.  enable = 2 (segment mode): events only where
 * the pass moves from the encoder to the GNN, from the GNN to the assignment
 * step, and at the end, so the GNN's launches run chained as without timing.
 * enable = 0 turns timing off; other values return SG_ERR_INVALID_ARG.
 * After the stream has been synchronised, sg_profile_read sums the event
 * intervals of the last sg_match by class: 0 encoder, 1 q|k|v GEMM,
 * 2 attention, 3 update-MLP layer 1 GEMM, 4 update-MLP layer 2 GEMM, 5 final
 * projection GEMM, 6 score GEMM, 7 Sinkhorn + extraction (or the
 * double-softmax head), 8 the whole GNN segment, classes 1-6 back to back
 * (segment mode only; classes 1-6 stay 0 there).  launches_by_class counts the
 * intervals.  ms_by_class and launches_by_class need n_classes >= 8 entries
 * (class 8 is written when n_classes >= 9); returns the number of classes
 * written, or -1.
 */
sg_status_t sg_profile(sg_handle* h, int enable);
int sg_profile_read(sg_handle* h, float* ms_by_class, int* launches_by_class, int n_classes);

/*
 * Steps 4-5 (transport + extraction, as sg_optimal_transport) for callers that
 * cannot allocate device memory: a runtime without a device allocator, a plugin
 * whose host application owns every allocation, or code running after memory
 * was reserved up front.  No handle is needed and nothing is allocated: the
 * scratch is a 4 MiB static device array inside the library, which every GPU
 * that loads the library holds until the process exits.  The paper has no
 * counterpart of this entry point; it exists for those callers.
 *   scores: device B x M x N float32; outputs as for sg_match (out_logP may be
 *   NULL); status: device word the caller zeroes, where device-side errors are
 *   OR-ed in (1 = a bounded wait ran out, 2 = non-finite value).
 * Returns SG_ERR_SHAPE if N > 3072 or the call needs more scratch than the
 * static array holds (about 40 bytes per score-matrix column and per row of
 * every pair).  The first call on a device does a one-time set-up (kernel
 * attributes and the array's device address); make it before any stream
 * capture.  Every call shares the one array and leaves its contents behind
 * (the parts that must start at zero are cleared on the stream by each call),
 * so calls that overlap on the GPU race: serialise them, e.g. on one stream.
 */
sg_status_t sg_optimal_transport_static(int B, int M, int N, const float* scores,
                                        float bin_score, int sinkhorn_iters,
                                        float match_threshold, float* out_logP,
                                        int32_t* matches0, int32_t* matches1,
                                        float* mscores0, float* mscores1,
                                        unsigned* status, void* stream);

/* Static description of a status code. */
const char* sg_strerror(sg_status_t s);

/* Number of kernel launches one sg_match(B, M, N) enqueues (for accounting). */
int sg_launches_per_match(const sg_handle* h, int B, int M, int N);

#ifdef __cplusplus
}
#endif
#endif /* SG_H */
