"""Float64 CPU oracle of the SuperGlue matcher forward pass.

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow, step-by-step
definition that the CUDA path is checked against.  Only the tests, the smoke
check and the benchmark's CPU-baseline leg may import it; the library itself
never does, and it shares no code, table or helper with the CUDA sources.

Every step is written in float64 NumPy in the order and notation of the pages:

* keypoint normalisation: "SuperGlue_Code_Learning / SuperGlue_model_forward_learning"
  (Jazihars notes), the ``normalize_keypoints`` walkthrough;
* keypoint encoder x = d + MLP_enc(x, y, c): "笔记：SuperGlue:Learning Feature
  Matching with Graph Neural Networks论文阅读" (realcat notes), section 特征点Encode;
  "SuperGlue 的注意力图神经网络怎样传递信息" (huluoboge blog), section
  SuperGlue 的两类边分别带来什么;
* attention q/k/v, softmax(q.k/sqrt(d_head)), message = sum alpha v: huluoboge
  blog, section Attention 让节点自己选择消息来源; realcat notes, section
  Attentional Aggregation;
* residual update x <- x + MLP([x || m]) with self/cross alternation: realcat
  notes, section 多层GNN; huluoboge blog, section 多轮消息怎样回到同一幅图;
* final projection, score S = <f_A, f_B> / sqrt(D): realcat notes, section
  匹配层 / 匹配得分预测; Jazihars notes, forward() walkthrough (score scaling);
* dustbin augmentation and marginals a = [1_M; N], b = [1_N; M]: realcat notes,
  section 遮挡以及可见性;
* log-domain Sinkhorn: realcat notes, section Sinkhorn Algorithm (the author's
  log-space optimal transport);
* mutual nearest neighbour extraction with threshold: Jazihars notes,
  forward() walkthrough (matches / matching scores).

Readings of points the pages leave open (each is also listed in the design
notes): BatchNorm eps = 1e-5; head h uses channels [64h, 64h+64); the heads are
merged by a 256->256 linear layer with bias; argmax ties go to the lowest index.

Parity status: see the header of each function ("pinned by" lines name the
test that pins it).
"""
from __future__ import annotations

import math

import numpy as np

F64 = np.float64


def _as64(a):
    return np.asarray(a, dtype=F64)


# --------------------------------------------------------------------------- boundary
def normalize_keypoints(kpts, width, height, mode=0):
    """(kpt - (W/2, H/2)) / (0.7 * max(W, H))   [Jazihars notes, normalize_keypoints].

    mode 1 divides by max(W, H)/2 instead (a long-side [-1, 1] normalisation).
    Pinned by: the printed input/output values of the notes (tests/golden).
    """
    k = _as64(kpts)
    center = np.array([width / 2.0, height / 2.0], F64)
    if mode == 0:
        scaling = max(width, height) * 0.7
    else:
        scaling = max(width, height) / 2.0
    return (k - center) / scaling


# --------------------------------------------------------------------------- MLP blocks
def batchnorm_eval(z, gamma, beta, mean, var, eps):
    """Eval-mode BatchNorm1d per channel: gamma (z - mean) / sqrt(var + eps) + beta.

    z is (points, channels).  Pinned by: torch.nn.BatchNorm1d in eval mode.
    """
    return _as64(gamma) * (z - _as64(mean)) / np.sqrt(_as64(var) + eps) + _as64(beta)


def linear(z, W, b):
    """Kernel-size-1 Conv1d on point-major data: z (n, c_in) -> z W^T + b."""
    out = z @ _as64(W).T
    if b is not None:
        out = out + _as64(b)
    return out


def mlp(z, Ws, bs, bns, eps):
    """Conv1d(k=1) layers; BatchNorm + ReLU after every layer except the last
    [realcat notes, section 特征点Encode, the MLP builder].
    Pinned by: torch Conv1d/BatchNorm1d/ReLU Sequential with the same weights."""
    n = len(Ws)
    for l in range(n):
        z = linear(z, Ws[l], bs[l])
        if l < n - 1:
            z = batchnorm_eval(z, *bns[l], eps)
            z = np.maximum(z, 0.0)
    return z


def keypoint_encoder(kpts_norm, conf, desc, weights, eps):
    """x0 = d + MLP_enc([x, y, c]), MLP channels 3-32-64-128-256-256, last bias 0
    [realcat notes, section 特征点Encode; huluoboge blog, x^(0) = d + MLP_enc(p)].
    Input order (x, y, c): keypoints first, then the confidence."""
    p = np.concatenate([_as64(kpts_norm), _as64(conf)[:, None]], axis=1)
    enc = mlp(p, weights["enc_W"], weights["enc_b"], weights["enc_bn"], eps)
    return _as64(desc) + enc


# --------------------------------------------------------------------------- attention
def softmax(e, axis=-1):
    """exp(e) / sum exp(e), max-shifted.  Pinned by the worked example of the
    huluoboge blog (scores [2, 1, 0])."""
    e = _as64(e)
    m = np.max(e, axis=axis, keepdims=True)
    x = np.exp(e - m)
    return x / np.sum(x, axis=axis, keepdims=True)


def attend(q, k, v):
    """One head: alpha_ij = softmax_j(q_i . k_j / sqrt(d_k)); m_i = sum_j alpha_ij v_j
    [huluoboge blog, section Attention 让节点自己选择消息来源].
    Returns (message, alpha)."""
    dk = q.shape[-1]
    e = (q @ k.T) / math.sqrt(dk)
    alpha = softmax(e, axis=1)
    return alpha @ v, alpha


def multi_head_attention(x, src, st, heads):
    """q = Wq x + bq (query image), k = Wk s + bk, v = Wv s + bv (source image);
    head h reads channels [dh*h, dh*(h+1)); the concatenated heads go through the
    merge layer Wm, bm [realcat notes, section Attentional Aggregation].
    Pinned by: torch.nn.MultiheadAttention with the same projections."""
    q = linear(x, st["Wq"], st["bq"])
    k = linear(src, st["Wk"], st["bk"])
    v = linear(src, st["Wv"], st["bv"])
    d = q.shape[1]
    dh = d // heads
    msg = np.empty((x.shape[0], d), F64)
    for h in range(heads):
        sl = slice(h * dh, (h + 1) * dh)
        msg[:, sl], _ = attend(q[:, sl], k[:, sl], v[:, sl])
    return linear(msg, st["Wm"], st["bm"])


def bidirectional_cross_attention(x0, x1, st, heads):
    """Cross attention with one similarity matrix for both directions [LightGlue
    review, section 2.3 交叉注意力, the CrossBlock forward listing]: a point has
    one projection qk = Wqk x + bqk (here st["Wq"], st["bq"]) and a value
    v = Wv x + bv; per head, sim = (qk0 s)(qk1 s)^T with s = d_head^(-1/4);
    softmax over the rows of sim gives the messages to image 0 from the values
    of image 1, softmax over the rows of sim^T the messages to image 1; the
    concatenated heads go through the merge layer.  Returns (m0, m1)."""
    qk0 = linear(x0, st["Wq"], st["bq"])
    qk1 = linear(x1, st["Wq"], st["bq"])
    v0 = linear(x0, st["Wv"], st["bv"])
    v1 = linear(x1, st["Wv"], st["bv"])
    d = qk0.shape[1]
    dh = d // heads
    s = dh ** -0.25
    m0 = np.empty((x0.shape[0], d), F64)
    m1 = np.empty((x1.shape[0], d), F64)
    for h in range(heads):
        sl = slice(h * dh, (h + 1) * dh)
        sim = (qk0[:, sl] * s) @ (qk1[:, sl] * s).T
        m0[:, sl] = softmax(sim, axis=1) @ v1[:, sl]
        m1[:, sl] = softmax(sim.T, axis=1) @ v0[:, sl]
    return linear(m0, st["Wm"], st["bm"]), linear(m1, st["Wm"], st["bm"])


def attentional_propagation(x, src, st, heads, eps):
    """delta = MLP([x || message]), MLP 512-512-256 with BN+ReLU in the middle
    and last bias 0 [realcat notes, section 多层GNN, AttentionalPropagation]."""
    m = multi_head_attention(x, src, st, heads)
    z = np.concatenate([x, m], axis=1)
    return mlp(z, [st["W1"], st["W2"]], [st["b1"], st["b2"]], [st["bn1"]], eps)


def stage_names(n_stages):
    """['self', 'cross'] repeated: self first [realcat notes, section 多层GNN]."""
    return ["self" if s % 2 == 0 else "cross" for s in range(n_stages)]


def attentional_gnn(x0, x1, weights, heads, eps, n_stages=None, bidirectional=False):
    """Stages alternate self (A<-A, B<-B) and cross (A<-B, B<-A); both deltas are
    computed from the pre-stage states and then added [realcat notes, section
    多层GNN, AttentionalGNN].  bidirectional=True: the cross stages take their
    messages from bidirectional_cross_attention (one qk projection, one
    similarity for both directions [LightGlue review, section 2.3]) and feed
    them to the same update MLP."""
    stages = weights["stages"]
    if n_stages is None:
        n_stages = len(stages)
    for s, name in enumerate(stage_names(n_stages)):
        if name == "cross" and bidirectional:
            st = stages[s]
            m0, m1 = bidirectional_cross_attention(x0, x1, st, heads)
            d0 = mlp(np.concatenate([x0, m0], axis=1), [st["W1"], st["W2"]], [st["b1"], st["b2"]], [st["bn1"]], eps)
            d1 = mlp(np.concatenate([x1, m1], axis=1), [st["W1"], st["W2"]], [st["b1"], st["b2"]], [st["bn1"]], eps)
            x0, x1 = x0 + d0, x1 + d1
            continue
        if name == "cross":
            src0, src1 = x1, x0
        else:
            src0, src1 = x0, x1
        d0 = attentional_propagation(x0, src0, stages[s], heads, eps)
        d1 = attentional_propagation(x1, src1, stages[s], heads, eps)
        x0, x1 = x0 + d0, x1 + d1
    return x0, x1


# --------------------------------------------------------------------------- matching layer
def score_matrix(x0, x1, Wf, bf):
    """f = Wf x + bf for both images; S_ij = <f_i^A, f_j^B> / sqrt(D)
    [realcat notes, section 匹配得分预测; Jazihars notes, forward(), scaling by
    descriptor_dim ** 0.5]."""
    f0 = linear(x0, Wf, bf)
    f1 = linear(x1, Wf, bf)
    return (f0 @ f1.T) / math.sqrt(f0.shape[1])


def augment_dustbin(S, alpha):
    """S_bar = [[S, alpha 1], [alpha 1^T, alpha]] [realcat notes, section 遮挡以及可见性]."""
    M, N = S.shape
    Z = np.full((M + 1, N + 1), float(alpha), F64)
    Z[:M, :N] = S
    return Z


def logsumexp(x, axis):
    """log sum exp along an axis, max-shifted (all entries are finite here)."""
    m = np.max(x, axis=axis, keepdims=True)
    return np.squeeze(m, axis=axis) + np.log(np.sum(np.exp(x - m), axis=axis))


def log_marginals(M, N):
    """log mu = [norm]*M ++ [log N + norm], log nu = [norm]*N ++ [log M + norm],
    norm = -log(M + N): the marginals a = [1_M; N], b = [1_N; M] divided by M+N
    [realcat notes, sections 遮挡以及可见性 and Sinkhorn Algorithm]."""
    norm = -math.log(M + N)
    log_mu = np.full(M + 1, norm, F64)
    log_mu[M] = math.log(N) + norm
    log_nu = np.full(N + 1, norm, F64)
    log_nu[N] = math.log(M) + norm
    return log_mu, log_nu, norm


def log_sinkhorn(Z, log_mu, log_nu, iters):
    """u = v = 0; repeat: u = log mu - LSE_j(Z + v); v = log nu - LSE_i(Z + u).
    Returns Z + u + v [realcat notes, section Sinkhorn Algorithm].
    Pinned by: the 1x1 closed form, the constant-score closed form, the exact
    column marginals, and brute-force optimal partial assignments."""
    u = np.zeros(Z.shape[0], F64)
    v = np.zeros(Z.shape[1], F64)
    for _ in range(iters):
        u = log_mu - logsumexp(Z + v[None, :], axis=1)
        v = log_nu - logsumexp(Z + u[:, None], axis=0)
    return Z + u[:, None] + v[None, :]


def log_optimal_transport(S, alpha, iters):
    """Dustbin-augmented log-domain optimal transport; the result is multiplied
    by M + N (i.e. -norm added) so that its marginals are a and b."""
    M, N = S.shape
    Z = augment_dustbin(S, alpha)
    log_mu, log_nu, norm = log_marginals(M, N)
    return log_sinkhorn(Z, log_mu, log_nu, iters) - norm


def extract_matches(logP, threshold):
    """Mutual nearest neighbours on the real block of log P_bar [Jazihars notes,
    forward(), "Get the matches with score above match_threshold"]:
    idx0 = argmax_j, idx1 = argmax_i (lowest index on ties); mutual0_i iff
    idx1[idx0[i]] == i; mscore0 = exp(max0) if mutual0 else 0; mscore1_j =
    mscore0[idx1_j] if mutual1 else 0; valid0 = mutual0 and mscore0 > threshold;
    valid1 = mutual1 and valid0[idx1_j]; invalid entries are -1.
    Pinned by: hand-built matrices (ties, dustbin-best rows, non-mutual pairs,
    values at the threshold)."""
    P = _as64(logP)[:-1, :-1]
    M, N = P.shape
    idx0 = np.argmax(P, axis=1)          # numpy argmax returns the first maximum
    idx1 = np.argmax(P, axis=0)
    max0 = P[np.arange(M), idx0]
    mutual0 = idx1[idx0] == np.arange(M)
    mutual1 = idx0[idx1] == np.arange(N)
    mscores0 = np.where(mutual0, np.exp(max0), 0.0)
    mscores1 = np.where(mutual1, mscores0[idx1], 0.0)
    valid0 = mutual0 & (mscores0 > threshold)
    valid1 = mutual1 & valid0[idx1]
    matches0 = np.where(valid0, idx0, -1).astype(np.int32)
    matches1 = np.where(valid1, idx1, -1).astype(np.int32)
    return matches0, matches1, mscores0, mscores1


# --------------------------------------------------------------------------- double-softmax head
def log_sigmoid(x):
    """log(1 / (1 + exp(-x))) = min(x, 0) - log(1 + exp(-|x|)) (stable form)."""
    x = _as64(x)
    return np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))


def log_softmax(x, axis):
    """x - log sum exp along `axis`."""
    x = _as64(x)
    return x - np.expand_dims(logsumexp(x, axis), axis)


def double_softmax_log_assignment(sim, z0, z1):
    """The matching head that replaces the dustbin and Sinkhorn ("论文解读:LightGlue,
    让稀疏特征匹配随难度自适应地快" (LightGlue review), section 2.4 匹配头, the
    sigmoid_log_double_softmax listing): an (M+1) x (N+1) log assignment whose real
    block is log_softmax over j (each row) + log_softmax over i (each column) +
    log sigmoid(z0_i) + log sigmoid(z1_j); the last column is log sigmoid(-z0_i),
    the last row log sigmoid(-z1_j), the corner 0.
    Pinned by: torch log_softmax / logsigmoid in float64, a 2 x 2 closed form, the
    dustbin complement exp(last column) = 1 - sigmoid(z0), planted mistakes."""
    sim = _as64(sim)
    z0, z1 = _as64(z0), _as64(z1)
    M, N = sim.shape
    out = np.zeros((M + 1, N + 1), F64)
    out[:M, :N] = (log_softmax(sim, 1) + log_softmax(sim, 0)
                   + log_sigmoid(z0)[:, None] + log_sigmoid(z1)[None, :])
    out[:M, N] = log_sigmoid(-z0)
    out[M, :N] = log_sigmoid(-z1)
    return out


def double_softmax_head(x0, x1, Wp, bp, wz, bz):
    """Similarity and matchability of the double-softmax head (LightGlue review,
    section 2.4, MatchAssignment.forward): m = final_proj(x) / D^(1/4) for both
    images, sim_ij = <m0_i, m1_j>; z = matchability(x) = x . wz + bz on the GNN
    states themselves (not on m).  Returns (log assignment, sim, z0, z1).
    Pinned by: the torch MatchAssignment composition in float64."""
    x0, x1 = _as64(x0), _as64(x1)
    d = x0.shape[1]
    m0 = linear(x0, Wp, bp) / d ** 0.25
    m1 = linear(x1, Wp, bp) / d ** 0.25
    sim = m0 @ m1.T
    z0 = x0 @ _as64(wz) + float(bz)
    z1 = x1 @ _as64(wz) + float(bz)
    return double_softmax_log_assignment(sim, z0, z1), sim, z0, z1


# --------------------------------------------------------------------------- training-side derivatives
def nll_loss(logP, matches, unmatched0, unmatched1):
    """Negative log-likelihood of the augmented assignment: -sum log P_ij over the
    true matches, -sum log P_i,N+1 over the unmatched points of A, -sum
    log P_M+1,j over those of B [realcat notes, section Loss]."""
    logP = _as64(logP)
    M, N = logP.shape[0] - 1, logP.shape[1] - 1
    loss = -sum(logP[i, j] for i, j in matches)
    loss -= sum(logP[i, N] for i in unmatched0)
    loss -= sum(logP[M, j] for j in unmatched1)
    return float(loss)


def nll_loss_grad(shape, matches, unmatched0, unmatched1):
    """d nll_loss / d log P: -1 at every entry the loss reads."""
    g = np.zeros(shape, F64)
    M, N = shape[0] - 1, shape[1] - 1
    for i, j in matches:
        g[i, j] -= 1.0
    for i in unmatched0:
        g[i, N] -= 1.0
    for j in unmatched1:
        g[M, j] -= 1.0
    return g


def attend_backward(q, k, v, g):
    """Gradients of m = softmax(q k^T / sqrt(d)) v for the upstream gradient g =
    dL/dm: dL/de_ij = alpha_ij g_i . (v_j - m_i) for the scores e [huluoboge
    blog, the derivation of how the loss changes attention], then through
    e = q k^T / sqrt(d) and m = alpha v.  Returns (dq, dk, dv)."""
    q, k, v, g = _as64(q), _as64(k), _as64(v), _as64(g)
    d = q.shape[1]
    m, a = attend(q, k, v)
    de = a * (g @ v.T - np.sum(g * m, axis=1, keepdims=True))
    dq = de @ k / math.sqrt(d)
    dk = de.T @ q / math.sqrt(d)
    dv = a.T @ g
    return dq, dk, dv


def log_sinkhorn_backward(Z, log_mu, log_nu, iters, G):
    """dL/dZ for out = log_sinkhorn(Z, ...) and the upstream gradient G = dL/dout,
    by reverse mode through the T iterations: out = Z + u_T + v_T; v_t = log nu -
    LSE_i(Z + u_t) gives dv_t/dZ_ij = dv_t/du_t,i = -Pc_ij (Pc the softmax of Z + u_t
    over i); u_t = log mu - LSE_j(Z + v_{t-1}) gives -Pr_ij (Pr the softmax of
    Z + v_{t-1} over j); v_0 = 0."""
    Z, G = _as64(Z), _as64(G)
    us, vs = [], [np.zeros(Z.shape[1], F64)]
    u = np.zeros(Z.shape[0], F64)
    v = vs[0]
    for _ in range(iters):
        u = log_mu - logsumexp(Z + v[None, :], axis=1)
        v = log_nu - logsumexp(Z + u[:, None], axis=0)
        us.append(u)
        vs.append(v)
    dZ = G.copy()
    if iters == 0:
        return dZ
    gu = G.sum(axis=1)
    gv = G.sum(axis=0)
    for t in range(iters, 0, -1):
        u_t, v_prev = us[t - 1], vs[t - 1]
        x = Z + u_t[:, None]
        pc = np.exp(x - logsumexp(x, axis=0)[None, :])          # columns sum to 1
        dZ -= pc * gv[None, :]
        gu = gu - (pc * gv[None, :]).sum(axis=1)
        y = Z + v_prev[None, :]
        pr = np.exp(y - logsumexp(y, axis=1)[:, None])          # rows sum to 1
        dZ -= pr * gu[:, None]
        gv = -(pr * gu[:, None]).sum(axis=0)
        gu = np.zeros_like(gu)
    return dZ


# --------------------------------------------------------------------------- adaptive depth
def confidence_threshold(layer, n_layers):
    """Per-layer exit threshold lambda_l = clip(0.8 + 0.1 exp(-4 l / L), 0, 1)
    [LightGlue review, section 2.6 自适应深度, confidence_threshold].
    Pinned by the two values the section prints (l = 1 and l = 9 of L = 9)."""
    return float(np.clip(0.8 + 0.1 * math.exp(-4.0 * layer / n_layers), 0.0, 1.0))


def token_confidence(x, w, b):
    """Per-point confidence c_i = sigmoid(w . x_i + b) of the classifier after a
    layer [LightGlue review, section 2.6: one confidence per point after every
    layer but the last; section 2.5: the classifier is a linear layer and a
    sigmoid on the layer's state]."""
    z = _as64(x) @ _as64(w) + float(b)
    e = np.exp(-np.abs(z))                       # no overflow for large |z|
    return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def check_if_stop(confidences, layer, n_layers, depth_confidence, num_points):
    """Stop after `layer` when the share of points whose confidence is not below
    the layer's threshold exceeds depth_confidence (strict) [LightGlue review,
    section 2.6, check_if_stop]: ratio = 1 - #(c < lambda_l) / num_points."""
    lam = confidence_threshold(layer, n_layers)
    ratio = 1.0 - float(np.sum(np.asarray(confidences) < lam)) / float(num_points)
    return ratio > depth_confidence


def attentional_gnn_adaptive(xs0, xs1, weights, heads, eps, depth_confidence, n_stages=None,
                             width_confidence=None, pruning_threshold=1536):
    """The stages of attentional_gnn for a batch of pairs (lists of states), with
    the adaptive-depth exit [LightGlue review, section 2.6] and, when
    width_confidence > 0, point pruning [section 2.7].  A layer is one (self,
    cross) pair of stages.  After layer l < L - 1:

    * exit: the confidences of every remaining point of every pair decide one
      stop for the whole batch; the share is 1 - #(c < lambda_l) / num_points
      with num_points the original point count (the listing passes m + n, so a
      pruned point counts as confident).  Reading: for a batch, num_points is
      all B (M + N) original points; for B = 1 it is the pages' m + n.
    * pruning (if the run goes on): each image of each pair with more than
      pruning_threshold remaining points keeps the points that
      get_pruning_mask keeps (matchability from the layer's head,
      weights["mt_w"][l], weights["mt_b"][l]; confidences only when the exit
      is enabled); the others leave every later layer (as queries and keys).

    Returns (xs0, xs1, kept0, kept1, layers_run); kept* are the original
    indices of the points still present, in order."""
    stages = weights["stages"]
    if n_stages is None:
        n_stages = len(stages)
    n_layers = n_stages // 2
    depth = depth_confidence is not None and depth_confidence > 0
    width = width_confidence is not None and width_confidence > 0
    xs0, xs1 = list(xs0), list(xs1)
    kept0 = [np.arange(len(x)) for x in xs0]
    kept1 = [np.arange(len(x)) for x in xs1]
    num_points = sum(len(x) for x in xs0) + sum(len(x) for x in xs1)
    for layer in range(n_layers):
        if any(len(x) == 0 for x in xs0) or any(len(x) == 0 for x in xs1):
            # a pair without points left: no more layers (reading: the count
            # reported is the layers that ran)
            return xs0, xs1, kept0, kept1, layer
        for s in (2 * layer, 2 * layer + 1):
            for b in range(len(xs0)):
                x0, x1 = xs0[b], xs1[b]
                src0, src1 = (x1, x0) if s % 2 == 1 else (x0, x1)
                d0 = attentional_propagation(x0, src0, stages[s], heads, eps)
                d1 = attentional_propagation(x1, src1, stages[s], heads, eps)
                xs0[b], xs1[b] = x0 + d0, x1 + d1
        if layer == n_layers - 1:
            continue                             # no exit and no pruning after the last layer
        conf0 = conf1 = None
        if depth:
            conf0 = [token_confidence(x, weights["tc_w"][layer], weights["tc_b"][layer]) for x in xs0]
            conf1 = [token_confidence(x, weights["tc_w"][layer], weights["tc_b"][layer]) for x in xs1]
            if check_if_stop(np.concatenate(conf0 + conf1), layer, n_layers, depth_confidence, num_points):
                return xs0, xs1, kept0, kept1, layer + 1
        if width:
            for b in range(len(xs0)):
                for xs, kept, conf in ((xs0, kept0, conf0), (xs1, kept1, conf1)):
                    if len(xs[b]) <= pruning_threshold:
                        continue
                    scores = matchability(xs[b], weights["mt_w"][layer], weights["mt_b"][layer])
                    keep = get_pruning_mask(None if conf is None else conf[b], scores, layer, n_layers,
                                            width_confidence)
                    xs[b], kept[b] = xs[b][keep], kept[b][keep]
    return xs0, xs1, kept0, kept1, n_layers


def matchability(x, w, b):
    """sigmoid(w . x + b): the matchability of the layer's assignment head
    [LightGlue review, section 2.4, MatchAssignment.get_matchability]."""
    z = _as64(x) @ _as64(w) + float(b)
    e = np.exp(-np.abs(z))
    return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def get_pruning_mask(confidences, scores, layer, n_layers, width_confidence):
    """Points kept for the next layer: matchability above 1 - width_confidence,
    and every point whose confidence is not above the layer's threshold (an
    uncertain point is never pruned) [LightGlue review, section 2.7,
    get_pruning_mask]."""
    keep = np.asarray(scores) > (1.0 - width_confidence)
    if confidences is not None:
        keep = keep | (np.asarray(confidences) <= confidence_threshold(layer, n_layers))
    return keep


# --------------------------------------------------------------------------- whole pass
def matching_head(x0, x1, weights, head="sinkhorn", iters=100, threshold=0.2):
    """Score matrix + dustbin + log-Sinkhorn, or the double-softmax head, then the
    mutual extraction, on the final GNN states of one pair."""
    if head == "double_softmax":
        logP, sim, z0, z1 = double_softmax_head(x0, x1, weights["lg_Wp"], weights["lg_bp"],
                                                weights["lg_wz"], weights["lg_bz"])
        m0, m1, s0, s1 = extract_matches(logP, threshold)
        return {"log_P": logP, "matches0": m0, "matches1": m1, "mscores0": s0, "mscores1": s1,
                "scores": sim, "z0": z0, "z1": z1}
    S = score_matrix(x0, x1, weights["Wf"], weights["bf"])
    logP = log_optimal_transport(S, float(weights["bin_score"]), iters)
    m0, m1, s0, s1 = extract_matches(logP, threshold)
    return {"log_P": logP, "matches0": m0, "matches1": m1, "mscores0": s0, "mscores1": s1,
            "scores": S}


def superglue_pair(kpts0, conf0, desc0, kpts1, conf1, desc1, weights,
                   img_w=640.0, img_h=480.0, heads=4, iters=100,
                   threshold=0.2, eps=1e-5, norm_mode=0, n_stages=None, head="sinkhorn"):
    """One pair through the whole matcher.  Inputs point-major: kpts (n, 2) px,
    conf (n,), desc (n, D).  Returns a dict with log_P ((M+1) x (N+1)),
    matches0/1, mscores0/1.  head="double_softmax" replaces the score matrix,
    dustbin and Sinkhorn by the double-softmax head on the same GNN states
    (extraction unchanged; LightGlue's default threshold is 0.1).

    Empty input (M == 0 or N == 0): matches -1 and scores 0, no log_P
    [Jazihars notes, forward(), the "no keypoints" early return]."""
    M, N = len(kpts0), len(kpts1)
    if M == 0 or N == 0:
        return {"log_P": None,
                "matches0": np.full(M, -1, np.int32), "matches1": np.full(N, -1, np.int32),
                "mscores0": np.zeros(M, F64), "mscores1": np.zeros(N, F64)}
    k0 = normalize_keypoints(kpts0, img_w, img_h, norm_mode)
    k1 = normalize_keypoints(kpts1, img_w, img_h, norm_mode)
    x0 = keypoint_encoder(k0, conf0, desc0, weights, eps)
    x1 = keypoint_encoder(k1, conf1, desc1, weights, eps)
    x0, x1 = attentional_gnn(x0, x1, weights, heads, eps, n_stages)
    return matching_head(x0, x1, weights, head, iters, threshold)


def superglue_batch_adaptive(batch, weights, depth_confidence, img_w=640.0, img_h=480.0, heads=4,
                             iters=100, threshold=0.2, eps=1e-5, norm_mode=0, n_stages=None,
                             head="sinkhorn", width_confidence=None, pruning_threshold=1536):
    """A whole batch (pairs of equal, non-zero M and N) with the adaptive-depth
    exit decided over the batch and optional point pruning; returns (list of
    per-pair results, layers run).  With pruning, the head runs on the points
    left after the last layer and its matches are mapped back to the original
    indices [LightGlue review, section 2.7: prune0/prune1 and the map back];
    a pruned point is unmatched (-1, score 0); log_P covers the points left,
    listed in "kept0" / "kept1"."""
    B = batch["kpts0"].shape[0]
    xs0, xs1 = [], []
    for b in range(B):
        k0 = normalize_keypoints(batch["kpts0"][b], img_w, img_h, norm_mode)
        k1 = normalize_keypoints(batch["kpts1"][b], img_w, img_h, norm_mode)
        xs0.append(keypoint_encoder(k0, batch["conf0"][b], batch["desc0"][b], weights, eps))
        xs1.append(keypoint_encoder(k1, batch["conf1"][b], batch["desc1"][b], weights, eps))
    M, N = len(xs0[0]), len(xs1[0])
    xs0, xs1, kept0, kept1, layers = attentional_gnn_adaptive(
        xs0, xs1, weights, heads, eps, depth_confidence, n_stages, width_confidence, pruning_threshold)
    out = []
    for b in range(B):
        m0 = np.full(M, -1, np.int32)
        m1 = np.full(N, -1, np.int32)
        s0 = np.zeros(M, F64)
        s1 = np.zeros(N, F64)
        res = {"log_P": None, "kept0": kept0[b], "kept1": kept1[b]}
        if len(kept0[b]) and len(kept1[b]):
            r = matching_head(xs0[b], xs1[b], weights, head, iters, threshold)
            sub0, sub1 = r["matches0"], r["matches1"]
            m0[kept0[b]] = np.where(sub0 >= 0, kept1[b][np.maximum(sub0, 0)], -1)
            m1[kept1[b]] = np.where(sub1 >= 0, kept0[b][np.maximum(sub1, 0)], -1)
            s0[kept0[b]] = r["mscores0"]
            s1[kept1[b]] = r["mscores1"]
            res.update({k: v for k, v in r.items() if k not in ("matches0", "matches1", "mscores0", "mscores1")})
        res.update({"matches0": m0, "matches1": m1, "mscores0": s0, "mscores1": s1})
        out.append(res)
    return out, layers


def superglue_batch(batch, weights, pairs=None, **kw):
    """Run superglue_pair on the pairs of a stacked batch (all, or a subset)."""
    B = batch["kpts0"].shape[0]
    idx = range(B) if pairs is None else pairs
    return [superglue_pair(batch["kpts0"][b], batch["conf0"][b], batch["desc0"][b],
                           batch["kpts1"][b], batch["conf1"][b], batch["desc1"][b],
                           weights, **kw) for b in idx]
