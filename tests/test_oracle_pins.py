"""Pins of the float64 oracle against things other than itself: values the pages
print, library routines (torch float64 modules), closed forms, invariants and
brute force.  CPU only."""
import itertools
import math

import numpy as np
import pytest
import torch

from conftest import golden_path
from oracle import superglue_oracle as O
from learned_sparse_feature_b200 import synth


def _read_golden(name):
    rows = []
    with open(golden_path(name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# --------------------------------------------------------------------------- printed values
def test_normalize_keypoints_printed_values():
    rows = np.array(_read_golden("normalize_keypoints_427x640.txt"), float)
    out = O.normalize_keypoints(rows[:, :2], width=640.0, height=427.0, mode=0)
    # outputs printed to 5 significant digits, inputs to 1e-4 px (/448 px)
    tol = 5e-5 * np.abs(rows[:, 2:]) + 1.2e-7
    assert np.all(np.abs(out - rows[:, 2:]) <= tol)


def test_normalize_mode1_is_long_side_unit_range():
    corners = np.array([[0.0, 0.0], [640.0, 480.0]])
    out = O.normalize_keypoints(corners, 640.0, 480.0, mode=1)
    np.testing.assert_allclose(out, [[-1.0, -0.75], [1.0, 0.75]], rtol=0, atol=1e-15)


def test_attention_worked_example():
    g = {r[0]: [float(v) for v in r[1:]] for r in _read_golden("attention_worked_example.txt")
         if r[0] != "value"}
    values = np.array([[float(v) for v in r[1:]] for r in _read_golden("attention_worked_example.txt")
                       if r[0] == "value"])
    w = O.softmax(np.array(g["scores"]))
    np.testing.assert_allclose(w, g["weights"], atol=5e-4)
    # same example through one attention head: d_k = 1, q = 1, k_j = score_j
    q = np.array([[1.0]])
    k = np.array(g["scores"])[:, None]
    msg, alpha = O.attend(q, k, values)
    np.testing.assert_allclose(alpha[0], g["weights"], atol=5e-4)
    np.testing.assert_allclose(msg[0], g["message"], atol=5e-4)


def test_attention_scale_uses_key_width():
    # d_k = 4: q.k = 8 for the first key -> e = 8 / sqrt(4) = 4
    q = np.array([[1.0, 1.0, 1.0, 1.0]])
    k = np.array([[2.0, 2.0, 2.0, 2.0], [0.0, 0.0, 0.0, 0.0]])
    _, alpha = O.attend(q, k, np.eye(2))
    np.testing.assert_allclose(alpha[0, 0], 1.0 / (1.0 + math.exp(-4.0)), rtol=1e-14)


# --------------------------------------------------------------------------- library pins
def _torch_mlp(Ws, bs, bns, eps):
    layers = []
    n = len(Ws)
    for l in range(n):
        conv = torch.nn.Conv1d(Ws[l].shape[1], Ws[l].shape[0], kernel_size=1, bias=True).double()
        conv.weight.data = torch.tensor(np.asarray(Ws[l], float))[:, :, None]
        conv.bias.data = torch.tensor(np.asarray(bs[l], float))
        layers.append(conv)
        if l < n - 1:
            bn = torch.nn.BatchNorm1d(Ws[l].shape[0], eps=eps).double()
            g, b, m, v = (torch.tensor(np.asarray(a, float)) for a in bns[l])
            bn.weight.data, bn.bias.data = g, b
            bn.running_mean.data, bn.running_var.data = m, v
            layers.append(bn)
            layers.append(torch.nn.ReLU())
    return torch.nn.Sequential(*layers).eval()


def test_batchnorm_matches_torch(weights):
    rng = np.random.default_rng(1)
    z = rng.standard_normal((50, 32))
    stats = weights["enc_bn"][0]
    bn = torch.nn.BatchNorm1d(32, eps=1e-5).double().eval()
    bn.weight.data, bn.bias.data = (torch.tensor(np.asarray(a, float)) for a in stats[:2])
    bn.running_mean.data, bn.running_var.data = (torch.tensor(np.asarray(a, float)) for a in stats[2:])
    with torch.no_grad():
        ref = bn(torch.tensor(z)).numpy()
    np.testing.assert_allclose(O.batchnorm_eval(z, *stats, 1e-5), ref, rtol=1e-13, atol=1e-13)


def test_batchnorm_identity_stats_is_plain_scaling():
    z = np.linspace(-3, 3, 12).reshape(4, 3)
    one, zero = np.ones(3), np.zeros(3)
    np.testing.assert_allclose(O.batchnorm_eval(z, one, zero, zero, one, 1e-5),
                               z / math.sqrt(1.0 + 1e-5), rtol=1e-15)


def test_encoder_mlp_matches_torch_modules(weights):
    rng = np.random.default_rng(2)
    p = rng.uniform(-0.7, 0.7, (40, 3))
    net = _torch_mlp(weights["enc_W"], weights["enc_b"], weights["enc_bn"], 1e-5)
    with torch.no_grad():
        ref = net(torch.tensor(p.T[None]))[0].numpy().T      # channels-first in torch
    out = O.mlp(p, weights["enc_W"], weights["enc_b"], weights["enc_bn"], 1e-5)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_keypoint_encoder_adds_descriptor(weights):
    rng = np.random.default_rng(3)
    k = rng.uniform(-0.7, 0.7, (10, 2))
    c = rng.uniform(0, 1, 10)
    d = rng.standard_normal((10, 256))
    net = _torch_mlp(weights["enc_W"], weights["enc_b"], weights["enc_bn"], 1e-5)
    inp = torch.cat([torch.tensor(k.T[None]), torch.tensor(c[None, None])], dim=1)
    with torch.no_grad():
        ref = d + net(inp)[0].numpy().T
    np.testing.assert_allclose(O.keypoint_encoder(k, c, d, weights, 1e-5), ref, rtol=1e-12, atol=1e-12)


def _torch_mha(st, d=256, heads=4):
    mha = torch.nn.MultiheadAttention(d, heads, bias=True, batch_first=True).double().eval()
    W = np.concatenate([st["Wq"], st["Wk"], st["Wv"]]).astype(float)
    b = np.concatenate([st["bq"], st["bk"], st["bv"]]).astype(float)
    mha.in_proj_weight.data = torch.tensor(W)
    mha.in_proj_bias.data = torch.tensor(b)
    mha.out_proj.weight.data = torch.tensor(np.asarray(st["Wm"], float))
    mha.out_proj.bias.data = torch.tensor(np.asarray(st["bm"], float))
    return mha


def test_multi_head_attention_matches_torch(weights):
    rng = np.random.default_rng(4)
    x = rng.standard_normal((17, 256)) * 0.3
    src = rng.standard_normal((23, 256)) * 0.3
    st = weights["stages"][0]
    mha = _torch_mha(st)
    with torch.no_grad():
        ref, _ = mha(torch.tensor(x[None]), torch.tensor(src[None]), torch.tensor(src[None]))
    np.testing.assert_allclose(O.multi_head_attention(x, src, st, 4), ref[0].numpy(),
                               rtol=1e-11, atol=1e-12)


def test_attentional_propagation_matches_torch(weights):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((19, 256)) * 0.3
    src = rng.standard_normal((11, 256)) * 0.3
    st = weights["stages"][3]
    mha = _torch_mha(st)
    net = _torch_mlp([st["W1"], st["W2"]], [st["b1"], st["b2"]], [st["bn1"]], 1e-5)
    with torch.no_grad():
        m, _ = mha(torch.tensor(x[None]), torch.tensor(src[None]), torch.tensor(src[None]))
        z = torch.cat([torch.tensor(x[None]), m], dim=2).transpose(1, 2)
        ref = net(z)[0].numpy().T
    np.testing.assert_allclose(O.attentional_propagation(x, src, st, 4, 1e-5), ref,
                               rtol=1e-10, atol=1e-12)


def test_sinkhorn_logsumexp_matches_torch():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((7, 9)) * 30
    np.testing.assert_allclose(O.logsumexp(x, 1), torch.logsumexp(torch.tensor(x), 1).numpy(), rtol=1e-14)
    np.testing.assert_allclose(O.logsumexp(x, 0), torch.logsumexp(torch.tensor(x), 0).numpy(), rtol=1e-14)


# --------------------------------------------------------------------------- GNN structure
def _pair(n0, n1, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((n0, 256)) * 0.3, rng.standard_normal((n1, 256)) * 0.3)


def test_self_stage_reads_only_own_image(weights):
    x0, x1 = _pair(9, 7, 7)
    a0, _ = O.attentional_gnn(x0, x1, weights, 4, 1e-5, n_stages=1)
    b0, _ = O.attentional_gnn(x0, x1 * 2.0 + 0.1, weights, 4, 1e-5, n_stages=1)
    np.testing.assert_array_equal(a0, b0)


def test_cross_stage_reads_other_image(weights):
    x0, x1 = _pair(9, 7, 8)
    a0, _ = O.attentional_gnn(x0, x1, weights, 4, 1e-5, n_stages=2)
    b0, _ = O.attentional_gnn(x0, x1 * 2.0 + 0.1, weights, 4, 1e-5, n_stages=2)
    assert np.abs(a0 - b0).max() > 1e-3


def test_gnn_is_symmetric_in_the_two_images(weights):
    # shared weights + simultaneous update: swapping the images swaps the outputs
    x0, x1 = _pair(9, 7, 9)
    a0, a1 = O.attentional_gnn(x0, x1, weights, 4, 1e-5, n_stages=4)
    b1, b0 = O.attentional_gnn(x1, x0, weights, 4, 1e-5, n_stages=4)
    np.testing.assert_allclose(a0, b0, rtol=0, atol=1e-13)
    np.testing.assert_allclose(a1, b1, rtol=0, atol=1e-13)


def test_cross_stage_equals_self_stage_on_the_other_source(weights):
    # a single cross stage on (x0, x1) gives A the delta a self stage would give
    # a query set x0 attending to x1, i.e. attentional_propagation(x0, x1)
    x0, x1 = _pair(6, 8, 10)
    st = weights["stages"][1]
    y0, y1 = O.attentional_gnn(x0, x1, {"stages": [weights["stages"][0], st]}, 4, 1e-5, n_stages=2)
    s0, s1 = O.attentional_gnn(x0, x1, weights, 4, 1e-5, n_stages=1)
    np.testing.assert_allclose(y0 - s0, O.attentional_propagation(s0, s1, st, 4, 1e-5), atol=1e-13)
    np.testing.assert_allclose(y1 - s1, O.attentional_propagation(s1, s0, st, 4, 1e-5), atol=1e-13)


# --------------------------------------------------------------------------- Sinkhorn
def test_marginals_sum_to_one():
    for M, N in [(1, 1), (5, 3), (64, 100)]:
        lm, ln, norm = O.log_marginals(M, N)
        assert abs(np.exp(lm).sum() - 1) < 1e-14 and abs(np.exp(ln).sum() - 1) < 1e-14
        assert abs(norm + math.log(M + N)) < 1e-15


@pytest.mark.parametrize("s,z", [(3.0, 1.0), (-2.0, 1.0), (0.5, -4.0)])
def test_sinkhorn_one_by_one_closed_form(s, z):
    # S_bar = [[s, z], [z, z]], all marginals 1: fixed point [[p, 1-p], [1-p, p]]
    # with cross-ratio p^2 / (1-p)^2 = exp(s - z), i.e. p = sigmoid((s - z) / 2)
    P = np.exp(O.log_optimal_transport(np.array([[s]]), z, iters=200))
    p = 1.0 / (1.0 + math.exp(-(s - z) / 2.0))
    np.testing.assert_allclose(P, [[p, 1 - p], [1 - p, p]], rtol=0, atol=1e-12)


@pytest.mark.parametrize("T", [1, 7])
def test_sinkhorn_constant_scores_closed_form(T):
    M, N, z = 5, 3, 0.7
    logP = O.log_optimal_transport(np.full((M, N), z), z, iters=T)
    a = np.r_[np.ones(M), N]
    b = np.r_[np.ones(N), M]
    np.testing.assert_allclose(np.exp(logP), np.outer(a, b) / (M + N), rtol=1e-13)


def test_sinkhorn_column_marginals_exact_and_rows_converge():
    rng = np.random.default_rng(11)
    M, N = 13, 9
    S = rng.standard_normal((M, N)) * 3
    a = np.r_[np.ones(M), N]
    b = np.r_[np.ones(N), M]
    prev = np.inf
    for T in (1, 3, 10, 30, 100):
        P = np.exp(O.log_optimal_transport(S, 1.0, T))
        np.testing.assert_allclose(P.sum(0), b, rtol=1e-12)       # v is updated last
        res = np.abs(P.sum(1) - a).max()
        assert res <= prev + 1e-15
        prev = res
    assert prev < 1e-6


def _best_partial_assignment(S, z):
    """Brute force: the partial injection maximising sum (S_ij - z)."""
    M, N = S.shape
    best, arg = -np.inf, None
    for k in range(0, min(M, N) + 1):
        for rows in itertools.combinations(range(M), k):
            for cols in itertools.permutations(range(N), k):
                val = sum(S[i, j] - z for i, j in zip(rows, cols))
                if val > best + 1e-12:
                    best, arg = val, dict(zip(rows, cols))
    return best, arg


def _second_best_gap(S, z, best):
    M, N = S.shape
    vals = []
    for k in range(0, min(M, N) + 1):
        for rows in itertools.combinations(range(M), k):
            for cols in itertools.permutations(range(N), k):
                vals.append(sum(S[i, j] - z for i, j in zip(rows, cols)))
    vals = np.sort(np.array(vals))[::-1]
    return best - vals[1] if len(vals) > 1 else np.inf


def test_sinkhorn_low_temperature_is_optimal_partial_assignment():
    rng = np.random.default_rng(12)
    eps, z = 0.02, 1.0
    checked = 0
    for trial in range(200):
        M, N = rng.integers(1, 5), rng.integers(1, 5)
        S = rng.uniform(-1.0, 4.0, (M, N))
        best, assign = _best_partial_assignment(S, z)
        if _second_best_gap(S, z, best) < 0.5:
            continue
        P = np.exp(O.log_optimal_transport(S / eps, z / eps, iters=3000))
        for i in range(M):
            j = assign.get(i, N)                       # N = dustbin column
            assert P[i, j] > 0.95, (trial, i, j, P)
        for j in range(N):
            i = {c: r for r, c in assign.items()}.get(j, M)
            assert P[i, j] > 0.95
        checked += 1
        if checked >= 25:
            break
    assert checked >= 25


# --------------------------------------------------------------------------- extraction
def test_extraction_hand_built():
    thr = 0.2
    # real block 4 x 4 (+ dustbin row/col).  Probabilities, then log.
    P = np.full((5, 5), 1e-3)
    P[0, 1] = 0.90      # row 0 <-> col 1 mutual, above threshold
    P[1, 0] = 0.15      # row 1 <-> col 0 mutual, below threshold
    P[1, 4] = 0.80      # row 1's best is the dustbin; real argmax still col 0
    P[2, 2] = 0.50      # row 2 -> col 2, but col 2's best is row 3: not mutual
    P[3, 2] = 0.60
    P[3, 3] = 0.55      # row 3 -> col 2 (0.60 > 0.55); col 3 -> row 3 (not mutual for col 3)
    P[2, 3] = 0.30
    logP = np.log(P)
    m0, m1, s0, s1 = O.extract_matches(logP, thr)
    np.testing.assert_array_equal(m0, [1, -1, -1, 2])
    np.testing.assert_array_equal(m1, [-1, 0, 3, -1])
    np.testing.assert_allclose(s0, [0.90, 0.15, 0.0, 0.60], rtol=1e-12)
    np.testing.assert_allclose(s1, [0.15, 0.90, 0.60, 0.0], rtol=1e-12)


def test_extraction_ties_take_lowest_index_and_threshold_is_strict():
    P = np.full((3, 3), 0.01)
    P[0, 0] = P[0, 1] = 0.5     # tie in row 0 -> col 0; col 0 -> row 0 (mutual)
    logP = np.log(P)
    at = float(np.exp(logP[0, 0]))                   # the score row 0 will get
    m0, m1, s0, _ = O.extract_matches(logP, at)      # exactly at threshold: rejected
    assert m0[0] == -1 and s0[0] == at
    m0, m1, _, _ = O.extract_matches(logP, 0.49)
    assert m0[0] == 0 and m1[0] == 0 and m1[1] == -1


def test_empty_input(weights):
    r = O.superglue_pair(np.zeros((0, 2)), np.zeros(0), np.zeros((0, 256)),
                         np.ones((3, 2)), np.ones(3), np.ones((3, 256)), weights)
    assert r["log_P"] is None
    np.testing.assert_array_equal(r["matches1"], [-1, -1, -1])
    np.testing.assert_array_equal(r["mscores1"], [0, 0, 0])
    assert r["matches0"].shape == (0,)


# --------------------------------------------------------------------------- whole network
def test_full_network_permutation_equivariance(weights):
    batch = synth.make_batch("pair64_fp32")
    k0, c0, d0 = batch["kpts0"][0], batch["conf0"][0], batch["desc0"][0]
    k1, c1, d1 = batch["kpts1"][0][:48], batch["conf1"][0][:48], batch["desc1"][0][:48]
    ref = O.superglue_pair(k0, c0, d0, k1, c1, d1, weights, n_stages=4)
    rng = np.random.default_rng(13)
    pa, pb = rng.permutation(len(k0)), rng.permutation(len(k1))
    out = O.superglue_pair(k0[pa], c0[pa], d0[pa], k1[pb], c1[pb], d1[pb], weights, n_stages=4)
    ra = np.r_[pa, len(k0)]
    rb = np.r_[pb, len(k1)]
    np.testing.assert_allclose(out["log_P"], ref["log_P"][np.ix_(ra, rb)], rtol=0, atol=1e-10)
    inv_b = np.argsort(pb)
    inv_a = np.argsort(pa)
    exp0 = np.where(ref["matches0"][pa] >= 0, inv_b[np.maximum(ref["matches0"][pa], 0)], -1)
    exp1 = np.where(ref["matches1"][pb] >= 0, inv_a[np.maximum(ref["matches1"][pb], 0)], -1)
    np.testing.assert_array_equal(out["matches0"], exp0)
    np.testing.assert_array_equal(out["matches1"], exp1)


def test_score_matrix_scale_matches_library_attention(weights):
    # softmax_j(S_ij) with S = <f_i^A, f_j^B> / sqrt(D) is exactly what the library's
    # scaled-dot-product attention computes for q = f^A, k = f^B, v = I (default
    # scale 1/sqrt(D)).  Softmax is shift- but not scale-invariant, so this pins
    # the 1/sqrt(D) factor and the operand order.
    rng = np.random.default_rng(14)
    x0 = rng.standard_normal((6, 256)) * 0.3
    x1 = rng.standard_normal((9, 256)) * 0.3
    S = O.score_matrix(x0, x1, weights["Wf"], weights["bf"])
    f0 = O.linear(x0, weights["Wf"], weights["bf"])
    f1 = O.linear(x1, weights["Wf"], weights["bf"])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(f0[None]), torch.tensor(f1[None]), torch.eye(9, dtype=torch.float64)[None])[0]
    np.testing.assert_allclose(O.softmax(S, axis=1), ref.numpy(), rtol=1e-10, atol=1e-13)


# --------------------------------------------------------------------------- double-softmax head
def _dsm_inputs(seed=3, M=5, N=4):
    rng = np.random.default_rng(seed)
    return rng.normal(0, 2.0, (M, N)), rng.normal(0, 1.5, M), rng.normal(0, 1.5, N)


def test_double_softmax_matches_torch_log_softmax_and_logsigmoid():
    import torch.nn.functional as F
    sim, z0, z1 = _dsm_inputs()
    M, N = sim.shape
    got = O.double_softmax_log_assignment(sim, z0, z1)
    s = torch.from_numpy(sim)
    a, b = torch.from_numpy(z0), torch.from_numpy(z1)
    real = F.log_softmax(s, 1) + F.log_softmax(s, 0) + F.logsigmoid(a)[:, None] + F.logsigmoid(b)[None, :]
    np.testing.assert_allclose(got[:M, :N], real.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[:M, N], F.logsigmoid(-a).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[M, :N], F.logsigmoid(-b).numpy(), rtol=0, atol=1e-12)
    assert got[M, N] == 0.0


def test_double_softmax_two_by_two_closed_form():
    # sim = [[1, 0], [0, 2]], z0 = (0, ln 3), z1 = (ln 2, 0): every entry by hand
    sim = np.array([[1.0, 0.0], [0.0, 2.0]])
    z0 = np.array([0.0, math.log(3.0)])
    z1 = np.array([math.log(2.0), 0.0])
    e = math.e
    sig = lambda t: 1.0 / (1.0 + math.exp(-t))
    row = [[e / (e + 1), 1 / (e + 1)], [1 / (1 + e * e), e * e / (1 + e * e)]]
    col = [[e / (e + 1), 1 / (1 + e * e)], [1 / (e + 1), e * e / (1 + e * e)]]
    got = np.exp(O.double_softmax_log_assignment(sim, z0, z1))
    for i in range(2):
        for j in range(2):
            want = row[i][j] * col[i][j] * sig(z0[i]) * sig(z1[j])
            assert abs(got[i, j] - want) < 1e-14
    assert abs(got[0, 2] - 0.5) < 1e-15 and abs(got[1, 2] - 0.25) < 1e-15
    assert abs(got[2, 0] - 1.0 / 3.0) < 1e-15 and abs(got[2, 1] - 0.5) < 1e-15
    assert got[2, 2] == 1.0


def test_log_sigmoid_is_stable_and_complements():
    x = np.array([-60.0, -5.0, -1e-3, 0.0, 2.0, 60.0])
    ls = O.log_sigmoid(x)
    assert np.all(np.isfinite(ls))
    assert abs(ls[0] - (-60.0 - math.exp(-60.0))) < 1e-12
    assert abs(ls[-1] + math.exp(-60.0)) < 1e-30
    np.testing.assert_allclose(np.exp(ls) + np.exp(O.log_sigmoid(-x)), 1.0, rtol=0, atol=1e-15)


def test_double_softmax_head_matches_torch_modules(weights):
    rng = np.random.default_rng(11)
    x0 = rng.normal(0, 1, (7, synth.D))
    x1 = rng.normal(0, 1, (6, synth.D))
    logP, sim, z0, z1 = O.double_softmax_head(x0, x1, weights["lg_Wp"], weights["lg_bp"],
                                              weights["lg_wz"], weights["lg_bz"])
    with torch.no_grad():
        proj = torch.nn.Linear(synth.D, synth.D).double()
        proj.weight.copy_(torch.from_numpy(np.asarray(weights["lg_Wp"], np.float64)))
        proj.bias.copy_(torch.from_numpy(np.asarray(weights["lg_bp"], np.float64)))
        mz = torch.nn.Linear(synth.D, 1).double()
        mz.weight.copy_(torch.from_numpy(np.asarray(weights["lg_wz"], np.float64))[None, :])
        mz.bias.fill_(float(weights["lg_bz"]))
        t0, t1 = torch.from_numpy(x0), torch.from_numpy(x1)
        m0 = proj(t0) / synth.D ** 0.25
        m1 = proj(t1) / synth.D ** 0.25
        want_sim = torch.einsum("md,nd->mn", m0, m1).numpy()
        want_z0 = mz(t0)[:, 0].numpy()
        want_z1 = mz(t1)[:, 0].numpy()
    np.testing.assert_allclose(sim, want_sim, rtol=1e-12, atol=1e-10)
    np.testing.assert_allclose(z0, want_z0, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z1, want_z1, rtol=1e-12, atol=1e-12)


def test_double_softmax_recovers_a_planted_permutation():
    # a sharp permutation similarity and confident points: the head's mutual
    # argmax is the permutation, each with probability near 1
    perm = np.array([2, 0, 3, 1])
    sim = np.full((4, 4), -10.0)
    sim[np.arange(4), perm] = 10.0
    logP = O.double_softmax_log_assignment(sim, np.full(4, 20.0), np.full(4, 20.0))
    m0, m1, s0, _ = O.extract_matches(logP, 0.1)
    np.testing.assert_array_equal(m0, perm)
    np.testing.assert_array_equal(m1[perm], np.arange(4))
    assert np.all(s0 > 0.99)


# --------------------------------------------------------------------------- adaptive depth
def test_confidence_threshold_printed_values():
    # the two thresholds the LightGlue review prints (section 2.6), to 3 decimals,
    # and the l = 0 closed form 0.8 + 0.1
    for row in _read_golden("confidence_threshold_lightglue.txt"):
        _, layer, n_layers, value = row
        assert abs(O.confidence_threshold(int(layer), int(n_layers)) - float(value)) < 5e-4
    assert O.confidence_threshold(0, 9) == pytest.approx(0.9, abs=1e-15)
    seq = [O.confidence_threshold(l, 9) for l in range(10)]
    assert all(a > b for a, b in zip(seq, seq[1:]))


def test_check_if_stop_counts_strictly():
    lam = O.confidence_threshold(2, 9)
    # 20 points: 19 at exactly the threshold (not below it: confident) and one below
    conf = np.full(20, lam)
    conf[3] = lam - 1e-9
    assert O.check_if_stop(conf, 2, 9, 0.9, 20)          # ratio 0.95 > 0.9
    assert not O.check_if_stop(conf, 2, 9, 0.95, 20)     # ratio 0.95 is not above 0.95
    assert not O.check_if_stop(conf, 2, 9, 0.96, 20)
    assert O.check_if_stop(np.full(5, 1.0), 8, 9, 0.99, 5)
    assert not O.check_if_stop(np.full(5, 0.5), 0, 9, 0.0, 5)   # every point below 0.9


def test_token_confidence_matches_torch_linear_sigmoid():
    rng = np.random.default_rng(41)
    x = rng.standard_normal((33, 256))
    w = rng.standard_normal(256) * 0.1
    b = 0.37
    lin = torch.nn.Linear(256, 1).double()
    with torch.no_grad():
        lin.weight.copy_(torch.from_numpy(w)[None])
        lin.bias.fill_(b)
        ref = torch.sigmoid(lin(torch.from_numpy(x)))[:, 0].numpy()
    np.testing.assert_allclose(O.token_confidence(x, w, b), ref, rtol=0, atol=1e-15)


def _adaptive_inputs(weights, B=2, M=9, N=7, seed=5):
    rng = np.random.default_rng(seed)
    xs0 = [rng.standard_normal((M, 256)) for _ in range(B)]
    xs1 = [rng.standard_normal((N, 256)) for _ in range(B)]
    return xs0, xs1


def test_adaptive_gnn_that_never_stops_is_the_fixed_depth_gnn(weights):
    xs0, xs1 = _adaptive_inputs(weights)
    # ratio > 1 is impossible: every layer runs
    a0, a1, _, _, layers = O.attentional_gnn_adaptive(xs0, xs1, weights, 4, 1e-5, 1.0, n_stages=6)
    assert layers == 3
    for b in range(2):
        r0, r1 = O.attentional_gnn(xs0[b], xs1[b], weights, 4, 1e-5, n_stages=6)
        np.testing.assert_allclose(a0[b], r0, rtol=0, atol=1e-12)
        np.testing.assert_allclose(a1[b], r1, rtol=0, atol=1e-12)


def test_adaptive_gnn_stops_after_the_planted_layer(weights):
    xs0, xs1 = _adaptive_inputs(weights)
    w = dict(weights)
    w["tc_w"] = [np.zeros(256) for _ in range(9)]
    for k in (0, 1, 2):
        # classifiers certain "not confident" before layer k, "confident" at k
        w["tc_b"] = [-50.0 if l < k else 50.0 for l in range(9)]
        a0, a1, _, _, layers = O.attentional_gnn_adaptive(xs0, xs1, w, 4, 1e-5, 0.95, n_stages=8)
        assert layers == k + 1
        for b in range(2):
            r0, r1 = O.attentional_gnn(xs0[b], xs1[b], w, 4, 1e-5, n_stages=2 * k + 2)
            np.testing.assert_allclose(a0[b], r0, rtol=0, atol=1e-12)
            np.testing.assert_allclose(a1[b], r1, rtol=0, atol=1e-12)
    # no exit check after the last layer: a confident last layer changes nothing
    w["tc_b"] = [-50.0, -50.0, -50.0, 50.0] + [50.0] * 5
    assert O.attentional_gnn_adaptive(xs0, xs1, w, 4, 1e-5, 0.95, n_stages=8)[4] == 4


def test_adaptive_decision_pools_the_points_of_the_batch(weights):
    # pair 0's points all confident, pair 1's points all below the threshold
    # (through the sign of one input channel): the pooled share is M0+N0 over
    # all points, so the exit flips exactly where depth_confidence crosses it
    w = dict(weights)
    tw = np.zeros(256)
    tw[0] = 100.0
    w["tc_w"] = [tw] * 9
    w["tc_b"] = [0.0] * 9
    xs0, xs1 = _adaptive_inputs(weights, B=2, M=6, N=4)
    xs0 = [np.abs(xs0[0]) + 50.0, -np.abs(xs0[1]) - 50.0]
    xs1 = [np.abs(xs1[0]) + 50.0, -np.abs(xs1[1]) - 50.0]
    # one stage pair changes the states, so look at the layer-0 confidences
    # after the first layer, as the gnn does
    a0, a1, _, _, _ = O.attentional_gnn_adaptive(xs0, xs1, w, 4, 1e-5, 1.0, n_stages=2)
    conf = np.concatenate([O.token_confidence(np.concatenate([a0[b], a1[b]]), tw, 0.0) for b in range(2)])
    share = 1.0 - np.mean(conf < O.confidence_threshold(0, 2))
    assert 0.0 < share < 1.0
    assert O.attentional_gnn_adaptive(xs0, xs1, w, 4, 1e-5, share - 1e-9, n_stages=4)[4] == 1
    assert O.attentional_gnn_adaptive(xs0, xs1, w, 4, 1e-5, share, n_stages=4)[4] == 2


# --------------------------------------------------------------------------- point pruning
def test_pruning_mask_hand_built():
    lam = O.confidence_threshold(1, 9)
    scores = np.array([0.5, 0.01, 0.001, 0.001, 0.001, 0.0100001])
    conf = np.array([0.99, 0.99, lam, lam + 1e-9, 0.2, 0.99])
    # score above 1 - 0.99 keeps; a confidence not above lambda keeps (never pruned)
    keep = O.get_pruning_mask(conf, scores, 1, 9, 0.99)
    assert keep.tolist() == [True, False, True, False, True, True]
    # without confidences (the exit disabled) only the score decides
    assert O.get_pruning_mask(None, scores, 1, 9, 0.99).tolist() == [True, False, False, False, False, True]
    # strictly above 1 - width_confidence (0.5 is exact in binary)
    assert O.get_pruning_mask(None, np.array([0.5, 0.5000001]), 1, 9, 0.5).tolist() == [False, True]


def test_matchability_matches_torch_linear_sigmoid():
    rng = np.random.default_rng(43)
    x = rng.standard_normal((21, 256))
    w = rng.standard_normal(256) * 0.2
    lin = torch.nn.Linear(256, 1).double()
    with torch.no_grad():
        lin.weight.copy_(torch.from_numpy(w)[None])
        lin.bias.fill_(-0.3)
        ref = torch.sigmoid(lin(torch.from_numpy(x)))[:, 0].numpy()
    np.testing.assert_allclose(O.matchability(x, w, -0.3), ref, rtol=0, atol=1e-15)


def _pruning_weights(weights, n_layers=9):
    # matchability sigmoid(1e4 x[0]): about 1 where channel 0 of the state is
    # positive and about 0 where it is negative (beyond 5e-4 either way)
    w = dict(weights)
    mw = np.zeros(256)
    mw[0] = 1e4
    w["mt_w"] = [mw] * n_layers
    w["mt_b"] = [0.0] * n_layers
    return w


def test_pruning_that_keeps_everything_is_the_unpruned_pass(weights):
    xs0, xs1 = _adaptive_inputs(weights, B=2, M=9, N=7)
    w = weights                                  # generated matchability: every score is above 0
    a = O.attentional_gnn_adaptive(xs0, xs1, w, 4, 1e-5, None, 6, width_confidence=1.0, pruning_threshold=0)
    r = O.attentional_gnn_adaptive(xs0, xs1, w, 4, 1e-5, None, 6)
    for b in range(2):
        np.testing.assert_array_equal(a[2][b], np.arange(9))
        np.testing.assert_allclose(a[0][b], r[0][b], rtol=0, atol=1e-12)
        np.testing.assert_allclose(a[1][b], r[1][b], rtol=0, atol=1e-12)
    # an image with no more points than the threshold is never pruned
    w = _pruning_weights(weights)
    a = O.attentional_gnn_adaptive(xs0, xs1, w, 4, 1e-5, None, 6, width_confidence=0.99, pruning_threshold=9)
    assert all(len(k) == 9 for k in a[2]) and all(len(k) == 7 for k in a[3])


def _pruned_reference(xs0, xs1, w, keep_channel_positive=True):
    """Layer 0 on every point, then layer 1 on the points whose channel 0 is
    positive after layer 0: the pruned two-layer pass written as a composition
    of the fixed-depth GNN."""
    refs = []
    stages_rest = dict(w)
    stages_rest["stages"] = w["stages"][2:]
    for x0, x1 in zip(xs0, xs1):
        y0, y1 = O.attentional_gnn(x0, x1, w, 4, 1e-5, n_stages=2)
        k0, k1 = np.where(y0[:, 0] > 0)[0], np.where(y1[:, 0] > 0)[0]
        margin = min(np.abs(y0[:, 0]).min(), np.abs(y1[:, 0]).min())
        z0, z1 = O.attentional_gnn(y0[k0], y1[k1], stages_rest, 4, 1e-5, n_stages=2)
        refs.append((z0, z1, k0, k1, margin))
    return refs


def test_pruned_points_leave_the_later_layers(weights):
    xs0, xs1 = _adaptive_inputs(weights, B=2, M=12, N=10, seed=8)
    w = _pruning_weights(weights)
    # two layers: pruning after layer 0 only (never after the last layer)
    a0, a1, k0, k1, layers = O.attentional_gnn_adaptive(xs0, xs1, w, 4, 1e-5, None, 4,
                                                          width_confidence=0.99, pruning_threshold=0)
    assert layers == 2
    for b, (z0, z1, r0, r1, margin) in enumerate(_pruned_reference(xs0, xs1, w)):
        assert margin > 2e-3                     # sigmoid(1e4 x) is decidable on both sides
        assert 0 < len(r0) < 12 and 0 < len(r1) < 10
        np.testing.assert_array_equal(k0[b], r0)
        np.testing.assert_array_equal(k1[b], r1)
        np.testing.assert_allclose(a0[b], z0, rtol=0, atol=1e-12)
        np.testing.assert_allclose(a1[b], z1, rtol=0, atol=1e-12)


def test_pruned_points_are_unmatched_and_matches_map_back(weights):
    rng = np.random.default_rng(21)
    pairs = [synth.make_pair(rng, 12, 10, 0.6) for _ in range(2)]
    batch = {k: np.stack([p[k] for p in pairs]) for k in ("kpts0", "conf0", "desc0", "kpts1", "conf1", "desc1")}
    w = _pruning_weights(weights)
    out, layers = O.superglue_batch_adaptive(batch, w, None, n_stages=4, width_confidence=0.99,
                                             pruning_threshold=0)
    for b, res in enumerate(out):
        k0, k1 = res["kept0"], res["kept1"]
        gone0 = np.setdiff1d(np.arange(12), k0)
        gone1 = np.setdiff1d(np.arange(10), k1)
        assert np.all(res["matches0"][gone0] == -1) and np.all(res["mscores0"][gone0] == 0)
        assert np.all(res["matches1"][gone1] == -1) and np.all(res["mscores1"][gone1] == 0)
        assert res["log_P"].shape == (len(k0) + 1, len(k1) + 1)
        # the head on the points left, in their own indices, agrees after the map
        sub = O.extract_matches(res["log_P"], 0.2)
        for p, i in enumerate(k0):
            j = res["matches0"][i]
            assert (j == -1) == (sub[0][p] == -1)
            if j >= 0:
                assert j == k1[sub[0][p]] and res["matches1"][j] == i


def test_exit_share_counts_pruned_points_as_confident(weights):
    # layer 0: confident where channel 1 is positive (about half), matchability
    # 0 everywhere, so exactly the confident points are pruned and the share at
    # layer 0 stays below depth_confidence; layer 1: confident where channel 2
    # is positive.  With the original point count a pruned point counts as
    # confident, which puts the share at layer 1 above the one of the points
    # left alone
    xs0, xs1 = _adaptive_inputs(weights, B=1, M=16, N=14, seed=12)
    w = dict(weights)
    w["mt_w"] = [np.zeros(256)] * 9
    w["mt_b"] = [-50.0] * 9
    t0, t1 = np.zeros(256), np.zeros(256)
    t0[1], t1[2] = 100.0, 100.0
    w["tc_w"] = [t0, t1] + [np.zeros(256)] * 7
    w["tc_b"] = [0.0] * 9
    total = 30
    a0, a1, k0, k1, _ = O.attentional_gnn_adaptive(xs0, xs1, w, 4, 1e-5, 1.0, 4, width_confidence=0.99,
                                                   pruning_threshold=0)
    left = len(k0[0]) + len(k1[0])
    assert 0 < left < total
    # confidences of the points left after layer 1 (the run above never exits)
    y0, y1, _, _, _ = O.attentional_gnn_adaptive(xs0, xs1, w, 4, 1e-5, 1.0, 6, width_confidence=0.99,
                                                 pruning_threshold=0)
    c = O.token_confidence(np.concatenate([y0[0], y1[0]]), t1, 0.0)
    low = int(np.sum(c < O.confidence_threshold(1, 3)))
    share_all, share_left = 1.0 - low / total, 1.0 - low / left
    share0 = 1.0 - (total - (total - left)) / total     # layer 0: the pruned points were the confident ones
    assert share0 < share_all
    d = (max(share0, share_left) + share_all) / 2.0 if share_left < share_all else None
    if d is None or not (share0 < d < share_all):
        pytest.skip(f"no separating depth_confidence: {share0}, {share_left}, {share_all}")
    assert O.attentional_gnn_adaptive(xs0, xs1, w, 4, 1e-5, d, 6, width_confidence=0.99,
                                      pruning_threshold=0)[4] == 2


# --------------------------------------------------------------------------- bidirectional cross attention
def test_bidirectional_cross_attention_is_tied_cross_attention_in_torch(weights):
    # with one projection for queries and keys, the two directions of torch's
    # MultiheadAttention are the row softmax of sim and the row softmax of sim^T
    rng = np.random.default_rng(44)
    x0 = rng.standard_normal((13, 256)) * 0.3
    x1 = rng.standard_normal((9, 256)) * 0.3
    st = dict(weights["stages"][1])
    st["Wk"], st["bk"] = st["Wq"], st["bq"]
    mha = _torch_mha(st)
    with torch.no_grad():
        r0, _ = mha(torch.tensor(x0[None]), torch.tensor(x1[None]), torch.tensor(x1[None]))
        r1, _ = mha(torch.tensor(x1[None]), torch.tensor(x0[None]), torch.tensor(x0[None]))
    m0, m1 = O.bidirectional_cross_attention(x0, x1, st, 4)
    np.testing.assert_allclose(m0, r0[0].numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(m1, r1[0].numpy(), rtol=1e-11, atol=1e-12)


def test_bidirectional_cross_attention_on_one_point_each():
    # one point per image: every softmax is over a single entry, so each
    # message is the other point's value through the merge layer
    rng = np.random.default_rng(45)
    st = {k: rng.standard_normal((8, 8)) for k in ("Wq", "Wv", "Wm")}
    st.update({k: rng.standard_normal(8) for k in ("bq", "bv", "bm")})
    x0, x1 = rng.standard_normal((1, 8)), rng.standard_normal((1, 8))
    m0, m1 = O.bidirectional_cross_attention(x0, x1, st, 2)
    np.testing.assert_allclose(m0[0], (st["Wv"] @ x1[0] + st["bv"]) @ st["Wm"].T + st["bm"], rtol=1e-12)
    np.testing.assert_allclose(m1[0], (st["Wv"] @ x0[0] + st["bv"]) @ st["Wm"].T + st["bm"], rtol=1e-12)


# --------------------------------------------------------------------------- training-side derivatives
def test_nll_loss_hand_built():
    logP = np.log(np.array([[0.5, 0.2, 0.3], [0.1, 0.6, 0.3], [0.4, 0.2, 1.4]]))
    loss = O.nll_loss(logP, [(0, 0)], [1], [1])
    assert loss == pytest.approx(-(math.log(0.5) + math.log(0.3) + math.log(0.2)), abs=1e-15)
    g = O.nll_loss_grad(logP.shape, [(0, 0)], [1], [1])
    assert g[0, 0] == -1 and g[1, 2] == -1 and g[2, 1] == -1 and np.count_nonzero(g) == 3


def test_attend_backward_matches_autograd():
    rng = np.random.default_rng(46)
    q, k, v = rng.standard_normal((7, 16)), rng.standard_normal((9, 16)), rng.standard_normal((9, 16))
    g = rng.standard_normal((7, 16))
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    a = torch.softmax(tq @ tk.T / 4.0, dim=1)
    (a @ tv).backward(torch.tensor(g))
    dq, dk, dv = O.attend_backward(q, k, v, g)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-12, atol=1e-13)


def test_attention_score_gradient_formula_of_the_pages():
    # dL/de_ij = alpha_ij g_i . (v_j - m_i): autograd through softmax(e) v
    rng = np.random.default_rng(47)
    e, v, g = rng.standard_normal((5, 6)), rng.standard_normal((6, 3)), rng.standard_normal((5, 3))
    te = torch.tensor(e, requires_grad=True)
    (torch.softmax(te, 1) @ torch.tensor(v)).backward(torch.tensor(g))
    a = np.exp(e - e.max(1, keepdims=True))
    a /= a.sum(1, keepdims=True)
    m = a @ v
    formula = np.array([[a[i, j] * g[i] @ (v[j] - m[i]) for j in range(6)] for i in range(5)])
    np.testing.assert_allclose(te.grad.numpy(), formula, rtol=1e-12, atol=1e-14)


def test_log_sinkhorn_backward_matches_autograd():
    rng = np.random.default_rng(48)
    S = rng.standard_normal((4, 5)) * 2.0
    Z = O.augment_dustbin(S, 0.7)
    log_mu, log_nu, _ = O.log_marginals(4, 5)
    G = rng.standard_normal(Z.shape)
    tz = torch.tensor(Z, requires_grad=True)
    tmu, tnu = torch.tensor(log_mu), torch.tensor(log_nu)
    u = torch.zeros(5, dtype=torch.float64)
    v = torch.zeros(6, dtype=torch.float64)
    for _ in range(7):
        u = tmu - torch.logsumexp(tz + v[None, :], dim=1)
        v = tnu - torch.logsumexp(tz + u[:, None], dim=0)
    (tz + u[:, None] + v[None, :]).backward(torch.tensor(G))
    np.testing.assert_allclose(O.log_sinkhorn_backward(Z, log_mu, log_nu, 7, G), tz.grad.numpy(),
                               rtol=1e-11, atol=1e-12)
    # no iterations: the identity
    np.testing.assert_allclose(O.log_sinkhorn_backward(Z, log_mu, log_nu, 0, G), G, rtol=0, atol=0)


def test_log_sinkhorn_backward_by_finite_differences():
    # the NLL loss of a planted match through 20 iterations, central differences
    rng = np.random.default_rng(49)
    Z = O.augment_dustbin(rng.standard_normal((3, 3)), 1.0)
    log_mu, log_nu, _ = O.log_marginals(3, 3)
    matches, un0, un1 = [(0, 1), (2, 0)], [1], [2]
    loss = lambda z: O.nll_loss(O.log_sinkhorn(z, log_mu, log_nu, 20), matches, un0, un1)
    G = O.nll_loss_grad(Z.shape, matches, un0, un1)
    grad = O.log_sinkhorn_backward(Z, log_mu, log_nu, 20, G)
    h = 1e-6
    for i, j in [(0, 0), (0, 1), (1, 3), (3, 2), (2, 0)]:
        zp, zm = Z.copy(), Z.copy()
        zp[i, j] += h
        zm[i, j] -= h
        assert abs((loss(zp) - loss(zm)) / (2 * h) - grad[i, j]) < 1e-6


def test_bidirectional_gnn_with_tied_projections_is_the_standard_gnn(weights):
    # with Wk = Wq (and bk = bq) in every cross stage, the bidirectional cross
    # stages compute the same messages as the standard ones
    rng = np.random.default_rng(50)
    x0 = rng.standard_normal((8, 256)) * 0.3
    x1 = rng.standard_normal((6, 256)) * 0.3
    w = dict(weights)
    w["stages"] = [dict(st) for st in weights["stages"][:4]]
    for st in w["stages"]:
        st["Wk"], st["bk"] = st["Wq"], st["bq"]
    a0, a1 = O.attentional_gnn(x0, x1, w, 4, 1e-5, n_stages=4, bidirectional=True)
    r0, r1 = O.attentional_gnn(x0, x1, w, 4, 1e-5, n_stages=4)
    np.testing.assert_allclose(a0, r0, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(a1, r1, rtol=1e-11, atol=1e-12)
    # and untied projections differ (the bidirectional stage ignores Wk)
    u0, _ = O.attentional_gnn(x0, x1, weights, 4, 1e-5, n_stages=2, bidirectional=True)
    s0, _ = O.attentional_gnn(x0, x1, weights, 4, 1e-5, n_stages=2)
    assert np.abs(u0 - s0).max() > 1e-6


def test_pruning_every_point_of_an_image_ends_the_layers(weights):
    # matchability 0 everywhere and no exit classifier: after layer 0 every
    # point is pruned, the next layer does not run and nothing is matched
    rng = np.random.default_rng(22)
    pairs = [synth.make_pair(rng, 6, 5, 0.5)]
    batch = {k: np.stack([p[k] for p in pairs]) for k in ("kpts0", "conf0", "desc0", "kpts1", "conf1", "desc1")}
    w = dict(weights)
    w["mt_w"] = [np.zeros(256)] * 9
    w["mt_b"] = [-50.0] * 9
    out, layers = O.superglue_batch_adaptive(batch, w, None, n_stages=6, width_confidence=0.99,
                                             pruning_threshold=0)
    assert layers == 1                           # only layer 0 ran
    res = out[0]
    assert len(res["kept0"]) == 0 and len(res["kept1"]) == 0 and res["log_P"] is None
    assert np.all(res["matches0"] == -1) and np.all(res["matches1"] == -1)
    assert np.all(res["mscores0"] == 0) and np.all(res["mscores1"] == 0)


def test_batch_adaptive_without_exit_or_pruning_is_the_pair_pass(weights):
    # the batch driver (encoder, lockstep layers, head, map back) reduces to
    # superglue_pair for every pair when nothing exits and nothing is pruned
    rng = np.random.default_rng(23)
    pairs = [synth.make_pair(rng, 10, 8, 0.5) for _ in range(2)]
    batch = {k: np.stack([p[k] for p in pairs]) for k in ("kpts0", "conf0", "desc0", "kpts1", "conf1", "desc1")}
    out, layers = O.superglue_batch_adaptive(batch, weights, None, n_stages=4)
    assert layers == 2
    for b in range(2):
        ref = O.superglue_pair(*(batch[k][b] for k in ("kpts0", "conf0", "desc0", "kpts1", "conf1", "desc1")),
                               weights, n_stages=4)
        np.testing.assert_array_equal(out[b]["log_P"], ref["log_P"])
        for k in ("matches0", "matches1", "mscores0", "mscores1"):
            np.testing.assert_array_equal(out[b][k], ref[k])
