"""Plant plausible mistakes in the oracle (on the CPU) and check that at least one
pin catches each of them.  This is what makes the pins evidence: a dropped term,
a wrong sign or index, a swapped operand anywhere in the oracle must fail one."""
import math

import numpy as np
import pytest

import test_oracle_pins as pins
from oracle import superglue_oracle as O

_extract_matches = O.extract_matches

PIN_TESTS = [
    (pins.test_normalize_keypoints_printed_values, False),
    (pins.test_attention_worked_example, False),
    (pins.test_attention_scale_uses_key_width, False),
    (pins.test_batchnorm_matches_torch, True),
    (pins.test_encoder_mlp_matches_torch_modules, True),
    (pins.test_keypoint_encoder_adds_descriptor, True),
    (pins.test_multi_head_attention_matches_torch, True),
    (pins.test_attentional_propagation_matches_torch, True),
    (pins.test_self_stage_reads_only_own_image, True),
    (pins.test_cross_stage_reads_other_image, True),
    (pins.test_gnn_is_symmetric_in_the_two_images, True),
    (pins.test_cross_stage_equals_self_stage_on_the_other_source, True),
    (pins.test_marginals_sum_to_one, False),
    (lambda: pins.test_sinkhorn_one_by_one_closed_form(3.0, 1.0), False),
    (lambda: pins.test_sinkhorn_constant_scores_closed_form(7), False),
    (pins.test_sinkhorn_column_marginals_exact_and_rows_converge, False),
    (pins.test_extraction_hand_built, False),
    (pins.test_extraction_ties_take_lowest_index_and_threshold_is_strict, False),
    (pins.test_score_matrix_scale_matches_library_attention, True),
    (pins.test_double_softmax_matches_torch_log_softmax_and_logsigmoid, False),
    (pins.test_double_softmax_two_by_two_closed_form, False),
    (pins.test_log_sigmoid_is_stable_and_complements, False),
    (pins.test_double_softmax_head_matches_torch_modules, True),
    (pins.test_double_softmax_recovers_a_planted_permutation, False),
    (pins.test_confidence_threshold_printed_values, False),
    (pins.test_check_if_stop_counts_strictly, False),
    (pins.test_token_confidence_matches_torch_linear_sigmoid, False),
    (pins.test_adaptive_gnn_that_never_stops_is_the_fixed_depth_gnn, True),
    (pins.test_adaptive_gnn_stops_after_the_planted_layer, True),
    (pins.test_adaptive_decision_pools_the_points_of_the_batch, True),
    (pins.test_pruning_mask_hand_built, False),
    (pins.test_matchability_matches_torch_linear_sigmoid, False),
    (pins.test_pruning_that_keeps_everything_is_the_unpruned_pass, True),
    (pins.test_pruned_points_leave_the_later_layers, True),
    (pins.test_pruned_points_are_unmatched_and_matches_map_back, True),
    (pins.test_exit_share_counts_pruned_points_as_confident, True),
    (pins.test_bidirectional_cross_attention_is_tied_cross_attention_in_torch, True),
    (pins.test_bidirectional_cross_attention_on_one_point_each, False),
    (pins.test_nll_loss_hand_built, False),
    (pins.test_attend_backward_matches_autograd, False),
    (pins.test_log_sinkhorn_backward_matches_autograd, False),
    (pins.test_log_sinkhorn_backward_by_finite_differences, False),
]


def _some_pin_fails(weights):
    for fn, needs_w in PIN_TESTS:
        try:
            fn(weights) if needs_w else fn()
        except (AssertionError, ValueError, IndexError):
            return True
    return False


def _attend_wrong_scale(q, k, v):
    e = (q @ k.T) / math.sqrt(4 * q.shape[-1])
    a = O.softmax(e, axis=1)
    return a @ v, a


def _attend_wrong_axis(q, k, v):
    e = (q @ k.T) / math.sqrt(q.shape[-1])
    a = O.softmax(e, axis=0)
    return a @ v, a


def _bn_eps_outside(z, g, b, m, v, eps):
    return np.asarray(g, float) * (z - m) / (np.sqrt(np.asarray(v, float)) + eps) + b


def _mlp_relu_before_bn(z, Ws, bs, bns, eps):
    n = len(Ws)
    for l in range(n):
        z = O.linear(z, Ws[l], bs[l])
        if l < n - 1:
            z = np.maximum(z, 0.0)
            z = O.batchnorm_eval(z, *bns[l], eps)
    return z


def _gnn_cross_uses_self(x0, x1, weights, heads, eps, n_stages=None):
    st = weights["stages"]
    n_stages = len(st) if n_stages is None else n_stages
    for s in range(n_stages):
        d0 = O.attentional_propagation(x0, x0, st[s], heads, eps)
        d1 = O.attentional_propagation(x1, x1, st[s], heads, eps)
        x0, x1 = x0 + d0, x1 + d1
    return x0, x1


def _gnn_sequential_update(x0, x1, weights, heads, eps, n_stages=None):
    st = weights["stages"]
    n_stages = len(st) if n_stages is None else n_stages
    for s, name in enumerate(O.stage_names(n_stages)):
        x0 = x0 + O.attentional_propagation(x0, x1 if name == "cross" else x0, st[s], heads, eps)
        x1 = x1 + O.attentional_propagation(x1, x0 if name == "cross" else x1, st[s], heads, eps)
    return x0, x1


def _gnn_cross_first(x0, x1, weights, heads, eps, n_stages=None):
    st = weights["stages"]
    n_stages = len(st) if n_stages is None else n_stages
    for s in range(n_stages):
        cross = s % 2 == 0
        d0 = O.attentional_propagation(x0, x1 if cross else x0, st[s], heads, eps)
        d1 = O.attentional_propagation(x1, x0 if cross else x1, st[s], heads, eps)
        x0, x1 = x0 + d0, x1 + d1
    return x0, x1


def _sinkhorn_v_first(Z, log_mu, log_nu, iters):
    u = np.zeros(Z.shape[0])
    v = np.zeros(Z.shape[1])
    for _ in range(iters):
        v = log_nu - O.logsumexp(Z + u[:, None], axis=0)
        u = log_mu - O.logsumexp(Z + v[None, :], axis=1)
    return Z + u[:, None] + v[None, :]


def _marginals_swapped(M, N):
    norm = -math.log(M + N)
    lm = np.full(M + 1, norm)
    lm[M] = math.log(M) + norm
    ln = np.full(N + 1, norm)
    ln[N] = math.log(N) + norm
    return lm, ln, norm


def _augment_zero_corner(S, alpha):
    Z = np.full((S.shape[0] + 1, S.shape[1] + 1), float(alpha))
    Z[:-1, :-1] = S
    Z[-1, -1] = 0.0
    return Z


def _lot_no_renorm(S, alpha, iters):
    M, N = S.shape
    Z = O.augment_dustbin(S, alpha)
    lm, ln, _ = O.log_marginals(M, N)
    return O.log_sinkhorn(Z, lm, ln, iters)


def _extract_ge(logP, threshold):
    P = np.asarray(logP)[:-1, :-1]
    M, N = P.shape
    i0, i1 = P.argmax(1), P.argmax(0)
    mu0, mu1 = i1[i0] == np.arange(M), i0[i1] == np.arange(N)
    s0 = np.where(mu0, np.exp(P[np.arange(M), i0]), 0.0)
    s1 = np.where(mu1, s0[i1], 0.0)
    v0 = mu0 & (s0 >= threshold)
    v1 = mu1 & v0[i1]
    return np.where(v0, i0, -1), np.where(v1, i1, -1), s0, s1


def _extract_last_tie(logP, threshold):
    P = np.asarray(logP)[:-1, :-1]
    flipped = P[:, ::-1][::-1, :]
    m0, m1, s0, s1 = _extract_matches(np.pad(flipped, ((0, 1), (0, 1))), threshold)
    M, N = P.shape
    m0 = np.where(m0[::-1] >= 0, N - 1 - m0[::-1], -1)
    m1 = np.where(m1[::-1] >= 0, M - 1 - m1[::-1], -1)
    return m0, m1, s0[::-1], s1[::-1]


def _normalize_hw_swapped(kpts, width, height, mode=0):
    return (np.asarray(kpts, float) - np.array([height / 2, width / 2])) / (0.7 * max(width, height))


def _score_unscaled(x0, x1, Wf, bf):
    return O.linear(x0, Wf, bf) @ O.linear(x1, Wf, bf).T


def _mha_interleaved_heads(x, src, st, heads):
    q = O.linear(x, st["Wq"], st["bq"])
    k = O.linear(src, st["Wk"], st["bk"])
    v = O.linear(src, st["Wv"], st["bv"])
    msg = np.empty_like(q)
    for h in range(heads):
        sl = slice(h, None, heads)
        msg[:, sl], _ = O.attend(q[:, sl], k[:, sl], v[:, sl])
    return O.linear(msg, st["Wm"], st["bm"])


def _prop_message_first(x, src, st, heads, eps):
    m = O.multi_head_attention(x, src, st, heads)
    z = np.concatenate([m, x], axis=1)
    return O.mlp(z, [st["W1"], st["W2"]], [st["b1"], st["b2"]], [st["bn1"]], eps)


_dsm_assign = O.double_softmax_log_assignment


def _dsm_same_axis_twice(sim, z0, z1):
    out = _dsm_assign(sim, z0, z1)
    M, N = np.shape(sim)
    out[:M, :N] += O.log_softmax(sim, 1) - O.log_softmax(sim, 0)
    return out


def _dsm_no_certainty(sim, z0, z1):
    out = _dsm_assign(sim, z0, z1)
    M, N = np.shape(sim)
    out[:M, :N] -= O.log_sigmoid(z0)[:, None] + O.log_sigmoid(z1)[None, :]
    return out


def _dsm_dustbin_sign(sim, z0, z1):
    out = _dsm_assign(sim, z0, z1)
    M, N = np.shape(sim)
    out[:M, N] = O.log_sigmoid(z0)
    out[M, :N] = O.log_sigmoid(z1)
    return out


def _dsm_corner_one(sim, z0, z1):
    out = _dsm_assign(sim, z0, z1)
    out[-1, -1] = 1.0
    return out


def _head_sqrt_scale(x0, x1, Wp, bp, wz, bz):
    x0, x1 = np.asarray(x0, float), np.asarray(x1, float)
    d = x0.shape[1]
    m0 = O.linear(x0, Wp, bp) / d ** 0.5
    m1 = O.linear(x1, Wp, bp) / d ** 0.5
    sim = m0 @ m1.T
    z0 = x0 @ np.asarray(wz, float) + float(bz)
    z1 = x1 @ np.asarray(wz, float) + float(bz)
    return O.double_softmax_log_assignment(sim, z0, z1), sim, z0, z1


def _head_matchability_on_projection(x0, x1, Wp, bp, wz, bz):
    x0, x1 = np.asarray(x0, float), np.asarray(x1, float)
    d = x0.shape[1]
    m0 = O.linear(x0, Wp, bp) / d ** 0.25
    m1 = O.linear(x1, Wp, bp) / d ** 0.25
    sim = m0 @ m1.T
    z0 = m0 @ np.asarray(wz, float) + float(bz)
    z1 = m1 @ np.asarray(wz, float) + float(bz)
    return O.double_softmax_log_assignment(sim, z0, z1), sim, z0, z1


def _threshold_growing(layer, n_layers):
    return float(np.clip(0.8 + 0.1 * math.exp(4.0 * layer / n_layers), 0.0, 1.0))


def _stop_counts_equal_as_low(confidences, layer, n_layers, depth_confidence, num_points):
    lam = O.confidence_threshold(layer, n_layers)
    ratio = 1.0 - float(np.sum(np.asarray(confidences) <= lam)) / float(num_points)
    return ratio > depth_confidence


def _stop_at_equal_share(confidences, layer, n_layers, depth_confidence, num_points):
    lam = O.confidence_threshold(layer, n_layers)
    ratio = 1.0 - float(np.sum(np.asarray(confidences) < lam)) / float(num_points)
    return ratio >= depth_confidence


def _confidence_without_bias(x, w, b):
    z = np.asarray(x, float) @ np.asarray(w, float)
    return 1.0 / (1.0 + np.exp(-z))


def _adaptive_last_pair_only(xs0, xs1, weights, heads, eps, depth_confidence, n_stages=None,
                             width_confidence=None, pruning_threshold=1536):
    stages = weights["stages"]
    n_stages = len(stages) if n_stages is None else n_stages
    n_layers = n_stages // 2
    xs0, xs1 = list(xs0), list(xs1)
    for layer in range(n_layers):
        for s in (2 * layer, 2 * layer + 1):
            for b in range(len(xs0)):
                x0, x1 = xs0[b], xs1[b]
                src0, src1 = (x1, x0) if s % 2 == 1 else (x0, x1)
                d0 = O.attentional_propagation(x0, src0, stages[s], heads, eps)
                d1 = O.attentional_propagation(x1, src1, stages[s], heads, eps)
                xs0[b], xs1[b] = x0 + d0, x1 + d1
        if layer == n_layers - 1 or depth_confidence is None or depth_confidence <= 0:
            continue
        b = len(xs0) - 1
        conf = O.token_confidence(np.concatenate([xs0[b], xs1[b]]), weights["tc_w"][layer],
                                  weights["tc_b"][layer])
        if O.check_if_stop(conf, layer, n_layers, depth_confidence, conf.size):
            return xs0, xs1, None, None, layer + 1
    return xs0, xs1, None, None, n_layers


def _mask_keeps_equal_score(confidences, scores, layer, n_layers, width_confidence):
    keep = np.asarray(scores) >= (1.0 - width_confidence)
    if confidences is not None:
        keep = keep | (np.asarray(confidences) <= O.confidence_threshold(layer, n_layers))
    return keep


def _mask_prunes_uncertain(confidences, scores, layer, n_layers, width_confidence):
    keep = np.asarray(scores) > (1.0 - width_confidence)
    if confidences is not None:
        keep = keep | (np.asarray(confidences) < O.confidence_threshold(layer, n_layers))
    return keep


_adaptive = O.attentional_gnn_adaptive


def _adaptive_prunes_after_last_layer(xs0, xs1, weights, heads, eps, depth_confidence, n_stages=None,
                                      width_confidence=None, pruning_threshold=1536):
    xs0, xs1, kept0, kept1, layers = _adaptive(xs0, xs1, weights, heads, eps, depth_confidence, n_stages,
                                               width_confidence, pruning_threshold)
    if width_confidence is not None and width_confidence > 0:
        last = layers - 1
        n_layers = (len(weights["stages"]) if n_stages is None else n_stages) // 2
        for b in range(len(xs0)):
            for xs, kept in ((xs0, kept0), (xs1, kept1)):
                if len(xs[b]) > pruning_threshold:
                    s = O.matchability(xs[b], weights["mt_w"][last], weights["mt_b"][last])
                    keep = O.get_pruning_mask(None, s, last, n_layers, width_confidence)
                    xs[b], kept[b] = xs[b][keep], kept[b][keep]
    return xs0, xs1, kept0, kept1, layers


def _stop_over_points_left(confidences, layer, n_layers, depth_confidence, num_points):
    c = np.asarray(confidences)
    lam = O.confidence_threshold(layer, n_layers)
    return 1.0 - float(np.sum(c < lam)) / float(c.size) > depth_confidence


def _matchability_negated(x, w, b):
    z = -(np.asarray(x, float) @ np.asarray(w, float) + float(b))
    return 1.0 / (1.0 + np.exp(-z))


def _bidir_same_softmax_axis(x0, x1, st, heads):
    qk0 = O.linear(x0, st["Wq"], st["bq"])
    qk1 = O.linear(x1, st["Wq"], st["bq"])
    v0 = O.linear(x0, st["Wv"], st["bv"])
    v1 = O.linear(x1, st["Wv"], st["bv"])
    d = qk0.shape[1]
    dh = d // heads
    s = dh ** -0.25
    m0 = np.empty((x0.shape[0], d))
    m1 = np.empty((x1.shape[0], d))
    for h in range(heads):
        sl = slice(h * dh, (h + 1) * dh)
        sim = (qk0[:, sl] * s) @ (qk1[:, sl] * s).T
        a = O.softmax(sim, axis=1)
        m0[:, sl] = a @ v1[:, sl]
        m1[:, sl] = a.T @ v0[:, sl]             # the row softmax reused for the other direction
    return O.linear(m0, st["Wm"], st["bm"]), O.linear(m1, st["Wm"], st["bm"])


def _nll_matches_only(logP, matches, unmatched0, unmatched1):
    logP = np.asarray(logP, float)
    return float(-sum(logP[i, j] for i, j in matches))


def _attend_backward_no_mean(q, k, v, g):
    d = q.shape[1]
    m, a = O.attend(q, k, v)
    de = a * (g @ v.T)
    return de @ k / math.sqrt(d), de.T @ q / math.sqrt(d), a.T @ g


_sk_bwd = O.log_sinkhorn_backward


def _sinkhorn_backward_last_iteration_only(Z, log_mu, log_nu, iters, G):
    return _sk_bwd(Z, log_mu, log_nu, min(iters, 1), G)


MUTATIONS = {
    "NLL loss without the unmatched terms": ("nll_loss", _nll_matches_only),
    "attention gradient without the mean message": ("attend_backward", _attend_backward_no_mean),
    "Sinkhorn gradient through one iteration": ("log_sinkhorn_backward", _sinkhorn_backward_last_iteration_only),
    "bidirectional: one softmax axis for both directions": ("bidirectional_cross_attention", _bidir_same_softmax_axis),
    "pruning keeps a score equal to 1 - width": ("get_pruning_mask", _mask_keeps_equal_score),
    "uncertain points at the threshold pruned": ("get_pruning_mask", _mask_prunes_uncertain),
    "pruning after the last layer": ("attentional_gnn_adaptive", _adaptive_prunes_after_last_layer),
    "exit share over the points left": ("check_if_stop", _stop_over_points_left),
    "matchability of the negated logit": ("matchability", _matchability_negated),
    "exit threshold grows with depth": ("confidence_threshold", _threshold_growing),
    "confidence at the threshold counted as low": ("check_if_stop", _stop_counts_equal_as_low),
    "exit when the share equals depth_confidence": ("check_if_stop", _stop_at_equal_share),
    "token confidence without its bias": ("token_confidence", _confidence_without_bias),
    "exit decided on the last pair only": ("attentional_gnn_adaptive", _adaptive_last_pair_only),
    "double softmax over one axis twice": ("double_softmax_log_assignment", _dsm_same_axis_twice),
    "double softmax without certainties": ("double_softmax_log_assignment", _dsm_no_certainty),
    "double softmax dustbin sign": ("double_softmax_log_assignment", _dsm_dustbin_sign),
    "double softmax corner not zero": ("double_softmax_log_assignment", _dsm_corner_one),
    "head scaled by D^(1/2)": ("double_softmax_head", _head_sqrt_scale),
    "matchability on the projection": ("double_softmax_head", _head_matchability_on_projection),
    "attention scale 1/sqrt(D)": ("attend", _attend_wrong_scale),
    "softmax over queries": ("attend", _attend_wrong_axis),
    "BN eps outside sqrt": ("batchnorm_eval", _bn_eps_outside),
    "ReLU before BN": ("mlp", _mlp_relu_before_bn),
    "cross stage reads own image": ("attentional_gnn", _gnn_cross_uses_self),
    "sequential A-then-B update": ("attentional_gnn", _gnn_sequential_update),
    "cross stage first": ("attentional_gnn", _gnn_cross_first),
    "Sinkhorn column update first": ("log_sinkhorn", _sinkhorn_v_first),
    "dustbin marginals swapped": ("log_marginals", _marginals_swapped),
    "dustbin corner zero": ("augment_dustbin", _augment_zero_corner),
    "missing M+N rescale": ("log_optimal_transport", _lot_no_renorm),
    "threshold not strict": ("extract_matches", _extract_ge),
    "ties to the last index": ("extract_matches", _extract_last_tie),
    "width/height swapped": ("normalize_keypoints", _normalize_hw_swapped),
    "score without 1/sqrt(D)": ("score_matrix", _score_unscaled),
    "interleaved head channels": ("multi_head_attention", _mha_interleaved_heads),
    "[m || x] concatenation": ("attentional_propagation", _prop_message_first),
}


def test_unmutated_oracle_passes_every_pin(weights):
    assert not _some_pin_fails(weights)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_each_planted_mistake_is_caught(name, weights, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    assert _some_pin_fails(weights), f"no pin catches: {name}"
