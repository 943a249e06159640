"""Adaptive depth (the LightGlue review, section 2.6) on the GPU through the C ABI
against the float64 oracle: exits planted with a wide margin in both
precisions, the no-exit case against the fixed-depth pass, the batch-wide
decision, and a decision on the classifier weights of the generator where the
oracle's share is far enough from depth_confidence to be decidable."""
import numpy as np
import pytest

from gpu_util import BF16_AGREEMENT, BF16_TOL, FP32_TOL, assert_pair_parity
from learned_sparse_feature_b200 import synth
from oracle import superglue_oracle as O

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

STAGES = 8          # four (self, cross) layers: exit checks after layers 0, 1, 2


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from learned_sparse_feature_b200 import build
    build.build()
    return torch.device("cuda:0")


def _batch(B, M, N, seed, inlier=0.5):
    rng = np.random.default_rng(seed)
    pairs = [synth.make_pair(rng, M, N, inlier) for _ in range(B)]
    return {k: np.ascontiguousarray(np.stack([p[k] for p in pairs]))
            for k in ("kpts0", "conf0", "desc0", "kpts1", "conf1", "desc1")}


def _planted(weights, k):
    # confidences sigmoid(-30) before layer k and sigmoid(30) at it: the share of
    # confident points is 0 or 1, far from any depth_confidence in (0, 1)
    w = dict(weights)
    w["tc_w"] = [np.zeros(256, np.float32) for _ in range(9)]
    w["tc_b"] = [np.float32(-30.0 if l < k else 30.0) for l in range(9)]
    return w


def _run(weights, batch, precision, depth_confidence, n_stages=STAGES):
    from learned_sparse_feature_b200.binding import Matcher, match_batch
    B, M, N = batch["kpts0"].shape[0], batch["kpts0"].shape[1], batch["kpts1"].shape[1]
    m = Matcher(weights, B, M, N, precision=precision, n_stages=n_stages, depth_confidence=depth_confidence)
    out = match_batch(m, batch, True)
    assert m.status() == 0
    layers = m.layers_run()
    m.close()
    return out, layers


def _check(out, refs, precision):
    for b, ref in enumerate(refs):
        pair = {k: v[b] for k, v in out.items()}
        if precision == "fp32":
            assert_pair_parity(pair, ref, FP32_TOL, thr=synth.MATCH_THRESHOLD)
        else:
            assert_pair_parity(pair, ref, BF16_TOL, thr=synth.MATCH_THRESHOLD, exact_matches=False,
                               agreement=BF16_AGREEMENT)


@pytest.mark.parametrize("precision,B,M,N,k", [("bf16", 2, 200, 150, 0), ("bf16", 1, 129, 255, 2),
                                               ("fp32", 1, 64, 48, 1)])
def test_planted_exit_matches_the_oracle(dev, weights, precision, B, M, N, k):
    w = _planted(weights, k)
    batch = _batch(B, M, N, seed=300 + k)
    out, layers = _run(w, batch, precision, 0.95)
    refs, ref_layers = O.superglue_batch_adaptive(batch, w, 0.95, n_stages=STAGES)
    assert ref_layers == k + 1
    assert layers == k + 1
    _check(out, refs, precision)


def test_no_exit_equals_the_fixed_depth_pass(dev, weights):
    w = _planted(weights, 9)                     # never confident: every layer runs
    batch = _batch(1, 150, 170, seed=77)
    out, layers = _run(w, batch, "bf16", 0.95)
    assert layers == STAGES // 2
    ref, full_layers = _run(weights, batch, "bf16", -1.0)
    assert full_layers == STAGES // 2
    # the Sinkhorn column sums are fp32 atomics: equal to rounding, not bitwise
    np.testing.assert_allclose(out["log_P"], ref["log_P"], rtol=0, atol=2e-5)
    assert (out["matches0"] == ref["matches0"]).mean() > 0.99


def test_exit_after_the_last_layer_is_never_taken(dev, weights):
    w = _planted(weights, 3)                     # confident only at the last layer (3 of 0..3)
    batch = _batch(1, 90, 70, seed=5)
    _, layers = _run(w, batch, "bf16", 0.95)
    assert layers == STAGES // 2


def _oracle_shares(batch, weights, n_layers):
    """Share of confident points after each checked layer, and how many points
    lie within 1e-2 of the threshold (where bf16 states may decide otherwise)."""
    B = batch["kpts0"].shape[0]
    xs = []
    for b in range(B):
        k0 = O.normalize_keypoints(batch["kpts0"][b], 640.0, 480.0)
        k1 = O.normalize_keypoints(batch["kpts1"][b], 640.0, 480.0)
        xs.append((O.keypoint_encoder(k0, batch["conf0"][b], batch["desc0"][b], weights, 1e-5),
                   O.keypoint_encoder(k1, batch["conf1"][b], batch["desc1"][b], weights, 1e-5)))
    shares, near = [], []
    for layer in range(n_layers - 1):
        conf = []
        for b in range(B):
            x0, x1 = O.attentional_gnn(xs[b][0], xs[b][1], weights, 4, 1e-5, n_stages=2 * layer + 2)
            conf.append(O.token_confidence(np.concatenate([x0, x1]), weights["tc_w"][layer],
                                           weights["tc_b"][layer]))
        conf = np.concatenate(conf)
        lam = O.confidence_threshold(layer, n_layers)
        shares.append(1.0 - np.mean(conf < lam))
        near.append(np.mean(np.abs(conf - lam) < 1e-2))
    return np.array(shares), np.array(near)


def test_decision_on_generated_classifier_weights(dev, weights):
    # classifier biases raised so that a good share of points is confident
    w = dict(weights)
    w["tc_b"] = [np.float32(b + 2.0) for b in weights["tc_b"]]
    batch = _batch(2, 96, 80, seed=11)
    shares, near = _oracle_shares(batch, w, STAGES // 2)
    # a depth_confidence between the shares: exit at the first layer whose share
    # clears it, each side by more than the share of undecidable points
    picked = None
    for d in np.linspace(0.02, 0.98, 97):
        margin = np.abs(shares - d) - near
        if np.all(margin > 1e-3):
            picked = d
            if np.any(shares > d):
                break
    if picked is None:
        pytest.skip(f"no decidable depth_confidence for shares {shares} (near {near})")
    out, layers = _run(w, batch, "bf16", float(picked))
    refs, ref_layers = O.superglue_batch_adaptive(batch, w, float(np.float32(picked)), n_stages=STAGES)
    assert layers == ref_layers, (picked, shares, near)
    _check(out, refs, "bf16")


def test_odd_stage_count_is_refused(dev, weights):
    from learned_sparse_feature_b200.binding import Matcher, SgError
    with pytest.raises(SgError):
        Matcher(weights, 1, 16, 16, n_stages=7, depth_confidence=0.95)


def test_layers_run_after_an_empty_call_is_zero(dev, weights):
    from learned_sparse_feature_b200.binding import Matcher
    w = _planted(weights, 1)
    m = Matcher(w, 1, 16, 16, n_stages=STAGES, depth_confidence=0.95)
    k0, c0, d0 = torch.zeros((1, 0, 2), device=dev), torch.zeros((1, 0), device=dev), torch.zeros((1, 0, 256), device=dev)
    k1, c1, d1 = torch.zeros((1, 5, 2), device=dev), torch.zeros((1, 5), device=dev), torch.zeros((1, 5, 256), device=dev)
    m0 = torch.empty((1, 0), dtype=torch.int32, device=dev)
    m1 = torch.empty((1, 5), dtype=torch.int32, device=dev)
    s0, s1 = torch.empty((1, 0), device=dev), torch.empty((1, 5), device=dev)
    m.match(k0, c0, d0, k1, c1, d1, None, m0, m1, s0, s1)
    assert m.status() == 0
    assert m.layers_run() == 0
    assert (m1 == -1).all()
    m.close()
