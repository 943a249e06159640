"""Seeded synthetic workloads for the SuperGlue matcher: keypoint pairs and weights.

This module only draws random numbers and builds planted correspondences. It
holds none of the matcher's arithmetic, so that the float64 oracle (test
infrastructure) and the CUDA path can both take their inputs from it.

Workload shapes follow the pages' benchmarks: 640x480 images with 512, 1024,
2048 and 4096 keypoints per image ("论文解读:LightGlue,让稀疏特征匹配随难度自适应地快",
section on runtime vs. number of keypoints; "笔记：SuperGlue:Learning Feature
Matching with Graph Neural Networks论文阅读", section 网络耗时). Planted matches
come from a random homography, which is the geometry of the homography
self-supervision the SuperGlue notes describe. No item of any public benchmark
is reproduced: every value is drawn from the seeds below.

All arrays are float32 (what the C ABI takes); the oracle promotes them to
float64 exactly.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

IMG_W = 640.0
IMG_H = 480.0
D = 256          # descriptor / state width
H = 4            # attention heads
N_STAGES = 18    # 9 x (self, cross)
SINKHORN_ITERS = 100
MATCH_THRESHOLD = 0.2
BIN_SCORE = 1.0
BN_EPS = 1e-5
ENC_CHANNELS = (3, 32, 64, 128, 256, 256)

# Kaiming-uniform bound g * sqrt(3 / fan_in) per layer family.  Chosen so that the
# score matrix has a non-degenerate spread (|S| of order 10): the literal ReLU
# gain on every layer makes the residual stream explode, 1/sqrt(fan_in) makes
# the assignment uniform.
GAIN_RELU = math.sqrt(2.0)
GAIN_LINEAR = 1.0
GAIN_RESIDUAL_OUT = 0.05
GAIN_FINAL_PROJ = 12.0


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    M: int
    N: int
    precision: str          # "fp32" or "bf16"
    inlier: object          # None, a ratio, or (lo, hi) drawn per pair
    seed: int


WORKLOADS = {
    w.name: w
    for w in (
        Workload("pair64_fp32", 1, 64, 64, "fp32", None, 1000),
        Workload("pair512", 1, 512, 512, "bf16", 0.6, 1001),
        Workload("pair2048", 1, 2048, 2048, "bf16", 0.4, 1002),
        Workload("batch32_pair1024", 32, 1024, 1024, "bf16", (0.1, 0.8), 1003),
        Workload("batch8_pair4096x3072", 8, 4096, 3072, "bf16", 0.3, 1004),
    )
}


def _f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


# --------------------------------------------------------------------------- weights
def _kaiming_uniform(rng, out_ch, in_ch, gain):
    bound = gain * math.sqrt(3.0 / in_ch)
    return _f32(rng.uniform(-bound, bound, size=(out_ch, in_ch)))


def _bias(rng, out_ch, in_ch):
    bound = 1.0 / math.sqrt(in_ch)
    return _f32(rng.uniform(-bound, bound, size=(out_ch,)))


def _bn_stats(rng, ch):
    """(gamma, beta, running_mean, running_var), non-trivial so the fold is exercised."""
    return (
        _f32(rng.uniform(0.8, 1.2, ch)),
        _f32(rng.uniform(-0.1, 0.1, ch)),
        _f32(rng.uniform(-0.1, 0.1, ch)),
        _f32(rng.uniform(0.8, 1.2, ch)),
    )


def make_weights(seed: int = 0, n_stages: int = N_STAGES, d: int = D,
                 gain_final_proj: float = GAIN_FINAL_PROJ,
                 gain_residual_out: float = GAIN_RESIDUAL_OUT) -> dict:
    """Random-init weights for the whole matcher (no trained checkpoint exists).

    Layout: every linear layer is (out_channels, in_channels), i.e. the weight of
    a kernel-size-1 Conv1d with the trailing 1 dropped.
    """
    rng = np.random.default_rng(seed)
    w = {"enc_W": [], "enc_b": [], "enc_bn": []}
    ch = ENC_CHANNELS
    n_enc = len(ch) - 1
    for l in range(n_enc):
        last = l == n_enc - 1
        gain = gain_residual_out if last else GAIN_RELU
        w["enc_W"].append(_kaiming_uniform(rng, ch[l + 1], ch[l], gain))
        w["enc_b"].append(np.zeros(ch[l + 1], np.float32) if last else _bias(rng, ch[l + 1], ch[l]))
        if not last:
            w["enc_bn"].append(_bn_stats(rng, ch[l + 1]))
    stages = []
    for _ in range(n_stages):
        s = {}
        for nm in ("q", "k", "v", "m"):
            s["W" + nm] = _kaiming_uniform(rng, d, d, GAIN_LINEAR)
            s["b" + nm] = _bias(rng, d, d)
        s["W1"] = _kaiming_uniform(rng, 2 * d, 2 * d, GAIN_RELU)
        s["b1"] = _bias(rng, 2 * d, 2 * d)
        s["bn1"] = _bn_stats(rng, 2 * d)
        s["W2"] = _kaiming_uniform(rng, d, 2 * d, gain_residual_out)
        s["b2"] = np.zeros(d, np.float32)
        stages.append(s)
    w["stages"] = stages
    w["Wf"] = _kaiming_uniform(rng, d, d, gain_final_proj)
    w["bf"] = _bias(rng, d, d)
    w["bin_score"] = np.float32(BIN_SCORE)
    # double-softmax matching head (projection and matchability), from a stream
    # of its own so that the weights above do not depend on it
    rng_h = np.random.default_rng([seed, 1])
    w["lg_Wp"] = _kaiming_uniform(rng_h, d, d, gain_final_proj)
    w["lg_bp"] = _bias(rng_h, d, d)
    w["lg_wz"] = _kaiming_uniform(rng_h, 1, d, gain_final_proj)[0]
    w["lg_bz"] = np.float32(_bias(rng_h, 1, d)[0])
    # adaptive depth: one token-confidence classifier (linear + sigmoid) after
    # every (self, cross) layer, from a third stream
    rng_c = np.random.default_rng([seed, 2])
    n_layers = n_stages // 2
    w["tc_w"] = [_kaiming_uniform(rng_c, 1, d, 1.0)[0] for _ in range(n_layers)]
    w["tc_b"] = [np.float32(_bias(rng_c, 1, d)[0]) for _ in range(n_layers)]
    # point pruning: the matchability of every layer's assignment head, a fourth stream
    rng_m = np.random.default_rng([seed, 3])
    w["mt_w"] = [_kaiming_uniform(rng_m, 1, d, 1.0)[0] for _ in range(n_layers)]
    w["mt_b"] = [np.float32(_bias(rng_m, 1, d)[0]) for _ in range(n_layers)]
    return w


# --------------------------------------------------------------------------- pairs
def _random_points(rng, n):
    xy = np.stack([rng.uniform(0.0, IMG_W, n), rng.uniform(0.0, IMG_H, n)], axis=1)
    return xy


def _random_descriptors(rng, n, d):
    x = rng.standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def _homography_from_corners(src, dst):
    """4-point DLT: H (3x3, H[2,2]=1) with dst ~ H @ src (input geometry only)."""
    A = []
    rhs = []
    for (x, y), (u, v) in zip(src, dst):
        A.append([x, y, 1, 0, 0, 0, -u * x, -u * y])
        rhs.append(u)
        A.append([0, 0, 0, x, y, 1, -v * x, -v * y])
        rhs.append(v)
    h = np.linalg.solve(np.asarray(A, float), np.asarray(rhs, float))
    return np.append(h, 1.0).reshape(3, 3)


def _apply_h(Hm, xy):
    p = np.concatenate([xy, np.ones((len(xy), 1))], axis=1) @ Hm.T
    return p[:, :2] / p[:, 2:3]


def make_pair(rng, M: int, N: int, inlier_ratio, d: int = D) -> dict:
    """One keypoint pair.  Image A: M uniform points, U[0,1] confidences, unit
    Gaussian descriptors.  Image B: round(r*N) planted points (homography image
    of A points + N(0,1px) noise, descriptor + N(0,0.1^2) re-normalised, fresh
    confidence) and N-K fresh points, in a shuffled order."""
    k0 = _random_points(rng, M)
    c0 = rng.uniform(0.0, 1.0, M)
    d0 = _random_descriptors(rng, M, d)
    gt = np.zeros((0, 2), np.int64)
    if inlier_ratio is None or N == 0 or M == 0:
        k1 = _random_points(rng, N)
        c1 = rng.uniform(0.0, 1.0, N)
        d1 = _random_descriptors(rng, N, d)
    else:
        corners = np.array([[0, 0], [IMG_W, 0], [IMG_W, IMG_H], [0, IMG_H]], float)
        pert = rng.uniform(-0.15, 0.15, (4, 2)) * np.array([IMG_W, IMG_H])
        Hm = _homography_from_corners(corners, corners + pert)
        K = int(round(inlier_ratio * N))
        K = min(K, M)
        proj = _apply_h(Hm, k0)
        inside = np.nonzero((proj[:, 0] >= 0) & (proj[:, 0] < IMG_W)
                            & (proj[:, 1] >= 0) & (proj[:, 1] < IMG_H))[0]
        K = min(K, len(inside))          # shortfall is recorded in the GT length
        src = rng.choice(inside, size=K, replace=False)
        kp = proj[src] + rng.standard_normal((K, 2))
        dp = d0[src] + 0.1 * rng.standard_normal((K, d))
        dp /= np.linalg.norm(dp, axis=1, keepdims=True)
        cp = rng.uniform(0.0, 1.0, K)
        kf = _random_points(rng, N - K)
        cf = rng.uniform(0.0, 1.0, N - K)
        df = _random_descriptors(rng, N - K, d)
        k1 = np.concatenate([kp, kf])
        c1 = np.concatenate([cp, cf])
        d1 = np.concatenate([dp, df])
        perm = rng.permutation(N)
        k1, c1, d1 = k1[perm], c1[perm], d1[perm]
        inv = np.empty(N, np.int64)
        inv[perm] = np.arange(N)
        gt = np.stack([src, inv[np.arange(K)]], axis=1)
    return {
        "kpts0": _f32(k0.reshape(M, 2)), "conf0": _f32(c0), "desc0": _f32(d0.reshape(M, d)),
        "kpts1": _f32(k1.reshape(N, 2)), "conf1": _f32(c1), "desc1": _f32(d1.reshape(N, d)),
        "gt_matches": gt,
    }


def make_batch(workload, first_pair: int = 0, n_pairs=None, d: int = D) -> dict:
    """Pairs [first_pair, first_pair+n_pairs) of a workload, stacked as B x n x ...

    Pair p of a workload is drawn from default_rng([workload.seed, p]) alone, so
    any subset of the batch can be regenerated independently.
    """
    w = WORKLOADS[workload] if isinstance(workload, str) else workload
    if n_pairs is None:
        n_pairs = w.B - first_pair
    pairs = []
    for p in range(first_pair, first_pair + n_pairs):
        rng = np.random.default_rng([w.seed, p])
        r = w.inlier
        if isinstance(r, tuple):
            r = float(rng.uniform(r[0], r[1]))
        pairs.append(make_pair(rng, w.M, w.N, r, d))
    out = {}
    for key in ("kpts0", "conf0", "desc0", "kpts1", "conf1", "desc1"):
        out[key] = np.ascontiguousarray(np.stack([p[key] for p in pairs]))
    out["gt_matches"] = [p["gt_matches"] for p in pairs]
    return out
