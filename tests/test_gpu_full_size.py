"""The bench workloads at their full sizes, in the launch configuration bench.py
times (one handle sized for the workload, bf16, the whole batch in one call),
against the float64 oracle on sampled pairs, plus properties that hold for
every pair of the batch: after the last column update of Sinkhorn each real
column of exp(log P) sums to 1 and the dustbin column to M."""
import numpy as np
import pytest

from gpu_util import BF16_AGREEMENT, BF16_TOL, assert_pair_parity
from learned_sparse_feature_b200 import synth
from oracle import superglue_oracle as O

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from learned_sparse_feature_b200 import build
    build.build()
    return torch.device("cuda:0")


def _run_workload(weights, name):
    from learned_sparse_feature_b200.binding import Matcher, match_batch
    w = synth.WORKLOADS[name]
    batch = synth.make_batch(w, 0, w.B)
    m = Matcher(weights, w.B, w.M, w.N, precision=w.precision)
    out = match_batch(m, batch, True)
    assert m.status() == 0
    m.close()
    return w, batch, out


def _check_marginals(logP, M):
    P = np.exp(np.asarray(logP, np.float64))
    cols = P[:, :-1].sum(axis=0)
    assert np.abs(cols - 1.0).max() < 1e-3, np.abs(cols - 1.0).max()
    assert abs(P[:, -1].sum() - M) < 1e-3 * M


def _check_pair(batch, weights, out, b, w):
    ref = O.superglue_pair(batch["kpts0"][b], batch["conf0"][b], batch["desc0"][b],
                           batch["kpts1"][b], batch["conf1"][b], batch["desc1"][b], weights)
    pair = {k: v[b] for k, v in out.items()}
    assert_pair_parity(pair, ref, BF16_TOL, thr=synth.MATCH_THRESHOLD, exact_matches=False,
                       agreement=BF16_AGREEMENT)


def test_pair2048_full(dev, weights):
    w, batch, out = _run_workload(weights, "pair2048")
    _check_marginals(out["log_P"][0], w.M)
    _check_pair(batch, weights, out, 0, w)


def test_batch32_pair1024_full(dev, weights):
    w, batch, out = _run_workload(weights, "batch32_pair1024")
    for b in range(w.B):
        _check_marginals(out["log_P"][b], w.M)
    for b in (0, 17):
        _check_pair(batch, weights, out, b, w)


def test_batch8_pair4096x3072_full(dev, weights):
    w, batch, out = _run_workload(weights, "batch8_pair4096x3072")
    for b in range(w.B):
        _check_marginals(out["log_P"][b], w.M)
    _check_pair(batch, weights, out, 5, w)
