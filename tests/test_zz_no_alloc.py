"""The allocation-free transport entry point (sg_optimal_transport_static),
through the C ABI, against the handle-based sg_optimal_transport on the same
scores.  It is for callers that cannot allocate device memory; its scratch is a
static array inside the library.  Kept in a file of its own that pytest
collects last."""
import numpy as np
import pytest

from gpu_util import FP32_TOL

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _outs(B, M, N, dev):
    return (torch.empty((B, M + 1, N + 1), device=dev), torch.empty((B, M), dtype=torch.int32, device=dev),
            torch.empty((B, N), dtype=torch.int32, device=dev), torch.empty((B, M), device=dev),
            torch.empty((B, N), device=dev))


def test_static_scratch_entry_point_matches_handle_entry_point(weights):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from learned_sparse_feature_b200 import build
    build.build()
    from learned_sparse_feature_b200.binding import Matcher, optimal_transport_static
    dev = torch.device("cuda:0")
    B, M, N = 2, 300, 257
    rng = np.random.default_rng(21)
    m = Matcher(weights, B, M, N, precision="fp32", n_stages=1)
    for call in range(2):                       # two calls in a row share the static scratch
        S = torch.from_numpy((rng.standard_normal((B, M, N)) * 3).astype(np.float32)).to(dev)
        ref = _outs(B, M, N, dev)
        m.optimal_transport(S, *ref)
        assert m.status() == 0
        got = _outs(B, M, N, dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        optimal_transport_static(S, *got, status, bin_score=float(weights["bin_score"]))
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        np.testing.assert_allclose(got[0].cpu().numpy(), ref[0].cpu().numpy(), rtol=0, atol=FP32_TOL)
        for g, r in zip(got[1:3], ref[1:3]):
            assert (g.cpu().numpy() == r.cpu().numpy()).mean() > 0.99
        np.testing.assert_allclose(got[3].cpu().numpy(), ref[3].cpu().numpy(), rtol=0, atol=FP32_TOL)
    m.close()
