"""CUDA path (through the C ABI) against the float64 oracle on the same seeded
inputs.  Needs a B200 and the built library."""
import numpy as np
import pytest

from gpu_util import BF16_AGREEMENT, BF16_TOL, FP32_TOL, assert_pair_parity
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


def _matcher(weights, B, M, N, precision, **kw):
    from learned_sparse_feature_b200.binding import Matcher
    return Matcher(weights, B, M, N, precision=precision, **kw)


def _run(m, batch, with_logP=True):
    from learned_sparse_feature_b200.binding import match_batch
    return match_batch(m, batch, with_logP)


def _pair(out, b):
    return {k: (v[b] if v is not None else None) for k, v in out.items()}


def _oracle(batch, weights, b, **kw):
    return O.superglue_pair(batch["kpts0"][b], batch["conf0"][b], batch["desc0"][b],
                            batch["kpts1"][b], batch["conf1"][b], batch["desc1"][b], weights, **kw)


def _random_batch(B, M, N, seed, inlier=0.5):
    rng = np.random.default_rng(seed)
    pairs = [synth.make_pair(rng, M, N, inlier) for _ in range(B)]
    return {k: np.ascontiguousarray(np.stack([p[k] for p in pairs]))
            for k in ("kpts0", "conf0", "desc0", "kpts1", "conf1", "desc1")}


# --------------------------------------------------------------------------- transport only
@pytest.mark.parametrize("B,M,N", [(1, 1, 1), (1, 63, 65), (2, 127, 129), (1, 3, 700), (1, 512, 512),
                                   (3, 700, 5), (1, 2047, 2049)])
def test_sinkhorn_extraction_parity(dev, weights, B, M, N):
    rng = np.random.default_rng(100 + M + N)
    S = (rng.standard_normal((B, M, N)) * 2.5).astype(np.float32)
    # plant a few strong matches so that the extraction has work to do
    for b in range(B):
        k = min(M, N) // 3
        S[b, np.arange(k), rng.permutation(N)[:k]] += 9.0
    m = _matcher(weights, B, M, N, "fp32", n_stages=1)
    St = torch.from_numpy(S).to(dev)
    lp = torch.empty((B, M + 1, N + 1), device=dev)
    m0 = torch.empty((B, M), dtype=torch.int32, device=dev)
    m1 = torch.empty((B, N), dtype=torch.int32, device=dev)
    s0 = torch.empty((B, M), device=dev)
    s1 = torch.empty((B, N), device=dev)
    m.optimal_transport(St, lp, m0, m1, s0, s1)
    assert m.status() == 0
    for b in range(B):
        ref_lp = O.log_optimal_transport(S[b].astype(np.float64), 1.0, 100)
        r0, r1, q0, q1 = O.extract_matches(ref_lp, 0.2)
        ref = {"log_P": ref_lp, "matches0": r0, "matches1": r1, "mscores0": q0, "mscores1": q1}
        out = {"log_P": lp[b].cpu().numpy(), "matches0": m0[b].cpu().numpy(),
               "matches1": m1[b].cpu().numpy(), "mscores0": s0[b].cpu().numpy(),
               "mscores1": s1[b].cpu().numpy()}
        assert_pair_parity(out, ref, FP32_TOL)
    m.close()


def test_sinkhorn_column_marginals_exact(dev, weights):
    # v is updated last, so the columns of exp(log P) sum to b = [1_N; M]
    rng = np.random.default_rng(7)
    M, N = 300, 200
    S = (rng.standard_normal((1, M, N)) * 3).astype(np.float32)
    m = _matcher(weights, 1, M, N, "fp32", n_stages=1)
    lp = torch.empty((1, M + 1, N + 1), device=dev)
    outs = [torch.empty((1, M), dtype=torch.int32, device=dev), torch.empty((1, N), dtype=torch.int32, device=dev),
            torch.empty((1, M), device=dev), torch.empty((1, N), device=dev)]
    m.optimal_transport(torch.from_numpy(S).to(dev), lp, *outs)
    P = np.exp(lp[0].double().cpu().numpy())
    np.testing.assert_allclose(P.sum(0), np.r_[np.ones(N), M], rtol=2e-4)
    m.close()


def test_sinkhorn_extreme_scores_take_exact_fallback(dev, weights):
    # scores spread over +-60 make the predicted shifts underflow on the first
    # iterations; the exact recomputation must keep the result on the oracle
    rng = np.random.default_rng(8)
    M, N = 40, 50
    S = (rng.uniform(-60, 60, (1, M, N))).astype(np.float32)
    m = _matcher(weights, 1, M, N, "fp32", n_stages=1)
    lp = torch.empty((1, M + 1, N + 1), device=dev)
    outs = [torch.empty((1, M), dtype=torch.int32, device=dev), torch.empty((1, N), dtype=torch.int32, device=dev),
            torch.empty((1, M), device=dev), torch.empty((1, N), device=dev)]
    m.optimal_transport(torch.from_numpy(S).to(dev), lp, *outs)
    assert m.status() == 0
    ref = O.log_optimal_transport(S[0].astype(np.float64), 1.0, 100)
    got = lp[0].double().cpu().numpy()
    # compare where the plan carries mass (log P > -60): elsewhere fp32 exp underflows
    mask = ref > -60
    assert np.abs(got - ref)[mask].max() <= 5e-3
    m.close()


# --------------------------------------------------------------------------- whole pass
def test_full_pass_fp32_tiny_pair(dev, weights):
    batch = synth.make_batch("pair64_fp32")
    m = _matcher(weights, 1, 64, 64, "fp32")
    out = _run(m, batch)
    ref = _oracle(batch, weights, 0)
    assert_pair_parity(_pair(out, 0), ref, FP32_TOL)
    m.close()


@pytest.mark.parametrize("B,M,N,stages", [(2, 37, 91, 4), (1, 130, 1, 2), (1, 1, 65, 2), (3, 129, 127, 3)])
def test_full_pass_fp32_ragged(dev, weights, B, M, N, stages):
    batch = _random_batch(B, M, N, seed=M * 7 + N)
    m = _matcher(weights, B, M, N, "fp32", n_stages=stages)
    out = _run(m, batch)
    for b in range(B):
        assert_pair_parity(_pair(out, b), _oracle(batch, weights, b, n_stages=stages), FP32_TOL)
    m.close()


@pytest.mark.parametrize("B,M,N,stages", [(2, 200, 333, 4), (1, 129, 255, 18)])
def test_full_pass_bf16_ragged(dev, weights, B, M, N, stages):
    batch = _random_batch(B, M, N, seed=M + 3 * N)
    m = _matcher(weights, B, M, N, "bf16", n_stages=stages)
    out = _run(m, batch)
    for b in range(B):
        assert_pair_parity(_pair(out, b), _oracle(batch, weights, b, n_stages=stages), BF16_TOL,
                           exact_matches=False, agreement=BF16_AGREEMENT)
    m.close()


def test_full_pass_bf16_pair512(dev, weights):
    batch = synth.make_batch("pair512")
    m = _matcher(weights, 1, 512, 512, "bf16")
    out = _run(m, batch)
    ref = _oracle(batch, weights, 0)
    assert_pair_parity(_pair(out, 0), ref, BF16_TOL, exact_matches=False, agreement=BF16_AGREEMENT)
    m.close()


def test_scores_entry_point(dev, weights):
    batch = _random_batch(2, 70, 50, seed=5)
    m = _matcher(weights, 2, 70, 50, "fp32", n_stages=2)
    t = {k: torch.from_numpy(v).to(dev) for k, v in batch.items()}
    S = torch.empty((2, 70, 50), device=dev)
    m.scores(t["kpts0"], t["conf0"], t["desc0"], t["kpts1"], t["conf1"], t["desc1"], S)
    for b in range(2):
        ref = _oracle(batch, weights, b, n_stages=2)["scores"]
        np.testing.assert_allclose(S[b].double().cpu().numpy(), ref, atol=2e-4, rtol=0)
    m.close()


def test_host_buffer_entry_point_matches_device_entry_point(dev, weights):
    batch = _random_batch(2, 100, 80, seed=6)
    m = _matcher(weights, 2, 100, 80, "bf16", n_stages=2)
    dev_out = _run(m, batch)
    host = {k: np.ascontiguousarray(batch[k]) for k in ("kpts0", "conf0", "desc0", "kpts1", "conf1", "desc1")}
    lp = np.empty((2, 101, 81), np.float32)
    m0 = np.empty((2, 100), np.int32)
    m1 = np.empty((2, 80), np.int32)
    s0 = np.empty((2, 100), np.float32)
    s1 = np.empty((2, 80), np.float32)
    m.match_host(host["kpts0"], host["conf0"], host["desc0"], host["kpts1"], host["conf1"], host["desc1"],
                 lp, m0, m1, s0, s1)
    # the Sinkhorn column sums are fp32 atomics: run-to-run differences are
    # rounding-level, not bitwise zero
    np.testing.assert_allclose(lp, dev_out["log_P"], rtol=0, atol=2e-5)
    assert (m0 == dev_out["matches0"]).mean() > 0.99
    assert (m1 == dev_out["matches1"]).mean() > 0.99
    m.close()


# --------------------------------------------------------------------------- edge cases
def test_empty_inputs_give_unmatched(dev, weights):
    m = _matcher(weights, 2, 16, 16, "bf16", n_stages=2)
    for M, N in [(0, 5), (7, 0), (0, 0)]:
        k0 = torch.zeros((2, M, 2), device=dev)
        c0 = torch.zeros((2, M), device=dev)
        d0 = torch.zeros((2, M, 256), device=dev)
        k1 = torch.zeros((2, N, 2), device=dev)
        c1 = torch.zeros((2, N), device=dev)
        d1 = torch.zeros((2, N, 256), device=dev)
        m0 = torch.full((2, M), 7, dtype=torch.int32, device=dev)
        m1 = torch.full((2, N), 7, dtype=torch.int32, device=dev)
        s0 = torch.full((2, M), 7.0, device=dev)
        s1 = torch.full((2, N), 7.0, device=dev)
        m.match(k0, c0, d0, k1, c1, d1, None, m0, m1, s0, s1)
        assert m.status() == 0
        assert (m0 == -1).all() and (m1 == -1).all() and (s0 == 0).all() and (s1 == 0).all()
    m.close()


def test_shape_errors_are_reported(dev, weights):
    from learned_sparse_feature_b200.binding import SgError
    m = _matcher(weights, 1, 16, 16, "fp32", n_stages=1)
    batch = _random_batch(1, 17, 16, seed=9)
    with pytest.raises(SgError) as e:
        _run(m, batch)
    assert e.value.code == 2
    m.close()


def test_barrier_wait_times_out_and_context_survives(dev, weights):
    m = _matcher(weights, 1, 64, 64, "fp32")
    assert m.selftest_barrier_timeout(20000) == 5      # SG_ERR_TIMEOUT
    assert m.status() == 0                              # cleared once read
    batch = synth.make_batch("pair64_fp32")
    out = _run(m, batch)                                # the context is still usable
    assert_pair_parity(_pair(out, 0), _oracle(batch, weights, 0), FP32_TOL)
    m.close()


def test_non_finite_input_is_reported(dev, weights):
    M, N = 20, 30
    S = np.zeros((1, M, N), np.float32)
    S[0, 3, 4] = np.nan
    m = _matcher(weights, 1, M, N, "fp32", n_stages=1)
    lp = torch.empty((1, M + 1, N + 1), device=dev)
    outs = [torch.empty((1, M), dtype=torch.int32, device=dev), torch.empty((1, N), dtype=torch.int32, device=dev),
            torch.empty((1, M), device=dev), torch.empty((1, N), device=dev)]
    m.optimal_transport(torch.from_numpy(S).to(dev), lp, *outs)
    assert m.status() == 6                              # SG_ERR_NUMERIC
    m.close()


@pytest.mark.parametrize("B,M,N", [(1, 300, 200), (2, 128, 256), (3, 65, 190)])
def test_tensor_core_path_matches_cuda_core_path(dev, weights, B, M, N, monkeypatch):
    # same bf16 operands, fp32 accumulation in both: only the summation order differs
    batch = _random_batch(B, M, N, seed=B * 1000 + M)
    t = {k: torch.from_numpy(v).to(dev) for k, v in batch.items()}
    out = []
    for force_simt in (False, True):
        if force_simt:
            monkeypatch.setenv("SG_FORCE_SIMT", "1")
        m = _matcher(weights, B, M, N, "bf16", n_stages=2)
        S = torch.empty((B, M, N), device=dev)
        m.scores(t["kpts0"], t["conf0"], t["desc0"], t["kpts1"], t["conf1"], t["desc1"], S)
        assert m.status() == 0
        out.append(S.double().cpu().numpy())
        m.close()
    assert np.abs(out[0] - out[1]).max() < 2e-2 * max(1.0, np.abs(out[1]).max() / 10)
    for b in range(B):
        ref = _oracle(batch, weights, b, n_stages=2)["scores"]
        assert np.abs(out[0][b] - ref).max() < 5e-2


@pytest.mark.parametrize("B,M,N,cross_only", [(1, 300, 200, False), (2, 129, 257, False), (1, 1, 700, False)])
def test_tensor_core_attention_matches_cuda_core_attention(dev, weights, B, M, N, cross_only, monkeypatch):
    batch = _random_batch(B, M, N, seed=B * 77 + N)
    t = {k: torch.from_numpy(v).to(dev) for k, v in batch.items()}
    out = []
    for simt in (False, True):
        if simt:
            monkeypatch.setenv("SG_SIMT_ATTENTION", "1")
        m = _matcher(weights, B, M, N, "bf16", n_stages=2)
        S = torch.empty((B, M, N), device=dev)
        m.scores(t["kpts0"], t["conf0"], t["desc0"], t["kpts1"], t["conf1"], t["desc1"], S)
        assert m.status() == 0
        out.append(S.double().cpu().numpy())
        m.close()
    assert np.abs(out[0] - out[1]).max() < 2e-2 * max(1.0, np.abs(out[1]).max() / 10)


@pytest.mark.gpu
def test_fma_pipe_exp2_against_float64_and_cuda_exp2(dev):
    from learned_sparse_feature_b200 import binding
    xs = np.concatenate([np.linspace(-125.0, 126.0, 200001), np.linspace(-1.0, 1.0, 4001),
                         np.array([0.0, 0.5, -0.5, 1e-7, -1e-7, 63.5, 64.49, -124.999])]).astype(np.float32)
    x = torch.from_numpy(xs).to(dev)
    y = torch.empty_like(x)
    binding.selftest_exp2_poly(x, y)
    torch.cuda.synchronize()
    got = y.double().cpu().numpy()
    ref = np.exp2(xs.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1e-4, (rel.max(), xs[rel.argmax()])
    # and against CUDA's own exp2 (fp32) on the same inputs
    cu = torch.exp2(x).double().cpu().numpy()
    assert np.abs(got / cu - 1.0).max() < 1.1e-4
    # clamping: far outside [-125, 126] the result saturates at the clamp values
    xo = torch.tensor([-1e4, -300.0, 300.0, 1e4, float("-inf")], device=dev)
    yo = torch.empty_like(xo)
    binding.selftest_exp2_poly(xo, yo)
    torch.cuda.synchronize()
    vo = yo.double().cpu().numpy()
    assert np.all(np.abs(vo[[0, 1, 4]] / 2.0 ** -125 - 1) < 1e-4)
    assert np.all(np.abs(vo[[2, 3]] / 2.0 ** 126 - 1) < 1e-4)
    # odd length: the last element is computed, nothing past it is written
    x3 = torch.tensor([1.0, 2.0, 3.0], device=dev)
    y3 = torch.full((4,), -7.0, device=dev)
    binding.selftest_exp2_poly(x3, y3[:3])
    torch.cuda.synchronize()
    v3 = y3.cpu().numpy()
    assert np.allclose(v3[:3], [2.0, 4.0, 8.0], rtol=1e-4) and v3[3] == -7.0


@pytest.mark.gpu
@pytest.mark.parametrize("emu", ["2", "3", "4"])
def test_attention_exp_share_variants_agree(dev, weights, emu, monkeypatch):
    # the split of exponentials between MUFU and FMA pipe changes rounding only
    B, M, N = 2, 200, 333
    batch = _random_batch(B, M, N, seed=4242)
    t = {k: torch.from_numpy(v).to(dev) for k, v in batch.items()}
    out = []
    for share in ("0", emu):
        monkeypatch.setenv("SG_ATTN_EXP_EMU", share)
        m = _matcher(weights, B, M, N, "bf16", n_stages=2)
        S = torch.empty((B, M, N), device=dev)
        m.scores(t["kpts0"], t["conf0"], t["desc0"], t["kpts1"], t["conf1"], t["desc1"], S)
        assert m.status() == 0
        out.append(S.double().cpu().numpy())
        m.close()
    assert np.abs(out[0] - out[1]).max() < 2e-2 * max(1.0, np.abs(out[1]).max() / 10)
    for b in range(B):
        ref = _oracle(batch, weights, b, n_stages=2)["scores"]
        assert np.abs(out[1][b] - ref).max() < 5e-2


@pytest.mark.gpu
def test_attention_max_renewal_path(dev, weights, monkeypatch):
    # with the bound on a tile's sum lowered to 1, nearly every key tile renews
    # its rows' reference max and rescales the TMEM output rows; the result must
    # not change beyond rounding
    B, M, N = 1, 300, 700
    batch = _random_batch(B, M, N, seed=777)
    t = {k: torch.from_numpy(v).to(dev) for k, v in batch.items()}
    out = []
    for lim in ("64", "0"):
        monkeypatch.setenv("SG_ATTN_BLIND_LIMIT_LOG2", lim)
        m = _matcher(weights, B, M, N, "bf16", n_stages=2)
        S = torch.empty((B, M, N), device=dev)
        m.scores(t["kpts0"], t["conf0"], t["desc0"], t["kpts1"], t["conf1"], t["desc1"], S)
        assert m.status() == 0
        out.append(S.double().cpu().numpy())
        m.close()
    assert np.abs(out[0] - out[1]).max() < 2e-2 * max(1.0, np.abs(out[1]).max() / 10)
    ref = _oracle(batch, weights, 0, n_stages=2)["scores"]
    assert np.abs(out[1][0] - ref).max() < 5e-2


# --------------------------------------------------------------------------- timing hooks
def test_profile_modes_record_classes_and_segments(dev, weights):
    batch = _random_batch(1, 200, 150, seed=8)
    m = _matcher(weights, 1, 200, 150, "bf16", n_stages=4)
    ref = _run(m, batch)
    m.profile(True)
    out = _run(m, batch)
    per_kernel = m.profile_read()
    m.profile(True, segments=True)
    out_seg = _run(m, batch)
    per_seg = m.profile_read()
    m.profile(False)
    # timing events do not change the results
    for o in (out, out_seg):
        np.testing.assert_array_equal(o["matches0"], ref["matches0"])
    assert per_kernel["attention"][1] == 4 and per_kernel["qkv_gemm"][1] == 4
    assert per_kernel["gnn"] == (0.0, 0)
    # segment mode: encoder, the GNN as one interval, the assignment step
    assert per_seg["gnn"][1] == 1 and per_seg["gnn"][0] > 0
    assert per_seg["encoder"][1] == 1 and per_seg["sinkhorn"][1] == 1
    for k in ("qkv_gemm", "attention", "mlp1_gemm", "mlp2_gemm", "proj_gemm", "score_gemm"):
        assert per_seg[k] == (0.0, 0)
    assert m.lib.sg_profile(m.h, 3) == 1          # SG_ERR_INVALID_ARG
    m.close()
