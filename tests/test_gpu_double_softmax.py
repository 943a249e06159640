"""The double-softmax matching head on the GPU (through the C ABI) against the
float64 oracle: the assignment step on given similarities and matchability
logits, and whole passes with the head in fp32 and bf16."""
import numpy as np
import pytest

from gpu_util import BF16_AGREEMENT, BF16_TOL, FP32_TOL, assert_pair_parity
from learned_sparse_feature_b200 import synth
from oracle import superglue_oracle as O

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

THR = 0.1   # the LightGlue review's default filter threshold


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from learned_sparse_feature_b200 import build
    build.build()
    return torch.device("cuda:0")


def _matcher(weights, B, M, N, precision, **kw):
    from learned_sparse_feature_b200.binding import Matcher
    return Matcher(weights, B, M, N, precision=precision, head="double_softmax", match_threshold=THR, **kw)


@pytest.mark.parametrize("B,M,N", [(1, 1, 1), (1, 63, 65), (2, 127, 129), (1, 3, 700), (3, 700, 5),
                                   (1, 2047, 2049)])
def test_assignment_parity_on_given_inputs(dev, weights, B, M, N):
    rng = np.random.default_rng(500 + M + 3 * N)
    sim = (rng.standard_normal((B, M, N)) * 2.0).astype(np.float32)
    for b in range(B):
        k = min(M, N) // 3
        sim[b, np.arange(k), rng.permutation(N)[:k]] += 8.0     # planted strong pairs
    z0 = (rng.standard_normal((B, M)) * 2.0).astype(np.float32)
    z1 = (rng.standard_normal((B, N)) * 2.0).astype(np.float32)
    m = _matcher(weights, B, M, N, "fp32", n_stages=1)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    lp = torch.empty((B, M + 1, N + 1), device=dev)
    m0 = torch.empty((B, M), dtype=torch.int32, device=dev)
    m1 = torch.empty((B, N), dtype=torch.int32, device=dev)
    s0 = torch.empty((B, M), device=dev)
    s1 = torch.empty((B, N), device=dev)
    m.assign_double_softmax(t(sim), t(z0), t(z1), lp, m0, m1, s0, s1)
    torch.cuda.synchronize()
    assert m.status() == 0
    for b in range(B):
        logP = O.double_softmax_log_assignment(sim[b], z0[b], z1[b])
        r0, r1, rs0, rs1 = O.extract_matches(logP, THR)
        ref = {"log_P": logP, "matches0": r0, "matches1": r1, "mscores0": rs0, "mscores1": rs1}
        out = {"log_P": lp[b].cpu().numpy(), "matches0": m0[b].cpu().numpy(), "matches1": m1[b].cpu().numpy(),
               "mscores0": s0[b].cpu().numpy(), "mscores1": s1[b].cpu().numpy()}
        # float32 log-sum-exps over up to 2049 terms: well inside the fp32 bound
        err = assert_pair_parity(out, ref, 1e-4, thr=THR)
        assert err <= 1e-4
    m.close()


def test_assignment_without_log_p_and_rejections(dev, weights):
    B, M, N = 1, 40, 30
    rng = np.random.default_rng(9)
    sim = torch.from_numpy((rng.standard_normal((B, M, N)) * 3).astype(np.float32)).to(dev)
    z0 = torch.zeros((B, M), device=dev)
    z1 = torch.zeros((B, N), device=dev)
    m = _matcher(weights, B, M, N, "fp32", n_stages=1)
    outs = [torch.empty((B, M), dtype=torch.int32, device=dev), torch.empty((B, N), dtype=torch.int32, device=dev),
            torch.empty((B, M), device=dev), torch.empty((B, N), device=dev)]
    m.assign_double_softmax(sim, z0, z1, None, *outs)          # log P not requested
    torch.cuda.synchronize()
    logP = O.double_softmax_log_assignment(sim[0].cpu().numpy(), np.zeros(M), np.zeros(N))
    r0, _, _, _ = O.extract_matches(logP, THR)
    np.testing.assert_array_equal(outs[0][0].cpu().numpy(), r0)
    from learned_sparse_feature_b200.binding import SgError
    big = torch.zeros((B, M + 1, N), device=dev)
    with pytest.raises(SgError):
        m.assign_double_softmax(big, torch.zeros((B, M + 1), device=dev), z1, None, *outs)
    m.close()


def _run_pass(weights, batch, precision, n_stages=None):
    from learned_sparse_feature_b200.binding import match_batch
    B, M, N = batch["kpts0"].shape[0], batch["kpts0"].shape[1], batch["kpts1"].shape[1]
    kw = {} if n_stages is None else {"n_stages": n_stages}
    m = _matcher(weights, B, M, N, precision, **kw)
    out = match_batch(m, batch, True)
    assert m.status() == 0
    m.close()
    return out


def _oracle(batch, weights, b, **kw):
    return O.superglue_pair(batch["kpts0"][b], batch["conf0"][b], batch["desc0"][b],
                            batch["kpts1"][b], batch["conf1"][b], batch["desc1"][b], weights,
                            head="double_softmax", threshold=THR, **kw)


def test_full_pass_fp32_tiny_pair(dev, weights):
    w = synth.WORKLOADS["pair64_fp32"]
    batch = synth.make_batch(w, 0, 1)
    out = _run_pass(weights, batch, "fp32")
    ref = _oracle(batch, weights, 0)
    pair = {k: v[0] for k, v in out.items()}
    assert_pair_parity(pair, ref, FP32_TOL, thr=THR)


@pytest.mark.parametrize("B,M,N,stages", [(2, 200, 333, 2), (1, 129, 255, 18)])
def test_full_pass_bf16(dev, weights, B, M, N, stages):
    # The head counts the similarity twice (two log-softmaxes, each shifting by a
    # log-sum-exp that moves by at most the largest similarity error), so an
    # error d in sim bounds |d log P| by 4 d: the bf16 bound of this head is
    # that, taken on the similarity the same pass produced, and never above
    # twice the Sinkhorn head's bf16 bound.
    rng = np.random.default_rng(77 + M)
    pairs = [synth.make_pair(rng, M, N, 0.5) for _ in range(B)]
    batch = {k: np.ascontiguousarray(np.stack([p[k] for p in pairs]))
             for k in ("kpts0", "conf0", "desc0", "kpts1", "conf1", "desc1")}
    out = _run_pass(weights, batch, "bf16", n_stages=stages)
    m = _matcher(weights, B, M, N, "bf16", n_stages=stages)
    t = {k: torch.from_numpy(v).to(dev) for k, v in batch.items()}
    S = torch.empty((B, M, N), device=dev)
    m.scores(t["kpts0"], t["conf0"], t["desc0"], t["kpts1"], t["conf1"], t["desc1"], S)
    torch.cuda.synchronize()
    sim = S.double().cpu().numpy()
    m.close()
    for b in range(B):
        ref = _oracle(batch, weights, b, n_stages=stages)
        d_sim = np.abs(sim[b] - ref["scores"]).max()
        tol = min(4.0 * d_sim + 2e-3, 2.0 * BF16_TOL)
        pair = {k: v[b] for k, v in out.items()}
        assert_pair_parity(pair, ref, tol, thr=THR, exact_matches=False, agreement=BF16_AGREEMENT)


def test_scores_entry_returns_the_similarity(dev, weights):
    # with the double-softmax head, sg_scores gives sim = <m0, m1> (D^(1/4) folded)
    w = synth.WORKLOADS["pair64_fp32"]
    batch = synth.make_batch(w, 0, 1)
    M, N = batch["kpts0"].shape[1], batch["kpts1"].shape[1]
    m = _matcher(weights, 1, M, N, "fp32")
    t = {k: torch.from_numpy(np.ascontiguousarray(batch[k])).to(dev)
         for k in ("kpts0", "conf0", "desc0", "kpts1", "conf1", "desc1")}
    S = torch.empty((1, M, N), device=dev)
    m.scores(t["kpts0"], t["conf0"], t["desc0"], t["kpts1"], t["conf1"], t["desc1"], S)
    torch.cuda.synchronize()
    ref = _oracle(batch, weights, 0)["scores"]
    assert np.abs(S[0].double().cpu().numpy() - ref).max() < 1e-3 * max(1.0, np.abs(ref).max())
    m.close()
