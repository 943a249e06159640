"""Helpers shared by the GPU parity tests: comparison rules of the parity bar."""
import numpy as np

FP32_TOL = 1e-3      # |d log P| bound of the float32 path
BF16_TOL = 3e-2      # |d log P| bound of the bf16-operand path
MARGIN = 1e-3        # matches are unique only where the decisions have this margin
BF16_AGREEMENT = 0.99


def top2_margins(logP):
    """Per-row and per-column top-1 minus top-2 of the real block."""
    P = np.asarray(logP, np.float64)[:-1, :-1]
    r = np.sort(P, axis=1)
    c = np.sort(P, axis=0)
    m0 = r[:, -1] - r[:, -2] if P.shape[1] > 1 else np.full(P.shape[0], np.inf)
    m1 = c[-1, :] - c[-2, :] if P.shape[0] > 1 else np.full(P.shape[1], np.inf)
    return m0, m1


def decidable_rows(ref, thr, margin0, margin1):
    """Rows of A whose match is uniquely decided: a clear row argmax, a clear
    column argmax for the chosen column, and a score away from the threshold."""
    P = np.asarray(ref["log_P"], np.float64)[:-1, :-1]
    j = P.argmax(1)
    ms = np.exp(P[np.arange(P.shape[0]), j])
    return (margin0 > MARGIN) & (margin1[j] > MARGIN) & (np.abs(ms - thr) > MARGIN)


def decidable_cols(ref, thr, margin0, margin1):
    P = np.asarray(ref["log_P"], np.float64)[:-1, :-1]
    i = P.argmax(0)
    ms = np.exp(P[i, np.arange(P.shape[1])])
    return (margin1 > MARGIN) & (margin0[i] > MARGIN) & (np.abs(ms - thr) > MARGIN)


def assert_pair_parity(out, ref, tol, thr=0.2, exact_matches=True, agreement=None, logP_rows=None):
    """out: GPU outputs of one pair; ref: oracle outputs (log_P may be row-sampled
    via logP_rows)."""
    lp = np.asarray(out["log_P"], np.float64)
    rl = np.asarray(ref["log_P"], np.float64)
    if logP_rows is not None:
        lp = lp[logP_rows]
    d = np.abs(lp - rl)
    assert np.isfinite(lp).all()
    assert d.max() <= tol, f"max |d log P| = {d.max():.3e} > {tol}"
    if "margin0" in ref:
        m0, m1 = ref["margin0"], ref["margin1"]
    else:
        m0, m1 = top2_margins(rl)
    if exact_matches:
        rows = ref["decidable0"] if "decidable0" in ref else decidable_rows(ref, thr, m0, m1)
        cols = ref["decidable1"] if "decidable1" in ref else decidable_cols(ref, thr, m0, m1)
        np.testing.assert_array_equal(out["matches0"][rows], ref["matches0"][rows])
        np.testing.assert_array_equal(out["matches1"][cols], ref["matches1"][cols])
        valid = rows & (ref["matches0"] >= 0)
        np.testing.assert_allclose(out["mscores0"][valid], ref["mscores0"][valid], rtol=2 * tol)
    if agreement is not None:
        agree = np.concatenate([out["matches0"] == ref["matches0"], out["matches1"] == ref["matches1"]])
        assert agree.mean() >= agreement, f"match agreement {agree.mean():.4f} < {agreement}"
    return d.max()
