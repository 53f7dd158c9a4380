"""GPU codec fit (lla_fit_codec) against the oracle's FP64 SVD fit.

[LLA §3, "Initialisation and conversion"]: mu is the mean of the calibration stacks and W_down
the top-r right singular vectors of the centred stacks, each column's largest-magnitude entry
positive.  The GPU fit is an iteration (subspace iteration + Rayleigh-Ritz in fp64), so the bar
is stated per quantity:
  - mu within float rounding of the oracle's mean;
  - the top-r singular values within 2e-6 of the largest;
  - the fitted subspace: the reconstruction objective ||Xc - Xc W Wᵀ||² within 1e-5 (relative)
    of the optimum (the oracle's tail energy) plus float rounding of W;
  - single columns where the spectrum has a clear gap (both neighbours >= 1% of sigma_0 away):
    equal to the oracle's column, sign included, within 1e-4.
Inputs are the seeded smooth loop stacks (rank-R trajectories plus noise) of the test configs,
on both sides of the Gram choice (n >= S: S x S Gram; n < S: n x n Gram).
"""

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import decode_attention_lla_b200 as lla  # noqa: E402
import lla_synth as syn  # noqa: E402
from oracle import lla_oracle as O  # noqa: E402

DEV = "cuda"

CASES = [
    # (problems, n, T, d, R, noise_var, r)
    (3, 512, 4, 16, 6, 1e-3, 4),      # the tiny config's K rank (lossy: r < R)
    (3, 512, 4, 16, 6, 1e-3, 8),      # its V rank (r > R: noise columns included)
    (2, 300, 4, 32, 12, 1e-2, 16),
    (2, 200, 8, 64, 24, 1e-2, 40),    # n < S: the n x n Gram and back-projection
    (2, 1024, 4, 128, 24, 1e-2, 96),  # the ratio-4 K rank at S = 512
    (1, 1024, 4, 128, 24, 1e-2, 160), # the ratio-4 V rank
    (2, 256, 1, 2048, 24, 1e-2, 64),  # a 2D-like stack over 16 heads x 128 (S = 2048), n < S
    (2, 40, 2, 8, 3, 1e-3, 1),        # rank 1; the block is the whole space (k = m = 16)
]


def _stacks(tag, P, n, T, d, R, noise):
    X = np.stack([syn.smooth_stacks(f"{tag}/{p}", n, T, d, R, noise, syn.gaussian(f"{tag}/mu/{p}", T * d, 0.1))
                  for p in range(P)])
    return X.astype(np.float32)


def _fit_gpu(X, r, iters=0):
    P, n, S = X.shape
    Xd = torch.from_numpy(X).to(DEV)
    mu = torch.empty(P, S, device=DEV)
    W = torch.empty(P, S, r, device=DEV)
    sig = torch.empty(P, r, device=DEV)
    ws = torch.empty(lla.fit_codec_workspace_bytes(P, n, S, r), dtype=torch.uint8, device=DEV)
    lla.fit_codec(P, n, S, r, Xd, mu, W, sig, ws, iters=iters)
    torch.cuda.synchronize()
    return (mu.cpu().numpy().astype(np.float64), W.cpu().numpy().astype(np.float64),
            sig.cpu().numpy().astype(np.float64), lla.workspace_flags(ws))


@pytest.mark.parametrize("case", CASES)
def test_fit_matches_oracle(case):
    P, n, T, d, R, noise, r = case
    S = T * d
    X = _stacks(f"fit/{n}/{S}/{r}", P, n, T, d, R, noise)
    mu_g, W_g, sig_g, flags = _fit_gpu(X, r)
    assert flags == 0
    for p in range(P):
        Xp = X[p].astype(np.float64)
        mu_o, W_o, s_o = O.fit_codec_svd(Xp, r)
        assert np.abs(mu_g[p] - mu_o).max() <= 1e-6 * np.abs(mu_o).max() + 1e-7
        assert np.abs(sig_g[p] - s_o[:r]).max() <= 2e-6 * s_o[0], (p, np.abs(sig_g[p] - s_o[:r]).max() / s_o[0])
        Xc = Xp - mu_o
        W = W_g[p]
        e_gpu = np.linalg.norm(Xc - Xc @ W @ W.T) ** 2
        e_opt = float(np.sum(s_o[r:] ** 2))
        total = float(np.sum(s_o ** 2))
        assert e_gpu - e_opt <= 1e-5 * e_opt + 1e-6 * total, (p, e_gpu, e_opt)
        # columns with a clear gap on both sides are unique up to sign, and the sign is fixed
        gap = np.abs(np.diff(s_o[:r + 1])) / s_o[0]
        for a in range(r):
            if (a == 0 or gap[a - 1] >= 1e-2) and gap[a] >= 1e-2:
                assert np.abs(W[:, a] - W_o[:, a]).max() <= 1e-4, (p, a)
        # sign convention on every column: the entry of largest magnitude is positive
        top = np.abs(W).argmax(axis=0)
        vals = W[top, np.arange(r)]
        second = np.sort(np.abs(W), axis=0)[-2]
        assert np.all((vals > 0) | (np.abs(vals) - second <= 1e-6))


def test_fit_full_rank_is_exact():
    """r = min(n, S): the fitted basis spans every centred stack, so the objective is zero."""
    X = _stacks("fit/full", 2, 96, 2, 24, 5, 1e-2)  # S = 48 < n
    _, W, sig, flags = _fit_gpu(X, 48)
    assert flags == 0
    for p in range(2):
        Xc = X[p].astype(np.float64) - X[p].astype(np.float64).mean(0)
        assert np.linalg.norm(Xc - Xc @ W[p] @ W[p].T) <= 1e-5 * np.linalg.norm(Xc)
        assert np.abs(W[p].T @ W[p] - np.eye(48)).max() <= 1e-5
        s = np.linalg.svd(Xc, compute_uv=False)
        assert np.abs(sig[p] - s).max() <= 2e-6 * s[0]


def test_fit_more_iterations_do_not_hurt():
    X = _stacks("fit/iters", 1, 300, 4, 32, 12, 1e-2)
    r = 16
    s = np.linalg.svd(X[0].astype(np.float64) - X[0].astype(np.float64).mean(0), compute_uv=False)
    errs = []
    for it in (4, 16, 40):
        _, _, sig, _ = _fit_gpu(X, r, iters=it)
        errs.append(np.abs(sig[0] - s[:r]).max() / s[0])
    assert errs[2] <= errs[0] + 1e-7 and errs[2] <= 2e-6


def test_fit_argument_errors():
    buf = torch.zeros(1 << 12, device=DEV)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=DEV)
    with pytest.raises(lla.LLAError) as e:  # r above min(n, S)
        lla.fit_codec(1, 10, 8, 9, buf, buf, buf, None, ws)
    assert e.value.status == 1
    with pytest.raises(lla.LLAError) as e:  # a block of more than 1024 columns
        lla.fit_codec(1, 4096, 4096, 600, buf, buf, buf, None, ws)
    assert e.value.status == 2
    with pytest.raises(lla.LLAError) as e:  # workspace too small
        lla.fit_codec(4, 512, 512, 32, buf, buf, buf, None, ws)
    assert e.value.status == 6
    lla.fit_codec(0, 512, 512, 32, buf, buf, buf, None, ws)  # no problems: nothing to do


def test_fit_full_size_sampled():
    """All 384 (layer, head) problems of the ratio-4 V axis (1024 stacks of S = 512, r = 160) in one
    call, as bench.py --mode fit runs them: four distinct seeded sets repeated over the batch.  Each
    problem starts its iteration from its own pseudo-random block, so repeats agree to the
    iteration's accuracy; one of each set is checked against the oracle."""
    P, n, T, d, R, r = 384, 1024, 4, 128, 24, 160
    base = _stacks("fit/fullsize", 4, n, T, d, R, 1e-2)
    X = np.concatenate([base] * (P // 4))
    mu_g, W_g, sig_g, flags = _fit_gpu(X, r)
    assert flags == 0
    for p in (0, 1, 2, 3):
        Xp = base[p].astype(np.float64)
        mu_o, W_o, s_o = O.fit_codec_svd(Xp, r)
        for rep in (p + 4, p + 4 * 57, p + 4 * 95):
            assert np.array_equal(mu_g[rep], mu_g[p])
            assert np.abs(sig_g[rep] - sig_g[p]).max() <= 4e-6 * s_o[0]
        assert np.abs(mu_g[p] - mu_o).max() <= 1e-6 * np.abs(mu_o).max() + 1e-7
        assert np.abs(sig_g[p] - s_o[:r]).max() <= 2e-6 * s_o[0]
        Xc = Xp - mu_o
        e_gpu = np.linalg.norm(Xc - Xc @ W_g[p] @ W_g[p].T) ** 2
        e_opt = float(np.sum(s_o[r:] ** 2))
        assert e_gpu - e_opt <= 1e-5 * e_opt + 1e-6 * float(np.sum(s_o ** 2))
