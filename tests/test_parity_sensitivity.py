"""The GPU parity inputs can fail: planted score-path mistakes miss the acceptance bar.

For every decode input set the GPU tests compare with the oracle (``parity_cases.decode_sets``,
full-size samples included) and for the full-cache comparator's sets, the oracle's own output
under a planted mistake is fed to the same error measures the GPU tests assert on.  Each mistake
must miss the bar by a factor of two, so that a kernel making it fails even if its rounding error
(up to the bar) happened to pull toward the reference.

The mistakes are the plausible slips in the score path [LLA §3 eq. (3), then RoPE after
reconstruction, "RoPE and reconstruction"; softmax attention]: the query rotated one position
off either way, a sequence's last cached token left out, the softmax scale 10% off, uniform
attention (scores ignored), and keys rotated at positions 1..n instead of 0..n-1.  They are
planted in the oracle on the CPU.
"""

from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest

import parity_cases as PC
from lla_testutil import MAX_ABS_TOL, REL_L2_TOL
from oracle import lla_oracle as O

MARGIN = 2.0


def _keys_one_position_late(q, cK, cV, muK_t, WupK_t, muV_t, WupV_t, pos_q, scale, base, k_self=None, v_self=None):
    """The oracle's per-head decode with keys rotated at 1..n (a planted mistake)."""
    n = np.asarray(cK).shape[0]
    K_rot = O.apply_rope(O.reconstruct(cK, WupK_t, muK_t), np.arange(1, n + 1), base)
    V_hat = O.reconstruct(cV, WupV_t, muV_t)
    q_rot = O.apply_rope(q, pos_q, base)
    if k_self is not None:
        K_rot = np.vstack([K_rot, O.apply_rope(k_self, pos_q, base)[None]])
        V_hat = np.vstack([V_hat, np.asarray(v_self, np.float64)[None]])
    return O.softmax_attention(q_rot, K_rot, V_hat, scale)


def _reference_and_mutations(case):
    """The oracle's output and its outputs under each planted mistake.  The oracle's NumPy loops
    release the GIL, so the calls that change only arguments run on threads; the one that swaps
    an oracle function runs alone afterwards."""
    calls = {"reference": {},
             "query position +1": dict(qpos=[p + 1 for p in case.qpos]),
             "query position -1": dict(qpos=[p - 1 for p in case.qpos]),
             "last cached token dropped": dict(lens=[max(0, n - 1) for n in case.lens]),
             "softmax scale x0.9": dict(scale=0.9 * case.scale),
             "uniform attention": dict(scale=0.0)}
    with ThreadPoolExecutor(len(calls)) as ex:
        futs = {k: ex.submit(case.reference, **kw) for k, kw in calls.items()}
        outs = {k: f.result() for k, f in futs.items()}
    orig = O.lla_decode_head
    O.lla_decode_head = _keys_one_position_late
    try:
        outs["keys at positions 1..n"] = case.reference()
    finally:
        O.lla_decode_head = orig
    return outs.pop("reference"), outs


def _misses_bar(errs) -> bool:
    e_out, e_att, m = errs
    return max(e_out, e_att) >= MARGIN * REL_L2_TOL or m >= MARGIN * MAX_ABS_TOL


SETS = PC.decode_sets()


@pytest.mark.parametrize("name", list(SETS))
def test_planted_score_path_mistakes_miss_the_bar(name):
    for case in SETS[name]():
        ref, muts = _reference_and_mutations(case)
        mv = case.mu_v()
        assert np.isfinite(ref).all()
        for what, out in muts.items():
            errs = PC.decode_errors(out, ref, mv)
            assert _misses_bar(errs), (f"{case.name}: '{what}' gives rel_l2={errs[0]:.2e} "
                                       f"rel_l2(out-mu_v)={errs[1]:.2e} max_abs={errs[2]:.2e}")


@pytest.mark.parametrize("ci", range(len(PC.FULL_CACHE)))
def test_planted_mistakes_miss_the_bar_on_the_full_cache(ci):
    c, Kr, V, q, qpos, scale = PC.full_cache_inputs(ci)
    layer = c["L"] - 1
    lens = c["lens"]
    run = lambda lens=lens, qpos=qpos, scale=scale: O.full_decode(q, Kr[:, layer], V[:, layer], lens, qpos, scale,
                                                                  PC.ROPE_BASE)
    ref = run()
    zero = np.zeros((c["H"], 128))
    muts = {"last cached token dropped": run(lens=[max(0, n - 1) for n in lens])}
    if max(lens) > 1:  # with one cached token the softmax weight is 1 whatever the score
        muts.update({"query position +1": run(qpos=[p + 1 for p in qpos]),
                     "query position -1": run(qpos=[p - 1 for p in qpos]),
                     "softmax scale x0.9": run(scale=0.9 * scale),
                     "uniform attention": run(scale=0.0)})
    for what, out in muts.items():
        errs = PC.decode_errors(out, ref, zero)
        assert _misses_bar(errs), f"full cache {ci}: '{what}' gives {errs}"


def test_planted_mistakes_miss_the_bar_on_the_full_size_full_cache():
    f = PC.full_cache_full_size_sample()
    K = f["K"].transpose(0, 2, 1, 3)  # [sample][token][head][d], the oracle's order
    V = f["V"].transpose(0, 2, 1, 3)
    run = lambda lens=f["lens"], qpos=f["qpos"], scale=f["scale"]: O.full_decode(f["q"], K, V, lens, qpos, scale,
                                                                                PC.ROPE_BASE)
    ref = run()
    zero = np.zeros(f["q"].shape[1:])
    muts = {"last cached token dropped": run(lens=[n - 1 for n in f["lens"]]),
            "query position +1": run(qpos=[p + 1 for p in f["qpos"]]),
            "query position -1": run(qpos=[p - 1 for p in f["qpos"]]),
            "softmax scale x0.9": run(scale=0.9 * f["scale"]),
            "uniform attention": run(scale=0.0)}
    for what, out in muts.items():
        errs = PC.decode_errors(out, ref, zero)
        assert _misses_bar(errs), f"full cache, full size: '{what}' gives {errs}"
