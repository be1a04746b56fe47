"""Plant plausible mistakes in a copy of the oracle and check that the pins catch each one.

The copy is made from the oracle's source text with one substitution; the
real oracle module is never modified.
"""
import importlib.util
import inspect
import types

import pytest

import oracle
from tests import test_oracle_lloyd as lloyd_pins
from tests import test_oracle_pins as pins
from tests import test_oracle_sip as sip_pins
from tests import test_oracle_spread as spread_pins

MUTATIONS = {
    "wrong distance sign": ("diff = K[s:e, None, :] - Cn[None, :, :]", "diff = K[s:e, None, :] + Cn[None, :, :]"),
    "argmax instead of argmin": ("a = np.argmin(dist, axis=1)", "a = np.argmax(dist, axis=1)"),
    "ties to the highest index": ("a = np.argmin(dist, axis=1)",
                                  "a = dist.shape[1] - 1 - np.argmin(dist[:, ::-1], axis=1)"),
    "histogram off by one cluster": ("hist[j, a[k]] += 1", "hist[j, (a[k] + 1) % C] += 1"),
    "block sums skip first key": ("for k in range(s, e):\n        i = pos[int(a[k])]",
                                  "for k in range(s + 1, e):\n        i = pos[int(a[k])]"),
    "totals transposed value column": ("weights=Vf[:, t], minlength=C) for t in range(Vf.shape[1])], axis=1)\n    return n, S",
                                       "weights=Vf[:, -1 - t], minlength=C) for t in range(Vf.shape[1])], axis=1)\n    return n, S"),
    "log2 count weight": ("+ np.log(nU[live])[None, :]", "+ np.log2(nU[live])[None, :]"),
    "count weight dropped": ("+ np.log(nU[live])[None, :]", "+ 0.0"),
    "raw count instead of log": ("+ np.log(nU[live])[None, :]", "+ nU[live][None, :].astype(float)"),
    "clusters compensate selected keys too": ("U = ~in_sel", "U = np.ones_like(in_sel)"),
    "cluster sum instead of mean": ("vbar[nz] = SU[nz] / nU[nz, None]", "vbar[nz] = SU[nz]"),
    "scale dropped on exact logits": ("ell = s * (q @ Kf[in_sel].T)", "ell = (q @ Kf[in_sel].T)"),
    "scale dropped on centroid logits": ("lam = s * (q @ Cf[live].T)", "lam = (q @ Cf[live].T)"),
    "centroid term missing from denominator": ("den = pe.sum(axis=1) + pl.sum(axis=1)", "den = pe.sum(axis=1)"),
    "exact term missing from numerator": ("num = pe @ Vf[in_sel] + pl @ vbar[live]", "num = pl @ vbar[live]"),
    "values of the wrong keys": ("num = pe @ Vf[in_sel]", "num = pe @ Vf[in_sel][::-1]"),
    "Lloyd: sum instead of mean": ("new[live] = S[live] / n[live][:, None]", "new[live] = S[live]"),
    "Lloyd: empty cluster sent to the origin": ("new = Cf.copy()", "new = np.zeros_like(Cf)"),
    "Lloyd: mean of the wrong keys": ("np.add.at(S, a, Kf)", "np.add.at(S, a, Kf[::-1])"),
    "k-means objective without the square": ("((Kf - Cf[a]) ** 2).sum()", "np.abs(Kf - Cf[a]).sum()"),
    "spread: factor 1 instead of 1/2": ("lam = lam + 0.5 * s * s *", "lam = lam + 1.0 * s * s *"),
    "spread: s instead of s^2": ("lam = lam + 0.5 * s * s *", "lam = lam + 0.5 * s *"),
    "spread: wrong sign": ("lam = lam + 0.5 * s * s *", "lam = lam - 0.5 * s * s *"),
    "spread about the mean of all keys": ("dev2 = (Kf - Cf[a]) ** 2", "dev2 = (Kf - Kf.mean(axis=0)) ** 2"),
    "spread: sum instead of mean": ("D[nz] = tot[nz] / n[nz, None]", "D[nz] = tot[nz]"),
    "inclusion weight pi instead of 1/pi": ("s * (q @ Kf[bs:be].T) - math.log(float(p))",
                                             "s * (q @ Kf[bs:be].T) + math.log(float(p))"),
    "inclusion weight dropped": ("s * (q @ Kf[bs:be].T) - math.log(float(p))", "s * (q @ Kf[bs:be].T)"),
    "inclusion weights replaced by one common weight": ("s * (q @ Kf[bs:be].T) - math.log(float(p))",
                                                        "s * (q @ Kf[bs:be].T) - math.log(float(sum(incl)))"),
}

PINS = [
    (pins.test_reassign_hand_fixture, {}),
    (pins.test_reassign_matches_library_distance, {"seed": 0}),
    (pins.test_reassign_ties_go_to_lowest_index, {}),
    (pins.test_stats_hand_fixture, {}),
    (pins.test_histogram_against_library_and_invariants, {"N": 250, "block": 64}),
    (pins.test_block_sums_against_one_hot_matmul, {}),
    (pins.test_attention_hand_fixture, {"name": "attention_1d_a"}),
    (pins.test_attention_hand_fixture, {"name": "attention_1d_b"}),
    (pins.test_full_plan_is_dense_attention, {}),
    (pins.test_keys_on_centroids_compensation_is_exact, {"p": 0.3}),
    (pins.test_empty_plan_is_centroid_attention, {}),
    (pins.test_zero_queries_give_mean_value_for_any_plan, {}),
    (pins.test_per_key_correction_form, {}),
    (pins.test_brute_force_tiny, {}),
    (lloyd_pins.test_hand_example_one_step, {}),
    (lloyd_pins.test_matches_scikit_learn_lloyd, {}),
    (lloyd_pins.test_means_are_a_fixed_point, {}),
    (lloyd_pins.test_empty_cluster_keeps_its_centroid, {}),
    (lloyd_pins.test_objective_never_increases, {}),
    (lloyd_pins.test_objective_hand_value, {}),
    (spread_pins.test_offset_keys_give_the_squared_offset, {}),
    (spread_pins.test_corrected_logit_matches_the_cluster_log_sum_exp_to_fourth_order, {"seed": 0}),
    (sip_pins.test_certain_inclusion_of_every_block_is_dense_attention, {}),
    (sip_pins.test_sums_are_unbiased_over_all_subsets, {"seed": 1}),
    (sip_pins.test_equal_weights_cancel, {}),
]


def _mutant(src_old, src_new):
    src = inspect.getsource(oracle)
    assert src.count(src_old) >= 1, f"mutation anchor not found: {src_old!r}"
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(src_old, src_new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    old, new = MUTATIONS[name]
    mutant = _mutant(old, new)
    monkeypatch.setattr(pins, "oracle", mutant)
    monkeypatch.setattr(lloyd_pins, "oracle", mutant)
    monkeypatch.setattr(spread_pins, "oracle", mutant)
    monkeypatch.setattr(sip_pins, "oracle", mutant)
    caught = []
    for fn, kw in PINS:
        try:
            fn(**kw)
        except Exception:      # AssertionError or a crash both count as caught
            caught.append(fn.__name__)
    assert caught, f"no pin caught the planted mistake '{name}'"


def test_unmutated_oracle_passes_every_pin():
    for fn, kw in PINS:
        fn(**kw)
