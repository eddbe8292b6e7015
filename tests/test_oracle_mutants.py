"""Planted mistakes in the CPU oracle: each must fail at least one of its pins.

A mutant is the oracle's source with one plausible mistake written in (a wrong shift in the
generator, an off-by-one in the shuffle, a dropped sign, a transposed index, the wrong
block's tables, a missing 1/c), loaded as a separate module and put in place of the oracle
while the pins of tests/test_oracle_pins.py run. The unmutated oracle must pass every pin.

Most mutants must be caught by a pin tied to something outside the oracle: the published
SplitMix64 vector, permutation statistics, table invariants, hand-worked values, closed
forms, or the agreement of the definition with the two-step route. Two mutants change a
free convention of the hash reading (which bit gives the sign, how a block's stream key is
offset). Nothing outside the oracle fixes those, so only the frozen regression tables catch
them. The CUDA table generator, written separately from the same reading, is compared with
these tables bit for bit on the GPU.

Everything here runs on the CPU; nothing calls the CUDA library.
"""

import os
import types

import pytest

import oracle
from tests import test_oracle_pins as P

ORACLE_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "ss1_oracle.py")

REGRESSION = "tables_regression"

# (name, text in the oracle, replacement, kind); kind "pinned" = an independent pin must fail,
# "convention" = the regression tables must fail
MUTANTS = [
    ("mixer_shift", "z = z ^ (z >> _U64(27))", "z = z ^ (z >> _U64(28))", "pinned"),
    ("mixer_constant", "z = z * _U64(_MUL1)", "z = z * _U64(_MUL2)", "pinned"),
    ("draw_index_off_by_one", "state = key + _U64((t + 1) * GAMMA % (1 << 64))",
     "state = key + _U64(t * GAMMA % (1 << 64))", "pinned"),
    ("sattolo_shuffle", "* _U64(i + 1)) >> _U64(32)).astype(np.int64)", "* _U64(i)) >> _U64(32)).astype(np.int64)",
     "pinned"),
    ("naive_shuffle", "* _U64(i + 1)) >> _U64(32)).astype(np.int64)", "* _U64(BK)) >> _U64(32)).astype(np.int64)",
     "pinned"),
    ("swap_loses_value", "perm[rows, j] = pi", "perm[rows, j] = perm[:, i]", "pinned"),
    ("signs_reuse_shuffle_draws", "r = splitmix64_draws(keys, BK - 1 + k)", "r = splitmix64_draws(keys, k)", "pinned"),
    ("fold_by_division", "hl = perm % S", "hl = perm // c", "pinned"),
    ("no_chunk_offset", "hglob = hl + (kc * S)[:, None]", "hglob = hl + 0 * (kc * S)[:, None]", "pinned"),
    ("no_identity_at_c1", "    if c == 1:\n        h[:] = np.arange", "    if c == 0:\n        h[:] = np.arange", "pinned"),
    ("expand_drops_sign", "return Wc_blk[:, h[nb].astype(np.int64)] * g[nb].astype(np.float64)[None, :]",
     "return Wc_blk[:, h[nb].astype(np.int64)]", "pinned"),
    ("expand_uses_block0_tables", "return Wc_blk[:, h[nb].astype(np.int64)] * g[nb].astype(np.float64)[None, :]",
     "return Wc_blk[:, h[0].astype(np.int64)] * g[0].astype(np.float64)[None, :]", "pinned"),
    ("forward_reversed_inputs", "Y[:, nb * BN:(nb + 1) * BN] = X @ Wf.T", "Y[:, nb * BN:(nb + 1) * BN] = X[:, ::-1] @ Wf.T",
     "pinned"),
    ("sketch_overwrites_collisions", "np.add.at(Xs_t, h[nb].astype(np.int64), signed_t)",
     "Xs_t[h[nb].astype(np.int64)] = signed_t", "pinned"),
    ("sketch_uses_block0_weights", "Y[:, nb * BN:(nb + 1) * BN] = Xs_t.T @ Wc[nb * BN:(nb + 1) * BN].T",
     "Y[:, nb * BN:(nb + 1) * BN] = Xs_t.T @ Wc[:BN].T", "pinned"),
    ("sketch_operator_drops_sign", "Sk[np.arange(K), h[nb].astype(np.int64)] = g[nb].astype(np.float64)",
     "Sk[np.arange(K), h[nb].astype(np.int64)] = 1.0", "pinned"),
    ("projection_without_1_over_c", "(W[nb * BN:(nb + 1) * BN] @ Sk) / c", "(W[nb * BN:(nb + 1) * BN] @ Sk)", "pinned"),
    ("rows_sample_ignores_rows", "Ys = ss1_forward(X[rows], Wc, h, g, BN)", "Ys = ss1_forward(X[:len(rows)], Wc, h, g, BN)",
     "pinned"),
    ("backward_input_transposed_block", "dX += dY[:, nb * BN:(nb + 1) * BN] @ Wf",
     "dX += dY[:, nb * BN:(nb + 1) * BN] @ Wf[::-1]", "pinned"),
    ("backward_input_uses_block0_weights", "Wf = expand_weight(Wc, h, g, BN, nb)                   # [BN, K]",
     "Wf = expand_weight(Wc, h, g, BN, 0)                   # [BN, K]", "pinned"),
    ("backward_weight_drops_sign", "signed = dWfull[rows] * g[nb].astype(np.float64)[None, :]",
     "signed = dWfull[rows] * 1.0", "pinned"),
    ("backward_weight_overwrites_collisions", "dWc[rows, h[nb, k]] += signed[:, k]", "dWc[rows, h[nb, k]] = signed[:, k]",
     "pinned"),
    ("backward_weight_block0_tables", "dWc[rows, h[nb, k]] += signed[:, k]", "dWc[rows, h[0, k]] += signed[:, k]",
     "pinned"),
    ("e4m3_bias_8", "(1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)",
     "(1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 8.0)", "pinned"),
    ("e4m3_subnormal_scale", "np.where(e == 0, m / 8.0 * 2.0 ** -6", "np.where(e == 0, m / 8.0 * 2.0 ** -7", "pinned"),
    ("e4m3_ties_to_odd", "((d_hi == d_lo) & (hi % 2 == 0))", "((d_hi == d_lo) & (hi % 2 == 1))", "pinned"),
    ("e4m3_encode_drops_sign", "return (code | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)",
     "return code.astype(np.uint8)", "pinned"),
    ("quantize_scale_not_448", "amax / np.float32(E4M3_MAX)", "amax / np.float32(240.0)", "pinned"),
    ("fp8_forward_drops_scale", "Wd = e4m3_decode(Wq) * np.asarray(scale, dtype=np.float64)[:, None]",
     "Wd = e4m3_decode(Wq)", "pinned"),
    ("relu_is_identity", "return np.maximum(v, 0.0)", "return v", "pinned"),
    ("gelu_without_sqrt2", "return 0.5 * v * (1.0 + np.vectorize(erf)(v / sqrt(2.0)))",
     "return 0.5 * v * (1.0 + np.vectorize(erf)(v))", "pinned"),
    ("bias_dropped", "Y = Y + np.asarray(bias, dtype=np.float64)[None, :]", "Y = Y + 0.0", "pinned"),
    ("chain_drops_activation", "cur = ss1_forward_bias_act(cur, Wc, h, g, BN, bias, act)",
     "cur = ss1_forward_bias_act(cur, Wc, h, g, BN, bias, ACT_NONE)", "pinned"),
    ("sign_from_low_bit", "np.where((r >> _U64(63)) != 0, -1, 1)", "np.where((r & _U64(1)) != 0, -1, 1)", "convention"),
    ("block_key_without_offset", "^ mix64(ids + _U64(1))", "^ mix64(ids)", "convention"),
]


def _mutant_module(old: str, new: str) -> types.ModuleType:
    with open(ORACLE_SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"the oracle no longer holds exactly one {old!r}"
    mod = types.ModuleType("ss1_oracle_mutant")
    exec(compile(src.replace(old, new), "ss1_oracle_mutant", "exec"), mod.__dict__)
    return mod


def _pins(golden_dir):
    """Every pin of tests/test_oracle_pins.py with the parameters it runs with there."""
    pins = [
        ("splitmix64_published_vector", lambda: P.test_splitmix64_published_vector(golden_dir)),
        ("draws_are_counter_based", P.test_draws_are_counter_based),
        ("fisher_yates_is_uniform", P.test_fisher_yates_is_uniform),
        ("fisher_yates_positions_uniform", P.test_fisher_yates_positions_uniform_bk128),
        ("signs_balanced", P.test_signs_balanced),
        ("signs_independent_of_permutation", P.test_signs_independent_of_permutation),
        ("tables_independent_per_block_and_seed", P.test_tables_independent_per_block_and_seed),
        ("fold_is_mod_S", P.test_fold_is_mod_S),
        (REGRESSION, lambda: P.test_tables_regression(golden_dir)),
        ("handworked_examples", lambda: P.test_handworked_examples(golden_dir)),
        ("c1_is_dense_gemm", P.test_c1_is_dense_gemm),
        ("one_hot_probe_structure", P.test_one_hot_probe_structure),
        ("linearity_and_sign_symmetry", P.test_linearity_and_sign_symmetry),
        ("rows_sample_matches_full", P.test_rows_sample_matches_full),
        ("projection_at_c1_is_identity", P.test_projection_at_c1_is_identity),
        ("projection_recovers_tied_weights", P.test_projection_recovers_tied_weights),
    ]
    for args in [(768, 768, 2, 64, 64, 0), (1280, 512, 4, 128, 128, 2), (1024, 256, 8, 256, 128, 3),
                 (512, 256, 8, 128, 128, 4), (512, 256, 1, 128, 128, 4)]:
        pins.append((f"table_invariants{args}", lambda a=args: P.test_table_invariants(*a)))
    for c in (1, 2, 4, 8):
        pins.append((f"sketch_gram_identity[{c}]", lambda c=c: P.test_sketch_gram_identity(c)))
        pins.append((f"frobenius_identity[{c}]", lambda c=c: P.test_frobenius_identity(c)))
    for args in [(64, 32, 2, 16, 8), (256, 256, 4, 64, 64), (512, 256, 8, 256, 128), (768, 768, 2, 64, 64)]:
        pins.append((f"two_routes_agree{args}", lambda a=args: P.test_two_routes_agree(*a)))
    for args in [(2, 8, 4), (4, 8, 8), (1, 4, 4), (8, 16, 4)]:
        pins.append((f"backward_input_fd{args}", lambda a=args: P.test_backward_input_finite_differences(*a)))
        pins.append((f"backward_weight_fd{args}", lambda a=args: P.test_backward_weight_finite_differences(*a)))
    pins.append(("backward_c1", P.test_backward_c1_is_plain_matrix_calculus))
    pins.append(("e4m3_decode", P.test_e4m3_decode_matches_library_and_closed_forms))
    pins.append(("e4m3_encode", P.test_e4m3_encode_round_trip_ties_and_saturation))
    pins.append(("quantize_rows_fp8_forward", P.test_quantize_rows_and_fp8_forward))
    pins.append(("activations", P.test_activations_closed_forms))
    pins.append(("bias_act_layer", P.test_bias_act_layer))
    pins.append(("chain_composition", P.test_chain_is_composition))
    pins.append(("backward_weight_vs_projection", P.test_backward_weight_is_c_times_projection_of_dense_gradient))
    return pins


def _failing_pins(monkeypatch, mod, golden_dir):
    """Names of the pins that fail while `mod` stands in for the oracle."""
    with monkeypatch.context() as mp:
        for name in oracle.__all__:
            mp.setattr(oracle, name, getattr(mod, name))
        failed = []
        for name, pin in _pins(golden_dir):
            try:
                pin()
            except Exception:   # an assertion, or a mutant that no longer runs on the pin's input
                failed.append(name)
    return failed


def test_unmutated_oracle_passes_every_pin(monkeypatch, golden_dir):
    """The harness itself: the oracle's own source, loaded the same way, fails nothing."""
    assert _failing_pins(monkeypatch, _mutant_module("import numpy as np", "import numpy as np"), golden_dir) == []


@pytest.mark.parametrize("name,old,new,kind", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(monkeypatch, golden_dir, name, old, new, kind):
    failed = _failing_pins(monkeypatch, _mutant_module(old, new), golden_dir)
    if kind == "pinned":
        independent = [f for f in failed if f != REGRESSION]
        assert independent, f"mutant {name} passes every independent pin"
    else:
        assert REGRESSION in failed, f"mutant {name} passes the regression tables"
