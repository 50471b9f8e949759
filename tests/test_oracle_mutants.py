"""Planted mistakes in the oracle must each fail at least one pin.

Each mutant is one textual edit of oracle/mlra_oracle.py (a dropped term, a
wrong sign, a wrong axis or index, a missing scale), executed as a separate
module on the CPU.  The edit must match the source exactly once, so this test
fails loudly if the oracle is rewritten without updating the mutants.
"""
import pathlib
import types

import pytest

from tests import oracle_pins

SRC = (pathlib.Path(__file__).parents[1] / "oracle" / "mlra_oracle.py").read_text()

MUTANTS = {
    "rope_term_dropped": ("return q_rope_s @ kr.T", "return 0.0 * (q_rope_s @ kr.T)"),
    "rope_term_sign": ("return sigma * (q_blk @ c_blk.T + rope)", "return sigma * (q_blk @ c_blk.T - rope)"),
    "sigma_skips_rope": ("return sigma * (q_blk @ c_blk.T + rope)", "return sigma * q_blk @ c_blk.T + rope"),
    "max_wrong_axis": ("m = scores.max(axis=-1, keepdims=True)", "m = scores.max(axis=0, keepdims=True)"),
    "no_max_shift": ("e = np.exp(scores - m)", "e = np.exp(scores)"),
    "unnormalised": ("return e / z, (m + np.log(z))[..., 0]", "return e, (m + np.log(z))[..., 0]"),
    "lse_without_max": ("return e / z, (m + np.log(z))[..., 0]", "return e / z, np.log(z)[..., 0]"),
    "positions_misaligned": ("return p @ c_blk", "return p[:, ::-1] @ c_blk"),
    "wrong_query_block": ("scores = _branch_scores(q_lat_s[:, cols],",
                          "scores = _branch_scores(q_lat_s[:, slice(((b + 1) % B) * d, ((b + 1) % B + 1) * d)],"),
    "query_block_reversed": ("scores = _branch_scores(q_lat_s[:, cols],", "scores = _branch_scores(q_lat_s[:, cols][:, ::-1],"),
    "gamma_dropped": ("outs.append(gamma * _apply_probs(p, c_rows[:, cols]))", "outs.append(_apply_probs(p, c_rows[:, cols]))"),
    "summed_is_mean": ("np.sum(outs, axis=0)", "np.mean(outs, axis=0)"),
    "page_offset_index": ("pt[s, j // page_size] * page_size + j % page_size",
                          "pt[s, j // page_size] * page_size + j // page_size"),
    "contiguous_pitch": ("return s * np.int64(max_seq_len) + j", "return s * np.int64(max_seq_len + 1) + j"),
    "empty_lse_zero": ("lse = np.full((hq, B), -np.inf)", "lse = np.zeros((hq, B))"),
    "probs_from_other_branch": ("probs.append(p)", "probs.append(p if b == 0 else probs[0])"),
    "project_transposed_weight": ('np.einsum("hkd,shd->shk", to_f64(w_uv), to_f64(out))',
                                  'np.einsum("hkd,shk->shd", to_f64(w_uv), to_f64(out)[..., :w_uv.shape[1]])'),
    "project_first_branch_only": ('np.einsum("hkd,shd->shk", to_f64(w_uv), to_f64(out))',
                                  'np.einsum("hkd,shd->shk", to_f64(w_uv)[..., :8], to_f64(out)[..., :8])'),
    "absorb_transposed": ('np.einsum("hkd,shk->shd", to_f64(w_uk), to_f64(q_nope))',
                          'np.einsum("hkd,shd->shk", to_f64(w_uk), to_f64(q_nope)[..., :w_uk.shape[2]])'),
    "rope_sin_sign": ("y[..., 0::2] = x0 * c - x1 * s_", "y[..., 0::2] = x0 * c + x1 * s_"),
    "rope_pairs_halves": ("x0, x1 = x[..., 0::2], x[..., 1::2]", "x0, x1 = x[..., : d // 2], x[..., d // 2:]"),
    "rope_frequency_exponent": ("theta = base ** (-2.0 * i / d)", "theta = base ** (-1.0 * i / d)"),
    "append_off_by_one": ("        p = int(lens[s])\n", "        p = max(int(lens[s]) - 1, 0)\n"),
    "multi_token_causal_off_by_one": ("lens_t = np.maximum(lens - (q - 1 - t), 0)",
                                      "lens_t = np.maximum(lens - (q - t), 0)"),
    "multi_token_reversed": ("o, l = decode(q_lat[:, t], q_rope[:, t], c_kv, k_rope, lens_t,",
                             "o, l = decode(q_lat[:, q - 1 - t], q_rope[:, q - 1 - t], c_kv, k_rope, lens_t,"),
    "project_head_shift": ('np.einsum("hkd,shd->shk", to_f64(w_uv), to_f64(out))',
                           'np.einsum("hkd,shd->shk", np.roll(to_f64(w_uv), 1, axis=0), to_f64(out))'),
}


def _mutant(name):
    old, new = MUTANTS[name]
    assert SRC.count(old) == 1, f"mutant {name}: snippet not found exactly once"
    mod = types.ModuleType(f"oracle_mutant_{name}")
    exec(compile(SRC.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    mod = _mutant(name)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mod)
        except Exception as e:  # AssertionError or a shape error both count as caught
            caught.append((pin.__name__, type(e).__name__))
    assert caught, f"no pin catches the planted mistake {name}"


def test_unmutated_source_passes():
    mod = types.ModuleType("oracle_copy")
    exec(compile(SRC, "<copy>", "exec"), mod.__dict__)
    for pin in oracle_pins.ALL_PINS:
        pin(mod)
