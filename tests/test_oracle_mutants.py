"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that the
pins catch every one of them. This is what makes the oracle trustworthy as the
parity reference: a dropped term, a wrong sign, a wrong index or a transposed
operand anywhere in it fails at least one pin of tests/pins.py."""
import os

import pytest

import oracle
import pins

# (name, original text, replacement); each original occurs in attn_oracle.cpp.
MUTATIONS = [
    ("logits_without_scale", "s[j] = scale * acc;", "s[j] = acc;"),
    ("causal_drops_diagonal", "if (causal && j > i) return false;",
     "if (causal && j >= i) return false;"),
    ("causal_ignored", "if (causal && j > i) return false;", ""),
    ("window_left_off_by_one", "if (left >= 0 && j < i - left) return false;",
     "if (left >= 0 && j <= i - left) return false;"),
    ("window_right_ignored", "if (right >= 0 && j > i + right) return false;", ""),
    ("window_sides_swapped", "if (left >= 0 && j < i - left) return false;",
     "if (left >= 0 && j < i - right) return false;"),
    ("block_mask_transposed", "blocks[(i / kBlock) * nb + j / kBlock]",
     "blocks[(j / kBlock) * nb + i / kBlock]"),
    ("philox_wrong_multiplier", "static_cast<uint64_t>(0xD2511F53u) * x0",
     "static_cast<uint64_t>(0xD2511F55u) * x0"),
    ("philox_no_key_bump", "k0 += 0x9E3779B9u;", ""),
    ("dropout_no_rescale", "return keep(bh, i, j) ? 256.0 / (256.0 - threshold) : 0.0;",
     "return keep(bh, i, j) ? 1.0 : 0.0;"),
    ("dropout_rescale_unrounded_p", "return keep(bh, i, j) ? 256.0 / (256.0 - threshold) : 0.0;",
     "return keep(bh, i, j) ? 1.0 / (1.0 - p) : 0.0;"),
    ("dropout_word_index", "(w[i % 4] >> (8 * (j % 4)))", "(w[j % 4] >> (8 * (j % 4)))"),
    ("dropout_byte_index", "(w[i % 4] >> (8 * (j % 4)))", "(w[i % 4] >> (8 * (i % 4)))"),
    ("dropout_counter_swapped", "static_cast<uint32_t>(j / 4), static_cast<uint32_t>(i / 4),",
     "static_cast<uint32_t>(i / 4), static_cast<uint32_t>(j / 4),"),
    ("dropout_dP_without_Z", "dsi[j] = acc * drop.factor(bh, i, j);", "dsi[j] = acc;"),
    ("dropout_dV_without_Z", "const double p = P[i * N + j] * drop.factor(bh, i, j);",
     "const double p = P[i * N + j];"),
    ("dkdv_rows_ignore_masks", "if (!vis.sees(i, j)) continue;", ""),
    ("dkdv_rows_wrong_sign", "const double dsij = pij * (dpij * f - D[i]);",
     "const double dsij = pij * (dpij * f + D[i]);"),
    ("dkdv_rows_dV_without_Z", "gv[c] += pij * f * goi[c];", "gv[c] += pij * goi[c];"),
    ("dq_rows_without_scale", "for (int64_t c = 0; c < d; ++c) g[c] *= scale;", ""),
    ("dq_rows_dP_without_Z", "dp[j] = acc * drop.factor(bh, i, j);", "dp[j] = acc;"),
    ("forward_rows_without_Z", "const double pd = p[j] * drop.factor(bh, i, j);",
     "const double pd = p[j];"),
    ("block_mask_ignored", "if (blocks && !blocks[(i / kBlock) * nb + j / kBlock]) return false;",
     ""),
    ("no_max_subtraction", "p[j] = std::exp(s[j] - m);", "p[j] = std::exp(s[j]);"),
    ("no_normalisation", "for (int64_t j = 0; j < N; ++j) p[j] /= sum;", ""),
    ("lse_without_log", "return m + std::log(sum);", "return m + sum;"),
    ("lse_without_max", "return m + std::log(sum);", "return std::log(sum);"),
    ("output_from_keys", "const double* vj = v + j * d;\n        for (int64_t c = 0; c < d; ++c) oi[c]",
     "const double* vj = k + j * d;\n        for (int64_t c = 0; c < d; ++c) oi[c]"),
    ("dS_wrong_sign", "dsi[j] = pi[j] * (dsi[j] - Di);", "dsi[j] = pi[j] * (dsi[j] + Di);"),
    ("dS_without_D", "dsi[j] = pi[j] * (dsi[j] - Di);", "dsi[j] = pi[j] * dsi[j];"),
    ("dQ_without_scale", "for (int64_t c = 0; c < d; ++c) gqi[c] *= scale;", ""),
    ("dK_without_scale", "for (int64_t c = 0; c < d; ++c) gkj[c] *= scale;", ""),
    ("dK_transposed_dS", "const double ds = dS[i * N + j];", "const double ds = dS[j * N + i];"),
    ("dV_from_dS", "gvj[c] += p * goi[c];", "gvj[c] += ds * goi[c];"),
    ("dV_not_transposed", "const double p = P[i * N + j] * drop.factor(bh, i, j);",
     "const double p = P[j * N + i] * drop.factor(bh, i, j);"),
    ("dQ_uses_Q", "gqi[c] += dsi[j] * kj[c];", "gqi[c] += dsi[j] * q[j * d + c];"),
]


@pytest.fixture(scope="module")
def source():
    with open(oracle.SOURCE) as f:
        return f.read()


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(tmp_path, source, name, old, new):
    assert old in source, f"mutation {name}: text not found in the oracle source"
    mutant = oracle.Oracle.from_source(source.replace(old, new, 1), str(tmp_path / name))
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(mutant)
        except AssertionError as e:
            failed.append((pin.__name__, str(e).splitlines()[0]))
            break
    assert failed, f"planted mistake {name} passed every pin"
