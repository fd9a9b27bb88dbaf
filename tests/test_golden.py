"""The oracle against the regression fixtures in tests/golden/ (written by
tests/golden/make_golden.py from the oracle and the seeded input generator).

The pages print no worked example, so these values are not independent pins.
They catch an unintended change to the oracle or to the inputs. Bits that
are exact by construction (rotated Q, cache words, rotary table, batch
lengths) must match exactly. Attention outputs are compared to 1e-12, because
the order of the float64 sums may differ with the BLAS thread count."""
import importlib.util
import json
import os

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _gen():
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(HERE, "make_golden.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _stored():
    with open(os.path.join(HERE, "oracle_regression.json")) as f:
        return json.load(f)


def test_tiny_pass_matches_the_fixture():
    want, got = _stored()["tiny_pass"], _gen().tiny_pass()
    for key in ("q_rot_sha256", "cache_blocks_sha256", "cache_block_ids"):
        assert got[key] == want[key], key
    for (t, h, e, v), (t2, h2, e2, v2) in zip(got["out_samples"], want["out_samples"]):
        assert (t, h, e) == (t2, h2, e2)
        assert abs(float(v) - float(v2)) <= 1e-12
    assert abs(float(got["out_sum"]) - float(want["out_sum"])) <= 1e-9


def test_headline_snapshot_matches_the_fixture():
    assert _gen().headline_snapshot() == _stored()["headline_snapshot"]


def test_rotary_rows_match_the_fixture():
    assert _gen().rope_rows() == _stored()["rope_rows"]


def test_first_token_of_a_fresh_prompt_attends_only_to_itself():
    """The fixture's first sample is token 0 of a prompt at context 0: one
    admitted key, so its output is exactly that token's V value."""
    from oracle import bf16_bits_to_f64
    from ragged_paged_kv_b200 import workloads as W
    w = W.config1()
    assert int(w.ctx_lens[0]) == 0
    _, _, v = w.qkv()
    t, h, e, val = _stored()["tiny_pass"]["out_samples"][0]
    assert (t, h, e) == (0, 0, 0)
    assert float(val) == float(bf16_bits_to_f64(v[0, h // (w.n_q_heads // w.n_kv_heads), e]))
