"""The pins catch plausible mistakes: each test plants one mistake in the
oracle (CPU only, through monkeypatch) and checks that a pin that should
catch it now fails."""
import math

import numpy as np
import pytest

import oracle.attention as oatt
import oracle.bf16 as obf
import oracle.paged_cache as opc
import oracle.rotary as orot
from tests import test_oracle_attention as T_att
from tests import test_oracle_bf16 as T_bf16
from tests import test_oracle_rotary as T_rot


def _fails(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


# --------------------------------------------------------------- rotary
def _rotate_with(mut):
    def rotate(x_bits, positions, theta, exact=False):
        x_bits = np.asarray(x_bits)
        x = orot.bf16_bits_to_f64(x_bits) if x_bits.dtype == np.uint16 else x_bits.astype(np.float64)
        d = x.shape[-1]
        h = d // 2
        c, s = orot.rope_table(theta, d, positions, exact=exact)
        c = c.astype(np.float64)[:, None, :]
        s = s.astype(np.float64)[:, None, :]
        y = mut(x, c, s, h)
        return y if exact else orot.f64_to_bf16_bits(y)
    return rotate


def _sign_flip(x, c, s, h):
    y = np.empty_like(x)
    y[..., :h] = x[..., :h] * c + x[..., h:] * s
    y[..., h:] = x[..., h:] * c - x[..., :h] * s
    return y


def _interleaved(x, c, s, h):  # pairs (2i, 2i+1) instead of (i, i + d/2)
    y = np.empty_like(x)
    x1, x2 = x[..., 0::2], x[..., 1::2]
    y[..., 0::2] = x1 * c - x2 * s
    y[..., 1::2] = x2 * c + x1 * s
    return y


@pytest.mark.parametrize("mut", [_sign_flip, _interleaved], ids=["sign", "interleaved"])
def test_rotation_mistakes_are_caught(monkeypatch, mut):
    monkeypatch.setattr(T_rot, "rotate_half", _rotate_with(mut))
    _fails(T_rot.test_matches_huggingface_rotate_half)
    _fails(T_rot.test_equals_complex_rotation_rounded_once)


def test_frequency_exponent_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(T_rot, "inv_freq",
                        lambda theta, d: [1.0 / (theta ** (i / d)) for i in range(d // 2)])
    _fails(T_rot.test_inv_freq_closed_form)


# ------------------------------------------------------------------ bf16
def test_rounding_through_float32_is_caught(monkeypatch):
    def via_f32(x):
        x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
        b = x32.view(np.uint32)
        return ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)
    monkeypatch.setattr(T_bf16, "f64_to_bf16_bits", via_f32)
    _fails(T_bf16.test_exact_midpoints_round_to_even_and_off_midpoints_do_not)


def test_truncating_rounding_is_caught(monkeypatch):
    def trunc(x):
        x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
        return (x32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    monkeypatch.setattr(T_bf16, "f64_to_bf16_bits", trunc)
    _fails(T_bf16.test_random_doubles_match_brute_force)


# ------------------------------------------------------------- attention
def _attend_with(window_mut=None, scale_mut=None):
    orig = oatt.attend_contiguous

    def attend(q, positions, K, V, scale, window=0):
        q = np.asarray(q, dtype=np.float64)
        positions = np.asarray(positions, dtype=np.int64)
        sc = scale_mut(scale) if scale_mut else scale
        if window_mut is None:
            return orig(q, positions, K, V, sc, window)
        lo = np.maximum(0, positions - window) if window > 0 else np.zeros_like(positions)  # off by one
        keys = np.arange(K.shape[0])
        z = sc * (q @ K.T)
        ok = (keys[None, :] >= lo[:, None]) & (keys[None, :] <= positions[:, None])
        z = np.where(ok, z, -np.inf)
        w = np.exp(z - z.max(axis=1, keepdims=True))
        return (w @ V) / w.sum(axis=1, keepdims=True)
    return attend


def test_window_off_by_one_is_caught(monkeypatch):
    monkeypatch.setattr(oatt, "attend_contiguous", _attend_with(window_mut=True))
    _fails(T_att.test_brute_force_dense_attention, 16, 4, 1, 5)


def test_missing_softmax_scale_is_caught(monkeypatch):
    monkeypatch.setattr(oatt, "attend_contiguous", _attend_with(scale_mut=lambda s: 1.0))
    _fails(T_att.test_brute_force_dense_attention, 64, 4, 4, 0)


def test_wrong_group_mapping_is_caught(monkeypatch):
    def ragged(cache, block_tables, q_lens, ctx_lens, q_rot_bits, scale, window=0, tokens=None):
        q_all = np.asarray(q_rot_bits)
        T, Hq, d = q_all.shape
        Hkv = cache.n_kv_heads
        out = np.full((T, Hq, d), np.nan)
        start = 0
        for s in range(len(q_lens)):
            qs, cs = int(q_lens[s]), int(ctx_lens[s])
            rows = np.arange(start, start + qs)
            start += qs
            pos = cs + np.arange(qs)
            Kw, Vw = cache.gather(block_tables[s], cs + qs)
            for h in range(Hq):
                hk = h % Hkv                     # should be h // (Hq // Hkv)
                K = oatt.bf16_bits_to_f64(Kw[:, hk, :])
                V = oatt.bf16_bits_to_f64(Vw[:, hk, :])
                out[rows, h] = oatt.attend_contiguous(oatt.bf16_bits_to_f64(q_all[rows, h]), pos, K, V, scale, window)
        return out
    monkeypatch.setattr(T_att, "ragged_attention", ragged)
    _fails(T_att.test_brute_force_dense_attention, 64, 4, 2, 0)


def test_append_slot_off_by_one_is_caught(monkeypatch):
    orig = opc.PagedCache.write_positions

    def shifted(self, bt_row, positions, k_bits, v_bits):
        return orig(self, bt_row, (np.asarray(positions) + 1) % self.block_size + 0 * np.asarray(positions), k_bits, v_bits)
    monkeypatch.setattr(opc.PagedCache, "write_positions", shifted)
    _fails(T_att.test_append_is_a_bit_copy_and_leaves_other_slots)


# ----------------------------------------------------------- projection
def _linear_with(mut):
    def linear(x_bits, w_bits):
        x = obf.bf16_bits_to_f64(np.asarray(x_bits, dtype=np.uint16))
        w = obf.bf16_bits_to_f64(np.asarray(w_bits, dtype=np.uint16))
        return mut(x, w)
    return linear


def _dropped_term(x, w):
    return obf.f64_to_bf16_bits(x[:, :-1] @ w[:, :-1].T)


def _through_float32(x, w):
    return obf.f64_to_bf16_bits((x @ w.T).astype(np.float32).astype(np.float64))


def _truncated(x, w):
    y = (x @ w.T).astype(np.float32)
    return (y.view(np.uint32) >> 16).astype(np.uint16)


def _sequential_float64(x, w):
    # an ordinary float64 sum, term after term, rounded to bf16 at the end
    acc = np.zeros((x.shape[0], w.shape[0]))
    for i in range(x.shape[1]):
        acc = acc + np.outer(x[:, i], w[:, i])
    return obf.f64_to_bf16_bits(acc)


@pytest.mark.parametrize("mut,pin", [(_dropped_term, "test_linear_against_term_by_term_sums"),
                                     (_through_float32, "test_linear_rounds_the_exact_sum_once"),
                                     (_truncated, "test_linear_against_term_by_term_sums"),
                                     (_sequential_float64, "test_linear_sums_4096_terms_exactly")],
                         ids=["dropped_term", "float32_sum", "truncation", "sequential_float64_sum"])
def test_linear_mistakes_are_caught(monkeypatch, mut, pin):
    import oracle
    monkeypatch.setattr(oracle, "linear", _linear_with(mut))
    _fails(getattr(T_att, pin))
