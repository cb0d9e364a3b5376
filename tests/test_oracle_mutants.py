"""Each planted mistake in the CPU oracle must fail at least one pin.

The mistakes are planted in the oracle on the CPU (monkeypatch), never in the
CUDA library. A mutant that every pin accepts would mean the pins cannot see
that kind of error.
"""

import numpy as np
import pytest

import oracle_checks as oc
from oracle import attention as oatt
from oracle import blocks as oblk
from oracle import quant as oq


def _fails_some_check(golden):
    failed = []
    for check in oc.BLOCK_CHECKS:
        try:
            check(golden)
        except Exception:  # noqa: BLE001 - any failure counts as caught
            failed.append(check.__name__)
    for check in oc.PLAIN_BLOCK_CHECKS + oc.ATTENTION_CHECKS:
        try:
            check()
        except Exception:  # noqa: BLE001
            failed.append(check.__name__)
    return failed


def _softmax_no_scale(q_vec, keys, values, scale):
    x = np.asarray(keys, np.float64) @ np.asarray(q_vec, np.float64)
    w = np.exp(x - x.max())
    return (w / w.sum()) @ np.asarray(values, np.float64)


def _softmax_unnormalised(q_vec, keys, values, scale):
    x = scale * (np.asarray(keys, np.float64) @ np.asarray(q_vec, np.float64))
    return np.exp(x - x.max()) @ np.asarray(values, np.float64)


def _softmax_keys_as_values(q_vec, keys, values, scale):
    x = scale * (np.asarray(keys, np.float64) @ np.asarray(q_vec, np.float64))
    w = np.exp(x - x.max())
    return (w / w.sum()) @ np.asarray(keys, np.float64)


def _softmax_drop_last(q_vec, keys, values, scale):
    keys, values = np.asarray(keys, np.float64), np.asarray(values, np.float64)
    if len(keys) > 1:
        keys, values = keys[:-1], values[:-1]
    x = scale * (keys @ np.asarray(q_vec, np.float64))
    w = np.exp(x - x.max())
    return (w / w.sum()) @ values


def _e4m3_flush_subnormals(x):
    import oracle.quant as q
    x = np.asarray(x, dtype=np.float32)
    out = _ORIG_E4M3(x)
    return np.where(np.abs(x) < 2.0 ** -6, out & 0x80, out).astype(np.uint8)


_ORIG_E4M3 = oq.e4m3_encode


def _swap_wrong_index(dk, dv, sk, sv, mapping):
    k, v = np.array(dk, copy=True), np.array(dv, copy=True)
    for src, dst in np.asarray(mapping).reshape(-1, 2).tolist():
        k[int(src) % len(k)] = sk[int(src)]
        v[int(src) % len(v)] = sv[int(src)]
    return k, v


def _quantize_times_scale(x, scale):
    return _ORIG_E4M3(np.asarray(x, np.float32) * np.asarray(scale, np.float32))


def _quantize_float64(x, scale):
    # divides in float64 and picks the nearest E4M3 value of that quotient with
    # no rounding to float32 in between (nearest finite code by magnitude)
    q = np.asarray(x, np.float32).astype(np.float64) / np.asarray(scale, np.float64)
    codes = np.arange(0x7F, dtype=np.uint8)
    mags = oq.e4m3_decode(codes)
    near = codes[np.argmin(np.abs(np.abs(q)[..., None] - mags), axis=-1)]
    return (near | (np.signbit(q).astype(np.uint8) << 7)).astype(np.uint8)


def _dequantize_divides(codes, scale):
    return oq.e4m3_decode(codes) / np.asarray(scale, np.float64)


def _quantize_first_scale_only(x, scale):
    return _ORIG_E4M3(np.asarray(x, np.float32) / np.asarray(scale, np.float32).ravel()[0])


MUTANTS = {
    "quantize_multiplies_by_scale": (oq, "quantize", _quantize_times_scale),
    "quantize_divides_in_float64": (oq, "quantize", _quantize_float64),
    "quantize_ignores_head_scales": (oq, "quantize", _quantize_first_scale_only),
    "dequantize_divides_by_scale": (oq, "dequantize", _dequantize_divides),
    "prefill_diagonal_hidden": (oatt, "causal_visible",
                                lambda L, pos: np.arange(L)[None, :] < np.asarray(pos)[:, None]),
    "prefill_unmasked": (oatt, "causal_visible",
                         lambda L, pos: np.ones((len(pos), L), dtype=bool)),
    "prefill_positions_from_zero": (oatt, "chunk_positions", lambda L, n: np.arange(n)),
    "e4m3_round_half_up": (oq, "_round_half_even", lambda v: np.floor(np.asarray(v) + 0.5)),
    "e4m3_no_subnormals": (oq, "e4m3_encode", lambda x: _e4m3_flush_subnormals(x)),
    "gqa_heads_interleaved": (oatt, "kv_head_of", lambda j, g: j % g),
    "gqa_always_head0": (oatt, "kv_head_of", lambda j, g: 0),
    "offset_off_by_one": (oblk, "logical_position", lambda t, bs: (t // bs, (t + 1) % bs)),
    "block_index_swapped": (oblk, "logical_position", lambda t, bs: (t % bs, t // bs)),
    "blocks_floor": (oblk, "blocks_for", lambda n, bs: n // bs),
    "blocks_one_extra": (oblk, "blocks_for", lambda n, bs: n // bs + 1),
    "kv_bytes_no_v": (oblk, "kv_bytes_per_token", lambda L, h, d, e: L * h * d * e),
    "scale_dropped": (oatt, "softmax_attention", _softmax_no_scale),
    "softmax_not_normalised": (oatt, "softmax_attention", _softmax_unnormalised),
    "keys_used_as_values": (oatt, "softmax_attention", _softmax_keys_as_values),
    "last_token_dropped": (oatt, "softmax_attention", _softmax_drop_last),
    "swap_writes_source_index": (oatt, "swap_blocks", lambda dk, dv, sk, sv, m: (
        _swap_wrong_index(dk, dv, sk, sv, m))),
    "slot_without_block_size": (oblk, "slot_of",
                                lambda table, t, bs: int(table[t // bs]) + t % bs),
}


# a mutant that masks a whole row makes the softmax subtract -inf from -inf
@pytest.mark.filterwarnings("ignore:invalid value encountered in subtract:RuntimeWarning")
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, golden, monkeypatch):
    module, attr, bad = MUTANTS[name]
    monkeypatch.setattr(module, attr, bad)
    assert _fails_some_check(golden), f"mutant {name} passed every pin"


def test_unmutated_oracle_passes_every_check(golden):
    assert _fails_some_check(golden) == []
