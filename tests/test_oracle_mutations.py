"""Mistakes planted in the oracle, on the CPU: each must fail at least one pin
of tests/test_oracle_pins.py.

This is the evidence that the pins constrain every step of the oracle: a
dropped term, a wrong sign, index or offset, a transposed operand or a wrong
rounding rule anywhere in it shows up as a failing pin.  Each mutation
replaces one oracle function (the pins and the oracle's own internal calls
both look the name up at call time) and then every pin is run directly.
"""
import inspect

import numpy as np
import pytest

from oracle import hca_oracle as O
from tests import test_oracle_pins as P

ORIG = {name: getattr(O, name) for name in dir(O) if callable(getattr(O, name))}


def _pin_calls():
    """Every pin of test_oracle_pins with its parameter sets expanded."""
    calls = []
    for name, fn in inspect.getmembers(P, inspect.isfunction):
        if not name.startswith("test_") or fn.__module__ != P.__name__:
            continue
        sets = [{}]
        for mark in getattr(fn, "pytestmark", []):
            if mark.name != "parametrize":
                continue
            names = [a.strip() for a in mark.args[0].split(",")] if isinstance(mark.args[0], str) else mark.args[0]
            new = []
            for base in sets:
                for vals in mark.args[1]:
                    vals = vals if len(names) > 1 else (vals,)
                    new.append({**base, **dict(zip(names, vals))})
            sets = new
        calls += [(name, fn, kw) for kw in sets]
    return calls


PINS = _pin_calls()


def _failing_pins():
    """Pins whose assertions fail (an exception of another kind does not count:
    a mistake must be caught by a checked property, not by a crash)."""
    failed = []
    for name, fn, kw in PINS:
        try:
            with np.errstate(all="ignore"):
                fn(**kw)
        except AssertionError:
            failed.append(name)
        except Exception:
            pass
    return failed


# --------------------------------------------------------------- the mistakes
def rope_sign(x, pos, rd, theta=10000.0, inverse=False):
    return ORIG["rope"](x, pos, rd, theta, not inverse)


def rope_frequency(x, pos, rd, theta=10000.0, inverse=False):
    # theta^(-i/rd) instead of theta^(-2i/rd)
    return ORIG["rope"](x, pos, rd, theta ** 0.5, inverse)


def rope_half_split_pairs(x, pos, rd, theta=10000.0, inverse=False):
    # pairs (i, i + rd/2) instead of (2i, 2i+1)
    x = np.asarray(x, np.float64)
    if rd == 0:
        return x.copy()
    c = x.shape[-1]
    perm = np.arange(c)
    half = np.arange(rd // 2)
    perm[c - rd + 2 * half] = c - rd + half
    perm[c - rd + 2 * half + 1] = c - rd // 2 + half
    y = ORIG["rope"](x[..., perm], pos, rd, theta, inverse)
    out = np.empty_like(y)
    out[..., perm] = y
    return out


def rmsnorm_no_sqrt(x, gamma=None, eps=1e-6):
    x = np.asarray(x, np.float64)
    y = x / (np.mean(x * x, axis=-1, keepdims=True) + eps)
    return y if gamma is None else y * gamma


def compress_without_bias(Ca_blk, Za_blk, Ba, Cb_prev=None, Zb_prev=None, Bb=None):
    return ORIG["compress_entry"](Ca_blk, Za_blk, np.zeros_like(np.asarray(Ba, np.float64)), Cb_prev, Zb_prev,
                                  None if Bb is None else np.zeros_like(np.asarray(Bb, np.float64)))


def compress_b_rows_reversed(Ca_blk, Za_blk, Ba, Cb_prev=None, Zb_prev=None, Bb=None):
    if Cb_prev is None:
        return ORIG["compress_entry"](Ca_blk, Za_blk, Ba)
    return ORIG["compress_entry"](Ca_blk, Za_blk, Ba, np.asarray(Cb_prev)[::-1], Zb_prev, Bb)


def compress_softmax_over_channels(Ca_blk, Za_blk, Ba, Cb_prev=None, Zb_prev=None, Bb=None):
    L = [np.asarray(Za_blk, np.float64) + Ba]
    V = [np.asarray(Ca_blk, np.float64)]
    if Cb_prev is not None:
        L.append(np.asarray(Zb_prev, np.float64) + Bb)
        V.append(np.asarray(Cb_prev, np.float64))
    L, V = np.concatenate(L), np.concatenate(V)
    S = np.exp(L - L.max(axis=1, keepdims=True))
    S = S / S.sum(axis=1, keepdims=True)
    return (S * V).sum(axis=0)


def compress_prefill_no_overlap(Ca, Za, Ba, m, Cb=None, Zb=None, Bb=None):
    return ORIG["compress_prefill"](Ca, Za, Ba, m)


def compress_prefill_b_from_same_block(Ca, Za, Ba, m, Cb=None, Zb=None, Bb=None):
    n, E = Ca.shape[0], Ca.shape[0] // m
    out = np.zeros((E, Ca.shape[1]))
    for i in range(E):
        blk = slice(m * i, m * (i + 1))
        if Cb is not None and i > 0:
            out[i] = ORIG["compress_entry"](Ca[blk], Za[blk], Ba, Cb[blk], Zb[blk], Bb)
        else:
            out[i] = ORIG["compress_entry"](Ca[blk], Za[blk], Ba)
    return out


def epilogue_at_block_end(entries, m, first_entry=0, gamma=None, eps=1e-6, rd=0, theta=10000.0, norm=True):
    x = np.asarray(entries, np.float64)
    if norm:
        x = O.rmsnorm(x, gamma, eps)
    return O.rope(x, (first_entry + np.arange(x.shape[0])) * m + m - 1, rd, theta)


def visible_one_early(t, m):
    return (t + 2) // m


def visible_one_late(t, m):
    return t // m


def index_without_relu(qI_t, w_t, KI, V):
    dots = np.asarray(KI, np.float64)[:V] @ np.asarray(qI_t, np.float64).T
    return (dots * np.asarray(w_t, np.float64)[None, :]).sum(axis=1)


def index_relu_after_weighting(qI_t, w_t, KI, V):
    dots = np.asarray(KI, np.float64)[:V] @ np.asarray(qI_t, np.float64).T
    return np.maximum(dots * np.asarray(w_t, np.float64)[None, :], 0.0).sum(axis=1)


def topk_ties_to_higher_index(scores, k):
    s = np.asarray(scores, np.float64)
    V = s.shape[0]
    order = np.lexsort((-np.arange(V), -s))
    out = np.full(k, -1, dtype=np.int32)
    kept = np.sort(order[:min(k, V)])
    out[:kept.shape[0]] = kept
    return out


def topk_in_score_order(scores, k):
    s = np.asarray(scores, np.float64)
    V = s.shape[0]
    order = np.lexsort((np.arange(V), -s))[:min(k, V)]
    out = np.full(k, -1, dtype=np.int32)
    out[:order.shape[0]] = order
    return out


def window_without_own_token(t, w):
    return np.arange(max(0, t - w), t)


def attend_without_sink(q_t, rows, sink, scale):
    return ORIG["attend_token"](q_t, rows, np.full_like(np.asarray(sink, np.float64), -np.inf), scale)


def attend_sink_scaled(q_t, rows, sink, scale):
    return ORIG["attend_token"](q_t, rows, np.asarray(sink, np.float64) * scale, scale)


def attend_without_scale(q_t, rows, sink, scale):
    return ORIG["attend_token"](q_t, rows, sink, 1.0)


def output_rotated_forward(q_t, rows, sink, scale, t, rd, theta=10000.0):
    return O.rope(O.attend_token(q_t, rows, sink, scale), t, rd, theta, inverse=False)


def e4m3_truncating(x):
    x = np.clip(np.asarray(x, np.float64), -448, 448)
    codes = np.arange(256)
    vals = O.e4m3_to_f64(codes)
    ok = ~np.isnan(vals) & (codes != 0x80)
    codes, vals = codes[ok], vals[ok]
    best = np.where(np.abs(vals[None, :]) <= np.abs(x)[..., None] + 0 * vals, np.abs(vals[None, :]), -1)
    best = np.where(np.sign(vals[None, :]) * np.sign(x)[..., None] >= 0, best, -1)
    return codes[np.argmax(best, axis=-1)].astype(np.uint8)


def bf16_ties_away(x):
    x = np.asarray(x, np.float64)
    m, e = np.frexp(x)
    q = np.ldexp(np.trunc(np.ldexp(m, 8) + np.copysign(0.5, m)), e - 8)
    return (q.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def kv_quant_scale_240(row, rd, block=64):
    # block amax / 240 (the fnuz format's maximum) instead of / 448
    x = np.asarray(row, np.float64)
    nq = x.shape[-1] - rd
    xb = x[..., :nq].astype(np.float32).reshape(*x.shape[:-1], nq // block, block)
    scale = (np.abs(xb).max(axis=-1, keepdims=True) / np.float32(240.0)).astype(np.float32)
    quot = (xb / np.where(scale > 0, scale, np.float32(1.0))).astype(np.float32)
    codes = O.e4m3_encode(quot.astype(np.float64)).reshape(*x.shape[:-1], nq)
    return codes, scale[..., 0], O.bf16_encode(x[..., nq:])


def kv_dequant_without_scale(codes, scales, rope_bits, block=64):
    return ORIG["kv_row_dequant"](codes, np.ones_like(np.asarray(scales, np.float64)), rope_bits, block)


def e2m1_ties_away(x):
    x = np.asarray(x, np.float64)
    a = np.minimum(np.abs(x), 6.0)
    mags = O.E2M1_MAGNITUDES
    d = np.abs(a[..., None] - mags)
    mag = np.argmin(d + 1e-12 * (7 - np.arange(8)), axis=-1)      # ties to the larger magnitude
    return (np.where((x < 0) & (mag > 0), 8, 0) + mag).astype(np.uint8)


def hadamard_unnormalised(n):
    return ORIG["hadamard"](n) * np.sqrt(n)


def fp4_scale_one_bit_low(x, block=32):
    x = np.asarray(x, np.float64)
    n = x.shape[-1]
    xb = x.reshape(*x.shape[:-1], n // block, block)
    amax = np.abs(xb).max(axis=-1)
    e = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 1, 0).astype(np.int64)
    codes = O.e2m1_encode(xb / np.ldexp(1.0, e)[..., None])
    return codes.reshape(x.shape), e


def oproj_groups_interleaved(o, wo_a, wo_b, g):
    # heads dealt to groups round-robin instead of in consecutive runs
    o = np.asarray(o, np.float64)
    n_h = o.shape[-2]
    perm = np.concatenate([np.arange(i, n_h, g) for i in range(g)])
    return ORIG["output_projection"](o[..., perm, :], wo_a, wo_b, g)


def oproj_wo_b_transposed(o, wo_a, wo_b, g):
    # only a square wo_b can be transposed without a shape error
    wo_b = np.asarray(wo_b, np.float64)
    return ORIG["output_projection"](o, wo_a, wo_b.T if wo_b.shape[0] == wo_b.shape[1] else wo_b, g)


def decode_emit_at_block_start(pos, m, cur_Ca, cur_Za, Ba, prev_Cb=None, prev_Zb=None, Bb=None):
    if pos % m != 0:
        return None
    r = np.asarray(cur_Ca).shape[0]          # the rows present so far, their biases only
    return O.compress_entry(cur_Ca, cur_Za, np.asarray(Ba)[:r], prev_Cb, prev_Zb, Bb)


def e4m3_bias_8(bits):
    b = np.asarray(bits).astype(np.int64) & 0xFF
    s = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 3) & 0xF
    f = (b & 7).astype(np.float64)
    v = s * np.where(e == 0, np.ldexp(f / 8.0, -7), np.ldexp(1.0 + f / 8.0, (e - 8).astype(np.int64)))
    return np.where((e == 15) & ((b & 7) == 7), np.nan, v)


def bf16_decode_shift_15(bits):
    b = np.asarray(bits).astype(np.uint32) << np.uint32(15)
    return b.view(np.float32).astype(np.float64)


def fp4_scores_keys_not_rotated(qI_t, w_t, KI, V):
    qr = O.fp4_simulate(O.hadamard_rotate(qI_t))
    kr = O.fp4_simulate(np.asarray(KI, np.float64)[:V])
    return O.bf16_bits_to_f64(O.bf16_encode(O.index_scores(qr, w_t, kr, V)))


def fp4_scores_not_rounded(qI_t, w_t, KI, V):
    qr = O.fp4_simulate(O.hadamard_rotate(qI_t))
    kr = O.fp4_simulate(O.hadamard_rotate(np.asarray(KI, np.float64)[:V]))
    return O.index_scores(qr, w_t, kr, V)


def fp4_blocks_of_16(x, block=32):
    return ORIG["fp4_block_quant"](x, 16)


def kv_quant_blocks_of_32(row, rd, block=64):
    return ORIG["kv_row_quant"](row, rd, 32)


def topk_pads_with_low_scores(scores, k):
    # keeps k entries even when fewer are visible (indices past the visible set)
    s = np.asarray(scores, np.float64)
    V = s.shape[0]
    order = np.lexsort((np.arange(V), -s))
    kept = np.sort(order[:min(k, V)])
    out = np.arange(k, dtype=np.int32) + V
    out[:kept.shape[0]] = kept
    return out


def compress_entry0_with_zero_row(Ca_blk, Za_blk, Ba, Cb_prev=None, Zb_prev=None, Bb=None):
    # entry 0's missing b-half as a zero value with logit 0 instead of -inf
    if Cb_prev is None and np.asarray(Ca_blk).shape[0] > 1:
        z = np.zeros((1, np.asarray(Ca_blk).shape[1]))
        return ORIG["compress_entry"](Ca_blk, Za_blk, Ba, z, z, np.zeros_like(z))
    return ORIG["compress_entry"](Ca_blk, Za_blk, Ba, Cb_prev, Zb_prev, Bb)


def e2m1_sign_bit_2(codes):
    c = np.asarray(codes).astype(np.int64) & 0xF
    return np.where(c & 4, -1.0, 1.0) * O.E2M1_MAGNITUDES[c & 7]


MUTATIONS = {
    "decode: emission at the block start": ("decode_new_entry", decode_emit_at_block_start),
    "e4m3: exponent bias 8": ("e4m3_to_f64", e4m3_bias_8),
    "bf16: decoded with a 15-bit shift": ("bf16_bits_to_f64", bf16_decode_shift_15),
    "fp4 scores: keys not rotated": ("index_scores_fp4", fp4_scores_keys_not_rotated),
    "fp4 scores: not rounded to bf16": ("index_scores_fp4", fp4_scores_not_rounded),
    "fp4: blocks of 16": ("fp4_block_quant", fp4_blocks_of_16),
    "mixed KV: blocks of 32": ("kv_row_quant", kv_quant_blocks_of_32),
    "top-k: padded with invisible entries": ("topk_select", topk_pads_with_low_scores),
    "compress: entry 0 with a zero b row": ("compress_entry", compress_entry0_with_zero_row),
    "e2m1: sign in bit 2": ("e2m1_to_f64", e2m1_sign_bit_2),
    "rope: rotation sign": ("rope", rope_sign),
    "rope: frequency theta^(-i/rd)": ("rope", rope_frequency),
    "rope: half-split pairs": ("rope", rope_half_split_pairs),
    "rmsnorm: no square root": ("rmsnorm", rmsnorm_no_sqrt),
    "compress: biases dropped": ("compress_entry", compress_without_bias),
    "compress: b rows in reverse": ("compress_entry", compress_b_rows_reversed),
    "compress: softmax over channels": ("compress_entry", compress_softmax_over_channels),
    "compress: overlap ignored": ("compress_prefill", compress_prefill_no_overlap),
    "compress: b series from the same block": ("compress_prefill", compress_prefill_b_from_same_block),
    "epilogue: RoPE at the block end": ("entry_epilogue", epilogue_at_block_end),
    "visibility: one token early": ("visible_entries", visible_one_early),
    "visibility: one token late": ("visible_entries", visible_one_late),
    "index: ReLU dropped": ("index_scores", index_without_relu),
    "index: ReLU after the weight": ("index_scores", index_relu_after_weighting),
    "top-k: ties to the higher index": ("topk_select", topk_ties_to_higher_index),
    "top-k: output in score order": ("topk_select", topk_in_score_order),
    "window: own token left out": ("window_positions", window_without_own_token),
    "attend: sink dropped": ("attend_token", attend_without_sink),
    "attend: sink scaled": ("attend_token", attend_sink_scaled),
    "attend: logit scale dropped": ("attend_token", attend_without_scale),
    "attend: output rotated forward": ("attend_output", output_rotated_forward),
    "e4m3: truncating encoder": ("e4m3_encode", e4m3_truncating),
    "bf16: ties away from zero": ("bf16_encode", bf16_ties_away),
    "mixed KV: scale amax/240": ("kv_row_quant", kv_quant_scale_240),
    "mixed KV: reader drops the scale": ("kv_row_dequant", kv_dequant_without_scale),
    "e2m1: ties away from zero": ("e2m1_encode", e2m1_ties_away),
    "hadamard: not normalised": ("hadamard", hadamard_unnormalised),
    "fp4: block scale one bit low": ("fp4_block_quant", fp4_scale_one_bit_low),
    "output projection: heads dealt round-robin": ("output_projection", oproj_groups_interleaved),
    "output projection: wo_b transposed": ("output_projection", oproj_wo_b_transposed),
}


def test_pins_pass_unmutated():
    assert _failing_pins() == []


@pytest.mark.parametrize("label", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(monkeypatch, label):
    name, fn = MUTATIONS[label]
    monkeypatch.setattr(O, name, fn)
    failed = _failing_pins()
    assert failed, f"no pin catches the planted mistake '{label}'"
