"""The oracle's pins have teeth (CPU only): each case plants one plausible mistake in
the oracle (a dropped term, a sign, a missing scale, a wrong index or a missing step,
patched into the oracle module for the duration of the case) and checks that the pin
meant to guard that step now fails.  Nothing here touches the product path."""
import numpy as np
import pytest

from oracle import bf16, codebooks, layer, model, quant
from tests import test_oracle_bf16 as F
from tests import test_oracle_layer as P
from tests import test_oracle_quant as Q


def _rmsnorm_bwd_dropped_term(x, w, r, dy):
    return r * dy * w                         # the - x r^3 <w dy, x> / H term is gone


def _rope_sign_flip(x, cos, sin):
    h = x.shape[-1] // 2
    x1, x2 = x[..., :h], x[..., h:]
    c, s = cos[None, :, None, :], sin[None, :, None, :]
    return np.concatenate([x1 * c + x2 * s, x2 * c - x1 * s], axis=-1)   # rotates the other way


def _attention_no_scale(q, k, v):
    return _orig_attention(q * np.sqrt(q.shape[-1]), k, v)               # forgets 1/sqrt(d)


def _attention_gqa_interleaved(q, k, v):
    # query head h read kv head h % n_kv instead of h // (n_q / n_kv)
    nq, nkv = q.shape[2], k.shape[2]
    order = [(h % nkv) * (nq // nkv) + h // nkv for h in range(nq)]
    o, Pr = _orig_attention(q[:, :, order], k, v)
    inv = np.argsort(order)
    return o[:, :, inv], Pr[:, inv]


def _attention_bwd_dk_without_q(q, k, v, Pr, do):
    dq, dk, dv = _orig_attention_bwd(q, k, v, Pr, do)
    return dq, dk * 0.5, dv                                              # a halved dK


def _silu_as_sigmoid(x):
    return layer.sigmoid(x)                                              # x * sigmoid(x) lost its x


def _ce_unshifted(logits, ids, batch, seq, rnd=True):
    ids = np.asarray(ids).reshape(batch, seq)
    shifted = np.concatenate([ids[:, :1], ids[:, :-1]], axis=1)         # targets one position late
    return _orig_ce(logits, shifted, batch, seq, rnd)


def _adamw_no_bias_correction(p, g, m, v, step, lr=2e-4, b1=0.9, b2=0.999, eps=1e-8, wd=0.0):
    m = b1 * m + (1 - b1) * g
    v = b2 * v + (1 - b2) * g * g
    return p - lr * (m / (np.sqrt(v) + eps) + wd * p), m, v


def _nearest_off_by_one(u, table):
    idx = _orig_nearest(u, table)
    if len(table) == 16:                                                 # every 7th NF4 code one too high
        idx = np.minimum(idx + (np.arange(idx.size).reshape(idx.shape) % 7 == 3), 15)
    return idx


def _quantize_swapped_nibbles(w):
    q = dict(_orig_quantize(w))
    p = q["packed"]
    q["packed"] = (((p & 0x0F) << 4) | (p >> 4)).astype(np.uint8)   # element 2j in the low nibble
    return q


def _quantize_offset_off(w):
    q = dict(_orig_quantize(w))
    q["offset"] = np.float32(q["offset"] * 1.01)
    return q


def _bf16_truncating(x):
    b = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32)
    return (b >> np.uint32(16)).astype(np.uint16)                       # drops the low half: rounds toward 0


def _bf16_ties_away(x):
    b = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32).astype(np.uint64)
    return ((b + np.uint64(0x8000)) >> np.uint64(16)).astype(np.uint16)  # halfway cases go up in magnitude


def _round_f64_ties_away(x):
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    b = a.view(np.uint64)
    b = (b + np.uint64(1 << 44)) & ~np.uint64((1 << 45) - 1)
    return b.view(np.float64)


def _block_scales_group_of_64(q):
    code8 = codebooks.code8_table()
    gidx = np.minimum(np.arange(q["q8"].size) // 64, q["nested"].size - 1)   # groups of 64 blocks
    prod = (code8[q["q8"].astype(np.int64)] * q["nested"][gidx]).astype(np.float32)
    return (prod + np.float32(q["offset"])).astype(np.float32)


_orig_nearest = codebooks.nearest_index
_orig_quantize = quant.quantize
_orig_attention = layer.attention
_orig_attention_bwd = layer.attention_bwd
_orig_ce = model.cross_entropy

CASES = [
    ("rmsnorm_bwd", layer, "rmsnorm_bwd", _rmsnorm_bwd_dropped_term,
     [P.test_rmsnorm_backward_matches_torch_autograd]),
    ("rope sign", layer, "rope", _rope_sign_flip,
     [P.test_rope_matches_complex_rotation_and_its_adjoint]),
    ("attention scale", layer, "attention", _attention_no_scale,
     [P.test_attention_matches_torch_sdpa,
      lambda: P.test_layer_forward_matches_transformers_llama_decoder_layer(False)]),
    ("attention GQA mapping", layer, "attention", _attention_gqa_interleaved,
     [P.test_attention_matches_torch_sdpa]),
    ("attention dK", layer, "attention_bwd", _attention_bwd_dk_without_q,
     [P.test_attention_backward_matches_torch_autograd,
      lambda: P.test_layer_backward_finite_differences(1, 8)]),
    ("SiLU", layer, "silu", _silu_as_sigmoid,
     [lambda: P.test_layer_forward_matches_transformers_llama_decoder_layer(True)]),
    ("cross-entropy shift", model, "cross_entropy", _ce_unshifted,
     [P.test_cross_entropy_gradient_matches_torch_autograd, P.test_model_step_matches_transformers_llama_autograd]),
    ("AdamW bias correction", model, "adamw", _adamw_no_bias_correction, [P.test_adamw_matches_torch]),
    ("NF4 code off by one", codebooks, "nearest_index", _nearest_off_by_one,
     [Q.test_quantizer_properties, lambda: Q.test_quantizer_brute_force(64 * 4, 0)]),
    ("nibble order", quant, "quantize", _quantize_swapped_nibbles,
     [Q.test_quantizer_properties, Q.test_nibble_order_high_first]),
    ("offset", quant, "quantize", _quantize_offset_off,
     [Q.test_quantizer_properties, lambda: Q.test_quantizer_brute_force(64 * 4, 0)]),
    ("bf16 truncation", bf16, "f32_to_bf16_bits", _bf16_truncating,
     [F.test_f32_to_bf16_bits_matches_torch_on_constructed_patterns, F.test_f32_to_bf16_ties_go_to_even,
      Q.test_dequant_across_nested_groups_with_different_scales]),
    ("bf16 ties away", bf16, "f32_to_bf16_bits", _bf16_ties_away,
     [F.test_f32_to_bf16_bits_matches_torch_on_constructed_patterns, F.test_f32_to_bf16_ties_go_to_even]),
    ("float64 bf16 ties away", bf16, "round_f64", _round_f64_ties_away,
     [F.test_round_f64_ties_and_near_ties]),
    ("nested group of 64 blocks", quant, "block_scales", _block_scales_group_of_64,
     [Q.test_dequant_across_nested_groups_with_different_scales]),
]


@pytest.mark.parametrize("name,mod,attr,bad,pins", CASES, ids=[c[0] for c in CASES])
def test_pins_catch_planted_mistake(monkeypatch, name, mod, attr, bad, pins):
    for pin in pins:
        pin()                                        # holds on the oracle as it is
    monkeypatch.setattr(mod, attr, bad)
    for pin in pins:
        with pytest.raises(AssertionError):
            pin()
