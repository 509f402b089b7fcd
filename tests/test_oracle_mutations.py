"""The oracle's pins are not vacuous: each test here plants one plausible
mistake in the oracle (on the CPU, through monkeypatch, for the duration of
the test only) and checks that at least one of the pins written for that
part of the method then fails."""

import numpy as np
import pytest

from oracle import awq, moe, nvfp4, razor
from oracle.formats import e4m3_to_f64, f32_to_e2m1, f32_to_e4m3

from tests import test_oracle_moe as tm
from tests import test_oracle_quant as tq
from tests import test_oracle_razor as tr


def _fails(pin) -> bool:
    try:
        pin()
    except Exception:  # an assertion, or a shape / index error the mistake causes
        return True
    return False


# --- mutants -----------------------------------------------------------------

def _silu_sign(g):
    return g / (1.0 + np.exp(g))


def _swap_gate_up(orig):
    return lambda x, wg, wu, wd: orig(x, wu, wg, wd)


def _down_untransposed(x, wg, wu, wd):
    h = moe.silu(np.asarray(x) @ np.asarray(wg).T) * (np.asarray(x) @ np.asarray(wu).T)
    return h @ np.asarray(wd), h


def _route_unnormalised(orig):
    def route(x, w_router, bias, k, extra=0):
        r = orig(x, w_router, bias, k, extra)
        r["w"] = np.take_along_axis(r["p"], r["idx"][:, :k], axis=1)
        return r
    return route


def _order_ties_high(p):
    E = p.shape[-1]
    return (E - 1) - np.argsort(-p[..., ::-1], axis=-1, kind="stable")


def _layer_without_shared(orig):
    return lambda x, w_router, bias, k, ew, shared_weights=None, extra=0, shared_gate_w=None: orig(
        x, w_router, bias, k, ew, None, extra, shared_gate_w)


def _permute_tokens_descending(idx, E):
    idx = np.asarray(idx, np.int64)
    T, ks = idx.shape
    flat = idx.reshape(-1)
    key = flat * (T * ks) + (T * ks - 1 - np.arange(T * ks))  # tokens descending inside an expert
    order = np.argsort(key, kind="stable")
    counts = np.bincount(flat, minlength=E)
    offsets = np.zeros(E + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    slot_row = np.empty(T * ks, np.int64)
    slot_row[order] = np.arange(T * ks)
    return dict(offsets=offsets, row_token=order // ks, slot_row=slot_row.reshape(T, ks), counts=counts)


def _literal_without_promoted(f_rows, slot_row, idx, p, k):
    T, H = idx.shape[0], f_rows.shape[1]
    out = np.zeros((T, k, H))
    for t in range(T):
        pS = np.array([p[t, idx[t, j]] for j in range(k)])
        y = (pS / pS.sum()) @ np.stack([f_rows[slot_row[t, j]] for j in range(k)])
        for j in range(k):
            slots = [s for s in range(k) if s != j]  # the rank-(k+1) expert is not promoted
            p2 = np.array([p[t, idx[t, s]] for s in slots])
            out[t, j] = (p2 / p2.sum()) @ np.stack([f_rows[slot_row[t, s]] for s in slots]) - y
    return out


def _closed_form_without_promoted(f_rows, slot_row, idx, p, k):
    pk = np.take_along_axis(p, idx[:, : k + 1], axis=1)
    F = f_rows[slot_row[:, : k + 1]]
    Z = pk[:, :k].sum(1)
    U = np.einsum("tj,tjh->th", pk[:, :k], F[:, :k])
    out = np.empty((idx.shape[0], k, F.shape[2]))
    for j in range(k):
        Zp = Z - pk[:, j] + pk[:, k]
        out[:, j] = (U - pk[:, j:j + 1] * F[:, j]) / Zp[:, None] - U / Z[:, None]  # p_r f_r dropped
    return out


def _select_ascending(sum_sq, count, keep):
    s = razor.scores(sum_sq, count)
    ranking = np.lexsort((np.arange(len(s)), s))
    return np.sort(ranking[:keep]), ranking, s


def _pack_reversed(codes):
    c = np.asarray(codes, np.int64)
    c = c.reshape(*c.shape[:-1], c.shape[-1] // 8, 8)
    word = np.zeros(c.shape[:-1], np.int64)
    for i in range(8):
        word |= c[..., i] << (4 * (7 - i))
    return word.astype(np.uint32).view(np.int32)


def _dequant_group16(qweight, qzeros, scales, mode="fp16"):
    q, z = awq.unpack_nibbles(qweight), awq.unpack_nibbles(qzeros)
    s = np.asarray(scales, np.float16).astype(np.float64)
    g = np.arange(q.shape[0]) // 16  # wrong group size
    return awq.f64_to_f16((q - z[g]) * s[g]).astype(np.float64)


def _dequant_bf16_unrounded_scale(orig):
    def dequant(qweight, qzeros, scales, mode="fp16"):
        if mode != "bf16":
            return orig(qweight, qzeros, scales, mode)
        q, z = awq.unpack_nibbles(qweight), awq.unpack_nibbles(qzeros)
        s = np.asarray(scales, np.float16).astype(np.float64)
        g = np.arange(q.shape[0]) // awq.GROUP
        return awq.bf16_round((q - z[g]) * s[g])  # the FP16 scale not rounded to BF16 first
    return dequant


def _quantize_4sg(v, s_g=None):
    v = np.asarray(v, np.float32)
    rows, K = v.shape
    s_g = nvfp4.global_scale(v) if s_g is None else np.float32(s_g)
    blocks = v.reshape(rows, K // 16, 16)
    t = np.float32(np.float32(4.0) * s_g)  # 4 instead of 6: the block max no longer maps to code 6
    sb_code = f32_to_e4m3((np.max(np.abs(blocks), axis=2) / t).astype(np.float32))
    denom = (e4m3_to_f64(sb_code).astype(np.float32) * s_g).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(denom[:, :, None] > 0, (blocks / denom[:, :, None]).astype(np.float32), np.float32(0))
    return f32_to_e2m1(q).reshape(rows, K), sb_code, s_g


def _awq_halves_swapped(qw_gu, qz_gu, sc_gu, qw_d, qz_d, sc_d, e, I, mode="fp16"):
    wgu = awq.dequant(qw_gu[e], qz_gu[e], sc_gu[e], mode)
    wd = awq.dequant(qw_d[e], qz_d[e], sc_d[e], mode)
    return wgu[:, I:].T, wgu[:, :I].T, wd.T  # up taken as gate and gate as up


def _nvfp4_shared_gate_up_scale(w_gate_up, w_down):
    E, I2, _ = w_gate_up.shape
    I = I2 // 2
    raw, deq = {}, {}
    for e in range(E):
        c, sb, g = nvfp4.quantize(w_gate_up[e].astype(np.float32))  # gate and up as one tensor
        raw[(e, "gate")], raw[(e, "up")] = (c[:I], sb[:I], g), (c[I:], sb[I:], g)
        raw[(e, "down")] = nvfp4.quantize(w_down[e].astype(np.float32))
        for name in ("gate", "up", "down"):
            deq[(e, name)] = nvfp4.dequant(*raw[(e, name)])
    return (lambda e: (deq[(e, "gate")], deq[(e, "up")], deq[(e, "down")])), raw


MUTATIONS = [
    ("silu sign", lambda mp: mp.setattr(moe, "silu", _silu_sign),
     [tm.test_softmax_and_silu_vs_torch, tm.test_single_expert_layer_is_textbook_swiglu]),
    ("gate and up swapped", lambda mp: mp.setattr(moe, "swiglu_expert", _swap_gate_up(moe.swiglu_expert)),
     [tm.test_single_expert_layer_is_textbook_swiglu]),
    ("down projection not transposed", lambda mp: mp.setattr(moe, "swiglu_expert", _down_untransposed),
     [tm.test_single_expert_layer_is_textbook_swiglu]),
    ("selected weights not renormalised", lambda mp: mp.setattr(moe, "route", _route_unnormalised(moe.route)),
     [tm.test_route_weights_sum_to_one_and_follow_probabilities]),
    ("ties to the higher index", lambda mp: mp.setattr(moe, "expert_order", _order_ties_high),
     [tm.test_route_topk_matches_brute_force_with_ties]),
    ("shared expert left out", lambda mp: mp.setattr(moe, "moe_layer", _layer_without_shared(moe.moe_layer)),
     [tm.test_single_expert_layer_is_textbook_swiglu]),
    ("tokens descending inside an expert", lambda mp: mp.setattr(moe, "permute", _permute_tokens_descending),
     [tm.test_permute_structure_and_brute_force]),
    ("shared gate sign", lambda mp: mp.setattr(moe, "shared_gate", lambda x, w: 1.0 / (1.0 + np.exp(x @ w))),
     [tm.test_shared_gate_closed_forms_and_library]),
    ("RMSNorm gain w instead of 1 + w",
     lambda mp: mp.setattr(moe, "rmsnorm", lambda x, w, eps=1e-6: x / np.sqrt(np.mean(x * x, -1, keepdims=True) + eps) * w),
     [tm.test_rmsnorm_against_torch_and_closed_forms]),
    ("Refill: promoted expert dropped (definition)",
     lambda mp: mp.setattr(razor, "refill_deltas_literal", _literal_without_promoted),
     [tr.test_refill_definition_equals_knockout_reevaluation]),
    ("Refill: promoted term dropped (closed form)",
     lambda mp: mp.setattr(razor, "refill_deltas_closed_form", _closed_form_without_promoted),
     [tr.test_refill_closed_form_equals_definition]),
    ("ranking ascending", lambda mp: mp.setattr(razor, "select", _select_ascending),
     [tr.test_select_hand_example_and_brute_force]),
    ("router norm as an L1 norm",
     lambda mp: mp.setattr(razor, "router_norm", lambda w: np.sum(np.abs(np.asarray(w, np.float64)), axis=1)),
     [tr.test_router_norm_hand_example_and_library]),
    ("slice in reversed order", lambda mp: mp.setattr(razor, "slice_experts",
                                                      lambda a, kept: np.asarray(a)[np.asarray(kept)[::-1]]),
     [tr.test_sliced_layer_equals_layer_with_removed_experts_masked]),
    ("AWQ nibble order reversed", lambda mp: mp.setattr(awq, "pack_nibbles", _pack_reversed),
     [tq.test_awq_pack_layout_and_round_trip]),
    ("AWQ group of 16 rows", lambda mp: mp.setattr(awq, "dequant", _dequant_group16),
     [tq.test_awq_dequant_zero_at_zero_point_and_vs_torch_half]),
    ("AWQ BF16 mode without scale rounding", lambda mp: mp.setattr(awq, "dequant", _dequant_bf16_unrounded_scale(awq.dequant)),
     [tq.test_awq_dequant_bf16_mode_vs_torch_bfloat16]),
    ("AWQ gate and up halves swapped", lambda mp: mp.setattr(awq, "expert_weights_out_in", _awq_halves_swapped),
     [tq.test_awq_expert_bank_split_and_orientation]),
    ("NVFP4 one global scale shared by gate and up",
     lambda mp: mp.setattr(nvfp4, "quantize_expert_weights", _nvfp4_shared_gate_up_scale),
     [tq.test_nvfp4_expert_weights_one_global_scale_per_projection]),
    ("block input not rounded to 16 bits",
     lambda mp: mp.setattr(moe, "block_input", lambda x, w, eps=1e-6, dtype="bf16": moe.rmsnorm(x, w, eps)),
     [tm.test_block_input_is_the_rounded_norm]),
    ("BF16 rounding by truncation", lambda mp: mp.setattr(
        __import__("oracle.formats", fromlist=["formats"]), "f64_to_bf16_values",
        lambda x: np.ldexp(np.trunc(np.frexp(np.asarray(x, np.float64))[0] * 256.0) / 256.0,
                           np.frexp(np.asarray(x, np.float64))[1])),
     [tm.test_bf16_rounding_from_float64]),
    ("NVFP4 block scale from 4 s_g", lambda mp: mp.setattr(nvfp4, "quantize", _quantize_4sg),
     [tq.test_nvfp4_grid_values_round_trip_exactly, tq.test_nvfp4_error_bound_and_block_max]),
]


@pytest.mark.parametrize("name,plant,pins", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_fails_a_pin(monkeypatch, name, plant, pins):
    for pin in pins:
        assert not _fails(pin), f"{pin.__name__} fails on the unmodified oracle"
    plant(monkeypatch)
    assert any(_fails(pin) for pin in pins), f"no pin catches: {name}"
