"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in the oracle (on the CPU, by replacing one
function of ``oracle`` for the duration of the case) and runs the pins that
should see it; at least one of them must fail.  A planted mistake that every
pin accepts would mean the oracle is pinned to nothing at that point."""
import numpy as np
import pytest

import oracle
import oracle.fp8
import oracle.moe
from tests import test_oracle_backward as PB
from tests import test_oracle_dispatch_expert as PD
from tests import test_oracle_e5m2 as PE
from tests import test_oracle_fp8 as PF
from tests import test_oracle_fp8_backward as PFB
from tests import test_oracle_layer_backward as PL
from tests import test_oracle_route as PR

ORIG = {name: getattr(oracle.moe, name) for name in (
    "route", "group_scores", "biased_scores", "bias_update", "combine", "swiglu_expert",
    "dispatch", "swiglu_expert_backward", "route_backward", "dispatch_backward",
    "combine_backward", "round_bf16", "affinity")}
ORIG_E4M3 = oracle.fp8.e4m3_encode
ORIG_E5M2 = oracle.fp8.e5m2_encode


# ---- the planted mistakes -------------------------------------------------------------

def gates_from_biased_scores(x, router, bias, G, topG, K):
    r = dict(ORIG["route"](x, router, bias, G, topG, K))
    sel = np.take_along_axis(r["sb"], r["idx"], axis=1)
    r["gate"] = sel / sel.sum(axis=1, keepdims=True)
    return r


def group_score_top1(sb, G):
    T, N = sb.shape
    gs = N // G
    return np.stack([sb[:, g * gs:(g + 1) * gs].max(axis=1) for g in range(G)], axis=1)


def bias_ignored(s, bias):
    return np.asarray(s, dtype=np.float64)


def bias_update_sign_flipped(bias, counts, T, K, gamma):
    return ORIG["bias_update"](bias, counts, T, K, -gamma)


def combine_without_shared(shared, routed, idx, gate, tokens):
    return ORIG["combine"](np.zeros_like(np.asarray(shared, np.float64)), routed, idx, gate,
                           tokens)


def swiglu_roles_swapped(a, w1, w3, w2, h_round="none"):
    return ORIG["swiglu_expert"](a, w3, w1, w2, h_round)


def dispatch_tokens_descending(idx, N):
    idx = np.asarray(idx)
    d = ORIG["dispatch"](idx[::-1], N)
    T = idx.shape[0]
    perm = (T - 1) - d["perm_tok"]
    return dict(offsets=d["offsets"], perm_tok=perm, slot=d["slot"][::-1].copy(),
                counts=d["counts"])


def silu_derivative_missing_term(a, w1, w3, w2, dy, gu_round="none", dgu_round="none"):
    a = np.asarray(a, np.float64)
    w1, w3, w2 = (np.asarray(w, np.float64) for w in (w1, w3, w2))
    dy = np.asarray(dy, np.float64)
    g, u = a @ w1.T, a @ w3.T
    sig = 1.0 / (1.0 + np.exp(-g))
    h = g * sig * u
    dh = dy @ w2
    dg = dh * u * sig                      # the g (1 - sigma) term dropped
    du = dh * g * sig
    return dict(da=dg @ w1 + du @ w3, dw1=dg.T @ a, dw3=du.T @ a, dw2=dy.T @ h, dg=dg, du=du,
                dh=dh)


def gate_gradient_without_normalisation(x, router, idx, dgate):
    r = dict(ORIG["route_backward"](x, router, idx, np.zeros(np.asarray(idx).shape)))
    x = np.asarray(x, np.float64)
    R = np.asarray(router, np.float64)
    s, S = r["s"], r["s"].sum(axis=1, keepdims=True)
    dz = np.asarray(dgate, np.float64) / S * s * (1.0 - s)   # the mean term dropped
    r["dz"] = dz
    r["dx"] = np.einsum("tk,tkd->td", dz, R[np.asarray(idx)])
    drouter = np.zeros_like(R)
    for t in range(dz.shape[0]):
        for k in range(dz.shape[1]):
            drouter[idx[t, k]] += dz[t, k] * x[t]
    r["drouter"] = drouter
    return r


def dispatch_backward_drops_router_path(dx_perm, dx_shared, slot, dx_route=None):
    return ORIG["dispatch_backward"](dx_perm, dx_shared, slot, None)


def combine_backward_ignores_gate(dy, y_perm, slot, gate):
    return ORIG["combine_backward"](dy, y_perm, slot, np.ones_like(np.asarray(gate, np.float64)))


def round_bf16_truncates(v):
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    e = np.maximum(e, -125)
    step_exp = e - 8
    return np.ldexp(np.trunc(np.ldexp(v, -step_exp)), step_exp)


def e4m3_ties_away(v):
    v = np.asarray(v, dtype=np.float64)
    return ORIG_E4M3(v * (1.0 + 1e-9))


# ---- which pins must see each mistake ---------------------------------------------------

ROUTE_PINS = [
    PR.test_hand_worked_fixture,
    lambda: PR.test_brute_force_selection(40, 16, 16, 4, 2, 3),
    PR.test_brute_force_tiny_config,
    lambda: PR.test_invariants(1),
    PR.test_bias_moves_selection_not_gates,
    PR.test_special_cases,
]
EXPERT_PINS = [PD.test_dense_brute_force_moe, PD.test_silu_glu_special_case_matches_torch,
               PD.test_combine_weights_and_order]
LAYER_BWD_PINS = [lambda: PL.test_dx_matches_finite_differences(0),
                  PL.test_drouter_matches_finite_differences,
                  PL.test_combine_backward_is_the_derivative_of_combine,
                  PL.test_uniform_gate_gradient_moves_nothing]

CASES = [
    ("route", gates_from_biased_scores, ROUTE_PINS),
    ("group_scores", group_score_top1, ROUTE_PINS),
    ("biased_scores", bias_ignored, ROUTE_PINS),
    ("bias_update", bias_update_sign_flipped, [PD.test_bias_update_closed_form]),
    ("combine", combine_without_shared, EXPERT_PINS),
    ("swiglu_expert", swiglu_roles_swapped, EXPERT_PINS),
    ("dispatch", dispatch_tokens_descending, [PD.test_dispatch_is_lexicographic_sort]),
    ("swiglu_expert_backward", silu_derivative_missing_term,
     [lambda: PB.test_gradients_match_central_differences(3, 5, 4)]),
    ("route_backward", gate_gradient_without_normalisation, LAYER_BWD_PINS),
    ("dispatch_backward", dispatch_backward_drops_router_path, LAYER_BWD_PINS),
    ("combine_backward", combine_backward_ignores_gate, LAYER_BWD_PINS),
    ("round_bf16", round_bf16_truncates, [PD.test_round_bf16_matches_torch_from_float32]),
]


def _fails(pins):
    caught = []
    for pin in pins:
        try:
            pin()
        except (AssertionError, RuntimeError, ValueError, IndexError, KeyError):
            caught.append(pin)
    return caught


@pytest.mark.parametrize("name,mutant,pins", CASES, ids=[c[0] + ":" + c[1].__name__
                                                         for c in CASES])
def test_planted_mistake_is_caught(monkeypatch, name, mutant, pins):
    monkeypatch.setattr(oracle.moe, name, mutant)
    monkeypatch.setattr(oracle, name, mutant)
    assert _fails(pins), f"no pin caught {mutant.__name__}"


def test_planted_e4m3_rounding_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(oracle.fp8, "e4m3_encode", e4m3_ties_away)
    monkeypatch.setattr(oracle, "e4m3_encode", e4m3_ties_away)
    assert _fails([PF.test_exhaustive_code_table, PF.test_midpoints_round_to_even_and_saturate,
                   PF.test_encode_matches_torch_in_range])


def e5m2_ties_away(v):
    v = np.asarray(v, dtype=np.float64)
    return ORIG_E5M2(v * (1.0 + 1e-9))


def e5m2_overflow_to_inf(v):
    c = ORIG_E5M2(v)
    big = np.abs(np.asarray(v, dtype=np.float64)) > 57344.0
    return np.where(big, (c & 0x80) | 0x7C, c).astype(np.uint8)


@pytest.mark.parametrize("mutant", [e5m2_ties_away, e5m2_overflow_to_inf])
def test_planted_e5m2_mistake_is_caught(monkeypatch, mutant):
    monkeypatch.setattr(oracle.fp8, "e5m2_encode", mutant)
    monkeypatch.setattr(oracle, "e5m2_encode", mutant)
    assert _fails([PE.test_exhaustive_code_table, PE.test_midpoints_round_to_even_and_saturate,
                   PE.test_encode_matches_torch_in_range])


ORIG_FP8_BWD = oracle.fp8.fp8_swiglu_expert_backward_dx


def fp8_backward_weights_swapped(a, w1, w3, w2, dy, quant=True):
    return ORIG_FP8_BWD(a, w3, w1, w2, dy, quant)


def test_planted_fp8_backward_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(oracle.fp8, "fp8_swiglu_expert_backward_dx", fp8_backward_weights_swapped)
    monkeypatch.setattr(oracle, "fp8_swiglu_expert_backward_dx", fp8_backward_weights_swapped)
    assert _fails([lambda: PFB.test_without_quantisation_it_is_the_exact_backward(0),
                   lambda: PFB.test_fp8_error_stays_within_the_formats_precision(2)])


def test_the_unmodified_oracle_passes_the_same_pins():
    """Control: with nothing planted every pin used above passes."""
    pins = set()
    for _, _, ps in CASES:
        pins.update(ps)
    assert not _fails(list(pins))


# ---- FP8 forward expert: four plausible composition mistakes ----------------------------

from tests import test_oracle_fp8_expert as PFX  # noqa: E402

ORIG_FP8_FWD = oracle.fp8.fp8_swiglu_expert


def fp8_gate_and_up_swapped(a, w1, w3, w2, quant=True):
    return ORIG_FP8_FWD(a, w3, w1, w2, quant)


def _fp8_expert_with(a, w1, w3, w2, h_quant, w2_scales=lambda s: s):
    F = oracle.fp8
    qa, sa = F.quant_rows_1x128(a)
    q1, s1 = F.quant_blocks_128(w1)
    q3, s3 = F.quant_blocks_128(w3)
    q2, s2 = F.quant_blocks_128(w2)
    h = oracle.moe.silu(F.fp8_gemm_ref(qa, sa, q1, s1)) * F.fp8_gemm_ref(qa, sa, q3, s3)
    return h_quant(h.astype(np.float32), q2, w2_scales(s2))


def fp8_h_not_quantised(a, w1, w3, w2, quant=True):
    if not quant:
        return ORIG_FP8_FWD(a, w1, w3, w2, quant)
    def keep_h(h, q2, s2):
        W2 = oracle.fp8.e4m3_decode(q2) * np.kron(s2.astype(np.float64), np.ones((128, 128)))
        return h.astype(np.float64) @ W2.T
    return _fp8_expert_with(a, w1, w3, w2, keep_h)


def fp8_h_quantised_per_column(a, w1, w3, w2, quant=True):
    if not quant:
        return ORIG_FP8_FWD(a, w1, w3, w2, quant)
    def h_by_columns(h, q2, s2):
        qh, sh = oracle.fp8.quant_cols_1x128(h)                     # 128-row tiles along M
        H = oracle.fp8.e4m3_decode(qh) * np.repeat(sh.astype(np.float64), 128, axis=0)[:h.shape[0]]
        W2 = oracle.fp8.e4m3_decode(q2) * np.kron(s2.astype(np.float64), np.ones((128, 128)))
        return H @ W2.T
    return _fp8_expert_with(a, w1, w3, w2, h_by_columns)


def fp8_w2_scales_transposed(a, w1, w3, w2, quant=True):
    if not quant:
        return ORIG_FP8_FWD(a, w1, w3, w2, quant)
    def rows(h, q2, s2):
        qh, sh = oracle.fp8.quant_rows_1x128(h)
        return oracle.fp8.fp8_gemm_ref(qh, sh, q2, s2)
    # W2 is [d, f]: its scale grid is [d/128, f/128]; read it the other way round
    return _fp8_expert_with(a, w1, w3, w2, rows,
                            lambda s: np.ascontiguousarray(s.T).reshape(s.shape))


FP8_FWD_PINS = [lambda: PFX.test_without_quantisation_it_is_the_exact_expert(0),
                PFX.test_lossless_operands_leave_the_1x128_quantisation_of_h_along_f,
                lambda: PFX.test_error_stays_within_e4m3_precision(2),
                PFX.test_rows_are_independent,
                PFX.test_equals_swiglu_of_the_dequantised_operands]


@pytest.mark.parametrize("mutant", [fp8_gate_and_up_swapped, fp8_h_not_quantised,
                                    fp8_h_quantised_per_column, fp8_w2_scales_transposed])
def test_planted_fp8_forward_mistake_is_caught(monkeypatch, mutant):
    monkeypatch.setattr(oracle.fp8, "fp8_swiglu_expert", mutant)
    monkeypatch.setattr(oracle, "fp8_swiglu_expert", mutant)
    assert _fails(FP8_FWD_PINS), f"no pin caught {mutant.__name__}"


def test_the_unmodified_fp8_forward_passes_its_pins():
    assert not _fails(FP8_FWD_PINS)
