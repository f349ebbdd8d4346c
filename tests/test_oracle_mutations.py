"""The oracle's pins catch plausible mistakes: each case plants one mistake in a copy of an
oracle function (on the CPU, by a textual edit of its source), installs it, and checks that at
least one pin of ``test_oracle_pins`` fails."""
import inspect
import textwrap

import pytest

from oracle import swimba_oracle as O
import tests.test_oracle_block_pins as BP
import tests.test_oracle_pins as P

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

PINS = [
    P.test_softplus_special_values_and_library,
    P.test_silu_identities,
    lambda: P.test_route_brute_force(5, 3),
    lambda: P.test_route_brute_force(4, 2),
    P.test_route_top1_gate_is_exactly_one,
    P.test_projection_unit_vector_selects_weight_row,
    P.test_projection_brute_force_loops,
    P.test_mixing_streams_equals_mixing_weights,
    P.test_zero_dt_projection_leaves_mixed_bias,
    P.test_scan_closed_form_constant_inputs_scalar_state,
    lambda: P.test_scan_brute_force_unrolled_sum(5),
    P.test_identical_experts_reduce_to_dense_scan,
    P.test_invariants_and_bibo_bound_under_fast_switching,
    P.test_skip_path_alone_when_injection_or_readout_is_zero,
    P.test_free_decay_of_the_initial_state,
    P.test_chunk_split_and_step_by_step_equal_prefill,
    P.test_gate_placement_out_is_y_times_silu_z,
    lambda: BP.test_conv1d_matches_library_convolution(4),
    BP.test_conv1d_impulse_taps_are_identity_and_shift,
    BP.test_conv1d_zero_state_when_absent,
    lambda: BP.test_conv1d_state_handoff_equals_whole(2),
    BP.test_round_bf16_matches_torch,
    BP.test_block_is_residual_when_W_out_is_zero,
    BP.test_block_zero_gate_branch_gives_residual,
    BP.test_block_zero_convolution_gives_residual,
    BP.test_block_ssm_branch_takes_the_first_half_of_W_in,
    BP.test_block_is_causal,
    lambda: BP.test_block_split_and_decode_equal_whole(2),
    BP.test_block_output_minus_residual_is_linear_in_W_out,
    BP.test_block_bf16_stores_bf16_values,
    P.test_summary_closed_form_constant_inputs_scalar_state,
    lambda: P.test_summary_brute_force(3),
    P.test_chain_of_piece_summaries_gives_the_prefix_states,
    P.test_separate_moe_one_expert_is_the_selective_scan,
    lambda: P.test_separate_moe_brute_force(4),
    P.test_separate_moe_unchosen_expert_keeps_its_state_and_switching_differs_from_one_trajectory,
    P.test_zoh_is_the_exact_solution_for_held_inputs,
    lambda: P.test_zoh_brute_force_and_small_step_limit(3),
]

MUTATIONS = {
    "skip term dropped": ("selective_scan", " + D_skip[None, :] * x[:, t, :]", ""),
    "no delta in injection": ("selective_scan", "u = d_t[:, :, None] * B_mix", "u = 1.0 * B_mix"),
    "no delta in decay": ("selective_scan", "np.exp(d_t[:, :, None] * A_t)", "np.exp(A_t)"),
    "injection decayed too": ("selective_scan", "h = a_bar * h + u", "h = a_bar * (h + u)"),
    "readout before update": (
        "selective_scan",
        ["h = a_bar * h + u\n", "+ D_skip[None, :] * x[:, t, :]\n"],
        ["h_next = a_bar * h + u\n", "+ D_skip[None, :] * x[:, t, :]\n        h = h_next\n"],
    ),
    "exp instead of softplus": ("selective_scan", "delta = softplus(dt_mix)", "delta = np.exp(dt_mix)"),
    "gate z not SiLU": ("selective_scan", "out = y * silu(z)", "out = y * z"),
    "A mixed without gates": ("selective_scan", "g[:, t, j, None, None] * A[idx", "(1.0 / idx.shape[2]) * A[idx"),
    "h0 ignored": ("selective_scan", "if h0 is None else np.array(h0, dtype=np.float64)", "if True else None"),
    "sign of A flipped": ("selective_scan", "np.exp(d_t[:, :, None] * A_t)", "np.exp(-d_t[:, :, None] * A_t)"),
    "ties to the higher index": (
        "route",
        'order = np.argsort(-logits, axis=-1, kind="stable")[..., :k]',
        'order = (E - 1 - np.argsort(-logits[..., ::-1], axis=-1, kind="stable"))[..., :k]',
    ),
    "gates not normalised": ("route", "gates = w / w.sum(axis=-1, keepdims=True)", "gates = w"),
    "ascending order": ("route", "np.argsort(-logits", "np.argsort(logits"),
    "dt bias dropped": ("expert_projections", "@ W_dt[e] + b_dt[e]", "@ W_dt[e]"),
    "B and C swapped": (
        "expert_projections",
        'np.einsum("tj,tjn->tn", g, xdbl[:, :, R:R + N])',
        'np.einsum("tj,tjn->tn", g, xdbl[:, :, R + N:R + 2 * N])',
    ),
    "wrong expert table": ("expert_projections", "v = x[rows] @ W_x[e]", "v = x[rows] @ W_x[(e + 1) % E]"),
    "dt from the wrong columns": ("expert_projections", "v[:, :R] @ W_dt[e]", "v[:, N:N + R] @ W_dt[e]"),
    "softplus without max(v,0)": ("softplus", "np.maximum(v, 0.0) + ", ""),
    "silu as sigmoid": ("silu", "return z / (1.0 + np.exp(-z))", "return 1.0 / (1.0 + np.exp(-z))"),
    "conv taps reversed": ("causal_conv1d", "w[None, :, i] * p[:, t + i, :]", "w[None, :, W - 1 - i] * p[:, t + i, :]"),
    "conv state ignored": ("causal_conv1d", "if state is None:", "if True:"),
    "conv bias dropped": ("causal_conv1d", "acc = np.array(b, dtype=np.float64)", "acc = 0.0 * np.array(b, dtype=np.float64)"),
    "conv without SiLU": ("causal_conv1d", "return c, silu(c), p[:, L:, :].copy()", "return c, c, p[:, L:, :].copy()"),
    "conv state from the first rows": ("causal_conv1d", "p[:, L:, :].copy()", "p[:, :W - 1, :].copy()"),
    "conv reads one token late": ("causal_conv1d", "p[:, t + i, :]", "p[:, max(t + i - 1, 0), :]"),
    "x and z halves swapped": (
        "block_branches",
        "x_pre, z = store(xz[..., :D]), store(xz[..., D:])",
        "z, x_pre = store(xz[..., :D]), store(xz[..., D:])",
    ),
    "residual dropped": ("block_forward", "@ np.asarray(BW[\"W_out\"], dtype=np.float64) + u)", "@ np.asarray(BW[\"W_out\"], dtype=np.float64))"),
    "block conv state not carried": ("block_branches", "BW[\"conv_b\"], conv_state)", "BW[\"conv_b\"], None)"),
    "block h0 not carried": ("block_forward", "layer_forward(x, z, BW, k, h0=h0)", "layer_forward(x, z, BW, k, h0=None)"),
    "block layer on x_pre": ("block_forward", "layer_forward(x, z, BW, k", "layer_forward(x_pre, z, BW, k"),
    "summary decay without delta": ("scan_summary", "log_decay += d_t[:, :, None] * A_t", "log_decay += A_t"),
    "summary injection without delta": ("scan_summary", "h + d_t[:, :, None] * B_mix[:, t, None, :] * x[:, t, :, None]",
                                        "h + B_mix[:, t, None, :] * x[:, t, :, None]"),
    "summary injection decayed too": ("scan_summary",
                                      "h = np.exp(d_t[:, :, None] * A_t) * h + d_t",
                                      "h = np.exp(d_t[:, :, None] * A_t) * h * 0.5 + d_t"),
    "chain adds before decaying": ("chain_summaries", "np.exp(log_decay[p]) * H[p] + h_zero[p]",
                                   "np.exp(log_decay[p]) * (H[p] + h_zero[p])"),
    "chain ignores h0": ("chain_summaries", "if h0 is not None:", "if False:"),
    "chain uses the next piece's decay": ("chain_summaries", "np.exp(log_decay[p])",
                                          "np.exp(log_decay[min(p + 1, P - 1)])"),
    "separate: one shared trajectory": ("separate_ssm_moe", "e = idx[b, t, j]", "e = 0"),
    "separate: outputs not gated": ("separate_ssm_moe", "y_t[b] += g[b, t, j] * (", "y_t[b] += 1.0 * ("),
    "separate: first slot's step for every slot": ("separate_ssm_moe", "d_bj = delta[b, t, j]", "d_bj = delta[b, t, 0]"),
    "separate: skip dropped": ("separate_ssm_moe", "y_t = D_skip[None, :] * x[:, t, :]", "y_t = 0.0 * x[:, t, :]"),
    "separate: first slot's readout for every slot": ("separate_ssm_moe", "(h[e, b] @ C_j[b, t, j])",
                                                       "(h[e, b] @ C_j[b, t, 0])"),
    "zoh without the transition's inverse": ("selective_scan", "np.expm1(d_t[:, :, None] * A_t) / A_t",
                                             "np.expm1(d_t[:, :, None] * A_t)"),
    "zoh with exp instead of expm1": ("selective_scan", "np.expm1(d_t[:, :, None] * A_t) / A_t",
                                      "np.exp(d_t[:, :, None] * A_t) / A_t"),
    "zoh falls back to Euler": ("selective_scan", 'if injection == "zoh":', 'if injection == "never":'),
    "bf16 rounding toward zero": ("round_bf16", "np.rint(m * 256.0)", "np.trunc(m * 256.0)"),
    "bf16 rounding with 7 bits": ("round_bf16", "np.ldexp(np.rint(m * 256.0), e - 8)", "np.ldexp(np.rint(m * 128.0), e - 7)"),
}


def _mutant(fn_name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(O, fn_name)))
    olds, news = (old, new) if isinstance(old, list) else ([old], [new])
    for o, n in zip(olds, news):
        assert o in src, f"mutation target not found in {fn_name}: {o!r}"
        src = src.replace(o, n, 1)
    ns = dict(vars(O))
    exec(compile(src, f"<mutant {fn_name}>", "exec"), ns)
    return ns[fn_name]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    fn_name, old, new = MUTATIONS[name]
    monkeypatch.setattr(O, fn_name, _mutant(fn_name, old, new))
    failed = []
    for pin in PINS:
        try:
            pin()
        except Exception as exc:  # an assertion, or an error the mistake provokes
            failed.append(exc)
            break
    assert failed, f"no pin fails with the planted mistake: {name}"


# ---- the Mamba-2 SSD form (oracle/swimba_ssd_oracle.py) ----------------------------------------

from oracle import swimba_ssd_oracle as SSD  # noqa: E402
import tests.test_oracle_ssd_pins as SP  # noqa: E402

SSD_PINS = [
    lambda: SP.test_ssd_brute_force_unrolled_sum(5),
    SP.test_one_channel_per_head_reduces_to_the_selective_scan,
    SP.test_identical_experts_equal_one_expert,
    SP.test_superposition_in_X_and_the_state,
    SP.test_state_decays_freely_without_input,
    lambda: SP.test_chunked_form_equals_sequential(4),
    SP.test_chunked_zero_state_when_absent,
]

SSD_MUTATIONS = {
    "decay without delta": ("ssd_scan_sequential", "a = np.exp(delta[t] * A)", "a = np.exp(A)"),
    "injection without delta": ("ssd_scan_sequential", "S = a[:, None, None] * S + delta[t][:, None, None] * inj",
                                "S = a[:, None, None] * S + inj"),
    "injection decayed too": ("ssd_scan_sequential", "S = a[:, None, None] * S + delta[t][:, None, None] * inj",
                              "S = a[:, None, None] * (S + delta[t][:, None, None] * inj)"),
    "readout with the first expert's C": ("ssd_scan_sequential", "c_mix = g[t] @ C[t]", "c_mix = C[t, 0]"),
    "skip on the first expert's X": ("ssd_scan_sequential", 'x_mix = np.einsum("j,jhp->hp", g[t], X[t])',
                                     "x_mix = X[t, 0]"),
    "injection ungated": ("ssd_scan_sequential", "inj += g[t, j] * X[t, j]", "inj += X[t, j]"),
    "chunk mask transposed": ("ssd_scan_chunked", "np.tril(np.ones((n, n)))", "np.triu(np.ones((n, n)))"),
    "carried state undecayed in the readout": ("ssd_scan_chunked",
                                               'y_c += np.exp(cum)[:, :, None] * np.einsum("hpn,in->ihp", S, c_mix)',
                                               'y_c += np.einsum("hpn,in->ihp", S, c_mix)'),
    "state passed without the tail decay": ("ssd_scan_chunked", "tail = np.exp(cum[-1][None, :] - cum)",
                                            "tail = np.ones_like(cum)"),
    "in-chunk term without the gate": ("ssd_scan_chunked", "(cb * (g[c0:c1, j])[None, :])", "(cb * 1.0)"),
}


def _ssd_mutant(fn_name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(SSD, fn_name)))
    assert old in src, f"mutation target not found in {fn_name}: {old!r}"
    src = src.replace(old, new, 1)
    ns = dict(vars(SSD))
    exec(compile(src, f"<mutant {fn_name}>", "exec"), ns)
    return ns[fn_name]


@pytest.mark.parametrize("name", sorted(SSD_MUTATIONS))
def test_ssd_pins_catch_planted_mistake(name, monkeypatch):
    fn_name, old, new = SSD_MUTATIONS[name]
    monkeypatch.setattr(SSD, fn_name, _ssd_mutant(fn_name, old, new))
    failed = []
    for pin in SSD_PINS:
        try:
            pin()
        except Exception as exc:
            failed.append(exc)
            break
    assert failed, f"no pin fails with the planted mistake: {name}"


# ---- the backward pass (oracle/swimba_backward_oracle.py) --------------------------------------

from oracle import swimba_backward_oracle as BO  # noqa: E402
import tests.test_oracle_backward_pins as BWP  # noqa: E402

BWD_PINS = [
    lambda: BWP.test_scan_backward_matches_finite_differences(0),
    BWP.test_scan_backward_one_token_closed_form,
    lambda: BWP.test_projection_backward_matches_finite_differences(0),
    BWP.test_softplus_backward_matches_finite_differences,
    BWP.test_route_backward_matches_finite_differences,
]

BWD_MUTATIONS = {
    "adjoint not carried back": ("scan_backward", "carry = a_ts[t] * lam", "carry = 0.0 * lam"),
    "adjoint carried without the decay": ("scan_backward", "carry = a_ts[t] * lam", "carry = lam"),
    "readout gradient from the previous state": ("scan_backward", 'dC[:, t, :] = np.einsum("bd,bdn->bn", dy[:, t, :], hs[t])',
                                                 'dC[:, t, :] = np.einsum("bd,bdn->bn", dy[:, t, :], h_prev[t])'),
    "step gradient without the decay term": ("scan_backward", 'np.einsum("bdn,bdn->bd", lam, A_ts[t] * a_ts[t] * h_prev[t]) + \\\n',
                                             '0.0 * np.einsum("bdn,bdn->bd", lam, A_ts[t] * a_ts[t] * h_prev[t]) + \\\n'),
    "step gradient without the injection term": ("scan_backward", 'np.einsum("bdn,bn->bd", lam, B_mix[:, t, :]) * x[:, t, :]\n',
                                                 '0.0 * x[:, t, :]\n'),
    "gate gradient through the wrong table": ("scan_backward", "dg[b, t, j] += np.sum(dA_t[b] * A[e[b]])",
                                              "dg[b, t, j] += np.sum(dA_t[b] * A[0])"),
    "A gradient ungated": ("scan_backward", "dA[e[b]] += gates[b, t, j] * dA_t[b]", "dA[e[b]] += dA_t[b]"),
    "SiLU derivative as sigmoid": ("silu_grad", "return s * (1.0 + np.asarray(z, dtype=np.float64) * (1.0 - s))",
                                   "return s"),
    "input gradient without the skip": ("scan_backward", "dx[:, t, :] = D_skip[None, :] * dy[:, t, :] + ",
                                        "dx[:, t, :] = "),
    "projection: bias gradient ungated": ("projection_backward", "d_dtj = gates[:, j, None] * g_dtmix",
                                          "d_dtj = g_dtmix"),
    "projection: W_dt gradient transposed use": ("projection_backward", "dv_e[:, :R] = d_dtj[rows] @ W_dt[e].T",
                                                 "dv_e[:, :R] = d_dtj[rows] @ W_dt[(e + 1) % W_x.shape[0]].T"),
    "projection: gate gradient without B": ("projection_backward", "np.sum(g_B * xdbl[:, j, R:R + N], axis=1)",
                                            "0.0"),
    "softplus derivative as exp": ("softplus_backward", "* sigmoid(dt_mix)", "* np.exp(dt_mix)"),
    "router: softmax Jacobian without the mean": ("route_backward",
                                                  "d_sel = gates * (g_gates - np.sum(gates * g_gates, axis=1, keepdims=True))",
                                                  "d_sel = gates * g_gates"),
}


def _bwd_mutant(fn_name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(BO, fn_name)))
    assert old in src, f"mutation target not found in {fn_name}: {old!r}"
    src = src.replace(old, new, 1)
    ns = dict(vars(BO))
    exec(compile(src, f"<mutant {fn_name}>", "exec"), ns)
    return ns[fn_name]


@pytest.mark.parametrize("name", sorted(BWD_MUTATIONS))
def test_backward_pins_catch_planted_mistake(name, monkeypatch):
    fn_name, old, new = BWD_MUTATIONS[name]
    mutant = _bwd_mutant(fn_name, old, new)
    monkeypatch.setattr(BO, fn_name, mutant)
    failed = []
    for pin in BWD_PINS:
        try:
            pin()
        except Exception as exc:
            failed.append(exc)
            break
    assert failed, f"no pin fails with the planted mistake: {name}"
