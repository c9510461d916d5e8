"""The oracles' pins are not vacuous: a plausible mistake planted in a copy of an oracle
(on the CPU; the oracle files themselves are untouched) makes at least one pin fail.

Each case rewrites one line of the oracle's source, loads the result as a separate module,
points the pin tests at it and expects a failure (an assertion, or an exception for a
shape error)."""
import inspect
import sys
import types

import pytest

import oracle.indexer_kl_oracle as IKO
import oracle.sfa_oracle as SFO


def mutant(module, old, new):
    src = inspect.getsource(module)
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    src = src.replace(old, new).replace("from .sfa_oracle import", "from oracle.sfa_oracle import")
    name = f"{module.__name__}_mutant_{abs(hash((old, new)))}"
    mod = types.ModuleType(name)
    sys.modules[name] = mod  # dataclasses resolve annotations through sys.modules
    exec(compile(src, f"<{name}>", "exec"), mod.__dict__)
    return mod


def fails(fn, *args):
    try:
        fn(*args)
    except Exception:  # an assertion or a shape error: the pin caught the mistake
        return True
    return False


# ---------------------------------------------------------------------------
# sparse attention oracle: finite differences, torch SDPA, hand-worked index cases
SFA_MUTATIONS = {
    "dq_scale_dropped": ("dqt[where[t]] = scale * (ds @ kt)", "dqt[where[t]] = (ds @ kt)"),
    "ds_sign_flipped": ("ds = p * (dp - dsum[:, None])  # stage 2", "ds = p * (dsum[:, None] - dp)  # stage 2"),
    "rowsum_of_do_with_itself": ("dsum = (do * _row(out, t, dtype)).sum(axis=1)",
                          "dsum = (do * _row(out, t, dtype)).sum(axis=1) * 0 + (do * do).sum(axis=1)"),
    "dk_scatter_overwrites": ("np.add.at(dkt, g, scale * (ds.T @ qt))", "dkt[g] = scale * (ds.T @ qt)"),
    "dv_uses_ds": ("np.add.at(dv, g, p.T @ do)", "np.add.at(dv, g, (p * (dp - dp.mean())).T @ do)"),
    "causal_off_by_one": ("if sparse_mode == 3 and j > q_pos + kv_len - q_len:",
                          "if sparse_mode == 3 and j >= q_pos + kv_len - q_len:"),
    "causal_top_left": ("if sparse_mode == 3 and j > q_pos + kv_len - q_len:",
                        "if sparse_mode == 3 and j > q_pos:"),
    "block_rows_not_cut_at_sequence_end": ("            if j >= kv_len:\n                break\n", ""),
}


@pytest.mark.parametrize("name", sorted(SFA_MUTATIONS))
def test_sfa_oracle_mistake_is_caught(name, monkeypatch):
    import test_oracle_pins as pins
    mod = mutant(SFO, *SFA_MUTATIONS[name])
    monkeypatch.setattr(pins, "O", mod)
    checks = [
        (pins.test_fd_gradients_bsnd, 1, 3, "causal"),
        (pins.test_fd_gradients_tnd_messy_duplicates,),
        (pins.test_sdpa_special_case_forward_and_backward,),
        (pins.test_selected_rows_hand_cases,),
    ]
    assert any(fails(c[0], *c[1:]) for c in checks), f"planted mistake {name} passed every pin"


# ---------------------------------------------------------------------------
# dense FA oracle: finite differences with GQA and the bottom-right causal mask, torch SDPA
# with is_causal, the page's all-ones worked example
FA_MUTATIONS = {
    "gqa_head_map": ("            hk = h // g\n", "            hk = h % Nkv\n"),
    "dq_scale_dropped": ("dq[qs, h] = scale * (ds @ k[ks, hk])", "dq[qs, h] = ds @ k[ks, hk]"),
    "dk_overwrites_heads": ("dk[ks, hk] += scale * (ds.T @ q[qs, h])", "dk[ks, hk] = scale * (ds.T @ q[qs, h])"),
    "causal_top_left": ("return j <= i + (kv_len - q_len)", "return j <= i"),
}


@pytest.mark.parametrize("name", sorted(FA_MUTATIONS))
def test_fa_oracle_mistake_is_caught(name, monkeypatch):
    import test_oracle_pins as pins
    mod = mutant(SFO, *FA_MUTATIONS[name])
    monkeypatch.setattr(pins, "O", mod)
    checks = [
        (pins.test_fa_oracle_fd_gqa_bottom_right_causal,),
        (pins.test_fa_oracle_sdpa_causal_square,),
        (pins.test_fa_oracle_sdpa_lower_right_causal_nonsquare,),
        (pins.test_page2_worked_example_all_ones,),
    ]
    assert any(fails(c[0], *c[1:]) for c in checks), f"planted mistake {name} passed every pin"


# ---------------------------------------------------------------------------
# indexer-gradient oracle: finite differences of the loss, torch autograd with kl_div
IKO_MUTATIONS = {
    "target_not_normalised": ("p = prob.sum(axis=0) / N1", "p = prob.sum(axis=0) / (2 * N1)"),
    "relu_mask_dropped_in_ds": ("ds = di[None, :] * w[:, None] * (s > 0)", "ds = di[None, :] * w[:, None]"),
    "relu_dropped_in_dw": ("d_weights[t] = np.maximum(s, 0.0) @ di", "d_weights[t] = s @ di"),
    "dk_sign_flipped": ("dk_index[rows] += ds.T @ np.asarray(q_index[t], dtype)",
                        "dk_index[rows] -= ds.T @ np.asarray(q_index[t], dtype)"),
    "entropy_term_dropped": ("loss_t[t] = np.sum(p[pos_p] * (np.log(p[pos_p]) - log_si[pos_p]))",
                             "loss_t[t] = np.sum(p[pos_p] * (-log_si[pos_p]))"),
    "indexer_scores_transposed_weights": ("return s, w @ np.maximum(s, 0.0)", "return s, w @ s"),
}


@pytest.mark.parametrize("name", sorted(IKO_MUTATIONS))
def test_indexer_oracle_mistake_is_caught(name, monkeypatch):
    import test_indexer_oracle_pins as pins
    mod = mutant(IKO, *IKO_MUTATIONS[name])
    monkeypatch.setattr(pins, "indexer_kl_grad_problem", mod.indexer_kl_grad_problem)
    monkeypatch.setattr(pins, "indexer_softmax_stats", mod.indexer_softmax_stats)
    monkeypatch.setattr(pins, "visible_keys", mod.visible_keys)
    checks = [
        (pins.test_finite_differences, "tnd_causal"),
        (pins.test_torch_autograd_special_case, "tnd_causal"),
        (pins.test_zero_divergence_when_distributions_match,),
    ]
    assert any(fails(c[0], *c[1:]) for c in checks), f"planted mistake {name} passed every pin"


def test_unmutated_oracles_pass_the_same_checks():
    """Control: the same checks pass on the oracles as they are."""
    import test_indexer_oracle_pins as ipins
    import test_oracle_pins as spins
    assert not fails(spins.test_fd_gradients_bsnd, 1, 3, "causal")
    assert not fails(spins.test_sdpa_special_case_forward_and_backward)
    assert not fails(spins.test_fa_oracle_fd_gqa_bottom_right_causal)
    assert not fails(spins.test_fa_oracle_sdpa_causal_square)
    assert not fails(spins.test_fa_oracle_sdpa_lower_right_causal_nonsquare)
    assert not fails(ipins.test_finite_differences, "tnd_causal")
    assert not fails(ipins.test_torch_autograd_special_case, "tnd_causal")
