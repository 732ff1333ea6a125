"""The oracle's pins catch plausible slips.  Each test plants one slip in a
copy of the PyTorch restatement of the oracle (on the CPU: one function
replaced, the rest untouched) and runs an existing pin of
tests/test_oracle_pins.py against it; the pin must fail.  A last test runs
the same pins on the unmodified copy, which must pass."""
import types

import pytest
import torch

import oracle
import test_oracle_pins as pins

F64 = torch.float64
REF = oracle.torch_ref


def _copy(**replaced):
    ns = types.SimpleNamespace(**{n: getattr(REF, n) for n in REF.__all__})
    for k, v in replaced.items():
        setattr(ns, k, v)
    return ns


# ------------------------------------------------------------------ selection
def _select(slip):
    def select_experts(s, b, k):
        s = torch.as_tensor(s, dtype=F64)
        b = torch.as_tensor(b, dtype=F64)
        key = s.clone() if slip == "bias_ignored" else s + b
        T, E = key.shape
        rows = []
        for t in range(T):
            tie = (lambda e: -e) if slip == "ties_to_higher_index" else (lambda e: e)
            rows.append(sorted(range(E), key=lambda e: (-key[t, e].item(), tie(e)))[:k])
        idx = torch.tensor(rows, dtype=torch.int64)
        num = torch.gather(key if slip == "biased_mixture" else s, 1, idx)
        p = num / num.sum(dim=1, keepdim=True)
        srt = torch.sort(key, dim=1, descending=True).values
        margin = srt[:, k - 1] - srt[:, k] if k < E else torch.full((T,), float("inf"), dtype=F64)
        return idx, p, margin
    return select_experts


@pytest.mark.parametrize("slip", ["ties_to_higher_index", "biased_mixture", "bias_ignored"])
def test_selection_pins_catch(slip):
    O = _copy(select_experts=_select(slip))
    failed = 0
    for E, k in [(6, 3), (8, 4), (12, 4)]:
        try:
            pins.test_select_experts_brute_force(O, E, k)
        except AssertionError:
            failed += 1
    try:
        pins.test_mixture_weights_use_unbiased_scores(O)
    except AssertionError:
        failed += 1
    assert failed > 0


def test_router_pin_catches_a_transposed_weight():
    O = _copy(router_scores=lambda x, Wr: REF.sigmoid(x @ Wr))
    with pytest.raises(AssertionError):
        pins.test_router_orientation(O)


# ------------------------------------------------------------------ experts
@pytest.mark.parametrize("slip", ["no_sigmoid", "no_cap_on_v", "cap_without_1_over_c"])
def test_situ_glu_pin_catches(slip):
    def situ_glu(g, v, c):
        if slip == "no_sigmoid":
            return (c * torch.tanh(g / c)) * (c * torch.tanh(v / c))
        if slip == "no_cap_on_v":
            return torch.sigmoid(g) * (c * torch.tanh(g / c)) * v
        return torch.sigmoid(g) * (c * torch.tanh(g)) * (c * torch.tanh(v))
    with pytest.raises(AssertionError):
        pins.test_situ_glu_properties(_copy(situ_glu=situ_glu))


@pytest.mark.parametrize("slip", ["gate_up_swapped", "h_not_rounded"])
def test_expert_pin_catches(slip):
    def expert_forward(z, Wg, Wv, Wo, c, rnd, act=None):
        g, v = z @ Wg.T, z @ Wv.T
        if slip == "gate_up_swapped":
            g, v = v, g
        h = REF.situ_glu(g, v, c)
        return (h if slip == "h_not_rounded" else rnd(h)) @ Wo.T
    with pytest.raises(AssertionError):
        pins.test_expert_forward_orientation(_copy(expert_forward=expert_forward))


# ------------------------------------------------------------------ combine, RMSNorm, permute
@pytest.mark.parametrize("slip", ["slots_reversed", "weights_ignored"])
def test_combine_pin_catches(slip):
    def combine(y, p):
        if slip == "weights_ignored":
            return y.mean(dim=1)
        return torch.einsum("tj,tjl->tl", p, y.flip(1))
    with pytest.raises(AssertionError):
        pins.test_combine_one_hot_and_linear(_copy(combine=combine))


@pytest.mark.parametrize("slip", ["eps_outside_sqrt", "sum_not_mean", "gain_ignored"])
def test_rms_norm_pin_catches(slip):
    def rms_norm(u, gamma, eps):
        ms = (u * u).sum(dim=1, keepdim=True) if slip == "sum_not_mean" else (u * u).mean(dim=1, keepdim=True)
        d = torch.sqrt(ms) + eps if slip == "eps_outside_sqrt" else torch.sqrt(ms + eps)
        return u / d if slip == "gain_ignored" else gamma[None] * u / d
    with pytest.raises(AssertionError):
        pins.test_rms_norm_closed_forms(_copy(rms_norm=rms_norm))


def test_permute_pin_catches_an_unstable_order():
    def permute(idx, E):
        counts, offsets, perm_token, inv_perm = REF.permute(idx, E)
        perm_token = perm_token.copy()
        for e in range(E):  # tokens of each expert in descending order
            perm_token[offsets[e]:offsets[e + 1]] = perm_token[offsets[e]:offsets[e + 1]][::-1]
        return counts, offsets, perm_token, inv_perm
    with pytest.raises(AssertionError):
        pins.test_permute_invariants_and_library_sort(_copy(permute=permute))


def test_the_unmodified_copy_passes_the_same_pins():
    O = _copy()
    for E, k in [(6, 3), (8, 4), (12, 4)]:
        pins.test_select_experts_brute_force(O, E, k)
    pins.test_mixture_weights_use_unbiased_scores(O)
    pins.test_router_orientation(O)
    pins.test_situ_glu_properties(O)
    pins.test_expert_forward_orientation(O)
    pins.test_combine_one_hot_and_linear(O)
    pins.test_rms_norm_closed_forms(O)
    pins.test_permute_invariants_and_library_sort(O)
