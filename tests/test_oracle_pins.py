"""Pins of the CPU oracle against facts other than itself: published tables,
closed forms, invariants, library routines and brute force on tiny inputs.
Each test would fail on a plausible slip in the oracle (a dropped term, a
wrong sign, a transposed operand, a wrong tie rule)."""
import itertools
import math

import numpy as np
import pytest
import scipy.special
import torch

import gen
import oracle
from conftest import read_golden
from oracle import inputs as oin

F64 = torch.float64


@pytest.fixture(params=["cpp", "torch"])
def O(request):
    """Each pin runs on both restatements of the method: the fp64 C++ oracle
    and the fp64 PyTorch one."""
    return oracle if request.param == "cpp" else oracle.torch_ref


# ---------------------------------------------------------------- number formats
def test_bf16_round_matches_torch_on_fp32_values(O):
    a = torch.randn(100_000, generator=torch.Generator().manual_seed(1), dtype=torch.float32) * 37.0
    want = a.to(torch.bfloat16).to(F64)
    got = O.bf16_round(a.to(F64))
    assert torch.equal(got, want)


def test_bf16_round_is_nearest_even_on_fp64_values(O):
    rng = np.random.default_rng(3)
    x = rng.standard_normal(20_000) * 10.0 ** rng.integers(-5, 5, 20_000)
    # include exact midpoints between bf16 neighbours
    mid = np.array([1.0 + 2.0**-8, 1.0 + 3 * 2.0**-8, -(2.0 + 2.0**-7)])
    x = np.concatenate([x, mid])
    r = O.bf16_round(torch.from_numpy(x)).numpy()
    for xi, ri in zip(x, r):
        e = math.frexp(abs(xi))[1]  # |x| in [2^(e-1), 2^e)
        ulp = 2.0 ** (e - 1 - 7)
        lo = math.floor(abs(xi) / ulp) * ulp
        hi = lo + ulp
        d_lo, d_hi = abs(xi) - lo, hi - abs(xi)
        if d_lo < d_hi:
            want = lo
        elif d_hi < d_lo:
            want = hi
        else:
            want = lo if (round(lo / ulp) % 2 == 0) else hi
        assert abs(ri) == want and (ri == 0 or np.sign(ri) == np.sign(xi))


def test_e2m1_dequant_matches_ocp_table(O):
    tab = {int(r[0]): float(r[1]) for r in read_golden("e2m1_ocp_mx.txt")}
    for s in (1, 100, 120, 127, 130, 200):
        codes = np.array([[c | (d << 4) for c, d in zip(range(0, 16, 2), range(1, 16, 2))] * 4], np.uint8)
        scales = np.full((1, 2), s, np.uint8)
        v = O.mxfp4_dequant(codes, scales)[0].numpy()
        for k in range(32):
            assert v[k] == tab[k % 16] * 2.0 ** (s - 127)
    nan = O.mxfp4_dequant(np.zeros((1, 16), np.uint8), np.full((1, 1), 255, np.uint8))
    assert torch.isnan(nan).all()


def test_mxfp4_dequant_of_generator_output_is_bf16_exact(O):
    # E2M1 x 2^e needs at most 2 significant bits: exact in bfloat16.
    c, s = gen.fill_host_mxfp4(0, 7, 0, 8, 512, 512**-0.5)
    v = O.mxfp4_dequant(c, s)
    assert torch.equal(O.bf16_round(v), v)


# ---------------------------------------------------------------- router
def test_e4m3_decode_matches_torch_float8(O):
    """All 256 E4M3 codes decode as PyTorch's float8_e4m3fn (a library
    implementation of the same OCP format), NaN codes included."""
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(F64)
    got = O.e4m3_decode(codes)
    assert torch.equal(torch.isnan(got), torch.isnan(want))
    assert torch.equal(torch.nan_to_num(got, nan=0.0), torch.nan_to_num(want, nan=0.0))
    assert got[0x7E].item() == 448.0 and got[0x01].item() == 2.0**-9 and got[0x08].item() == 2.0**-6


def test_e4m3_encode_matches_torch_cast_and_tie_rules(O):
    """Nearest-even encoding: PyTorch's fp32 -> float8_e4m3fn cast on values in
    range (fp32-exact, so one rounding), exact midpoints, saturation and the
    sign of zero."""
    g = torch.Generator().manual_seed(11)
    v = torch.randn(50_000, generator=g, dtype=torch.float64) * torch.exp2(
        torch.randint(-14, 9, (50_000,), generator=g).to(F64))
    v = v.to(torch.float32).clamp(-448, 448).to(F64)
    # midpoints between neighbouring E4M3 values (normal and subnormal ranges)
    vals = O.e4m3_decode(np.arange(0, 0x7E, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2
    v = torch.cat([v, mids, -mids])
    want = v.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(v), want)
    sat = O.e4m3_encode(torch.tensor([448.0, 463.9, 464.0, 1e6, -500.0, 0.0, -0.0], dtype=F64))
    assert list(sat) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x00, 0x80]


def test_mx8_scale_rule_closed_forms(O):
    """OCP MX v1.0 shared scale s = floor(log2 max|v|) - 8, clamped to the
    E8M0 range; codes of v / 2^s."""
    def q(block):
        c, s = O.mx8_quantize(torch.tensor([block], dtype=F64))
        return c[0], int(s[0, 0])

    c, s = q([1.0] * 32)                      # s = -8: 1 -> 256 = 2^8, code 0x78
    assert s == 119 and set(c) == {0x78}
    c, s = q([1.9375] + [0.0] * 31)           # 1.9375 * 2^8 = 496 saturates to 448
    assert s == 119 and c[0] == 0x7E and set(c[1:]) == {0}
    c, s = q([0.0] * 32)                      # all-zero block: the lowest scale
    assert s == 0 and set(c) == {0}
    c, s = q([2.0**-130] + [0.0] * 31)        # clamped at -127: 2^-130 * 2^127 = 2^-3
    assert s == 0 and c[0] == (4 << 3)
    c, s = q([2.0**127] * 32)                 # s = 119 (byte 246): 2^127 / 2^119 = 2^8
    assert s == 246 and set(c) == {0x78}
    c, s = q([-3.0, 0.75] + [0.0] * 30)       # max 3 -> s = -7: -3 * 128 = -384, 0.75 * 128 = 96
    assert s == 120 and c[0] == 0x80 | (15 << 3) | 4 and c[1] == (13 << 3) | 4
    v = torch.tensor([[2.0**-20] * 16 + [5.0] * 16], dtype=F64)  # tiny elements flush within the block
    assert O.mx8_round(v)[0, 0].item() == 0.0


def test_mx8_round_is_idempotent_and_within_half_a_step(O):
    """Quantising MXFP8 values again changes nothing, and each element moves by
    at most half an E4M3 step: 2^-4 of itself in the normal range, 2^-10 of
    the block scale below it; only elements above 448 units clip."""
    g = torch.Generator().manual_seed(12)
    x = torch.randn(64, 256, generator=g, dtype=F64) * torch.exp2(torch.randint(-20, 20, (64, 8), generator=g)
                                                                   .to(F64)).repeat_interleave(32, dim=1)
    x = x.to(torch.bfloat16).to(F64)
    r = O.mx8_round(x)
    assert torch.equal(O.mx8_round(r), r)
    _, s = O.mx8_quantize(x)
    scale = torch.exp2(torch.from_numpy(s.astype(np.int64) - 127).to(F64)).repeat_interleave(32, dim=1)
    units = (x / scale).abs()
    bound = torch.where(units >= 2.0**-6, x.abs() * 2.0**-4, scale * 2.0**-10)
    clipped = units > 448
    assert bool(((r - x).abs() <= bound + 1e-300)[~clipped].all())
    assert bool((r.abs()[clipped] == 448 * scale[clipped]).all())


def test_cpp_and_torch_mx8_agree_bit_for_bit():
    x = torch.randn(200, 1024, generator=torch.Generator().manual_seed(13), dtype=F64).to(torch.bfloat16).to(F64)
    x = x * torch.exp2(torch.randint(-40, 40, (200, 1), generator=torch.Generator().manual_seed(14)).to(F64))
    a = oracle.mx8_quantize(x)
    b = oracle.torch_ref.mx8_quantize(x)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_expert_forward_mx8_rounds_both_inputs(O):
    """act="mxfp8": the expert sees the MXFP8 values of its z rows and of h.  With
    z already MXFP8-exact the gate/up inputs are unchanged, so the result is
    W_o applied to mx8_round(h); with an identity-like W_o that is h's MXFP8
    rounding itself, which differs from the unquantised expert."""
    g = torch.Generator().manual_seed(15)
    L, I, n = 64, 64, 5
    z = O.mx8_round(torch.randn(n, L, generator=g, dtype=F64))
    Wg = torch.randn(I, L, generator=g, dtype=F64) / 8
    Wv = torch.randn(I, L, generator=g, dtype=F64) / 8
    Wo = torch.eye(L, I, dtype=F64)
    y8 = O.expert_forward(z, Wg, Wv, Wo, 10.0, O.bf16_round, act="mxfp8")
    h = O.bf16_round(O.situ_glu(z @ Wg.T, z @ Wv.T, 10.0))
    assert torch.equal(y8, O.mx8_round(h))
    y = O.expert_forward(z, Wg, Wv, Wo, 10.0, O.bf16_round)
    assert torch.equal(y, h) and not torch.equal(y, y8)


def _e2m1_table():
    """Code -> value of the 16 E2M1 codes, from the OCP table (golden file)."""
    tab = {int(r[0]): float(r[1]) for r in read_golden("e2m1_ocp_mx.txt")}
    return np.array([tab[c] for c in range(16)])


def _pin_e2m1_encode(encode):
    """Brute force over the OCP table: every value maps to the code whose value
    is nearest (magnitudes beyond 6 to +-6), a tie going to the even code; the
    sign is kept, -0 included.  Midpoints of every neighbour pair are in the
    sample, so a wrong tie rule or spacing fails."""
    tab = _e2m1_table()
    mags = tab[:8]
    mids = (mags[:-1] + mags[1:]) / 2
    rng = np.random.default_rng(21)
    v = np.concatenate([mags, mids, np.nextafter(mids, 0), np.nextafter(mids, 10), rng.uniform(0, 9, 5000),
                        [6.5, 7.0, 100.0, 1e300]])
    v = np.concatenate([v, -v])
    got = encode(torch.from_numpy(v))
    for x, c in zip(v, got):
        a = min(abs(x), 6.0)
        d = np.abs(mags - a)
        best = np.flatnonzero(d == d.min())
        want = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert c == (want | (8 if np.signbit(x) else 0)), (x, c)
    assert list(encode(torch.tensor([0.0, -0.0], dtype=F64))) == [0, 8]
    assert np.array_equal(encode(torch.from_numpy(tab[np.r_[0:8, 9:16]])), np.r_[0:8, 9:16])


def test_e2m1_encode_is_the_nearest_code_ties_to_even(O):
    _pin_e2m1_encode(O.e2m1_encode)


def _pin_mx4_scale_rule(quantize):
    """OCP MX v1.0 shared scale of an MXFP4 block, s = floor(log2 max|v|) - 2,
    clamped to the E8M0 range; codes of v / 2^s packed two per byte, the even
    element in the low nibble."""
    def q(block):
        c, s = quantize(torch.tensor([block], dtype=F64))
        return c[0], int(s[0, 0])

    c, s = q([1.0] * 32)                      # s = -2: 1 -> 4, code 6
    assert s == 125 and set(c) == {0x66}
    c, s = q([7.0] + [0.0] * 31)              # s = 0: 7 saturates to 6 (code 7)
    assert s == 127 and c[0] == 0x07 and set(c[1:]) == {0}
    c, s = q([0.0] * 32)                      # all-zero block: the lowest scale
    assert s == 0 and set(c) == {0}
    c, s = q([-3.0, 0.75] + [0.0] * 30)       # max 3 -> s = -1: -6 (code 15), 1.5 (code 3)
    assert s == 126 and c[0] == (3 << 4) | 15
    c, s = q([0.0, 6.0 * 2.0**100] + [0.0] * 30)  # s = 100: 6 in the high nibble
    assert s == 227 and c[0] == 0x70
    c, s = q([2.0**-130] + [0.0] * 31)        # clamped at -127: 2^-130 * 2^127 = 0.125 rounds to 0
    assert s == 0 and set(c) == {0}
    c, s = q([0.2] * 16 + [5.0] * 16)         # s = 0: 0.2 -> 0 (nearest of 0, 0.5), 5 -> 4 (tie, even code 6)
    assert s == 127 and set(c[:8]) == {0} and set(c[8:]) == {0x66}


def test_mx4_scale_rule_closed_forms(O):
    _pin_mx4_scale_rule(O.mx4_quantize)


# Plausible slips, planted in copies of the oracle's encoders on the CPU: each
# must fail the pins above.
def _e2m1_mutant(kind):
    def encode(v):
        v = torch.as_tensor(v).to(F64)
        neg = torch.signbit(v)
        a = torch.clamp(v.abs(), max=4.0 if kind == "saturate_at_4" else 6.0)
        _, ex = torch.frexp(a)
        q = torch.clamp(ex.to(torch.int64) - 1, min=0)
        x = torch.ldexp(a, (1 - q).to(torch.int64))
        units = torch.floor(x + 0.5) if kind == "ties_away" else torch.round(x)
        if kind == "subnormal_spacing":  # below 1 the step taken as 1 instead of 0.5
            units = torch.where(q == 0, 2 * torch.round(x / 2), units)
        carry = (q >= 1) & (units >= 4)
        q = torch.where(carry, q + 1, q)
        units = torch.where(carry, units / 2, units).to(torch.int64)
        code = torch.where(q == 0, units, ((q + 1) << 1) | (units - 2))
        if kind != "sign_dropped":
            code = torch.where(neg, code | 8, code)
        return code.to(torch.uint8).numpy()
    return encode


def _mx4_mutant(kind):
    def quantize(v):
        v = torch.as_tensor(v).to(F64)
        R, K = v.shape
        blocks = v.reshape(R, K // 32, 32)
        amax = blocks.abs().amax(dim=2)
        _, ex = torch.frexp(amax)
        emax = {"emax_1": 1, "emax_3": 3}.get(kind, 2)
        fl = ex.to(torch.int64) - 1
        if kind == "round_log2":
            fl = torch.round(torch.log2(torch.where(amax > 0, amax, torch.ones_like(amax)))).to(torch.int64)
        s = torch.clamp(fl - emax, min=-127, max=127)
        s = torch.where(amax == 0, torch.full_like(s, 0 if kind == "zero_block_scale_1" else -127), s)
        nib = oracle.torch_ref.e2m1_encode(torch.ldexp(blocks, (-s)[:, :, None].expand(R, K // 32, 32)).reshape(R, K))
        lo, hi = (nib[:, 1::2], nib[:, 0::2]) if kind == "nibbles_swapped" else (nib[:, 0::2], nib[:, 1::2])
        return (lo | (hi << 4)).astype(np.uint8), (s + 127).to(torch.uint8).numpy()
    return quantize


@pytest.mark.parametrize("kind", ["ties_away", "saturate_at_4", "subnormal_spacing", "sign_dropped"])
def test_e2m1_pin_catches_a_planted_slip(kind):
    with pytest.raises(AssertionError):
        _pin_e2m1_encode(_e2m1_mutant(kind))


@pytest.mark.parametrize("kind", ["emax_1", "emax_3", "round_log2", "zero_block_scale_1", "nibbles_swapped"])
def test_mx4_pin_catches_a_planted_slip(kind):
    with pytest.raises(AssertionError):
        _pin_mx4_scale_rule(_mx4_mutant(kind))


def test_unmutated_copies_pass_the_pins():
    """The copies the slips are planted in are faithful without a slip."""
    _pin_e2m1_encode(_e2m1_mutant("none"))
    _pin_mx4_scale_rule(_mx4_mutant("none"))


def test_mx4_round_is_the_nearest_block_value_and_idempotent(O):
    """Each element of mx4_round(x) is, brute force, the nearest of the 15
    values +-E2M1 * 2^s of its block to x (ties to the even code), and
    quantising the result again changes nothing."""
    g = torch.Generator().manual_seed(22)
    x = torch.randn(16, 128, generator=g, dtype=F64) * torch.exp2(torch.randint(-20, 20, (16, 4), generator=g)
                                                                   .to(F64)).repeat_interleave(32, dim=1)
    r = O.mx4_round(x)
    assert torch.equal(O.mx4_round(r), r)
    _, s = O.mx4_quantize(x)
    tab = _e2m1_table()
    for i in range(x.shape[0]):
        for k in range(x.shape[1]):
            sc = 2.0 ** (int(s[i, k // 32]) - 127)
            cand = tab * sc
            d = np.abs(cand - x[i, k].item())
            best = np.flatnonzero(d == d.min())
            best = [b for b in best if b % 2 == 0] or list(best)
            assert r[i, k].item() in cand[best], (i, k)


def test_cpp_and_torch_mx4_agree_bit_for_bit():
    x = torch.randn(200, 1024, generator=torch.Generator().manual_seed(23), dtype=F64).to(torch.bfloat16).to(F64)
    x = x * torch.exp2(torch.randint(-40, 40, (200, 1), generator=torch.Generator().manual_seed(24)).to(F64))
    a = oracle.mx4_quantize(x)
    b = oracle.torch_ref.mx4_quantize(x)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_expert_forward_mx4_rounds_both_inputs(O):
    """act="mxfp4": as for MXFP8, with the MXFP4 values of z and of h."""
    g = torch.Generator().manual_seed(25)
    L, I, n = 64, 64, 5
    z = O.mx4_round(torch.randn(n, L, generator=g, dtype=F64))
    Wg = torch.randn(I, L, generator=g, dtype=F64) / 8
    Wv = torch.randn(I, L, generator=g, dtype=F64) / 8
    Wo = torch.eye(L, I, dtype=F64)
    y4 = O.expert_forward(z, Wg, Wv, Wo, 10.0, O.bf16_round, act="mxfp4")
    h = O.bf16_round(O.situ_glu(z @ Wg.T, z @ Wv.T, 10.0))
    assert torch.equal(y4, O.mx4_round(h))
    assert not torch.equal(y4, O.expert_forward(z, Wg, Wv, Wo, 10.0, O.bf16_round, act="mxfp8"))


def test_sigmoid_matches_scipy(O):
    x = torch.linspace(-30, 30, 2001, dtype=F64)
    assert torch.allclose(O.sigmoid(x), torch.from_numpy(scipy.special.expit(x.numpy())), rtol=1e-15, atol=0)


def test_router_orientation(O):
    # W_r = a row permutation: logit e = x[perm[e]]
    H = 7
    perm = [3, 0, 6, 1, 5, 2, 4]
    Wr = torch.zeros(H, H, dtype=F64)
    for e, h in enumerate(perm):
        Wr[e, h] = 1.0
    x = torch.randn(5, H, dtype=F64, generator=torch.Generator().manual_seed(0))
    s = O.router_scores(x, Wr)
    want = torch.from_numpy(scipy.special.expit(x[:, perm].numpy()))
    assert torch.allclose(s, want, rtol=1e-15, atol=0)


def _brute_force_topk(key, k):
    """Best k-subset by total key; among equal totals the lexicographically
    smallest sorted index tuple.  Slots then in (key desc, index asc)."""
    E = len(key)
    best, best_set = None, None
    for sub in itertools.combinations(range(E), k):
        tot = sum(key[i] for i in sub)
        if best is None or tot > best or (tot == best and sub < best_set):
            best, best_set = tot, sub
    return sorted(best_set, key=lambda i: (-key[i], i))


@pytest.mark.parametrize("E,k", [(6, 1), (6, 3), (8, 4), (10, 2), (12, 4)])
def test_select_experts_brute_force(O, E, k):
    rng = np.random.default_rng(E * 100 + k)
    for trial in range(40):
        # quantised values produce exact ties in s + b
        s = rng.integers(1, 8, size=E) / 8.0
        b = rng.integers(-2, 3, size=E) / 8.0
        key = s + b
        idx, p, margin = O.select_experts(torch.tensor(s[None]), torch.tensor(b), k)
        want = _brute_force_topk(list(key), k)
        assert idx[0].tolist() == want
        # mixture weights: unbiased scores renormalised over the chosen set
        assert torch.allclose(p[0], torch.tensor(s[want] / s[want].sum()), rtol=0, atol=1e-15)
        srt = sorted(key, reverse=True)
        assert margin[0].item() == pytest.approx(srt[k - 1] - srt[k]) if k < E else True


def test_mixture_weights_use_unbiased_scores(O):
    s = torch.tensor([[0.9, 0.2, 0.3, 0.1]], dtype=F64)
    b = torch.tensor([-1.0, 0.5, 0.0, 0.0], dtype=F64)  # the bias reorders the selection
    idx, p, _ = O.select_experts(s, b, 2)
    assert idx[0].tolist() == [1, 2]  # keys 0.7, 0.3 beat -0.1 and 0.1
    assert torch.allclose(p[0], torch.tensor([0.2 / 0.5, 0.3 / 0.5], dtype=F64))
    assert abs(p.sum().item() - 1.0) < 1e-15


def test_select_from_f32_scores_uses_fp32_key(O):
    # 0.5 + 2^-30 rounds to 0.5 in fp32: the keys tie there and the lower
    # index wins, although in fp64 the tiny bias decides.
    s2 = np.array([[0.5, 0.5]], np.float32)
    b2 = np.array([0.0, np.float32(2.0**-30)], np.float32)
    idx2, _ = O.select_experts_from_f32_scores(s2, b2, 1)
    assert idx2[0, 0].item() == 0
    idx3, _, _ = O.select_experts(torch.tensor(s2, dtype=F64), torch.tensor(b2, dtype=F64), 1)
    assert idx3[0, 0].item() == 1  # in fp64 the tiny bias decides


def test_permute_invariants_and_library_sort(O):
    rng = np.random.default_rng(5)
    T, E, k = 300, 17, 4
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)])
    counts, offsets, perm_token, inv_perm = O.permute(idx, E)
    assert counts.sum() == T * k and np.all(np.diff(offsets) >= 0) and offsets[-1] == T * k
    assert np.array_equal(np.bincount(idx.ravel(), minlength=E), counts)
    # stable library sort of the flattened expert ids gives the same order
    order = np.argsort(idx.ravel(), kind="stable")
    assert np.array_equal(perm_token, order // k)
    inv = np.empty(T * k, np.int64)
    inv[order] = np.arange(T * k)
    assert np.array_equal(inv_perm, inv)
    for e in range(E):
        seg = perm_token[offsets[e] : offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)
        assert all(e in idx[t] for t in seg)
    # inv_perm o perm = identity on the pairs
    for t in range(T):
        for j in range(k):
            assert perm_token[inv_perm[t * k + j]] == t


# ---------------------------------------------------------------- experts
def test_situ_glu_properties(O):
    g = torch.linspace(-40, 40, 801, dtype=F64)[:, None]
    v = torch.linspace(-40, 40, 161, dtype=F64)[None, :]
    c = 10.0
    h = O.situ_glu(g, v, c)
    assert torch.allclose(O.situ_glu(g, -v, c), -h, rtol=0, atol=0)  # odd in v
    assert h.abs().max() <= c * c
    # c -> infinity gives SwiGLU (library silu)
    big = O.situ_glu(g, v, 1e6)
    sw = torch.nn.functional.silu(g) * v
    assert torch.allclose(big, sw, rtol=1e-8, atol=1e-12)
    # small arguments: 0 <= 1 - h/swiglu <= (g^2 + v^2) / (3 c^2)
    gs = torch.linspace(-2, 2, 41, dtype=F64)[:, None]
    vs = torch.linspace(-2, 2, 41, dtype=F64)[None, :]
    hs = O.situ_glu(gs, vs, c)
    sws = torch.nn.functional.silu(gs) * vs
    mask = sws.abs() > 1e-12
    rel = 1.0 - hs[mask] / sws[mask]
    bound = ((gs**2 + vs**2) / (3 * c * c)).expand_as(hs)[mask]
    assert (rel >= -1e-15).all() and (rel <= bound + 1e-15).all()
    # the cap binds: large positive g, v -> c^2
    assert abs(O.situ_glu(torch.tensor(1e3, dtype=F64), torch.tensor(1e3, dtype=F64), c).item() - c * c) < 1e-9


def test_expert_forward_orientation(O):
    # permutation weights: g = z[pg], v = z[pv], y = h[po]
    L = I = 6
    rng = np.random.default_rng(0)
    pg, pv, po = rng.permutation(L), rng.permutation(L), rng.permutation(I)

    def P(p):
        m = torch.zeros(len(p), len(p), dtype=F64)
        m[torch.arange(len(p)), torch.as_tensor(p)] = 1.0
        return m

    z = torch.randn(3, L, dtype=F64, generator=torch.Generator().manual_seed(2))
    y = O.expert_forward(z, P(pg), P(pv), P(po), 10.0, lambda t: t)
    h = O.situ_glu(z[:, pg], z[:, pv], 10.0)
    assert torch.equal(y, h[:, po])
    # the stored h is rounded before the down projection
    yb = O.expert_forward(z, P(pg), P(pv), P(po), 10.0, O.bf16_round)
    assert torch.equal(yb, O.bf16_round(h)[:, po])


def test_shared_experts_orientation(O):
    # two shared experts with permutation weights on a square hidden size
    H = 5
    rng = np.random.default_rng(9)
    ps = [(rng.permutation(H), rng.permutation(H), rng.permutation(H)) for _ in range(2)]

    def P(p):
        m = torch.zeros(len(p), len(p), dtype=F64)
        m[torch.arange(len(p)), torch.as_tensor(p)] = 1.0
        return m

    Wsg = torch.stack([P(a) for a, _, _ in ps])
    Wsv = torch.stack([P(b) for _, b, _ in ps])
    Wso = torch.stack([P(c) for _, _, c in ps])
    x = torch.randn(4, H, dtype=F64, generator=torch.Generator().manual_seed(3))
    y = O.shared_experts(x, Wsg, Wsv, Wso, 10.0, lambda t: t)
    want = sum(O.situ_glu(x[:, a], x[:, b], 10.0)[:, c] for a, b, c in ps)
    assert torch.allclose(y, want, rtol=1e-15, atol=1e-15)


def test_combine_one_hot_and_linear(O):
    y = torch.randn(4, 3, 5, dtype=F64, generator=torch.Generator().manual_seed(4))
    for j in range(3):
        p = torch.zeros(4, 3, dtype=F64)
        p[:, j] = 1.0
        assert torch.equal(O.combine(y, p), y[:, j])
    p = torch.rand(4, 3, dtype=F64, generator=torch.Generator().manual_seed(5))
    want = torch.einsum("tj,tjl->tl", p, y)
    assert torch.allclose(O.combine(y, p), want, rtol=1e-14, atol=1e-15)


def test_rms_norm_closed_forms(O):
    gam = torch.ones(8, dtype=F64)
    for a in (1e-3, 0.5, 7.0, -3.0):
        u = torch.full((1, 8), a, dtype=F64)
        n = O.rms_norm(u, gam, 1e-6)
        assert torch.allclose(n, torch.full((1, 8), a / math.sqrt(a * a + 1e-6), dtype=F64), rtol=1e-15)
    u = torch.randn(6, 64, dtype=F64, generator=torch.Generator().manual_seed(7))
    n = O.rms_norm(u, torch.ones(64, dtype=F64), 0.0)
    assert torch.allclose(n, O.rms_norm(u * 123.0, torch.ones(64, dtype=F64), 0.0), rtol=1e-14)
    assert torch.allclose((n * n).mean(dim=1), torch.ones(6, dtype=F64), rtol=1e-14)
    g = torch.randn(64, dtype=F64, generator=torch.Generator().manual_seed(8))
    assert torch.allclose(O.rms_norm(u, g, 0.0), g[None] * n, rtol=1e-14)
    ms = (u * u).mean(dim=1)
    n1 = O.rms_norm(u, torch.ones(64, dtype=F64), 0.25)
    assert torch.allclose((n1 * n1).mean(dim=1), ms / (ms + 0.25), rtol=1e-14)


# ---------------------------------------------------------------- whole layer
def _tiny_weights(cfg):
    return oin.all_weights(cfg)


def test_identical_experts_reduce_to_dense_glu(O):
    """Zero bias and identical experts: the routed mixture is one dense GLU
    (the renormalised weights sum to one), for any routing."""
    cfg = gen.CONFIGS["tiny"]
    w = _tiny_weights(cfg)
    w["bias"] = torch.zeros(cfg.E, dtype=F64)
    for name in ("Wg", "Wv", "Wo"):
        w[name] = w[name][:1].expand_as(w[name]).clone()
    x = oin.x_rows(cfg, range(cfg.T))
    out = O.layer_forward(cfg, w, x)
    rnd = O.storage_round(cfg.act)
    z = rnd(x @ w["Wdown"].T)
    u_dense = O.expert_forward(z, w["Wg"][0], w["Wv"][0], w["Wo"][0], cfg.situ_c, rnd)
    assert torch.allclose(out["u"], u_dense, rtol=1e-12, atol=1e-13)
    n = rnd(O.rms_norm(u_dense, w["gamma"], cfg.rms_eps))
    y = O.shared_experts(x, w["Wsg"], w["Wsv"], w["Wso"], cfg.situ_c, rnd) + n @ w["Wup"].T
    assert torch.allclose(out["y"], y, rtol=1e-12, atol=1e-12)


def test_latent_projection_orientation(O):
    """W_down = [I | 0] selects the first L hidden coordinates of x."""
    cfg = gen.CONFIGS["tiny"]
    w = _tiny_weights(cfg)
    w["Wdown"] = torch.zeros(cfg.L, cfg.H, dtype=F64)
    w["Wdown"][torch.arange(cfg.L), torch.arange(cfg.L)] = 1.0
    x = oin.x_rows(cfg, range(8))
    out = O.layer_forward(cfg, w, x)
    assert torch.equal(out["z"], x[:, : cfg.L])


def test_top1_routing_uses_the_selected_expert_only(O):
    """k = 1: p = 1 and u is the chosen expert's output."""
    cfg = gen.CONFIGS["tiny"].with_(k=1)
    w = _tiny_weights(cfg)
    x = oin.x_rows(cfg, range(16))
    out = O.layer_forward(cfg, w, x)
    assert torch.equal(out["p"], torch.ones(16, 1, dtype=F64))
    rnd = O.storage_round(cfg.act)
    for t in range(16):
        e = out["idx"][t, 0].item()
        ye = O.expert_forward(out["z"][t : t + 1], w["Wg"][e], w["Wv"][e], w["Wo"][e], cfg.situ_c, rnd)
        assert torch.allclose(out["u"][t : t + 1], ye, rtol=1e-14, atol=1e-15)


def test_streamed_forward_equals_in_memory_forward(O):
    cfg = gen.CONFIGS["tiny"]
    w = _tiny_weights(cfg)
    x = oin.x_rows(cfg, range(cfg.T))
    a = O.layer_forward(cfg, w, x)
    b = O.layer_forward_streamed(cfg, w, x, lambda e: (w["Wg"][e], w["Wv"][e], w["Wo"][e]))
    assert torch.equal(a["idx"], b["idx"]) and torch.allclose(a["y"], b["y"], rtol=1e-14, atol=1e-14)


def test_storage_rounding_points(O):
    """bf16 workloads: z, n (and h, shared h) are bf16 values; u, y are not."""
    cfg = gen.CONFIGS["mid"].with_(T=16)
    w = oin.dense_weights(cfg)
    x = oin.x_rows(cfg, range(16))
    out = O.layer_forward_streamed(cfg, w, x, lambda e: oin.expert_weights(cfg, e))
    assert torch.equal(O.bf16_round(out["z"]), out["z"])
    assert torch.equal(O.bf16_round(out["n"]), out["n"])
    assert not torch.equal(O.bf16_round(out["u"]), out["u"])
    assert not torch.equal(O.bf16_round(out["y"]), out["y"])


def test_k3_parameter_count_matches_the_published_total():
    """3-matrix GLU experts in the latent space, shared intermediate 3072 and
    93 MoE layers give 2.770T parameters, within 0.5% of the printed 2.78T."""
    t = {r[0]: float(r[1]) for r in read_golden("k3_model_table.txt")}
    cfg = gen.CONFIGS["prefill"]
    assert (cfg.H, cfg.L, cfg.E, cfg.k, cfg.I, cfg.S) == (
        t["hidden"], t["latent"], t["routed_experts"], t["top_k"], t["expert_intermediate"], t["shared_experts"])
    per_layer = cfg.E * 3 * cfg.L * cfg.I + cfg.S * 3 * cfg.H * cfg.Is + 2 * cfg.H * cfg.L + cfg.E * cfg.H
    total = per_layer * t["layers"]
    assert abs(total / t["total_params"] - 1.0) < 0.005
    active = (cfg.k * 3 * cfg.L * cfg.I + cfg.S * 3 * cfg.H * cfg.Is + 2 * cfg.H * cfg.L + cfg.E * cfg.H) * t["layers"]
    assert active < t["active_params"]  # the rest is attention and embeddings


# ---------------------------------------------------------------- the two restatements
def test_cpp_oracle_reads_raw_weight_bits_exactly():
    """The C++ oracle decodes bf16 bit patterns and MXFP4 (codes, scales)
    itself; the results equal those from exactly decoded fp64 weights."""
    for name in ("mid", "mxfp4-small"):
        cfg = gen.CONFIGS[name]
        dense = oin.dense_weights(cfg)
        x = oin.x_rows(cfg, range(8))
        a = oracle.layer_forward_streamed(cfg, dense, x, lambda e: oin.expert_weights_raw(cfg, e))
        b = oracle.layer_forward_streamed(cfg, dense, x, lambda e: oin.expert_weights(cfg, e))
        for key in ("s", "idx", "p", "z", "u", "n", "y"):
            assert torch.equal(a[key], b[key]), key


def test_cpp_and_torch_oracles_agree_on_a_bf16_layer():
    """Independent restatements (C++ loops, PyTorch ops) of the same layer:
    identical selections, outputs equal up to fp64 summation order (and the
    bf16 storage roundings that order can flip, one step at most)."""
    cfg = gen.CONFIGS["mid"]
    dense = oin.dense_weights(cfg)
    x = oin.x_rows(cfg, range(24))
    a = oracle.layer_forward_streamed(cfg, dense, x, lambda e: oin.expert_weights_raw(cfg, e))
    b = oracle.torch_ref.layer_forward_streamed(cfg, dense, x, lambda e: oin.expert_weights(cfg, e))
    assert torch.equal(a["idx"], b["idx"])
    assert torch.allclose(a["s"], b["s"], rtol=1e-13, atol=0)
    assert torch.allclose(a["p"], b["p"], rtol=1e-13, atol=0)
    for key in ("u", "y"):
        rms = b[key].pow(2).mean().sqrt()
        assert ((a[key] - b[key]).abs().max() / rms).item() < 1e-4, key


def test_cpp_oracle_thread_count_is_the_host_core_count():
    import os

    assert oracle.num_threads() == (int(os.environ["MOE_ORACLE_THREADS"]) if os.environ.get("MOE_ORACLE_THREADS")
                                    else os.cpu_count())
