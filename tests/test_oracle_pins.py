"""Pins of the CPU oracle to facts outside itself (no GPU needed).

Each test checks the oracle against something it does not compute itself: the number formats
against torch's own casts, exact sums against math.fsum, the RMSNorm of the "MoE update" page
against closed forms, the router reading against constructed cases, and the whole layer
against special cases that reduce to a dense SwiGLU MLP evaluated here with torch matmuls.
Shapes are deliberately non-square (d != inter) and W1 != W3, so a transposed operand or
swapped projection fails.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synthetic
from oracle import bf16_bits_to_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def to_bf16_bits(v64: np.ndarray) -> np.ndarray:
    return bits(torch.from_numpy(np.asarray(v64, np.float64)).to(torch.bfloat16))


def ulp_bf16(v):
    v = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(v, 2.0 ** -126)))
    return 2.0 ** (e - 7)


# ----------------------------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------------------------
def test_bf16_round_to_nearest_even_matches_torch():
    g = torch.Generator().manual_seed(1)
    v = torch.randn(20000, generator=g, dtype=torch.float64) * torch.exp2(torch.randint(-140, 120, (20000,), generator=g).double())
    v32 = v.float()
    # halfway cases: bf16 value + half quantum (exactly representable in fp32)
    base = torch.randn(2000, generator=g).to(torch.bfloat16).float()
    half = base + base.abs() * 0 + torch.ldexp(torch.ones(2000), torch.frexp(base)[1] - 9)
    v32 = torch.cat([v32, half, torch.tensor([0.0, -0.0, 3.0e38, -3.4e38, 1e-40, -1e-45])])
    want = bits(v32.to(torch.bfloat16))
    got = oracle.f64_to_bf16(v32.double().numpy())
    assert np.array_equal(got, want)
    back = oracle.bf16_to_f64(want[:500])
    assert np.array_equal(back, v32.to(torch.bfloat16).double().numpy()[:500])


def test_e4m3_all_codes_and_rounding_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = oracle.e4m3_to_f64(codes)
    finite = ~np.isnan(want)
    assert np.array_equal(np.isnan(got), ~finite)
    assert np.array_equal(got[finite], want[finite])
    # rounding: random values inside the finite range plus every midpoint between neighbours
    g = torch.Generator().manual_seed(2)
    v = (torch.rand(20000, generator=g, dtype=torch.float64) * 2 - 1) * torch.exp2(torch.randint(-12, 9, (20000,), generator=g).double())
    v = v.clamp(-448, 448)
    fin = np.sort(np.unique(want[finite]))
    mids = (fin[:-1] + fin[1:]) / 2
    v = torch.cat([v, torch.from_numpy(mids)]).float()
    want_c = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got_c = oracle.f64_to_e4m3(v.double().numpy())
    # +0 / -0 share value 0: compare decoded values and signs of non-zeros
    assert np.array_equal(oracle.e4m3_to_f64(got_c), oracle.e4m3_to_f64(want_c))
    # saturation (satfinite) beyond the largest finite value, per the OCP FP8 definition
    assert list(oracle.f64_to_e4m3([449.0, 1e6, -470.0])) == [0x7E, 0x7E, 0xFE]


def test_exact_sum_of_squares_matches_fsum():
    g = torch.Generator().manual_seed(3)
    for n in (1, 7, 256, 7168):
        s = (torch.randn(n, generator=g) * torch.exp2(torch.randint(-30, 30, (n,), generator=g).float())).numpy()
        ss = math.fsum(float(x) * float(x) for x in s)     # exact sum, correctly rounded to double
        assert oracle.mean_square(s) == np.float32(ss / n)
    # order independence
    s = torch.randn(7168, generator=g).numpy()
    assert oracle.mean_square(s) == oracle.mean_square(s[::-1].copy())


# ----------------------------------------------------------------------------------------------
# RMSNorm ("MoE update" page, RMSNorm excerpt): closed forms
# ----------------------------------------------------------------------------------------------
@pytest.mark.parametrize("c", [1.0, -2.5, 0.001, 37.0])
def test_norm_constant_input_closed_form(c):
    d = 256
    half = torch.full((d,), c / 2, dtype=torch.float64)
    x = half.to(torch.bfloat16)
    r = (torch.full((d,), c, dtype=torch.float64) - x.double()).to(torch.bfloat16)
    s = (x.float() + r.float()).double()                     # the fp32 sum is exact here
    gain = torch.linspace(0.5, 1.5, d).float()
    xn, ro, x64, x32 = oracle.norm_token(bits(x), bits(r), gain.numpy())
    # eps is float32 1e-6 in the page's module
    want64 = gain.double().numpy() * s.numpy() / np.sqrt(s.numpy() ** 2 + float(np.float32(1e-6)))
    assert np.allclose(x64, want64, rtol=1e-12, atol=0)
    got = bf16_bits_to_f64(xn)
    assert np.all(np.abs(got - want64) <= ulp_bf16(want64))   # one bf16 rounding away
    assert np.array_equal(ro, bits(s.to(torch.bfloat16)))


def test_norm_one_hot_and_zero_closed_forms():
    d = 7168
    a = 3.0
    x = torch.zeros(d, dtype=torch.bfloat16)
    x[123] = a
    r = torch.zeros(d, dtype=torch.bfloat16)
    g = np.ones(d, np.float32) * 2.0
    xn, ro, x64, x32 = oracle.norm_token(bits(x), bits(r), g)
    want = 2.0 * a / math.sqrt(a * a / d + float(np.float32(1e-6)))
    assert abs(x64[123] - want) <= 1e-12 * want
    assert abs(bf16_bits_to_f64(xn[123:124])[0] - want) <= ulp_bf16(want)
    assert np.all(bf16_bits_to_f64(np.delete(xn, 123)) == 0)
    # zero input: eps keeps the result finite and zero
    z = torch.zeros(d, dtype=torch.bfloat16)
    xn, ro, x64, _ = oracle.norm_token(bits(z), bits(z), g)
    assert np.all(bf16_bits_to_f64(xn) == 0) and np.all(np.isfinite(x64))
    # no residual: s = x alone, and the residual add matters when present
    xn2, _, x64b, _ = oracle.norm_token(bits(x), None, g)
    assert abs(x64b[123] - want) <= 1e-12 * want
    r2 = torch.zeros(d, dtype=torch.bfloat16)
    r2[5] = 1.0
    _, _, x64c, _ = oracle.norm_token(bits(x), bits(r2), g)
    assert x64c[5] != 0 and abs(x64c[123] - want) > 1e-6


def test_norm_residual_out_matches_torch_add():
    g = torch.Generator().manual_seed(4)
    x = torch.randn(2048, generator=g).to(torch.bfloat16)
    r = (torch.randn(2048, generator=g) * 2).to(torch.bfloat16)
    _, ro, x64, x32 = oracle.norm_token(bits(x), bits(r), np.ones(2048, np.float32))
    assert np.array_equal(ro, bits((x.float() + r.float()).to(torch.bfloat16)))
    assert np.allclose(x32, x64, rtol=1e-6)


# ----------------------------------------------------------------------------------------------
# FP8 activation quant
# ----------------------------------------------------------------------------------------------
def test_act_quant_matches_torch_and_bounds():
    g = torch.Generator().manual_seed(5)
    v = torch.randn(1024, generator=g).to(torch.bfloat16).double()
    v[256:384] = 0.0                                    # an all-zero group
    q, sc, dq = oracle.act_quant(v.numpy())
    vv = v.float().view(8, 128)
    amax = vv.abs().amax(1)
    want_sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    assert np.array_equal(sc, want_sc.numpy())
    want_q = (vv / want_sc[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).view(-1).numpy()
    want_q = np.where(np.repeat(amax.numpy() > 0, 128), want_q, 0)
    assert np.array_equal(oracle.e4m3_to_f64(q), oracle.e4m3_to_f64(want_q))
    # the group maximum lands exactly on +-448; error at most half an e4m3 step of the value
    for gi in range(8):
        if amax[gi] > 0:
            j = int(torch.argmax(vv[gi].abs()))
            assert abs(oracle.e4m3_to_f64([q[gi * 128 + j]])[0]) == 448.0
    err = np.abs(dq - v.numpy())
    bound = np.maximum(np.abs(v.numpy()) * 2.0 ** -4, np.repeat(sc, 128) * 2.0 ** -10)
    assert np.all(err <= bound * (1 + 1e-12))
    assert np.all(dq[256:384] == 0)


# ----------------------------------------------------------------------------------------------
# router (reading: sigmoid scores, top-k, lower index wins ties, normalised weights)
# ----------------------------------------------------------------------------------------------
def test_gate_zero_weights_tie_break():
    d, E, k = 256, 8, 3
    xn = torch.randn(d).to(torch.bfloat16)
    sc, idx, w, m = oracle.gate_token(bits(xn), bits(torch.zeros(E, d, dtype=torch.bfloat16)), None, k)
    assert np.all(sc == 0.5)
    assert list(idx) == [0, 1, 2]
    assert np.allclose(w, 1.0 / k, rtol=0, atol=1e-15)
    assert m == 0.0


def test_gate_bias_selects_sigmoid_normalised():
    d, E, k = 256, 8, 2
    xn = torch.randn(d).to(torch.bfloat16)
    bias = np.array([0.0, -1.0, 2.0, 0.5, 3.0, -4.0, 1.0, 0.0], np.float32)
    sc, idx, w, m = oracle.gate_token(bits(xn), bits(torch.zeros(E, d, dtype=torch.bfloat16)), bias, k)
    s = 1.0 / (1.0 + np.exp(-bias.astype(np.float64)))
    assert list(idx) == [4, 2]
    assert np.allclose(w, s[[4, 2]] / s[[4, 2]].sum(), rtol=1e-15)
    assert abs(m - (s[2] - s[6])) < 1e-15


def test_gate_topk_equals_full_sort_brute_force():
    shape = synthetic.CONFIGS["C1"]
    inp = synthetic.generate(shape, with_experts=False)
    for t in range(16):
        xn, _, _, _ = oracle.norm_token(bits(inp["x"][t]), bits(inp["residual"][t]), inp["norm_w"].numpy())
        sc, idx, w, m = oracle.gate_token(xn, bits(inp["gate_w"]), None, shape.k)
        z = bf16_bits_to_f64(bits(inp["gate_w"])) @ bf16_bits_to_f64(xn)
        s = 1.0 / (1.0 + np.exp(-z))
        order = np.lexsort((np.arange(shape.E), -s))     # score desc, index asc
        assert list(idx) == list(order[:shape.k])
        assert np.allclose(sc, s, rtol=1e-13)
        assert abs(w.sum() - 1) < 1e-14


# ----------------------------------------------------------------------------------------------
# the whole layer: special cases that reduce to a dense SwiGLU MLP
# ----------------------------------------------------------------------------------------------
def _dequant(w, s):
    """block-scaled e4m3 [rows, cols] -> float64, by expanding the scale grid (independent path)."""
    v = torch.from_numpy(np.asarray(w)).view(torch.float8_e4m3fn).double()
    ss = torch.from_numpy(np.asarray(s, np.float32)).double()
    ss = ss.repeat_interleave(128, 0)[: v.shape[0]].repeat_interleave(128, 1)[:, : v.shape[1]]
    return v * ss


def _w(t, s=None):
    t = t.cpu()
    if t.dtype == torch.uint8:
        return _dequant(t.numpy(), s.cpu().numpy())
    return t.double()


def _rb(v):  # round to bf16 and back (torch's cast)
    return v.to(torch.bfloat16).double()


def _textbook_swiglu(a, w1, w3, w2):
    """w2(silu(w1 a) * w3 a), with the Linear outputs rounded to bf16 as the expert excerpt implies and
    silu * mul in float32 (silu correctly rounded to float32, float32 product)."""
    g = _rb(w1 @ a)
    u = _rb(w3 @ a)
    h = (torch.nn.functional.silu(g).float() * u.float()).to(torch.bfloat16).double()
    return _rb(w2 @ h)


def _close(got, want, terms):
    """got (bf16) equals the rounded sum of ``terms``, allowing one bf16 step on each term (the
    expert outputs are themselves bf16 roundings of float64 sums taken in another order) and
    one on the result."""
    tol = ulp_bf16(want.numpy()) + sum(ulp_bf16(t.numpy()) for t in terms)
    err = (got - want).abs().numpy()
    assert np.all(err <= tol), float((err / tol).max())
    # and most elements agree exactly after rounding
    assert np.mean(got.numpy() == want.to(torch.bfloat16).double().numpy()) > 0.95


def _small_shape(E, k, wtype="bf16", d=256, I=384, Is=128):
    return synthetic.MoEShape("pin", T=24, d=d, I=I, E=E, k=k, n_shared=1, shared_inter=Is, wtype=wtype, seed=11)


def _layer(shape, **over):
    inp = synthetic.generate(shape)
    inp.update(over)
    return inp


def _xn_all(o):
    r = o.forward(route_only=True)
    return torch.from_numpy(bf16_bits_to_f64(r["xn"]))


@pytest.mark.parametrize("wtype", ["bf16", "fp8"])
def test_single_expert_is_textbook_swiglu_plus_shared(wtype):
    shape = _small_shape(E=1, k=1, wtype=wtype)
    inp = _layer(shape)
    o = oracle.Oracle(shape, inp, act_fp8=False)
    r = o.forward()
    xn = _xn_all(o)
    w1, w3, w2 = _w(inp["w1"][0], inp["s1"] if inp["s1"] is None else inp["s1"][0]), \
        _w(inp["w3"][0], None if inp["s3"] is None else inp["s3"][0]), \
        _w(inp["w2"][0], None if inp["s2"] is None else inp["s2"][0])
    sw1, sw3, sw2 = _w(inp["sw1"], inp["ss1"]), _w(inp["sw3"], inp["ss3"]), _w(inp["sw2"], inp["ss2"])
    ye = torch.stack([_textbook_swiglu(a, w1, w3, w2) for a in xn])
    ys = torch.stack([_textbook_swiglu(a, sw1, sw3, sw2) for a in xn])
    got = torch.from_numpy(bf16_bits_to_f64(r["out"]))
    _close(got, ye + ys, [ye, ys])
    assert np.all(r["idx"] == 0) and np.allclose(r["w"], 1.0)


def test_k_equals_E_with_zero_gate_is_dense_mean():
    shape = _small_shape(E=4, k=4)
    inp = _layer(shape, gate_w=torch.zeros(4, 256, dtype=torch.bfloat16))
    o = oracle.Oracle(shape, inp)
    r = o.forward()
    xn = _xn_all(o)
    terms = [torch.stack([_textbook_swiglu(a, _w(inp["w1"][e]), _w(inp["w3"][e]), _w(inp["w2"][e])) for a in xn]) / 4
             for e in range(4)]
    terms.append(torch.stack([_textbook_swiglu(a, _w(inp["sw1"]), _w(inp["sw3"]), _w(inp["sw2"])) for a in xn]))
    got = torch.from_numpy(bf16_bits_to_f64(r["out"]))
    _close(got, sum(terms), terms)
    assert np.all(r["idx"] == np.arange(4)) and np.allclose(r["w"], 0.25)


@pytest.mark.parametrize("wtype", ["bf16", "fp8"])
def test_zero_routed_weights_gives_shared_only(wtype):
    shape = _small_shape(E=6, k=2, wtype=wtype)
    inp = _layer(shape)
    inp["w2"] = torch.zeros_like(inp["w2"])
    o = oracle.Oracle(shape, inp, act_fp8=False)
    r = o.forward()
    xn = _xn_all(o)
    want = torch.stack([_textbook_swiglu(a, _w(inp["sw1"], inp["ss1"]), _w(inp["sw3"], inp["ss3"]),
                                         _w(inp["sw2"], inp["ss2"])) for a in xn])
    got = torch.from_numpy(bf16_bits_to_f64(r["out"]))
    _close(got, want, [want])


def test_identical_experts_make_routing_irrelevant():
    shape = _small_shape(E=5, k=2)
    inp = _layer(shape)
    for n in ("w1", "w3", "w2"):
        inp[n] = inp[n][:1].expand_as(inp[n]).contiguous()
    o1 = oracle.Oracle(shape, inp).forward()
    inp2 = dict(inp)
    inp2["gate_w"] = (-inp["gate_w"].float()).to(torch.bfloat16)
    o2 = oracle.Oracle(shape, inp2).forward()
    assert not np.array_equal(np.sort(o1["idx"], 1), np.sort(o2["idx"], 1))
    a = bf16_bits_to_f64(o1["out"])
    b = bf16_bits_to_f64(o2["out"])
    assert np.all(np.abs(a - b) <= 2 * ulp_bf16(np.maximum(np.abs(a), np.abs(b))) + 1e-12)  # + exact cancellations
    assert np.mean(a == b) > 0.9     # the rest sit on exact bf16 midpoints of y + y_shared


def test_token_permutation_equivariance():
    shape = _small_shape(E=6, k=2, wtype="fp8")
    inp = _layer(shape)
    perm = torch.randperm(shape.T, generator=torch.Generator().manual_seed(9))
    inp_p = dict(inp)
    inp_p["x"] = inp["x"][perm].contiguous()
    inp_p["residual"] = inp["residual"][perm].contiguous()
    for act in (False, True):
        a = oracle.Oracle(shape, inp, act_fp8=act).forward()
        b = oracle.Oracle(shape, inp_p, act_fp8=act).forward()
        assert np.array_equal(a["out"][perm.numpy()], b["out"])
        assert np.array_equal(a["idx"][perm.numpy()], b["idx"])


def test_fp8_activation_mode_close_to_bf16_mode():
    shape = _small_shape(E=6, k=2, wtype="fp8")
    inp = _layer(shape)
    a = bf16_bits_to_f64(oracle.Oracle(shape, inp, act_fp8=False).forward()["out"])
    b = bf16_bits_to_f64(oracle.Oracle(shape, inp, act_fp8=True).forward()["out"])
    rel = np.sqrt(np.mean((a - b) ** 2)) / np.sqrt(np.mean(a ** 2))
    assert 1e-4 < rel < 0.1          # quant noise present but bounded


def test_parameter_accounting_from_pages():
    gold = json.load(open(os.path.join(GOLDEN, "param_counts.json")))
    d, I, E = gold["dim"], gold["moe_inter_dim"], gold["n_routed_experts"]
    # 256 routed + 1 shared SwiGLU (3 matrices each), the [E, d] router weight and E more router
    # parameters (read as a per-expert bias)
    assert 3 * d * I * (E + gold["n_shared_swiglus"]) + E * d + E == gold["moe_params_per_block"]
    assert d * I == gold["w1_params_per_expert"]
    assert d * I * E == gold["w1_params_all_routed"]
    assert 2 * d == gold["rmsnorm_params_per_block"]
    assert round(gold["moe_params_per_block"] / 2 ** 30, 1) == gold["moe_fp8_gib_per_block_rounded"]
    s = synthetic.CONFIGS["C3"]
    assert (s.d, s.I, s.E, s.Is) == (d, I, E, I)


@pytest.mark.parametrize("wtype", ["bf16", "fp8"])
def test_dense_block_is_textbook_swiglu_and_matches_the_single_expert_route(wtype):
    """A dense block ("MoE update" page, Block excerpt: MLP(dim, inter_dim) in the first blocks) has
    no router: out = MLP(ffn_norm(x)).  Pinned to the SwiGLU evaluated here with torch matmuls, and
    bit-for-bit to the routed path with one expert, top-1 (weight exactly 1) holding the same MLP."""
    d, Is = 256, 384
    dense = synthetic.MoEShape("pin-dense", T=24, d=d, I=128, E=0, k=0, n_shared=1, shared_inter=Is,
                               wtype=wtype, seed=12)
    inp = _layer(dense)
    assert inp["gate_w"] is None and inp["w1"] is None
    o = oracle.Oracle(dense, inp, act_fp8=False)
    r = o.forward()
    assert r["idx"].shape == (24, 0) and np.all(np.isinf(r["margin"]))
    xn = _xn_all(o)
    y = torch.stack([_textbook_swiglu(a, _w(inp["sw1"], inp["ss1"]), _w(inp["sw3"], inp["ss3"]),
                                      _w(inp["sw2"], inp["ss2"])) for a in xn])
    _close(torch.from_numpy(bf16_bits_to_f64(r["out"])), y, [y])
    # the same MLP as the only routed expert, no shared expert, in both activation modes
    routed = synthetic.MoEShape("pin-dense-routed", T=24, d=d, I=Is, E=1, k=1, n_shared=0, shared_inter=0,
                                wtype=wtype, seed=12)
    rin = dict(inp, gate_w=torch.zeros(1, d, dtype=torch.bfloat16), w1=inp["sw1"][None], w3=inp["sw3"][None],
               w2=inp["sw2"][None], s1=None if inp["ss1"] is None else inp["ss1"][None],
               s3=None if inp["ss3"] is None else inp["ss3"][None], s2=None if inp["ss2"] is None else inp["ss2"][None],
               sw1=None, sw3=None, sw2=None, ss1=None, ss3=None, ss2=None)
    for act8 in ([False, True] if wtype == "fp8" else [False]):
        a = oracle.Oracle(dense, inp, act_fp8=act8).forward()
        b = oracle.Oracle(routed, rin, act_fp8=act8).forward()
        assert np.array_equal(a["out"], b["out"]) and np.array_equal(a["residual_out"], b["residual_out"])
