"""Pins for the fp64 oracle: checks that do not reuse the oracle's code.

Each pin takes an ``oracle.Oracle`` and raises AssertionError when it disagrees with
what the pages and the mathematics fix:
  - exact rational arithmetic (Python ``fractions``) for the quantizer,
  - closed forms (uniform router, a softmax with a known value, zero weights,
    one-hot activations, exact scaling by 2),
  - special cases that reduce to library routines (a MoE whose two experts are
    identical is one dense SwiGLU MLP, computed with torch's silu and matmul),
  - brute force on tiny inputs (every expert evaluated densely, gated by a
    numpy argsort of numpy logits),
  - invariants (two distinct experts per token, weights in (0, 1] summing to at
    most 1, |w - q*s| <= s/2).
``test_oracle_pins.py`` runs them on the oracle; ``test_oracle_mutants.py`` runs
them on deliberately broken copies of the oracle and expects each copy to fail.
"""
from fractions import Fraction

import numpy as np
import torch

import synth

# ------------------------------------------------------------------ helpers


def f32_nearest(fr: Fraction) -> float:
    """The fp32 value nearest to a positive rational (ties to even), by integer arithmetic."""
    assert fr > 0
    e = fr.numerator.bit_length() - fr.denominator.bit_length()
    while fr >= Fraction(2) ** (e + 1):
        e += 1
    while fr < Fraction(2) ** e:
        e -= 1
    assert -126 <= e <= 127, "outside fp32's normal range"
    m = round(fr / Fraction(2) ** (e - 23))  # round() on a Fraction: nearest, ties to even
    v = float(m) * 2.0 ** (e - 23)
    assert float(np.float32(v)) == v
    return v


def bf16_bits(values) -> np.ndarray:
    """bf16 bit patterns of values that are exactly representable in bf16."""
    f = np.asarray(values, dtype=np.float32)
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(synth.bf16_bits_to_f32(bits), f), "value not exact in bf16"
    return bits


def random_bf16(rng, shape, std):
    return synth.f32_to_bf16_bits((rng.standard_normal(shape) * std).astype(np.float32))


def dequant(q, s):
    return q.astype(np.float64) * s.astype(np.float64)[..., None]


def swiglu_torch(x, w1, w3, w2):
    """Dense SwiGLU MLP with torch's own silu and matmul, fp64: W2 (silu(W1 x) * W3 x)."""
    x = torch.as_tensor(x, dtype=torch.float64)
    w1, w3, w2 = (torch.as_tensor(a, dtype=torch.float64) for a in (w1, w3, w2))
    h = torch.nn.functional.silu(x @ w1.T) * (x @ w3.T)
    return (h @ w2.T).numpy(), h.numpy()


def tiny_layer(rng, T=5, d=32, F=48, E=16, wstd=0.05, rstd=0.3):
    """A small random layer built directly as int8 codes and fp32 scales, so that the forward
    pins do not depend on the quantizer under test."""
    x = random_bf16(rng, (T, d), 1.0)
    wr = (rng.standard_normal((E, d)) * rstd).astype(np.float32)
    q1 = rng.integers(-127, 128, (E, F, d), dtype=np.int8)
    q3 = rng.integers(-127, 128, (E, F, d), dtype=np.int8)
    q2 = rng.integers(-127, 128, (E, d, F), dtype=np.int8)
    s1 = (rng.uniform(0.5, 1.5, (E, F)) * wstd / 127).astype(np.float32)
    s3 = (rng.uniform(0.5, 1.5, (E, F)) * wstd / 127).astype(np.float32)
    s2 = (rng.uniform(0.5, 1.5, (E, d)) * wstd / 127).astype(np.float32)
    return dict(x=x, wr=wr, q1=q1, s1=s1, q3=q3, s3=s3, q2=q2, s2=s2)


def fwd(orc, L, bias=None, **kw):
    return orc.moe_forward(L["x"], L["wr"], bias, L["q1"], L["s1"], L["q3"], L["s3"], L["q2"], L["s2"], **kw)


# ----------------------------------------------------------- quantization


def pin_quantize_exact_rational(orc):
    rng = np.random.default_rng(11)
    w = random_bf16(rng, (12, 40), 0.02)
    w[3, 7] = bf16_bits([0.90625])[0]      # an outlier row
    w[5, :] = random_bf16(rng, (40,), 3e-5)  # a row of tiny values
    q, s = orc.quantize(w)
    wf = synth.bf16_bits_to_f32(w)
    for r in range(w.shape[0]):
        amax = max(abs(Fraction(float(v))) for v in wf[r])
        s_exact = f32_nearest(amax / 127)
        assert float(s[r]) == s_exact, (r, float(s[r]), s_exact)
        for c in range(w.shape[1]):
            qe = round(Fraction(float(wf[r, c])) / Fraction(s_exact))
            qe = max(-127, min(127, qe))
            assert int(q[r, c]) == qe, (r, c, int(q[r, c]), qe)


def pin_quantize_roundtrip_pow2(orc):
    rng = np.random.default_rng(12)
    for k in (-14, -7, 0, 3):
        qq = rng.integers(-127, 128, (6, 33))
        qq[:, 5] = 127
        qq[2, 5] = -127
        w = bf16_bits(qq.astype(np.float32) * np.float32(2.0 ** k))
        q, s = orc.quantize(w)
        assert np.all(s == np.float32(2.0 ** k)), (k, s)
        assert np.array_equal(q.astype(np.int64), qq)


def pin_quantize_halfway(orc):
    # amax = 127 * 2^k gives scale = 2^k exactly; (n + 1/2) * 2^k are exact ties, which go to the even n.
    k = -6
    vals = [127, 0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, 125.5, 126.5, -126.5, 0.25, 0.75, 0]
    expect = [127, 0, 2, 2, 4, 0, -2, -2, 126, 126, -126, 0, 1, 0]
    w = bf16_bits(np.array(vals, dtype=np.float32) * np.float32(2.0 ** k))[None, :]
    q, s = orc.quantize(w)
    assert float(s[0]) == 2.0 ** k
    assert q[0].tolist() == expect, q[0].tolist()


def pin_quantize_zero_row(orc):
    w = np.zeros((3, 16), dtype=np.uint16)
    w[1, 3] = bf16_bits([0.25])[0]
    w[2, :] = 0x8000  # negative zeros
    q, s = orc.quantize(w)
    assert float(s[0]) == 1.0 and float(s[2]) == 1.0
    assert not q[0].any() and not q[2].any()
    assert int(q[1, 3]) == 127


def pin_quantize_invariants(orc):
    rng = np.random.default_rng(13)
    w = random_bf16(rng, (64, 257), 0.02)
    q, s = orc.quantize(w)
    wf = synth.bf16_bits_to_f32(w).astype(np.float64)
    err = np.abs(wf - q.astype(np.float64) * s.astype(np.float64)[:, None])
    assert np.all(err <= s.astype(np.float64)[:, None] / 2)
    assert q.min() >= -127 and q.max() <= 127
    am = np.argmax(np.abs(wf), axis=1)
    assert np.all(np.abs(q[np.arange(64), am]) == 127)


# ---------------------------------------------------------------- routing


def pin_route_uniform(orc):
    x = random_bf16(np.random.default_rng(1), (4, 8), 1.0)
    ids, w = orc.route(x, np.zeros((16, 8), np.float32))
    assert np.all(ids[:, 0] == 0) and np.all(ids[:, 1] == 1)
    assert np.all(w == 1.0 / 16)


def pin_route_closed_form_half(orc):
    # z_0 = ln 15, z_others = 0: p_0 = 15 / (15 + 15) = 1/2, p_e = 1/30; ties among the zeros -> expert 1.
    x = bf16_bits([1.0])[None, :]
    wr = np.zeros((16, 1), np.float32)
    wr[0, 0] = np.float32(np.log(15.0))
    ids, w = orc.route(x, wr)
    assert ids[0].tolist() == [0, 1]
    assert abs(w[0, 0] - 0.5) < 1e-7 and abs(w[0, 1] - 1.0 / 30) < 1e-8


def pin_route_ties_and_order(orc):
    x = bf16_bits([1.0])[None, :]
    z = np.zeros((16, 1), np.float32)
    z[:4, 0] = [1.0, 3.0, 3.0, 2.0]
    ids, _ = orc.route(x, z)
    assert ids[0].tolist() == [1, 2]
    z[:4, 0] = [1.0, 2.0, 3.0, 2.5]
    ids, w = orc.route(x, z)
    assert ids[0].tolist() == [2, 3] and w[0, 0] > w[0, 1]


def pin_route_bias(orc):
    rng = np.random.default_rng(2)
    x = random_bf16(rng, (6, 16), 1.0)
    wr = (rng.standard_normal((16, 16)) * 0.1).astype(np.float32)
    b = np.zeros(16, np.float32)
    b[5] = 40.0
    ids, w = orc.route(x, wr, b)
    assert np.all(ids[:, 0] == 5) and np.all(w[:, 0] > 0.999999)
    ids0, w0 = orc.route(x, wr)
    ids1, w1 = orc.route(x, wr, np.full(16, 3.0, np.float32))  # a common shift changes nothing
    assert np.array_equal(ids0, ids1) and np.allclose(w0, w1, rtol=1e-12, atol=0)


def pin_route_bruteforce(orc):
    rng = np.random.default_rng(3)
    x = random_bf16(rng, (200, 24), 1.0)
    wr = (rng.standard_normal((16, 24)) * 0.3).astype(np.float32)
    b = (rng.standard_normal(16)).astype(np.float32)
    ids, w, z = orc.route(x, wr, b, want_logits=True)
    zz = synth.bf16_bits_to_f32(x).astype(np.float64) @ wr.astype(np.float64).T + b.astype(np.float64)
    assert np.allclose(z, zz, rtol=1e-13, atol=1e-13)
    order = np.argsort(-zz, axis=1, kind="stable")[:, :2]
    assert np.array_equal(ids, order)
    p = torch.softmax(torch.as_tensor(zz), dim=1).numpy()
    assert np.allclose(w, np.take_along_axis(p, order, 1), rtol=1e-12, atol=0)
    # invariants
    assert np.all(ids[:, 0] != ids[:, 1]) and ids.min() >= 0 and ids.max() < 16
    assert np.all(w[:, 0] >= w[:, 1]) and np.all(w[:, 1] > 0) and np.all(w.sum(1) <= 1.0)


# ---------------------------------------------------------------- experts


def pin_forward_zero_gate_or_up(orc):
    L = tiny_layer(np.random.default_rng(4))
    for key in ("q1", "q3"):
        M = dict(L)
        M[key] = np.zeros_like(L[key])
        assert not np.any(fwd(orc, M)["y"]), key


def pin_forward_exact_scaling(orc):
    L = tiny_layer(np.random.default_rng(5))
    y = fwd(orc, L)["y"]
    for key in ("s2", "s3"):
        M = dict(L)
        M[key] = L[key] * np.float32(2.0)
        assert np.array_equal(fwd(orc, M)["y"], 2.0 * y), key


def pin_forward_identical_experts_is_dense_mlp(orc):
    # With E = 2 and K = 2 both experts are always chosen and their softmax weights sum to one,
    # so two identical experts make the layer one dense SwiGLU MLP.
    L = tiny_layer(np.random.default_rng(6), T=7, d=24, F=40, E=2)
    for k in ("q1", "q3", "q2", "s1", "s3", "s2"):
        L[k] = np.ascontiguousarray(np.repeat(L[k][:1], 2, axis=0))
    out = fwd(orc, L)
    y_ref, _ = swiglu_torch(synth.bf16_bits_to_f32(L["x"]), dequant(L["q1"][0], L["s1"][0]),
                            dequant(L["q3"][0], L["s3"][0]), dequant(L["q2"][0], L["s2"][0]))
    assert np.allclose(out["y"], y_ref, rtol=1e-12, atol=1e-15)


def pin_forward_bruteforce_dense_gating(orc):
    rng = np.random.default_rng(7)
    L = tiny_layer(rng, T=9, d=32, F=48, E=16)
    b = rng.standard_normal(16).astype(np.float32)
    out = fwd(orc, L, bias=b, want_hidden=True)
    xf = synth.bf16_bits_to_f32(L["x"]).astype(np.float64)
    z = xf @ L["wr"].astype(np.float64).T + b
    p = torch.softmax(torch.as_tensor(z), 1).numpy()
    top = np.argsort(-z, axis=1, kind="stable")[:, :2]
    y_ref = np.zeros_like(xf)
    for e in range(16):  # every expert on every token; the gate is zero off the top two
        ye, he = swiglu_torch(xf, dequant(L["q1"][e], L["s1"][e]), dequant(L["q3"][e], L["s3"][e]),
                              dequant(L["q2"][e], L["s2"][e]))
        g = np.where((top == e).any(1), p[:, e], 0.0)
        y_ref += g[:, None] * ye
        for k in range(2):
            sel = top[:, k] == e
            assert np.allclose(out["h"][sel, k], he[sel], rtol=1e-12, atol=1e-15)
    assert np.array_equal(out["ids"], top)
    assert np.allclose(out["y"], y_ref, rtol=1e-11, atol=1e-14)


def pin_forward_one_hot(orc):
    # x = e_i: a1_j = q1[j][i] s1[j] and a3_j = q3[j][i] s3[j] exactly.
    L = tiny_layer(np.random.default_rng(8), T=1, d=16, F=24)
    i = 9
    x = np.zeros((1, 16), np.float32)
    x[0, i] = 1.0
    L["x"] = bf16_bits(x)
    out = fwd(orc, L, want_hidden=True)
    for k in range(2):
        e = out["ids"][0, k]
        a1 = torch.as_tensor(L["q1"][e][:, i].astype(np.float64) * L["s1"][e].astype(np.float64))
        a3 = L["q3"][e][:, i].astype(np.float64) * L["s3"][e].astype(np.float64)
        assert np.allclose(out["h"][0, k], torch.nn.functional.silu(a1).numpy() * a3, rtol=1e-14, atol=0)


def pin_forward_token_subset_and_expert_permutation(orc):
    rng = np.random.default_rng(9)
    L = tiny_layer(rng, T=11)
    full = fwd(orc, L)["y"]
    sub = [7, 0, 3]
    assert np.array_equal(fwd(orc, L, tokens=sub)["y"], full[sub])
    perm = rng.permutation(16)
    M = {k: (np.ascontiguousarray(v[perm]) if k != "x" else v) for k, v in L.items()}
    outp = fwd(orc, M)
    # the softmax denominator sums the experts in another order: equal up to that rounding
    assert np.allclose(outp["y"], full, rtol=1e-13, atol=1e-16)


# ---------------------------------------------------------- bf16-weight layer


def pin_bf16w_equals_int8_when_weights_are_codes_times_pow2(orc):
    # bf16 weights w = q * 2^k are exact; with scales 2^k the int8 layer computes the same products
    rng = np.random.default_rng(21)
    L = tiny_layer(rng, T=6, d=32, F=40)
    for key, sk in (("q1", "s1"), ("q3", "s3"), ("q2", "s2")):
        L[sk] = np.full_like(L[sk], np.float32(2.0 ** -9))
    w = {key: bf16_bits(L[key].astype(np.float32) * np.float32(2.0 ** -9)) for key in ("q1", "q3", "q2")}
    a = fwd(orc, L, want_hidden=True)
    b = orc.moe_forward_bf16w(L["x"], L["wr"], None, w["q1"], w["q3"], w["q2"], want_hidden=True)
    assert np.array_equal(a["ids"], b["ids"]) and np.array_equal(a["h"], b["h"]) and np.array_equal(a["y"], b["y"])


def pin_bf16w_identical_experts_is_dense_mlp(orc):
    rng = np.random.default_rng(22)
    T, d, F = 5, 24, 36
    x = random_bf16(rng, (T, d), 1.0)
    wr = (rng.standard_normal((2, d)) * 0.3).astype(np.float32)
    w1, w3 = random_bf16(rng, (F, d), 0.05), random_bf16(rng, (F, d), 0.05)
    w2 = random_bf16(rng, (d, F), 0.05)
    rep = lambda a: np.ascontiguousarray(np.repeat(a[None], 2, axis=0))  # noqa: E731
    out = orc.moe_forward_bf16w(x, wr, None, rep(w1), rep(w3), rep(w2))
    f = synth.bf16_bits_to_f32
    y_ref, _ = swiglu_torch(f(x), f(w1), f(w3), f(w2))
    assert np.allclose(out["y"], y_ref, rtol=1e-12, atol=1e-15)


# ------------------------------------------------------------- dense MLP


def tiny_mlp(rng, T=6, d=32, F=40, wstd=0.05):
    L = tiny_layer(rng, T=T, d=d, F=F, E=1, wstd=wstd)
    return {k: (np.ascontiguousarray(v[0]) if k not in ("x", "wr") else v) for k, v in L.items()}


def mlp(orc, L, **kw):
    return orc.mlp_forward(L["x"], L["q1"], L["s1"], L["q3"], L["s3"], L["q2"], L["s2"], **kw)


def pin_mlp_matches_torch_swiglu(orc):
    L = tiny_mlp(np.random.default_rng(31), T=7, d=40, F=56)
    out = mlp(orc, L, want_hidden=True)
    y_ref, h_ref = swiglu_torch(synth.bf16_bits_to_f32(L["x"]), dequant(L["q1"], L["s1"]),
                                dequant(L["q3"], L["s3"]), dequant(L["q2"], L["s2"]))
    assert np.allclose(out["h"], h_ref, rtol=1e-12, atol=1e-15)
    assert np.allclose(out["y"], y_ref, rtol=1e-12, atol=1e-15)


def pin_mlp_zero_gate_or_up_and_exact_scaling(orc):
    L = tiny_mlp(np.random.default_rng(32))
    y = mlp(orc, L)["y"]
    for key in ("q1", "q3"):
        M = dict(L)
        M[key] = np.zeros_like(L[key])
        assert not np.any(mlp(orc, M)["y"]), key
    for key in ("s2", "s3"):
        M = dict(L)
        M[key] = L[key] * np.float32(2.0)
        assert np.array_equal(mlp(orc, M)["y"], 2.0 * y), key


def pin_mlp_one_hot_and_token_subset(orc):
    L = tiny_mlp(np.random.default_rng(33), T=9, d=16, F=24)
    full = mlp(orc, L)["y"]
    sub = [8, 2, 5]
    assert np.array_equal(mlp(orc, L, tokens=sub)["y"], full[sub])
    i = 5
    x = np.zeros((1, 16), np.float32)
    x[0, i] = 1.0
    M = dict(L)
    M["x"] = bf16_bits(x)
    out = mlp(orc, M, want_hidden=True)
    a1 = torch.as_tensor(L["q1"][:, i].astype(np.float64) * L["s1"].astype(np.float64))
    a3 = L["q3"][:, i].astype(np.float64) * L["s3"].astype(np.float64)
    assert np.allclose(out["h"][0], torch.nn.functional.silu(a1).numpy() * a3, rtol=1e-14, atol=0)


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
