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


# ------------------------------------------------------------- FP8 (E4M3) layer


def torch_e4m3(v):
    """torch's own float8_e4m3fn cast (nearest, ties to even; no saturation: |v| must be < 464)."""
    t = torch.as_tensor(np.asarray(v, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy(), t.to(torch.float64).numpy()


E4M3_VALUES = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def pin_e4m3_rounding_against_torch(orc):
    rng = np.random.default_rng(41)
    finite = E4M3_VALUES[np.isfinite(E4M3_VALUES)]
    pos = np.unique(finite[finite >= 0])
    mids = (pos[1:] + pos[:-1]) / 2  # every tie, between every pair of neighbours
    v = np.concatenate([rng.standard_normal(20000) * 30, rng.standard_normal(4000) * 1e-2,
                        rng.uniform(-2e-3, 2e-3, 2000), mids, -mids, pos, -pos, [447.9, -447.9, 1e-30]])
    v = v.astype(np.float32).astype(np.float64)  # exact in fp32, so torch's cast rounds once
    codes, vals = orc.e4m3_round(v)
    tc, tv = torch_e4m3(v)
    assert np.array_equal(codes, tc)
    assert np.array_equal(vals, tv)
    # saturation (torch gives NaN there): +-448
    c2, v2 = orc.e4m3_round(np.array([448.0, 463.9, 464.0, 1e6, -500.0]))
    assert v2.tolist() == [448.0, 448.0, 448.0, 448.0, -448.0] and c2.tolist() == [0x7E] * 4 + [0xFE]


def pin_quantize_fp8_exact_rational(orc):
    rng = np.random.default_rng(42)
    w = random_bf16(rng, (10, 48), 0.02)
    w[2, 5] = bf16_bits([0.90625])[0]
    w[4] = 0
    q, s = orc.quantize_fp8(w)
    finite = np.isfinite(E4M3_VALUES)
    table = [(Fraction(float(E4M3_VALUES[c])), c) for c in range(256) if finite[c]]
    for r in range(w.shape[0]):
        vals = [Fraction(float(v)) for v in synth.bf16_bits_to_f32(w[r])]
        amax = max(abs(v) for v in vals)
        if amax == 0:
            assert s[r] == 1.0 and not q[r].any()
            continue
        scale = f32_nearest(amax / 448)
        assert float(s[r]) == scale
        for i, v in enumerate(vals):
            quot = v / Fraction(scale)
            best = min(abs(quot - tv) for tv, _ in table)
            cands = sorted({c for tv, c in table if abs(quot - tv) == best and not (tv == 0 and c == 0x80)})
            if len(cands) > 1:  # a tie: the even code (zero is +0 unless the value is negative zero)
                cands = [c for c in cands if c % 2 == 0]
            assert q[r, i] == cands[0] or (quot == 0 and q[r, i] in (0, 0x80)), (r, i)


def fp8_layer(rng, T=6, d=32, F=40, E=16):
    """Random FP8 codes (finite) and scales for a small layer, built directly."""
    finite = np.flatnonzero(np.isfinite(E4M3_VALUES)).astype(np.uint8)
    L = tiny_layer(rng, T=T, d=d, F=F, E=E)
    for k in ("q1", "q3", "q2"):
        L[k] = rng.choice(finite, size=L[k].shape).astype(np.uint8)
    for k in ("s1", "s3", "s2"):
        L[k] = (L[k] * np.float32(127 / 448 / 8)).astype(np.float32)
    return L


def torch_fp8_ffn(xf, q1, s1, q3, s3, q2, s2):
    """One FP8 expert on every row of xf with torch's float8 cast for the activations and for h
    (held in bf16 first, torch's casts): per-row scales amax / 448 in fp32."""
    def quant_rows(a):
        amax = np.abs(a).max(axis=1).astype(np.float32)
        sc = np.where(amax == 0, np.float32(1), amax / np.float32(448)).astype(np.float32)
        _, v = torch_e4m3((a / sc[:, None].astype(np.float64)).astype(np.float32))
        return v * sc[:, None].astype(np.float64)
    w = lambda q, s: E4M3_VALUES[q] * s.astype(np.float64)[:, None]  # noqa: E731
    xd = quant_rows(xf)
    a1, a3 = xd @ w(q1, s1).T, xd @ w(q3, s3).T
    h = torch.nn.functional.silu(torch.as_tensor(a1)).numpy() * a3
    hb = torch.as_tensor(h).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()  # h held in bf16
    return quant_rows(hb) @ w(q2, s2).T, h


def pin_fp8_forward_against_torch_float8(orc):
    # every expert on every token with torch's float8 casts and matmul, gated by numpy top-2
    rng = np.random.default_rng(43)
    L = fp8_layer(rng, T=7, d=32, F=48)
    out = orc.moe_forward_fp8(L["x"], L["wr"], None, L["q1"], L["s1"], L["q3"], L["s3"], L["q2"], L["s2"],
                              want_hidden=True)
    xf = synth.bf16_bits_to_f32(L["x"]).astype(np.float64)
    z = xf @ L["wr"].astype(np.float64).T
    p = torch.softmax(torch.as_tensor(z), 1).numpy()
    top = np.argsort(-z, axis=1, kind="stable")[:, :2]
    y_ref = np.zeros_like(xf)
    for e in range(16):
        ye, he = torch_fp8_ffn(xf, L["q1"][e], L["s1"][e], L["q3"][e], L["s3"][e], L["q2"][e], L["s2"][e])
        y_ref += np.where((top == e).any(1), p[:, e], 0.0)[:, None] * ye
        for k in range(2):
            sel = top[:, k] == e
            assert np.allclose(out["h"][sel, k], he[sel], rtol=1e-12, atol=1e-15)
    assert np.array_equal(out["ids"], top)
    assert np.allclose(out["y"], y_ref, rtol=1e-10, atol=1e-13)


def pin_fp8_forward_zero_gate_and_exact_grid(orc):
    rng = np.random.default_rng(44)
    L = fp8_layer(rng)
    M = dict(L)
    M["q1"] = np.zeros_like(L["q1"])
    out = orc.moe_forward_fp8(M["x"], M["wr"], None, M["q1"], M["s1"], M["q3"], M["s3"], M["q2"], M["s2"])
    assert not np.any(out["y"])
    # activations already on the E4M3 grid with amax 448 * 2^-6: quantizing them is exact
    vals = E4M3_VALUES[np.isfinite(E4M3_VALUES)]
    x = rng.choice(vals[np.abs(vals) <= 448], size=(3, 32)) * 2.0 ** -6
    x[:, 0] = 448 * 2.0 ** -6
    L["x"] = bf16_bits(x.astype(np.float32))
    q, sx = orc.quantize_fp8(L["x"])
    assert np.all(sx == np.float32(2.0 ** -6)) and np.array_equal(E4M3_VALUES[q] * 2.0 ** -6, x)


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
