"""Pins for the FP64 CPU oracle: it is checked against things other than itself.

Each pin is a fact the pages or the mathematics fix, not a retyping of the
oracle's own code:
  * a hand-worked example of the definition (tests/golden/hand_gemm_2x3x2.json);
  * the address formula of the view API evaluated by hand
    ("DeepGEMM: a recalibration of the compute paradigm", §2.3; byte strides §3.2);
  * closed forms: all-ones (C = K), ones-B (row sums), arithmetic series,
    rank-one products, identity and permutation gathers;
  * exact-rational brute force on tiny inputs whose values are decoded by
    numpy/torch, not by the oracle;
  * format tables: every FP16 / BF16 / E4M3 code against numpy's and torch's
    casts and the E4M3 landmarks (448, 2^-9, NaN codes);
  * the pages' strided example (1,128,7,7), strides (0,196,28,4) FP32, against
    numpy's matmul of the reshaped arrays;
  * linearity in alpha/beta, the alpha = 0 and beta = 0 cases, scales applied once;
  * the rounding scale S = |alpha sa sb| sum_k |a b| (the oracle's second output,
    which every GPU tolerance multiplies): worked by hand on a mixed-sign case
    with a negative alpha and scales (tests/golden/hand_gemm_bound_signed.json),
    exact rationals in the brute-force pin, E4M3 powers of two, and the
    one-by-one evaluation equal to the full one;
  * the fused epilogue (Inner discipline page, §3.3): a hand-worked bias + ReLU
    case that fixes the bias to the output column and the activation after
    beta*C (tests/golden/hand_gemm_bias_relu.json); GeLU's tanh form within its
    4.73e-4 approximation error of z*Phi(z) (Phi from libm's erf), its odd-part
    identity g(z) - g(-z) = z, slope 1/2 at 0 and limits; ReLU's closed forms.
The last test plants mistakes in a copy of the oracle source and checks that
some pin catches every one of them.
"""
import json
import math
import os
import shutil
import subprocess
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _problem(A, B, C, alpha=1.0, beta=0.0, sa=None, sb=None, bias=None, act="none"):
    return W.Problem("pin", A, B, C, alpha, beta, sa, sb, bias=bias, act=act)


def _f32(x):
    return W.row_major(torch.tensor(x, dtype=torch.float32), "f32")


# ------------------------------------------------------------------ pins
# Each pin takes an Oracle instance so it can also be run against planted
# mistakes (see test_pins_catch_planted_mistakes).

def pin_hand_example(orc):
    g = json.load(open(os.path.join(GOLDEN, "hand_gemm_2x3x2.json")))
    p = _problem(_f32(g["A"]), _f32(g["B"]), _f32(g["C"]), g["alpha"], g["beta"])
    out, bound = orc.gemm(p, want_bound=True)
    assert np.array_equal(out, np.array(g["expected"]))
    assert np.array_equal(bound, np.array(g["expected_bound"]))


def pin_hand_bound_signed(orc):
    # mixed-sign products, a negative alpha and per-row / per-column scales:
    # the rounding scale S = |alpha sa sb| sum_k |a b| worked by hand
    g = json.load(open(os.path.join(GOLDEN, "hand_gemm_bound_signed.json")))
    p = _problem(_f32(g["A"]), _f32(g["B"]), _f32(g["C"]), g["alpha"], g["beta"],
                 torch.tensor(g["scale_a"]), torch.tensor(g["scale_b"]))
    out, bound = orc.gemm(p, want_bound=True)
    assert np.array_equal(out, np.array(g["expected"]))
    assert np.array_equal(bound, np.array(g["expected_bound"]))
    pts, pbound = orc.gemm_points(p, [0, 0, 1, 1], [0, 1, 0, 1])
    assert np.array_equal(pts, np.array(g["expected"]).reshape(-1))
    assert np.array_equal(pbound, np.array(g["expected_bound"]).reshape(-1))


def pin_view_address(orc):
    g = json.load(open(os.path.join(GOLDEN, "view_address_p2.json")))
    t = torch.zeros(2 * 3 * 4, dtype=torch.float32)
    for row_dims in (1, 2):
        op = W.Operand(t, tuple(g["shape"]), tuple(g["stride"]), row_dims, "f32")
        for i, j, k, want in g["cases"]:
            if row_dims == 1:
                r, c = i, j * 4 + k
            else:
                r, c = i * 3 + j, k
            assert orc.offset(op, r, c) == want


def pin_all_ones(orc):
    for dt in ("f16", "bf16", "e4m3", "f32"):
        M, N, K = 5, 7, 37
        A = W.row_major(torch.ones(M, K).to(W.TORCH_DTYPE[dt]), dt)
        B = W.row_major(torch.ones(K, N).to(W.TORCH_DTYPE[dt]), dt)
        out = orc.gemm(_problem(A, B, W.empty_out(M, N, "f32")), want_bound=False)
        assert np.all(out == K)


def pin_row_sums(orc):
    g = torch.Generator().manual_seed(7)
    M, N, K = 6, 3, 50
    a = torch.randint(-8, 9, (M, K), generator=g).to(torch.float16)
    out = orc.gemm(_problem(W.row_major(a, "f16"), W.row_major(torch.ones(K, N, dtype=torch.float16), "f16"),
                            W.empty_out(M, N, "f32")), want_bound=False)
    sums = a.double().sum(dim=1).numpy()
    assert np.array_equal(out, np.repeat(sums[:, None], N, axis=1))


def pin_index_series(orc):
    # a(m,k) = m + 2k and b(k,n) = 3k + n (small integers, exact in FP16) make a
    # transposed operand or a swapped index give a different closed form:
    # sum_k (m + 2k)(3k + n) = K*m*n + 3m*S1 + 2n*S1 + 6*S2, S1 = sum k, S2 = sum k^2.
    M, N, K = 4, 5, 6
    m = torch.arange(M)[:, None]
    k = torch.arange(K)
    n = torch.arange(N)[None, :]
    a = (m + 2 * k[None, :]).to(torch.float16)
    b = (3 * k[:, None] + n).to(torch.float16)
    out = orc.gemm(_problem(W.row_major(a, "f16"), W.row_major(b, "f16"), W.empty_out(M, N, "f32")),
                   want_bound=False)
    S1, S2 = K * (K - 1) // 2, (K - 1) * K * (2 * K - 1) // 6
    mm, nn = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    want = K * mm * nn + 3 * mm * S1 + 2 * nn * S1 + 6 * S2
    assert np.array_equal(out, want.astype(np.float64))


def pin_rank_one(orc):
    # a(m,k) = u_m, b(k,n) = v_n  =>  C = K * u_m * v_n exactly (small integers).
    M, N, K = 3, 4, 9
    u = torch.tensor([1.0, -2.0, 3.0])
    v = torch.tensor([0.5, 4.0, -1.0, 2.0])
    a = u[:, None].expand(M, K).contiguous().to(torch.bfloat16)
    b = v[None, :].expand(K, N).contiguous().to(torch.bfloat16)
    out = orc.gemm(_problem(W.row_major(a, "bf16"), W.row_major(b, "bf16"), W.empty_out(M, N, "f32")),
                   want_bound=False)
    assert np.array_equal(out, K * np.outer(u.numpy(), v.numpy()))


def pin_identity_and_permutation(orc):
    g = torch.Generator().manual_seed(3)
    M, K = 9, 12
    a = (torch.rand(M, K, generator=g) * 2 - 1).to(torch.bfloat16)
    eye = torch.eye(K, dtype=torch.bfloat16)
    out = orc.gemm(_problem(W.row_major(a, "bf16"), W.row_major(eye, "bf16"), W.empty_out(M, K, "f32")),
                   want_bound=False)
    assert np.array_equal(out, a.double().numpy())
    perm = torch.randperm(K, generator=g)
    P = torch.zeros(K, K, dtype=torch.bfloat16)
    P[perm, torch.arange(K)] = 1  # column j of P selects row perm[j]: (aP)[:, j] = a[:, perm[j]]
    out = orc.gemm(_problem(W.row_major(a, "bf16"), W.row_major(P, "bf16"), W.empty_out(M, K, "f32")),
                   want_bound=False)
    assert np.array_equal(out, a.double().numpy()[:, perm.numpy()])


def _exact_values(t: torch.Tensor, dt: str):
    """Decode with numpy/torch (not the oracle) into Python Fractions."""
    if dt == "f16":
        vals = t.numpy().astype(np.float64)
    else:
        vals = t.to(torch.float64).numpy()
    return [[Fraction(float(x)) for x in row] for row in vals]


def pin_brute_force(orc):
    g = torch.Generator().manual_seed(11)
    for dt in ("f16", "bf16", "e4m3"):
        for (M, N, K) in ((1, 1, 1), (2, 3, 4), (3, 2, 5), (4, 4, 16)):
            a32 = torch.randn(M, K, generator=g)
            b32 = torch.randn(K, N, generator=g)
            c32 = torch.randn(M, N, generator=g)
            a = a32.to(W.TORCH_DTYPE[dt])
            b = b32.to(W.TORCH_DTYPE[dt])
            sa = torch.rand(M, generator=g) + 0.5
            sb = torch.rand(N, generator=g) + 0.5
            alpha, beta = (0.75 if M % 2 else -0.75), -1.25
            p = _problem(W.row_major(a, dt), W.row_major(b, dt), W.row_major(c32.contiguous(), "f32"),
                         alpha, beta, sa, sb)
            out, bound = orc.gemm(p, want_bound=True)
            A = _exact_values(a, dt)
            B = _exact_values(b, dt)
            for i in range(M):
                for j in range(N):
                    acc = sum(A[i][k] * B[k][j] for k in range(K))
                    mag = sum(abs(A[i][k] * B[k][j]) for k in range(K))
                    s = Fraction(alpha) * Fraction(float(sa[i])) * Fraction(float(sb[j]))
                    r = s * acc + Fraction(beta) * Fraction(float(c32[i, j]))
                    # FP64 rounding of a K-term sum plus the scale and beta steps
                    tol = (K + 4) * 2.0 ** -52 * float(abs(s) * mag + abs(Fraction(beta) * Fraction(float(c32[i, j]))))
                    assert abs(out[i, j] - float(r)) <= tol, (dt, M, N, K, i, j)
                    # the rounding scale S = |alpha sa sb| sum_k |a b|, exact up to FP64 rounding
                    S = abs(s) * mag
                    assert abs(bound[i, j] - float(S)) <= (K + 4) * 2.0 ** -52 * float(S), (dt, M, N, K, i, j)


def pin_f16_bf16_tables(orc):
    codes = np.arange(65536, dtype=np.uint16)
    f16 = codes.view(np.float16).astype(np.float64)
    bf16 = torch.from_numpy(codes.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    for i in range(0, 65536, 97):  # a spread of codes incl. subnormals, infs, nans
        raw = int(codes[i]).to_bytes(2, "little")
        for dt, ref in (("f16", f16[i]), ("bf16", bf16[i])):
            got = orc.decode(dt, raw)
            assert (math.isnan(got) and math.isnan(ref)) or got == ref, (dt, i, got, ref)
    # landmarks
    assert orc.decode("f16", (0x0001).to_bytes(2, "little")) == 2.0 ** -24
    assert orc.decode("f16", (0x7BFF).to_bytes(2, "little")) == 65504.0
    assert orc.decode("f16", (0x7C00).to_bytes(2, "little")) == math.inf
    assert orc.decode("bf16", (0x3F80).to_bytes(2, "little")) == 1.0
    assert orc.decode("bf16", (0xC000).to_bytes(2, "little")) == -2.0


def pin_e4m3_table(orc):
    codes = torch.arange(256, dtype=torch.int16).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = orc.decode_e4m3(c)
        assert (math.isnan(got) and math.isnan(ref[c])) or got == ref[c], (c, got, ref[c])
    assert orc.decode_e4m3(0x7E) == 448.0  # largest finite
    assert orc.decode_e4m3(0x01) == 2.0 ** -9  # smallest subnormal
    assert orc.decode_e4m3(0x08) == 2.0 ** -6  # smallest normal
    assert orc.decode_e4m3(0x38) == 1.0
    assert orc.decode_e4m3(0xB8) == -1.0
    assert math.isnan(orc.decode_e4m3(0x7F)) and math.isnan(orc.decode_e4m3(0xFF))


def pin_pages_strided_example(orc):
    # Q and K of shape (1,128,7,7) with strides (0,196,28,4) bytes, FP32,
    # matmul(Q, K^T) over the (128, 49) matrices: the recalibration page, §2.2.
    g = torch.Generator().manual_seed(5)
    q = torch.randn(128 * 49, generator=g)
    k = torch.randn(128 * 49, generator=g)
    Q = W.Operand(q, (1, 128, 7, 7), (0, 196, 28, 4), 2, "f32")
    # K^T as a [49, 128] view: rows are (h, w), columns are channels.
    KT = W.Operand(k, (7, 7, 1, 128), (28, 4, 0, 196), 2, "f32")
    out = orc.gemm(_problem(Q, KT, W.empty_out(128, 128, "f32")), want_bound=False)
    ref = q.double().numpy().reshape(128, 49) @ k.double().numpy().reshape(128, 49).T
    assert np.allclose(out, ref, rtol=0, atol=1e-12)


def pin_strided_equals_contiguous(orc):
    g = torch.Generator().manual_seed(9)
    x = torch.rand(2, 8, 3, 5, generator=g).to(torch.bfloat16)  # NCHW
    b = torch.rand(8, 6, generator=g).to(torch.bfloat16)
    strided = W.nchw_as_rows(x, "bf16")
    dense = W.row_major(x.permute(0, 2, 3, 1).reshape(2 * 3 * 5, 8).contiguous(), "bf16")
    B = W.row_major(b, "bf16")
    o1 = orc.gemm(_problem(strided, B, W.empty_out(30, 6, "f32")), want_bound=False)
    o2 = orc.gemm(_problem(dense, B, W.empty_out(30, 6, "f32")), want_bound=False)
    assert np.array_equal(o1, o2)
    kt = torch.rand(6, 8, generator=g).to(torch.bfloat16)
    o3 = orc.gemm(_problem(dense, W.transposed(kt, "bf16"), W.empty_out(30, 6, "f32")), want_bound=False)
    o4 = orc.gemm(_problem(dense, W.row_major(kt.t().contiguous(), "bf16"), W.empty_out(30, 6, "f32")),
                  want_bound=False)
    assert np.array_equal(o3, o4)


def pin_linearity_alpha_beta(orc):
    p = W.cfg_small(M=16, N=24, K=40)
    c0 = torch.randn(16, 24, generator=torch.Generator().manual_seed(2))
    C = W.row_major(c0.contiguous(), "f32")
    base = orc.gemm(_problem(p.A, p.B, C, 1.0, 0.0), want_bound=False)
    for alpha, beta in ((2.0, 0.0), (-0.5, 1.0), (0.25, -3.0)):
        out = orc.gemm(_problem(p.A, p.B, C, alpha, beta), want_bound=False)
        assert np.allclose(out, alpha * base + beta * c0.double().numpy(), rtol=1e-14, atol=1e-13)


def pin_alpha_zero_beta_zero(orc):
    M, N, K = 3, 4, 5
    a = torch.ones(M, K, dtype=torch.float16)
    a[1, 2] = float("inf")
    b = torch.ones(K, N, dtype=torch.float16)
    c = torch.arange(M * N, dtype=torch.float32).reshape(M, N)
    out = orc.gemm(_problem(W.row_major(a, "f16"), W.row_major(b, "f16"), W.row_major(c, "f32"), 0.0, 2.0),
                   want_bound=False)
    assert np.array_equal(out, 2.0 * c.double().numpy())  # beta still applied, A never read
    cn = torch.full((M, N), float("nan"))
    a[1, 2] = 1.0
    out = orc.gemm(_problem(W.row_major(a, "f16"), W.row_major(b, "f16"), W.row_major(cn, "f32"), 1.0, 0.0),
                   want_bound=False)
    assert np.all(out == K)  # C is not read when beta == 0


def pin_scales_once(orc):
    M, N, K = 4, 6, 8
    a = torch.ones(M, K).to(torch.float8_e4m3fn)
    b = torch.ones(K, N).to(torch.float8_e4m3fn)
    sa = torch.tensor([2.0 ** j for j in range(M)])
    sb = torch.tensor([2.0 ** -j for j in range(N)])
    out = orc.gemm(_problem(W.row_major(a, "e4m3"), W.row_major(b, "e4m3"), W.empty_out(M, N, "f32"),
                            1.0, 0.0, sa, sb), want_bound=False)
    want = K * np.outer(sa.numpy(), sb.numpy())
    assert np.array_equal(out, want)
    # E4M3 codes of +-1 and -2 with alpha = -2: the output and its rounding
    # scale both carry |alpha sa sb| exactly once (powers of two: exact)
    a = torch.ones(M, K)
    a[:, ::2] = -2.0
    a = a.to(torch.float8_e4m3fn)
    out, bound = orc.gemm(_problem(W.row_major(a, "e4m3"), W.row_major(b, "e4m3"), W.empty_out(M, N, "f32"),
                                   -2.0, 0.0, sa, sb), want_bound=True)
    row_sum = (K // 2) * (-2.0) + (K // 2) * 1.0       # sum_k a b
    row_mag = (K // 2) * 2.0 + (K // 2) * 1.0          # sum_k |a b|
    assert np.array_equal(out, -2.0 * row_sum * np.outer(sa.numpy(), sb.numpy()))
    assert np.array_equal(bound, 2.0 * row_mag * np.outer(sa.numpy(), sb.numpy()))


def pin_points_match_full(orc):
    p = W.cfg_strided(n=2, c=24, h=5, w=7, N=40)
    full = orc.gemm(p, want_bound=False)
    ms = [0, 1, 34, 69, 35]
    ns = [0, 39, 7, 20, 1]
    pts, _ = orc.gemm_points(p, ms, ns)
    assert np.array_equal(pts, full[ms, ns])
    # the one-by-one evaluation gives the same output and rounding scale as
    # the full oracle on a scaled E4M3 problem with a negative alpha and beta != 0
    g = torch.Generator().manual_seed(21)
    M, N, K = 7, 9, 40
    qa, sa = W.quantise_e4m3(W.normal((M, K), g), dim=1)
    qb, sb = W.quantise_e4m3(W.normal((K, N), g), dim=0)
    q = _problem(W.row_major(qa, "e4m3"), W.row_major(qb, "e4m3"), W.row_major(W.uniform((M, N), g), "f32"),
                 -1.5, 0.5, sa, sb)
    full, fbound = orc.gemm(q, want_bound=True)
    ms = np.repeat(np.arange(M), N)
    ns = np.tile(np.arange(N), M)
    pts, pbound = orc.gemm_points(q, ms, ns)
    assert np.array_equal(pts, full.reshape(-1))
    assert np.array_equal(pbound, fbound.reshape(-1))


# ------------------------------------------------------ the fused epilogue

def pin_epilogue_hand(orc):
    g = json.load(open(os.path.join(GOLDEN, "hand_gemm_bias_relu.json")))
    p = _problem(_f32(g["A"]), _f32(g["B"]), _f32(g["C"]), g["alpha"], g["beta"],
                 bias=torch.tensor(g["bias"]), act=g["act"])
    out, bound, pre = orc.gemm(p, want_bound=True, want_pre=True)
    assert np.array_equal(pre, np.array(g["expected_pre"]))
    assert np.array_equal(out, np.array(g["expected"]))
    assert np.array_equal(bound, np.array([[58.0, 64.0], [139.0, 154.0]]))  # S has no bias or C term


def _phi(z):
    return 0.5 * (1.0 + math.erf(z / math.sqrt(2.0)))


def pin_gelu_closed_forms(orc):
    # GeLU(z) = z Phi(z); the tanh form (Inner discipline page, §3.3) is within
    # 4.73e-4 of it everywhere (the approximation's published maximum error);
    # Phi comes from libm's erf, an independent special function.
    g = lambda z: orc.activation("gelu_tanh", z)  # noqa: E731
    assert g(0.0) == 0.0
    for i in range(-800, 801):
        z = i / 100.0
        assert abs(g(z) - z * _phi(z)) <= 5e-4, z
        # z Phi(z) - (-z) Phi(-z) = z since Phi(z) + Phi(-z) = 1; the tanh form keeps it (tanh is odd)
        assert abs((g(z) - g(-z)) - z) <= 4e-16 * max(1.0, abs(z)), z
    assert g(20.0) == 20.0 and abs(g(-20.0)) <= 1e-300
    h = 1e-6  # slope 1/2 at 0: Phi(0) = 1/2
    assert abs((g(h) - g(-h)) / (2 * h) - 0.5) <= 1e-9
    assert math.isnan(g(float("nan")))


def pin_relu_closed_forms(orc):
    r = lambda z: orc.activation("relu", z)  # noqa: E731
    for z in (-3.5, -1e-30, 0.0, 2.5, 1e30):
        assert r(z) - r(-z) == z and r(z) >= 0.0
    assert r(-2.0) == 0.0 and r(7.25) == 7.25
    assert math.isnan(r(float("nan")))  # a NaN of the sum still reaches C
    assert orc.activation("none", -4.5) == -4.5


def _epi_problem(act, seed=13, bias=True):
    g = torch.Generator().manual_seed(seed)
    M, N, K = 6, 10, 24
    a = W.cast(W.normal((M, K), g), "bf16")
    b = W.cast(W.normal((K, N), g), "bf16")
    c = W.uniform((M, N), g)
    bv = W.normal((N,), g)  # drawn either way, so the scales below are the same draws
    return _problem(W.row_major(a, "bf16"), W.row_major(b, "bf16"), W.row_major(c.contiguous(), "f32"),
                    0.5, -1.5, torch.rand(M, generator=g) + 0.5, torch.rand(N, generator=g) + 0.5,
                    bv if bias else None, act)


def pin_bias_per_column_and_activation_last(orc):
    # the bias is added once per output column, to every row
    with_b = orc.gemm(_epi_problem("none"), want_bound=False)
    without = orc.gemm(_epi_problem("none", bias=False), want_bound=False)
    bias = _epi_problem("none").bias.double().numpy()
    assert np.allclose(with_b - without, np.broadcast_to(bias, with_b.shape), rtol=0, atol=1e-13)
    # the activation acts on the whole sum (product, beta*C and bias)
    relu = orc.gemm(_epi_problem("relu"), want_bound=False)
    assert np.array_equal(relu, np.where(with_b < 0, 0.0, with_b))
    gelu = orc.gemm(_epi_problem("gelu_tanh"), want_bound=False)
    exact = np.vectorize(lambda z: z * _phi(z))(with_b)
    assert np.all(np.abs(gelu - exact) <= 5e-4)
    # the one-by-one evaluation agrees, including the value before the activation
    ms = np.repeat(np.arange(6), 10)
    ns = np.tile(np.arange(10), 6)
    pts, _, pre = orc.gemm_points(_epi_problem("gelu_tanh"), ms, ns, want_pre=True)
    assert np.array_equal(pts, gelu.reshape(-1))
    assert np.array_equal(pre, with_b.reshape(-1))


PINS = [pin_hand_example, pin_hand_bound_signed, pin_view_address, pin_all_ones, pin_row_sums, pin_index_series,
        pin_rank_one, pin_identity_and_permutation, pin_brute_force, pin_f16_bf16_tables,
        pin_e4m3_table, pin_pages_strided_example, pin_strided_equals_contiguous,
        pin_linearity_alpha_beta, pin_alpha_zero_beta_zero, pin_scales_once, pin_points_match_full,
        pin_epilogue_hand, pin_gelu_closed_forms, pin_relu_closed_forms, pin_bias_per_column_and_activation_last]


@pytest.mark.parametrize("pin", PINS, ids=[f.__name__ for f in PINS])
def test_pin(pin):
    pin(oracle.default())


# Plausible mistakes, planted in a copy of the oracle source.  Each must make
# at least one pin fail.
MUTANTS = {
    "beta_dropped": ("if (beta != 0.0) r += beta * elem(C, m, n);", "(void)beta;"),
    "alpha_ignored": ("double s = alpha * s_m * s_n;", "double s = s_m * s_n;"),
    "b_transposed": ("bt[n * K + k] = elem(B, k, n);", "bt[n * K + k] = elem(B, n % K, k % N);"),
    "col_major_unflatten": ("for (int d = v->row_dims - 1; d >= 0; --d) {",
                            "for (int d = 0; d < v->row_dims; ++d) {"),
    "e4m3_bias_8": ("v = ldexp(1.0 + (double)f / 8.0, e - 7);", "v = ldexp(1.0 + (double)f / 8.0, e - 8);"),
    "e4m3_no_subnormal": ("v = ldexp((double)f, -9);", "v = ldexp(1.0 + (double)f / 8.0, -6);"),
    "scale_twice": ("double s = alpha * s_m * s_n;", "double s = alpha * s_m * s_n * s_m;"),
    "k_dropped_last": ("for (int64_t k = 0; k < K; ++k) {\n                    double p",
                       "for (int64_t k = 0; k + 1 < K; ++k) {\n                    double p"),
    "f16_bias_14": ("v = ldexp(1.0 + (double)f / 1024.0, e - 15);", "v = ldexp(1.0 + (double)f / 1024.0, e - 14);"),
    "beta_zero_reads_c": ("if (beta != 0.0) r += beta * elem(C, m, n);", "r += beta * elem(C, m, n);"),
    # the rounding scale S = |alpha sa sb| sum_k |a b| that every GPU tolerance multiplies
    "bound_is_mag": ("bound[m * N + n] = (a ? fabs(s) * mag : 0.0);", "bound[m * N + n] = (a ? mag : 0.0);"),
    "bound_no_alpha": ("bound[m * N + n] = (a ? fabs(s) * mag : 0.0);",
                       "bound[m * N + n] = (a ? fabs(s_m * s_n) * mag : 0.0);"),
    "bound_signed_scale": ("bound[m * N + n] = (a ? fabs(s) * mag : 0.0);", "bound[m * N + n] = (a ? s * mag : 0.0);"),
    "mag_signed_products": ("acc += p;\n                    mag += fabs(p);", "acc += p;\n                    mag += p;"),
    "points_bound_is_mag": ("bound[i] = use_ab ? fabs(s) * mag : 0.0;", "bound[i] = use_ab ? mag : 0.0;"),
    "points_mag_signed": ("acc += p;\n                mag += fabs(p);", "acc += p;\n                mag += p;"),
    # the fused epilogue: bias, activation and their order
    "bias_per_row": ("if (bias) r += (double)bias[n];\n            out[m * N + n]",
                     "if (bias) r += (double)bias[m % N];\n            out[m * N + n]"),
    "activation_before_beta_c": (
        "if (beta != 0.0) r += beta * elem(C, m, n);\n            if (bias) r += (double)bias[n];\n"
        "            out[m * N + n] = dgo_activation(act, r);",
        "if (bias) r += (double)bias[n];\n"
        "            out[m * N + n] = dgo_activation(act, r) + (beta != 0.0 ? beta * elem(C, m, n) : 0.0);"),
    "activation_dropped": ("out[m * N + n] = dgo_activation(act, r);", "out[m * N + n] = r;"),
    "gelu_no_cubic": ("tanh(c * (z + 0.044715 * z * z * z))", "tanh(c * z)"),
    "gelu_no_half": ("return 0.5 * z * (1.0 + tanh", "return z * (1.0 + tanh"),
    "gelu_wrong_constant": ("sqrt(2.0 / acos(-1.0))", "sqrt(2.0 * acos(-1.0))"),
    "relu_abs": ("case DGO_ACT_RELU: return z < 0.0 ? 0.0 : z;", "case DGO_ACT_RELU: return fabs(z);"),
    "points_bias_dropped": ("if (bias) r += (double)bias[n];\n        out[i]", "out[i]"),
}


def _pins_pass(orc) -> bool:
    for pin in PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError):
            return False
    return True


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_pins_catch_planted_mistakes(tmp_path):
    src = open(oracle._SRC).read()
    for name, (old, new) in MUTANTS.items():
        assert src.count(old) >= 1, f"mutation site for {name} not found"
        path = tmp_path / f"{name}.c"
        path.write_text(src.replace(old, new, 1))
        lib = tmp_path / f"lib{name}.so"
        subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", str(path), "-o",
                        str(lib), "-lm"], check=True)
        assert not _pins_pass(oracle.Oracle(str(lib))), f"no pin caught the planted mistake {name}"
