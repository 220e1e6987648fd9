"""Pins for the CPU oracle: checks against what the pages and the mathematics fix, never
against the oracle's own formulas retyped.

Scan ("Why Gated DeltaNet Survives 4-Bit Quantization", abstract, mechanisms ii-iii):
  overwrite along the key, identity gates, geometric forgetting (closed form and
  contraction bound), associative recall from orthonormal keys, the d = 1 closed form,
  an independently derived chunked (WY/UT) form, composition of prefix + suffix, GQA and
  variable-length equivalences, gates against torch's softplus/sigmoid.
Tail ("Red Lite dev15d - DeltaNet gated tail", Pinned graph semantics): one shared weight
  (head permutation), reduction to torch's rms_norm, the mean-square identity.
NVFP4 (16-element block scaling, E2M1 values, E4M3 scales): E4M3 against torch's
  float8_e4m3fn, E2M1 against the decision thresholds of the format, the exact round trip
  of grid values, nibble order, the block error bound, GEMM against brute force in exact
  rational arithmetic.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads

RNG = np.random.default_rng(1234)
BIG = 40.0      # sigmoid(40) == 1.0 exactly in fp64
NEG = -1000.0   # exp(-1000) == 0.0 exactly in fp64


def _unit(shape, rng):
    x = rng.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _scan(q, k, v, a, b, A_log, dt_bias, **kw):
    return oracle.gdn_scan(q, k, v, a, b, A_log, dt_bias, **kw)


# ------------------------------------------------------------------------ gates ----

def test_gates_match_torch_softplus_sigmoid():
    rng = np.random.default_rng(1)
    for _ in range(200):
        a, b = rng.normal() * 4, rng.normal() * 6
        A_log, dt = rng.uniform(-2, 3), rng.normal()
        g, alpha, beta = oracle.gates(a, b, A_log, dt)
        t_sp = torch.nn.functional.softplus(torch.tensor(a + dt, dtype=torch.float64)).item()
        assert g == pytest.approx(-math.exp(A_log) * t_sp, rel=1e-13, abs=1e-300)
        assert alpha == pytest.approx(math.exp(g), rel=1e-13)
        assert beta == pytest.approx(torch.sigmoid(torch.tensor(b, dtype=torch.float64)).item(),
                                     rel=1e-13)


def test_gate_special_values():
    # softplus(0) = ln 2 and exp(0) = 1, so alpha = exp(-ln 2) = 1/2; sigmoid(0) = 1/2
    g, alpha, beta = oracle.gates(0.0, 0.0, 0.0, 0.0)
    assert alpha == pytest.approx(0.5, rel=1e-15) and beta == 0.5
    # large arguments: softplus(x) -> x, so log(alpha) = -exp(A_log) * x
    g, _, _ = oracle.gates(500.0, 0.0, math.log(3.0), 0.0)
    assert g == pytest.approx(-1500.0, rel=1e-15)
    # the saturating special cases used by the pins below
    assert oracle.gates(0.3, BIG, 0.0, 0.0)[2] == 1.0
    assert oracle.gates(0.3, NEG, 0.0, 0.0)[2] == 0.0
    assert oracle.gates(0.3, 0.0, NEG, 0.0)[1] == 1.0


# ------------------------------------------------------------------------- scan ----

@pytest.mark.parametrize("steps", [1, 5])
def test_write_overwrites_along_key(steps):
    """beta = 1 and a unit key: after the write, S k = v, so reading with q = k returns v,
    whatever the previous state and decay (mechanism iii)."""
    rng = np.random.default_rng(2)
    D = 24
    T = steps
    k = _unit((T, 1, D), rng)
    q = k.copy()
    v = rng.standard_normal((T, 1, D))
    a = rng.standard_normal((T, 1))
    b = np.full((T, 1), BIG)
    S0 = rng.standard_normal((1, 1, D, D))
    o, S = _scan(q, k, v, a, b, [0.7], [0.1], initial_state=S0, eps=0.0)
    np.testing.assert_allclose(o[:, 0, :], v[:, 0, :].astype(np.float32), rtol=0, atol=1e-12)
    np.testing.assert_allclose(S[0, 0] @ k[-1, 0].astype(np.float32).astype(np.float64),
                               v[-1, 0].astype(np.float32), atol=1e-12)


def test_identity_gates_leave_state_unchanged():
    """alpha = 1, beta = 0: S stays bit-for-bit; o_t = S0 q_t."""
    rng = np.random.default_rng(3)
    T, D = 9, 16
    q = rng.standard_normal((T, 1, D)).astype(np.float32)
    k = rng.standard_normal((T, 1, D)).astype(np.float32)
    v = rng.standard_normal((T, 1, D)).astype(np.float32)
    a = rng.standard_normal((T, 1))
    b = np.full((T, 1), NEG)
    S0 = rng.standard_normal((1, 1, D, D))
    o, S = _scan(q, k, v, a, b, [NEG], [0.0], initial_state=S0, qk_l2norm=False)
    assert np.array_equal(S, S0)
    np.testing.assert_allclose(o[:, 0, :], q[:, 0, :].astype(np.float64) @ S0[0, 0].T,
                               rtol=1e-14, atol=1e-14)


def test_forgetting_closed_form():
    """beta = 0 and alpha = 1/2 each step (a = 0, A_log = 0): S_T = 2^-T S0 exactly."""
    rng = np.random.default_rng(4)
    T, D = 12, 8
    q = rng.standard_normal((T, 1, D)).astype(np.float32)
    k = rng.standard_normal((T, 1, D)).astype(np.float32)
    v = rng.standard_normal((T, 1, D)).astype(np.float32)
    S0 = rng.standard_normal((1, 1, D, D))
    o, S = _scan(q, k, v, np.zeros((T, 1)), np.full((T, 1), NEG), [0.0], [0.0],
                 initial_state=S0, qk_l2norm=False)
    np.testing.assert_allclose(S, S0 * 2.0 ** -T, rtol=1e-13)
    for t in range(T):
        np.testing.assert_allclose(o[t, 0], (S0[0, 0] @ q[t, 0].astype(np.float64)) * 2.0 ** -(t + 1),
                                   rtol=1e-12, atol=1e-15)


def test_impulse_decays_geometrically():
    """Two runs that differ only in S0: ||dS_t||_2 <= prod(alpha) ||dS0||_2, because
    ||I - beta k k^T||_2 <= 1 for a unit key and beta in [0, 1]."""
    rng = np.random.default_rng(5)
    T, D = 300, 16
    q = rng.standard_normal((T, 1, D)).astype(np.float32)
    k = rng.standard_normal((T, 1, D)).astype(np.float32)
    v = rng.standard_normal((T, 1, D)).astype(np.float32)
    a = (rng.standard_normal((T, 1)) - 1.0)
    b = rng.standard_normal((T, 1))
    A_log = [math.log(0.2)]     # mean decay per step ~ exp(-0.06): a timescale of ~16 steps
    S0 = rng.standard_normal((1, 1, D, D))
    dS0 = rng.standard_normal((1, 1, D, D))
    logs = []
    bound0 = np.linalg.norm(dS0[0, 0], 2)
    prod_log = 0.0
    for t_end in (1, 10, 50, 150, 300):
        o1, S1 = _scan(q[:t_end], k[:t_end], v[:t_end], a[:t_end], b[:t_end], A_log, [0.0],
                       initial_state=S0, eps=0.0)
        o2, S2 = _scan(q[:t_end], k[:t_end], v[:t_end], a[:t_end], b[:t_end], A_log, [0.0],
                       initial_state=S0 + dS0, eps=0.0)
        prod_log = sum(oracle.gates(float(a[t, 0]), 0.0, A_log[0], 0.0)[0] for t in range(t_end))
        diff = np.linalg.norm(S2[0, 0] - S1[0, 0], 2)
        assert diff <= math.exp(prod_log) * bound0 * (1 + 1e-9) + 1e-300
        logs.append(diff)
    # the impulse is forgotten: after 300 steps it is below 1e-6 of its size
    assert logs[-1] < 1e-6 * bound0
    assert all(x >= y for x, y in zip(logs, logs[1:]))


def test_associative_recall_orthonormal_keys():
    """alpha = 1, beta = 1, keys e_1..e_d, S0 = 0: S = sum_t v_t e_t^T; q = e_i reads v_i."""
    rng = np.random.default_rng(6)
    D = 16
    k = np.eye(D, dtype=np.float32)[:, None, :]
    v = rng.standard_normal((D, 1, D)).astype(np.float32)
    o, S = _scan(k, k, v, np.zeros((D, 1)), np.full((D, 1), BIG), [NEG], [0.0], eps=0.0)
    np.testing.assert_allclose(S[0, 0], v[:, 0, :].T.astype(np.float64), atol=1e-15)
    # read every slot back after all writes (continue from S with identity gates)
    o2, _ = _scan(k[::-1], k, v, np.zeros((D, 1)), np.full((D, 1), NEG), [NEG], [0.0],
                  initial_state=S, eps=0.0)
    np.testing.assert_allclose(o2[:, 0, :], v[::-1, 0, :].astype(np.float64), atol=1e-15)


def test_scalar_closed_form():
    """Dk = Dv = 1: k_hat = sign(k), so S_t = alpha_t (1 - beta_t) S_{t-1} + beta_t v_t sign(k_t)
    and o_t = S_t sign(q_t)."""
    rng = np.random.default_rng(7)
    T = 40
    q = rng.standard_normal((T, 1, 1)).astype(np.float32)
    k = rng.standard_normal((T, 1, 1)).astype(np.float32)
    v = rng.standard_normal((T, 1, 1)).astype(np.float32)
    a = rng.standard_normal((T, 1)).astype(np.float32)
    b = rng.standard_normal((T, 1)).astype(np.float32)
    A_log, dt = float(np.float32(0.3)), float(np.float32(0.2))   # the oracle reads fp32 gates
    o, S = _scan(q, k, v, a, b, [A_log], [dt], eps=0.0)
    s = 0.0
    for t in range(T):
        alpha = math.exp(-math.exp(A_log) * math.log1p(math.exp(float(a[t, 0]) + dt)))
        beta = 1.0 / (1.0 + math.exp(-float(b[t, 0])))
        s = alpha * (1.0 - beta) * s + beta * float(v[t, 0, 0]) * math.copysign(1.0, float(k[t, 0, 0]))
        assert o[t, 0, 0] == pytest.approx(s * math.copysign(1.0, float(q[t, 0, 0])), rel=1e-12, abs=1e-14)
    assert S[0, 0, 0, 0] == pytest.approx(s, rel=1e-12)


def _chunked_reference(qh, kh, v, g, beta, S0, C):
    """Chunked (WY / UT transform) form of the same recurrence, derived independently:
    with gamma_r = exp(G_r) (G = in-chunk cumulative log decay), u_r = beta_r (v_r - alpha_r
    S_{r-1} k_r) solves (I + A) U = diag(beta) V - diag(beta gamma) K S0^T, where
    A_rs = beta_r exp(G_r - G_s) k_r.k_s for s < r. Then O = diag(gamma) Q S0^T +
    (Q K^T * Gamma) U and S_C = gamma_C S0 + U^T diag(gamma_C / gamma) K."""
    T = qh.shape[0]
    S = S0.copy()
    O = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        sl = slice(c0, min(T, c0 + C))
        Q, K, V, gg, bb = qh[sl], kh[sl], v[sl], g[sl], beta[sl]
        L = Q.shape[0]
        G = np.cumsum(gg)
        diff = G[:, None] - G[None, :]
        mask = np.tril(np.ones((L, L), dtype=bool))
        Gam = np.where(mask, np.exp(np.where(mask, diff, 0.0)), 0.0)
        A = np.tril(bb[:, None] * Gam * (K @ K.T), -1)
        Tm = np.linalg.inv(np.eye(L) + A)
        W = Tm @ ((bb * np.exp(G))[:, None] * K)
        Ut = Tm @ (bb[:, None] * V)
        U = Ut - W @ S.T
        O[sl] = np.exp(G)[:, None] * (Q @ S.T) + ((Q @ K.T) * Gam) @ U
        S = np.exp(G[-1]) * S + U.T @ (np.exp(G[-1] - G)[:, None] * K)
    return O, S


@pytest.mark.parametrize("T,C", [(64, 64), (150, 64), (37, 16), (200, 32)])
def test_chunked_form_matches_recurrence(T, C):
    rng = np.random.default_rng(T + C)
    D = 16
    q = rng.standard_normal((T, 1, D)).astype(np.float32)
    k = rng.standard_normal((T, 1, D)).astype(np.float32)
    v = rng.standard_normal((T, 1, D)).astype(np.float32)
    a = rng.standard_normal((T, 1)).astype(np.float32)
    b = rng.standard_normal((T, 1)).astype(np.float32)
    A_log, dt = [float(np.float32(math.log(2.5)))], [float(np.float32(0.1))]  # fp32 gate inputs
    S0 = rng.standard_normal((1, 1, D, D)) * 0.1
    o, S = _scan(q, k, v, a, b, A_log, dt, initial_state=S0, scale=0.5)
    qq = q[:, 0].astype(np.float64)
    kk = k[:, 0].astype(np.float64)
    qh = 0.5 * qq / np.sqrt((qq ** 2).sum(-1, keepdims=True) + oracle.EPS_QK)
    kh = kk / np.sqrt((kk ** 2).sum(-1, keepdims=True) + oracle.EPS_QK)
    at = torch.tensor(a[:, 0].astype(np.float64) + dt[0])
    g = (-math.exp(A_log[0]) * torch.nn.functional.softplus(at)).numpy()
    beta = torch.sigmoid(torch.tensor(b[:, 0].astype(np.float64))).numpy()
    Oc, Sc = _chunked_reference(qh, kh, v[:, 0].astype(np.float64), g, beta, S0[0, 0], C)
    np.testing.assert_allclose(o[:, 0], Oc, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(S[0, 0], Sc, rtol=1e-10, atol=1e-11)


def test_prefix_suffix_composition_and_single_steps():
    w = workloads.custom("c", (70,), 2, 4, 16, io="f32", s0_std=0.1, seed=11)
    x = workloads.generate(w)
    args = [x[n] for n in ("q", "k", "v", "a", "b", "A_log", "dt_bias")]
    o, S = _scan(*args, initial_state=x["initial_state"])
    t = 29
    o1, S1 = _scan(*[y[:t] for y in args[:5]], *args[5:], initial_state=x["initial_state"])
    o2, S2 = _scan(*[y[t:] for y in args[:5]], *args[5:], initial_state=S1)
    np.testing.assert_allclose(np.concatenate([o1, o2]), o, rtol=0, atol=0)
    np.testing.assert_allclose(S2, S, rtol=0, atol=0)
    Sd = x["initial_state"].astype(np.float64)
    for tt in range(70):
        od, Sd = _scan(*[y[tt:tt + 1] for y in args[:5]], *args[5:], initial_state=Sd)
        np.testing.assert_array_equal(od[0], o[tt])
    np.testing.assert_array_equal(Sd, S)


def test_gqa_mapping_equals_duplicated_keys():
    w = workloads.custom("g", (33,), 2, 6, 8, io="f32", seed=12)
    x = workloads.generate(w)
    o, S = _scan(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"])
    idx = np.arange(6) // 3
    o2, S2 = _scan(x["q"][:, idx], x["k"][:, idx], x["v"], x["a"], x["b"], x["A_log"],
                   x["dt_bias"])
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(S, S2)


def test_varlen_equals_separate_runs():
    w = workloads.custom("v", (5, 1, 40, 17), 1, 2, 8, io="f32", s0_std=0.1, seed=13)
    x = workloads.generate(w)
    o, S = _scan(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                 cu_seqlens=x["cu_seqlens"], initial_state=x["initial_state"])
    cu = x["cu_seqlens"]
    for n in range(4):
        sl = slice(cu[n], cu[n + 1])
        on, Sn = _scan(x["q"][sl], x["k"][sl], x["v"][sl], x["a"][sl], x["b"][sl], x["A_log"],
                       x["dt_bias"], initial_state=x["initial_state"][n:n + 1])
        np.testing.assert_array_equal(o[sl], on)
        np.testing.assert_array_equal(S[n], Sn[0])


# ------------------------------------------------------------------------- tail ----

def test_gated_norm_shared_weight_head_permutation():
    rng = np.random.default_rng(20)
    M, H, D = 5, 4, 128
    o = rng.standard_normal((M, H, D)).astype(np.float32)
    z = rng.standard_normal((M, H, D)).astype(np.float32)
    w = rng.uniform(0.5, 1.5, D).astype(np.float32)
    y = oracle.gated_rmsnorm_silu(o, z, w).reshape(M, H, D)
    perm = rng.permutation(H)
    yp = oracle.gated_rmsnorm_silu(o[:, perm], z[:, perm], w).reshape(M, H, D)
    np.testing.assert_array_equal(yp, y[:, perm])


def test_gated_norm_reduces_to_torch_rms_norm():
    rng = np.random.default_rng(21)
    M, H, D = 3, 2, 128
    o = rng.standard_normal((M, H, D)).astype(np.float32)
    z = np.full((M, H, D), BIG, dtype=np.float32)
    w = np.ones(D, dtype=np.float32)
    y = oracle.gated_rmsnorm_silu(o, z, w, eps=1e-6).reshape(M, H, D)
    ref = torch.nn.functional.rms_norm(torch.tensor(o, dtype=torch.float64), (D,), eps=1e-6) * BIG
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-13)


def test_gated_norm_mean_square_identity():
    rng = np.random.default_rng(22)
    M, H, D = 4, 3, 128
    o = rng.standard_normal((M, H, D)).astype(np.float32)
    z = rng.standard_normal((M, H, D)).astype(np.float32) + 3.0
    w = rng.uniform(0.5, 1.5, D).astype(np.float32)
    y = oracle.gated_rmsnorm_silu(o, z, w, eps=1e-6).reshape(M, H, D)
    silu = z.astype(np.float64) / (1.0 + np.exp(-z.astype(np.float64)))
    r = y / (w.astype(np.float64) * silu)
    ms = (o.astype(np.float64) ** 2).mean(-1)
    np.testing.assert_allclose((r ** 2).mean(-1), ms / (ms + 1e-6), rtol=1e-12)


# ------------------------------------------------------------------------ NVFP4 ----

def test_e4m3_decode_matches_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    got = oracle.e4m3_decode(codes)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    m = ~np.isnan(ref)
    assert np.array_equal(ref[m], got[m])


def test_e4m3_encode_matches_torch_rounding():
    rng = np.random.default_rng(30)
    vals = np.sort(oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8)))
    mids = (vals[:-1].astype(np.float64) + vals[1:]) / 2
    mids = mids.astype(np.float32)
    near = np.concatenate([np.nextafter(mids, np.float32(0)), mids,
                           np.nextafter(mids, np.float32(1000))])
    rand = np.exp(rng.uniform(math.log(1e-4), math.log(448.0), 200000)).astype(np.float32)
    bf = torch.arange(0, 0x43E0, dtype=torch.int16).view(torch.bfloat16).float().numpy()
    x = np.concatenate([vals, near, rand, bf[(bf >= 0) & (bf <= 448)], [0.0, 1e-30, 448.0]])
    x = x.astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(x)
    assert np.array_equal(ref, got)
    # satfinite: above the largest finite value the scale saturates to 448 (0x7E)
    assert np.all(oracle.e4m3_encode(np.array([449.0, 464.0, 1e6, 3e38], np.float32)) == 0x7E)


def test_e2m1_grid_and_thresholds():
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(oracle.e2m1_decode(np.arange(8))) == grid
    assert list(oracle.e2m1_decode(np.arange(8, 16))) == [-g for g in grid]
    for c in range(16):
        assert oracle.e2m1_encode(oracle.e2m1_decode([c]))[0] == c
    # decision points of round-to-nearest-even over {0,.5,1,1.5,2,3,4,6}:
    # (boundary, code at the boundary (tie -> even code), code below, code above)
    table = [(0.25, 0, 0, 1), (0.75, 2, 1, 2), (1.25, 2, 2, 3), (1.75, 4, 3, 4),
             (2.5, 4, 4, 5), (3.5, 6, 5, 6), (5.0, 6, 6, 7)]
    for bnd, at, below, above in table:
        f = np.float32(bnd)
        x = np.array([f, np.nextafter(f, np.float32(0)), np.nextafter(f, np.float32(10))],
                     dtype=np.float32)
        got = oracle.e2m1_encode(x)
        assert list(got) == [at, below, above], bnd
        assert list(oracle.e2m1_encode(-x)) == [at | 8, below | 8, above | 8]
    assert list(oracle.e2m1_encode(np.array([6.5, 1e9, -7.0], np.float32))) == [7, 7, 15]
    assert list(oracle.e2m1_encode(np.array([0.0, -0.0, -0.1], np.float32))) == [0, 8, 8]


def test_nvfp4_nibble_order_and_scale_layout():
    # one block with amax 6 and gs = 1: scale 1.0 (E4M3 0x38), codes are the grid values
    x = np.zeros((1, 32), np.float32)
    x[0, :16] = [1.0, 6.0, 0.5, -2.0] + [0.0] * 12
    x[0, 16:] = [3.0] + [0.0] * 15
    xq, xs = oracle.nvfp4_quantize(x, 1.0)
    assert xs.shape == (1, 2) and xq.shape == (1, 16)
    assert xs[0, 0] == 0x38          # 1.0
    assert xq[0, 0] == (2 | (7 << 4))      # element 0 -> low nibble, element 1 -> high
    assert xq[0, 1] == (1 | ((4 | 8) << 4))
    # block 2: amax 3 -> s = 0.5 (0x30); 3 * (1 / 0.5) = 6 -> code 7
    assert xs[0, 1] == 0x30 and xq[0, 8] == 7


def _scale_order_cases():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_scale_order.txt")
    cases = []
    with open(path) as fh:
        for line in fh:
            if line.strip() and not line.startswith("#"):
                amax, gs_bits, want, alt1, alt2 = line.split()
                gs = np.array([int(gs_bits, 16)], np.uint32).view(np.float32)[0]
                cases.append((float(amax), gs, int(want, 16), int(alt1, 16), int(alt2, 16)))
    return cases


@pytest.mark.parametrize("case", _scale_order_cases())
def test_nvfp4_block_scale_order_of_operations(case):
    """The block scale is (amax / 6) * gs in two fp32 roundings, then E4M3 ties-to-even
    (tests/golden/nvfp4_scale_order.txt): each case sits on an E4M3 tie, where the other orders
    of the same operations give a different code, so a wrong order fails here."""
    amax, gs, want, alt1, alt2 = case
    # the fixture's three codes, re-derived with torch's fp32 arithmetic and its E4M3 rounding
    t = lambda x: torch.tensor(x, dtype=torch.float32)
    e4 = lambda s: int(s.reshape(1).to(torch.float8_e4m3fn).view(torch.uint8)[0])
    a, g = t(amax), t(float(gs))
    assert e4((a / 6.0) * g) == want
    assert e4(a * (g / 6.0)) == alt1 and e4((a * g) / 6.0) == alt2
    assert want != alt1 and want != alt2
    # the oracle on one block whose largest magnitude is amax (the sign must not matter)
    x = np.zeros((2, 16), np.float32)
    x[0, :4] = [0.25 * amax, -amax, 0.5, 0.0]
    x[1, 7] = amax
    xq, xs = oracle.nvfp4_quantize(x, gs)
    assert int(xs[0, 0]) == want and int(xs[1, 0]) == want


def test_nvfp4_exact_round_trip_of_grid_values():
    rng = np.random.default_rng(31)
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float32)
    M, K = 64, 256
    codes = rng.integers(0, 8, size=(M, K))
    sign = np.where(rng.random((M, K)) < 0.5, -1.0, 1.0).astype(np.float32)
    x = grid[codes] * sign
    x.reshape(M, K // 16, 16)[:, :, 3] = 6.0            # every block's amax is 6
    e = rng.integers(-9, 9, size=(M, K // 16, 1)).astype(np.float32)
    x = (x.reshape(M, K // 16, 16) * np.exp2(e)).reshape(M, K).astype(np.float32)
    xq, xs = oracle.nvfp4_quantize(x, 1.0)
    back = oracle.nvfp4_dequantize(xq, xs, 1.0)
    np.testing.assert_array_equal(back, x.astype(np.float64))


def test_nvfp4_block_error_bound():
    x = workloads.activations(128, 512, seed=32)
    amax = float(np.abs(x).max())
    gs = np.float32(448.0 * 6.0 / amax)
    xq, xs = oracle.nvfp4_quantize(x, gs)
    back = oracle.nvfp4_dequantize(xq, xs, gs)
    sc = oracle.e4m3_decode(xs.ravel()).reshape(xs.shape).astype(np.float64) / float(gs)
    step = np.repeat(sc, 16, axis=1)        # dequant step of each element's block
    ax = np.abs(x.astype(np.float64))
    with np.errstate(divide="ignore", invalid="ignore"):
        rel = np.where(step > 0, ax / step, 0.0)
    half_gap = np.where(rel <= 2, 0.25, np.where(rel <= 4, 0.5, 1.0))
    bound = np.where(rel <= 6, half_gap, rel - 6.0) * step
    err = np.abs(back - x)
    assert np.all(err <= bound * (1 + 1e-6) + 1e-300)
    # where the block scale is a normal E4M3 (code >= 8) it is at most 2^-4 below amax / 6,
    # so no scaled value passes 6 / (1 - 2^-4); subnormal scales round more coarsely
    normal = np.repeat(xs >= 8, 16, axis=1)
    assert np.all(rel[normal] <= 6.0 / (1 - 2.0 ** -4) + 1e-9)
    assert normal.mean() > 0.9
    # all-zero blocks get a zero scale and zero codes
    zero_blocks = np.all(x.reshape(128, 32, 16) == 0, axis=2)
    assert zero_blocks.any()
    assert np.all(xs[zero_blocks] == 0)


def test_nvfp4_gemm_brute_force_exact():
    """Oracle GEMM (fp64 product of dequantised operands) against an exact rational
    triple loop over the codes and scales."""
    rng = np.random.default_rng(33)
    for (M, N, K) in [(3, 2, 32), (64, 16, 32)]:
        A = workloads.activations(M, K, seed=int(rng.integers(1 << 30)))
        B = workloads.round_bf16(rng.standard_normal((N, K)).astype(np.float32) * 0.02)
        gsa = np.float32(448 * 6 / np.abs(A).max())
        gsb = np.float32(448 * 6 / np.abs(B).max())
        aq, as_ = oracle.nvfp4_quantize(A, gsa)
        bq, bs = oracle.nvfp4_quantize(B, gsb)
        Y = oracle.nvfp4_gemm(aq, as_, gsa, bq, bs, gsb)
        grid = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2),
                Fraction(3), Fraction(4), Fraction(6)]

        def val(q, s, r, kk):
            byte = int(q[r, kk // 2])
            c = (byte >> 4) if kk % 2 else (byte & 15)
            m = grid[c & 7] * (-1 if c & 8 else 1)
            return m * Fraction(float(torch.tensor(int(s[r, kk // 16]), dtype=torch.uint8)
                                      .view(torch.float8_e4m3fn).float()))
        rows = range(M) if M <= 3 else [0, 17, 63]
        for i in rows:
            for j in range(N):
                acc = sum(val(aq, as_, i, kk) * val(bq, bs, j, kk) for kk in range(K))
                exact = acc / (Fraction(float(gsa)) * Fraction(float(gsb)))
                assert Y[i, j] == pytest.approx(float(exact), rel=1e-13, abs=1e-13)


# --------------------------------------------------------------- page facts ----

def test_tail_shapes_from_the_pages():
    """The gated tail of page 3 maps 32 value heads x 128 -> 4096 -> 2048 with one F32 [128]
    norm weight (golden/tail_shapes.txt)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tail_shapes.txt")
    facts = {}
    for line in open(path):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = line.split("=")
            facts[k.strip()] = int(v)
    w = workloads.PREFILL_LONG
    assert w.Hv == facts["value_heads"] and w.D == facts["head_dim"]
    assert w.K == facts["flat_width"] and w.n_out == facts["hidden"]
    x = workloads.generate(workloads.custom("t", (2,), 16, facts["value_heads"],
                                            facts["head_dim"], seed=3, n_out=facts["hidden"]))
    assert x["norm_weight"].shape == (facts["norm_weight_len"],)
    y = oracle.gated_rmsnorm_silu(x["v"], x["z"], x["norm_weight"])
    assert y.shape == (2, facts["flat_width"])
    aq, as_ = oracle.nvfp4_quantize(y.astype(np.float32), 1.0)
    assert as_.shape[1] * facts["nvfp4_block"] == facts["flat_width"]
