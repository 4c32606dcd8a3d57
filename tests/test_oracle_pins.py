"""Pins of the fp64 oracle against things other than itself (CPU only).

Each pin is chosen so that a plausible slip in the oracle -- a dropped term, a
wrong sign, a transposed operand, a wrong rounding -- fails at least one of
them; ``test_planted_mistakes_are_caught`` plants such slips in a copy of the
oracle source and checks exactly that.
"""
import os
import shutil
import struct
import subprocess
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import l2model
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------- bf16


def _torch_bf16_bits_of_f32(vals_f32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(vals_f32.astype(np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_bf16_decode_exhaustive_matches_torch():
    """Every one of the 65,536 bf16 patterns decodes to the value torch gives."""
    bits = np.arange(65536, dtype=np.uint16)
    ours = oracle.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_bf16_round_trip_exhaustive():
    """decode -> round is the identity on every non-NaN pattern (signed zeros kept)."""
    bits = np.arange(65536, dtype=np.uint16)
    vals = oracle.bf16_to_f64(bits)
    back = oracle.round_bf16(vals)
    nan = np.isnan(vals)
    assert np.array_equal(back[~nan], bits[~nan])
    assert np.all((back[nan] & 0x7FFF) > 0x7F80)  # NaN stays NaN


def test_rne_matches_torch_on_fp32_values():
    """On values exactly representable in fp32, rounding straight from fp64
    must agree with torch's fp32->bf16 conversion (round to nearest even)."""
    rng = np.random.default_rng(1)
    vals = rng.standard_normal(200000).astype(np.float32) * np.float32(3.0)
    # exact midpoints between neighbouring bf16 values (ties), and their neighbours
    base = rng.integers(0, 0x7F7F, 50000).astype(np.uint32)
    lo = (base << 16).view(np.float32)
    hi = ((base + 1) << 16).view(np.float32)
    mid = ((lo.astype(np.float64) + hi.astype(np.float64)) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (lo.astype(np.float64) + hi.astype(np.float64)) / 2)
    up = np.nextafter(mid, np.float32(np.inf))
    dn = np.nextafter(mid, np.float32(-np.inf))
    edge = np.array([0.0, -0.0, 1e-40, -1e-40, 1e-45, 3.3895314e38, -3.3895314e38,
                     3.4e38, np.float32(3.4028235e38)], dtype=np.float32)
    allv = np.concatenate([vals, mid, -mid, up, dn, edge])
    ours = oracle.round_bf16(allv.astype(np.float64))
    ref = _torch_bf16_bits_of_f32(allv)
    assert np.array_equal(ours, ref)


def test_rne_ties_go_to_even():
    """Constructed halfway cases: 1 + 2^-8 lies between 1 (even) and 1 + 2^-7
    (odd) and must round down; 1 + 3*2^-8 lies between 1 + 2^-7 (odd) and
    1 + 2^-6 (even) and must round up."""
    r = oracle.round_bf16(np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2 ** 128, -(2 ** 128)]))
    assert list(r) == [0x3F80, 0x3F82, 0xBF80, 0x7F80, 0xFF80]


def test_rne_overflow_threshold():
    """Largest finite bf16 is (2 - 2^-7) 2^127; the midpoint to 2^128 rounds to inf."""
    maxf = (2 - 2 ** -7) * 2.0 ** 127
    mid = (2 - 2 ** -8) * 2.0 ** 127
    r = oracle.round_bf16(np.array([maxf, np.nextafter(mid, 0), mid]))
    assert list(r) == [0x7F7F, 0x7F7F, 0x7F80]


def test_rne_double_values_not_fp32():
    """Rounding is done once, from fp64: a value just above a bf16 midpoint by
    less than fp32 resolution must round up (double rounding through fp32
    would land on the midpoint and round to even instead)."""
    v = 1 + 2 ** -8 + 2 ** -40
    assert oracle.round_bf16(np.array([v]))[0] == 0x3F81
    assert _torch_bf16_bits_of_f32(np.array([v], dtype=np.float32))[0] == 0x3F80


# --------------------------------------------------------------------------- GEMM


def _exact_gemm(X, W):
    """Exact rational product over the bf16 values (brute force)."""
    xf = X.to(torch.float64).numpy()
    wf = W.to(torch.float64).numpy()
    M, K = xf.shape
    N = wf.shape[0]
    out = [[sum((Fraction(float(xf[m, k])) * Fraction(float(wf[n, k])) for k in range(K)), Fraction(0))
            for n in range(N)] for m in range(M)]
    return out


def _rne_exact(q: Fraction) -> int:
    """bf16 RNE of an exact rational, by exhaustive neighbour search."""
    if q == 0:
        return 0
    sign = 0x8000 if q < 0 else 0
    a = abs(q)
    # bracket with float, then check neighbours exactly
    cand = int(oracle.round_bf16(np.array([float(a)]))[0])
    best = None
    for c in (cand - 1, cand, cand + 1):
        if c < 0 or c >= 0x7F80:
            continue
        v = Fraction(struct.unpack("<f", struct.pack("<I", c << 16))[0])
        d = abs(v - a)
        key = (d, c & 1)  # nearest, ties to even significand
        if best is None or key < best[0]:
            best = (key, c)
    return sign | best[1]


@pytest.mark.parametrize("M,N,K,seed", [(1, 1, 1, 0), (1, 3, 16, 1), (2, 4, 64, 2), (4, 4, 64, 3), (3, 2, 40, 4)])
def test_brute_force_exact(M, N, K, seed):
    """Tiny shapes whose fp64 sums are exact: the oracle equals the exact
    rational product, and its single rounding equals the exact RNE."""
    X, W = synth.make_binade_xw(M, N, K, seed)
    Y, S = oracle.gemm_ref(X, W)
    ex = _exact_gemm(X, W)
    for m in range(M):
        for n in range(N):
            assert Fraction(Y[m, n]) == ex[m][n]
    rb = oracle.round_bf16(Y)
    for m in range(M):
        for n in range(N):
            assert int(rb[m, n]) == _rne_exact(ex[m][n])
    # S is the sum of |products|
    sabs = [[sum(abs(Fraction(float(a)) * Fraction(float(b))) for a, b in
                 zip(X[m].double().tolist(), W[n].double().tolist())) for n in range(N)] for m in range(M)]
    for m in range(M):
        for n in range(N):
            assert Fraction(S[m, n]) == sabs[m][n]


@pytest.mark.parametrize("M,N,K", [(1, 17, 96), (5, 33, 257 * 8), (8, 64, 1024), (16, 40, 4096)])
def test_integer_inputs_match_int64_matmul(M, N, K):
    X, W = synth.make_int_xw(M, N, K, seed=M + N)
    Y, S = oracle.gemm_ref(X, W)
    xi = X.to(torch.int64).numpy()
    wi = W.to(torch.int64).numpy()
    assert np.array_equal(Y, (xi @ wi.T).astype(np.float64))
    assert np.array_equal(S, (np.abs(xi) @ np.abs(wi).T).astype(np.float64))


def test_identity_and_permutation():
    K = 256
    X, _ = synth.make_xw(4, K, K, seed=7)
    I = torch.eye(K, dtype=torch.bfloat16)
    Y, _ = oracle.gemm_ref(X, I)
    assert np.array_equal(Y, X.to(torch.float64).numpy())
    P, p = synth.make_permutation_w(K, seed=3)
    Y, _ = oracle.gemm_ref(X, P)
    # Y[m, n] = X[m, p[n]]
    assert np.array_equal(Y, X.to(torch.float64).numpy()[:, p.numpy()])


def test_onehot_rows_select_w_rows():
    M, N, K = 6, 50, 384
    X, idx = synth.make_onehot_x(M, K, seed=5)
    _, W = synth.make_xw(1, N, K, seed=9)
    Y, _ = oracle.gemm_ref(X, W)
    assert np.array_equal(Y, W.to(torch.float64).numpy()[:, idx.numpy()].T)


@pytest.mark.parametrize("K", [1, 8, 64, 256])
def test_all_ones_gives_k(K):
    X = torch.ones(3, K, dtype=torch.bfloat16)
    W = torch.ones(5, K, dtype=torch.bfloat16)
    Y, _ = oracle.gemm_ref(X, W)
    assert np.all(Y == K)
    assert np.all(oracle.round_bf16(Y) == _torch_bf16_bits_of_f32(np.full(1, K, np.float32))[0])


def test_linearity_exact_on_integers():
    M, N, K = 4, 48, 512
    X1, W = synth.make_int_xw(M, N, K, seed=11)
    X2, _ = synth.make_int_xw(M, N, K, seed=12)
    Y1, _ = oracle.gemm_ref(X1, W)
    Y2, _ = oracle.gemm_ref(X2, W)
    Y12, _ = oracle.gemm_ref((X1.float() + X2.float()).to(torch.bfloat16), W)
    assert np.array_equal(Y12, Y1 + Y2)


@pytest.mark.parametrize("M,N,K", [(1, 300, 4096), (8, 129, 1000), (16, 64, 12288)])
def test_random_matches_numpy_fp64_within_bound(M, N, K):
    """Against numpy's fp64 product (a library routine with another summation
    order): both are within K * 2^-53 * S of the exact value."""
    X, W = synth.make_xw(M, N, K, seed=M)
    Y, S = oracle.gemm_ref(X, W)
    ref = X.to(torch.float64).numpy() @ W.to(torch.float64).numpy().T
    bound = 2 * K * 2.0 ** -53 * S + 1e-300
    assert np.all(np.abs(Y - ref) <= bound)
    sref = np.abs(X.to(torch.float64).numpy()) @ np.abs(W.to(torch.float64).numpy()).T
    assert np.all(np.abs(S - sref) <= bound)


def test_sampled_equals_full():
    M, N, K = 7, 91, 777 * 8
    X, W = synth.make_xw(M, N, K, seed=4)
    Y, S = oracle.gemm_ref(X, W)
    rng = np.random.default_rng(0)
    ms = rng.integers(0, M, 200)
    ns = rng.integers(0, N, 200)
    Ys, Ss = oracle.gemm_ref_sampled(X, W, ms, ns)
    assert np.array_equal(Ys, Y[ms, ns])
    assert np.array_equal(Ss, S[ms, ns])


def test_thread_count_does_not_change_results():
    X, W = synth.make_xw(4, 257, 4096, seed=2)
    prev = oracle.set_threads(0)
    oracle.set_threads(1)
    Y1, S1 = oracle.gemm_ref(X, W)
    oracle.set_threads(max(2, os.cpu_count() or 2))
    Y2, S2 = oracle.gemm_ref(X, W)
    oracle.set_threads(prev)
    assert np.array_equal(Y1, Y2) and np.array_equal(S1, S2)


def test_chain_ref_is_per_task():
    tasks = [synth.make_xw(2, 40, 64, seed=s) for s in range(3)]
    outs = oracle.chain_ref(tasks)
    for (X, W), (Y, S) in zip(tasks, outs):
        Y1, S1 = oracle.gemm_ref(X, W)
        assert np.array_equal(Y, Y1) and np.array_equal(S, S1)


def test_synth_recipe():
    """The input recipe: one generator draws X then W; W has std 1/sqrt(K)."""
    X, W = synth.make_xw(3, 4096, 1024, seed=0)
    g = torch.Generator().manual_seed(0)
    x = torch.randn(3, 1024, generator=g)
    w = torch.randn(4096, 1024, generator=g) / 32.0
    assert torch.equal(X, x.to(torch.bfloat16)) and torch.equal(W, w.to(torch.bfloat16))
    assert abs(W.float().std().item() - 1 / 32.0) < 1e-3
    # chain task seeds
    lay = synth.chain_layout(layers=2, M=16)
    assert [c.seed for c in lay] == list(range(8))
    assert [(c.K, c.N) for c in lay[:4]] == [(4096, 6144), (4096, 4096), (4096, 24576), (12288, 4096)]


# --------------------------------------------------------------------------- Eq.(1)


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(v) for v in line.split()])
    return rows


def test_eq1_worked_table():
    for B, mt, R, pct in _read_table("eq1_l2_hit_table.txt"):
        B, mt, R = int(B), int(mt), int(R)
        assert l2model.m_tiles(B, 16) == mt
        assert l2model.sharers(B, 31, 16) == R
        assert l2model.weight_hit(B, 31, 16) == Fraction(int(pct), 100)


def test_eq1_limits_and_monotone():
    # B -> infinity: hit -> (W-1)/W = 30/31
    assert l2model.weight_hit(10 ** 6, 31, 16) == Fraction(30, 31)
    prev = Fraction(0)
    for B in range(1, 2000, 7):
        h = l2model.weight_hit(B, 31, 16)
        assert h >= prev
        prev = h


def test_ai_eff_worked_values():
    for B, pct, printed, tol in _read_table("eq1_ai_eff.txt"):
        v = l2model.ai_eff(int(B), Fraction(int(pct), 100))
        assert abs(v - printed) <= tol * printed + 1e-12


def test_one_hbm_fetch_per_column():
    for B in (16, 32, 64):
        for tm in (16, 32):
            assert l2model.hbm_weight_bytes(1000, B, 31, tm) == 1000


# --------------------------------------------------------------------------- mutations


MUTATIONS = {
    # transposed operand: index W by (k, n) instead of (n, k)
    "transposed_w": ("const uint16_t *wr = W + (size_t)n * K;\n        double acc = 0.0, sabs = 0.0;\n        for (int k = 0; k < K; ++k) {\n            double p = wsmo_bf16_to_f64(xr[k]) * wsmo_bf16_to_f64(wr[k]);",
                     "const uint16_t *wr = W + (size_t)n;\n        double acc = 0.0, sabs = 0.0;\n        for (int k = 0; k < K; ++k) {\n            double p = wsmo_bf16_to_f64(xr[k]) * wsmo_bf16_to_f64(wr[(size_t)k * N]);"),
    # dropped last term
    "dropped_term": ("for (int k = 0; k < K; ++k) {\n            double p = wsmo_bf16_to_f64(xr[k]) * wsmo_bf16_to_f64(wr[k]);\n            acc += p;\n            sabs += fabs(p);\n        }\n        Y_ref[idx] = acc;",
                     "for (int k = 0; k < K - 1; ++k) {\n            double p = wsmo_bf16_to_f64(xr[k]) * wsmo_bf16_to_f64(wr[k]);\n            acc += p;\n            sabs += fabs(p);\n        }\n        Y_ref[idx] = acc;"),
    # sign slip
    "sign": ("acc += p;\n            sabs += fabs(p);\n        }\n        Y_ref[idx] = acc;",
             "acc -= p;\n            sabs += fabs(p);\n        }\n        Y_ref[idx] = acc;"),
    # rounding: ties away from zero instead of to even
    "ties_away": ("if (frac > 0.5 || (frac == 0.5 && fmod(n, 2.0) != 0.0))", "if (frac >= 0.5)"),
    # rounding: truncation
    "truncate": ("if (frac > 0.5 || (frac == 0.5 && fmod(n, 2.0) != 0.0))", "if (0)"),
    # decode: wrong shift (fp16-like placement)
    "decode_shift": ("uint32_t bits = (uint32_t)h << 16;", "uint32_t bits = (uint32_t)h << 13;"),
}


def _pins_pass(lib) -> bool:
    """A compact run of the pins above against a given oracle build."""
    try:
        # decode + round trip
        bits = np.arange(0, 65536, 7, dtype=np.uint16)
        vals = np.array([lib.wsmo_bf16_to_f64(int(b)) for b in bits])
        ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
        ok = np.isnan(ref)
        if not np.array_equal(vals[~ok], ref[~ok]):
            return False
        r = oracle.round_bf16(np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -9 * 3]), lib=lib)
        if list(r) != [0x3F80, 0x3F82, 0x3F81]:
            return False
        # integer product
        X, W = synth.make_int_xw(3, 20, 64, seed=1)
        Y, _ = oracle.gemm_ref(X, W, lib=lib)
        if not np.array_equal(Y, (X.to(torch.int64).numpy() @ W.to(torch.int64).numpy().T).astype(np.float64)):
            return False
        # permutation
        Xp, _ = synth.make_xw(2, 64, 64, seed=2)
        P, p = synth.make_permutation_w(64, seed=3)
        Y, _ = oracle.gemm_ref(Xp, P, lib=lib)
        if not np.array_equal(Y, Xp.to(torch.float64).numpy()[:, p.numpy()]):
            return False
        return True
    except Exception:
        return False


def test_pins_pass_on_real_oracle():
    assert _pins_pass(oracle.load())


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes_are_caught(name, tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc missing")
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()
    old, new = MUTATIONS[name]
    assert old in src, f"mutation anchor for {name} not found in oracle.c"
    mutated = tmp_path / f"oracle_{name}.c"
    mutated.write_text(src.replace(old, new, 1))
    so = tmp_path / f"liboracle_{name}.so"
    subprocess.run(["gcc", *oracle.CFLAGS, "-o", str(so), str(mutated), "-lm"], check=True)
    lib = oracle.load(str(so))
    assert not _pins_pass(lib), f"planted mistake '{name}' was not caught by the pins"


# --------------------------------------------------------------------------- fused epilogues
#
# The pins below take the functions under test as parameters, so the same pins
# can be run against deliberately wrong variants (planted in the test, on the
# CPU) to show that each plausible slip is caught.

SIGMOID_1 = 0.7310585786300049          # logistic(1) = e / (1 + e), to 16 digits


def _silu_pins(silu):
    z = np.random.default_rng(0).normal(0, 4, 4096)
    if silu(np.array([0.0]))[0] != 0.0:
        return False
    if abs(silu(np.array([1.0]))[0] - SIGMOID_1) > 1e-15:
        return False
    # silu(z) - silu(-z) = z  (sigmoid(z) + sigmoid(-z) = 1)
    if np.max(np.abs(silu(z) - silu(-z) - z) / np.maximum(1.0, np.abs(z))) > 1e-14:
        return False
    big = silu(np.array([40.0, 1000.0, -40.0, -1000.0]))
    if not (abs(big[0] - 40.0) < 1e-14 and big[1] == 1000.0 and abs(big[2]) < 1e-15 and big[3] == 0.0):
        return False
    return not np.isnan(big).any()


def _interleave_by_reshape(Wg, Wu):
    """Fused gate+up weight built independently of gate_up_rows: blocks of 8
    gate rows then the matching 8 up rows."""
    I, K = Wg.shape
    g = Wg.reshape(I // 8, 8, K)
    u = Wu.reshape(I // 8, 8, K)
    return torch.stack([g, u], dim=1).reshape(2 * I, K).contiguous()


def _silu_mul_pins(silu_mul_ref):
    M, I, K = 3, 32, 96
    X, Wg = synth.make_xw(M, I, K, seed=70)
    _, Wu = synth.make_xw(1, I, K, seed=71)
    H, G, U, Sg, Su = silu_mul_ref(X, _interleave_by_reshape(Wg, Wu))
    Gr, Sgr = oracle.gemm_ref(X, Wg)
    Ur, Sur = oracle.gemm_ref(X, Wu)
    if not (np.array_equal(G, Gr) and np.array_equal(U, Ur) and np.array_equal(Sg, Sgr) and np.array_equal(Su, Sur)):
        return False
    return np.array_equal(H, oracle.silu(Gr) * Ur)


def _residual_pins(residual_ref):
    X, W = synth.make_int_xw(3, 40, 64, seed=72)
    R = synth.make_x(3, 40, seed=73)                 # any bf16 [3, 40]
    Y, S = residual_ref(X, W, R)
    Y0, S0 = oracle.gemm_ref(X, W)
    # R widened exactly (torch's bf16 -> fp64) and added once
    if not np.array_equal(Y - Y0, R.to(torch.float64).numpy()) or not np.array_equal(S, S0):
        return False
    Yz, _ = residual_ref(X, W, torch.zeros(3, 40, dtype=torch.bfloat16))
    return np.array_equal(Yz, Y0)


def test_silu_pins():
    assert _silu_pins(oracle.silu)


def test_silu_mul_pins():
    assert _silu_mul_pins(oracle.silu_mul_ref)


def test_residual_pins():
    assert _residual_pins(oracle.residual_ref)


def test_gate_up_rows_cover_every_row_once():
    gi, ui = oracle.gate_up_rows(64)
    assert sorted(np.concatenate([gi, ui]).tolist()) == list(range(128))
    assert np.all(ui - gi == 8) and np.all((gi % 16) < 8)


def test_silu_derivative_bound():
    """The constant 1.1 of fused_bounds: |silu'| <= 1.1 on a fine grid (its
    extremes are ~1.0998 near z = 2.4 and ~-0.0998 near z = -2.4)."""
    z = np.linspace(-30, 30, 600001)
    d = np.gradient(oracle.silu(z), z)
    assert d.max() < 1.1 and d.min() > -1.1
    assert abs(d.max() - 1.0998) < 1e-3 and abs(d.min() + 0.0998) < 1e-3


def test_fused_bound_covers_perturbed_inputs():
    """Any G, U moved by at most their GEMM bounds changes silu(G) * U by no
    more than the silu_mul bound (corners of the box, many random points)."""
    rng = np.random.default_rng(5)
    G = rng.normal(0, 3, 20000)
    U = rng.normal(0, 3, 20000)
    Sg = np.abs(G) * rng.uniform(1, 50, G.size)
    Su = np.abs(U) * rng.uniform(1, 50, U.size)
    b = oracle.fused_bounds("silu_mul", G=G, U=U, Sg=Sg, Su=Su)
    H = oracle.silu(G) * U
    dg, du = 1e-3 * Sg + 1e-6, 1e-3 * Su + 1e-6
    for sg in (-1, 1):
        for su in (-1, 1):
            Hp = oracle.silu(G + sg * dg) * (U + su * du)
            assert np.all(np.abs(Hp - H) <= b)
    # the bound is not vacuous: the worst corner uses a good part of it
    Hp = np.maximum.reduce([np.abs(oracle.silu(G + a * dg) * (U + c * du) - H) for a in (-1, 1) for c in (-1, 1)])
    assert np.median(Hp / b) > 0.3


FUSED_MUTATIONS = {
    # exp(+z) instead of exp(-z)
    "silu_sign": ("silu", lambda z: np.asarray(z, np.float64) / (1.0 + np.exp(np.asarray(z, np.float64)))),
    # sigmoid without the factor z
    "silu_no_z": ("silu", lambda z: 1.0 / (1.0 + np.exp(-np.asarray(z, np.float64)))),
    # gate and up swapped
    "swap_gate_up": ("silu_mul", lambda X, W: (lambda Y, S: (
        oracle.silu(Y[:, oracle.gate_up_rows(Y.shape[1] // 2)[1]]) * Y[:, oracle.gate_up_rows(Y.shape[1] // 2)[0]],
        Y[:, oracle.gate_up_rows(Y.shape[1] // 2)[1]], Y[:, oracle.gate_up_rows(Y.shape[1] // 2)[0]],
        S[:, oracle.gate_up_rows(Y.shape[1] // 2)[1]], S[:, oracle.gate_up_rows(Y.shape[1] // 2)[0]]))(
        *oracle.gemm_ref(X, W))),
    # halves layout (gate rows first, then up rows) instead of blocks of 8
    "halves_layout": ("silu_mul", lambda X, W: (lambda Y, S, I: (
        oracle.silu(Y[:, :I]) * Y[:, I:], Y[:, :I], Y[:, I:], S[:, :I], S[:, I:]))(
        *oracle.gemm_ref(X, W), W.shape[0] // 2)),
    # residual dropped / subtracted
    "residual_dropped": ("residual", lambda X, W, R: oracle.gemm_ref(X, W)),
    "residual_sign": ("residual", lambda X, W, R: (lambda Y, S: (Y - R.to(torch.float64).numpy(), S))(
        *oracle.gemm_ref(X, W))),
}


@pytest.mark.parametrize("name", sorted(FUSED_MUTATIONS))
def test_fused_planted_mistakes_are_caught(name):
    kind, fn = FUSED_MUTATIONS[name]
    pins = {"silu": _silu_pins, "silu_mul": _silu_mul_pins, "residual": _residual_pins}[kind]
    assert not pins(fn), f"planted mistake '{name}' was not caught"
