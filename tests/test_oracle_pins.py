"""Pins of the CPU oracle against facts that do not come from the oracle itself:
the e4m3 format definition and torch's converter, hand-worked INT4 rows, fp64
means, algebraic identities of the two smoothing steps, fp64 attention (when
the quantizers are swapped for the identity), brute force on single tiles and
the N=1 / uniform-attention closed forms."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import sage2_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------- e4m3
def _torch_e4m3_decode_all():
    codes = torch.arange(256, dtype=torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_table_matches_torch_decoder():
    mine = orc.e4m3_value_table()
    ref = _torch_e4m3_decode_all()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert nan.sum() == 2                       # 0x7F and 0xFF only
    assert np.array_equal(mine[~nan], ref[~nan])


def test_e4m3_golden_points():
    for line in open(os.path.join(GOLDEN, "e4m3_points.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        val, code = line.split()[:2]
        got = int(orc.e4m3_encode(np.array([float(val)]))[0])
        assert got == int(code, 16), (val, hex(got), code)


def test_e4m3_roundtrip_all_codes():
    vals = orc.e4m3_value_table()
    for c in range(256):
        if np.isnan(vals[c]):
            continue
        back = int(orc.e4m3_encode(np.array([vals[c]]))[0])
        if vals[c] == 0:
            assert back in (0x00, 0x80)
        else:
            assert back == c


def test_e4m3_midpoints_round_to_even():
    vals = orc.e4m3_value_table()
    pos = sorted(set(v for v in vals if not np.isnan(v) and v >= 0))
    for a, b in zip(pos[:-1], pos[1:]):
        mid = (a + b) / 2
        got = orc.e4m3_decode(orc.e4m3_encode(np.array([mid])))[0]
        ca = int(orc.e4m3_encode(np.array([a]))[0])
        cb = int(orc.e4m3_encode(np.array([b]))[0])
        even = a if (ca & 1) == 0 else b
        assert (ca & 1) != (cb & 1)
        assert got == even, (a, b, got)


def test_e4m3_encode_matches_torch_converter_random():
    rng = np.random.default_rng(5)
    x = np.concatenate([
        rng.standard_normal(200000) * 50,
        rng.uniform(-464, 464, 100000),
        rng.standard_normal(100000) * 1e-3,
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = orc.e4m3_encode(x.astype(np.float64))
    # the two signed zeros are the same value
    same = (mine == ref) | (((mine & 0x7F) == 0) & ((ref & 0x7F) == 0))
    assert same.all(), x[~same][:10]


def test_e4m3_neighbours_differ_only_near_boundaries():
    # exactly representable -> one value; a boundary -> both neighbours
    lo, hi = orc.e4m3_neighbours(np.array([1.0, 1.0625, 368.0, 368.0 * (1 + 2 ** -10)]), 2 ** -12)
    assert lo[0] == hi[0] == 1.0
    assert (lo[1], hi[1]) == (1.0, 1.125)
    assert (lo[2], hi[2]) == (352.0, 384.0)
    assert lo[3] == hi[3] == 384.0


def _band_case(rng, n, d, cmag):
    """Random scores of one row as the kernel forms them: exact integer S,
    fp32 scales, a correction of magnitude cmag, and its error bound."""
    S = rng.integers(-49 * d // 4, 49 * d // 4 + 1, n).astype(np.float64)
    sq = np.float32(rng.uniform(0.05, 3.0))
    sk = rng.uniform(0.05, 3.0, n).astype(np.float32)
    C = (rng.standard_normal(n) * cmag).astype(np.float64)
    cb = d * orc.U32 * np.abs(C) * rng.uniform(1.0, 4.0, n)
    return S, sq, sk, C, cb


def _f32(x):
    return np.asarray(x, np.float64).astype(np.float32).astype(np.float64)


@pytest.mark.parametrize("seed", range(6))
def test_p448_band_covers_an_fp32_evaluation(seed):
    """The band must contain what an fp32 evaluation of the kernel's formula
    gives: sk*S and the fused multiply-add rounded to fp32, a correction
    anywhere within its error bound, the running maximum taken over the fp32
    scores, the argument x'L - mL + log2 448 in fp32 (L itself rounded), and
    an exp2 off by up to EX2_REL."""
    rng = np.random.default_rng(300 + seed)
    d = 128
    sm = 1.0 / math.sqrt(d) * rng.uniform(0.5, 4.0)
    L = sm * orc.LOG2E
    Lf = _f32(_f32(sm) * _f32(orc.LOG2E))
    worst = 0.0
    for _ in range(40):
        S, sq, sk, C, cb = _band_case(rng, 256, d, rng.choice([0.1, 10.0, 1000.0]))
        A = np.float64(sq) * sk.astype(np.float64) * S
        X = A + C
        M = np.array([X.max()])
        e_m = np.array([np.max(orc.U32 * (2 * np.abs(A) + np.abs(X)) + cb)])
        band_all = orc.p448_band(A[None], X[None], M, e_m, cb[None], L)[0]
        y = 448.0 * np.exp2(L * (X - M[0]))
        for trial in range(4):
            Cf = _f32(C + cb * rng.uniform(-1, 1, C.size))
            t = _f32(sk.astype(np.float64) * S)
            xk = _f32(np.float64(sq) * t + Cf)
            mk = xk.max()
            nb = _f32(_f32(orc.LOG2_448) - _f32(mk * Lf))
            arg = _f32(xk * Lf + nb)
            yk = np.exp2(arg) * (1 + orc.EX2_REL * rng.uniform(-1, 1, arg.size))
            live = y > 448.0 * 2.0 ** -40
            rel = np.abs(yk[live] / y[live] - 1)
            band = band_all[live]
            assert (rel <= band).all(), (rel / band).max()
            worst = max(worst, float((rel / band).max()))
    assert worst > 0.01          # the band is not vacuously wide


def test_p448_band_grows_with_each_error_source():
    A = np.array([[100.0]]); X = np.array([[90.0]]); M = np.array([95.0]); L = 0.2
    base = orc.p448_band(A, X, M, np.array([0.0]), np.array([[0.0]]), L)[0, 0]
    assert orc.p448_band(A, X, M, np.array([1e-3]), np.array([[0.0]]), L)[0, 0] > base
    assert orc.p448_band(A, X, M, np.array([0.0]), np.array([[1e-3]]), L)[0, 0] > base
    assert orc.p448_band(A * 10, X, M, np.array([0.0]), np.array([[0.0]]), L)[0, 0] > base
    assert base >= orc.EX2_REL


# --------------------------------------------------------------------- INT4
def test_int4_golden_rows():
    for line in open(os.path.join(GOLDEN, "int4_rows.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        xs, qs, sc = [s.split() for s in line.split("|")]
        x = np.array([float(v) for v in xs], np.float32)[None]
        q, s = orc.quant_int4_rows(x)
        assert q[0].tolist() == [int(v) for v in qs], (xs, q)
        assert s[0] == np.float32(float(sc[0]))


def test_int4_bounds_random():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((500, 128)) * rng.uniform(0.01, 100, (500, 1))).astype(np.float32)
    q, s = orc.quant_int4_rows(x)
    assert np.abs(q).max() <= 7
    err = np.abs(x.astype(np.float64) - q * s[:, None].astype(np.float64))
    assert (err <= s[:, None] * (0.5 + 1e-5)).all()
    # the element carrying the amax maps to +-7
    arg = np.abs(x).argmax(axis=1)
    assert (np.abs(q[np.arange(500), arg]) == 7).all()


# --------------------------------------------------------------- the means
def test_k_mean_close_to_fp64_mean():
    rng = np.random.default_rng(2)
    for N in (1, 127, 128, 129, 300, 1000):
        K = (rng.standard_normal((N, 64)) * 3 + 5).astype(np.float32)
        got = orc.k_mean(K).astype(np.float64)
        ref = K.astype(np.float64).mean(axis=0)
        assert np.allclose(got, ref, rtol=2e-6, atol=1e-6)


def test_k_mean_exact_on_integer_data():
    # integer sums are exact in fp32 and N a power of two makes /N exact
    rng = np.random.default_rng(3)
    K = rng.integers(-8, 9, (256, 32)).astype(np.float32)
    assert np.array_equal(orc.k_mean(K), (K.astype(np.float64).mean(0)).astype(np.float32))


def test_q_block_means_tail_uses_valid_rows_only():
    rng = np.random.default_rng(4)
    Q = rng.standard_normal((300, 64)).astype(np.float32)
    qb = orc.q_block_means(Q)
    assert qb.shape == (3, 64)
    for b, (r0, r1) in enumerate([(0, 128), (128, 256), (256, 300)]):
        assert np.allclose(qb[b], Q[r0:r1].astype(np.float64).mean(0), rtol=1e-5, atol=1e-6)


# ---------------------------------------------------- smoothing identities
def test_q_smoothing_reconstruction_fp64():
    """Q K_s^T = Q_s K_s^T + C - qbar.kbar (exact algebra, fp64)."""
    rng = np.random.default_rng(6)
    N, d = 300, 64
    Q = (rng.standard_normal((N, d)) + rng.normal(0, 2, d)).astype(np.float32)
    K = (rng.standard_normal((N, d)) + rng.normal(0, 3, d)).astype(np.float32)
    pay = orc.smooth_quant_qk(Q, K)
    C = orc.qk_correction(pay["q_mean"], K)
    qbar = pay["q_mean"].astype(np.float64)
    kbar = pay["k_mean"].astype(np.float64)
    blk = np.arange(N) // orc.BM
    Qs = Q - qbar[blk]
    Ks = K - kbar
    lhs = Q.astype(np.float64) @ Ks.T
    rhs = Qs @ Ks.T + C[blk][:, :N] - (qbar @ kbar)[blk][:, None]
    assert np.allclose(lhs, rhs, rtol=0, atol=1e-10)


def test_k_smoothing_is_softmax_invariant():
    rng = np.random.default_rng(7)
    N, d = 200, 64
    Q = rng.standard_normal((N, d))
    K = rng.standard_normal((N, d)) + rng.normal(0, 5, d)
    V = rng.standard_normal((N, d))
    kbar = K.mean(0)
    for causal in (False, True):
        a = orc.attn_fp64(Q, K, V, causal, 0.125)
        b = orc.attn_fp64(Q, K - kbar, V, causal, 0.125)
        assert np.abs(a - b).max() < 1e-12


# ---------------------------------------- tiling / online softmax / masking
def _identity_payload(Q, K, V):
    pay = orc.smooth_quant_qk(Q, K)
    blk = np.arange(Q.shape[0]) // orc.BM
    return dict(q_s=Q.astype(np.float64) - pay["q_mean"].astype(np.float64)[blk],
                k_s=K.astype(np.float64) - pay["k_mean"].astype(np.float64),
                v=V.astype(np.float64),
                C=orc.qk_correction(pay["q_mean"], K))


@pytest.mark.parametrize("N", [1, 7, 128, 129, 300, 513])
@pytest.mark.parametrize("causal", [False, True])
def test_online_softmax_identity_quant_equals_fp64(N, causal):
    rng = np.random.default_rng(100 + N)
    d = 64
    Q = (rng.standard_normal((N, d)) + rng.normal(0, 1, d)).astype(np.float32)
    K = (rng.standard_normal((N, d)) + rng.normal(0, 3, d)).astype(np.float32)
    V = rng.standard_normal((N, d)).astype(np.float32)
    sm = 1 / math.sqrt(d)
    O, amb, rows = orc.attn_quantized(_identity_payload(Q, K, V), N, causal, sm, quantize=False)
    ref = orc.attn_fp64(Q, K, V, causal, sm)
    assert np.array_equal(rows, np.arange(N))
    assert np.abs(O - ref).max() < 1e-11
    assert (amb == 0).all()


def _golden():
    vals = {}
    for line in open(os.path.join(GOLDEN, "two_tile_recurrence.txt")):
        line = line.split("#")[0].strip()
        if line:
            key, val = line.split()
            vals[key] = float(val)
    return vals


def scripted_payload(x_tile0, x_tile1, v0, v1, d=64):
    """One head, N = 256, not causal: Q^ = K^ = 0 with unit scales, so the
    score of key j (in log2 units, with sm_scale = 1) is the correction
    alone; x_tile*: [128] scores; v0, v1: per-channel V values of each tile
    (exact e4m3 values, v_scale 1).  The same scores for both query blocks."""
    N = 256
    x = np.concatenate([x_tile0, x_tile1])
    vt = np.zeros((d, N), np.uint8)
    vt[:, :128] = orc.e4m3_encode(np.asarray(v0, np.float64))[:, None]
    vt[:, 128:] = orc.e4m3_encode(np.asarray(v1, np.float64))[:, None]
    return dict(q_i4=np.zeros((N, d), np.int8), q_scale=np.ones(N, np.float32),
                k_i4=np.zeros((N, d), np.int8), k_scale=np.ones(N, np.float32),
                C=np.repeat((x / orc.LOG2E)[None, :], 2, axis=0), v_t=vt,
                v_scale=np.ones(d, np.float32))


def scenario_a(d=64):
    x0 = np.r_[np.zeros(64), np.full(64, -0.3)]
    x1 = np.r_[np.full(32, 0.7), np.full(96, 0.2)]
    v1 = np.where(np.arange(d) % 2 == 0, 2.0, -0.5)
    return scripted_payload(x0, x1, np.ones(d), v1, d)


def scenario_b(d=64):
    x0 = np.full(128, -30.0)
    x0[0] = 0.0
    x0[1] = math.log2(368.0 / 448.0) + math.log2(1 + 2.0 ** -22)
    x1 = np.full(128, -30.0)
    x1[0] = 0.5
    v0 = np.where(np.arange(d) % 2 == 0, 1.0, -2.0)
    return scripted_payload(x0, x1, v0, np.full(d, 0.5), d)


def test_two_tile_recurrence_golden():
    """Rounding P~ per tile against the running maximum, then rescaling by
    alpha into the outer accumulator, against the hand-worked values."""
    g = _golden()
    O, amb, rows = orc.attn_quantized(scenario_a(), 256, False, 1.0)
    assert np.array_equal(rows, np.arange(256))
    assert np.allclose(O[:, 0::2], g["A_O_even"], rtol=1e-12, atol=0)
    assert np.allclose(O[:, 1::2], g["A_O_odd"], rtol=1e-12, atol=0)
    assert (amb == 0).all()                # no score near a boundary


def test_ambiguous_code_and_its_flip_golden():
    """One 448p sits 2^-22 above an e4m3 boundary: the oracle rounds it up,
    lists it as its only ambiguous code, and gives the hand-worked change of
    the output when it is rounded down instead."""
    g = _golden()
    O, amb, rows, flips = orc.attn_quantized(scenario_b(), 256, False, 1.0, explain_rows=[0, 200])
    assert np.allclose(O[:, 0::2], g["B_O_even"], rtol=1e-12, atol=0)
    assert np.allclose(O[:, 1::2], g["B_O_odd"], rtol=1e-12, atol=0)
    for row in (0, 200):
        f = flips[row]
        assert f.shape == (1, 64)
        assert np.allclose(f[0, 0::2], g["B_delta_even"], rtol=1e-12, atol=0)
        assert np.allclose(f[0, 1::2], g["B_delta_odd"], rtol=1e-12, atol=0)
    assert np.allclose(amb[0], np.abs(flips[0][0]), rtol=1e-12)


@pytest.mark.parametrize("N", [1, 5, 100, 128])
def test_single_tile_brute_force(N):
    """One key tile: the online recurrence reduces to the direct formula."""
    rng = np.random.default_rng(200 + N)
    d = 64
    Q = rng.standard_normal((N, d)).astype(np.float32)
    K = (rng.standard_normal((N, d)) + 2).astype(np.float32)
    V = (rng.standard_normal((N, d)) + 1).astype(np.float32)
    sm = 1 / math.sqrt(d)
    pay, O, amb, rows = orc.sage2_head(Q, K, V, causal=False, sm_scale=sm)
    S = np.zeros((N, N), np.int64)
    for i in range(N):                       # naive integer dot products
        for j in range(N):
            S[i, j] = sum(int(a) * int(b) for a, b in zip(pay["q_i4"][i], pay["k_i4"][j]))
    x = (pay["q_scale"][:N, None].astype(np.float64) * pay["k_scale"][None, :N] * S
         + pay["C"][0][:N][None, :]) * sm * orc.LOG2E
    p = np.exp2(x - x.max(1, keepdims=True))
    vh = orc.e4m3_decode(pay["v_t"][:, :N]).T * pay["v_scale"][None, :]
    ref = (orc.e4m3_round(448 * p) @ vh) / (448 * p.sum(1, keepdims=True))
    assert np.abs(O - ref).max() < 1e-12


def test_qk_int_matches_naive_loop():
    rng = np.random.default_rng(8)
    q = rng.integers(-7, 8, (5, 64)).astype(np.int8)
    k = rng.integers(-7, 8, (6, 64)).astype(np.int8)
    S = orc.qk_int(q, k)
    for i in range(5):
        for j in range(6):
            assert S[i, j] == sum(int(q[i, c]) * int(k[j, c]) for c in range(64))


def test_n1_closed_form():
    rng = np.random.default_rng(9)
    Q, K, V = (rng.standard_normal((1, 128)).astype(np.float32) for _ in range(3))
    pay, O, _, _ = orc.sage2_head(Q, K, V, causal=True)
    vh = orc.e4m3_decode(pay["v_t"][:, 0]) * pay["v_scale"]
    assert np.array_equal(O[0], vh)


@pytest.mark.parametrize("causal", [False, True])
def test_uniform_attention_closed_form(causal):
    """Identical keys give identical scores in a row: P~ = 448 everywhere, so
    O_i is the plain mean of the dequantized V over the visible keys."""
    rng = np.random.default_rng(10)
    N, d = 300, 64
    Q = rng.standard_normal((N, d)).astype(np.float32)
    K = np.repeat(rng.standard_normal((1, d)).astype(np.float32), N, axis=0)
    V = (rng.standard_normal((N, d)) + 3).astype(np.float32)
    pay, O, amb, rows = orc.sage2_head(Q, K, V, causal=causal)
    vh = orc.e4m3_decode(pay["v_t"][:, :N]).T * pay["v_scale"][None, :]
    for i in (0, 1, 127, 128, 255, 299):
        ref = vh[: i + 1].mean(0) if causal else vh.mean(0)
        assert np.abs(O[i] - ref).max() < 1e-12
    assert (amb == 0).all()


def test_causal_row0_sees_only_key0():
    rng = np.random.default_rng(11)
    Q, K, V = (rng.standard_normal((200, 64)).astype(np.float32) for _ in range(3))
    pay, O, _, _ = orc.sage2_head(Q, K, V, causal=True)
    assert np.array_equal(O[0], orc.e4m3_decode(pay["v_t"][:, 0]) * pay["v_scale"])


# ------------------------------------------------------------- V quantizer
def test_quant_v_properties():
    rng = np.random.default_rng(12)
    N, d = 300, 64
    V = (rng.standard_normal((N, d)) * rng.uniform(0.1, 10, d)).astype(np.float32)
    V[:, 5] = 0
    vt, sv = orc.quant_v(V)
    assert vt.shape == (d, 384) and (vt[:, N:] == 0).all()
    assert sv[5] == 0 and (vt[5] == 0).all()
    arg = np.abs(V).argmax(0)
    top = vt[np.arange(d), arg]
    ok = np.arange(d) != 5
    assert ((top[ok] & 0x7F) == 0x7E).all()
    deq = orc.e4m3_decode(vt[:, :N]).T * sv[None, :]
    rel = np.abs(deq - V) / (np.abs(V) + 1e-30)
    big = np.abs(V) * (448 / np.maximum(np.abs(V).max(0), 1e-30)) >= 2 ** -6
    assert (rel[big] <= 2 ** -4 * (1 + 1e-6)).all()      # half of 3-bit mantissa step


# ------------------------------------------------- sanity against fp64 attention
def test_quantized_close_to_fp64_small():
    rng = np.random.default_rng(13)
    N, d = 256, 64
    Q = rng.standard_normal((N, d)).astype(np.float32)
    K = (rng.standard_normal((N, d)) + rng.normal(0, 3, d)).astype(np.float32)
    V = (rng.standard_normal((N, d)) + 1).astype(np.float32)
    _, O, _, _ = orc.sage2_head(Q, K, V, causal=False)
    ref = orc.attn_fp64(Q, K, V, False, 1 / math.sqrt(d))
    cos = (O * ref).sum() / np.linalg.norm(O) / np.linalg.norm(ref)
    assert cos > 0.98
