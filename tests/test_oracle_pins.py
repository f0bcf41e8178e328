"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- a library e4m3 cast (torch.float8_e4m3fn), closed forms, values
printed on the pages (tests/golden/pages_values.json), invariants of the scale
rule, and exact-rational brute force on tiny inputs.  CPU only."""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from fp8_block_scaled_11_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_values.json")


def torch_e4m3_bits(v):
    """Library cast (RNE, not saturating: valid for |v| <= 448 only)."""
    return torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def torch_e4m3_value(b):
    return torch.from_numpy(np.ascontiguousarray(b, dtype=np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def f32_from_bits(u):
    return np.asarray(u, dtype=np.uint32).view(np.float32)


def bits_from_f32(f):
    return np.asarray(f, dtype=np.float32).view(np.uint32)


# --------------------------------------------------------------------------- #
# e4m3 codec
# --------------------------------------------------------------------------- #
def test_decode_all_codes_vs_library(oracle_mod):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    ours = oracle_mod.e4m3_decode(codes)
    lib = torch_e4m3_value(codes)
    assert np.array_equal(ours, lib)
    assert np.array_equal(np.signbit(ours), np.signbit(lib))
    assert np.isnan(oracle_mod.e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()


def test_decode_closed_forms(oracle_mod):
    cases = {0x7E: 448.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
             0x38: 1.0, 0x77: 240.0, 0x3C: 1.5, 0xB8: -1.0, 0xFE: -448.0}
    for c, v in cases.items():
        assert oracle_mod.e4m3_decode(np.array([c], np.uint8))[0] == v
    z = oracle_mod.e4m3_decode(np.array([0x80], np.uint8))[0]
    assert z == 0.0 and math.copysign(1.0, z) < 0


def test_decode_encode_roundtrip_all_codes(oracle_mod):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = oracle_mod.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(oracle_mod.e4m3_encode(vals), codes)


def _grid_neighbourhood(radius=64):
    """fp32 patterns within +-radius ulps of every e4m3 value and of every
    midpoint between consecutive e4m3 magnitudes (the rounding boundaries)."""
    mags = np.unique(torch_e4m3_value(np.arange(0, 0x7F, dtype=np.uint8)))
    mids = (mags[:-1] + mags[1:]) / 2.0                  # exact in fp64 and fp32
    centres = np.concatenate([mags, mids]).astype(np.float32)
    base = bits_from_f32(centres).astype(np.int64)
    offs = np.arange(-radius, radius + 1, dtype=np.int64)
    pats = (base[:, None] + offs[None, :]).reshape(-1)
    pats = pats[(pats >= 0)]
    v = f32_from_bits(pats.astype(np.uint32))
    v = v[np.abs(v) <= 448.0]
    return np.concatenate([v, -v])


def test_encode_vs_library_at_rounding_boundaries(oracle_mod):
    v = _grid_neighbourhood()
    assert np.array_equal(oracle_mod.e4m3_encode(v), torch_e4m3_bits(v))


def test_encode_vs_library_random_patterns(oracle_mod):
    rng = np.random.default_rng(123)
    pats = rng.integers(0, 0x43E00001, size=4_000_000, dtype=np.int64).astype(np.uint32)  # |v| <= 448
    v = f32_from_bits(pats)
    v = np.concatenate([v, -v])
    assert np.array_equal(oracle_mod.e4m3_encode(v), torch_e4m3_bits(v))


def test_encode_vs_library_strided_sweep(oracle_mod):
    # every 97th fp32 pattern in [0, 448], both signs (~11M values)
    pats = np.arange(0, 0x43E00001, 97, dtype=np.uint32)
    v = f32_from_bits(pats)
    assert np.array_equal(oracle_mod.e4m3_encode(v), torch_e4m3_bits(v))
    assert np.array_equal(oracle_mod.e4m3_encode(-v), torch_e4m3_bits(-v))


def test_encode_saturates(oracle_mod):
    big = np.array([448.0001, 464.0, 479.9, 480.0, 1e6, 3.0e38, np.inf], np.float32)
    assert (oracle_mod.e4m3_encode(big) == 0x7E).all()
    assert (oracle_mod.e4m3_encode(-big) == 0xFE).all()


def test_encode_keeps_sign_of_zero(oracle_mod):
    tiny = np.array([-0.0, -1e-30, -(2.0 ** -11), -(2.0 ** -10)], np.float32)   # -2^-10 is a tie -> even (0)
    assert (oracle_mod.e4m3_encode(tiny) == 0x80).all()
    assert oracle_mod.e4m3_encode(np.array([-(2.0 ** -10) * (1 + 2.0 ** -23)], np.float32))[0] == 0x81
    assert oracle_mod.e4m3_encode(np.array([0.0], np.float32))[0] == 0x00


# --------------------------------------------------------------------------- #
# Quantization: the scale rule s = 448/amax, q = e4m3(x*s), stored r = 1/s
# --------------------------------------------------------------------------- #
def _e4m3_grid_values(rng, n):
    codes = rng.integers(0, 0x7E, size=n).astype(np.uint8) | (rng.integers(0, 2, size=n).astype(np.uint8) << 7)
    return torch_e4m3_value(codes).astype(np.float32)


def test_quant_amax_448_is_identity_on_representable_values(oracle_mod):
    rng = np.random.default_rng(1)
    x = _e4m3_grid_values(rng, 4 * 256).reshape(4, 256)
    x[:, 0] = 448.0
    x[:, 128] = -448.0
    q, r = oracle_mod.quant_1x128(x)
    assert np.array_equal(r, np.ones_like(r))
    assert np.array_equal(torch_e4m3_value(q).astype(np.float32), x)


@pytest.mark.parametrize("amax,s", [(224.0, 2.0), (7.0, 64.0), (3.5, 128.0), (0.4375, 1024.0), (896.0, 0.5)])
def test_quant_power_of_two_scale_closed_form(oracle_mod, amax, s):
    rng = np.random.default_rng(int(amax * 16))
    x = (rng.uniform(-1.0, 1.0, size=(3, 128)) * amax).astype(np.float32)
    x[:, 5] = amax
    q, r = oracle_mod.quant_1x128(x)
    assert np.all(r == np.float32(1.0 / s))
    # x*s is exact (power-of-two s), so q is the library cast of x*s
    assert np.array_equal(q, torch_e4m3_bits(x * np.float32(s)))


def test_quant_all_zero_group(oracle_mod):
    x = np.zeros((2, 256), np.float32)
    x[1, :128] = -0.0
    x[1, 128:] = 3.0
    q, r = oracle_mod.quant_1x128(x)
    assert (q[0] == 0).all() and (q[1, :128] == 0x80).all()
    s0 = np.float32(448.0) / np.float32(1e-12)     # reading: amax clamped to 1e-12
    assert r[0, 0] == np.float32(1.0) / s0 and r[1, 0] == r[0, 0]
    assert (q[1, 128:] == 0x7E).all() and abs(float(r[1, 1]) * 448.0 / 3.0 - 1.0) < 1e-6


def _check_group_invariants(oracle_mod, x_groups, q_groups, r):
    """Per group: the largest code is +-448 (amax*s rounds to 448), every
    element is within half an e4m3 step of x*s, and r*s = 1 to fp32 rounding."""
    xs = x_groups.astype(np.float64)
    amax = np.abs(xs).max(axis=1)
    s = (np.float32(448.0) / np.maximum(amax, 1e-12).astype(np.float32)).astype(np.float64)
    d = torch_e4m3_value(q_groups)
    nz = amax > 0
    assert np.all(np.abs(d[nz]).max(axis=1) == 448.0)
    t = xs * s[:, None]
    step = np.where(np.abs(t) < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(t), 2.0 ** -6))) - 3))
    err = np.abs(d - np.clip(t, -448, 448))
    assert np.all(err <= step / 2 + np.abs(t) * 2.0 ** -23)
    assert np.all(np.abs(r.astype(np.float64) * s - 1.0) <= 2.0 ** -23)
    assert np.array_equal(np.signbit(d), np.signbit(xs))


def test_quant_1x128_invariants_bf16(oracle_mod):
    x = inputs.random_matrix(64, 1024, seed=7).view(torch.uint16).numpy()
    q, r = oracle_mod.quant_1x128(x)
    xf = inputs.random_matrix(64, 1024, seed=7).float().numpy()
    _check_group_invariants(oracle_mod, xf.reshape(-1, 128), q.reshape(-1, 128), r.reshape(-1))


def test_quant_128x128_invariants_and_layout(oracle_mod):
    x = inputs.random_matrix(256, 384, seed=8).float().numpy()
    x[128:, 256:] *= 1000.0
    q, r = oracle_mod.quant_128x128(x)
    assert r.shape == (2, 3)
    tiles_x = x.reshape(2, 128, 3, 128).transpose(0, 2, 1, 3).reshape(6, -1)
    tiles_q = q.reshape(2, 128, 3, 128).transpose(0, 2, 1, 3).reshape(6, -1)
    _check_group_invariants(oracle_mod, tiles_x, tiles_q, r.reshape(-1))
    # each tile equals a whole-tensor quantization of that tile (a separate code path)
    for bi in range(2):
        for bj in range(3):
            t = np.ascontiguousarray(x[128 * bi:128 * bi + 128, 128 * bj:128 * bj + 128])
            qt, rt = oracle_mod.quant_tensor(t)
            assert np.array_equal(qt, q[128 * bi:128 * bi + 128, 128 * bj:128 * bj + 128])
            assert rt[0] == r[bi, bj]


def test_quant_1x128_matches_rowwise_per_group_and_ragged(oracle_mod):
    x = inputs.random_matrix(37, 200, seed=9).view(torch.uint16).numpy()    # ragged rows and cols
    q, r = oracle_mod.quant_1x128(x)
    assert r.shape == (37, 2)
    q0, r0 = oracle_mod.quant_rowwise(np.ascontiguousarray(x[:, :128]))
    q1, r1 = oracle_mod.quant_rowwise(np.ascontiguousarray(x[:, 128:]))
    assert np.array_equal(q[:, :128], q0) and np.array_equal(q[:, 128:], q1)
    assert np.array_equal(r[:, 0], r0) and np.array_equal(r[:, 1], r1)


def test_quant_transposed_equals_quant_of_transpose(oracle_mod):
    x = inputs.random_matrix(300, 96, seed=10).view(torch.uint16).numpy()
    qt, rt = oracle_mod.quant_1x128(x, transpose=True)
    q2, r2 = oracle_mod.quant_1x128(np.ascontiguousarray(x.T))
    assert np.array_equal(qt, q2) and np.array_equal(rt, r2)
    qb, rb = oracle_mod.quant_128x128(x, transpose=True)
    qb2, rb2 = oracle_mod.quant_128x128(np.ascontiguousarray(x.T))
    assert np.array_equal(qb, qb2) and np.array_equal(rb, rb2)


def test_quant_sampled_rows_match_full(oracle_mod):
    x = inputs.random_matrix(300, 256, seed=11).view(torch.uint16).numpy()
    q, r = oracle_mod.quant_1x128(x)
    rows = [0, 7, 128, 299]
    qs, rs = oracle_mod.quant_1x128(x, rows=rows)
    assert np.array_equal(qs, q[rows]) and np.array_equal(rs, r[rows])
    qb, rb = oracle_mod.quant_128x128(x)
    qbs, rbs = oracle_mod.quant_128x128(x, rblocks=[2])
    assert np.array_equal(qbs[:300 - 256], qb[256:]) and np.array_equal(rbs[0], rb[2])


# --------------------------------------------------------------------------- #
# GEMM
# --------------------------------------------------------------------------- #
def _rand_scales(rng, shape):
    return (2.0 ** rng.uniform(-12, 2, size=shape)).astype(np.float32)


def test_gemm_per_tensor_equals_integer_dot(oracle_mod):
    """Per-tensor scaling: C = rA rB 2^-18 sum_k int(qA 2^9) int(qB 2^9), an exact
    integer dot product (numpy int64 matmul as the library routine)."""
    rng = np.random.default_rng(5)
    M, N, K = 24, 40, 640
    A = inputs.random_e4m3_bytes(M, K, seed=21).numpy()
    B = inputs.random_e4m3_bytes(N, K, seed=22).numpy()
    sa, sb = _rand_scales(rng, (1,)), _rand_scales(rng, (1,))
    Ai = (torch_e4m3_value(A) * 512).astype(np.int64)
    Bi = (torch_e4m3_value(B) * 512).astype(np.int64)
    assert np.array_equal(Ai.astype(np.float64), torch_e4m3_value(A) * 512)   # integer-valued
    scale = float(sa[0]) * float(sb[0]) * 2.0 ** -18
    exact = (Ai @ Bi.T).astype(np.float64) * scale
    mag = (np.abs(Ai) @ np.abs(Bi).T).astype(np.float64) * scale     # sum of |terms|
    for blocks in (False, True):
        C = oracle_mod.gemm(A, B, sa, sb, oracle_mod.SCALE_TENSOR, exact_blocks=blocks)
        assert np.all(np.abs(C - exact) <= 1e-14 * mag)


def _brute(A, B, sa, sb, mode):
    """Exact rational evaluation of the definition, element by element."""
    M, K = A.shape
    N = B.shape[0]
    dA = torch_e4m3_value(A)
    dB = torch_e4m3_value(B)
    C = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                kb = k // 128
                if mode == 0:
                    ra, rb = sa[0], sb[0]
                elif mode == 1:
                    ra, rb = sa[m], sb[n]
                elif mode == 2:
                    ra, rb = sa[m, kb], sb[n // 128, kb]
                else:
                    ra, rb = sa[m, kb], sb[n, kb]
                acc += Fraction(float(dA[m, k])) * Fraction(float(ra)) * Fraction(float(dB[n, k])) * Fraction(float(rb))
            C[m, n] = float(acc)
    return C


@pytest.mark.parametrize("mode", [0, 1, 2, 3])
@pytest.mark.parametrize("MNK", [(3, 4, 32), (4, 2, 128), (2, 3, 208), (4, 4, 384)])
def test_gemm_brute_force_rational(oracle_mod, mode, MNK):
    M, N, K = MNK
    rng = np.random.default_rng(100 * mode + K)
    A = inputs.random_e4m3_bytes(M, K, seed=K + mode).numpy()
    B = inputs.random_e4m3_bytes(N, K, seed=K + mode + 1000).numpy()
    Kb = (K + 127) // 128
    if mode == 0:
        sa, sb = _rand_scales(rng, (1,)), _rand_scales(rng, (1,))
    elif mode == 1:
        sa, sb = _rand_scales(rng, (M,)), _rand_scales(rng, (N,))
    elif mode == 2:
        sa, sb = _rand_scales(rng, (M, Kb)), _rand_scales(rng, ((N + 127) // 128, Kb))
    else:
        sa, sb = _rand_scales(rng, (M, Kb)), _rand_scales(rng, (N, Kb))
    exact = _brute(A, B, sa, sb, mode)
    mag = np.abs(torch_e4m3_value(A)).max() * np.abs(torch_e4m3_value(B)).max() * sa.max() * sb.max() * K
    for blocks in (False, True):
        C = oracle_mod.gemm(A, B, sa, sb, mode, exact_blocks=blocks)
        assert np.all(np.abs(C - exact) <= 1e-14 * mag)


def test_gemm_two_readings_agree_and_sampled_rows(oracle_mod):
    rng = np.random.default_rng(9)
    M, N, K = 130, 260, 1000
    A = inputs.random_e4m3_bytes(M, K, seed=31).numpy()
    B = inputs.random_e4m3_bytes(N, K, seed=32).numpy()
    Kb = (K + 127) // 128
    sa, sb = _rand_scales(rng, (M, Kb)), _rand_scales(rng, ((N + 127) // 128, Kb))
    C1 = oracle_mod.gemm(A, B, sa, sb, 2)
    C2 = oracle_mod.gemm(A, B, sa, sb, 2, exact_blocks=True)
    assert np.linalg.norm(C1 - C2) <= 1e-13 * np.linalg.norm(C2)
    rows = [0, 64, 129]
    assert np.array_equal(oracle_mod.gemm(A, B, sa, sb, 2, rows=rows), C1[rows])


# --------------------------------------------------------------------------- #
# SQNR and the pages' printed values
# --------------------------------------------------------------------------- #
def test_sqnr_reproduces_printed_collapse_values(oracle_mod):
    g = json.load(open(GOLDEN))["long_k_repro"]
    rng = np.random.default_rng(3)
    for i in (1, 2):
        ref_norm, out_norm, want = g["fp32_ref_norm"][i], g["collapsed_scaled_mm_norm"][i], g["collapsed_scaled_mm_sqnr_db"][i]
        ref = rng.standard_normal(4096)
        ref *= ref_norm / np.linalg.norm(ref)
        d = rng.standard_normal(4096)
        d -= d.dot(ref) / ref.dot(ref) * ref                       # orthogonal to ref
        d *= math.sqrt(out_norm ** 2 - ref_norm ** 2) / np.linalg.norm(d)   # ||ref + d|| = out_norm
        assert round(oracle_mod.sqnr(ref, ref + d), 2) == want


def test_bf16_output_conversion_vs_library(oracle_mod):
    rng = np.random.default_rng(4)
    c = rng.standard_normal(100000) * 10.0 ** rng.uniform(-3, 3, 100000)
    ours = oracle_mod.to_bf16_bits(c)
    lib = torch.from_numpy(c.astype(np.float32)).to(torch.bfloat16).view(torch.uint16).numpy()
    assert np.array_equal(ours, lib)


def _long_k_case(oracle_mod, K, rows):
    goT, x = inputs.long_k(K)
    qa, ra = oracle_mod.quant_1x128(goT.view(torch.uint16).numpy(), rows=rows)
    xb = x.view(torch.uint16).numpy()
    qb, rb = oracle_mod.quant_128x128(xb, transpose=True)            # x^T: 512 x K, 128x128 tiles
    C = oracle_mod.gemm(qa, qb, ra, rb, oracle_mod.SCALE_BLOCK_1x128_128x128)
    ref = oracle_mod.matmul_ref(goT[rows].view(torch.uint16).numpy(),
                                np.ascontiguousarray(x.t().contiguous().view(torch.uint16).numpy()))
    qb2, rb2 = oracle_mod.quant_1x128(xb, transpose=True)
    C2 = oracle_mod.gemm(qa, qb2, ra, rb2, oracle_mod.SCALE_BLOCK_1x128_1x128)
    # the same GEMM through a library matmul of the dequantized operands
    dA = torch_e4m3_value(qa) * np.repeat(ra.astype(np.float64), 128, axis=1)[:, :K]
    dB = torch_e4m3_value(qb) * np.kron(rb.astype(np.float64), np.ones((128, 128)))[:, :K]
    assert np.linalg.norm(dA @ dB.T - C) <= 1e-12 * np.linalg.norm(C)
    return ref, C, C2


def test_long_k_sqnr_and_norm_vs_pages(oracle_mod):
    """Long-K workload at k_blocks 1000 and 1001.  Pins: the fp32 reference
    norm the pages print (3273.87 at K=128128); no collapse between k_blocks
    1000 and 1001 (the pages' correct path moves by 0.07 dB); the 28 dB floor
    for both recipes.  The pages' absolute ~31.1 dB is not reproduced: with
    both operands random each one's e4m3 error is ~31.8 dB and the two add to
    ~28.9 dB; the pages' own inputs are not given."""
    g = json.load(open(GOLDEN))["long_k_repro"]
    rows = np.arange(0, 256, 16)                                     # 16 sampled rows
    sq = {}
    for K in (128000, 128128):
        ref, C, C2 = _long_k_case(oracle_mod, K, rows)
        sq[K] = oracle_mod.sqnr(ref, C)
        assert sq[K] >= 28.0 and oracle_mod.sqnr(ref, C2) >= 28.0
        i = g["k"].index(K)
        if g["fp32_ref_norm"][i] is not None:
            est_norm = np.linalg.norm(ref) * math.sqrt(256 / len(rows))
            assert abs(est_norm / g["fp32_ref_norm"][i] - 1.0) < 0.03
    assert abs(sq[128000] - sq[128128]) < 0.2


# --------------------------------------------------------------------------- power-of-two scales
# The scale rule of hardware block scaling (UE8M0 scale factors): the largest
# power of two not above the method's fp32 scale 448/amax.  Used only by the
# fast-accumulation ablation below.
def _pow2_rule_quant(oracle, x_bits):
    with oracle.scale_rule(oracle.SCALE_RULE_POW2):
        return oracle.quant_1x128(x_bits)


def test_pow2_scales_are_powers_of_two_below_the_fp32_scale(oracle_mod):
    oracle = oracle_mod
    g = torch.Generator().manual_seed(31)
    x = (torch.randn(64, 1024, generator=g) * torch.logspace(-3, 3, 64).unsqueeze(1)).to(torch.bfloat16)
    xb = x.view(torch.uint16).numpy()
    _, r2 = _pow2_rule_quant(oracle, xb)
    _, r32 = oracle.quant_1x128(xb)
    s2 = (1.0 / r2.astype(np.float64))
    s32 = (1.0 / r32.astype(np.float64))
    bits = r2.astype(np.float32).view(np.uint32)
    assert np.all(bits & 0x7FFFFF == 0), "reciprocal scale not a power of two"
    assert np.all(s2 <= s32 * (1 + 1e-7)) and np.all(s32 < 2 * s2 * (1 + 1e-7))


def test_pow2_scales_closed_forms(oracle_mod):
    oracle = oracle_mod
    # amax = 448, 224, 112: 448/amax is a power of two, both rules agree
    for amax, s in ((448.0, 1.0), (224.0, 2.0), (112.0, 4.0), (300.0, 1.0), (100.0, 4.0), (0.75, 512.0)):
        x = np.zeros((1, 128), dtype=np.float32)
        x[0, 5] = amax
        x[0, 6] = -amax / 3
        q, r = _pow2_rule_quant(oracle, x)
        assert r[0, 0] == np.float32(1.0 / s), (amax, r[0, 0])
        # x * s is exact (power of two): q is the e4m3 rounding of x*s, here via torch's cast
        want = torch.from_numpy(x * np.float32(s)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(q, want), amax


def test_pow2_scales_keep_the_group_maximum_in_the_top_binade(oracle_mod):
    oracle = oracle_mod
    g = torch.Generator().manual_seed(32)
    x = torch.randn(32, 1024, generator=g) * 3.7
    q, r = _pow2_rule_quant(oracle, x.numpy())
    d = oracle.e4m3_decode(q).reshape(q.shape)
    gmax = np.abs(d).reshape(32, 8, 128).max(axis=2)
    assert np.all(gmax <= 448) and np.all(gmax >= 224)


def test_fast_accumulation_ablation_sqnr(oracle_mod):
    """The accuracy cost of the variant without software promotion: on B200
    that is hardware block scaling, which takes power-of-two block scales.  On
    the long-K workload (sampled rows, k_blocks 1000/1001/1002, both recipes)
    the power-of-two rule stays within 1 dB of the method's fp32 scales and
    above 27.5 dB (the method's own recipe is held to 28 dB elsewhere)."""
    oracle = oracle_mod
    rows = list(range(0, 256, 64))
    for K in inputs.LONG_K_VALUES:
        goT, x = inputs.long_k(K)
        gb, xb = goT.view(torch.uint16).numpy(), x.view(torch.uint16).numpy()
        ref = oracle.matmul_ref(gb[rows], x.t().contiguous().view(torch.uint16).numpy())
        res = {}
        for rule in (oracle.SCALE_RULE_FP32, oracle.SCALE_RULE_POW2):
            with oracle.scale_rule(rule):
                qa, sa = oracle.quant_1x128(gb, rows=rows)
                qb, sb = oracle.quant_128x128(xb, transpose=True)
            res[rule] = oracle.sqnr(ref, oracle.gemm(qa, qb, sa, sb, oracle.SCALE_BLOCK_1x128_128x128))
        assert res[oracle.SCALE_RULE_FP32] >= 28.0
        assert res[oracle.SCALE_RULE_POW2] >= 27.5
        assert res[oracle.SCALE_RULE_FP32] - res[oracle.SCALE_RULE_POW2] <= 1.0, (K, res)
