"""Pins of the host oracle to facts outside itself (no GPU).

Each test ties one part of the oracle to something other than the oracle: hand-written bit
patterns, a library routine (numpy's float16 decoder, numpy integer/float matmul) on special
cases where the method reduces to a plain product, closed forms, and invariants (parallel-k
additivity, per-channel == one group). The mutation test at the end rebuilds the oracle with
one plausible mistake at a time and checks that some pin here rejects it.
"""
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
from gemv_w4a16_w8a8_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fixture_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            *vals, word = line.split()
            rows.append(([int(v) for v in vals], int(word, 16)))
    return rows


# ---- binary16 decoding ---------------------------------------------------------------------

def check_half_decoder(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = orc.half_to_double(bits)
    want = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    # signed zeros keep their sign
    assert np.signbit(got[0x8000]) and not np.signbit(got[0])


def test_half_decoder_all_bit_patterns():
    check_half_decoder(oracle.get())


# ---- packing ----------------------------------------------------------------------------------

def check_pack_fixtures(orc):
    for codes, word in _fixture_rows("pack_int4.txt"):
        got = orc.pack_int4(np.array([codes], dtype=np.uint8))
        assert got.shape == (1, 1) and int(got[0, 0]) == word, (codes, hex(int(got[0, 0])))
        back = orc.unpack_int4(np.array([[word]], dtype=np.uint32), 8)
        assert back.tolist() == [codes]
    for vals, word in _fixture_rows("pack_int2.txt"):
        got = orc.pack_int2(np.array([vals], dtype=np.int8))
        assert int(got[0, 0]) == word, (vals, hex(int(got[0, 0])))
        back = orc.unpack_int2(np.array([[word]], dtype=np.uint32), 16)
        assert back.tolist() == [vals]


def test_pack_golden_words():
    check_pack_fixtures(oracle.get())


def check_pack_interleaved(orc):
    for codes, word in _fixture_rows("pack_int4_interleaved.txt"):
        got = orc.pack_int4_interleaved(np.array([codes], dtype=np.uint8))
        assert int(got[0, 0]) == word, (codes, hex(int(got[0, 0])))
        assert orc.unpack_int4_interleaved(np.array([[word]], dtype=np.uint32), 8).tolist() == [codes]
    # the same codes in both layouts: a fixed permutation of the nibbles of every word
    codes = synth.uniform_int((7, 64), 0, 15, 8, synth.TID_W, np.uint8)
    nat = orc.pack_int4(codes)
    ilv = orc.pack_int4_interleaved(codes)
    assert np.array_equal(orc.unpack_int4_interleaved(ilv, 64), codes)
    perm = [0, 2, 4, 6, 1, 3, 5, 7]           # nibble i of the interleaved word = code perm[i]
    for i, e in enumerate(perm):
        assert np.array_equal((ilv >> (4 * i)) & 0xF, (nat >> (4 * e)) & 0xF)


def test_pack_interleaved():
    check_pack_interleaved(oracle.get())


def check_pack_int2_interleaved(orc):
    for vals, word in _fixture_rows("pack_int2_interleaved.txt"):
        got = orc.pack_int2_interleaved(np.array([vals], dtype=np.int8))
        assert int(got[0, 0]) == word, (vals, hex(int(got[0, 0])))
        back = orc.unpack_int2_interleaved(np.array([[word]], dtype=np.uint32), 16)
        assert back.tolist() == [vals]
    # the same values in both layouts: a fixed permutation of the 2-bit fields of every word
    vals = synth.uniform_int((5, 128), -2, 1, 9, synth.TID_W, np.int8)
    nat = orc.pack_int2(vals)
    ilv = orc.pack_int2_interleaved(vals)
    assert np.array_equal(orc.unpack_int2_interleaved(ilv, 128), vals)
    perm = [0, 4, 1, 5, 2, 6, 3, 7, 8, 12, 9, 13, 10, 14, 11, 15]   # field f holds value perm[f]
    for f, e in enumerate(perm):
        assert np.array_equal((ilv >> (2 * f)) & 3, (nat >> (2 * e)) & 3)


def test_pack_int2_interleaved():
    check_pack_int2_interleaved(oracle.get())


def test_pack_roundtrip_random():
    codes = synth.uniform_int((37, 256), 0, 15, 3, synth.TID_W, np.uint8)
    assert np.array_equal(oracle.unpack_int4(oracle.pack_int4(codes), 256), codes)
    vals = synth.uniform_int((19, 512), -2, 1, 4, synth.TID_W, np.int8)
    assert np.array_equal(oracle.unpack_int2(oracle.pack_int2(vals), 512), vals)
    # every packed word is a bijection of its fields: random words survive unpack -> pack
    words = synth.bits(5, 9, 0, 64).astype(np.uint32).reshape(4, 16)
    assert np.array_equal(oracle.pack_int4(oracle.unpack_int4(words, 128)), words)
    assert np.array_equal(oracle.pack_int2(oracle.unpack_int2(words, 256)), words)


def check_pack_masks_high_bits(orc):
    # codes above 15 keep only their low nibble (the packing definition masks with 0xF)
    codes = np.array([[0x1F, 0x20, 0, 0, 0, 0, 0, 0xFF]], dtype=np.uint8)
    assert int(orc.pack_int4(codes)[0, 0]) == 0xF000000F
    # int2 keeps the low two bits of each int8 (its two's-complement field)
    vals = np.array([[-2, 5, -1, 0] + [0] * 12], dtype=np.int8)
    assert int(orc.pack_int2(vals)[0, 0]) == 0b11_01_10


def test_pack_masks_high_bits():
    check_pack_masks_high_bits(oracle.get())


# ---- W4A16 --------------------------------------------------------------------------------------

def _w4_case(M, N, K, gs, has_zero, seed):
    d = synth.w4a16_inputs(M, N, K, gs, has_zero, seed)
    d["Wq"] = oracle.pack_int4(d["codes"])
    return d


def check_w4_unit_scale_is_plain_matmul(orc):
    """s = 1, z = 0: C is A times the code matrix, a plain product numpy can do."""
    M, N, K, gs = 5, 7, 96, 32
    d = synth.w4a16_inputs(M, N, K, gs, False, 11)
    Wq = orc.pack_int4(d["codes"])
    ones = np.ones((N, K // gs), dtype=np.float16)
    # integer-valued activations keep every partial sum exact in fp64: equality is exact
    Aint = synth.uniform_int((M, K), -2, 1, 12, synth.TID_A, np.int8).astype(np.float16)
    got = orc.w4a16(Aint, Wq, ones, None, K, gs)
    want = Aint.astype(np.float64) @ d["codes"].astype(np.float64).T
    assert np.array_equal(got, want)
    # random-normal activations: equal up to fp64 summation order
    got = orc.w4a16(d["A"], Wq, ones, None, K, gs)
    want = d["A"].astype(np.float64) @ d["codes"].astype(np.float64).T
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_w4_unit_scale_is_plain_matmul():
    check_w4_unit_scale_is_plain_matmul(oracle.get())


def check_w4_one_hot_reads_single_weight(orc):
    """A = e_k0: C[m, n] = (q[n,k0] - z[n,g(k0)]) * s[n,g(k0)], for k0 in every group."""
    N, K, gs = 9, 256, 64
    G = K // gs
    codes = synth.uniform_int((N, K), 0, 15, 21, synth.TID_W, np.uint8)
    s = synth.uniform_f16((N, G), 0.001, 0.01, 21, synth.TID_SCALE)
    z = synth.uniform_int((N, G), 0, 15, 21, synth.TID_ZERO, np.int8).astype(np.float16)
    Wq = orc.pack_int4(codes)
    k0s = [0, 1, 7, 8, 63, 64, 65, 130, 200, 255]
    A = np.zeros((len(k0s), K), dtype=np.float16)
    for i, k0 in enumerate(k0s):
        A[i, k0] = 1.0
    got = orc.w4a16(A, Wq, s, z, K, gs)
    for i, k0 in enumerate(k0s):
        g = k0 // gs
        want = (codes[:, k0].astype(np.float64) - z[:, g].astype(np.float64)) * s[:, g].astype(np.float64)
        assert np.array_equal(got[i], want), k0
    # without zeros the same read gives q * s
    got = orc.w4a16(A, Wq, s, None, K, gs)
    for i, k0 in enumerate(k0s):
        g = k0 // gs
        assert np.array_equal(got[i], codes[:, k0] * s[:, g].astype(np.float64))


def test_w4_one_hot_reads_single_weight():
    check_w4_one_hot_reads_single_weight(oracle.get())


def check_w4_constant_closed_form(orc):
    """A = 1, every code q, per-group s_g and z_g: C = sum_g gs * (q - z_g) * s_g."""
    M, N, K, gs = 2, 3, 512, 128
    G = K // gs
    q = 11
    codes = np.full((N, K), q, dtype=np.uint8)
    s = np.array([[0.5, 0.25, 0.125, 2.0]] * N, dtype=np.float16)
    z = np.array([[8.0, 3.0, 0.0, 15.0]] * N, dtype=np.float16)
    A = np.ones((M, K), dtype=np.float16)
    got = orc.w4a16(A, orc.pack_int4(codes), s, z, K, gs)
    want = sum(gs * (q - float(z[0, g])) * float(s[0, g]) for g in range(G))
    assert np.all(got == want), (got, want)
    # W = 0 (codes equal to the zero point) gives C = 0
    zq = np.full((N, G), q, dtype=np.float16)
    assert np.all(orc.w4a16(A, orc.pack_int4(codes), s, zq, K, gs) == 0.0)


def test_w4_constant_closed_form():
    check_w4_constant_closed_form(oracle.get())


def check_w4_per_channel_equals_one_group(orc):
    M, N, K = 3, 5, 128
    d = _w4_case(M, N, K, -1, True, 31)
    assert d["scales"].shape == (N, 1)
    a = orc.w4a16(d["A"], d["Wq"], d["scales"], d["zeros"], K, -1)
    b = orc.w4a16(d["A"], d["Wq"], d["scales"], d["zeros"], K, K)
    assert np.array_equal(a, b)


def test_w4_per_channel_equals_one_group():
    check_w4_per_channel_equals_one_group(oracle.get())


def check_w4_parallel_k_additivity(orc):
    """Split K into parts (hidet issue #364, parallel-k): the parts' sums add to the total."""
    M, N, K, gs = 3, 6, 384, 128
    d = _w4_case(M, N, K, gs, True, 41)
    full = orc.w4a16(d["A"], d["Wq"], d["scales"], d["zeros"], K, gs)
    parts = 0.0
    for k0 in range(0, K, gs):
        g0 = k0 // gs
        Wq = orc.pack_int4(d["codes"][:, k0:k0 + gs])
        parts = parts + orc.w4a16(d["A"][:, k0:k0 + gs], Wq, d["scales"][:, g0:g0 + 1],
                                  d["zeros"][:, g0:g0 + 1], gs, gs)
    np.testing.assert_allclose(parts, full, rtol=1e-12, atol=1e-12)


def test_w4_parallel_k_additivity():
    check_w4_parallel_k_additivity(oracle.get())


def check_w4_elementwise_matches_full(orc):
    M, N, K, gs = 4, 33, 256, 64
    d = _w4_case(M, N, K, gs, True, 51)
    full = orc.w4a16(d["A"], d["Wq"], d["scales"], d["zeros"], K, gs)
    ms, ns = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    at = orc.w4a16_at(d["A"], d["Wq"], d["scales"], d["zeros"], K, gs, ms.ravel(), ns.ravel())
    assert np.array_equal(at.reshape(M, N), full)


def test_w4_elementwise_matches_full():
    check_w4_elementwise_matches_full(oracle.get())


def test_w4_rejects_bad_group():
    d = _w4_case(1, 2, 96, 32, False, 1)
    with pytest.raises(ValueError):
        oracle.w4a16(d["A"], d["Wq"], d["scales"], None, 96, 64)   # 96 % 64 != 0


# ---- dense fp16 ----------------------------------------------------------------------------------

def check_dense_is_numpy_matmul(orc):
    d = synth.dense_inputs(6, 10, 200, 61)
    got = orc.dense_f16(d["A"], d["W"])
    want = d["A"].astype(np.float64) @ d["W"].astype(np.float64).T
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-15)
    ms = np.array([0, 5, 3]); ns = np.array([9, 0, 4])
    assert np.array_equal(orc.dense_f16_at(d["A"], d["W"], ms, ns), got[ms, ns])


def test_dense_is_numpy_matmul():
    check_dense_is_numpy_matmul(oracle.get())


# ---- integer paths --------------------------------------------------------------------------------

def check_w8a8_is_integer_matmul(orc):
    d = synth.w8a8_inputs(7, 13, 320, 71)
    got = orc.w8a8(d["A"], d["W"])
    want = d["A"].astype(np.int64) @ d["W"].astype(np.int64).T
    assert np.array_equal(got, want)
    ms = np.array([6, 0]); ns = np.array([0, 12])
    assert np.array_equal(orc.w8a8_at(d["A"], d["W"], ms, ns), want[ms, ns])


def test_w8a8_is_integer_matmul():
    check_w8a8_is_integer_matmul(oracle.get())


def test_w8a8_extreme_closed_form():
    K = 16384
    A = np.full((1, K), -128, dtype=np.int8)
    W = np.full((2, K), -128, dtype=np.int8)
    assert np.all(oracle.w8a8(A, W) == K * 16384)
    W[1] = 127
    assert oracle.w8a8(A, W)[0, 1] == -128 * 127 * K


def check_w2a8_is_integer_matmul(orc):
    d = synth.w2a8_inputs(5, 11, 256, 81)
    Wq = orc.pack_int2(d["Wv"])
    got = orc.w2a8(d["A"], Wq)
    want = d["A"].astype(np.int64) @ d["Wv"].astype(np.int64).T
    assert np.array_equal(got, want)
    ms = np.array([4, 1]); ns = np.array([10, 3])
    assert np.array_equal(orc.w2a8_at(d["A"], Wq, ms, ns), want[ms, ns])


def test_w2a8_is_integer_matmul():
    check_w2a8_is_integer_matmul(oracle.get())


def test_int_parallel_k_additivity():
    d = synth.w8a8_inputs(3, 4, 512, 91)
    full = oracle.w8a8(d["A"], d["W"])
    parts = sum(oracle.w8a8(d["A"][:, k:k + 128], d["W"][:, k:k + 128]) for k in range(0, 512, 128))
    assert np.array_equal(parts, full)
    e = synth.w2a8_inputs(3, 4, 512, 92)
    full = oracle.w2a8(e["A"], oracle.pack_int2(e["Wv"]))
    parts = sum(oracle.w2a8(e["A"][:, k:k + 64], oracle.pack_int2(e["Wv"][:, k:k + 64]))
                for k in range(0, 512, 64))
    assert np.array_equal(parts, full)


# ---- the acceptance rule ----------------------------------------------------------------------------

def test_fp16_close_rule():
    ref = np.linspace(-4, 4, 1000)
    ok, _ = oracle.fp16_close(ref.astype(np.float16), ref)
    assert ok
    bad = ref.copy(); bad[17] += 0.5
    assert not oracle.fp16_close(bad, ref)[0]                       # one element out of bound
    drift = ref * (1 + 8e-3)
    assert not oracle.fp16_close(drift, ref)[0]                     # Frobenius bound
    nan = ref.copy(); nan[3] = np.nan
    assert not oracle.fp16_close(nan, ref)[0]


# ---- fp16 encoding and round-to-nearest int4 quantisation ------------------------------------------

def check_float_to_half(orc):
    """Against numpy's float32 -> float16 conversion (round to nearest even): every float16 value,
    the midpoints between neighbours (ties), values just off them, subnormals and overflow."""
    rng = np.random.default_rng(3)
    halves = np.arange(0, 0x7C00, 97, dtype=np.uint16).view(np.float16)
    exact = halves.astype(np.float32)
    nxt = np.nextafter(halves, np.float16(np.inf)).astype(np.float32)
    mids = ((exact.astype(np.float64) + nxt.astype(np.float64)) / 2).astype(np.float32)
    off = np.concatenate([np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    rand = (rng.standard_normal(2000) * np.exp2(rng.integers(-26, 17, 2000))).astype(np.float32)
    edge = np.array([0.0, -0.0, 65504.0, 65519.9, 65520.0, 1e9, 2.0**-24, 2.0**-25, 3 * 2.0**-26,
                     2.0**-26, -2.0**-14, np.inf, -np.inf], dtype=np.float32)
    xs = np.concatenate([exact, mids, off, rand, -rand, edge])
    got = orc.float_to_half(xs)
    want = xs.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want), np.flatnonzero(got != want)[:5]
    assert (orc.float_to_half(np.array([np.nan], np.float32))[0] & 0x7C00) == 0x7C00


def test_float_to_half_matches_numpy():
    check_float_to_half(oracle.get())


def _rtn_fixture():
    path = os.path.join(os.path.dirname(__file__), "golden", "rtn_int4.txt")
    gs, rows = None, []
    with open(path) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            if key == "gs":
                gs = int(vals[0])
            elif key == "row":
                rows.append({})
            elif key == "w":
                rows[-1]["w"] = np.array([float(v) for v in vals], dtype=np.float16)
            elif key == "q":
                rows[-1]["q"] = np.array([int(v) for v in vals], dtype=np.uint8)
            else:
                rows[-1][key] = np.array([int(v, 16) for v in vals], dtype=np.uint16)
    return gs, rows


def check_rtn_golden(orc):
    gs, rows = _rtn_fixture()
    for r in rows:
        codes, S, Z = orc.rtn_int4(r["w"][None, :], gs)
        assert np.array_equal(codes[0], r["q"]), (codes[0], r["q"])
        assert np.array_equal(S[0].view(np.uint16), r["s"]), S[0].view(np.uint16)
        assert np.array_equal(Z[0].view(np.uint16), r["z"]), Z[0].view(np.uint16)


def test_rtn_golden_fixture():
    check_rtn_golden(oracle.get())


def check_rtn_error_bound(orc):
    """(q - z) s is within s/2 of w wherever the code is not clamped, within s everywhere; the
    group's extreme values take the codes 0 and 15 whenever the group straddles 0."""
    rng = np.random.default_rng(5)
    N, K, gs = 64, 512, 128
    W = (rng.standard_normal((N, K)) * np.exp2(rng.integers(-6, 4, (N, 1)))).astype(np.float16)
    W[:8] = np.abs(W[:8])          # all-positive rows
    W[8:16] = -np.abs(W[8:16])     # all-negative rows
    codes, S, Z = orc.rtn_int4(W, gs)
    s = np.repeat(S.astype(np.float64), gs, axis=1)
    z = np.repeat(Z.astype(np.float64), gs, axis=1)
    err = np.abs(W.astype(np.float64) - (codes.astype(np.float64) - z) * s)
    inner = (codes > 0) & (codes < 15)
    assert np.all(err[inner] <= 0.5 * s[inner] * (1 + 1e-6))
    assert np.all(err <= s * (1 + 1e-6))
    assert codes.max() <= 15 and np.all(Z.astype(np.float64) == np.rint(Z.astype(np.float64)))
    g = W.reshape(N, K // gs, gs).astype(np.float64)
    c = codes.reshape(N, K // gs, gs)
    straddle = (g.min(axis=2) < 0) & (g.max(axis=2) > 0)
    lo_code = np.take_along_axis(c, g.argmin(axis=2)[..., None], axis=2)[..., 0]
    hi_code = np.take_along_axis(c, g.argmax(axis=2)[..., None], axis=2)[..., 0]
    assert np.all(lo_code[straddle] == 0) and np.all(hi_code[straddle] >= 14)


def test_rtn_error_bound():
    check_rtn_error_bound(oracle.get())


def check_rtn_closed_forms(orc):
    """Constant groups: 0 -> (s 1, z 0, q 0); c > 0 -> (s = c/15, z 0, q 15); c < 0 ->
    (s = -c/15, z 15, q 0). Scaling W by 2 doubles s exactly and keeps codes and zeros."""
    gs = 32
    W = np.concatenate([np.zeros(gs), np.full(gs, 3.0), np.full(gs, -1.5)]).astype(np.float16)
    codes, S, Z = orc.rtn_int4(W[None, :], gs)
    assert np.array_equal(codes[0], np.repeat(np.array([0, 15, 0], np.uint8), gs))
    assert np.array_equal(S[0].astype(np.float64),
                          np.array([1.0, np.float16(np.float32(3.0) / np.float32(15.0)),
                                    np.float16(np.float32(1.5) / np.float32(15.0))]))
    assert np.array_equal(Z[0].astype(np.float64), np.array([0.0, 0.0, 15.0]))
    rng = np.random.default_rng(6)
    W = (rng.standard_normal((16, 256))).astype(np.float16)
    c1, s1, z1 = orc.rtn_int4(W, 64)
    c2, s2, z2 = orc.rtn_int4((W.astype(np.float32) * 2).astype(np.float16), 64)
    assert np.array_equal(c1, c2) and np.array_equal(z1, z2)
    assert np.array_equal(s2.astype(np.float64), 2 * s1.astype(np.float64))
    # one group spanning K equals group_size = K
    assert all(np.array_equal(a, b) for a, b in zip(orc.rtn_int4(W, -1), orc.rtn_int4(W, 256)))


def test_rtn_closed_forms():
    check_rtn_closed_forms(oracle.get())


# ---- W8A8 with int8 requantised output ---------------------------------------------------------------

def check_w8a8_requant(orc):
    """Closed forms on hand-built operands: with one-hot activations C[m, n] = W[n, k]; a
    multiplier of 1 returns it, 0.5 halves it with ties to even (W odd -> x.5), 4 saturates at
    both ends, and the multiplier is indexed by the output channel n."""
    K = 16
    W = np.array([[-128, -7, -5, -3, -1, 0, 1, 3, 5, 7, 9, 31, 33, 63, 64, 127]], np.int8).T
    W = np.repeat(W, K, axis=1)                       # row n is the constant W[n]
    A = np.zeros((1, K), np.int8)
    A[0, 5] = 1                                        # one-hot: C[0, n] = W[n, 5] = W[n]
    w = W[:, 0].astype(np.int64)
    N = W.shape[0]
    assert np.array_equal(orc.w8a8_requant(A, W, np.ones(N, np.float32))[0], w)
    half = orc.w8a8_requant(A, W, np.full(N, 0.5, np.float32))[0].astype(np.int64)
    want = np.array([-64, -4, -2, -2, 0, 0, 0, 2, 2, 4, 4, 16, 16, 32, 32, 64])   # ties to even
    assert np.array_equal(half, want), half
    four = orc.w8a8_requant(A, W, np.full(N, 4.0, np.float32))[0].astype(np.int64)
    assert np.array_equal(four, np.clip(4 * w, -128, 127))
    mult = np.arange(N, dtype=np.float32) / 16
    got = orc.w8a8_requant(A, W, mult)[0].astype(np.int64)
    assert np.array_equal(got, np.clip(np.rint(w.astype(np.float32) * mult), -128, 127))
    # a large accumulator: A = W = -128 over K = 256 gives 4194304, times 2^-15 = 128 -> 127
    A2 = np.full((1, 256), -128, np.int8)
    W2 = np.full((2, 256), -128, np.int8)
    out = orc.w8a8_requant(A2, W2, np.array([2.0**-15, -2.0**-15], np.float32))[0]
    assert out.tolist() == [127, -128]


def test_w8a8_requant_closed_forms():
    check_w8a8_requant(oracle.get())


# ---- mutation check: each plausible mistake fails at least one pin ------------------------------------

MUTANTS = [
    ("wrong nibble order", "(4 * (k % 8))", "(4 * (7 - k % 8))"),
    ("zero point dropped", "w[k] = ((double)int4_code(Wq, K, n, k) - z) * s;",
     "w[k] = ((double)int4_code(Wq, K, n, k)) * s;"),
    ("zero point sign flipped", "w[k] = ((double)int4_code(Wq, K, n, k) - z) * s;",
     "w[k] = ((double)int4_code(Wq, K, n, k) + z) * s;"),
    ("scale groups reversed", "double s = orc_half_to_double(S[n * G + g]);",
     "double s = orc_half_to_double(S[n * G + (G - 1 - g)]);"),
    ("zero read from the scale array", "orc_half_to_double(Z[n * G + g])",
     "orc_half_to_double(S[n * G + g])"),
    ("group index off by one", "int64_t g = k / gs;\n        double s",
     "int64_t g = (k + 1) / gs < G ? (k + 1) / gs : G - 1;\n        double s"),
    ("activation transposed", "C[m * N + n] = dot_f64(Ad + m * K, w, K);",
     "C[m * N + n] = dot_f64(Ad + n % (M ? M : 1) * K, w, K);"),
    ("int2 sign extension wrong", "return u - 4 * (u >> 1);", "return u;"),
    ("int2 field order", "(2 * (k % 16))) & 3u", "(2 * (15 - k % 16))) & 3u"),
    ("half exponent bias", "ldexp((double)(1024 + f), e - 25)", "ldexp((double)(1024 + f), e - 24)"),
    ("half subnormal scale", "ldexp((double)f, -24)", "ldexp((double)f, -25)"),
    ("int8 weight widened unsigned", "w[k] = W8[n * K + k];", "w[k] = (uint8_t)W8[n * K + k];"),
    ("pack order reversed", "<< (4 * i);", "<< (4 * (7 - i));"),
    ("pack code not masked", "(uint32_t)(codes[n * K + 8 * j + i] & 0xF)",
     "(uint32_t)(codes[n * K + 8 * j + i])"),
    ("interleaved layout wrong", "static const int ILV_POS[8] = {0, 4, 1, 5, 2, 6, 3, 7};",
     "static const int ILV_POS[8] = {0, 1, 2, 3, 4, 5, 6, 7};"),
    ("interleaved unpack shift", "(4 * ILV_POS[k % 8])) & 0xF)", "(4 * (k % 8))) & 0xF)"),
    ("int2 interleaved layout wrong",
     "static const int ILV2_POS[16] = {0, 2, 4, 6, 1, 3, 5, 7, 8, 10, 12, 14, 9, 11, 13, 15};",
     "static const int ILV2_POS[16] = {0, 4, 8, 12, 1, 5, 9, 13, 2, 6, 10, 14, 3, 7, 11, 15};"),
    ("int2 interleaved unpack ignores the layout", "(2 * ILV2_POS[k % 16])) & 3u)",
     "(2 * (k % 16))) & 3u)"),
    ("int2 interleaved unpack sign", "vals[n * K + k] = (int8_t)(u - 4 * (u >> 1));",
     "vals[n * K + k] = (int8_t)u;"),
    ("int2 pack not masked", "((uint8_t)vals[n * K + 16 * j + i] & 3u)",
     "((uint8_t)vals[n * K + 16 * j + i])"),
    ("half encoding ties away from zero", "(rem == halfway && (q & 1u))", "(rem == halfway)"),
    ("half encoding drops the exponent carry", "q = 1024u;\n            ++he;", "q = 1023u;"),
    ("rtn truncates", "float q = rintf(v / s) + z;", "float q = truncf(v / s) + z;"),
    ("rtn range not widened to 0", "float lo = 0.0f, hi = 0.0f;",
     "float lo = (float)orc_half_to_double(w[0]), hi = lo;"),
    ("rtn zero sign", "float z = rintf(0.0f - lo / s);", "float z = rintf(lo / s);"),
    ("rtn sixteen steps", "range / 15.0f", "range / 16.0f"),
    ("rtn scale not rounded to fp16", "const float s = (float)orc_half_to_double(s16);",
     "const float s = s32;"),
    ("requant rounds half away", "float r = rintf(x);", "float r = roundf(x);"),
    ("requant saturates asymmetrically", "if (r < -128.0f) r = -128.0f;", "if (r < -127.0f) r = -127.0f;"),
    ("requant multiplier by row", "* mult[n];", "* mult[m];"),
]

PINS = [check_half_decoder, check_pack_fixtures, check_pack_interleaved,
        check_pack_int2_interleaved, check_pack_masks_high_bits, check_w4_unit_scale_is_plain_matmul,
        check_w4_one_hot_reads_single_weight, check_w4_constant_closed_form,
        check_w4_per_channel_equals_one_group, check_w4_parallel_k_additivity,
        check_w4_elementwise_matches_full, check_dense_is_numpy_matmul,
        check_w8a8_is_integer_matmul, check_w2a8_is_integer_matmul, check_float_to_half,
        check_rtn_golden, check_rtn_error_bound, check_rtn_closed_forms, check_w8a8_requant]


def _build_mutant(src: str, tmpdir: str, idx: int):
    c = os.path.join(tmpdir, f"mutant{idx}.c")
    so = os.path.join(tmpdir, f"mutant{idx}.so")
    with open(c, "w") as f:
        f.write(src)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", so, c, "-lm",
                    ], check=True, capture_output=True)
    return oracle.Oracle(so)


def _caught(orc) -> bool:
    for pin in PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError):
            return True
    return False


def test_pins_catch_planted_mistakes():
    with open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")) as f:
        src = f.read()
    # the unmutated source passes every pin
    with tempfile.TemporaryDirectory() as tmp:
        assert not _caught(_build_mutant(src, tmp, 999))
        escaped = []
        for i, (name, old, new) in enumerate(MUTANTS):
            assert old in src, f"mutation site for '{name}' not found"
            mutant = _build_mutant(src.replace(old, new, 1), tmp, i)
            if not _caught(mutant):
                escaped.append(name)
        assert not escaped, f"mutants not caught by any pin: {escaped}"
