"""Pins for the CPU oracle: checks against what the pages and the mathematics
fix, never against the oracle itself.

Each test names what it pins and which plausible mistake it would catch
(a dropped term, a wrong sign or index, a transposed operand, a wrong
rounding).  Sources: TinyGPT "Quantization Expansion" (GPTQ format, dequant
recipe, smoke test; QAT quantizer), metrale_gpu_runtime/mlx_int8.rs (MLX 8-bit
layout), Hugging Face "Metal" quantization (affine packed layout, bits 2/4/8),
executorch PR #24467 (W4A8 scheme).
"""
import os

import numpy as np
import pytest
import torch

import gwb_synth as synth
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _bf16(v):
    return synth.bits16(torch.tensor(v, dtype=torch.float32).to(torch.bfloat16))


def _f16(v):
    return synth.bits16(torch.tensor(v, dtype=torch.float32).to(torch.float16))


# --------------------------------------------------------------------- 16-bit formats
def test_bf16_rounding_matches_torch():
    """Pins fp32->bf16 round-to-nearest-even (ties, carries, subnormals) against torch's cast."""
    rng = np.random.default_rng(0)
    vals = rng.standard_normal(20000).astype(np.float32) * np.float32(3.0)
    # exact ties: low 16 bits = 0x8000 with even and odd kept lsb, and carry into the exponent
    ties = np.array([0x3f808000, 0x3f818000, 0x3fffffff, 0x3f7f8000, 0x00018000, 0x80008000,
                     0x7f7fffff, 0x007fffff], dtype=np.uint32).view(np.float32)
    vals = np.concatenate([vals, ties, np.float32([0.0, -0.0, 1e-40, -3.5e-39])])
    ref = synth.bits16(torch.from_numpy(vals).to(torch.bfloat16))
    got = np.array([oracle.f32_to_bf16(v) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_f16_codec_matches_torch():
    """Pins binary16 decode (all 63488 finite patterns) and fp64->fp16 RNE incl. subnormals/overflow."""
    pats = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    finite = pats[(pats & 0x7c00) != 0x7c00]
    ref = torch.from_numpy(finite.view(np.int16)).view(torch.float16).double().numpy()
    got = np.array([oracle.f16_to_f64(int(h)) for h in finite])
    assert np.array_equal(got, ref)
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(5000) * 1e3, rng.standard_normal(5000) * 1e-6,
                        [65504.0, 65519.99, 65520.0, -70000.0, 2.0 ** -25, 2.0 ** -25 * 3, 2.0 ** -24,
                         1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 2048.0 + 1.0, 0.0]])
    ref = synth.bits16(torch.from_numpy(v).to(torch.float16))
    got = np.array([oracle.f64_to_f16(x) for x in v], dtype=np.uint16)
    assert np.array_equal(got, ref)


# --------------------------------------------------------------------- MLX packing
def test_mlx_word_order_golden():
    """Pins low-bits-first column order for 2/4/8-bit words (mlx_int8.rs layout doc)."""
    for row in _golden_lines("mlx_word_order.txt"):
        bits, word, codes = int(row[0]), int(row[1], 16), [int(c) for c in row[2:]]
        K = 32 // bits
        got = oracle.unpack_affine(np.array([[word]], np.uint32), 1, K, bits)
        assert got[0].tolist() == codes, (bits, hex(word))
        back = oracle.pack_affine(np.array([codes], np.int32), bits)
        assert int(back[0, 0]) == word


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_pack_unpack_bijection(bits):
    """unpack(pack(c)) == c and pack(unpack(w)) == w on random data (catches overlapping fields)."""
    rng = np.random.default_rng(bits)
    N, K = 5, 4 * 32
    words = rng.integers(0, 1 << 32, size=(N, K * bits // 32), dtype=np.uint64).astype(np.uint32)
    codes = oracle.unpack_affine(words, N, K, bits)
    assert codes.min() >= 0 and codes.max() <= (1 << bits) - 1
    assert np.array_equal(oracle.pack_affine(codes, bits), words)
    c2 = rng.integers(0, 1 << bits, size=(N, K)).astype(np.int32)
    assert np.array_equal(oracle.unpack_affine(oracle.pack_affine(c2, bits), N, K, bits), c2)


def test_dequant_affine_hand_case():
    """w = byte * scale + bias with per-group scale/bias selection (mlx_int8.rs formula).
    Two groups of 4 columns with different scale/bias catch a wrong c/G index."""
    codes = np.array([[1, 2, 3, 4, 0, 1, 128, 255]], np.int32)
    wq = oracle.pack_affine(codes, 8)
    sc = np.concatenate([_bf16([0.5]), _bf16([-2.0])]).reshape(1, 2)
    bi = np.concatenate([_bf16([-1.0]), _bf16([3.0])]).reshape(1, 2)
    w = oracle.dequant_affine_f64(wq, sc, bi, 1, 8, 8, 4)
    assert w[0].tolist() == [-0.5, 0.0, 0.5, 1.0, 3.0, 1.0, -253.0, -507.0]


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_dequant_every_code_from_hand_packed_words(bits):
    """Every code 0 .. 2^b - 1 of a bit width, packed into words by hand (numpy shifts written
    here, lowest bits = lowest column), dequantizes to code * s + b exactly, with a different
    power-of-two scale and bias per group: a wrong mask, shift or group index fails it."""
    per = 32 // bits
    ncode = 1 << bits
    K = max(ncode, 64)
    codes = np.arange(K) % ncode
    words = np.zeros(K // per, np.uint64)
    for k in range(K):
        words[k // per] |= np.uint64(int(codes[k]) << ((k % per) * bits))
    gs = 32
    G = K // gs
    s = 2.0 ** -np.arange(1, G + 1)
    b = -(2.0 ** np.arange(G))
    W = oracle.dequant_affine_f64(words.astype(np.uint32).reshape(1, -1), _bf16(s).reshape(1, G),
                                  _bf16(b).reshape(1, G), 1, K, bits, gs)
    g = np.arange(K) // gs
    assert np.array_equal(W[0], codes * s[g] + b[g])


# --------------------------------------------------------------------- affine quantizer
@pytest.mark.parametrize("bits,gs", [(2, 32), (4, 64), (8, 128), (4, 32)])
def test_qpack_affine_nearest_grid_bruteforce(bits, gs):
    """Brute force: every code is the nearest grid point mn + c*s over all c in [0, 2^b-1]
    (fp32 s and mn), each group's min maps to 0 and max to 2^b-1, and the stored
    scale/bias are the bf16 roundings of (max-min)/(2^b-1) and min."""
    N, K = 6, 2 * gs
    w = synth.weights(N, K, seed=7).numpy()
    wq, sc, bi, codes = oracle.qpack_affine(w, bits, gs)
    assert np.array_equal(oracle.unpack_affine(wq, N, K, bits), codes)
    qmax = (1 << bits) - 1
    grid = np.arange(qmax + 1, dtype=np.float64)
    for n in range(N):
        for g in range(K // gs):
            seg = w[n, g * gs:(g + 1) * gs]
            mn, mx = np.float32(seg.min()), np.float32(seg.max())
            s = np.float32(np.float32(mx - mn) / np.float32(qmax))
            assert sc[n, g] == _bf16([s])[0] and bi[n, g] == _bf16([mn])[0]
            c = codes[n, g * gs:(g + 1) * gs]
            assert c[np.argmin(seg)] == 0 and c[np.argmax(seg)] == qmax
            dist = np.abs(seg.astype(np.float64)[:, None] - (float(mn) + grid[None, :] * float(s)))
            best = dist.min(axis=1)
            chosen = dist[np.arange(gs), c]
            # equal to the nearest grid point up to the fp32 rounding of (w-mn)/s
            assert np.all(chosen <= best + 4e-7 * float(s) * qmax + 1e-12)


def test_qpack_affine_degenerate_group():
    """A constant group (max == min) gives scale 0, bias = min, all codes 0 and exact dequant."""
    w = np.full((2, 64), 0.375, np.float32)
    w[1, :32] = -1.25
    w[1, 32:] = np.linspace(0, 1, 32, dtype=np.float32)
    wq, sc, bi, codes = oracle.qpack_affine(w, 4, 32)
    assert np.all(codes[0] == 0) and np.all(codes[1, :32] == 0)
    deq = oracle.dequant_affine_f64(wq, sc, bi, 2, 64, 4, 32)
    assert np.all(deq[0] == 0.375) and np.all(deq[1, :32] == -1.25)
    assert sc[0, 0] == 0 and sc[1, 0] == 0


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_qpack_affine_error_bound(bits):
    """|w - dequant(quant(w))| <= s/2 plus the bf16 rounding of s and of the bias."""
    N, K, gs = 8, 256, 64
    w = synth.weights(N, K, seed=3).numpy()
    wq, sc, bi, _ = oracle.qpack_affine(w, bits, gs)
    deq = oracle.dequant_affine_f64(wq, sc, bi, N, K, bits, gs)
    s = np.repeat(oracle.bf16_array_to_f64(sc), gs, axis=1)
    b = np.repeat(oracle.bf16_array_to_f64(bi), gs, axis=1)
    qmax = (1 << bits) - 1
    slack = s / 2 * (1 + 2.0 ** -7) + qmax * s * 2.0 ** -8 + np.abs(b) * 2.0 ** -8
    assert np.all(np.abs(deq - w) <= slack)


def test_dequant_bf16_single_rounding():
    """The standalone dequant's bf16 output is the exact value rounded to fp32 then bf16
    (torch's RNE casts as the library routine)."""
    N, K, gs = 16, 128, 32
    w = synth.weights(N, K, seed=11).numpy()
    wq, sc, bi, codes = oracle.qpack_affine(w, 4, gs)
    got = oracle.dequant_affine_bf16(wq, sc, bi, N, K, 4, gs)
    exact = codes.astype(np.float64) * np.repeat(oracle.bf16_array_to_f64(sc), gs, 1) \
        + np.repeat(oracle.bf16_array_to_f64(bi), gs, 1)
    ref = synth.bits16(torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16))
    assert np.array_equal(got, ref)


# --------------------------------------------------------------------- qmm (affine)
@pytest.mark.parametrize("bits,gs", [(4, 64), (8, 32), (2, 128)])
def test_qmm_affine_against_numpy_matmul(bits, gs):
    """With power-of-two scales and small integer biases everything is exact in fp64, so
    the oracle must equal numpy's x @ W^T on the dequantized matrix built from the known
    codes (catches x.W vs W.x, wrong group index, dropped bias term)."""
    rng = np.random.default_rng(5)
    M, N, K = 3, 7, 2 * gs
    codes = rng.integers(0, 1 << bits, size=(N, K)).astype(np.int32)
    G = K // gs
    s = 2.0 ** rng.integers(-4, 2, size=(N, G))
    b = rng.integers(-9, 9, size=(N, G)).astype(np.float64)
    x = rng.integers(-6, 7, size=(M, K)).astype(np.float32) * np.float32(0.25)
    wq = oracle.pack_affine(codes, bits)
    W = codes * np.repeat(s, gs, 1) + np.repeat(b, gs, 1)
    y = oracle.qmm_affine(_bf16(x).reshape(M, K), wq, _bf16(s).reshape(N, G), _bf16(b).reshape(N, G),
                          N, K, bits, gs)
    assert np.array_equal(y, x.astype(np.float64) @ W.T)
    # row sampling returns exactly the selected rows
    y2 = oracle.qmm_affine(_bf16(x).reshape(M, K), wq, _bf16(s).reshape(N, G), _bf16(b).reshape(N, G),
                           N, K, bits, gs, rows=[2, 0])
    assert np.array_equal(y2, y[[2, 0]])


def test_qmm_unit_scale_is_integer_matmul():
    """scale 1, bias 0: the qmm is the integer product of x and the raw codes."""
    rng = np.random.default_rng(9)
    M, N, K, gs = 2, 5, 64, 64
    codes = rng.integers(0, 16, size=(N, K)).astype(np.int32)
    x = rng.integers(-20, 21, size=(M, K)).astype(np.float32)
    y = oracle.qmm_affine(_bf16(x).reshape(M, K), oracle.pack_affine(codes, 4),
                          _bf16(np.ones((N, 1))).reshape(N, 1), _bf16(np.zeros((N, 1))).reshape(N, 1),
                          N, K, 4, gs)
    assert np.array_equal(y, (x.astype(np.int64) @ codes.T.astype(np.int64)).astype(np.float64))


# --------------------------------------------------------------------- GPTQ
def test_gptq_worked_example_golden():
    """The page's smoke test: W[0,:] = [-1, 0, 1, ..., 14] (pins nibble order along IN,
    the +1 zero convention and the sign of int4 - zero)."""
    rows = {r[0]: r[1:] for r in _golden_lines("gptq_worked_example.txt")}
    K, gs = int(rows["in_features"][0]), int(rows["group_size"][0])
    N = 8
    expected = np.array([float(v) for v in rows["row0"]])
    qweight = np.zeros((K // 8, N), np.int64)
    qweight[0, 0] = 0x76543210           # codes 0..7 for in-features 0..7
    qweight[1, 0] = 0xFEDCBA98           # codes 8..15 for in-features 8..15
    qweight = qweight.astype(np.uint32).view(np.int32)
    qzeros = np.zeros((K // gs, N // 8), np.int32)   # stored zero 0 -> zero 1
    scales = _f16(np.ones((K // gs, N)))
    W = oracle.gptq_dequant_f64(qweight, scales, qzeros, None, K, N, gs)
    assert np.array_equal(W[0], expected)
    W16 = oracle.gptq_dequant_f16(qweight, scales, qzeros, None, K, N, gs)
    assert np.array_equal(np.array([oracle.f16_to_f64(h) for h in W16[0]]), expected)


def test_gptq_zero_nibble_selects_out_column():
    """qzeros is packed along OUT: column o reads nibble o % 8 of word o // 8.  Distinct
    stored zeros per column give W[o, i] = scale * (i - (z_o + 1)) in closed form."""
    K, N, gs = 8, 16, 8
    qweight = np.full((1, N), 0x76543210, np.int64).astype(np.uint32).view(np.int32)  # codes 0..7
    z = np.array([3, 0, 15, 7, 1, 2, 9, 4, 5, 6, 8, 10, 11, 12, 13, 14])
    words = [sum(int(z[8 * w + j]) << (4 * j) for j in range(8)) for w in range(2)]
    qzeros = np.array([words], np.int64).astype(np.uint32).view(np.int32)
    scales = _f16(np.full((1, N), 0.5))
    W = oracle.gptq_dequant_f64(qweight, scales, qzeros, None, K, N, gs)
    i = np.arange(K)
    for o in range(N):
        assert np.array_equal(W[o], 0.5 * (i - (z[o] + 1)))


def test_gptq_g_idx_selects_group_per_in_feature():
    """g = g_idx[i], not i // gs: with the two groups swapped, in-features 0..7 take group 1's
    scale (2.0) and 8..15 group 0's (1.0)."""
    K, N, gs = 16, 8, 8
    qweight = np.zeros((2, N), np.int64)
    qweight[0, :] = 0x76543210
    qweight[1, :] = 0xFEDCBA98
    qweight = qweight.astype(np.uint32).view(np.int32)
    qzeros = np.zeros((2, 1), np.int32)
    scales = _f16(np.array([[1.0] * N, [2.0] * N]))
    g_idx = np.array([1] * 8 + [0] * 8, np.int32)
    W = oracle.gptq_dequant_f64(qweight, scales, qzeros, g_idx, K, N, gs)
    i = np.arange(K)
    assert np.array_equal(W[0], np.where(i < 8, 2.0, 1.0) * (i - 1))
    Wid = oracle.gptq_dequant_f64(qweight, scales, qzeros, None, K, N, gs)
    assert np.array_equal(Wid[0], np.where(i < 8, 1.0, 2.0) * (i - 1))


def test_gptq_equals_mlx_affine_cross_layout():
    """GPTQ with stored zero 7 (zero 8) and scale s equals MLX affine with the same codes,
    scale s and bias -8s: two layouts transposed against each other must give one W."""
    rng = np.random.default_rng(21)
    K, N, gs = 128, 16, 32
    codes = rng.integers(0, 16, size=(N, K)).astype(np.int64)            # [out, in]
    s = 2.0 ** rng.integers(-6, -2, size=(K // gs, N))                    # [groups, out]
    qweight = np.zeros((K // 8, N), np.int64)
    for j in range(8):
        qweight |= codes.T.reshape(K // 8, 8, N)[:, j, :] << (4 * j)
    qweight = qweight.astype(np.uint32).view(np.int32)
    qzeros = np.full((K // gs, N // 8), 0x77777777, np.int64).astype(np.uint32).view(np.int32)
    Wg = oracle.gptq_dequant_f64(qweight, _f16(s).reshape(K // gs, N), qzeros, None, K, N, gs)
    wq = oracle.pack_affine(codes.astype(np.int32), 4)
    Wm = oracle.dequant_affine_f64(wq, _bf16(s.T).reshape(N, K // gs), _bf16(-8 * s.T).reshape(N, K // gs),
                                   N, K, 4, gs)
    assert np.array_equal(Wg, Wm)


def test_gptq_qmm_against_numpy_and_permutation_invariance():
    """y = x . W^T (numpy matmul on the oracle's own dequantized W, exact inputs), and
    permuting in-features of x together with qweight rows and g_idx leaves y unchanged."""
    K, N, gs = 64, 16, 16
    qweight, scales, qzeros, g_idx = synth.gptq_quartet(K, N, gs, seed=4, permuted=True)
    rng = np.random.default_rng(2)
    x = (rng.integers(-8, 9, size=(3, K)) * 0.125).astype(np.float32)
    xb = _f16(x).reshape(3, K)
    args = (qweight.numpy(), synth.bits16(scales), qzeros.numpy())
    y = oracle.gptq_qmm(xb, *args, g_idx.numpy(), K, N, gs)
    W = oracle.gptq_dequant_f64(*args, g_idx.numpy(), K, N, gs)
    assert np.allclose(y, x.astype(np.float64) @ W.T, rtol=1e-13, atol=1e-13)
    # swap in-feature octets 0 and 1 (whole qweight rows) with their g_idx entries and x columns
    perm = np.r_[8:16, 0:8, 16:K]
    qw2 = qweight.numpy()[np.r_[1, 0, 2:K // 8]]
    y2 = oracle.gptq_qmm(_f16(x[:, perm]).reshape(3, K), qw2, args[1], args[2],
                         g_idx.numpy()[perm], K, N, gs)
    assert np.allclose(y2, y, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------- AWQ zero convention
def test_awq_worked_example_without_plus_one():
    """The GPTQ smoke-test inputs read with the AWQ convention: the page says AWQ does not
    re-add the 1, so the printed row [-1, ..., 14] moves up by exactly one to [0, ..., 15]."""
    rows = {r[0]: r[1:] for r in _golden_lines("gptq_worked_example.txt")}
    K, gs = int(rows["in_features"][0]), int(rows["group_size"][0])
    N = 8
    expected = np.array([float(v) for v in rows["row0"]]) + 1.0
    qweight = np.zeros((K // 8, N), np.int64)
    qweight[0, 0] = 0x76543210
    qweight[1, 0] = 0xFEDCBA98
    qweight = qweight.astype(np.uint32).view(np.int32)
    qzeros = np.zeros((K // gs, N // 8), np.int32)   # stored zero 0 -> zero 0
    scales = _f16(np.ones((K // gs, N)))
    assert np.array_equal(oracle.awq_dequant_f64(qweight, scales, qzeros, K, N, gs)[0], expected)
    W16 = oracle.awq_dequant_f16(qweight, scales, qzeros, K, N, gs)
    assert np.array_equal(np.array([oracle.f16_to_f64(h) for h in W16[0]]), expected)


def test_awq_zero_nibble_closed_form():
    """qzeros packed along OUT, zero taken as stored: W[o, i] = s_g * (i - z_o) for codes
    0..7, with a different scale per group (pins the group index i // gs and the nibble
    index o % 8 of word o // 8)."""
    K, N, gs = 16, 16, 8
    qweight = np.full((2, N), 0x76543210, np.int64).astype(np.uint32).view(np.int32)  # codes i % 8
    z = np.array([3, 0, 15, 7, 1, 2, 9, 4, 5, 6, 8, 10, 11, 12, 13, 14])
    words = [sum(int(z[8 * w + j]) << (4 * j) for j in range(8)) for w in range(2)]
    qzeros = np.array([words, words], np.int64).astype(np.uint32).view(np.int32)
    scales = _f16(np.array([[0.5] * N, [-2.0] * N]))
    W = oracle.awq_dequant_f64(qweight, scales, qzeros, K, N, gs)
    i = np.arange(K)
    for o in range(N):
        assert np.array_equal(W[o], np.where(i < 8, 0.5, -2.0) * (i % 8 - z[o]))


def test_awq_equals_gptq_with_stored_zero_minus_one():
    """The one stated difference: AWQ with stored zero z is GPTQ with stored zero z - 1
    (z >= 1, no g_idx), for every weight and for the matmul."""
    rng = np.random.default_rng(31)
    K, N, gs = 128, 24, 32
    qweight = rng.integers(0, 2**32, size=(K // 8, N), dtype=np.uint64).astype(np.uint32).view(np.int32)
    z = rng.integers(1, 16, size=(K // gs, N))
    pack = lambda zz: sum(zz.reshape(K // gs, N // 8, 8)[:, :, j].astype(np.int64) << (4 * j) for j in range(8))
    qz_awq = pack(z).astype(np.uint32).view(np.int32)
    qz_gptq = pack(z - 1).astype(np.uint32).view(np.int32)
    scales = _f16(rng.standard_normal((K // gs, N)) * 0.01).reshape(K // gs, N)
    Wa = oracle.awq_dequant_f64(qweight, scales, qz_awq, K, N, gs)
    assert np.array_equal(Wa, oracle.gptq_dequant_f64(qweight, scales, qz_gptq, None, K, N, gs))
    assert np.array_equal(oracle.awq_dequant_f16(qweight, scales, qz_awq, K, N, gs),
                          oracle.gptq_dequant_f16(qweight, scales, qz_gptq, None, K, N, gs))
    x = _f16((rng.integers(-8, 9, size=(3, K)) * 0.125).astype(np.float32)).reshape(3, K)
    ya = oracle.awq_qmm(x, qweight, scales, qz_awq, K, N, gs)
    assert np.array_equal(ya, oracle.gptq_qmm(x, qweight, scales, qz_gptq, None, K, N, gs))
    xf = np.array([[oracle.f16_to_f64(h) for h in row] for row in x])
    assert np.allclose(ya, xf @ Wa.T, rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------- W4A8
def test_quant_per_token_i8_properties():
    """Per token: sx = amax/127 (fp32), the argmax hits +-127, codes are the nearest grid
    point, negating x negates the codes, an all-zero row gives sx = 0 and q = 0."""
    x = synth.activations(6, 512, seed=5, outlier_frac=0.01)
    x[3] = 0
    xb = synth.bits16(x)
    qx, sx = oracle.quant_per_token_i8(xb)
    xf = x.float().numpy()
    for m in range(6):
        amax = np.float32(np.abs(xf[m]).max())
        assert sx[m] == np.float32(amax / np.float32(127.0))
        if amax == 0:
            assert np.all(qx[m] == 0)
            continue
        assert abs(int(qx[m, np.argmax(np.abs(xf[m]))])) == 127
        dist = np.abs(xf[m].astype(np.float64)[:, None] - np.arange(-127, 128)[None, :] * float(sx[m]))
        chosen = dist[np.arange(512), qx[m].astype(np.int64) + 127]
        assert np.all(chosen <= dist.min(axis=1) + 1e-6 * float(sx[m]))
    qn, sn = oracle.quant_per_token_i8(synth.bits16(-x))
    assert np.array_equal(qn, -qx) and np.array_equal(sn, sx)


def test_qpack_sym_i4_nibbles_and_grid():
    """Two's-complement nibbles, lowest k first ([0..7] -> 0x76543210, seven -1 then 7 ->
    0x7FFFFFFF, a constant -1 row -> all -7 = 0x99999999), sw = max|w|/7, and each code is
    the nearest point of s*[-8..7]."""
    w = np.array([[0, 1, 2, 3, 4, 5, 6, 7], [-1] * 7 + [7], [7, -7, 0, 0, 0, 0, 0, 0], [-1] * 8],
                 np.float32)
    wq, sw, codes = oracle.qpack_sym_i4(w)
    assert wq[:, 0].tolist() == [0x76543210, 0x7FFFFFFF, 0x00000097, 0x99999999]
    assert sw.tolist() == [1.0, 1.0, 1.0, np.float32(np.float32(1.0) / np.float32(7.0))]
    W = synth.weights(16, 256, seed=8).numpy()
    wq, sw, codes = oracle.qpack_sym_i4(W)
    grid = np.arange(-8, 8, dtype=np.float64)
    for n in range(16):
        assert sw[n] == np.float32(np.float32(np.abs(W[n]).max()) / np.float32(7.0))
        dist = np.abs(W[n].astype(np.float64)[:, None] - grid[None, :] * float(sw[n]))
        chosen = dist[np.arange(256), codes[n] + 8]
        assert np.all(chosen <= dist.min(axis=1) + 1e-6 * float(sw[n]))
    assert codes.min() >= -7 and codes.max() <= 7     # |w/sw| <= 7, so -8 never occurs


def test_gemm_i8i4_integer_product_and_overflow_flag():
    """acc equals numpy's int64 product of the known int8 and int4 codes (pins signed nibble
    decoding and the K-index pairing); y = acc*sx*sw; the flag reports int32 overflow."""
    rng = np.random.default_rng(3)
    M, N, K = 4, 9, 64
    qx = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    cw = rng.integers(-8, 8, size=(N, K)).astype(np.int64)
    wq = np.zeros((N, K // 8), np.int64)
    for j in range(8):
        wq |= (cw.reshape(N, K // 8, 8)[:, :, j] & 0xF) << (4 * j)
    wq = wq.astype(np.uint32)
    sx = rng.random(M).astype(np.float32)
    sw = rng.random(N).astype(np.float32)
    acc, y, ovf = oracle.gemm_i8i4(qx, sx, wq, sw, N, K)
    ref = qx.astype(np.int64) @ cw.T
    assert np.array_equal(acc, ref) and not ovf
    assert np.allclose(y, ref * sx.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :],
                       rtol=1e-15, atol=0)
    Kb = 1 << 22          # 127 * 8 * 2^22 > 2^31 - 1
    acc2, _, ovf2 = oracle.gemm_i8i4(np.full((1, Kb), -127, np.int8), np.ones(1, np.float32),
                                     np.full((1, Kb // 8), 0x88888888, np.uint32), np.ones(1, np.float32),
                                     1, Kb)
    assert ovf2 and acc2[0, 0] == 127 * 8 * Kb


def test_symmetric_quant_error_bounds():
    """Symmetric quantizers (QAT section): every element is within half a step of its
    reconstruction, i.e. the code is the nearest grid point of s*[-qMax..qMax]."""
    W = synth.weights(64, 512, seed=12).numpy()
    wq, sw, codes = oracle.qpack_sym_i4(W)
    # half a step, plus the fp32 rounding of the step itself magnified by |q|
    err = np.abs(codes * sw[:, None].astype(np.float64) - W)
    assert np.all(err <= sw[:, None] * (0.5 + np.abs(codes) * 2.0 ** -23))
    x = torch.from_numpy(W / 0.02).to(torch.bfloat16)
    qx, sx = oracle.quant_per_token_i8(synth.bits16(x))
    xf = x.float().numpy()
    q = qx.astype(np.float64)
    assert np.all(np.abs(q * sx[:, None] - xf) <= sx[:, None] * (0.5 + np.abs(q) * 2.0 ** -23))


# --------------------------------------------------------------------- W8A8
def test_qpack_sym_i8_hand_values():
    """Per-row symmetric int8 with qMax = 127 (QAT section, bits = 8): a row whose max is 127
    has sw = 1, so codes are the row itself rounded half to even (63.5 -> 64, 0.5 -> 0,
    -2.5 -> -2, 1.5 -> 2); a constant -1 row maps to -127; a zero row gives sw = 0, codes 0;
    clipping is to [-127, 127] (never -128)."""
    w = np.zeros((3, 16), np.float32)
    w[0, :8] = [127, -127, 63.5, 0.5, -2.5, 1.5, -0.25, 100.49]
    w[1, :] = -1.0
    wq, sw = oracle.qpack_sym_i8(w)
    assert sw.tolist() == [1.0, np.float32(np.float32(1.0) / np.float32(127.0)), 0.0]
    assert wq[0, :8].tolist() == [127, -127, 64, 0, -2, 2, 0, 100]
    assert np.all(wq[0, 8:] == 0) and np.all(wq[1] == -127) and np.all(wq[2] == 0)


def test_qpack_sym_i8_nearest_grid_point():
    """Every code is the nearest point of sw*[-127..127] (so the reconstruction error is at
    most half a step, the page's 1/qMax bound), the row max maps to +-127, and negating the
    row negates the codes."""
    W = synth.weights(16, 384, seed=13).numpy()
    wq, sw = oracle.qpack_sym_i8(W)
    grid = np.arange(-127, 128, dtype=np.float64)
    for n in range(16):
        assert sw[n] == np.float32(np.float32(np.abs(W[n]).max()) / np.float32(127.0))
        assert abs(int(wq[n, np.argmax(np.abs(W[n]))])) == 127
        dist = np.abs(W[n].astype(np.float64)[:, None] - grid[None, :] * float(sw[n]))
        chosen = dist[np.arange(384), wq[n].astype(np.int64) + 127]
        # the decision is taken on the fp32 quotient w/sw, off by up to 127 * 2^-24 steps
        assert np.all(chosen <= dist.min(axis=1) + 2.0 ** -16 * float(sw[n]))
    wn, sn = oracle.qpack_sym_i8(-W)
    assert np.array_equal(wn, -wq) and np.array_equal(sn, sw)


def test_gemm_i8i8_integer_product_and_overflow_flag():
    """acc equals numpy's int64 product of the int8 codes (pins the K pairing and the [N, K]
    weight orientation: a transposed operand fails for N != M); y = acc*sx*sw; the flag
    reports int32 overflow."""
    rng = np.random.default_rng(4)
    M, N, K = 5, 7, 96
    qx = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    sx = rng.random(M).astype(np.float32)
    sw = rng.random(N).astype(np.float32)
    acc, y, ovf = oracle.gemm_i8i8(qx, sx, wq, sw, N, K)
    ref = qx.astype(np.int64) @ wq.astype(np.int64).T
    assert np.array_equal(acc, ref) and not ovf
    assert np.allclose(y, ref * sx.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :],
                       rtol=1e-15, atol=0)
    Kb = 1 << 18          # 127 * 127 * 2^18 > 2^31 - 1
    acc2, _, ovf2 = oracle.gemm_i8i8(np.full((1, Kb), 127, np.int8), np.ones(1, np.float32),
                                     np.full((1, Kb), -127, np.int8), np.ones(1, np.float32), 1, Kb)
    assert ovf2 and acc2[0, 0] == -127 * 127 * Kb


# --------------------------------------------------------------------- fused decode products
def test_silu_mul_closed_forms():
    """silu(g) = g * sigmoid(g): silu(0) = 0, silu(ln 3) = (3/4) ln 3, silu(-ln 3) = -(1/4) ln 3
    (sigmoid(ln 3) = 3/4), silu(g) - silu(-g) = g for every g (sigmoid(g) + sigmoid(-g) = 1),
    and the up factor multiplies (gate and up are not interchangeable)."""
    ln3 = np.log(3.0)
    g = np.array([0.0, ln3, -ln3, 2.0, -2.0, 0.5], np.float32)
    gb = _bf16(g)
    gv = np.array([oracle.bf16_to_f64(h) for h in gb])          # the bf16 values actually used
    one = _bf16(np.ones_like(g))
    h = oracle.silu_mul(gb, one)
    assert h[0] == 0.0
    assert np.isclose(h[1], gv[1] / (1 + 1 / np.exp(gv[1])), rtol=1e-15)
    assert np.isclose(h[1], 0.75 * gv[1], rtol=2e-2)            # bf16(ln 3) is ln 3 to 2^-8
    assert np.isclose(h[2], -0.25 * (-gv[2]), rtol=2e-2)
    assert np.allclose(h[[1, 3]] - h[[2, 4]], gv[[1, 3]], rtol=1e-15, atol=0)
    up = _bf16(np.full_like(g, -3.0))
    assert np.allclose(oracle.silu_mul(gb, up), -3.0 * h, rtol=1e-15, atol=0)
    # swapping gate and up changes the product: silu(2) * 1 != silu(1) * 2
    a = oracle.silu_mul(_bf16(np.array([2.0], np.float32)), _bf16(np.array([1.0], np.float32)))
    b = oracle.silu_mul(_bf16(np.array([1.0], np.float32)), _bf16(np.array([2.0], np.float32)))
    assert abs(a[0] - b[0]) > 0.1


def _identity_affine(n, bits, gs):
    """Packed MLX weights of the n x n identity: code 1 on the diagonal, scale 1, bias 0."""
    codes = np.eye(n, dtype=np.int32)
    wq = oracle.pack_affine(codes, bits)
    G = n // gs
    return wq, _bf16(np.ones((n, G))).reshape(n, G), _bf16(np.zeros((n, G))).reshape(n, G)


def test_qmv_silu_gate_identity_weight_and_residual():
    """With W = I, y[t, n] = silu(gate[t, n]) * up[t, n] exactly (pins the elementwise product and
    the [out, in] orientation); the residual adds resid[t, n] to every output."""
    n, bits, gs = 64, 4, 32
    wq, sc, bi = _identity_affine(n, bits, gs)
    rng = np.random.default_rng(7)
    gate = _bf16(rng.standard_normal((3, n)).astype(np.float32) * 2).reshape(3, n)
    up = _bf16(rng.standard_normal((3, n)).astype(np.float32)).reshape(3, n)
    y = oracle.qmv_silu_gate(gate, up, wq, sc, bi, n, n, bits, gs)
    assert np.array_equal(y, oracle.silu_mul(gate, up))
    res = _bf16(rng.standard_normal((3, n)).astype(np.float32)).reshape(3, n)
    yr = oracle.qmv_silu_gate(gate, up, wq, sc, bi, n, n, bits, gs, resid_bf16=res)
    rv = np.array([[oracle.bf16_to_f64(h) for h in row] for row in res])
    assert np.allclose(yr - y, rv, rtol=0, atol=1e-12)


def test_qmv_silu_gate_is_matmul_of_silu_product():
    """A general weight: y = (silu(gate) * up) . W^T (numpy matmul on the oracle's dequantized W),
    for two row samples."""
    N, K, bits, gs = 24, 128, 8, 64
    w = synth.weights(N, K, seed=17).numpy()
    wq, sc, bi, _ = oracle.qpack_affine(w, bits, gs)
    rng = np.random.default_rng(8)
    gate = _bf16(rng.standard_normal((4, K)).astype(np.float32)).reshape(4, K)
    up = _bf16(rng.standard_normal((4, K)).astype(np.float32)).reshape(4, K)
    W = oracle.dequant_affine_f64(wq, sc, bi, N, K, bits, gs)
    y = oracle.qmv_silu_gate(gate, up, wq, sc, bi, N, K, bits, gs, rows=[3, 1])
    assert np.allclose(y, oracle.silu_mul(gate, up)[[3, 1]] @ W.T, rtol=1e-12, atol=1e-14)


def test_w4a8_fused_exact_grid_case():
    """x on the exact int8 grid of its own scale: x = q * 2^-3 with max|q| = 127 gives sx = 2^-3 and
    the codes q back unchanged; acc = q . c^T for known int4 codes; y = acc * sx * sw."""
    q = np.array([[127, -64, 0, 1, -127, 5, 3, -2] * 4, [-127, 2, 2, 2, 2, 2, 2, 2] * 4], np.int64)
    K = q.shape[1]
    x = _bf16((q * 0.125).astype(np.float32)).reshape(2, K)
    rng = np.random.default_rng(9)
    codes = rng.integers(-8, 8, size=(3, K)).astype(np.int64)
    wq = np.zeros((3, K // 8), np.int64)
    for j in range(8):
        wq |= (codes.reshape(3, K // 8, 8)[:, :, j] & 0xF) << (4 * j)
    sw = np.array([0.5, 0.25, 2.0], np.float32)
    acc, y, ovf = oracle.w4a8_fused(x, wq.astype(np.uint32), sw, 3, K)
    assert not ovf and np.array_equal(acc, q @ codes.T)
    assert np.array_equal(y, (q @ codes.T) * 0.125 * sw.astype(np.float64)[None, :])
