"""Pins of the scalar CPU oracle to facts outside itself (no GPU needed).

Each test ties one oracle function to something the pages or mathematics
fix: hand-worked examples from the bitnet-cpu page's definitions (golden
files), brute force over tiny inputs, closed forms, library special cases
(torch / numpy evaluations of the same definition), and invariants.
"""
import itertools
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32_to_bf16_bits_np(f):
    """Independent RNE narrowing in numpy (for building inputs only)."""
    u = np.asarray(f, np.float32).view(np.uint32).astype(np.uint64)
    lower = u & 0xFFFF
    upper = u >> 16
    up = (lower > 0x8000) | ((lower == 0x8000) & ((upper & 1) == 1))
    return (upper + up.astype(np.uint64)).astype(np.uint16)


def bf16_to_f32(bits):
    return synth.bf16_bits_to_f32(np.asarray(bits, np.uint16))


# --------------------------------------------------------------------- pack

def _pack_golden():
    rows = []
    with open(os.path.join(GOLDEN, "pack_examples.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            *w, b = line.split()
            rows.append(([int(v) for v in w], int(b, 16)))
    return rows


def test_pack_golden_examples():
    rows = _pack_golden()
    assert len(rows) >= 5
    for w, byte in rows:
        got = oracle.pack(np.array([w], np.int8))
        assert got.shape == (1, 1)
        assert int(got[0, 0]) == byte, (w, hex(int(got[0, 0])), hex(byte))


def test_pack_brute_force_all_81_tuples():
    tuples = list(itertools.product((-1, 0, 1), repeat=4))
    w = np.array(tuples, np.int8)              # [81, 4] -> one byte per row
    packed = oracle.pack(w)[:, 0]
    assert len(set(packed.tolist())) == 81     # injective
    for t, b in zip(tuples, packed.tolist()):
        fields = [(b >> (2 * i)) & 3 for i in range(4)]
        assert all(f in (1, 2, 3) for f in fields)
        assert [f - 2 for f in fields] == list(t)  # element i in bits 2i..2i+1


def test_pack_row_layout_and_roundtrip():
    k = synth.key(99, 0, synth.T_WEIGHT)
    w = synth.ternary(k, 37, 96)
    p = oracle.pack(w)
    assert p.shape == (37, 24) and p.dtype == np.uint8
    # byte j of row n covers elements 4j..4j+3 of that row only
    for n in (0, 5, 36):
        for j in (0, 7, 23):
            assert int(p[n, j]) == int(oracle.pack(w[n:n + 1, 4 * j:4 * j + 4])[0, 0])
    assert np.array_equal(oracle.unpack(p, 96), w)


def test_pack_of_unpack_is_identity_on_valid_bytes():
    rng = np.random.default_rng(3)
    fields = rng.integers(1, 4, size=(16, 32, 4))
    bytes_ = (fields[..., 0] | fields[..., 1] << 2 | fields[..., 2] << 4
              | fields[..., 3] << 6).astype(np.uint8)
    assert np.array_equal(oracle.pack(oracle.unpack(bytes_, 128)), bytes_)


def test_pack_rejects_out_of_range_and_bad_k():
    with pytest.raises(oracle.OracleError):
        oracle.pack(np.array([[0, 2, 0, 0]], np.int8))
    with pytest.raises(oracle.OracleError):
        oracle.pack(np.array([[0, -2, 0, 0]], np.int8))
    with pytest.raises(oracle.OracleError):
        oracle.pack(np.zeros((2, 6), np.int8))


def test_unpack_code_zero_decodes_to_minus_two():
    # 0b00 is never produced by pack; decode is code - 2 for every code.
    assert oracle.unpack(np.array([[0x00]], np.uint8), 4).tolist() == [[-2] * 4]
    assert oracle.unpack(np.array([[0xE4]], np.uint8), 4).tolist() == [[-2, -1, 0, 1]]


# ----------------------------------------------------------------- quantize

def _quant_golden():
    rows = []
    with open(os.path.join(GOLDEN, "quantize_examples.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            xs, qs, ss = [p.split(":", 1)[1].strip() for p in line.split("|")]
            rows.append(([float(v) for v in xs.split()],
                         [int(v) for v in qs.split()], int(ss, 16)))
    return rows


def test_quantize_golden_examples():
    rows = _quant_golden()
    assert len(rows) >= 5
    for xs, qs, sbits in rows:
        bits = f32_to_bf16_bits_np(np.array([xs], np.float32))
        q, s = oracle.quantize(bits)
        assert q[0].tolist() == qs, (xs, q[0].tolist(), qs)
        assert int(s[0]) == sbits, (xs, hex(int(s[0])), hex(sbits))


def test_quantize_invariants_random_rows():
    k = synth.key(98, 0, synth.T_ACT)
    x = synth.act_bf16(k, 64, 1000)
    q, s = oracle.quantize(x)
    xf = bf16_to_f32(x).astype(np.float64)
    absmax = np.maximum(np.abs(xf).max(axis=1), 1e-5)
    s32 = (np.float32(1) * absmax.astype(np.float32)) / np.float32(127)
    assert np.all(np.abs(q.astype(np.int32)) <= 127)
    assert np.all(np.abs(q).max(axis=1) == 127)           # the absmax maps to 127
    err = np.abs(xf / s32.astype(np.float64)[:, None] - q)
    assert err.max() <= 0.5 + 1e-5                          # round to nearest
    # stored scale is the bf16 rounding of absmax / 127 (within half a bf16 ulp)
    sf = bf16_to_f32(s).astype(np.float64)
    rel = np.abs(sf - absmax / 127.0) / (absmax / 127.0)
    assert rel.max() <= 2.0 ** -8 + 1e-7


def test_quantize_matches_torch_fp32_evaluation():
    """Library special case: the page's torch expression evaluated in fp32."""
    torch = pytest.importorskip("torch")
    k = synth.key(97, 0, synth.T_ACT)
    x = synth.act_bf16(k, 257, 2048)
    # add exact ties: entries equal to (j + 0.5) * scale for a power-of-two scale
    x[0, :8] = f32_to_bf16_bits_np(np.array([127, 0.5, 1.5, 2.5, -0.5, -1.5, 3.5, -2.5], np.float32))
    q, s = oracle.quantize(x)
    xt = torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).float()
    absmax = xt.abs().amax(dim=-1, keepdim=True).clamp(min=1e-5)
    scale = absmax / 127.0
    qt = (xt / scale).round().clamp(-127, 127).to(torch.int8)
    st = scale.squeeze(-1).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(qt.numpy(), q)
    assert np.array_equal(st, s)


def test_quantize_f32_golden_examples():
    """fp32 rows (the bitnet-cpu page also takes float32 activations), worked
    by hand from the page's quantize_activation: s = absmax / 127."""
    x = np.array([[254.0, 3.0, -5.0, 1.0],            # s = 2: 1.5 -> 2, -2.5 -> -2, 0.5 -> 0
                  [127.0, 0.3, -63.5, 1.0000001],     # s = 1: -63.5 -> -64 (even), 0.3 -> 0
                  [0.0, 0.0, 0.0, 0.0]], np.float32)  # clamped absmax: q = 0
    q, s = oracle.quantize_f32(x)
    assert q.tolist() == [[127, 2, -2, 0], [127, 0, -64, 1], [0, 0, 0, 0]]
    assert s[0] == 0x4000 and s[1] == 0x3F80
    assert s[2] == f32_to_bf16_bits_np(np.float32(1e-5) / np.float32(127.0))


def test_quantize_f32_matches_torch_fp32_evaluation():
    """Library special case: the page's expression on float32 tensors."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(11)
    x = rng.standard_normal((129, 1536)).astype(np.float32)
    x[:, ::97] *= 20.0
    x[0, :8] = np.array([127, 0.5, 1.5, 2.5, -0.5, -1.5, 3.5, -2.5], np.float32)  # exact ties
    q, s = oracle.quantize_f32(x)
    xt = torch.from_numpy(x.copy())
    absmax = xt.abs().amax(dim=-1, keepdim=True).clamp(min=1e-5)
    scale = absmax / 127.0
    qt = (xt / scale).round().clamp(-127, 127).to(torch.int8)
    st = scale.squeeze(-1).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(qt.numpy(), q)
    assert np.array_equal(st, s)


def test_quantize_f32_agrees_with_bf16_path_on_bf16_values():
    """Rows whose values are bf16 give the same codes and scales either way."""
    x = synth.act_bf16(synth.key(97, 3, synth.T_ACT), 33, 640)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    assert [a.tolist() for a in oracle.quantize(x)] == [a.tolist() for a in oracle.quantize_f32(xf)]
    p = oracle.pack(synth.ternary(synth.key(97, 3, synth.T_WEIGHT), 40, 640))
    sw = np.array([0.05], np.float32)
    assert np.array_equal(oracle.linear(x, p, sw), oracle.linear_f32(xf, p, sw))


def test_f32_to_bf16_matches_torch_rounding():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(5)
    u = rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32)
    u[:4000] = (u[:4000] & 0xFFFF0000) | 0x8000      # exact ties
    f = u.view(np.float32)
    f = f[np.isfinite(f)]
    ours = np.array([oracle.f32_to_bf16(float(v)) for v in f[:6000]], np.uint16)
    ref = torch.from_numpy(f[:6000].copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# ---------------------------------------------------------------------- acc

def _brute_acc(q, w):
    M, K = q.shape
    N = w.shape[0]
    out = np.zeros((M, N), np.int64)
    for m in range(M):
        for n in range(N):
            s = 0
            for k in range(K):
                s += int(q[m, k]) * int(w[n, k])
            out[m, n] = s
    return out


@pytest.mark.parametrize("M,N,K", [(1, 1, 4), (3, 5, 8), (7, 2, 64), (8, 8, 32)])
def test_acc_brute_force_tiny(M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    q = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    w = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    got = oracle.acc(q, oracle.pack(w))
    assert np.array_equal(got, _brute_acc(q, w))


def test_acc_exhaustive_k4():
    # every ternary 4-vector against a fixed set of activation rows
    w = np.array(list(itertools.product((-1, 0, 1), repeat=4)), np.int8)
    q = np.array([[1, 2, 3, 4], [-127, 127, -127, 127], [5, -7, 0, 9]], np.int8)
    assert np.array_equal(oracle.acc(q, oracle.pack(w)), _brute_acc(q, w))


def test_acc_matches_float64_matmul():
    """Library special case: integer-valued float64 matmul is exact here."""
    k = synth.key(96, 0, synth.T_WEIGHT)
    w = synth.ternary(k, 96, 512)
    rng = np.random.default_rng(9)
    q = rng.integers(-127, 128, size=(13, 512)).astype(np.int8)
    ref = q.astype(np.float64) @ w.astype(np.float64).T
    assert np.array_equal(oracle.acc(q, oracle.pack(w)), ref.astype(np.int64))


def test_acc_special_cases():
    rng = np.random.default_rng(11)
    K = 64
    q = rng.integers(-127, 128, size=(5, K)).astype(np.int8)
    zero = np.zeros((K, K), np.int8)
    eye = np.eye(K, dtype=np.int8)
    ones = np.ones((3, K), np.int8)
    assert np.all(oracle.acc(q, oracle.pack(zero)) == 0)
    assert np.array_equal(oracle.acc(q, oracle.pack(eye)), q.astype(np.int32))
    assert np.array_equal(oracle.acc(q, oracle.pack(-eye)), -q.astype(np.int32))
    rs = q.astype(np.int32).sum(axis=1)
    assert np.array_equal(oracle.acc(q, oracle.pack(ones)), np.repeat(rs[:, None], 3, 1))


def test_acc_extreme_magnitude():
    K = 11008
    q = np.full((1, K), -127, np.int8)
    w = np.full((2, K), 1, np.int8)
    w[1] = -1
    got = oracle.acc(q, oracle.pack(w))
    assert got.tolist() == [[-127 * K, 127 * K]]


# ----------------------------------------------------------------- epilogue

def test_epilogue_power_of_two_scales_closed_form():
    # acc * 2^a * 2^b is exact in fp32, so out = bf16_rne(acc * 2^(a+b)).
    rng = np.random.default_rng(12)
    acc = rng.integers(-2 ** 20, 2 ** 20, size=(4, 64)).astype(np.int32)
    sa = f32_to_bf16_bits_np(np.array([2.0 ** -7, 2.0 ** -3, 1.0, 2.0 ** 4], np.float32))
    sw = np.array([2.0 ** -5], np.float32)
    out = oracle.epilogue(acc, sa, sw)
    exact = acc.astype(np.float64) * np.array([2.0 ** -12, 2.0 ** -8, 2.0 ** -5, 2.0 ** -1])[:, None]
    assert np.array_equal(out, f32_to_bf16_bits_np(exact.astype(np.float32)))


def test_epilogue_within_one_ulp_of_exact_product():
    rng = np.random.default_rng(13)
    acc = rng.integers(-200000, 200000, size=(16, 256)).astype(np.int32)
    sa = f32_to_bf16_bits_np(rng.uniform(0.001, 0.2, 16).astype(np.float32))
    sw = rng.uniform(0.01, 0.1, 256).astype(np.float32)
    out = oracle.epilogue(acc, sa, sw)
    exact = acc.astype(np.float64) * bf16_to_f32(sa).astype(np.float64)[:, None] * sw.astype(np.float64)[None, :]
    got = bf16_to_f32(out).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact), 1e-30))) - 7)
    assert np.all(np.abs(got - exact) <= ulp + 1e-30)
    # per-column scale is honoured (len N) and a scalar is broadcast (len 1)
    out1 = oracle.epilogue(acc, sa, sw[:1])
    outN = oracle.epilogue(acc, sa, np.full(256, sw[0], np.float32))
    assert np.array_equal(out1, outN)


# --------------------------------------------------------------- composition

def test_linear_is_quantize_then_gemm():
    kw = synth.key(95, 0, synth.T_WEIGHT)
    kx = synth.key(95, 0, synth.T_ACT)
    w = synth.ternary(kw, 200, 256)
    x = synth.act_bf16(kx, 9, 256)
    sw = synth.scale_wt(synth.key(95, 0, synth.T_SCALE_WT))
    p = oracle.pack(w)
    q, sa = oracle.quantize(x)
    assert np.array_equal(oracle.linear(x, p, sw), oracle.gemm(q, p, sa, sw))
    assert np.array_equal(oracle.linear(x, p, sw, threads=4), oracle.linear(x, p, sw))
    assert np.array_equal(oracle.gemm_threads(q, p, sa, sw, 3), oracle.gemm(q, p, sa, sw))
    assert np.array_equal(oracle.linear_cols_threads(x, p, sw, 7), oracle.linear(x, p, sw))
    swn = synth.uniform_f32(synth.key(95, 1, 3), 200, 0.01, 0.1)
    assert np.array_equal(oracle.linear_cols_threads(x, p, swn, 5), oracle.linear(x, p, swn))


def test_linear_close_to_float64_dequantised_product():
    """The whole layer tracks the real-valued product of its quantised parts."""
    kw = synth.key(94, 0, synth.T_WEIGHT)
    kx = synth.key(94, 0, synth.T_ACT)
    w = synth.ternary(kw, 64, 512)
    x = synth.act_bf16(kx, 4, 512)
    sw = np.array([0.05], np.float32)
    p = oracle.pack(w)
    q, sa = oracle.quantize(x)
    y = bf16_to_f32(oracle.linear(x, p, sw)).astype(np.float64)
    ref = (q.astype(np.float64) @ w.astype(np.float64).T) * bf16_to_f32(sa)[:, None] * 0.05
    assert np.allclose(y, ref, rtol=2 ** -7, atol=1e-6)


# --------------------------------------------------- absmean ternarisation

def test_ternarize_golden_example():
    """Worked by hand from BitLinear.from_dense on the bitnet-cpu page:
    mean|w| = 4.1 / 4 = 1.025; w / gamma = 0.49, -1.46, 0.098, 1.95."""
    w = np.array([[0.5, -1.5, 0.1, 2.0], [0.0, 0.0, 0.0, 0.0]], np.float32)
    wt, sc = oracle.ternarize_absmean(w)
    assert wt.tolist() == [[0, -1, 0, 1], [0, 0, 0, 0]]
    assert sc[0] == np.float32(1.0234375)                        # bf16(1.025)
    bits = f32_to_bf16_bits_np(np.float32(1e-8))                 # zero row: gamma = eps
    assert sc[1] == (np.uint32(bits) << 16).view(np.float32)
    wt, sc = oracle.ternarize_absmean(w, per_row=False)          # mean over 8 = 0.5125
    assert wt.tolist() == [[1, -1, 0, 1], [0, 0, 0, 0]]          # 0.5 / 0.5125 = 0.976 -> 1
    assert sc[0] == np.float32(0.51171875)                       # bf16(0.5125)


def test_ternarize_recovers_scaled_ternary_matrices():
    """w = gamma_n * t with t ternary: mean|w| = gamma_n * nnz / K <= gamma_n,
    so w / mean is 0 or at least 1 in magnitude and the codes are t."""
    rng = np.random.default_rng(3)
    t = rng.choice(np.array([-1, 0, 1], np.int8), size=(64, 320), p=[0.3, 0.4, 0.3])
    t[:, 0] = 1
    g = rng.uniform(0.01, 0.5, size=(64, 1)).astype(np.float32)
    wt, _ = oracle.ternarize_absmean(t.astype(np.float32) * g)
    assert np.array_equal(wt, t)
    wt, _ = oracle.ternarize_absmean(t.astype(np.float32) * np.float32(0.07), per_row=False)
    assert np.array_equal(wt, t)


def test_ternarize_matches_float64_definition():
    """Library special case: for ordinary weights the float64 sum of |w| is
    exact, so gamma = max(float32(sum / K), eps) and the codes follow with a
    float32 division and round-half-even."""
    rng = np.random.default_rng(9)
    w = (rng.standard_normal((96, 2560)) * 0.02).astype(np.float32)
    w[0, :4] = [0.0, 0.0, 0.0, 0.0]
    for per_row, eps in ((True, 1e-8), (False, 1e-5)):
        wt, sc = oracle.ternarize_absmean(w, per_row=per_row)
        a = np.abs(w).astype(np.float64)
        mean = a.sum(axis=1) / w.shape[1] if per_row else np.array([a.sum() / w.size])
        gamma = np.maximum(mean.astype(np.float32), np.float32(eps))
        gb = (f32_to_bf16_bits_np(gamma).astype(np.uint32) << 16).view(np.float32)
        assert np.array_equal(sc, gb)
        ref = np.clip(np.rint(w / gamma.reshape(-1, 1)), -1, 1).astype(np.int8)
        assert np.array_equal(wt, ref)


def test_ternarize_rejects_non_finite():
    w = np.zeros((2, 8), np.float32)
    w[1, 3] = np.inf
    with pytest.raises(Exception):
        oracle.ternarize_absmean(w)


# --------------------------------------------------------------- bias


def test_linear_bias_rounding_worked_examples():
    """y + bias in bf16 (BitLinear.forward on the bitnet-cpu page). The layer
    outputs exactly +1.0 or -1.0 (one input 127 -> q = 127 at scale 1.0, one
    weight +1 or -1, scale_wt = 1/127: 127 * fl(1/127) rounds to bf16 1.0).
    bf16 has 8 significant bits, so an ulp at 1.0 is 2^-7 and:
    bias 2^-9 (a quarter ulp) -> 1.0; 2^-8 (half an ulp, a tie) -> 1.0, the
    even neighbour; 2^-7 -> 1.0078125; 0.5 -> 1.5; -1.0 + 0 -> -1.0."""
    K = 32
    x = np.zeros((1, K), np.uint16)
    x[0, 0] = f32_to_bf16_bits_np(np.float32(127.0))
    w = np.zeros((5, K), np.int8)
    w[:4, 0] = 1
    w[4, 0] = -1
    p = oracle.pack(w)
    sw = np.array([np.float32(1.0) / np.float32(127.0)], np.float32)
    bias = f32_to_bf16_bits_np(np.array([2 ** -9, 2 ** -8, 2 ** -7, 0.5, 0.0], np.float32))
    yb = (oracle.linear(x, p, sw).astype(np.uint32) << 16).view(np.float32)[0]
    assert yb.tolist() == [1.0, 1.0, 1.0, 1.0, -1.0]
    y = (oracle.linear_bias(x, p, sw, bias).astype(np.uint32) << 16).view(np.float32)[0]
    assert y.tolist() == [1.0, 1.0, 1.0078125, 1.5, -1.0]


def test_linear_bias_matches_torch_bf16_addition():
    torch = pytest.importorskip("torch")
    x = synth.act_bf16(synth.key(91, 0, synth.T_ACT), 9, 256)
    p = oracle.pack(synth.ternary(synth.key(91, 0, synth.T_WEIGHT), 70, 256))
    sw = synth.uniform_f32(synth.key(91, 0, 3), 70, 0.01, 0.1)
    bias = f32_to_bf16_bits_np(np.random.default_rng(4).standard_normal(70).astype(np.float32))
    bias[:3] = [0x0000, 0x8000, 0x3F80]
    y = torch.from_numpy(oracle.linear(x, p, sw).view(np.int16).copy()).view(torch.bfloat16)
    b = torch.from_numpy(bias.view(np.int16).copy()).view(torch.bfloat16)
    ref = (y + b).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.linear_bias(x, p, sw, bias), ref)


# ------------------------------------------------------ RMSNorm -> quantise

def test_rmsnorm_worked_example():
    """x = [3, 4], g = 1, eps = 0: mean(x^2) = 12.5, r = 1/sqrt(12.5) =
    0.28284271; x * r = 0.84852814, 1.13137085 -> bf16 0.84765625, 1.1328125;
    the quantiser's s = 1.1328125 / 127, so q = [round(95.03), 127]."""
    x = f32_to_bf16_bits_np(np.array([[3.0, 4.0]], np.float32))
    g = f32_to_bf16_bits_np(np.array([1.0, 1.0], np.float32))
    z = (oracle.rmsnorm(x, g, 0.0).astype(np.uint32) << 16).view(np.float32)
    assert z.tolist() == [[0.84765625, 1.1328125]]
    q, s = oracle.rmsnorm_quantize(x, g, 0.0)
    assert q.tolist() == [[95, 127]]
    assert s[0] == f32_to_bf16_bits_np(np.float32(1.1328125) / np.float32(127.0))


def test_rmsnorm_invariant_under_power_of_two_scaling():
    """With eps = 0 every step scales exactly by powers of two, so x * 2^k
    gives the same normalised row, bit for bit."""
    x = synth.act_bf16(synth.key(89, 0, synth.T_ACT), 6, 512)
    g = f32_to_bf16_bits_np(np.random.default_rng(2).uniform(0.5, 1.5, 512).astype(np.float32))
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    z0 = oracle.rmsnorm(x, g, 0.0)
    for k in (-3, 5):
        xs = f32_to_bf16_bits_np(xf * np.float32(2.0 ** k))
        assert np.array_equal(oracle.rmsnorm(xs, g, 0.0), z0)


def test_rmsnorm_matches_torch_fp32_evaluation():
    """The usual RMSNorm in fp32 (as the transformers BitNet module writes
    it), on rows where torch's fp32 mean of squares is exact (small integer
    values, K a power of two)."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(8)
    xf = rng.integers(-8, 9, size=(17, 64)).astype(np.float32)
    xf[3] = 0.0
    gf = rng.uniform(0.25, 2.0, 64).astype(np.float32)
    x = f32_to_bf16_bits_np(xf)
    g = f32_to_bf16_bits_np(gf)
    eps = 1e-5
    xt = torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16)
    gt = torch.from_numpy(g.view(np.int16).copy()).view(torch.bfloat16)
    h = xt.float()
    var = h.pow(2).mean(-1, keepdim=True)
    y = (h * torch.rsqrt(var + eps)).to(torch.bfloat16)
    ref = (gt * y).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.rmsnorm(x, g, eps), ref)


def test_rmsnorm_zero_weight_gives_zero_codes():
    x = synth.act_bf16(synth.key(89, 1, synth.T_ACT), 3, 256)
    g = np.zeros(256, np.uint16)
    q, _ = oracle.rmsnorm_quantize(x, g, 1e-5)
    assert not q.any()


@pytest.mark.parametrize("M,N,K,threads", [(1, 37, 64, 8), (5, 3, 128, 8), (16, 300, 256, 7),
                                           (2, 1, 32, 4)])
def test_acc_threads_is_the_brute_force_sum(M, N, K, threads):
    """The threaded driver of the contraction (used by the full-size parity
    tests) against an int64 brute-force sum of the unpacked weights: the
    split over weight rows, including more threads than rows, changes no
    output."""
    rng = np.random.default_rng(M * 100 + N + K)
    q = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    w = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    ref = q.astype(np.int64) @ w.astype(np.int64).T
    got = oracle.acc_threads(q, oracle.pack(w), threads)
    assert got.dtype == np.int32
    assert np.array_equal(got.astype(np.int64), ref)
