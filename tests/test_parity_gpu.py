"""Parity of the CUDA path (through the C ABI) with the scalar CPU oracle.

Integer stages (packed bytes, int8 codes, bf16 scale bits, int32
accumulators) must match bit for bit. The method's stated tolerance for the
bf16 outputs is 1 bf16 ulp (relative error <= 2^-8); with round-half-even,
IEEE division and the epilogue's two fp32 products in a fixed order every
stage is a function of its inputs, so the kernels are held to exact equality
with the oracle's bf16 outputs (the tolerance stays the documented contract).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads as W
import bit_gemm_bitnet_b200 as bn
from helpers import bf16_bits, bf16_ulp_diff, f32_to_bf16_bits, to_dev

pytestmark = pytest.mark.gpu

BF16_ULP_TOL = 1


@pytest.fixture(autouse=True)
def _gpu(cuda_ok):
    yield
    bn.bitnet_device_status()


def weights(wl, layer, N, K, tensor=synth.T_WEIGHT, variant=0):
    return synth.ternary(synth.key(wl, layer, tensor, variant), N, K)


def acts(wl, layer, M, K, outliers=True, variant=0):
    return synth.act_bf16(synth.key(wl, layer, synth.T_ACT, variant), M, K,
                          outliers=outliers)


def sw_of(wl, layer, variant=0):
    return synth.scale_wt(synth.key(wl, layer, synth.T_SCALE_WT, variant))


def assert_bf16_close(got_bits, ref_bits):
    """Exact bf16 equality (the ulp distance is reported on a mismatch)."""
    d = bf16_ulp_diff(got_bits, ref_bits)
    assert d.max() <= BF16_ULP_TOL, f"max ulp {d.max()} at {np.unravel_index(d.argmax(), d.shape)}"
    assert np.array_equal(got_bits, ref_bits), (
        f"{int((d > 0).sum())} outputs differ by one ulp from the oracle")


# ------------------------------------------------------------------- pack

@pytest.mark.parametrize("N,K", [(1, 4), (7, 12), (512, 512), (640, 2560), (33, 6912)])
def test_pack_bitexact(N, K):
    w = weights(90, 0, N, K)
    got = bn.bitnet_pack_weights(to_dev(w)).cpu().numpy()
    assert np.array_equal(got, oracle.pack(w))


def test_pack_rejects_bad_values():
    w = weights(90, 1, 16, 64)
    w[3, 5] = 2
    with pytest.raises(bn.BitnetValueError):
        bn.bitnet_pack_weights(to_dev(w))


def test_pack_empty():
    out = bn.bitnet_pack_weights(torch.zeros((0, 8), dtype=torch.int8, device="cuda"))
    assert out.shape == (0, 2)


# --------------------------------------------------------------- quantise

@pytest.mark.parametrize("M,K", [(1, 32), (3, 96), (17, 512), (300, 2560), (64, 4096),
                                 (5, 11008), (2, 16416), (3, 20000)])
def test_quantize_bitexact(M, K):
    x = acts(91, K, M, K)
    q_ref, s_ref = oracle.quantize(x)
    q, s = bn.bitnet_quantize_act(to_dev(x, torch.bfloat16))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(bf16_bits(s), s_ref)


def test_quantize_ties_and_edge_rows():
    K = 256
    rows = []
    # exact ties: absmax 127 * 2^e makes the scale exactly 2^e
    for e in (-3, 0, 2):
        r = np.zeros(K, np.float32)
        r[0] = 127 * 2.0 ** e
        r[1:129] = (np.arange(128) - 64 + 0.5) * 2.0 ** e   # (j + 0.5) * s
        rows.append(r)
    rows.append(np.zeros(K, np.float32))                    # all-zero row
    r = np.zeros(K, np.float32); r[7] = 1e-6; rows.append(r)  # absmax < eps
    r = np.full(K, -3.0, np.float32); rows.append(r)         # constant negative
    # near-ties: values within a few ulp of (j + 0.5) * s for an inexact s
    rng = np.random.default_rng(0)
    r = rng.standard_normal(K).astype(np.float32)
    r[0] = 10.0
    s = np.float32(10.0) / np.float32(127.0)
    j = rng.integers(-126, 126, K // 2)
    r[1:K // 2 + 1] = ((j + 0.5) * s).astype(np.float32)
    rows.append(r)
    x = f32_to_bf16_bits(np.stack(rows))
    q_ref, s_ref = oracle.quantize(x)
    q, sc = bn.bitnet_quantize_act(to_dev(x, torch.bfloat16))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(bf16_bits(sc), s_ref)


def test_quantize_rejects_bad_shape():
    with pytest.raises(bn.BitnetValueError):
        bn.bitnet_quantize_act(torch.zeros((2, 48), dtype=torch.bfloat16, device="cuda"))


# ------------------------------------------------------------ fused GEMV

GEMV_CASES = [(1, 512, 512), (4, 512, 512), (1, 2560, 640), (2, 96, 40), (3, 160, 33),
              (15, 4096, 300), (8, 11008, 130), (1, 2560, 128256 // 16), (5, 6912, 2560),
              (1, 32, 1), (9, 1024, 4099), (12, 2112, 77), (10, 64, 5), (14, 8256, 260)]


@pytest.mark.parametrize("M,K,N", GEMV_CASES)
def test_gemv_fused_debug_bitexact(M, K, N):
    x = acts(92, K, M, K)
    w = weights(92, N, N, K)
    p = oracle.pack(w)
    q_ref, s_ref = oracle.quantize(x)
    acc_ref = oracle.acc(q_ref, p)
    acc, q, s = bn.bitnet_gemv_fused_debug(to_dev(x, torch.bfloat16), to_dev(p))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(bf16_bits(s), s_ref)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)


@pytest.mark.parametrize("M,K,N", GEMV_CASES)
@pytest.mark.parametrize("per_row_scale", [False, True])
def test_gemv_fused_matches_oracle(M, K, N, per_row_scale):
    x = acts(93, K, M, K)
    w = weights(93, N, N, K)
    p = oracle.pack(w)
    sw = (synth.uniform_f32(synth.key(93, N, 3), N, 0.01, 0.1) if per_row_scale
          else sw_of(93, N))
    ref = oracle.linear(x, p, sw)
    got = bn.bitnet_gemv_fused(to_dev(x, torch.bfloat16), to_dev(p), to_dev(sw))
    assert_bf16_close(bf16_bits(got), ref)


def test_gemv_fused_rejects_m16_and_big_mk():
    x = torch.zeros((16, 512), dtype=torch.bfloat16, device="cuda")
    p = torch.zeros((8, 128), dtype=torch.uint8, device="cuda")
    with pytest.raises(bn.BitnetValueError):
        bn.bitnet_gemv_fused(x, p, 1.0)
    x = torch.zeros((15, 16384), dtype=torch.bfloat16, device="cuda")
    p = torch.zeros((8, 4096), dtype=torch.uint8, device="cuda")
    with pytest.raises(bn.BitnetValueError):
        bn.bitnet_gemv_fused(x, p, 1.0)


# ------------------------------------------------------------------ GEMM

GEMM_CASES = [(4, 512, 512), (1, 128, 256), (130, 384, 300), (128, 4096, 256),
              (257, 2560, 520), (64, 11008, 384), (300, 256, 1000), (37, 96, 77),
              (200, 160, 64), (16, 6912, 2560)]


@pytest.mark.parametrize("M,K,N", GEMM_CASES)
def test_gemm_acc_bitexact(M, K, N):
    rng = np.random.default_rng(M * 7 + K + N)
    q = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    w = weights(94, N, N, K)
    p = oracle.pack(w)
    acc = bn.bitnet_gemm_acc_i32(to_dev(q), to_dev(p))
    assert np.array_equal(acc.cpu().numpy(), oracle.acc(q, p))


@pytest.mark.parametrize("M,K,N", GEMM_CASES)
def test_gemm_matches_oracle(M, K, N):
    x = acts(95, K, M, K, outliers=False)
    q, sa = oracle.quantize(x)
    w = weights(95, N, N, K)
    p = oracle.pack(w)
    sw = synth.uniform_f32(synth.key(95, N, 3), N, 0.01, 0.1)
    ref = oracle.gemm(q, p, sa, sw)
    got = bn.bitnet_gemm(to_dev(q), to_dev(p), to_dev(sa, torch.bfloat16), to_dev(sw))
    assert_bf16_close(bf16_bits(got), ref)


# M <= 128 takes the few-row kernel (512-wide K stages; the K loop split over
# a cluster of up to 8 CTAs where the tiles do not fill the GPU), 128 < M <=
# 256 the split-K kernel's 256-row tile: ragged last K stages, ragged N,
# every activation-row width (16 ... 256) and a few splits.
SK_CASES = [(33, 4096, 128), (2, 192, 130), (17, 640, 1000), (64, 8256, 200),
            (256, 1024, 4096), (100, 2560, 131), (1, 11008, 4099), (129, 64, 256),
            (16, 4096, 11008)]


@pytest.mark.parametrize("M,K,N", SK_CASES)
def test_gemm_split_k_bitexact_and_oracle(M, K, N):
    rng = np.random.default_rng(M * 31 + K + N)
    q = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    w = weights(99, N, N, K)
    p = oracle.pack(w)
    pd = to_dev(p)
    acc = bn.bitnet_gemm_acc_i32(to_dev(q), pd)
    assert np.array_equal(acc.cpu().numpy(), oracle.acc(q, p))
    sa = f32_to_bf16_bits(rng.uniform(0.001, 0.05, size=M).astype(np.float32))
    sw = synth.uniform_f32(synth.key(99, N, 3), N, 0.01, 0.1)
    got = bn.bitnet_gemm(to_dev(q), pd, to_dev(sa, torch.bfloat16), to_dev(sw))
    assert_bf16_close(bf16_bits(got), oracle.gemm(q, p, sa, sw))


def test_gemm_extreme_accumulators():
    # |acc| = 127 * K at the largest K of the workloads
    K, M, N = 11008, 3, 256
    q = np.full((M, K), 127, np.int8)
    q[1] = -127
    w = np.ones((N, K), np.int8)
    w[1::2] = -1
    p = oracle.pack(w)
    acc = bn.bitnet_gemm_acc_i32(to_dev(q), to_dev(p)).cpu().numpy()
    assert np.array_equal(acc, oracle.acc(q, p))


@pytest.mark.parametrize("M,N", [(150, 9600), (192, 11008)])
def test_gemm_one_wave_rows_bitexact(M, N):
    # 129..192 rows with at least 74 weight tiles take the persistent kernel
    # (one 192-row tile per weight tile); its int32 sums and bf16 outputs,
    # natural order (bitnet_gemm) and permuted (bitnet_linear), match the
    # oracle exactly
    K = 1024
    x = acts(131, M, M, K)
    w = weights(131, M, N, K)
    p = oracle.pack(w)
    q, sa = oracle.quantize(x)
    acc = bn.bitnet_gemm_acc_i32(to_dev(q), to_dev(p)).cpu().numpy()
    assert np.array_equal(acc, oracle.acc(q, p))
    sw = sw_of(131, M)
    got = bn.bitnet_linear(to_dev(x, torch.bfloat16), to_dev(p), to_dev(sw))
    assert_bf16_close(bf16_bits(got), oracle.linear(x, p, sw))


@pytest.mark.parametrize("M", [2, 130])
@pytest.mark.parametrize("K", [131008, 131072])
def test_gemm_scaled_weight_limit(M, K):
    # The natural-order few-row and split-K kernels sum 64 * w in int32. At
    # their largest K, x = -128 against code 0 (w = -2) gives 64 * 256 * K just
    # below 2^31; one step beyond, the call takes the persistent kernel. Both
    # are exact.
    N = 128 if M <= 2 else 64
    q = np.full((M, K), -128, np.int8)
    q[1] = 127
    p = np.random.default_rng(K).integers(0, 256, (N, K // 4), dtype=np.uint8)
    p[0] = 0x00  # code 0 everywhere: w = -2
    p[1] = 0xFF  # code 3 everywhere: w = +1
    acc = bn.bitnet_gemm_acc_i32(to_dev(q), to_dev(p)).cpu().numpy()
    assert np.array_equal(acc, oracle.acc(q, p))
    assert acc[0, 0] == 256 * K and acc[1, 1] == 127 * K


def test_gemm_empty_and_sentinel():
    # M = 0 is a no-op; outputs outside [M, N] are never written
    p = torch.zeros((64, 128), dtype=torch.uint8, device="cuda")
    q = torch.zeros((0, 512), dtype=torch.int8, device="cuda")
    sa = torch.zeros((0,), dtype=torch.bfloat16, device="cuda")
    out = bn.bitnet_gemm(q, p, sa, 1.0)
    assert out.shape == (0, 64)
    M, K, N = 5, 256, 40
    buf = torch.full((M * N + 64,), 0x7F7F, dtype=torch.int16, device="cuda")
    out = buf[:M * N].view(torch.bfloat16).view(M, N)
    x = acts(96, 0, M, K)
    q, sa = oracle.quantize(x)
    w = weights(96, 0, N, K)
    pk = oracle.pack(w)
    bn.bitnet_gemm(to_dev(q), to_dev(pk), to_dev(sa, torch.bfloat16), 0.05, out=out)
    assert torch.all(buf[M * N:] == 0x7F7F)
    assert_bf16_close(bf16_bits(out), oracle.gemm(q, pk, sa, np.array([0.05], np.float32)))


# ---------------------------------------------------------------- linear

@pytest.mark.parametrize("M", [1, 4, 15, 16, 17, 129])
def test_linear_dispatch_matches_oracle(M):
    K, N = 1024, 384
    x = acts(97, M, M, K)
    w = weights(97, M, N, K)
    p = oracle.pack(w)
    sw = sw_of(97, M)
    got = bn.bitnet_linear(to_dev(x, torch.bfloat16), to_dev(p), to_dev(sw))
    assert_bf16_close(bf16_bits(got), oracle.linear(x, p, sw))


def test_gemv_and_gemm_paths_agree_tiny_config():
    """Tiny workload through both the fused GEMV and the GEMM (bit-exact)."""
    M, K, N = W.TINY["M"], W.TINY["K"], W.TINY["N"]
    x = acts(W.W_TINY, 0, M, K)
    w = weights(W.W_TINY, 0, N, K)
    sw = sw_of(W.W_TINY, 0)
    p = bn.bitnet_pack_weights(to_dev(w))
    xd = to_dev(x, torch.bfloat16)
    y1 = bn.bitnet_gemv_fused(xd, p, to_dev(sw))
    q, sa = bn.bitnet_quantize_act(xd)
    y2 = bn.bitnet_gemm(q, p, sa, to_dev(sw))
    ref = oracle.linear(x, oracle.pack(w), sw)
    assert np.array_equal(bf16_bits(y1), bf16_bits(y2))
    assert_bf16_close(bf16_bits(y1), ref)


def test_linear_workspace_errors():
    x = torch.zeros((32, 512), dtype=torch.bfloat16, device="cuda")
    p = torch.zeros((64, 128), dtype=torch.uint8, device="cuda")
    sw = torch.ones(1, dtype=torch.float32, device="cuda")
    out = torch.empty((32, 64), dtype=torch.bfloat16, device="cuda")
    L = bn.lib()
    import ctypes
    st = L.bitnet_linear(ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(x.data_ptr()), 0,
                         ctypes.c_void_p(p.data_ptr()), ctypes.c_void_p(sw.data_ptr()), 1,
                         32, 64, 512, None, 0, None)
    assert st == bn.ERR_WORKSPACE


@pytest.mark.parametrize("M,K,N", [(130, 384, 300), (257, 2560, 520), (16, 11008, 256),
                                   (200, 160, 64), (129, 4096, 4099), (256, 2560, 640),
                                   (31, 6912, 2560), (64, 4160, 96)])
def test_linear_split_path_ragged(M, K, N):
    """M >= 16: quantise into the workspace, then the GEMM (tensor-core path
    with transposed groups and row sums when K % 64 == 0, SIMT otherwise)."""
    x = acts(98, M + K, M, K)
    w = weights(98, N + K, N, K)
    p = oracle.pack(w)
    sw = synth.uniform_f32(synth.key(98, N, 3), N, 0.01, 0.1)
    got = bn.bitnet_linear(to_dev(x, torch.bfloat16), to_dev(p), to_dev(sw))
    assert_bf16_close(bf16_bits(got), oracle.linear(x, p, sw))


# -------------------------------------------------------------- grouped GEMV

@pytest.mark.parametrize("M", [1, 2, 4, 15])
def test_gemv_fused_grouped_matches_oracle_and_single_calls(M):
    shapes = [(2560, 2560), (2560, 640), (6912, 300), (96, 40), (512, 1), (4096, 1000),
              (128, 77), (2112, 130), (8192, 64)]
    xs, wps, sws, host = [], [], [], []
    for i, (K, N) in enumerate(shapes):
        x = acts(99, 10 * M + i, M, K)
        w = weights(99, 10 * M + i, N, K)
        sw = synth.uniform_f32(synth.key(99, 10 * M + i, 3), N if i % 2 else 1, 0.01, 0.1)
        p = oracle.pack(w)
        host.append((x, p, sw))
        xs.append(to_dev(x, torch.bfloat16))
        wps.append(to_dev(p))
        sws.append(to_dev(sw))
    outs = bn.bitnet_gemv_fused_grouped(xs, wps, sws)
    for (x, p, sw), o, xd, wd, sd in zip(host, outs, xs, wps, sws):
        single = bn.bitnet_gemv_fused(xd, wd, sd)
        assert np.array_equal(bf16_bits(o), bf16_bits(single))
        assert_bf16_close(bf16_bits(o), oracle.linear(x, p, sw))


def test_gemv_fused_grouped_more_than_one_launch():
    # 300 problems: two launches of the grouped kernel
    xs, wps, sws, refs = [], [], [], []
    for i in range(300):
        K, N = (128, 16 + i % 50) if i % 3 else (256, 33)
        x = acts(100, i, 1, K)
        w = weights(100, i, N, K)
        p = oracle.pack(w)
        sw = sw_of(100, i)
        refs.append(oracle.linear(x, p, sw))
        xs.append(to_dev(x, torch.bfloat16))
        wps.append(to_dev(p))
        sws.append(to_dev(sw))
    outs = bn.bitnet_gemv_fused_grouped(xs, wps, sws)
    for o, r in zip(outs, refs):
        assert_bf16_close(bf16_bits(o), r)


# ---------------------------------------------------------- float32 input

F32_CASES = [(1, 512, 512), (4, 2560, 640), (15, 4096, 300), (9, 1024, 131), (3, 96, 40),
             (16, 1024, 384), (64, 2560, 520), (300, 4096, 256), (37, 160, 77)]


def acts_f32(layer, M, K):
    rng = np.random.default_rng(layer * 7919 + M * 31 + K)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, ::101] *= 20.0
    if M > 1:
        x[1, :6] = np.array([127.0, 0.5, 1.5, -2.5, 3.5, -0.5], np.float32)  # exact ties
    return x


@pytest.mark.parametrize("M,K,N", F32_CASES)
def test_float32_activations_match_oracle(M, K, N):
    """float32 activations (the dtype the bitnet-cpu page accepts besides
    bf16) through the quantiser, the fused GEMV and bitnet_linear."""
    x = acts_f32(M, M, K)
    w = weights(93, M + K, N, K)
    p = oracle.pack(w)
    sw = sw_of(93, M)
    xd = to_dev(x)
    q_ref, s_ref = oracle.quantize_f32(x)
    xq, sa = bn.bitnet_quantize_act(xd)
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(bf16_bits(sa), s_ref)
    ref = oracle.linear_f32(x, p, sw)
    pd = to_dev(p)
    assert_bf16_close(bf16_bits(bn.bitnet_linear(xd, pd, to_dev(sw))), ref)
    assert_bf16_close(bf16_bits(bn.bitnet_linear_noalloc(xd, pd, to_dev(sw))), ref)
    if M < 16:
        assert_bf16_close(bf16_bits(bn.bitnet_gemv_fused(xd, pd, to_dev(sw))), ref)


# --------------------------------------------------- absmean ternarisation

TERN_CASES = [(64, 320), (300, 4096), (4096, 2560), (7, 96), (1, 16)]


def dense_weights(N, K, seed):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[0, : min(K, 8)] = 0.0
    if N > 2:
        w[2] = 0.0                        # an all-zero row: gamma = eps
    if N > 4:
        # magnitudes whose |w| * 2^64 is truncated (2^-60 .. 2^-45) or far
        # below the rest of their group (the exact sum's general case)
        w[3, ::7] *= np.float32(2.0 ** -40)
        w[4, 1::5] *= np.float32(2.0 ** -110)
        w[4, ::9] *= np.float32(2.0 ** 30)
    return w


@pytest.mark.parametrize("per_row", [True, False])
@pytest.mark.parametrize("N,K", TERN_CASES)
def test_ternarize_absmean_bitexact(N, K, per_row):
    w = dense_weights(N, K, N * 17 + K)
    wt_ref, sc_ref = oracle.ternarize_absmean(w, per_row=per_row)
    wt, sc = bn.bitnet_ternarize_absmean(to_dev(w), per_row=per_row)
    assert np.array_equal(wt.cpu().numpy(), wt_ref)
    assert np.array_equal(sc.cpu().numpy(), sc_ref)


def test_ternarize_then_pack_and_linear_match_oracle():
    """The load-time chain the page's BitLinear.from_dense runs: ternarise,
    pack, then the layer, against the oracle's chain."""
    N, K, M = 384, 1024, 20
    w = dense_weights(N, K, 5)
    wt, sc = bn.bitnet_ternarize_absmean(to_dev(w))
    p = bn.bitnet_pack_weights(wt)
    x = acts(92, 0, M, K)
    wt_ref, sc_ref = oracle.ternarize_absmean(w)
    ref = oracle.linear(x, oracle.pack(wt_ref), sc_ref)
    assert_bf16_close(bf16_bits(bn.bitnet_linear(to_dev(x, torch.bfloat16), p, sc)), ref)


def test_ternarize_rejects_non_finite():
    w = torch.zeros((4, 64), dtype=torch.float32, device="cuda")
    w[1, 5] = float("nan")
    with pytest.raises(bn.BitnetValueError):
        bn.bitnet_ternarize_absmean(w)
    w[1, 5] = 2.0 ** 48
    with pytest.raises(bn.BitnetValueError):
        bn.bitnet_ternarize_absmean(w, per_row=False)


# ----------------------------------------------------------- fused bias

@pytest.mark.parametrize("M,K,N", [(1, 2560, 640), (3, 96, 40), (8, 4096, 300), (12, 2112, 77),
                                   (20, 1024, 384), (300, 4096, 256), (37, 160, 77),
                                   (2048, 2560, 1000)])
def test_linear_bias_matches_oracle(M, K, N):
    """The layer with its bf16 bias fused into every kernel's epilogue: the
    fused dp4a and tensor-core GEMVs, the split-K and persistent GEMMs and
    the SIMT path, against the oracle's y + bias."""
    x = acts(90, M + K, M, K)
    w = weights(90, N + K, N, K)
    p = oracle.pack(w)
    sw = synth.uniform_f32(synth.key(90, N, 3), N, 0.01, 0.1)
    bias = f32_to_bf16_bits(np.random.default_rng(M + N).standard_normal(N).astype(np.float32))
    bias[:2] = [0x0000, 0x8000]
    got = bn.bitnet_linear(to_dev(x, torch.bfloat16), to_dev(p), to_dev(sw),
                           bias=to_dev(bias, torch.bfloat16))
    rows = np.arange(M) if M <= 64 else np.unique(np.r_[np.random.default_rng(M).choice(M, 40, replace=False), 0, M - 1])
    ref = oracle.linear_bias(x[rows], p, sw, bias)
    assert_bf16_close(bf16_bits(got)[rows], ref)
    # without the bias the result is bitnet_linear's
    plain = bn.bitnet_linear(to_dev(x, torch.bfloat16), to_dev(p), to_dev(sw))
    assert_bf16_close(bf16_bits(plain)[rows], oracle.linear(x[rows], p, sw))


# ------------------------------------------------------ RMSNorm -> quantise

RMS_CASES = [(1, 64), (2, 96), (7, 2560), (64, 4096), (300, 2560), (3, 8192), (5, 11008),
             (2, 16384), (2, 16416), (1, 27648)]


def norm_weight(K, seed):
    """bf16 norm weights around 1 with a zero, a negative and a 2 in front."""
    g = (1.0 + 0.25 * np.random.default_rng(seed).standard_normal(K)).astype(np.float32)
    g[:3] = [0.0, -1.0, 2.0]
    return f32_to_bf16_bits(g)


def norm_inputs(M, K, seed):
    """Activations with a zero row (r = 1/sqrt(eps)), a row scaled by 2^12
    (large squares), a row scaled by 2^-70 (squares below 2^-64), and rows
    mixing magnitudes far apart (the exact sum's general case)."""
    x = acts(95, seed, M, K)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    if M > 2:
        x[2] = 0
    if M > 3:
        x[3] = f32_to_bf16_bits(xf[3] * np.float32(2.0 ** 12))
    if M > 4:
        x[4] = f32_to_bf16_bits(xf[4] * np.float32(2.0 ** -70))
    if M > 5:  # squares in [2^-64, 2^-50): truncated at 2^-64
        x[5, ::3] = f32_to_bf16_bits(xf[5, ::3] * np.float32(2.0 ** -28))
    if M > 6:  # exponents spread over more than 21 binades
        x[6, ::5] = f32_to_bf16_bits(xf[6, ::5] * np.float32(2.0 ** -24))
        x[6, 1::7] = f32_to_bf16_bits(xf[6, 1::7] * np.float32(2.0 ** 16))
    return x


@pytest.mark.parametrize("eps", [1e-5, 1e-6])
@pytest.mark.parametrize("M,K", RMS_CASES)
def test_rmsnorm_quantize_bitexact(M, K, eps):
    x = norm_inputs(M, K, M + K)
    g = norm_weight(K, M * 3 + K)
    q_ref, s_ref = oracle.rmsnorm_quantize(x, g, eps)
    q, s = bn.bitnet_rmsnorm_quantize_act(to_dev(x, torch.bfloat16), to_dev(g, torch.bfloat16),
                                          eps)
    bn.bitnet_device_status()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(bf16_bits(s), s_ref)


@pytest.mark.parametrize("M,K,N", [(1, 2560, 640), (2, 96, 40), (2, 16384, 130), (1, 11008, 300),
                                   (3, 4096, 200), (12, 2112, 77), (64, 4096, 300),
                                   (16, 11008, 256), (300, 2560, 520), (2048, 2560, 256)])
def test_linear_rmsnorm_matches_oracle(M, K, N):
    """Norm, quantiser and the layer in one call: the norm inside the fused
    GEMV's staging (M <= 2), the norm kernel in front of the fused GEMV
    (3 <= M < 16), the tensor-core GEMMs (permuted workspace plus code sums)
    and the SIMT path (K % 64 != 0)."""
    x = norm_inputs(M, K, M * 5 + K)
    g = norm_weight(K, N + K)
    w = weights(96, N + K, N, K)
    p = oracle.pack(w)
    sw = synth.uniform_f32(synth.key(96, N, 3), N, 0.01, 0.1)
    got = bn.bitnet_linear_rmsnorm(to_dev(x, torch.bfloat16), to_dev(g, torch.bfloat16), 1e-6,
                                   to_dev(p), to_dev(sw))
    bn.bitnet_device_status()
    rows = np.arange(M) if M <= 64 else np.unique(np.r_[np.random.default_rng(M).choice(M, 40, replace=False), 0, 2, 3, 4, M - 1])
    ref = oracle.linear_rmsnorm(x[rows], g, 1e-6, p, sw)
    assert_bf16_close(bf16_bits(got)[rows], ref)


def test_rmsnorm_flags_out_of_range_input():
    """|x| >= 2^23 (whose square the exact sum does not take) and NaN are
    reported by bitnet_device_status; the flag is cleared after it is read."""
    K = 256
    g = to_dev(norm_weight(K, 1), torch.bfloat16)
    for bad in (2.0 ** 24, float("nan")):
        x = torch.ones((3, K), dtype=torch.bfloat16, device="cuda")
        x[1, 7] = bad
        bn.bitnet_rmsnorm_quantize_act(x, g, 1e-5)
        with pytest.raises(bn.BitnetValueError):
            bn.bitnet_device_status()
        bn.bitnet_device_status()
    # the same check inside the fused GEMV's staging (one row)
    w = to_dev(oracle.pack(weights(97, 1, 64, K)))
    xb = torch.ones((1, K), dtype=torch.bfloat16, device="cuda")
    xb[0, 3] = 2.0 ** 24
    bn.bitnet_linear_rmsnorm(xb, g, 1e-5, w, torch.tensor([0.05], device="cuda"))
    with pytest.raises(bn.BitnetValueError):
        bn.bitnet_device_status()
    bn.bitnet_device_status()
    with pytest.raises(bn.BitnetValueError):
        bn.bitnet_rmsnorm_quantize_act(x, g, 0.0)
    with pytest.raises(ValueError):
        bn.bitnet_rmsnorm_quantize_act(x, g[:128], 1e-5)


@pytest.mark.parametrize("M", [1, 2, 4, 8])
def test_gemv_grouped_wide_rows(M):
    """Grouped problems with ragged N, K from 128 to 7680 (units of one or two
    rows per warp), per-row and per-tensor weight scales, against the oracle
    and the single-problem kernel."""
    shapes = [(2560, 2560), (2560, 640), (6912, 300), (128, 77), (4096, 1000), (256, 1),
              (7680, 130), (1152, 200)]
    xs, wps, sws, host = [], [], [], []
    for i, (K, N) in enumerate(shapes):
        x = acts(101, 10 * M + i, M, K)
        w = weights(101, 10 * M + i, N, K)
        sw = synth.uniform_f32(synth.key(101, 10 * M + i, 3), N if i % 2 else 1, 0.01, 0.1)
        p = oracle.pack(w)
        host.append((x, p, sw))
        xs.append(to_dev(x, torch.bfloat16))
        wps.append(to_dev(p))
        sws.append(to_dev(sw))
    outs = bn.bitnet_gemv_fused_grouped(xs, wps, sws)
    bn.bitnet_device_status()
    for (x, p, sw), o, xd, wd, sd in zip(host, outs, xs, wps, sws):
        assert_bf16_close(bf16_bits(o), oracle.linear(x, p, sw))
        assert np.array_equal(bf16_bits(o), bf16_bits(bn.bitnet_gemv_fused(xd, wd, sd)))


# ------------------------------------------- accumulators of every product path
#
# bitnet_linear_acc_i32 and bitnet_gemv_fused_grouped_acc_i32 run the
# product's own dispatch and kernels with the epilogue replaced by an int32
# store (and the quantised codes and scales written out), so the exact sums
# of every kernel the product runs are compared with the oracle bit for bit.

# (M, K, N, the kernel instantiation the product reaches)
LINEAR_PATHS = [
    (1, 2560, 640, "gemv_kernel MB=1 (register-cached staging)"),
    (1, 4096, 32768, "gemv_grouped_kernel, one-problem launch (32 MB layer)"),
    (2, 2560, 52432, "gemv_grouped_kernel MB=2, one-problem launch, ragged units"),
    (2, 4096, 300, "gemv_kernel MB=2"),
    (1, 96, 40, "gemv_kernel MB=1, K % 64 != 0 (8-byte copies)"),
    (3, 160, 33, "gemv_kernel MB=4, K % 64 != 0"),
    (7, 4096, 130, "gemv_kernel MB=8"),
    (4, 27648, 64, "gemv_kernel MB=4, K past the cached staging"),
    (8, 4096, 300, "gemv_i8_skq_kernel, M = 8"),
    (12, 2112, 77, "gemv_i8_skq_kernel, ragged N"),
    (15, 11008, 130, "gemv_i8_skq_kernel, M = 15"),
    (9, 1024, 4099, "gemv_i8_skq_kernel, N % 4 != 0"),
    (16, 4096, 256, "gemm_i8_fr_kernel<16, perm>"),
    (33, 4096, 130, "gemm_i8_fr_kernel<64, perm>, ragged N"),
    (100, 2560, 131, "gemm_i8_fr_kernel<128, perm>, ragged last K stage"),
    (64, 11008, 4096, "gemm_i8_fr_kernel<64, perm>, one CTA per tile"),
    (20, 64, 300, "gemm_i8_fr_kernel<32, perm>, K below one stage"),
    (256, 1024, 4096, "gemm_i8_sk_kernel<256, perm>"),
    (129, 64, 256, "gemm_i8_sk_kernel<256, perm>, one K block of 64"),
    (257, 2560, 520, "gemm_i8_ts_kernel<perm>, ragged M and N tiles"),
    (300, 4096, 1000, "gemm_i8_ts_kernel<perm>"),
    (37, 160, 77, "SIMT path (gemv_kernel on pre-quantised rows), K % 64 != 0"),
    (200, 96, 64, "SIMT path, many row chunks"),
]


@pytest.mark.parametrize("M,K,N,path", LINEAR_PATHS)
def test_linear_accumulators_every_path(M, K, N, path):
    x = acts(102, M + K, M, K)
    w = weights(102, N + K, N, K)
    p = oracle.pack(w)
    sw = synth.uniform_f32(synth.key(102, N, 3), N, 0.01, 0.1)
    xd, pd = to_dev(x, torch.bfloat16), to_dev(p)
    acc, xq, sa, _ = bn.bitnet_linear_acc_i32(xd, pd)
    q_ref, s_ref = oracle.quantize(x)
    assert np.array_equal(xq.cpu().numpy(), q_ref), path
    assert np.array_equal(bf16_bits(sa), s_ref), path
    acc_ref = oracle.acc(q_ref, p)
    assert np.array_equal(acc.cpu().numpy(), acc_ref), path
    y = bn.bitnet_linear(xd, pd, to_dev(sw))
    assert_bf16_close(bf16_bits(y), oracle.epilogue(acc_ref, s_ref, sw))


@pytest.mark.parametrize("M,K,N", [(1, 512, 512), (9, 1024, 131), (64, 2560, 520),
                                   (300, 4096, 256), (37, 160, 77)])
def test_linear_accumulators_float32(M, K, N):
    """float32 rows through the same hooks (the fp32 quantisers)."""
    xf = acts_f32(M + 7, M, K)
    w = weights(103, N + K, N, K)
    p = oracle.pack(w)
    acc, xq, sa, _ = bn.bitnet_linear_acc_i32(to_dev(xf), to_dev(p))
    q_ref, s_ref = oracle.quantize_f32(xf)
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(bf16_bits(sa), s_ref)
    assert np.array_equal(acc.cpu().numpy(), oracle.acc(q_ref, p))


@pytest.mark.parametrize("M", [1, 2, 4, 8, 15])
def test_grouped_accumulators(M):
    """The grouped kernel's exact sums, codes and scales for every problem of
    a group, including problems that take their own launch (K % 64 != 0)."""
    shapes = [(2560, 2560), (2560, 640), (6912, 300), (128, 77), (4096, 1000), (256, 1),
              (7680, 130), (96, 40), (1152, 200)]
    xs, wps, host = [], [], []
    for i, (K, N) in enumerate(shapes):
        x = acts(104, 10 * M + i, M, K)
        w = weights(104, 10 * M + i, N, K)
        p = oracle.pack(w)
        host.append((x, p))
        xs.append(to_dev(x, torch.bfloat16))
        wps.append(to_dev(p))
    res = bn.bitnet_gemv_fused_grouped_acc_i32(xs, wps)
    bn.bitnet_device_status()
    for i, ((x, p), (acc, xq, sa)) in enumerate(zip(host, res)):
        q_ref, s_ref = oracle.quantize(x)
        assert np.array_equal(xq.cpu().numpy(), q_ref), f"problem {i}"
        assert np.array_equal(bf16_bits(sa), s_ref), f"problem {i}"
        assert np.array_equal(acc.cpu().numpy(), oracle.acc(q_ref, p)), f"problem {i}"


# ----------------------------------------------------------------- guard bands

POISON = 0x7F7F


def poisoned(rows, cols, pad=256):
    """A bf16 [rows, cols] view inside a buffer of 0x7F7F words, `pad` words
    of which lie on each side of it."""
    buf = torch.full((rows * cols + 2 * pad,), POISON, dtype=torch.int16, device="cuda")
    return buf, buf[pad:pad + rows * cols].view(torch.bfloat16).view(rows, cols), pad


def assert_fences(buf, n, pad):
    b = buf.cpu().numpy().view(np.uint16)
    assert np.all(b[:pad] == POISON), "written before the output"
    assert np.all(b[pad + n:] == POISON), "written past the output"


@pytest.mark.parametrize("M,K,N,path", [
    (3, 512, 33, "gemv_kernel"), (12, 2112, 77, "gemv_i8_skq_kernel"),
    (100, 2560, 131, "gemm_i8_sk_kernel"), (300, 4096, 1000, "gemm_i8_ts_kernel"),
    (37, 160, 77, "SIMT path")])
def test_guard_bands_linear(M, K, N, path):
    """Outputs of ragged tiles stay inside [M, N]: the words around the
    output keep their poison."""
    x = acts(105, M + K, M, K)
    w = weights(105, N + K, N, K)
    p = oracle.pack(w)
    sw = sw_of(105, N)
    buf, out, pad = poisoned(M, N)
    bn.bitnet_linear(to_dev(x, torch.bfloat16), to_dev(p), to_dev(sw), out=out)
    torch.cuda.synchronize()
    assert_fences(buf, M * N, pad)
    assert_bf16_close(bf16_bits(out), oracle.linear(x, p, sw))


@pytest.mark.parametrize("M", [1, 4, 15])
def test_guard_bands_grouped(M):
    """Problems of a group written back to back with poison between them:
    the ragged last unit of each problem stays inside its own output."""
    shapes = [(2560, 33), (4096, 1000), (128, 77), (6912, 300), (256, 1), (2560, 641)]
    pad = 64
    total = sum(M * N + pad + 8 for _, N in shapes) + pad
    buf = torch.full((total,), POISON, dtype=torch.int16, device="cuda")
    xs, wps, sws, outs, host, spans = [], [], [], [], [], []
    off = pad
    for i, (K, N) in enumerate(shapes):
        x = acts(106, 10 * M + i, M, K)
        w = weights(106, 10 * M + i, N, K)
        p = oracle.pack(w)
        sw = sw_of(106, i)
        host.append((x, p, sw))
        xs.append(to_dev(x, torch.bfloat16))
        wps.append(to_dev(p))
        sws.append(to_dev(sw))
        # 16-byte aligned starts: the offset in words is a multiple of 8
        off = (off + 7) // 8 * 8
        outs.append(buf[off:off + M * N].view(torch.bfloat16).view(M, N))
        spans.append((off, off + M * N))
        off += M * N + pad
    bn.bitnet_gemv_fused_grouped(xs, wps, sws, outs)
    torch.cuda.synchronize()
    b = buf.cpu().numpy().view(np.uint16)
    mask = np.ones(b.shape, bool)
    for a, e in spans:
        mask[a:e] = False
    assert np.all(b[mask] == POISON), "a problem wrote outside its output"
    for (x, p, sw), o in zip(host, outs):
        assert_bf16_close(bf16_bits(o), oracle.linear(x, p, sw))


def test_wrong_output_buffers_are_refused_before_launch():
    """A caller's `out` of the wrong shape, dtype or device is refused by the
    binding before anything is launched: the buffer keeps its contents."""
    M, K, N = 20, 512, 256
    x = to_dev(acts(107, 0, M, K), torch.bfloat16)
    p = to_dev(oracle.pack(weights(107, 0, N, K)))
    bad = [torch.full((M, N - 8), 7.0, dtype=torch.bfloat16, device="cuda"),
           torch.full((M, N), 7.0, dtype=torch.float32, device="cuda"),
           torch.full((M, N), 7.0, dtype=torch.bfloat16)]
    for out in bad:
        for fn in (lambda o: bn.bitnet_linear(x, p, 0.05, out=o),
                   lambda o: bn.bitnet_linear_noalloc(x, p, 0.05, out=o),
                   lambda o: bn.bitnet_gemv_fused(x[:4], p, 0.05, out=o[:4])):
            with pytest.raises((ValueError, TypeError)):
                fn(out)
        torch.cuda.synchronize()
        assert torch.all(out == 7.0)
    q, sa = bn.bitnet_quantize_act(x)
    with pytest.raises(ValueError):
        bn.bitnet_gemm(q, p, sa, 0.05, out=torch.empty((M + 1, N), dtype=torch.bfloat16,
                                                        device="cuda"))
    with pytest.raises(ValueError):
        bn.bitnet_gemv_fused_grouped([x[:1]], [p], [0.05],
                                     [torch.empty((1, N + 1), dtype=torch.bfloat16,
                                                  device="cuda")])
