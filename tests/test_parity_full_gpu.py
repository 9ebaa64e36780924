"""Parity at the workloads' full sizes, in the launch configuration the bench
times. Outputs the oracle can afford are compared in full; at prefill sizes
a seeded sample of rows (quantisation and the contraction are row-local, so
the oracle computes those rows alone) plus the last, ragged row."""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads as W
import bit_gemm_bitnet_b200 as bn
from helpers import bf16_bits, bf16_ulp_diff, f32_to_bf16_bits, to_dev

pytestmark = pytest.mark.gpu
THREADS = max(1, min(32, os.cpu_count() or 1))


@pytest.fixture(autouse=True)
def _gpu(cuda_ok):
    yield
    bn.bitnet_device_status()


def close(got, ref):
    """Exact bf16 equality with the oracle (the stated contract is 1 ulp;
    every stage is a function of its inputs, so the outputs must agree)."""
    d = bf16_ulp_diff(got, ref)
    assert d.max() <= 1, f"max ulp {d.max()}"
    assert np.array_equal(got, ref), f"{int((d > 0).sum())} outputs differ by one ulp"


def test_decode_sweep_graph_matches_oracle():
    """Two layers of the 2B decode sweep plus the LM head, issued as the
    bench issues them (C-ABI calls captured in one CUDA graph)."""
    names = [n for n, _, _ in W.DECODE_2B_LAYER]
    calls = [(layer, names.index(n), K, N) for layer in (0, 29) for n, K, N in W.DECODE_2B_LAYER]
    calls.append((30, len(names), W.DECODE_2B_LM_HEAD[1], W.DECODE_2B_LM_HEAD[2]))
    host, dev = [], []
    for layer, v, K, N in calls:
        w = synth.ternary(synth.key(W.W_DECODE_2B, layer, synth.T_WEIGHT, v), N, K)
        sw = synth.scale_wt(synth.key(W.W_DECODE_2B, layer, synth.T_SCALE_WT, v))
        x = synth.act_bf16(synth.key(W.W_DECODE_2B, layer, synth.T_ACT, v), 1, K)
        p = oracle.pack(w)
        host.append((x, p, sw))
        dev.append((to_dev(x, torch.bfloat16), bn.bitnet_pack_weights(to_dev(w)), to_dev(sw),
                    torch.empty((1, N), dtype=torch.bfloat16, device="cuda")))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for x, p, sw, o in dev:
                bn.bitnet_gemv_fused(x, p, sw, out=o)
        for o in (d[3] for d in dev):
            o.fill_(0)
        g.replay()
        g.replay()
    torch.cuda.synchronize()
    for (x, p, sw), d in zip(host, dev):
        close(bf16_bits(d[3]), oracle.linear_cols_threads(x, p, sw, THREADS))


@pytest.mark.parametrize("M", W.LLAMA_GEMV_M)
@pytest.mark.parametrize("shape", W.LLAMA_GEMV_SHAPES)
def test_llama_gemv_full(M, shape):
    name, K, N = shape
    v = [s[0] for s in W.LLAMA_GEMV_SHAPES].index(name)
    w = synth.ternary(synth.key(W.W_LLAMA_GEMV, M, synth.T_WEIGHT, v), N, K)
    x = synth.act_bf16(synth.key(W.W_LLAMA_GEMV, M, synth.T_ACT, v), M, K)
    sw = synth.scale_wt(synth.key(W.W_LLAMA_GEMV, M, synth.T_SCALE_WT, v))
    p = oracle.pack(w)
    xd, pd = to_dev(x, torch.bfloat16), bn.bitnet_pack_weights(to_dev(w))
    got = bn.bitnet_gemv_fused(xd, pd, to_dev(sw))
    # the same dispatch with int32 sums: gemv_kernel for M < 8, the
    # tensor-core gemv_i8_skq_kernel for M = 8 and 15
    acc, xq, sa, _ = bn.bitnet_linear_acc_i32(xd, pd)
    q_ref, s_ref = oracle.quantize(x)
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(bf16_bits(sa), s_ref)
    acc_ref = oracle.acc_threads(q_ref, p, THREADS)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    close(bf16_bits(got), oracle.epilogue(acc_ref, s_ref, sw))


@pytest.mark.parametrize("M", W.MIDBATCH_M)
@pytest.mark.parametrize("KN", W.MIDBATCH_SHAPES)
def test_midbatch_gemm(M, KN):
    K, N = KN
    x = synth.act_bf16(synth.key(W.W_MIDBATCH, M, synth.T_ACT, N), M, K, outliers=False)
    q, sa = oracle.quantize(x)
    w = synth.ternary(synth.key(W.W_MIDBATCH, M, synth.T_WEIGHT, N), N, K)
    sw = synth.scale_wt(synth.key(W.W_MIDBATCH, M, synth.T_SCALE_WT, N))
    p = oracle.pack(w)
    pd = bn.bitnet_pack_weights(to_dev(w))
    got = bn.bitnet_gemm(to_dev(q), pd, to_dev(sa, torch.bfloat16), to_dev(sw))
    # every row: gemm_i8_sk_kernel's int32 sums (its accumulator-hook
    # instantiation) and bf16 outputs
    acc_ref = oracle.acc_threads(q, p, THREADS)
    acc = bn.bitnet_gemm_acc_i32(to_dev(q), pd).cpu().numpy()
    assert np.array_equal(acc, acc_ref)
    close(bf16_bits(got), oracle.epilogue(acc_ref, sa, sw))


@pytest.mark.parametrize("M", W.PREFILL_M)
@pytest.mark.parametrize("KN", W.PREFILL_SHAPES)
def test_prefill_linear(M, KN):
    """bitnet_linear at prefill sizes: the permuted-layout quantiser and
    gemm_i8_ts_kernel<perm>. Every row at M = 2048; at M = 8192 a seeded
    sample of 512 rows plus the first and last (quantisation and the
    contraction are row-local, so the oracle computes those rows alone).
    Codes, scales and int32 sums come from the accumulator hook (the same
    quantiser and GEMM kernel with an int32 store)."""
    K, N = KN
    x = synth.act_bf16(synth.key(W.W_PREFILL, M, synth.T_ACT, K), M, K)
    w = synth.ternary(synth.key(W.W_PREFILL, M, synth.T_WEIGHT, K), N, K)
    sw = synth.scale_wt(synth.key(W.W_PREFILL, M, synth.T_SCALE_WT, K))
    p = oracle.pack(w)
    xd = to_dev(x, torch.bfloat16)
    pd = bn.bitnet_pack_weights(to_dev(w))
    y = bf16_bits(bn.bitnet_linear(xd, pd, to_dev(sw)))
    acc, xq, sa, _ = bn.bitnet_linear_acc_i32(xd, pd)
    acc, xq, sa = acc.cpu().numpy(), xq.cpu().numpy(), bf16_bits(sa)
    if M <= 2048:
        rows = np.arange(M)
    else:
        rows = np.unique(np.r_[np.random.default_rng(M + K).choice(M, 512, replace=False), 0, M - 1])
    q_ref, s_ref = oracle.quantize(x[rows])
    assert np.array_equal(xq[rows], q_ref)
    assert np.array_equal(sa[rows], s_ref)
    acc_ref = oracle.acc_threads(q_ref, p, THREADS)
    assert np.array_equal(acc[rows], acc_ref)
    close(y[rows], oracle.epilogue(acc_ref, s_ref, sw))


def test_decode_sweep_grouped_graph_matches_oracle():
    """All 211 calls of the 2B decode sweep as one grouped call, captured in a
    CUDA graph as the bench does. Every problem is checked against the
    oracle: its bf16 outputs, and through the accumulator hook (the same
    partition and gemv_grouped_kernel with an int32 store) its int32 sums,
    codes and scale. The CTA ranges cut across problem boundaries, so every
    unit boundary of every problem is covered."""
    names = [n for n, _, _ in W.DECODE_2B_LAYER]
    calls = [(layer, names.index(n), K, N) for layer in range(W.DECODE_2B_LAYERS)
             for n, K, N in W.DECODE_2B_LAYER]
    calls.append((30, len(names), W.DECODE_2B_LM_HEAD[1], W.DECODE_2B_LM_HEAD[2]))
    xs, wps, sws, outs, host = [], [], [], [], []
    for i, (layer, v, K, N) in enumerate(calls):
        w = synth.ternary(synth.key(W.W_DECODE_2B, layer, synth.T_WEIGHT, v), N, K)
        sw = synth.scale_wt(synth.key(W.W_DECODE_2B, layer, synth.T_SCALE_WT, v))
        x = synth.act_bf16(synth.key(W.W_DECODE_2B, layer, synth.T_ACT, v), 1, K)
        xs.append(to_dev(x, torch.bfloat16))
        wps.append(bn.bitnet_pack_weights(to_dev(w)))
        sws.append(to_dev(sw))
        outs.append(torch.zeros((1, N), dtype=torch.bfloat16, device="cuda"))
        host.append((x, oracle.pack(w), sw))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        bn.bitnet_gemv_fused_grouped(xs, wps, sws, outs)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            bn.bitnet_gemv_fused_grouped(xs, wps, sws, outs)
        for o in outs:
            o.fill_(0)
        g.replay()
        res = bn.bitnet_gemv_fused_grouped_acc_i32(xs, wps)
    torch.cuda.synchronize()
    bn.bitnet_device_status()
    for i, ((x, p, sw), o, (acc, xq, sa)) in enumerate(zip(host, outs, res)):
        q_ref, s_ref = oracle.quantize(x)
        assert np.array_equal(xq.cpu().numpy(), q_ref), f"problem {i}"
        assert np.array_equal(bf16_bits(sa), s_ref), f"problem {i}"
        acc_ref = oracle.acc_threads(q_ref, p, THREADS)
        assert np.array_equal(acc.cpu().numpy(), acc_ref), f"problem {i}"
        close(bf16_bits(o), oracle.epilogue(acc_ref, s_ref, sw))


# ------------------------------------- the widened rows at the bench's sizes

def _ffn_weights(N=11008, K=4096):
    w = synth.ternary(synth.key(W.W_PREFILL, 1, synth.T_WEIGHT, N), N, K)
    return w, oracle.pack(w), bn.bitnet_pack_weights(to_dev(w))


def _sample(M, seed):
    return np.unique(np.r_[np.random.default_rng(seed).choice(M, 40, replace=False), 0, M - 1])


@pytest.mark.parametrize("per_row", [True, False])
def test_ternarize_bench_size(per_row):
    """11008 x 4096 float32 weights, as the bench ternarises them."""
    w = (np.random.default_rng(7).standard_normal((11008, 4096)) * 0.02).astype(np.float32)
    wt_ref, sc_ref = oracle.ternarize_absmean(w, per_row=per_row)
    wt, sc = bn.bitnet_ternarize_absmean(to_dev(w), per_row=per_row)
    assert np.array_equal(wt.cpu().numpy(), wt_ref)
    assert np.array_equal(sc.cpu().numpy(), sc_ref)


def test_float32_gemv_and_linear_bench_size():
    """float32 activations: the decode GEMV at M = 1 (every output) and
    bitnet_linear at M = 2048 (sampled rows), 4096 -> 11008."""
    w, p, pd = _ffn_weights()
    sw = np.array([0.05], np.float32)
    x1 = np.random.default_rng(11).standard_normal((1, 4096)).astype(np.float32)
    close(bf16_bits(bn.bitnet_gemv_fused(to_dev(x1), pd, to_dev(sw))), oracle.linear_f32(x1, p, sw))
    x = np.random.default_rng(12).standard_normal((2048, 4096)).astype(np.float32)
    y = bn.bitnet_linear(to_dev(x), pd, to_dev(sw))
    rows = _sample(2048, 12)
    close(bf16_bits(y)[rows], oracle.linear_f32(x[rows], p, sw))


def test_linear_bias_bench_size():
    w, p, pd = _ffn_weights()
    sw = synth.uniform_f32(synth.key(W.W_PREFILL, 2, 3), 11008, 0.01, 0.1)
    x = synth.act_bf16(synth.key(W.W_PREFILL, 2048, synth.T_ACT, 11008), 2048, 4096)
    bias = f32_to_bf16_bits((np.random.default_rng(13).standard_normal(11008) * 0.1).astype(np.float32))
    y = bn.bitnet_linear(to_dev(x, torch.bfloat16), pd, to_dev(sw), bias=to_dev(bias, torch.bfloat16))
    rows = _sample(2048, 13)
    close(bf16_bits(y)[rows], oracle.linear_bias(x[rows], p, sw, bias))


def test_rmsnorm_bench_size():
    """RMSNorm + quantiser over 2048 rows of 4096 (every code and scale), and
    bitnet_linear_rmsnorm at M = 2048 (sampled rows) and M = 1."""
    K = 4096
    x = synth.act_bf16(synth.key(W.W_PREFILL, 2048, synth.T_ACT, K), 2048, K)
    g = f32_to_bf16_bits((1.0 + 0.1 * np.random.default_rng(14).standard_normal(K)).astype(np.float32))
    xd, gd = to_dev(x, torch.bfloat16), to_dev(g, torch.bfloat16)
    q_ref, s_ref = oracle.rmsnorm_quantize(x, g, 1e-6)
    q, s = bn.bitnet_rmsnorm_quantize_act(xd, gd, 1e-6)
    bn.bitnet_device_status()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(bf16_bits(s), s_ref)
    w, p, pd = _ffn_weights()
    sw = np.array([0.05], np.float32)
    y = bn.bitnet_linear_rmsnorm(xd, gd, 1e-6, pd, to_dev(sw))
    rows = _sample(2048, 14)
    close(bf16_bits(y)[rows], oracle.linear_rmsnorm(x[rows], g, 1e-6, p, sw))
    y1 = bn.bitnet_linear_rmsnorm(xd[:1], gd, 1e-6, pd, to_dev(sw))
    close(bf16_bits(y1), oracle.linear_rmsnorm(x[:1], g, 1e-6, p, sw))
