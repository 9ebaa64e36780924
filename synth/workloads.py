"""Shapes of the BitNet b1.58 W1.58A8 workloads (K -> N, and M).

Taken from the bitnet-tc announcement's benchmark shapes: the
microsoft/bitnet-b1.58-2B-4T projections (decode) and the LLaMA-7B
projections, plus the mid-batch and prefill regimes it discusses.
Keys for the generator are (workload id, layer, tensor, variant).
"""

# 0: tiny correctness case, through both the fused GEMV and the GEMM
TINY = dict(M=4, K=512, N=512)

# 1: BitNet-b1.58-2B decode at M = 1: 30 layers x 7 BitLinears + LM head
DECODE_2B_LAYER = (
    ("q", 2560, 2560), ("k", 2560, 640), ("v", 2560, 640), ("o", 2560, 2560),
    ("gate", 2560, 6912), ("up", 2560, 6912), ("down", 6912, 2560),
)
DECODE_2B_LAYERS = 30
DECODE_2B_LM_HEAD = ("lm_head", 2560, 128256)

# 2: LLaMA-7B projections through the fused GEMV at small M
LLAMA_GEMV_M = (1, 4, 8, 15)
LLAMA_GEMV_SHAPES = (("attn", 4096, 4096), ("gate_up", 4096, 11008),
                     ("down", 11008, 4096))

# 3: mid-batch GEMM on pre-quantised activations (no outliers)
MIDBATCH_M = (32, 64, 128, 256)
MIDBATCH_SHAPES = ((4096, 4096), (4096, 11008))

# 4: prefill GEMM, activations quantised per token
PREFILL_M = (2048, 8192)
PREFILL_SHAPES = ((4096, 11008), (11008, 4096), (2560, 6912), (6912, 2560))

W_TINY, W_DECODE_2B, W_LLAMA_GEMV, W_MIDBATCH, W_PREFILL = range(5)


def decode_2b_sweep():
    """The 211 calls of one decode sweep, in order: (layer, name, K, N)."""
    calls = []
    for layer in range(DECODE_2B_LAYERS):
        for name, K, N in DECODE_2B_LAYER:
            calls.append((layer, name, K, N))
    name, K, N = DECODE_2B_LM_HEAD
    calls.append((DECODE_2B_LAYERS, name, K, N))
    return calls


def decode_2b_packed_bytes():
    return sum(N * K // 4 for _, _, K, N in decode_2b_sweep())
