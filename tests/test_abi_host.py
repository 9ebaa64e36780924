"""The C ABI library loads, exports what include/bitnet.h declares, and its
argument validation rejects bad calls before touching the GPU (no device
needed: every call here returns before any CUDA work)."""
import ctypes
import os
import re

import pytest

import bit_gemm_bitnet_b200 as bn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitnet.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bitnet_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = header_functions()
    for n in ("bitnet_pack_weights", "bitnet_quantize_act", "bitnet_gemm",
              "bitnet_gemv_fused", "bitnet_linear"):
        assert n in names
    assert set(names) == set(bn.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = bn.lib()
    for n in header_functions():
        assert hasattr(L, n), n


def test_status_strings():
    for s in range(9):
        assert bn.status_string(s).startswith("BITNET_")
    assert "UNKNOWN" in bn.status_string(99)


def test_workspace_bytes():
    assert bn.bitnet_linear_workspace_bytes(1, 4096) == 0
    assert bn.bitnet_linear_workspace_bytes(15, 4096) == 0
    assert bn.bitnet_linear_workspace_bytes(16, 4096) == 16 * 4096 + 256 + 256
    assert bn.bitnet_linear_workspace_bytes(8192, 11008) == 8192 * 11008 + 16384 + 32768
    # M * K over the fused GEMV's on-chip limit takes the split path
    assert bn.bitnet_linear_workspace_bytes(15, 16384) > 0
    assert bn.bitnet_linear_workspace_bytes(0, 4096) == 0


P = ctypes.c_void_p
FAKE = P(0x10000)        # 16-byte aligned, never dereferenced: calls fail first
ODD = P(0x10008)


@pytest.mark.parametrize("call,expect", [
    (lambda L: L.bitnet_gemm(None, FAKE, FAKE, FAKE, FAKE, 1, 4, 4, 64, None), bn.ERR_NULL),
    (lambda L: L.bitnet_gemm(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, 4, 48, None), bn.ERR_SHAPE),
    (lambda L: L.bitnet_gemm(FAKE, FAKE, FAKE, FAKE, FAKE, 1, -1, 4, 64, None), bn.ERR_SHAPE),
    (lambda L: L.bitnet_gemm(FAKE, FAKE, FAKE, FAKE, FAKE, 3, 4, 4, 64, None), bn.ERR_SHAPE),
    (lambda L: L.bitnet_gemm(FAKE, FAKE, FAKE, FAKE, None, 1, 4, 4, 64, None), bn.ERR_NULL),
    (lambda L: L.bitnet_gemm(ODD, FAKE, FAKE, FAKE, FAKE, 1, 4, 4, 64, None), bn.ERR_ALIGN),
    (lambda L: L.bitnet_gemm(FAKE, FAKE, ODD, FAKE, FAKE, 1, 4, 4, 64, None), bn.ERR_ALIGN),
    (lambda L: L.bitnet_gemv_fused(FAKE, FAKE, 0, FAKE, FAKE, 1, 16, 4, 64, None), bn.ERR_SHAPE),
    (lambda L: L.bitnet_gemv_fused(FAKE, FAKE, 0, FAKE, FAKE, 1, 0, 4, 64, None), bn.ERR_SHAPE),
    (lambda L: L.bitnet_gemv_fused(FAKE, FAKE, 2, FAKE, FAKE, 1, 1, 4, 64, None), bn.ERR_DTYPE),
    # float32 activations (dtype 1) are validated like bf16 ones
    (lambda L: L.bitnet_gemv_fused(FAKE, ODD, 1, FAKE, FAKE, 1, 1, 4, 64, None), bn.ERR_ALIGN),
    (lambda L: L.bitnet_quantize_act(FAKE, FAKE, FAKE, 1, 2, 40, None), bn.ERR_SHAPE),
    (lambda L: L.bitnet_linear(FAKE, FAKE, 1, FAKE, FAKE, 1, 32, 4, 64, None, 0, None),
     bn.ERR_WORKSPACE),
    (lambda L: L.bitnet_gemv_fused(FAKE, ODD, 0, FAKE, FAKE, 1, 1, 4, 64, None), bn.ERR_ALIGN),
    (lambda L: L.bitnet_gemv_fused(FAKE, FAKE, 0, FAKE, FAKE, 1, 15, 4, 16384, None), bn.ERR_SHAPE),
    (lambda L: L.bitnet_quantize_act(FAKE, FAKE, FAKE, 0, 2, 40, None), bn.ERR_SHAPE),
    (lambda L: L.bitnet_quantize_act(FAKE, FAKE, None, 0, 2, 64, None), bn.ERR_NULL),
    (lambda L: L.bitnet_quantize_act(FAKE, FAKE, FAKE, 2, 2, 64, None), bn.ERR_DTYPE),
    (lambda L: L.bitnet_pack_weights(FAKE, FAKE, 4, 6, None), bn.ERR_SHAPE),
    (lambda L: L.bitnet_ternarize_absmean(FAKE, FAKE, FAKE, 4, 6, 1, None), bn.ERR_SHAPE),
    (lambda L: L.bitnet_ternarize_absmean(FAKE, FAKE, FAKE, 4, 8, 0, None), bn.ERR_SHAPE),
    (lambda L: L.bitnet_ternarize_absmean(None, FAKE, FAKE, 4, 16, 1, None), bn.ERR_NULL),
    (lambda L: L.bitnet_ternarize_absmean(FAKE, FAKE, ODD, 4, 16, 1, None), bn.ERR_ALIGN),
    (lambda L: L.bitnet_pack_weights(None, FAKE, 4, 8, None), bn.ERR_NULL),
    (lambda L: L.bitnet_linear(FAKE, FAKE, 0, FAKE, FAKE, 1, 32, 4, 64, None, 0, None),
     bn.ERR_WORKSPACE),
    (lambda L: L.bitnet_linear(FAKE, FAKE, 0, FAKE, FAKE, 1, 32, 4, 64, P(0x10010), 1 << 20,
                               None), bn.ERR_ALIGN),
    (lambda L: L.bitnet_linear(FAKE, FAKE, 0, FAKE, FAKE, 1, 32, 4, 65, FAKE, 1 << 20, None),
     bn.ERR_SHAPE),
    (lambda L: L.bitnet_gemm_acc_i32(FAKE, None, FAKE, 4, 4, 64, None), bn.ERR_NULL),
    (lambda L: L.bitnet_linear_bias(FAKE, FAKE, 0, FAKE, FAKE, 1, None, 4, 4, 64, None, 0, None),
     bn.ERR_NULL),
    (lambda L: L.bitnet_linear_bias(FAKE, FAKE, 0, FAKE, FAKE, 1, P(0x10001), 4, 4, 64, None, 0,
                                    None),
     bn.ERR_ALIGN),
    (lambda L: L.bitnet_gemv_fused_debug(FAKE, FAKE, None, FAKE, 0, FAKE, 1, 4, 64, None),
     bn.ERR_NULL),
    (lambda L: L.bitnet_rmsnorm_quantize_act(FAKE, FAKE, FAKE, FAKE, 1e-5, 4, 48, None),
     bn.ERR_SHAPE),
    (lambda L: L.bitnet_rmsnorm_quantize_act(FAKE, FAKE, FAKE, FAKE, 0.0, 4, 64, None),
     bn.ERR_VALUE),
    (lambda L: L.bitnet_rmsnorm_quantize_act(FAKE, FAKE, FAKE, FAKE, float("nan"), 4, 64, None),
     bn.ERR_VALUE),
    (lambda L: L.bitnet_rmsnorm_quantize_act(FAKE, FAKE, FAKE, FAKE, float("inf"), 4, 64, None),
     bn.ERR_VALUE),
    (lambda L: L.bitnet_rmsnorm_quantize_act(FAKE, FAKE, FAKE, None, 1e-5, 4, 64, None),
     bn.ERR_NULL),
    (lambda L: L.bitnet_rmsnorm_quantize_act(FAKE, FAKE, P(0x10008), FAKE, 1e-5, 4, 64, None),
     bn.ERR_ALIGN),
    (lambda L: L.bitnet_linear_rmsnorm(FAKE, FAKE, FAKE, -1.0, FAKE, FAKE, 1, 4, 4, 64, FAKE,
                                       1 << 20, None), bn.ERR_VALUE),
    (lambda L: L.bitnet_linear_rmsnorm(FAKE, FAKE, FAKE, 1e-5, FAKE, FAKE, 1, 4, 4, 64, FAKE, 500,
                                       None), bn.ERR_WORKSPACE),
    (lambda L: L.bitnet_linear_rmsnorm(FAKE, FAKE, FAKE, 1e-5, FAKE, FAKE, 1, 32, 4, 64, FAKE,
                                       2559, None), bn.ERR_WORKSPACE),
    (lambda L: L.bitnet_linear_rmsnorm(FAKE, FAKE, None, 1e-5, FAKE, FAKE, 1, 4, 4, 64, FAKE,
                                       1 << 20, None), bn.ERR_NULL),
    (lambda L: L.bitnet_linear_rmsnorm(FAKE, FAKE, FAKE, 1e-5, FAKE, FAKE, 1, 4, 4, 96,
                                       P(0x10080), 1 << 20, None), bn.ERR_ALIGN),
    # the accumulator hooks validate like the product entries
    (lambda L: L.bitnet_linear_acc_i32(FAKE, None, FAKE, FAKE, 0, FAKE, 4, 4, 64, None, 0, None),
     bn.ERR_NULL),
    (lambda L: L.bitnet_linear_acc_i32(ODD, FAKE, FAKE, FAKE, 0, FAKE, 4, 4, 64, None, 0, None),
     bn.ERR_ALIGN),
    (lambda L: L.bitnet_linear_acc_i32(FAKE, FAKE, FAKE, FAKE, 0, FAKE, 32, 4, 64, None, 0, None),
     bn.ERR_WORKSPACE),
    (lambda L: L.bitnet_linear_acc_i32(FAKE, FAKE, FAKE, FAKE, 3, FAKE, 4, 4, 64, None, 0, None),
     bn.ERR_DTYPE),
    (lambda L: L.bitnet_gemv_fused_grouped_acc_i32(FAKE, None, FAKE, 1, 1, 0, None), bn.ERR_NULL),
    # the allocation-free linear refuses a shape whose activations do not fit
    # its built-in scratch before any CUDA call (M = 4096, K = 8192 needs 32 MiB)
    (lambda L: L.bitnet_linear_noalloc(FAKE, FAKE, 0, FAKE, FAKE, 1, 4096, 256, 8192, None),
     bn.ERR_WORKSPACE),
])
def test_validation_rejects_before_launch(call, expect):
    assert call(bn.lib()) == expect


def test_failure_path_switch_only_in_the_test_library():
    """The stage-skipping switch and the 1 ms wait limit live in the test
    library alone; the product library exports none of its entry points."""
    assert not hasattr(bn.lib(), "bitnet_wait_test_gemv")
    path = os.path.join(os.path.dirname(bn.LIB_PATH), "libbitnet_b200_waittest.so")
    T = ctypes.CDLL(path)
    assert hasattr(T, "bitnet_wait_test_gemv") and hasattr(T, "bitnet_wait_test_status")
    T.bitnet_wait_test_gemv.argtypes = [P, P, P, P, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_int, P]
    # validation happens before any CUDA call
    assert T.bitnet_wait_test_gemv(FAKE, FAKE, FAKE, FAKE, 64, 96, -1, None) == bn.ERR_SHAPE
    assert T.bitnet_wait_test_gemv(None, FAKE, FAKE, FAKE, 64, 128, -1, None) == bn.ERR_NULL


def test_rmsnorm_workspace_size():
    """Rows the fused GEMV takes: the bf16 normalised rows. Otherwise int8
    codes, bf16 scales and int32 code sums. Each part rounded up to 256 bytes."""
    L = bn.lib()
    assert L.bitnet_linear_rmsnorm_workspace_bytes(3, 64) == 512
    assert L.bitnet_linear_rmsnorm_workspace_bytes(32, 64) == 2048 + 256 + 256
    assert L.bitnet_linear_rmsnorm_workspace_bytes(300, 2560) == 768000 + 768 + 1280
    assert L.bitnet_linear_rmsnorm_workspace_bytes(0, 64) == 0
    # one or two rows the fused GEMV takes are normalised inside it: no scratch
    assert L.bitnet_linear_rmsnorm_workspace_bytes(1, 4096) == 0
    assert L.bitnet_linear_rmsnorm_workspace_bytes(2, 16384) == 0
    assert L.bitnet_linear_rmsnorm_workspace_bytes(3, 4096) == 3 * 4096 * 2


def test_noop_sizes_return_ok_without_work():
    L = bn.lib()
    assert L.bitnet_gemm(None, None, None, None, None, 1, 0, 4, 64, None) == bn.OK
    assert L.bitnet_gemm(None, None, None, None, None, 1, 4, 0, 64, None) == bn.OK
    assert L.bitnet_pack_weights(None, None, 0, 8, None) == bn.OK
    assert L.bitnet_quantize_act(None, None, None, 0, 0, 64, None) == bn.OK
    assert L.bitnet_linear(None, None, 0, None, None, 1, 0, 4, 64, None, 0, None) == bn.OK
    # the widened rows' entries: empty inputs are no-ops too
    assert L.bitnet_ternarize_absmean(None, None, None, 0, 64, 1, None) == bn.OK
    assert L.bitnet_ternarize_absmean(None, None, None, 0, 64, 0, None) == bn.OK
    assert L.bitnet_linear_bias(None, None, 0, None, None, 1, FAKE, 0, 4, 64, None, 0, None) == bn.OK
    assert L.bitnet_rmsnorm_quantize_act(None, None, None, None, 1e-5, 0, 64, None) == bn.OK
    assert L.bitnet_linear_rmsnorm(None, None, None, 1e-5, None, None, 1, 0, 4, 64, None, 0,
                                   None) == bn.OK
    assert L.bitnet_linear_rmsnorm(None, None, None, 1e-5, None, None, 1, 4, 0, 64, None, 0,
                                   None) == bn.OK


def test_grouped_validation_before_launch():
    L = bn.lib()
    arr = (bn.GemvProblem * 2)()
    for i in range(2):
        arr[i] = bn.GemvProblem(0x10000, 0x10000, 0x10000, 0x10000, 1, 64, 128)
    p = ctypes.cast(arr, ctypes.c_void_p)
    assert L.bitnet_gemv_fused_grouped(p, 0, 1, 0, None) == bn.OK
    assert L.bitnet_gemv_fused_grouped(None, 2, 1, 0, None) == bn.ERR_NULL
    assert L.bitnet_gemv_fused_grouped(p, -1, 1, 0, None) == bn.ERR_SHAPE
    assert L.bitnet_gemv_fused_grouped(p, 2, 16, 0, None) == bn.ERR_SHAPE
    assert L.bitnet_gemv_fused_grouped(p, 2, 1, 2, None) == bn.ERR_DTYPE
    arr[1] = bn.GemvProblem(0x10000, 0x10000, 0x10000, 0x10000, 1, 64, 48)   # K % 32
    assert L.bitnet_gemv_fused_grouped(p, 2, 1, 0, None) == bn.ERR_SHAPE
    arr[1] = bn.GemvProblem(0x10008, 0x10000, 0x10000, 0x10000, 1, 64, 128)  # out align
    assert L.bitnet_gemv_fused_grouped(p, 2, 1, 0, None) == bn.ERR_ALIGN
    arr[1] = bn.GemvProblem(0x10000, 0x10000, 0x10000, 0x10000, 3, 64, 128)  # scale len
    assert L.bitnet_gemv_fused_grouped(p, 2, 1, 0, None) == bn.ERR_SHAPE


def test_bench_traffic_record_names_existing_sources():
    """The bench reports the recorded DRAM traffic only while the kernel's
    sources hash as they did at capture; every header it hashes must exist,
    and the record must name a summary that is committed."""
    import json
    import os
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    csrc = os.path.join(root, "bit_gemm_bitnet_b200", "csrc")
    for kernel, files in bench.KERNEL_SOURCES.items():
        for f in files:
            assert os.path.exists(os.path.join(csrc, f)), (kernel, f)
        assert len(bench.source_hash(kernel)) == 16
    rec = json.load(open(os.path.join(root, "profiles", "ncu_traffic.json")))
    for kernel, r in rec.items():
        assert os.path.exists(os.path.join(root, r["summary"])), r["summary"]
        assert r["bytes"] > 0
