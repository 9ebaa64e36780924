"""BitNet b1.58 W1.58A8 linear layer on B200: Python binding of libbitnet_b200.

A thin ctypes layer over the C ABI declared in ``include/bitnet.h``. It only
marshals arguments: it checks tensor dtypes, devices and contiguity, allocates
outputs with torch, passes raw device pointers and the current CUDA stream,
and turns status codes into exceptions. Every step of the computation runs in
the library's CUDA kernels; there is no fallback of any kind. If the library
is missing, every call raises.

Function names follow the C entry points (and the bitnet-cpu page's API:
pack_weights, quantize_activation, bitnet_gemm, bitnet_gemv_fused,
bitnet_linear).
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitnet_b200.so")

OK, ERR_NULL, ERR_SHAPE, ERR_DTYPE, ERR_ALIGN, ERR_VALUE, ERR_WORKSPACE, \
    ERR_CUDA, ERR_TIMEOUT = range(9)
BF16 = 0
F32 = 1

# every symbol include/bitnet.h declares
EXPORTS = (
    "bitnet_ternarize_absmean", "bitnet_pack_weights", "bitnet_quantize_act", "bitnet_gemm",
    "bitnet_gemv_fused", "bitnet_linear_workspace_bytes", "bitnet_linear",
    "bitnet_device_status", "bitnet_status_string", "bitnet_gemm_acc_i32",
    "bitnet_gemv_fused_debug", "bitnet_linear_noalloc", "bitnet_gemv_fused_grouped",
    "bitnet_linear_bias", "bitnet_rmsnorm_quantize_act", "bitnet_linear_rmsnorm_workspace_bytes",
    "bitnet_linear_rmsnorm", "bitnet_linear_acc_i32", "bitnet_gemv_fused_grouped_acc_i32",
)


class GemvProblem(ctypes.Structure):
    """bitnet_gemv_problem of include/bitnet.h."""
    _fields_ = [("out", ctypes.c_void_p), ("x", ctypes.c_void_p),
                ("w_packed", ctypes.c_void_p), ("scale_wt", ctypes.c_void_p),
                ("scale_wt_len", ctypes.c_int64), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64)]

_lib = None


class BitnetError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


class BitnetValueError(BitnetError, ValueError):
    pass


def lib():
    """Load libbitnet_b200.so (built in-tree); raise if it is absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"libbitnet_b200.so not found at {LIB_PATH}; build it with "
                "`python -m bit_gemm_bitnet_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, SZ, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
        F = ctypes.c_float
        sig = {
            "bitnet_pack_weights": [P, P, I64, I64, P],
            "bitnet_ternarize_absmean": [P, P, P, I64, I64, I, P],
            "bitnet_quantize_act": [P, P, P, I, I64, I64, P],
            "bitnet_gemm": [P, P, P, P, P, I64, I64, I64, I64, P],
            "bitnet_gemv_fused": [P, P, I, P, P, I64, I64, I64, I64, P],
            "bitnet_linear": [P, P, I, P, P, I64, I64, I64, I64, P, SZ, P],
            "bitnet_linear_bias": [P, P, I, P, P, I64, P, I64, I64, I64, P, SZ, P],
            "bitnet_linear_noalloc": [P, P, I, P, P, I64, I64, I64, I64, P],
            "bitnet_rmsnorm_quantize_act": [P, P, P, P, F, I64, I64, P],
            "bitnet_linear_rmsnorm": [P, P, P, F, P, P, I64, I64, I64, I64, P, SZ, P],
            "bitnet_gemv_fused_grouped": [P, I64, I64, I, P],
            "bitnet_device_status": [P],
            "bitnet_gemm_acc_i32": [P, P, P, I64, I64, I64, P],
            "bitnet_gemv_fused_debug": [P, P, P, P, I, P, I64, I64, I64, P],
            "bitnet_linear_acc_i32": [P, P, P, P, I, P, I64, I64, I64, P, SZ, P],
            "bitnet_gemv_fused_grouped_acc_i32": [P, P, P, I64, I64, I, P],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.bitnet_linear_workspace_bytes.argtypes = [I64, I64]
        L.bitnet_linear_workspace_bytes.restype = SZ
        L.bitnet_linear_rmsnorm_workspace_bytes.argtypes = [I64, I64]
        L.bitnet_linear_rmsnorm_workspace_bytes.restype = SZ
        L.bitnet_status_string.argtypes = [ctypes.c_int]
        L.bitnet_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(status):
    return lib().bitnet_status_string(int(status)).decode()


def _check(status, what):
    if status == OK:
        return
    if status in (ERR_NULL, ERR_SHAPE, ERR_DTYPE, ERR_ALIGN, ERR_VALUE, ERR_WORKSPACE):
        raise BitnetValueError(status, what)
    raise BitnetError(status, what)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _act_dt(t, name, ndim=None):
    """Activations: bf16 or float32; returns the C dtype code."""
    if isinstance(t, torch.Tensor) and t.dtype == torch.float32:
        _need(t, torch.float32, name, ndim)
        return F32
    _need(t, torch.bfloat16, name, ndim)
    return BF16


def _need(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-D, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _out(out, dtype, shape, device, name="out"):
    """A caller-supplied output buffer, checked before anything is launched
    (dtype, device, shape, contiguity), or a new one."""
    if out is None:
        return torch.empty(shape, dtype=dtype, device=device)
    _need(out, dtype, name)
    if tuple(out.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(out.shape)}")
    if out.device != torch.device(device):
        raise ValueError(f"{name} is on {out.device}, expected {device}")
    return out


def _out_rows(out, orig, M, N, device):
    """bf16 output of the linear entries: shape (M, N) or the input's leading
    dimensions followed by N; returned as an (M, N) view."""
    if out is None:
        return torch.empty((M, N), dtype=torch.bfloat16, device=device)
    if tuple(out.shape) == tuple(orig[:-1]) + (N,):
        _need(out, torch.bfloat16, "out")
        out = out.view(M, N)
    return _out(out, torch.bfloat16, (M, N), device)


def _scale_wt(scale_wt, N, device):
    """fp32 weight scale of length 1 or N (bf16 [N] is widened exactly)."""
    if not isinstance(scale_wt, torch.Tensor):
        scale_wt = torch.tensor([float(scale_wt)], dtype=torch.float32, device=device)
    if scale_wt.dtype == torch.bfloat16:
        scale_wt = scale_wt.float()
    sw = scale_wt.reshape(-1).contiguous()
    _need(sw, torch.float32, "scale_wt")
    if sw.numel() not in (1, N):
        raise ValueError(f"scale_wt must have 1 or N={N} elements, got {sw.numel()}")
    return sw


# ---------------------------------------------------------------- entries

def bitnet_pack_weights(w, out=None):
    """int8 [N, K] in {-1, 0, +1} -> uint8 [N, K/4] (synchronises)."""
    _need(w, torch.int8, "w", 2)
    N, K = w.shape
    out = _out(out, torch.uint8, (N, K // 4), w.device)
    _check(lib().bitnet_pack_weights(_ptr(out), _ptr(w), N, K, _stream(w.device)),
           "bitnet_pack_weights")
    return out


def bitnet_ternarize_absmean(w, per_row=True, w_t=None, scale_wt=None):
    """float32 [N, K] weights -> (int8 ternary [N, K], float32 scale [N] or
    [1]): absmean ternarisation (BitLinear.from_dense per row; BitLinearKernel
    per tensor), ready for bitnet_pack_weights."""
    _need(w, torch.float32, "w", 2)
    N, K = w.shape
    w_t = _out(w_t, torch.int8, (N, K), w.device, "w_t")
    scale_wt = _out(scale_wt, torch.float32, (N if per_row else 1,), w.device, "scale_wt")
    _check(lib().bitnet_ternarize_absmean(_ptr(w_t), _ptr(scale_wt), _ptr(w), N, K,
                                          1 if per_row else 0, _stream(w.device)),
           "bitnet_ternarize_absmean")
    return w_t, scale_wt


def bitnet_quantize_act(x, x_q=None, scale_act=None):
    """bf16 or float32 [..., K] -> (int8 [M, K], bf16 [M])."""
    x2 = x.reshape(-1, x.shape[-1])
    dt = _act_dt(x2, "x", 2)
    M, K = x2.shape
    x_q = _out(x_q, torch.int8, (M, K), x.device, "x_q")
    scale_act = _out(scale_act, torch.bfloat16, (M,), x.device, "scale_act")
    _check(lib().bitnet_quantize_act(_ptr(x_q), _ptr(scale_act), _ptr(x2), dt, M, K,
                                     _stream(x.device)), "bitnet_quantize_act")
    return x_q, scale_act


def bitnet_gemm(x_q, w_packed, scale_act, scale_wt, out=None):
    """int8 [M, K] x packed [N, K/4] -> bf16 [M, N]."""
    _need(x_q, torch.int8, "x_q", 2)
    _need(w_packed, torch.uint8, "w_packed", 2)
    _need(scale_act, torch.bfloat16, "scale_act", 1)
    M, K = x_q.shape
    N = w_packed.shape[0]
    if w_packed.shape[1] * 4 != K:
        raise ValueError(f"w_packed {tuple(w_packed.shape)} does not match K={K}")
    if scale_act.numel() != M:
        raise ValueError(f"scale_act has {scale_act.numel()} elements, expected M={M}")
    sw = _scale_wt(scale_wt, N, x_q.device)
    out = _out(out, torch.bfloat16, (M, N), x_q.device)
    _check(lib().bitnet_gemm(_ptr(out), _ptr(x_q), _ptr(w_packed), _ptr(scale_act),
                             _ptr(sw), sw.numel(), M, N, K, _stream(x_q.device)),
           "bitnet_gemm")
    return out


def bitnet_gemv_fused(x, w_packed, scale_wt, out=None):
    """bf16 or float32 [M, K] (M < 16) -> bf16 [M, N], quantisation fused."""
    dt = _act_dt(x, "x", 2)
    _need(w_packed, torch.uint8, "w_packed", 2)
    M, K = x.shape
    N = w_packed.shape[0]
    if w_packed.shape[1] * 4 != K:
        raise ValueError(f"w_packed {tuple(w_packed.shape)} does not match K={K}")
    sw = _scale_wt(scale_wt, N, x.device)
    out = _out(out, torch.bfloat16, (M, N), x.device)
    _check(lib().bitnet_gemv_fused(_ptr(out), _ptr(x), dt, _ptr(w_packed), _ptr(sw),
                                   sw.numel(), M, N, K, _stream(x.device)),
           "bitnet_gemv_fused")
    return out


def gemv_problems(xs, w_packeds, scale_wts, outs):
    """ctypes array of problem descriptors (the tensors must stay alive)."""
    arr = (GemvProblem * len(xs))()
    for i, (x, wp, sw, o) in enumerate(zip(xs, w_packeds, scale_wts, outs)):
        arr[i] = GemvProblem(o.data_ptr(), x.data_ptr(), wp.data_ptr(), sw.data_ptr(),
                             sw.numel(), wp.shape[0], x.shape[1])
    return arr


def bitnet_gemv_fused_grouped(xs, w_packeds, scale_wts, outs=None):
    """Independent fused GEMV problems with the same M in one call:
    xs[i] bf16 [M, K_i], w_packeds[i] uint8 [N_i, K_i/4] -> bf16 [M, N_i]."""
    if not (len(xs) == len(w_packeds) == len(scale_wts)):
        raise ValueError("xs, w_packeds and scale_wts must have the same length")
    if len(xs) == 0:
        return []
    M = xs[0].shape[0]
    sws, new_outs = [], []
    for i, (x, wp, sw) in enumerate(zip(xs, w_packeds, scale_wts)):
        _need(x, torch.bfloat16, f"xs[{i}]", 2)
        _need(wp, torch.uint8, f"w_packeds[{i}]", 2)
        if x.shape[0] != M:
            raise ValueError("every problem of a group has the same M")
        if wp.shape[1] * 4 != x.shape[1]:
            raise ValueError(f"w_packeds[{i}] {tuple(wp.shape)} does not match K={x.shape[1]}")
        sws.append(_scale_wt(sw, wp.shape[0], x.device))
        if outs is None:
            new_outs.append(torch.empty((M, wp.shape[0]), dtype=torch.bfloat16, device=x.device))
    if outs is None:
        outs = new_outs
    else:
        if len(outs) != len(xs):
            raise ValueError("outs must have one tensor per problem")
        for i, (o, wp) in enumerate(zip(outs, w_packeds)):
            _out(o, torch.bfloat16, (M, wp.shape[0]), xs[0].device, f"outs[{i}]")
    arr = gemv_problems(xs, w_packeds, sws, outs)
    _check(lib().bitnet_gemv_fused_grouped(ctypes.cast(arr, ctypes.c_void_p), len(xs), M, BF16,
                                           _stream(xs[0].device)),
           "bitnet_gemv_fused_grouped")
    return outs


def bitnet_linear_workspace_bytes(M, K):
    return int(lib().bitnet_linear_workspace_bytes(M, K))


def bitnet_linear(x, w_packed, scale_wt, out=None, workspace=None, bias=None):
    """bf16 or float32 [..., K] -> bf16 [..., N]; dispatches by M like the
    page's bitnet_linear (fused GEMV for M < 16, else quantise + GEMM).
    bias (bf16 [N]), if given, is added in the epilogue as the page's
    BitLinear.forward adds it to the bf16 output."""
    orig = x.shape
    K = orig[-1]
    x2 = x.reshape(-1, K)
    dt = _act_dt(x2, "x", 2)
    _need(w_packed, torch.uint8, "w_packed", 2)
    M = x2.shape[0]
    N = w_packed.shape[0]
    if w_packed.shape[1] * 4 != K:
        raise ValueError(f"w_packed {tuple(w_packed.shape)} does not match K={K}")
    sw = _scale_wt(scale_wt, N, x.device)
    out = _out_rows(out, orig, M, N, x.device)
    need = bitnet_linear_workspace_bytes(M, K)
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty((need,), dtype=torch.uint8, device=x.device)
    wsp = _ptr(workspace) if need else None
    if bias is None:
        _check(lib().bitnet_linear(_ptr(out), _ptr(x2), dt, _ptr(w_packed), _ptr(sw),
                                   sw.numel(), M, N, K, wsp, need, _stream(x.device)),
               "bitnet_linear")
    else:
        _need(bias, torch.bfloat16, "bias", 1)
        if bias.numel() != N:
            raise ValueError(f"bias has {bias.numel()} elements, expected N={N}")
        _check(lib().bitnet_linear_bias(_ptr(out), _ptr(x2), dt, _ptr(w_packed), _ptr(sw),
                                        sw.numel(), _ptr(bias), M, N, K, wsp, need,
                                        _stream(x.device)),
               "bitnet_linear_bias")
    return out.view(*orig[:-1], N)


def bitnet_linear_noalloc(x, w_packed, scale_wt, out=None):
    """bitnet_linear without a workspace argument: for M >= 16 the library
    keeps the quantised activations in its built-in 16 MiB scratch (see
    include/bitnet.h); calls that may overlap on the GPU must not share it."""
    orig = x.shape
    K = orig[-1]
    x2 = x.reshape(-1, K)
    dt = _act_dt(x2, "x", 2)
    _need(w_packed, torch.uint8, "w_packed", 2)
    M = x2.shape[0]
    N = w_packed.shape[0]
    if w_packed.shape[1] * 4 != K:
        raise ValueError(f"w_packed {tuple(w_packed.shape)} does not match K={K}")
    sw = _scale_wt(scale_wt, N, x.device)
    out = _out_rows(out, orig, M, N, x.device)
    _check(lib().bitnet_linear_noalloc(_ptr(out), _ptr(x2), dt, _ptr(w_packed), _ptr(sw),
                                       sw.numel(), M, N, K, _stream(x.device)),
           "bitnet_linear_noalloc")
    return out.view(*orig[:-1], N)


def bitnet_rmsnorm_quantize_act(x, g, eps, x_q=None, scale_act=None):
    """bf16 [M, K] -> RMSNorm with weight g (bf16 [K]) and epsilon eps, then
    the per-token quantiser: int8 [M, K] codes, bf16 [M] scales."""
    _need(x, torch.bfloat16, "x", 2)
    _need(g, torch.bfloat16, "g", 1)
    M, K = x.shape
    if g.numel() != K:
        raise ValueError(f"g has {g.numel()} elements, expected K={K}")
    x_q = _out(x_q, torch.int8, (M, K), x.device, "x_q")
    scale_act = _out(scale_act, torch.bfloat16, (M,), x.device, "scale_act")
    _check(lib().bitnet_rmsnorm_quantize_act(_ptr(x_q), _ptr(scale_act), _ptr(x), _ptr(g),
                                             float(eps), M, K, _stream(x.device)),
           "bitnet_rmsnorm_quantize_act")
    return x_q, scale_act


def bitnet_linear_rmsnorm_workspace_bytes(M, K):
    return int(lib().bitnet_linear_rmsnorm_workspace_bytes(M, K))


def bitnet_linear_rmsnorm(x, g, eps, w_packed, scale_wt, out=None, workspace=None):
    """RMSNorm (weight g, epsilon eps), the quantiser and the ternary GEMM:
    bf16 [..., K] -> bf16 [..., N]."""
    orig = x.shape
    K = orig[-1]
    x2 = x.reshape(-1, K)
    _need(x2, torch.bfloat16, "x", 2)
    _need(g, torch.bfloat16, "g", 1)
    _need(w_packed, torch.uint8, "w_packed", 2)
    M = x2.shape[0]
    N = w_packed.shape[0]
    if w_packed.shape[1] * 4 != K:
        raise ValueError(f"w_packed {tuple(w_packed.shape)} does not match K={K}")
    if g.numel() != K:
        raise ValueError(f"g has {g.numel()} elements, expected K={K}")
    sw = _scale_wt(scale_wt, N, x.device)
    out = _out_rows(out, orig, M, N, x.device)
    need = bitnet_linear_rmsnorm_workspace_bytes(M, K)
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty((need,), dtype=torch.uint8, device=x.device)
    _check(lib().bitnet_linear_rmsnorm(_ptr(out), _ptr(x2), _ptr(g), float(eps), _ptr(w_packed),
                                       _ptr(sw), sw.numel(), M, N, K,
                                       _ptr(workspace) if need else None, need,
                                       _stream(x.device)),
           "bitnet_linear_rmsnorm")
    return out.view(*orig[:-1], N)


def bitnet_device_status(device=None):
    """Synchronise the current stream; raise if a kernel gave up a wait."""
    dev = device if device is not None else torch.cuda.current_device()
    _check(lib().bitnet_device_status(_stream(dev)), "bitnet_device_status")


# ------------------------------------------------------------- test hooks

def bitnet_gemm_acc_i32(x_q, w_packed, out=None):
    _need(x_q, torch.int8, "x_q", 2)
    _need(w_packed, torch.uint8, "w_packed", 2)
    M, K = x_q.shape
    N = w_packed.shape[0]
    out = _out(out, torch.int32, (M, N), x_q.device)
    _check(lib().bitnet_gemm_acc_i32(_ptr(out), _ptr(x_q), _ptr(w_packed), M, N, K,
                                     _stream(x_q.device)), "bitnet_gemm_acc_i32")
    return out


def bitnet_gemv_fused_debug(x, w_packed):
    """-> (int32 acc [M, N], int8 codes [M, K], bf16 scales [M])."""
    _need(x, torch.bfloat16, "x", 2)
    _need(w_packed, torch.uint8, "w_packed", 2)
    M, K = x.shape
    N = w_packed.shape[0]
    acc = torch.empty((M, N), dtype=torch.int32, device=x.device)
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    sa = torch.empty((M,), dtype=torch.bfloat16, device=x.device)
    _check(lib().bitnet_gemv_fused_debug(_ptr(acc), _ptr(xq), _ptr(sa), _ptr(x), BF16,
                                         _ptr(w_packed), M, N, K, _stream(x.device)),
           "bitnet_gemv_fused_debug")
    return acc, xq, sa


def bitnet_linear_acc_i32(x, w_packed, workspace=None):
    """bitnet_linear's dispatch and kernels with int32 sums stored instead of
    the epilogue -> (int32 acc [M, N], int8 codes [M, K], bf16 scales [M],
    the workspace used or None)."""
    dt = _act_dt(x, "x", 2)
    _need(w_packed, torch.uint8, "w_packed", 2)
    M, K = x.shape
    N = w_packed.shape[0]
    if w_packed.shape[1] * 4 != K:
        raise ValueError(f"w_packed {tuple(w_packed.shape)} does not match K={K}")
    acc = torch.empty((M, N), dtype=torch.int32, device=x.device)
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    sa = torch.empty((M,), dtype=torch.bfloat16, device=x.device)
    need = bitnet_linear_workspace_bytes(M, K)
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty((need,), dtype=torch.uint8, device=x.device)
    _check(lib().bitnet_linear_acc_i32(_ptr(acc), _ptr(xq), _ptr(sa), _ptr(x), dt,
                                       _ptr(w_packed), M, N, K,
                                       _ptr(workspace) if need else None, need,
                                       _stream(x.device)), "bitnet_linear_acc_i32")
    return acc, xq, sa, (workspace if need else None)


def bitnet_gemv_fused_grouped_acc_i32(xs, w_packeds):
    """bitnet_gemv_fused_grouped's dispatch and kernel with int32 sums stored
    -> a list of (int32 acc [M, N_i], int8 codes [M, K_i], bf16 scales [M])."""
    if len(xs) != len(w_packeds):
        raise ValueError("xs and w_packeds must have the same length")
    if len(xs) == 0:
        return []
    M = xs[0].shape[0]
    dev = xs[0].device
    res, keep = [], []
    for i, (x, wp) in enumerate(zip(xs, w_packeds)):
        _need(x, torch.bfloat16, f"xs[{i}]", 2)
        _need(wp, torch.uint8, f"w_packeds[{i}]", 2)
        if x.shape[0] != M or wp.shape[1] * 4 != x.shape[1]:
            raise ValueError(f"problem {i}: shapes {tuple(x.shape)}, {tuple(wp.shape)}")
        res.append((torch.empty((M, wp.shape[0]), dtype=torch.int32, device=dev),
                    torch.empty((M, x.shape[1]), dtype=torch.int8, device=dev),
                    torch.empty((M,), dtype=torch.bfloat16, device=dev)))
        keep.append(torch.ones(1, dtype=torch.float32, device=dev))
    arr = gemv_problems(xs, w_packeds, keep, [r[0] for r in res])
    qs = (ctypes.c_void_p * len(xs))(*[r[1].data_ptr() for r in res])
    sas = (ctypes.c_void_p * len(xs))(*[r[2].data_ptr() for r in res])
    _check(lib().bitnet_gemv_fused_grouped_acc_i32(ctypes.cast(arr, ctypes.c_void_p),
                                                   ctypes.cast(qs, ctypes.c_void_p),
                                                   ctypes.cast(sas, ctypes.c_void_p), len(xs), M,
                                                   BF16, _stream(dev)),
           "bitnet_gemv_fused_grouped_acc_i32")
    return res


# the page's Python names
pack_weights = bitnet_pack_weights
quantize_activation = bitnet_quantize_act
