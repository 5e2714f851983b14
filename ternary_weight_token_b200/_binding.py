"""ctypes marshalling for ``libbitnet_b200.so`` (argument passing only)."""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libbitnet_b200.so"

BITNET_OK = 0
BITNET_ERR_INVALID_ARG = 1
BITNET_ERR_UNSUPPORTED = 2
BITNET_ERR_CUDA = 3
BITNET_ERR_WORKSPACE = 4
BITNET_ERR_TIMEOUT = 5

BITNET_F32, BITNET_BF16, BITNET_I32 = 0, 1, 2
BITNET_PRELUDE_NONE, BITNET_PRELUDE_RMSNORM, BITNET_PRELUDE_FWHT = 0, 1, 2
BITNET_EPI_TYPE_MASK = 0x0F
BITNET_EPI_RESIDUAL = 0x10
BITNET_EPI_SILU = 0x20
BITNET_LAUNCH_PDL = 0x100
BITNET_LAUNCH_PDL_INPUTS = 0x200
BITNET_FFN_RELU2_GLU, BITNET_FFN_HADAMARD_SILU = 0, 1
BITNET_FFN_SINGLE_LAUNCH = 0x200
(BITNET_PLAN_STREAM, BITNET_PLAN_FLAT, BITNET_PLAN_GEMV_TC, BITNET_PLAN_GEMV,
 BITNET_PLAN_GEMM_TC) = 1, 2, 3, 4, 5

_DTYPE_CODE = {torch.float32: BITNET_F32, torch.bfloat16: BITNET_BF16, torch.int32: BITNET_I32}


class BitnetError(RuntimeError):
    def __init__(self, code, message):
        super().__init__(f"bitnet error {code}: {message}")
        self.code = code


_lib = None


def library_path():
    return os.path.join(_HERE, _LIB_NAME)


def library():
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(f"{_LIB_NAME} is not built; run ternary_weight_token_b200/build.py "
                          "(the BitLinear path has no CPU fallback)")
    lib = ctypes.CDLL(path)
    P, I, U, S, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t, ctypes.c_float
    sigs = {
        "bitnet_packed_row_bytes": (S, [I]),
        "bitnet_pack_workspace_size": (S, [I, I]),
        "bitnet_pack_weights": (I, [P, I, I, I, P, P, P, S, P]),
        "bitnet_export_tw2": (I, [P, I, I, P, P]),
        "bitnet_linear_multi": (I, [P, P, P, I, P, P, P, I, I, P, I, P]),
        "bitnet_import_tw2": (I, [P, I, I, P, P]),
        "bitnet_quant_act": (I, [P, I, I, I, I, P, F, P, P, P, P]),
        "bitnet_linear": (I, [P, P, P, P, P, I, I, I, P, I, P, P]),
        "bitnet_plan_linear": (I, [I, I, I, I, I, P]),
        "bitnet_ffn_workspace_size": (S, [I, I, I, I]),
        "bitnet_ffn": (I, [P, I, I, I, I, P, P, P, P, P, P, P, P, F, I, P, I, P, S, P]),
        "bitnet_ffn_noalloc": (I, [P, I, I, I, I, P, P, P, P, P, P, P, P, F, I, P, I, P]),
        "bitnet_block_tail_workspace_size": (S, [I, I, I]),
        "bitnet_block_tail": (I, [P, P, I, I, I, I, P, P, P, P, P, P, P, P, P, P, P, F, P, P, P,
                                  S, P]),
        "bitnet_last_error": (ctypes.c_char_p, []),
        "bitnet_check_device_error": (I, [P]),
        "bitnet_debug_wait_timeout": (I, [U, P]),
        "bitnet_release_cache": (None, []),
        "bitnet_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the BitLinear library must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the BitLinear library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


_RAW_STREAM = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream):
    if stream is None:
        if _RAW_STREAM is not None:          # the current stream's handle, without a Stream object
            return ctypes.c_void_p(_RAW_STREAM(torch.cuda.current_device()))
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype(t):
    try:
        return _DTYPE_CODE[t.dtype]
    except KeyError:
        raise ValueError(f"unsupported dtype {t.dtype}") from None


def _check(code):
    if code != BITNET_OK:
        raise BitnetError(code, bitnet_last_error())


# --------------------------------------------------------------- host calls

def bitnet_packed_row_bytes(K):
    return int(library().bitnet_packed_row_bytes(int(K)))


def bitnet_pack_workspace_size(N, K):
    return int(library().bitnet_pack_workspace_size(int(N), int(K)))


def bitnet_ffn_workspace_size(M, H, I, variant=BITNET_FFN_RELU2_GLU):
    return int(library().bitnet_ffn_workspace_size(int(M), int(H), int(I), int(variant)))


def bitnet_last_error():
    return library().bitnet_last_error().decode()


def bitnet_version():
    return library().bitnet_version().decode()


def bitnet_release_cache():
    library().bitnet_release_cache()


def bitnet_plan_linear(M, N, K, epilogue=BITNET_BF16, sms=148):
    """The launch plan bitnet_linear() follows for one projection on a device
    with `sms` SMs (host logic only): a dict with the kernel (BITNET_PLAN_*),
    its token tile, CTAs and two kernel-specific values (see the header)."""
    out = (ctypes.c_int * 5)()
    _check(library().bitnet_plan_linear(int(M), int(N), int(K), int(epilogue), int(sms), out))
    return {"kernel": out[0], "tokens": out[1], "grid": out[2], "a": out[3], "b": out[4]}


# ------------------------------------------------------------- device calls

def bitnet_pack_weights(W, packed, gamma, workspace, stream=None):
    """Ternarise W [N][K] (fp32/bf16) into packed codes and gamma (fp32[1])."""
    N, K = W.shape
    _check(library().bitnet_pack_weights(_ptr(W), _dtype(W), N, K, _ptr(packed), _ptr(gamma),
                                         _ptr(workspace), workspace.numel() * workspace.element_size(),
                                         _stream(stream)))


def bitnet_linear_multi(Xq, x_scale, x_rowsum, packed, gamma, K, Y, epilogue=None, stream=None):
    """Several projections of one quantised input: packed, gamma and Y are
    lists (one entry per projection, outputs [M][N_i])."""
    count = len(packed)
    if not (len(gamma) == len(Y) == count):
        raise ValueError("packed, gamma and Y need one entry per projection")
    ptrs = lambda ts: (ctypes.c_void_p * count)(*[_ptr(t) for t in ts])
    Ns = (ctypes.c_int * count)(*[int(y.shape[1]) for y in Y])
    if epilogue is None:
        epilogue = _dtype(Y[0])
    _check(library().bitnet_linear_multi(_ptr(Xq), _ptr(x_scale), _ptr(x_rowsum), count,
                                         ptrs(packed), ptrs(gamma), Ns, Xq.shape[0], int(K),
                                         ptrs(Y), int(epilogue), _stream(stream)))


def bitnet_export_tw2(packed, K, tw2, stream=None):
    """Device-layout packed weights [N][packed_row_bytes(K)] -> the canonical
    exchange layout TW2 [N][K/4] (four codes to a byte, low bits first)."""
    _check(library().bitnet_export_tw2(_ptr(packed), packed.shape[0], int(K), _ptr(tw2),
                                       _stream(stream)))


def bitnet_import_tw2(tw2, K, packed, stream=None):
    """TW2 [N][K/4] -> device-layout packed weights [N][packed_row_bytes(K)]."""
    _check(library().bitnet_import_tw2(_ptr(tw2), tw2.shape[0], int(K), _ptr(packed),
                                       _stream(stream)))


def bitnet_quant_act(X, Xq, x_scale, x_rowsum=None, prelude=BITNET_PRELUDE_NONE, norm_gain=None,
                     eps=1e-5, stream=None):
    """Per-token int8 codes (and scales / code sums) of X [M][K] after the prelude."""
    M, K = X.shape
    _check(library().bitnet_quant_act(_ptr(X), _dtype(X), M, K, int(prelude), _ptr(norm_gain),
                                      float(eps), _ptr(Xq), _ptr(x_scale), _ptr(x_rowsum),
                                      _stream(stream)))


def bitnet_linear(Xq, x_scale, x_rowsum, packed, gamma, K, Y, epilogue=None, residual=None,
                  stream=None):
    """Y [M][N] = dequant(Xq . t^T) with the fused epilogue (type taken from Y)."""
    M = Xq.shape[0]
    N = Y.shape[1]
    if epilogue is None:
        epilogue = _dtype(Y) | (BITNET_EPI_RESIDUAL if residual is not None else 0)
    _check(library().bitnet_linear(_ptr(Xq), _ptr(x_scale), _ptr(x_rowsum), _ptr(packed),
                                   _ptr(gamma), M, N, int(K), _ptr(Y), int(epilogue),
                                   _ptr(residual), _stream(stream)))


def bitnet_ffn(X, W_gate, gamma_gate, W_up, gamma_up, W_down, gamma_down, Y, workspace,
               variant=BITNET_FFN_RELU2_GLU, pre_norm_gain=None, sub_norm_gain=None, eps=1e-5,
               stream=None):
    """One BitLinear FFN (see include/bitnet.h for the two variants)."""
    M, H = X.shape
    I = W_gate.shape[0]
    _check(library().bitnet_ffn(_ptr(X), _dtype(X), M, H, I, _ptr(W_gate), _ptr(gamma_gate),
                                _ptr(W_up), _ptr(gamma_up), _ptr(W_down), _ptr(gamma_down),
                                _ptr(pre_norm_gain), _ptr(sub_norm_gain), float(eps), int(variant),
                                _ptr(Y), _dtype(Y), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream)))


def bitnet_block_tail_workspace_size(M, H, I):
    return int(library().bitnet_block_tail_workspace_size(int(M), int(H), int(I)))


def bitnet_block_tail(A, X, W_o, gamma_o, W_gate, gamma_gate, W_up, gamma_up, W_down,
                      gamma_down, Y, workspace, H_out=None, attn_norm_gain=None,
                      post_norm_gain=None, sub_norm_gain=None, eps=1e-5, stream=None):
    """The block after attention at decode sizes, one launch (include/bitnet.h)."""
    M, H = X.shape
    I = W_gate.shape[0]
    _check(library().bitnet_block_tail(
        _ptr(A), _ptr(X), _dtype(X), M, H, I, _ptr(W_o), _ptr(gamma_o), _ptr(W_gate),
        _ptr(gamma_gate), _ptr(W_up), _ptr(gamma_up), _ptr(W_down), _ptr(gamma_down),
        _ptr(attn_norm_gain), _ptr(post_norm_gain), _ptr(sub_norm_gain), float(eps),
        _ptr(H_out), _ptr(Y), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def alloc_block_tail_workspace(M, H, I, device="cuda"):
    return torch.empty(max(1, bitnet_block_tail_workspace_size(M, H, I)), dtype=torch.uint8,
                       device=device)


BITNET_FFN_NOALLOC_SCRATCH_BYTES = 8 << 20


def bitnet_ffn_noalloc(X, W_gate, gamma_gate, W_up, gamma_up, W_down, gamma_down, Y,
                       variant=BITNET_FFN_RELU2_GLU, pre_norm_gain=None, sub_norm_gain=None,
                       eps=1e-5, stream=None):
    """bitnet_ffn on the library's built-in scratch (no workspace argument)."""
    M, H = X.shape
    I = W_gate.shape[0]
    _check(library().bitnet_ffn_noalloc(_ptr(X), _dtype(X), M, H, I, _ptr(W_gate),
                                        _ptr(gamma_gate), _ptr(W_up), _ptr(gamma_up),
                                        _ptr(W_down), _ptr(gamma_down), _ptr(pre_norm_gain),
                                        _ptr(sub_norm_gain), float(eps), int(variant), _ptr(Y),
                                        _dtype(Y), _stream(stream)))


def bitnet_check_device_error(stream=None):
    """Synchronise and return the device error status (BITNET_OK or an error code)."""
    return int(library().bitnet_check_device_error(_stream(stream)))


def bitnet_debug_wait_timeout(timeout_us, stream=None):
    _check(library().bitnet_debug_wait_timeout(int(timeout_us), _stream(stream)))


# ------------------------------------------------------------ allocations

def alloc_packed(N, K, device="cuda"):
    """(packed uint8 [N][row_bytes], gamma fp32 [1], workspace uint8) for an N x K weight."""
    packed = torch.empty((N, bitnet_packed_row_bytes(K)), dtype=torch.uint8, device=device)
    gamma = torch.empty(1, dtype=torch.float32, device=device)
    ws = torch.empty(bitnet_pack_workspace_size(N, K), dtype=torch.uint8, device=device)
    return packed, gamma, ws


def alloc_quant(M, K, device="cuda"):
    """(codes int8 [M][K], scales fp32 [M], code sums int32 [M])."""
    return (torch.empty((M, K), dtype=torch.int8, device=device),
            torch.empty(M, dtype=torch.float32, device=device),
            torch.empty(M, dtype=torch.int32, device=device))


def alloc_ffn_workspace(M, H, I, variant=BITNET_FFN_RELU2_GLU, device="cuda"):
    return torch.empty(max(1, bitnet_ffn_workspace_size(M, H, I, variant)), dtype=torch.uint8,
                       device=device)
