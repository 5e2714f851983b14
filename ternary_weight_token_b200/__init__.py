"""B200 BitLinear (W1.58A8): Python binding of the C ABI in ``include/bitnet.h``.

The binding only marshals arguments: every step of the path (ternarise and
pack, prelude and per-token quant, int8 x ternary contraction, epilogue) runs
in the CUDA kernels of ``libbitnet_b200.so``.  PyTorch supplies device memory
and the current stream.  There is no CPU fallback: if the library is missing
or no CUDA device is present the calls raise.

Functions carry the C names and take torch tensors plus explicit outputs:

    bitnet_pack_weights(W, packed, gamma, workspace)
    bitnet_quant_act(X, Xq, x_scale, x_rowsum, prelude=..., norm_gain=None, eps=1e-5)
    bitnet_linear(Xq, x_scale, x_rowsum, packed, gamma, K, Y, epilogue=..., residual=None)
    bitnet_ffn(X, W_gate, gamma_gate, W_up, gamma_up, W_down, gamma_down, Y, workspace, ...)

``alloc_*`` helpers size the outputs with torch.
"""
from ._binding import (  # noqa: F401
    BITNET_BF16,
    BITNET_EPI_RESIDUAL,
    BITNET_EPI_SILU,
    BITNET_EPI_TYPE_MASK,
    BITNET_FFN_SINGLE_LAUNCH,
    BITNET_ERR_CUDA,
    BITNET_ERR_INVALID_ARG,
    BITNET_ERR_TIMEOUT,
    BITNET_ERR_UNSUPPORTED,
    BITNET_ERR_WORKSPACE,
    BITNET_F32,
    BITNET_FFN_HADAMARD_SILU,
    BITNET_FFN_RELU2_GLU,
    BITNET_I32,
    BITNET_LAUNCH_PDL,
    BITNET_LAUNCH_PDL_INPUTS,
    BITNET_OK,
    BITNET_PLAN_FLAT,
    BITNET_PLAN_GEMM_TC,
    BITNET_PLAN_GEMV,
    BITNET_PLAN_GEMV_TC,
    BITNET_PLAN_STREAM,
    BITNET_PRELUDE_FWHT,
    BITNET_PRELUDE_NONE,
    BITNET_PRELUDE_RMSNORM,
    BitnetError,
    alloc_block_tail_workspace,
    alloc_ffn_workspace,
    alloc_packed,
    alloc_quant,
    bitnet_block_tail,
    bitnet_block_tail_workspace_size,
    bitnet_check_device_error,
    bitnet_debug_wait_timeout,
    bitnet_export_tw2,
    bitnet_ffn,
    bitnet_ffn_noalloc,
    BITNET_FFN_NOALLOC_SCRATCH_BYTES,
    bitnet_ffn_workspace_size,
    bitnet_last_error,
    bitnet_import_tw2,
    bitnet_linear,
    bitnet_linear_multi,
    bitnet_pack_weights,
    bitnet_pack_workspace_size,
    bitnet_packed_row_bytes,
    bitnet_plan_linear,
    bitnet_quant_act,
    bitnet_release_cache,
    bitnet_version,
    library,
    library_path,
)
