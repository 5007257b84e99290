"""B200-native residual-compression activation codec (libcf) and its binding.

The codec: per communicated activation tensor and per denoising step, form the
residual against the base tensor, add the error-feedback buffer, compress it
(k-bit group quantisation or rank-r subspace iteration), and decompress into
the receiver's reconstruction cache ("Accelerating Parallel Diffusion Model
Serving with Residual Compression", arXiv 2507.17511: abstract; reproducibility
table, "Dataset Splits" and "Pseudocode" rows).

All arithmetic runs in the sm_100a kernels of ``libcf.so``; this package only
builds the library and marshals arguments.
"""
from ._cf import (  # noqa: F401
    CF_E_ALIGN, CF_E_ARG, CF_E_CUDA, CF_E_NOMEM, CF_E_NONFINITE, CF_E_SHAPE, CF_E_STATE, CF_E_TIMEOUT,
    CF_MODE_LOWRANK, CF_MODE_QUANT, CF_OK, CF_PRECISION_AUTO, CF_PRECISION_SPLIT, CF_PRECISION_TF32, EXPORTED,
    KV, CfError, Context, Slot, cf_check, cf_compress, cf_config, cf_create, cf_kv, cf_decompress, cf_destroy, cf_loopback, cf_lowrank, cf_lowrank_noalloc, cf_payload_bytes, lib,
    NOALLOC_SCRATCH_BYTES,
)
from .state import HostStreamCodec, QuantState, alloc_quant_state  # noqa: F401
