"""Activation-sparse FFN decode (PowerInfer's neuron-aware sparse FFN) for B200 / sm_100a.

The work runs in hand-written CUDA kernels behind the C ABI declared in
include/pi_sparse_ffn.h (libpi.so).  This package is the thin Python binding: it passes
torch tensors' device pointers and the current stream to the library.  It has no CPU or
PyTorch fallback; importing it fails if libpi.so has not been built.
"""
from ._abi import (PI_F16, PI_F32, PI_MAX_BATCH, PI_NOALLOC_SCRATCH_BYTES, PI_Q4_0, PI_RELU, PI_RELU2, PI_REGLU, EXPORTS,
                   Layer, LayerDesc, LayerWeights, PiError, Trace, Workspace, abi_version, compact_active,
                   decode_stack, decode_stack_host, diag_barrier_timeout, get_perm, kernel_launches, lib, load_layer,
                   make_desc, predict, predict_noalloc, reorder_hot_prefix, sparse_ffn, status_str)

# the C names, for readers coming from the header
pi_load_layer = load_layer
pi_reorder_hot_prefix = reorder_hot_prefix
pi_get_perm = get_perm
pi_predict = predict
pi_predict_noalloc = predict_noalloc
pi_compact_active = compact_active
pi_sparse_ffn = sparse_ffn
pi_decode_stack = decode_stack
pi_decode_stack_host = decode_stack_host
pi_status_str = status_str
pi_kernel_launches = kernel_launches
