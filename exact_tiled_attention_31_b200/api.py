"""ctypes binding of libfa.so (include/fa.h).

Two layers:

* ``fa_*`` (every name in ``EXPORTS``: forward, packed forward, the
  backward and its three launches, the packed and allocation-free
  backwards, dropout forward/backward, decode, status and error helpers):
  the C entry points under the same names, taking raw device pointers (ints)
  and sizes, returning the ``fa_status`` code (or a size).
* ``forward``, ``forward_varlen``, ``backward``, ``backward_varlen``,
  ``backward_noalloc``, ``decode``: tensor conveniences that check
  shapes/dtypes, allocate outputs and workspace with torch unless given
  (device memory and streams are all torch provides) and raise ``FAError``
  on a non-zero status.

Every step of the attention itself runs in the library's CUDA kernels; there
is no fallback.  If ``libfa.so`` is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(5)
FA_BF16, FA_FP16 = 0, 1

EXPORTS = ("fa_fwd", "fa_fwd_varlen", "fa_bwd_workspace_size", "fa_bwd", "fa_bwd_preprocess", "fa_bwd_main",
           "fa_bwd_finish", "fa_bwd_noalloc", "fa_bwd_varlen_workspace_size", "fa_bwd_varlen", "fa_status_string",
           "fa_check_device_error", "fa_launch_count", "fa_selftest_timeout", "fa_decode_num_splits",
           "fa_decode_workspace_size", "fa_decode", "fa_fwd_dropout", "fa_bwd_dropout", "fa_fwd_varlen_dropout",
           "fa_bwd_varlen_dropout")

# Fixed scratch size of fa_bwd_noalloc (FA_BWD_NOALLOC_SCRATCH_BYTES in include/fa.h).
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024

_lib = None


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {fa_status_string(status)} ({status})")
        self.status = status


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfa.so once; raise loudly if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m exact_tiled_attention_31_b200.build` "
            "(there is no non-CUDA implementation to fall back to)")
    lib = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
    lib.fa_fwd.restype = i
    lib.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
    lib.fa_fwd_varlen.restype = i
    lib.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    lib.fa_bwd_workspace_size.restype = sz
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, vp, sz, vp]
    lib.fa_bwd.restype = i
    lib.fa_bwd_preprocess.argtypes = [vp, vp, vp, i, i, i, i, i, vp, sz, vp]
    lib.fa_bwd_preprocess.restype = i
    lib.fa_bwd_main.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, vp, sz, vp]
    lib.fa_bwd_main.restype = i
    lib.fa_bwd_finish.argtypes = [vp, i, i, i, i, f, i, i, vp, sz, vp]
    lib.fa_bwd_finish.restype = i
    lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, vp]
    lib.fa_bwd_noalloc.restype = i
    lib.fa_bwd_varlen_workspace_size.argtypes = [i, i, i, i, i]
    lib.fa_bwd_varlen_workspace_size.restype = sz
    lib.fa_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp, sz, vp]
    lib.fa_bwd_varlen.restype = i
    lib.fa_status_string.argtypes = [i]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_check_device_error.argtypes = [vp]
    lib.fa_check_device_error.restype = i
    lib.fa_selftest_timeout.argtypes = [vp]
    lib.fa_selftest_timeout.restype = i
    lib.fa_decode_num_splits.argtypes = [i, i, i]
    lib.fa_decode_num_splits.restype = i
    lib.fa_decode_workspace_size.argtypes = [i, i, i, i]
    lib.fa_decode_workspace_size.restype = sz
    lib.fa_decode.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, sz, vp]
    lib.fa_decode.restype = i
    u64 = ctypes.c_uint64
    lib.fa_fwd_dropout.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, i, f, u64, u64, vp]
    lib.fa_fwd_dropout.restype = i
    lib.fa_bwd_dropout.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, f, u64, u64, vp, sz, vp]
    lib.fa_bwd_dropout.restype = i
    lib.fa_fwd_varlen_dropout.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, f, u64, u64, vp]
    lib.fa_fwd_varlen_dropout.restype = i
    lib.fa_bwd_varlen_dropout.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, f, u64,
                                          u64, vp, sz, vp]
    lib.fa_bwd_varlen_dropout.restype = i
    lib.fa_launch_count.argtypes = []
    lib.fa_launch_count.restype = ctypes.c_uint64
    _lib = lib
    return lib


# ---------------------------------------------------------------- raw entry points

def fa_fwd(q, k, v, o, lse, B, H, S, D, scale, causal, dt, stream) -> int:
    return load_library().fa_fwd(q, k, v, o, lse, B, H, S, D, scale, int(causal), dt, stream)


def fa_fwd_varlen(q, k, v, o, lse, cu_seqlens, nseq, max_seqlen, total, H, D, scale, causal, dt, stream) -> int:
    return load_library().fa_fwd_varlen(q, k, v, o, lse, cu_seqlens, nseq, max_seqlen, total, H, D, scale,
                                        int(causal), dt, stream)


def fa_bwd_workspace_size(B, H, S, D) -> int:
    return load_library().fa_bwd_workspace_size(B, H, S, D)


def fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, S, D, scale, causal, dt, deterministic, workspace,
           workspace_bytes, stream) -> int:
    return load_library().fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, S, D, scale, int(causal), dt,
                                 int(deterministic), workspace, workspace_bytes, stream)


def fa_bwd_preprocess(o, dO, lse, B, H, S, D, dt, workspace, workspace_bytes, stream) -> int:
    return load_library().fa_bwd_preprocess(o, dO, lse, B, H, S, D, dt, workspace, workspace_bytes, stream)


def fa_bwd_main(q, k, v, dO, dk, dv, B, H, S, D, scale, causal, dt, deterministic, workspace, workspace_bytes,
                stream) -> int:
    return load_library().fa_bwd_main(q, k, v, dO, dk, dv, B, H, S, D, scale, int(causal), dt, int(deterministic),
                                      workspace, workspace_bytes, stream)


def fa_bwd_finish(dq, B, H, S, D, scale, dt, deterministic, workspace, workspace_bytes, stream) -> int:
    return load_library().fa_bwd_finish(dq, B, H, S, D, scale, dt, int(deterministic), workspace, workspace_bytes,
                                        stream)


def fa_bwd_noalloc(q, k, v, o, dO, lse, dq, dk, dv, B, H, S, D, scale, causal, dt, deterministic,
                   stream) -> int:
    return load_library().fa_bwd_noalloc(q, k, v, o, dO, lse, dq, dk, dv, B, H, S, D, scale, int(causal), dt,
                                         int(deterministic), stream)


def fa_bwd_varlen_workspace_size(nseq, max_seqlen, total, H, D) -> int:
    return load_library().fa_bwd_varlen_workspace_size(nseq, max_seqlen, total, H, D)


def fa_bwd_varlen(q, k, v, o, dO, lse, dq, dk, dv, cu_seqlens, nseq, max_seqlen, total, H, D, scale, causal, dt,
                  deterministic, workspace, workspace_bytes, stream) -> int:
    return load_library().fa_bwd_varlen(q, k, v, o, dO, lse, dq, dk, dv, cu_seqlens, nseq, max_seqlen, total, H, D,
                                        scale, int(causal), dt, int(deterministic), workspace, workspace_bytes,
                                        stream)


def fa_fwd_dropout(q, k, v, o, lse, B, H, S, D, scale, causal, dt, dropout_p, seed, offset, stream) -> int:
    return load_library().fa_fwd_dropout(q, k, v, o, lse, B, H, S, D, scale, int(causal), dt, dropout_p, seed, offset,
                                         stream)


def fa_bwd_dropout(q, k, v, o, dO, lse, dq, dk, dv, B, H, S, D, scale, causal, dt, deterministic, dropout_p, seed,
                   offset, workspace, workspace_bytes, stream) -> int:
    return load_library().fa_bwd_dropout(q, k, v, o, dO, lse, dq, dk, dv, B, H, S, D, scale, int(causal), dt,
                                         int(deterministic), dropout_p, seed, offset, workspace, workspace_bytes,
                                         stream)


def fa_fwd_varlen_dropout(q, k, v, o, lse, cu_seqlens, nseq, max_seqlen, total, H, D, scale, causal, dt, dropout_p,
                          seed, offset, stream) -> int:
    return load_library().fa_fwd_varlen_dropout(q, k, v, o, lse, cu_seqlens, nseq, max_seqlen, total, H, D, scale,
                                                int(causal), dt, dropout_p, seed, offset, stream)


def fa_bwd_varlen_dropout(q, k, v, o, dO, lse, dq, dk, dv, cu_seqlens, nseq, max_seqlen, total, H, D, scale, causal,
                          dt, deterministic, dropout_p, seed, offset, workspace, workspace_bytes, stream) -> int:
    return load_library().fa_bwd_varlen_dropout(q, k, v, o, dO, lse, dq, dk, dv, cu_seqlens, nseq, max_seqlen, total,
                                                H, D, scale, int(causal), dt, int(deterministic), dropout_p, seed,
                                                offset, workspace, workspace_bytes, stream)


def fa_decode_num_splits(B, Hkv, L_max) -> int:
    return load_library().fa_decode_num_splits(B, Hkv, L_max)


def fa_decode_workspace_size(B, Hq, n_splits, D) -> int:
    return load_library().fa_decode_workspace_size(B, Hq, n_splits, D)


def fa_decode(q, k_cache, v_cache, seq_lens, o, lse, B, Hq, Hkv, L_max, D, scale, dt, n_splits, workspace,
              workspace_bytes, stream) -> int:
    return load_library().fa_decode(q, k_cache, v_cache, seq_lens, o, lse, B, Hq, Hkv, L_max, D, scale, dt, n_splits,
                                    workspace, workspace_bytes, stream)


def fa_status_string(status: int) -> str:
    return load_library().fa_status_string(status).decode()


def fa_check_device_error(stream) -> int:
    return load_library().fa_check_device_error(stream)


def fa_selftest_timeout(stream) -> int:
    return load_library().fa_selftest_timeout(stream)


def fa_launch_count() -> int:
    return load_library().fa_launch_count()


# ---------------------------------------------------------------- tensor conveniences

def _dt(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return FA_BF16
    if t.dtype == torch.float16:
        return FA_FP16
    raise TypeError(f"expected bf16 or fp16 tensors, got {t.dtype}")


def _check(ts, shape):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"shape {tuple(t.shape)} != {tuple(shape)}")
        if t.dtype != ts[0].dtype:
            raise TypeError("all tensors must share one dtype")


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def forward(q, k, v, causal: bool, scale: float | None = None, out=None, lse=None, stream=None,
            dropout_p: float = 0.0, seed: int = 0, offset: int = 0):
    """O, LSE of [B, H, S, D] inputs; LSE is fp32 [B, H, S].  ``dropout_p`` > 0
    drops attention probabilities with the counter-based mask of (seed, offset)."""
    import torch
    B, H, S, D = q.shape
    _check((q, k, v), q.shape)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, S), device=q.device, dtype=torch.float32) if lse is None else lse
    if dropout_p:
        st = fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, S, D,
                            scale, causal, _dt(q), float(dropout_p), int(seed), int(offset), _stream(stream))
        if st != FA_OK:
            raise FAError(st, "fa_fwd_dropout")
        return o, lse
    st = fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, S, D, scale,
                causal, _dt(q), _stream(stream))
    if st != FA_OK:
        raise FAError(st, "fa_fwd")
    return o, lse


def forward_varlen(q, k, v, cu_seqlens, max_seqlen: int, causal: bool, scale: float | None = None,
                   stream=None, dropout_p: float = 0.0, seed: int = 0, offset: int = 0):
    """Packed [H, T, D] forward; ``cu_seqlens`` is a device int32 tensor.
    ``dropout_p`` > 0 drops P with sequence s taking the mask of batch index
    s of a dense batch (fa_fwd_varlen_dropout)."""
    import torch
    H, T, D = q.shape
    _check((q, k, v), q.shape)
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda:
        raise TypeError("cu_seqlens must be a CUDA int32 tensor")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    o = torch.empty_like(q)
    lse = torch.empty((H, T), device=q.device, dtype=torch.float32)
    if dropout_p:
        st = fa_fwd_varlen_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                   cu_seqlens.data_ptr(), cu_seqlens.numel() - 1, int(max_seqlen), T, H, D, scale,
                                   causal, _dt(q), float(dropout_p), int(seed), int(offset), _stream(stream))
        if st != FA_OK:
            raise FAError(st, "fa_fwd_varlen_dropout")
        return o, lse
    st = fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                       cu_seqlens.data_ptr(), cu_seqlens.numel() - 1, int(max_seqlen), T, H, D, scale, causal,
                       _dt(q), _stream(stream))
    if st != FA_OK:
        raise FAError(st, "fa_fwd_varlen")
    return o, lse


def backward(q, k, v, o, do, lse, causal: bool, scale: float | None = None, deterministic: bool = False,
             workspace=None, stream=None, dropout_p: float = 0.0, seed: int = 0, offset: int = 0, out=None):
    """dQ, dK, dV of [B, H, S, D] inputs given the forward's O and LSE (and
    the forward's dropout_p, seed and offset, if it dropped).  ``out`` may
    give the three output tensors to fill."""
    import torch
    B, H, S, D = q.shape
    _check((q, k, v, o, do), q.shape)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if out is None:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    else:
        dq, dk, dv = out
        _check((q, dq, dk, dv), q.shape)
    nbytes = fa_bwd_workspace_size(B, H, S, D)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(max(nbytes, 1), device=q.device, dtype=torch.uint8)
    if dropout_p:
        st = fa_bwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, S, D, scale, causal, _dt(q),
                            deterministic, float(dropout_p), int(seed), int(offset), workspace.data_ptr(),
                            workspace.numel(), _stream(stream))
        if st != FA_OK:
            raise FAError(st, "fa_bwd_dropout")
        return dq, dk, dv
    st = fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, S, D, scale, causal, _dt(q), deterministic,
                workspace.data_ptr(), workspace.numel(), _stream(stream))
    if st != FA_OK:
        raise FAError(st, "fa_bwd")
    return dq, dk, dv


def backward_varlen(q, k, v, o, do, lse, cu_seqlens, max_seqlen: int, causal: bool, scale: float | None = None,
                    deterministic: bool = False, workspace=None, stream=None, dropout_p: float = 0.0, seed: int = 0,
                    offset: int = 0):
    """dQ, dK, dV of a packed [H, T, D] batch given fa_fwd_varlen's O and LSE
    (with the forward's dropout_p, seed and offset, if it dropped)."""
    import torch
    H, T, D = q.shape
    _check((q, k, v, o, do), q.shape)
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda:
        raise TypeError("cu_seqlens must be a CUDA int32 tensor")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    nseq = cu_seqlens.numel() - 1
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nbytes = fa_bwd_varlen_workspace_size(nseq, int(max_seqlen), T, H, D)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(max(nbytes, 1), device=q.device, dtype=torch.uint8)
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(), dq.data_ptr(),
            dk.data_ptr(), dv.data_ptr(), cu_seqlens.data_ptr(), nseq, int(max_seqlen), T, H, D, scale, causal, _dt(q),
            deterministic)
    if dropout_p:
        st = fa_bwd_varlen_dropout(*args, float(dropout_p), int(seed), int(offset), workspace.data_ptr(),
                                   workspace.numel(), _stream(stream))
        if st != FA_OK:
            raise FAError(st, "fa_bwd_varlen_dropout")
        return dq, dk, dv
    st = fa_bwd_varlen(*args, workspace.data_ptr(), workspace.numel(), _stream(stream))
    if st != FA_OK:
        raise FAError(st, "fa_bwd_varlen")
    return dq, dk, dv


def backward_noalloc(q, k, v, o, do, lse, dq, dk, dv, causal: bool, scale: float | None = None,
                     deterministic: bool = False, stream=None):
    """Backward into caller-provided dq, dk, dv with no allocation at all:
    the library's fixed device scratch replaces the workspace (for callers
    that must not allocate device memory; sizes beyond the scratch raise)."""
    B, H, S, D = q.shape
    _check((q, k, v, o, do, dq, dk, dv), q.shape)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    st = fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, S, D, scale, causal, _dt(q),
                        deterministic, _stream(stream))
    if st != FA_OK:
        raise FAError(st, "fa_bwd_noalloc")
    return dq, dk, dv


def decode(q, k_cache, v_cache, seq_lens, scale: float | None = None, n_splits: int | None = None, out=None,
           lse=None, workspace=None, stream=None):
    """One decode step: q [B, Hq, D] against caches [B, Hkv, L_max, D] holding
    ``seq_lens`` (CUDA int32 [B]) valid keys each.  Returns O [B, Hq, D] and
    fp32 LSE [B, Hq].  ``n_splits`` defaults to the library's choice."""
    import torch
    B, Hq, D = q.shape
    _check((q,), q.shape)
    _check((k_cache, v_cache), k_cache.shape)
    if k_cache.dtype != q.dtype:
        raise TypeError("q and the caches must share one dtype")
    Bk, Hkv, L, Dk = k_cache.shape
    if Bk != B or Dk != D:
        raise ValueError(f"cache shape {tuple(k_cache.shape)} does not match q {tuple(q.shape)}")
    if not seq_lens.is_cuda or seq_lens.dtype != torch.int32 or tuple(seq_lens.shape) != (B,):
        raise ValueError("seq_lens must be a CUDA int32 tensor of shape [B]")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    n = fa_decode_num_splits(B, Hkv, L) if n_splits is None else int(n_splits)
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq), device=q.device, dtype=torch.float32) if lse is None else lse
    need = fa_decode_workspace_size(B, Hq, n, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=q.device, dtype=torch.uint8)
    st = fa_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seq_lens.data_ptr(), o.data_ptr(),
                   lse.data_ptr(), B, Hq, Hkv, L, D, scale, _dt(q), n, workspace.data_ptr(), workspace.numel(),
                   _stream(stream))
    if st != FA_OK:
        raise FAError(st, "fa_decode")
    return o, lse


def check_device_error(stream=None):
    """Synchronise and raise FAError if a kernel recorded an error (a wait
    that timed out, or split backward calls that disagreed on the mode)."""
    st = fa_check_device_error(_stream(stream))
    if st != FA_OK:
        raise FAError(st, "device")
