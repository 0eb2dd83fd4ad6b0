"""Python binding of libfa, exact IO-aware attention for NVIDIA B200 (sm_100a).

The C ABI (include/fa.h) is the product boundary; this module only marshals
arguments to it.  Two layers:

* ``fa_fwd``, ``fa_bwd``, ``fa_fwd_varlen``, ``fa_bwd_varlen``, ``fa_fwd_splitkv``, ``fa_fwd_kvcache``,
  their fp16 twins ``fa_*_f16``, ``fa_fwd_f32``, ``fa_bwd_f32``,
  ``fa_bwd_workspace_size``, ``fa_fwd_splitkv_workspace_size``,
  ``fa_get_device_status``, ``fa_status_string``: the C entry points under the
  same names, taking raw device pointers (ints) and sizes, returning the
  status code.
* ``attention_forward`` / ``attention_backward`` / ``attention_forward_varlen`` /
  ``attention_backward_varlen`` /
  ``attention_forward_splitkv`` / ``attention_forward_kvcache``:
  the same calls on torch CUDA tensors (torch only allocates the outputs and
  the workspace and supplies the current stream); bf16 or fp16 tensors pick
  the bf16 or fp16 entry point.

There is no fallback: if libfa.so cannot be loaded or built, importing the
tensor API raises, and every computation runs in the library's CUDA kernels.
"""
import ctypes
import math
import os

__all__ = [
    "FAError", "load_library", "library_path",
    "fa_fwd", "fa_bwd", "fa_bwd_noalloc", "fa_fwd_f32", "fa_bwd_f32", "fa_bwd_workspace_size",
    "fa_fwd_varlen", "fa_bwd_varlen", "fa_fwd_splitkv", "fa_fwd_splitkv_workspace_size", "fa_fwd_kvcache",
    "fa_fwd_kvcache_workspace_size", "fa_fwd_f16", "fa_bwd_f16", "fa_fwd_varlen_f16",
    "fa_bwd_varlen_f16", "fa_fwd_splitkv_f16", "fa_fwd_kvcache_f16", "fa_fwd_blocksparse",
    "fa_fwd_blocksparse_f16", "attention_forward_blocksparse", "fa_bwd_blocksparse",
    "fa_bwd_blocksparse_f16", "attention_backward_blocksparse",
    "fa_get_device_status", "fa_status_string", "fa_trace_enable", "fa_trace_read",
    "KERNEL_KINDS", "attention_forward", "attention_backward", "attention_forward_splitkv",
    "attention_forward_kvcache", "attention_forward_varlen", "attention_backward_varlen",
    "fa_lse_merge", "fa_lse_merge_f16", "fa_grad_accumulate", "fa_grad_accumulate_f16",
    "lse_merge", "grad_accumulate", "fa_test_withhold_next_load",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libfa.so")
_lib = None

FA_OK = 0


class FAError(RuntimeError):
    """A libfa entry point returned a non-zero status."""

    def __init__(self, name, status):
        super().__init__("%s failed: %s (%d)" % (name, fa_status_string(status), status))
        self.status = status


def library_path():
    return _LIB_PATH


def load_library():
    """Load libfa.so from the package directory, building it with nvcc if it is
    missing.  Raises if neither works: there is no other implementation."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        from . import build as _build
        _build.build()
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    sz = ctypes.c_size_t
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i, vp]
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i,
                           vp, sz, vp]
    lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i,
                                   i, vp]
    lib.fa_fwd_f32.argtypes = lib.fa_fwd.argtypes
    lib.fa_bwd_f32.argtypes = lib.fa_bwd.argtypes
    lib.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    lib.fa_bwd_workspace_size.restype = sz
    lib.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i, i, vp, sz, vp]
    lib.fa_fwd_splitkv_workspace_size.argtypes = [i, i, i, i, i, i, i, i, i, i]
    lib.fa_fwd_splitkv_workspace_size.restype = sz
    lib.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, i, i, i, vp]
    lib.fa_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i,
                                  f, i, i, i, vp, sz, vp]
    lib.fa_fwd_kvcache_workspace_size.argtypes = [i, i, i, i, i, i, i, i, i, i, i]
    lib.fa_fwd_kvcache_workspace_size.restype = sz
    lib.fa_fwd_kvcache.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i, i,
                                   i, vp, sz, vp]
    lib.fa_get_device_status.argtypes = [vp]
    lib.fa_status_string.argtypes = [i]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_trace_enable.argtypes = [i]
    lib.fa_trace_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong)]
    ll = ctypes.c_longlong
    lib.fa_fwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, ll, ll, i, i, i, i, i, i, f, i, i, i, vp]
    lib.fa_fwd_blocksparse.restype = i
    lib.fa_bwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ll, ll, i, i, i, i, i,
                                       i, f, i, i, i, vp, sz, vp]
    lib.fa_bwd_blocksparse.restype = i
    for base in ("fa_fwd", "fa_bwd", "fa_fwd_varlen", "fa_bwd_varlen", "fa_fwd_splitkv",
                 "fa_fwd_kvcache", "fa_fwd_blocksparse", "fa_bwd_blocksparse"):
        getattr(lib, base + "_f16").argtypes = getattr(lib, base).argtypes
        getattr(lib, base + "_f16").restype = i
    lib.fa_test_withhold_next_load.argtypes = []
    lib.fa_test_withhold_next_load.restype = i
    for name in ("fa_lse_merge", "fa_lse_merge_f16"):
        getattr(lib, name).argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
        getattr(lib, name).restype = i
    for name in ("fa_grad_accumulate", "fa_grad_accumulate_f16"):
        getattr(lib, name).argtypes = [vp, vp, vp, i, i, i, i, ll, i, vp]
        getattr(lib, name).restype = i
    for name in ("fa_fwd", "fa_bwd", "fa_bwd_noalloc", "fa_fwd_f32", "fa_bwd_f32", "fa_fwd_splitkv", "fa_fwd_kvcache", "fa_fwd_varlen", "fa_bwd_varlen",
                 "fa_get_device_status",
                 "fa_trace_enable", "fa_trace_read"):
        getattr(lib, name).restype = i
    _lib = lib
    return lib


# ----------------------------------------------------------- C entry points

def fa_fwd(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l, win_r, stream):
    return load_library().fa_fwd(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, scale, causal,
                                 win_l, win_r, stream)


def fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l,
           win_r, workspace, workspace_bytes, stream):
    return load_library().fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, d, scale,
                                 causal, win_l, win_r, workspace, workspace_bytes, stream)


def fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l,
                   win_r, stream):
    """fa_bwd for callers that cannot allocate device memory (no workspace
    argument; the library's fixed scratch array is used instead)."""
    return load_library().fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, d,
                                         scale, causal, win_l, win_r, stream)


def fa_fwd_splitkv(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l, win_r, n_splits,
                   workspace, workspace_bytes, stream):
    """Forward for few query rows over a long key range, split across CTAs."""
    return load_library().fa_fwd_splitkv(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, scale, causal,
                                         win_l, win_r, n_splits, workspace, workspace_bytes, stream)


def fa_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k,
                  total_q, total_k, Hq, Hkv, d, scale, causal, win_l, win_r, stream):
    """Forward over packed variable-length sequences."""
    return load_library().fa_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q,
                                        max_seqlen_k, total_q, total_k, Hq, Hkv, d, scale, causal,
                                        win_l, win_r, stream)


def fa_bwd_varlen(q, k, v, o, lse, dO, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q,
                  max_seqlen_k, total_q, total_k, Hq, Hkv, d, scale, causal, win_l, win_r,
                  workspace, workspace_bytes, stream):
    """Backward over packed variable-length sequences (deterministic)."""
    return load_library().fa_bwd_varlen(q, k, v, o, lse, dO, dq, dk, dv, cu_seqlens_q, cu_seqlens_k,
                                        B, max_seqlen_q, max_seqlen_k, total_q, total_k, Hq, Hkv, d,
                                        scale, causal, win_l, win_r, workspace, workspace_bytes,
                                        stream)


def fa_fwd_kvcache(q, k_cache, v_cache, k_new, v_new, cache_seqlens, o, lse, B, Nq, Nk, n_new, Hq,
                   Hkv, d, scale, causal, win_l, win_r, n_splits, workspace, workspace_bytes, stream):
    """fa_fwd_splitkv over a key/value cache, appending n_new keys/values in place."""
    return load_library().fa_fwd_kvcache(q, k_cache, v_cache, k_new, v_new, cache_seqlens, o, lse,
                                         B, Nq, Nk, n_new, Hq, Hkv, d, scale, causal, win_l, win_r,
                                         n_splits, workspace, workspace_bytes, stream)


def fa_fwd_kvcache_workspace_size(B, Nq, Nk, Hq, Hkv, d, causal, win_l, win_r, n_splits,
                                  with_seqlens):
    return load_library().fa_fwd_kvcache_workspace_size(B, Nq, Nk, Hq, Hkv, d, causal, win_l,
                                                        win_r, n_splits, int(bool(with_seqlens)))


def fa_fwd_splitkv_workspace_size(B, Nq, Nk, Hq, Hkv, d, causal, win_l, win_r, n_splits):
    return load_library().fa_fwd_splitkv_workspace_size(B, Nq, Nk, Hq, Hkv, d, causal, win_l,
                                                        win_r, n_splits)


def fa_fwd_f32(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l, win_r, stream):
    return load_library().fa_fwd_f32(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, scale, causal,
                                     win_l, win_r, stream)


def fa_bwd_f32(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l,
               win_r, workspace, workspace_bytes, stream):
    return load_library().fa_bwd_f32(q, k, v, o, lse, dO, dq, dk, dv, B, Nq, Nk, Hq, Hkv, d,
                                     scale, causal, win_l, win_r, workspace, workspace_bytes,
                                     stream)


def _f16_twin(name):
    def call(*args):
        return getattr(load_library(), name)(*args)
    call.__name__ = name
    call.__doc__ = "fp16 twin of %s (same arguments, fp16 tensors)." % name[:-4]
    return call


fa_fwd_f16 = _f16_twin("fa_fwd_f16")
fa_bwd_f16 = _f16_twin("fa_bwd_f16")
fa_fwd_varlen_f16 = _f16_twin("fa_fwd_varlen_f16")
fa_bwd_varlen_f16 = _f16_twin("fa_bwd_varlen_f16")
fa_fwd_splitkv_f16 = _f16_twin("fa_fwd_splitkv_f16")
fa_fwd_kvcache_f16 = _f16_twin("fa_fwd_kvcache_f16")
fa_fwd_blocksparse_f16 = _f16_twin("fa_fwd_blocksparse_f16")
fa_bwd_blocksparse_f16 = _f16_twin("fa_bwd_blocksparse_f16")


def fa_bwd_blocksparse(q, k, v, o, lse, dO, dq, dk, dv, block_mask, mask_stride_b, mask_stride_h,
                       B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l, win_r, workspace,
                       workspace_bytes, stream):
    """Gradients of fa_fwd_blocksparse with the same block mask."""
    return load_library().fa_bwd_blocksparse(q, k, v, o, lse, dO, dq, dk, dv, block_mask,
                                             mask_stride_b, mask_stride_h, B, Nq, Nk, Hq, Hkv, d,
                                             scale, causal, win_l, win_r, workspace,
                                             workspace_bytes, stream)


def fa_fwd_blocksparse(q, k, v, o, lse, block_mask, mask_stride_b, mask_stride_h, B, Nq, Nk, Hq,
                       Hkv, d, scale, causal, win_l, win_r, stream):
    """Block-sparse forward: 128 x 128 tiles that block_mask marks zero are skipped."""
    return load_library().fa_fwd_blocksparse(q, k, v, o, lse, block_mask, mask_stride_b,
                                             mask_stride_h, B, Nq, Nk, Hq, Hkv, d, scale, causal,
                                             win_l, win_r, stream)


def fa_bwd_workspace_size(B, Nq, Hq, d):
    return load_library().fa_bwd_workspace_size(B, Nq, Hq, d)


def fa_get_device_status(stream=None):
    return load_library().fa_get_device_status(stream)


def fa_status_string(status):
    return load_library().fa_status_string(int(status)).decode()


def fa_lse_merge(o_acc, lse_acc, o_part, lse_part, o_out, B, Nq, H, d, Nq_acc, row0, first, stream):
    """Fold one partial forward result (bf16 O, fp32 LSE) into rows row0 ..
    row0 + Nq - 1 of a running fp32 one."""
    return load_library().fa_lse_merge(o_acc, lse_acc, o_part, lse_part, o_out, B, Nq, H, d, Nq_acc, row0, first,
                                       stream)


def fa_lse_merge_f16(o_acc, lse_acc, o_part, lse_part, o_out, B, Nq, H, d, Nq_acc, row0, first, stream):
    return load_library().fa_lse_merge_f16(o_acc, lse_acc, o_part, lse_part, o_out, B, Nq, H, d, Nq_acc, row0,
                                           first, stream)


def fa_grad_accumulate(acc, part, out, B, rows_acc, row0, rows, row_elems, first, stream):
    """acc (fp32) = (first ? 0 : acc) + part (bf16) on rows row0 .. row0 + rows - 1;
    out (bf16) = rounded acc on the same rows."""
    return load_library().fa_grad_accumulate(acc, part, out, B, rows_acc, row0, rows, row_elems, first, stream)


def fa_test_withhold_next_load():
    """Test only: the next dense forward launch's first CTA withholds a key/value
    load, so its bounded wait runs out (see include/fa.h)."""
    return load_library().fa_test_withhold_next_load()


def fa_grad_accumulate_f16(acc, part, out, B, rows_acc, row0, rows, row_elems, first, stream):
    return load_library().fa_grad_accumulate_f16(acc, part, out, B, rows_acc, row0, rows, row_elems, first, stream)


KERNEL_KINDS = ("fwd", "bwd_prep", "bwd_dq", "bwd_dkdv", "f32", "decode", "kvcache_append",
                "bwd_call", "merge")


def fa_trace_enable(on):
    return load_library().fa_trace_enable(int(bool(on)))


def fa_trace_read():
    """Return ({kind: device ms}, {kind: launches}) accumulated since the last read."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_longlong * n)()
    _check("fa_trace_read", load_library().fa_trace_read(ms, cnt))
    return dict(zip(KERNEL_KINDS, ms)), dict(zip(KERNEL_KINDS, cnt))


# ------------------------------------------------------------ tensor layer

def _check(name, st):
    if st != FA_OK:
        raise FAError(name, st)


def _dims(q, k, v):
    import torch
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, N, H, d]")
    B, Nq, Hq, d = q.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[3] != d:
        raise ValueError("k and v must be [B, Nk, Hkv, d] with q's B and d")
    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
        if t.dtype not in (torch.bfloat16, torch.float16, torch.float32) or t.dtype != q.dtype:
            raise ValueError("tensors must all be bf16, all fp16 or all fp32")
    return B, Nq, k.shape[1], Hq, k.shape[2], d


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _window(causal, window):
    wl, wr = (-1, -1) if window is None else window
    return int(bool(causal)), int(wl), int(wr)


def attention_forward(q, k, v, scale=None, causal=False, window=(-1, -1), out=None, lse=None):
    """O, LSE = attention(q, k, v) on the current CUDA stream.

    q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d] contiguous, all bf16 (fa_fwd) or all fp32
    (fa_fwd_f32).  Returns (o like q, lse [B,Hq,Nq] fp32).  ``window`` is
    (left, right), negative = unbounded; ``causal`` aligns bottom-right.
    """
    import torch
    B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    c, wl, wr = _window(causal, window)
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    fn = {torch.bfloat16: fa_fwd, torch.float16: fa_fwd_f16}.get(q.dtype, fa_fwd_f32)
    _check(fn.__name__, fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                           B, Nq, Nk, Hq, Hkv, d, scale, c, wl, wr, _stream()))
    return o, lse


def attention_forward_splitkv(q, k, v, scale=None, causal=False, window=(-1, -1), n_splits=0,
                              out=None, lse=None, workspace=None):
    """O, LSE = attention(q, k, v) through fa_fwd_splitkv (bf16 only).

    Meant for few query rows against many keys (decoding with a KV cache):
    the keys are split across CTAs and the splits merged by their LSE.
    ``n_splits`` 0 lets the library choose.  ``workspace``: optional uint8
    CUDA tensor of at least ``fa_fwd_splitkv_workspace_size(...)`` bytes,
    allocated here if omitted and needed.
    """
    import torch
    B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
    if q.dtype not in (torch.bfloat16, torch.float16):
        raise ValueError("fa_fwd_splitkv takes bf16 or fp16 tensors")
    fn = fa_fwd_splitkv if q.dtype == torch.bfloat16 else fa_fwd_splitkv_f16
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    c, wl, wr = _window(causal, window)
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    wsb = fa_fwd_splitkv_workspace_size(B, Nq, Nk, Hq, Hkv, d, c, wl, wr, int(n_splits))
    if workspace is None:
        workspace = torch.empty(max(wsb, 16), dtype=torch.uint8, device=q.device)
    _check(fn.__name__,
           fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                          B, Nq, Nk, Hq, Hkv, d, scale, c, wl, wr, int(n_splits),
                          workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                          _stream()))
    return o, lse


BLOCK_SPARSE_TILE = 128


def _block_mask_arg(m, B, Hq, Nq, Nk):
    """(tensor, batch stride, head stride) of a block mask for the C ABI."""
    import torch
    nqb, nkb = -(-Nq // BLOCK_SPARSE_TILE), -(-Nk // BLOCK_SPARSE_TILE)
    if m.dtype == torch.bool:
        m = m.to(torch.uint8)
    if m.dtype != torch.uint8 or not m.is_cuda or m.dim() != 4:
        raise ValueError("block_mask must be a 4-D uint8 or bool CUDA tensor")
    if m.shape[2:] != (nqb, nkb) or m.shape[0] not in (1, B) or m.shape[1] not in (1, Hq):
        raise ValueError("block_mask must be [B or 1, Hq or 1, %d, %d]" % (nqb, nkb))
    if m.stride(3) != 1 or m.stride(2) != nkb:
        m = m.contiguous()
    sb = 0 if m.shape[0] == 1 else m.stride(0)
    sh = 0 if m.shape[1] == 1 else m.stride(1)
    return m, sb, sh


def attention_backward_blocksparse(q, k, v, o, lse, do, block_mask, scale=None, causal=False,
                                   window=(-1, -1), dq=None, dk=None, dv=None, workspace=None):
    """dQ, dK, dV of attention_forward_blocksparse (same block mask)."""
    import torch
    B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
    if q.dtype not in (torch.bfloat16, torch.float16):
        raise ValueError("fa_bwd_blocksparse takes bf16 or fp16 tensors")
    m, sb, sh = _block_mask_arg(block_mask, B, Hq, Nq, Nk)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    c, wl, wr = _window(causal, window)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    wsb = fa_bwd_workspace_size(B, Nq, Hq, d)
    if workspace is None:
        workspace = torch.empty(max(wsb, 16), dtype=torch.uint8, device=q.device)
    fn = fa_bwd_blocksparse if q.dtype == torch.bfloat16 else fa_bwd_blocksparse_f16
    _check(fn.__name__, fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                           do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), m.data_ptr(),
                           sb, sh, B, Nq, Nk, Hq, Hkv, d, scale, c, wl, wr, workspace.data_ptr(),
                           workspace.numel() * workspace.element_size(), _stream()))
    return dq, dk, dv


def attention_forward_blocksparse(q, k, v, block_mask, scale=None, causal=False, window=(-1, -1),
                                  out=None, lse=None):
    """O, LSE with 128 x 128 (query block, key block) tiles left out where
    block_mask is zero.  q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d] bf16 or fp16;
    block_mask: uint8 (or bool) CUDA tensor [B, Hq, ceil(Nq/128), ceil(Nk/128)]
    whose batch / head dims may be broadcast (size 1, or expanded with stride 0)."""
    import torch
    B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
    if q.dtype not in (torch.bfloat16, torch.float16):
        raise ValueError("fa_fwd_blocksparse takes bf16 or fp16 tensors")
    m, sb, sh = _block_mask_arg(block_mask, B, Hq, Nq, Nk)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    c, wl, wr = _window(causal, window)
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    fn = fa_fwd_blocksparse if q.dtype == torch.bfloat16 else fa_fwd_blocksparse_f16
    _check(fn.__name__, fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                           m.data_ptr(), sb, sh, B, Nq, Nk, Hq, Hkv, d, scale, c, wl, wr,
                           _stream()))
    return o, lse


def attention_forward_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                             scale=None, causal=False, window=(-1, -1), out=None, lse=None):
    """O, LSE for packed sequences through fa_fwd_varlen (bf16 only).

    q [total_q, Hq, d], k/v [total_k, Hkv, d] contiguous; cu_seqlens_q/k int32
    CUDA tensors of B + 1 offsets.  Returns (o like q, lse [Hq, total_q])."""
    import torch
    if q.dim() != 3 or k.dim() != 3 or v.dim() != 3 or k.shape != v.shape or k.shape[2] != q.shape[2]:
        raise ValueError("q must be [total_q, Hq, d] and k, v [total_k, Hkv, d]")
    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous() or t.dtype not in (torch.bfloat16, torch.float16) \
                or t.dtype != q.dtype:
            raise ValueError("q, k, v must be contiguous CUDA tensors, all bf16 or all fp16")
    for t in (cu_seqlens_q, cu_seqlens_k):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous() or t.dim() != 1:
            raise ValueError("cu_seqlens must be contiguous int32 CUDA vectors")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both hold B + 1 offsets")
    total_q, Hq, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    B = cu_seqlens_q.numel() - 1
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    c, wl, wr = _window(causal, window)
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device) if lse is None else lse
    fn = fa_fwd_varlen if q.dtype == torch.bfloat16 else fa_fwd_varlen_f16
    _check(fn.__name__,
           fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                         cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, int(max_seqlen_q),
                         int(max_seqlen_k), total_q, total_k, Hq, Hkv, d, scale, c, wl, wr,
                         _stream()))
    return o, lse


def attention_backward_varlen(q, k, v, o, lse, do, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                              max_seqlen_k, scale=None, causal=False, window=(-1, -1), dq=None,
                              dk=None, dv=None, workspace=None):
    """dQ, dK, dV for packed sequences through fa_bwd_varlen (bf16 only), in
    the layouts of attention_forward_varlen."""
    import torch
    total_q, Hq, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    B = cu_seqlens_q.numel() - 1
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    c, wl, wr = _window(causal, window)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    wsb = fa_bwd_workspace_size(B, int(max_seqlen_q), Hq, d)
    if workspace is None:
        workspace = torch.empty(max(wsb, 16), dtype=torch.uint8, device=q.device)
    fn = fa_bwd_varlen if q.dtype == torch.bfloat16 else fa_bwd_varlen_f16
    _check(fn.__name__,
           fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                         do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                         cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, int(max_seqlen_q),
                         int(max_seqlen_k), total_q, total_k, Hq, Hkv, d, scale, c, wl, wr,
                         workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                         _stream()))
    return dq, dk, dv


def attention_forward_kvcache(q, k_cache, v_cache, k_new=None, v_new=None, cache_seqlens=None,
                              scale=None, causal=False, window=(-1, -1), n_splits=0, out=None,
                              lse=None, workspace=None):
    """O, LSE through fa_fwd_kvcache (bf16 only): k_new / v_new [B, n_new,
    Hkv, d] are written into k_cache / v_cache [B, Nk, Hkv, d] in place at
    rows cache_seqlens[b] .. + n_new - 1, then q [B, Nq, Hq, d] attends to
    the first cache_seqlens[b] + n_new keys of each sequence.
    ``cache_seqlens``: int32 CUDA tensor [B], or None for full caches (then no
    k_new / v_new)."""
    import torch
    B, Nq, Nk, Hq, Hkv, d = _dims(q, k_cache, v_cache)
    if q.dtype not in (torch.bfloat16, torch.float16):
        raise ValueError("fa_fwd_kvcache takes bf16 or fp16 tensors")
    fn = fa_fwd_kvcache if q.dtype == torch.bfloat16 else fa_fwd_kvcache_f16
    n_new = 0
    if k_new is not None or v_new is not None:
        if k_new is None or v_new is None or k_new.shape != v_new.shape:
            raise ValueError("k_new and v_new must be given together, with equal shapes")
        if k_new.dim() != 4 or k_new.shape[0] != B or k_new.shape[2:] != k_cache.shape[2:]:
            raise ValueError("k_new must be [B, n_new, Hkv, d]")
        if not (k_new.is_contiguous() and v_new.is_contiguous()) or k_new.dtype != q.dtype:
            raise ValueError("k_new / v_new must be contiguous, of q's dtype")
        n_new = int(k_new.shape[1])
    if cache_seqlens is not None:
        if cache_seqlens.dtype != torch.int32 or not cache_seqlens.is_cuda or \
                cache_seqlens.numel() != B or not cache_seqlens.is_contiguous():
            raise ValueError("cache_seqlens must be a contiguous int32 CUDA tensor of B entries")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    c, wl, wr = _window(causal, window)
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    wsb = fa_fwd_kvcache_workspace_size(B, Nq, Nk, Hq, Hkv, d, c, wl, wr, int(n_splits),
                                        cache_seqlens is not None)
    if workspace is None:
        workspace = torch.empty(max(wsb, 16), dtype=torch.uint8, device=q.device)
    ptr = lambda t: None if t is None else t.data_ptr()
    _check(fn.__name__,
           fn(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), ptr(k_new),
                          ptr(v_new), ptr(cache_seqlens), o.data_ptr(), lse.data_ptr(), B, Nq, Nk,
                          n_new, Hq, Hkv, d, scale, c, wl, wr, int(n_splits), workspace.data_ptr(),
                          workspace.numel() * workspace.element_size(), _stream()))
    return o, lse


def attention_backward(q, k, v, o, lse, do, scale=None, causal=False, window=(-1, -1),
                       dq=None, dk=None, dv=None, workspace=None):
    """dQ, dK, dV of sum(do * o) on the current CUDA stream (deterministic).

    ``workspace``: optional uint8 CUDA tensor of at least
    ``fa_bwd_workspace_size(B, Nq, Hq, d)`` bytes; allocated here if omitted.
    """
    import torch
    B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    c, wl, wr = _window(causal, window)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    wsb = fa_bwd_workspace_size(B, Nq, Hq, d)
    if workspace is None:
        workspace = torch.empty(max(wsb, 16), dtype=torch.uint8, device=q.device)
    fn = {torch.bfloat16: fa_bwd, torch.float16: fa_bwd_f16}.get(q.dtype, fa_bwd_f32)
    _check(fn.__name__, fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                           do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Nq, Nk,
                           Hq, Hkv, d, scale, c, wl, wr, workspace.data_ptr(),
                           workspace.numel() * workspace.element_size(), _stream()))
    return dq, dk, dv


def _need(cond, what):
    if not cond:
        raise ValueError(what)


def lse_merge(o_acc, lse_acc, o_part, lse_part, first=False, out=None, row0=0):
    """Fold (o_part [B, Nq, H, d] bf16/fp16, lse_part [B, H, Nq] fp32) into
    rows row0 .. row0 + Nq - 1 of the running fp32 result (o_acc [B, Nq_acc, H,
    d], lse_acc [B, H, Nq_acc]), in place; with ``out`` given (o_acc's shape),
    also write those merged rows of O rounded to out's type.  Returns ``out``."""
    import torch
    B, Nq, H, d = o_part.shape
    Nq_acc = o_acc.shape[1]
    _need(o_acc.shape == (B, Nq_acc, H, d) and lse_acc.shape == (B, H, Nq_acc) and lse_part.shape == (B, H, Nq)
          and (out is None or out.shape == o_acc.shape), "lse_merge: mismatched shapes")
    _need(0 <= row0 <= Nq_acc - Nq, "lse_merge: rows out of range")
    _need(o_acc.dtype == torch.float32 and lse_acc.dtype == torch.float32 and lse_part.dtype == torch.float32
          and o_part.dtype in (torch.bfloat16, torch.float16) and (out is None or out.dtype == o_part.dtype),
          "lse_merge: dtypes")
    _need(all(t.is_contiguous() for t in (o_acc, lse_acc, o_part, lse_part) + ((out,) if out is not None else ())),
          "lse_merge: tensors must be contiguous")
    fn = fa_lse_merge_f16 if o_part.dtype == torch.float16 else fa_lse_merge
    _check(fn.__name__, fn(o_acc.data_ptr(), lse_acc.data_ptr(), o_part.data_ptr(), lse_part.data_ptr(),
                           out.data_ptr() if out is not None else None, B, Nq, H, d, Nq_acc, int(row0),
                           int(bool(first)), _stream()))
    return out


def grad_accumulate(acc, part=None, first=False, out=None, row0=0):
    """acc (fp32) = (first ? 0 : acc) + part (bf16/fp16), in place; with ``out``
    given (acc's shape), also write acc rounded to out's type.  Returns ``out``.
    A 1-D acc is one flat sum.  Otherwise acc is [B, rows_acc, ...] and part
    [B, rows, ...] covers acc's rows row0 .. row0 + rows - 1 (without part, every
    row from row0 on is converted)."""
    import math as _m
    import torch
    ref = part if part is not None else out
    _need(ref is not None, "grad_accumulate: part or out needed")
    _need(acc.dtype == torch.float32 and ref.dtype in (torch.bfloat16, torch.float16)
          and (part is None or out is None or out.dtype == part.dtype), "grad_accumulate: dtypes")
    _need(all(t.is_contiguous() for t in (acc, part, out) if t is not None), "grad_accumulate: tensors must be contiguous")
    _need(out is None or out.shape == acc.shape, "grad_accumulate: out must have acc's shape")
    if acc.dim() == 1:
        _need(row0 == 0 and (part is None or part.shape == acc.shape), "grad_accumulate: mismatched shapes")
        B, rows_acc, rows, row_elems = 1, 1, 1, acc.numel()
    else:
        B, rows_acc = acc.shape[0], acc.shape[1]
        row_elems = _m.prod(acc.shape[2:])
        rows = part.shape[1] if part is not None else rows_acc - row0
        _need(part is None or part.shape == (B, rows) + tuple(acc.shape[2:]), "grad_accumulate: mismatched shapes")
        _need(0 <= row0 and 1 <= rows and row0 + rows <= rows_acc, "grad_accumulate: rows out of range")
    fn = fa_grad_accumulate_f16 if ref.dtype == torch.float16 else fa_grad_accumulate
    _check(fn.__name__, fn(acc.data_ptr(), part.data_ptr() if part is not None else None,
                           out.data_ptr() if out is not None else None, B, rows_acc, int(row0), rows, row_elems,
                           int(bool(first)), _stream()))
    return out
