"""Dynamic bifocal RoPE attention (Jet-Long) on B200 -- Python binding.

Thin ctypes layer over ``libjetlong.so`` (C ABI declared in include/jetlong.h):
it checks tensor dtypes/devices/shapes, passes raw device pointers, sizes and
the current CUDA stream, and turns a non-OK status into an exception.  Every
step of the computation runs in the library's sm_100a kernels; there is no
fallback.  If the shared library is missing, the first call raises.

PyTorch is used only for device memory and streams.
"""
import ctypes
import os

import torch

__all__ = [
    "NO_BIFOCAL", "DEVICE_POS", "ROTATE_KEYS_ONCE", "DEBUG_SKIP_ARRIVE", "JetLongError", "group_size",
    "bifocal_prefill", "prefill_rotated_keys_bytes",
    "prefill_workspace_size", "decode_workspace_size", "bifocal_decode",
    "bifocal_prefill_3pass", "prefill_3pass_workspace_size",
    "bifocal_decode_batched", "decode_batched_workspace_size",
    "bifocal_prefill_chunk", "prefill_chunk_workspace_size",
    "bifocal_decode_noalloc", "bifocal_decode_paged",
    "check_device_status", "finalize", "library_path", "load",
]

NO_BIFOCAL = 1 << 0  # JL_FLAG_NO_BIFOCAL
DEVICE_POS = 1 << 1  # JL_FLAG_DEVICE_POS (set by the bindings when pos is a CUDA tensor)
ROTATE_KEYS_ONCE = 1 << 2  # JL_FLAG_ROTATE_KEYS_ONCE (prefill: rotated keys in a workspace)
DEBUG_SKIP_ARRIVE = 1 << 31  # JL_FLAG_DEBUG_SKIP_ARRIVE (tests of the bounded waits only)

_BF16, _F32 = 0, 1
_STATUS = {0: "JL_OK", 1: "JL_ERR_INVALID_ARG", 2: "JL_ERR_UNSUPPORTED",
           3: "JL_ERR_CUDA", 4: "JL_ERR_TIMEOUT"}

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None


class JetLongError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


def library_path() -> str:
    return os.environ.get("JETLONG_LIB", os.path.join(_HERE, "libjetlong.so"))


def load():
    """Load libjetlong.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(
            f"libjetlong.so not found at {path}; build it with "
            "`python -m long_context_attention_bifocal_b200.build` (there is no fallback)")
    L = ctypes.CDLL(path)
    p, i, d, u, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_uint,
                      ctypes.c_size_t)
    L.jl_group_size.restype = ctypes.c_longlong
    L.jl_group_size.argtypes = [ctypes.c_longlong, ctypes.c_longlong]
    L.jl_bifocal_prefill.restype = i
    L.jl_bifocal_prefill.argtypes = [p, p, p, p, p, i, i, i, i, i, i, i, d, p]
    L.jl_bifocal_prefill_workspace_size.restype = sz
    L.jl_bifocal_prefill_workspace_size.argtypes = [i, i, i, i, i]
    L.jl_bifocal_prefill_rotated_keys_bytes.restype = sz
    L.jl_bifocal_prefill_rotated_keys_bytes.argtypes = [i, i, i, i]
    L.jl_bifocal_prefill_ex.restype = i
    L.jl_bifocal_prefill_ex.argtypes = [p, p, p, p, p, i, i, i, i, i, i, i, d, i,
                                        ctypes.c_float, u, p, sz, p]
    L.jl_bifocal_prefill_3pass_workspace_size.restype = sz
    L.jl_bifocal_prefill_3pass_workspace_size.argtypes = [i, i, i, i, i]
    L.jl_bifocal_prefill_3pass.restype = i
    L.jl_bifocal_prefill_3pass.argtypes = [p, p, p, p, p, i, i, i, i, i, i, i, d, u, p, sz, p]
    L.jl_bifocal_prefill_chunk_workspace_size.restype = sz
    L.jl_bifocal_prefill_chunk_workspace_size.argtypes = [i, i, i, i, i]
    L.jl_bifocal_prefill_chunk.restype = i
    L.jl_bifocal_prefill_chunk.argtypes = [p, p, p, i, i, p, p, i, i, i, i, i, i, i, d, u, p,
                                           sz, p]
    L.jl_bifocal_decode_workspace_size.restype = sz
    L.jl_bifocal_decode_workspace_size.argtypes = [i, i, i, i, i]
    L.jl_bifocal_decode.restype = i
    L.jl_bifocal_decode.argtypes = [p, p, p, i, i, p, p, p, sz, i, i, i, i, i, i, d,
                                    u, p]
    L.jl_bifocal_decode_batched_workspace_size.restype = sz
    L.jl_bifocal_decode_batched_workspace_size.argtypes = [i, i, i, i]
    L.jl_bifocal_decode_batched.restype = i
    L.jl_bifocal_decode_batched.argtypes = [p, p, p, p, i, p, p, p, sz, i, i, i, i, i, i, d,
                                            u, p]
    L.jl_bifocal_decode_paged.restype = i
    L.jl_bifocal_decode_paged.argtypes = [p, p, p, i, i, p, i, p, p, p, p, sz, i, i, i, i, i, i,
                                          d, u, p]
    L.jl_bifocal_decode_noalloc.restype = i
    L.jl_bifocal_decode_noalloc.argtypes = [p, p, p, i, i, p, p, i, i, i, i, i, i, d, u, p]
    L.jl_last_error.restype = ctypes.c_char_p
    L.jl_last_error.argtypes = []
    L.jl_check_device_status.restype = i
    L.jl_check_device_status.argtypes = [p]
    L.jl_finalize.restype = None
    L.jl_finalize.argtypes = []
    _lib = L
    return L


def _check(status):
    if status != 0:
        msg = load().jl_last_error().decode(errors="replace")
        raise JetLongError(status, msg)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _positions(pos, B, flags):
    """Host positions (a sequence of ints) as a C array, or a CUDA int32 tensor
    of B positions passed by pointer with JL_FLAG_DEVICE_POS."""
    if isinstance(pos, torch.Tensor) and pos.is_cuda:
        _need(pos, "pos", torch.int32, (B,))
        return ctypes.c_void_p(pos.data_ptr()), int(flags) | DEVICE_POS
    pos = [int(x) for x in pos]
    if len(pos) != B:
        raise ValueError(f"pos must hold {B} positions, got {len(pos)}")
    return (ctypes.c_int * B)(*pos), int(flags)


def group_size(L: int, w_pretrained: int) -> int:
    """G = max(1, ceil(L / w_pretrained)) as the library computes it."""
    return int(load().jl_group_size(L, w_pretrained))


def prefill_workspace_size(B, L, Hkv, D, dtype=torch.bfloat16) -> int:
    code = _BF16 if dtype == torch.bfloat16 else _F32
    return int(load().jl_bifocal_prefill_workspace_size(B, L, Hkv, D, code))


def prefill_rotated_keys_bytes(B, L, Hkv, D) -> int:
    """Workspace bytes of a bf16 prefill with ROTATE_KEYS_ONCE."""
    return int(load().jl_bifocal_prefill_rotated_keys_bytes(B, L, Hkv, D))


def bifocal_prefill(q, k, v, *, w_local, w_pretrained, rope_base, out=None, lse=None,
                    softmax_scale=0.0, flags=0, workspace=None, stream=None):
    """Bifocal causal prefill.  q [B,L,Hq,D], k/v [B,L,Hkv,D] (pre-RoPE),
    bf16 (D=128) or fp32 (D in {64,128}).  Returns (out [B,L,Hq,D], lse [B,Hq,L] fp32).
    With flags | ROTATE_KEYS_ONCE (bf16) the keys are rotated once into a
    workspace (allocated here when none is given) instead of in the kernel.
    """
    dtype = q.dtype
    if dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("q must be bfloat16 or float32")
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    _need(q, "q", dtype)
    _need(k, "k", dtype, (B, L, Hkv, D))
    _need(v, "v", dtype, (B, L, Hkv, D))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    _need(out, "out", dtype, (B, L, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq, L))
    ws_ptr, ws_bytes = None, 0
    if workspace is None and (flags & ROTATE_KEYS_ONCE) and dtype == torch.bfloat16:
        workspace = torch.empty(prefill_rotated_keys_bytes(B, L, Hkv, D), dtype=torch.uint8,
                                device=q.device)
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8)
        ws_ptr, ws_bytes = _ptr(workspace), workspace.numel()
    with torch.cuda.device(q.device):
        _check(load().jl_bifocal_prefill_ex(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, L, Hq, Hkv, D,
            int(w_local), int(w_pretrained), float(rope_base),
            _BF16 if dtype == torch.bfloat16 else _F32, float(softmax_scale),
            int(flags), ws_ptr, ws_bytes, _stream(stream)))
    return out, lse


def prefill_3pass_workspace_size(B, L, Hq, Hkv, D) -> int:
    return int(load().jl_bifocal_prefill_3pass_workspace_size(B, L, Hq, Hkv, D))


def bifocal_prefill_3pass(q, k, v, *, w_local, w_pretrained, rope_base, out=None, lse=None,
                          flags=0, workspace=None, stream=None):
    """The pages' unfused three-call formulation (A + B - C, LSE merge) of the
    same bifocal prefill; bf16, D=128.  Returns (out, lse) like bifocal_prefill."""
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    _need(q, "q", torch.bfloat16)
    _need(k, "k", torch.bfloat16, (B, L, Hkv, D))
    _need(v, "v", torch.bfloat16, (B, L, Hkv, D))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.bfloat16, (B, L, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq, L))
    if workspace is None:
        workspace = torch.empty(prefill_3pass_workspace_size(B, L, Hq, Hkv, D),
                                dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace", torch.uint8)
    with torch.cuda.device(q.device):
        _check(load().jl_bifocal_prefill_3pass(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, L, Hq, Hkv, D, int(w_local),
            int(w_pretrained), float(rope_base), int(flags), _ptr(workspace),
            workspace.numel(), _stream(stream)))
    return out, lse


def prefill_chunk_workspace_size(B, q_offset, Lq, Hkv, D) -> int:
    return int(load().jl_bifocal_prefill_chunk_workspace_size(B, q_offset, Lq, Hkv, D))


def bifocal_prefill_chunk(q, k_cache, v_cache, q_offset, *, w_local, w_pretrained, rope_base,
                          out=None, lse=None, flags=0, workspace=None, stream=None):
    """Chunked prefill: q [B,Lq,Hq,D] pre-RoPE bf16 at positions q_offset + r
    against caches [B,cap,Hkv,D] bf16 (keys rotated at original positions,
    slots 0..q_offset+Lq-1 valid).  Returns (out [B,Lq,Hq,D], lse [B,Hq,Lq])."""
    B, Lq, Hq, D = q.shape
    cap, Hkv = k_cache.shape[1], k_cache.shape[2]
    _need(q, "q", torch.bfloat16)
    _need(k_cache, "k_cache", torch.bfloat16, (B, cap, Hkv, D))
    _need(v_cache, "v_cache", torch.bfloat16, (B, cap, Hkv, D))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.bfloat16, (B, Lq, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq, Lq))
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8)
        ws_ptr, ws_bytes = _ptr(workspace), workspace.numel()
    with torch.cuda.device(q.device):
        _check(load().jl_bifocal_prefill_chunk(
            _ptr(q), _ptr(k_cache), _ptr(v_cache), int(q_offset), cap, _ptr(out), _ptr(lse), B,
            Lq, Hq, Hkv, D, int(w_local), int(w_pretrained), float(rope_base), int(flags),
            ws_ptr, ws_bytes, _stream(stream)))
    return out, lse


def decode_workspace_size(B, Hq, Hkv, D, pos) -> int:
    return int(load().jl_bifocal_decode_workspace_size(B, Hq, Hkv, D, pos))


def bifocal_decode(q_new, k_cache, v_cache, pos, *, w_local, w_pretrained, rope_base,
                   out=None, lse=None, workspace=None, flags=0, stream=None):
    """Single-token decode at position `pos`.  q_new [B,Hq,D] pre-RoPE bf16;
    caches [B,cap,Hkv,D] bf16 with keys rotated at their original positions.
    Returns (out [B,Hq,D] bf16, lse [B,Hq] fp32)."""
    B, Hq, D = q_new.shape
    cap, Hkv = k_cache.shape[1], k_cache.shape[2]
    _need(q_new, "q_new", torch.bfloat16)
    _need(k_cache, "k_cache", torch.bfloat16, (B, cap, Hkv, D))
    _need(v_cache, "v_cache", torch.bfloat16, (B, cap, Hkv, D))
    if out is None:
        out = torch.empty_like(q_new)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q_new.device)
    _need(out, "out", torch.bfloat16, (B, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq))
    if workspace is None:
        n = decode_workspace_size(B, Hq, Hkv, D, pos)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q_new.device)
    _need(workspace, "workspace", torch.uint8)
    with torch.cuda.device(q_new.device):
        _check(load().jl_bifocal_decode(
            _ptr(q_new), _ptr(k_cache), _ptr(v_cache), int(pos), cap, _ptr(out),
            _ptr(lse), _ptr(workspace), workspace.numel(), B, Hq, Hkv, D, int(w_local),
            int(w_pretrained), float(rope_base), int(flags), _stream(stream)))
    return out, lse


def decode_batched_workspace_size(B, Hq, Hkv, D) -> int:
    return int(load().jl_bifocal_decode_batched_workspace_size(B, Hq, Hkv, D))


def bifocal_decode_batched(q_new, k_cache, v_cache, pos, *, w_local, w_pretrained, rope_base,
                           out=None, lse=None, workspace=None, flags=0, stream=None):
    """Single-token decode of B sequences, sequence b at position pos[b]: a
    sequence of B ints, or a CUDA int32 tensor of B positions (the plan is then
    made on the GPU and the call can be captured in a CUDA graph).  q_new
    [B,Hq,D] pre-RoPE bf16; caches [B,cap,Hkv,D] bf16 with keys rotated at
    their original positions.  Returns (out, lse)."""
    B, Hq, D = q_new.shape
    cap, Hkv = k_cache.shape[1], k_cache.shape[2]
    _need(q_new, "q_new", torch.bfloat16)
    _need(k_cache, "k_cache", torch.bfloat16, (B, cap, Hkv, D))
    _need(v_cache, "v_cache", torch.bfloat16, (B, cap, Hkv, D))
    pos_arr, flags = _positions(pos, B, flags)
    if out is None:
        out = torch.empty_like(q_new)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q_new.device)
    _need(out, "out", torch.bfloat16, (B, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq))
    if workspace is None:
        workspace = torch.empty(max(decode_batched_workspace_size(B, Hq, Hkv, D), 16),
                                dtype=torch.uint8, device=q_new.device)
    _need(workspace, "workspace", torch.uint8)
    with torch.cuda.device(q_new.device):
        _check(load().jl_bifocal_decode_batched(
            _ptr(q_new), _ptr(k_cache), _ptr(v_cache), pos_arr, cap, _ptr(out), _ptr(lse),
            _ptr(workspace), workspace.numel(), B, Hq, Hkv, D, int(w_local), int(w_pretrained),
            float(rope_base), int(flags), _stream(stream)))
    return out, lse


def bifocal_decode_paged(q_new, k_pages, v_pages, block_table, pos, *, w_local, w_pretrained,
                         rope_base, out=None, lse=None, workspace=None, flags=0, stream=None):
    """Single-token decode of B sequences over a paged cache.  k_pages, v_pages
    [num_pages, page_size, Hkv, D] bf16 (keys rotated at their original
    positions); block_table [B, max_pages_per_seq] int32 on the device (page of
    keys page_size*i .. page_size*(i+1)-1 of sequence b); pos a sequence of B
    ints or a CUDA int32 tensor (as in bifocal_decode_batched).  Returns
    (out, lse)."""
    B, Hq, D = q_new.shape
    num_pages, page_size, Hkv = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    _need(q_new, "q_new", torch.bfloat16)
    _need(k_pages, "k_pages", torch.bfloat16, (num_pages, page_size, Hkv, D))
    _need(v_pages, "v_pages", torch.bfloat16, (num_pages, page_size, Hkv, D))
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError(f"block_table must be [B={B}, max_pages_per_seq]")
    _need(block_table, "block_table", torch.int32)
    pos_arr, flags = _positions(pos, B, flags)
    if out is None:
        out = torch.empty_like(q_new)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q_new.device)
    _need(out, "out", torch.bfloat16, (B, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq))
    if workspace is None:
        workspace = torch.empty(max(decode_batched_workspace_size(B, Hq, Hkv, D), 16),
                                dtype=torch.uint8, device=q_new.device)
    _need(workspace, "workspace", torch.uint8)
    with torch.cuda.device(q_new.device):
        _check(load().jl_bifocal_decode_paged(
            _ptr(q_new), _ptr(k_pages), _ptr(v_pages), num_pages, page_size, _ptr(block_table),
            block_table.shape[1], pos_arr, _ptr(out), _ptr(lse), _ptr(workspace),
            workspace.numel(), B, Hq, Hkv, D, int(w_local), int(w_pretrained), float(rope_base),
            int(flags), _stream(stream)))
    return out, lse


def bifocal_decode_noalloc(q_new, k_cache, v_cache, pos, *, w_local, w_pretrained,
                           rope_base, out=None, lse=None, flags=0, stream=None):
    """bifocal_decode without a workspace, for callers that cannot allocate
    device memory: the library uses a fixed 4 MiB array of its own for the split
    partials and allocates nothing (include/jetlong.h states the limits).  Passing
    out/lse avoids the only allocations this wrapper would make."""
    B, Hq, D = q_new.shape
    cap, Hkv = k_cache.shape[1], k_cache.shape[2]
    _need(q_new, "q_new", torch.bfloat16)
    _need(k_cache, "k_cache", torch.bfloat16, (B, cap, Hkv, D))
    _need(v_cache, "v_cache", torch.bfloat16, (B, cap, Hkv, D))
    if out is None:
        out = torch.empty_like(q_new)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q_new.device)
    _need(out, "out", torch.bfloat16, (B, Hq, D))
    _need(lse, "lse", torch.float32, (B, Hq))
    with torch.cuda.device(q_new.device):
        _check(load().jl_bifocal_decode_noalloc(
            _ptr(q_new), _ptr(k_cache), _ptr(v_cache), int(pos), cap, _ptr(out), _ptr(lse),
            B, Hq, Hkv, D, int(w_local), int(w_pretrained), float(rope_base), int(flags),
            _stream(stream)))
    return out, lse


def check_device_status(stream=None):
    """Synchronise `stream`; raise JetLongError if a kernel abandoned a bounded wait."""
    _check(load().jl_check_device_status(_stream(stream)))


def finalize():
    load().jl_finalize()
