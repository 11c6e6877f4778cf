"""ctypes binding of the C ABI in ``include/fa.h`` (argument marshalling only).

Each function checks tensor dtypes / devices / shapes, allocates outputs with
torch on the inputs' device, passes raw device pointers and the current CUDA
stream to the library, and raises ``FAError`` on a non-zero status.  Every
step of the computation runs in the library's kernels.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa_sm100.so")

FA_OK = 0
_STATUS = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_CUDA", 4: "FA_ERR_TIMEOUT"}

_lib = None


class FAError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what} failed: {_STATUS.get(status, status)}")


def load_library(path=None):
    """Loads (once) and returns the ctypes handle of libfa_sm100.so."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m exact_io_aware_49_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, f, u64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_uint64, ctypes.c_size_t
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, f, u64, vp]
    lib.fa_fwd.restype = i
    lib.fa_fwd_ex.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, f, u64, i, vp]
    lib.fa_fwd_ex.restype = i
    lib.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    lib.fa_bwd_workspace_size.restype = sz
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, f, u64, vp, sz, vp]
    lib.fa_bwd.restype = i
    lib.fa_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, f, u64, i, vp, sz, vp]
    lib.fa_bwd_ex.restype = i
    lib.fa_fwd_qk.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, f, u64, i, vp]
    lib.fa_fwd_qk.restype = i
    lib.fa_bwd_qk_workspace_size.argtypes = [i, i, i, i, i]
    lib.fa_bwd_qk_workspace_size.restype = sz
    lib.fa_bwd_qk.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, f, u64, i, i, vp, sz, vp]
    lib.fa_bwd_qk.restype = i
    lib.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, f, u64, i, vp]
    lib.fa_fwd_varlen.restype = i
    lib.fa_bwd_varlen_workspace_size.argtypes = [i, i, i, i, i, i]
    lib.fa_bwd_varlen_workspace_size.restype = sz
    lib.fa_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, f, u64, i,
                                  i, vp, sz, vp]
    lib.fa_bwd_varlen.restype = i
    lib.fa_bwd_prepare.argtypes = [vp, vp, vp, i, i, i, i, vp, sz, vp]
    lib.fa_bwd_prepare.restype = i
    lib.fa_bwd_tiles.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, f, u64, vp, sz, vp]
    lib.fa_bwd_tiles.restype = i
    lib.fa_bwd_finish.argtypes = [vp, i, i, i, i, f, vp, sz, vp]
    lib.fa_bwd_finish.restype = i
    lib.fa_fwd_bwd_host_workspace_size.argtypes = [i, i, i, i, i]
    lib.fa_fwd_bwd_host_workspace_size.restype = sz
    lib.fa_fwd_bwd_host.argtypes = [vp] * 9 + [i, i, i, i, i, f, f, u64, i, i, vp, sz, ctypes.POINTER(vp)]
    lib.fa_fwd_bwd_host.restype = i
    lib.fa_decode_num_splits.argtypes = [i, i, i, i, i]
    lib.fa_decode_num_splits.restype = i
    lib.fa_decode_workspace_size.argtypes = [i, i, i, i, i]
    lib.fa_decode_workspace_size.restype = sz
    lib.fa_decode_paged.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, i, f, i, i, vp, sz, vp]
    lib.fa_decode_paged.restype = i
    lib.fa_dropout_mask.argtypes = [vp, i, i, i, f, u64, vp]
    lib.fa_dropout_mask.restype = i
    lib.fa_selftest_wait_timeout.argtypes = [ctypes.c_uint32, vp]
    lib.fa_selftest_wait_timeout.restype = i
    lib.fa_last_device_error.argtypes = []
    lib.fa_last_device_error.restype = i
    lib.fa_status_string.argtypes = [i]
    lib.fa_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _stream(t):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _guard(t):
    """Makes ``t``'s device the current one for the call: the library sets kernel
    attributes and launches on the current device."""
    return torch.cuda.device(t.device)


def _on_device(device):
    """The same for an explicit device (calls whose tensors are on the host)."""
    return torch.cuda.device(device)


# element types of the ``_ex`` entry points (fa_dtype)
FA_DTYPE = {torch.bfloat16: 0, torch.float16: 1}


def _check_device(name, t, device):
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device} like q")


def _check_bhnd(name, t, shape=None, dtype=None, device=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    _check_device(name, t, device)
    if t.dtype not in FA_DTYPE:
        raise ValueError(f"{name} must be bf16 or fp16")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} is {t.dtype}, expected {dtype} like q")
    if t.dim() != 4 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous [B, H, N, d] tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _check_f32(name, t, shape, device):
    if not t.is_cuda or t.dtype != torch.float32 or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous fp32 CUDA tensor of shape {tuple(shape)}")
    _check_device(name, t, device)


def _ws_args(workspace, device):
    """(pointer, bytes) of a caller's workspace (None -> (None, 0))."""
    if workspace is None:
        return None, 0
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    _check_device("workspace", workspace, device)
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


def _raise(st, what):
    if st != FA_OK:
        raise FAError(st, what)


def fa_fwd(q, k, v, causal, scale=None, p_drop=0.0, seed=0, out=None, lse=None):
    """(O, LSE) of exact attention on one CUDA device: q [B, H, Nq, d], k and v
    [B, H, Nk, d], all bf16 or all fp16.  Square bf16 problems go to fa_fwd,
    square fp16 ones to fa_fwd_ex, Nq != Nk to fa_fwd_qk."""
    lib = load_library()
    _check_bhnd("q", q)
    B, H, Nq, d = q.shape
    dev = q.device
    _check_bhnd("k", k, None, q.dtype, dev)
    Nk = k.shape[2]
    if (k.shape[0], k.shape[1], k.shape[3]) != (B, H, d):
        raise ValueError(f"k has shape {tuple(k.shape)}, expected [{B}, {H}, Nk, {d}]")
    _check_bhnd("v", v, k.shape, q.dtype, dev)
    scale = d ** -0.5 if scale is None else scale
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, Nq), device=dev, dtype=torch.float32) if lse is None else lse
    _check_bhnd("out", out, q.shape, q.dtype, dev)
    _check_f32("lse", lse, (B, H, Nq), dev)
    ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr())
    tail = (d, int(bool(causal)), float(scale), float(p_drop), int(seed) & (2**64 - 1))
    with _guard(q):
        if Nq != Nk:
            _raise(lib.fa_fwd_qk(*ptrs, B, H, Nq, Nk, *tail, FA_DTYPE[q.dtype], _stream(q)), "fa_fwd_qk")
        elif q.dtype == torch.bfloat16:
            _raise(lib.fa_fwd(*ptrs, B, H, Nq, *tail, _stream(q)), "fa_fwd")
        else:
            _raise(lib.fa_fwd_ex(*ptrs, B, H, Nq, *tail, FA_DTYPE[q.dtype], _stream(q)), "fa_fwd_ex")
    return out, lse


def fa_bwd_workspace_size(B, H, N, d):
    return int(load_library().fa_bwd_workspace_size(B, H, N, d))


def fa_bwd(q, k, v, o, do, lse, causal, scale=None, p_drop=0.0, seed=0, workspace=None, dq=None, dk=None,
           dv=None, deterministic=False):
    """(dQ, dK, dV) of sum(dO * O) by recomputation; same arguments as the matching fa_fwd call
    (square bf16 tensors go to fa_bwd, square fp16 ones to fa_bwd_ex, Nq != Nk or
    ``deterministic`` -- a fixed order of the dQ additions -- to fa_bwd_qk)."""
    lib = load_library()
    _check_bhnd("q", q)
    B, H, Nq, d = q.shape
    dev = q.device
    for name, t in (("o", o), ("do", do)):
        _check_bhnd(name, t, q.shape, q.dtype, dev)
    _check_bhnd("k", k, None, q.dtype, dev)
    Nk = k.shape[2]
    if (k.shape[0], k.shape[1], k.shape[3]) != (B, H, d):
        raise ValueError(f"k has shape {tuple(k.shape)}, expected [{B}, {H}, Nk, {d}]")
    _check_bhnd("v", v, k.shape, q.dtype, dev)
    scale = d ** -0.5 if scale is None else scale
    _check_f32("lse", lse, (B, H, Nq), dev)
    det = int(bool(deterministic))
    ws_bytes = int(lib.fa_bwd_qk_workspace_size(B, H, Nq, d, det))
    if workspace is None:
        workspace = torch.empty(ws_bytes, device=dev, dtype=torch.uint8)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(k) if dv is None else dv
    _check_bhnd("dq", dq, q.shape, q.dtype, dev)
    _check_bhnd("dk", dk, k.shape, q.dtype, dev)
    _check_bhnd("dv", dv, k.shape, q.dtype, dev)
    ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(), dq.data_ptr(),
            dk.data_ptr(), dv.data_ptr())
    tail = (d, int(bool(causal)), float(scale), float(p_drop), int(seed) & (2**64 - 1))
    with _guard(q):
        ws = (*_ws_args(workspace, dev), _stream(q))
        if Nq != Nk or det:
            _raise(lib.fa_bwd_qk(*ptrs, B, H, Nq, Nk, *tail, FA_DTYPE[q.dtype], det, *ws), "fa_bwd_qk")
        elif q.dtype == torch.bfloat16:
            _raise(lib.fa_bwd(*ptrs, B, H, Nq, *tail, *ws), "fa_bwd")
        else:
            _raise(lib.fa_bwd_ex(*ptrs, B, H, Nq, *tail, FA_DTYPE[q.dtype], *ws), "fa_bwd_ex")
    return dq, dk, dv


def _check_packed(name, t, dtype=None, rows=None, H=None, d=None, device=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    _check_device(name, t, device)
    if t.dtype not in FA_DTYPE or (dtype is not None and t.dtype != dtype):
        raise ValueError(f"{name} must be bf16 or fp16, the type of q")
    if t.dim() != 3 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous [total, H, d] tensor")
    if (rows is not None and t.shape[0] != rows) or (H is not None and t.shape[1] != H) or \
            (d is not None and t.shape[2] != d):
        raise ValueError(f"{name} has shape {tuple(t.shape)}")


def _check_cu(name, cu, B, device=None):
    if not cu.is_cuda or cu.dtype != torch.int32 or cu.dim() != 1 or cu.numel() != B + 1 or not cu.is_contiguous():
        raise ValueError(f"{name} must be a contiguous int32 CUDA tensor of B + 1 offsets")
    _check_device(name, cu, device)


def fa_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal, scale=None, p_drop=0.0,
                  seed=0, out=None, lse=None):
    """(O [total_q, H, d], LSE [H, total_q]) of B packed sequences: q [total_q, H, d],
    k, v [total_k, H, d], int32 offsets cu_seqlens_q / cu_seqlens_k [B + 1] on the device."""
    lib = load_library()
    _check_packed("q", q)
    total_q, H, d = q.shape
    dev = q.device
    _check_packed("k", k, q.dtype, None, H, d, dev)
    total_k = k.shape[0]
    _check_packed("v", v, q.dtype, total_k, H, d, dev)
    B = cu_seqlens_q.numel() - 1
    _check_cu("cu_seqlens_q", cu_seqlens_q, B, dev)
    _check_cu("cu_seqlens_k", cu_seqlens_k, B, dev)
    scale = d ** -0.5 if scale is None else scale
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((H, total_q), device=dev, dtype=torch.float32) if lse is None else lse
    _check_packed("out", out, q.dtype, total_q, H, d, dev)
    _check_f32("lse", lse, (H, total_q), dev)
    with _guard(q):
        _raise(lib.fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                 cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, H, total_q, total_k,
                                 int(max_seqlen_q), int(max_seqlen_k), d, int(bool(causal)), float(scale),
                                 float(p_drop), int(seed) & (2**64 - 1), FA_DTYPE[q.dtype], _stream(q)),
               "fa_fwd_varlen")
    return out, lse


def fa_bwd_varlen(q, k, v, o, do, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal, scale=None,
                  p_drop=0.0, seed=0, workspace=None, dq=None, dk=None, dv=None, deterministic=False):
    """(dQ, dK, dV) of the matching fa_fwd_varlen call, in the same packed layouts
    (``deterministic``: fixed order of the dQ additions)."""
    lib = load_library()
    _check_packed("q", q)
    total_q, H, d = q.shape
    dev = q.device
    _check_packed("k", k, q.dtype, None, H, d, dev)
    total_k = k.shape[0]
    _check_packed("v", v, q.dtype, total_k, H, d, dev)
    _check_packed("o", o, q.dtype, total_q, H, d, dev)
    _check_packed("do", do, q.dtype, total_q, H, d, dev)
    B = cu_seqlens_q.numel() - 1
    _check_cu("cu_seqlens_q", cu_seqlens_q, B, dev)
    _check_cu("cu_seqlens_k", cu_seqlens_k, B, dev)
    _check_f32("lse", lse, (H, total_q), dev)
    scale = d ** -0.5 if scale is None else scale
    det = int(bool(deterministic))
    ws_bytes = int(lib.fa_bwd_varlen_workspace_size(B, H, total_q, int(max_seqlen_q), d, det))
    if workspace is None:
        workspace = torch.empty(ws_bytes, device=dev, dtype=torch.uint8)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(k) if dv is None else dv
    _check_packed("dq", dq, q.dtype, total_q, H, d, dev)
    _check_packed("dk", dk, q.dtype, total_k, H, d, dev)
    _check_packed("dv", dv, q.dtype, total_k, H, d, dev)
    with _guard(q):
        _raise(lib.fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                 lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), cu_seqlens_q.data_ptr(),
                                 cu_seqlens_k.data_ptr(), B, H, total_q, total_k, int(max_seqlen_q),
                                 int(max_seqlen_k), d, int(bool(causal)), float(scale), float(p_drop),
                                 int(seed) & (2**64 - 1), FA_DTYPE[q.dtype], det, *_ws_args(workspace, dev),
                                 _stream(q)), "fa_bwd_varlen")
    return dq, dk, dv


def fa_bwd_stages(q, k, v, o, do, lse, causal, scale=None, p_drop=0.0, seed=0, workspace=None, dq=None, dk=None,
                  dv=None, between=None):
    """fa_bwd as its three ABI stages (prepare, tiles, finish).  ``between(i)``, if
    given, is called before stage i and after the last (i = 0..3) -- e.g. to
    record CUDA events around the tiles kernel."""
    lib = load_library()
    _check_bhnd("q", q, None, torch.bfloat16)
    dev = q.device
    for name, t in (("k", k), ("v", v), ("o", o), ("do", do)):
        _check_bhnd(name, t, q.shape, torch.bfloat16, dev)
    B, H, N, d = q.shape
    _check_f32("lse", lse, (B, H, N), dev)
    scale = d ** -0.5 if scale is None else scale
    if workspace is None:
        workspace = torch.empty(fa_bwd_workspace_size(B, H, N, d), device=dev, dtype=torch.uint8)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _check_bhnd(name, t, q.shape, torch.bfloat16, dev)
    seed = int(seed) & (2**64 - 1)
    ws, wsb = _ws_args(workspace, dev)
    with _guard(q):
        st = _stream(q)
        if between:
            between(0)
        _raise(lib.fa_bwd_prepare(o.data_ptr(), do.data_ptr(), lse.data_ptr(), B, H, N, d, ws, wsb, st),
               "fa_bwd_prepare")
        if between:
            between(1)
        _raise(lib.fa_bwd_tiles(q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(), dk.data_ptr(),
                                dv.data_ptr(), B, H, N, d, int(bool(causal)), float(scale), float(p_drop), seed, ws,
                                wsb, st), "fa_bwd_tiles")
        if between:
            between(2)
        _raise(lib.fa_bwd_finish(dq.data_ptr(), B, H, N, d, float(scale), ws, wsb, st), "fa_bwd_finish")
        if between:
            between(3)
    return dq, dk, dv


def fa_decode_paged(q, k_cache, v_cache, block_table, seqlens_k, max_seqlen_k, causal, scale=None, num_splits=0,
                    out=None, lse=None, workspace=None):
    """(O [B, H, Nq, d], LSE [B, H, Nq]) of q over a paged key/value cache:
    k_cache, v_cache [num_pages, page_size, H_kv, d]; block_table int32 [B, max_pages];
    seqlens_k int32 [B] (all on the device); num_splits = 0 chooses the split count."""
    lib = load_library()
    _check_bhnd("q", q)
    B, H, Nq, d = q.shape
    dev = q.device
    for name, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        if not t.is_cuda or t.dtype != q.dtype or t.dim() != 4 or not t.is_contiguous() or t.shape[3] != d:
            raise ValueError(f"{name} must be a contiguous [num_pages, page_size, H_kv, d] tensor of q's type")
        _check_device(name, t, dev)
    if tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("v_cache must have k_cache's shape")
    num_pages, page, H_kv, _ = k_cache.shape
    for name, t, shape in (("block_table", block_table, (B, block_table.shape[-1])), ("seqlens_k", seqlens_k, (B,))):
        if not t.is_cuda or t.dtype != torch.int32 or tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous int32 CUDA tensor of shape {shape}")
        _check_device(name, t, dev)
    scale = d ** -0.5 if scale is None else scale
    splits = int(num_splits) or int(lib.fa_decode_num_splits(B, H_kv, H, Nq, int(max_seqlen_k)))
    ws_bytes = int(lib.fa_decode_workspace_size(B, H, Nq, d, splits)) if splits > 0 else 0
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, device=dev, dtype=torch.uint8)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, Nq), device=dev, dtype=torch.float32) if lse is None else lse
    _check_bhnd("out", out, q.shape, q.dtype, dev)
    _check_f32("lse", lse, (B, H, Nq), dev)
    with _guard(q):
        _raise(lib.fa_decode_paged(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_table.data_ptr(),
                                   seqlens_k.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H, H_kv, Nq, d, num_pages,
                                   page, block_table.shape[1], int(max_seqlen_k), int(bool(causal)), float(scale),
                                   splits, FA_DTYPE[q.dtype], *_ws_args(workspace, dev), _stream(q)),
               "fa_decode_paged")
    return out, lse


def fa_dropout_mask(B, H, N, p_drop, seed, device="cuda"):
    """uint8 [B, H, N, N] keep mask generated by the device Philox (test/inspection export)."""
    lib = load_library()
    mask = torch.empty((B, H, N, N), device=device, dtype=torch.uint8)
    with _guard(mask):
        st = lib.fa_dropout_mask(mask.data_ptr(), B, H, N, float(p_drop), int(seed) & (2**64 - 1), _stream(mask))
    _raise(st, "fa_dropout_mask")
    return mask


def fa_selftest_wait_timeout(limit_us=1000, device="cuda"):
    """Runs the bounded-wait self-test kernel (a wait that can only time out)."""
    lib = load_library()
    dev = torch.device(device)
    with torch.cuda.device(dev):
        st = torch.cuda.current_stream(dev)
        _raise(lib.fa_selftest_wait_timeout(int(limit_us), ctypes.c_void_p(st.cuda_stream)),
               "fa_selftest_wait_timeout")


def fa_last_device_error():
    """Synchronises; returns the status of bounded device waits since the last call."""
    return int(load_library().fa_last_device_error())


def _check_host(name, t, shape, dtype):
    if t.is_cuda or t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} CPU tensor of shape {tuple(shape)}")


def fa_fwd_bwd_host_workspace_size(B, H, N, d, groups):
    return int(load_library().fa_fwd_bwd_host_workspace_size(B, H, N, d, groups))


def fa_fwd_bwd_host(q, k, v, do, causal, scale=None, p_drop=0.0, seed=0, groups=8, device=None, workspace=None,
                    streams=None, out=None, lse=None, dq=None, dk=None, dv=None):
    """Forward and backward of attention on HOST tensors (the C ABI's
    fa_fwd_bwd_host): q, k, v, do are CPU [B, H, N, d] bf16 or fp16 tensors
    (pin them for the copies to overlap the kernels); returns CPU
    (O, LSE, dQ, dK, dV).  The work is cut into ``groups`` groups of (b, h)
    units copied in, computed and copied out on three CUDA streams of
    ``device`` (``streams``: three torch.cuda.Stream, created if omitted).
    Returns once the work is enqueued; synchronise ``streams[2]`` (or the
    device) before reading the outputs."""
    lib = load_library()
    if q.dtype not in FA_DTYPE or q.dim() != 4:
        raise ValueError("q must be a [B, H, N, d] bf16 or fp16 tensor")
    B, H, N, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("do", do)):
        _check_host(name, t, q.shape, q.dtype)
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    scale = d ** -0.5 if scale is None else scale
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, N), dtype=torch.float32) if lse is None else lse
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    for name, t in (("out", out), ("dq", dq), ("dk", dk), ("dv", dv)):
        _check_host(name, t, q.shape, q.dtype)
    _check_host("lse", lse, (B, H, N), torch.float32)
    ws_bytes = fa_fwd_bwd_host_workspace_size(B, H, N, d, groups)
    if workspace is None:
        workspace = torch.empty(ws_bytes, device=device, dtype=torch.uint8)
    if streams is None:
        streams = [torch.cuda.Stream(device) for _ in range(3)]
    if len(streams) != 3:
        raise ValueError("streams must hold three CUDA streams")
    handles = (ctypes.c_void_p * 3)(*[ctypes.c_void_p(st.cuda_stream) for st in streams])
    ws, wsb = _ws_args(workspace, device)
    if wsb < ws_bytes:
        raise ValueError(f"workspace holds {wsb} bytes, fa_fwd_bwd_host needs {ws_bytes}")
    with _on_device(device):
        _raise(lib.fa_fwd_bwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(), out.data_ptr(),
                                   lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, N, d,
                                   int(bool(causal)), float(scale), float(p_drop), int(seed) & (2**64 - 1),
                                   FA_DTYPE[q.dtype], int(groups), ws, wsb, handles), "fa_fwd_bwd_host")
    return out, lse, dq, dk, dv
