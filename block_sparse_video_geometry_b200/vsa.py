"""ctypes binding of libvsa (C ABI in include/vsa.h).

Argument marshalling only: every step of the computation runs in the CUDA
library. torch tensors are used as device buffers and torch streams as CUDA
streams. The library is loaded on first use; if it is missing the call raises,
there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvsa.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE_TOO_SMALL, ERR_CUDA, ERR_TIMEOUT, ERR_NOT_UPLOADED = range(7)
SEG_TEXT, SEG_REF_IMAGE, SEG_REF_AUDIO, SEG_OTHER_COND, SEG_VIDEO = range(5)
SELECT_TOPK, SELECT_ADAPTIVE = 0, 1
SINK_EXACT_KV, SINK_EXACT_KV_AND_ROWS, SINK_OFF = 0, 1, 2
COARSE_MEAN, COARSE_REWEIGHT = 0, 1
OUT_F32, OUT_BF16 = 0, 1
TILE, HEAD_DIM = 64, 128
MAX_EXTRA_TOKENS = 64


class VSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = "%s: %s (status %d)" % (where, status_string(status), status)
        if status == ERR_CUDA:
            msg += ": " + lib().vsa_last_error_detail().decode()
        super().__init__(msg)


class Segment(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("grid_t", ctypes.c_int32), ("grid_h", ctypes.c_int32),
                ("grid_w", ctypes.c_int32), ("start", ctypes.c_int64), ("length", ctypes.c_int64)]


class Params(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("keep", ctypes.c_float), ("tau", ctypes.c_float),
                ("sink", ctypes.c_int32), ("scale", ctypes.c_float), ("coarse", ctypes.c_int32),
                ("extra_tokens", ctypes.c_int32)]


class LayoutInfo(ctypes.Structure):
    _fields_ = [("seq_len", ctypes.c_int64), ("n_cond_tiles", ctypes.c_int32),
                ("n_video_tiles", ctypes.c_int32), ("n_tiles", ctypes.c_int32),
                ("grid_t", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
                ("video_start", ctypes.c_int64), ("device_bytes", ctypes.c_size_t)]


_lib = None
_P = ctypes.c_void_p
_I32, _I64, _SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t

_SIGNATURES = {
    "vsa_layout_build": (_I32, [ctypes.POINTER(Segment), _I32, _I64, _P, _SZ, _P, ctypes.POINTER(_P)]),
    "vsa_layout_upload": (_I32, [_P, _P, _SZ, _P]),
    "vsa_layout_query": (_I32, [_P, ctypes.POINTER(LayoutInfo)]),
    "vsa_layout_copy_tables": (_I32, [_P, _P, _P, _P, _P]),
    "vsa_layout_free": (None, [_P]),
    "vsa_select_kmax": (_I32, [_P, ctypes.POINTER(Params), ctypes.POINTER(_I32)]),
    "vsa_coarse_select_workspace_size": (_I32, [_P, _I32, _I32, ctypes.POINTER(Params), ctypes.POINTER(_SZ)]),
    "vsa_coarse_select": (_I32, [_P, ctypes.POINTER(Params), _I32, _I32, _P, _P, _P, _I64, _I64, _I64,
                                 _P, _P, _P, _P, _SZ, _P]),
    "vsa_coarse_select_noalloc": (_I32, [_P, ctypes.POINTER(Params), _I32, _I32, _P, _P, _P, _I64, _I64, _I64,
                                         _P, _P, _P, _P]),
    "vsa_coarse_select_workspace_init": (_I32, [_P, _P]),
    "vsa_coarse_select_status": (_I32, [_P, _P]),
    "vsa_coarse_select_failed_calls": (_I32, [_P, _P, ctypes.POINTER(ctypes.c_uint32)]),
    "vsa_coarse_select_noalloc_status": (_I32, [_P]),
    "vsa_debug_inject_select_wait_timeout": (_I32, [ctypes.c_uint64]),
    "vsa_sparse_attn_workspace_size": (_I32, [_P, _I32, _I32, ctypes.POINTER(Params), ctypes.POINTER(_SZ)]),
    "vsa_sparse_attn_fwd": (_I32, [_P, ctypes.POINTER(Params), _I32, _I32, _P, _P, _P, _I64, _I64, _I64,
                                   _P, _I64, _I64, _I64, _I64, _P, _P, _I32, _P, _P, _P, _P, _I32, _I64, _I64,
                                   _I64, _P, _SZ, _P]),
    "vsa_extra_tokens_workspace_size": (_I32, [_P, _I32, _I32, ctypes.POINTER(Params), ctypes.POINTER(_SZ)]),
    "vsa_extra_tokens_select": (_I32, [_P, ctypes.POINTER(Params), _I32, _I32, _P, _P, _I64, _I64, _I64,
                                       _P, _P, _I32, _P, _P, _P, _SZ, _P]),
    "vsa_extra_tokens_status": (_I32, [_P, _P]),
    "vsa_sparse_attn_bwd_workspace_size": (_I32, [_P, _I32, _I32, ctypes.POINTER(Params), ctypes.POINTER(_SZ)]),
    "vsa_sparse_attn_bwd": (_I32, [_P, ctypes.POINTER(Params), _I32, _I32, _P, _P, _P, _I64, _I64, _I64,
                                   _P, _I64, _I64, _I64, _I64, _P, _P, _I32, _P, _P, _I64, _I64, _I64,
                                   _P, _P, _P, _I64, _I64, _I64, _P, _I64, _I64, _I64, _I64, _P, _SZ, _P]),
    "vsa_sparse_attn_bwd_status": (_I32, [_P, _P]),
    "vsa_sparse_attn_status": (_I32, [_P, _P]),
    "vsa_sparse_attn_workspace_init": (_I32, [_P, _P]),
    "vsa_sparse_attn_failed_calls": (_I32, [_P, _P, ctypes.POINTER(ctypes.c_uint32)]),
    "vsa_debug_inject_wait_timeout": (_I32, [ctypes.c_uint64]),
    "vsa_status_string": (ctypes.c_char_p, [_I32]),
    "vsa_version": (_I32, []),
    "vsa_last_error_detail": (ctypes.c_char_p, []),
}


def lib() -> ctypes.CDLL:
    """Loads libvsa.so (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libvsa.so is missing: build it with "
                               "`python -m block_sparse_video_geometry_b200.build_ext`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().vsa_status_string(status).decode()


def version() -> int:
    return lib().vsa_version()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise VSAError(status, where)


def make_params(mode: int = SELECT_TOPK, keep: float = 0.1, tau: float = 1.0,
                sink: int = SINK_EXACT_KV, scale: float = 0.0, coarse: int = 0, extra_tokens: int = 0) -> Params:
    return Params(mode, keep, tau, sink, scale, coarse, extra_tokens)


def _stream_handle(stream) -> int:
    if stream is None:
        return 0
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream        # torch.cuda.Stream


class Layout:
    """Owned vsa_layout handle. `segments` is a list of (kind, start, length,
    (t, h, w) or None) in sequence order."""

    def __init__(self, segments, seq_len: int):
        arr = (Segment * len(segments))()
        for i, (kind, start, length, grid) in enumerate(segments):
            t, h, w = grid if grid is not None else (0, 0, 0)
            arr[i] = Segment(kind, t, h, w, start, length)
        handle = _P()
        _check(lib().vsa_layout_build(arr, len(segments), seq_len, None, 0, None, ctypes.byref(handle)),
               "vsa_layout_build")
        self._h = handle
        self.info = LayoutInfo()
        _check(lib().vsa_layout_query(self._h, ctypes.byref(self.info)), "vsa_layout_query")
        self._dev = None

    @property
    def handle(self):
        return self._h

    def __del__(self):
        h = getattr(self, "_h", None)
        if h and _lib is not None:
            _lib.vsa_layout_free(h)
            self._h = None

    def tables(self):
        """Host copies: perm [n_tiles, 64], inv [S], tile_count [n_tiles], tile_kind [n_tiles]."""
        i = self.info
        perm = np.empty(i.n_tiles * TILE, dtype=np.int32)
        inv = np.empty(i.seq_len, dtype=np.int32)
        cnt = np.empty(i.n_tiles, dtype=np.int32)
        kind = np.empty(i.n_tiles, dtype=np.int32)
        _check(lib().vsa_layout_copy_tables(self._h, perm.ctypes.data, inv.ctypes.data, cnt.ctypes.data,
                                            kind.ctypes.data), "vsa_layout_copy_tables")
        return perm.reshape(-1, TILE), inv, cnt, kind

    def upload(self, dev_buf, stream=None) -> None:
        """Uploads the device tables into `dev_buf` (a torch uint8 CUDA tensor
        of at least info.device_bytes bytes, kept alive by this object)."""
        _check(lib().vsa_layout_upload(self._h, dev_buf.data_ptr(), dev_buf.numel() * dev_buf.element_size(),
                                       _stream_handle(stream)), "vsa_layout_upload")
        self._dev = dev_buf

    def kmax(self, params: Params) -> int:
        k = _I32()
        _check(lib().vsa_select_kmax(self._h, ctypes.byref(params), ctypes.byref(k)), "vsa_select_kmax")
        return k.value

    def coarse_select_workspace_size(self, B: int, H: int, params: Params) -> int:
        n = _SZ()
        _check(lib().vsa_coarse_select_workspace_size(self._h, B, H, ctypes.byref(params), ctypes.byref(n)),
               "vsa_coarse_select_workspace_size")
        return n.value

    def extra_tokens_workspace_size(self, B: int, H: int, params: Params) -> int:
        n = _SZ()
        _check(lib().vsa_extra_tokens_workspace_size(self._h, B, H, ctypes.byref(params), ctypes.byref(n)),
               "vsa_extra_tokens_workspace_size")
        return n.value

    def sparse_attn_bwd_workspace_size(self, B: int, H: int, params: Params) -> int:
        n = _SZ()
        _check(lib().vsa_sparse_attn_bwd_workspace_size(self._h, B, H, ctypes.byref(params), ctypes.byref(n)),
               "vsa_sparse_attn_bwd_workspace_size")
        return n.value

    def sparse_attn_workspace_size(self, B: int, H: int, params: Params) -> int:
        n = _SZ()
        _check(lib().vsa_sparse_attn_workspace_size(self._h, B, H, ctypes.byref(params), ctypes.byref(n)),
               "vsa_sparse_attn_workspace_size")
        return n.value


def _qkv_strides(q, k, v):
    if not (q.stride() == k.stride() == v.stride()):
        raise ValueError("q, k and v must share strides")
    if q.dim() != 4 or q.shape[-1] != HEAD_DIM or q.stride(-1) != 1:
        raise ValueError("q, k, v must be [B, S, H, 128] with a contiguous head dim")
    return q.stride(0), q.stride(1), q.stride(2)


def coarse_select(layout: Layout, params: Params, q, k, v, idx, cnt, o_coarse, workspace, stream=None) -> None:
    """vsa_coarse_select on torch tensors (bf16 q/k/v [B, S, H, 128])."""
    B, S, H, _ = q.shape
    sb, ss, sh = _qkv_strides(q, k, v)
    _check(lib().vsa_coarse_select(layout.handle, ctypes.byref(params), B, H, q.data_ptr(), k.data_ptr(),
                                   v.data_ptr(), sb, ss, sh, idx.data_ptr(), cnt.data_ptr(),
                                   o_coarse.data_ptr(), workspace.data_ptr(),
                                   workspace.numel() * workspace.element_size(), _stream_handle(stream)),
           "vsa_coarse_select")


def coarse_select_noalloc(layout: Layout, params: Params, q, k, v, idx, cnt, o_coarse, stream=None) -> None:
    """vsa_coarse_select_noalloc: the selection call for callers that cannot
    provide scratch memory (the library's built-in 32 MiB buffer is used)."""
    B, S, H, _ = q.shape
    sb, ss, sh = _qkv_strides(q, k, v)
    _check(lib().vsa_coarse_select_noalloc(layout.handle, ctypes.byref(params), B, H, q.data_ptr(), k.data_ptr(),
                                           v.data_ptr(), sb, ss, sh, idx.data_ptr(), cnt.data_ptr(),
                                           o_coarse.data_ptr(), _stream_handle(stream)),
           "vsa_coarse_select_noalloc")


def coarse_select_workspace_init(workspace, stream=None) -> None:
    """Zeroes the selection workspace header (and its count of failed calls)."""
    _check(lib().vsa_coarse_select_workspace_init(workspace.data_ptr(), _stream_handle(stream)),
           "vsa_coarse_select_workspace_init")


def coarse_select_status(workspace, stream=None) -> int:
    """Synchronises the stream and returns the selection call's status word (OK or ERR_TIMEOUT)."""
    return lib().vsa_coarse_select_status(workspace.data_ptr(), _stream_handle(stream))


def coarse_select_failed_calls(workspace, stream=None) -> int:
    """Synchronises the stream; selection calls that recorded an error since the header was zeroed."""
    n = ctypes.c_uint32()
    _check(lib().vsa_coarse_select_failed_calls(workspace.data_ptr(), _stream_handle(stream), ctypes.byref(n)),
           "vsa_coarse_select_failed_calls")
    return n.value


def coarse_select_noalloc_status(stream=None) -> int:
    """coarse_select_status of the built-in buffer of coarse_select_noalloc (current device)."""
    return lib().vsa_coarse_select_noalloc_status(_stream_handle(stream))


def extra_tokens_select(layout: Layout, params: Params, q, k, idx, cnt, kmax: int, extra_idx, extra_cnt,
                        workspace, stream=None) -> None:
    """vsa_extra_tokens_select: extra_idx int32 [B, H, n_tiles, E], extra_cnt int32 [B, H, n_tiles] out."""
    B, S, H, _ = q.shape
    sb, ss, sh = _qkv_strides(q, k, k)
    _check(lib().vsa_extra_tokens_select(layout.handle, ctypes.byref(params), B, H, q.data_ptr(), k.data_ptr(),
                                         sb, ss, sh, idx.data_ptr(), cnt.data_ptr(), kmax, extra_idx.data_ptr(),
                                         extra_cnt.data_ptr(), workspace.data_ptr(),
                                         workspace.numel() * workspace.element_size(), _stream_handle(stream)),
           "vsa_extra_tokens_select")


def extra_tokens_status(workspace, stream=None) -> int:
    """Synchronises the stream; the status word of the extra-token selection (OK or ERR_TIMEOUT)."""
    return lib().vsa_extra_tokens_status(workspace.data_ptr(), _stream_handle(stream))


def sparse_attn_fwd(layout: Layout, params: Params, q, k, v, g, idx, cnt, kmax: int, o_coarse, out,
                    workspace, stream=None, extra_idx=None, extra_cnt=None) -> None:
    """vsa_sparse_attn_fwd on torch tensors; out is float32 or bfloat16 [B, S, H, 128];
    g is bf16 [B, S, H] (one gate per token and head) or [B, S, H, 128] (one per channel);
    extra_idx / extra_cnt from extra_tokens_select when params.extra_tokens > 0."""
    import torch
    B, S, H, _ = q.shape
    if g.dim() == 3:
        g_sd = 0
    elif g.dim() == 4 and g.shape[3] == HEAD_DIM:
        g_sd = g.stride(3)
    else:
        raise ValueError("g must be [B, S, H] or [B, S, H, 128]")
    sb, ss, sh = _qkv_strides(q, k, v)
    if out.dtype == torch.float32:
        od = OUT_F32
    elif out.dtype == torch.bfloat16:
        od = OUT_BF16
    else:
        raise ValueError("out must be float32 or bfloat16")
    _check(lib().vsa_sparse_attn_fwd(layout.handle, ctypes.byref(params), B, H, q.data_ptr(), k.data_ptr(),
                                     v.data_ptr(), sb, ss, sh, g.data_ptr(), g.stride(0), g.stride(1),
                                     g.stride(2), g_sd, idx.data_ptr(), cnt.data_ptr(), kmax, o_coarse.data_ptr(),
                                     None if extra_idx is None else extra_idx.data_ptr(),
                                     None if extra_cnt is None else extra_cnt.data_ptr(),
                                     out.data_ptr(), od, out.stride(0), out.stride(1), out.stride(2),
                                     workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                     _stream_handle(stream)), "vsa_sparse_attn_fwd")


def sparse_attn_bwd(layout: Layout, params: Params, q, k, v, g, idx, cnt, kmax: int, o_coarse, dout,
                    dq, dk, dv, dg, workspace, stream=None) -> None:
    """vsa_sparse_attn_bwd on torch tensors: dout bf16 [B, S, H, 128]; dq, dk, dv
    float32 [B, S, H, 128] and dg float32 shaped like g (outputs)."""
    B, S, H, _ = q.shape
    sb, ss, sh = _qkv_strides(q, k, v)
    if dout.dim() != 4 or dout.stride(-1) != 1:
        raise ValueError("dout must be [B, S, H, 128] with a contiguous head dim")
    if not (dq.stride() == dk.stride() == dv.stride()):
        raise ValueError("dq, dk and dv must share strides")
    g_sd = g.stride(3) if g.dim() == 4 else 0
    dg_sd = dg.stride(3) if dg.dim() == 4 else 0
    _check(lib().vsa_sparse_attn_bwd(layout.handle, ctypes.byref(params), B, H, q.data_ptr(), k.data_ptr(),
                                     v.data_ptr(), sb, ss, sh, g.data_ptr(), g.stride(0), g.stride(1), g.stride(2),
                                     g_sd, idx.data_ptr(), cnt.data_ptr(), kmax, o_coarse.data_ptr(),
                                     dout.data_ptr(), dout.stride(0), dout.stride(1), dout.stride(2),
                                     dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), dq.stride(0), dq.stride(1),
                                     dq.stride(2), dg.data_ptr(), dg.stride(0), dg.stride(1), dg.stride(2), dg_sd,
                                     workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                     _stream_handle(stream)), "vsa_sparse_attn_bwd")


def sparse_attn_bwd_status(workspace, stream=None) -> int:
    """Synchronises the stream; the backward pass's status (OK or ERR_TIMEOUT)."""
    return lib().vsa_sparse_attn_bwd_status(workspace.data_ptr(), _stream_handle(stream))


def sparse_attn_status(workspace, stream=None) -> int:
    """Synchronises the stream and returns the kernel's status word (OK or ERR_TIMEOUT)."""
    return lib().vsa_sparse_attn_status(workspace.data_ptr(), _stream_handle(stream))


def sparse_attn_workspace_init(workspace, stream=None) -> None:
    """Zeroes the attention workspace header (and its count of failed calls)."""
    _check(lib().vsa_sparse_attn_workspace_init(workspace.data_ptr(), _stream_handle(stream)),
           "vsa_sparse_attn_workspace_init")


def sparse_attn_failed_calls(workspace, stream=None) -> int:
    """Synchronises the stream; number of calls that recorded an error since the header was zeroed."""
    n = ctypes.c_uint32()
    _check(lib().vsa_sparse_attn_failed_calls(workspace.data_ptr(), _stream_handle(stream), ctypes.byref(n)),
           "vsa_sparse_attn_failed_calls")
    return n.value


def debug_inject_wait_timeout(timeout_ns):
    """Test hook: while timeout_ns > 0, each sparse_attn_fwd runs into a bounded
    wait that nothing completes and reports ERR_TIMEOUT (see vsa.h); 0 disarms."""
    lib().vsa_debug_inject_wait_timeout(int(timeout_ns))


def debug_inject_select_wait_timeout(timeout_ns):
    """Test hook: while timeout_ns > 0, each coarse_select (mean coarse branch)
    runs into a bounded wait that nothing completes and reports ERR_TIMEOUT
    through coarse_select_status; 0 disarms."""
    lib().vsa_debug_inject_select_wait_timeout(int(timeout_ns))


class Forward:
    """Holds the buffers of one shape and runs the two calls of the forward
    pass (caller-owned torch buffers; no allocation inside the calls)."""

    def __init__(self, layout: Layout, params: Params, B: int, H: int, device="cuda",
                 out_dtype=None, stream=None):
        import torch
        self.layout, self.params, self.B, self.H = layout, params, B, H
        info = layout.info
        if layout._dev is None:
            buf = torch.empty(info.device_bytes, dtype=torch.uint8, device=device)
            layout.upload(buf, stream)
        self.kmax = layout.kmax(params)
        self.idx = torch.empty((B, H, info.n_tiles, self.kmax), dtype=torch.int32, device=device)
        self.cnt = torch.empty((B, H, info.n_tiles), dtype=torch.int32, device=device)
        self.o_coarse = torch.empty((B, H, info.n_tiles, HEAD_DIM), dtype=torch.float32, device=device)
        self.ws_select = torch.empty(layout.coarse_select_workspace_size(B, H, params), dtype=torch.uint8,
                                     device=device)
        self.ws_attn = torch.empty(layout.sparse_attn_workspace_size(B, H, params), dtype=torch.uint8,
                                   device=device)
        sparse_attn_workspace_init(self.ws_attn, stream)
        coarse_select_workspace_init(self.ws_select, stream)
        self.out_dtype = out_dtype or torch.float32
        self.stream = stream
        self.extra_idx = self.extra_cnt = self.ws_extra = None
        if params.extra_tokens > 0:
            self.extra_idx = torch.empty((B, H, info.n_tiles, params.extra_tokens), dtype=torch.int32, device=device)
            self.extra_cnt = torch.empty((B, H, info.n_tiles), dtype=torch.int32, device=device)
            self.ws_extra = torch.empty(layout.extra_tokens_workspace_size(B, H, params), dtype=torch.uint8,
                                        device=device)

    def __call__(self, q, k, v, g, out=None):
        import torch
        if out is None:
            out = torch.empty(q.shape, dtype=self.out_dtype, device=q.device)
        coarse_select(self.layout, self.params, q, k, v, self.idx, self.cnt, self.o_coarse, self.ws_select,
                      self.stream)
        if self.params.extra_tokens > 0:
            extra_tokens_select(self.layout, self.params, q, k, self.idx, self.cnt, self.kmax, self.extra_idx,
                                self.extra_cnt, self.ws_extra, self.stream)
        sparse_attn_fwd(self.layout, self.params, q, k, v, g, self.idx, self.cnt, self.kmax, self.o_coarse,
                        out, self.ws_attn, self.stream, self.extra_idx, self.extra_cnt)
        return out

    def pooled(self):
        """Pooled means [3, B, H, n_tiles, 128] left in the selection workspace (from byte 256)."""
        import torch
        n = 3 * self.B * self.H * self.layout.info.n_tiles * HEAD_DIM
        return self.ws_select[256: 256 + 4 * n].view(torch.float32).view(3, self.B, self.H, self.layout.info.n_tiles,
                                                                HEAD_DIM)
