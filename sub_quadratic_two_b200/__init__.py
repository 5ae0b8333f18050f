"""SQuad-Attention on NVIDIA B200: Python binding of the C-ABI library libsquad.

The operator is the two-pass O(n sqrt n) attention of "SQuad: Sub-Quadratic
Attention Distillation for Efficient Video Generation" (gist.science technical
summary, Methodology section 1): softmax attention inside each tT x tH x tW
window of a T x H x W token grid, then softmax attention across windows among
tokens with the same in-window position, with the first pass's output as
values (attention_multi composes more passes over nested tiles). All
arithmetic runs in the CUDA kernels of libsquad.so; this module
only checks and marshals arguments (PyTorch supplies device memory and
streams). There is no CPU fallback: without the built library every call
raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

__all__ = [
    "SquadError", "attention", "squad_attn_fwd", "squad_attn_bwd", "workspace_size",
    "poll_device_error", "library_path", "load_library", "SQUAD_F32", "SQUAD_BF16", "squad_attn_fwd_pass",
    "plan_info", "make_desc", "attention_multi", "squad_attn_multi_fwd", "squad_attn_multi_bwd",
    "multi_fwd_workspace_size", "attention_host",
    "tmap_cache_stats",
]

SQUAD_F32 = 0
SQUAD_BF16 = 1
_STATUS = {0: "SQUAD_OK", 1: "SQUAD_ERR_INVALID_ARG", 2: "SQUAD_ERR_SHAPE", 3: "SQUAD_ERR_ALIGN",
           4: "SQUAD_ERR_UNSUPPORTED", 5: "SQUAD_ERR_CUDA", 6: "SQUAD_ERR_TIMEOUT", 7: "SQUAD_ERR_WORKSPACE",
           8: "SQUAD_ERR_INDEX"}

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None


class SquadError(RuntimeError):
    def __init__(self, status: int, where: str, cuda_error: int = 0):
        self.status = status
        msg = f"{where}: {_STATUS.get(status, status)}"
        if status == 5:
            msg += f" (CUDA error {cuda_error})"
        super().__init__(msg)


class SquadDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("heads", ctypes.c_int), ("d", ctypes.c_int),
                ("T", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("tT", ctypes.c_int), ("tH", ctypes.c_int), ("tW", ctypes.c_int),
                ("dtype", ctypes.c_int), ("scale", ctypes.c_float)]


def library_path() -> str:
    return os.path.join(_HERE, "libsquad.so")


def load_library():
    """Load libsquad.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m sub_quadratic_two_b200.build`")
        lib = ctypes.CDLL(path)
        vp, sz, fp = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p
        dp = ctypes.POINTER(SquadDesc)
        lib.squad_attn_workspace_size.argtypes = [dp, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]
        lib.squad_attn_fwd.argtypes = [dp, vp, vp, vp, vp, vp, fp, fp, vp, sz, vp]
        lib.squad_attn_bwd.argtypes = [dp, vp, vp, vp, vp, vp, fp, fp, vp, vp, vp, vp, vp, sz, vp]
        lib.squad_attn_fwd_pass.argtypes = [dp, ctypes.c_int, vp, vp, vp, vp, fp, vp]
        lib.squad_attn_fwd_host_workspace_size.argtypes = [dp, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]
        lib.squad_attn_fwd_host.argtypes = [dp, vp, vp, vp, vp, ctypes.c_int, vp, sz, vp, vp, vp]
        lib.squad_plan_info.argtypes = [dp, ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
        ip = ctypes.POINTER(ctypes.c_int)
        lib.squad_attn_multi_fwd_workspace_size.argtypes = [dp, ctypes.c_int, ip, ctypes.c_int,
                                                            ctypes.POINTER(ctypes.c_size_t)]
        lib.squad_attn_multi_fwd.argtypes = [dp, ctypes.c_int, ip, vp, vp, vp, vp, vp, fp, vp, sz, vp]
        lib.squad_attn_multi_bwd_workspace_size.argtypes = [dp, ctypes.c_int, ip, ctypes.POINTER(ctypes.c_size_t)]
        lib.squad_attn_multi_bwd.argtypes = [dp, ctypes.c_int, ip, vp, vp, vp, vp, vp, fp, vp, vp, vp, vp, vp,
                                             sz, vp]
        lib.squad_poll_device_error.argtypes = [vp]
        ull = ctypes.POINTER(ctypes.c_ulonglong)
        lib.squad_tmap_cache_stats.argtypes = [ull, ull]
        lib.squad_strerror.argtypes = [ctypes.c_int]
        lib.squad_strerror.restype = ctypes.c_char_p
        for f in ("squad_attn_workspace_size", "squad_attn_fwd", "squad_attn_bwd", "squad_poll_device_error",
                  "squad_attn_fwd_pass", "squad_plan_info", "squad_attn_fwd_host_workspace_size",
                  "squad_attn_fwd_host", "squad_attn_multi_fwd_workspace_size", "squad_attn_multi_fwd",
                  "squad_attn_multi_bwd_workspace_size", "squad_attn_multi_bwd",
                  "squad_last_cuda_error", "squad_version", "squad_tmap_cache_stats"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise SquadError(status, where, load_library().squad_last_cuda_error())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SQUAD_F32
    if t.dtype == torch.bfloat16:
        return SQUAD_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def make_desc(q: torch.Tensor, grid: Sequence[int], tile: Sequence[int], scale: Optional[float]) -> SquadDesc:
    if q.dim() != 4:
        raise ValueError("expected [B, heads, n, d] tensors")
    B, h, n, d = q.shape
    T, H, W = (int(x) for x in grid)
    tT, tH, tW = (int(x) for x in tile)
    if T * H * W != n:
        raise ValueError(f"n={n} but T*H*W={T * H * W}")
    return SquadDesc(B, h, d, T, H, W, tT, tH, tW, _dtype_code(q), float(scale or 0.0))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream: Optional[torch.cuda.Stream], dev: torch.device):
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    return ctypes.c_void_p(s.cuda_stream)


def _check_inputs(*ts: torch.Tensor):
    ref = ts[0]
    for t in ts:
        if not t.is_cuda:
            raise ValueError("libsquad needs CUDA tensors (there is no CPU path)")
        if not t.is_contiguous():
            raise ValueError("libsquad needs contiguous [B, heads, n, d] tensors")
        if t.dtype != ref.dtype or t.device != ref.device or t.shape != ref.shape:
            raise ValueError("q, k, v (and gradients) must share shape, dtype and device")


def _check_aux(t: torch.Tensor, shape, dtype, device, name: str):
    """A saved tensor handed back to the library: its extent is implied by the descriptor,
    so a wrong shape, dtype or device would make a kernel read outside it."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be a CUDA tensor on {device}")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be {dtype} of shape {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def workspace_size(desc: SquadDesc, which: int) -> int:
    out = ctypes.c_size_t(0)
    _check(load_library().squad_attn_workspace_size(ctypes.byref(desc), which, ctypes.byref(out)),
           "squad_attn_workspace_size")
    return int(out.value)


def squad_attn_fwd(q, k, v, grid, tile, scale: Optional[float] = None, save: bool = True,
                   stream: Optional[torch.cuda.Stream] = None, out: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None):
    """Forward through the C ABI. Returns (o, o1, lse1, lse2); o1/lse are None when save=False.

    With save=False the local-pass output lives in a workspace (``workspace``
    if given, else a fresh allocation of ``workspace_size(desc, 0)`` bytes).
    """
    lib = load_library()
    _check_inputs(q, k, v)
    desc = make_desc(q, grid, tile, scale)
    if out is not None:
        _check_aux(out, q.shape, q.dtype, q.device, "out")
    if workspace is not None and (not workspace.is_cuda or workspace.device != q.device
                                  or not workspace.is_contiguous()):
        raise ValueError(f"workspace must be a contiguous CUDA tensor on {q.device}")
    o = torch.empty_like(q) if out is None else out
    if save:
        o1 = torch.empty_like(q)
        lse1 = torch.empty(q.shape[:3], device=q.device, dtype=torch.float32)
        lse2 = torch.empty(q.shape[:3], device=q.device, dtype=torch.float32)
        ws_bytes = workspace_size(desc, 2)
        ws = workspace if workspace is not None else torch.empty(ws_bytes, device=q.device, dtype=torch.uint8)
        if ws.numel() * ws.element_size() < ws_bytes:
            raise ValueError("workspace too small")
    else:
        o1 = lse1 = lse2 = None
        ws_bytes = workspace_size(desc, 0)
        ws = workspace if workspace is not None else torch.empty(ws_bytes, device=q.device, dtype=torch.uint8)
        if ws.numel() * ws.element_size() < ws_bytes:
            raise ValueError("workspace too small")
    with torch.cuda.device(q.device):
        st = _stream_handle(stream, q.device)
        _check(lib.squad_attn_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(o1), _ptr(lse1),
                                  _ptr(lse2), _ptr(ws), ws_bytes, st), "squad_attn_fwd")
    return o, o1, lse1, lse2


def squad_attn_fwd_pass(stage: int, q, k, val, out, grid, tile, scale: Optional[float] = None,
                        lse: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None):
    """One pass of the forward (stage 1: local, values V; stage 2: global, values O1) into ``out``."""
    lib = load_library()
    _check_inputs(q, k, val, out)
    if lse is not None:
        _check_aux(lse, q.shape[:3], torch.float32, q.device, "lse")
    desc = make_desc(q, grid, tile, scale)
    with torch.cuda.device(q.device):
        st = _stream_handle(stream, q.device)
        _check(lib.squad_attn_fwd_pass(ctypes.byref(desc), int(stage), _ptr(q), _ptr(k), _ptr(val), _ptr(out),
                                       _ptr(lse), st), "squad_attn_fwd_pass")
    return out


def plan_info(desc: SquadDesc, stage: int):
    """Tiling of one pass: dict with rows, problems, tiles, box_rows, box (a, b, c), key_tiles_per_group."""
    info = (ctypes.c_int * 8)()
    _check(load_library().squad_plan_info(ctypes.byref(desc), int(stage), info), "squad_plan_info")
    v = list(info)
    return dict(rows=v[0], problems=v[1], tiles=v[2], box_rows=v[3], box=(v[4], v[5], v[6]), key_tiles_per_group=v[7])


def squad_attn_bwd(q, k, v, o, o1, lse1, lse2, dout, grid, tile, scale: Optional[float] = None,
                   stream: Optional[torch.cuda.Stream] = None):
    """Backward through the C ABI. Returns (dq, dk, dv)."""
    lib = load_library()
    _check_inputs(q, k, v, o, o1, dout)
    for t, name in ((lse1, "lse1"), (lse2, "lse2")):
        _check_aux(t, q.shape[:3], torch.float32, q.device, name)
    desc = make_desc(q, grid, tile, scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = workspace_size(desc, 1)
    ws = torch.empty(ws_bytes, device=q.device, dtype=torch.uint8)
    with torch.cuda.device(q.device):
        st = _stream_handle(stream, q.device)
        _check(lib.squad_attn_bwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(o1),
                                  _ptr(lse1), _ptr(lse2), _ptr(dout), _ptr(dq), _ptr(dk),
                                  _ptr(dv), _ptr(ws), ws_bytes, st), "squad_attn_bwd")
    return dq, dk, dv


def selftest_wait_timeout(timeout_ns: int = 10_000_000, stream: Optional[torch.cuda.Stream] = None):
    """Launch the device timeout self-test (a bounded wait that nothing satisfies)."""
    lib = load_library()
    lib.squad_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, ctypes.c_void_p]
    lib.squad_selftest_wait_timeout.restype = ctypes.c_int
    dev = torch.device("cuda", torch.cuda.current_device())
    _check(lib.squad_selftest_wait_timeout(int(timeout_ns), _stream_handle(stream, dev)), "squad_selftest_wait_timeout")


def tmap_cache_stats() -> Tuple[int, int]:
    """(hits, misses) of the library's tensor-map cache since it was loaded."""
    hits, misses = ctypes.c_ulonglong(0), ctypes.c_ulonglong(0)
    _check(load_library().squad_tmap_cache_stats(ctypes.byref(hits), ctypes.byref(misses)), "squad_tmap_cache_stats")
    return int(hits.value), int(misses.value)


def poll_device_error(stream: Optional[torch.cuda.Stream] = None, device=None):
    """Synchronise and raise SquadError(SQUAD_ERR_TIMEOUT) if a kernel gave up on a wait."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _check(load_library().squad_poll_device_error(_stream_handle(stream, dev)), "squad_poll_device_error")


class _SquadAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, grid, tile, scale):
        need = any(ctx.needs_input_grad[:3])
        o, o1, lse1, lse2 = squad_attn_fwd(q, k, v, grid, tile, scale, save=need)
        if need:
            ctx.save_for_backward(q, k, v, o, o1, lse1, lse2)
        ctx.geom = (tuple(grid), tuple(tile), scale)
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, o, o1, lse1, lse2 = ctx.saved_tensors
        grid, tile, scale = ctx.geom
        dq, dk, dv = squad_attn_bwd(q, k, v, o, o1, lse1, lse2, dout.contiguous(), grid, tile, scale)
        return dq, dk, dv, None, None, None


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid: Tuple[int, int, int],
              tile: Tuple[int, int, int], scale: Optional[float] = None) -> torch.Tensor:
    """SQuad-Attention of [B, heads, T*H*W, d] CUDA tensors (float32 or bfloat16), differentiable."""
    return _SquadAttention.apply(q, k, v, tuple(grid), tuple(tile), scale)


_side_streams = {}


def attention_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid, tile, scale: Optional[float] = None,
                   out: Optional[torch.Tensor] = None, slices_per_chunk: int = 4,
                   device: Optional[torch.device] = None, synchronize: bool = True) -> torch.Tensor:
    """SQuad-Attention forward of HOST tensors [B, heads, n, d] through squad_attn_fwd_host.

    The copies to and from the device overlap the forward, chunk by chunk of
    (batch, head) slices (pinned host tensors for the overlap). Returns the
    output as a host tensor (``out``, pinned, when not given). With
    synchronize=False the call returns once everything is enqueued on the
    device's current stream; ``out`` is complete after that stream synchronises.
    """
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        if t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous 4-D host tensor")
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("q, k and v must have the same shape and dtype")
    desc = make_desc(q, grid, tile, scale)
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    elif out.is_cuda or not out.is_contiguous() or out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must be a contiguous host tensor of q's shape and dtype")
    nb = ctypes.c_size_t(0)
    _check(lib.squad_attn_fwd_host_workspace_size(ctypes.byref(desc), int(slices_per_chunk), ctypes.byref(nb)),
           "squad_attn_fwd_host_workspace_size")
    with torch.cuda.device(dev):
        ws = torch.empty(int(nb.value), device=dev, dtype=torch.uint8)
        if dev.index not in _side_streams:
            _side_streams[dev.index] = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
        s_in, s_out = _side_streams[dev.index]
        cur = torch.cuda.current_stream(dev)
        _check(lib.squad_attn_fwd_host(ctypes.byref(desc), ctypes.c_void_p(q.data_ptr()),
                                       ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
                                       ctypes.c_void_p(out.data_ptr()), int(slices_per_chunk), _ptr(ws), int(nb.value),
                                       ctypes.c_void_p(cur.cuda_stream), ctypes.c_void_p(s_in.cuda_stream),
                                       ctypes.c_void_p(s_out.cuda_stream)), "squad_attn_fwd_host")
        ws.record_stream(s_in)
        ws.record_stream(s_out)
        if synchronize:
            cur.synchronize()
    return out


def squad_attn_fwd_noalloc(q, k, v, grid, tile, scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                           lse1: Optional[torch.Tensor] = None, lse2: Optional[torch.Tensor] = None,
                           stream: Optional[torch.cuda.Stream] = None):
    """Forward for callers that cannot give the library scratch memory.

    The C entry point squad_attn_fwd_noalloc allocates nothing: the local-pass
    output lives in a fixed 32 MiB device array inside libsquad, so only inputs
    and outputs are passed (here ``out`` is created with torch when not given).
    Problems whose local-pass output does not fit are rejected with
    SQUAD_ERR_WORKSPACE. Calls on one device share that array: do not let two of
    them run on the GPU at the same time (different streams or threads).
    """
    lib = load_library()
    fn = lib.squad_attn_fwd_noalloc
    fn.argtypes = [ctypes.POINTER(SquadDesc), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    _check_inputs(q, k, v)
    desc = make_desc(q, grid, tile, scale)
    if out is not None:
        _check_aux(out, q.shape, q.dtype, q.device, "out")
    for t, name in ((lse1, "lse1"), (lse2, "lse2")):
        if t is not None:
            _check_aux(t, q.shape[:3], torch.float32, q.device, name)
    o = torch.empty_like(q) if out is None else out
    with torch.cuda.device(q.device):
        st = _stream_handle(stream, q.device)
        _check(fn(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse1), _ptr(lse2), st),
               "squad_attn_fwd_noalloc")
    return o


# ---------------------------------------------------------------- more than two passes

def _tiles_arg(tiles: Sequence[Sequence[int]]):
    flat = [int(x) for t in tiles for x in t]
    if len(tiles) < 1 or any(len(t) != 3 for t in tiles):
        raise ValueError("tiles: a non-empty sequence of (tT, tH, tW), innermost first")
    return len(tiles), (ctypes.c_int * len(flat))(*flat)


def squad_attn_multi_fwd(q, k, v, grid, tiles, scale: Optional[float] = None,
                         stream: Optional[torch.cuda.Stream] = None, one_launch: Optional[bool] = None,
                         save: bool = True, out: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None):
    """k = len(tiles) + 1 passes over nested tiles (innermost first) through the C ABI.

    Returns (o, inter, lse): inter is [k-1, B, heads, n, d] (outputs of passes
    1..k-1), lse is [k, B, heads, n] fp32. one_launch: on bf16, run all passes in
    one launch (passes a counter workspace); False runs one launch per pass; None
    (default) picks one launch for save=False (same time, intermediates never
    written to DRAM) and one launch per pass otherwise (measured 3% faster).
    save=False (inference): the intermediate outputs and the LSE are not kept
    (inter and lse are None; the intermediates live in the workspace and, on bf16,
    leave L2 without a write-back once read). out / workspace: optional
    preallocated output and workspace (at least the size the library asks for).
    """
    lib = load_library()
    _check_inputs(q, k, v)
    desc = make_desc(q, grid, tiles[0], scale)
    nt, tarr = _tiles_arg(tiles)
    if out is not None:
        _check_aux(out, tuple(q.shape), q.dtype, q.device, "out")
    o = torch.empty_like(q) if out is None else out
    inter = torch.empty((nt,) + tuple(q.shape), device=q.device, dtype=q.dtype) if save else None
    lse = torch.empty((nt + 1,) + tuple(q.shape[:3]), device=q.device, dtype=torch.float32) if save else None
    if one_launch is None:
        one_launch = not save
    ws, ws_n = None, 0
    if one_launch or not save:
        nb = ctypes.c_size_t(0)
        _check(lib.squad_attn_multi_fwd_workspace_size(ctypes.byref(desc), nt, tarr, int(save), ctypes.byref(nb)),
               "squad_attn_multi_fwd_workspace_size")
        ws_n = int(nb.value)
        if workspace is not None:
            if workspace.device != q.device or not workspace.is_contiguous() or workspace.numel() * workspace.element_size() < ws_n:
                raise ValueError(f"workspace must be a contiguous tensor of at least {ws_n} bytes on {q.device}")
            ws = workspace
            ws_n = workspace.numel() * workspace.element_size()
        else:
            ws = torch.empty(ws_n, device=q.device, dtype=torch.uint8)
    with torch.cuda.device(q.device):
        st = _stream_handle(stream, q.device)
        _check(lib.squad_attn_multi_fwd(ctypes.byref(desc), nt, tarr, _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                        _ptr(inter), _ptr(lse), _ptr(ws), ws_n, st), "squad_attn_multi_fwd")
    return o, inter, lse


def squad_attn_multi_bwd(q, k, v, o, inter, lse, dout, grid, tiles, scale: Optional[float] = None,
                         stream: Optional[torch.cuda.Stream] = None):
    """Backward of squad_attn_multi_fwd through the C ABI. Returns (dq, dk, dv)."""
    lib = load_library()
    _check_inputs(q, k, v, o, dout)
    desc = make_desc(q, grid, tiles[0], scale)
    nt, tarr = _tiles_arg(tiles)
    _check_aux(inter, (nt,) + tuple(q.shape), q.dtype, q.device, "inter")
    _check_aux(lse, (nt + 1,) + tuple(q.shape[:3]), torch.float32, q.device, "lse")
    ws_bytes = ctypes.c_size_t(0)
    _check(lib.squad_attn_multi_bwd_workspace_size(ctypes.byref(desc), nt, tarr, ctypes.byref(ws_bytes)),
           "squad_attn_multi_bwd_workspace_size")
    ws = torch.empty(int(ws_bytes.value), device=q.device, dtype=torch.uint8)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    with torch.cuda.device(q.device):
        st = _stream_handle(stream, q.device)
        _check(lib.squad_attn_multi_bwd(ctypes.byref(desc), nt, tarr, _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                        _ptr(inter), _ptr(lse), _ptr(dout), _ptr(dq),
                                        _ptr(dk), _ptr(dv), _ptr(ws), int(ws_bytes.value), st),
               "squad_attn_multi_bwd")
    return dq, dk, dv


def multi_fwd_workspace_size(q: torch.Tensor, grid, tiles, save: bool = True, scale: Optional[float] = None) -> int:
    """Bytes of workspace squad_attn_multi_fwd asks for (save: the caller keeps the intermediates)."""
    lib = load_library()
    desc = make_desc(q, grid, tiles[0], scale)
    nt, tarr = _tiles_arg(tiles)
    nb = ctypes.c_size_t(0)
    _check(lib.squad_attn_multi_fwd_workspace_size(ctypes.byref(desc), nt, tarr, int(save), ctypes.byref(nb)),
           "squad_attn_multi_fwd_workspace_size")
    return int(nb.value)


class _SquadAttentionMulti(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, grid, tiles, scale):
        o, inter, lse = squad_attn_multi_fwd(q, k, v, grid, tiles, scale)
        if any(ctx.needs_input_grad[:3]):
            ctx.save_for_backward(q, k, v, o, inter, lse)
        ctx.geom = (tuple(grid), tuple(tuple(t) for t in tiles), scale)
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, o, inter, lse = ctx.saved_tensors
        grid, tiles, scale = ctx.geom
        dq, dk, dv = squad_attn_multi_bwd(q, k, v, o, inter, lse, dout.contiguous(), grid, tiles, scale)
        return dq, dk, dv, None, None, None


def attention_multi(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid: Tuple[int, int, int],
                    tiles: Sequence[Tuple[int, int, int]], scale: Optional[float] = None) -> torch.Tensor:
    """k = len(tiles) + 1 passes over nested tiles (innermost first), differentiable.

    Pass j attends among the tokens of one t_j-window at the same position inside
    their t_{j-1}-window (t_0 = one token, the last window the whole grid); one
    tile gives attention(q, k, v, grid, tiles[0]).
    """
    return _SquadAttentionMulti.apply(q, k, v, tuple(grid), tuple(tuple(t) for t in tiles), scale)
