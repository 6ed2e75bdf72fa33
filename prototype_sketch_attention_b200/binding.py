"""ctypes binding of libsa_sketch.so (argument marshalling only).

The functions named ``sa_*`` mirror the C ABI in include/sa_sketch.h one to one.
They take raw device pointers (ints), sizes and a stream handle, and return the
library's status code. ``forward`` and ``backward`` are conveniences for torch
users: they allocate outputs and workspace with torch (the library itself
allocates nothing), call the C ABI on the current stream and raise on errors.
Every step of the computation runs in the library's CUDA kernels. There is no
fallback: if the library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsa_sketch.so")

SA_F32 = 0
SA_BF16 = 1
SA_OK = 0
SA_ERR_INVALID_ARG = 1
SA_ERR_UNSUPPORTED = 2
SA_ERR_WORKSPACE = 3
SA_ERR_CUDA = 4
SA_ERR_TIMEOUT = 5
SA_ERR_BAD_OFFSETS = 6
SA_ERR_NO_DEVICE = 7

EXPORTED = ("sa_sketch_workspace_size", "sa_sketch_forward", "sa_sketch_backward",
            "sa_sketch_get_device_status", "sa_status_string", "sa_sketch_debug_wait_timeout",
            "sa_sketch_profile_events", "sa_sketch_forward_noalloc", "sa_sketch_combine",
            "sa_sketch_debug_gemm", "sa_stca_workspace_size", "sa_stca_forward",
            "sa_stca_backward", "sa_sketch_pack", "sa_sketch_unpack",
            "sa_sketch_forward_host_buffer_size", "sa_sketch_forward_host",
            "sa_sketch_forward_host_status", "sa_sketch_host_parts", "sa_sketch_forward_grid",
            "sa_stca_keys_workspace_size", "sa_stca_keys_forward", "sa_stca_keys_backward",
            "sa_stca_recent_ranges")
SA_CODEC_BF16 = 0
SA_CODEC_FP8 = 1


class SketchAttentionError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {sa_status_string(status)} ({status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is not built; run `python -m prototype_sketch_attention_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    lib.sa_sketch_workspace_size.restype = sz
    lib.sa_sketch_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32]
    lib.sa_sketch_forward.restype = i32
    lib.sa_sketch_forward.argtypes = [vp, vp, i32, i64, i32, vp, i32, vp, vp, i32,
                                      vp, vp, vp, vp, vp, sz, vp]
    lib.sa_sketch_backward.restype = i32
    lib.sa_sketch_backward.argtypes = [vp, vp, i32, i64, i32, vp, i32, vp, vp, i32,
                                       vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.sa_sketch_debug_gemm.restype = i32
    lib.sa_sketch_debug_gemm.argtypes = [vp, i32, vp, i32, i32, i32, i32, i32, vp, vp, vp]
    lib.sa_sketch_combine.restype = i32
    lib.sa_sketch_combine.argtypes = [vp, vp, i32, i32, i32, vp, i32, vp, vp]
    lib.sa_sketch_get_device_status.restype = i32
    lib.sa_sketch_get_device_status.argtypes = [vp, vp]
    lib.sa_status_string.restype = ctypes.c_char_p
    lib.sa_status_string.argtypes = [i32]
    lib.sa_sketch_debug_wait_timeout.restype = i32
    lib.sa_sketch_debug_wait_timeout.argtypes = [vp, ctypes.c_longlong, vp]
    lib.sa_sketch_profile_events.restype = i32
    lib.sa_sketch_profile_events.argtypes = [vp, vp]
    lib.sa_sketch_forward_noalloc.restype = i32
    lib.sa_sketch_forward_noalloc.argtypes = [vp, vp, i32, i64, i32, vp, i32, vp, vp, i32,
                                              vp, vp, vp, vp, vp, vp]
    lib.sa_stca_workspace_size.restype = sz
    lib.sa_stca_workspace_size.argtypes = [i32, i64, i32, i32, i32]
    lib.sa_sketch_pack.restype = i32
    lib.sa_sketch_pack.argtypes = [vp, i64, i32, i32, vp, vp, vp]
    lib.sa_sketch_unpack.restype = i32
    lib.sa_sketch_unpack.argtypes = [vp, vp, i64, i32, i32, vp, vp]
    lib.sa_stca_backward.restype = i32
    lib.sa_stca_backward.argtypes = [vp, vp, vp, i32, i64, i32, vp, i32, vp, vp, vp, vp, vp, vp,
                                     vp, vp, vp, vp, sz, vp]
    lib.sa_stca_forward.restype = i32
    lib.sa_stca_forward.argtypes = [vp, vp, i32, i64, i32, vp, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.sa_sketch_forward_host_buffer_size.restype = sz
    lib.sa_sketch_forward_host_buffer_size.argtypes = [i32, i64, i32, i32, i32, i32]
    lib.sa_sketch_forward_host.restype = i32
    lib.sa_sketch_forward_host.argtypes = [vp, vp, i32, i64, i32, vp, i32, vp, vp, i32, vp, vp,
                                           vp, sz, i32, vp, vp, vp]
    lib.sa_sketch_forward_host_status.restype = i32
    lib.sa_sketch_forward_host_status.argtypes = [vp, i32, i64, i32, i32, i32, i32, vp]
    lib.sa_sketch_forward_grid.restype = i32
    lib.sa_sketch_forward_grid.argtypes = [i32, i32, i32, vp, vp, vp, vp]
    lib.sa_sketch_host_parts.restype = i32
    lib.sa_sketch_host_parts.argtypes = [vp, i32, i32, vp]
    lib.sa_stca_keys_workspace_size.restype = sz
    lib.sa_stca_keys_workspace_size.argtypes = [i32, i64, i32, i32]
    lib.sa_stca_keys_forward.restype = i32
    lib.sa_stca_keys_forward.argtypes = [vp, vp, i32, i64, i32, vp, i64, vp, vp, vp, vp, vp, vp,
                                         vp, vp, sz, vp]
    lib.sa_stca_keys_backward.restype = i32
    lib.sa_stca_keys_backward.argtypes = [vp, vp, i32, i64, i32, vp, i64, vp, vp, vp, vp, vp, vp,
                                          vp, vp, i32, vp, vp, vp, vp, sz, vp]
    lib.sa_stca_recent_ranges.restype = i32
    lib.sa_stca_recent_ranges.argtypes = [vp, i32, i64, vp, vp, vp]
    return lib


_lib = _load()


# ---------------------------------------------------------------- raw C ABI
def sa_sketch_workspace_size(R: int, n_total: int, k: int, d: int, dt: int, backward: int) -> int:
    return int(_lib.sa_sketch_workspace_size(R, n_total, k, d, dt, backward))


def sa_sketch_forward(X, offsets, R, n_total, d, P, k, Wk, Wv, dt, sketch, mass, lse, xsketch,
                      workspace, ws_bytes, stream) -> int:
    return int(_lib.sa_sketch_forward(X, offsets, R, n_total, d, P, k, Wk, Wv, dt, sketch, mass,
                                      lse, xsketch, workspace, ws_bytes, stream))


def sa_sketch_backward(X, offsets, R, n_total, d, P, k, Wk, Wv, dt, sketch, mass, lse, xsketch,
                       dsketch, dmass, dX, dP, dWk, dWv, workspace, ws_bytes, stream) -> int:
    return int(_lib.sa_sketch_backward(X, offsets, R, n_total, d, P, k, Wk, Wv, dt, sketch, mass,
                                       lse, xsketch, dsketch, dmass, dX, dP, dWk, dWv, workspace,
                                       ws_bytes, stream))


def sa_sketch_debug_gemm(A, a_mn, B, b_mn, M, N, K, splits, out, workspace, stream) -> int:
    return int(_lib.sa_sketch_debug_gemm(A, a_mn, B, b_mn, M, N, K, splits, out, workspace, stream))


def sa_sketch_combine(xsketch, mass, R, k, d, Wv, dt, sketch, stream) -> int:
    return int(_lib.sa_sketch_combine(xsketch, mass, R, k, d, Wv, dt, sketch, stream))


def sa_stca_workspace_size(R: int, n_cand: int, k: int, d: int, backward: int = 0) -> int:
    return int(_lib.sa_stca_workspace_size(R, n_cand, k, d, backward))


def sa_stca_backward(Q, cand_offsets, cand_offsets_host, R, n_cand, d, S, k, Wq, WK, WV, dout, dQ,
                     dS, dWq, dWK, dWV, workspace, ws_bytes, stream) -> int:
    return int(_lib.sa_stca_backward(Q, cand_offsets, cand_offsets_host, R, n_cand, d, S, k, Wq, WK,
                                     WV, dout, dQ, dS, dWq, dWK, dWV, workspace, ws_bytes, stream))


def sa_stca_forward(Q, cand_offsets, R, n_cand, d, S, k, Wq, WK, WV, out, lse, workspace,
                    ws_bytes, stream) -> int:
    return int(_lib.sa_stca_forward(Q, cand_offsets, R, n_cand, d, S, k, Wq, WK, WV, out, lse,
                                    workspace, ws_bytes, stream))


def sa_stca_keys_workspace_size(R: int, n_cand: int, d: int, backward: int = 0) -> int:
    return int(_lib.sa_stca_keys_workspace_size(R, n_cand, d, backward))


def sa_stca_keys_forward(Q, cand_offsets, R, n_cand, d, Kx, n_keys, key_begin, key_end, Wq, WK,
                         WV, out, lse, workspace, ws_bytes, stream) -> int:
    return int(_lib.sa_stca_keys_forward(Q, cand_offsets, R, n_cand, d, Kx, n_keys, key_begin,
                                         key_end, Wq, WK, WV, out, lse, workspace, ws_bytes,
                                         stream))


def sa_stca_keys_backward(Q, cand_offsets, R, n_cand, d, Kx, n_keys, key_begin, key_end, Wq, WK,
                          WV, dout, dQ, dKx, accumulate, dWq, dWK, dWV, workspace, ws_bytes,
                          stream) -> int:
    return int(_lib.sa_stca_keys_backward(Q, cand_offsets, R, n_cand, d, Kx, n_keys, key_begin,
                                          key_end, Wq, WK, WV, dout, dQ, dKx, int(accumulate),
                                          dWq, dWK, dWV, workspace, ws_bytes, stream))


def sa_stca_recent_ranges(offsets, R, L, key_begin, key_end, stream) -> int:
    return int(_lib.sa_stca_recent_ranges(offsets, R, L, key_begin, key_end, stream))


def sa_sketch_forward_host_buffer_size(R, n_total, k, d, dt, parts) -> int:
    return int(_lib.sa_sketch_forward_host_buffer_size(R, n_total, k, d, dt, parts))


def sa_sketch_forward_host(X_host, offsets_host, R, n_total, d, P, k, Wk, Wv, dt, sketch_host,
                           mass_host, device_buffer, device_bytes, parts, stream, h2d_stream,
                           d2h_stream) -> int:
    return int(_lib.sa_sketch_forward_host(X_host, offsets_host, R, n_total, d, P, k, Wk, Wv, dt,
                                           sketch_host, mass_host, device_buffer, device_bytes,
                                           parts, stream, h2d_stream, d2h_stream))


def sa_sketch_forward_host_status(device_buffer, R, n_total, k, d, dt, parts, stream) -> int:
    return int(_lib.sa_sketch_forward_host_status(device_buffer, R, n_total, k, d, dt, parts,
                                                  stream))


def sa_sketch_forward_grid(k, d, dt, clusters, cluster_size, helpers=None, helper_share=None) -> int:
    return int(_lib.sa_sketch_forward_grid(k, d, dt, clusters, cluster_size, helpers, helper_share))


def forward_grid(k: int, d: int, dtype=torch.bfloat16) -> tuple[int, int, int, int]:
    """(clusters, cluster_size, helpers, helper_share) of the bf16 forward on the current
    device: tile ranges as sa_sketch_forward_grid describes."""
    c, s, h, f = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    st = sa_sketch_forward_grid(k, d, SA_BF16 if dtype == torch.bfloat16 else SA_F32,
                                ctypes.addressof(c), ctypes.addressof(s), ctypes.addressof(h),
                                ctypes.addressof(f))
    if st != SA_OK:
        raise SketchAttentionError(st, "sa_sketch_forward_grid")
    return c.value, s.value, h.value, f.value


def sa_sketch_host_parts(offsets_host, R, parts, bounds) -> int:
    return int(_lib.sa_sketch_host_parts(offsets_host, R, parts, bounds))


def sa_sketch_pack(sketch, rows, d, fmt, codes, scales, stream) -> int:
    return int(_lib.sa_sketch_pack(sketch, rows, d, fmt, codes, scales, stream))


def sa_sketch_unpack(codes, scales, rows, d, fmt, sketch, stream) -> int:
    return int(_lib.sa_sketch_unpack(codes, scales, rows, d, fmt, sketch, stream))


def sketch_pack(S: torch.Tensor, fmt: int = SA_CODEC_FP8, stream=None) -> dict:
    """Packs fp32 sketches [..., d] (contiguous, CUDA) for the cache: codes (uint8 for
    fp8, bfloat16 for bf16) and, for fp8, one fp32 scale per row."""
    where = "sketch_pack"
    _require(isinstance(S, torch.Tensor) and S.dim() >= 2, where, "S must be [..., d]")
    d = S.shape[-1]
    rows = S.numel() // d if d else 0
    _check_tensor(where, "S", S, tuple(S.shape), torch.float32, S.device)
    _check_cuda(where, S)
    dt = torch.uint8 if fmt == SA_CODEC_FP8 else torch.bfloat16
    out = {"codes": torch.empty(S.shape, dtype=dt, device=S.device),
           "scales": (torch.empty(S.shape[:-1], dtype=torch.float32, device=S.device)
                      if fmt == SA_CODEC_FP8 else None), "format": fmt}
    with torch.cuda.device(S.device):
        st = sa_sketch_pack(_ptr(S), rows, d, fmt, _ptr(out["codes"]), _ptr(out["scales"]),
                            _stream(stream, S.device))
    if st != SA_OK:
        raise SketchAttentionError(st, "sa_sketch_pack")
    return out


def sketch_unpack(packed: dict, stream=None) -> torch.Tensor:
    """The fp32 sketches back from sketch_pack's output."""
    codes, fmt = packed["codes"], packed["format"]
    d = codes.shape[-1]
    S = torch.empty(codes.shape, dtype=torch.float32, device=codes.device)
    with torch.cuda.device(codes.device):
        st = sa_sketch_unpack(_ptr(codes), _ptr(packed.get("scales")), codes.numel() // d, d, fmt,
                              _ptr(S), _stream(stream, codes.device))
    if st != SA_OK:
        raise SketchAttentionError(st, "sa_sketch_unpack")
    return S


def sa_sketch_get_device_status(workspace, stream) -> int:
    return int(_lib.sa_sketch_get_device_status(workspace, stream))


def sa_status_string(status: int) -> str:
    return _lib.sa_status_string(int(status)).decode()


def sa_sketch_debug_wait_timeout(workspace, budget_cycles: int, stream) -> int:
    return int(_lib.sa_sketch_debug_wait_timeout(workspace, int(budget_cycles), stream))


def sa_sketch_forward_noalloc(X, offsets, R, n_total, d, P, k, Wk, Wv, dt, sketch, mass, lse,
                              xsketch, device_status, stream) -> int:
    """Forward without a workspace (see include/sa_sketch.h). `device_status` is a host
    pointer (ctypes) or None."""
    return int(_lib.sa_sketch_forward_noalloc(X, offsets, R, n_total, d, P, k, Wk, Wv, dt, sketch,
                                              mass, lse, xsketch, device_status, stream))


def sa_sketch_profile_events(start_event, stop_event) -> int:
    return int(_lib.sa_sketch_profile_events(start_event, stop_event))


# ---------------------------------------------------------------- torch conveniences
def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def _dt(x: torch.Tensor) -> int:
    if x.dtype == torch.bfloat16:
        return SA_BF16
    if x.dtype == torch.float32:
        return SA_F32
    raise TypeError(f"X must be bfloat16 or float32, got {x.dtype}")


def _stream(stream, device=None) -> int:
    s = torch.cuda.current_stream(device) if stream is None else stream
    return s.cuda_stream


def _require(cond: bool, where: str, what: str) -> None:
    if not cond:
        raise SketchAttentionError(SA_ERR_INVALID_ARG, f"{where}: {what}")


def _check_tensor(where: str, name: str, t: torch.Tensor | None, shape: tuple, dtype,
                  device=None, optional: bool = False) -> None:
    """The C ABI sees only a pointer: shape, dtype, memory layout and device are the
    caller's promise, so the torch conveniences check them here."""
    if t is None:
        _require(optional, where, f"{name} is required")
        return
    _require(isinstance(t, torch.Tensor), where, f"{name} must be a tensor")
    _require(tuple(t.shape) == tuple(shape), where,
             f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    _require(t.dtype == dtype, where, f"{name} has dtype {t.dtype}, expected {dtype}")
    _require(t.is_contiguous(), where, f"{name} must be contiguous")
    if device is not None:
        _require(t.device == device, where, f"{name} is on {t.device}, expected {device}")


def _check_cuda(where: str, X: torch.Tensor) -> None:
    _require(X.is_cuda, where, f"inputs are on {X.device}; the library runs on CUDA devices only")


def _check_forward_inputs(where, X, offsets, P, Wk, Wv):
    _require(isinstance(X, torch.Tensor) and X.dim() == 2, where, "X must be a 2-D tensor")
    _require(isinstance(P, torch.Tensor) and P.dim() == 2, where, "P must be a 2-D tensor")
    _require(isinstance(offsets, torch.Tensor) and offsets.dim() == 1 and offsets.numel() >= 1,
             where, "offsets must be a 1-D tensor with R + 1 entries")
    n_total, d = X.shape
    k = P.shape[0]
    _dt(X)
    dev = X.device
    _check_tensor(where, "X", X, (n_total, d), X.dtype, dev)
    _check_tensor(where, "offsets", offsets, (offsets.numel(),), torch.int64, dev)
    _check_tensor(where, "P", P, (k, d), X.dtype, dev)
    _check_tensor(where, "Wk", Wk, (d, d), X.dtype, dev)
    _check_tensor(where, "Wv", Wv, (d, d), X.dtype, dev)


def workspace(R: int, n_total: int, k: int, d: int, dtype: torch.dtype, backward: bool = False,
              device=None) -> torch.Tensor:
    """A workspace tensor large enough for one call with these sizes."""
    dt = SA_BF16 if dtype == torch.bfloat16 else SA_F32
    n = sa_sketch_workspace_size(R, n_total, k, d, dt, int(backward))
    if n == 0:
        raise SketchAttentionError(SA_ERR_UNSUPPORTED, "sa_sketch_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def forward(X: torch.Tensor, offsets: torch.Tensor, P: torch.Tensor, Wk: torch.Tensor,
            Wv: torch.Tensor, *, want_lse: bool = True, want_xsketch: bool = True,
            ws: torch.Tensor | None = None, out: dict | None = None, stream=None) -> dict:
    """Sketch Attention forward on the GPU. Returns sketch, mass (and lse, xsketch).

    X [n_total, d] bf16/fp32, offsets [R+1] int64, P [k, d], Wk, Wv [d, d] (same dtype
    as X), all contiguous on one CUDA device. `out`, if given, holds fp32 sketch [R, k, d]
    and mass [R, k], and optionally lse [n_total] and xsketch [R, k, d].
    """
    where = "forward"
    _check_forward_inputs(where, X, offsets, P, Wk, Wv)
    n_total, d = X.shape
    k = P.shape[0]
    R = offsets.shape[0] - 1
    dt = _dt(X)
    dev = X.device
    if out is None:
        out = {"sketch": torch.empty(R, k, d, device=dev, dtype=torch.float32),
               "mass": torch.empty(R, k, device=dev, dtype=torch.float32)}
        if want_lse:
            out["lse"] = torch.empty(n_total, device=dev, dtype=torch.float32)
        if want_xsketch:
            out["xsketch"] = torch.empty(R, k, d, device=dev, dtype=torch.float32)
    f32 = torch.float32
    _check_tensor(where, "sketch", out.get("sketch"), (R, k, d), f32, dev)
    _check_tensor(where, "mass", out.get("mass"), (R, k), f32, dev)
    _check_tensor(where, "lse", out.get("lse"), (n_total,), f32, dev, optional=True)
    _check_tensor(where, "xsketch", out.get("xsketch"), (R, k, d), f32, dev, optional=True)
    _check_cuda(where, X)
    with torch.cuda.device(dev):
        if ws is None:
            ws = workspace(R, n_total, k, d, X.dtype, False, dev)
        _require(ws.device == dev and ws.is_contiguous(), where,
                 "ws must be contiguous on X's device")
        st = sa_sketch_forward(_ptr(X), _ptr(offsets), R, n_total, d, _ptr(P), k, _ptr(Wk),
                               _ptr(Wv), dt, _ptr(out["sketch"]), _ptr(out["mass"]),
                               _ptr(out.get("lse")), _ptr(out.get("xsketch")), _ptr(ws),
                               ws.nbytes, _stream(stream, dev))
    if st != SA_OK:
        raise SketchAttentionError(st, "sa_sketch_forward")
    out["_ws"] = ws
    return out


def backward(X, offsets, P, Wk, Wv, fwd: dict, dsketch: torch.Tensor, dmass=None, *,
             ws: torch.Tensor | None = None, stream=None) -> dict:
    """Gradients dX, dP, dWk, dWv given dL/dsketch (and optionally dL/dmass).

    `fwd` holds the forward's fp32 sketch [R, k, d], mass [R, k] and xsketch [R, k, d]
    (lse [n_total] optional); dsketch [R, k, d] and dmass [R, k] are fp32."""
    where = "backward"
    _check_forward_inputs(where, X, offsets, P, Wk, Wv)
    n_total, d = X.shape
    k = P.shape[0]
    R = offsets.shape[0] - 1
    dt = _dt(X)
    dev = X.device
    f32 = torch.float32
    _check_tensor(where, "sketch", fwd.get("sketch"), (R, k, d), f32, dev)
    _check_tensor(where, "mass", fwd.get("mass"), (R, k), f32, dev)
    _check_tensor(where, "xsketch", fwd.get("xsketch"), (R, k, d), f32, dev)
    _check_tensor(where, "lse", fwd.get("lse"), (n_total,), f32, dev, optional=True)
    _check_tensor(where, "dsketch", dsketch, (R, k, d), f32, dev)
    _check_tensor(where, "dmass", dmass, (R, k), f32, dev, optional=True)
    _check_cuda(where, X)
    out = {"dX": torch.empty(n_total, d, device=dev, dtype=f32),
           "dP": torch.empty(k, d, device=dev, dtype=f32),
           "dWk": torch.empty(d, d, device=dev, dtype=f32),
           "dWv": torch.empty(d, d, device=dev, dtype=f32)}
    with torch.cuda.device(dev):
        if ws is None:
            ws = workspace(R, n_total, k, d, X.dtype, True, dev)
        _require(ws.device == dev and ws.is_contiguous(), where,
                 "ws must be contiguous on X's device")
        st = sa_sketch_backward(_ptr(X), _ptr(offsets), R, n_total, d, _ptr(P), k, _ptr(Wk),
                                _ptr(Wv), dt, _ptr(fwd["sketch"]), _ptr(fwd["mass"]),
                                _ptr(fwd.get("lse")), _ptr(fwd["xsketch"]), _ptr(dsketch),
                                _ptr(dmass), _ptr(out["dX"]), _ptr(out["dP"]), _ptr(out["dWk"]),
                                _ptr(out["dWv"]), _ptr(ws), ws.nbytes, _stream(stream, dev))
    if st != SA_OK:
        raise SketchAttentionError(st, "sa_sketch_backward")
    out["_ws"] = ws
    return out


def combine(xsketch: torch.Tensor, mass: torch.Tensor, Wv: torch.Tensor, *,
            out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """sketch = (xsketch Wv) / mass for users whose partial xsketch and mass (from
    forward calls over parts of their tokens) have been summed. xsketch [R, k, d] and
    mass [R, k] fp32, Wv [d, d] bf16/fp32, all on one CUDA device."""
    where = "combine"
    _require(isinstance(xsketch, torch.Tensor) and xsketch.dim() == 3, where,
             "xsketch must be a 3-D tensor")
    R, k, d = xsketch.shape
    dev = xsketch.device
    f32 = torch.float32
    _check_tensor(where, "xsketch", xsketch, (R, k, d), f32, dev)
    _check_tensor(where, "mass", mass, (R, k), f32, dev)
    _require(isinstance(Wv, torch.Tensor), where, "Wv must be a tensor")
    _check_tensor(where, "Wv", Wv, (d, d), Wv.dtype, dev)
    dt = _dt(Wv)
    if out is None:
        out = torch.empty(R, k, d, device=dev, dtype=f32)
    _check_tensor(where, "out", out, (R, k, d), f32, dev)
    _check_cuda(where, xsketch)
    with torch.cuda.device(dev):
        st = sa_sketch_combine(_ptr(xsketch), _ptr(mass), R, k, d, _ptr(Wv), dt, _ptr(out),
                               _stream(stream, dev))
    if st != SA_OK:
        raise SketchAttentionError(st, "sa_sketch_combine")
    return out


def stca_forward(Q: torch.Tensor, cand_offsets: torch.Tensor, S: torch.Tensor, Wq: torch.Tensor,
                 WK: torch.Tensor, WV: torch.Tensor, *, want_lse: bool = True,
                 ws: torch.Tensor | None = None, stream=None) -> dict:
    """Candidate-to-sketch cross attention on the GPU: every candidate of user u attends
    over the k rows of u's sketch. Q [n_cand, d] bf16, cand_offsets [R+1] int64,
    S [R, k, d] fp32 (the forward's sketch), Wq, WK, WV [d, d] bf16, all contiguous on one
    CUDA device. Returns out [n_cand, d] fp32 (and lse [n_cand])."""
    where = "stca_forward"
    _require(isinstance(Q, torch.Tensor) and Q.dim() == 2, where, "Q must be a 2-D tensor")
    _require(isinstance(S, torch.Tensor) and S.dim() == 3, where, "S must be a 3-D tensor")
    _require(isinstance(cand_offsets, torch.Tensor) and cand_offsets.dim() == 1
             and cand_offsets.numel() >= 1, where, "cand_offsets must be a 1-D tensor with R + 1 entries")
    n_cand, d = Q.shape
    R, k = cand_offsets.numel() - 1, S.shape[1]
    dev = Q.device
    bf = torch.bfloat16
    _check_tensor(where, "Q", Q, (n_cand, d), bf, dev)
    _check_tensor(where, "cand_offsets", cand_offsets, (R + 1,), torch.int64, dev)
    _check_tensor(where, "S", S, (R, k, d), torch.float32, dev)
    for name, W in (("Wq", Wq), ("WK", WK), ("WV", WV)):
        _check_tensor(where, name, W, (d, d), bf, dev)
    _check_cuda(where, Q)
    out = {"out": torch.empty(n_cand, d, device=dev, dtype=torch.float32)}
    if want_lse:
        out["lse"] = torch.empty(n_cand, device=dev, dtype=torch.float32)
    with torch.cuda.device(dev):
        if ws is None:
            nb = sa_stca_workspace_size(R, n_cand, k, d, 0)
            if nb == 0:
                raise SketchAttentionError(SA_ERR_UNSUPPORTED, "sa_stca_workspace_size")
            ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        st = sa_stca_forward(_ptr(Q), _ptr(cand_offsets), R, n_cand, d, _ptr(S), k, _ptr(Wq),
                             _ptr(WK), _ptr(WV), _ptr(out["out"]), _ptr(out.get("lse")),
                             _ptr(ws), ws.nbytes, _stream(stream, dev))
    if st != SA_OK:
        raise SketchAttentionError(st, "sa_stca_forward")
    out["_ws"] = ws
    return out


def stca_backward(Q: torch.Tensor, cand_offsets: torch.Tensor, S: torch.Tensor, Wq: torch.Tensor,
                  WK: torch.Tensor, WV: torch.Tensor, dout: torch.Tensor, *,
                  cand_offsets_host: torch.Tensor | None = None,
                  ws: torch.Tensor | None = None, stream=None) -> dict:
    """Gradients of stca_forward given dL/dout [n_cand, d] fp32: dQ, dS (into each
    user's sketch), dWq, dWK, dWV. Inputs as for stca_forward; cand_offsets_host, a CPU
    copy of cand_offsets, saves the device-to-host copy (and lets the call be captured
    into a CUDA graph)."""
    where = "stca_backward"
    _require(isinstance(Q, torch.Tensor) and Q.dim() == 2, where, "Q must be a 2-D tensor")
    _require(isinstance(S, torch.Tensor) and S.dim() == 3, where, "S must be a 3-D tensor")
    _require(isinstance(cand_offsets, torch.Tensor) and cand_offsets.dim() == 1
             and cand_offsets.numel() >= 1, where, "cand_offsets must be a 1-D tensor with R + 1 entries")
    n_cand, d = Q.shape
    R, k = cand_offsets.numel() - 1, S.shape[1]
    dev = Q.device
    bf, f32 = torch.bfloat16, torch.float32
    _check_tensor(where, "Q", Q, (n_cand, d), bf, dev)
    _check_tensor(where, "cand_offsets", cand_offsets, (R + 1,), torch.int64, dev)
    _check_tensor(where, "S", S, (R, k, d), f32, dev)
    for name, W in (("Wq", Wq), ("WK", WK), ("WV", WV)):
        _check_tensor(where, name, W, (d, d), bf, dev)
    _check_tensor(where, "dout", dout, (n_cand, d), f32, dev)
    _check_cuda(where, Q)
    if cand_offsets_host is None:
        coff_h = cand_offsets.cpu().contiguous()
    else:
        _check_tensor(where, "cand_offsets_host", cand_offsets_host, (R + 1,), torch.int64,
                      torch.device("cpu"))
        coff_h = cand_offsets_host
    out = {"dQ": torch.empty(n_cand, d, device=dev, dtype=f32),
           "dS": torch.empty(R, k, d, device=dev, dtype=f32),
           "dWq": torch.empty(d, d, device=dev, dtype=f32),
           "dWK": torch.empty(d, d, device=dev, dtype=f32),
           "dWV": torch.empty(d, d, device=dev, dtype=f32)}
    with torch.cuda.device(dev):
        if ws is None:
            nb = sa_stca_workspace_size(R, n_cand, k, d, 1)
            if nb == 0:
                raise SketchAttentionError(SA_ERR_UNSUPPORTED, "sa_stca_workspace_size")
            ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        st = sa_stca_backward(_ptr(Q), _ptr(cand_offsets), _ptr(coff_h), R, n_cand, d, _ptr(S), k,
                              _ptr(Wq), _ptr(WK), _ptr(WV), _ptr(dout), _ptr(out["dQ"]),
                              _ptr(out["dS"]), _ptr(out["dWq"]), _ptr(out["dWK"]),
                              _ptr(out["dWV"]), _ptr(ws), ws.nbytes, _stream(stream, dev))
    if st != SA_OK:
        raise SketchAttentionError(st, "sa_stca_backward")
    out["_ws"] = ws
    return out


def recent_ranges(offsets: torch.Tensor, L: int, *, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """The recent branch's key ranges over a history laid out by `offsets` [R+1] (int64,
    CUDA): each user's last min(n_u, L) rows. Returns (key_begin, key_end), int64 [R]."""
    where = "recent_ranges"
    _require(isinstance(offsets, torch.Tensor) and offsets.dim() == 1 and offsets.numel() >= 1,
             where, "offsets must be a 1-D tensor with R + 1 entries")
    R = offsets.numel() - 1
    dev = offsets.device
    _check_tensor(where, "offsets", offsets, (R + 1,), torch.int64, dev)
    _check_cuda(where, offsets)
    kb = torch.empty(R, dtype=torch.int64, device=dev)
    ke = torch.empty(R, dtype=torch.int64, device=dev)
    with torch.cuda.device(dev):
        st = sa_stca_recent_ranges(_ptr(offsets), R, int(L), _ptr(kb), _ptr(ke),
                                   _stream(stream, dev))
    if st != SA_OK:
        raise SketchAttentionError(st, "sa_stca_recent_ranges")
    return kb, ke


def _check_keys_inputs(where, Q, cand_offsets, Kx, key_begin, key_end, Wq, WK, WV):
    _require(isinstance(Q, torch.Tensor) and Q.dim() == 2, where, "Q must be a 2-D tensor")
    _require(isinstance(Kx, torch.Tensor) and Kx.dim() == 2, where, "Kx must be a 2-D tensor")
    _require(isinstance(cand_offsets, torch.Tensor) and cand_offsets.dim() == 1
             and cand_offsets.numel() >= 1, where, "cand_offsets must be a 1-D tensor with R + 1 entries")
    n_cand, d = Q.shape
    R = cand_offsets.numel() - 1
    dev = Q.device
    bf = torch.bfloat16
    _check_tensor(where, "Q", Q, (n_cand, d), bf, dev)
    _check_tensor(where, "Kx", Kx, (Kx.shape[0], d), bf, dev)
    _check_tensor(where, "cand_offsets", cand_offsets, (R + 1,), torch.int64, dev)
    _check_tensor(where, "key_begin", key_begin, (R,), torch.int64, dev)
    _check_tensor(where, "key_end", key_end, (R,), torch.int64, dev)
    for name, W in (("Wq", Wq), ("WK", WK), ("WV", WV)):
        _check_tensor(where, name, W, (d, d), bf, dev)
    _check_cuda(where, Q)
    return n_cand, d, R, Kx.shape[0], dev


def stca_keys_forward(Q: torch.Tensor, cand_offsets: torch.Tensor, Kx: torch.Tensor,
                      key_begin: torch.Tensor, key_end: torch.Tensor, Wq: torch.Tensor,
                      WK: torch.Tensor, WV: torch.Tensor, *, want_lse: bool = True,
                      ws: torch.Tensor | None = None, stream=None) -> dict:
    """Cross attention from user u's candidates to the key rows Kx[key_begin[u]:key_end[u]]
    (the recent branch: Kx = the history X, ranges from recent_ranges). Q [n_cand, d] bf16,
    cand_offsets [R+1] int64, Kx [n_keys, d] bf16, key_begin / key_end [R] int64,
    Wq, WK, WV [d, d] bf16, all on one CUDA device. Returns out [n_cand, d] fp32 (and
    lse [n_cand])."""
    where = "stca_keys_forward"
    n_cand, d, R, n_keys, dev = _check_keys_inputs(where, Q, cand_offsets, Kx, key_begin, key_end,
                                                   Wq, WK, WV)
    out = {"out": torch.empty(n_cand, d, device=dev, dtype=torch.float32)}
    if want_lse:
        out["lse"] = torch.empty(n_cand, device=dev, dtype=torch.float32)
    with torch.cuda.device(dev):
        if ws is None:
            nb = sa_stca_keys_workspace_size(R, n_cand, d, 0)
            if nb == 0:
                raise SketchAttentionError(SA_ERR_UNSUPPORTED, "sa_stca_keys_workspace_size")
            ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        st = sa_stca_keys_forward(_ptr(Q), _ptr(cand_offsets), R, n_cand, d, _ptr(Kx), n_keys,
                                  _ptr(key_begin), _ptr(key_end), _ptr(Wq), _ptr(WK), _ptr(WV),
                                  _ptr(out["out"]), _ptr(out.get("lse")), _ptr(ws), ws.nbytes,
                                  _stream(stream, dev))
    if st != SA_OK:
        raise SketchAttentionError(st, "sa_stca_keys_forward")
    out["_ws"] = ws
    return out


def stca_keys_backward(Q: torch.Tensor, cand_offsets: torch.Tensor, Kx: torch.Tensor,
                       key_begin: torch.Tensor, key_end: torch.Tensor, Wq: torch.Tensor,
                       WK: torch.Tensor, WV: torch.Tensor, dout: torch.Tensor, *,
                       dKx: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                       stream=None) -> dict:
    """Gradients of stca_keys_forward given dL/dout [n_cand, d] fp32: dQ, dKx [n_keys, d]
    (into the key rows), dWq, dWK, dWV. Inputs as for stca_keys_forward. With dKx given
    (fp32 [n_keys, d]), the key rows' gradient is added into it instead of a new tensor
    (for the recent branch: into the history gradient)."""
    where = "stca_keys_backward"
    n_cand, d, R, n_keys, dev = _check_keys_inputs(where, Q, cand_offsets, Kx, key_begin, key_end,
                                                   Wq, WK, WV)
    f32 = torch.float32
    _check_tensor(where, "dout", dout, (n_cand, d), f32, dev)
    _check_tensor(where, "dKx", dKx, (n_keys, d), f32, dev, optional=True)
    accumulate = dKx is not None
    out = {"dQ": torch.empty(n_cand, d, device=dev, dtype=f32),
           "dKx": dKx if accumulate else torch.empty(n_keys, d, device=dev, dtype=f32),
           "dWq": torch.empty(d, d, device=dev, dtype=f32),
           "dWK": torch.empty(d, d, device=dev, dtype=f32),
           "dWV": torch.empty(d, d, device=dev, dtype=f32)}
    with torch.cuda.device(dev):
        if ws is None:
            nb = sa_stca_keys_workspace_size(R, n_cand, d, 1)
            if nb == 0:
                raise SketchAttentionError(SA_ERR_UNSUPPORTED, "sa_stca_keys_workspace_size")
            ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        st = sa_stca_keys_backward(_ptr(Q), _ptr(cand_offsets), R, n_cand, d, _ptr(Kx), n_keys,
                                   _ptr(key_begin), _ptr(key_end), _ptr(Wq), _ptr(WK), _ptr(WV),
                                   _ptr(dout), _ptr(out["dQ"]), _ptr(out["dKx"]), accumulate,
                                   _ptr(out["dWq"]), _ptr(out["dWK"]), _ptr(out["dWV"]),
                                   _ptr(ws), ws.nbytes, _stream(stream, dev))
    if st != SA_OK:
        raise SketchAttentionError(st, "sa_stca_keys_backward")
    out["_ws"] = ws
    return out


def user_chunks(offsets_host: torch.Tensor, chunks: int) -> list[tuple[int, int]]:
    """The library's cut of users [0, R) into at most `chunks` consecutive parts of about
    equal token count (sa_sketch_host_parts). offsets_host: int64 [R + 1] on the host."""
    _require(isinstance(offsets_host, torch.Tensor) and offsets_host.dtype == torch.int64
             and offsets_host.device.type == "cpu" and offsets_host.dim() == 1,
             "user_chunks", "offsets_host must be a host int64 [R + 1] tensor")
    off = offsets_host.contiguous()
    R = off.numel() - 1
    bounds = (ctypes.c_int * (max(int(chunks), 1) + 1))()
    np_ = sa_sketch_host_parts(off.data_ptr(), R, int(chunks), ctypes.addressof(bounds))
    if np_ < 0:
        raise SketchAttentionError(-np_, "sa_sketch_host_parts")
    return [(bounds[i], bounds[i + 1]) for i in range(np_)]


def forward_from_host(Xh: torch.Tensor, offsets_h: torch.Tensor, P: torch.Tensor,
                      Wk: torch.Tensor, Wv: torch.Tensor, *, chunks: int = 4,
                      state: dict | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """Forward from host X and offsets to host sketch and mass through
    sa_sketch_forward_host, which cuts the users into `chunks` parts and overlaps each
    part's copy to the device with the previous part's forward (the library owns the
    pipeline; this function only marshals). Xh and offsets_h should be pinned. P, Wk, Wv
    live on the device. `state` (a dict the caller keeps) holds the device buffer, the
    pinned outputs and the two copy streams between calls. The outputs are complete once
    the current stream reaches the end of this call's work; the returned host tensors are
    the state's staging, which the next call with the same `state` overwrites."""
    where = "forward_from_host"
    _require(isinstance(Xh, torch.Tensor) and Xh.dim() == 2 and Xh.device.type == "cpu"
             and Xh.is_contiguous(), where, "Xh must be a contiguous 2-D host tensor")
    _require(isinstance(offsets_h, torch.Tensor) and offsets_h.dim() == 1
             and offsets_h.numel() >= 1 and offsets_h.dtype == torch.int64
             and offsets_h.device.type == "cpu", where, "offsets_h must be host int64 [R + 1]")
    _require(isinstance(P, torch.Tensor) and P.is_cuda, where, "P, Wk, Wv must be on the GPU")
    _require(int(chunks) >= 1, where, "chunks must be at least 1")
    R = offsets_h.numel() - 1
    n_total, d = Xh.shape
    k = P.shape[0]
    dev = P.device
    dt = _dt(Xh)
    _check_tensor(where, "P", P, (k, d), Xh.dtype, dev)
    _check_tensor(where, "Wk", Wk, (d, d), Xh.dtype, dev)
    _check_tensor(where, "Wv", Wv, (d, d), Xh.dtype, dev)
    st = {} if state is None else state
    key = (R, n_total, k, d, Xh.dtype, int(chunks), dev)
    if st.get("key") != key:
        st.clear()
        with torch.cuda.device(dev):
            nb = sa_sketch_forward_host_buffer_size(R, n_total, k, d, dt, int(chunks))
            if nb == 0:
                raise SketchAttentionError(SA_ERR_UNSUPPORTED, "sa_sketch_forward_host_buffer_size")
            st.update(key=key, buf=torch.empty(nb, dtype=torch.uint8, device=dev),
                      sk_h=torch.empty(R, k, d, dtype=torch.float32).pin_memory(),
                      ms_h=torch.empty(R, k, dtype=torch.float32).pin_memory(),
                      s_h2d=torch.cuda.Stream(dev), s_d2h=torch.cuda.Stream(dev))
    off = offsets_h.contiguous()
    cur = torch.cuda.current_stream(dev)
    with torch.cuda.device(dev):
        rc = sa_sketch_forward_host(_ptr(Xh), off.data_ptr(), R, n_total, d, _ptr(P), k, _ptr(Wk),
                                    _ptr(Wv), dt, _ptr(st["sk_h"]), _ptr(st["ms_h"]),
                                    _ptr(st["buf"]), st["buf"].nbytes, int(chunks),
                                    cur.cuda_stream, st["s_h2d"].cuda_stream,
                                    st["s_d2h"].cuda_stream)
    if rc != SA_OK:
        raise SketchAttentionError(rc, "sa_sketch_forward_host")
    return st["sk_h"], st["ms_h"]


def forward_from_host_status(state: dict, stream=None) -> int:
    """Device status of the last forward_from_host call made with `state` (synchronises)."""
    R, n_total, k, d, dtype, chunks, dev = state["key"]
    return sa_sketch_forward_host_status(_ptr(state["buf"]), R, n_total, k, d,
                                         SA_BF16 if dtype == torch.bfloat16 else SA_F32, chunks,
                                         _stream(stream, dev))


def device_status(ws: torch.Tensor, stream=None) -> int:
    return sa_sketch_get_device_status(_ptr(ws), _stream(stream))
