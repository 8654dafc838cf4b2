"""ctypes binding of ``libssm_scan_b200.so`` (C ABI: ``include/ssm_scan.h``).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, their data pointers and the current CUDA stream are passed to
the library, and every step of the scan runs in the library's kernels.
There is no fallback: if the library is missing, loading fails loudly.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssm_scan_b200.so")

# ssm_status
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_MISALIGNED, ERR_CUDA, ERR_TIMEOUT, ERR_OOM = range(7)
# ssm_dtype
F32, BF16 = 0, 1
# flags
HAS_Z, HAS_D, DELTA_SOFTPLUS, HAS_DELTA_BIAS, HAS_H0, WANT_HLAST, A_DIRECT = 1, 2, 4, 8, 16, 32, 64
ZOH = 128  # zero-order-hold input matrix: Bbar = (exp(Delta A) - 1) / A * B
CONV_X = 256  # x branch through the causal conv front-end (ssm_scan_fwd_conv)
CONV_WIDTH = 4

_TORCH_TO_SSM = {torch.float32: F32, torch.bfloat16: BF16}


class SsmError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


class Desc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("dim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
                ("flags", ctypes.c_uint32)]


class Info(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("lanes_per_chan", ctypes.c_int),
                ("warps_per_cta", ctypes.c_int), ("tile_t", ctypes.c_int), ("stages", ctypes.c_int),
                ("stages_per_row", ctypes.c_int), ("chans_per_cta", ctypes.c_int),
                ("grid", ctypes.c_int), ("rows", ctypes.c_int64), ("units", ctypes.c_int64),
                ("parts_per_row", ctypes.c_int), ("stages_per_part", ctypes.c_int),
                ("smem_bytes", ctypes.c_size_t), ("workspace_bytes", ctypes.c_size_t),
                ("chans_per_lane", ctypes.c_int), ("segments", ctypes.c_int),
                ("stages_per_segment", ctypes.c_int), ("carry_grid", ctypes.c_int),
                ("launches_per_call", ctypes.c_int), ("scan_loop", ctypes.c_int),
                ("carry_lanes_per_chan", ctypes.c_int), ("carry_loop", ctypes.c_int),
                ("bwd_warps_per_cta", ctypes.c_int), ("carry_chans_per_lane", ctypes.c_int),
                ("bwd_segments", ctypes.c_int)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


class Config(ctypes.Structure):
    _fields_ = [("lanes_per_chan", ctypes.c_int), ("warps_per_cta", ctypes.c_int),
                ("grid", ctypes.c_int), ("tile_t", ctypes.c_int),
                ("chans_per_lane", ctypes.c_int), ("segments", ctypes.c_int),
                ("scan_loop", ctypes.c_int), ("carry_lanes_per_chan", ctypes.c_int),
                ("carry_loop", ctypes.c_int), ("bwd_warps_per_cta", ctypes.c_int),
                ("carry_chans_per_lane", ctypes.c_int), ("bwd_segments", ctypes.c_int)]


class Variant(ctypes.Structure):
    _fields_ = [("dstate", ctypes.c_int), ("lanes_per_chan", ctypes.c_int),
                ("chans_per_lane", ctypes.c_int), ("warps_per_cta", ctypes.c_int),
                ("tile_t", ctypes.c_int), ("zoh", ctypes.c_int), ("carry", ctypes.c_int),
                ("conv", ctypes.c_int), ("opt", ctypes.c_int)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


_lib = None
_lib_lock = threading.Lock()
_vp = ctypes.c_void_p


def load_library(path: str | None = None):
    """Load the CUDA library (once).  Raises if it has not been built."""
    global _lib
    with _lib_lock:
        if _lib is not None:
            return _lib
        path = path or LIB_PATH
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m selective_state_space_31_b200.build`")
        lib = ctypes.CDLL(path)
        st = ctypes.c_int
        lib.ssm_scan_create.argtypes = [ctypes.POINTER(_vp), ctypes.POINTER(Desc), ctypes.c_int]
        lib.ssm_scan_create.restype = st
        lib.ssm_scan_destroy.argtypes = [_vp]
        lib.ssm_scan_destroy.restype = st
        lib.ssm_scan_fwd.argtypes = [_vp] * 13
        lib.ssm_scan_fwd.restype = st
        lib.ssm_scan_step_host.argtypes = [_vp] * 11 + [ctypes.c_int64, _vp]
        lib.ssm_scan_step_host.restype = st
        lib.ssm_scan_fwd_host.argtypes = [_vp] * 12 + [ctypes.c_int64, _vp]
        lib.ssm_scan_fwd_host.restype = st
        lib.ssm_scan_fwd_conv.argtypes = [_vp] * 16
        lib.ssm_scan_fwd_conv.restype = st
        lib.ssm_scan_seq_map.argtypes = [_vp] * 9
        lib.ssm_scan_seq_map.restype = st
        lib.ssm_scan_fold_maps.argtypes = [_vp, ctypes.c_int] + [_vp] * 6
        lib.ssm_scan_fold_maps.restype = st
        lib.ssm_scan_step.argtypes = [_vp] * 12
        lib.ssm_scan_step.restype = st
        lib.ssm_scan_bwd.argtypes = [_vp] * 22
        lib.ssm_scan_bwd.restype = st
        lib.ssm_scan_get_status.argtypes = [_vp]
        lib.ssm_scan_get_status.restype = st
        lib.ssm_scan_get_info.argtypes = [_vp, ctypes.POINTER(Info)]
        lib.ssm_scan_get_info.restype = st
        lib.ssm_scan_set_config.argtypes = [_vp, ctypes.POINTER(Config)]
        lib.ssm_scan_set_config.restype = st
        lib.ssm_scan_set_debug.argtypes = [_vp, ctypes.c_uint64, ctypes.c_int64]
        lib.ssm_scan_set_debug.restype = st
        lib.ssm_status_string.argtypes = [ctypes.c_int]
        lib.ssm_status_string.restype = ctypes.c_char_p
        lib.ssm_scan_version.argtypes = []
        lib.ssm_scan_version.restype = ctypes.c_int
        lib.ssm_scan_fwd_noalloc.argtypes = [ctypes.POINTER(Desc)] + [_vp] * 12
        lib.ssm_scan_fwd_noalloc.restype = st
        lib.ssm_scan_noalloc_status.argtypes = []
        lib.ssm_scan_noalloc_status.restype = st
        lib.ssm_scan_noalloc_set_debug.argtypes = [ctypes.c_uint64, ctypes.c_int64]
        lib.ssm_scan_noalloc_set_debug.restype = st
        lib.ssm_probe_peak.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int, _vp,
                                       ctypes.POINTER(ctypes.c_int64), _vp]
        lib.ssm_probe_peak.restype = st
        lib.ssm_probe_exp2.argtypes = [_vp, _vp, _vp, ctypes.c_int64, _vp]
        lib.ssm_probe_exp2.restype = st
        lib.ssm_scan_list_variants.argtypes = [ctypes.c_int, ctypes.c_int,
                                               ctypes.POINTER(Variant), ctypes.c_int]
        lib.ssm_scan_list_variants.restype = ctypes.c_int
        _lib = lib
        return lib


def status_string(s: int) -> str:
    return load_library().ssm_status_string(int(s)).decode()


def _check(rc: int, what: str):
    if rc != OK:
        raise SsmError(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t, name, shape, dtype, device):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


class Plan:
    """One problem shape on one device (wraps ``ssm_scan_plan``)."""

    def __init__(self, batch, seqlen, dim, dstate, in_dtype=torch.bfloat16, out_dtype=None,
                 flags=0, device=None):
        self._lib = load_library()
        self.device = torch.device(device if device is not None else "cuda", )
        if self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        out_dtype = out_dtype or in_dtype
        self.desc = Desc(int(batch), int(seqlen), int(dim), int(dstate),
                         _TORCH_TO_SSM[in_dtype], _TORCH_TO_SSM[out_dtype], int(flags))
        self.in_dtype, self.out_dtype, self.flags = in_dtype, out_dtype, int(flags)
        h = _vp()
        _check(self._lib.ssm_scan_create(ctypes.byref(h), ctypes.byref(self.desc),
                                         self.device.index), "ssm_scan_create")
        self._h = h

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            self._lib.ssm_scan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def info(self) -> dict:
        i = Info()
        _check(self._lib.ssm_scan_get_info(self._h, ctypes.byref(i)), "ssm_scan_get_info")
        return i.as_dict()

    def set_config(self, lanes_per_chan=0, warps_per_cta=0, grid=0, tile_t=0,
                   chans_per_lane=0, segments=0, scan_loop=0, carry_lanes_per_chan=0,
                   carry_loop=0, bwd_warps_per_cta=0, carry_chans_per_lane=0, bwd_segments=0):
        c = Config(lanes_per_chan, warps_per_cta, grid, tile_t, chans_per_lane, segments,
                   scan_loop, carry_lanes_per_chan, carry_loop, bwd_warps_per_cta,
                   carry_chans_per_lane, bwd_segments)
        _check(self._lib.ssm_scan_set_config(self._h, ctypes.byref(c)), "ssm_scan_set_config")

    def set_debug(self, wait_timeout_ns=0, drop_unit=-1):
        _check(self._lib.ssm_scan_set_debug(self._h, int(wait_timeout_ns), int(drop_unit)),
               "ssm_scan_set_debug")

    def status(self) -> int:
        """Synchronise and return (and clear) the device-side status."""
        return self._lib.ssm_scan_get_status(self._h)

    # -- calls -------------------------------------------------------------
    def fwd(self, x, delta, A, B, C, D=None, z=None, delta_bias=None, h0=None, y=None,
            h_last=None):
        d, f, dev = self.desc, self.flags, self.device
        Bz, L, Dm, N = d.batch, d.seqlen, d.dim, d.dstate
        if f & A_DIRECT:
            _need(A, "A", (Bz, L, Dm), self.in_dtype, dev)
            _need(h0, "h0", (Bz, Dm), torch.float32, dev)
            hshape = (Bz, Dm)
        else:
            _need(delta, "delta", (Bz, L, Dm), self.in_dtype, dev)
            _need(A, "A", (Dm, N), torch.float32, dev)
            _need(D, "D", (Dm,), torch.float32, dev)
            _need(z, "z", (Bz, L, Dm), self.in_dtype, dev)
            _need(delta_bias, "delta_bias", (Dm,), torch.float32, dev)
            _need(h0, "h0", (Bz, Dm, N), torch.float32, dev)
            hshape = (Bz, Dm, N)
        _need(x, "x", (Bz, L, Dm), self.in_dtype, dev)
        bshape = (Bz, L, Dm) if f & A_DIRECT else (Bz, L, N)
        _need(B, "B", bshape, self.in_dtype, dev)
        _need(C, "C", bshape, self.in_dtype, dev)
        if y is None:
            y = torch.empty((Bz, L, Dm), dtype=self.out_dtype, device=dev)
        _need(y, "y", (Bz, L, Dm), self.out_dtype, dev)
        if f & WANT_HLAST and h_last is None:
            h_last = torch.empty(hshape, dtype=torch.float32, device=dev)
        _need(h_last, "h_last", hshape, torch.float32, dev)
        rc = self._lib.ssm_scan_fwd(self._h, _ptr(x), _ptr(delta), _ptr(delta_bias), _ptr(A),
                                    _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(h0), _ptr(y),
                                    _ptr(h_last), _stream(dev))
        _check(rc, "ssm_scan_fwd")
        return y, h_last

    def fwd_host(self, x, delta, A, B, C, D=None, z=None, delta_bias=None, h0=None, y=None,
                 h_last=None, chunk_tokens=0, stream=None):
        """Forward pass on CPU tensors (pinned for overlapped copies): the
        library streams the sequence through the plan's device in chunks of
        tokens (ssm_scan_fwd_host).  Returns (y, h_last) as CPU tensors; they
        are complete once `stream` (default: the device's current stream)
        has been synchronised."""
        d, f = self.desc, self.flags
        if f & (A_DIRECT | CONV_X):
            raise ValueError("fwd_host takes neither A_DIRECT nor CONV_X plans")
        Bz, L, Dm, N = d.batch, d.seqlen, d.dim, d.dstate
        cpu = torch.device("cpu")
        for name, t, shape, dt in (("x", x, (Bz, L, Dm), self.in_dtype),
                                   ("delta", delta, (Bz, L, Dm), self.in_dtype),
                                   ("z", z, (Bz, L, Dm), self.in_dtype),
                                   ("B", B, (Bz, L, N), self.in_dtype),
                                   ("C", C, (Bz, L, N), self.in_dtype),
                                   ("A", A, (Dm, N), torch.float32),
                                   ("D", D, (Dm,), torch.float32),
                                   ("delta_bias", delta_bias, (Dm,), torch.float32),
                                   ("h0", h0, (Bz, Dm, N), torch.float32)):
            _need(t, name, shape, dt, cpu)
        if y is None:
            y = torch.empty((Bz, L, Dm), dtype=self.out_dtype).pin_memory()
        _need(y, "y", (Bz, L, Dm), self.out_dtype, cpu)
        if f & WANT_HLAST and h_last is None:
            h_last = torch.empty((Bz, Dm, N), dtype=torch.float32).pin_memory()
        _need(h_last, "h_last", (Bz, Dm, N), torch.float32, cpu)
        st = ctypes.c_void_p(stream.cuda_stream if stream is not None
                             else torch.cuda.current_stream(self.device).cuda_stream)
        rc = self._lib.ssm_scan_fwd_host(self._h, _ptr(x), _ptr(delta), _ptr(delta_bias),
                                         _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(h0),
                                         _ptr(y), _ptr(h_last), int(chunk_tokens), st)
        _check(rc, "ssm_scan_fwd_host")
        return y, h_last

    def fwd_conv(self, x_in, conv_w, delta, A, B, C, conv_b=None, D=None, z=None,
                 delta_bias=None, h0=None, y=None, h_last=None, x_conv=None):
        """Forward pass with the causal conv front-end of the x branch: x_in
        (B, L, D) in_dtype, conv_w (D, 4) fp32, conv_b (D,) fp32.  x_conv,
        when given ((B, L, D) out dtype), receives silu(conv(x_in)).
        Returns (y, h_last)."""
        d, f, dev = self.desc, self.flags, self.device
        if not f & CONV_X:
            raise ValueError("the plan was created without CONV_X")
        Bz, L, Dm, N = d.batch, d.seqlen, d.dim, d.dstate
        _need(x_in, "x_in", (Bz, L, Dm), self.in_dtype, dev)
        _need(conv_w, "conv_w", (Dm, CONV_WIDTH), torch.float32, dev)
        _need(conv_b, "conv_b", (Dm,), torch.float32, dev)
        _need(delta, "delta", (Bz, L, Dm), self.in_dtype, dev)
        _need(A, "A", (Dm, N), torch.float32, dev)
        _need(D, "D", (Dm,), torch.float32, dev)
        _need(z, "z", (Bz, L, Dm), self.in_dtype, dev)
        _need(delta_bias, "delta_bias", (Dm,), torch.float32, dev)
        _need(h0, "h0", (Bz, Dm, N), torch.float32, dev)
        _need(B, "B", (Bz, L, N), self.in_dtype, dev)
        _need(C, "C", (Bz, L, N), self.in_dtype, dev)
        if y is None:
            y = torch.empty((Bz, L, Dm), dtype=self.out_dtype, device=dev)
        _need(y, "y", (Bz, L, Dm), self.out_dtype, dev)
        if f & WANT_HLAST and h_last is None:
            h_last = torch.empty((Bz, Dm, N), dtype=torch.float32, device=dev)
        _need(h_last, "h_last", (Bz, Dm, N), torch.float32, dev)
        _need(x_conv, "x_conv", (Bz, L, Dm), self.out_dtype, dev)
        rc = self._lib.ssm_scan_fwd_conv(self._h, _ptr(x_in), _ptr(conv_w), _ptr(conv_b),
                                         _ptr(delta), _ptr(delta_bias), _ptr(A), _ptr(B),
                                         _ptr(C), _ptr(D), _ptr(z), _ptr(h0), _ptr(y),
                                         _ptr(h_last), _ptr(x_conv), _stream(dev))
        _check(rc, "ssm_scan_fwd_conv")
        return y, h_last

    def seq_map(self, x, delta, A, B, delta_bias=None, map_h=None, map_s=None):
        """Map of the plan's whole sequence: (map_h (B, D, N) = the state
        reached from 0, map_s (B, D) = the sum of Delta), fp32."""
        d, dev = self.desc, self.device
        Bz, L, Dm, N = d.batch, d.seqlen, d.dim, d.dstate
        _need(x, "x", (Bz, L, Dm), self.in_dtype, dev)
        _need(delta, "delta", (Bz, L, Dm), self.in_dtype, dev)
        _need(A, "A", (Dm, N), torch.float32, dev)
        _need(B, "B", (Bz, L, N), self.in_dtype, dev)
        _need(delta_bias, "delta_bias", (Dm,), torch.float32, dev)
        if map_h is None:
            map_h = torch.empty((Bz, Dm, N), dtype=torch.float32, device=dev)
        if map_s is None:
            map_s = torch.empty((Bz, Dm), dtype=torch.float32, device=dev)
        _need(map_h, "map_h", (Bz, Dm, N), torch.float32, dev)
        _need(map_s, "map_s", (Bz, Dm), torch.float32, dev)
        _check(self._lib.ssm_scan_seq_map(self._h, _ptr(x), _ptr(delta), _ptr(delta_bias),
                                          _ptr(A), _ptr(B), _ptr(map_h), _ptr(map_s),
                                          _stream(dev)), "ssm_scan_seq_map")
        return map_h, map_s

    def fold_maps(self, count, maps_h, maps_s, A, h0=None, h_out=None):
        """Compose the first `count` maps (maps_h (>= count, B, D, N), maps_s
        (>= count, B, D)) in order onto h0 (None = 0); returns h (B, D, N)."""
        d, dev = self.desc, self.device
        Bz, Dm, N = d.batch, d.dim, d.dstate
        _need(A, "A", (Dm, N), torch.float32, dev)
        _need(h0, "h0", (Bz, Dm, N), torch.float32, dev)
        for name, t, tail in (("maps_h", maps_h, (Bz, Dm, N)), ("maps_s", maps_s, (Bz, Dm))):
            if count > 0:
                if t.dtype != torch.float32 or t.device != dev or not t.is_contiguous() or \
                        tuple(t.shape[1:]) != tail or t.shape[0] < count:
                    raise ValueError(f"{name} must be contiguous fp32 (>= {count}, {tail})")
        if h_out is None:
            h_out = torch.empty((Bz, Dm, N), dtype=torch.float32, device=dev)
        _need(h_out, "h_out", (Bz, Dm, N), torch.float32, dev)
        _check(self._lib.ssm_scan_fold_maps(self._h, int(count),
                                            _ptr(maps_h) if count > 0 else None,
                                            _ptr(maps_s) if count > 0 else None, _ptr(A),
                                            _ptr(h0), _ptr(h_out), _stream(dev)),
               "ssm_scan_fold_maps")
        return h_out

    def bwd(self, x, delta, A, B, C, dy, D=None, z=None, delta_bias=None, h0=None,
            dh_last=None, want_dh0=True):
        """Gradients of the forward pass for dL/dy = dy (out dtype) and
        dL/dh_last = dh_last (fp32, or None for 0).  Returns a dict of fp32
        tensors keyed like the inputs (x, delta, A, B, C, and D, z,
        delta_bias, h0 where present)."""
        d, f, dev = self.desc, self.flags, self.device
        Bz, L, Dm, N = d.batch, d.seqlen, d.dim, d.dstate
        for name, t in (("x", x), ("delta", delta), ("z", z)):
            _need(t, name, (Bz, L, Dm), self.in_dtype, dev)
        _need(B, "B", (Bz, L, N), self.in_dtype, dev)
        _need(C, "C", (Bz, L, N), self.in_dtype, dev)
        _need(A, "A", (Dm, N), torch.float32, dev)
        _need(D, "D", (Dm,), torch.float32, dev)
        _need(delta_bias, "delta_bias", (Dm,), torch.float32, dev)
        _need(h0, "h0", (Bz, Dm, N), torch.float32, dev)
        _need(dy, "dy", (Bz, L, Dm), self.out_dtype, dev)
        _need(dh_last, "dh_last", (Bz, Dm, N), torch.float32, dev)
        f32 = dict(dtype=torch.float32, device=dev)
        g = {"x": torch.empty((Bz, L, Dm), **f32), "delta": torch.empty((Bz, L, Dm), **f32),
             "A": torch.empty((Dm, N), **f32), "B": torch.empty((Bz, L, N), **f32),
             "C": torch.empty((Bz, L, N), **f32)}
        if D is not None:
            g["D"] = torch.empty((Dm,), **f32)
        if z is not None:
            g["z"] = torch.empty((Bz, L, Dm), **f32)
        if delta_bias is not None:
            g["delta_bias"] = torch.empty((Dm,), **f32)
        if want_dh0:
            g["h0"] = torch.empty((Bz, Dm, N), **f32)
        rc = self._lib.ssm_scan_bwd(self._h, _ptr(x), _ptr(delta), _ptr(delta_bias), _ptr(A),
                                    _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(h0), _ptr(dy),
                                    _ptr(dh_last), _ptr(g["x"]), _ptr(g["delta"]),
                                    _ptr(g.get("delta_bias")), _ptr(g["A"]), _ptr(g["B"]),
                                    _ptr(g["C"]), _ptr(g.get("D")), _ptr(g.get("z")),
                                    _ptr(g.get("h0")), _stream(dev))
        _check(rc, "ssm_scan_bwd")
        return g

    def step(self, state, x, delta, A, B, C, D=None, z=None, delta_bias=None, y=None):
        d, dev = self.desc, self.device
        Bz, Dm, N = d.batch, d.dim, d.dstate
        _need(state, "state", (Bz, Dm, N), torch.float32, dev)
        for name, t in (("x", x), ("delta", delta), ("z", z)):
            _need(t, name, (Bz, Dm), self.in_dtype, dev)
        _need(A, "A", (Dm, N), torch.float32, dev)
        _need(B, "B", (Bz, N), self.in_dtype, dev)
        _need(C, "C", (Bz, N), self.in_dtype, dev)
        _need(D, "D", (Dm,), torch.float32, dev)
        _need(delta_bias, "delta_bias", (Dm,), torch.float32, dev)
        if y is None:
            y = torch.empty((Bz, Dm), dtype=self.out_dtype, device=dev)
        _need(y, "y", (Bz, Dm), self.out_dtype, dev)
        rc = self._lib.ssm_scan_step(self._h, _ptr(x), _ptr(delta), _ptr(delta_bias), _ptr(A),
                                     _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(state), _ptr(y),
                                     _stream(dev))
        _check(rc, "ssm_scan_step")
        return y

    def step_host(self, state, x, delta, A, B, C, D=None, z=None, delta_bias=None, y=None,
                  chunk_rows=0, stream=None):
        """One decode step with the token's inputs and y on the host (CPU
        tensors, pinned for overlapped copies) and the state, A, D,
        delta_bias on the device (ssm_scan_step_host).  Returns y (CPU),
        complete once `stream` (default: the current stream) is synchronised."""
        d, dev = self.desc, self.device
        Bz, Dm, N = d.batch, d.dim, d.dstate
        cpu = torch.device("cpu")
        _need(state, "state", (Bz, Dm, N), torch.float32, dev)
        for name, t in (("x", x), ("delta", delta), ("z", z)):
            _need(t, name, (Bz, Dm), self.in_dtype, cpu)
        _need(B, "B", (Bz, N), self.in_dtype, cpu)
        _need(C, "C", (Bz, N), self.in_dtype, cpu)
        _need(A, "A", (Dm, N), torch.float32, dev)
        _need(D, "D", (Dm,), torch.float32, dev)
        _need(delta_bias, "delta_bias", (Dm,), torch.float32, dev)
        if y is None:
            y = torch.empty((Bz, Dm), dtype=self.out_dtype).pin_memory()
        _need(y, "y", (Bz, Dm), self.out_dtype, cpu)
        st = ctypes.c_void_p(stream.cuda_stream if stream is not None
                             else torch.cuda.current_stream(dev).cuda_stream)
        rc = self._lib.ssm_scan_step_host(self._h, _ptr(x), _ptr(delta), _ptr(delta_bias),
                                          _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                                          _ptr(state), _ptr(y), int(chunk_rows), st)
        _check(rc, "ssm_scan_step_host")
        return y


def list_variants(in_dtype=torch.bfloat16, out_dtype=None) -> list:
    """The compiled variants of the fused kernel for a dtype pair (dicts)."""
    lib = load_library()
    a, b = _TORCH_TO_SSM[in_dtype], _TORCH_TO_SSM[out_dtype or in_dtype]
    n = lib.ssm_scan_list_variants(a, b, None, 0)
    arr = (Variant * max(n, 1))()
    lib.ssm_scan_list_variants(a, b, arr, n)
    return [arr[i].as_dict() for i in range(n)]


def probe_peak(kind: int, iters: int, blocks: int, sink, stream=None) -> int:
    """Launch the library's throughput probe (kind 0 = ex2.approx, 1 = fp32
    FMA) on the current stream; returns the operation count it launched."""
    ops = ctypes.c_int64(0)
    dev = sink.device
    st = ctypes.c_void_p(stream.cuda_stream if stream is not None
                         else torch.cuda.current_stream(dev).cuda_stream)
    _check(load_library().ssm_probe_peak(int(kind), int(iters), int(blocks), _ptr(sink),
                                         ctypes.byref(ops), st), "ssm_probe_peak")
    return ops.value


def probe_exp2(x):
    """The kernels' two 2^x implementations on the fp32 device tensor x:
    returns (FMA-pipe polynomial, ex2.approx) as tensors shaped like x."""
    _need(x, "x", tuple(x.shape), torch.float32, x.device)
    y_fma, y_sfu = torch.empty_like(x), torch.empty_like(x)
    st = ctypes.c_void_p(torch.cuda.current_stream(x.device).cuda_stream)
    _check(load_library().ssm_probe_exp2(_ptr(x), _ptr(y_fma), _ptr(y_sfu), x.numel(), st),
           "ssm_probe_exp2")
    return y_fma, y_sfu


def flags_for(*, z=None, D=None, delta_bias=None, h0=None, delta_softplus=True,
              want_h_last=True, zoh=False, conv=False) -> int:
    return ((HAS_Z if z is not None else 0) | (HAS_D if D is not None else 0)
            | (DELTA_SOFTPLUS if delta_softplus else 0)
            | (HAS_DELTA_BIAS if delta_bias is not None else 0)
            | (HAS_H0 if h0 is not None else 0) | (WANT_HLAST if want_h_last else 0)
            | (ZOH if zoh else 0) | (CONV_X if conv else 0))


_plans: dict = {}
_plans_lock = threading.Lock()


def _plan_for(key, make):
    with _plans_lock:
        p = _plans.get(key)
        if p is None:
            p = make()
            _plans[key] = p
        return p


def fwd(x, delta, A, B, C, D=None, z=None, delta_bias=None, h0=None, delta_softplus=True,
        want_h_last=True, out_dtype=None, zoh=False):
    """Selective-scan forward.  x, delta, z: (B, L, D); B, C: (B, L, N);
    A: (D, N) fp32; D, delta_bias: (D,) fp32; h0: (B, D, N) fp32.
    zoh selects the zero-order-hold input matrix (exp(Delta A) - 1) / A * B.
    Returns (y, h_last) (h_last is None when not requested)."""
    Bz, L, Dm = x.shape
    N = A.shape[1]
    flags = flags_for(z=z, D=D, delta_bias=delta_bias, h0=h0, delta_softplus=delta_softplus,
                      want_h_last=want_h_last, zoh=zoh)
    out_dtype = out_dtype or x.dtype
    key = ("fwd", Bz, L, Dm, N, x.dtype, out_dtype, flags, x.device)
    plan = _plan_for(key, lambda: Plan(Bz, L, Dm, N, x.dtype, out_dtype, flags, x.device))
    return plan.fwd(x, delta, A, B, C, D=D, z=z, delta_bias=delta_bias, h0=h0)


def step(state, x, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
         out_dtype=None, zoh=False):
    """One decode step: updates ``state`` (B, D, N) fp32 in place, returns y (B, D)."""
    Bz, Dm, N = state.shape
    flags = flags_for(z=z, D=D, delta_bias=delta_bias, delta_softplus=delta_softplus,
                      want_h_last=False, zoh=zoh)
    out_dtype = out_dtype or x.dtype
    key = ("step", Bz, Dm, N, x.dtype, out_dtype, flags, x.device)
    plan = _plan_for(key, lambda: Plan(Bz, 1, Dm, N, x.dtype, out_dtype, flags, x.device))
    return plan.step(state, x, delta, A, B, C, D=D, z=z, delta_bias=delta_bias)


def direct(x, A, B, C, h0=None, want_h_last=True, out_dtype=None):
    """Elementwise variant (N = 1, transition A_t given): all of x, A, B, C
    are (B, L, D); h0 (B, D) fp32.  Returns (y, h_last)."""
    Bz, L, Dm = x.shape
    flags = A_DIRECT | (HAS_H0 if h0 is not None else 0) | (WANT_HLAST if want_h_last else 0)
    out_dtype = out_dtype or x.dtype
    key = ("direct", Bz, L, Dm, x.dtype, out_dtype, flags, x.device)
    plan = _plan_for(key, lambda: Plan(Bz, L, Dm, 1, x.dtype, out_dtype, flags, x.device))
    return plan.fwd(x, None, A, B, C, h0=h0)
