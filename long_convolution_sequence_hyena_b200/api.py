"""Torch-facing convenience layer over the C ABI (``capi``).

PyTorch supplies device memory and the current CUDA stream; every step of the
operator runs in ``libhyena.so``. Errors from the library raise ``HyenaError``.
"""
from __future__ import annotations

import torch

from . import capi

_DT = {torch.float32: capi.HYENA_F32, torch.bfloat16: capi.HYENA_BF16}


class HyenaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__("%s failed: %s (%s)" % (what, capi.hyena_status_string(status),
                                                 capi.STATUS_NAMES.get(status, status)))
        self.status = status


def _check(status: int, what: str):
    if status != capi.HYENA_OK:
        raise HyenaError(status, what)


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def implicit_params(p: dict) -> capi.hyena_implicit_params_t:
    """C struct from a dict of device fp32 tensors (W1 b1 W2 b2 W3 b3 and alpha or sigma) and scalars.
    The caller keeps the tensors alive while the struct is used."""
    window = p["alpha"] if "alpha" in p else p["sigma"]
    return capi.hyena_implicit_params_t(
        p["W1"].data_ptr(), p["b1"].data_ptr(), p["W2"].data_ptr(), p["b2"].data_ptr(),
        p["W3"].data_ptr(), p["b3"].data_ptr(), window.data_ptr(),
        int(p["width"]), int(p.get("num_freqs", 0)), float(p["omega0"]), float(p["omega_hidden"]))


class Plan:
    """A plan for one geometry: shape (L,), (H, W) or (Dz, H, W), channels, order, io dtype, and the
    activation layout of 1D plans: "bdl" ([B, D, L], the default) or "bld" ([B, L, D],
    channels-last, read and written in place). radix3: a 1D plan may pad to M = 6 * 2^j
    when that is below the power of two."""

    def __init__(self, shape, channels: int, order: int, dtype=torch.bfloat16, layout: str = "bdl",
                 radix3: bool = False):
        shape = tuple(int(s) for s in shape)
        self.ndim = len(shape)
        self.shape = shape
        self.channels = int(channels)
        self.order = int(order)
        self.dtype = dtype
        st, h = capi.hyena_plan_create_ex(self.ndim, shape, self.channels, self.order, _DT[dtype],
                                          1 if self.ndim == 1 else 0, capi.HYENA_PLAN_RADIX3 if radix3 else 0)
        _check(st, "hyena_plan_create")
        self.handle = h
        st, self.fft_len, self.spectrum_elems, self.path = capi.hyena_plan_info(h)
        _check(st, "hyena_plan_info")
        self.layout = layout
        if layout != "bdl":
            lay = {"bld": capi.HYENA_LAYOUT_BLD}.get(layout)
            if lay is None:
                self.close()
                raise ValueError("layout must be 'bdl' or 'bld'")
            _check(capi.hyena_plan_set_layout(h, lay), "hyena_plan_set_layout")

    def close(self):
        if getattr(self, "handle", None):
            capi.hyena_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def spectrum_shape(self):
        if self.ndim == 1:
            return (self.order, self.channels, self.spectrum_elems)
        if self.ndim == 3:
            return (self.order, self.channels) + tuple(2 * e for e in self.shape)   # bin (kz, ky, kx) natural order
        H, W = self.shape
        return (self.order, self.channels, W + 1, 2 * H)   # bin (ky, kx) at [kx][ky]

    def workspace_bytes(self, batch: int) -> int:
        return capi.hyena_workspace_bytes(self.handle, batch)

    def implicit_filter(self, params: dict, out=None, stream=None):
        if out is None:
            shp = ((self.order, self.channels, self.shape[0]) if self.ndim == 1 else
                   (self.order, self.channels) + tuple(2 * e for e in self.shape))
            out = torch.empty(shp, dtype=torch.float32, device="cuda")
        c = implicit_params(params)
        _check(capi.hyena_implicit_filter(self.handle, c, out.data_ptr(), _stream(stream)), "hyena_implicit_filter")
        return out

    def filter_spectrum(self, h=None, implicit: dict | None = None, out=None, stream=None, workspace=None):
        """Spectra as a complex64 tensor of ``spectrum_shape``. ``workspace``: a uint8 device tensor
        of at least ``spectrum_workspace_bytes()`` for the transforms, so that calls on one plan
        from several threads overlap (None: the plan's own scratch, one call at a time)."""
        if out is None:
            out = torch.empty(self.spectrum_shape, dtype=torch.complex64, device="cuda")
        c = implicit_params(implicit) if implicit is not None else None
        if h is not None:
            h = h.contiguous()
        if workspace is None:
            _check(capi.hyena_filter_spectrum(self.handle, _ptr(h), c, out.data_ptr(), _stream(stream)),
                   "hyena_filter_spectrum")
        else:
            _check(capi.hyena_filter_spectrum_ws(self.handle, _ptr(h), c, out.data_ptr(), workspace.data_ptr(),
                                                 workspace.numel() * workspace.element_size(), _stream(stream)),
                   "hyena_filter_spectrum_ws")
        return out

    def spectrum_workspace_bytes(self) -> int:
        return capi.lib.hyena_filter_spectrum_workspace_bytes(self.handle)

    def forward(self, v, gates, H, dskip=None, out=None, workspace=None, stream=None):
        if out is None:
            out = torch.empty_like(v)
        ws = workspace
        need = self.workspace_bytes(v.shape[0])
        if ws is None and need:
            ws = torch.empty(need, dtype=torch.uint8, device=v.device)
        st = capi.hyena_forward(self.handle, v.shape[0], v.data_ptr(), [g.data_ptr() for g in gates],
                                H.data_ptr(), _ptr(dskip), out.data_ptr(), _ptr(ws),
                                0 if ws is None else ws.numel(), _stream(stream))
        _check(st, "hyena_forward")
        return out

    def forward_gated(self, q, k, gates, H, dskip=None, out=None, workspace=None, stream=None):
        """The HyenaND gate sandwich: y = SiLU(x^N) (K^N * (... SiLU(x^1) (K^1 * (q SiLU(k)))));
        with one order, (K * (q SiLU(k))) SiLU(v) for gates = [v]."""
        if out is None:
            out = torch.empty_like(q)
        ws = workspace
        need = self.workspace_bytes(q.shape[0])
        if ws is None and need:
            ws = torch.empty(need, dtype=torch.uint8, device=q.device)
        st = capi.hyena_forward_gated(self.handle, q.shape[0], q.data_ptr(), k.data_ptr(),
                                      [g.data_ptr() for g in gates], H.data_ptr(), _ptr(dskip), out.data_ptr(),
                                      _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream))
        _check(st, "hyena_forward_gated")
        return out

    def host_workspace_bytes(self, batch: int) -> int:
        return capi.hyena_forward_host_workspace_bytes(self.handle, batch)

    def forward_host(self, v_host, gates_host, H, dskip=None, out=None, workspace=None, stream=None):
        """Forward on page-locked CPU tensors (``tensor.pin_memory()``): the library copies v and
        the gates in and y out, pipelined over the batch, on ``stream``. H and dskip are device
        tensors. Returns the page-locked output; it is complete once ``stream`` reaches the end of
        the call (synchronize before reading it)."""
        if out is None:
            out = torch.empty_like(v_host).pin_memory()
        ws = workspace
        if ws is None:
            ws = torch.empty(max(1, self.host_workspace_bytes(v_host.shape[0])), dtype=torch.uint8, device=H.device)
        st = capi.hyena_forward_host(self.handle, v_host.shape[0], v_host.data_ptr(),
                                     [g.data_ptr() for g in gates_host], H.data_ptr(), _ptr(dskip), out.data_ptr(),
                                     ws.data_ptr(), ws.numel(), _stream(stream))
        _check(st, "hyena_forward_host")
        return out
