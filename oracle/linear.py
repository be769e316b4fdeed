"""Oracle composition of the FP8 delayed-scaling linear layer (test infrastructure only).

The steps follow the pages in their order:

* forward ("CPU Overhead of te.Linear FP8 Layers", repro script; "[PyTorch]
  Refactor FP8 workspaces in linear modules"): cast the input with the scale in
  its meta and record its amax; when the weight cache must be refreshed
  (``is_first_microbatch`` is None or True, or nothing is cached yet) cast the
  weight and its transpose with the weight meta's scale, record the weight amax
  and keep the scale_inv the weight was cast with; then the FP8 GEMM with the
  two private scale_invs (the torch._scaled_mm contract on the PyTorch FP8 page).
* backward (HYBRID format: e4m3 forward tensors, e5m2 gradients): cast the
  output gradient to e5m2 with its transpose and record its amax; dgrad
  dX = dY . W from dY8 and the cached W8^T; wgrad dW = dY^T . X from dY8^T and
  X8^T.
* once per step: the delayed-scaling update over every meta.

GEMM results are exact (fp64); the caller rounds them when a stored dtype is
wanted (``round_bf16`` for bf16 outputs).
"""
import numpy as np

from . import (E4M3, E5M2, cast_transpose_amax, gemm, update_scales)


class OracleMeta:
    """Packed meta of T FP8 tensors: history [H, T], scale [T], scale_inv [T], formats [T]."""

    def __init__(self, fmts, hist_len=16):
        self.fmts = np.ascontiguousarray(fmts, dtype=np.uint8)
        T = self.fmts.size
        self.hist = np.zeros((hist_len, T), np.float32)
        self.scale = np.ones(T, np.float32)
        self.scale_inv = np.ones(T, np.float32)

    def record(self, t, amax):
        self.hist[0, t] = amax

    def update(self, algo=0):
        self.hist, self.scale, self.scale_inv = update_scales(
            self.hist, self.scale, self.scale_inv, self.fmts, algo)


class OracleLinear:
    """One linear layer y = x . W^T + b with an FP8 weight cache."""

    def __init__(self, w, bias, meta_in, meta_w, meta_grad):
        self.w = np.ascontiguousarray(w, dtype=np.float32)      # [out, in] fp32 master
        self.bias = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
        self.meta_in, self.meta_w, self.meta_grad = meta_in, meta_w, meta_grad
        self.w8 = self.w8t = None
        self.w_scale_inv = None

    def _refresh_weight(self, meta):
        t = self.meta_w
        self.w8, self.w8t, am, self.w_scale_inv = cast_transpose_amax(
            self.w, E4M3, meta.scale[t], meta.hist[0, t])
        meta.record(t, am)

    def fwd(self, x, meta, is_first_microbatch=None, rows=None):
        """Returns (y fp64 [rows, out], saved) with saved = (x8, x8t, x_scale_inv)."""
        t = self.meta_in
        x8, x8t, am, x_si = cast_transpose_amax(x, E4M3, meta.scale[t], meta.hist[0, t])
        meta.record(t, am)
        if is_first_microbatch is None or is_first_microbatch or self.w8 is None:
            self._refresh_weight(meta)
        y = gemm(x8, E4M3, self.w8, E4M3, x_si, self.w_scale_inv, self.bias, rows=rows)
        return y, (x8, x8t, x_si)

    def bwd(self, dy, meta, saved, rows_dgrad=None, rows_wgrad=None, want_dgrad=True):
        """Returns (dx fp64 or None, dw fp64, (dy8, dy8t, dy_scale_inv))."""
        x8, x8t, x_si = saved
        t = self.meta_grad
        dy8, dy8t, am, dy_si = cast_transpose_amax(dy, E5M2, meta.scale[t], meta.hist[0, t])
        meta.record(t, am)
        dx = None
        if want_dgrad:
            dx = gemm(dy8, E5M2, self.w8t, E4M3, dy_si, self.w_scale_inv, None, rows=rows_dgrad)
        dw = gemm(dy8t, E5M2, x8t, E4M3, dy_si, x_si, None, rows=rows_wgrad)
        return dx, dw, (dy8, dy8t, dy_si)
