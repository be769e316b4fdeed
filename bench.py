"""Benchmark of the FP8 delayed-scaling linear hot path on B200.

One step = one pass of the whole path over one batch: the forward and
backward of the MLP pair 2048 -> 8192 -> 2048 at 8192 tokens (batch 8 x seq
1024) with the HYBRID recipe (e4m3 forward tensors, e5m2 gradients), weights
recast into the FP8 cache every step (is_first_microbatch=True), and one
multi-tensor delayed-scaling update of all 6 metas (history 16).  The step
is laid out for B200:
- H (fc1's output) and dH (fc2's dgrad) are handed to the next GEMM in FP8.
  The GEMM epilogue casts them with the consumer's delayed scale and records
  the amax (fp8_linear_fwd_ex / fp8_linear_bwd_ex).
- No FP8 transpose is written: the wgrads and dgrads read X8, H8, dY8, dH8
  and the weight caches MN-major, since tcgen05 reads 8-bit operands in
  either order.
The results are identical to the unfused, transpose-based calls.

Per step: 4 casts with amax (X, W1, W2, dY) in 2 launches (the weight-cache
refresh of both linears with X as an extra cast, then dY in the backward),
6 FP8 GEMMs (fwd, dgrad, wgrad of both linears; 1.649 TFLOP), 1 update
launch.  The unfused step (every linear casts its own input and gradient with
transposes, 6 casts in 5 launches) is timed beside it and reported as
"unfused_step".  Under torchrun every rank runs its
own batch (data parallel, weak scaling) and the ranks max-reduce the current
amaxes over NCCL before the update (the amax sync of delayed scaling).

Printed (rank 0, one compact JSON line): whole-job GEMM TFLOP/s of the step,
the cast-transpose-amax workload bf16 [8192, 2048] -> e4m3/e5m2 in GB/s, the
roofline of the dominant kernel (the GEMM) from CUDA events over the timed
region, the end-to-end figure through the public linear API with pinned host
inputs, the TEBlock forward over four microbatches and the 32-block forward
(576 metas), the oracle's CPU baseline on a bounded sample, and the SM clocks
sampled during the timed region.  --detail PATH also writes the per-kernel
breakdown and the notes on how each figure was taken.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from fp8_delayed_scaling_cast_b200 import inputs  # noqa: E402

METRIC = "FP8 GEMM TFLOP/s & cast-transpose-amax GB/s, % of B200 roofline"
TOKENS, HIDDEN, FFN = inputs.TOKENS, inputs.HIDDEN, inputs.MLP_RATIO * inputs.HIDDEN
GEMM_FLOP = 2.0 * TOKENS * FFN * HIDDEN          # every GEMM of the step has this size
STEP_GEMMS = 6
STEP_FLOP = STEP_GEMMS * GEMM_FLOP
# Algorithmic DRAM bytes of the native step's six GEMM launches: both FP8
# operands read once (1 B per element) and the output written once -- FP8
# codes (1 B) for fc1 fwd and fc2 dgrad, bf16 (2 B) for fc2 fwd and fc1
# dgrad, fp32 (4 B) for the wgrads.  Mean per launch.
_T, _H, _F = TOKENS, HIDDEN, FFN
GEMM_ALG_BYTES = (
    (_T * _H + _F * _H + _T * _F)              # fc1 fwd:   X8, W1_8 -> H8
    + (_T * _F + _H * _F + 2 * _T * _H)        # fc2 fwd:   H8, W2_8 -> Y bf16
    + (_T * _H + _F * _H + _T * _F)            # fc2 dgrad: dY8, W2_8 (MN) -> dH8
    + (_H * _T + _F * _T + 4 * _H * _F)        # fc2 wgrad: dY8 (MN), H8 (MN) -> dW2 fp32
    + (_T * _F + _H * _F + 2 * _T * _H)        # fc1 dgrad: dH8, W1_8 (MN) -> dX bf16
    + (_F * _T + _H * _T + 4 * _F * _H)        # fc1 wgrad: dH8 (MN), X8 (MN) -> dW1 fp32
) / 6.0
# cast+transpose+amax algorithmic bytes: read input + write y + write yt
CAST_BYTES = {
    "x": TOKENS * HIDDEN * (4 + 2), "w1": FFN * HIDDEN * (4 + 2), "h": TOKENS * FFN * (2 + 2),
    "w2": HIDDEN * FFN * (4 + 2), "dy": TOKENS * HIDDEN * (2 + 2), "dh": TOKENS * FFN * (2 + 2),
}
STEP_CAST_BYTES = sum(CAST_BYTES.values())
# With the FP8 hand-over, H and dH are cast inside the GEMM epilogues (fc1
# forward, fc2 dgrad), which write FP8 codes + transpose (2 B per element)
# instead of bf16 (2 B): the separate H and dH casts disappear.
FUSED_CASTS = ("x", "w1", "w2", "dy")
# the native step writes no transposes: read input + write y only
CAST_BYTES_NATIVE = {
    "x": TOKENS * HIDDEN * (4 + 1), "w1": FFN * HIDDEN * (4 + 1), "w2": HIDDEN * FFN * (4 + 1),
    "dy": TOKENS * HIDDEN * (2 + 1),
}
STEP_CAST_BYTES_FUSED = sum(CAST_BYTES_NATIVE[k] for k in FUSED_CASTS)
C2_ROWS, C2_COLS = TOKENS, HIDDEN                  # cast-transpose-amax workload
C2_BYTES = C2_ROWS * C2_COLS * (2 + 1 + 1)
META_NAMES = ["fc1.in", "fc1.w", "fc1.grad", "fc2.in", "fc2.w", "fc2.grad"]
META_FMTS = ["e4m3", "e4m3", "e5m2", "e4m3", "e4m3", "e5m2"]


def step_config(world):
    """The workload both arms name in their JSON line."""
    return {
        "workload": "MLP pair 2048->8192->2048 fwd+bwd at 8192 tokens (batch 8 x seq 1024), "
                    "HYBRID delayed scaling, amax history 16, weights recast every step, "
                    "H and dH handed over in FP8 from the GEMM epilogues, no FP8 transposes "
                    "(MN-major operand reads)",
        "tokens": TOKENS, "hidden": HIDDEN, "ffn": FFN, "gemms_per_step": STEP_GEMMS,
        "parallelism": "dp%d" % world,
        "l2": "inputs larger than L2: about 1.5 GB touched per step, X/dY rotate over 2 sets",
    }


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm": p["hbm_gbs"], "bf16": p["bf16_tflops"], "bf16_sus": p["bf16_tflops_sustained"],
                "src": "measured"}
    except Exception:
        return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sus": 1400.0, "src": "fallback"}


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """SM clock and clock-event reasons sampled during the timed region.

    NVML is polled every 2 ms on a host thread; only the samples taken between
    mark_start() and mark_end() (host times around the timed launches and the
    synchronize that ends them) count.  Without NVML it falls back to
    `nvidia-smi -lms 20` over the same window.
    """

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    SMI_FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        import threading
        self.samples = []           # (host time, sm MHz, set of reason names)
        self.t0 = self.t1 = None
        self.max_mhz = None
        self.src = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            uuid = None
        self.uuid = uuid
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.src = "nvml"
        except Exception:
            self.nv = None

    def _poll_nvml(self):
        nv = self.nv
        bits = [(name, getattr(nv, attr)) for name, attr in self.REASONS]
        while not self._stop.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, {n for n, b in bits if r & b}))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        import threading
        if self.nv is not None:
            self._thread = threading.Thread(target=self._poll_nvml, daemon=True)
            self._thread.start()
            return
        cmd = ["nvidia-smi", "--query-gpu=" + self.SMI_FIELDS, "--format=csv,noheader,nounits", "-lms", "20"]
        if self.uuid:
            cmd[1:1] = ["-i", self.uuid]
        try:
            self._out = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
            self._proc = subprocess.Popen(cmd, stdout=self._out, stderr=subprocess.DEVNULL)
            self._proc_t0 = time.perf_counter()
            self.src = "nvidia-smi"
        except Exception:
            self._proc = None

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def _read_smi(self):
        # nvidia-smi lines carry no host time: spread them evenly over the
        # sampler's lifetime and keep those inside the window
        self._proc.terminate()
        try:
            self._proc.wait(timeout=5)
        except Exception:
            self._proc.kill()
        t_end = time.perf_counter()
        self._out.flush()
        self._out.seek(0)
        lines = [ln for ln in self._out.read().splitlines() if ln.count(",") >= 5]
        os.unlink(self._out.name)
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for idx, line in enumerate(lines):
            parts = [p.strip() for p in line.split(",")]
            try:
                mhz, mx = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            self.max_mhz = mx if self.max_mhz is None else max(self.max_mhz, mx)
            t = self._proc_t0 + (t_end - self._proc_t0) * (idx + 0.5) / len(lines)
            self.samples.append((t, mhz, {n for n, v in zip(names, parts[2:6]) if v.lower().startswith("active")}))

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        elif self._proc is not None:
            self._read_smi()
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"]}
        inside = [(m, r) for t, m, r in self.samples
                  if self.t0 is not None and self.t1 is not None and self.t0 <= t <= self.t1]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples in the timed region"],
                    "source": self.src}
        reasons = set()
        for _, r in inside:
            reasons |= r
        return {"sm_mhz": statistics.median(m for m, _ in inside), "sm_min_mhz": min(m for m, _ in inside),
                "sm_max_mhz": self.max_mhz, "samples": len(inside), "reasons": sorted(reasons),
                "source": self.src}


# --------------------------------------------------------------- the step --

class MlpStep:
    """Device state of the MLP-pair training step (all buffers preallocated).

    Two layouts of the same step:
    - native (the headline): H and dH pass between the linears in FP8 from the
      GEMM epilogues, and no FP8 transpose exists anywhere -- casts write no
      yt, weight caches no w8t, and the wgrads / dgrads read X8, H8, dY8, dH8
      and the weights MN-major (fc1n, fc2n: linears without transposes);
    - unfused: every linear casts its own input and gradient with their
      transposes and reads K-major operands only (fc1, fc2), the layout of
      the pages' Hopper-era designs.
    """

    def __init__(self, fp8, device, n_input_sets=2, seed=0):
        self.fp8 = fp8
        dev = device
        w1, b1, w2, b2 = inputs.mlp_pair(seed)
        w1, b1, w2, b2 = w1.to(dev), b1.to(dev), w2.to(dev), b2.to(dev)
        self.meta = fp8.Fp8Meta(META_FMTS, hist_len=16, device=dev)
        self.fc1 = fp8.Fp8Linear(w1, b1, 0, 1, 2)
        self.fc2 = fp8.Fp8Linear(w2, b2, 3, 4, 5)
        self.fc1n = fp8.Fp8Linear(w1, b1, 0, 1, 2, transpose=False)
        self.fc2n = fp8.Fp8Linear(w2, b2, 3, 4, 5, transpose=False)
        self.host_inputs = [inputs.mlp_step_inputs(s, seed) for s in range(n_input_sets)]
        self.xs = [x.to(dev) for x, _ in self.host_inputs]
        self.dys = [dy.to(dev) for _, dy in self.host_inputs]
        u8, bf, f32 = torch.uint8, torch.bfloat16, torch.float32
        e = lambda *s, dt=u8: torch.empty(*s, dtype=dt, device=dev)  # noqa: E731
        self.x8, self.x8t = e(TOKENS, HIDDEN), e(HIDDEN, TOKENS)
        self.h = e(TOKENS, FFN, dt=bf)
        self.h8, self.h8t = e(TOKENS, FFN), e(FFN, TOKENS)
        self.y = e(TOKENS, HIDDEN, dt=bf)
        self.dy8, self.dy8t = e(TOKENS, HIDDEN), e(HIDDEN, TOKENS)
        self.dh = e(TOKENS, FFN, dt=bf)
        self.dh8, self.dh8t = e(TOKENS, FFN), e(FFN, TOKENS)
        self.dx = e(TOKENS, HIDDEN, dt=bf)
        self.dw1 = e(FFN, HIDDEN, dt=f32)
        self.dw2 = e(HIDDEN, FFN, dt=f32)
        self.si = e(4, dt=f32)  # private scale_invs of x8, h8, dy8, dh8
        # the native step casts X, W1 and W2 in one launch: the weight-cache
        # refresh of both linears with X as an extra cast (job arrays built once)
        self.group = fp8.LinearGroup([self.fc1n, self.fc2n])
        self._xjobs = {}

    def xjob(self, x):
        """The X cast of the native step as a job array (built once per input
        buffer)."""
        key = x.data_ptr()
        if key not in self._xjobs:
            amax = self.meta.amax_history[0]
            self._xjobs[key] = (x, self.fp8.cast_jobs([self.fp8.cast_job(x, "e4m3", self.meta.scale[0:1], self.x8,
                                                                         None, amax[0:1], self.si[0:1])]))
        return self._xjobs[key][1]

    def run_linear_api(self, i, sync_amax=None, fused=True):
        """The step through the public linear API (what a user calls).  fused:
        the native step (fp8_linear_fwd_ex / fp8_linear_bwd_ex, FP8 hand-over,
        no transposes); otherwise the unfused step (fp8_linear_fwd / bwd)."""
        fp8, m = self.fp8, self.meta
        x, dy = self.xs[i % len(self.xs)], self.dys[i % len(self.dys)]
        if fused:
            fc1, fc2 = self.fc1n, self.fc2n
            fp8.fp8_linear_refresh_weights(self.group, m, self.xjob(x))
            fp8.fp8_linear_fwd_ex(fc1, m, None, None, False, self.x8, None, self.si[0:1], in_cast=True,
                                  out_meta=3, out8=self.h8, out_scale_inv=self.si[1:2])
            fp8.fp8_linear_fwd_ex(fc2, m, None, self.y, False, self.h8, None, self.si[1:2], in_cast=True)
            fp8.fp8_linear_bwd_ex(fc2, m, dy, None, self.si[1:2], self.dw2, self.dy8, None, self.si[2:3],
                                  out_meta=2, out8=self.dh8, out_scale_inv=self.si[3:4], x8=self.h8)
            fp8.fp8_linear_bwd_ex(fc1, m, None, None, self.si[0:1], self.dw1, self.dh8, None, self.si[3:4],
                                  dx=self.dx, in_cast=True, x8=self.x8)
            if sync_amax is not None:
                sync_amax(m)
            m.update()
            return
        fp8.fp8_linear_fwd(self.fc1, m, x, self.h, True, self.x8, self.x8t, self.si[0:1])
        fp8.fp8_linear_fwd(self.fc2, m, self.h, self.y, True, self.h8, self.h8t, self.si[1:2])
        fp8.fp8_linear_bwd(self.fc2, m, dy, self.h8t, self.si[1:2], self.dw2, self.dy8, self.dy8t,
                           self.si[2:3], dx=self.dh)
        fp8.fp8_linear_bwd(self.fc1, m, self.dh, self.x8t, self.si[0:1], self.dw1, self.dh8, self.dh8t,
                           self.si[3:4], dx=self.dx)
        if sync_amax is not None:
            sync_amax(m)
        m.update()

    def run_casts(self, i):
        """The native step's delayed-scaling casts alone (X, W1 and W2 from
        fp32 in one launch, as the step issues them; dY from bf16; y only, no
        transpose), on step i's inputs."""
        fp8, m, fc2 = self.fp8, self.meta, self.fc2n
        x, dy = self.xs[i % len(self.xs)], self.dys[i % len(self.dys)]
        amax = m.amax_history[0]
        fp8.fp8_linear_refresh_weights(self.group, m, self.xjob(x))
        fp8.fp8_cast_transpose_amax(dy, "e5m2", m.scale[5:6], self.dy8, None, amax[5:6], self.si[2:3])

    def run_gemms(self):
        """The native step's six GEMM launches alone, in step order, on the
        step's own operands, outputs, layouts and epilogues, with nothing
        between them."""
        fp8, m, fc1, fc2 = self.fp8, self.meta, self.fc1n, self.fc2n
        fp8.fp8_gemm_cast(self.x8, "e4m3", self.si[0:1], fc1.w8, "e4m3", fc1.w_scale_inv, "e4m3", m.scale[3:4],
                          self.h8, None, m.amax_history[0, 3:4], self.si[1:2], bias=fc1.bias)
        fp8.fp8_gemm(self.h8, "e4m3", self.si[1:2], fc2.w8, "e4m3", fc2.w_scale_inv, self.y, bias=fc2.bias)
        fp8.fp8_gemm_cast(self.dy8, "e5m2", self.si[2:3], fc2.w8, "e4m3", fc2.w_scale_inv, "e5m2", m.scale[2:3],
                          self.dh8, None, m.amax_history[0, 2:3], self.si[3:4], b_major="mn")
        fp8.fp8_gemm_major(self.dy8, "e5m2", "mn", self.si[2:3], self.h8, "e4m3", "mn", self.si[1:2], self.dw2)
        fp8.fp8_gemm_major(self.dh8, "e5m2", "k", self.si[3:4], fc1.w8, "e4m3", "mn", fc1.w_scale_inv, self.dx)
        fp8.fp8_gemm_major(self.dh8, "e5m2", "mn", self.si[3:4], self.x8, "e4m3", "mn", self.si[0:1], self.dw1)

    def run_kernels(self, i, ev=None, sync_amax=None):
        """The native step's launches, one C call per kernel so that CUDA
        events can bracket each one.  ev(kind, key) returns a callable
        recorded after the launch, or None."""
        fp8, m = self.fp8, self.meta
        x, dy = self.xs[i % len(self.xs)], self.dys[i % len(self.dys)]
        mark = ev if ev is not None else (lambda kind, key: None)

        def timed(kind, key, fn):
            h0 = mark(kind, key)
            fn()
            if h0:
                h0()

        fc1, fc2 = self.fc1n, self.fc2n
        amax = m.amax_history[0]
        # X, W1 and W2 in one launch
        timed("cast", "x+w1+w2", lambda: fp8.fp8_linear_refresh_weights(self.group, m, self.xjob(x)))
        timed("gemm", "fc1.fwd", lambda: fp8.fp8_gemm_cast(
            self.x8, "e4m3", self.si[0:1], fc1.w8, "e4m3", fc1.w_scale_inv, "e4m3", m.scale[3:4], self.h8, None,
            amax[3:4], self.si[1:2], bias=fc1.bias))
        timed("gemm", "fc2.fwd", lambda: fp8.fp8_gemm(self.h8, "e4m3", self.si[1:2], fc2.w8, "e4m3",
                                                       fc2.w_scale_inv, self.y, bias=fc2.bias))
        timed("cast", "dy", lambda: fp8.fp8_cast_transpose_amax(dy, "e5m2", m.scale[5:6], self.dy8, None, amax[5:6],
                                                                 self.si[2:3]))
        timed("gemm", "fc2.dgrad", lambda: fp8.fp8_gemm_cast(
            self.dy8, "e5m2", self.si[2:3], fc2.w8, "e4m3", fc2.w_scale_inv, "e5m2", m.scale[2:3], self.dh8, None,
            amax[2:3], self.si[3:4], b_major="mn"))
        timed("gemm", "fc2.wgrad", lambda: fp8.fp8_gemm_major(self.dy8, "e5m2", "mn", self.si[2:3], self.h8, "e4m3",
                                                               "mn", self.si[1:2], self.dw2))
        timed("gemm", "fc1.dgrad", lambda: fp8.fp8_gemm_major(self.dh8, "e5m2", "k", self.si[3:4], fc1.w8, "e4m3",
                                                               "mn", fc1.w_scale_inv, self.dx))
        timed("gemm", "fc1.wgrad", lambda: fp8.fp8_gemm_major(self.dh8, "e5m2", "mn", self.si[3:4], self.x8, "e4m3",
                                                               "mn", self.si[0:1], self.dw1))
        if sync_amax is not None:
            sync_amax(m)
        timed("update", "update", m.update)


class TeblockForward:
    """Forward of `blocks` TEBlocks (six linears each: 2048 -> 12288 (+bias),
    6144, 2048, 4096, 8192 (+bias), and 8192 -> 2048 (+bias)) at 8192 tokens,
    fp32 master weights ~ N(0, 0.02) and input X ~ U[0,1) fp32 drawn on the
    device from a seeded generator, bf16 outputs, HYBRID e4m3, history 16.
    The path per block, through the public API:
      - one fp8_cast_transpose_amax_multi launch casts X for the five K = 2048
        linears, each with its own meta (the pages' te.Linear casts its own
        input);
      - the six GEMMs (fp8_linear_fwd_ex with in_cast); fc1 hands H to fc2 in
        FP8 from its epilogue (no bf16 H, no separate H cast);
    plus, per step, the weight-cache refresh of every linear in one launch
    (fp8_linear_refresh_weights) when the weights are recast, and one
    fp8_update_scales over all 18 * blocks metas.  Native B200 layout: no FP8
    transposes (the backward would read X8, H8 and the weights MN-major)."""

    def __init__(self, fp8, device, blocks, seed=0):
        self.fp8 = fp8
        L = 6 * blocks
        self.blocks = blocks
        self.meta = fp8.Fp8Meta(["e4m3", "e4m3", "e5m2"] * L, hist_len=16, device=device)
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        self.lins = []
        for i in range(L):
            out_f, in_f, has_bias = inputs.TEBLOCK_LINEARS[i % 6]
            w = torch.randn(out_f, in_f, generator=g, device=device) * 0.02
            bias = torch.randn(out_f, generator=g, device=device) * 0.02 if has_bias else None
            self.lins.append(fp8.Fp8Linear(w, bias, 3 * i, 3 * i + 1, 3 * i + 2, transpose=False))
        self.group = fp8.LinearGroup(self.lins)
        self.x = torch.rand(TOKENS, HIDDEN, generator=g, device=device)
        u8, bf = torch.uint8, torch.bfloat16
        self.x8 = [torch.empty(TOKENS, HIDDEN, dtype=u8, device=device) for _ in range(5)]
        self.h8 = torch.empty(TOKENS, FFN, dtype=u8, device=device)
        self.ys = [torch.empty(TOKENS, out_f, dtype=bf, device=device) for out_f, _, _ in inputs.TEBLOCK_LINEARS]
        self.si = torch.zeros(6, dtype=torch.float32, device=device)   # private scale_invs of the inputs
        amax = self.meta.amax_history[0]
        self.xjobs = []
        for b in range(blocks):
            jobs = []
            for j in range(5):
                t = 3 * (6 * b + j)
                jobs.append(fp8.cast_job(self.x, "e4m3", self.meta.scale[t:t + 1], self.x8[j], None,
                                         amax[t:t + 1], self.si[j:j + 1]))
            self.xjobs.append(fp8.cast_jobs(jobs))
        self.flop = blocks * sum(2.0 * TOKENS * o * i for o, i, _ in inputs.TEBLOCK_LINEARS)

    def launches(self, refresh):
        return (1 if refresh else 0) + self.blocks * (1 + 6) + 1

    def run(self, refresh):
        fp8, m = self.fp8, self.meta
        if refresh:
            fp8.fp8_linear_refresh_weights(self.group, m)
        for b in range(self.blocks):
            fp8.fp8_cast_transpose_amax_multi(self.xjobs[b])
            lins = self.lins[6 * b:6 * b + 6]
            for j in range(4):
                fp8.fp8_linear_fwd_ex(lins[j], m, None, self.ys[j], False, self.x8[j], None, self.si[j:j + 1],
                                      in_cast=True)
            fp8.fp8_linear_fwd_ex(lins[4], m, None, None, False, self.x8[4], None, self.si[4:5], in_cast=True,
                                  out_meta=lins[5]._c.meta_in, out8=self.h8, out_scale_inv=self.si[5:6])
            fp8.fp8_linear_fwd_ex(lins[5], m, None, self.ys[5], False, self.h8, None, self.si[5:6], in_cast=True)
        m.update()


def time_teblock_microbatches(fp8, device, rounds):
    """The TEBlock forward over 4 microbatches (is_first_microbatch True, then
    False x3: the weight caches are refreshed at microbatch 0 and reused), the
    update after each microbatch; CUDA events around every microbatch, over
    `rounds` rounds after one warm-up round."""
    tb = TeblockForward(fp8, device, blocks=1)
    for mb in range(4):
        tb.run(mb == 0)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(rounds)]
    for r in range(rounds):
        ev[r][0].record()
        for mb in range(4):
            tb.run(mb == 0)
            ev[r][mb + 1].record()
    torch.cuda.synchronize()
    per_mb = [[ev[r][mb].elapsed_time(ev[r][mb + 1]) for r in range(rounds)] for mb in range(4)]
    refresh_ms = statistics.mean(per_mb[0])
    reuse_ms = statistics.mean(per_mb[1] + per_mb[2] + per_mb[3])
    out = {"refresh_mb_ms": refresh_ms, "reuse_mb_ms": reuse_ms,
           "reuse_tflops": tb.flop / (reuse_ms * 1e-3) / 1e12, "refresh_tflops": tb.flop / (refresh_ms * 1e-3) / 1e12,
           "launches_refresh_mb": tb.launches(True), "launches_reuse_mb": tb.launches(False)}
    del tb
    torch.cuda.empty_cache()
    return out


def time_toy_model(fp8, device, steps):
    """The 32-block forward (192 linears, 576 metas, weights recast every
    step): device ms per step issued eagerly, the host time to issue one
    step into an idle queue (median of 3), and the same step captured once in
    a CUDA graph and replayed (device ms and host us per replay)."""
    toy = TeblockForward(fp8, device, blocks=32)
    for _ in range(2):
        toy.run(True)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        toy.run(True)
    e1.record()
    torch.cuda.synchronize()
    eager_ms = e0.elapsed_time(e1) / steps
    # host time to issue one step into an idle queue (back to back, the
    # launch queue fills and the host waits on the GPU)
    host = []
    for _ in range(3):
        torch.cuda.synchronize()
        h0 = time.perf_counter()
        toy.run(True)
        host.append(time.perf_counter() - h0)
    torch.cuda.synchronize()
    host_s = statistics.median(host) * steps
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        toy.run(True)
    graph.replay()
    torch.cuda.synchronize()
    e0.record()
    h0 = time.perf_counter()
    for _ in range(steps):
        graph.replay()
    ghost_s = time.perf_counter() - h0
    e1.record()
    torch.cuda.synchronize()
    graph_ms = e0.elapsed_time(e1) / steps
    status = fp8.fp8ds_device_status()
    out = {"ms_per_step": eager_ms, "tflops": toy.flop / (eager_ms * 1e-3) / 1e12,
           "host_us_per_step": 1e6 * host_s / steps, "graph_ms_per_step": graph_ms,
           "graph_host_us_per_step": 1e6 * ghost_s / steps, "launches_per_step": toy.launches(True),
           "device_status": status}
    del graph, toy
    torch.cuda.empty_cache()
    return out


# native step: 2 cast launches (X with W1 and W2, dY), 6 GEMMs, 1 update
LAUNCHES_PER_STEP = 2 + 6 + 1
# unfused step: X with W1, H, W2, dY, dH casts, 6 GEMMs, 1 update
LAUNCHES_PER_STEP_UNFUSED = 5 + 6 + 1


class EventLog:
    """Pairs of CUDA events recorded on the launching (current) stream."""

    def __init__(self):
        self.pairs = []

    def __call__(self, kind, key):
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        self.pairs.append((kind, key, s, e))
        return e.record

    def summary(self):
        out = {}
        for kind, key, s, e in self.pairs:
            out.setdefault(kind, []).append((key, s.elapsed_time(e)))
        return out


def barrier_sync(world):
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()


def max_over_ranks(v, world, device):
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------- measurements --

def graph_time_us(run, reps):
    """Mean device time per call of run(i), i = 0 .. reps-1, with the calls
    captured once in a CUDA graph and the graph replayed between two CUDA
    events on the launching stream.  Short kernels issued one by one from
    Python wait on the host (about 10-17 us per call on these boxes); in the
    graph they run back to back as they would behind a long kernel."""
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(reps):
            run(i)
    graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    graph.replay()
    e1.record()
    torch.cuda.synchronize()
    del graph
    return 1e3 * e0.elapsed_time(e1) / reps


def host_issue_time_us(run, reps):
    """The same calls issued one by one from Python, CUDA events around the
    loop: the host's per-call cost when it exceeds the kernel's."""
    for i in range(3):
        run(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(reps):
        run(i)
    e1.record()
    torch.cuda.synchronize()
    return 1e3 * e0.elapsed_time(e1) / reps


def time_cast_workload(fp8, device, reps=100):
    """bf16 [8192, 2048] (0.1% spikes) -> e4m3 and e5m2 with transpose and amax,
    over 8 rotating input buffers (268 MB > L2); per-launch device times of
    graph-replayed launches, plus the host-issued loop for context."""
    base = inputs.spiky_bf16().to(device)
    xs = [base] + [base.roll(i * 17, dims=1).contiguous() for i in range(1, 8)]
    y = torch.empty(C2_ROWS, C2_COLS, dtype=torch.uint8, device=device)
    yt = torch.empty(C2_COLS, C2_ROWS, dtype=torch.uint8, device=device)
    s = torch.ones(1, device=device)
    am = torch.zeros(1, device=device)
    si = torch.zeros(1, device=device)
    res = {}
    for fmt in ("e4m3", "e5m2"):
        def cast(i, fmt=fmt):
            fp8.fp8_cast_transpose_amax(xs[i % 8], fmt, s, y, yt, am, si)
        for i in range(5):
            cast(i)
        res[fmt] = {"us_mean": graph_time_us(cast, reps), "us_host_issued": host_issue_time_us(cast, reps)}
    # dynamic scaling of the same tensors (amax pass, scale, cast: the input
    # is read twice) for comparison with the delayed cast above
    sd = torch.ones(1, device=device)

    def dyn(i):
        fp8.fp8_cast_transpose_amax_dynamic(xs[i % 8], "e4m3", sd, y, yt, am, si)
    for i in range(5):
        dyn(i)
    res["dynamic_e4m3"] = {"us_mean": graph_time_us(dyn, reps)}
    return res


def time_update_576(fp8, device, reps=200):
    """One fp8_update_scales launch over the 576 metas of the 32-block model
    (32 blocks x 6 linears x input/weight/grad), history 16, launched back to
    back from a CUDA graph (the history starts filled with amaxes; every
    launch reads and rewrites all 16 slots of every meta).  Mean per launch."""
    T = 32 * 6 * 3
    meta = fp8.Fp8Meta(["e4m3", "e4m3", "e5m2"] * (T // 3), hist_len=16, device=device)
    g = torch.Generator(device="cpu").manual_seed(11)
    meta.amax_history.copy_(torch.rand(16, T, generator=g).to(device) * 10)
    for _ in range(10):
        meta.update()
    return graph_time_us(lambda i: meta.update(), reps)


def time_headline_gemm(fp8, device, reps=50, warmup=10):
    """8192x2048x8192 and 8192x8192x2048 e4m3 GEMMs (bf16 out), timed alone:
    10 warm-up and 50 timed launches.  torch._scaled_mm (a library GEMM) is
    timed on the same operands as context only; it is not part of the path."""
    out = {}
    for (M, N, K) in [(8192, 2048, 8192), (8192, 8192, 2048)]:
        g = torch.Generator(device="cpu").manual_seed(3)
        a = torch.randint(0, 0x7F, (M, K), generator=g, dtype=torch.uint8).to(device)
        b = torch.randint(0, 0x7F, (N, K), generator=g, dtype=torch.uint8).to(device)
        sa = torch.full((1,), 2.0 ** -10, device=device)
        d = torch.empty(M, N, dtype=torch.bfloat16, device=device)

        def timed(fn):
            for _ in range(warmup):
                fn()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record()
            for _ in range(reps):
                fn()
            e1.record()
            torch.cuda.synchronize()
            return 1e3 * e0.elapsed_time(e1) / reps

        us = timed(lambda: fp8.fp8_gemm(a, "e4m3", sa, b, "e4m3", sa, d))
        row = {"us_mean": us, "tflops": 2.0 * M * N * K / (us * 1e-6) / 1e12}
        try:
            a8, b8 = a.view(torch.float8_e4m3fn), b.view(torch.float8_e4m3fn)
            s0 = sa.reshape(())
            us_lib = timed(lambda: torch._scaled_mm(a8, b8.t(), scale_a=s0, scale_b=s0, out_dtype=torch.bfloat16))
            row["context_torch_scaled_mm"] = {"us_mean": us_lib,
                                              "tflops": 2.0 * M * N * K / (us_lib * 1e-6) / 1e12}
        except Exception as exc:  # context only
            row["context_torch_scaled_mm"] = {"unavailable": str(exc)[:120]}
        out["%dx%dx%d" % (M, N, K)] = row
    return out


class OracleStepSample:
    """The oracle's pass over the whole path on a sample of the workload: the
    same MLP-pair step at `tokens` of the 8192 tokens, full weights (weight
    casts, both forward GEMMs, dgrads, wgrads, grad casts, the update).
    Inputs are drawn once; run() returns (GEMM FLOP computed, seconds)."""

    def __init__(self, tokens=128, seed=0):
        w1, b1, w2, b2 = inputs.mlp_pair(seed)
        x, dy = inputs.mlp_step_inputs(0, seed)
        self.tokens = tokens
        self.w1, self.b1, self.w2, self.b2 = w1.numpy(), b1.numpy(), w2.numpy(), b2.numpy()
        self.x = x[:tokens].numpy().copy()
        self.dyb = inputs.bf16_bits(dy[:tokens]).copy()
        self.cores = 1  # the oracle is single-threaded C

    def run(self):
        import oracle as o
        t0 = time.perf_counter()
        meta = o.OracleMeta([0, 0, 1, 0, 0, 1], 16)
        fc1 = o.OracleLinear(self.w1, self.b1, 0, 1, 2)
        fc2 = o.OracleLinear(self.w2, self.b2, 3, 4, 5)
        h, s1 = fc1.fwd(self.x, meta, True)
        _, s2 = fc2.fwd(o.round_bf16(h), meta, True)
        dh, _, _ = fc2.bwd(self.dyb, meta, s2)
        fc1.bwd(o.round_bf16(dh), meta, s1)
        meta.update()
        dt = time.perf_counter() - t0
        return 6 * 2.0 * self.tokens * FFN * HIDDEN, dt


def e2e_linear_api(fp8, step, device, steps, warmup):
    """End to end through the public linear API: every step copies its X (fp32)
    and dY (bf16) from pinned host memory (side stream, double-buffered) and
    reads the updated meta (history, scales) back to the host."""
    hx = [x.pin_memory() for x, _ in step.host_inputs]
    hdy = [dy.pin_memory() for _, dy in step.host_inputs]
    dx_buf = [torch.empty_like(step.xs[0]) for _ in range(2)]
    ddy_buf = [torch.empty_like(step.dys[0]) for _ in range(2)]
    meta_host = torch.empty(step.meta.amax_history.numel() + 2 * step.meta.num_tensors,
                            dtype=torch.float32).pin_memory()
    copy = torch.cuda.Stream(device)
    comp = torch.cuda.current_stream(device)
    ready = [torch.cuda.Event() for _ in range(2)]
    free = [torch.cuda.Event() for _ in range(2)]
    for j in range(2):
        free[j].record(comp)
    saved_x, saved_dy = step.xs, step.dys
    h2d = hx[0].numel() * 4 + hdy[0].numel() * 2
    d2h = meta_host.numel() * 4

    def issue_copy(i):
        j = i % 2
        with torch.cuda.stream(copy):
            copy.wait_event(free[j])
            dx_buf[j].copy_(hx[i % len(hx)], non_blocking=True)
            ddy_buf[j].copy_(hdy[i % len(hdy)], non_blocking=True)
            ready[j].record(copy)

    def one(i):
        j = i % 2
        comp.wait_event(ready[j])
        step.xs, step.dys = [dx_buf[j]], [ddy_buf[j]]
        step.run_linear_api(0)
        free[j].record(comp)
        n = step.meta.amax_history.numel()
        T = step.meta.num_tensors
        meta_host[:n].copy_(step.meta.amax_history.view(-1), non_blocking=True)
        meta_host[n:n + T].copy_(step.meta.scale, non_blocking=True)
        meta_host[n + T:].copy_(step.meta.scale_inv, non_blocking=True)

    issue_copy(0)
    for i in range(warmup):
        issue_copy(i + 1)
        one(i)
    torch.cuda.synchronize()
    issue_copy(0)
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(comp)
    for i in range(steps):
        if i + 1 < steps:
            issue_copy(i + 1)
        one(i)
    e.record(comp)
    torch.cuda.synchronize()
    step.xs, step.dys = saved_x, saved_dy
    ms = s.elapsed_time(e) / steps
    return ms, h2d, d2h


TRAFFIC_PROFILE = os.path.join("profiles", "gemm_traffic_mlp_pair_step.md")
GEMM_SOURCE = os.path.join("fp8_delayed_scaling_cast_b200", "csrc", "gemm_sm100.cu")


def committed_gemm_traffic(root):
    """Mean DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per GEMM
    launch of the step, from the committed ncu summary -- only if that capture
    was taken on the current GEMM source (its SHA-256 is recorded beside the
    number); otherwise None and the reason."""
    import hashlib
    try:
        text = open(os.path.join(root, TRAFFIC_PROFILE)).read()
        sha = hashlib.sha256(open(os.path.join(root, GEMM_SOURCE), "rb").read()).hexdigest()
    except OSError:
        return None, "no capture"
    fields = {}
    for line in text.splitlines():
        if ":" in line and line.split(":", 1)[0] in ("gemm_source_sha256", "traffic_bytes_per_launch"):
            k, v = line.split(":", 1)
            fields[k] = v.strip()
    if fields.get("gemm_source_sha256") != sha:
        return None, "GEMM source changed since the ncu capture"
    return float(fields["traffic_bytes_per_launch"]), "ncu capture of the step's 6 GEMM launches (%s)" % TRAFFIC_PROFILE


def time_graph_step(step, steps, device):
    """The fused step captured once in a CUDA graph and replayed `steps` times
    (no host work per step beyond the replay call).  The graph reads the
    first input set.  Blocks of graph replays alternate with blocks of the
    same step issued eagerly on the same input set, so that both see the
    same clock (the power cap lowers it as the run goes on); the SM clock is
    sampled over the section.  Returns device ms per step for both, and the
    host us per replay."""
    saved = step.xs, step.dys
    step.xs, step.dys = saved[0][:1], saved[1][:1]
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step.run_linear_api(0)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(device)
    clocks.start()
    time.sleep(0.1)
    clocks.mark_start()
    graph_ms, eager_ms, host_s = [], [], 0.0
    for _ in range(2):
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(steps):
            step.run_linear_api(0)
        e.record()
        torch.cuda.synchronize()
        eager_ms.append(s.elapsed_time(e) / steps)
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        h0 = time.perf_counter()
        s.record()
        for _ in range(steps):
            graph.replay()
        e.record()
        host_s += time.perf_counter() - h0
        torch.cuda.synchronize()
        graph_ms.append(s.elapsed_time(e) / steps)
    clocks.mark_end()
    clock_info = clocks.stop()
    step.xs, step.dys = saved
    del graph
    ms = statistics.mean(graph_ms)
    return {"ms_per_step": ms, "value": STEP_FLOP / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "host_us_per_step": 1e6 * host_s / (2 * steps),
            "eager_same_section_ms_per_step": statistics.mean(eager_ms),
            "blocks_ms": {"eager": eager_ms, "graph": graph_ms}, "clocks": clock_info}


def single_kernel(args):
    """One kernel alone on its workload: 2 warm-up launches then --reps timed
    ones (used under ncu with -s 2)."""
    from fp8_delayed_scaling_cast_b200 import binding as fp8
    dev = torch.device("cuda", 0)
    if args.kernel == "castmulti":
        # the step's X, W1 and W2 casts (fp32 [8192, 2048], [8192, 2048],
        # [2048, 8192] -> e4m3, y only) in one fp8_cast_transpose_amax_multi
        # launch; 201 MB read per launch, more than L2
        g = torch.Generator(device=dev)
        g.manual_seed(5)
        srcs = [torch.rand(TOKENS, HIDDEN, generator=g, device=dev),
                torch.randn(FFN, HIDDEN, generator=g, device=dev) * 0.02,
                torch.randn(HIDDEN, FFN, generator=g, device=dev) * 0.02]
        outs = [torch.empty(t.shape, dtype=torch.uint8, device=dev) for t in srcs]
        sc = torch.ones(3, device=dev)
        am = torch.zeros(3, device=dev)
        si = torch.zeros(3, device=dev)
        jobs = fp8.cast_jobs([fp8.cast_job(t, "e4m3", sc[i:i + 1], o, None, am[i:i + 1], si[i:i + 1])
                              for i, (t, o) in enumerate(zip(srcs, outs))])
        run = lambda: fp8.fp8_cast_transpose_amax_multi(jobs)  # noqa: E731
        work, unit = sum(t.numel() * 5 for t in srcs) / 1e9, "GB/s"
    elif args.kernel in ("gemm", "gemmcast"):
        M, N, K = (int(v) for v in args.shape.split("x"))
        g = torch.Generator(device="cpu").manual_seed(3)
        a = torch.randint(0, 0x7F, (M, K), generator=g, dtype=torch.uint8).to(dev)
        b = torch.randint(0, 0x7F, (N, K), generator=g, dtype=torch.uint8).to(dev)
        sa = torch.full((1,), 2.0 ** -10, device=dev)
        if args.kernel == "gemm":
            d = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            am, bm = args.major.split(",")
            if (am, bm) == ("k", "k"):
                run = lambda: fp8.fp8_gemm(a, "e4m3", sa, b, "e4m3", sa, d)  # noqa: E731
            else:
                a_st = a.t().contiguous() if am == "mn" else a      # stored [K, M]
                b_st = b.t().contiguous() if bm == "mn" else b      # stored [K, N]
                run = lambda: fp8.fp8_gemm_major(a_st, "e4m3", am, sa, b_st, "e4m3", bm, sa, d)  # noqa: E731
        else:
            # FP8 output and amax (the native step's hand-over epilogue: no transpose)
            d8 = torch.empty(M, N, dtype=torch.uint8, device=dev)
            so = torch.full((1,), 0.5, device=dev)
            am = torch.zeros(1, device=dev)
            si = torch.zeros(1, device=dev)
            run = lambda: fp8.fp8_gemm_cast(a, "e4m3", sa, b, "e4m3", sa, "e4m3", so, d8, None, am, si)  # noqa: E731
        work, unit = 2.0 * M * N * K / 1e12, "TFLOP/s"
    else:
        # the bf16 [8192, 2048] workload, or (--cast-in f32) the fp32 input
        # of the same shape that the step's X and weight casts read; --no-yt
        # writes y only, as the native step does
        base = inputs.spiky_bf16().to(dev)
        if args.cast_in == "f32":
            base = base.float()
        xs = [base] + [base.roll(i * 17, dims=1).contiguous() for i in range(1, 8)]
        y = torch.empty(C2_ROWS, C2_COLS, dtype=torch.uint8, device=dev)
        yt = None
        if not args.no_yt and args.kernel != "quantize":
            yt = torch.empty(C2_COLS, C2_ROWS, dtype=torch.uint8, device=dev)
        s = torch.ones(1, device=dev)
        am = torch.zeros(1, device=dev)
        si = torch.zeros(1, device=dev)
        it = iter(range(1 << 30))
        if args.kernel == "quantize":                    # the flat (1-D) cast of the same bytes
            run = lambda: fp8.fp8_quantize(xs[next(it) % 8], args.fmt, s, y, am, si)  # noqa: E731
        else:
            run = lambda: fp8.fp8_cast_transpose_amax(xs[next(it) % 8], args.fmt, s, y, yt, am, si)  # noqa: E731
        work = C2_ROWS * C2_COLS * (base.element_size() + 1 + (0 if yt is None else 1)) / 1e9
        unit = "GB/s"
    for _ in range(2):
        run()
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    for _ in range(args.reps):
        run()
    s1.record()
    torch.cuda.synchronize()
    us = 1e3 * s0.elapsed_time(s1) / args.reps
    print(json.dumps({"kernel": args.kernel, "shape": args.shape if args.kernel.startswith("gemm") else None,
                      "cast_in": args.cast_in, "yt": not args.no_yt, "us": us, "rate": work / (us * 1e-6), "unit": unit,
                      "status": fp8.fp8ds_device_status()}))


# -------------------------------------------------------------------- main --

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-tokens", type=int, default=None,
                    help="tokens of the oracle's sample (default 128; 8 per step for --impl reference)")
    ap.add_argument("--kernel", choices=["gemm", "gemmcast", "cast", "castmulti", "quantize"], default=None,
                    help="run one kernel alone (2 warm-up + --reps launches), for profilers")
    ap.add_argument("--shape", default="8192x2048x8192", help="MxNxK for --kernel gemm")
    ap.add_argument("--major", default="k,k", help="operand layouts a,b for --kernel gemm: k or mn each")
    ap.add_argument("--fmt", default="e4m3", help="FP8 format for --kernel cast")
    ap.add_argument("--cast-in", default="bf16", choices=["bf16", "f32"], help="input dtype for --kernel cast")
    ap.add_argument("--no-yt", action="store_true", help="--kernel cast writes y only (no transpose)")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--detail", default=None, help="also write the per-kernel breakdown and notes (JSON) here")
    ap.add_argument("--no-models", action="store_true", help="skip the TEBlock and 32-block forward timings")
    args = ap.parse_args()
    if args.kernel:
        return single_kernel(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        # The reference arm is the oracle (plain CPU C), timed on the host
        # cores on a bounded sample of the same step; rank 0 alone.
        if rank != 0:
            return
        args.cpu_tokens = args.cpu_tokens or 8
        sample = OracleStepSample(args.cpu_tokens)
        cores = sample.cores
        for _ in range(args.warmup):
            sample.run()
        times = []
        for _ in range(args.steps):
            flop, dt = sample.run()
            times.append(dt)
        ms = 1e3 * statistics.mean(times)
        v = flop / (ms * 1e-3) / 1e12
        sample = "oracle step (6 casts, 6 fp64 GEMMs, update) at %d of %d tokens, full weights" % (
            args.cpu_tokens, TOKENS)
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": step_config(world),
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }))
        return

    assert args.warmup >= 3, "at least 3 warm-up steps"
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)

    from fp8_delayed_scaling_cast_b200 import binding as fp8
    pk = peaks()
    step = MlpStep(fp8, device)

    from fp8_delayed_scaling_cast_b200.dist import sync_amax
    sync = sync_amax if world > 1 else None

    # warm-up (both variants of the step)
    for i in range(args.warmup):
        step.run_linear_api(i, sync_amax=sync, fused=False)
    for i in range(args.warmup):
        step.run_linear_api(i, sync_amax=sync)
    barrier_sync(world)

    # timed region: K steps through the public linear API, launched back to
    # back (no host sync, no events between kernels)
    clocks = ClockSampler(device) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.1)
    barrier_sync(world)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if clocks:
        clocks.mark_start()
    t_start.record()
    h0 = time.perf_counter()
    for i in range(args.steps):
        step.run_linear_api(i, sync_amax=sync)
    host_us = 1e6 * (time.perf_counter() - h0) / args.steps
    t_end.record()
    barrier_sync(world)
    if clocks:
        clocks.mark_end()
    clock_info = clocks.stop() if clocks else None
    ms_local = t_start.elapsed_time(t_end) / args.steps
    ms = max_over_ranks(ms_local, world, device)
    status = fp8.fp8ds_device_status()

    # the same step with each linear casting its own input and gradient
    barrier_sync(world)
    t_start.record()
    for i in range(args.steps):
        step.run_linear_api(i, sync_amax=sync, fused=False)
    t_end.record()
    barrier_sync(world)
    ms_unfused = max_over_ranks(t_start.elapsed_time(t_end) / args.steps, world, device)

    # the fused step replayed from a CUDA graph (one GPU: the amax sync of
    # several ranks is not captured)
    graph_info = time_graph_step(step, args.steps, device) if world == 1 else None

    # per-kernel durations: the same launches, one C call per kernel, each
    # bracketed by CUDA events on the launching stream (K more steps)
    log = EventLog()
    for i in range(args.steps):
        step.run_kernels(i, ev=log, sync_amax=sync)
    barrier_sync(world)

    # the dominant kernel's launch duration: the step's six GEMM launches
    # back to back (PDL between them, as in the step), K rounds, CUDA events
    # around the whole loop on the launching stream; across a round the GEMMs
    # touch ~2 GB of distinct operands and outputs, far more than L2
    for _ in range(2):
        step.run_gemms()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gclocks = ClockSampler(device) if rank == 0 else None
    if gclocks:
        gclocks.start()
        time.sleep(0.1)
    barrier_sync(world)
    if gclocks:
        gclocks.mark_start()
    g0.record()
    for _ in range(args.steps):
        step.run_gemms()
    g1.record()
    barrier_sync(world)
    if gclocks:
        gclocks.mark_end()
    gemm_clock_info = gclocks.stop() if gclocks else None
    gemm_b2b_ms = g0.elapsed_time(g1) / (STEP_GEMMS * args.steps)

    # the step's cast launches back to back, K rounds over the rotating inputs
    # (234 MB read per round, more than L2), replayed from a CUDA graph: the
    # cast kernels' own rate in the step's shapes, free of host issue gaps
    for i in range(2):
        step.run_casts(i)
    barrier_sync(world)
    cast_b2b_ms = max_over_ranks(graph_time_us(step.run_casts, args.steps) * 1e-3, world, device)

    per = log.summary()
    gemm_ms = [t for _, t in per["gemm"]]
    gemm_by_key = {}
    for key, t in per["gemm"]:
        gemm_by_key.setdefault(key, []).append(t)
    cast_ms = {}
    for key, t in per["cast"]:
        cast_ms.setdefault(key, []).append(t)
    upd_ms = [t for _, t in per["update"]]
    gemm_avg = statistics.mean(gemm_ms)
    gemm_avg_b2b = max_over_ranks(gemm_b2b_ms, world, device)
    gemm_tflops = GEMM_FLOP / (gemm_avg_b2b * 1e-3) / 1e12
    fp8_peak = 2.0 * pk["bf16"]                       # nominal fp8:bf16 ratio 4.5 / 2.25
    fp8_peak_sus = 2.0 * pk["bf16_sus"]
    # The burst peak applies to a kernel running at full clock; if the SM
    # clock sampled over the GEMM loop sat more than 10 % below its maximum
    # (the power cap engaged), the sustained peak is the denominator.
    gemm_peak, gemm_peak_kind = fp8_peak, "burst"
    if gemm_clock_info and gemm_clock_info.get("sm_mhz") and gemm_clock_info.get("sm_max_mhz"):
        if gemm_clock_info["sm_mhz"] < 0.9 * gemm_clock_info["sm_max_mhz"]:
            gemm_peak, gemm_peak_kind = fp8_peak_sus, "sustained"
    cast_total_ms = sum(sum(v) for v in cast_ms.values()) / args.steps
    kernel_ms = (sum(gemm_ms) + sum(upd_ms)) / args.steps + cast_total_ms
    cast_gbs_step = STEP_CAST_BYTES_FUSED / (cast_b2b_ms * 1e-3) / 1e9
    cast_gbs_bracketed = STEP_CAST_BYTES_FUSED / (cast_total_ms * 1e-3) / 1e9
    value = world * STEP_FLOP / (ms * 1e-3) / 1e12

    # standalone: cast-transpose-amax workload and the headline GEMM shapes
    c2 = time_cast_workload(fp8, device)
    c2_us = statistics.mean([c2["e4m3"]["us_mean"], c2["e5m2"]["us_mean"]])
    c2_gbs = C2_BYTES / (c2_us * 1e-6) / 1e9
    heads = time_headline_gemm(fp8, device)
    upd576_us = time_update_576(fp8, device)

    # end to end through the public API with host buffers
    e2e_ms, h2d, d2h = e2e_linear_api(fp8, step, device, max(10, args.steps // 2), 3)
    e2e_ms = max_over_ranks(e2e_ms, world, device)
    status = status or fp8.fp8ds_device_status()

    # the TEBlock forward (4 microbatches, cache refreshed at the first) and
    # the 32-block forward (576 metas): rank 0's GPU only, after the step
    teblock = toy = None
    if world == 1 and not args.no_models:
        del step
        torch.cuda.empty_cache()
        teblock = time_teblock_microbatches(fp8, device, rounds=max(3, min(args.steps, 10)))
        toy = time_toy_model(fp8, device, steps=max(3, min(args.steps, 10)))
        status = status or toy["device_status"]

    if world > 1:
        barrier_sync(world)
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    traffic, traffic_note = committed_gemm_traffic(os.path.dirname(os.path.abspath(__file__)))
    cpu = None
    args.cpu_tokens = args.cpu_tokens or 128
    if not args.no_cpu_baseline and world == 1:
        sample = OracleStepSample(args.cpu_tokens)
        flop, dt = sample.run()
        cpu = {"value": flop / dt / 1e12, "unit": "TFLOP/s", "cores": sample.cores, "kind": "oracle",
               "sample": "oracle step (6 casts, 6 fp64 GEMMs, update) at %d of %d tokens, full "
                         "weights; %.1f s" % (args.cpu_tokens, TOKENS, dt)}

    r3 = lambda v: None if v is None else round(v, 3)  # noqa: E731
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8(e4m3,e5m2)xfp8->f32",
        "data": "synthetic",
        "config": step_config(world),
        "cast_transpose_amax": {
            "bf16_8192x2048_e4m3_us": r3(c2["e4m3"]["us_mean"]), "e5m2_us": r3(c2["e5m2"]["us_mean"]),
            "gbs": r3(c2_gbs), "peak_gbs": pk["hbm"], "frac": r3(c2_gbs / pk["hbm"]),
            "in_step_us": r3(1e3 * cast_b2b_ms), "in_step_gbs": r3(cast_gbs_step),
            "in_step_frac": r3(cast_gbs_step / pk["hbm"]), "dynamic_e4m3_us": r3(c2["dynamic_e4m3"]["us_mean"]),
        },
        "roofline": {
            "bound": "tensor", "achieved": r3(gemm_tflops), "peak": gemm_peak, "unit": "TFLOP/s",
            "frac": r3(gemm_tflops / gemm_peak), "traffic": traffic,
            "kernel": "fp8_gemm_2sm_kernel", "launch_us": r3(1e3 * gemm_avg_b2b), "peak_kind": gemm_peak_kind,
            "peak_src": pk["src"], "frac_burst": r3(gemm_tflops / fp8_peak),
        },
        "e2e": {"value": r3(world * STEP_FLOP / (e2e_ms * 1e-3) / 1e12), "unit": "TFLOP/s",
                "ms_per_step": r3(e2e_ms), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "gpu_launches_per_step": LAUNCHES_PER_STEP,
        "gemm_alone": {k: {"us": r3(v["us_mean"]), "tflops": r3(v["tflops"]),
                           "torch_scaled_mm_us": r3(v["context_torch_scaled_mm"].get("us_mean"))}
                       for k, v in heads.items()},
        "teblock_fwd_4mb": None if teblock is None else {k: r3(v) for k, v in teblock.items()},
        "toy32_fwd": None if toy is None else {k: r3(v) for k, v in toy.items() if k != "device_status"},
        "graph_step": None if graph_info is None else {"ms_per_step": r3(graph_info["ms_per_step"]),
                                                      "eager_ms_same_section": r3(
                                                          graph_info["eager_same_section_ms_per_step"]),
                                                      "host_us_per_step": r3(graph_info["host_us_per_step"])},
        "host_us_per_step": r3(host_us),
        "unfused_step_ms": r3(ms_unfused),
        "update_576_metas_us": r3(upd576_us),
        "step_roofline_frac": r3(((STEP_FLOP / (fp8_peak * 1e12)) + (STEP_CAST_BYTES_FUSED / (pk["hbm"] * 1e9))) /
                                 (ms * 1e-3)),
        "device_status": status,
        "clocks": clock_info,
        "cpu_baseline": cpu,
    }
    if args.detail:
        detail = {
            "gemm_event_bracketed_us": {k: 1e3 * statistics.mean(v) for k, v in gemm_by_key.items()},
            "cast_event_bracketed_us": {k: 1e3 * statistics.mean(v) for k, v in cast_ms.items()},
            "update_event_bracketed_us": 1e3 * statistics.mean(upd_ms),
            "kernels_event_bracketed_sum_ms_per_step": kernel_ms,
            "event_bracketed_note": "each launch bracketed by CUDA events: the events break the PDL overlap and "
                                    "add host gaps, so these run 5-20% above the back-to-back figures and their "
                                    "sum exceeds ms_per_step",
            "roofline_timing": "the step's 6 GEMM launches (same operands, outputs, epilogues) back to back for K "
                               "rounds, CUDA events around the loop on the launching stream; mean per launch",
            "roofline_traffic_note": traffic_note, "gemm_algorithmic_bytes_per_launch": GEMM_ALG_BYTES,
            "gemm_clocks": gemm_clock_info,
            "peak_note": "fp8 dense = 2 x measured bf16 (%s): burst %.1f, sustained %.1f TFLOP/s; sustained is "
                         "used when the SM clock over the GEMM loop sat >10%% below max" % (
                             pk["src"], fp8_peak, fp8_peak_sus),
            "cast_workload": c2,
            "cast_in_step_event_bracketed_gbs": cast_gbs_bracketed,
            "cast_timing": "100 launches over 8 rotating inputs captured in a CUDA graph, replayed between CUDA "
                           "events; us_host_issued: the same launches issued one by one from Python; in_step: the "
                           "step's 2 cast launches (X+W1+W2 fp32 in one, dY bf16; y only) back to back, K rounds, "
                           "replayed from a CUDA graph",
            "graph_step": graph_info,
            "gemm_alone": heads,
            "teblock_fwd_4mb": teblock,
            "toy32_fwd": toy,
            "e2e_api": "fp8_linear_refresh_weights + fp8_linear_fwd_ex/bwd_ex + fp8_update_scales, pinned host "
                       "X/dY, double-buffered copies",
        }
        with open(args.detail, "w") as f:
            json.dump(detail, f, indent=1)
    print(json.dumps(line))


if __name__ == "__main__":
    main()
