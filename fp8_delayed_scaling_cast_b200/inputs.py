"""Seeded synthetic inputs for the FP8 delayed-scaling linear workloads.

This module draws random tensors and nothing else: it holds none of the
method's arithmetic (no cast, amax, scale or GEMM), so both the CUDA path and
the CPU oracle can consume its output.  Every tensor is drawn on the host from
``torch.Generator('cpu')`` seeded as stated, in the order listed, so the same
bytes reach both sides.

Workload shapes follow the pages: the TEBlock of "CPU Overhead of te.Linear
FP8 Layers" (hidden 2048, mlp_ratio 4, batch 8 x seq 1024 = 8192 tokens; six
linears 2048->12288 (+bias), 2048->6144, 2048->2048, 2048->4096, 2048->8192
(+bias), 8192->2048 (+bias)), fp32 master weights, inputs ~ U[0,1), weights
~ N(0, 0.02).
"""
import torch

HIDDEN = 2048
MLP_RATIO = 4
TOKENS = 8 * 1024

# (out_features, in_features, has_bias) of the six TEBlock linears, in order.
TEBLOCK_LINEARS = (
    (6 * HIDDEN, HIDDEN, True),            # timestep modulation
    (3 * HIDDEN, HIDDEN, False),           # self-attention qkv
    (HIDDEN, HIDDEN, False),               # cross-attention q
    (2 * HIDDEN, HIDDEN, False),           # cross-attention kv
    (MLP_RATIO * HIDDEN, HIDDEN, True),    # mlp fc1
    (HIDDEN, MLP_RATIO * HIDDEN, True),    # mlp fc2
)


def gen(seed):
    g = torch.Generator("cpu")
    g.manual_seed(int(seed))
    return g


def uniform(shape, g):
    return torch.rand(*shape, generator=g, dtype=torch.float32)


def normal(shape, g, std=1.0):
    return torch.randn(*shape, generator=g, dtype=torch.float32) * std


def single_linear(seed=0, m=128, k=256, n=512):
    """Single linear, two delayed-scaling steps: X ~ U[0,1) [m,k], W ~ N(0,0.02) [n,k]."""
    g = gen(seed)
    x = uniform((m, k), g)
    w = normal((n, k), g, 0.02)
    return x, w


def spiky_bf16(rows=TOKENS, cols=HIDDEN, seed=0, spike_frac=1e-3, spike_mult=1000.0):
    """bf16 [rows, cols] ~ N(0,1) with a fraction of entries multiplied (saturation probes).

    Drawn as fp32 then stored as bf16 (the storage dtype of the workload).
    """
    g = gen(seed)
    x = normal((rows, cols), g)
    mask = uniform((rows, cols), g) < spike_frac
    x[mask] *= spike_mult
    return x.to(torch.bfloat16)


def iter_teblock_weights(seed=0, blocks=1, scale=1):
    """Yield (fp32 master weight [out, in], bias or None) of `blocks` TEBlocks,
    block-major, one linear at a time (so a large model need not sit on the
    host all at once).

    `scale` divides every feature size (tests use it to shrink the block while
    keeping its structure).  Biases come from a second generator (seed + 1).
    """
    g = gen(seed)
    gb = gen(seed + 1)
    for _ in range(blocks):
        for out_f, in_f, has_bias in TEBLOCK_LINEARS:
            w = normal((out_f // scale, in_f // scale), g, 0.02)
            yield w, (normal((out_f // scale,), gb, 0.02) if has_bias else None)


def teblock_weights(seed=0, blocks=1, scale=1):
    """Lists (weights, biases) of iter_teblock_weights (same bytes)."""
    ws, bs = [], []
    for w, b in iter_teblock_weights(seed, blocks, scale):
        ws.append(w)
        bs.append(b)
    return ws, bs


def teblock_microbatch(mb, seed=0, tokens=TOKENS, hidden=HIDDEN):
    """TEBlock input of microbatch `mb`: X ~ U[0,1) fp32 [tokens, hidden] from
    generator 2000 + mb + seed (each microbatch can be regenerated alone)."""
    return uniform((tokens, hidden), gen(2000 + mb + seed))


def toy_step_input(step, seed=0, tokens=TOKENS, hidden=HIDDEN):
    """Input of forward step `step` of the 32-block model: X ~ U[0,1) fp32
    [tokens, hidden] from generator 3000 + step + seed."""
    return uniform((tokens, hidden), gen(3000 + step + seed))


def mlp_pair(seed=0, tokens=TOKENS, hidden=HIDDEN, ratio=MLP_RATIO):
    """MLP pair hidden -> ratio*hidden -> hidden: W1 [4h,h], W2 [h,4h], biases (seed+1)."""
    g = gen(seed)
    gb = gen(seed + 1)
    w1 = normal((ratio * hidden, hidden), g, 0.02)
    w2 = normal((hidden, ratio * hidden), g, 0.02)
    b1 = normal((ratio * hidden,), gb, 0.02)
    b2 = normal((hidden,), gb, 0.02)
    return w1, b1, w2, b2


def mlp_step_inputs(step, seed=0, tokens=TOKENS, hidden=HIDDEN, grad_std=1e-3, spike_step=None,
                    spike_mult=8.0):
    """Per-step X ~ U[0,1) fp32 [tokens, hidden] and dY ~ N(0, grad_std) bf16 [tokens, hidden].

    Each step has its own generator (seed 1000 + 2*step + seed) so a step can be
    regenerated alone.  If `step == spike_step` dY is multiplied by `spike_mult`
    (an amax spike that enters and later leaves the history window).
    """
    g = gen(1000 + 2 * step + seed)
    x = uniform((tokens, hidden), g)
    dy = normal((tokens, hidden), g, grad_std)
    if spike_step is not None and step == spike_step:
        dy = dy * spike_mult
    return x, dy.to(torch.bfloat16)


def fp8_codes(shape, seed=0, fmt_max_code=0x7E):
    """Random finite FP8 byte codes (both signs) as uint8, for GEMM-only tests."""
    g = gen(seed)
    mag = torch.randint(0, fmt_max_code + 1, shape, generator=g, dtype=torch.int32)
    sign = torch.randint(0, 2, shape, generator=g, dtype=torch.int32) * 128
    return (mag + sign).to(torch.uint8)


def bf16_bits(t):
    """Raw uint16 bit patterns of a bf16 tensor (numpy), for byte-level consumers."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")
