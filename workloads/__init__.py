"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module only draws random numbers and lays out shapes.  It holds none of
the quantization arithmetic (no scales, codes, packing or products), so both
the CUDA path and the CPU oracle can take their inputs from here without
sharing any of the method's code.

Workloads (all synthetic; the pages measure on Qwen-class weights that are not
available here, so Gaussian weights with the stated spreads stand in for them):

* ``single``   -- W 256x512 ~ N(0, 0.02^2), seed 0, b=5, x 1x512 ~ N(0,1).
* ``decode``   -- W 4096x4096 ~ N(0, 0.02^2) with 0.1% of the entries scaled by
                  20 (outliers), b in {4,5,6,7,8,10,12}, x with M in {1,4,16}.
* ``mlp27b``   -- up/gate W 17408x5120 and down W 5120x17408 ~ N(0, 0.015^2),
                  b in {5,6}, M in {1,8,32}.
* ``recipe``   -- 64 layers x 7 linears of a 27B-class decoder, mixed bits
                  (283 at 6, 98 at 5, 34 at 7, 33 at 8), M=1 chained.
* ``prefill``  -- x 2048x5120 ~ N(0,1); W 17408x5120 and 5120x5120
                  ~ N(0, 0.02^2), b in {5,6,8,10,12}.
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------
# workload table
# ----------------------------------------------------------------------------

SINGLE = dict(name="single", N=256, K=512, sigma=0.02, bits=[5], Ms=[1],
              w_seed=0, x_seed=0)
DECODE = dict(name="decode", N=4096, K=4096, sigma=0.02,
              bits=[4, 5, 6, 7, 8, 10, 12], Ms=[1, 4, 16],
              outlier_frac=0.001, outlier_scale=20.0, w_seed=0, x_seed=1)
MLP27B = dict(name="mlp27b", shapes=[("up", 17408, 5120), ("gate", 17408, 5120),
                                     ("down", 5120, 17408)],
              sigma=0.015, bits=[5, 6], Ms=[1, 8, 32], w_seed=0, x_seed=1)
PREFILL = dict(name="prefill", M=2048, shapes=[("up", 17408, 5120), ("o", 5120, 5120)],
               sigma=0.02, bits=[5, 6, 8, 10, 12], w_seed=0, x_seed=1)

# One decoder layer of the 27B-class recipe stack, in execution order.
# (name, N = out features, K = in features)
RECIPE_LAYER = [
    ("q", 6144, 5120),
    ("k", 1024, 5120),
    ("v", 1024, 5120),
    ("o", 5120, 6144),
    ("gate", 17408, 5120),
    ("up", 17408, 5120),
    ("down", 5120, 17408),
]
RECIPE_LAYERS = 64
RECIPE = dict(name="recipe", layers=RECIPE_LAYERS, sigma=0.02, M=1,
              bit_counts={6: 283, 5: 98, 7: 34, 8: 33}, bits_seed=0, w_seed=0,
              x_seed=1)


def recipe_shapes(layers: int = RECIPE_LAYERS):
    """(layer, name, N, K) for every linear of the recipe stack, in order."""
    out = []
    for layer in range(layers):
        for name, n, k in RECIPE_LAYER:
            out.append((layer, name, n, k))
    return out


def recipe_bits(seed: int = RECIPE["bits_seed"], counts=None):
    """Per-matrix bit widths of the recipe stack.

    The multiset is 283 matrices at 6 bits, 98 at 5 and the remaining 67
    split 34 at 7 / 33 at 8 bits; it is shuffled by a seeded permutation and
    read in (layer, q, k, v, o, gate, up, down) order.
    """
    counts = counts or RECIPE["bit_counts"]
    bits = []
    for b in sorted(counts):
        bits += [b] * counts[b]
    bits = np.array(bits, dtype=np.int64)
    perm = np.random.default_rng(seed).permutation(len(bits))
    return [int(v) for v in bits[perm]]


# ----------------------------------------------------------------------------
# generators
# ----------------------------------------------------------------------------

def gen_weight(N: int, K: int, sigma: float, seed: int,
               outlier_frac: float = 0.0, outlier_scale: float = 20.0) -> np.ndarray:
    """W[N, K] float32 ~ N(0, sigma^2), optionally with outliers.

    Outliers: round(outlier_frac * N * K) distinct flat indices, drawn without
    replacement from the same generator after W, are multiplied by
    ``outlier_scale``.
    """
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((N, K), dtype=np.float32)
    W *= np.float32(sigma)
    n_out = int(round(outlier_frac * N * K))
    if n_out > 0:
        idx = rng.choice(N * K, size=n_out, replace=False)
        flat = W.reshape(-1)
        flat[idx] *= np.float32(outlier_scale)
    return W


def gen_x(M: int, K: int, seed: int):
    """x[M, K] ~ N(0,1) rounded to bfloat16 (round-to-nearest-even).

    Returns a CPU ``torch.bfloat16`` tensor.  ``x.float().numpy()`` holds the
    same values exactly.
    """
    import torch

    rng = np.random.default_rng(seed)
    a = rng.standard_normal((M, K), dtype=np.float32)
    return torch.from_numpy(a).to(torch.bfloat16)


def gen_weight_torch(N: int, K: int, sigma: float, seed: int, device="cuda"):
    """W[N, K] float32 ~ N(0, sigma^2) drawn by torch's generator on ``device``.

    Used for the 448-matrix recipe stack, whose 21.8 G weights are too many to
    draw on the host.  Deterministic for a given seed, shape and device type.
    """
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    W = torch.randn((N, K), generator=g, device=device, dtype=torch.float32)
    W.mul_(sigma)
    return W


def special_rows(K: int, seed: int = 7) -> np.ndarray:
    """A small W with the degenerate rows the quantizer must handle.

    Row 0: all zeros.  Row 1: one nonzero entry.  Row 2: the smallest positive
    subnormal in every slot.  Row 3: a few subnormals of different sizes.
    Row 4: a constant row.  Row 5: negative maximum.  Row 6: values spanning
    2^-30 .. 2^30.  Row 7: Gaussian.
    """
    rng = np.random.default_rng(seed)
    W = np.zeros((8, K), dtype=np.float32)
    W[1, K // 2] = np.float32(-3.25)
    W[2, :] = np.float32(np.finfo(np.float32).smallest_subnormal)
    sub = np.finfo(np.float32).smallest_subnormal
    W[3, :] = (rng.integers(-40, 41, size=K).astype(np.float64) * sub).astype(np.float32)
    W[4, :] = np.float32(0.125)
    W[5, :] = rng.standard_normal(K).astype(np.float32) * np.float32(0.01)
    W[5, 0] = np.float32(-7.0)
    W[6, :] = (np.exp2(rng.uniform(-30, 30, size=K)) *
               rng.choice([-1.0, 1.0], size=K)).astype(np.float32)
    W[7, :] = rng.standard_normal(K).astype(np.float32)
    return W


# ----------------------------------------------------------------------------
# recipe stack data flow
# ----------------------------------------------------------------------------

# Activation slots of the chained decode pass.  The pages give no data flow
# between the linears of a layer; this one follows a decoder layer's shape
# (q/k/v read the hidden state, o reads the attention-side output, gate/up
# read o's output, down reads up's output) with an RMS normalisation on every
# linear's input after the first, which keeps 64 chained layers in range.
SLOT_H, SLOT_Q, SLOT_K, SLOT_V, SLOT_O, SLOT_G, SLOT_U, SLOT_D = range(8)
SLOT_WIDTH = {SLOT_H: 5120, SLOT_Q: 6144, SLOT_K: 1024, SLOT_V: 1024, SLOT_O: 5120,
              SLOT_G: 17408, SLOT_U: 17408, SLOT_D: 5120}


def recipe_links(layers: int = RECIPE_LAYERS):
    """(in_slot, out_slot, norm_input) for every linear, in recipe order.

    Layer 0's q/k/v read x0 (slot H) as is; later layers read the previous
    layer's down output (slot D) normalised.
    """
    out = []
    for layer in range(layers):
        h = SLOT_H if layer == 0 else SLOT_D
        hn = layer > 0
        out += [(h, SLOT_Q, hn), (h, SLOT_K, hn), (h, SLOT_V, hn),
                (SLOT_Q, SLOT_O, True), (SLOT_O, SLOT_G, True), (SLOT_O, SLOT_U, True),
                (SLOT_U, SLOT_D, True)]
    return out


def recipe_weight_seed(index: int) -> int:
    """Seed of the index-th matrix of the recipe stack."""
    return 1000 * RECIPE["w_seed"] + 17 + index
