"""Seeded synthetic workloads for Log-linear Sparse Attention (LLSA).

This module only describes shapes and draws input values.  It holds none of the
method's arithmetic (no pooling, scoring, selection or attention), so both the
CPU oracle and the CUDA path may take their inputs from it.

Input recipe (image-like values in Z-order, one generator for every shape):
  * every (tensor, batch, head, channel) of Q, K and V is a sum of four
    low-frequency 2D sinusoids  a * sin(2*pi*(fx*x/W + fy*y/H) + phi)  over the
    pixel grid, with a ~ U(0,1), fx, fy ~ U(-4,4) cycles per image and
    phi ~ U(0, 2*pi), plus N(0, 0.5) noise (0.5 is the standard deviation);
  * dO ~ N(0, 1);
  * values are drawn in fp32 and rounded to bf16 (round to nearest even) for
    bf16 workloads; the returned float32 arrays hold those rounded values;
  * the random stream is numpy's default_rng(seed), drawn in a fixed order.

Token order is Z-order (Morton order): token t sits at pixel (x, y) where x is
made of the even bits of t and y of the odd bits, so every 16 consecutive
tokens form a 4x4 pixel tile, every 256 a 16x16 tile, and so on.  This is the
"group 2x2, then 4x4" index reordering of "Trainable Log-linear Sparse
Attention for Efficient Diffusion Transformers" (howistudyai explainer,
Step 5: Index Reordering for Images).
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

BLOCK = 16  # tokens per query/key block and pooling factor per level


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic LLSA problem (shapes, levels, Top-K, dtype, seed)."""

    name: str
    B: int
    H: int
    N: int
    D: int
    dtype: str  # "f32" or "bf16"
    L: int  # number of pooled levels (level 1 = 16-token blocks)
    topk: int
    seed: int
    backward: bool = True

    @property
    def side(self) -> int:
        s = int(round(math.sqrt(self.N)))
        assert s * s == self.N
        return s

    def n_level(self, l: int) -> int:
        """Tokens at level l (level 0 = the N fine tokens)."""
        return self.N // BLOCK**l

    def k_eff(self) -> list[int]:
        """K_eff(l) for l = 0..L (index 0 unused): min(K, candidates at l)."""
        k = [0] * (self.L + 1)
        k[self.L] = min(self.topk, self.n_level(self.L))
        for l in range(self.L - 1, 0, -1):
            k[l] = min(self.topk, BLOCK * k[l + 1], self.n_level(l))
        return k

    def keys_per_query(self) -> int:
        k = self.k_eff()
        return BLOCK * k[1] + sum(k[2:])


# Five workloads: a 32x32 fp32 correctness case, 64x64, 128x128, the 256x256
# headline (N = 65536) and the 512x512 scaling case at two Top-K values.
WORKLOADS = {
    "tiny_32x32_f32": Workload("tiny_32x32_f32", 1, 2, 1024, 64, "f32", 2, 4, 1001),
    "img64_bf16": Workload("img64_bf16", 2, 8, 4096, 64, "bf16", 3, 8, 1002),
    "img128_bf16": Workload("img128_bf16", 2, 12, 16384, 64, "bf16", 3, 8, 1003),
    "img256_bf16": Workload("img256_bf16", 1, 16, 65536, 64, "bf16", 3, 8, 1004),
    "img512_k8_bf16": Workload("img512_k8_bf16", 1, 8, 262144, 128, "bf16", 4, 8, 1005, backward=False),
    "img512_k32_bf16": Workload("img512_k32_bf16", 1, 8, 262144, 128, "bf16", 4, 32, 1005, backward=False),
}
HEADLINE = "img256_bf16"


def zorder_decode(t: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Pixel (x, y) of Z-order token t: x from the even bits, y from the odd bits."""
    t = np.asarray(t, dtype=np.int64)
    x = np.zeros_like(t)
    y = np.zeros_like(t)
    for b in range(31):
        x |= ((t >> (2 * b)) & 1) << b
        y |= ((t >> (2 * b + 1)) & 1) << b
    return x, y


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    # finite inputs only: the largest finite pattern plus 0x8000 stays below 2^32
    u = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return u.view(np.float32)


def _sinusoid_field(rng, B, H, D, side, x, y):
    """[B,H,N,D] sum of four random low-frequency sinusoids over pixels (x, y)."""
    a = rng.uniform(0.0, 1.0, size=(B, H, D, 4))
    fx = rng.uniform(-4.0, 4.0, size=(B, H, D, 4))
    fy = rng.uniform(-4.0, 4.0, size=(B, H, D, 4))
    ph = rng.uniform(0.0, 2.0 * np.pi, size=(B, H, D, 4))
    coord = np.arange(side, dtype=np.float64) / side
    flat = x * side + y
    out = np.empty((B, H, x.size, D), dtype=np.float32)
    for b in range(B):
        for h in range(H):
            # sin(A + B) = sin A cos B + cos A sin B with A a function of x only
            # and B of y only: each channel image is a rank-8 product of tables.
            A = 2.0 * np.pi * fx[b, h, :, :, None] * coord + ph[b, h, :, :, None]
            Bv = 2.0 * np.pi * fy[b, h, :, :, None] * coord
            ux = np.concatenate([a[b, h, :, :, None] * np.sin(A), a[b, h, :, :, None] * np.cos(A)], axis=1)
            vy = np.concatenate([np.cos(Bv), np.sin(Bv)], axis=1)
            img = np.matmul(ux.transpose(0, 2, 1), vy)  # [D, side_x, side_y]
            out[b, h] = img.reshape(D, -1)[:, flat].T
    return out


def make_inputs(w: Workload, heads: slice | None = None, with_dout: bool = True):
    """Seeded Q, K, V (and dO) as float32 numpy arrays [B,H,N,D] in Z-order.

    For bf16 workloads the values are already rounded to bf16.  ``heads``
    returns a head slice of the same draw (the full draw is made and sliced,
    so a slice equals the same heads of the full problem).
    """
    rng = np.random.default_rng(w.seed)
    x, y = zorder_decode(np.arange(w.N))
    out = {}
    for name in ("q", "k", "v"):
        field = _sinusoid_field(rng, w.B, w.H, w.D, w.side, x, y)
        field += rng.standard_normal(size=field.shape, dtype=np.float32) * np.float32(0.5)
        out[name] = field
    if with_dout:
        out["do"] = rng.standard_normal(size=(w.B, w.H, w.N, w.D), dtype=np.float32)
    if w.dtype == "bf16":
        for name in out:
            out[name] = round_to_bf16(out[name])
    if heads is not None:
        out = {k: np.ascontiguousarray(v[:, heads]) for k, v in out.items()}
    return out
