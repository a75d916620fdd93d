"""The seeded input generator shared by the tests and the bench: bf16
rounding against torch's own conversion, the Z-order decode against the
oracle's encode, determinism, head slices, and the image-like structure the
selection relies on (nearby tokens are more alike than distant ones)."""

import numpy as np
import torch

import oracle
from hierarchical_top_sparse_llsa_b200 import workloads


def test_round_to_bf16_matches_torch():
    rng = np.random.default_rng(90)
    a = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 10.0 ** rng.integers(-6, 6, 10000),
                        # exact ties between two bf16 values, both parities
                        np.array([1.0 + 2.0**-8, 1.0 + 3 * 2.0**-8, -(1.0 + 2.0**-8), 0.0, -0.0], np.float32)])
    ours = workloads.round_to_bf16(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).float().numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_zorder_decode_inverts_the_oracle_encode():
    side = 32
    z = oracle.zorder_index(side, side)  # Z-order token of raster position y * side + x
    x, y = workloads.zorder_decode(z)
    pos = np.arange(side * side)
    assert np.array_equal(x, pos % side) and np.array_equal(y, pos // side)


def test_inputs_are_deterministic_and_sliceable():
    w = workloads.WORKLOADS["img64_bf16"]
    a = workloads.make_inputs(w)
    b = workloads.make_inputs(w)
    for k in ("q", "k", "v", "do"):
        assert a[k].shape == (w.B, w.H, w.N, w.D) and a[k].dtype == np.float32
        assert np.array_equal(a[k], b[k])
        assert np.array_equal(a[k], workloads.round_to_bf16(a[k]))  # already bf16 values
    s = workloads.make_inputs(w, heads=[2, 5])
    for k in ("q", "k", "v", "do"):
        assert np.array_equal(s[k], a[k][:, [2, 5]])


def test_inputs_are_image_like():
    # tokens of one 16-token block (a 4x4 pixel tile) differ less than tokens
    # drawn far apart, which is what makes pooled blocks informative
    w = workloads.WORKLOADS["img64_bf16"]
    q = workloads.make_inputs(w, with_dout=False)["q"][0, 0]  # [N, D]
    near = np.mean(np.abs(q[0::16] - q[1::16]))
    far = np.mean(np.abs(q[: w.N // 2] - q[w.N // 2:]))
    assert near < 0.8 * far
