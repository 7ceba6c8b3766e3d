"""Pins of the layer oracle (CPU): its bf16 rounding against torch's conversion,
the identity reduction -- with W_in = I and W_o selecting the mixer output, the
layer is the (pinned) prefill oracle on the column blocks of x -- and the
orientation of both projections (permutation matrices move columns, x W and
o W, not rows)."""
import numpy as np
import torch

import oracle
from oracle import layer


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(5000) * 10.0 ** rng.integers(-6, 6, 5000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 65504.0, -3.0e-39])]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    np.testing.assert_array_equal(layer.bf16_round(x), want)
    np.testing.assert_array_equal(layer.bits_to_f64(want), torch.from_numpy(want.view(np.int16)).view(
        torch.bfloat16).double().numpy())


def test_identity_projections_reduce_to_the_mixer():
    rng = np.random.default_rng(1)
    H, dk, dv, n = 2, 4, 3, 19
    c_in = H * (2 * dk + 2 * dv) + 2 * H
    x = layer.bf16_round(rng.standard_normal((n, c_in)))
    w_in = layer.bf16_round(np.eye(c_in))
    w_o = layer.bf16_round(np.eye(H * dv, c_in))                 # y[:, :H dv] = mixer output
    conv_w = (rng.standard_normal((H * (2 * dk + dv), 4)) * 0.5).astype(np.float32)
    A = np.log(rng.uniform(1, 16, H)).astype(np.float32)
    b_alpha = np.zeros(H, np.float32)
    norm_w = (0.1 * rng.standard_normal(dv)).astype(np.float32)
    cu = np.array([0, 11, 19], np.int32)
    y, S = layer.layer_forward(x, w_in, conv_w, A, b_alpha, norm_w, w_o, H, dk, dv, cu_seqlens=cu)
    cols = np.cumsum([H * dk, H * dk, H * dv, H * dv, H])
    q, k, v, z, a, b = np.split(x, cols, axis=1)
    out, S_ref = oracle.prefill(q.reshape(n, H, dk).copy(), k.reshape(n, H, dk).copy(), v.reshape(n, H, dv).copy(),
                                conv_w, a.copy(), b.copy(), A, b_alpha, z.reshape(n, H, dv).copy(), norm_w,
                                cu_seqlens=cu)
    np.testing.assert_array_equal(y[:, :H * dv], layer.bits_to_f64(layer.bf16_round(out)).reshape(n, H * dv))
    assert not np.any(y[:, H * dv:])
    np.testing.assert_array_equal(S, S_ref)


def _small_layer(rng, H=2, dk=4, dv=3):
    conv_w = (rng.standard_normal((H * (2 * dk + dv), 4)) * 0.5).astype(np.float32)
    A = np.log(rng.uniform(1, 16, H)).astype(np.float32)
    return conv_w, A, np.zeros(H, np.float32), (0.1 * rng.standard_normal(dv)).astype(np.float32)


def test_projections_are_right_multiplications():
    """W_in = P (a permutation) equals the identity layer on x P; W_o = E Q (E selects
    the mixer output, Q permutes) places the output at the columns Q sends it to."""
    rng = np.random.default_rng(2)
    H, dk, dv, n = 2, 4, 3, 13
    c_in = H * (2 * dk + 2 * dv) + 2 * H
    conv_w, A, b_alpha, norm_w = _small_layer(rng, H, dk, dv)
    x = layer.bf16_round(rng.standard_normal((n, c_in)))
    perm = rng.permutation(c_in)
    P = np.eye(c_in)[:, perm]                                    # (x P)[:, j] = x[:, perm[j]]
    E = np.eye(H * dv, c_in)
    Q = np.eye(c_in)[:, rng.permutation(c_in)]
    y1, S1 = layer.layer_forward(x, layer.bf16_round(P), conv_w, A, b_alpha, norm_w, layer.bf16_round(E @ Q), H,
                                 dk, dv, num_seqs=1)
    xp = layer.bf16_round(layer.bits_to_f64(x)[:, perm])
    y2, S2 = layer.layer_forward(xp, layer.bf16_round(np.eye(c_in)), conv_w, A, b_alpha, norm_w,
                                 layer.bf16_round(E), H, dk, dv, num_seqs=1)
    np.testing.assert_array_equal(S1, S2)
    np.testing.assert_array_equal(y1, y2 @ Q)
    assert np.any(y1 != y2)                                     # the output permutation did move columns
