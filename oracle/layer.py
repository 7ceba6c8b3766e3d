"""fp64 CPU oracle of the GDN layer from the hidden states -- TEST INFRASTRUCTURE.

Only the tests, the smoke check in the package entry file and bench.py's
CPU-baseline leg may import this module; it shares no code with the CUDA path.

The layer (slinene.github.io write-up of "On the Design of Qwen3.8-Next
Architecture", 模块 A, 参数化): q, k, v, z and the two gate logits are linear
projections of the hidden state x, the mixer maps them to
sigmoid(z) * RMSNorm(y) (the prefill oracle), and W_o projects that back.
The layer stores its projections and the mixer output in bf16 (the inputs of
the next step); the products themselves are exact here (fp64).
"""
import numpy as np

from . import prefill as _prefill


def bits_to_f64(bits):
    """bf16 bit patterns (uint16) -> float64 (exact)."""
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_round(x):
    """float -> the nearest bf16 (ties to even) as bit patterns; values are first
    rounded to fp32."""
    u = np.ascontiguousarray(np.asarray(x, np.float64).astype(np.float32)).view(np.uint32).astype(np.uint64)
    return (((u + 0x7FFF + ((u >> 16) & 1)) >> 16) & 0xFFFF).astype(np.uint16)


def layer_forward(x_bits, w_in_bits, conv_w, A, b_alpha, norm_w, w_o_bits, H, dk, dv, S0=None,
                  cu_seqlens=None, num_seqs=None):
    """x [N, d_model], w_in [d_model, H(2dk + 2dv) + 2H] (column blocks q, k, v, z,
    a, b), w_o [H dv, d_model], all bf16 bits.  Returns (y [N, d_model] float64,
    S_final float64)."""
    x = bits_to_f64(x_bits)
    P = bf16_round(x @ bits_to_f64(w_in_bits))                # the projections, stored in bf16
    n = x.shape[0]
    widths = [H * dk, H * dk, H * dv, H * dv, H, H]
    q, k, v, z, a, b = np.split(P, np.cumsum(widths)[:-1], axis=1)
    out, S_final = _prefill(np.ascontiguousarray(q.reshape(n, H, dk)), np.ascontiguousarray(k.reshape(n, H, dk)),
                            np.ascontiguousarray(v.reshape(n, H, dv)), conv_w, np.ascontiguousarray(a),
                            np.ascontiguousarray(b), A, b_alpha, np.ascontiguousarray(z.reshape(n, H, dv)), norm_w,
                            S0=S0, cu_seqlens=cu_seqlens, num_seqs=num_seqs)
    o = bits_to_f64(bf16_round(out)).reshape(n, H * dv)      # the mixer output, stored in bf16
    return o @ bits_to_f64(w_o_bits), S_final
