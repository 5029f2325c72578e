"""Helpers shared by the GPU parity tests: host copies, tolerance normalisers.

The parity rule (staged, because a 1-ulp float difference upstream can flip a
later int8):
  P1 quantized activations / packed weights: int8 quants and fp16 scales bit-exact;
  P2 per-block int32 dots bit-exact;
  P3 fp32 matmul outputs, given the same quantized inputs:
     |y_gpu - y_oracle| <= 1e-5 * S, S = sum_b |d_w d_x| sum_i |q_w q_x|
     (sum |w * x| of the dequantized operands; 1e-5 is the relative bound the
     method's description fixes for float outputs);
  P4 SwiGLU on the GPU's own g and u: |h - silu(g) u| <= 1e-5 (|silu(g) u| + tiny);
  P5 h -> Q8_0: the oracle quantizer on the GPU's fp32 h equals the GPU's hq bit-exactly.
"""
import numpy as np
import torch

TOL = 1e-5
QK = 32


def bits(d: torch.Tensor) -> np.ndarray:
    """fp16 scale tensor (device or host) -> numpy uint16 bit patterns."""
    return d.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def canon_d(d: torch.Tensor, k: int) -> np.ndarray:
    """Packed scales [rows, ld_d] -> canonical [rows, k/32] bit patterns."""
    b = bits(d)
    return np.ascontiguousarray(b[..., : k // QK])


def deq_abs(q: np.ndarray, d: np.ndarray) -> np.ndarray:
    """|d * q| per element in float64 (numpy float16 conversion)."""
    s = np.abs(d.view(np.float16).astype(np.float64))
    return np.abs(q.astype(np.float64)) * np.repeat(s, QK, axis=-1)


def S_norm(wq, wd, xq, xd) -> np.ndarray:
    """sum |w x| per (activation row, weight row): [n_x, n_w]."""
    return deq_abs(xq.reshape(-1, xq.shape[-1]), xd.reshape(-1, xd.shape[-1])) @ \
        deq_abs(wq.reshape(-1, wq.shape[-1]), wd.reshape(-1, wd.shape[-1])).T


def assert_p3(y_gpu: np.ndarray, y_ref: np.ndarray, S: np.ndarray, what: str = ""):
    y_gpu = np.asarray(y_gpu, np.float64)
    err = np.abs(y_gpu - y_ref)
    bound = TOL * S + 1e-30
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"P3 {what}: {bad.sum()} of {bad.size} outside 1e-5*S; first at "
                             f"{tuple(i)}: gpu={y_gpu[tuple(i)]!r} ref={y_ref[tuple(i)]!r} "
                             f"S={S[tuple(i)]!r}")
    return float((err / (S + 1e-30)).max())
