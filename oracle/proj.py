"""fp64 oracle for the projections around the attention: the fused QKV projection with
rotary position embedding, and the output projection.

TEST INFRASTRUCTURE ONLY (imported by ``tests/`` and ``bench.py``'s CPU leg); it shares
no code with the CUDA path.

What it computes (Mage-Flow page, "DiT Block" data flow: x -> AdaLayerNorm -> [Q,K,V]
projection -> RoPE -> attention -> output projection; "fusion strategy one": one GEMM
with the stacked weight W_qkv, then a split of its output into q, k, v):
    qkv = x W_qkv^T                  x [T, C], W_qkv [3*H*d, C] (rows: q heads, k heads, v heads)
    q, k, v = the three [T, H, d] slices of qkv
    q, k rotated by RoPE at each token's position inside its own image,
    y = o W_o^T                      o [T, H*d], W_o [C_out, H*d]
RoPE (reading: the pages name it without a formula; this is the standard rotary embedding
with the rotate-half pairing): for i in [0, d/2), theta_i = theta^(-2i/d) and the position
p = token index - first token of its segment,
    (x_i, x_{i+d/2}) -> (x_i cos(p theta_i) - x_{i+d/2} sin(p theta_i),
                         x_i sin(p theta_i) + x_{i+d/2} cos(p theta_i)).
All in fp64; bf16 inputs are widened exactly.
"""
import numpy as np


def _f64(x):
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        return x.double().numpy()
    if hasattr(x, "numpy") and not isinstance(x, np.ndarray):
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def positions(cu_seqlens, total):
    """Position of every token inside its segment."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    pos = np.zeros(int(total), dtype=np.int64)
    for i in range(len(cu) - 1):
        pos[cu[i]:cu[i + 1]] = np.arange(cu[i + 1] - cu[i])
    return pos


def rope(x, pos, theta):
    """Rotate-half RoPE of x [T, H, d] at positions pos [T] (fp64)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    inv = theta ** (-2.0 * np.arange(half, dtype=np.float64) / d)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]          # [T, d/2]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def qkv_rope(x, w_qkv, cu_seqlens, heads, head_dim, theta):
    """q, k, v [T, H, d] (fp64) of the fused projection; theta <= 0: no rotation."""
    xa, wa = _f64(x), _f64(w_qkv)
    T = xa.shape[0]
    qkv = xa @ wa.T                                                          # [T, 3*H*d]
    q, k, v = (qkv[:, i * heads * head_dim:(i + 1) * heads * head_dim].reshape(T, heads, head_dim)
               for i in range(3))
    if theta > 0:
        pos = positions(cu_seqlens, T)
        q, k = rope(q, pos, theta), rope(k, pos, theta)
    return q, k, v


def linear(x, w):
    """y = x w^T in fp64 (x [rows, in], w [out, in])."""
    return _f64(x) @ _f64(w).T
