"""Seeded synthetic inputs for packed variable-length attention.

This module holds input generators only: it draws q/k/v, builds ``cu_seqlens``
from image sizes and picks sampled query rows. It contains none of the
attention arithmetic, so both the CPU oracle (``oracle/``) and the CUDA path
(``dit_resolution_packed_b200``) may be fed from it without sharing code.

Conventions (Mage-Flow page, "Native-resolution sequence packing"):
  * q, k, v are ``[total_tokens, heads, head_dim]``, images concatenated;
  * ``cu_seqlens`` is int32 ``[B+1]`` = [0, L0, L0+L1, ...];
  * an image h x w at patch size 16 contributes (h/16)*(w/16) tokens.

Values are i.i.d. N(0, 1), drawn in fp32 on the CPU with
``torch.Generator().manual_seed(seed)`` in the order q, k, v and rounded once
to bf16.
"""
import json
import math
import os

import numpy as np
import torch

PATCH = 16
_HERE = os.path.dirname(os.path.abspath(__file__))
CONFIG_NAMES = ("tiny", "mixed", "training", "interactive", "long")
# packs of the short-segment (HBM-bound) regime, measured beside the configurations above
SHORT_PACK_NAMES = ("many_short", "thumbnails")


def tokens_for_image(h, w, patch=PATCH):
    """Token count of an h x w image patchified at ``patch`` (Mage-Flow page, packing section)."""
    if h % patch or w % patch:
        raise ValueError(f"image {h}x{w} is not a multiple of the patch size {patch}")
    return (h // patch) * (w // patch)


def cu_seqlens_from_lengths(lengths):
    """[0, L0, L0+L1, ...] as int32 (Mage-Flow page, ``packed_attention`` listing)."""
    cu = [0]
    for n in lengths:
        if n < 0:
            raise ValueError("negative segment length")
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32)


def load_config(name):
    with open(os.path.join(_HERE, "configs", name + ".json")) as f:
        return json.load(f)


def all_configs():
    return [load_config(n) for n in CONFIG_NAMES]


def valid_flops(segments, heads, head_dim):
    """Valid block-diagonal FLOPs of one forward: 4 * sum(L_i^2) * d * H (two GEMMs, 2 FLOP per MAC)."""
    return 4.0 * float(sum(int(n) * int(n) for n in segments)) * head_dim * heads


def random_qkv(total_tokens, heads, head_dim, seed, v_dim=None):
    """q, k, v drawn N(0,1) in fp32 (order q, k, v) from one seeded CPU generator, then rounded to bf16."""
    v_dim = head_dim if v_dim is None else v_dim
    g = torch.Generator().manual_seed(int(seed))
    q = torch.randn(total_tokens, heads, head_dim, generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn(total_tokens, heads, head_dim, generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(total_tokens, heads, v_dim, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return q, k, v, g


def make_inputs(cfg):
    """Inputs of a frozen workload: dict with q, k, v (bf16 CPU), cu_seqlens (int32 CPU), max_seqlen, scale."""
    segs = [int(n) for n in cfg["segments"]]
    T, H, d = sum(segs), int(cfg["heads"]), int(cfg["head_dim"])
    q, k, v, g = random_qkv(T, H, d, cfg["seed"])
    out = dict(q=q, k=k, v=v, cu_seqlens=cu_seqlens_from_lengths(segs),
               max_seqlen=max(segs) if segs else 0, scale=float(cfg["scale"]),
               segments=segs, heads=H, head_dim=d)
    if "key_outliers" in cfg:
        # 1% of key token rows (all heads) multiplied by the factor after the bf16 draw;
        # x8 is a power of two, so the product is exact in bf16.
        n_out = int(math.floor(cfg["key_outliers"]["fraction"] * T))
        idx = torch.randperm(T, generator=g)[:n_out]
        k[idx] = (k[idx].float() * cfg["key_outliers"]["factor"]).to(torch.bfloat16)
        out["outlier_rows"] = idx
    return out


def sampled_rows(cfg, per_head=None):
    """(token, head) pairs of the sampled query rows of a workload, as int64 / int32 CPU tensors.

    Per head h, ``per_head`` distinct token indices from
    ``torch.randperm(T, generator=manual_seed(seed_base + h))``.
    """
    T, H = int(sum(cfg["segments"])), int(cfg["heads"])
    spec = cfg.get("sampled_rows", dict(per_head=512, seed_base=1000 + int(cfg["seed"])))
    n = int(spec["per_head"] if per_head is None else per_head)
    n = min(n, T)
    toks, heads = [], []
    for h in range(H):
        g = torch.Generator().manual_seed(int(spec["seed_base"]) + h)
        idx = torch.randperm(T, generator=g)[:n]
        toks.append(idx.to(torch.int64))
        heads.append(torch.full((n,), h, dtype=torch.int32))
    return torch.cat(toks), torch.cat(heads)


def packing_layouts(lengths, bucket_size=4):
    """The same image mix laid out three ways (Mage-Flow page, the table after "Packing +
    Flash Attention varlen": padding to the longest, bucket grouping, native packing).

    Returns {scheme: dict(segments=[...], token_utilisation=u)} where ``segments`` are the
    sequence lengths a kernel processes: every image padded to the longest ("padded");
    images sorted by length and cut into groups of ``bucket_size``, each padded to its
    group's longest ("bucketed"); the images as they are ("packed").  The token
    utilisation is real tokens / processed tokens.
    """
    lengths = [int(n) for n in lengths if int(n) > 0]
    real = sum(lengths)
    longest = max(lengths)
    padded = [longest] * len(lengths)
    srt = sorted(lengths)
    bucketed = []
    for i in range(0, len(srt), bucket_size):
        grp = srt[i:i + bucket_size]
        bucketed += [max(grp)] * len(grp)
    out = {}
    for name, segs in (("padded", padded), ("bucketed", bucketed), ("packed", list(lengths))):
        out[name] = dict(segments=segs, token_utilisation=real / float(sum(segs)))
    return out


def random_dout(shape, seed):
    """The upstream gradient dL/dout of a backward workload: N(0,1) in fp32 from its own
    seeded CPU generator, rounded to bf16."""
    g = torch.Generator().manual_seed(int(seed))
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def random_pack(lengths, heads, head_dim, seed, scale=None):
    """An ad-hoc pack of the given segment lengths with seeded N(0,1) bf16 inputs."""
    lengths = [int(n) for n in lengths]
    T = sum(lengths)
    q, k, v, _ = random_qkv(T, heads, head_dim, seed)
    return dict(q=q, k=k, v=v, cu_seqlens=cu_seqlens_from_lengths(lengths),
                max_seqlen=max(lengths) if lengths else 0,
                scale=(1.0 / math.sqrt(head_dim)) if scale is None else float(scale),
                segments=lengths, heads=heads, head_dim=head_dim)


def sparseattn_worked_example():
    """Inputs of the worked example on the SparseAttn page ("AIGC fundamentals: SparseAttn", section 04).

    The page builds a toy video of 4 frames x (4x4) positions = 64 tokens, flattened
    frame-major (token i = frame*16 + position). Two heads with d = 4 + 16 = 20:
    head 0 carries amplitude 6 in the one-hot dimension of the token's frame,
    head 1 in dimension 4 + position; then N(0, 0.15) noise of shape (2, 64, 20)
    is added, k equals q, and v ~ N(0, 1) of shape (64, 3) is shared by both heads.
    Random numbers: ``numpy.random.default_rng(7)``, noise drawn before v.

    The construction follows the input lines of the script printed on that page
    (section 04) in the same order: the seeded draws must come in the page's order
    to reproduce its printed digits.  The rest of that script (masks, block costs,
    the result table) is not reproduced here.

    Returns fp64 numpy arrays q (2, 64, 20), k (2, 64, 20), v (64, 3) and the
    frame / position index of every token.
    """
    rng = np.random.default_rng(7)
    frames, positions = 4, 16
    n, d = frames * positions, frames + positions
    frame = np.repeat(np.arange(frames), positions)
    position = np.tile(np.arange(positions), frames)
    q = np.zeros((2, n, d), dtype=np.float64)
    q[0, np.arange(n), frame] = 6.0
    q[1, np.arange(n), frames + position] = 6.0
    q = q + rng.normal(0.0, 0.15, size=q.shape)
    k = q.copy()
    v = rng.normal(size=(n, 3))
    return dict(q=q, k=k, v=v, frame=frame, position=position)
