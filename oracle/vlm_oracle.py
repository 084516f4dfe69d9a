"""CPU oracle for the image half of the Mistral 3 / Pixtral multimodal forward.

TEST INFRASTRUCTURE. Only the tests, `__graft_entry__.smoke()` and the
`cpu_baseline` / reference leg of `bench.py` may import or run this module.
The product path (the C-ABI library and its Python binding) never calls it
and shares no code with it.

What it computes, step by step, as plain numpy in float64 (matmul is the only
library primitive used as a step):

  vision tower ("Mistral 3", KerasFormers, API: `Mistral3VisionModel`:
  conv patch embed -> RMS pre-norm -> 2D-rotary blocks over a packed
  variable-resolution patch sequence)
    a1  pixel normalisation with the processor's mean/std
        ("Mistral 3", API: `Mistral3ImageProcessor`)
    a2  patch embedding: a convolution with kernel = stride = patch size,
        no bias (reading: the pages give no bias)
    a3  `ln_pre` RMSNorm
    a4..a10  per block: RMSNorm -> q,k,v -> 2D RoPE on q,k -> attention within
        each image only -> o-projection + residual -> RMSNorm -> SiLU-gated MLP
        + residual
  patch-merging projector ("Mistral 3", API: `Mistral3Model`:
  `spatial_merge_size` 2, `projector_bias` False)
    a12 RMSNorm per patch, a13 2x2 unfold + concat -> merge linear,
    a14 linear -> GELU -> linear
  a15 masked scatter of the image rows into the text embeddings at
      `image_token_id` positions (vllm.cpp issue "Mistral3ForConditionalGeneration
      ...", "What we would contribute", item 2: gated so text rows stay
      byte-identical)

Readings taken where the pages are silent (each one is listed in the design
notes): no biases anywhere; eps 1e-5 for every vision RMSNorm (the pages give
1e-5 for the text model only); `ln_pre` plus pre-norm blocks and no final
norm; SiLU-gated MLP; RoPE frequencies w_k = theta^(-2k/64), even k to the
patch row, odd k to the patch column, rotation pairs (i, i+32); positions
restart at (0, 0) in every image or tile; the projector RMSNorm is applied per
patch before the merge; merged features in `unfold` channel-major order
c*m*m + dy*m + dx; GELU in its erf form.

Every function below is pinned by `tests/test_oracle_pins.py` against closed
forms, library routines or brute force. The composition (`tower_block`,
`tower`, `encode_merge_project`) is pinned by `tests/test_oracle_tower_pin.py`
against the same steps rebuilt from torch primitives (conv2d, rms_norm, a
complex-rotation RoPE, masked scaled_dot_product_attention, silu, unfold,
gelu), with planted composition mistakes that must fail. Nothing here is
"parity unpinned" except the end-to-end numbers of real trained weights,
which do not exist in this environment.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

# "Mistral 3" (KerasFormers), API table `Mistral3Model`: vision_embed_dim 1024,
# vision_mlp_dim 4096, vision_num_layers 24, vision_num_heads 16, patch_size 14,
# vision_rope_theta 10000, spatial_merge_size 2, image_token_id 10; text
# embed_dim 5120 is the projector's output width.
MISTRAL3 = dict(layers=24, width=1024, heads=16, head_dim=64, mlp=4096, patch=14,
                merge=2, proj_out=5120, image_token_id=10, rope_theta=1.0e4, eps=1.0e-5)

# "Pixtral-12B-2409": ViT, 24 layers, hidden 1024, 16 heads, patch_size 16,
# image_size 1024, intermediate 4096, rope_theta 1e4, no spatial merge.
PIXTRAL12B = dict(MISTRAL3, patch=16, merge=1)

# "Mistral 3" (KerasFormers), API table `Mistral3ImageProcessor`.
IMAGE_MEAN = (0.48145466, 0.4578275, 0.40821073)
IMAGE_STD = (0.26862954, 0.26130258, 0.27577711)
LONGEST_EDGE = 1540
PIXTRAL_TILE = 1024


# ---------------------------------------------------------------------------
# a0: shapes and positions
# ---------------------------------------------------------------------------

def patch_grid(height: int, width: int, patch: int) -> tuple:
    """(h, w) patches of an image that lies on the patch grid.

    "Mistral 3" intro: images are resized so they stay on the patch grid;
    off-grid sizes are rejected here (reading: no padding or cropping).
    """
    if height <= 0 or width <= 0 or height % patch or width % patch:
        raise ValueError(f"image {height}x{width} is not on the {patch}-pixel patch grid")
    return height // patch, width // patch


def merged_grid(h: int, w: int, merge: int) -> tuple:
    """(h/m, w/m) merged tokens; `spatial_merge_size` m ("Mistral 3", `Mistral3Model`)."""
    if h % merge or w % merge:
        raise ValueError(f"patch grid {h}x{w} is not divisible by merge {merge}")
    return h // merge, w // merge


def tile_count(height: int, width: int, tile: int = PIXTRAL_TILE) -> int:
    """Number of tile x tile tiles ("Pixtral-12B-2409", VISION TOKENS: 4096^2 -> 4x4 grid)."""
    if height % tile or width % tile:
        raise ValueError("image is not a whole number of tiles")
    return (height // tile) * (width // tile)


def positions(grids) -> tuple:
    """Per-token (row, col) patch positions and block boundaries.

    Patches are concatenated image after image, row-major inside each image
    ("Mistral 3", `Mistral3VisionModel`: packed variable-resolution sequence).
    Positions restart at (0, 0) in each image (reading).
    Returns (rows int64 [T], cols int64 [T], cu_seqlens int64 [n+1]).
    """
    rows, cols, cu = [], [], [0]
    for h, w in grids:
        rr, cc = np.meshgrid(np.arange(h), np.arange(w), indexing="ij")
        rows.append(rr.reshape(-1))
        cols.append(cc.reshape(-1))
        cu.append(cu[-1] + h * w)
    return (np.concatenate(rows).astype(np.int64), np.concatenate(cols).astype(np.int64),
            np.asarray(cu, dtype=np.int64))


# ---------------------------------------------------------------------------
# Image front end (before the path): resize onto the grid, Pixtral tiling
# ---------------------------------------------------------------------------

def pixels_from_u8(image_hwc: np.ndarray) -> np.ndarray:
    """Decoded u8 RGB [H, W, 3] -> float [3, H, W] in [0, 1] (value / 255).

    Reading: "Mistral 3", API `Mistral3ImageProcessor` gives the mean/std in
    [0, 1] units, so pixels enter the normalisation as u8 / 255.
    """
    x = np.asarray(image_hwc)
    if x.ndim != 3 or x.shape[2] != 3:
        raise ValueError("expected [H, W, 3]")
    return x.astype(np.float64).transpose(2, 0, 1) / 255.0


def resized_hw(height: int, width: int, longest_edge: int, grid: int) -> tuple:
    """Target size of the processor's resize.

    "Mistral 3" intro: the processor scales an image down until its longer
    side is at most longest_edge and keeps both sides on the patch grid.
    Reading: shrink (never enlarge) by r = max(H, W) / longest_edge when
    r > 1, flooring each side, then round each side up to a multiple of
    `grid` (patch size times the merge size, so the merge always finds whole
    2x2 blocks). Rounding up stays within longest_edge only when longest_edge
    is itself a multiple of grid, so any other longest_edge is rejected.
    """
    if height <= 0 or width <= 0 or longest_edge <= 0 or grid <= 0:
        raise ValueError("sizes must be positive")
    if longest_edge % grid:
        raise ValueError(f"longest_edge {longest_edge} is not a multiple of the grid {grid}")
    ratio = max(height, width) / longest_edge
    if ratio > 1.0:
        height, width = int(height // ratio), int(width // ratio)
    height, width = max(height, 1), max(width, 1)
    return -(-height // grid) * grid, -(-width // grid) * grid


def resize_bilinear(image: np.ndarray, out_h: int, out_w: int) -> np.ndarray:
    """Bilinear resampling with half-pixel centres (no antialiasing).

    Output pixel (y, x) samples the input at ((y + 1/2) H/out_h - 1/2,
    (x + 1/2) W/out_w - 1/2), clamped to the image, interpolating the four
    neighbours (reading: the pages do not name the filter).
    """
    x = np.asarray(image, dtype=np.float64)
    c, h, w = x.shape

    def axis(n_out, n_in):
        src = (np.arange(n_out) + 0.5) * (n_in / n_out) - 0.5
        src = np.clip(src, 0.0, n_in - 1)
        i0 = np.floor(src).astype(np.int64)
        i1 = np.minimum(i0 + 1, n_in - 1)
        return i0, i1, src - i0

    y0, y1, fy = axis(out_h, h)
    x0, x1, fx = axis(out_w, w)
    top = x[:, y0][:, :, x0] * (1 - fx) + x[:, y0][:, :, x1] * fx
    bot = x[:, y1][:, :, x0] * (1 - fx) + x[:, y1][:, :, x1] * fx
    return top * (1 - fy)[None, :, None] + bot * fy[None, :, None]


def tile_image(image: np.ndarray, tile: int = PIXTRAL_TILE) -> list:
    """Split [3, H, W] into tile x tile tiles, row-major over the tile grid
    ("Pixtral-12B-2409", VISION TOKENS: 4096^2 -> a 4x4 grid of 1024^2 tiles)."""
    c, h, w = image.shape
    tile_count(h, w, tile)
    return [np.asarray(image[:, i:i + tile, j:j + tile]) for i in range(0, h, tile) for j in range(0, w, tile)]


def expand_placeholders(input_ids, marker_id: int, counts, image_token_id: int) -> np.ndarray:
    """Each occurrence of marker_id, in order, becomes counts[k] copies of
    image_token_id; every other id is kept ("Mistral 3", "Several images in one
    conversation": the processor expands each image marker to that image's own
    token count). Raises if the number of markers differs from len(counts)."""
    out, k = [], 0
    for t in np.asarray(input_ids).reshape(-1):
        if t == marker_id:
            if k >= len(counts):
                raise ValueError("more markers than images")
            out.extend([image_token_id] * int(counts[k]))
            k += 1
        else:
            out.append(int(t))
    if k != len(counts):
        raise ValueError(f"{k} markers for {len(counts)} images")
    return np.asarray(out, dtype=np.int64)


# ---------------------------------------------------------------------------
# a1, a2: processor normalisation and patch embedding
# ---------------------------------------------------------------------------

def normalize_pixels(image: np.ndarray) -> np.ndarray:
    """(x - mean_c) / std_c per channel ("Mistral 3", `Mistral3ImageProcessor`)."""
    x = np.asarray(image, dtype=np.float64)
    mean = np.asarray(IMAGE_MEAN, dtype=np.float64)[:, None, None]
    std = np.asarray(IMAGE_STD, dtype=np.float64)[:, None, None]
    return (x - mean) / std


def im2col(image: np.ndarray, patch: int) -> np.ndarray:
    """[h*w, 3*p*p] patch rows; row = r*w + c, column = ch*p*p + ky*p + kx."""
    c, height, width = image.shape
    h, w = patch_grid(height, width, patch)
    x = np.asarray(image, dtype=np.float64).reshape(c, h, patch, w, patch)
    return x.transpose(1, 3, 0, 2, 4).reshape(h * w, c * patch * patch)


def patch_embed(image: np.ndarray, w_pe: np.ndarray) -> np.ndarray:
    """Conv with kernel = stride = p and no bias, as im2col . W_pe^T.

    "Mistral 3", `Mistral3VisionModel`: conv patch embed. w_pe is [D, 3, p, p].
    """
    d, _, p, _ = w_pe.shape
    return im2col(image, p) @ np.asarray(w_pe, dtype=np.float64).reshape(d, -1).T


# ---------------------------------------------------------------------------
# a3/a4/a9/a12: RMSNorm
# ---------------------------------------------------------------------------

def rms_norm(x: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * gain over the last axis ("RMS pre-norm")."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(gain, dtype=np.float64)


# ---------------------------------------------------------------------------
# a6: 2D rotary position embedding
# ---------------------------------------------------------------------------

def rope_frequencies(theta: float, head_dim: int) -> np.ndarray:
    """w_k = theta^(-2k/head_dim), k = 0 .. head_dim/2 - 1 (vision_rope_theta 1e4)."""
    k = np.arange(head_dim // 2, dtype=np.float64)
    return theta ** (-2.0 * k / head_dim)


def rope_angles(rows, cols, theta: float, head_dim: int) -> np.ndarray:
    """[T, head_dim/2] angles: pair i < head_dim/4 turns by row * w_{2i},
    pair i >= head_dim/4 by col * w_{2(i - head_dim/4) + 1} (reading: frequencies
    split between the patch's row and column index, even ones to the row)."""
    omega = rope_frequencies(theta, head_dim)
    rows = np.asarray(rows, dtype=np.float64)
    cols = np.asarray(cols, dtype=np.float64)
    return np.concatenate([np.outer(rows, omega[0::2]), np.outer(cols, omega[1::2])], axis=1)


def apply_rope(x: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """Rotate each pair (x_i, x_{i+half}) of every head by angles[:, i].

    x is [T, heads, head_dim]; angles is [T, head_dim/2].
    """
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    cos = np.cos(angles)[:, None, :]
    sin = np.sin(angles)[:, None, :]
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * cos - b * sin, b * cos + a * sin], axis=-1)


# ---------------------------------------------------------------------------
# a7: block-diagonal attention
# ---------------------------------------------------------------------------

def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, cu_seqlens) -> np.ndarray:
    """Bidirectional softmax attention where token t attends only to tokens of
    its own block [cu[b], cu[b+1]) (one block per image or tile).

    q, k, v are [T, heads, head_dim]; scores are scaled by 1/sqrt(head_dim);
    the softmax subtracts the row maximum before exponentiating.
    Returns [T, heads * head_dim], heads concatenated in order.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    t_total, heads, dh = q.shape
    out = np.zeros((t_total, heads, dh), dtype=np.float64)
    scale = 1.0 / math.sqrt(dh)
    for b in range(len(cu_seqlens) - 1):
        lo, hi = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
        for h in range(heads):
            kb, vb = k[lo:hi, h, :], v[lo:hi, h, :]
            for q0 in range(lo, hi, 2048):  # query chunks bound the score matrix's memory
                q1 = min(q0 + 2048, hi)
                s = (q[q0:q1, h, :] @ kb.T) * scale
                s -= s.max(axis=1, keepdims=True)
                p = np.exp(s)
                p /= p.sum(axis=1, keepdims=True)
                out[q0:q1, h, :] = p @ vb
    return out.reshape(t_total, heads * dh)


def attention_rows(q, k, v, cu_seqlens, rows) -> np.ndarray:
    """attention() evaluated for the listed query rows only (for sampled checks)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    _, heads, dh = q.shape
    cu = np.asarray(cu_seqlens)
    scale = 1.0 / math.sqrt(dh)
    out = np.zeros((len(rows), heads * dh), dtype=np.float64)
    for i, t in enumerate(rows):
        b = int(np.searchsorted(cu, t, side="right") - 1)
        lo, hi = int(cu[b]), int(cu[b + 1])
        for h in range(heads):
            s = (k[lo:hi, h, :] @ q[t, h, :]) * scale
            s -= s.max()
            p = np.exp(s)
            p /= p.sum()
            out[i, h * dh:(h + 1) * dh] = p @ v[lo:hi, h, :]
    return out


# ---------------------------------------------------------------------------
# a10, a14: activations
# ---------------------------------------------------------------------------

def silu(z):
    """z * sigmoid(z) = z / (1 + e^-z)."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def gelu(z):
    """Exact (erf) GELU: z * (1 + erf(z / sqrt 2)) / 2 (reading: the form is unstated)."""
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + _erf(z / math.sqrt(2.0)))


# ---------------------------------------------------------------------------
# a4..a10: one tower block, and the tower
# ---------------------------------------------------------------------------

def tower_block(x: np.ndarray, lw: dict, angles: np.ndarray, cu_seqlens, cfg: dict) -> np.ndarray:
    """x + attn(norm(x)), then + MLP(norm(.)) with pre-norm RMSNorms.

    lw holds wq, wk, wv, wo [D, D], w_gate, w_up [F, D], w_down [D, F],
    g_attn, g_ffn [D] (nn.Linear [out, in] layouts, y = x W^T).
    """
    t_total = x.shape[0]
    heads, dh, eps = cfg["heads"], cfg["head_dim"], cfg["eps"]
    xn = rms_norm(x, lw["g_attn"], eps)
    q = (xn @ lw["wq"].T).reshape(t_total, heads, dh)
    k = (xn @ lw["wk"].T).reshape(t_total, heads, dh)
    v = (xn @ lw["wv"].T).reshape(t_total, heads, dh)
    q = apply_rope(q, angles)
    k = apply_rope(k, angles)
    x = x + attention(q, k, v, cu_seqlens) @ lw["wo"].T
    xn = rms_norm(x, lw["g_ffn"], eps)
    hidden = silu(xn @ lw["w_gate"].T) * (xn @ lw["w_up"].T)
    return x + hidden @ lw["w_down"].T


def block_keys_values(x: np.ndarray, lw: dict, angles: np.ndarray, cfg: dict) -> tuple:
    """The part of tower_block shared by every query row: the attention-norm
    input of all rows and their rotated keys and values ([T, heads, head_dim])."""
    t_total = x.shape[0]
    heads, dh = cfg["heads"], cfg["head_dim"]
    xn = rms_norm(x, lw["g_attn"], cfg["eps"])
    k = apply_rope((xn @ lw["wk"].T).reshape(t_total, heads, dh), angles)
    v = (xn @ lw["wv"].T).reshape(t_total, heads, dh)
    return xn, k, v


def tower_block_rows(x: np.ndarray, lw: dict, angles: np.ndarray, cu_seqlens, cfg: dict, rows,
                     kv: tuple | None = None) -> np.ndarray:
    """tower_block() evaluated for the listed rows only: every step of the block
    is row-wise except attention, whose keys and values come from all rows of
    the row's block (pass `kv` from block_keys_values to reuse them)."""
    rows = np.asarray(rows)
    heads, dh, eps = cfg["heads"], cfg["head_dim"], cfg["eps"]
    xn, k, v = block_keys_values(x, lw, angles, cfg) if kv is None else kv
    q = apply_rope((xn[rows] @ lw["wq"].T).reshape(len(rows), heads, dh), angles[rows])
    qfull = np.zeros((x.shape[0], heads, dh))
    qfull[rows] = q
    xr = x[rows] + attention_rows(qfull, k, v, cu_seqlens, rows) @ lw["wo"].T
    xrn = rms_norm(xr, lw["g_ffn"], eps)
    hidden = silu(xrn @ lw["w_gate"].T) * (xrn @ lw["w_up"].T)
    return xr + hidden @ lw["w_down"].T


def layer_weights(tw: dict, layer: int) -> dict:
    names = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down", "g_attn", "g_ffn")
    return {n: np.asarray(tw[n][layer], dtype=np.float64) for n in names}


def tower(images, tw: dict, cfg: dict, layers: int | None = None, normalize: bool = True) -> np.ndarray:
    """Vision tower over a packed sequence of images.

    images: list of fp [3, H, W] arrays (raw U[0,1) pixels if `normalize`).
    tw: w_pe [D,3,p,p], g_pre [D], stacked per-layer tensors [L, ...].
    Returns the residual stream after the last block, [T, D] (no final norm).
    """
    p, eps = cfg["patch"], cfg["eps"]
    n_layers = cfg["layers"] if layers is None else layers
    grids = [patch_grid(im.shape[1], im.shape[2], p) for im in images]
    rows, cols, cu = positions(grids)
    w_pe = np.asarray(tw["w_pe"], dtype=np.float64)
    x = np.concatenate([patch_embed(normalize_pixels(im) if normalize else np.asarray(im, np.float64), w_pe)
                        for im in images], axis=0)
    x = rms_norm(x, tw["g_pre"], eps)
    angles = rope_angles(rows, cols, cfg["rope_theta"], cfg["head_dim"])
    for layer in range(n_layers):
        x = tower_block(x, layer_weights(tw, layer), angles, cu, cfg)
    return x


# ---------------------------------------------------------------------------
# FP8 (E4M3) tower GEMMs: the deployments the pages describe run FP8-native
# checkpoints ("Mistral 3" intro; vllm.cpp issue). Reading: weights quantised
# per output row with scale amax/448, activations with one static scale per
# GEMM input; the four tower GEMMs of every block run on E4M3 operands with
# fp32 accumulation; attention, norms, the patch embed and the projector stay
# as in the bf16 path.
# ---------------------------------------------------------------------------
E4M3_MAX = 448.0


def e4m3_round(x) -> np.ndarray:
    """Nearest value of the OCP FP8 E4M3 format (finite variant: 4 exponent
    bits with bias 7, 3 mantissa bits, largest finite 448, no infinities),
    ties to even, saturating to +-448. Normals cover [2^-6, 448] with 8
    steps per binade; below 2^-6 the step is the subnormal quantum 2^-9."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e = np.frexp(a)                       # a = f * 2^e, f in [0.5, 1)
    e = np.clip(e - 1, -6, 8)                # binade exponent, subnormals share 2^-6's step
    quantum = np.ldexp(1.0, (e - 3).astype(np.int64))
    q = np.minimum(np.round(a / quantum) * quantum, E4M3_MAX)  # np.round: half to even
    return np.where(np.isnan(x), np.nan, np.copysign(q, x))


def quantize_weight_rows(w) -> tuple:
    """Per-output-row E4M3 weights: s[n] = fp32(amax_n / 448) (1 for an all-zero
    row), q = e4m3(fp32(w / s[n])) with fp32 division. Returns (q, s) as
    float64 [N, K] and float32 [N]."""
    w32 = np.asarray(w, dtype=np.float32)
    amax = np.max(np.abs(w32), axis=1)
    sc = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    sc = np.where(sc > 0, sc, np.float32(1.0)).astype(np.float32)
    return e4m3_round((w32 / sc[:, None]).astype(np.float32)), sc


def fp8_linear(a, q_w: np.ndarray, s_w: np.ndarray, s_a: float) -> np.ndarray:
    """y = x W^T with both operands in E4M3: q_a = e4m3(fp32(a) * fp32(1/s_a)),
    y[:, n] = (q_a q_w^T)[:, n] * fp32(s_a * s_w[n])."""
    inv = np.float32(1.0 / np.float64(np.float32(s_a)))
    q_a = e4m3_round(np.asarray(a, dtype=np.float32) * inv)
    colscale = (np.float32(s_a) * np.asarray(s_w, dtype=np.float32)).astype(np.float64)
    return (q_a @ np.asarray(q_w, dtype=np.float64).T) * colscale[None, :]


def quantize_layer(lw: dict) -> dict:
    """E4M3 copies of one layer's GEMM weights (q and per-row scales)."""
    out = dict(lw)
    for n in ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down"):
        out[n + "_q"], out[n + "_s"] = quantize_weight_rows(lw[n])
    return out


def tower_block_fp8(x: np.ndarray, lq: dict, act_scales, angles: np.ndarray, cu_seqlens, cfg: dict) -> np.ndarray:
    """tower_block() with its four GEMMs (QKV, O, gate/up, down) on E4M3
    operands; act_scales = (s_attn_norm, s_attn_out, s_ffn_norm, s_hidden),
    the static scales of those four GEMM inputs."""
    t_total = x.shape[0]
    heads, dh, eps = cfg["heads"], cfg["head_dim"], cfg["eps"]
    xn = rms_norm(x, lq["g_attn"], eps)
    q = fp8_linear(xn, lq["wq_q"], lq["wq_s"], act_scales[0]).reshape(t_total, heads, dh)
    k = fp8_linear(xn, lq["wk_q"], lq["wk_s"], act_scales[0]).reshape(t_total, heads, dh)
    v = fp8_linear(xn, lq["wv_q"], lq["wv_s"], act_scales[0]).reshape(t_total, heads, dh)
    q = apply_rope(q, angles)
    k = apply_rope(k, angles)
    x = x + fp8_linear(attention(q, k, v, cu_seqlens), lq["wo_q"], lq["wo_s"], act_scales[1])
    xn = rms_norm(x, lq["g_ffn"], eps)
    hidden = silu(fp8_linear(xn, lq["w_gate_q"], lq["w_gate_s"], act_scales[2])) * \
        fp8_linear(xn, lq["w_up_q"], lq["w_up_s"], act_scales[2])
    return x + fp8_linear(hidden, lq["w_down_q"], lq["w_down_s"], act_scales[3])


def tower_fp8(images, tw: dict, act_scales, cfg: dict, layers: int | None = None,
              normalize: bool = True) -> np.ndarray:
    """tower() with tower_block_fp8 blocks; act_scales[l] holds layer l's four
    static activation scales."""
    p, eps = cfg["patch"], cfg["eps"]
    n_layers = cfg["layers"] if layers is None else layers
    grids = [patch_grid(im.shape[1], im.shape[2], p) for im in images]
    rows, cols, cu = positions(grids)
    w_pe = np.asarray(tw["w_pe"], dtype=np.float64)
    x = np.concatenate([patch_embed(normalize_pixels(im) if normalize else np.asarray(im, np.float64), w_pe)
                        for im in images], axis=0)
    x = rms_norm(x, tw["g_pre"], eps)
    angles = rope_angles(rows, cols, cfg["rope_theta"], cfg["head_dim"])
    for layer in range(n_layers):
        x = tower_block_fp8(x, quantize_layer(layer_weights(tw, layer)), act_scales[layer], angles, cu, cfg)
    return x


# ---------------------------------------------------------------------------
# NVFP4 (E2M1 with E4M3 block scales) GEMM operands: the deployment on the
# vllm.cpp issue ("Why this one is smaller than it looks", the quantisation
# loaders bullet) loads NVFP4 weights: packed 4-bit values with a scale per
# block. Reading: a block is 16 consecutive values of a row along K, its
# scale is one E4M3 number, and the tensor has one fp32 global scale, so
# x ~ q * s_block * s_global. Both GEMM operands take this format (the
# block-scaled FP4 tensor-core product needs both in FP4): weights with
# s_global = amax(W) / (6 * 448), activations with a static s_global per GEMM
# input and block scales computed from the data. Every scaling step below is
# one fp32 operation, so an implementation in fp32 reaches the same codes.
# ---------------------------------------------------------------------------
E2M1_MAX = 6.0
NVFP4_BLOCK = 16


def e2m1_round(x) -> np.ndarray:
    """Nearest value of the E2M1 format (1 sign, 2 exponent bits with bias 1,
    1 mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), ties to the even
    mantissa, saturating to +-6. Binade [2^e, 2^(e+1)) has step 2^(e-1);
    below 1 the step is the subnormal quantum 0.5."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e = np.frexp(a)                       # a = f * 2^e, f in [0.5, 1)
    e = np.clip(e - 1, 0, 2)                 # binade exponent; subnormals share binade 0's step
    quantum = np.ldexp(1.0, (e - 1).astype(np.int64))
    q = np.minimum(np.round(a / quantum) * quantum, E2M1_MAX)  # np.round: half to even
    return np.where(np.isnan(x), np.nan, np.copysign(q, x))


def nvfp4_global_scale(x) -> np.float32:
    """Per-tensor scale that maps the tensor's largest magnitude onto the
    largest block scale times the largest element: fp32(amax / 2688)."""
    amax = np.float32(np.max(np.abs(np.asarray(x, dtype=np.float32))))
    return np.float32(amax / np.float32(E2M1_MAX * E4M3_MAX))


def quantize_nvfp4(x, s_global) -> tuple:
    """Rows of x [R, K] (K a multiple of 16) to NVFP4 with the given fp32
    global scale. Per block of 16: s_b = e4m3(fp32(amax_b / fp32(6 s_g)));
    r = fp32(1 / fp32(s_b s_g)) (0 when s_b is 0); q = e2m1(fp32(x r)).
    Returns (q float64 [R, K] on the E2M1 grid, s_b float64 [R, K/16])."""
    x32 = np.asarray(x, dtype=np.float32)
    r_, k_ = x32.shape
    assert k_ % NVFP4_BLOCK == 0
    sg = np.float32(s_global)
    blocks = x32.reshape(r_, k_ // NVFP4_BLOCK, NVFP4_BLOCK)
    amax = np.max(np.abs(blocks), axis=2)
    s_b = e4m3_round((amax / np.float32(np.float32(E2M1_MAX) * sg)).astype(np.float32))
    denom = (s_b.astype(np.float32) * sg).astype(np.float32)
    with np.errstate(divide="ignore"):
        recip = np.where(denom > 0, np.float32(1.0) / np.where(denom > 0, denom, np.float32(1.0)),
                         np.float32(0.0)).astype(np.float32)
    q = e2m1_round((blocks * recip[:, :, None]).astype(np.float32))
    return q.reshape(r_, k_), s_b


def dequantize_nvfp4(q, s_b, s_global) -> np.ndarray:
    """q * s_b (each scale repeated over its 16 values) * s_g, in float64."""
    q = np.asarray(q, dtype=np.float64)
    return q * np.repeat(np.asarray(s_b, dtype=np.float64), NVFP4_BLOCK, axis=1) * np.float64(np.float32(s_global))


def nvfp4_linear(q_a, s_a, g_a, q_w, s_w, g_w) -> np.ndarray:
    """y = A W^T on NVFP4 operands: the blocked products summed exactly, then
    the one fp32 factor fp32(g_a * g_w) for both global scales."""
    a = np.asarray(q_a, np.float64) * np.repeat(np.asarray(s_a, np.float64), NVFP4_BLOCK, axis=1)
    w = np.asarray(q_w, np.float64) * np.repeat(np.asarray(s_w, np.float64), NVFP4_BLOCK, axis=1)
    alpha = np.float64(np.float32(np.float32(g_a) * np.float32(g_w)))
    return (a @ w.T) * alpha


# The four tower GEMMs as they are executed: [Wq; Wk; Wv], Wo, [W_gate; W_up], W_down.
NVFP4_GEMMS = (("qkv", ("wq", "wk", "wv")), ("o", ("wo",)), ("gate_up", ("w_gate", "w_up")), ("down", ("w_down",)))


def quantize_layer_nvfp4(lw: dict) -> dict:
    """NVFP4 copies of one layer's GEMM weights: one global scale per executed
    GEMM weight (QKV and gate/up each as one tensor), block scales per 16 values
    of a row. Entry name -> (q, s_b, s_g)."""
    out = dict(lw)
    for name, parts in NVFP4_GEMMS:
        w = np.concatenate([np.asarray(lw[n], dtype=np.float32) for n in parts])
        g = nvfp4_global_scale(w)
        q, sb = quantize_nvfp4(w, g)
        out[name] = (q, sb, g)
    return out


def _nvfp4_gemm(a, lq: dict, name: str, g_a) -> np.ndarray:
    q_w, s_w, g_w = lq[name]
    q_a, s_a = quantize_nvfp4(np.asarray(a, dtype=np.float32), g_a)
    return nvfp4_linear(q_a, s_a, g_a, q_w, s_w, g_w)


def tower_block_nvfp4(x: np.ndarray, lq: dict, act_scales, angles: np.ndarray, cu_seqlens, cfg: dict) -> np.ndarray:
    """tower_block() with its four GEMMs on NVFP4 operands: each GEMM input is
    rounded to fp32 and quantised with its static global scale
    act_scales = (g_attn_norm, g_attn_out, g_ffn_norm, g_hidden), the weights
    as quantize_layer_nvfp4 left them. Attention, norms and RoPE as in bf16."""
    t_total = x.shape[0]
    heads, dh, eps, d = cfg["heads"], cfg["head_dim"], cfg["eps"], cfg["width"]
    xn = rms_norm(x, lq["g_attn"], eps)
    qkv = _nvfp4_gemm(xn, lq, "qkv", act_scales[0])
    q = apply_rope(qkv[:, :d].reshape(t_total, heads, dh), angles)
    k = apply_rope(qkv[:, d:2 * d].reshape(t_total, heads, dh), angles)
    v = qkv[:, 2 * d:].reshape(t_total, heads, dh)
    x = x + _nvfp4_gemm(attention(q, k, v, cu_seqlens), lq, "o", act_scales[1])
    xn = rms_norm(x, lq["g_ffn"], eps)
    gu = _nvfp4_gemm(xn, lq, "gate_up", act_scales[2])
    f = gu.shape[1] // 2
    return x + _nvfp4_gemm(silu(gu[:, :f]) * gu[:, f:], lq, "down", act_scales[3])


def tower_nvfp4(images, tw: dict, act_scales, cfg: dict, layers: int | None = None,
                normalize: bool = True) -> np.ndarray:
    """tower() with tower_block_nvfp4 blocks; act_scales[l] holds layer l's four
    static activation global scales, the weights are quantised per layer as
    quantize_layer_nvfp4 does."""
    p, eps = cfg["patch"], cfg["eps"]
    n_layers = cfg["layers"] if layers is None else layers
    grids = [patch_grid(im.shape[1], im.shape[2], p) for im in images]
    rows, cols, cu = positions(grids)
    w_pe = np.asarray(tw["w_pe"], dtype=np.float64)
    x = np.concatenate([patch_embed(normalize_pixels(im) if normalize else np.asarray(im, np.float64), w_pe)
                        for im in images], axis=0)
    x = rms_norm(x, tw["g_pre"], eps)
    angles = rope_angles(rows, cols, cfg["rope_theta"], cfg["head_dim"])
    for layer in range(n_layers):
        x = tower_block_nvfp4(x, quantize_layer_nvfp4(layer_weights(tw, layer)), act_scales[layer], angles, cu, cfg)
    return x


# ---------------------------------------------------------------------------
# a12..a14: patch-merging projector
# ---------------------------------------------------------------------------

def merge_unfold(x: np.ndarray, grids, merge: int) -> np.ndarray:
    """2x2 (m x m) unfold + concat per image.

    For image b with patch grid (h, w) and merged position (i, j):
    z[c*m*m + dy*m + dx] = x[off_b + (m*i + dy)*w + (m*j + dx), c]
    (channel-major order of an unfold with kernel = stride = m). Merged tokens
    are row-major per image, images concatenated.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[1]
    out, off = [], 0
    for h, w in grids:
        hm, wm = merged_grid(h, w, merge)
        img = x[off:off + h * w].reshape(hm, merge, wm, merge, d)  # [i, dy, j, dx, c]
        out.append(img.transpose(0, 2, 4, 1, 3).reshape(hm * wm, d * merge * merge))
        off += h * w
    return np.concatenate(out, axis=0)


def projector(x_tower: np.ndarray, grids, pw: dict, cfg: dict) -> np.ndarray:
    """RMSNorm per patch -> m x m merge -> merge linear -> W1 -> GELU -> W2, no biases.

    ("Mistral 3", `Mistral3Model`: 2x2 patch-merging projector, projector_bias
    False, text width 5120.) pw: g_proj [D], w_merge [D, m*m*D], w1 [E, D],
    w2 [E, E].
    cfg["norm_after_merge"] (default False) takes the other reading of the
    pages' order: merge -> merge linear -> RMSNorm over the merged D-vector ->
    W1 -> GELU -> W2 (the same g_proj; with merge 1 both readings coincide).
    """
    eps, m = cfg["eps"], cfg["merge"]
    after = bool(cfg.get("norm_after_merge", False)) and m > 1
    xn = np.asarray(x_tower, dtype=np.float64) if after else rms_norm(x_tower, pw["g_proj"], eps)
    z = merge_unfold(xn, grids, m) if m > 1 else xn
    y = z @ np.asarray(pw["w_merge"], dtype=np.float64).T if m > 1 else z
    if after:
        y = rms_norm(y, pw["g_proj"], eps)
    return gelu(y @ np.asarray(pw["w1"], dtype=np.float64).T) @ np.asarray(pw["w2"], dtype=np.float64).T


# ---------------------------------------------------------------------------
# a15: masked scatter
# ---------------------------------------------------------------------------

def scatter(input_ids: np.ndarray, image_rows: np.ndarray, text_rows: np.ndarray,
            image_token_id: int) -> np.ndarray:
    """Copy image row k into the k-th position whose id equals image_token_id.

    Rows are copied as raw bits (any dtype); every other row is left as it
    was. Raises if the placeholder count differs from the number of image rows.
    """
    ids = np.asarray(input_ids).reshape(-1)
    out = np.array(text_rows, copy=True)
    k = 0
    for i in range(ids.shape[0]):
        if ids[i] == image_token_id:
            if k < image_rows.shape[0]:
                out[i] = image_rows[k]
            k += 1
    if k != image_rows.shape[0]:
        raise ValueError(f"{k} placeholders for {image_rows.shape[0]} image rows")
    return out


# ---------------------------------------------------------------------------
# The whole image half
# ---------------------------------------------------------------------------

def encode_merge_project(images, tw: dict, pw: dict, cfg: dict, layers: int | None = None,
                         normalize: bool = True) -> tuple:
    """(tower output [T, D], projected image embeddings [T_m, E])."""
    grids = [patch_grid(im.shape[1], im.shape[2], cfg["patch"]) for im in images]
    xt = tower(images, tw, cfg, layers=layers, normalize=normalize)
    return xt, projector(xt, grids, pw, cfg)


def flops(cfg: dict, grids, layers: int | None = None) -> float:
    """Algorithmic FLOPs (2 per multiply-add) of tower + merge + projector.

    Attention is counted over each block's own L_b^2 query-key pairs only.
    """
    d, f, e, m, p = cfg["width"], cfg["mlp"], cfg["proj_out"], cfg["merge"], cfg["patch"]
    n_layers = cfg["layers"] if layers is None else layers
    total = 0.0
    for h, w in grids:
        lb = h * w
        per_layer = lb * 2 * (3 * d * d + d * d + 3 * d * f) + 4 * lb * lb * d
        total += n_layers * per_layer + lb * 2 * 3 * p * p * d
        tm = lb // (m * m)
        total += tm * (2 * (m * m * d) * d if m > 1 else 0) + tm * 2 * (d * e + e * e)
    return total
