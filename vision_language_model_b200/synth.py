"""Seeded synthetic inputs for the image half of the Mistral 3 / Pixtral forward.

This module only draws random numbers and lays them out in the shapes the
pages describe. It holds no step of the method's arithmetic, so both the CPU
oracle (via the tests) and the CUDA path (via the tests and the bench) take
their inputs from here.

Recipe (one torch CPU generator per named tensor, so every tensor is
reproducible on its own and independent of call order):

* matrices: N(0, 0.02), rounded to bf16 (round-to-nearest-even);
* RMSNorm gains: 1 + N(0, 0.02), rounded to bf16 and kept as fp32 values;
* pixels: U[0, 1) per channel, fp32, before the processor's mean/std
  normalisation (which belongs to the path, not to this module);
* text ids: uniform in [11, 131072); text embeddings: N(0, 1) in bf16.

Image shapes follow the pages' workloads: Mistral 3's default 1540x1540
image at patch 14 (KerasFormers "Mistral 3", API table `Mistral3Model`),
Pixtral-12B's 1024x1024 tiles at patch 16 ("Pixtral-12B-2409", VISION
TOKENS), and packed variable-resolution batches whose sides are multiples of
28 (patch 14 times merge 2, so every image lands on the merged grid).
"""
from __future__ import annotations

import torch

_MASK64 = (1 << 64) - 1


def _fnv1a64(text: str) -> int:
    h = 0xCBF29CE484222325
    for byte in text.encode("utf-8"):
        h ^= byte
        h = (h * 0x100000001B3) & _MASK64
    return h


def _splitmix64(x: int) -> int:
    x = (x + 0x9E3779B97F4A7C15) & _MASK64
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & _MASK64
    return x ^ (x >> 31)


def stream_seed(seed: int, name: str) -> int:
    """63-bit seed of the generator that draws tensor `name` under `seed`."""
    return _splitmix64((seed & _MASK64) ^ _fnv1a64(name)) >> 1


def generator(seed: int, name: str) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(stream_seed(seed, name))
    return g


def randn_bf16(seed: int, name: str, shape, std: float = 0.02) -> torch.Tensor:
    """bf16 tensor of N(0, std) draws (CPU)."""
    t = torch.randn(tuple(shape), generator=generator(seed, name), dtype=torch.float32)
    return (t * std).to(torch.bfloat16)


def gain(seed: int, name: str, shape, std: float = 0.02) -> torch.Tensor:
    """fp32 tensor of 1 + N(0, std), rounded through bf16 so both sides see the same value."""
    t = torch.randn(tuple(shape), generator=generator(seed, name), dtype=torch.float32)
    return (1.0 + std * t).to(torch.bfloat16).to(torch.float32)


def pixels_u01(seed: int, name: str, height: int, width: int) -> torch.Tensor:
    """fp32 [3, H, W] image with U[0, 1) channels (before normalisation)."""
    return torch.rand((3, height, width), generator=generator(seed, name), dtype=torch.float32)


def photo_u8(seed: int, name: str, height: int, width: int) -> torch.Tensor:
    """uint8 [H, W, 3] RGB image as a decoder returns it: per channel a mean
    level plus three random low-frequency plane waves (1-4 periods across the
    image, like the slow shading of a photograph) plus uniform +-24 grain,
    rounded and clipped to [0, 255]."""
    g = generator(seed, name)
    y = torch.arange(height, dtype=torch.float64)[:, None] / height
    x = torch.arange(width, dtype=torch.float64)[None, :] / width
    chans = []
    for _ in range(3):
        p = torch.rand(10, generator=g, dtype=torch.float64)
        field = 60.0 + 135.0 * p[0]
        for k in range(3):
            fy, fx, ph = 1.0 + 3.0 * p[1 + 3 * k], 1.0 + 3.0 * p[2 + 3 * k], 6.283185307179586 * p[3 + 3 * k]
            field = field + 30.0 * torch.sin(6.283185307179586 * (fy * y + fx * x) + ph)
        grain = (torch.rand((height, width), generator=g, dtype=torch.float64) - 0.5) * 48.0
        chans.append(field + grain)
    return torch.stack(chans, -1).clamp(0, 255).round().to(torch.uint8).contiguous()


# ---------------------------------------------------------------------------
# Model hyperparameters of the synthetic towers (shapes only)
# ---------------------------------------------------------------------------

def tower_weights(seed: int, layers: int, width: int, mlp: int, patch: int,
                  qk_scale: float = 1.0) -> dict:
    """Random tower weights in the natural nn.Linear [out, in] layouts.

    `qk_scale` multiplies Wq and Wk (a "peaked" variant: with N(0, 0.02)
    weights attention scores are near zero and softmax is near uniform).
    """
    d, f, p = width, mlp, patch
    w = {
        "w_pe": randn_bf16(seed, "w_pe", (d, 3, p, p)),
        "g_pre": gain(seed, "g_pre", (d,)),
        "wq": randn_bf16(seed, "wq", (layers, d, d), 0.02 * qk_scale),
        "wk": randn_bf16(seed, "wk", (layers, d, d), 0.02 * qk_scale),
        "wv": randn_bf16(seed, "wv", (layers, d, d)),
        "wo": randn_bf16(seed, "wo", (layers, d, d)),
        "w_gate": randn_bf16(seed, "w_gate", (layers, f, d)),
        "w_up": randn_bf16(seed, "w_up", (layers, f, d)),
        "w_down": randn_bf16(seed, "w_down", (layers, d, f)),
        "g_attn": gain(seed, "g_attn", (layers, d)),
        "g_ffn": gain(seed, "g_ffn", (layers, d)),
    }
    return w


def fp8_act_scales(layers: int) -> list:
    """Static E4M3 activation scales per layer for the synthetic towers: the
    GEMM inputs' ranges under N(0, 0.02) weights and ~1 gains are about
    |normed x| <= 8, |attention output| <= 4 (the values of v) and |gated
    hidden| <= 16; each scale maps that bound to 448."""
    return [[8.0 / 448.0, 4.0 / 448.0, 8.0 / 448.0, 16.0 / 448.0] for _ in range(layers)]


def nvfp4_act_scales(layers: int) -> list:
    """Static NVFP4 activation global scales per layer for the synthetic towers:
    the same bounds as fp8_act_scales (8, 4, 8, 16), each mapped to the largest
    E2M1 value times the largest E4M3 block scale, 6 * 448 = 2688."""
    return [[8.0 / 2688.0, 4.0 / 2688.0, 8.0 / 2688.0, 16.0 / 2688.0] for _ in range(layers)]


def projector_weights(seed: int, width: int, merge: int, proj_out: int) -> dict:
    d, e, m = width, proj_out, merge
    return {
        "g_proj": gain(seed, "g_proj", (d,)),
        "w_merge": randn_bf16(seed, "w_merge", (d, d * m * m)),
        "w1": randn_bf16(seed, "w1", (e, d)),
        "w2": randn_bf16(seed, "w2", (e, e)),
    }


# ---------------------------------------------------------------------------
# Image batches
# ---------------------------------------------------------------------------

def packed_sizes(seed: int, n_images: int, lo_units: int = 10, hi_units: int = 55,
                 unit: int = 28) -> list:
    """Sides drawn independently and uniformly from unit * {lo..hi} (aspect free)."""
    g = generator(seed, "packed_sizes")
    units = torch.randint(lo_units, hi_units + 1, (n_images, 2), generator=g)
    return [(int(a) * unit, int(b) * unit) for a, b in units.tolist()]


def images(seed: int, sizes) -> list:
    """One U[0,1) fp32 [3,H,W] tensor per (H, W)."""
    return [pixels_u01(seed, f"image{i}", h, w) for i, (h, w) in enumerate(sizes)]


def tile_sizes(height: int, width: int, tile: int = 1024) -> list:
    """Sizes of the tiles a large image is split into (row-major tile order)."""
    return [(tile, tile)] * ((height // tile) * (width // tile))


def text_sequences(seed: int, n_seq: int, seq_len: int, runs, image_token_id: int = 10,
                   vocab: int = 131072, lo_id: int = 11) -> torch.Tensor:
    """int64 [n_seq, seq_len] ids U[lo_id, vocab) with placeholder runs.

    `runs[s]` is the list of run lengths that sequence `s` carries; each run
    starts at a seeded offset and runs do not overlap.
    """
    g = generator(seed, "text_ids")
    ids = torch.randint(lo_id, vocab, (n_seq, seq_len), generator=g, dtype=torch.int64)
    g_off = generator(seed, "placeholder_offsets")
    for s, seq_runs in enumerate(runs):
        total = sum(seq_runs)
        if total > seq_len:
            raise ValueError("placeholder runs longer than the sequence")
        free = seq_len - total
        # split the free slots into len(runs)+1 gaps at seeded cut points
        cuts = sorted(torch.randint(0, free + 1, (len(seq_runs),), generator=g_off).tolist())
        pos, prev = 0, 0
        for run, cut in zip(seq_runs, cuts):
            pos += cut - prev
            prev = cut
            ids[s, pos:pos + run] = image_token_id
            pos += run
    return ids


def prompt_with_markers(seed: int, n_text: int, n_images: int, marker_id: int, vocab: int = 131072,
                        lo_id: int = 11) -> torch.Tensor:
    """int64 [n_text + n_images] ids: U[lo_id, vocab) text with one marker_id
    per image at seeded, distinct positions (a prompt before expansion)."""
    g = generator(seed, "prompt_ids")
    n = n_text + n_images
    ids = torch.randint(lo_id, vocab, (n,), generator=g, dtype=torch.int64)
    where = torch.randperm(n, generator=generator(seed, "marker_positions"))[:n_images]
    ids[where] = marker_id
    return ids


def text_embeddings(seed: int, n_tokens: int, width: int) -> torch.Tensor:
    return randn_bf16(seed, "text_embeds", (n_tokens, width), 1.0)
