"""Thin ctypes binding of libvlm_b200.so (include/vlm.h, include/vlm_kernels.h).

Argument marshalling only: torch supplies device memory and the current CUDA
stream; every step of the path runs in the library's sm_100a kernels. There
is no fallback: if the library is missing or a tensor is not on a CUDA
device, the call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

# VLM_B200_LIBRARY selects another build of the library, such as the
# index-checked libvlm_b200_debug.so beside this file.
_LIB_PATH = os.environ.get("VLM_B200_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)),
                                                                "libvlm_b200.so")
DEBUG_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvlm_b200_debug.so")
_lib = None

# vlm_status values (include/vlm.h)
OK, ERR_INVALID_ARG, ERR_BAD_SHAPE, ERR_WORKSPACE, ERR_COUNT_MISMATCH, ERR_TIMEOUT, ERR_CUDA, ERR_UNSUPPORTED = \
    0, -1, -2, -3, -4, -5, -6, -7
# epilogues (include/vlm_kernels.h)
EPI_BF16, EPI_F32, EPI_RESID, EPI_SWIGLU, EPI_ROPE, EPI_GELU = range(6)
# profiling kernel classes
KCLASS = {"gemm": 0, "attention": 1, "rmsnorm": 2, "im2col": 3, "merge": 4, "scatter": 5, "setup": 6, "pack": 7,
          "resize": 8, "expand": 9}


class VlmError(RuntimeError):
    def __init__(self, rc: int, what: str):
        self.rc = rc
        super().__init__(f"{what}: {status_string(rc)} ({rc})")


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("layers", "width", "heads", "head_dim", "mlp", "patch", "merge", "proj_out", "image_token_id")] + \
               [("rope_theta", ctypes.c_float), ("eps", ctypes.c_float), ("normalize", ctypes.c_int32),
                ("norm_after_merge", ctypes.c_int32), ("sm_budget", ctypes.c_int32)]

    def as_dict(self) -> dict:
        return {n: getattr(self, n) for n, _ in self._fields_}


class TowerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w_pe", "g_pre", "wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down", "g_attn", "g_ffn")]


class ProjectorWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("g_proj", "w_merge", "w1", "w2")]


def _torch_empty(shape, dtype, device) -> torch.Tensor:
    return torch.empty(shape, dtype=dtype, device=device)


# Every device buffer this module allocates (outputs, workspaces, packed
# weights, status words) comes from here; a test harness may install its own
# allocator, for example one that surrounds each buffer with guard bytes.
_alloc = _torch_empty


def set_allocator(fn=None):
    """Install fn(shape, dtype, device) -> tensor as the allocator of this
    module's device buffers (None restores torch.empty); returns the old one."""
    global _alloc
    old, _alloc = _alloc, (fn or _torch_empty)
    return old


def _empty(shape, dtype, device) -> torch.Tensor:
    return _alloc(shape, dtype, device)


def _zeros(shape, dtype, device) -> torch.Tensor:
    return _alloc(shape, dtype, device).zero_()


def lib_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with `python -m vision_language_model_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        P, I32, I64, SZ, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
        CP = ctypes.POINTER(Config)
        sig = {
            "vlm_status_string": (ctypes.c_char_p, [I32]),
            "vlm_status_sync": (I32, [P, P]),
            "vlm_config_preset": (I32, [I32, CP]),
            "vlm_tower_packed_bytes": (SZ, [CP]),
            "vlm_pack_tower": (I32, [CP, ctypes.POINTER(TowerWeights), P, SZ, P]),
            "vlm_projector_packed_bytes": (SZ, [CP]),
            "vlm_pack_projector": (I32, [CP, ctypes.POINTER(ProjectorWeights), P, SZ, P]),
            "vlm_num_patches": (I64, [CP, P, I32]),
            "vlm_num_merged": (I64, [CP, P, I32]),
            "vlm_encode_workspace_size": (SZ, [CP, P, I32]),
            "vlm_encode": (I32, [CP, P, P, I32, P, P, P, SZ, P, P]),
            "vlm_merge_project_workspace_size": (SZ, [CP, P, I32]),
            "vlm_merge_project": (I32, [CP, P, P, I32, P, P, P, SZ, P, P]),
            "vlm_merge_project_scatter_workspace_size": (SZ, [CP, P, I32, I64]),
            "vlm_merge_project_scatter": (I32, [CP, P, P, I32, P, P, I64, P, P, SZ, P, P]),
            "vlm_scatter_workspace_size": (SZ, [I64]),
            "vlm_scatter": (I32, [P, I64, I64, P, I64, P, I64, P, SZ, P, P]),
            "vlm_resize_target": (I32, [I32, I32, I32, I32, ctypes.POINTER(ctypes.c_int32),
                                        ctypes.POINTER(ctypes.c_int32)]),
            "vlm_preprocess": (I32, [P, P, I32, P, I32, P, P]),
            "vlm_expand_placeholders_workspace_size": (SZ, [I64, I32]),
            "vlm_expand_placeholders": (I32, [P, I64, I64, P, I32, I64, P, I64, ctypes.POINTER(I64), P, SZ, P, P]),
            "vlm_tower_fp8_packed_bytes": (SZ, [CP]),
            "vlm_pack_tower_fp8": (I32, [CP, ctypes.POINTER(TowerWeights), P, P, SZ, P]),
            "vlm_encode_fp8": (I32, [CP, P, P, I32, P, P, P, P, SZ, P, P]),
            "vlm_tower_nvfp4_packed_bytes": (SZ, [CP]),
            "vlm_pack_tower_nvfp4": (I32, [CP, ctypes.POINTER(TowerWeights), P, P, SZ, P]),
            "vlm_encode_nvfp4_workspace_size": (SZ, [CP, P, I32]),
            "vlm_encode_nvfp4": (I32, [CP, P, P, I32, P, P, P, P, SZ, P, P]),
            "vlm_gemm_fp8": (I32, [I32, P, P, P, F, I64, I64, I64, P, P, P, P, I64, P, P]),
            "vlm_rmsnorm_fp8": (I32, [P, P, P, P, I64, I32, F, F, P]),
            "vlm_nvfp4_sf_bytes": (SZ, [I64, I64]),
            "vlm_amax_scale": (I32, [P, I32, I64, F, P, P]),
            "vlm_quant_nvfp4": (I32, [P, I32, I64, I64, P, P, P, P]),
            "vlm_gemm_nvfp4": (I32, [I32, P, P, P, P, P, P, I64, I64, I64, P, P, P]),
            "vlm_gemm_nvfp4_ex": (I32, [I32, P, P, P, P, P, P, I64, I64, I64, P, P, F, P, P, I64, P, P]),
            "vlm_rmsnorm_nvfp4": (I32, [P, P, P, P, P, I64, I32, F, F, P]),
            "vlm_attention_nvfp4": (I32, [P, I64, I32, I32, P, I32, P, P, F, P, SZ, P, P]),
            "vlm_patch_embed": (I32, [CP, P, P, I32, P, P, P, SZ, P, P]),
            "vlm_launch_count": (I64, []),
            "vlm_profile_enable": (I32, [I32]),
            "vlm_profile_query": (I32, [I32, ctypes.POINTER(I64), ctypes.POINTER(ctypes.c_double)]),
            "vlm_gemm": (I32, [I32, P, P, I64, I64, I64, P, P, P, P, I64, P, P]),
            "vlm_rope_table": (I32, [F, I32, I32, P, P]),
            "vlm_attention_workspace_size": (SZ, [I32]),
            "vlm_attention": (I32, [P, I64, I32, I32, P, I32, P, P, SZ, P, P]),
            "vlm_rmsnorm": (I32, [P, P, P, P, I64, I32, F, P]),
            "vlm_selftest_wait_timeout": (I32, [I64, P, P]),
            "vlm_debug_build": (I32, []),
            "vlm_debug_checks": (I32, [ctypes.POINTER(ctypes.c_int32)]),
            "vlm_debug_selftest_bounds": (I32, [P, I32, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(rc: int) -> str:
    return lib().vlm_status_string(int(rc)).decode()


def _check(rc: int, what: str) -> None:
    if rc != OK:
        raise VlmError(rc, what)


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dev(t: torch.Tensor | None, name: str) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _hw_array(image_hw) -> tuple:
    flat = [int(v) for hw in image_hw for v in hw]
    arr = (ctypes.c_int32 * max(1, len(flat)))(*flat)
    return arr, len(flat) // 2


# ---------------------------------------------------------------------------
# Configs
# ---------------------------------------------------------------------------

def preset(name: str = "mistral3", **overrides) -> Config:
    cfg = Config()
    _check(lib().vlm_config_preset({"mistral3": 0, "pixtral12b": 1}[name], ctypes.byref(cfg)), "vlm_config_preset")
    for k, v in overrides.items():
        setattr(cfg, k, v)
    return cfg


def num_patches(cfg: Config, image_hw) -> int:
    arr, n = _hw_array(image_hw)
    t = lib().vlm_num_patches(ctypes.byref(cfg), arr, n)
    if t < 0:
        raise VlmError(int(t), "vlm_num_patches")
    return int(t)


def num_merged(cfg: Config, image_hw) -> int:
    arr, n = _hw_array(image_hw)
    t = lib().vlm_num_merged(ctypes.byref(cfg), arr, n)
    if t < 0:
        raise VlmError(int(t), "vlm_num_merged")
    return int(t)


def new_status(device=None) -> torch.Tensor:
    return _zeros(1, dtype=torch.int32, device=device or "cuda")


def status_sync(status: torch.Tensor, stream=None) -> int:
    return int(lib().vlm_status_sync(_dev(status, "status"), _stream(stream)))


# ---------------------------------------------------------------------------
# Weight packing
# ---------------------------------------------------------------------------

def pack_tower(cfg: Config, w: dict, stream=None) -> torch.Tensor:
    """w: device tensors named as in vlm_tower_weights (bf16 matrices, fp32 gains)."""
    L = lib()
    tw = TowerWeights(**{k: _dev(w[k], k) for k, _ in TowerWeights._fields_})
    nbytes = L.vlm_tower_packed_bytes(ctypes.byref(cfg))
    if nbytes == 0:
        raise VlmError(ERR_INVALID_ARG, "vlm_tower_packed_bytes")
    packed = _empty(nbytes, dtype=torch.uint8, device=w["wq"].device)
    _check(L.vlm_pack_tower(ctypes.byref(cfg), ctypes.byref(tw), packed.data_ptr(), nbytes, _stream(stream)),
           "vlm_pack_tower")
    return packed


def pack_projector(cfg: Config, w: dict, stream=None) -> torch.Tensor:
    L = lib()
    pw = ProjectorWeights(g_proj=_dev(w["g_proj"], "g_proj"), w_merge=_dev(w.get("w_merge"), "w_merge"),
                          w1=_dev(w["w1"], "w1"), w2=_dev(w["w2"], "w2"))
    nbytes = L.vlm_projector_packed_bytes(ctypes.byref(cfg))
    if nbytes == 0:
        raise VlmError(ERR_INVALID_ARG, "vlm_projector_packed_bytes")
    packed = _empty(nbytes, dtype=torch.uint8, device=w["w1"].device)
    _check(L.vlm_pack_projector(ctypes.byref(cfg), ctypes.byref(pw), packed.data_ptr(), nbytes, _stream(stream)),
           "vlm_pack_projector")
    return packed


# ---------------------------------------------------------------------------
# The three calls of the path
# ---------------------------------------------------------------------------

def encode_workspace_size(cfg: Config, image_hw) -> int:
    arr, n = _hw_array(image_hw)
    return int(lib().vlm_encode_workspace_size(ctypes.byref(cfg), arr, n))


def encode(cfg: Config, pixels: torch.Tensor, image_hw, packed_tower: torch.Tensor, out=None, workspace=None,
           status=None, stream=None) -> torch.Tensor:
    """Vision tower: pixels (device fp32, CHW blocks concatenated) -> bf16 [T, width]."""
    L = lib()
    arr, n = _hw_array(image_hw)
    T = num_patches(cfg, image_hw)
    dev = pixels.device
    if out is None:
        out = _empty((T, cfg.width), dtype=torch.bfloat16, device=dev)
    ws_need = L.vlm_encode_workspace_size(ctypes.byref(cfg), arr, n)
    if workspace is None:
        workspace = _empty(ws_need, dtype=torch.uint8, device=dev)
    if status is None:
        status = new_status(dev)
    _check(L.vlm_encode(ctypes.byref(cfg), _dev(pixels, "pixels"), arr, n, _dev(packed_tower, "packed_tower"),
                        _dev(out, "out"), _dev(workspace, "workspace"), workspace.numel(), _dev(status, "status"),
                        _stream(stream)), "vlm_encode")
    return out


def merge_project_workspace_size(cfg: Config, image_hw) -> int:
    arr, n = _hw_array(image_hw)
    return int(lib().vlm_merge_project_workspace_size(ctypes.byref(cfg), arr, n))


def merge_project(cfg: Config, tower_out: torch.Tensor, image_hw, packed_projector: torch.Tensor, out=None,
                  workspace=None, status=None, stream=None) -> torch.Tensor:
    """Projector: bf16 [T, width] -> bf16 [T_m, proj_out]."""
    L = lib()
    arr, n = _hw_array(image_hw)
    Tm = num_merged(cfg, image_hw)
    dev = tower_out.device
    if out is None:
        out = _empty((Tm, cfg.proj_out), dtype=torch.bfloat16, device=dev)
    if workspace is None:
        workspace = _empty(L.vlm_merge_project_workspace_size(ctypes.byref(cfg), arr, n), dtype=torch.uint8,
                                device=dev)
    if status is None:
        status = new_status(dev)
    _check(L.vlm_merge_project(ctypes.byref(cfg), _dev(tower_out, "tower_out"), arr, n,
                               _dev(packed_projector, "packed_projector"), _dev(out, "out"),
                               _dev(workspace, "workspace"), workspace.numel(), _dev(status, "status"),
                               _stream(stream)), "vlm_merge_project")
    return out


def merge_project_scatter_workspace_size(cfg: Config, image_hw, n_tokens: int) -> int:
    arr, n = _hw_array(image_hw)
    return int(lib().vlm_merge_project_scatter_workspace_size(ctypes.byref(cfg), arr, n, int(n_tokens)))


def merge_project_scatter(cfg: Config, tower_out: torch.Tensor, image_hw, packed_projector: torch.Tensor,
                          input_ids: torch.Tensor, text_embeds: torch.Tensor, workspace=None, status=None,
                          stream=None) -> torch.Tensor:
    """Projector with the masked scatter fused into its last linear: rows of
    text_embeds (bf16 [n_tokens, proj_out]) at cfg.image_token_id positions <-
    the projected merged tokens, in order; no [T_m, proj_out] buffer."""
    L = lib()
    if input_ids.dtype != torch.int64:
        raise ValueError("input_ids must be int64")
    n = input_ids.numel()
    if text_embeds.dtype != torch.bfloat16 or text_embeds.dim() != 2 or tuple(text_embeds.shape) != (n, cfg.proj_out):
        raise ValueError("text_embeds must be bf16 [n_tokens, proj_out]")
    arr, n_img = _hw_array(image_hw)
    dev = text_embeds.device
    if workspace is None:
        workspace = _empty(max(256, L.vlm_merge_project_scatter_workspace_size(ctypes.byref(cfg), arr, n_img, n)),
                           dtype=torch.uint8, device=dev)
    if status is None:
        status = new_status(dev)
    _check(L.vlm_merge_project_scatter(ctypes.byref(cfg), _dev(tower_out, "tower_out"), arr, n_img,
                                       _dev(packed_projector, "packed_projector"), _dev(input_ids, "input_ids"), n,
                                       _dev(text_embeds, "text_embeds"), _dev(workspace, "workspace"),
                                       workspace.numel(), _dev(status, "status"), _stream(stream)),
           "vlm_merge_project_scatter")
    return text_embeds


def scatter_workspace_size(n_tokens: int) -> int:
    return int(lib().vlm_scatter_workspace_size(int(n_tokens)))


def scatter(input_ids: torch.Tensor, image_embeds: torch.Tensor, text_embeds: torch.Tensor, image_token_id: int = 10,
            workspace=None, status=None, stream=None) -> torch.Tensor:
    """In place: rows of text_embeds at image_token_id positions <- image_embeds rows, in order."""
    L = lib()
    if input_ids.dtype != torch.int64:
        raise ValueError("input_ids must be int64")
    n = input_ids.numel()
    if text_embeds.shape[0] != n:
        raise ValueError("text_embeds must have one row per id")
    row_bytes = text_embeds[0].numel() * text_embeds.element_size()
    if image_embeds.numel() and image_embeds[0].numel() * image_embeds.element_size() != row_bytes:
        raise ValueError("image and text rows differ in size")
    dev = text_embeds.device
    if workspace is None:
        workspace = _empty(max(256, L.vlm_scatter_workspace_size(n)), dtype=torch.uint8, device=dev)
    if status is None:
        status = new_status(dev)
    _check(L.vlm_scatter(_dev(input_ids, "input_ids"), n, int(image_token_id), _dev(image_embeds, "image_embeds"),
                         image_embeds.shape[0], _dev(text_embeds, "text_embeds"), row_bytes,
                         _dev(workspace, "workspace"), workspace.numel(), _dev(status, "status"), _stream(stream)),
           "vlm_scatter")
    return text_embeds


# ---------------------------------------------------------------------------
# Per-kernel entry points
# ---------------------------------------------------------------------------

# ---------------------------------------------------------------------------
# FP8 (E4M3) tower GEMMs
# ---------------------------------------------------------------------------

def _act_array(cfg: Config, act_scales):
    flat = [float(v) for row in act_scales for v in row]
    if len(flat) != 4 * cfg.layers:
        raise ValueError(f"act_scales needs {cfg.layers} rows of 4 scales")
    return (ctypes.c_float * max(1, len(flat)))(*flat)


def pack_tower_fp8(cfg: Config, w: dict, act_scales, stream=None) -> torch.Tensor:
    """E4M3 tower (per-row weight scales, static activation scales act_scales[l][0..3])."""
    L = lib()
    tw = TowerWeights(**{k: _dev(w[k], k) for k, _ in TowerWeights._fields_})
    nbytes = L.vlm_tower_fp8_packed_bytes(ctypes.byref(cfg))
    if nbytes == 0:
        raise VlmError(ERR_INVALID_ARG, "vlm_tower_fp8_packed_bytes")
    packed = _empty(nbytes, dtype=torch.uint8, device=w["wq"].device)
    _check(L.vlm_pack_tower_fp8(ctypes.byref(cfg), ctypes.byref(tw), _act_array(cfg, act_scales), packed.data_ptr(),
                                nbytes, _stream(stream)), "vlm_pack_tower_fp8")
    return packed


def encode_fp8(cfg: Config, pixels: torch.Tensor, image_hw, packed_tower_fp8: torch.Tensor, act_scales, out=None,
               workspace=None, status=None, stream=None) -> torch.Tensor:
    """vlm_encode with the E4M3 tower GEMMs."""
    L = lib()
    arr, n = _hw_array(image_hw)
    T = num_patches(cfg, image_hw)
    dev = pixels.device
    if out is None:
        out = _empty((T, cfg.width), dtype=torch.bfloat16, device=dev)
    if workspace is None:
        workspace = _empty(L.vlm_encode_workspace_size(ctypes.byref(cfg), arr, n), dtype=torch.uint8, device=dev)
    if status is None:
        status = new_status(dev)
    _check(L.vlm_encode_fp8(ctypes.byref(cfg), _dev(pixels, "pixels"), arr, n, _dev(packed_tower_fp8, "packed"),
                            _act_array(cfg, act_scales), _dev(out, "out"), _dev(workspace, "workspace"),
                            workspace.numel(), _dev(status, "status"), _stream(stream)), "vlm_encode_fp8")
    return out


def pack_tower_nvfp4(cfg: Config, w: dict, act_scales, stream=None) -> torch.Tensor:
    """NVFP4 tower (block-scaled E2M1 weights, static activation global scales act_scales[l][0..3])."""
    L = lib()
    tw = TowerWeights(**{k: _dev(w[k], k) for k, _ in TowerWeights._fields_})
    nbytes = L.vlm_tower_nvfp4_packed_bytes(ctypes.byref(cfg))
    if nbytes == 0:
        raise VlmError(ERR_INVALID_ARG, "vlm_tower_nvfp4_packed_bytes")
    packed = _empty(nbytes, dtype=torch.uint8, device=w["wq"].device)
    _check(L.vlm_pack_tower_nvfp4(ctypes.byref(cfg), ctypes.byref(tw), _act_array(cfg, act_scales),
                                  packed.data_ptr(), nbytes, _stream(stream)), "vlm_pack_tower_nvfp4")
    return packed


def patch_embed(cfg: Config, pixels: torch.Tensor, image_hw, packed_tower: torch.Tensor, status=None,
                stream=None) -> torch.Tensor:
    """The patch features fp32 [T, width] (gather + patch-embed GEMM, before ln_pre)."""
    L = lib()
    arr, n = _hw_array(image_hw)
    T = num_patches(cfg, image_hw)
    dev = pixels.device
    x = _empty((T, cfg.width), dtype=torch.float32, device=dev)
    ws = _empty(L.vlm_encode_workspace_size(ctypes.byref(cfg), arr, n), dtype=torch.uint8, device=dev)
    if status is None:
        status = new_status(dev)
    _check(L.vlm_patch_embed(ctypes.byref(cfg), _dev(pixels, "pixels"), arr, n, _dev(packed_tower, "packed"),
                             _dev(x, "x"), _dev(ws, "workspace"), ws.numel(), _dev(status, "status"), _stream(stream)),
           "vlm_patch_embed")
    return x


def encode_nvfp4_workspace_size(cfg: Config, image_hw) -> int:
    arr, n = _hw_array(image_hw)
    return lib().vlm_encode_nvfp4_workspace_size(ctypes.byref(cfg), arr, n)


def encode_nvfp4(cfg: Config, pixels: torch.Tensor, image_hw, packed_tower_nvfp4: torch.Tensor, act_scales,
                 out=None, workspace=None, status=None, stream=None) -> torch.Tensor:
    """vlm_encode with the NVFP4 tower GEMMs."""
    L = lib()
    arr, n = _hw_array(image_hw)
    T = num_patches(cfg, image_hw)
    dev = pixels.device
    if out is None:
        out = _empty((T, cfg.width), dtype=torch.bfloat16, device=dev)
    if workspace is None:
        workspace = _empty(encode_nvfp4_workspace_size(cfg, image_hw), dtype=torch.uint8, device=dev)
    if status is None:
        status = new_status(dev)
    _check(L.vlm_encode_nvfp4(ctypes.byref(cfg), _dev(pixels, "pixels"), arr, n, _dev(packed_tower_nvfp4, "packed"),
                              _act_array(cfg, act_scales), _dev(out, "out"), _dev(workspace, "workspace"),
                              workspace.numel(), _dev(status, "status"), _stream(stream)), "vlm_encode_nvfp4")
    return out


def gemm_fp8(epilogue: int, a: torch.Tensor, b: torch.Tensor, colscale: torch.Tensor, out: torch.Tensor,
             out_scale: float = 1.0, out_bf16=None, pos=None, rope=None, rope_cols: int = 0, status=None,
             stream=None) -> torch.Tensor:
    """E4M3 GEMM: a [M, K], b [N, K] as uint8 or float8_e4m3fn tensors."""
    M, K = a.shape
    N = b.shape[0]
    if status is None:
        status = new_status(a.device)
    _check(lib().vlm_gemm_fp8(epilogue, _dev(a, "a"), _dev(b, "b"), _dev(colscale, "colscale"), float(out_scale),
                              M, N, K, _dev(out, "out"), _dev(out_bf16, "out_bf16"), _dev(pos, "pos"),
                              _dev(rope, "rope"), rope_cols, _dev(status, "status"), _stream(stream)), "vlm_gemm_fp8")
    return out


def rmsnorm_fp8(x: torch.Tensor, g1: torch.Tensor, f8_scale: float, g0=None, eps: float = 1e-5, out=None,
                stream=None) -> torch.Tensor:
    rows, width = x.shape
    if out is None:
        out = _empty((rows, width), dtype=torch.uint8, device=x.device)
    _check(lib().vlm_rmsnorm_fp8(_dev(x, "x"), _dev(g0, "g0"), _dev(g1, "g1"), _dev(out, "out"), rows, width,
                                 float(eps), float(f8_scale), _stream(stream)), "vlm_rmsnorm_fp8")
    return out


# ---------------------------------------------------------------------------
# NVFP4 operands (E2M1 codes, E4M3 block scales, fp32 global scale)
# ---------------------------------------------------------------------------
DTYPE_BF16, DTYPE_F32 = 0, 1
NVFP4_GLOBAL_DIVISOR = 6.0 * 448.0


def nvfp4_sf_bytes(rows: int, k: int) -> int:
    """Bytes of block scales for `rows` rows of K values (host only)."""
    return int(lib().vlm_nvfp4_sf_bytes(rows, k))


def _dtype_code(x: torch.Tensor) -> int:
    if x.dtype == torch.bfloat16:
        return DTYPE_BF16
    if x.dtype == torch.float32:
        return DTYPE_F32
    raise TypeError(f"bf16 or fp32 expected, got {x.dtype}")


def amax_scale(x: torch.Tensor, divisor: float = NVFP4_GLOBAL_DIVISOR, out=None, stream=None) -> torch.Tensor:
    """Device fp32 [1] = max |x| / divisor (an NVFP4 global scale by default)."""
    if out is None:
        out = _empty(1, dtype=torch.float32, device=x.device)
    _check(lib().vlm_amax_scale(_dev(x, "x"), _dtype_code(x), x.numel(), float(divisor), _dev(out, "out"),
                                _stream(stream)), "vlm_amax_scale")
    return out


def quant_nvfp4(x: torch.Tensor, s_global: torch.Tensor, q=None, sf=None, stream=None) -> tuple:
    """x [rows, K] (bf16 or fp32) -> (codes uint8 [rows, K/2], block scales uint8
    [nvfp4_sf_bytes(rows, K)]) with the device global scale s_global [1]."""
    rows, k = x.shape
    if q is None:
        q = _empty((rows, k // 2), dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = _empty(max(nvfp4_sf_bytes(rows, k), 1), dtype=torch.uint8, device=x.device)
    _check(lib().vlm_quant_nvfp4(_dev(x, "x"), _dtype_code(x), rows, k, _dev(s_global, "s_global"), _dev(q, "q"),
                                 _dev(sf, "sf"), _stream(stream)), "vlm_quant_nvfp4")
    return q, sf


def gemm_nvfp4(epilogue: int, a: tuple, b: tuple, out: torch.Tensor, status=None, stream=None) -> torch.Tensor:
    """out (bf16, or fp32 += for EPI_RESID) = fp32(g_a g_b) * A . B^T, where a and
    b are (codes [rows, K/2], block scales, global scale [1]) triples."""
    (qa, sfa, ga), (qb, sfb, gb) = a, b
    M, N, K = qa.shape[0], qb.shape[0], 2 * qa.shape[1]
    if status is None:
        status = new_status(qa.device)
    _check(lib().vlm_gemm_nvfp4(epilogue, _dev(qa, "a"), _dev(sfa, "a_sf"), _dev(ga, "g_a"), _dev(qb, "b"),
                                _dev(sfb, "b_sf"), _dev(gb, "g_b"), M, N, K, _dev(out, "out"), _dev(status, "status"),
                                _stream(stream)), "vlm_gemm_nvfp4")
    return out


def gemm_nvfp4_rope(a: tuple, b: tuple, out: torch.Tensor, pos: torch.Tensor, rope_table: torch.Tensor,
                    rope_cols: int, status=None, stream=None) -> torch.Tensor:
    """gemm_nvfp4 with the ROPE epilogue: out bf16 [M, N], columns below
    rope_cols rotated (pos: int32 [M] = row << 16 | col; rope_table from rope_table())."""
    (qa, sfa, ga), (qb, sfb, gb) = a, b
    M, N, K = qa.shape[0], qb.shape[0], 2 * qa.shape[1]
    if status is None:
        status = new_status(qa.device)
    _check(lib().vlm_gemm_nvfp4_ex(EPI_ROPE, _dev(qa, "a"), _dev(sfa, "a_sf"), _dev(ga, "g_a"), _dev(qb, "b"),
                                   _dev(sfb, "b_sf"), _dev(gb, "g_b"), M, N, K, _dev(out, "out"), None, 1.0,
                                   _dev(pos, "pos"), _dev(rope_table, "rope"), int(rope_cols), _dev(status, "status"),
                                   _stream(stream)), "vlm_gemm_nvfp4_ex")
    return out


def gemm_nvfp4_swiglu(a: tuple, b: tuple, out_sg: float, q=None, sf=None, status=None, stream=None) -> tuple:
    """gemm_nvfp4 with the SWIGLU epilogue (B rows gate / up interleaved by 16):
    returns the NVFP4 codes [M, N/4] and block scales of silu(gate) * up with
    global scale out_sg (the scales of padding rows are zero when sf is None)."""
    (qa, sfa, ga), (qb, sfb, gb) = a, b
    M, N, K = qa.shape[0], qb.shape[0], 2 * qa.shape[1]
    if q is None:
        q = _empty((M, N // 4), dtype=torch.uint8, device=qa.device)
    if sf is None:
        sf = _zeros(nvfp4_sf_bytes(M, N // 2), dtype=torch.uint8, device=qa.device)
    if status is None:
        status = new_status(qa.device)
    _check(lib().vlm_gemm_nvfp4_ex(EPI_SWIGLU, _dev(qa, "a"), _dev(sfa, "a_sf"), _dev(ga, "g_a"), _dev(qb, "b"),
                                   _dev(sfb, "b_sf"), _dev(gb, "g_b"), M, N, K, _dev(q, "out"), _dev(sf, "out_sf"),
                                   float(out_sg), None, None, 0, _dev(status, "status"), _stream(stream)),
           "vlm_gemm_nvfp4_ex")
    return q, sf


def rmsnorm_nvfp4(x: torch.Tensor, g1: torch.Tensor, s_global: float, g0=None, eps: float = 1e-5, stream=None) -> tuple:
    """rmsnorm whose output is NVFP4 with global scale s_global: (codes, block scales)."""
    rows, width = x.shape
    q = _empty((rows, width // 2), dtype=torch.uint8, device=x.device)
    sf = _zeros(nvfp4_sf_bytes(rows, width), dtype=torch.uint8, device=x.device)
    _check(lib().vlm_rmsnorm_nvfp4(_dev(x, "x"), _dev(g0, "g0"), _dev(g1, "g1"), _dev(q, "q"), _dev(sf, "sf"), rows,
                                   width, float(eps), float(s_global), _stream(stream)), "vlm_rmsnorm_nvfp4")
    return q, sf


# ---------------------------------------------------------------------------
# Image front end and placeholder expansion
# ---------------------------------------------------------------------------

def resize_target(height: int, width: int, longest_edge: int = 1540, grid: int = 28) -> tuple:
    """The processor's resize size (host only): see vlm_resize_target."""
    oh, ow = ctypes.c_int32(), ctypes.c_int32()
    _check(lib().vlm_resize_target(int(height), int(width), int(longest_edge), int(grid), ctypes.byref(oh),
                                   ctypes.byref(ow)), "vlm_resize_target")
    return oh.value, ow.value


def preprocess(images_u8: torch.Tensor, src_hw, out_hw, tile: int = 0, out=None, stream=None) -> torch.Tensor:
    """Bilinear resize of decoded u8 RGB HWC images (concatenated, flat) onto out_hw.

    Returns fp32 [3*sum(oh*ow)] CHW blocks in [0, 1]; with tile > 0 each image
    is written as its row-major tiles of [3, tile, tile].
    """
    if images_u8.dtype != torch.uint8:
        raise ValueError("images_u8 must be uint8")
    src_arr, n = _hw_array(src_hw)
    out_arr, n_out = _hw_array(out_hw)
    if n != n_out:
        raise ValueError("src_hw and out_hw must list the same images")
    need_src = sum(3 * int(h) * int(w) for h, w in src_hw)
    if images_u8.numel() != need_src:
        raise ValueError(f"images_u8 holds {images_u8.numel()} bytes, the sizes need {need_src}")
    total = sum(3 * int(h) * int(w) for h, w in out_hw)
    if out is None:
        out = _empty(total, dtype=torch.float32, device=images_u8.device)
    elif out.numel() < total or out.dtype != torch.float32:
        raise ValueError("out must be fp32 with room for every output pixel")
    _check(lib().vlm_preprocess(_dev(images_u8, "images_u8"), src_arr, n, out_arr, int(tile), _dev(out, "out"),
                                _stream(stream)), "vlm_preprocess")
    return out


def tiled_hw(out_hw, tile: int) -> list:
    """Image table that vlm_encode takes for the output of preprocess(..., tile)."""
    return [(tile, tile)] * sum((int(h) // tile) * (int(w) // tile) for h, w in out_hw)


def expand_placeholders_workspace_size(n_ids: int, n_images: int) -> int:
    return int(lib().vlm_expand_placeholders_workspace_size(int(n_ids), int(n_images)))


def expand_placeholders(input_ids: torch.Tensor, marker_id: int, counts, image_token_id: int = 10, out=None,
                        workspace=None, status=None, stream=None) -> torch.Tensor:
    """Each marker_id (in order) becomes counts[k] copies of image_token_id; returns int64 ids."""
    L = lib()
    n_ids = input_ids.numel()
    n_img = len(counts)
    carr = (ctypes.c_int64 * max(1, n_img))(*[int(c) for c in counts])
    total = n_ids - n_img + sum(int(c) for c in counts)
    if out is None:
        out = _empty(max(total, 0), dtype=torch.int64, device=input_ids.device)
    ws_need = L.vlm_expand_placeholders_workspace_size(n_ids, n_img)
    if workspace is None:
        workspace = _empty(max(ws_need, 256), dtype=torch.uint8, device=input_ids.device)
    if status is None:
        status = new_status(input_ids.device)
    out_len = ctypes.c_int64()
    _check(L.vlm_expand_placeholders(_dev(input_ids, "input_ids"), n_ids, int(marker_id), carr, n_img,
                                     int(image_token_id), _dev(out, "out"), out.numel(), ctypes.byref(out_len),
                                     _dev(workspace, "workspace"), workspace.numel(), _dev(status, "status"),
                                     _stream(stream)), "vlm_expand_placeholders")
    return out[:out_len.value]


def gemm(epilogue: int, a: torch.Tensor, b: torch.Tensor, out: torch.Tensor, out_bf16=None, pos=None,
         rope_table=None, rope_cols: int = 0, status=None, stream=None) -> torch.Tensor:
    M, K = a.shape
    N = b.shape[0]
    if status is None:
        status = new_status(a.device)
    _check(lib().vlm_gemm(epilogue, _dev(a, "a"), _dev(b, "b"), M, N, K, _dev(out, "out"), _dev(out_bf16, "out_bf16"),
                          _dev(pos, "pos"), _dev(rope_table, "rope_table"), rope_cols, _dev(status, "status"),
                          _stream(stream)), "vlm_gemm")
    return out


def rope_table(theta: float, head_dim: int, max_pos: int, device="cuda", stream=None) -> torch.Tensor:
    tab = _empty((max_pos, head_dim // 2, 2), dtype=torch.float32, device=device)
    _check(lib().vlm_rope_table(float(theta), head_dim, max_pos, tab.data_ptr(), _stream(stream)), "vlm_rope_table")
    return tab


def attention(qkv: torch.Tensor, cu_seqlens, heads: int, out=None, status=None, stream=None) -> torch.Tensor:
    L = lib()
    T = qkv.shape[0]
    cu = (ctypes.c_int32 * len(cu_seqlens))(*[int(c) for c in cu_seqlens])
    nb = len(cu_seqlens) - 1
    if out is None:
        out = _empty((T, heads * 64), dtype=torch.bfloat16, device=qkv.device)
    ws = _empty(max(256, L.vlm_attention_workspace_size(nb)), dtype=torch.uint8, device=qkv.device)
    if status is None:
        status = new_status(qkv.device)
    _check(L.vlm_attention(_dev(qkv, "qkv"), T, heads, 64, cu, nb, _dev(out, "out"), ws.data_ptr(), ws.numel(),
                           _dev(status, "status"), _stream(stream)), "vlm_attention")
    return out


def attention_nvfp4(qkv: torch.Tensor, cu_seqlens, heads: int, s_global: float, status=None, stream=None) -> tuple:
    """attention whose output is NVFP4 with global scale s_global: (codes, block scales)."""
    L = lib()
    T = qkv.shape[0]
    cu = (ctypes.c_int32 * len(cu_seqlens))(*[int(c) for c in cu_seqlens])
    nb = len(cu_seqlens) - 1
    q = _empty((T, heads * 32), dtype=torch.uint8, device=qkv.device)
    sf = _zeros(nvfp4_sf_bytes(T, heads * 64), dtype=torch.uint8, device=qkv.device)
    ws = _empty(max(256, L.vlm_attention_workspace_size(nb)), dtype=torch.uint8, device=qkv.device)
    if status is None:
        status = new_status(qkv.device)
    _check(L.vlm_attention_nvfp4(_dev(qkv, "qkv"), T, heads, 64, cu, nb, _dev(q, "q"), _dev(sf, "sf"), float(s_global),
                                 ws.data_ptr(), ws.numel(), _dev(status, "status"), _stream(stream)),
           "vlm_attention_nvfp4")
    return q, sf


def rmsnorm(x: torch.Tensor, g1: torch.Tensor, g0=None, eps: float = 1e-5, out=None, stream=None) -> torch.Tensor:
    rows, width = x.shape
    if out is None:
        out = _empty((rows, width), dtype=torch.bfloat16, device=x.device)
    _check(lib().vlm_rmsnorm(_dev(x, "x"), _dev(g0, "g0"), _dev(g1, "g1"), _dev(out, "out"), rows, width, float(eps),
                             _stream(stream)), "vlm_rmsnorm")
    return out


def selftest_wait_timeout(budget_cycles: int, status: torch.Tensor, stream=None) -> None:
    _check(lib().vlm_selftest_wait_timeout(int(budget_cycles), _dev(status, "status"), _stream(stream)),
           "vlm_selftest_wait_timeout")


def debug_build() -> bool:
    """True when the loaded library is the index-checked debug build."""
    return bool(lib().vlm_debug_build())


def debug_checks() -> int:
    """Synchronises the device; the first failing index check's code
    (file id << 16 | line), or 0, and clears the record (debug builds only)."""
    code = ctypes.c_int32(0)
    _check(lib().vlm_debug_checks(ctypes.byref(code)), "vlm_debug_checks")
    return int(code.value)


def debug_selftest_bounds(buf: torch.Tensor, n: int, stream=None) -> None:
    """Debug builds: the deliberate out-of-range writes into buf[n:2n] are
    caught by the index check and skipped."""
    _check(lib().vlm_debug_selftest_bounds(_dev(buf, "buf"), int(n), _stream(stream)), "vlm_debug_selftest_bounds")


# ---------------------------------------------------------------------------
# Instrumentation
# ---------------------------------------------------------------------------

def launch_count() -> int:
    return int(lib().vlm_launch_count())


def profile_enable(on: bool = True) -> None:
    _check(lib().vlm_profile_enable(1 if on else 0), "vlm_profile_enable")


def profile_query(kclass: str) -> tuple:
    n = ctypes.c_int64()
    ms = ctypes.c_double()
    _check(lib().vlm_profile_query(KCLASS[kclass], ctypes.byref(n), ctypes.byref(ms)), "vlm_profile_query")
    return int(n.value), float(ms.value)


# ---------------------------------------------------------------------------
# A reusable pipeline: packed weights + workspaces for repeated calls
# ---------------------------------------------------------------------------

class ImagePipeline:
    """vlm_encode -> vlm_merge_project (-> vlm_scatter) with buffers kept between calls."""

    def __init__(self, cfg: Config, tower: dict, projector: dict, image_hw, device="cuda", fp8_act_scales=None,
                 nvfp4_act_scales=None):
        """fp8_act_scales: [layers][4] static activation scales for the E4M3 tower
        GEMMs (vlm_encode_fp8); nvfp4_act_scales: [layers][4] static activation
        global scales for the NVFP4 tower GEMMs (vlm_encode_nvfp4); neither: the
        bf16 tower."""
        if fp8_act_scales is not None and nvfp4_act_scales is not None:
            raise ValueError("choose one of fp8_act_scales and nvfp4_act_scales")
        self.cfg = cfg
        self.image_hw = [tuple(int(v) for v in hw) for hw in image_hw]
        self.fp8_act_scales = fp8_act_scales
        self.nvfp4_act_scales = nvfp4_act_scales
        if nvfp4_act_scales is not None:
            self.packed_tower = pack_tower_nvfp4(cfg, tower, nvfp4_act_scales)
        elif fp8_act_scales is not None:
            self.packed_tower = pack_tower_fp8(cfg, tower, fp8_act_scales)
        else:
            self.packed_tower = pack_tower(cfg, tower)
        self.packed_proj = pack_projector(cfg, projector)
        self.T = num_patches(cfg, self.image_hw)
        self.Tm = num_merged(cfg, self.image_hw)
        self.tower_out = _empty((self.T, cfg.width), dtype=torch.bfloat16, device=device)
        self.embeds = _empty((self.Tm, cfg.proj_out), dtype=torch.bfloat16, device=device)
        enc_ws = encode_nvfp4_workspace_size(cfg, self.image_hw) if nvfp4_act_scales is not None else \
            encode_workspace_size(cfg, self.image_hw)
        ws = max(enc_ws, merge_project_workspace_size(cfg, self.image_hw))
        self.workspace = _empty(ws, dtype=torch.uint8, device=device)
        self.status = new_status(device)
        self._fused_ws = None  # vlm_merge_project_scatter's workspace, sized on first use

    def encode(self, pixels: torch.Tensor, stream=None) -> torch.Tensor:
        """The tower alone: pixels -> self.tower_out."""
        if self.nvfp4_act_scales is not None:
            encode_nvfp4(self.cfg, pixels, self.image_hw, self.packed_tower, self.nvfp4_act_scales,
                         out=self.tower_out, workspace=self.workspace, status=self.status, stream=stream)
        elif self.fp8_act_scales is None:
            encode(self.cfg, pixels, self.image_hw, self.packed_tower, out=self.tower_out, workspace=self.workspace,
                   status=self.status, stream=stream)
        else:
            encode_fp8(self.cfg, pixels, self.image_hw, self.packed_tower, self.fp8_act_scales, out=self.tower_out,
                       workspace=self.workspace, status=self.status, stream=stream)
        return self.tower_out

    def __call__(self, pixels: torch.Tensor, stream=None) -> torch.Tensor:
        self.encode(pixels, stream)
        merge_project(self.cfg, self.tower_out, self.image_hw, self.packed_proj, out=self.embeds,
                      workspace=self.workspace, status=self.status, stream=stream)
        return self.embeds

    def embed_into(self, pixels: torch.Tensor, input_ids: torch.Tensor, text_embeds: torch.Tensor,
                   stream=None) -> torch.Tensor:
        """The whole image path written into the token embeddings in place:
        vlm_encode, then vlm_merge_project_scatter (the masked scatter fused
        into the projector's last linear; self.embeds is not written). Rows of
        text_embeds at cfg.image_token_id positions receive this batch's
        projected merged tokens in order; the others are left untouched."""
        self.encode(pixels, stream)
        need = merge_project_scatter_workspace_size(self.cfg, self.image_hw, input_ids.numel())
        if self._fused_ws is None or self._fused_ws.numel() < need:
            self._fused_ws = _empty(max(256, need), dtype=torch.uint8, device=self.tower_out.device)
        return merge_project_scatter(self.cfg, self.tower_out, self.image_hw, self.packed_proj, input_ids, text_embeds,
                                     workspace=self._fused_ws, status=self.status, stream=stream)


class GraphStep:
    """Captures every kernel a callable launches on the current stream into one
    CUDA graph and replays it: one host call per step instead of one per
    kernel. The callable's buffers must stay at the same addresses (an
    ImagePipeline's do); the kernels keep their programmatic-launch edges.
    """

    def __init__(self, fn, warmup: int = 1):
        self.fn = fn
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(warmup):
                fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        before = launch_count()
        with torch.cuda.graph(self.graph):
            fn()
        self.launches_per_replay = launch_count() - before

    def __call__(self) -> None:
        self.graph.replay()


class EncoderSideStream:
    """Runs the image path (vlm_encode + vlm_merge_project) on its own CUDA
    stream so it overlaps other work on the caller's stream; the caller's
    stream waits on an event before the scatter reads the embeddings.

    submit() orders the side stream after the caller's stream (the pixels were
    written there) and after the previous scatter (which read the previous
    embeddings from the same buffers), then enqueues the image path and
    records `ready`. scatter() makes the caller's stream wait on `ready`,
    scatters, and records `consumed`.
    """

    def __init__(self, pipeline: ImagePipeline, priority: int = 0):
        self.pipe = pipeline
        self.stream = torch.cuda.Stream(device=pipeline.embeds.device, priority=priority)
        self.ready = torch.cuda.Event()
        self.consumed = torch.cuda.Event()
        self.consumed.record(torch.cuda.current_stream())

    def submit(self, pixels: torch.Tensor) -> torch.cuda.Event:
        self.stream.wait_stream(torch.cuda.current_stream())
        self.stream.wait_event(self.consumed)
        with torch.cuda.stream(self.stream):
            self.pipe(pixels, stream=self.stream)
            self.ready.record(self.stream)
        pixels.record_stream(self.stream)
        return self.ready

    def scatter(self, input_ids: torch.Tensor, text_embeds: torch.Tensor, workspace=None, stream=None) -> None:
        main = stream if stream is not None else torch.cuda.current_stream()
        main.wait_event(self.ready)
        scatter(input_ids, self.pipe.embeds, text_embeds, self.pipe.cfg.image_token_id, workspace=workspace,
                status=self.pipe.status, stream=main)
        self.consumed.record(main)


class HostFedSteps:
    """Steps whose inputs come from pinned host memory and whose result goes
    back to it, with the copies overlapped with the compute: while step i runs
    on the current stream, a copy stream brings in step i+1's inputs and then
    takes out step i's result, ordered by events. Every device input and the
    result buffer are double-buffered, so a copy never touches a buffer a
    running step uses.

    step_fn(inputs, result) enqueues one step on the current stream, reading
    the device tensors `inputs` and writing the device tensor `result`.
    """

    def __init__(self, step_fn, input_templates, result_template: torch.Tensor):
        self.step_fn = step_fn
        dev = result_template.device
        self.inputs = [[torch.empty_like(t) for t in input_templates] for _ in range(2)]
        self.results = [result_template.clone(), result_template.clone()]
        self.copy = torch.cuda.Stream(device=dev)
        self.ev_in = [torch.cuda.Event(), torch.cuda.Event()]
        self.ev_done = [torch.cuda.Event(), torch.cuda.Event()]
        self.ev_out = [torch.cuda.Event(), torch.cuda.Event()]

    def run(self, host_inputs, host_result: torch.Tensor, steps: int) -> None:
        """`steps` steps, each on a fresh copy of host_inputs (pinned host
        tensors matching the input templates); each step's result is copied
        into host_result. Returns when everything is enqueued; the last copy is
        ordered before any later work on the current stream."""
        main = torch.cuda.current_stream()
        self.copy.wait_stream(main)
        with torch.cuda.stream(self.copy):
            for d, h in zip(self.inputs[0], host_inputs):
                d.copy_(h, non_blocking=True)
            self.ev_in[0].record(self.copy)
        for i in range(steps):
            b, nb = i % 2, 1 - i % 2
            main.wait_event(self.ev_in[b])
            if i >= 2:
                main.wait_event(self.ev_out[b])  # step i-2's result has left this buffer
            self.step_fn(self.inputs[b], self.results[b])
            self.ev_done[b].record(main)
            with torch.cuda.stream(self.copy):
                if i + 1 < steps:
                    if i >= 1:
                        self.copy.wait_event(self.ev_done[nb])  # step i-1 is done with these inputs
                    for d, h in zip(self.inputs[nb], host_inputs):
                        d.copy_(h, non_blocking=True)
                    self.ev_in[nb].record(self.copy)
                self.copy.wait_event(self.ev_done[b])
                host_result.copy_(self.results[b], non_blocking=True)
                self.ev_out[b].record(self.copy)
        main.wait_stream(self.copy)
