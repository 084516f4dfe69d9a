"""Helpers shared by the GPU parity tests: weights to device, comparisons."""
import numpy as np
import torch

# Tolerances of the floating-point parity checks: bf16 results against the
# fp64 oracle, max relative error measured as max|gpu - oracle| / max|oracle|
# over the tensor, and the cosine similarity of every row.
MAX_REL = 2e-2
MIN_COS = 0.999


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def compare(gpu, ref, max_rel=MAX_REL, min_cos=MIN_COS, what=""):
    g = to_np(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite GPU values"
    denom = np.abs(r).max()
    rel = np.abs(g - r).max() / (denom if denom > 0 else 1.0)
    g2 = g.reshape(g.shape[0], -1)
    r2 = r.reshape(r.shape[0], -1)
    num = (g2 * r2).sum(1)
    den = np.linalg.norm(g2, axis=1) * np.linalg.norm(r2, axis=1)
    ok = den > 0
    cos = np.where(ok, num / np.where(ok, den, 1.0), 1.0)
    assert rel <= max_rel, f"{what}: max relative error {rel:.3e} > {max_rel}"
    assert cos.min() >= min_cos, f"{what}: min row cosine {cos.min():.6f} < {min_cos}"
    return rel, float(cos.min())


def tower_to_device(tw: dict, device="cuda") -> dict:
    return {k: v.to(device).contiguous() for k, v in tw.items()}


def to_oracle(w: dict) -> dict:
    return {k: v.double().numpy() for k, v in w.items()}


def pixels_to_device(images) -> torch.Tensor:
    return torch.cat([im.reshape(-1) for im in images]).to("cuda").contiguous()


# ---------------------------------------------------------------------------
# Guard bands: every device buffer the binding allocates during a GPU test (and
# every buffer a test makes with `guarded` / `guarded_copy`) sits between two
# 4 KiB bands of a known byte; after the test the bands must be unchanged, so
# a kernel that writes past either end of a buffer fails the test.
# ---------------------------------------------------------------------------
GUARD_BYTES = 4096
GUARD_FILL = 0xA5


class Guard:
    def __init__(self):
        self.bufs = []

    def __call__(self, shape, dtype, device):
        shape = (shape,) if isinstance(shape, int) else tuple(shape)
        n = 1
        for d in shape:
            n *= int(d)
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        buf = torch.full((2 * GUARD_BYTES + nbytes,), GUARD_FILL, dtype=torch.uint8, device=device)
        self.bufs.append(buf)
        return buf[GUARD_BYTES:GUARD_BYTES + nbytes].view(dtype).view(shape)

    def check(self):
        torch.cuda.synchronize()
        bad = []
        for i, buf in enumerate(self.bufs):
            for name, band in (("before", buf[:GUARD_BYTES]), ("after", buf[buf.numel() - GUARD_BYTES:])):
                if not bool((band == GUARD_FILL).all()):
                    bad.append(f"buffer {i} ({buf.numel() - 2 * GUARD_BYTES} bytes): guard band {name} overwritten")
        self.bufs.clear()
        assert not bad, "; ".join(bad)


_active_guard = None


def guarded(shape, dtype, device="cuda") -> torch.Tensor:
    """An uninitialised device tensor inside guard bands (a plain tensor when no guard is active)."""
    if _active_guard is None:
        return torch.empty(shape, dtype=dtype, device=device)
    return _active_guard(shape, dtype, device)


def guarded_copy(t: torch.Tensor) -> torch.Tensor:
    """A device copy of t inside guard bands."""
    out = guarded(tuple(t.shape), t.dtype)
    out.copy_(t)
    return out


def guarded_zeros(shape, dtype, device="cuda") -> torch.Tensor:
    return guarded(shape, dtype, device).zero_()
