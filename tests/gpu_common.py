"""Helpers of the GPU parity tests: tolerances and conversions.

Tolerances
* attention (bf16 output, fp32 accumulation) against the fp64 oracle:
  max |err| <= 2e-2 and ||err||_2 / ||ref||_2 <= 5e-3 per checked tensor;
* RoPE output (fp32 rotation, one bf16 rounding): per element
  |err| <= 2^-8 |ref| + 2^-16 * |pair| (half a bf16 ulp is at most 2^-8 of
  the value; the fp32 products add well under 2^-16 of the pair norm);
* Euler (fp32 FMA): ||err||/||ref|| <= 1e-5 and per element
  |err| <= 1e-5 (|x| + |dsigma v|).
"""
import os

import numpy as np
import torch

ATTN_MAX_ABS = 2e-2
ATTN_REL_L2 = 5e-3

# worst attention errors seen per test (node id -> [max-abs, rel-L2]); the
# conftest prints them after the run, so that the margins to the bounds at
# every size are on record
MARGINS: dict = {}


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def assert_attn_close(gpu, ref, what=""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite output"
    mx = float(np.max(np.abs(gpu - ref)))
    rl = rel_l2(gpu, ref)
    node = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    worst = MARGINS.setdefault(node, [0.0, 0.0])
    worst[0], worst[1] = max(worst[0], mx), max(worst[1], rl)
    assert mx <= ATTN_MAX_ABS and rl <= ATTN_REL_L2, f"{what}: max-abs {mx:.3g}, rel-L2 {rl:.3g}"
    return mx, rl


def assert_lse_close(gpu, ref, what=""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    # lse is a log of a sum of positives: an absolute bound of 2e-2 covers the
    # bf16 rounding of q and k (about 2^-8 relative on each logit of size ~1)
    mx = float(np.max(np.abs(gpu - ref)))
    assert mx <= 2e-2, f"{what}: lse max-abs {mx:.3g}"


def assert_rope_close(gpu, ref, what=""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    pair = np.sqrt(ref[..., 0::2] ** 2 + ref[..., 1::2] ** 2)
    pair = np.repeat(pair, 2, axis=-1)
    tol = 2.0 ** -8 * np.abs(ref) + 2.0 ** -16 * pair
    bad = np.abs(gpu - ref) > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} elements outside the RoPE bound"


def cuda_sync():
    torch.cuda.synchronize()
