"""Shared test helpers: device transfer of synthetic inputs and the
tolerance checks of the parity tests."""
import re
import os

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# Tolerance (a): |gpu - exact| <= REL * sum_k |x_k * a_k| per element.
REL = 1e-3


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> CUDA bfloat16 tensor (same bits)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    """CUDA tensor -> numpy array of its raw bits (uint16 / uint32)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy().view(np.uint32)
    return t.numpy()


def assert_tol(gpu: np.ndarray, exact: np.ndarray, bound: np.ndarray, rel=REL, what=""):
    gpu = np.asarray(gpu, np.float64)
    err = np.abs(gpu - exact)
    lim = rel * bound
    bad = err > lim
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements outside |gpu-exact| <= {rel}*sum|x*a|; "
                           f"worst err {float(err.max()):.3e} at bound {float(lim.ravel()[np.argmax(err)]):.3e}")


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (as float64)."""
    f = np.abs(np.asarray(x, np.float64)).astype(np.float32)
    return np.spacing(f).astype(np.float64) * 65536.0


def header_functions():
    """Names of the functions declared in include/bi.h."""
    src = open(os.path.join(ROOT, "include", "bi.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bi_[a-z0-9_]+)\s*\(", src)))
