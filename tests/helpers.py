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


# Plan layout of bi_lora_plan (include/bi.h): perm[M], offsets[n_ad + 2],
# padding to a multiple of four words, then one 68-word record per 64-row
# tile of the segments in order: {adapter, rows, first position, 0, ids[64]}
# (ids past `rows` are -1; records past the last tile have adapter -1).
PLAN_TILE = 64
PLAN_REC = 4 + PLAN_TILE


def plan_table_word(M, n_ad):
    return (M + n_ad + 2 + 3) // 4 * 4


def plan_tiles(M, n_ad):
    return (M + PLAN_TILE - 1) // PLAN_TILE + n_ad + 1


def plan_words(M, n_ad):
    return plan_table_word(M, n_ad) + PLAN_REC * plan_tiles(M, n_ad)


def expected_plan_table(perm, offsets, n_ad):
    """Tile records (header rows [T][4], ids per record) that the layout
    above derives from a full perm (no-adapter tokens last) and offsets."""
    M = perm.size
    heads, ids = [], []
    for a in range(n_ad + 1):
        b, e = int(offsets[a]), int(offsets[a + 1])
        for j in range(b, e, PLAN_TILE):
            rows = min(PLAN_TILE, e - j)
            heads.append((a, rows, j, 0))
            ids.append(perm[j:j + rows])
    while len(heads) < plan_tiles(M, n_ad):
        heads.append((-1, 0, 0, 0))
        ids.append(np.empty(0, np.int32))
    return np.array(heads, np.int64), ids


def check_plan_table(plan_words_arr, perm, offsets, n_ad):
    """The device plan's table against expected_plan_table."""
    M = perm.size
    t0 = plan_table_word(M, n_ad)
    tab = plan_words_arr[t0:t0 + PLAN_REC * plan_tiles(M, n_ad)].reshape(-1, PLAN_REC)
    heads, ids = expected_plan_table(perm, offsets, n_ad)
    assert np.array_equal(tab[:, :4].astype(np.int64), heads)
    for i, want in enumerate(ids):
        assert np.array_equal(tab[i, 4:4 + want.size], want), i
        assert np.all(tab[i, 4 + want.size:] == -1), i
