"""ctypes binding of libbi.so (C ABI declared in include/bi.h).

Argument marshalling only: each function checks dtypes / shapes / devices of
the torch tensors it is given, passes raw device pointers, sizes and the
current CUDA stream to the entry point of the same name, and raises
``BiError`` on a non-OK status.  Every step of the computation runs in the
library's CUDA kernels; there is no fallback.  If libbi.so has not been
built, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbi.so")

OK = 0
STATUS_NAMES = {0: "BI_OK", 1: "BI_ERR_INVALID_ARG", 2: "BI_ERR_UNSUPPORTED_SHAPE",
                3: "BI_ERR_WORKSPACE", 4: "BI_ERR_CUDA", 5: "BI_ERR_TIMEOUT", 6: "BI_ERR_NO_DEVICE"}
MODES = {"unsplit": 0, "atomic": 1, "tree": 2}


class BiError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")


_lib = None

P, I, Z, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
_SIGS = {
    "bi_lora_shrink": (I, [P, P, P, I, I, I, I, I, P]),
    "bi_lora_plan_bytes": (Z, [I, I]),
    "bi_lora_plan": (I, [P, I, I, P, Z, P]),
    "bi_lora_shrink_segmented": (I, [P, P, P, I, P, I, I, I, I, I, P]),
    "bi_lora_shrink_segmented_noalloc": (I, [P, P, P, I, P, I, I, I, I, I, P]),
    "bi_lora_fused": (I, [P, P, P, P, I, P, P, I, I, I, I, I, I, P]),
    "bi_lora_expand": (I, [P, P, P, I, I, I, I, P]),
    "bi_lora_expand_segmented": (I, [P, P, P, I, P, I, I, I, I, P]),
    "bi_gemm": (I, [P, P, P, I, I, I, I, P]),
    "bi_addmm": (I, [P, P, P, P, I, I, I, I, P]),
    "bi_gemm_tree_ws_bytes": (Z, [I, I, I]),
    "bi_gemm_tree_partials": (I, [P, P, P, I, I, I, I, P]),
    "bi_gemm_tree": (I, [P, P, P, I, I, I, I, P, Z, P]),
    "bi_tree_combine": (I, [P, P, I, Z, P]),
    "bi_tree_combine_peers": (I, [ctypes.POINTER(ctypes.c_void_p), I, P, Z, Z, P]),
    "bi_rmsnorm": (I, [P, P, P, I, I, F, P]),
    "bi_log_softmax": (I, [P, P, I, I, P]),
    "bi_mean": (I, [P, P, I, I, P]),
    "bi_math_spec": (I, [P, P, Z, I, P]),
    "bi_attn_decode_ws_bytes": (Z, [I, I, I, I]),
    "bi_attn_decode": (I, [P, P, P, P, P, I, I, I, I, I, F, P, Z, P]),
    "bi_get_device_status": (I, [P]),
    "bi_status_string": (ctypes.c_char_p, [I]),
    "bi_selftest_bounded_wait": (I, [I, P]),
    "bi_debug_set_fault": (None, [I]),
}


def lib():
    """Load libbi.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m invariant_bi_lora_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(l, name)
            fn.restype = res
            fn.argtypes = args
        _lib = l
    return _lib


def _call(name, *args):
    st = getattr(lib(), name)(*args)
    if st != OK:
        raise BiError(name, st)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _check(t: torch.Tensor, name: str, dtype, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")


# --------------------------------------------------------------------- LoRA

def lora_shrink(x, A, y, splits=8, mode="tree", stream=None):
    """y[M,r] (fp32) = x[M,K] (bf16) . A^T-storage, A bf16 [r,K]."""
    _check(x, "x", torch.bfloat16, 2)
    _check(A, "A", torch.bfloat16, 2)
    _check(y, "y", torch.float32, 2)
    M, K = x.shape
    r = A.shape[0]
    if A.shape[1] != K or tuple(y.shape) != (M, r):
        raise ValueError("shape mismatch")
    _call("bi_lora_shrink", _ptr(x), _ptr(A), _ptr(y), M, K, r, splits, MODES[mode], _stream(stream))
    return y


def lora_plan_bytes(M, n_adapters):
    return int(lib().bi_lora_plan_bytes(M, n_adapters))


def lora_plan(ids, n_adapters, plan=None, stream=None):
    """Token plan (int32 tensor) grouping tokens by adapter id."""
    _check(ids, "ids", torch.int32, 1)
    M = ids.shape[0]
    nbytes = lora_plan_bytes(M, n_adapters)
    if plan is None:
        plan = torch.empty(nbytes // 4, dtype=torch.int32, device=ids.device)
    _check(plan, "plan", torch.int32, 1)
    _call("bi_lora_plan", _ptr(ids), M, n_adapters, _ptr(plan), plan.numel() * 4, _stream(stream))
    return plan


def lora_shrink_segmented(x, A, plan, y, splits=8, mode="tree", stream=None):
    """y[t] = x[t] . A_{id[t]}; A bf16 [n_ad, r, K]; plan from lora_plan."""
    _check(x, "x", torch.bfloat16, 2)
    _check(A, "A", torch.bfloat16, 3)
    _check(plan, "plan", torch.int32, 1)
    _check(y, "y", torch.float32, 2)
    M, K = x.shape
    n_ad, r, K2 = A.shape
    if K2 != K or tuple(y.shape) != (M, r):
        raise ValueError("shape mismatch")
    if plan.numel() * 4 < lora_plan_bytes(M, n_ad):
        raise ValueError("plan too small")
    _call("bi_lora_shrink_segmented", _ptr(x), _ptr(A), _ptr(plan), n_ad, _ptr(y), M, K, r,
          splits, MODES[mode], _stream(stream))
    return y


NOALLOC_MAX_TOKENS = 65536


def lora_shrink_segmented_noalloc(x, A, ids, y, splits=8, mode="tree", stream=None):
    """Segmented shrink that allocates nothing: ids int32 [M] go straight to
    the library, which builds the token plan in its own fixed device array
    (M <= NOALLOC_MAX_TOKENS).  Calls that overlap on the GPU race on that
    array; serialise them."""
    _check(x, "x", torch.bfloat16, 2)
    _check(A, "A", torch.bfloat16, 3)
    _check(ids, "ids", torch.int32, 1)
    _check(y, "y", torch.float32, 2)
    M, K = x.shape
    n_ad, r, K2 = A.shape
    if K2 != K or tuple(y.shape) != (M, r) or ids.shape[0] != M:
        raise ValueError("shape mismatch")
    _call("bi_lora_shrink_segmented_noalloc", _ptr(x), _ptr(A), _ptr(ids), n_ad, _ptr(y), M, K, r,
          splits, MODES[mode], _stream(stream))
    return y


def lora_fused(x, A, B, plan, out, y=None, splits=8, accumulate=False, stream=None):
    """Segmented shrink then expand in one launch: out[t] (+)= bf16(y[t]) .
    B_{id[t]}^T with y = x[t] . A_{id[t]} (split-K tree, or unsplit when
    splits = 1); y is also written when given.  A bf16 [n_ad, r, K],
    B bf16 [n_ad, N, r], out fp32 [M, N]."""
    _check(x, "x", torch.bfloat16, 2)
    _check(A, "A", torch.bfloat16, 3)
    _check(B, "B", torch.bfloat16, 3)
    _check(plan, "plan", torch.int32, 1)
    _check(out, "out", torch.float32, 2)
    M, K = x.shape
    n_ad, r, K2 = A.shape
    N = B.shape[1]
    if K2 != K or tuple(B.shape) != (n_ad, N, r) or tuple(out.shape) != (M, N):
        raise ValueError("shape mismatch")
    if y is not None:
        _check(y, "y", torch.float32, 2)
        if tuple(y.shape) != (M, r):
            raise ValueError("shape mismatch")
    if plan.numel() * 4 < lora_plan_bytes(M, n_ad):
        raise ValueError("plan too small")
    _call("bi_lora_fused", _ptr(x), _ptr(A), _ptr(B), _ptr(plan), n_ad, _ptr(y), _ptr(out), M, K, r, N,
          splits, int(bool(accumulate)), _stream(stream))
    return out


def lora_expand(y, B, out, accumulate=False, stream=None):
    """out[M,N] (+)= bf16(y[M,r]) . B^T, B bf16 [N, r]."""
    _check(y, "y", torch.float32, 2)
    _check(B, "B", torch.bfloat16, 2)
    _check(out, "out", torch.float32, 2)
    M, r = y.shape
    N = B.shape[0]
    if B.shape[1] != r or tuple(out.shape) != (M, N):
        raise ValueError("shape mismatch")
    _call("bi_lora_expand", _ptr(y), _ptr(B), _ptr(out), M, r, N, int(bool(accumulate)), _stream(stream))
    return out


def lora_expand_segmented(y, B, plan, out, accumulate=False, stream=None):
    """out[t] (+)= bf16(y[t]) . B_{id[t]}^T, B bf16 [n_ad, N, r]."""
    _check(y, "y", torch.float32, 2)
    _check(B, "B", torch.bfloat16, 3)
    _check(plan, "plan", torch.int32, 1)
    _check(out, "out", torch.float32, 2)
    M, r = y.shape
    n_ad, N, r2 = B.shape
    if r2 != r or tuple(out.shape) != (M, N):
        raise ValueError("shape mismatch")
    if plan.numel() * 4 < lora_plan_bytes(M, n_ad):
        raise ValueError("plan too small")
    _call("bi_lora_expand_segmented", _ptr(y), _ptr(B), _ptr(plan), n_ad, _ptr(out), M, r, N,
          int(bool(accumulate)), _stream(stream))
    return out


# --------------------------------------------------------------------- GEMM

def gemm(A, W, C, stream=None):
    """C[M,N] = A[M,K] . W[N,K]^T; C fp32 or bf16."""
    _check(A, "A", torch.bfloat16, 2)
    _check(W, "W", torch.bfloat16, 2)
    if C.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("C must be float32 or bfloat16")
    _check(C, "C", C.dtype, 2)
    M, K = A.shape
    N = W.shape[0]
    if W.shape[1] != K or tuple(C.shape) != (M, N):
        raise ValueError("shape mismatch")
    _call("bi_gemm", _ptr(A), _ptr(W), _ptr(C), M, N, K, int(C.dtype == torch.bfloat16), _stream(stream))
    return C


def addmm(bias, A, W, C, stream=None):
    """C[M,N] = bias[N] + A[M,K] . W[N,K]^T (torch.addmm); bias bf16, C fp32 or bf16."""
    _check(bias, "bias", torch.bfloat16, 1)
    _check(A, "A", torch.bfloat16, 2)
    _check(W, "W", torch.bfloat16, 2)
    if C.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("C must be float32 or bfloat16")
    _check(C, "C", C.dtype, 2)
    M, K = A.shape
    N = W.shape[0]
    if W.shape[1] != K or tuple(C.shape) != (M, N) or bias.shape[0] != N:
        raise ValueError("shape mismatch")
    _call("bi_addmm", _ptr(bias), _ptr(A), _ptr(W), _ptr(C), M, N, K, int(C.dtype == torch.bfloat16),
          _stream(stream))
    return C


def gemm_tree_ws_bytes(M, N, shards):
    return int(lib().bi_gemm_tree_ws_bytes(M, N, shards))


def gemm_tree_partials(A, W, partials, shards, stream=None):
    _check(A, "A", torch.bfloat16, 2)
    _check(W, "W", torch.bfloat16, 2)
    _check(partials, "partials", torch.float32, 3)
    M, K = A.shape
    N = W.shape[0]
    if W.shape[1] != K or tuple(partials.shape) != (shards, M, N):
        raise ValueError("shape mismatch")
    _call("bi_gemm_tree_partials", _ptr(A), _ptr(W), _ptr(partials), M, N, K, shards, _stream(stream))
    return partials


def gemm_tree(A, W, C, shards=1, ws=None, stream=None):
    _check(A, "A", torch.bfloat16, 2)
    _check(W, "W", torch.bfloat16, 2)
    _check(C, "C", torch.float32, 2)
    M, K = A.shape
    N = W.shape[0]
    if W.shape[1] != K or tuple(C.shape) != (M, N):
        raise ValueError("shape mismatch")
    need = gemm_tree_ws_bytes(M, N, shards)
    if need and ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=A.device)
    wsp, wsb = (None, 0) if ws is None else (_ptr(ws), ws.numel() * ws.element_size())
    _call("bi_gemm_tree", _ptr(A), _ptr(W), _ptr(C), M, N, K, shards, wsp, wsb, _stream(stream))
    return C


def tree_combine(partials, out, stream=None):
    """out = canonical tree over partials' first axis."""
    _check(partials, "partials", torch.float32)
    _check(out, "out", torch.float32)
    s = partials.shape[0]
    if partials.numel() != s * out.numel():
        raise ValueError("shape mismatch")
    _call("bi_tree_combine", _ptr(partials), _ptr(out), s, out.numel(), _stream(stream))
    return out


def tree_combine_peers(ptrs, out, begin=0, count=None, stream=None):
    """out[begin:begin+count] = canonical tree over the partials behind the
    device pointers `ptrs` (ints; each partial fp32 with out's numel, in this
    GPU's memory or a peer's), read with plain loads in one kernel."""
    _check(out, "out", torch.float32)
    count = out.numel() - begin if count is None else count
    if begin < 0 or count < 0 or begin + count > out.numel():
        raise ValueError("range outside out")
    arr = (ctypes.c_void_p * len(ptrs))(*[ctypes.c_void_p(int(q)) for q in ptrs])
    _call("bi_tree_combine_peers", arr, len(ptrs), _ptr(out), begin, count, _stream(stream))
    return out


# ----------------------------------------------------------------- row ops

def rmsnorm(x, w, y, eps=1e-6, stream=None):
    _check(x, "x", torch.bfloat16, 2)
    _check(w, "w", torch.bfloat16, 1)
    _check(y, "y", torch.bfloat16, 2)
    R, n = x.shape
    if w.shape[0] != n or y.shape != x.shape:
        raise ValueError("shape mismatch")
    _call("bi_rmsnorm", _ptr(x), _ptr(w), _ptr(y), R, n, float(eps), _stream(stream))
    return y


def log_softmax(x, out, stream=None):
    _check(x, "x", torch.float32, 2)
    _check(out, "out", torch.float32, 2)
    if out.shape != x.shape:
        raise ValueError("shape mismatch")
    R, n = x.shape
    _call("bi_log_softmax", _ptr(x), _ptr(out), R, n, _stream(stream))
    return out


def mean(x, out, stream=None):
    _check(x, "x", torch.float32, 2)
    _check(out, "out", torch.float32, 1)
    R, n = x.shape
    if out.shape[0] != R:
        raise ValueError("shape mismatch")
    _call("bi_mean", _ptr(x), _ptr(out), R, n, _stream(stream))
    return out


def math_spec(x, y, which, stream=None):
    """y = the library's exp (which='exp'), log ('log') or the exp shortcut
    log_softmax uses on [-87, 88] ('exp_fast'; 'exp_fast2' on packed two-lane
    instructions) of x."""
    _check(x, "x", torch.float32)
    _check(y, "y", torch.float32)
    _call("bi_math_spec", _ptr(x), _ptr(y), x.numel(), {"exp": 0, "log": 1, "exp_fast": 2, "exp_fast2": 3}[which],
          _stream(stream))
    return y


# ------------------------------------------------------------- attention

def attn_decode_ws_bytes(B, Hq, D, Lmax):
    return int(lib().bi_attn_decode_ws_bytes(B, Hq, D, Lmax))


def attn_decode(q, k, v, lens, out, scale=None, ws=None, stream=None):
    """Decode attention with a fixed-size KV split: q bf16 [B, Hq, D];
    k, v bf16 [B, Hkv, Lmax, D]; lens int32 [B]; out fp32 [B, Hq, D]."""
    _check(q, "q", torch.bfloat16, 3)
    _check(k, "k", torch.bfloat16, 4)
    _check(v, "v", torch.bfloat16, 4)
    _check(lens, "lens", torch.int32, 1)
    _check(out, "out", torch.float32, 3)
    B, Hq, D = q.shape
    B2, Hkv, Lmax, D2 = k.shape
    if B2 != B or D2 != D or v.shape != k.shape or lens.shape[0] != B or tuple(out.shape) != (B, Hq, D):
        raise ValueError("shape mismatch")
    if scale is None:
        scale = 1.0 / float(D) ** 0.5
    need = attn_decode_ws_bytes(B, Hq, D, Lmax)
    if ws is None:
        ws = torch.empty(max(need, 4), dtype=torch.uint8, device=q.device)
    _call("bi_attn_decode", _ptr(q), _ptr(k), _ptr(v), _ptr(lens), _ptr(out), B, Hq, Hkv, D, Lmax, float(scale),
          _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    return out


# ------------------------------------------------------------------ status

def get_device_status(stream=None) -> int:
    """Synchronise and return (and clear) the device status word."""
    return int(lib().bi_get_device_status(_stream(stream)))


def status_string(code: int) -> str:
    return lib().bi_status_string(code).decode()


def selftest_bounded_wait(max_polls=1000, stream=None):
    _call("bi_selftest_bounded_wait", int(max_polls), _stream(stream))


FAULT_NONE, FAULT_SKIP_STAGE = 0, 1


def debug_set_fault(code):
    """Test-only: FAULT_SKIP_STAGE makes the following GEMM calls leave one
    stage unloaded (their bounded wait reports BI_ERR_TIMEOUT); FAULT_NONE
    turns it off."""
    lib().bi_debug_set_fault(int(code))
