"""ctypes binding of libvgqa (include/varlen_gqa.h): argument marshalling only.

Every step of the attention runs in the library's CUDA kernels; this module
checks dtypes, shapes and devices of torch tensors, passes their device
pointers and the current CUDA stream, and turns ATTN_* codes into exceptions.
There is no fallback: if the library is missing or no sm_100 device is
present, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libvgqa.so")

ATTN_OK = 0
ATTN_VARIANT_AUTO, ATTN_VARIANT_SIMT, ATTN_VARIANT_MMA, ATTN_VARIANT_TC = 0, 1, 2, 3
ATTN_COMBINE_AUTO, ATTN_COMBINE_KERNEL, ATTN_COMBINE_FUSED = 0, 1, 2
ATTN_DEV_ERR_OFFSETS = 0x1
ATTN_DEV_ERR_Q_TOO_LONG = 0x2
ATTN_DEV_ERR_K_TOO_LONG = 0x4
ATTN_DEV_ERR_TIMEOUT = 0x8
ATTN_DEV_ERR_PAGE = 0x10

EXPORTED = ("attn_plan", "attn_plan_ex", "attn_plan_info", "attn_run", "attn_run_strided", "attn_run_paged",
            "attn_merge_lse", "attn_check_error", "attn_destroy", "attn_strerror")


class Overrides(ctypes.Structure):
    _fields_ = [("nsplit", ctypes.c_int), ("block_n", ctypes.c_int), ("variant", ctypes.c_int),
                ("stages", ctypes.c_int), ("combine", ctypes.c_int), ("ctas", ctypes.c_int),
                ("deterministic", ctypes.c_int), ("wait_limit_us", ctypes.c_int), ("test_stall", ctypes.c_int)]


class PlanDesc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "B_max", "s_max", "Hq", "Hkv", "D", "max_q", "G", "variant", "nsplit", "chunk", "block_n",
        "stages", "rows_per_block", "row_tiles", "grid_x", "grid_y", "grid_z", "ctas", "deterministic", "combine",
        "combine_blocks",
        "smem_bytes", "num_sms")] + [("scratch_bytes", ctypes.c_size_t)]


class AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} (code {code})")


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load libvgqa.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libvgqa.so not built ({LIB_PATH}); run "
                               "`python -m varlen_gqa_split_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, i32p = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
        L.attn_plan.argtypes = [ctypes.POINTER(vp), i, i, i, i, i, i]
        L.attn_plan.restype = i
        L.attn_plan_ex.argtypes = [ctypes.POINTER(vp), i, i, i, i, i, i, ctypes.POINTER(Overrides)]
        L.attn_plan_ex.restype = i
        L.attn_plan_info.argtypes = [vp, ctypes.POINTER(PlanDesc)]
        L.attn_plan_info.restype = i
        L.attn_run.argtypes = [vp, vp, vp, vp, i32p, i32p, vp, vp, vp]
        L.attn_run.restype = i
        L.attn_run_strided.argtypes = [vp, vp, vp, vp, i32p, i32p, vp, vp, ctypes.c_int64, ctypes.c_int64, vp]
        L.attn_run_strided.restype = i
        i64 = ctypes.c_int64
        L.attn_run_paged.argtypes = [vp, vp, vp, vp, i64, i64, i, i, i32p, i, i32p, i32p, vp, vp, vp]
        L.attn_run_paged.restype = i
        L.attn_merge_lse.argtypes = [i, vp, vp, i64, i32p, i, i, i, vp, vp, vp]
        L.attn_merge_lse.restype = i
        L.attn_check_error.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
        L.attn_check_error.restype = i
        L.attn_destroy.argtypes = [vp]
        L.attn_destroy.restype = None
        L.attn_strerror.argtypes = [i]
        L.attn_strerror.restype = ctypes.c_char_p
        _lib = L
        return L


def merge_lse(outs, lses, cu_q, out=None, lse=None, stream=None):
    """out, lse = merge_lse(outs, lses, cu_q[, out, lse, stream]): combine the
    attention results of n disjoint key ranges (attn_merge_lse).

    outs [n, T_q, Hq, D] bf16 and lses [n, T_q, Hq] fp32 contiguous CUDA
    tensors; cu_q int32 [B_max + 1]; only tokens [cu_q[0], cu_q[B_max]) are
    written."""
    if outs.dtype != torch.bfloat16 or not outs.is_cuda or not outs.is_contiguous() or outs.dim() != 4:
        raise ValueError("outs must be a contiguous bf16 CUDA tensor [n, T_q, Hq, D]")
    n, T_q, Hq, D = outs.shape
    if lses.dtype != torch.float32 or not lses.is_contiguous() or tuple(lses.shape) != (n, T_q, Hq):
        raise ValueError("lses must be a contiguous fp32 tensor [n, T_q, Hq]")
    if cu_q.dtype != torch.int32 or not cu_q.is_cuda or not cu_q.is_contiguous() or cu_q.dim() != 1:
        raise ValueError("cu_q must be a contiguous int32 CUDA tensor")
    if out is None:
        out = torch.empty(T_q, Hq, D, dtype=torch.bfloat16, device=outs.device)
    if lse is None:
        lse = torch.empty(T_q, Hq, dtype=torch.float32, device=outs.device)
    if out.dtype != torch.bfloat16 or tuple(out.shape) != (T_q, Hq, D) or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor [T_q, Hq, D]")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (T_q, Hq) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 tensor [T_q, Hq]")
    rc = lib().attn_merge_lse(int(n), outs.data_ptr(), lses.data_ptr(), int(T_q), cu_q.data_ptr(),
                              int(cu_q.numel() - 1), int(Hq), int(D), out.data_ptr(), lse.data_ptr(),
                              _stream_ptr(stream))
    _check(rc, "attn_merge_lse")
    return out, lse


def strerror(code: int) -> str:
    return lib().attn_strerror(int(code)).decode()


def _check(code: int, where: str):
    if code != ATTN_OK:
        raise AttnError(code, where)


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class Plan:
    """A plan: launch shape, split count and scratch fixed from constants.

    Plan(B_max, s_max, Hq, Hkv, D, max_q=1, *, nsplit=0, block_n=0, variant=0,
    stages=0, combine=0, ctas=0, deterministic=0, wait_limit_us=0, test_stall=0) -- the
    keyword choices override the planner (0 = its own; deterministic=1 asks
    for static tile shares, -1 for run-time balancing of shared units;
    wait_limit_us bounds one device wait; test_stall=1 is the test hook of
    attn_overrides that makes the first call's merge waits run out)."""

    def __init__(self, B_max, s_max, Hq, Hkv, D, max_q=1, *, nsplit=0, block_n=0, variant=0,
                 stages=0, combine=0, ctas=0, deterministic=0, wait_limit_us=0, test_stall=0):
        L = lib()
        h = ctypes.c_void_p()
        if nsplit or block_n or variant or stages or combine or ctas or deterministic or wait_limit_us or test_stall:
            o = Overrides(int(nsplit), int(block_n), int(variant), int(stages), int(combine), int(ctas),
                          int(deterministic), int(wait_limit_us), int(test_stall))
            rc = L.attn_plan_ex(ctypes.byref(h), int(B_max), int(s_max), int(Hq), int(Hkv), int(D),
                                int(max_q), ctypes.byref(o))
        else:
            rc = L.attn_plan(ctypes.byref(h), int(B_max), int(s_max), int(Hq), int(Hkv), int(D),
                             int(max_q))
        _check(rc, "attn_plan")
        self._h = h
        self.device = torch.cuda.current_device()
        self.info = self._info()

    def _info(self) -> dict:
        d = PlanDesc()
        _check(lib().attn_plan_info(self._h, ctypes.byref(d)), "attn_plan_info")
        return {name: getattr(d, name) for name, _ in PlanDesc._fields_}

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    def run(self, q, k, v, cu_q, cu_k, out=None, lse=None, stream=None):
        """out, lse = plan.run(q, k, v, cu_q, cu_k[, out, lse, stream]).

        q [T_q, Hq, D] bf16 contiguous CUDA tensor; k / v [T_kv, Hkv, D] bf16
        CUDA tensors whose heads are contiguous within a token -- packed, or
        views into a larger buffer with a token stride (e.g. the halves of a
        fused [T, 2, Hkv, D] cache), which go through attn_run_strided;
        cu_q / cu_k int32 CUDA tensors with B_max + 1 entries; out / lse are
        allocated when not given (pass them for graph capture)."""
        out, lse = self._check_common(q, cu_q, cu_k, out, lse, "attn_run")
        i = self.info
        for name, t in (("k", k), ("v", v)):
            if t.dtype != torch.bfloat16 or not t.is_cuda:
                raise TypeError(f"{name} must be a bf16 CUDA tensor")
            if t.dim() != 3 or t.shape[1:] != (i["Hkv"], i["D"]):
                raise ValueError(f"{name} must be [T_kv, {i['Hkv']}, {i['D']}]")
            if t.stride(2) != 1 or t.stride(1) != i["D"] or (t.shape[0] > 1 and t.stride(0) < i["Hkv"] * i["D"]):
                raise ValueError(f"{name} must keep each token's heads contiguous (strides (s, D, 1), s >= Hkv*D)")
        packed = i["Hkv"] * i["D"]
        ks = k.stride(0) if k.shape[0] > 1 else packed
        vs = v.stride(0) if v.shape[0] > 1 else packed
        if ks == packed and vs == packed:
            rc = lib().attn_run(self._h, q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_q.data_ptr(),
                                cu_k.data_ptr(), out.data_ptr(), lse.data_ptr(), _stream_ptr(stream))
            _check(rc, "attn_run")
        else:
            rc = lib().attn_run_strided(self._h, q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_q.data_ptr(),
                                        cu_k.data_ptr(), out.data_ptr(), lse.data_ptr(), ks, vs,
                                        _stream_ptr(stream))
            _check(rc, "attn_run_strided")
        return out, lse

    def run_paged(self, q, k_cache, v_cache, block_table, cu_q, cu_k, out=None, lse=None, stream=None):
        """out, lse = plan.run_paged(q, k_cache, v_cache, block_table, cu_q, cu_k[, out, lse, stream]).

        k_cache / v_cache [num_pages, page_size, Hkv, D] bf16 CUDA tensors
        (each token's heads contiguous; token and page strides free, so the
        halves of a [num_pages, 2, page_size, Hkv, D] cache work);
        block_table [B_max, n] int32 CUDA tensor, row b listing the pages of
        sequence b in key order (n >= ceil(s_max / page_size), row stride
        free); cu_k supplies the key lengths only.  Goes through
        attn_run_paged."""
        out, lse = self._check_common(q, cu_q, cu_k, out, lse, "attn_run_paged")
        i = self.info
        shape = None
        for name, t in (("k_cache", k_cache), ("v_cache", v_cache)):
            if t.dtype != torch.bfloat16 or not t.is_cuda:
                raise TypeError(f"{name} must be a bf16 CUDA tensor")
            if t.dim() != 4 or t.shape[2:] != (i["Hkv"], i["D"]):
                raise ValueError(f"{name} must be [num_pages, page_size, {i['Hkv']}, {i['D']}]")
            if t.stride(3) != 1 or t.stride(2) != i["D"]:
                raise ValueError(f"{name} must keep each token's heads contiguous")
            if shape is not None and (t.shape != shape or t.stride() != k_cache.stride()):
                raise ValueError("k_cache and v_cache must have the same shape and strides")
            shape = t.shape
        n_pages, page_size = int(shape[0]), int(shape[1])
        tok = k_cache.stride(1) if page_size > 1 else i["Hkv"] * i["D"]
        pstride = k_cache.stride(0) if n_pages > 1 else page_size * tok
        bt = block_table
        if bt.dtype != torch.int32 or not bt.is_cuda or bt.dim() != 2 or bt.shape[0] != i["B_max"] or bt.stride(1) != 1:
            raise ValueError("block_table must be an int32 CUDA tensor [B_max, n] with unit column stride")
        if bt.shape[1] * page_size < i["s_max"]:
            raise ValueError("block_table rows must cover s_max keys")
        rc = lib().attn_run_paged(self._h, q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), int(pstride),
                                  int(tok), page_size, n_pages, bt.data_ptr(), int(bt.stride(0)),
                                  cu_q.data_ptr(), cu_k.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                  _stream_ptr(stream))
        _check(rc, "attn_run_paged")
        return out, lse

    def _check_common(self, q, cu_q, cu_k, out, lse, where):
        if self._h is None:
            raise AttnError(-5, where)
        i = self.info
        if q.dtype != torch.bfloat16 or not q.is_cuda or not q.is_contiguous():
            raise TypeError("q must be a contiguous bf16 CUDA tensor")
        if q.dim() != 3 or q.shape[1:] != (i["Hq"], i["D"]):
            raise ValueError(f"q must be [T_q, {i['Hq']}, {i['D']}]")
        for name, t in (("cu_q", cu_q), ("cu_k", cu_k)):
            if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous() or t.numel() != i["B_max"] + 1:
                raise ValueError(f"{name} must be a contiguous int32 CUDA tensor of B_max+1 entries")
        if out is None:
            out = torch.empty_like(q)
        if lse is None:
            lse = torch.empty(q.shape[0], i["Hq"], dtype=torch.float32, device=q.device)
        if out.dtype != torch.bfloat16 or out.shape != q.shape or not out.is_contiguous():
            raise ValueError("out must be a contiguous bf16 tensor shaped like q")
        if lse.dtype != torch.float32 or lse.shape != (q.shape[0], i["Hq"]) or not lse.is_contiguous():
            raise ValueError("lse must be a contiguous fp32 tensor [T_q, Hq]")
        return out, lse

    def check_error(self, stream=None) -> int:
        """Synchronise, then read and clear the sticky device error bits."""
        f = ctypes.c_uint32(0)
        _check(lib().attn_check_error(self._h, _stream_ptr(stream), ctypes.byref(f)), "attn_check_error")
        return int(f.value)

    def close(self):
        if self._h is not None:
            lib().attn_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()
