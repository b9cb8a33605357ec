"""ctypes binding of liblighthouse.so, the C ABI in include/lighthouse.h.

Argument marshalling only: every function below checks that the tensors
have the dtype, size and device the C call expects, passes their device
pointers and torch's current CUDA stream, and raises LighthouseError if the
library returns an error.  All work runs in the library's CUDA kernels.
The library must be built (``python -m hierarchical_selection_attention_b200.build``);
importing this module without it raises at once, there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblighthouse.so")

LH_OK = 0
LH_ERR_INVALID_ARGUMENT = 1
LH_ERR_DEVICE_TIMEOUT = 5
LH_WAIT_TIMEOUT_CHECK_DETAIL = 900   # detail code of lh_check_wait_timeout
_STATUS = {0: "LH_OK", 1: "LH_ERR_INVALID_ARGUMENT", 2: "LH_ERR_UNSUPPORTED",
           3: "LH_ERR_WORKSPACE", 4: "LH_ERR_CUDA", 5: "LH_ERR_DEVICE_TIMEOUT",
           6: "LH_ERR_DEVICE_BOUNDS"}


class LighthouseError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {_STATUS.get(code, code)} ({_lib.lh_status_string(code).decode()})")


class lh_config(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("N", ctypes.c_int64), ("H", ctypes.c_int64),
                ("d", ctypes.c_int64), ("L", ctypes.c_int64), ("p", ctypes.c_int64),
                ("k", ctypes.c_int64), ("scale", ctypes.c_float),
                ("scatter_mode", ctypes.c_int32), ("select_mode", ctypes.c_int32),
                ("select_chunk", ctypes.c_int64)]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


class lh_gemm_operand(ctypes.Structure):
    _fields_ = [("a", ctypes.c_void_p), ("b", ctypes.c_void_p), ("k", ctypes.c_int64),
                ("lda", ctypes.c_int64), ("ldb", ctypes.c_int64)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m hierarchical_selection_attention_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    C = ctypes.POINTER(lh_config)
    sig = {
        "lh_config_check": (I32, [C]),
        "lh_subseq_len": (I64, [C]),
        "lh_total_entries": (I64, [C]),
        "lh_pooled_rows": (I64, [C]),
        "lh_workspace_bytes": (I32, [C, ctypes.POINTER(SZ), ctypes.POINTER(SZ), ctypes.POINTER(SZ)]),
        "lh_saved_offsets": (I32, [C, ctypes.POINTER(SZ)]),
        "lh_bwd_ws_offsets": (I32, [C, ctypes.POINTER(SZ)]),
        "lh_pyramid": (I32, [C, P, P, P, P, P, P, P, P, P]),
        "lh_score_topk": (I32, [C, P, P, P, P, P, SZ, P]),
        "lh_score_topk_noalloc": (I32, [C, P, P, P, P, P]),
        "lh_score_topk_noalloc_max_bytes": (SZ, []),
        "lh_gather": (I32, [C, P, P, P, P, P, P, P, P, P, P, P]),
        "lh_attn_fwd": (I32, [C, P, P, P, P, P, P, P]),
        "lh_attn_bwd": (I32, [C, P, P, P, P, P, P, P, P, P, P, P, SZ, P]),
        "lh_attn_bwd_dkdv": (I32, [C, P, P, P, P, P, P, P, P, P]),
        "lh_attn_bwd_dq": (I32, [C, P, P, P, P, P, P, P, P]),
        "lh_attn_fwd_block": (I32, [C, I32, I32, I32, P, P, P, P, P, P, P, P, P]),
        "lh_attn_bwd_dkdv_block": (I32, [C, I32, I32, I32, P, P, P, P, P, P, P, P, P, P, P]),
        "lh_attn_bwd_dq_block": (I32, [C, I32, I32, I32, P, P, P, P, P, P, P, P, P]),
        "lh_scatter": (I32, [C, P, P, P, P, SZ, P]),
        "lh_scatter_bwd": (I32, [C, P, P, P, P, P, P, P]),
        "lh_gather_bwd": (I32, [C, P, P, P, P, P, P, P, P]),
        "lh_forward": (I32, [C, P, P, P, P, P, SZ, P, SZ, P]),
        "lh_backward": (I32, [C, P, SZ, P, P, P, P, P, SZ, P]),
        "lh_forward_gather": (I32, [C, P, P, P, P, SZ, P, SZ, P]),
        "lh_forward_scatter": (I32, [C, P, SZ, P, P, SZ, P]),
        "lh_backward_scatter": (I32, [C, P, SZ, P, P, SZ, P]),
        "lh_backward_gather": (I32, [C, P, SZ, P, SZ, P, P, P, P]),
        "lh_check_wait_timeout": (I32, [P]),
        "lh_get_device_status": (I32, [P, ctypes.POINTER(I32)]),
        "lh_status_string": (ctypes.c_char_p, [I32]),
        "lh_forward_launches": (I32, [C]),
        "lh_backward_launches": (I32, [C]),
        "lh_gemm_ws_bytes": (SZ, [I64, I64, I32]),
        "lh_gemm": (I32, [I64, I64, I32, ctypes.POINTER(lh_gemm_operand), I32, I32, P, I64, I32, P,
                          SZ, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


_lib = _load()
EXPORTED = ("lh_config_check", "lh_subseq_len", "lh_total_entries", "lh_pooled_rows",
            "lh_workspace_bytes", "lh_saved_offsets", "lh_bwd_ws_offsets", "lh_pyramid", "lh_score_topk",
            "lh_score_topk_noalloc", "lh_score_topk_noalloc_max_bytes", "lh_gather",
            "lh_attn_fwd", "lh_attn_bwd", "lh_attn_bwd_dkdv", "lh_attn_bwd_dq",
            "lh_attn_fwd_block", "lh_attn_bwd_dkdv_block", "lh_attn_bwd_dq_block",
            "lh_scatter", "lh_scatter_bwd", "lh_gather_bwd",
            "lh_forward", "lh_backward", "lh_forward_gather", "lh_forward_scatter",
            "lh_backward_scatter", "lh_backward_gather", "lh_check_wait_timeout",
            "lh_get_device_status",
            "lh_status_string",
            "lh_forward_launches", "lh_backward_launches", "lh_gemm_ws_bytes", "lh_gemm")


def make_config(B, N, H, d, L, p, k, scale: float = 0.0, scatter_mode: int = 0,
                select_mode: int = 0, select_chunk: int = 0) -> lh_config:
    return lh_config(B, N, H, d, L, p, k, scale, scatter_mode, select_mode, select_chunk)


def _ck(code: int, where: str):
    if code != LH_OK:
        raise LighthouseError(code, where)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _p(t: torch.Tensor | None, dtype=None, numel=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if numel is not None and t.numel() * t.element_size() < numel:
        raise ValueError(f"{name} holds {t.numel() * t.element_size()} bytes, needs {numel}")
    return ctypes.c_void_p(t.data_ptr())


BF16, F32, I32 = torch.bfloat16, torch.float32, torch.int32


# ------------------------------------------------------------------ sizes --

def lh_config_check(cfg: lh_config) -> int:
    return _lib.lh_config_check(ctypes.byref(cfg))


def lh_subseq_len(cfg: lh_config) -> int:
    return _lib.lh_subseq_len(ctypes.byref(cfg))


def lh_total_entries(cfg: lh_config) -> int:
    return _lib.lh_total_entries(ctypes.byref(cfg))


def lh_pooled_rows(cfg: lh_config) -> int:
    return _lib.lh_pooled_rows(ctypes.byref(cfg))


def lh_workspace_bytes(cfg: lh_config):
    f, b, s = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _ck(_lib.lh_workspace_bytes(ctypes.byref(cfg), ctypes.byref(f), ctypes.byref(b),
                                ctypes.byref(s)), "lh_workspace_bytes")
    return f.value, b.value, s.value


def lh_saved_offsets(cfg: lh_config):
    arr = (ctypes.c_size_t * 8)()
    _ck(_lib.lh_saved_offsets(ctypes.byref(cfg), arr), "lh_saved_offsets")
    return list(arr)


def lh_bwd_ws_offsets(cfg: lh_config):
    arr = (ctypes.c_size_t * 5)()
    _ck(_lib.lh_bwd_ws_offsets(ctypes.byref(cfg), arr), "lh_bwd_ws_offsets")
    return list(arr)


def lh_forward_launches(cfg: lh_config) -> int:
    return _lib.lh_forward_launches(ctypes.byref(cfg))


def lh_backward_launches(cfg: lh_config) -> int:
    return _lib.lh_backward_launches(ctypes.byref(cfg))


# ------------------------------------------------------------------ stages --

def lh_pyramid(cfg, q, k, v, q_lv, k_lv, v_lv, qk, kq, stream=None):
    _ck(_lib.lh_pyramid(ctypes.byref(cfg), _p(q, BF16, name="q"), _p(k, BF16, name="k"),
                        _p(v, BF16, name="v"), _p(q_lv, BF16), _p(k_lv, BF16), _p(v_lv, BF16),
                        _p(qk, F32), _p(kq, F32), _stream(stream)), "lh_pyramid")


def lh_score_topk(cfg, qk, kq, sel_idx, slot_map, ws, stream=None):
    _ck(_lib.lh_score_topk(ctypes.byref(cfg), _p(qk, F32), _p(kq, F32), _p(sel_idx, I32),
                           _p(slot_map, I32), _p(ws), ws.numel() * ws.element_size(),
                           _stream(stream)), "lh_score_topk")


def lh_score_topk_noalloc(cfg, qk, kq, sel_idx, slot_map, stream=None):
    """lh_score_topk without a workspace argument: the scratch is the library's
    own fixed device array (see the header for the size limit and the rule
    that calls on one device must not overlap)."""
    _ck(_lib.lh_score_topk_noalloc(ctypes.byref(cfg), _p(qk, F32), _p(kq, F32),
                                   _p(sel_idx, I32), _p(slot_map, I32), _stream(stream)),
        "lh_score_topk_noalloc")


def lh_score_topk_noalloc_max_bytes() -> int:
    return _lib.lh_score_topk_noalloc_max_bytes()


def lh_gather(cfg, q, k, v, q_lv, k_lv, v_lv, sel_idx, qg, kg, vg, stream=None):
    _ck(_lib.lh_gather(ctypes.byref(cfg), _p(q, BF16), _p(k, BF16), _p(v, BF16), _p(q_lv, BF16),
                       _p(k_lv, BF16), _p(v_lv, BF16), _p(sel_idx, I32), _p(qg, BF16),
                       _p(kg, BF16), _p(vg, BF16), _stream(stream)), "lh_gather")


def lh_attn_fwd(cfg, qg, kg, vg, og, lse, og_lo=None, stream=None):
    _ck(_lib.lh_attn_fwd(ctypes.byref(cfg), _p(qg, BF16), _p(kg, BF16), _p(vg, BF16),
                         _p(og, BF16), _p(og_lo, BF16), _p(lse, F32), _stream(stream)),
        "lh_attn_fwd")


def lh_attn_bwd(cfg, qg, kg, vg, og, lse, dog, dqg, dkg, dvg, ws, og_lo=None, stream=None):
    _ck(_lib.lh_attn_bwd(ctypes.byref(cfg), _p(qg, BF16), _p(kg, BF16), _p(vg, BF16),
                         _p(og, BF16), _p(og_lo, BF16), _p(lse, F32), _p(dog, BF16),
                         _p(dqg, BF16), _p(dkg, BF16),
                         _p(dvg, BF16), _p(ws), ws.numel() * ws.element_size(),
                         _stream(stream)), "lh_attn_bwd")


def lh_attn_bwd_dkdv(cfg, qg, kg, vg, dog, lse, delta, dkg, dvg, stream=None):
    _ck(_lib.lh_attn_bwd_dkdv(ctypes.byref(cfg), _p(qg, BF16), _p(kg, BF16), _p(vg, BF16),
                              _p(dog, BF16), _p(lse, F32), _p(delta, F32), _p(dkg, BF16),
                              _p(dvg, BF16), _stream(stream)), "lh_attn_bwd_dkdv")


def lh_attn_bwd_dq(cfg, qg, kg, vg, dog, lse, delta, dqg, stream=None):
    _ck(_lib.lh_attn_bwd_dq(ctypes.byref(cfg), _p(qg, BF16), _p(kg, BF16), _p(vg, BF16),
                            _p(dog, BF16), _p(lse, F32), _p(delta, F32), _p(dqg, BF16),
                            _stream(stream)), "lh_attn_bwd_dq")


LH_BLOCK_DIAG, LH_BLOCK_FULL = 0, 1


def lh_attn_fwd_block(cfg, mode, first, last, qg, kg, vg, o_acc, lse2_acc, og, lse, og_lo=None,
                      stream=None):
    _ck(_lib.lh_attn_fwd_block(ctypes.byref(cfg), mode, int(first), int(last), _p(qg, BF16),
                               _p(kg, BF16), _p(vg, BF16), _p(o_acc, F32), _p(lse2_acc, F32),
                               _p(og, BF16), _p(og_lo, BF16), _p(lse, F32), _stream(stream)),
        "lh_attn_fwd_block")


def lh_attn_bwd_dkdv_block(cfg, mode, first, last, qg, kg, vg, dog, lse, delta, dk_acc, dv_acc,
                           dkg, dvg, stream=None):
    _ck(_lib.lh_attn_bwd_dkdv_block(ctypes.byref(cfg), mode, int(first), int(last), _p(qg, BF16),
                                    _p(kg, BF16), _p(vg, BF16), _p(dog, BF16), _p(lse, F32),
                                    _p(delta, F32), _p(dk_acc, F32), _p(dv_acc, F32),
                                    _p(dkg, BF16), _p(dvg, BF16), _stream(stream)),
        "lh_attn_bwd_dkdv_block")


def lh_attn_bwd_dq_block(cfg, mode, first, last, qg, kg, vg, dog, lse, delta, dq_acc, dqg,
                         stream=None):
    _ck(_lib.lh_attn_bwd_dq_block(ctypes.byref(cfg), mode, int(first), int(last), _p(qg, BF16),
                                  _p(kg, BF16), _p(vg, BF16), _p(dog, BF16), _p(lse, F32),
                                  _p(delta, F32), _p(dq_acc, F32), _p(dqg, BF16), _stream(stream)),
        "lh_attn_bwd_dq_block")


def lh_scatter(cfg, og, slot_map, o, ws=None, stream=None):
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    _ck(_lib.lh_scatter(ctypes.byref(cfg), _p(og, BF16), _p(slot_map, I32), _p(o, BF16),
                        _p(ws), nb, _stream(stream)), "lh_scatter")


def lh_scatter_bwd(cfg, dout, og, sel_idx, dog, delta, og_lo=None, stream=None):
    _ck(_lib.lh_scatter_bwd(ctypes.byref(cfg), _p(dout, BF16), _p(og, BF16), _p(og_lo, BF16),
                            _p(sel_idx, I32), _p(dog, BF16), _p(delta, F32), _stream(stream)),
        "lh_scatter_bwd")


def lh_gather_bwd(cfg, dqg, dkg, dvg, slot_map, dq, dk, dv, stream=None):
    _ck(_lib.lh_gather_bwd(ctypes.byref(cfg), _p(dqg, BF16), _p(dkg, BF16), _p(dvg, BF16),
                           _p(slot_map, I32), _p(dq, BF16), _p(dk, BF16), _p(dv, BF16),
                           _stream(stream)), "lh_gather_bwd")


def lh_forward(cfg, q, k, v, o, saved, ws, stream=None):
    _ck(_lib.lh_forward(ctypes.byref(cfg), _p(q, BF16), _p(k, BF16), _p(v, BF16), _p(o, BF16),
                        _p(saved), saved.numel() * saved.element_size(), _p(ws),
                        ws.numel() * ws.element_size(), _stream(stream)), "lh_forward")


def lh_backward(cfg, saved, dout, dq, dk, dv, ws, stream=None):
    _ck(_lib.lh_backward(ctypes.byref(cfg), _p(saved), saved.numel() * saved.element_size(),
                         _p(dout, BF16), _p(dq, BF16), _p(dk, BF16), _p(dv, BF16), _p(ws),
                         ws.numel() * ws.element_size(), _stream(stream)), "lh_backward")


def _nb(t):
    return t.numel() * t.element_size()


def lh_forward_gather(cfg, q, k, v, saved, ws, stream=None):
    _ck(_lib.lh_forward_gather(ctypes.byref(cfg), _p(q, BF16), _p(k, BF16), _p(v, BF16),
                               _p(saved), _nb(saved), _p(ws), _nb(ws), _stream(stream)),
        "lh_forward_gather")


def lh_forward_scatter(cfg, saved, o, ws, stream=None):
    _ck(_lib.lh_forward_scatter(ctypes.byref(cfg), _p(saved), _nb(saved), _p(o, BF16), _p(ws),
                                _nb(ws), _stream(stream)), "lh_forward_scatter")


def lh_backward_scatter(cfg, saved, dout, ws, stream=None):
    _ck(_lib.lh_backward_scatter(ctypes.byref(cfg), _p(saved), _nb(saved), _p(dout, BF16),
                                 _p(ws), _nb(ws), _stream(stream)), "lh_backward_scatter")


def lh_backward_gather(cfg, saved, ws, dq, dk, dv, stream=None):
    _ck(_lib.lh_backward_gather(ctypes.byref(cfg), _p(saved), _nb(saved), _p(ws), _nb(ws),
                                _p(dq, BF16), _p(dk, BF16), _p(dv, BF16), _stream(stream)),
        "lh_backward_gather")


def lh_get_device_status(stream=None):
    detail = ctypes.c_int32(0)
    code = _lib.lh_get_device_status(_stream(stream), ctypes.byref(detail))
    return code, detail.value


def lh_check_wait_timeout(stream=None):
    """Enqueue the bounded-wait check: one warp waits on an mbarrier nothing
    completes until the wait gives up (about 2 s) and records
    LH_ERR_DEVICE_TIMEOUT (detail LH_WAIT_TIMEOUT_CHECK_DETAIL); read it with
    lh_get_device_status."""
    _ck(_lib.lh_check_wait_timeout(_stream(stream)), "lh_check_wait_timeout")


def check_device_status(stream=None):
    code, detail = lh_get_device_status(stream)
    if code != LH_OK:
        raise LighthouseError(code, f"device status (detail {detail})")


# ------------------------------------------------------- buffer helpers --

def saved_views(cfg: lh_config, saved: torch.Tensor) -> dict:
    """Typed views into the saved buffer of lh_forward (no copies)."""
    off = lh_saved_offsets(cfg)
    B, H, d = cfg.B, cfg.H, cfg.d
    S, P = lh_subseq_len(cfg), lh_total_entries(cfg)

    def view(i, dtype, shape):
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        return saved[off[i]:off[i] + nbytes].view(dtype).view(*shape)

    return dict(sel_idx=view(0, I32, (B, H, S)), slot_map=view(1, I32, (B, H, P)),
                qg=view(2, BF16, (B, H, S, d)), kg=view(3, BF16, (B, H, S, d)),
                vg=view(4, BF16, (B, H, S, d)), og=view(5, BF16, (B, H, S, d)),
                og_lo=view(6, BF16, (B, H, S, d)), lse=view(7, F32, (B, H, S)))


def lh_gemm_ws_bytes(M, N, splits=1):
    return int(_lib.lh_gemm_ws_bytes(M, N, splits))


def lh_gemm(c, pairs, a_mn=0, b_mn=0, splits=1, ws=None, stream=None):
    """C[M, N] = sum_i A_i B_i^T into the bf16 matrix c (row-major, may be a
    row-slice view with its own stride).  pairs: list of (a, b, k) with a, b
    bf16 2-D tensors; a is [M, k] (a_mn=0) or [k, M] (a_mn=1), b is [N, k]
    (b_mn=0) or [k, N] (b_mn=1), each with unit inner stride."""
    M, N = c.shape
    ops = (lh_gemm_operand * len(pairs))()
    for i, (a, b, k) in enumerate(pairs):
        for t in (a, b):
            if t.dtype != BF16 or t.dim() != 2 or t.stride(1) != 1 or not t.is_cuda:
                raise LighthouseError(LH_ERR_INVALID_ARGUMENT, "lh_gemm operand")
        # the kernel reads exactly these extents (the C ABI cannot see allocations)
        if tuple(a.shape) != ((k, M) if a_mn else (M, k)) or tuple(b.shape) != ((k, N) if b_mn else (N, k)):
            raise LighthouseError(LH_ERR_INVALID_ARGUMENT, "lh_gemm operand shape")
        ops[i] = lh_gemm_operand(a.data_ptr(), b.data_ptr(), k, a.stride(0), b.stride(0))
    if c.dtype != BF16 or c.stride(1) != 1:
        raise LighthouseError(LH_ERR_INVALID_ARGUMENT, "lh_gemm output")
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    _ck(_lib.lh_gemm(M, N, len(pairs), ops, a_mn, b_mn, c.data_ptr(), c.stride(0), splits,
                     _p(ws), nb, _stream(stream)), "lh_gemm")
    return c


class LighthouseLayer:
    """Owns the saved and scratch buffers of one layer shape on one device.

    forward(q, k, v) -> o and backward(dout) -> (dq, dk, dv) call lh_forward and
    lh_backward on torch's current stream; tensors are [B, N, H, d] bf16.
    """

    def __init__(self, B, N, H, d, L, p, k, scale: float = 0.0, scatter_mode: int = 0,
                 device="cuda", select_mode: int = 0, select_chunk: int = 0):
        self.cfg = make_config(B, N, H, d, L, p, k, scale, scatter_mode, select_mode,
                               select_chunk)
        _ck(lh_config_check(self.cfg), "lh_config_check")
        fwd, bwd, saved = lh_workspace_bytes(self.cfg)
        self.device = torch.device(device)
        self.saved = torch.empty(saved, dtype=torch.uint8, device=self.device)
        self.ws_fwd = torch.empty(fwd, dtype=torch.uint8, device=self.device)
        self.ws_bwd = torch.empty(bwd, dtype=torch.uint8, device=self.device)
        self.S = lh_subseq_len(self.cfg)

    def forward(self, q, k, v, out=None):
        o = torch.empty_like(q) if out is None else out
        lh_forward(self.cfg, q, k, v, o, self.saved, self.ws_fwd)
        return o

    def backward(self, dout, grads=None):
        if grads is None:
            grads = tuple(torch.empty_like(dout) for _ in range(3))
        lh_backward(self.cfg, self.saved, dout, *grads, self.ws_bwd)
        return grads

    def views(self):
        return saved_views(self.cfg, self.saved)

    def bwd_views(self):
        """Typed views into the backward scratch as lh_backward leaves it:
        delta, dog, dqg, dkg, dvg (no copies)."""
        off = lh_bwd_ws_offsets(self.cfg)
        B, H, d, S = self.cfg.B, self.cfg.H, self.cfg.d, self.S

        def view(i, dtype, shape):
            n = 1
            for s in shape:
                n *= s
            nbytes = n * torch.tensor([], dtype=dtype).element_size()
            return self.ws_bwd[off[i]:off[i] + nbytes].view(dtype).view(*shape)

        return dict(delta=view(0, F32, (B, H, S)), dog=view(1, BF16, (B, H, S, d)),
                    dqg=view(2, BF16, (B, H, S, d)), dkg=view(3, BF16, (B, H, S, d)),
                    dvg=view(4, BF16, (B, H, S, d)))


class LighthouseProjectedLayer:
    """The layer with its projections (Sec. 3.1): per-head Q, K, V from the
    layer's own W_Q, W_K, W_V, the Lighthouse layer, the output projection:

        y = Lighthouse(x W_q^T, x W_k^T, x W_v^T) W_o^T

    x, y [B, N, Dm]; wq, wk, wv [H d, Dm]; wo [Dm, H d]; all bf16 and owned
    by the caller.  forward(x, wq, wk, wv, wo) -> y and backward(dy) ->
    (dx, dwq, dwk, dwv, dwo) run every product in lh_gemm and the layer in
    lh_forward / lh_backward, on torch's current stream.
    """

    def __init__(self, B, N, H, d, Dm, L, p, k, scale: float = 0.0, device="cuda",
                 select_mode: int = 0, select_chunk: int = 0):
        self.core = LighthouseLayer(B, N, H, d, L, p, k, scale, device=device,
                                    select_mode=select_mode, select_chunk=select_chunk)
        self.shape = (B, N, H, d, Dm)
        dev = self.core.device
        e = lambda *s: torch.empty(*s, dtype=BF16, device=dev)
        self.q, self.k, self.v, self.o = (e(B, N, H, d) for _ in range(4))
        self.do, self.dq, self.dk, self.dv = (e(B, N, H, d) for _ in range(4))
        # weight gradients: K = B N is long and there are few output tiles,
        # so the K range is split over enough CTAs to fill the GPU
        tiles = -(-(H * d) // 128) * -(-Dm // 256)
        self.wsplits = max(1, min(16, 2 * 148 // max(1, tiles)))
        nbytes = max(lh_gemm_ws_bytes(H * d, Dm, self.wsplits), lh_gemm_ws_bytes(Dm, H * d, self.wsplits))
        self.gemm_ws = torch.empty(max(1, nbytes), dtype=torch.uint8, device=dev)

    def forward(self, x, wq, wk, wv, wo, y=None):
        B, N, H, d, Dm = self.shape
        T, HD = B * N, H * d
        x2 = x.view(T, Dm)
        for dst, w in ((self.q, wq), (self.k, wk), (self.v, wv)):
            lh_gemm(dst.view(T, HD), [(x2, w, Dm)])
        self.core.forward(self.q, self.k, self.v, out=self.o)
        y = torch.empty(B, N, Dm, dtype=BF16, device=x.device) if y is None else y
        lh_gemm(y.view(T, Dm), [(self.o.view(T, HD), wo, HD)])
        self._saved = (x, wq, wk, wv, wo)
        return y

    def backward(self, dy, grads=None):
        B, N, H, d, Dm = self.shape
        T, HD = B * N, H * d
        x, wq, wk, wv, wo = self._saved
        dev = dy.device
        if grads is None:
            grads = (torch.empty(B, N, Dm, dtype=BF16, device=dev),
                     *(torch.empty(HD, Dm, dtype=BF16, device=dev) for _ in range(3)),
                     torch.empty(Dm, HD, dtype=BF16, device=dev))
        dx, dwq, dwk, dwv, dwo = grads
        dy2 = dy.view(T, Dm)
        lh_gemm(self.do.view(T, HD), [(dy2, wo, Dm)], b_mn=1)                  # dO = dy W_o
        lh_gemm(dwo, [(dy2, self.o.view(T, HD), T)], a_mn=1, b_mn=1,           # dW_o = dy^T O
                splits=self.wsplits, ws=self.gemm_ws)
        self.core.backward(self.do, grads=(self.dq, self.dk, self.dv))
        g = [t.view(T, HD) for t in (self.dq, self.dk, self.dv)]
        lh_gemm(dx.view(T, Dm), [(g[0], wq, HD), (g[1], wk, HD), (g[2], wv, HD)], b_mn=1)
        for dw, gi in zip((dwq, dwk, dwv), g):                                 # dW_i = dQ_i^T x
            lh_gemm(dw, [(gi, x.view(T, Dm), T)], a_mn=1, b_mn=1, splits=self.wsplits, ws=self.gemm_ws)
        return grads


class LighthouseAttention(torch.autograd.Function):
    """Autograd wrapper: y = Lighthouse(q, k, v); the selection is not differentiated."""

    @staticmethod
    def forward(ctx, q, k, v, layer: LighthouseLayer):
        ctx.layer = layer
        return layer.forward(q.contiguous(), k.contiguous(), v.contiguous())

    @staticmethod
    def backward(ctx, dout):
        dq, dk, dv = ctx.layer.backward(dout.contiguous())
        return dq, dk, dv, None
