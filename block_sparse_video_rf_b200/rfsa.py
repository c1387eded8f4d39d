"""ctypes binding of ``librfsa.so`` (see include/rfsa.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  Importing this module fails loudly when the library has not been
built (``python -m block_sparse_video_rf_b200.build``); there is no fallback.
Tensors are torch CUDA tensors; the stream defaults to torch's current
stream on the tensor's device.
"""

from __future__ import annotations

import ctypes
import math
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "librfsa.so")

RF_BSND, RF_BNSD = 0, 1
LAYOUTS = {"BSND": RF_BSND, "BNSD": RF_BNSD}
STATUS = {0: "RF_OK", 1: "RF_ERR_LAYOUT", 2: "RF_ERR_ARG", 3: "RF_ERR_UNSUPPORTED", 4: "RF_ERR_CUDA",
          5: "RF_ERR_WORKSPACE", 6: "RF_ERR_TIMEOUT"}

PLAN_FIELDS = ["S", "txt_len", "T", "H", "W", "Ha", "Wa", "n_promoted", "n_tail", "P", "P_pad", "nb", "ff", "k",
               "dense", "S_int", "n_tiles", "mask_words"]
WS_FIELDS = ["q_int", "k_int", "v_int", "pooled_q", "pooled_k", "mask", "kept", "margin", "counter", "status",
             "q8", "k8", "v8", "scales", "vmax", "redo", "total"]
RF_BF16, RF_F16 = 0, 1
PRECISIONS = {"native": 0, "fp8": 1}

# Every symbol include/rfsa.h declares.
EXPORTS = ["rf_plan", "rf_workspace_layout", "rf_workspace_size", "rf_sparse_attention", "rf_sparse_attention_ws",
           "rf_prepare", "rf_attend", "rf_unpermute", "rf_sparse_attention_host", "rf_read_status",
           "rf_debug_set_wait", "rf_debug_set_path", "rf_debug_set_stage_event", "rf_read_stats",
           "rf_block_mask_noalloc", "rf_last_error_string", "rf_workspace_layout_ex",
           "rf_workspace_size_ex", "rf_prepare_ex", "rf_attend_ex", "rf_sparse_attention_ex", "rf_plan_kv",
           "rf_read_stats_ex", "rf_debug_exp2_poly", "rf_sparse_attention_host_ex"]


class RfPlan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in PLAN_FIELDS]

    def as_dict(self):
        return {n: getattr(self, n) for n in PLAN_FIELDS}


class RfWsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in WS_FIELDS]


class RfStats(ctypes.Structure):
    _fields_ = [("kept_blocks", ctypes.c_longlong), ("query_blocks", ctypes.c_longlong),
                ("kept_pairs", ctypes.c_double), ("density", ctypes.c_double), ("near_ties", ctypes.c_int),
                ("redo_tiles", ctypes.c_int), ("status", ctypes.c_int)]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


class RfError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m block_sparse_video_rf_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    I, F, P, Z = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
    geo = [I, I, I, I, I, I, I, I]  # layout, B, S, N, D, txt_len, t, h ... (w appended below)
    sig = {
        "rf_plan": (I, [I, I, I, I, I, I, F, ctypes.POINTER(RfPlan)]),
        "rf_workspace_layout": (I, [I, I, I, ctypes.POINTER(RfPlan), ctypes.POINTER(RfWsLayout)]),
        "rf_workspace_size": (Z, [I, I, I, I, I, I, I, I]),
        "rf_sparse_attention": (I, [P, P, P] + geo + [I, I, F, F, P, P]),
        "rf_sparse_attention_ws": (I, [P, P, P] + geo + [I, I, F, F, P, P, Z, P]),
        "rf_prepare": (I, [P, P, P] + geo + [I, I, F, P, Z, P]),
        "rf_attend": (I, geo + [I, I, F, F, P, P, Z, P]),
        "rf_unpermute": (I, [P] + geo + [I, P, P]),
        "rf_sparse_attention_host": (I, [P, P, P] + geo + [I, I, F, F, P, P]),
        "rf_read_status": (I, [P, Z, I, I, I, ctypes.POINTER(RfPlan), ctypes.POINTER(I), P]),
        "rf_block_mask_noalloc": (I, [P, P] + geo + [I, I, F, P, P, P, P]),
        "rf_debug_set_wait": (I, [ctypes.c_longlong, I]),
        "rf_debug_set_path": (I, [I, F]),
        "rf_debug_set_stage_event": (I, [P]),
        "rf_read_stats": (I, [P, Z, I, I, I, ctypes.POINTER(RfPlan), ctypes.POINTER(RfStats), P]),
        "rf_read_stats_ex": (I, [I, P, Z, I, I, I, ctypes.POINTER(RfPlan), ctypes.POINTER(RfPlan),
                                 ctypes.POINTER(RfStats), P]),
        "rf_debug_exp2_poly": (I, [P, P, I, P]),
        "rf_last_error_string": (ctypes.c_char_p, []),
        "rf_plan_kv": (I, [I, I, I, I, I, I, I, I, I, I, F, ctypes.POINTER(RfPlan), ctypes.POINTER(RfPlan)]),
        "rf_workspace_layout_ex": (I, [I, I, I, I, ctypes.POINTER(RfPlan), ctypes.POINTER(RfPlan),
                                       ctypes.POINTER(RfWsLayout)]),
        "rf_workspace_size_ex": (Z, [I, I, I, I, I, I, I, I, I, I, I, I, I]),
        "rf_prepare_ex": (I, [P, P, P, I, I] + geo + [I, I, I, I, I, I, F, P, Z, P]),
        "rf_attend_ex": (I, [I, I] + geo + [I, I, I, I, I, I, F, F, P, P, Z, P]),
        "rf_sparse_attention_ex": (I, [P, P, P, I, I] + geo + [I, I, I, I, I, I, F, F, P, P, Z, P]),
        "rf_sparse_attention_host_ex": (I, [P, P, P, I, I] + geo + [I, I, I, I, I, I, F, F, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()


def _check(code: int):
    if code != 0:
        raise RfError(code, LIB.rf_last_error_string().decode())


def _dims(x, layout: str):
    if layout == "BSND":
        B, S, N, D = x.shape
    elif layout == "BNSD":
        B, N, S, D = x.shape
    else:
        raise RfError(1, "input layout must be BSND or BNSD")
    return B, S, N, D


def _check_tensors(layout: str, q, k=None, v=None, out=None, same_kv_len: bool = True, host: bool = False):
    """Checks, before any call into the library, what the C ABI cannot see
    from bare pointers: every tensor is a contiguous torch tensor of bf16 or
    fp16 (all of one type) on one CUDA device (host: in CPU memory); k and v
    have one shape, with q's batch, heads and head dim (and q's length unless
    k and v have a geometry of their own); out has q's shape.  Raises
    RfError(RF_ERR_ARG)."""
    dims = _dims(q, layout)
    tensors = [("q", q), ("k", k), ("v", v), ("out", out)]
    tensors = [(n, t) for n, t in tensors if t is not None]
    for name, t in tensors:
        if t.dim() != 4:
            raise RfError(2, f"{name} must have 4 dims ({layout}), got {tuple(t.shape)}")
        if t.dtype != q.dtype:
            raise RfError(2, f"{name} is {t.dtype}, q is {q.dtype}")
    _dtype(q)
    if k is not None and v is not None and k.shape != v.shape:
        raise RfError(2, f"k {tuple(k.shape)} and v {tuple(v.shape)} differ in shape")
    if k is not None:
        kd = _dims(k, layout)
        if (kd[0], kd[2], kd[3]) != (dims[0], dims[2], dims[3]) or (same_kv_len and kd[1] != dims[1]):
            raise RfError(2, f"k {tuple(k.shape)} does not match q {tuple(q.shape)} ({layout})")
    if out is not None and out.shape != q.shape:
        raise RfError(2, f"out {tuple(out.shape)} must have q's shape {tuple(q.shape)}")
    for name, t in tensors:
        if not t.is_contiguous():
            raise RfError(2, f"{name} must be contiguous")
    for name, t in tensors:
        if host and t.device.type != "cpu":
            raise RfError(2, f"{name} must be a CPU tensor, got {t.device}")
        if not host and (not t.is_cuda or t.device != q.device):
            raise RfError(2, f"{name} must be a CUDA tensor on q's device ({q.device}), got {t.device}")


def _stream(x, stream):
    if stream is not None:
        return ctypes.c_void_p(stream)
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream(x.device).cuda_stream)


def _ptr(x):
    return ctypes.c_void_p(x.data_ptr()) if x is not None else None


def _scale(scale):
    return float("nan") if scale is None else float(scale)


def _dtype(x) -> int:
    import torch
    if x.dtype == torch.bfloat16:
        return RF_BF16
    if x.dtype == torch.float16:
        return RF_F16
    raise RfError(2, f"q, k, v must be bfloat16 or float16 (got {x.dtype})")


def _prec(precision: str) -> int:
    if precision not in PRECISIONS:
        raise RfError(2, f"precision must be one of {sorted(PRECISIONS)}")
    return PRECISIONS[precision]


def _plain(x, precision: str) -> bool:
    """bf16 at native precision goes through the plain entry points."""
    return _dtype(x) == RF_BF16 and _prec(precision) == 0


def _nbytes(t):
    return t.numel() * t.element_size()


def _kv(k, layout: str, latent_k):
    """(S_kv, kv_t, kv_h, kv_w) of the _ex entry points: zeros when k and v share q's geometry."""
    if latent_k is None:
        return (0, 0, 0, 0)
    return (_dims(k, layout)[1], *latent_k)


def rf_plan(S: int, txt_len: int, latent, sparsity: float, block_size: int = 128) -> RfPlan:
    p = RfPlan()
    _check(LIB.rf_plan(S, txt_len, *latent, block_size, float(sparsity), ctypes.byref(p)))
    return p


def rf_plan_kv(S: int, txt_len: int, latent, S_kv: int, latent_k, sparsity: float, block_size: int = 128):
    """(query plan, key/value plan) of a call whose k and v have a geometry of their own."""
    p, pk = RfPlan(), RfPlan()
    _check(LIB.rf_plan_kv(S, txt_len, *latent, S_kv, *latent_k, block_size, float(sparsity), ctypes.byref(p),
                          ctypes.byref(pk)))
    return p, pk


def rf_workspace_layout(B: int, N: int, D: int, plan: RfPlan, precision: str = "native",
                        plan_kv: RfPlan | None = None) -> RfWsLayout:
    lay = RfWsLayout()
    if precision == "native" and plan_kv is None:
        _check(LIB.rf_workspace_layout(B, N, D, ctypes.byref(plan), ctypes.byref(lay)))
    else:
        _check(LIB.rf_workspace_layout_ex(_prec(precision), B, N, D, ctypes.byref(plan),
                                          ctypes.byref(plan_kv) if plan_kv is not None else None, ctypes.byref(lay)))
    return lay


def rf_workspace_size(B, S, N, D, txt_len, latent, precision: str = "native", S_kv: int = 0, latent_k=None) -> int:
    if precision == "native" and latent_k is None:
        return int(LIB.rf_workspace_size(B, S, N, D, txt_len, *latent))
    kv = (S_kv, *latent_k) if latent_k is not None else (0, 0, 0, 0)
    return int(LIB.rf_workspace_size_ex(_prec(precision), B, S, N, D, txt_len, *latent, *kv))


def rf_sparse_attention(q, k, v, layout: str, txt_len: int, latent, sparsity: float, scale=None, out=None,
                        block_size: int = 128, stream=None, precision: str = "native", latent_k=None):
    """The whole rf_v2 call on device tensors; returns ``out`` (shape, layout and type of q).

    q, k, v: bf16 or fp16; precision "native" or "fp8"; latent_k: the (t, h, w)
    of k and v when they have a geometry of their own (see include/rfsa.h)."""
    import torch
    B, S, N, D = _dims(q, layout)
    if out is None:
        out = torch.empty_like(q)
    _check_tensors(layout, q, k, v, out, same_kv_len=latent_k is None)
    lay = LAYOUTS.get(layout, -1)
    if _plain(q, precision) and latent_k is None:
        _check(LIB.rf_sparse_attention(_ptr(q), _ptr(k), _ptr(v), lay, B, S, N, D, txt_len, *latent, block_size,
                                       float(sparsity), _scale(scale), _ptr(out), _stream(q, stream)))
    else:
        _check(LIB.rf_sparse_attention_ex(_ptr(q), _ptr(k), _ptr(v), _dtype(q), _prec(precision), lay, B, S, N, D,
                                          txt_len, *latent, *_kv(k, layout, latent_k), block_size, float(sparsity),
                                          _scale(scale), _ptr(out), None, 0, _stream(q, stream)))
    return out


def rf_sparse_attention_ws(q, k, v, layout, txt_len, latent, sparsity, workspace, scale=None, out=None,
                           block_size=128, stream=None, precision: str = "native", latent_k=None):
    import torch
    B, S, N, D = _dims(q, layout)
    if out is None:
        out = torch.empty_like(q)
    _check_tensors(layout, q, k, v, out, same_kv_len=latent_k is None)
    lay = LAYOUTS.get(layout, -1)
    if _plain(q, precision) and latent_k is None:
        _check(LIB.rf_sparse_attention_ws(_ptr(q), _ptr(k), _ptr(v), lay, B, S, N, D, txt_len, *latent, block_size,
                                          float(sparsity), _scale(scale), _ptr(out), _ptr(workspace),
                                          _nbytes(workspace), _stream(q, stream)))
    else:
        _check(LIB.rf_sparse_attention_ex(_ptr(q), _ptr(k), _ptr(v), _dtype(q), _prec(precision), lay, B, S, N, D,
                                          txt_len, *latent, *_kv(k, layout, latent_k), block_size, float(sparsity),
                                          _scale(scale), _ptr(out), _ptr(workspace), _nbytes(workspace),
                                          _stream(q, stream)))
    return out


def rf_prepare(q, k, v, layout, txt_len, latent, sparsity, workspace, block_size=128, stream=None,
               precision: str = "native", latent_k=None):
    B, S, N, D = _dims(q, layout)
    _check_tensors(layout, q, k, v, same_kv_len=latent_k is None)
    lay = LAYOUTS.get(layout, -1)
    if _plain(q, precision) and latent_k is None:
        _check(LIB.rf_prepare(_ptr(q), _ptr(k), _ptr(v), lay, B, S, N, D, txt_len, *latent, block_size,
                              float(sparsity), _ptr(workspace), _nbytes(workspace), _stream(q, stream)))
    else:
        _check(LIB.rf_prepare_ex(_ptr(q), _ptr(k), _ptr(v), _dtype(q), _prec(precision), lay, B, S, N, D, txt_len,
                                 *latent, *_kv(k, layout, latent_k), block_size, float(sparsity), _ptr(workspace),
                                 _nbytes(workspace), _stream(q, stream)))


def rf_attend(out, layout, txt_len, latent, sparsity, workspace, scale=None, block_size=128, stream=None,
              precision: str = "native", S_kv: int = 0, latent_k=None):
    B, S, N, D = _dims(out, layout)
    _check_tensors(layout, out)
    lay = LAYOUTS.get(layout, -1)
    kv = (S_kv, *latent_k) if latent_k is not None else (0, 0, 0, 0)
    if _plain(out, precision) and latent_k is None:
        _check(LIB.rf_attend(lay, B, S, N, D, txt_len, *latent, block_size, float(sparsity), _scale(scale),
                             _ptr(out), _ptr(workspace), _nbytes(workspace), _stream(out, stream)))
    else:
        _check(LIB.rf_attend_ex(_dtype(out), _prec(precision), lay, B, S, N, D, txt_len, *latent, *kv, block_size,
                                float(sparsity), _scale(scale), _ptr(out), _ptr(workspace), _nbytes(workspace),
                                _stream(out, stream)))
    return out


def rf_unpermute(o_int, out, layout, txt_len, latent, stream=None):
    B, S, N, D = _dims(out, layout)
    _check_tensors(layout, out)
    if o_int.dtype != out.dtype or not o_int.is_contiguous() or not o_int.is_cuda:
        raise RfError(2, "o_int must be a contiguous CUDA tensor of out's type")
    plan = rf_plan(S, txt_len, latent, 0.0)
    if o_int.numel() < B * N * plan.S_int * D:
        raise RfError(2, f"o_int holds {o_int.numel()} values, the internal layout needs {B * N * plan.S_int * D}")
    _check(LIB.rf_unpermute(_ptr(o_int), LAYOUTS.get(layout, -1), B, S, N, D, txt_len, *latent, _ptr(out),
                            _stream(out, stream)))
    return out


def rf_sparse_attention_host(q, k, v, layout, txt_len, latent, sparsity, out, scale=None, block_size=128,
                             stream=None, precision: str = "native", latent_k=None):
    """The whole call through host buffers: q, k, v, out are contiguous CPU
    (ideally pinned) tensors of one 16-bit type, out shaped like q; the
    copies to and from the device happen inside the library."""
    import torch
    B, S, N, D = _dims(q, layout)
    if out is None:
        raise RfError(2, "out must be a CPU tensor shaped like q")
    _check_tensors(layout, q, k, v, out, same_kv_len=latent_k is None, host=True)
    st = ctypes.c_void_p(stream if stream is not None else torch.cuda.current_stream().cuda_stream)
    lay = LAYOUTS.get(layout, -1)
    if _plain(q, precision) and latent_k is None:
        _check(LIB.rf_sparse_attention_host(_ptr(q), _ptr(k), _ptr(v), lay, B, S, N, D, txt_len, *latent,
                                            block_size, float(sparsity), _scale(scale), _ptr(out), st))
    else:
        _check(LIB.rf_sparse_attention_host_ex(_ptr(q), _ptr(k), _ptr(v), _dtype(q), _prec(precision), lay, B, S, N,
                                               D, txt_len, *latent, *_kv(k, layout, latent_k), block_size,
                                               float(sparsity), _scale(scale), _ptr(out), st))
    return out


def rf_block_mask_noalloc(q, k, layout, txt_len, latent, sparsity, mask, kept, margin, block_size=128,
                          stream=None):
    """Block mask into caller buffers, with no device allocation (see include/rfsa.h).

    mask: int32 or uint32 [B, N, nb, ceil(nb / 32)], kept: int32 [B, N, nb],
    margin: float32 [B, N, nb], contiguous CUDA tensors (checked here: the
    library sees only their addresses)."""
    import torch
    B, S, N, D = _dims(q, layout)
    _check_tensors(layout, q, k)
    plan = rf_plan(S, txt_len, latent, float(sparsity), block_size)
    rows = B * N * plan.nb
    for name, t, n, types in (("mask", mask, rows * plan.mask_words, (torch.int32, torch.uint32)),
                              ("kept", kept, rows, (torch.int32,)), ("margin", margin, rows, (torch.float32,))):
        if t.dtype not in types or not t.is_contiguous() or not t.is_cuda or t.numel() < n:
            raise RfError(2, f"{name} must be a contiguous CUDA {types[0]} tensor of at least {n} values")
    _check(LIB.rf_block_mask_noalloc(_ptr(q), _ptr(k), LAYOUTS.get(layout, -1), B, S, N, D, txt_len, *latent,
                                     block_size, float(sparsity), _ptr(mask), _ptr(kept), _ptr(margin),
                                     _stream(q, stream)))


def sparse_attention(q, k, v, attn_mask=None, scale=None, is_causal=False, head_num=1, input_layout="BNSD",
                     inner_precise=0, sparse_type=None, txt_len=0, block_size=128, latent_shape_q=None,
                     latent_shape_k=None, keep_sink=True, keep_recent=True, cdf_threshold=1.0, sparsity=0.0,
                     **_kwargs):
    """The operation under the parameter list of MindSpore Lite's
    ``lite_boost.ops.sparse_attention`` (argument checks and marshalling
    only; the call is ``rf_sparse_attention``).

    - ``sparse_type=None``: dense softmax attention over the whole sequence;
      ``"rf_v2"``: block-sparse (token reorder, block pooling, top-k mask,
      attention, inverse reorder) with ``latent_shape_q`` (required) and
      ``latent_shape_k`` (default: the query's).  Any other value raises
      ValueError, as does an ``input_layout`` other than "BSND" / "BNSD"
      (the page's "Raises").
    - ``head_num`` must equal the tensors' head dimension.
    - ``scale`` None means head_dim ** -0.5.  ``sparsity`` in [0, 1].
    - ``attn_mask`` is reserved on the page and unused by rf_v2; ``keep_sink``,
      ``keep_recent`` and ``cdf_threshold`` belong to another mode and are
      not read; ``inner_precise`` selects nothing here (the arithmetic is
      the precision the inputs give).  A causal mask (``is_causal=True``) is
      not implemented and raises NotImplementedError.
    Returns the output, shaped like q."""
    if input_layout not in LAYOUTS:
        raise ValueError(f'input_layout must be "BSND" or "BNSD" (got {input_layout!r})')
    if sparse_type not in (None, "rf_v2"):
        raise ValueError(f'sparse_type must be None or "rf_v2" (got {sparse_type!r})')
    if is_causal:
        raise NotImplementedError("causal attention is not implemented")
    B, S, N, D = _dims(q, input_layout)
    if head_num != N:
        raise ValueError(f"head_num {head_num} does not match the tensors' {N} heads")
    if sparse_type is None:
        return rf_sparse_attention(q, k, v, input_layout, 0, (0, 0, 0), 0.0, scale=scale, block_size=block_size)
    if latent_shape_q is None:
        raise ValueError("the rf_v2 path needs latent_shape_q (t, h, w)")
    latent = tuple(int(x) for x in latent_shape_q)
    latent_k = None if latent_shape_k is None else tuple(int(x) for x in latent_shape_k)
    if latent_k == latent:
        latent_k = None
    return rf_sparse_attention(q, k, v, input_layout, int(txt_len), latent, float(sparsity), scale=scale,
                               block_size=int(block_size), latent_k=latent_k)


def rf_debug_set_wait(wait_limit_ns: int = 0, skip_first_q: int = 0):
    """Test control of the attention kernel's bounded waits (see include/rfsa.h)."""
    _check(LIB.rf_debug_set_wait(int(wait_limit_ns), int(skip_first_q)))


def rf_debug_set_path(path: int = 0, sum_limit: float = 0.0):
    """Test control of the attention path (see include/rfsa.h)."""
    _check(LIB.rf_debug_set_path(int(path), float(sum_limit)))


def rf_debug_set_stage_event(event=None):
    """While set, rf_prepare records ``event`` (a torch.cuda.Event that has been
    recorded once, so that its CUDA event exists) between K1 and the kernels
    after it; None clears the hook.  The caller keeps the event alive while it
    is set (see include/rfsa.h)."""
    handle = None
    if event is not None:
        handle = int(event.cuda_event)
        if not handle:
            raise ValueError("the event has no CUDA event yet: record it once first")
    _check(LIB.rf_debug_set_stage_event(ctypes.c_void_p(handle)))


def rf_read_status(workspace, B, N, D, plan, stream=None) -> int:
    st = ctypes.c_int(0)
    _check(LIB.rf_read_status(_ptr(workspace), workspace.numel() * workspace.element_size(), B, N, D,
                              ctypes.byref(plan), ctypes.byref(st), _stream(workspace, stream)))
    return st.value


def rf_read_stats(workspace, B, N, D, plan, stream=None, precision: str = "native", plan_kv=None) -> dict:
    """Statistics of the last call on a workspace (see include/rfsa.h)."""
    st = RfStats()
    if precision == "native" and plan_kv is None:
        _check(LIB.rf_read_stats(_ptr(workspace), workspace.numel() * workspace.element_size(), B, N, D,
                                 ctypes.byref(plan), ctypes.byref(st), _stream(workspace, stream)))
    else:
        _check(LIB.rf_read_stats_ex(_prec(precision), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    B, N, D, ctypes.byref(plan), ctypes.byref(plan_kv) if plan_kv is not None else None,
                                    ctypes.byref(st), _stream(workspace, stream)))
    return st.as_dict()


def rf_debug_exp2_poly(x, y=None, stream=None):
    """y = 2^x by the attention's FMA-pipe exponential (see include/rfsa.h);
    x, y: contiguous fp32 CUDA tensors of one size."""
    import torch
    if y is None:
        y = torch.empty_like(x)
    if x.dtype != torch.float32 or y.dtype != torch.float32 or x.numel() != y.numel():
        raise RfError(2, "x and y must be fp32 tensors of one size")
    if not (x.is_contiguous() and y.is_contiguous() and x.is_cuda and y.is_cuda):
        raise RfError(2, "x and y must be contiguous CUDA tensors")
    _check(LIB.rf_debug_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream(x, stream)))
    return y


def workspace_views(workspace, B, N, plan, dtype=None, precision: str = "native", plan_kv=None):
    """Typed torch views of the workspace regions (for inspection and tests).

    dtype: torch type of the internal q/k/v copies (the input type; default bf16).
    plan_kv: the key/value plan when k and v have a geometry of their own."""
    import torch
    dtype = dtype or torch.bfloat16
    lay = rf_workspace_layout(B, N, 128, plan, precision, plan_kv)
    pk = plan if plan_kv is None else plan_kv
    raw = workspace.view(torch.uint8)
    heads = B * N

    def view(off, count, dtype, shape):
        nbytes = count * torch.empty((), dtype=dtype).element_size()
        return raw[off:off + nbytes].view(dtype).view(shape)

    nb, nbk, words = plan.nb, pk.nb, pk.mask_words
    if precision == "fp8":
        nq, nk = plan.n_tiles, pk.n_tiles
        copies = {
            "q8": view(lay.q8, heads * plan.S_int * 128, torch.uint8, (B, N, plan.S_int, 128)),
            "k8": view(lay.k8, heads * pk.S_int * 128, torch.uint8, (B, N, pk.S_int, 128)),
            "v8": view(lay.v8, heads * pk.S_int * 128, torch.uint8, (B, N, nk, 128, 128)),
            "q_scales": view(lay.scales, heads * nq, torch.float32, (B, N, nq)),
            "k_scales": view(lay.scales + 4 * heads * nq, heads * nk, torch.float32, (B, N, nk)),
            "v_scales": view(lay.scales + 4 * heads * (nq + nk), heads * nk, torch.float32, (B, N, nk)),
            "vmax": view(lay.vmax, heads, torch.float32, (B, N)),
        }
    else:   # the 16-bit internal copies exist at native precision only
        copies = {
            "q_int": view(lay.q_int, heads * plan.S_int * 128, dtype, (B, N, plan.S_int, 128)),
            "k_int": view(lay.k_int, heads * pk.S_int * 128, dtype, (B, N, pk.S_int, 128)),
            "v_int": view(lay.v_int, heads * pk.S_int * 128, dtype, (B, N, pk.S_int, 128)),
        }
    return copies | {
        "pooled_q": view(lay.pooled_q, heads * nb * 128, torch.float32, (B, N, nb, 128)),
        "pooled_k": view(lay.pooled_k, heads * nbk * 128, torch.float32, (B, N, nbk, 128)),
        "mask": view(lay.mask, heads * nb * words, torch.int32, (B, N, nb, words)),
        "kept": view(lay.kept, heads * nb, torch.int32, (B, N, nb)),
        "margin": view(lay.margin, heads * nb, torch.float32, (B, N, nb)),
    } | {"redo": view(lay.redo, 2 + heads * plan.n_tiles, torch.int32, (2 + heads * plan.n_tiles,))}


def alloc_workspace(B, S, N, D, txt_len, latent, device="cuda", precision: str = "native", S_kv: int = 0,
                    latent_k=None):
    import torch
    n = rf_workspace_size(B, S, N, D, txt_len, latent, precision, S_kv, latent_k)
    if n == 0:
        raise RfError(2, "bad arguments for the workspace size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def kept_block_flops(plan: RfPlan, kept, B: int, N: int, D: int = 128) -> float:
    """Algorithmic FLOPs of one call: 4 * D * sum over query rows of |key set|.

    Dense rows (prefix, first-frame blocks, or everything in the dense
    fallback) read all S keys; a sparse block's 128 rows read the P prefix
    keys plus 128 per kept block.  ``kept`` is the per-row kept-count tensor
    (B, N, nb) from the workspace.
    """
    S = plan.S
    if plan.dense:
        return 4.0 * D * B * N * S * S
    dense_rows = plan.P + 128 * plan.ff
    sparse_keys = kept[..., plan.ff:].double().sum().item() * 128.0 + (plan.nb - plan.ff) * B * N * plan.P
    return 4.0 * D * (B * N * dense_rows * S + 128.0 * sparse_keys)


def default_scale(D: int = 128) -> float:
    return 1.0 / math.sqrt(D)
