"""ctypes binding of libsparseattn.so (C ABI in include/sparse_attn.h).

Argument marshalling only: every function below packs its arguments into the
C structs and calls the entry point of the same name; all computation runs in
the library's CUDA kernels.  Tensors are torch CUDA tensors (PyTorch provides
device memory and streams).  If the library is missing, loading fails with
an error that says how to build it: there is no other implementation.

``Pipeline`` strings the calls of one forward pass together (layout ->
reorder -> mask prediction -> block-sparse attention -> inverse reorder) and
owns the buffers it allocates through torch.
"""

from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsparseattn.so")

SA_OK, SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_WORKSPACE = 0, 1, 2, 3
SA_ERR_EMPTY_ROW, SA_ERR_TIMEOUT, SA_ERR_CUDA, SA_ERR_CAPACITY = 4, 5, 6, 7
SA_BF16, SA_FP32 = 0, 1
SA_ORDER = {"identity": 0, "window": 1, "hilbert": 2}
SA_FLAG_FORCE_SIMT = 1

STATUS_NAMES = {0: "SA_OK", 1: "SA_ERR_INVALID_ARG", 2: "SA_ERR_UNSUPPORTED", 3: "SA_ERR_WORKSPACE",
                4: "SA_ERR_EMPTY_ROW", 5: "SA_ERR_TIMEOUT", 6: "SA_ERR_CUDA", 7: "SA_ERR_CAPACITY"}

EXPORTS = ["sa_version", "sa_last_error", "sa_attn_kernel_path", "sa_attn_workspace", "sa_layout_workspace",
           "sa_layout_build", "sa_reorder", "sa_unreorder", "sa_predict_mask_workspace",
           "sa_predict_mask_ws_layout", "sa_order_group_hint", "sa_predict_mask", "sa_reorder_predict_mask",
           "sa_predict_mask_noalloc",
           "sa_mask_from_blocks_workspace",
           "sa_mask_from_blocks", "sa_block_sparse_attn", "sa_dense_attn", "sa_read_status", "sa_l1_error",
           "sa_head_placement", "sa_reorder_heads", "sa_rows_attn", "sa_rows_mse",
           "sa_quantize_blocks", "sa_attn_qk8_workspace", "sa_block_sparse_attn_qk8",
           "sa_reorder_predict_mask_q8", "sa_forward_host_workspace", "sa_forward_host"]


class SAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("Hq", ctypes.c_int64), ("Hkv", ctypes.c_int64),
                ("N", ctypes.c_int64), ("d", ctypes.c_int64), ("dv", ctypes.c_int64),
                ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class LayoutDesc(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int64), ("W", ctypes.c_int64),
                ("txt_len", ctypes.c_int64), ("sink_frames", ctypes.c_int64),
                ("win", ctypes.c_int64 * 3), ("mode", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class MaskParams(ctypes.Structure):
    _fields_ = [("bq", ctypes.c_int32), ("bk", ctypes.c_int32), ("tau", ctypes.c_float),
                ("theta", ctypes.c_float), ("sink_tokens", ctypes.c_int64),
                ("txt_len", ctypes.c_int64), ("local_window", ctypes.c_int64),
                ("anchor_tokens", ctypes.c_int64), ("causal", ctypes.c_int32),
                ("order_group", ctypes.c_int32)]


class Mask(ctypes.Structure):
    _fields_ = [("block_mask", ctypes.c_void_p), ("row_ptr", ctypes.c_void_p),
                ("col_idx", ctypes.c_void_p), ("order", ctypes.c_void_p),
                ("kept_total", ctypes.c_void_p), ("status", ctypes.c_void_p),
                ("col_capacity", ctypes.c_int64), ("nqb", ctypes.c_int64), ("nkb", ctypes.c_int64),
                ("bq", ctypes.c_int32), ("bk", ctypes.c_int32), ("causal", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} not found: build it with `python -m long_context_mean_b200.build` "
                           "(there is no fallback implementation)")
    lib = ctypes.CDLL(path)
    P, I32, I64, SZ, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    sig = {
        "sa_version": (ctypes.c_char_p, []),
        "sa_last_error": (ctypes.c_char_p, []),
        "sa_attn_kernel_path": (I32, [ctypes.POINTER(Shape), I32, I32, I32]),
        "sa_layout_workspace": (SZ, [ctypes.POINTER(LayoutDesc)]),
        "sa_layout_build": (I32, [ctypes.POINTER(LayoutDesc), P, P, P, SZ, P]),
        "sa_reorder": (I32, [P, P, P, I64, I64, I64, I32, P]),
        "sa_unreorder": (I32, [P, P, P, I64, I64, I64, I32, P]),
        "sa_predict_mask_workspace": (SZ, [ctypes.POINTER(Shape), ctypes.POINTER(MaskParams)]),
        "sa_predict_mask_ws_layout": (I32, [ctypes.POINTER(Shape), ctypes.POINTER(MaskParams),
                                            ctypes.POINTER(SZ * 6)]),
        "sa_order_group_hint": (I32, [ctypes.POINTER(Shape)]),
        "sa_predict_mask": (I32, [P, P, ctypes.POINTER(Shape), ctypes.POINTER(MaskParams), P, SZ,
                                  ctypes.POINTER(Mask), P]),
        "sa_reorder_predict_mask": (I32, [P, P, P, P, P, ctypes.POINTER(Shape), ctypes.POINTER(MaskParams), P,
                                          SZ, ctypes.POINTER(Mask), P]),
        "sa_predict_mask_noalloc": (I32, [P, P, ctypes.POINTER(Shape), ctypes.POINTER(MaskParams),
                                          ctypes.POINTER(Mask), P]),
        "sa_mask_from_blocks_workspace": (SZ, [ctypes.POINTER(Shape), I32, I32]),
        "sa_mask_from_blocks": (I32, [P, ctypes.POINTER(Shape), I32, I32, I32, P, SZ,
                                      ctypes.POINTER(Mask), P]),
        "sa_attn_workspace": (SZ, []),
        "sa_l1_error": (I32, [P, P, I64, I32, P, P]),
        "sa_head_placement": (I32, [I64, I64, I64, I64, P, I64, I32, I32, P, P, P, P]),
        "sa_reorder_heads": (I32, [P, P, P, I64, I64, I64, I32, P]),
        "sa_quantize_blocks": (I32, [P, I64, I64, I64, I32, I32, I32, P, P, P]),
        "sa_attn_qk8_workspace": (SZ, [ctypes.POINTER(Mask)]),
        "sa_reorder_predict_mask_q8": (I32, [P, P, P, I32, P, P, P, P, ctypes.POINTER(Shape),
                                             ctypes.POINTER(MaskParams), P, SZ, ctypes.POINTER(Mask), P]),
        "sa_block_sparse_attn_qk8": (I32, [P, P, P, P, I32, P, ctypes.POINTER(Shape), ctypes.POINTER(Mask), F,
                                           F, P, P, P, P, P, SZ, I32, P]),
        "sa_rows_mse": (I32, [P, P, P, I64, I64, I64, I64, I32, P, P, P]),
        "sa_rows_attn": (I32, [P, P, P, ctypes.POINTER(Shape), P, I64, P, P, I32, I32, F, P, P, P, P]),
        "sa_block_sparse_attn": (I32, [P, P, P, ctypes.POINTER(Shape), ctypes.POINTER(Mask), F, F,
                                       P, P, P, P, P, SZ, I32, P]),
        "sa_dense_attn": (I32, [P, P, P, ctypes.POINTER(Shape), I32, F, P, P, P, P, SZ, I32, P]),
        "sa_read_status": (I32, [P, P]),
        "sa_forward_host_workspace": (SZ, [ctypes.POINTER(Shape), ctypes.POINTER(LayoutDesc),
                                           ctypes.POINTER(MaskParams), I32]),
        "sa_forward_host": (I32, [P, P, P, P, P, ctypes.POINTER(Shape), ctypes.POINTER(LayoutDesc),
                                  ctypes.POINTER(MaskParams), F, F, I32, P, SZ, P, ctypes.POINTER(P * 3)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(code: int):
    if code != SA_OK:
        raise SAError(code, load().sa_last_error().decode(errors="replace"))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return SA_BF16
    if t.dtype == torch.float32:
        return SA_FP32
    raise ValueError(f"unsupported dtype {t.dtype}")


def make_shape(q, k, v) -> Shape:
    B, Hq, N, d = q.shape
    return Shape(B, Hq, k.shape[1], N, d, v.shape[3], dtype_code(q), 0)


def make_layout(T, H, W, txt_len=0, sink_frames=0, mode="identity", win=(1, 1, 1)) -> LayoutDesc:
    w = (ctypes.c_int64 * 3)(*[int(x) for x in win])
    return LayoutDesc(int(T), int(H), int(W), int(txt_len), int(sink_frames), w, SA_ORDER[mode], 0)


def make_params(bq, bk, tau, theta=0.0, sink_tokens=0, txt_len=0, local_window=0,
                anchor_tokens=0, causal=False, order_group=0) -> MaskParams:
    return MaskParams(int(bq), int(bk), float(tau), float(theta), int(sink_tokens), int(txt_len),
                      int(local_window), int(anchor_tokens), int(bool(causal)), int(order_group))


# ---------------------------------------------------------------------------
# Thin wrappers (one per entry point)
# ---------------------------------------------------------------------------

def version() -> str:
    return load().sa_version().decode()


def attn_kernel_path(shape: Shape, bq: int, bk: int, flags: int = 0) -> int:
    return int(load().sa_attn_kernel_path(ctypes.byref(shape), bq, bk, flags))


def layout_workspace(desc: LayoutDesc) -> int:
    return int(load().sa_layout_workspace(ctypes.byref(desc)))


def layout_build(desc: LayoutDesc, perm, inv, ws=None, stream=None):
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(load().sa_layout_build(ctypes.byref(desc), _ptr(perm), _ptr(inv), _ptr(ws), nbytes,
                                  _stream(stream)))


def reorder(perm, x, y, stream=None):
    """y[..., n, :] = x[..., perm[n], :] for x of shape [..., N, row]."""
    N, row = x.shape[-2], x.shape[-1]
    outer = x.numel() // (N * row)
    _check(load().sa_reorder(_ptr(perm), _ptr(x), _ptr(y), outer, N, row, dtype_code(x), _stream(stream)))


def unreorder(perm, y, x, stream=None):
    """x[..., perm[n], :] = y[..., n, :]."""
    N, row = y.shape[-2], y.shape[-1]
    outer = y.numel() // (N * row)
    _check(load().sa_unreorder(_ptr(perm), _ptr(y), _ptr(x), outer, N, row, dtype_code(y), _stream(stream)))


def predict_mask_workspace(shape: Shape, params: MaskParams) -> int:
    return int(load().sa_predict_mask_workspace(ctypes.byref(shape), ctypes.byref(params)))


def predict_mask_ws_layout(shape: Shape, params: MaskParams):
    off = (ctypes.c_size_t * 6)()
    _check(load().sa_predict_mask_ws_layout(ctypes.byref(shape), ctypes.byref(params), ctypes.byref(off)))
    return list(off)


def order_group_hint(shape: Shape) -> int:
    """The library's work-order grouping for a shape (MaskParams.order_group)."""
    g = int(load().sa_order_group_hint(ctypes.byref(shape)))
    if g < 0:
        raise SAError(SA_ERR_INVALID_ARG, "sa_order_group_hint: invalid shape")
    return g


def predict_mask(q, k, shape: Shape, params: MaskParams, ws, mask: Mask, stream=None):
    _check(load().sa_predict_mask(_ptr(q), _ptr(k), ctypes.byref(shape), ctypes.byref(params), _ptr(ws),
                                  ws.numel() * ws.element_size(), ctypes.byref(mask), _stream(stream)))


def reorder_predict_mask(perm, q, k, q_r, k_r, shape: Shape, params: MaskParams, ws, mask: Mask, stream=None):
    """Mask prediction on the permuted sequence with q, k in the original order;
    writes the reordered copies q_r, k_r in the same pass."""
    _check(load().sa_reorder_predict_mask(_ptr(perm), _ptr(q), _ptr(k), _ptr(q_r), _ptr(k_r), ctypes.byref(shape),
                                          ctypes.byref(params), _ptr(ws), ws.numel() * ws.element_size(),
                                          ctypes.byref(mask), _stream(stream)))


def predict_mask_noalloc(q, k, shape: Shape, params: MaskParams, mask: Mask, stream=None):
    """sa_predict_mask with the library's own fixed scratch array (no workspace argument)."""
    _check(load().sa_predict_mask_noalloc(_ptr(q), _ptr(k), ctypes.byref(shape), ctypes.byref(params),
                                          ctypes.byref(mask), _stream(stream)))


def mask_from_blocks_workspace(shape: Shape, bq: int, bk: int) -> int:
    return int(load().sa_mask_from_blocks_workspace(ctypes.byref(shape), bq, bk))


def mask_from_blocks(block_mask, shape: Shape, bq, bk, causal, ws, mask: Mask, stream=None):
    _check(load().sa_mask_from_blocks(_ptr(block_mask), ctypes.byref(shape), bq, bk, int(bool(causal)),
                                      _ptr(ws), ws.numel() * ws.element_size(), ctypes.byref(mask),
                                      _stream(stream)))


def attn_workspace() -> int:
    return int(load().sa_attn_workspace())


_attn_ws = {}


def _default_attn_ws(device):
    """A per-device attention workspace for callers that pass none (calls on
    one device then share it, so they must not overlap on the GPU)."""
    import torch
    key = str(device)
    if key not in _attn_ws:
        _attn_ws[key] = workspace(attn_workspace(), device)
    return _attn_ws[key]


def block_sparse_attn(q, k, v, shape: Shape, mask: Mask, lam, scale, out, lse=None, skip_log=None,
                      flags=0, stream=None, ws=None, out_perm=None):
    ws = ws if ws is not None else _default_attn_ws(q.device)
    _check(load().sa_block_sparse_attn(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(shape), ctypes.byref(mask),
                                       float(lam), float(scale), _ptr(out), _ptr(lse), _ptr(out_perm),
                                       _ptr(skip_log),
                                       _ptr(ws), ws.numel() * ws.element_size(), int(flags),
                                       _stream(stream)))


SA_Q_INT8, SA_Q_E4M3 = 0, 1
Q_FORMATS = {"int8": SA_Q_INT8, "e4m3": SA_Q_E4M3}


def quantize_blocks(x, rows, x8, scales, fmt="int8", stream=None):
    """Per-block 8-bit codes x8 ("int8" or "e4m3") and scales of a bf16
    [..., N, d] tensor, one scale per `rows` tokens of each head."""
    N, d = x.shape[-2], x.shape[-1]
    heads = x.numel() // (N * d)
    _check(load().sa_quantize_blocks(_ptr(x), heads, N, d, rows, dtype_code(x), Q_FORMATS[fmt], _ptr(x8),
                                     _ptr(scales), _stream(stream)))


def reorder_predict_mask_q8(perm, q, k, fmt, q8, q_scales, k8, k_scales, shape: Shape, params: MaskParams, ws,
                            mask: Mask, stream=None):
    """Mask prediction whose pooling pass writes the reordered 8-bit codes
    and block scales of Q and K (perm None: the original order)."""
    _check(load().sa_reorder_predict_mask_q8(_ptr(perm), _ptr(q), _ptr(k), Q_FORMATS[fmt], _ptr(q8), _ptr(q_scales),
                                             _ptr(k8), _ptr(k_scales), ctypes.byref(shape), ctypes.byref(params),
                                             _ptr(ws), ws.numel() * ws.element_size(), ctypes.byref(mask),
                                             _stream(stream)))


def attn_qk8_workspace(mask: Mask) -> int:
    return int(load().sa_attn_qk8_workspace(ctypes.byref(mask)))


def block_sparse_attn_qk8(q8, q_scales, k8, k_scales, v, shape: Shape, mask: Mask, lam, scale, out, ws, lse=None,
                          skip_log=None, flags=0, stream=None, out_perm=None, fmt="int8"):
    _check(load().sa_block_sparse_attn_qk8(_ptr(q8), _ptr(q_scales), _ptr(k8), _ptr(k_scales), Q_FORMATS[fmt],
                                           _ptr(v),
                                           ctypes.byref(shape), ctypes.byref(mask), float(lam), float(scale),
                                           _ptr(out), _ptr(lse), _ptr(out_perm), _ptr(skip_log), _ptr(ws),
                                           ws.numel() * ws.element_size(), int(flags), _stream(stream)))


def dense_attn(q, k, v, shape: Shape, causal, scale, out, lse=None, status=None, flags=0, stream=None,
               ws=None):
    ws = ws if ws is not None else _default_attn_ws(q.device)
    _check(load().sa_dense_attn(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(shape), int(bool(causal)),
                                float(scale), _ptr(out), _ptr(lse), _ptr(status), _ptr(ws),
                                ws.numel() * ws.element_size(), int(flags), _stream(stream)))


def l1_error(ref, x, sums, stream=None):
    """Enqueue sums[0] = sum |ref - x|, sums[1] = sum |ref| (sums: float64
    device tensor of 2)."""
    _check(load().sa_l1_error(_ptr(ref), _ptr(x), ref.numel(), dtype_code(ref), _ptr(sums), _stream(stream)))


SA_HEAD_SPATIAL, SA_HEAD_TEMPORAL = 0, 1


SA_FLAG_OUT_PERM_PER_HEAD = 2
SA_FLAG_TEST_STALL = 4   # testing the timeout path only (see the header)


def head_placement(T, H, W, txt_len, kinds, bq, bk, perms=None, block_mask=None, status=None, stream=None):
    """Per-head orders (perms [heads, N]) and tile covers (block_mask) of the
    spatial / temporal candidates; kinds: int32 device tensor [heads]."""
    _check(load().sa_head_placement(T, H, W, txt_len, _ptr(kinds), kinds.numel(), bq, bk, _ptr(perms),
                                    _ptr(block_mask), _ptr(status), _stream(stream)))


def reorder_heads(perms, x, y, stream=None):
    """y[o, n, :] = x[o, perms[o, n], :] for x of shape [..., N, row]."""
    N, row = x.shape[-2], x.shape[-1]
    outer = x.numel() // (N * row)
    _check(load().sa_reorder_heads(_ptr(perms), _ptr(x), _ptr(y), outer, N, row, dtype_code(x), _stream(stream)))


def rows_attn(q, k, v, shape: Shape, rows, out, lse=None, perms=None, block_mask=None, bq=128, bk=64, scale=0.0,
              status=None, stream=None):
    """Attention of the sampled query rows only: out [B*Hq, nrows, dv] and
    lse [B*Hq, nrows] (float32), over every key or over a candidate's kept
    tiles in each head's order (perms, block_mask from head_placement)."""
    _check(load().sa_rows_attn(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(shape), _ptr(rows), rows.numel(), _ptr(perms),
                               _ptr(block_mask), bq, bk, float(scale), _ptr(out), _ptr(lse), _ptr(status),
                               _stream(stream)))


def rows_mse(ref, x, rows, out, status=None, stream=None):
    """out[h] = mean (ref - x)^2 over the sampled rows of head h; ref/x
    [..., N, dv] device tensors, rows int32 device tensor, out float64 [BH]."""
    N, dv = ref.shape[-2], ref.shape[-1]
    BH = ref.numel() // (N * dv)
    _check(load().sa_rows_mse(_ptr(ref), _ptr(x), _ptr(rows), rows.numel(), BH, N, dv, dtype_code(ref), _ptr(out),
                              _ptr(status), _stream(stream)))


def read_status(status, stream=None) -> int:
    """Synchronises the stream and returns the device status code (no raise)."""
    return int(load().sa_read_status(_ptr(status), _stream(stream)))


# ---------------------------------------------------------------------------
# Buffers and the whole forward path
# ---------------------------------------------------------------------------

@dataclass
class MaskBuffers:
    block_mask: object
    row_ptr: object
    col_idx: object
    order: object
    kept_total: object
    status: object
    struct: Mask

    @classmethod
    def allocate(cls, B, Hq, N, bq, bk, device, capacity=None):
        import torch
        nqb, nkb = -(-N // bq), -(-N // bk)
        R = B * Hq * nqb
        cap = capacity if capacity is not None else R * nkb
        bm = torch.zeros(R * nkb, dtype=torch.uint8, device=device)
        rp = torch.zeros(R + 1, dtype=torch.int32, device=device)
        ci = torch.zeros(max(1, cap), dtype=torch.int32, device=device)
        od = torch.zeros(R, dtype=torch.int32, device=device)
        kt = torch.zeros(1, dtype=torch.int64, device=device)
        st = torch.zeros(1, dtype=torch.int32, device=device)
        m = Mask(bm.data_ptr(), rp.data_ptr(), ci.data_ptr(), od.data_ptr(), kt.data_ptr(), st.data_ptr(),
                 max(1, cap), nqb, nkb, bq, bk, 0, 0)
        return cls(bm, rp, ci, od, kt, st, m)


def workspace(nbytes, device):
    """A 256-byte aligned byte buffer (torch allocations are 512-byte aligned)."""
    import torch
    return torch.empty(max(256, int(nbytes)), dtype=torch.uint8, device=device)


class Pipeline:
    """One forward pass of the block-sparse path for a fixed problem.

    Allocates (through torch) the layout, reordered copies, workspace, mask
    lists and outputs once; ``run(q, k, v)`` then enqueues, on the current
    stream: layout build, mask prediction fused with the reorder of Q and K
    (the reorder of V runs beside it on a side stream), block-sparse
    attention with the inverse reorder of O and LSE fused into its store.  Inputs are BNSD in the original token order;
    ``out``/``lse`` come back in that order too.
    """

    def __init__(self, B, Hq, Hkv, N, d, dv, dtype, *, layout: LayoutDesc, params: MaskParams,
                 lam=-math.inf, scale=0.0, flags=0, device="cuda", log_skips=False, qk8=False):
        import torch
        tdt = torch.bfloat16 if dtype in ("bf16", SA_BF16) else torch.float32
        self.shape = Shape(B, Hq, Hkv, N, d, dv, SA_BF16 if tdt == torch.bfloat16 else SA_FP32, 0)
        self.layout, self.params = layout, params
        self.lam, self.scale, self.flags = lam, scale, flags
        self.identity = layout.mode == SA_ORDER["identity"]
        self.perm = torch.empty(N, dtype=torch.int32, device=device)
        self.inv = torch.empty(N, dtype=torch.int32, device=device)
        self.layout_ws = workspace(layout_workspace(layout), device)
        if not self.identity:
            if not qk8:   # the 8-bit path gets codes from the pooling pass instead
                self.qr = torch.empty(B, Hq, N, d, dtype=tdt, device=device)
                self.kr = torch.empty(B, Hkv, N, d, dtype=tdt, device=device)
            self.vr = torch.empty(B, Hkv, N, dv, dtype=tdt, device=device)
        self.out = torch.empty(B, Hq, N, dv, dtype=tdt, device=device)
        self.lse = torch.empty(B, Hq, N, 1, dtype=torch.float32, device=device)
        self.ws = workspace(predict_mask_workspace(self.shape, params), device)
        self.mask = MaskBuffers.allocate(B, Hq, N, params.bq, params.bk, device)
        # INT8 QK ([P3] 2.4): Q and K quantised per query / key block after
        # the prediction, the attention on the codes.
        self.qk8 = {True: "int8", False: None}.get(qk8, qk8)    # None, "int8" or "e4m3"
        if self.qk8:
            if self.qk8 not in Q_FORMATS:
                raise ValueError(f"qk8 must be one of {sorted(Q_FORMATS)}")
            nqb, nkb = self.mask.struct.nqb, self.mask.struct.nkb
            self.q8 = torch.empty(B, Hq, N, d, dtype=torch.uint8, device=device)
            self.k8 = torch.empty(B, Hkv, N, d, dtype=torch.uint8, device=device)
            self.q_scales = torch.empty(B * Hq * nqb, dtype=torch.float32, device=device)
            self.k_scales = torch.empty(B * Hkv * nkb, dtype=torch.float32, device=device)
            self.attn_ws = workspace(attn_qk8_workspace(self.mask.struct), device)
        else:
            self.attn_ws = workspace(attn_workspace(), device)
        self.skip_log = (torch.zeros(self.mask.col_idx.numel(), dtype=torch.uint8, device=device)
                         if log_skips else None)
        if not self.identity:
            # The V reorder runs on a side stream beside the prediction: both
            # need only the layout, and the prediction's scoring and list
            # kernels leave HBM bandwidth free.
            self.side = torch.cuda.Stream(device=torch.device(device))
            self.ev_layout = torch.cuda.Event()
            self.ev_v = torch.cuda.Event()

    def run(self, q, k, v, stream=None, out=None, lse=None):
        """Enqueue the path on ``stream`` (default: the current stream).
        ``out``/``lse`` (optional) receive the results instead of the
        pipeline's own buffers."""
        out = self.out if out is None else out
        lse = self.lse if lse is None else lse
        if self.identity:
            qr, kr, vr = q, k, v
            if self.qk8:
                self._predict_codes(None, q, k, stream)
            else:
                predict_mask(qr, kr, self.shape, self.params, self.ws, self.mask.struct, stream)
        else:
            import torch
            st = stream if stream is not None else torch.cuda.current_stream(q.device)
            layout_build(self.layout, self.perm, self.inv, self.layout_ws, st)
            # V on the side stream, after the layout (and after everything the
            # caller enqueued before, including the last pass's attention).
            self.ev_layout.record(st)
            self.side.wait_event(self.ev_layout)
            reorder(self.perm, v, self.vr, self.side)
            if not torch.cuda.is_current_stream_capturing():
                v.record_stream(self.side)   # the caller's v stays allocated until the side stream has read it
            self.ev_v.record(self.side)
            # Q and K are reordered (or reordered and quantised) by the
            # pooling pass of the prediction.
            if self.qk8:
                self._predict_codes(self.perm, q, k, st)
            else:
                reorder_predict_mask(self.perm, q, k, self.qr, self.kr, self.shape, self.params, self.ws,
                                     self.mask.struct, st)
            st.wait_event(self.ev_v)
            stream = st
            qr, kr, vr = (None, None, self.vr) if self.qk8 else (self.qr, self.kr, self.vr)
        # The inverse reorder of O and LSE is fused into the attention store
        # (out_perm); sa_unreorder stays available for standalone use.
        out_perm = None if self.identity else self.perm
        if self.qk8:
            block_sparse_attn_qk8(self.q8, self.q_scales, self.k8, self.k_scales, vr, self.shape, self.mask.struct,
                                  self.lam, self.scale, out, self.attn_ws, lse, self.skip_log, self.flags, stream,
                                  out_perm=out_perm, fmt=self.qk8)
        else:
            block_sparse_attn(qr, kr, vr, self.shape, self.mask.struct, self.lam, self.scale, out, lse,
                              self.skip_log, self.flags, stream, ws=self.attn_ws, out_perm=out_perm)
        return out, lse

    def capture(self, q, k, v):
        """Capture ``run(q, k, v)`` into a CUDA graph: the inputs and the
        pipeline's buffers are fixed, so ``replay()`` re-runs the whole path
        (every kernel, the side stream included) with one launch from the
        host.  q, k, v must stay allocated and keep their addresses while the
        graph is used; write new inputs into them in place."""
        import torch
        self.run(q, k, v)              # one-time library setup outside the capture
        torch.cuda.synchronize(q.device)
        self._graph_inputs = (q, k, v)
        self.graph = torch.cuda.CUDAGraph()
        # captured at high priority: the V reorder on the (default-priority)
        # side stream then fills the SM slots the prediction leaves free
        cap = torch.cuda.Stream(device=q.device, priority=torch.cuda.Stream.priority_range()[1])
        with torch.cuda.graph(self.graph, stream=cap, capture_error_mode="relaxed"):
            self.run(q, k, v)
        torch.cuda.synchronize(q.device)
        return self.graph

    def replay(self):
        """Re-run the captured path on the current stream (see ``capture``)."""
        self.graph.replay()
        return self.out, self.lse

    def _predict_codes(self, perm, q, k, stream):
        reorder_predict_mask_q8(perm, q, k, self.qk8, self.q8, self.q_scales, self.k8, self.k_scales, self.shape,
                                self.params, self.ws, self.mask.struct, stream)

    def status(self, stream=None) -> int:
        return read_status(self.mask.status, stream)


class HostPipeline:
    """End-to-end pass from pinned host buffers to pinned host buffers: the
    library's ``sa_forward_host`` (one C call per pass).

    Heads are independent, so the library cuts the problem into ``chunks``
    groups of (batch, head) rows; chunk i's host-to-device copy runs on a
    copy stream, its path on the compute stream and its copy back on a third
    stream, so the copies of one chunk overlap the kernels of its
    neighbours.  The workspace and the two copy streams are allocated here
    once (through torch).  ``run`` only enqueues: the caller waits on
    ``done`` (an event recorded on the compute stream after the call) or
    synchronises.
    """

    def __init__(self, B, Hq, Hkv, N, d, dv, dtype, *, layout: LayoutDesc, params: MaskParams,
                 lam=-math.inf, scale=0.0, flags=0, device="cuda", chunks=4):
        import torch
        if (B * Hkv) % chunks:
            raise ValueError(f"chunks={chunks} must divide the {B * Hkv} kv rows")
        self.device = torch.device(device)
        tdt = torch.bfloat16 if dtype in ("bf16", SA_BF16) else torch.float32
        self.shape = Shape(B, Hq, Hkv, N, d, dv, SA_BF16 if tdt == torch.bfloat16 else SA_FP32, 0)
        self.layout, self.params = layout, params
        self.lam, self.scale, self.chunks = lam, scale, chunks
        nbytes = load().sa_forward_host_workspace(ctypes.byref(self.shape), ctypes.byref(layout),
                                                  ctypes.byref(params), int(chunks))
        if nbytes == 0:
            raise SAError(SA_ERR_INVALID_ARG, load().sa_last_error().decode(errors="replace"))
        self.ws = workspace(nbytes, device)
        self.s_in = torch.cuda.Stream(device=self.device)
        self.s_out = torch.cuda.Stream(device=self.device)
        self.done = torch.cuda.Event()
        self.status_word = torch.zeros(1, dtype=torch.int32, device=device)   # worst status over chunks

    def run(self, q_host, k_host, v_host, out_host, lse_host, stream=None):
        """q_host [B, Hq, N, d], k_host/v_host [B, Hkv, N, d|dv], out_host
        [B, Hq, N, dv], lse_host [B, Hq, N] or [B, Hq, N, 1]: pinned CPU
        tensors.  Work is ordered after ``stream`` (default: current)."""
        import torch
        comp = stream if stream is not None else torch.cuda.current_stream(self.device)
        streams = (ctypes.c_void_p * 3)(comp.cuda_stream, self.s_in.cuda_stream, self.s_out.cuda_stream)
        _check(load().sa_forward_host(_ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(out_host), _ptr(lse_host),
                                      ctypes.byref(self.shape), ctypes.byref(self.layout), ctypes.byref(self.params),
                                      float(self.lam), float(self.scale), int(self.chunks), _ptr(self.ws),
                                      self.ws.numel() * self.ws.element_size(), _ptr(self.status_word),
                                      ctypes.byref(streams)))
        self.done.record(comp)

    def status(self) -> int:
        """Synchronises; the largest status code any chunk raised (0 = SA_OK)."""
        return read_status(self.status_word)


def params_for(w, order_group=None) -> MaskParams:
    """Mask parameters of a workload description, with the library's work-order
    grouping for its shape unless ``order_group`` is given."""
    if order_group is None:
        shape = Shape(w.B, w.Hq, w.Hkv, w.N, w.d, w.dv, SA_BF16 if w.dtype == "bf16" else SA_FP32, 0)
        order_group = order_group_hint(shape)
    return make_params(w.bq, w.bk, w.tau, w.theta, w.sink_tokens, w.txt_len, w.local_window,
                       w.anchor_tokens, w.causal, order_group)


def host_pipeline_for(w, device="cuda", chunks=4, order_group=None, **kw) -> HostPipeline:
    """HostPipeline for a workload description from ``inputs.WORKLOADS``."""
    lay = make_layout(w.T, w.H, w.W, w.txt_len, w.sink_frames, w.order, w.win)
    prm = params_for(w, order_group)
    return HostPipeline(w.B, w.Hq, w.Hkv, w.N, w.d, w.dv, w.dtype, layout=lay, params=prm, lam=w.lam,
                        device=device, chunks=chunks, **kw)


def pipeline_for(w, device="cuda", order_group=None, **kw) -> Pipeline:
    """Pipeline for a workload description from ``inputs.WORKLOADS``."""
    lay = make_layout(w.T, w.H, w.W, w.txt_len, w.sink_frames, w.order, w.win)
    prm = params_for(w, order_group)
    return Pipeline(w.B, w.Hq, w.Hkv, w.N, w.d, w.dv, w.dtype, layout=lay, params=prm, lam=w.lam,
                    device=device, **kw)
