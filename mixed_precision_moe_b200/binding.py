"""ctypes binding of libmoe (include/moe.h): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; this module turns
torch tensors into device pointers and the current torch stream into a
cudaStream_t, and raises ``MoeError`` on a non-zero status.  It fails loudly
when libmoe.so has not been built: there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

BF16, INT8, INT4 = 0, 1, 2
STATUS_BAD_EXPERT_ID = 0x1
STATUS_NONFINITE_LOGIT = 0x2
STATUS_WAIT_TIMEOUT = 0x4
STATUS_UNSET_EXPERT = 0x8
STATUS_BAD_ROW_INDEX = 0x10

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")

# name -> (restype, argtypes); mirrors include/moe.h
_P, _I, _S = C.c_void_p, C.c_int, C.c_size_t
SIGNATURES = {
    "moe_last_error": (C.c_char_p, []),
    "moe_abi_version": (_I, []),
    "moe_layer_create": (_I, [_I, _I, _I, _I, C.POINTER(_P)]),
    "moe_layer_destroy": (_I, [_P]),
    "moe_set_expert_precision": (_I, [_P, _I, _I, _P, _P]),
    "moe_get_expert_precision": (_I, [_P, _I, C.POINTER(_I)]),
    "moe_route_topk": (_I, [_P, _I, _I, _I, _I, _P, _P, _P]),
    "moe_router_topk": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    "moe_permute": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P]),
    "moe_ffn_workspace_bytes": (_I, [_P, _I, C.POINTER(_S)]),
    "moe_grouped_ffn_mixed": (_I, [_P, _P, _P, _I, _P, _P, _S, _P]),
    "moe_grouped_ffn_mixed_noalloc": (_I, [_P, _P, _P, _I, _P, _P]),
    "moe_ffn_noalloc_max_bytes": (_I, [C.POINTER(_S)]),
    "moe_ffn_noalloc_reset": (_I, []),
    "moe_combine": (_I, [_P, _P, _P, _I, _I, _I, _P, _P]),
    "moe_layer_forward": (_I, [_P, _P, _P, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P, _P]),
    "moe_layer_forward_hidden": (_I, [_P, _P, _P, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S,
                                      _P, _P]),
    "moe_quantize_weights": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "moe_get_device_status": (_I, [C.POINTER(C.c_uint)]),
    "moe_layer_set_hotness_counter": (_I, [_P, _P]),
    "moe_hot_set_size": (_I, [_P, _S, _I, C.POINTER(_I)]),
    "moe_select_hot_experts": (_I, [_P, _I, _I, _I, _P, _P]),
    "moe_layer_set_bf16_slots": (_I, [_P, _I, _P]),
    "moe_apply_hot_set": (_I, [_P, _P, _I, _I, _P]),
}


class MoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libmoe error {code}: {msg}")
        self.code = code


class _ExpertWeights(C.Structure):
    _fields_ = [("w13", _P), ("s13", _P), ("w2", _P), ("s2", _P)]


_lib = None


def lib():
    """Load libmoe.so (built in-tree by mixed_precision_moe_b200.build), or the
    library named by MOE_LIB_PATH (the profiling build of ffn_trace.py)."""
    global _lib
    if _lib is None:
        path = os.environ.get("MOE_LIB_PATH") or LIB_PATH
        if not os.path.exists(path):
            raise RuntimeError(f"libmoe.so is not built ({path}); run "
                               "`python -m mixed_precision_moe_b200.build`")
        L = C.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _check(rc: int):
    if rc != 0:
        raise MoeError(rc, lib().moe_last_error().decode())


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _need(t, dtype, name):
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor, got "
                         f"{t.dtype} on {t.device} (contiguous={t.is_contiguous()})")


# ----------------------------------------------------------- entry points --

def moe_route_topk(logits, k, renormalize=True, topk_idx=None, topk_w=None, stream=None):
    _need(logits, torch.float32, "logits")
    T, E = logits.shape
    if topk_idx is None:
        topk_idx = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    _check(lib().moe_route_topk(_ptr(logits), T, E, k, int(bool(renormalize)), _ptr(topk_idx),
                                _ptr(topk_w), _stream(stream)))
    return topk_idx, topk_w


def moe_router_topk(h, w_router, k, renormalize=True, logits=None, topk_idx=None, topk_w=None,
                    stream=None):
    """z = W_r h (fp32, written to `logits` if given) and its top-k; returns
    (topk_idx [T,k] int32, topk_w [T,k] fp32)."""
    _need(h, torch.bfloat16, "h")
    _need(w_router, torch.bfloat16, "w_router")
    T, H = h.shape
    E = w_router.shape[0]
    if w_router.shape[1] != H:
        raise ValueError("w_router must be [E, H]")
    if logits is not None:
        _need(logits, torch.float32, "logits")
        if tuple(logits.shape) != (T, E):
            raise ValueError("logits must be [T, E]")
    if topk_idx is None:
        topk_idx = torch.empty((T, k), dtype=torch.int32, device=h.device)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=h.device)
    _check(lib().moe_router_topk(_ptr(h), _ptr(w_router), T, H, E, k, int(bool(renormalize)),
                                 _ptr(logits), _ptr(topk_idx), _ptr(topk_w), _stream(stream)))
    return topk_idx, topk_w


def moe_permute(topk_idx, x, E, out=None, stream=None):
    """Returns (expert_offsets [E+1], perm_token [T*k], dest_row [T,k], x_perm [T*k,H])."""
    _need(topk_idx, torch.int32, "topk_idx")
    _need(x, torch.bfloat16, "x")
    T, k = topk_idx.shape
    H = x.shape[1]
    dev = x.device
    if out is None:
        out = (torch.empty(E + 1, dtype=torch.int32, device=dev),
               torch.empty(T * k, dtype=torch.int32, device=dev),
               torch.empty((T, k), dtype=torch.int32, device=dev),
               torch.empty((T * k, H), dtype=torch.bfloat16, device=dev))
    off, perm, dest, xp = out
    _check(lib().moe_permute(_ptr(topk_idx), _ptr(x), T, E, k, H, _ptr(off), _ptr(perm),
                             _ptr(dest), _ptr(xp), _stream(stream)))
    return out


def moe_ffn_workspace_bytes(layer, rows):
    n = C.c_size_t(0)
    _check(lib().moe_ffn_workspace_bytes(layer.handle, rows, C.byref(n)))
    return n.value


def moe_grouped_ffn_mixed(layer, x_perm, expert_offsets, y_perm=None, workspace=None,
                          stream=None):
    _need(x_perm, torch.bfloat16, "x_perm")
    _need(expert_offsets, torch.int32, "expert_offsets")
    rows = x_perm.shape[0]
    if y_perm is None:
        y_perm = torch.empty((rows, layer.H), dtype=torch.bfloat16, device=x_perm.device)
    if workspace is None:
        workspace = torch.empty(moe_ffn_workspace_bytes(layer, rows), dtype=torch.uint8,
                                device=x_perm.device)
    _check(lib().moe_grouped_ffn_mixed(layer.handle, _ptr(x_perm), _ptr(expert_offsets), rows,
                                       _ptr(y_perm), _ptr(workspace), workspace.numel(),
                                       _stream(stream)))
    return y_perm


def moe_grouped_ffn_mixed_noalloc(layer, x_perm, expert_offsets, y_perm=None, stream=None):
    """moe_grouped_ffn_mixed with the library's built-in scratch (no workspace);
    see include/moe.h for the size limit and the no-overlap rule."""
    _need(x_perm, torch.bfloat16, "x_perm")
    _need(expert_offsets, torch.int32, "expert_offsets")
    rows = x_perm.shape[0]
    if y_perm is None:
        y_perm = torch.empty((rows, layer.H), dtype=torch.bfloat16, device=x_perm.device)
    _check(lib().moe_grouped_ffn_mixed_noalloc(layer.handle, _ptr(x_perm), _ptr(expert_offsets),
                                               rows, _ptr(y_perm), _stream(stream)))
    return y_perm


def moe_ffn_noalloc_max_bytes() -> int:
    n = C.c_size_t(0)
    _check(lib().moe_ffn_noalloc_max_bytes(C.byref(n)))
    return n.value


def moe_ffn_noalloc_reset():
    """Forget the cached scratch address of the current device (after a device
    reset); the next no-alloc call looks it up again."""
    _check(lib().moe_ffn_noalloc_reset())


def moe_combine(y_perm, dest_row, topk_w, out=None, stream=None):
    _need(y_perm, torch.bfloat16, "y_perm")
    _need(dest_row, torch.int32, "dest_row")
    _need(topk_w, torch.float32, "topk_w")
    T, k = dest_row.shape
    H = y_perm.shape[1]
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=y_perm.device)
    _check(lib().moe_combine(_ptr(y_perm), _ptr(dest_row), _ptr(topk_w), T, k, H, _ptr(out),
                             _stream(stream)))
    return out


def moe_quantize_weights(w_bf16, precision, q_out=None, scales=None, stream=None):
    """bf16 [rows, K] -> (codes in the storage format, fp16 scales [K/128, rows])."""
    _need(w_bf16, torch.bfloat16, "w_bf16")
    rows, K = w_bf16.shape
    dev = w_bf16.device
    if q_out is None:
        q_out = (torch.empty((rows, K // 2), dtype=torch.uint8, device=dev) if precision == INT4
                 else torch.empty((rows, K), dtype=torch.int8, device=dev))
    if scales is None:
        scales = torch.empty((K // 128, rows), dtype=torch.float16, device=dev)
    _check(lib().moe_quantize_weights(_ptr(w_bf16), rows, K, precision, _ptr(q_out),
                                      _ptr(scales), _stream(stream)))
    return q_out, scales


def moe_select_hot_experts(counts, n_hot, zero_counts=True, hot_ids=None, stream=None):
    """counts: device uint32-as-int32 [E]; returns hot_ids (device int32 [n_hot])."""
    _need(counts, torch.int32, "counts")
    if hot_ids is None:
        hot_ids = torch.empty(n_hot, dtype=torch.int32, device=counts.device)
    _check(lib().moe_select_hot_experts(_ptr(counts), counts.numel(), n_hot, int(bool(zero_counts)),
                                        _ptr(hot_ids), _stream(stream)))
    return hot_ids


def moe_get_device_status() -> int:
    v = C.c_uint(0)
    _check(lib().moe_get_device_status(C.byref(v)))
    return v.value


# ------------------------------------------------------------ layer object --

class MoELayer:
    """One routed-expert layer: the library's layer handle plus the weight
    tensors it points to (kept alive here, as the C ABI requires)."""

    def __init__(self, H, I, E, k):
        h = C.c_void_p()
        _check(lib().moe_layer_create(H, I, E, k, C.byref(h)))
        self.handle = h
        self.H, self.I, self.E, self.k = H, I, E, k
        self._weights = [None] * E
        self._retired = []   # (event, tensors) kept until the event completes

    def set_expert(self, e, precision, w13, s13, w2, s2, stream=None):
        """Stream-ordered handle swap; the previous tensors of expert e are
        released once an event recorded after this call has completed."""
        w = _ExpertWeights(w13.data_ptr(), s13.data_ptr() if s13 is not None else None,
                           w2.data_ptr(), s2.data_ptr() if s2 is not None else None)
        _check(lib().moe_set_expert_precision(self.handle, e, precision, C.byref(w),
                                              _stream(stream)))
        old = self._weights[e]
        self._weights[e] = (w13, s13, w2, s2)
        if old is not None:
            ev = torch.cuda.Event()
            ev.record(stream if stream is not None else torch.cuda.current_stream())
            self._retired.append((ev, old))
        self._retired = [(ev, t) for ev, t in self._retired if not ev.query()]

    def set_hotness_counter(self, counts):
        """counts: device int32 [E] (read as uint32) or None; later forwards add
        their per-expert selection counts to it."""
        if counts is not None:
            _need(counts, torch.int32, "counts")
            assert counts.numel() == self.E
        self._hot = counts
        _check(lib().moe_layer_set_hotness_counter(self.handle, _ptr(counts)))

    def hot_set_size(self, budget_bytes, low=INT4) -> int:
        n = C.c_int(0)
        _check(lib().moe_hot_set_size(self.handle, int(budget_bytes), low, C.byref(n)))
        return n.value

    def set_bf16_slots(self, slots):
        """slots: list of (w13 bf16 [2I, H], w2 bf16 [H, I]) device tensors."""
        arr = (_ExpertWeights * max(1, len(slots)))()
        for i, (w13, w2) in enumerate(slots):
            _need(w13, torch.bfloat16, "slot w13")
            _need(w2, torch.bfloat16, "slot w2")
            arr[i] = _ExpertWeights(w13.data_ptr(), None, w2.data_ptr(), None)
        self._slots = list(slots)
        _check(lib().moe_layer_set_bf16_slots(self.handle, len(slots), arr))

    def apply_hot_set(self, hot_ids, n_hot, slot_base, stream=None):
        _need(hot_ids, torch.int32, "hot_ids")
        _check(lib().moe_apply_hot_set(self.handle, _ptr(hot_ids), n_hot, slot_base,
                                       _stream(stream)))

    def precision(self, e) -> int:
        p = C.c_int(0)
        _check(lib().moe_get_expert_precision(self.handle, e, C.byref(p)))
        return p.value

    def forward(self, logits, x, renormalize=True, bufs=None, stream=None):
        """route -> permute -> grouped FFN -> combine (one moe_layer_forward
        call); returns out [T, H] bf16."""
        _need(logits, torch.float32, "logits")
        _need(x, torch.bfloat16, "x")
        T = logits.shape[0]
        if bufs is None:
            bufs = self.alloc_buffers(T, logits.device)
        idx, w = bufs["route"]
        off, perm, dest, xp = bufs["permute"]
        y, ws = bufs["ffn"]
        out = bufs["out"]
        _check(lib().moe_layer_forward(self.handle, _ptr(logits), _ptr(x), T, int(bool(renormalize)),
                                       _ptr(idx), _ptr(w), _ptr(off), _ptr(perm), _ptr(dest),
                                       _ptr(xp), _ptr(y), _ptr(ws), ws.numel(), _ptr(out),
                                       _stream(stream)))
        return out

    def forward_hidden(self, x, w_router, renormalize=True, bufs=None, stream=None):
        """router (z = W_r x) -> route -> permute -> grouped FFN -> combine (one
        moe_layer_forward_hidden call); returns out [T, H] bf16.  The logits
        land in bufs["logits"]."""
        _need(x, torch.bfloat16, "x")
        _need(w_router, torch.bfloat16, "w_router")
        if tuple(w_router.shape) != (self.E, self.H):
            raise ValueError("w_router must be [E, H]")
        T = x.shape[0]
        if bufs is None:
            bufs = self.alloc_buffers(T, x.device)
        idx, w = bufs["route"]
        off, perm, dest, xp = bufs["permute"]
        y, ws = bufs["ffn"]
        out = bufs["out"]
        _check(lib().moe_layer_forward_hidden(
            self.handle, _ptr(x), _ptr(w_router), T, int(bool(renormalize)), _ptr(bufs["logits"]),
            _ptr(idx), _ptr(w), _ptr(off), _ptr(perm), _ptr(dest), _ptr(xp), _ptr(y), _ptr(ws),
            ws.numel(), _ptr(out), _stream(stream)))
        return out

    def alloc_buffers(self, T, device="cuda"):
        """Preallocated intermediates for forward(bufs=...), e.g. for graph capture."""
        k, H, E = self.k, self.H, self.E
        R = T * k
        i32 = dict(dtype=torch.int32, device=device)
        return {
            "route": (torch.empty((T, k), **i32), torch.empty((T, k), dtype=torch.float32,
                                                             device=device)),
            "permute": (torch.empty(E + 1, **i32), torch.empty(R, **i32),
                        torch.empty((T, k), **i32),
                        torch.empty((R, H), dtype=torch.bfloat16, device=device)),
            "ffn": (torch.empty((R, H), dtype=torch.bfloat16, device=device),
                    torch.empty(moe_ffn_workspace_bytes(self, R), dtype=torch.uint8,
                                device=device)),
            "out": torch.empty((T, H), dtype=torch.bfloat16, device=device),
            "logits": torch.empty((T, E), dtype=torch.float32, device=device),
        }

    def close(self):
        if self.handle:
            _check(lib().moe_layer_destroy(self.handle))
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
