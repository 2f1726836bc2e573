"""Python binding of libckl.so: the fused chunked KL-distillation loss on B200.

Argument marshalling only.  Every step of the loss runs in the CUDA library
(``csrc/``, declared in ``include/ckl.h``); PyTorch supplies device memory,
streams and events.  There is no CPU path: importing this package fails when
the library has not been built, and every call fails when no sm_100 device
is present.

    import chunked_kl_loss_ckl_b200 as ckl
    loss, lse = ckl.forward(H, W, idx, logp, mask, chunk=1024)
    dH, dW = ckl.backward(H, W, idx, logp, mask, lse, chunk=1024)
    loss = ckl.chunked_kl_loss(H, W, idx, logp, mask, chunk=1024)  # autograd
"""

from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "LIB_PATH", "CklError", "Trace", "KERNEL_NAMES", "lib", "workspace_bytes", "new_workspace",
    "forward", "backward", "read_device_status", "status_string", "chunked_kl_loss",
    "topk_cache", "single_pass_workspace_bytes", "forward_backward", "backward_plan",
    "DW_READY_FN", "forward_f32", "backward_f32", "selftest_wait_timeout", "dp_local_stats",
    "dp_finish", "forward_vocab_shard", "combine_vocab_shards", "backward_vocab_shard",
    "dh_to_bf16", "find_duplicate_ids",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libckl.so")

CKL_OK = 0
STATUS_NAMES = {
    0: "CKL_OK", 1: "CKL_ERR_INVALID_ARG", 2: "CKL_ERR_UNSUPPORTED", 3: "CKL_ERR_WORKSPACE",
    4: "CKL_ERR_CUDA", 5: "CKL_ERR_BAD_INDEX", 6: "CKL_ERR_BAD_LOGP", 7: "CKL_ERR_TIMEOUT",
    8: "CKL_ERR_TOPK_TIES", 9: "CKL_ERR_DUP_INDEX",
}
KERNEL_NAMES = {1: "prep", 2: "fwd_gemm", 3: "fwd_combine", 4: "bwd_dz", 5: "bwd_dhdw", 6: "other",
                7: "topk", 8: "sp_gemm", 9: "sp_rows"}


class CklError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)} ({status_string(code)})")


class _Trace(ctypes.Structure):
    _fields_ = [("capacity", ctypes.c_int32), ("count", ctypes.c_int32),
                ("events", ctypes.POINTER(ctypes.c_void_p)),
                ("kernel_id", ctypes.POINTER(ctypes.c_int32))]


# void (*)(int64_t v_begin, int64_t v_end, void* user)
DW_READY_FN = ctypes.CFUNCTYPE(None, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p)


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m chunked_kl_loss_ckl_b200._build` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    for name in ("ckl_forward", "ckl_backward", "ckl_backward_ex", "ckl_forward_backward",
                 "ckl_topk_cache"):
        if not hasattr(L, name):
            raise ImportError(f"{LIB_PATH} lacks {name}: it is older than its sources; rebuild "
                              "with `python -m chunked_kl_loss_ckl_b200._build --force`")
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    tr = ctypes.POINTER(_Trace)
    L.ckl_workspace_bytes.argtypes = [i64, i64, i64, i32, i64]
    L.ckl_workspace_bytes.restype = sz
    L.ckl_forward.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, i64, vp, vp, vp, sz, vp, tr]
    L.ckl_forward.restype = ctypes.c_int
    L.ckl_backward.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, i64, vp, vp, vp, vp, i32,
                               vp, sz, vp, tr]
    L.ckl_backward.restype = ctypes.c_int
    L.ckl_backward_ex.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, i64, vp, vp, vp, vp, i32,
                                  vp, sz, vp, tr, DW_READY_FN, vp]
    L.ckl_backward_ex.restype = ctypes.c_int
    L.ckl_backward_plan.argtypes = [i64, i64, i64, i32, i64, ctypes.POINTER(i64)]
    L.ckl_backward_plan.restype = ctypes.c_int
    L.ckl_workspace_bytes_f32.argtypes = [i64, i64, i64, i32, i64]
    L.ckl_workspace_bytes_f32.restype = sz
    L.ckl_forward_f32.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, i64, vp, vp, vp, sz, vp,
                                  tr]
    L.ckl_forward_f32.restype = ctypes.c_int
    L.ckl_backward_f32.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, i64, vp, vp, vp, vp,
                                   i32, vp, sz, vp, tr]
    L.ckl_backward_f32.restype = ctypes.c_int
    L.ckl_single_pass_workspace_bytes.argtypes = [i64, i64, i64, i32, i64]
    L.ckl_single_pass_workspace_bytes.restype = sz
    L.ckl_forward_backward.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, i64, vp, vp, vp, vp,
                                       vp, i32, vp, sz, vp, tr]
    L.ckl_forward_backward.restype = ctypes.c_int
    L.ckl_topk_cache.argtypes = [vp, i64, i64, i32, vp, vp, vp, vp]
    L.ckl_topk_cache.restype = ctypes.c_int
    L.ckl_find_duplicate_ids.argtypes = [vp, i64, i32, vp, vp]
    L.ckl_find_duplicate_ids.restype = ctypes.c_int
    L.ckl_selftest_wait_timeout.argtypes = [i64, vp, sz, vp]
    L.ckl_selftest_wait_timeout.restype = ctypes.c_int
    L.ckl_forward_vocab_shard.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i32, i64,
                                          vp, vp, sz, vp, tr]
    L.ckl_forward_vocab_shard.restype = ctypes.c_int
    L.ckl_combine_vocab_shards.argtypes = [vp, i32, vp, i64, i32, vp, vp, vp, sz, vp, tr]
    L.ckl_combine_vocab_shards.restype = ctypes.c_int
    L.ckl_backward_vocab_shard.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i32, i64,
                                           vp, vp, vp, vp, i32, vp, sz, vp, tr]
    L.ckl_backward_vocab_shard.restype = ctypes.c_int
    L.ckl_dh_to_bf16.argtypes = [vp, vp, i64, vp]
    L.ckl_dh_to_bf16.restype = ctypes.c_int
    L.ckl_dp_local_stats.argtypes = [vp, vp, vp]
    L.ckl_dp_local_stats.restype = ctypes.c_int
    L.ckl_dp_finish.argtypes = [vp, vp, vp, vp, vp]
    L.ckl_dp_finish.restype = ctypes.c_int
    L.ckl_read_device_status.argtypes = [vp, vp, ctypes.POINTER(i32)]
    L.ckl_read_device_status.restype = ctypes.c_int
    L.ckl_status_string.argtypes = [i32]
    L.ckl_status_string.restype = ctypes.c_char_p
    L.ckl_version.argtypes = []
    L.ckl_version.restype = i32
    return L


lib = _load()


def status_string(code: int) -> str:
    return lib.ckl_status_string(int(code)).decode()


class Trace:
    """Per-launch CUDA events recorded by the library around each kernel.

    ``durations()`` returns [(kernel name, ms)] after the stream has been
    synchronised.  Call ``reset()`` between steps to reuse the events.
    """

    def __init__(self, capacity: int = 256):
        self.capacity = capacity
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * capacity)]
        for e in self.events:  # create the underlying cudaEvent_t now
            e.record()
        torch.cuda.synchronize()
        self._handles = (ctypes.c_void_p * (2 * capacity))(*[e.cuda_event for e in self.events])
        self._ids = (ctypes.c_int32 * capacity)()
        self.c = _Trace(capacity, 0, ctypes.cast(self._handles, ctypes.POINTER(ctypes.c_void_p)),
                        ctypes.cast(self._ids, ctypes.POINTER(ctypes.c_int32)))

    def reset(self) -> None:
        self.c.count = 0

    @property
    def count(self) -> int:
        return int(self.c.count)

    def durations(self):
        return [(KERNEL_NAMES.get(self._ids[i], str(self._ids[i])),
                 self.events[2 * i].elapsed_time(self.events[2 * i + 1]))
                for i in range(self.count)]


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _trace_ptr(trace):
    return None if trace is None else ctypes.byref(trace.c)


_BF16 = (torch.bfloat16, torch.int16, torch.uint16)


def _check_inputs(H, W, idx, logp, mask, dtype=None):
    hw = _BF16 if dtype is None else (dtype,)
    for name, t, dts in (("H", H, hw), ("W", W, hw),
                         ("topk_idx", idx, (torch.int32,)), ("topk_logp", logp, (torch.float32,))):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.dtype not in dts:
            raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dts}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if mask is not None and (not mask.is_cuda or mask.dtype not in (torch.uint8, torch.bool)
                             or not mask.is_contiguous()):
        raise ValueError("mask must be a contiguous CUDA uint8/bool tensor")
    T, d = H.shape
    V, d2 = W.shape
    if d2 != d or idx.shape != logp.shape or idx.shape[0] != T:
        raise ValueError("shape mismatch: H [T,d], W [V,d], topk_idx/topk_logp [T,K]")
    if mask is not None and mask.shape != (T,):
        raise ValueError("mask must have shape [T]")
    return T, d, V, idx.shape[1]


def workspace_bytes(T: int, d: int, V: int, K: int, chunk: int) -> int:
    n = lib.ckl_workspace_bytes(T, d, V, K, chunk)
    if n == 0:
        raise CklError(1, "ckl_workspace_bytes")
    return int(n)


def new_workspace(T: int, d: int, V: int, K: int, chunk: int, device=None) -> torch.Tensor:
    n = workspace_bytes(T, d, V, K, chunk)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def forward(H, W, idx, logp, mask=None, chunk: int = 1024, workspace=None, stream=None,
            trace: Trace | None = None, out_loss=None, out_lse=None):
    """Mean KL over the positions that count, and lse for every row."""
    T, d, V, K = _check_inputs(H, W, idx, logp, mask)
    if workspace is None:
        workspace = new_workspace(T, d, V, K, chunk, H.device)
    loss = out_loss if out_loss is not None else torch.empty(1, dtype=torch.float32, device=H.device)
    lse = out_lse if out_lse is not None else torch.empty(T, dtype=torch.float32, device=H.device)
    rc = lib.ckl_forward(_ptr(H), _ptr(W), _ptr(idx), _ptr(logp), _ptr(mask), T, d, V, K, chunk,
                         _ptr(loss), _ptr(lse), _ptr(workspace), workspace.numel(),
                         _stream_handle(stream), _trace_ptr(trace))
    if rc != CKL_OK:
        raise CklError(rc, "ckl_forward")
    return loss, lse


def backward(H, W, idx, logp, mask, lse, grad_loss=None, chunk: int = 1024, dW=None,
             accumulate_dW: bool = False, workspace=None, stream=None,
             trace: Trace | None = None, out_dH=None, on_dw_ready=None):
    """dH (bf16, like H) and dW (fp32) by chunked recomputation.

    ``on_dw_ready(v_begin, v_end)``, when given, is called during the call as
    soon as the launches that last write dW rows [v_begin, v_end) have been
    enqueued on the stream (ckl_backward_ex); work it orders after them on
    the stream sees those rows final.
    """
    T, d, V, K = _check_inputs(H, W, idx, logp, mask)
    if workspace is None:
        workspace = new_workspace(T, d, V, K, chunk, H.device)
    dH = out_dH if out_dH is not None else torch.empty(T, d, dtype=torch.bfloat16, device=H.device)
    if dW is None:
        dW = torch.empty(V, d, dtype=torch.float32, device=H.device)
        accumulate_dW = False
    if grad_loss is not None and (grad_loss.dtype != torch.float32 or not grad_loss.is_cuda):
        raise TypeError("grad_loss must be a CUDA float32 tensor")
    if on_dw_ready is None:
        rc = lib.ckl_backward(_ptr(H), _ptr(W), _ptr(idx), _ptr(logp), _ptr(mask), T, d, V, K,
                              chunk, _ptr(lse), _ptr(grad_loss), _ptr(dH), _ptr(dW),
                              int(bool(accumulate_dW)), _ptr(workspace), workspace.numel(),
                              _stream_handle(stream), _trace_ptr(trace))
        if rc != CKL_OK:
            raise CklError(rc, "ckl_backward")
        return dH, dW
    errors = []

    def _cb(v0, v1, _user):
        if errors:
            return
        try:
            on_dw_ready(int(v0), int(v1))
        except BaseException as e:  # no exception may cross the C frames
            errors.append(e)

    cb = DW_READY_FN(_cb)
    rc = lib.ckl_backward_ex(_ptr(H), _ptr(W), _ptr(idx), _ptr(logp), _ptr(mask), T, d, V, K,
                             chunk, _ptr(lse), _ptr(grad_loss), _ptr(dH), _ptr(dW),
                             int(bool(accumulate_dW)), _ptr(workspace), workspace.numel(),
                             _stream_handle(stream), _trace_ptr(trace), cb, None)
    if errors:
        raise errors[0]
    if rc != CKL_OK:
        raise CklError(rc, "ckl_backward_ex")
    return dH, dW


def backward_plan(T: int, d: int, V: int, K: int, chunk: int):
    """(rows per row chunk, vocabulary columns per slab, slabs) of ckl_backward."""
    out = (ctypes.c_int64 * 3)()
    rc = lib.ckl_backward_plan(T, d, V, K, chunk, out)
    if rc != CKL_OK:
        raise CklError(rc, "ckl_backward_plan")
    return int(out[0]), int(out[1]), int(out[2])


def forward_f32(H, W, idx, logp, mask=None, chunk: int = 1024, workspace=None, stream=None,
                trace: Trace | None = None):
    """ckl_forward on fp32 H and W (tf32 tensor-core products)."""
    T, d, V, K = _check_inputs(H, W, idx, logp, mask, dtype=torch.float32)
    if workspace is None:
        n = lib.ckl_workspace_bytes_f32(T, d, V, K, chunk)
        if n == 0:
            raise CklError(1, "ckl_workspace_bytes_f32")
        workspace = torch.empty(n, dtype=torch.uint8, device=H.device)
    loss = torch.empty(1, dtype=torch.float32, device=H.device)
    lse = torch.empty(T, dtype=torch.float32, device=H.device)
    rc = lib.ckl_forward_f32(_ptr(H), _ptr(W), _ptr(idx), _ptr(logp), _ptr(mask), T, d, V, K,
                             chunk, _ptr(loss), _ptr(lse), _ptr(workspace), workspace.numel(),
                             _stream_handle(stream), _trace_ptr(trace))
    if rc != CKL_OK:
        raise CklError(rc, "ckl_forward_f32")
    return loss, lse


def backward_f32(H, W, idx, logp, mask, lse, grad_loss=None, chunk: int = 1024, dW=None,
                 accumulate_dW: bool = False, workspace=None, stream=None,
                 trace: Trace | None = None):
    """ckl_backward on fp32 H and W: dH and dW in fp32."""
    T, d, V, K = _check_inputs(H, W, idx, logp, mask, dtype=torch.float32)
    if workspace is None:
        n = lib.ckl_workspace_bytes_f32(T, d, V, K, chunk)
        if n == 0:
            raise CklError(1, "ckl_workspace_bytes_f32")
        workspace = torch.empty(n, dtype=torch.uint8, device=H.device)
    dH = torch.empty(T, d, dtype=torch.float32, device=H.device)
    if dW is None:
        dW = torch.empty(V, d, dtype=torch.float32, device=H.device)
        accumulate_dW = False
    if grad_loss is not None and (grad_loss.dtype != torch.float32 or not grad_loss.is_cuda):
        raise TypeError("grad_loss must be a CUDA float32 tensor")
    rc = lib.ckl_backward_f32(_ptr(H), _ptr(W), _ptr(idx), _ptr(logp), _ptr(mask), T, d, V, K,
                              chunk, _ptr(lse), _ptr(grad_loss), _ptr(dH), _ptr(dW),
                              int(bool(accumulate_dW)), _ptr(workspace), workspace.numel(),
                              _stream_handle(stream), _trace_ptr(trace))
    if rc != CKL_OK:
        raise CklError(rc, "ckl_backward_f32")
    return dH, dW


def single_pass_workspace_bytes(T: int, d: int, V: int, K: int, chunk: int) -> int:
    n = lib.ckl_single_pass_workspace_bytes(T, d, V, K, chunk)
    if n == 0:
        raise CklError(1, "ckl_single_pass_workspace_bytes")
    return int(n)


def forward_backward(H, W, idx, logp, mask=None, grad_loss=None, chunk: int = 1024, dW=None,
                     accumulate_dW: bool = False, workspace=None, stream=None,
                     trace: Trace | None = None, out_loss=None, out_lse=None, out_dH=None):
    """Single pass: loss, lse, dH and dW with each chunk's logits computed once.

    Returns (loss, lse, dH, dW).  The upstream gradient g (``grad_loss``, a
    CUDA float32 [1] tensor; None = 1) must be known before the call.
    """
    T, d, V, K = _check_inputs(H, W, idx, logp, mask)
    if workspace is None:
        n = single_pass_workspace_bytes(T, d, V, K, chunk)
        workspace = torch.empty(n, dtype=torch.uint8, device=H.device)
    loss = out_loss if out_loss is not None else torch.empty(1, dtype=torch.float32, device=H.device)
    lse = out_lse if out_lse is not None else torch.empty(T, dtype=torch.float32, device=H.device)
    dH = out_dH if out_dH is not None else torch.empty(T, d, dtype=torch.bfloat16, device=H.device)
    if dW is None:
        dW = torch.empty(V, d, dtype=torch.float32, device=H.device)
        accumulate_dW = False
    if grad_loss is not None and (grad_loss.dtype != torch.float32 or not grad_loss.is_cuda):
        raise TypeError("grad_loss must be a CUDA float32 tensor")
    rc = lib.ckl_forward_backward(_ptr(H), _ptr(W), _ptr(idx), _ptr(logp), _ptr(mask), T, d, V, K,
                                  chunk, _ptr(grad_loss), _ptr(loss), _ptr(lse), _ptr(dH),
                                  _ptr(dW), int(bool(accumulate_dW)), _ptr(workspace),
                                  workspace.numel(), _stream_handle(stream), _trace_ptr(trace))
    if rc != CKL_OK:
        raise CklError(rc, "ckl_forward_backward")
    return loss, lse, dH, dW


def topk_cache(logits, K: int, stream=None, status=None):
    """The teacher's offline cache from its logits ([T, V] bf16 on the GPU).

    Returns (ids [T, K] int32, log-probs [T, K] fp32, status [1] int32): per
    row the K most likely tokens by descending logit (equal logits: smaller
    id first) and their log-probabilities under the full softmax.  A non-zero
    status (bit 8) marks a row with more ties at its K-th logit than the
    kernel's sort holds.
    """
    if not logits.is_cuda or logits.dim() != 2 or not logits.is_contiguous():
        raise ValueError("logits must be a contiguous 2-D CUDA tensor")
    if logits.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError("logits must be bf16 (or its bits as int16/uint16)")
    T, V = logits.shape
    idx = torch.empty(T, K, dtype=torch.int32, device=logits.device)
    logp = torch.empty(T, K, dtype=torch.float32, device=logits.device)
    st = status if status is not None else torch.zeros(1, dtype=torch.int32, device=logits.device)
    rc = lib.ckl_topk_cache(_ptr(logits), T, V, K, _ptr(idx), _ptr(logp), _ptr(st),
                            _stream_handle(stream))
    if rc != CKL_OK:
        raise CklError(rc, "ckl_topk_cache")
    return idx, logp, st


def find_duplicate_ids(idx, stream=None):
    """ckl_find_duplicate_ids on a [T, K] int32 CUDA tensor of teacher ids:
    returns a [1] int32 device tensor holding the smallest row with a
    repeated id, or -1."""
    if not idx.is_cuda or idx.dim() != 2 or not idx.is_contiguous() or idx.dtype != torch.int32:
        raise ValueError("idx must be a contiguous 2-D int32 CUDA tensor")
    out = torch.empty(1, dtype=torch.int32, device=idx.device)
    rc = lib.ckl_find_duplicate_ids(_ptr(idx), idx.shape[0], idx.shape[1], _ptr(out),
                                    _stream_handle(stream))
    if rc != CKL_OK:
        raise CklError(rc, "ckl_find_duplicate_ids")
    return out


def selftest_wait_timeout(limit_s: float, workspace, stream=None) -> None:
    """Launch the bounded-wait self-test (ckl_selftest_wait_timeout); read the
    result with read_device_status(workspace)."""
    rc = lib.ckl_selftest_wait_timeout(int(limit_s * 1e9), _ptr(workspace), workspace.numel(),
                                       _stream_handle(stream))
    if rc != CKL_OK:
        raise CklError(rc, "ckl_selftest_wait_timeout")


def _check_shard(H, W_shard, idx, logp, mask, V, v_begin, v_end):
    T, d, Vs, K = _check_inputs(H, W_shard, idx, logp, mask)
    if not (0 <= v_begin < v_end <= V) or Vs != v_end - v_begin:
        raise ValueError("W_shard must hold rows [v_begin, v_end) of a V-row head")
    return T, d, Vs, K


def forward_vocab_shard(H, W_shard, idx, logp, mask, V: int, v_begin: int, v_end: int,
                        chunk: int = 1024, workspace=None, stream=None,
                        trace: Trace | None = None):
    """This vocabulary shard's per-row partials [T, 4] (ckl_forward_vocab_shard)
    and the workspace that ``combine_vocab_shards`` then reads."""
    T, d, Vs, K = _check_shard(H, W_shard, idx, logp, mask, V, v_begin, v_end)
    if workspace is None:
        workspace = new_workspace(T, d, Vs, K, chunk, H.device)
    part = torch.empty(T, 4, dtype=torch.float32, device=H.device)
    rc = lib.ckl_forward_vocab_shard(_ptr(H), _ptr(W_shard), _ptr(idx), _ptr(logp), _ptr(mask),
                                     T, d, V, v_begin, v_end, K, chunk, _ptr(part),
                                     _ptr(workspace), workspace.numel(), _stream_handle(stream),
                                     _trace_ptr(trace))
    if rc != CKL_OK:
        raise CklError(rc, "ckl_forward_vocab_shard")
    return part, workspace


def combine_vocab_shards(gathered, mask, K: int, workspace, stream=None,
                         trace: Trace | None = None):
    """(loss [1], lse [T]) from every shard's partials, gathered [g, T, 4]."""
    g, T, four = gathered.shape
    if four != 4 or gathered.dtype != torch.float32 or not gathered.is_contiguous():
        raise ValueError("gathered must be a contiguous float32 [g, T, 4] tensor")
    loss = torch.empty(1, dtype=torch.float32, device=gathered.device)
    lse = torch.empty(T, dtype=torch.float32, device=gathered.device)
    rc = lib.ckl_combine_vocab_shards(_ptr(gathered), g, _ptr(mask), T, K, _ptr(loss), _ptr(lse),
                                      _ptr(workspace), workspace.numel(), _stream_handle(stream),
                                      _trace_ptr(trace))
    if rc != CKL_OK:
        raise CklError(rc, "ckl_combine_vocab_shards")
    return loss, lse


def backward_vocab_shard(H, W_shard, idx, logp, mask, V: int, v_begin: int, v_end: int, lse,
                         grad_loss=None, chunk: int = 1024, dW=None, accumulate_dW: bool = False,
                         workspace=None, stream=None, trace: Trace | None = None):
    """(this shard's fp32 share of dH [T, d], dW of the shard's rows [Vs, d])."""
    T, d, Vs, K = _check_shard(H, W_shard, idx, logp, mask, V, v_begin, v_end)
    if workspace is None:
        workspace = new_workspace(T, d, Vs, K, chunk, H.device)
    if grad_loss is not None and (grad_loss.dtype != torch.float32 or not grad_loss.is_cuda):
        raise TypeError("grad_loss must be a CUDA float32 tensor")
    dHp = torch.empty(T, d, dtype=torch.float32, device=H.device)
    if dW is None:
        dW = torch.empty(Vs, d, dtype=torch.float32, device=H.device)
        accumulate_dW = False
    rc = lib.ckl_backward_vocab_shard(_ptr(H), _ptr(W_shard), _ptr(idx), _ptr(logp), _ptr(mask),
                                      T, d, V, v_begin, v_end, K, chunk, _ptr(lse),
                                      _ptr(grad_loss), _ptr(dHp), _ptr(dW),
                                      int(bool(accumulate_dW)), _ptr(workspace),
                                      workspace.numel(), _stream_handle(stream),
                                      _trace_ptr(trace))
    if rc != CKL_OK:
        raise CklError(rc, "ckl_backward_vocab_shard")
    return dHp, dW


def dh_to_bf16(src, stream=None):
    """bf16 copy (round to nearest even) of an fp32 CUDA tensor (ckl_dh_to_bf16)."""
    if src.dtype != torch.float32 or not src.is_cuda or not src.is_contiguous():
        raise ValueError("src must be a contiguous float32 CUDA tensor")
    dst = torch.empty(src.shape, dtype=torch.bfloat16, device=src.device)
    rc = lib.ckl_dh_to_bf16(_ptr(src), _ptr(dst), src.numel(), _stream_handle(stream))
    if rc != CKL_OK:
        raise CklError(rc, "ckl_dh_to_bf16")
    return dst


def dp_local_stats(workspace, stream=None):
    """[4] fp64 device tensor after ckl_forward with ``workspace``: (sum of KL
    over this rank's counted positions, N_r) twice; sum the first two over
    the ranks, keep the last two (ckl_dp_local_stats)."""
    stats = torch.empty(4, dtype=torch.float64, device=workspace.device)
    rc = lib.ckl_dp_local_stats(_ptr(workspace), _ptr(stats), _stream_handle(stream))
    if rc != CKL_OK:
        raise CklError(rc, "ckl_dp_local_stats")
    return stats


def dp_finish(stats, grad_loss=None, stream=None):
    """(global loss [1], this rank's upstream gradient g N_r / N [1]) from the
    stats whose first two entries were summed over the ranks (ckl_dp_finish)."""
    if stats.dtype != torch.float64 or not stats.is_cuda or stats.numel() != 4:
        raise ValueError("stats must be the [4] fp64 CUDA tensor of dp_local_stats")
    if grad_loss is not None and (grad_loss.dtype != torch.float32 or not grad_loss.is_cuda):
        raise TypeError("grad_loss must be a CUDA float32 tensor")
    loss = torch.empty(1, dtype=torch.float32, device=stats.device)
    g_local = torch.empty(1, dtype=torch.float32, device=stats.device)
    rc = lib.ckl_dp_finish(_ptr(stats), _ptr(grad_loss), _ptr(loss), _ptr(g_local),
                           _stream_handle(stream))
    if rc != CKL_OK:
        raise CklError(rc, "ckl_dp_finish")
    return loss, g_local


def read_device_status(workspace, stream=None):
    """(status code, raw device word) of the last call that used ``workspace``."""
    word = ctypes.c_int32(0)
    rc = lib.ckl_read_device_status(_ptr(workspace), _stream_handle(stream), ctypes.byref(word))
    return int(rc), int(word.value)


class _ChunkedKL(torch.autograd.Function):
    @staticmethod
    def forward(ctx, H, W, idx, logp, mask, chunk):
        loss, lse = forward(H, W, idx, logp, mask, chunk)
        ctx.save_for_backward(H, W, idx, logp, lse)
        ctx.mask = mask
        ctx.chunk = chunk
        return loss.reshape(())

    @staticmethod
    def backward(ctx, g):
        H, W, idx, logp, lse = ctx.saved_tensors
        gl = g.reshape(1).to(torch.float32).contiguous()
        dH, dW = backward(H, W, idx, logp, ctx.mask, lse, grad_loss=gl, chunk=ctx.chunk)
        return dH.to(H.dtype), dW.to(W.dtype), None, None, None, None


def chunked_kl_loss(H, W, idx, logp, mask=None, chunk: int = 1024):
    """Differentiable loss (gradients w.r.t. H and W; dW cast to W's dtype)."""
    return _ChunkedKL.apply(H, W, idx, logp, mask, chunk)
