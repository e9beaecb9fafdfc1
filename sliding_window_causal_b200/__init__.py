"""Sliding-window causal attention for B200 (sm_100a).

Query i attends to keys j with 0 <= i - j < W. The CUDA library behind include/swa.h
does all the work; these functions check torch tensors, pass their device pointers
and the current CUDA stream to the C ABI, and raise SwaError on a non-OK status.
PyTorch only supplies device memory and streams.

    forward(q, k, v, window, scale=None)  prefill, q/k/v [B,H,T,D] views (bf16 D 64|128, or
                                        fp32), any (b,h,t) strides, e.g. q.transpose(1, 2)
                                        of a [B,T,H,D] tensor
    band_weights(q, k, window)          the softmax weights of each band, [B,H,T,min(W,T)]
    decode(q, kring, vring, pos, window)  one query per stream over a W-slot ring
    chunk_forward(q, k, v, kring, vring, pos, window)  C new tokens per stream over the
                                        ring, then appended to it (streaming prefill)
    ring_append(k, v, kring, vring, pos, window)       write tokens into the ring
    mha_forward(x, wq, bq, wk, bk, wv, bv, wo, bo, num_heads, window)
                                        the multi-head module: projections (cuBLASLt)
                                        around the attention
    forward_lse(q, k, v, window)        (out, lse): the training forward
    backward(q, k, v, dout, window)     (dq, dk, dv) of the prefill (tensor cores for bf16)
    forward_host(...)                   prefill from pinned host tensors (copies included)
"""
import ctypes

from . import _native
from ._native import SWA_BF16, SWA_F32, SwaError, check

__all__ = ["forward", "forward_lse", "backward", "band_weights", "decode", "chunk_forward", "ring_append", "mha_forward",
           "mha_workspace_bytes", "forward_host", "device_status", "tile_class", "valid_slots",
           "split_plan", "set_wait_limit_ns", "timeout_probe", "work_item", "backward_cta_tile",
           "set_prefill_mode", "prefill_auto_state", "PREFILL_AUTO", "PREFILL_ADAPTIVE", "PREFILL_FAST",
           "SwaError"]


def _torch():
    import torch
    return torch


def _stream_ptr(device):
    torch = _torch()
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return SWA_BF16
    if t.dtype == torch.float32:
        return SWA_F32
    raise TypeError(f"unsupported dtype {t.dtype}: use bfloat16 or float32")


def _need_cuda(*ts, contiguous=True):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device (use forward_host for host tensors)")
        if contiguous and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if not contiguous and t.dim() > 0 and t.shape[-1] > 1 and t.stride(-1) != 1:
            raise ValueError("the head dimension must be contiguous (stride 1)")
    dev = ts[0].device
    if any(t.device != dev for t in ts):
        raise ValueError("tensors must be on one device")
    return dev


def _bht_strides(*ts):
    """(b, h, t) element strides of [B,H,T,D] views, flattened, as a ctypes int64 array."""
    vals = [x for t in ts for x in t.stride()[:3]]
    return (ctypes.c_int64 * len(vals))(*vals)


def forward(q, k, v, window, out=None, scale=None):
    """Sliding-window causal attention prefill. q, k, v: [B,H,T,D] CUDA tensors of one
    dtype (bf16 with D in {64, 128}, or fp32 with any D <= 4096), each with a contiguous
    head dimension and any (b,h,t) strides: a [B,T,H,D] tensor is passed as
    x.transpose(1, 2). A 3-D [B,T,D] input is treated as one head. scale defaults to
    1/sqrt(D). Returns out (same shape and dtype; allocated with q's strides if None)."""
    torch = _torch()
    squeeze = q.dim() == 3
    if squeeze:
        q, k, v = q.unsqueeze(1), k.unsqueeze(1), v.unsqueeze(1)
        if out is not None:
            out = out.unsqueeze(1)
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [B,H,T,D] shape")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    dev = _need_cuda(q, k, v, contiguous=False)
    if out is None:
        out = torch.empty_like(q)
    else:
        _need_cuda(out, contiguous=False)
        if out.shape != q.shape or out.dtype != q.dtype:
            raise ValueError("out must match q")
    B, H, T, D = q.shape
    lib = _native.lib()
    with torch.cuda.device(dev):
        if scale is None and all(t.is_contiguous() for t in (q, k, v, out)):
            check(lib.swa_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                  B, H, T, D, int(window), _dtype_code(q), _stream_ptr(dev)))
        else:
            sc = 1.0 / D ** 0.5 if scale is None else float(scale)
            check(lib.swa_forward_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                     B, H, T, D, int(window), sc, _bht_strides(q, k, v, out),
                                     _dtype_code(q), _stream_ptr(dev)))
    return out.squeeze(1) if squeeze else out


def forward_lse(q, k, v, window, scale=None):
    """Training forward: (out, lse) for contiguous [B,H,T,D] q, k, v; lse [B,H,T] fp32 is
    the natural log-sum-exp of each row's scaled scores (what backward needs)."""
    torch = _torch()
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [B,H,T,D] shape")
    dev = _need_cuda(q, k, v)
    B, H, T, D = q.shape
    out = torch.empty_like(q)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    sc = 1.0 / D ** 0.5 if scale is None else float(scale)
    with torch.cuda.device(dev):
        check(_native.lib().swa_forward_lse(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                            lse.data_ptr(), B, H, T, D, int(window), sc, _dtype_code(q),
                                            _stream_ptr(dev)))
    return out, lse


def backward(q, k, v, dout, window, scale=None, out=None, lse=None):
    """Gradients (dq, dk, dv) of the prefill output with respect to q, k, v, given the
    output gradient dout. All [B,H,T,D] contiguous CUDA tensors of one dtype. out and lse
    are the forward's (forward_lse); they are computed here when not given. bf16 with D
    64 or 128 runs on the tensor cores; other cases on the CUDA cores (D <= 512)."""
    torch = _torch()
    if q.dim() != 4 or any(t.shape != q.shape for t in (k, v, dout)):
        raise ValueError("q, k, v, dout must share one [B,H,T,D] shape")
    if any(t.dtype != q.dtype for t in (k, v, dout)):
        raise TypeError("q, k, v, dout must share one dtype")
    dev = _need_cuda(q, k, v, dout)
    B, H, T, D = q.shape
    tensor_cores = q.dtype == torch.bfloat16 and D in (64, 128)
    if tensor_cores and (out is None or lse is None):
        out, lse = forward_lse(q, k, v, window, scale)
    ptr = lambda t: None if t is None else t.data_ptr()
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    lib = _native.lib()
    ws = torch.empty(max(1, int(lib.swa_backward_workspace_bytes(B, H, T))), dtype=torch.uint8, device=dev)
    sc = 1.0 / D ** 0.5 if scale is None else float(scale)
    with torch.cuda.device(dev):
        check(lib.swa_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), ptr(out), dout.data_ptr(),
                               ptr(lse), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(),
                               ws.numel(), B, H, T, D, int(window), sc, _dtype_code(q), _stream_ptr(dev)))
    return dq, dk, dv


def band_weights(q, k, window, scale=None):
    """Softmax weights of every query's band: a [B,H,T,Wo] fp32 tensor, Wo = min(W, T),
    where [..., i, c] is the weight of key j = i - Wo + 1 + c (0 where j < 0). q, k as in
    forward (bf16 or fp32, strided views allowed). A debugging aid, not the prefill path."""
    torch = _torch()
    if q.dim() != 4 or k.shape != q.shape:
        raise ValueError("q and k must share one [B,H,T,D] shape")
    if k.dtype != q.dtype:
        raise TypeError("q and k must share one dtype")
    dev = _need_cuda(q, k, contiguous=False)
    B, H, T, D = q.shape
    Wo = min(int(window), T) if window >= 1 else int(window)
    w = torch.empty((B, H, T, max(Wo, 0)), dtype=torch.float32, device=dev)
    sc = 1.0 / D ** 0.5 if scale is None else float(scale)
    with torch.cuda.device(dev):
        check(_native.lib().swa_band_weights(q.data_ptr(), k.data_ptr(), w.data_ptr(), B, H, T, D,
                                             int(window), sc, _bht_strides(q, k), _dtype_code(q),
                                             _stream_ptr(dev)))
    return w


def decode(q, kring, vring, pos, window, out=None):
    """One new query per stream over a W-slot rolling KV buffer (slot = position mod W).
    q: [B,H,D] bf16; kring, vring: [B,H,W,D] bf16; pos: [B] int64 on the device (the
    0-based position of each stream's query, whose k/v are already in slot pos mod W)."""
    torch = _torch()
    if q.dim() != 3 or kring.dim() != 4:
        raise ValueError("q must be [B,H,D] and the rings [B,H,W,D]")
    B, H, D = q.shape
    if kring.shape != (B, H, window, D) or vring.shape != kring.shape:
        raise ValueError("rings must be [B,H,W,D] with W = window")
    if pos.shape != (B,) or pos.dtype != torch.int64:
        raise ValueError("pos must be int64 [B]")
    if q.dtype != torch.bfloat16 or kring.dtype != torch.bfloat16 or vring.dtype != torch.bfloat16:
        raise TypeError("decode takes bf16 q and rings")
    dev = _need_cuda(q, kring, vring, pos)
    if out is None:
        out = torch.empty_like(q)
    else:
        _need_cuda(out)
    with torch.cuda.device(dev):
        check(_native.lib().swa_decode(q.data_ptr(), kring.data_ptr(), vring.data_ptr(),
                                       pos.data_ptr(), out.data_ptr(), B, H, D, int(window),
                                       _stream_ptr(dev)))
    return out


def _stream_tensors(k, kring, vring, pos, window):
    torch = _torch()
    if k.dim() != 4 or kring.dim() != 4:
        raise ValueError("chunk tensors must be [B,H,C,D] and the rings [B,H,W,D]")
    B, H, C, D = k.shape
    if kring.shape != (B, H, window, D) or vring.shape != kring.shape:
        raise ValueError("rings must be [B,H,W,D] with W = window")
    if pos.shape != (B,) or pos.dtype != torch.int64:
        raise ValueError("pos must be int64 [B]")
    if any(t.dtype != torch.bfloat16 for t in (k, kring, vring)):
        raise TypeError("streaming calls take bf16 tensors")
    return B, H, C, D


def chunk_forward(q, k, v, kring, vring, pos, window, out=None):
    """Chunked streaming prefill: q, k, v [B,H,C,D] bf16 are C new tokens per stream at
    positions pos[b] .. pos[b]+C-1; kring, vring [B,H,W,D] hold each stream's last
    min(pos[b], W) positions (slot = position mod W). Returns out [B,H,C,D]; afterwards
    the rings also hold the chunk (updated in place)."""
    torch = _torch()
    B, H, C, D = _stream_tensors(k, kring, vring, pos, window)
    if q.shape != k.shape or v.shape != k.shape or q.dtype != k.dtype or v.dtype != k.dtype:
        raise ValueError("q, k, v must share one bf16 [B,H,C,D] shape")
    dev = _need_cuda(q, k, v, kring, vring, pos)
    if out is None:
        out = torch.empty_like(q)
    else:
        _need_cuda(out)
    with torch.cuda.device(dev):
        check(_native.lib().swa_chunk_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                              kring.data_ptr(), vring.data_ptr(), pos.data_ptr(),
                                              out.data_ptr(), B, H, C, D, int(window),
                                              _stream_ptr(dev)))
    return out


def ring_append(k, v, kring, vring, pos, window):
    """Write k, v [B,H,C,D] (positions pos[b] .. pos[b]+C-1) into the rings in place,
    position p into slot p mod W (only the last W tokens when C > W)."""
    torch = _torch()
    B, H, C, D = _stream_tensors(k, kring, vring, pos, window)
    if v.shape != k.shape or v.dtype != k.dtype:
        raise ValueError("k and v must share one bf16 [B,H,C,D] shape")
    dev = _need_cuda(k, v, kring, vring, pos)
    with torch.cuda.device(dev):
        check(_native.lib().swa_ring_append(k.data_ptr(), v.data_ptr(), kring.data_ptr(),
                                            vring.data_ptr(), pos.data_ptr(), B, H, C, D,
                                            int(window), _stream_ptr(dev)))


def mha_workspace_bytes(B, T, d_model, dtype):
    """Bytes of device workspace mha_forward needs."""
    torch = _torch()
    code = SWA_BF16 if dtype == torch.bfloat16 else SWA_F32
    return int(_native.lib().swa_mha_workspace_bytes(B, T, d_model, code))


def mha_forward(x, wq, bq, wk, bk, wv, bv, wo, bo, num_heads, window, out=None, workspace=None):
    """Sliding-window multi-head attention module: x [B,T,d] (or [T,d]); kernels [d,d]
    (input x output); biases [d] or None; all bf16 (head width d/num_heads of 64 or 128)
    or fp32. Returns out shaped like x. workspace: optional preallocated uint8 CUDA
    tensor of at least mha_workspace_bytes(...) bytes."""
    torch = _torch()
    squeeze = x.dim() == 2
    if squeeze:
        x = x.unsqueeze(0)
    if x.dim() != 3:
        raise ValueError("x must be [B,T,d] or [T,d]")
    B, T, d = x.shape
    mats = [wq, wk, wv, wo]
    biases = [bq, bk, bv, bo]
    if any(w.shape != (d, d) for w in mats) or any(b is not None and b.shape != (d,) for b in biases):
        raise ValueError("kernels must be [d,d] and biases [d]")
    if any(t.dtype != x.dtype for t in mats + [b for b in biases if b is not None]):
        raise TypeError("x, kernels and biases must share one dtype")
    dev = _need_cuda(x, *mats, *[b for b in biases if b is not None])
    if out is None:
        out = torch.empty_like(x)
    else:
        _need_cuda(out)
        out = out.view(B, T, d)
    need = mha_workspace_bytes(B, T, d, x.dtype)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    ptr = lambda t: None if t is None else t.data_ptr()
    with torch.cuda.device(dev):
        check(_native.lib().swa_mha_forward(x.data_ptr(), ptr(wq), ptr(bq), ptr(wk), ptr(bk), ptr(wv),
                                            ptr(bv), ptr(wo), ptr(bo), out.data_ptr(),
                                            workspace.data_ptr(), workspace.numel(), B, T, d,
                                            int(num_heads), int(window), _dtype_code(x),
                                            _stream_ptr(dev)))
    return out[0] if squeeze else out


def forward_host(q, k, v, window, out=None, device=None, staging=None, heads_per_group=0):
    """Prefill from host tensors through swa_forward_host: q, k, v are contiguous
    [B,H,T,D] CPU tensors (pinned memory lets the copies overlap); the result lands in
    `out` (a CPU tensor, allocated pinned if None). The (b,h) heads are copied in, computed
    and copied back in groups on the library's own streams, overlapped; the current
    stream waits for all of it. `staging` may hold preallocated device tensors
    (dq, dk, dv, dout) of the same shape. The copies are asynchronous: q, k, v and out
    must stay alive (and unchanged) until the current stream has passed this call, e.g.
    until a synchronize."""
    torch = _torch()
    device = torch.device(device or "cuda")
    for t in (q, k, v):
        if t.device.type != "cpu" or not t.is_contiguous() or t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("q, k, v must be contiguous CPU tensors of one shape and dtype")
    if q.dim() != 4:
        raise ValueError("q, k, v must be [B,H,T,D]")
    if staging is None:
        staging = tuple(torch.empty(q.shape, dtype=q.dtype, device=device) for _ in range(4))
    _need_cuda(*staging)
    if any(t.shape != q.shape or t.dtype != q.dtype for t in staging):
        raise ValueError("staging tensors must match q's shape and dtype")
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    if out.device.type != "cpu" or not out.is_contiguous() or out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must be a contiguous CPU tensor like q")
    B, H, T, D = q.shape
    dq, dk, dv, dout = staging
    with torch.cuda.device(device):
        check(_native.lib().swa_forward_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                             dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), dout.data_ptr(),
                                             B, H, T, D, int(window), int(heads_per_group), _dtype_code(q),
                                             _stream_ptr(device)))
    return out


def device_status(stream=None):
    """Synchronize the stream and return/clear the device status word (raises on error)."""
    torch = _torch()
    s = ctypes.c_void_p(stream if stream is not None else torch.cuda.current_stream().cuda_stream)
    return check(_native.lib().swa_device_status(s))


def tile_class(T, W, bm, bn, qt, kt):
    """0 not visited, 1 edge (masked), 2 full; -1 invalid. Host only, no GPU needed."""
    return _native.lib().swa_prefill_tile_class(T, W, bm, bn, qt, kt)


def work_item(u, B, H, T, W):
    """(b, h, pair) of the tensor-core prefill's u-th work item (see swa_prefill_work_item),
    or None for invalid arguments."""
    b, h, p = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    rc = _native.lib().swa_prefill_work_item(u, B, H, T, W, ctypes.byref(b), ctypes.byref(h), ctypes.byref(p))
    return None if rc != 0 else (b.value, h.value, p.value)


def backward_cta_tile(u, B, H, T, W, kv):
    """(b, h, tile) of the tensor-core backward's u-th CTA (see swa_backward_cta_tile): a
    key tile when kv, else a query tile; None for invalid arguments."""
    b, h, t = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    rc = _native.lib().swa_backward_cta_tile(u, B, H, T, W, 1 if kv else 0, ctypes.byref(b), ctypes.byref(h),
                                             ctypes.byref(t))
    return None if rc != 0 else (b.value, h.value, t.value)


PREFILL_AUTO, PREFILL_ADAPTIVE, PREFILL_FAST = 0, 1, 2


def set_prefill_mode(mode):
    """Set the bf16 prefill mode (PREFILL_AUTO, PREFILL_ADAPTIVE or PREFILL_FAST, see
    swa_set_prefill_mode) for later launches; returns the previous mode."""
    prev = _native.lib().swa_set_prefill_mode(int(mode))
    if prev < 0:
        raise SwaError(1, _native.lib().swa_last_error().decode())
    return prev


def prefill_auto_state(clear=False):
    """1 if PREFILL_AUTO has switched to adaptive on the current device, else 0; clear resets it."""
    v = _native.lib().swa_prefill_auto_state(1 if clear else 0)
    if v < 0:
        raise SwaError(4, _native.lib().swa_last_error().decode())
    return v


def valid_slots(pos, W):
    """Number of valid ring slots (slots 0..n-1) for a stream at position pos."""
    return _native.lib().swa_decode_valid_slots(pos, W)


def split_plan(B, H, D, W):
    """(splits, chunk) that swa_decode uses for these sizes."""
    s, c = ctypes.c_int32(), ctypes.c_int32()
    check(_native.lib().swa_decode_split_plan(B, H, D, W, ctypes.byref(s), ctypes.byref(c)))
    return s.value, c.value


def set_wait_limit_ns(ns):
    """Set the kernels' bounded-wait limit (0 = default); returns the previous limit."""
    return _native.lib().swa_set_wait_limit_ns(int(ns))


def timeout_probe():
    """Launch the kernel whose wait never completes, to exercise the timeout path."""
    torch = _torch()
    check(_native.lib().swa_timeout_probe(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)))
