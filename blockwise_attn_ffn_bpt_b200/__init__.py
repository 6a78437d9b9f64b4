"""Python binding of the B200 BPT layer-forward library (libbpt.so).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. torch is used for device memory and streams. There is no fallback:
if the built library is missing, or a call returns an error status, these
functions raise.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbpt.so")

BPT_DTYPE_BF16 = 0
BPT_DTYPE_F32 = 1
# FFN-side schedules (wave_rows): include/bpt.h
BPT_WAVE_DEFAULT = 0
BPT_WAVE_CHAINED = -1
BPT_WAVE_DEFAULT_WAVES = -2
BPT_WAVE_MEGA = -3

EXPORTED = (
    "bpt_status_string", "bpt_layer_forward", "bpt_layer_forward_f32", "bpt_layer_workspace_bytes",
    "bpt_layer_forward_ws", "bpt_layer_forward_noalloc", "bpt_layer_workspace_bytes_ffn", "bpt_layer_forward_ffn",
    "bpt_layer_forward_host", "bpt_convert_f32_to_bf16",
    "bpt_qkv_projection", "bpt_attention", "bpt_ffn_backward_workspace_bytes", "bpt_ffn_backward",
    "bpt_attention_lse", "bpt_attention_backward_workspace_bytes", "bpt_attention_backward",
    "bpt_layer_backward_workspace_bytes", "bpt_layer_backward", "bpt_layer_forward_save", "bpt_layer_backward_saved",
    "bpt_stream_status", "bpt_device_status", "bpt_wait_flag",
    "bpt_launch_count", "bpt_set_kernel_timing", "bpt_kernel_times",
)


class BPTError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int), ("total_ms", ctypes.c_double)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m blockwise_attn_ffn_bpt_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.bpt_status_string.restype = ctypes.c_char_p
    L.bpt_status_string.argtypes = [i]
    L.bpt_layer_forward.restype = i
    L.bpt_layer_forward.argtypes = [vp] * 9 + [i] * 7 + [vp, vp]
    L.bpt_layer_forward_f32.restype = i
    L.bpt_layer_forward_f32.argtypes = [vp] * 9 + [i] * 7 + [vp, vp]
    L.bpt_layer_workspace_bytes.restype = sz
    L.bpt_layer_workspace_bytes.argtypes = [i] * 8
    L.bpt_layer_forward_ws.restype = i
    L.bpt_layer_forward_ws.argtypes = [i] + [vp] * 9 + [i] * 8 + [vp, sz, vp, vp]
    L.bpt_layer_workspace_bytes_ffn.restype = sz
    L.bpt_layer_workspace_bytes_ffn.argtypes = [i] * 9
    L.bpt_layer_forward_ffn.restype = i
    L.bpt_layer_forward_ffn.argtypes = [i] + [vp] * 9 + [i] * 9 + [vp, sz, vp, vp]
    ll = ctypes.c_longlong
    L.bpt_convert_f32_to_bf16.restype = i
    L.bpt_convert_f32_to_bf16.argtypes = [vp, vp, ll, vp]
    L.bpt_layer_forward_host.restype = i
    L.bpt_layer_forward_host.argtypes = [i, vp, ll] + [vp] * 8 + [i] * 7 + [vp, ll, i, vp]
    L.bpt_qkv_projection.restype = i
    L.bpt_qkv_projection.argtypes = [vp] * 3 + [i] * 3 + [vp] * 4
    L.bpt_attention.restype = i
    L.bpt_attention.argtypes = [vp] * 3 + [i] * 7 + [vp, vp]
    L.bpt_ffn_backward_workspace_bytes.restype = sz
    L.bpt_ffn_backward_workspace_bytes.argtypes = [i] * 4
    L.bpt_ffn_backward.restype = i
    L.bpt_ffn_backward.argtypes = [vp] * 5 + [i] * 4 + [vp] * 6 + [sz, vp]
    L.bpt_attention_lse.restype = i
    L.bpt_attention_lse.argtypes = [vp] * 3 + [i] * 5 + [vp, vp, vp]
    L.bpt_attention_backward_workspace_bytes.restype = sz
    L.bpt_attention_backward_workspace_bytes.argtypes = [i] * 4
    L.bpt_attention_backward.restype = i
    L.bpt_attention_backward.argtypes = [vp] * 6 + [i] * 5 + [vp] * 4 + [sz, vp]
    L.bpt_layer_backward_workspace_bytes.restype = sz
    L.bpt_layer_backward_workspace_bytes.argtypes = [i] * 5
    L.bpt_layer_backward.restype = i
    L.bpt_layer_backward.argtypes = [vp] * 10 + [i] * 6 + [vp] * 10 + [sz, vp]
    L.bpt_layer_forward_save.restype = i
    L.bpt_layer_forward_save.argtypes = [vp] * 9 + [i] * 8 + [vp] * 4
    L.bpt_layer_backward_saved.restype = i
    L.bpt_layer_backward_saved.argtypes = [vp] * 12 + [i] * 6 + [vp] * 10 + [sz, vp]
    L.bpt_stream_status.restype = i
    L.bpt_stream_status.argtypes = [vp]
    L.bpt_device_status.restype = i
    L.bpt_device_status.argtypes = []
    L.bpt_wait_flag.restype = i
    L.bpt_wait_flag.argtypes = [vp, i, i, vp]
    L.bpt_launch_count.restype = ctypes.c_uint64
    L.bpt_launch_count.argtypes = []
    L.bpt_set_kernel_timing.restype = i
    L.bpt_set_kernel_timing.argtypes = [i]
    L.bpt_kernel_times.restype = i
    L.bpt_kernel_times.argtypes = [ctypes.POINTER(KernelTime), i]
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().bpt_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != 0:
        raise BPTError(status, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


PARAM_NAMES = ("Wqkv", "bqkv", "Wo", "bo", "W1", "b1", "W2", "b2")


def workspace_bytes(dtype: int, b: int, s: int, h: int, heads: int, q_block: int, kv_block: int,
                    wave_rows: int = 0, ffn: Optional[int] = None) -> int:
    """Workspace bytes of one call (0 for invalid arguments); ffn defaults to 4h."""
    if ffn is None:
        return int(lib().bpt_layer_workspace_bytes(dtype, b, s, h, heads, q_block, kv_block, wave_rows))
    return int(lib().bpt_layer_workspace_bytes_ffn(dtype, b, s, h, heads, ffn, q_block, kv_block, wave_rows))


def _param_shapes(h: int, ffn: int) -> dict:
    return {"Wqkv": (h, 3 * h), "bqkv": (3 * h,), "Wo": (h, h), "bo": (h,), "W1": (h, ffn), "b1": (ffn,),
            "W2": (ffn, h), "b2": (h,)}


def layer_forward(x: torch.Tensor, params: dict, heads: int, q_block: int, kv_block: int, causal: bool,
                  out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  wave_rows: int = 0, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """One BPT layer forward; x [b, s, h] (bf16 or fp32) on the GPU, params a
    dict of Wqkv [h,3h], bqkv, Wo [h,h], bo, W1 [h,f], b1, W2 [f,h], b2 of
    x's dtype, with FFN width f = W1's second dimension (4h in the pages; any
    multiple of 64). Returns out, fp32 [b, s, h].

    With workspace=None the library allocates its workspace stream-ordered;
    otherwise `workspace` (a uint8 CUDA tensor of at least workspace_bytes(...))
    is used and nothing is allocated.
    """
    b, s, h = x.shape
    if out is None:
        out = torch.empty((b, s, h), dtype=torch.float32, device=x.device)
    ps = [_ptr(params[k]) for k in PARAM_NAMES]
    if x.dtype == torch.bfloat16:
        dtype = BPT_DTYPE_BF16
    elif x.dtype == torch.float32:
        dtype = BPT_DTYPE_F32
    else:
        raise TypeError(f"unsupported dtype {x.dtype}")
    ffn = int(params["W1"].shape[-1])
    for k, shape in _param_shapes(h, ffn).items():
        if params[k].dtype != x.dtype:
            raise TypeError(f"{k} must have dtype {x.dtype}")
        if tuple(params[k].shape) != shape:
            raise ValueError(f"{k} has shape {tuple(params[k].shape)}, expected {shape}")
    st = _stream(stream)
    if ffn != 4 * h:
        ws_ptr, ws_n = (None, 0) if workspace is None else (_ptr(workspace), workspace.numel())
        r = lib().bpt_layer_forward_ffn(dtype, _ptr(x), *ps, b, s, h, heads, ffn, q_block, kv_block,
                                        int(bool(causal)), wave_rows, ws_ptr, ws_n, _ptr(out), st)
    elif workspace is None and wave_rows == 0:
        fn = lib().bpt_layer_forward if dtype == BPT_DTYPE_BF16 else lib().bpt_layer_forward_f32
        r = fn(_ptr(x), *ps, b, s, h, heads, q_block, kv_block, int(bool(causal)), _ptr(out), st)
    else:
        if workspace is None:
            nbytes = workspace_bytes(dtype, b, s, h, heads, q_block, kv_block, wave_rows)
            workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)
        r = lib().bpt_layer_forward_ws(dtype, _ptr(x), *ps, b, s, h, heads, q_block, kv_block, int(bool(causal)),
                                       wave_rows, _ptr(workspace), workspace.numel(), _ptr(out), st)
    _check(r, "bpt_layer_forward")
    return out


def layer_forward_host(x_host: torch.Tensor, params: dict, heads: int, q_block: int, kv_block: int, causal: bool,
                       out_host: Optional[torch.Tensor] = None, n_inputs: Optional[int] = None,
                       stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """End to end from host memory through bpt_layer_forward_host.

    x_host is a host tensor [n, b, s, h] of n inputs, or [b, s, h] used
    n_inputs times (default 1); bf16 or fp32, pinned for the copies to overlap
    the compute. Weights are on the GPU. Returns out_host (fp32, [n, b, s, h]
    or [b, s, h] holding the last result), after every result has arrived.
    """
    if x_host.is_cuda:
        raise ValueError("x_host must be in host memory")
    if x_host.dim() == 4:
        n, b, s, h = x_host.shape
        x_stride = b * s * h * x_host.element_size()
        shape = (n, b, s, h)
    else:
        b, s, h = x_host.shape
        n = 1 if n_inputs is None else int(n_inputs)
        x_stride = 0
        shape = (b, s, h)
    if out_host is None:
        out_host = torch.empty(shape, dtype=torch.float32, pin_memory=True)
    if tuple(out_host.shape) != shape or out_host.dtype != torch.float32 or out_host.is_cuda:
        raise ValueError(f"out_host must be a host fp32 tensor of shape {shape}")
    out_stride = b * s * h * 4 if x_host.dim() == 4 else 0
    if x_host.dtype == torch.bfloat16:
        dtype = BPT_DTYPE_BF16
    elif x_host.dtype == torch.float32:
        dtype = BPT_DTYPE_F32
    else:
        raise TypeError(f"unsupported dtype {x_host.dtype}")
    for k, shp in _param_shapes(h, 4 * h).items():
        if params[k].dtype != x_host.dtype or tuple(params[k].shape) != shp or not params[k].is_cuda:
            raise ValueError(f"{k} must be a CUDA {x_host.dtype} tensor of shape {shp}")
    ps = [_ptr(params[k]) for k in PARAM_NAMES]
    dev = params["Wqkv"].device
    st = (stream if stream is not None else torch.cuda.current_stream(dev)).cuda_stream
    r = lib().bpt_layer_forward_host(dtype, _ptr(x_host), x_stride, *ps, b, s, h, heads, q_block, kv_block,
                                     int(bool(causal)), _ptr(out_host), out_stride, n, st)
    _check(r, "bpt_layer_forward_host")
    return out_host


def convert_f32_to_bf16(src: torch.Tensor, out: Optional[torch.Tensor] = None,
                        stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """src (fp32, CUDA) rounded to bf16 by the library's kernel."""
    if src.dtype != torch.float32 or not src.is_cuda:
        raise TypeError("src must be a CUDA fp32 tensor")
    if out is None:
        out = torch.empty(src.shape, dtype=torch.bfloat16, device=src.device)
    if out.dtype != torch.bfloat16 or out.numel() != src.numel():
        raise ValueError("out must be a bf16 tensor with as many elements as src")
    _check(lib().bpt_convert_f32_to_bf16(_ptr(src), _ptr(out), src.numel(), _stream(stream)),
           "bpt_convert_f32_to_bf16")
    return out


def stack_forward(x: torch.Tensor, layers: list, heads: int, q_block: int, kv_block: int, causal: bool,
                  stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """A stack of BPT layers: x (bf16 [b, s, h], CUDA) through each parameter
    dict of `layers` in turn; between layers the fp32 output is rounded to
    bf16 on the device. Returns the last layer's fp32 output."""
    out = None
    cur = x
    for i, params in enumerate(layers):
        out = layer_forward(cur, params, heads, q_block, kv_block, causal, stream=stream)
        if i + 1 < len(layers):
            cur = convert_f32_to_bf16(out, stream=stream).view(x.shape)
    return out


def qkv_projection(x: torch.Tensor, Wqkv: torch.Tensor, bqkv: torch.Tensor,
                   stream: Optional[torch.cuda.Stream] = None):
    """Algorithm 1 step 1 alone: bf16 Q, K, V [b, s, h] from bf16 x [b, s, h]."""
    b, s, h = x.shape
    q = torch.empty((b, s, h), dtype=torch.bfloat16, device=x.device)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    r = lib().bpt_qkv_projection(_ptr(x), _ptr(Wqkv), _ptr(bqkv), b, s, h, _ptr(q), _ptr(k), _ptr(v),
                                 _stream(stream))
    _check(r, "bpt_qkv_projection")
    return q, k, v


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, heads: int, q_block: int, kv_block: int,
              causal: bool, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Algorithm 1 steps 2-10 alone: bf16 O [b, s, h] (heads concatenated)."""
    b, s, h = q.shape
    o = torch.empty((b, s, h), dtype=torch.bfloat16, device=q.device)
    r = lib().bpt_attention(_ptr(q), _ptr(k), _ptr(v), b, s, h, heads, q_block, kv_block, int(bool(causal)),
                            _ptr(o), _stream(stream))
    _check(r, "bpt_attention")
    return o


def attention_lse(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, heads: int, causal: bool,
                  stream: Optional[torch.cuda.Stream] = None):
    """Attention (as `attention`) and each row's log-sum-exp of the scaled
    scores in log2 units (bpt_attention_lse): returns (O bf16 [b, s, h], lse2
    fp32 [b, heads, s])."""
    b, s, h = q.shape
    o = torch.empty((b, s, h), dtype=torch.bfloat16, device=q.device)
    lse2 = torch.empty((b, heads, s), dtype=torch.float32, device=q.device)
    r = lib().bpt_attention_lse(_ptr(q), _ptr(k), _ptr(v), b, s, h, heads, int(bool(causal)), _ptr(o), _ptr(lse2),
                                _stream(stream))
    _check(r, "bpt_attention_lse")
    return o, lse2


def attention_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, dO: torch.Tensor,
                       lse2: torch.Tensor, heads: int, causal: bool,
                       stream: Optional[torch.cuda.Stream] = None) -> dict:
    """dQ, dK, dV (bf16 [b, s, h]) of the attention for dO = dL/dO, from the
    forward's o and lse2 (bpt_attention_backward). Returns {"dq", "dk", "dv"}."""
    b, s, h = q.shape
    for name, t in (("k", k), ("v", v), ("o", o), ("dO", dO)):
        if t.dtype != torch.bfloat16 or t.shape != q.shape:
            raise ValueError(f"{name} must be bf16 of shape {tuple(q.shape)}")
    if lse2.dtype != torch.float32 or tuple(lse2.shape) != (b, heads, s):
        raise ValueError(f"lse2 must be fp32 of shape {(b, heads, s)}")
    g = {"dq": torch.empty_like(q), "dk": torch.empty_like(q), "dv": torch.empty_like(q)}
    nbytes = int(lib().bpt_attention_backward_workspace_bytes(b, s, h, heads))
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    r = lib().bpt_attention_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse2), b, s, h, heads,
                                     int(bool(causal)), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(ws),
                                     ws.numel(), _stream(stream))
    _check(r, "bpt_attention_backward")
    return g


def layer_forward_save(x: torch.Tensor, params: dict, heads: int, q_block: int, kv_block: int, causal: bool,
                       stream: Optional[torch.cuda.Stream] = None):
    """The layer forward that also keeps the attention output O and each row's
    log-sum-exp for a later backward (bpt_layer_forward_save): bf16 x and
    params as for layer_forward. Returns (out fp32 [b, s, h], o bf16 [b, s, h],
    lse2 fp32 [b, heads, s]); pass (o, lse2) as layer_backward's `saved`."""
    b, s, h = x.shape
    ffn = int(params["W1"].shape[-1])
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bf16")
    for k, shape in _param_shapes(h, ffn).items():
        if params[k].dtype != torch.bfloat16 or tuple(params[k].shape) != shape:
            raise ValueError(f"{k} must be bf16 of shape {shape}")
    out = torch.empty((b, s, h), dtype=torch.float32, device=x.device)
    o = torch.empty((b, s, h), dtype=torch.bfloat16, device=x.device)
    lse2 = torch.empty((b, heads, s), dtype=torch.float32, device=x.device)
    r = lib().bpt_layer_forward_save(_ptr(x), *[_ptr(params[k]) for k in PARAM_NAMES], b, s, h, heads, ffn, q_block,
                                     kv_block, int(bool(causal)), _ptr(out), _ptr(o), _ptr(lse2), _stream(stream))
    _check(r, "bpt_layer_forward_save")
    return out, o, lse2


def layer_backward(x: torch.Tensor, params: dict, dy: torch.Tensor, heads: int, causal: bool,
                   stream: Optional[torch.cuda.Stream] = None, saved=None) -> dict:
    """Gradients of the layer's output (bpt_layer_backward) for dy = dL/dout
    (fp32 [b, s, h]): x bf16 [b, s, h] and params as for layer_forward (bf16,
    FFN width from W1). Returns {"dx", "dWqkv", "dbqkv", "dWo", "dbo", "dW1",
    "db1", "dW2", "db2"} (fp32). saved = (o, lse2) from layer_forward_save skips
    the attention's recomputation (bpt_layer_backward_saved)."""
    b, s, h = x.shape
    ffn = params["W1"].shape[-1]
    if x.dtype != torch.bfloat16 or dy.dtype != torch.float32 or dy.shape != x.shape:
        raise TypeError("x must be bf16 and dy fp32 of the same shape")
    shapes = {"Wqkv": (h, 3 * h), "bqkv": (3 * h,), "Wo": (h, h), "bo": (h,), "W1": (h, ffn), "b1": (ffn,),
              "W2": (ffn, h), "b2": (h,)}
    for name, shape in shapes.items():
        t = params[name]
        if t.dtype != torch.bfloat16 or tuple(t.shape) != shape:
            raise ValueError(f"{name} must be bf16 of shape {shape}")
    dev = x.device
    g = {"dx": torch.empty((b, s, h), dtype=torch.float32, device=dev)}
    for name, shape in shapes.items():
        g["d" + name] = torch.empty(shape, dtype=torch.float32, device=dev)
    nbytes = int(lib().bpt_layer_backward_workspace_bytes(b, s, h, heads, ffn))
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    p = params
    outs = [_ptr(g[k]) for k in ("dx", "dWqkv", "dbqkv", "dWo", "dbo", "dW1", "db1", "dW2", "db2")]
    if saved is None:
        r = lib().bpt_layer_backward(_ptr(x), _ptr(p["Wqkv"]), _ptr(p["bqkv"]), _ptr(p["Wo"]), _ptr(p["bo"]),
                                     _ptr(p["W1"]), _ptr(p["b1"]), _ptr(p["W2"]), _ptr(p["b2"]), _ptr(dy), b, s, h,
                                     heads, ffn, int(bool(causal)), *outs, _ptr(ws), ws.numel(), _stream(stream))
        _check(r, "bpt_layer_backward")
        return g
    o, lse2 = saved
    if o.dtype != torch.bfloat16 or tuple(o.shape) != (b, s, h):
        raise ValueError("saved o must be bf16 [b, s, h]")
    if lse2.dtype != torch.float32 or tuple(lse2.shape) != (b, heads, s):
        raise ValueError("saved lse2 must be fp32 [b, heads, s]")
    r = lib().bpt_layer_backward_saved(_ptr(x), _ptr(p["Wqkv"]), _ptr(p["bqkv"]), _ptr(p["Wo"]), _ptr(p["bo"]),
                                       _ptr(p["W1"]), _ptr(p["b1"]), _ptr(p["W2"]), _ptr(p["b2"]), _ptr(o),
                                       _ptr(lse2), _ptr(dy), b, s, h, heads, ffn, int(bool(causal)), *outs, _ptr(ws),
                                       ws.numel(), _stream(stream))
    _check(r, "bpt_layer_backward_saved")
    return g


def ffn_backward(hid: torch.Tensor, W1: torch.Tensor, b1: torch.Tensor, W2: torch.Tensor, dy: torch.Tensor,
                 chunk_rows: int = 0, stream: Optional[torch.cuda.Stream] = None) -> dict:
    """Gradients of the FFN block out = hid + max(0, hid W1 + b1) W2 + b2 for
    dy = dL/dout (bpt_ffn_backward): hid, dy fp32 [..., h] on the GPU; W1, b1,
    W2 bf16. Returns {"dhid", "dW1", "db1", "dW2", "db2"} (fp32)."""
    h = hid.shape[-1]
    ffn = W1.shape[-1]
    rows = hid.numel() // h
    if hid.dtype != torch.float32 or dy.dtype != torch.float32 or dy.shape != hid.shape:
        raise TypeError("hid and dy must be fp32 tensors of the same shape")
    for name, t, shape in (("W1", W1, (h, ffn)), ("b1", b1, (ffn,)), ("W2", W2, (ffn, h))):
        if t.dtype != torch.bfloat16 or tuple(t.shape) != shape:
            raise ValueError(f"{name} must be bf16 of shape {shape}")
    dev = hid.device
    g = {"dhid": torch.empty_like(hid), "dW1": torch.empty((h, ffn), dtype=torch.float32, device=dev),
         "db1": torch.empty(ffn, dtype=torch.float32, device=dev),
         "dW2": torch.empty((ffn, h), dtype=torch.float32, device=dev),
         "db2": torch.empty(h, dtype=torch.float32, device=dev)}
    nbytes = int(lib().bpt_ffn_backward_workspace_bytes(rows, h, ffn, chunk_rows))
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    r = lib().bpt_ffn_backward(_ptr(hid), _ptr(W1), _ptr(b1), _ptr(W2), _ptr(dy), rows, h, ffn, chunk_rows,
                               _ptr(g["dhid"]), _ptr(g["dW1"]), _ptr(g["db1"]), _ptr(g["dW2"]), _ptr(g["db2"]),
                               _ptr(ws), ws.numel(), _stream(stream))
    _check(r, "bpt_ffn_backward")
    return g


def stream_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronise `stream` (default: the current stream) and return, then
    clear, the status word of the library's work queued on it (0 = BPT_OK)."""
    return int(lib().bpt_stream_status(_stream(stream)))


def device_status() -> int:
    """Synchronise the whole device and return, then clear, the status words
    of every stream of it (0 = BPT_OK). Stalls every stream; prefer
    stream_status."""
    return int(lib().bpt_device_status())


def wait_flag(flag: torch.Tensor, value: int, timeout_us: int, stream: Optional[torch.cuda.Stream] = None) -> None:
    """Queue a bounded wait on `stream` until flag[0] (an int32 CUDA tensor)
    equals value; if it gives up after timeout_us, the stream's status word
    records BPT_ERR_TIMEOUT (a check of the status path)."""
    if flag.dtype != torch.int32 or not flag.is_cuda:
        raise TypeError("flag must be an int32 CUDA tensor")
    _check(lib().bpt_wait_flag(_ptr(flag), int(value), int(timeout_us), _stream(stream)), "bpt_wait_flag")


def launch_count() -> int:
    return int(lib().bpt_launch_count())


def set_kernel_timing(enable: bool) -> None:
    _check(lib().bpt_set_kernel_timing(int(bool(enable))), "bpt_set_kernel_timing")


def kernel_times(max_kinds: int = 32) -> dict:
    """{kernel name: (launches, total ms)} since timing was enabled or last read."""
    arr = (KernelTime * max_kinds)()
    n = lib().bpt_kernel_times(arr, max_kinds)
    if n < 0:
        raise BPTError(n, "bpt_kernel_times")
    return {arr[i].name.decode(): (arr[i].launches, arr[i].total_ms) for i in range(n)}
