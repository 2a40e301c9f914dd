"""Python binding of libmoe_mx.so: argument marshalling only.

Every function here has the name of the C entry point it calls (see
include/moe_mx.h) and passes device pointers (``tensor.data_ptr()``), sizes and
the current CUDA stream through ctypes; all computation happens in the
library's CUDA kernels.  PyTorch is used only for device memory and streams.

The library is loaded on first use.  If it is missing or fails to load, the
call raises ``RuntimeError`` -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_mx.so")

MOE_MX_OK = 0
MOE_MX_ERR_INVALID_ARG = -1
MOE_MX_ERR_UNSUPPORTED = -2
MOE_MX_ERR_CUDA = -3
MOE_MX_ERR_TIMEOUT = -4
MOE_MX_ERR_NO_MEMORY = -5
MOE_MX_ACT_BF16 = 0
MOE_MX_ACT_MXFP8 = 1
MOE_MX_OUT_BF16 = 0
MOE_MX_OUT_F32 = 1
MOE_MX_FMT_MXFP4 = 0
MOE_MX_FMT_MXFP8 = 1
MOE_MX_SCALES_ROW_MAJOR = 0
MOE_MX_SCALES_TILED = 1
MOE_MX_W1 = 0
MOE_MX_W2 = 1
MOE_MX_INTER_AQ = 0
MOE_MX_INTER_ASF = 1
MOE_MX_INTER_HQ = 2
MOE_MX_INTER_HSF = 3
MOE_MX_INTER_Y = 4

# Every symbol include/moe_mx.h declares: name -> (restype, argtypes)
_P, _I, _I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
SIGNATURES = {
    "moe_mx_create": (_I, [ctypes.POINTER(_P), _I, _I, _I, _I, _I, _I]),
    "moe_mx_create_ex": (_I, [ctypes.POINTER(_P), _I, _I, _I, _I, _I, _I, _I]),
    "moe_mx_forward": (_I, [_P, _P, _P, _I, _P, _P, _P, _P, _I, _I, _P, _P]),
    "moe_mx_forward_routed": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _P, _I, _P, _I, _P]),
    "moe_mx_forward_shard": (_I, [_P, _P, _P, _I, _I, _I, _P, _P, _P, _P, _I, _I, _P, _I, _P]),
    "moe_mx_destroy": (_I, [_P]),
    "moe_mx_last_error": (ctypes.c_char_p, []),
    "moe_mx_sync_status": (_I, [_P, _P]),
    "moe_mx_quantize": (_I, [_P, _I64, _I64, _I, _P, _P, _P]),
    "moe_mx_block_rows": (_I, []),
    "moe_mx_max_grouped_rows": (_I64, [_P, _I, _I]),
    "moe_mx_get_routing": (_I, [_P, _P, _P, _P, _P, _P, _P]),
    "moe_mx_debug_watchdog": (_I, [_P, _I, _P]),
    "moe_mx_set_stage_timing": (_I, [_P, _I]),
    "moe_mx_get_stage_times": (_I, [_P, _P]),
    "moe_mx_route_group_noalloc": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "moe_mx_prepare_scales": (_I, [_P, _I, _P, _P, _P]),
    "moe_mx_set_scale_layout": (_I, [_P, _I]),
    "moe_mx_get_intermediate": (_I, [_P, _I, _P, _P]),
    "moe_mx_launch_count": (ctypes.c_longlong, [_P]),
    "moe_mx_debug_encode_act": (_I, [_P, _I, _I, _I, _I, _P, _P, _P]),
}
STAGES = ("route", "gather", "fc1", "fc2", "combine")

_lock = threading.Lock()
_lib = None


class MoeMxError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"moe_mx error {code}: {msg}")
        self.code = code


def load_library(path: str = LIB_PATH):
    """Load libmoe_mx.so (built by ``python -m block_scaled_moe_softmax_b200.build``)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m block_scaled_moe_softmax_b200.build`;"
                               " there is no fallback implementation")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def _check(code: int):
    if code != MOE_MX_OK:
        raise MoeMxError(code, moe_mx_last_error())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def moe_mx_last_error() -> str:
    return load_library().moe_mx_last_error().decode()


def moe_mx_block_rows() -> int:
    return load_library().moe_mx_block_rows()


def moe_mx_create(hidden: int, inter: int, num_experts: int, max_tokens: int, max_top_k: int,
                  device: int = 0) -> int:
    h = ctypes.c_void_p()
    _check(load_library().moe_mx_create(ctypes.byref(h), hidden, inter, num_experts, max_tokens, max_top_k,
                                        device))
    return h.value


def moe_mx_create_ex(hidden: int, inter: int, num_experts: int, num_shared: int, max_tokens: int, max_top_k: int,
                     device: int = 0) -> int:
    h = ctypes.c_void_p()
    _check(load_library().moe_mx_create_ex(ctypes.byref(h), hidden, inter, num_experts, num_shared, max_tokens,
                                           max_top_k, device))
    return h.value


def moe_mx_destroy(handle: int) -> None:
    _check(load_library().moe_mx_destroy(handle))


def moe_mx_forward(handle: int, x, router_logits, num_tokens: int, w1, w1_scale, w2, w2_scale, top_k: int,
                   act_dtype: int, out, stream=None) -> None:
    _check(load_library().moe_mx_forward(handle, _ptr(x), _ptr(router_logits), num_tokens, _ptr(w1),
                                         _ptr(w1_scale), _ptr(w2), _ptr(w2_scale), top_k, act_dtype, _ptr(out),
                                         _stream(stream)))


def moe_mx_forward_routed(handle: int, x, topk_ids, topk_w, num_tokens: int, top_k: int, local_expert_offset: int,
                          w1, w1_scale, w2, w2_scale, act_dtype: int, out, out_dtype: int = MOE_MX_OUT_BF16,
                          stream=None) -> None:
    _check(load_library().moe_mx_forward_routed(handle, _ptr(x), _ptr(topk_ids), _ptr(topk_w), num_tokens, top_k,
                                                local_expert_offset, _ptr(w1), _ptr(w1_scale), _ptr(w2),
                                                _ptr(w2_scale), act_dtype, _ptr(out), out_dtype, _stream(stream)))


def moe_mx_forward_shard(handle: int, x, router_logits, num_tokens: int, num_experts_global: int,
                         local_expert_offset: int, w1, w1_scale, w2, w2_scale, top_k: int, act_dtype: int, out,
                         out_dtype: int = MOE_MX_OUT_F32, stream=None) -> None:
    _check(load_library().moe_mx_forward_shard(handle, _ptr(x), _ptr(router_logits), num_tokens, num_experts_global,
                                               local_expert_offset, _ptr(w1), _ptr(w1_scale), _ptr(w2),
                                               _ptr(w2_scale), top_k, act_dtype, _ptr(out), out_dtype,
                                               _stream(stream)))


def moe_mx_sync_status(handle: int, stream=None) -> int:
    """Returns the status code (does not raise on MOE_MX_ERR_TIMEOUT)."""
    return load_library().moe_mx_sync_status(handle, _stream(stream))


def moe_mx_quantize(src, rows: int, K: int, fmt: int, codes, scales, stream=None) -> None:
    _check(load_library().moe_mx_quantize(_ptr(src), rows, K, fmt, _ptr(codes), _ptr(scales), _stream(stream)))


def moe_mx_max_grouped_rows(handle: int, num_tokens: int, top_k: int) -> int:
    return load_library().moe_mx_max_grouped_rows(handle, num_tokens, top_k)


def moe_mx_get_routing(handle: int, topk_ids=None, topk_w=None, counts=None, pad_offsets=None, sorted_pair=None,
                       stream=None) -> None:
    _check(load_library().moe_mx_get_routing(handle, _ptr(topk_ids), _ptr(topk_w), _ptr(counts),
                                             _ptr(pad_offsets), _ptr(sorted_pair), _stream(stream)))


def moe_mx_route_group_noalloc(router_logits, num_tokens: int, num_experts: int, top_k: int, topk_ids, topk_w,
                               counts, pad_offsets, sorted_pair, pos_of_pair, stream=None) -> None:
    """Routing + grouping into caller buffers, with no handle and no device allocation (see the header)."""
    _check(load_library().moe_mx_route_group_noalloc(
        _ptr(router_logits), num_tokens, num_experts, top_k, _ptr(topk_ids), _ptr(topk_w), _ptr(counts),
        _ptr(pad_offsets), _ptr(sorted_pair), _ptr(pos_of_pair), _stream(stream)))


def moe_mx_launch_count(handle: int) -> int:
    """Kernels launched by the handle's forwards since it was created (host-side count)."""
    return load_library().moe_mx_launch_count(handle)


def moe_mx_get_intermediate(handle: int, which: int, dst, stream=None) -> None:
    """Copy one intermediate buffer of the last forward (MOE_MX_INTER_*) into dst (see the header)."""
    _check(load_library().moe_mx_get_intermediate(handle, which, _ptr(dst), _stream(stream)))


def moe_mx_debug_encode_act(src, rows: int, K: int, act_dtype: int, method: int, codes, scale_atoms,
                            stream=None) -> None:
    """The forward's activation encoders on float32 rows (see the header)."""
    _check(load_library().moe_mx_debug_encode_act(_ptr(src), rows, K, act_dtype, method, _ptr(codes),
                                                  _ptr(scale_atoms), _stream(stream)))


def moe_mx_prepare_scales(handle: int, which: int, src, dst, stream=None) -> None:
    """Rearrange one row-major E8M0 weight-scale tensor into the tiled layout (see the header)."""
    _check(load_library().moe_mx_prepare_scales(handle, which, _ptr(src), _ptr(dst), _stream(stream)))


def moe_mx_set_scale_layout(handle: int, layout: int) -> None:
    _check(load_library().moe_mx_set_scale_layout(handle, layout))


def moe_mx_debug_watchdog(handle: int, timeout_us: int, stream=None) -> None:
    _check(load_library().moe_mx_debug_watchdog(handle, timeout_us, _stream(stream)))


def moe_mx_set_stage_timing(handle: int, enable: bool) -> None:
    _check(load_library().moe_mx_set_stage_timing(handle, int(bool(enable))))


def moe_mx_get_stage_times(handle: int) -> dict:
    ms = (ctypes.c_float * len(STAGES))()
    _check(load_library().moe_mx_get_stage_times(handle, ctypes.cast(ms, ctypes.c_void_p)))
    return dict(zip(STAGES, [float(v) for v in ms]))


# ------------------------------------------------------------------ convenience wrappers
class MoeMxLayer:
    """Owns a moe_mx handle for fixed (H, I, E) and runs forwards on torch tensors."""

    def __init__(self, hidden: int, inter: int, num_experts: int, max_tokens: int, max_top_k: int,
                 device: int | None = None, num_shared: int = 0):
        """num_experts routed experts; num_shared > 0 adds a shared expert held as that many
        extra expert slots of the weights (see moe_mx_create_ex)."""
        self.H, self.I, self.E, self.S = hidden, inter, num_experts, num_shared
        self.device = torch.cuda.current_device() if device is None else device
        self.handle = moe_mx_create_ex(hidden, inter, num_experts, num_shared, max_tokens, max_top_k, self.device)

    def forward(self, x: torch.Tensor, router_logits: torch.Tensor, w1, w1_scale, w2, w2_scale, top_k: int,
                act_dtype: int = MOE_MX_ACT_BF16, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        T = x.shape[0]
        if out is None:
            out = torch.empty(T, self.H, dtype=torch.bfloat16, device=x.device)
        moe_mx_forward(self.handle, x, router_logits, T, w1, w1_scale, w2, w2_scale, top_k, act_dtype, out, stream)
        return out

    def forward_routed(self, x: torch.Tensor, topk_ids: torch.Tensor, topk_w: torch.Tensor, w1, w1_scale, w2,
                       w2_scale, local_expert_offset: int = 0, act_dtype: int = MOE_MX_ACT_BF16,
                       out_dtype: int = MOE_MX_OUT_BF16, out: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
        """The layer with the routing given (global ids, weights) for the local shard of E experts
        starting at global id local_expert_offset; MOE_MX_OUT_F32 returns the shard's float32
        partial output."""
        T, k = topk_ids.shape
        if out is None:
            dt = torch.float32 if out_dtype == MOE_MX_OUT_F32 else torch.bfloat16
            out = torch.empty(T, self.H, dtype=dt, device=x.device)
        moe_mx_forward_routed(self.handle, x, topk_ids, topk_w, T, k, local_expert_offset, w1, w1_scale, w2,
                              w2_scale, act_dtype, out, out_dtype, stream)
        return out

    def forward_shard(self, x: torch.Tensor, router_logits: torch.Tensor, w1, w1_scale, w2, w2_scale, top_k: int,
                      local_expert_offset: int, act_dtype: int = MOE_MX_ACT_BF16, out_dtype: int = MOE_MX_OUT_F32,
                      out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """The layer routed from the whole layer's logits [T, E_global], over this handle's shard of
        E experts starting at global id local_expert_offset: the shard's partial output (float32
        by default, for a sum over the expert-parallel group)."""
        T, E_global = router_logits.shape
        if out is None:
            dt = torch.float32 if out_dtype == MOE_MX_OUT_F32 else torch.bfloat16
            out = torch.empty(T, self.H, dtype=dt, device=x.device)
        moe_mx_forward_shard(self.handle, x, router_logits, T, E_global, local_expert_offset, w1, w1_scale, w2,
                             w2_scale, top_k, act_dtype, out, out_dtype, stream)
        return out

    def prepare_scales(self, w1_scale: torch.Tensor, w2_scale: torch.Tensor, stream=None):
        """Tiled copies of both weight-scale tensors; later forwards of this layer read that layout."""
        t1, t2 = torch.empty_like(w1_scale), torch.empty_like(w2_scale)
        moe_mx_prepare_scales(self.handle, MOE_MX_W1, w1_scale, t1, stream)
        moe_mx_prepare_scales(self.handle, MOE_MX_W2, w2_scale, t2, stream)
        moe_mx_set_scale_layout(self.handle, MOE_MX_SCALES_TILED)
        return t1, t2

    def routing(self, T: int, top_k: int, stream=None):
        """The routing/grouping state of the most recent forward (device tensors)."""
        dev = torch.device("cuda", self.device)
        rows = moe_mx_max_grouped_rows(self.handle, T, top_k)
        slots = top_k + self.S  # the routed slots, then the shared expert's chunks
        ids = torch.empty(T, slots, dtype=torch.int32, device=dev)
        w = torch.empty(T, slots, dtype=torch.float32, device=dev)
        counts = torch.empty(self.E + self.S, dtype=torch.int32, device=dev)
        pad = torch.empty(self.E + self.S + 1, dtype=torch.int32, device=dev)
        sp = torch.empty(rows, dtype=torch.int32, device=dev)
        moe_mx_get_routing(self.handle, ids, w, counts, pad, sp, stream)
        return ids, w, counts, pad, sp

    def intermediates(self, T: int, top_k: int, stream=None) -> dict:
        """The intermediate buffers of the most recent forward of T tokens (device tensors):
        aq [2, rows, H] / hq [2, rows, I] uint8 E4M3 codes, asf / hsf uint8 scale atoms,
        y float32 [rows, H]; rows = moe_mx_max_grouped_rows(T, top_k)."""
        dev = torch.device("cuda", self.device)
        rows = moe_mx_max_grouped_rows(self.handle, T, top_k)
        bufs = {
            "aq": torch.empty(2, rows, self.H, dtype=torch.uint8, device=dev),
            "asf": torch.empty(rows // 128 * (self.H // 128) * 1024, dtype=torch.uint8, device=dev),
            "hq": torch.empty(2, rows, self.I, dtype=torch.uint8, device=dev),
            "hsf": torch.empty(rows // 128 * (self.I // 128) * 1024, dtype=torch.uint8, device=dev),
            "y": torch.empty(rows, self.H, dtype=torch.float32, device=dev),
        }
        which = {"aq": MOE_MX_INTER_AQ, "asf": MOE_MX_INTER_ASF, "hq": MOE_MX_INTER_HQ, "hsf": MOE_MX_INTER_HSF,
                 "y": MOE_MX_INTER_Y}
        for name, t in bufs.items():
            moe_mx_get_intermediate(self.handle, which[name], t, stream)
        return bufs

    def sync_status(self, stream=None) -> int:
        return moe_mx_sync_status(self.handle, stream)

    def close(self):
        if getattr(self, "handle", None):
            moe_mx_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def quantize_mx(src: torch.Tensor, fmt: int = MOE_MX_FMT_MXFP4, stream=None):
    """GPU MX quantisation of a float32 CUDA tensor [..., K] along its last dim."""
    assert src.is_cuda and src.dtype == torch.float32 and src.is_contiguous()
    K = src.shape[-1]
    rows = src.numel() // K
    ncode = K // 2 if fmt == MOE_MX_FMT_MXFP4 else K
    codes = torch.empty(*src.shape[:-1], ncode, dtype=torch.uint8, device=src.device)
    scales = torch.empty(*src.shape[:-1], K // 32, dtype=torch.uint8, device=src.device)
    moe_mx_quantize(src, rows, K, fmt, codes, scales, stream)
    return codes, scales
