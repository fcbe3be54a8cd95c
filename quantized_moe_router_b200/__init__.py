"""Python binding of the quantized MoE expert block's C ABI (include/moe.h).

Argument marshalling only: every step of the block runs in the CUDA library
``libmoe_b200.so`` built in-tree by ``quantized_moe_router_b200/build.py``. PyTorch provides
device memory and streams. There is no fallback: if the library is missing or the device is
not an sm_100a GPU, the calls raise.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE_CHECK = range(6)
MODE_DECODE, MODE_PREFILL = 0, 1

# every C entry point of include/moe.h with its ctypes signature
_vp, _i, _sz, _u64 = C.c_void_p, C.c_int, C.c_size_t, C.c_uint64
SIGNATURES = {
    "moe_status_str": (C.c_char_p, [_i]),
    "moe_abi_version": (_i, []),
    "moe_packed_layer_bytes": (_sz, [_i, _i, _i, _vp]),
    "moe_pack_layer": (_i, [_vp, _i, _i, _i, _vp, _sz, _vp]),
    "moe_route_topk": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp]),
    "moe_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "moe_workspace_init": (_i, [_vp, _sz, _vp]),
    "moe_expert_forward_decode": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_expert_forward_prefill": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_expert_forward_decode_noalloc": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "moe_noalloc_get_device_status": (_i, [_vp]),
    "moe_prefill_route": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _sz, _vp]),
    "moe_prefill_experts": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _sz, _vp]),
    "moe_get_device_status": (_i, [_vp, _vp]),
    "moe_set_wait_limit_ns": (None, [_u64]),
    "moe_quantize_hqq": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_cache_pool_bytes": (_sz, [_i, _vp, _vp, _i]),
    "moe_cache_create": (_i, [_i, _vp, _vp, _i, _i, _vp, _sz, _vp]),
    "moe_cache_destroy": (None, [_vp]),
    "moe_cache_request": (_i, [_vp, _i, _vp, _i, _vp, _vp, _vp]),
    "moe_cache_commit": (_i, [_vp, _vp, _vp]),
    "moe_cache_slot_of": (_i, [_vp, _i, _i]),
    "moe_cache_stats": (_i, [_vp, _vp, _vp, _vp]),
}


class HqqParams(C.Structure):
    """moe_hqq_params_t"""
    _fields_ = [("lp_norm", C.c_double), ("beta", C.c_double), ("kappa", C.c_double),
                ("iters", C.c_int32)]


class ExpertSrc(C.Structure):
    """moe_expert_src_t"""
    _fields_ = [("codes", C.c_void_p * 3), ("scale", C.c_void_p * 3), ("zero", C.c_void_p * 3),
                ("bits", C.c_int32)]


class MoeError(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what} failed: {status_name(status)}")
        self.status = status


_lib: Optional[C.CDLL] = None


def lib() -> C.CDLL:
    """The loaded CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library {LIB_PATH} is missing; run quantized_moe_router_b200/build.py "
                               "(or __graft_entry__.build())")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_name(status: int) -> str:
    return lib().moe_status_str(status).decode()


def _check(status: int, what: str) -> None:
    if status != MOE_OK:
        raise MoeError(what, status)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _p(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _dev(t: Optional[torch.Tensor], name: str, dtype, shape=None, optional: bool = False) -> None:
    """Checks that a tensor handed to the library is a contiguous CUDA tensor of the expected
    dtype (and shape) on the current device. The C ABI takes raw device pointers, so a host
    tensor, another GPU's tensor or a strided view must be refused here, before any launch."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} must have dtype {dtype}, not {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}, but the current device is cuda:{torch.cuda.current_device()}")


_F16 = (torch.float16, torch.int16, torch.uint16) if hasattr(torch, "uint16") else (torch.float16, torch.int16)


def _x_shape(x: torch.Tensor, name: str = "x"):
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise ValueError(f"{name} must be a 2-D [T, H] tensor")
    return x.shape


def _check_block_args(x, w_router, bias, k, idx_out, w_out):
    T, H = _x_shape(x)
    _dev(x, "x", torch.bfloat16)
    if not isinstance(w_router, torch.Tensor) or w_router.dim() != 2:
        raise ValueError("w_router must be a 2-D [E, H] tensor")
    E = w_router.shape[0]
    _dev(w_router, "w_router", torch.float32, (E, H))
    _dev(bias, "bias", torch.float32, (E,), optional=True)
    _dev(idx_out, "idx_out", torch.int32, (T, k), optional=True)
    _dev(w_out, "w_out", torch.float32, (T, k), optional=True)
    return T, H, E


# ------------------------------------------------------------------------------ weights

def packed_layer_bytes(E: int, H: int, I: int, bits: Sequence[int]) -> int:
    arr = (C.c_int32 * E)(*[int(b) for b in bits])
    n = lib().moe_packed_layer_bytes(E, H, I, C.cast(arr, C.c_void_p))
    if n == 0:
        raise MoeError("moe_packed_layer_bytes", MOE_ERR_INVALID_ARG)
    return n


def pack_layer(experts: Sequence[dict], H: int, I: int, out: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """experts[e] = {"bits": b, "codes": [3 uint8 tensors], "scale": [3 fp16/int16 tensors],
    "zero": [...]} on the GPU, canonical layout. Returns the packed layer (uint8 tensor)."""
    E = len(experts)
    bits = [int(ex["bits"]) for ex in experts]
    nbytes = packed_layer_bytes(E, H, I, bits)
    for e, ex in enumerate(experts):
        for m, (rows, cols) in enumerate(((I, H), (I, H), (H, I))):
            _dev(ex["codes"][m], f"experts[{e}].codes[{m}]", torch.uint8, (rows, cols * bits[e] // 8))
            _dev(ex["scale"][m], f"experts[{e}].scale[{m}]", _F16, (rows, cols // 64))
            _dev(ex["zero"][m], f"experts[{e}].zero[{m}]", _F16, (rows, cols // 64))
    dev = experts[0]["codes"][0].device
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _dev(out, "out", torch.uint8)
    if out.numel() < nbytes:
        raise ValueError(f"out holds {out.numel()} bytes, the packed layer needs {nbytes}")
    src = (ExpertSrc * E)()
    for e, ex in enumerate(experts):
        for m in range(3):
            src[e].codes[m] = ex["codes"][m].data_ptr()
            src[e].scale[m] = ex["scale"][m].data_ptr()
            src[e].zero[m] = ex["zero"][m].data_ptr()
        src[e].bits = bits[e]
    _check(lib().moe_pack_layer(C.cast(src, C.c_void_p), E, H, I, out.data_ptr(), out.numel(), _stream(stream)),
           "moe_pack_layer")
    return out


HQQ_DEFAULTS = {"lp_norm": 0.7, "beta": 10.0, "kappa": 1.01, "iters": 20}


def quantize_hqq(w: torch.Tensor, bits: int, lp_norm: float = 0.7, beta: float = 10.0,
                 kappa: float = 1.01, iters: int = 20, with_iters: bool = False, stream=None):
    """HQQ-style quantisation of bf16 weights [rows, cols] (CUDA, contiguous) into the canonical
    format: returns (codes uint8 [rows, cols*bits//8], scale fp16 [rows, cols//64],
    zero fp16 [rows, cols//64]) and, with ``with_iters``, the int32 steps run per group."""
    rows, cols = _x_shape(w, "w")
    _dev(w, "w", torch.bfloat16)
    dev = w.device
    codes = torch.empty((rows, cols * bits // 8), dtype=torch.uint8, device=dev)
    scale = torch.empty((rows, cols // 64), dtype=torch.float16, device=dev)
    zero = torch.empty((rows, cols // 64), dtype=torch.float16, device=dev)
    it = torch.empty((rows, cols // 64), dtype=torch.int32, device=dev) if with_iters else None
    prm = HqqParams(float(lp_norm), float(beta), float(kappa), int(iters))
    _check(lib().moe_quantize_hqq(_p(w), rows, cols, bits, C.addressof(prm), _p(codes), _p(scale), _p(zero),
                                  _p(it), _stream(stream)), "moe_quantize_hqq")
    return (codes, scale, zero, it) if with_iters else (codes, scale, zero)


class ExpertCache:
    """Expert cache of include/moe.h (moe_cache_*): the packed layers stay in host memory
    (``host_layers``: 1-D uint8 CPU tensors as moe_pack_layer wrote them, ideally pinned) and a
    device pool of ``slots`` expert slots holds the experts that calls need, behind one packed
    header per layer. Marshalling only; the policy and the copies are the library's."""

    def __init__(self, host_layers: Sequence[torch.Tensor], slots: int, keep_recent: int = 1,
                 device="cuda"):
        for l, t in enumerate(host_layers):
            if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.uint8 or t.dim() != 1 \
                    or not t.is_contiguous():
                raise ValueError(f"host_layers[{l}] must be a contiguous 1-D uint8 CPU tensor")
        self.host_layers = list(host_layers)   # kept alive: the library reads them at every commit
        L = len(self.host_layers)
        self._ptrs = (C.c_void_p * L)(*[t.data_ptr() for t in self.host_layers])
        self._sizes = (C.c_size_t * L)(*[t.numel() for t in self.host_layers])
        n = lib().moe_cache_pool_bytes(L, C.cast(self._ptrs, C.c_void_p), C.cast(self._sizes, C.c_void_p), slots)
        if n == 0:
            raise MoeError("moe_cache_pool_bytes", MOE_ERR_INVALID_ARG)
        self.pool = torch.empty(n, dtype=torch.uint8, device=device)
        h = C.c_void_p()
        _check(lib().moe_cache_create(L, C.cast(self._ptrs, C.c_void_p), C.cast(self._sizes, C.c_void_p), slots,
                                      keep_recent, self.pool.data_ptr(), n, C.byref(h)), "moe_cache_create")
        self._h = h
        self.slots = slots

    def request(self, layer: int, experts: Sequence[int]):
        """Host work only: returns (missing experts, their slots) of this request."""
        ids = [int(e) for e in experts]
        arr = (C.c_int32 * max(1, len(ids)))(*ids)
        le = (C.c_int32 * max(1, len(ids)))()
        ls = (C.c_int32 * max(1, len(ids)))()
        nl = C.c_int()
        _check(lib().moe_cache_request(self._h, layer, C.cast(arr, C.c_void_p), len(ids), C.cast(le, C.c_void_p),
                                       C.cast(ls, C.c_void_p), C.byref(nl)), "moe_cache_request")
        return list(le[:nl.value]), list(ls[:nl.value])

    def commit(self, stream=None) -> torch.Tensor:
        """Copies of the current request and its layer's header, on `stream`; returns the layer's
        packed header as a uint8 view of the pool, for the forward calls."""
        out = C.c_void_p()
        _check(lib().moe_cache_commit(self._h, _stream(stream), C.byref(out)), "moe_cache_commit")
        return self.pool[out.value - self.pool.data_ptr():]

    def prepare(self, layer: int, experts: Sequence[int], stream=None) -> torch.Tensor:
        self.request(layer, experts)
        return self.commit(stream)

    def slot_of(self, layer: int, expert: int) -> int:
        return lib().moe_cache_slot_of(self._h, layer, expert)

    def stats(self):
        h, m, e = C.c_uint64(), C.c_uint64(), C.c_uint64()
        _check(lib().moe_cache_stats(self._h, C.byref(h), C.byref(m), C.byref(e)), "moe_cache_stats")
        return {"hits": h.value, "misses": m.value, "evictions": e.value}

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib().moe_cache_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001 - interpreter shutdown
            pass


# ------------------------------------------------------------------------------ routing

def route_topk(x: torch.Tensor, w_router: torch.Tensor, bias: Optional[torch.Tensor], k: int,
               idx_out: Optional[torch.Tensor] = None, w_out: Optional[torch.Tensor] = None, stream=None):
    T, H, E = _check_block_args(x, w_router, bias, k, idx_out, w_out)
    if idx_out is None:
        idx_out = torch.empty((T, k), dtype=torch.int32, device=x.device)
    if w_out is None:
        w_out = torch.empty((T, k), dtype=torch.float32, device=x.device)
    _check(lib().moe_route_topk(_p(x), _p(w_router), _p(bias), T, H, E, k, _p(idx_out), _p(w_out),
                                _stream(stream)), "moe_route_topk")
    return idx_out, w_out


# ------------------------------------------------------------------------------ expert block

def workspace_bytes(T: int, H: int, I: int, E: int, k: int, mode: int) -> int:
    n = lib().moe_workspace_bytes(T, H, I, E, k, mode)
    if n == 0:
        raise MoeError("moe_workspace_bytes", MOE_ERR_INVALID_ARG)
    return n


def workspace(T: int, H: int, I: int, E: int, k: int, mode: int, device="cuda", stream=None) -> torch.Tensor:
    ws = torch.empty(workspace_bytes(T, H, I, E, k, mode), dtype=torch.uint8, device=device)
    _check(lib().moe_workspace_init(ws.data_ptr(), ws.numel(), _stream(stream)), "moe_workspace_init")
    return ws


def _forward(fn, what, x, w_router, bias, packed, I, E, k, ws, out, idx_out, w_out, stream):
    T, H, E_r = _check_block_args(x, w_router, bias, k, idx_out, w_out)
    if E_r != E:
        raise ValueError(f"w_router has {E_r} rows, E = {E}")
    _dev(packed, "packed", torch.uint8)
    _dev(ws, "ws", torch.uint8)
    _dev(out, "out", torch.bfloat16, (T, H), optional=True)
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    _check(fn(_p(x), _p(w_router), _p(bias), _p(packed), T, H, I, E, k, _p(out), _p(idx_out), _p(w_out),
              _p(ws), ws.numel(), _stream(stream)), what)
    return out


def forward_decode(x, w_router, bias, packed, I, E, k, ws, out=None, idx_out=None, w_out=None, stream=None):
    """Decode-path expert block (T <= 32): returns out [T x H] bf16."""
    return _forward(lib().moe_expert_forward_decode, "moe_expert_forward_decode", x, w_router, bias, packed,
                    I, E, k, ws, out, idx_out, w_out, stream)


def forward_prefill(x, w_router, bias, packed, I, E, k, ws, out=None, idx_out=None, w_out=None, stream=None):
    """Prefill-path expert block (any T): returns out [T x H] bf16."""
    return _forward(lib().moe_expert_forward_prefill, "moe_expert_forward_prefill", x, w_router, bias, packed,
                    I, E, k, ws, out, idx_out, w_out, stream)


def prefill_route(x, w_router, bias, I, E, k, ws, idx_out=None, w_out=None, stream=None):
    """Routing and bucketing of the prefill path into the workspace `ws`."""
    T, H, E_r = _check_block_args(x, w_router, bias, k, idx_out, w_out)
    if E_r != E:
        raise ValueError(f"w_router has {E_r} rows, E = {E}")
    _dev(ws, "ws", torch.uint8)
    _check(lib().moe_prefill_route(_p(x), _p(w_router), _p(bias), T, H, I, E, k, _p(idx_out), _p(w_out), _p(ws),
                                   ws.numel(), _stream(stream)), "moe_prefill_route")


def prefill_experts(x, packed, I, E, k, ws, out=None, stream=None):
    """Expert GEMMs and combine over the buckets of the last prefill_route on `ws`; returns out."""
    T, H = _x_shape(x)
    _dev(x, "x", torch.bfloat16)
    _dev(packed, "packed", torch.uint8)
    _dev(ws, "ws", torch.uint8)
    _dev(out, "out", torch.bfloat16, (T, H), optional=True)
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    _check(lib().moe_prefill_experts(_p(x), _p(packed), T, H, I, E, k, _p(out), _p(ws), ws.numel(), _stream(stream)),
           "moe_prefill_experts")
    return out


def forward_decode_noalloc(x, w_router, bias, packed, I, E, k, out=None, idx_out=None, w_out=None, stream=None):
    """Decode-path expert block using the library's fixed device scratch (no workspace)."""
    T, H, E_r = _check_block_args(x, w_router, bias, k, idx_out, w_out)
    if E_r != E:
        raise ValueError(f"w_router has {E_r} rows, E = {E}")
    _dev(packed, "packed", torch.uint8)
    _dev(out, "out", torch.bfloat16, (T, H), optional=True)
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    _check(lib().moe_expert_forward_decode_noalloc(_p(x), _p(w_router), _p(bias), _p(packed), T, H, I, E, k,
                                                   _p(out), _p(idx_out), _p(w_out), _stream(stream)),
           "moe_expert_forward_decode_noalloc")
    return out


def noalloc_device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the status of the fixed scratch array
    that forward_decode_noalloc uses on the current device."""
    return lib().moe_noalloc_get_device_status(_stream(stream))


def device_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronises the stream and returns (and clears) the workspace's device status."""
    _dev(ws, "ws", torch.uint8)
    return lib().moe_get_device_status(ws.data_ptr(), _stream(stream))


def set_wait_limit_ns(ns: int) -> None:
    lib().moe_set_wait_limit_ns(int(ns))
