"""Python binding of libmoe_b200.so: one MoE layer's forward pass on a B200.

The functions ``moe_route``, ``moe_dispatch``, ``moe_experts``,
``moe_combine`` (and the helpers) carry the names of the C ABI in
``include/moe_b200.h`` and only marshal arguments: every step of the layer
runs in the library's CUDA kernels.  PyTorch supplies device memory and the
stream.  There is no fallback: if the library is missing or was built for
another GPU, the first call raises.

``MoELayerBuffers`` / ``moe_layer_forward`` chain the four stages the way the
DWDP README's "Runtime Integration Layer" orders them (router -> dispatcher
-> executor -> merger), with caller-owned buffers allocated once.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "MoEError", "lib_path", "load_library", "moe_abi_version", "moe_launch_count",
    "moe_last_error",
    "moe_route", "moe_route_grouped", "moe_dispatch_workspace_bytes", "moe_dispatch", "moe_dispatch_noalloc",
    "moe_experts_workspace_bytes",
    "moe_experts", "moe_experts_shared", "moe_combine", "moe_read_status", "moe_probe_wait_timeout",
    "MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_UNSUPPORTED", "MOE_ERR_CUDA", "MOE_ERR_TIMEOUT",
    "MOE_ERR_BAD_INDEX", "MOE_ERR_OVERFLOW", "MOE_F32", "MOE_BF16", "MOE_F16", "MoELayerBuffers",
    "moe_layer_forward", "moe_route_dispatch", "moe_route_gated", "route_dispatch_fits", "route_and_dispatch",
    "moe_layer_forward_host", "moe_gather", "moe_combine_range", "moe_finalize",
    "moe_ep_partition_workspace_bytes", "moe_ep_partition", "moe_ep_owner", "moe_ep_pack_ids",
    "MoELayerDesc", "MoELayer", "moe_test_set_wait_budget_ns",
]

(MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_TIMEOUT,
 MOE_ERR_BAD_INDEX, MOE_ERR_OVERFLOW) = range(7)
MOE_F32, MOE_BF16, MOE_F16 = 0, 1, 2

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None


class MoEError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[moe status {code}] {msg}")
        self.code = code


def lib_path() -> str:
    return os.path.join(_HERE, "libmoe_b200.so")


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t

_SIGS = {
    "moe_abi_version": (_I, []),
    "moe_launch_count": (ctypes.c_ulonglong, []),
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_route": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P]),
    "moe_dispatch_workspace_bytes": (_SZ, [_I, _I, _I]),
    "moe_dispatch": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "moe_dispatch_noalloc": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_experts_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I]),
    "moe_experts": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _SZ, _P, _P]),
    "moe_experts_shared": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _I, _P, _P, _I, _I, _I,
                                _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "moe_combine": (_I, [_P, _I, _P, _I, _I, _I, _P, _P, _I, _P, _P, _P]),
    "moe_read_status": (_I, [_P, _P, _P]),
    "moe_probe_wait_timeout": (_I, [_P, _I, _P]),
    "moe_gather": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P]),
    "moe_route_grouped": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P]),
    "moe_route_gated": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                             _P]),
    "moe_route_dispatch": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P,
                                _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_layer_workspace_bytes": (_SZ, [_P]),
    "moe_test_set_wait_budget_ns": (_I, [ctypes.c_ulonglong]),
    "moe_layer_create": (_I, [_P, _P, _SZ, _P, _P]),
    "moe_layer_destroy": (_I, [_P]),
    "moe_layer_forward": (_I, [_P, _P, _P, _P]),
    "moe_layer_forward_host": (_I, [_P, _P, _P, _P]),
    "moe_layer_join": (_I, [_P, _P]),
    "moe_layer_status": (_I, [_P, _P, _P]),
    "moe_layer_buffer": (_P, [_P, ctypes.c_char_p]),
    "moe_combine_range": (_I, [_P, _I, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _I, _P, _P, _P]),
    "moe_finalize": (_I, [_P, _I, _I, _I, _P, _P]),
    "moe_ep_partition_workspace_bytes": (_SZ, [_I, _I]),
    "moe_ep_owner": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "moe_ep_pack_ids": (_I, [_P, _P, _P, _I, _I, _I, _P, _P]),
    "moe_ep_partition": (_I, [_P, _SZ, _P, _SZ, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P,
                              _SZ, _P]),
}


def load_library():
    """Load libmoe_b200.so (once).  Raises if it is missing: no fallback exists."""
    global _LIB
    if _LIB is None:
        path = lib_path()
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m mixture_experts_layer_44_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    if t.dtype == torch.float32:
        return MOE_F32
    if t.dtype == torch.float16:
        return MOE_F16
    raise MoEError(MOE_ERR_INVALID_ARG, f"unsupported dtype {t.dtype}")


def _check(code: int):
    if code != MOE_OK:
        raise MoEError(code, load_library().moe_last_error().decode())


def moe_abi_version() -> int:
    return load_library().moe_abi_version()


def moe_launch_count() -> int:
    """Kernels this library has enqueued in this process so far."""
    return int(load_library().moe_launch_count())


def moe_last_error() -> str:
    return load_library().moe_last_error().decode()


def moe_route(x, W_gate, bias, k: int, renormalize: bool, logits, topk_ids=None, topk_w=None,
              status=None, stream=None):
    T, H = x.shape
    E = W_gate.shape[0]
    _check(load_library().moe_route(_ptr(x), _ptr(W_gate), _ptr(bias), T, H, E, k,
                                    int(bool(renormalize)), _dtype_code(x), _ptr(logits),
                                    _ptr(topk_ids), _ptr(topk_w), _ptr(status),
                                    _stream(stream)))


def moe_route_grouped(x, W_gate, bias, k: int, renormalize: bool, n_groups: int,
                      topk_groups: int, logits, topk_ids, topk_w, status=None, stream=None):
    """Group-limited router: top-k among the experts of the topk_groups best
    of n_groups consecutive-expert groups (a group scored by its best logit)."""
    T, H = x.shape
    E = W_gate.shape[0]
    _check(load_library().moe_route_grouped(
        _ptr(x), _ptr(W_gate), _ptr(bias), T, H, E, k, int(bool(renormalize)), n_groups,
        topk_groups, _dtype_code(x), _ptr(logits), _ptr(topk_ids), _ptr(topk_w), _ptr(status),
        _stream(stream)))


def route_dispatch_fits(T: int, H: int, E: int, k: int, gate: bool = False) -> bool:
    """Shapes moe_route_dispatch takes (one launch for router + dispatcher;
    with a shared expert's gate row, E + 1 rows)."""
    return 1 <= T <= 64 and 1 <= E and E + int(gate) <= 64 and H <= 32768 and 1 <= k <= min(E, 8)


def moe_route_dispatch(x, W_gate, bias, k: int, renormalize: bool, logits, topk_ids, topk_w,
                       counts, offsets, perm, inv_perm, packed_tok, packed_w, x_packed, counter,
                       status=None, stream=None, n_groups: int = 1, topk_groups: int = 1,
                       w_gate_shared=None, shared_gate_logit=None):
    """moe_route_grouped then moe_dispatch in one launch (T <= 64, E <= 64).
    ``counter``: one int32 on the device, zero before the first call.  With
    ``w_gate_shared`` [H] (a shared expert's gate row; E <= 63) the same launch
    also writes x . w_gate_shared into ``shared_gate_logit`` [T] f32."""
    T, H = x.shape
    E = W_gate.shape[0]
    _check(load_library().moe_route_dispatch(
        _ptr(x), _ptr(W_gate), _ptr(bias), _ptr(w_gate_shared), T, H, E, k,
        int(bool(renormalize)), n_groups, topk_groups, _dtype_code(x), _ptr(logits),
        _ptr(topk_ids), _ptr(topk_w), _ptr(shared_gate_logit), _ptr(counts), _ptr(offsets),
        _ptr(perm), _ptr(inv_perm), _ptr(packed_tok), _ptr(packed_w), _ptr(x_packed),
        _ptr(counter), _ptr(status), _stream(stream)))


def moe_route_gated(x, W_gate, bias, w_gate_shared, k: int, renormalize: bool, logits,
                    topk_ids, topk_w, shared_gate_logit, status=None, stream=None,
                    n_groups: int = 1, topk_groups: int = 1):
    """moe_route_grouped plus a shared expert's gate logit x . w_gate_shared
    into ``shared_gate_logit`` [T] f32, in the router's own launch where it
    has room for it."""
    T, H = x.shape
    E = W_gate.shape[0]
    _check(load_library().moe_route_gated(
        _ptr(x), _ptr(W_gate), _ptr(bias), _ptr(w_gate_shared), T, H, E, k,
        int(bool(renormalize)), n_groups, topk_groups, _dtype_code(x), _ptr(logits),
        _ptr(topk_ids), _ptr(topk_w), _ptr(shared_gate_logit), _ptr(status), _stream(stream)))


def moe_dispatch_workspace_bytes(T: int, k: int, E: int) -> int:
    return load_library().moe_dispatch_workspace_bytes(T, k, E)


def moe_dispatch(topk_ids, topk_w, x, E: int, counts, offsets, perm, inv_perm, packed_tok,
                 packed_w, x_packed, ws, status=None, stream=None):
    T, k = topk_ids.shape
    H = x.shape[1] if x is not None else 0
    dt = _dtype_code(x) if x is not None else MOE_BF16
    _check(load_library().moe_dispatch(
        _ptr(topk_ids), _ptr(topk_w), _ptr(x), T, H, E, k, dt, _ptr(counts), _ptr(offsets),
        _ptr(perm), _ptr(inv_perm), _ptr(packed_tok), _ptr(packed_w), _ptr(x_packed),
        _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0, _ptr(status),
        _stream(stream)))


def moe_dispatch_noalloc(topk_ids, topk_w, x, E: int, counts, offsets, perm, inv_perm,
                         packed_tok, packed_w, x_packed, status=None, stream=None):
    """moe_dispatch without a workspace, for callers that cannot allocate: the
    count table lives in a fixed array inside the library (limit
    ceil(T*k/2048)*E <= 32768).  Calls that overlap on the GPU race on it."""
    T, k = topk_ids.shape
    H = x.shape[1] if x is not None else 0
    dt = _dtype_code(x) if x is not None else MOE_BF16
    _check(load_library().moe_dispatch_noalloc(
        _ptr(topk_ids), _ptr(topk_w), _ptr(x), T, H, E, k, dt, _ptr(counts), _ptr(offsets),
        _ptr(perm), _ptr(inv_perm), _ptr(packed_tok), _ptr(packed_w), _ptr(x_packed),
        _ptr(status), _stream(stream)))


def moe_experts_workspace_bytes(N: int, H: int, I: int, E: int, dtype: int) -> int:
    return load_library().moe_experts_workspace_bytes(N, H, I, E, dtype)


def moe_experts(x_packed, offsets, packed_w, w13, w2, h, y_packed, ws=None, status=None,
                stream=None):
    N, H = x_packed.shape
    E = w13.shape[0]
    I = w13.shape[1] // 2
    _check(load_library().moe_experts(
        _ptr(x_packed), _ptr(offsets), _ptr(packed_w), _ptr(w13), _ptr(w2), N, H, I, E,
        _dtype_code(x_packed), _dtype_code(y_packed), _ptr(h), _ptr(y_packed), _ptr(ws),
        ws.numel() * ws.element_size() if ws is not None else 0, _ptr(status), _stream(stream)))


def moe_experts_shared(x_packed, offsets, packed_w, w13, w2, h, y_packed, x, w13s, w2s, h_s,
                       y_s, ws=None, status=None, stream=None):
    """moe_experts plus a shared expert (every row of x through w13s [2I_s,H],
    w2s [H,I_s] into h_s, y_s) in the same two launches (bf16 only)."""
    N, H = x_packed.shape
    E = w13.shape[0]
    I = w13.shape[1] // 2
    T = x.shape[0]
    I_s = w13s.shape[0] // 2
    _check(load_library().moe_experts_shared(
        _ptr(x_packed), _ptr(offsets), _ptr(packed_w), _ptr(w13), _ptr(w2), N, H, I, E,
        _ptr(x), T, _ptr(w13s), _ptr(w2s), I_s, _dtype_code(x_packed), _dtype_code(y_packed),
        _ptr(h), _ptr(y_packed),
        _ptr(h_s), _ptr(y_s), _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0,
        _ptr(status), _stream(stream)))


def moe_combine(y_packed, inv_perm, T: int, k: int, out, shared=None, shared_gate_logit=None,
                status=None, stream=None):
    H = out.shape[1]
    _check(load_library().moe_combine(
        _ptr(y_packed), _dtype_code(y_packed), _ptr(inv_perm), T, H, k, _ptr(shared),
        _ptr(shared_gate_logit),
        _dtype_code(out), _ptr(out), _ptr(status), _stream(stream)))


def moe_gather(x, packed_tok, offsets, expert_start: int, expert_end: int, x_packed,
               status=None, stream=None):
    """x_packed rows of the experts [expert_start, expert_end) only."""
    N, H = x_packed.shape
    E = offsets.shape[0] - 1
    _check(load_library().moe_gather(
        _ptr(x), _ptr(packed_tok), _ptr(offsets), E, expert_start, expert_end, N, H,
        _dtype_code(x), _ptr(x_packed), _ptr(status), _stream(stream)))


def moe_combine_range(y_packed, inv_perm, offsets, expert_start: int, expert_end: int, T: int,
                      k: int, out, shared=None, shared_gate_logit=None, status=None,
                      stream=None):
    """Masked-local merge: only the rows of experts [expert_start, expert_end)."""
    H = out.shape[1]
    E = offsets.shape[0] - 1
    _check(load_library().moe_combine_range(
        _ptr(y_packed), _dtype_code(y_packed), _ptr(inv_perm), _ptr(offsets), E, expert_start,
        expert_end, T, H, k,
        _ptr(shared), _ptr(shared_gate_logit), _dtype_code(out), _ptr(out), _ptr(status),
        _stream(stream)))


def moe_finalize(acc, out, stream=None):
    """out = acc (fp32 [T,H]) rounded once to out's dtype."""
    T, H = out.shape
    _check(load_library().moe_finalize(_ptr(acc), T, H, _dtype_code(out), _ptr(out),
                                       _stream(stream)))


def moe_ep_partition_workspace_bytes(num_tokens: int, top_k: int) -> int:
    return load_library().moe_ep_partition_workspace_bytes(num_tokens, top_k)


def moe_ep_partition(gate_indices, gate_weights, num_tokens: int, top_k: int,
                     local_expert_start: int, local_expert_end: int, local_token_indices,
                     local_expert_ids, local_weights, remote_token_indices, remote_expert_ids,
                     remote_weights, bucket_counts, ws=None, stream=None):
    """metrale's build_ep_routing_table on the device (see moe_b200.h)."""
    _check(load_library().moe_ep_partition(
        _ptr(gate_indices), gate_indices.numel(), _ptr(gate_weights), gate_weights.numel(),
        num_tokens, top_k, local_expert_start, local_expert_end, _ptr(local_token_indices),
        _ptr(local_expert_ids), _ptr(local_weights), _ptr(remote_token_indices),
        _ptr(remote_expert_ids), _ptr(remote_weights), _ptr(bucket_counts), _ptr(ws),
        ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream)))


def moe_ep_owner(ids, E: int, world: int, owner, status=None, stream=None):
    """owner[f] = rank owning expert ids[f] (contiguous split of E over world)."""
    _check(load_library().moe_ep_owner(_ptr(ids), ids.numel(), E, world, _ptr(owner),
                                       _ptr(status), _stream(stream)))


def moe_ep_pack_ids(ids, perm, offsets, E: int, world: int, local_ids, stream=None):
    """local_ids[p] = ids[perm[p]] minus its owner's first expert (rows p < offsets[world])."""
    _check(load_library().moe_ep_pack_ids(_ptr(ids), _ptr(perm), _ptr(offsets), ids.numel(), E,
                                          world, _ptr(local_ids), _stream(stream)))


def moe_read_status(status, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(load_library().moe_read_status(_ptr(status), _stream(stream), ctypes.byref(v)))
    return int(v.value)


def moe_test_set_wait_budget_ns(ns: int):
    """Testing hook: budget of the tensor-core kernels' main-loop waits (0 = default)."""
    _check(load_library().moe_test_set_wait_budget_ns(ns))


def moe_probe_wait_timeout(status, budget_us: int, stream=None):
    _check(load_library().moe_probe_wait_timeout(_ptr(status), budget_us, _stream(stream)))


class MoELayerDesc(ctypes.Structure):
    """ctypes mirror of moe_layer_desc (include/moe_b200.h)."""
    _fields_ = [("T", _I), ("H", _I), ("E", _I), ("k", _I), ("I", _I), ("dtype", _I),
                ("renormalize", _I), ("n_groups", _I), ("topk_groups", _I), ("W_gate", _P),
                ("bias", _P), ("w13", _P), ("w2", _P), ("I_s", _I), ("w13s", _P), ("w2s", _P),
                ("w_sg", _P), ("y_f32", _I)]


def _desc(params: dict, T: int, k: int, renormalize: bool, n_groups: int, topk_groups: int,
          y_f32: bool = False):
    W = params["W_gate"]
    E, H = W.shape
    I = params["w13"].shape[1] // 2
    d = MoELayerDesc(T=T, H=H, E=E, k=k, I=I, dtype=_dtype_code(W),
                     renormalize=int(bool(renormalize)), n_groups=n_groups,
                     topk_groups=topk_groups, W_gate=W.data_ptr(),
                     bias=params["bias"].data_ptr() if params.get("bias") is not None else None,
                     w13=params["w13"].data_ptr(), w2=params["w2"].data_ptr(),
                     y_f32=int(bool(y_f32)))
    if params.get("w13s") is not None:
        d.I_s = params["w13s"].shape[0] // 2
        d.w13s = params["w13s"].data_ptr()
        d.w2s = params["w2s"].data_ptr()
        d.w_sg = params["w_sg"].data_ptr()
    return d


class MoELayer:
    """moe_layer handle: the whole layer for batches of T tokens, its buffers in
    one device block (a torch tensor this object keeps).  ``params`` (device
    tensors) must stay alive as long as the layer."""

    def __init__(self, params: dict, T: int, k: int, renormalize: bool, n_groups: int = 1,
                 topk_groups: int = 1, stream=None, y_f32: bool = False):
        lib = load_library()
        self.params = params
        self.desc = _desc(params, T, k, renormalize, n_groups, topk_groups, y_f32)
        nbytes = lib.moe_layer_workspace_bytes(ctypes.byref(self.desc))
        if nbytes == 0:
            raise MoEError(MOE_ERR_INVALID_ARG, "moe_layer_workspace_bytes: invalid layer")
        self.ws = torch.empty(nbytes + 256, dtype=torch.uint8, device=params["W_gate"].device)
        off = (-self.ws.data_ptr()) % 256
        self.block = self.ws[off:off + nbytes]
        h = ctypes.c_void_p()
        _check(lib.moe_layer_create(ctypes.byref(self.desc), _ptr(self.block), nbytes,
                                    _stream(stream), ctypes.byref(h)))
        self.handle = h
        self.T, self.H = T, self.desc.H
        self.dtype = params["W_gate"].dtype

    def forward(self, x, out, stream=None):
        _check(load_library().moe_layer_forward(self.handle, _ptr(x), _ptr(out), _stream(stream)))
        return out

    def forward_host(self, x_host, out_host, stream=None):
        _check(load_library().moe_layer_forward_host(self.handle, ctypes.c_void_p(x_host.data_ptr()),
                                                     ctypes.c_void_p(out_host.data_ptr()),
                                                     _stream(stream)))
        return out_host

    def join(self, stream=None):
        _check(load_library().moe_layer_join(self.handle, _stream(stream)))

    def status(self, stream=None) -> int:
        v = ctypes.c_int32(0)
        _check(load_library().moe_layer_status(self.handle, _stream(stream), ctypes.byref(v)))
        return int(v.value)

    def buffer(self, name: str, shape, dtype) -> torch.Tensor:
        """A view of one of the layer's intermediate buffers (see moe_layer_buffer)."""
        p = load_library().moe_layer_buffer(self.handle, name.encode())
        if not p:
            raise MoEError(MOE_ERR_INVALID_ARG, f"no layer buffer named {name!r}")
        n = 1
        for d in shape:
            n *= d
        off = p - self.block.data_ptr()
        es = torch.empty(0, dtype=dtype).element_size()
        return self.block[off:off + n * es].view(dtype).view(*shape)

    def close(self):
        if getattr(self, "handle", None):
            load_library().moe_layer_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class MoELayerBuffers:
    """Every device buffer one forward pass of a layer needs, allocated once.

    Shapes follow the ABI: T tokens, N = T*k assignments.  With a shared
    expert the buffers also hold its packed input/output and gate logit.
    y_packed (and the shared expert's output) are fp16 for bf16 layers (half
    the bytes of fp32; an element beyond the fp16 range sets MOE_ERR_OVERFLOW)
    unless ``y_f32``, and fp32 for fp32 layers.
    """

    def __init__(self, T: int, H: int, E: int, k: int, I: int, dtype: torch.dtype,
                 device="cuda", shared_I: Optional[int] = None, y_f32: bool = False):
        N = T * k
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.T, self.H, self.E, self.k, self.I, self.N = T, H, E, k, I, N
        self.logits = torch.empty(T, E, **f32)
        self.ids = torch.empty(T, k, **i32)
        self.w = torch.empty(T, k, **f32)
        self.counts = torch.empty(E, **i32)
        self.offsets = torch.empty(E + 1, **i32)
        self.perm = torch.empty(N, **i32)
        self.inv_perm = torch.empty(N, **i32)
        self.packed_tok = torch.empty(N, **i32)
        self.packed_w = torch.empty(N, **f32)
        self.x_packed = torch.empty(N, H, dtype=dtype, device=dev)
        self.h = torch.empty(N, I, dtype=dtype, device=dev)
        self.y_dtype = torch.float16 if dtype == torch.bfloat16 and not y_f32 else torch.float32
        self.y_packed = torch.empty(N, H, dtype=self.y_dtype, device=dev)
        self.out = torch.empty(T, H, dtype=dtype, device=dev)
        self.ws = torch.empty(max(1, moe_dispatch_workspace_bytes(T, k, E)), dtype=torch.uint8,
                              device=dev)
        # zero-filled once; the split-K counters return to zero after every call
        self.ws_experts = torch.zeros(
            max(16, moe_experts_workspace_bytes(N, H, I, E, MOE_BF16 if dtype == torch.bfloat16
                                                else MOE_F32)), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, **i32)
        self.rd_counter = torch.zeros(1, **i32)    # ticket of moe_route_dispatch
        self.route_dispatch = route_dispatch_fits(T, H, E, k, gate=shared_I is not None)
        self.shared_I = shared_I
        # bf16 tensor-core layers run the shared expert inside the routed launches
        self.fuse_shared = bool(shared_I) and dtype == torch.bfloat16 and H % 256 == 0 and \
            I % 64 == 0 and shared_I % 64 == 0
        if shared_I:
            self.sg_logit = torch.empty(T, 1, **f32)
            self.sh_offsets = torch.tensor([0, T], **i32)
            self.sh_h = torch.empty(T, shared_I, dtype=dtype, device=dev)
            self.sh_y = torch.empty(T, H, dtype=self.y_dtype, device=dev)


def route_and_dispatch(x, params: dict, k: int, renormalize: bool, buf: MoELayerBuffers,
                       stream=None, n_groups: int = 1, topk_groups: int = 1) -> bool:
    """Router then dispatcher into ``buf``: one launch for decode batches
    (moe_route_dispatch), else moe_route_gated / moe_route[_grouped] and
    moe_dispatch.  With a shared expert (``params["w13s"]``) its gate logit
    goes to ``buf.sg_logit`` in the router's launch.  Returns whether the
    shared gate logit was written."""
    E = params["W_gate"].shape[0]
    if buf.route_dispatch:
        w_sg = params.get("w_sg") if params.get("w13s") is not None else None
        moe_route_dispatch(x, params["W_gate"], params.get("bias"), k, renormalize, buf.logits,
                           buf.ids, buf.w, buf.counts, buf.offsets, buf.perm, buf.inv_perm,
                           buf.packed_tok, buf.packed_w, buf.x_packed, buf.rd_counter,
                           status=buf.status, stream=stream, n_groups=n_groups,
                           topk_groups=topk_groups, w_gate_shared=w_sg,
                           shared_gate_logit=buf.sg_logit if w_sg is not None else None)
        return w_sg is not None
    gated = params.get("w13s") is not None
    if gated:
        moe_route_gated(x, params["W_gate"], params.get("bias"), params["w_sg"], k, renormalize,
                        buf.logits, buf.ids, buf.w, buf.sg_logit, status=buf.status,
                        stream=stream, n_groups=n_groups, topk_groups=topk_groups)
    elif n_groups > 1:
        moe_route_grouped(x, params["W_gate"], params.get("bias"), k, renormalize, n_groups,
                          topk_groups, buf.logits, buf.ids, buf.w, status=buf.status,
                          stream=stream)
    else:
        moe_route(x, params["W_gate"], params.get("bias"), k, renormalize, buf.logits, buf.ids,
                  buf.w, status=buf.status, stream=stream)
    moe_dispatch(buf.ids, buf.w, x, E, buf.counts, buf.offsets, buf.perm, buf.inv_perm,
                 buf.packed_tok, buf.packed_w, buf.x_packed, buf.ws, buf.status, stream=stream)
    return gated


def moe_layer_forward(x, params: dict, k: int, renormalize: bool, buf: MoELayerBuffers,
                      stream=None, n_groups: int = 1, topk_groups: int = 1):
    """Router -> dispatcher -> executor -> merger into ``buf.out`` (asynchronous).

    ``params``: W_gate [E,H], bias [E] f32 or None, w13 [E,2I,H], w2 [E,H,I] and,
    for a shared expert, w13s [2I_s,H], w2s [H,I_s], w_sg [H].  n_groups > 1
    routes group-limited (moe_route_grouped).
    """
    gate_done = route_and_dispatch(x, params, k, renormalize, buf, stream, n_groups, topk_groups)
    shared = sg = None
    if params.get("w13s") is None:
        moe_experts(buf.x_packed, buf.offsets, buf.packed_w, params["w13"], params["w2"], buf.h,
                    buf.y_packed, ws=buf.ws_experts, status=buf.status, stream=stream)
    else:
        if not gate_done:
            moe_route(x, params["w_sg"].view(1, -1), None, 0, False, buf.sg_logit,
                      status=buf.status, stream=stream)
        if buf.fuse_shared:
            moe_experts_shared(buf.x_packed, buf.offsets, buf.packed_w, params["w13"],
                               params["w2"], buf.h, buf.y_packed, x, params["w13s"],
                               params["w2s"], buf.sh_h, buf.sh_y, ws=buf.ws_experts,
                               status=buf.status, stream=stream)
        else:
            moe_experts(buf.x_packed, buf.offsets, buf.packed_w, params["w13"], params["w2"],
                        buf.h, buf.y_packed, ws=buf.ws_experts, status=buf.status,
                        stream=stream)
            moe_experts(x, buf.sh_offsets, None, params["w13s"].unsqueeze(0),
                        params["w2s"].unsqueeze(0), buf.sh_h, buf.sh_y, ws=buf.ws_experts,
                        status=buf.status, stream=stream)
        shared, sg = buf.sh_y, buf.sg_logit
    moe_combine(buf.y_packed, buf.inv_perm, buf.T, k, buf.out, shared, sg, status=buf.status,
                stream=stream)
    return buf.out


def moe_layer_forward_host(x_host, params: dict, k: int, renormalize: bool,
                           buf: MoELayerBuffers, out_host, stream=None):
    """The same layer called with HOST activations: copy x (pinned host) to the
    device, run the four stages, copy the output back into ``out_host``
    (pinned), all on one stream; returns after the copy back is enqueued."""
    if stream is None:
        stream = torch.cuda.current_stream()
    if not hasattr(buf, "x_dev"):
        buf.x_dev = torch.empty(x_host.shape, dtype=x_host.dtype, device=buf.out.device)
    with torch.cuda.stream(stream):
        buf.x_dev.copy_(x_host, non_blocking=True)
        moe_layer_forward(buf.x_dev, params, k, renormalize, buf, stream=stream)
        out_host.copy_(buf.out, non_blocking=True)
    return out_host
