"""moe_dispatch_noalloc: the dispatcher for callers that cannot allocate.

Some callers cannot call cudaMalloc where they dispatch (a C program whose
GPU memory belongs to someone else, a plugin without access to its host
framework's allocator, a serving loop that allocates nothing once running).
For them the library offers moe_dispatch_noalloc, which keeps its count table
in a fixed array inside the library instead of a caller workspace.  These
tests call it through the C ABI and require its outputs to equal, bit for
bit, those of moe_dispatch on the same inputs, on two calls in a row.  Both
calls are large enough (more than 8192 assignments) to take the multi-block
path whose per-block counts live in the shared array, so the second call
runs on the first call's leftovers there.  This file is collected last on
purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_layer_44_b200 as M

pytestmark = pytest.mark.gpu

KEYS = ("counts", "offsets", "perm", "inv_perm", "packed_tok", "packed_w", "x_packed")


def _ids(rng, T, k, E, p=None):
    return torch.tensor(np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]),
                        dtype=torch.int32, device="cuda")


def _buffers(T, k, E, H, dtype):
    N = T * k
    i32 = dict(dtype=torch.int32, device="cuda")
    return dict(counts=torch.full((E,), -3, **i32), offsets=torch.full((E + 1,), -3, **i32),
                perm=torch.full((N,), -3, **i32), inv_perm=torch.full((N,), -3, **i32),
                packed_tok=torch.full((N,), -3, **i32),
                packed_w=torch.full((N,), -3.0, device="cuda"),
                x_packed=torch.zeros(N, H, dtype=dtype, device="cuda"))


def _both(ids, w, x, E):
    T, k = ids.shape
    H = x.shape[1]
    ref = _buffers(T, k, E, H, x.dtype)
    ws = torch.empty(M.moe_dispatch_workspace_bytes(T, k, E), dtype=torch.uint8, device="cuda")
    st_ref = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_dispatch(ids, w, x, E, *(ref[key] for key in KEYS), ws, st_ref)
    got = _buffers(T, k, E, H, x.dtype)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_dispatch_noalloc(ids, w, x, E, *(got[key] for key in KEYS), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(st_ref.item()) == 0
    for key in KEYS:
        a, b = got[key], ref[key]
        assert torch.equal(a.view(torch.uint8) if a.dtype == torch.bfloat16 else a,
                           b.view(torch.uint8) if b.dtype == torch.bfloat16 else b), key


def test_noalloc_dispatch_equals_the_workspace_dispatch_on_two_calls_in_a_row():
    rng = np.random.default_rng(0)
    # call 1: the Qwen3-30B-A3B routing shape (131072 assignments, 128 experts, skewed)
    p = np.arange(1, 129, dtype=np.float64) ** -1.1
    p[-8:] = 0
    p /= p.sum()
    ids = _ids(rng, 16384, 8, 128, p)
    w = torch.rand(16384, 8, device="cuda")
    x = torch.randn(16384, 256, device="cuda").to(torch.bfloat16)
    _both(ids, w, x, 128)
    # call 2: a smaller, different problem right after, on the same shared array:
    # 5000 tokens x top-3 = 15000 assignments -> 8 count blocks x 60 experts of
    # the array, all of which still hold call 1's block bases
    ids = _ids(rng, 5000, 3, 60)
    w = torch.rand(5000, 3, device="cuda")
    x = torch.randn(5000, 64, device="cuda")
    _both(ids, w, x, 60)


def test_noalloc_dispatch_rejects_sizes_beyond_its_fixed_scratch():
    lib = M.load_library()
    P = ctypes.c_void_p(256)   # never dereferenced: the size check comes first
    # ceil(300000 * 8 / 2048) * 256 = 300288 count entries > 32768
    r = lib.moe_dispatch_noalloc(P, P, P, 300000, 64, 256, 8, M.MOE_BF16, P, P, P, P, P, P, P,
                                 None, None)
    assert r == M.MOE_ERR_INVALID_ARG
    assert "32768" in M.moe_last_error()
