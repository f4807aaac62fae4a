"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

import mixture_experts_layer_44_b200 as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(M.lib_path()):
        from mixture_experts_layer_44_b200 import build
        build.build()
    return M.load_library()


def test_header_declares_the_stage_calls():
    names = _declared()
    for n in ("moe_route", "moe_dispatch", "moe_experts", "moe_experts_shared", "moe_combine",
              "moe_dispatch_workspace_bytes", "moe_experts_workspace_bytes", "moe_read_status",
              "moe_probe_wait_timeout", "moe_last_error", "moe_abi_version", "moe_launch_count",
              "moe_route_gated"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", M.lib_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(\w+)$", out, flags=re.M))
    for n in _declared():
        assert n in exported, n
        assert hasattr(lib, n)


def test_library_is_built_for_sm100a_only():
    out = subprocess.run(["/usr/local/cuda/bin/cuobjdump", "--list-elf", M.lib_path()],
                         capture_output=True, text=True).stdout
    assert "sm_100a" in out
    assert "sm_90" not in out and "sm_80" not in out


def test_abi_version_and_workspace_queries(lib):
    assert M.moe_abi_version() == 5
    assert M.moe_launch_count() == 0     # nothing launched on a CPU-only host
    ws = M.moe_dispatch_workspace_bytes(16384, 8, 128)
    assert ws >= (16384 * 8 + 2047) // 2048 * 128 * 4
    assert M.moe_dispatch_workspace_bytes(0, 2, 8) == 0
    # up to T*k = 65536 the count and scatter CTAs take 1024 assignments each:
    # one count row per 1024, and at most 64 * E entries (inside the 128 KiB
    # of the allocation-free entry point even at E = 256)
    assert M.moe_dispatch_workspace_bytes(4096, 2, 64) >= 8 * 64 * 4
    assert M.moe_dispatch_workspace_bytes(65536, 1, 256) <= 128 * 1024
    assert M.moe_experts_workspace_bytes(100, 256, 128, 4, M.MOE_BF16) >= 4096 * 4 + 128 * 1024
    assert M.moe_experts_workspace_bytes(100, 256, 128, 4, M.MOE_F32) == 0


NULL = None
P = ctypes.c_void_p(16)   # an aligned non-null address that is never dereferenced


def _err(lib):
    return lib.moe_last_error().decode()


def test_route_rejects_bad_arguments_on_the_host(lib):
    r = lib.moe_route(P, P, NULL, 0, 64, 8, 2, 1, M.MOE_BF16, P, P, P, NULL, NULL)
    assert r == M.MOE_ERR_INVALID_ARG and "T and H" in _err(lib)
    r = lib.moe_route(P, P, NULL, 4, 64, 8, 9, 1, M.MOE_BF16, P, P, P, NULL, NULL)
    assert r == M.MOE_ERR_INVALID_ARG and "k must be" in _err(lib)
    r = lib.moe_route(P, P, NULL, 4, 64, 300, 2, 1, M.MOE_BF16, P, P, P, NULL, NULL)
    assert r == M.MOE_ERR_INVALID_ARG and "E must be" in _err(lib)
    r = lib.moe_route(P, P, NULL, 4, 60, 8, 2, 1, M.MOE_BF16, P, P, P, NULL, NULL)
    assert r == M.MOE_ERR_INVALID_ARG and "multiple of 8" in _err(lib)
    r = lib.moe_route(ctypes.c_void_p(24), P, NULL, 4, 64, 8, 2, 1, M.MOE_BF16, P, P, P, NULL, NULL)
    assert r == M.MOE_ERR_INVALID_ARG and "aligned" in _err(lib)
    r = lib.moe_route(P, P, NULL, 4, 64, 8, 2, 1, 7, P, P, P, NULL, NULL)
    assert r == M.MOE_ERR_INVALID_ARG and "dtype" in _err(lib)
    r = lib.moe_route(P, P, NULL, 4, 64, 8, 2, 1, M.MOE_BF16, P, NULL, P, NULL, NULL)
    assert r == M.MOE_ERR_INVALID_ARG


def test_dispatch_rejects_bad_arguments_on_the_host(lib):
    args = [P, P, P, 4, 64, 8, 2, M.MOE_BF16, P, P, P, P, P, P, P, P, 4096, NULL, NULL]
    a = list(args); a[6] = 0
    assert lib.moe_dispatch(*a) == M.MOE_ERR_INVALID_ARG
    a = list(args); a[15] = NULL          # ws missing
    assert lib.moe_dispatch(*a) == M.MOE_ERR_INVALID_ARG and "workspace" in _err(lib)
    a = list(args); a[16] = 4             # ws too small
    assert lib.moe_dispatch(*a) == M.MOE_ERR_INVALID_ARG
    a = list(args); a[14] = NULL          # x given but no x_packed
    assert lib.moe_dispatch(*a) == M.MOE_ERR_INVALID_ARG and "x_packed" in _err(lib)
    a = list(args); a[13] = NULL          # topk_w given but no packed_w
    assert lib.moe_dispatch(*a) == M.MOE_ERR_INVALID_ARG


def test_route_dispatch_rejects_bad_arguments_on_the_host(lib):
    # x, W, bias, w_sg, T, H, E, k, renorm, G, Mg, dtype, logits, ids, w, sg_logit, counts,
    # offsets, perm, inv_perm, packed_tok, packed_w, x_packed, counter, status, stream
    args = [P, P, NULL, NULL, 4, 64, 8, 2, 1, 1, 1, M.MOE_BF16, P, P, P, NULL, P, P, P, P, P, P,
            P, P, NULL, NULL]
    a = list(args); a[4] = 65             # more tokens than the one-launch path takes
    assert lib.moe_route_dispatch(*a) == M.MOE_ERR_INVALID_ARG and "T must be" in _err(lib)
    a = list(args); a[6] = 65; a[7] = 2   # more experts than it takes
    assert lib.moe_route_dispatch(*a) == M.MOE_ERR_INVALID_ARG and "E must be" in _err(lib)
    a = list(args); a[7] = 0              # it always dispatches: k >= 1
    assert lib.moe_route_dispatch(*a) == M.MOE_ERR_INVALID_ARG and "k must be" in _err(lib)
    a = list(args); a[23] = NULL          # no ticket word
    assert lib.moe_route_dispatch(*a) == M.MOE_ERR_INVALID_ARG and "counter" in _err(lib)
    a = list(args); a[9] = 3              # 3 groups do not divide 8 experts
    assert lib.moe_route_dispatch(*a) == M.MOE_ERR_INVALID_ARG and "n_groups" in _err(lib)
    a = list(args); a[5] = 32776          # H above 32768
    assert lib.moe_route_dispatch(*a) == M.MOE_ERR_INVALID_ARG and "H must be" in _err(lib)
    a = list(args); a[11] = 7
    assert lib.moe_route_dispatch(*a) == M.MOE_ERR_INVALID_ARG
    a = list(args); a[3] = P              # a gate row without its logit output
    assert lib.moe_route_dispatch(*a) == M.MOE_ERR_INVALID_ARG and "shared_gate_logit" in _err(lib)
    a = list(args); a[3] = P; a[15] = P; a[6] = 64   # 64 experts leave no row for the gate
    assert lib.moe_route_dispatch(*a) == M.MOE_ERR_INVALID_ARG and "E must be" in _err(lib)


def test_experts_rejects_bad_arguments_on_the_host(lib):
    base = [P, P, P, P, P, 100, 256, 128, 4, M.MOE_BF16, M.MOE_F16, P, P, NULL, 0, NULL, NULL]
    a = list(base); a[6] = 200            # H not a multiple of 256 on the bf16 path
    assert lib.moe_experts(*a) == M.MOE_ERR_UNSUPPORTED and "H % 256" in _err(lib)
    a = list(base); a[7] = 100            # I not a multiple of 8
    assert lib.moe_experts(*a) == M.MOE_ERR_INVALID_ARG
    a = list(base); a[8] = 0
    assert lib.moe_experts(*a) == M.MOE_ERR_INVALID_ARG
    a = list(base); a[5] = 0              # nothing to do: OK without touching the GPU
    assert lib.moe_experts(*a) == M.MOE_OK
    a = list(base); a[3] = NULL
    assert lib.moe_experts(*a) == M.MOE_ERR_INVALID_ARG
    a = list(base); a[9] = M.MOE_F32      # fp32 layers keep y_packed in fp32
    assert lib.moe_experts(*a) == M.MOE_ERR_UNSUPPORTED and "y_dtype" in _err(lib)
    a = list(base); a[10] = 5             # no such y type
    assert lib.moe_experts(*a) == M.MOE_ERR_INVALID_ARG
    a = list(base); a[10] = M.MOE_BF16    # y_packed is fp16 or fp32 only
    assert lib.moe_experts(*a) == M.MOE_ERR_INVALID_ARG and "y_dtype" in _err(lib)


def test_experts_shared_rejects_bad_arguments_on_the_host(lib):
    # routed part as above, then x, T, w13s, w2s, I_s, dtype, y_dtype, h, y, h_s, y_s, ws,
    # bytes, status, stream
    base = [P, P, P, P, P, 100, 256, 128, 4, P, 32, P, P, 512, M.MOE_BF16, M.MOE_F16, P, P, P,
            P, NULL, 0, NULL, NULL]
    a = list(base); a[13] = 100           # I_s not a multiple of 128
    assert lib.moe_experts_shared(*a) == M.MOE_ERR_UNSUPPORTED and "I_s" in _err(lib)
    a = list(base); a[10] = 0             # T < 1
    assert lib.moe_experts_shared(*a) == M.MOE_ERR_INVALID_ARG
    a = list(base); a[19] = NULL          # no y_s
    assert lib.moe_experts_shared(*a) == M.MOE_ERR_INVALID_ARG
    a = list(base); a[14] = M.MOE_F32     # fp32 runs the two experts separately
    a[15] = M.MOE_F32
    assert lib.moe_experts_shared(*a) == M.MOE_ERR_UNSUPPORTED
    a = list(base); a[6] = 200            # the routed rules still apply
    assert lib.moe_experts_shared(*a) == M.MOE_ERR_UNSUPPORTED and "H % 256" in _err(lib)


def test_combine_and_status_reject_bad_arguments_on_the_host(lib):
    B, F = M.MOE_BF16, M.MOE_F16
    assert lib.moe_combine(P, F, P, 4, 64, 0, NULL, NULL, B, P, NULL, NULL) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(P, F, P, 4, 63, 2, NULL, NULL, B, P, NULL, NULL) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(NULL, F, P, 4, 64, 2, NULL, NULL, B, P, NULL, NULL) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(P, 3, P, 4, 64, 2, NULL, NULL, B, P, NULL, NULL) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(P, B, P, 4, 64, 2, NULL, NULL, B, P, NULL, NULL) == M.MOE_ERR_INVALID_ARG
    assert "y_dtype" in _err(lib)
    v = ctypes.c_int32(0)
    assert lib.moe_read_status(NULL, NULL, ctypes.byref(v)) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_probe_wait_timeout(P, 0, NULL) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_probe_wait_timeout(P, 3_000_000, NULL) == M.MOE_ERR_INVALID_ARG


def test_python_binding_raises_with_the_library_message(lib):
    import torch
    x = torch.empty(0, 64)
    with pytest.raises(M.MoEError, match="moe_route: "):
        M.moe_route(x, torch.empty(8, 64), None, 2, True, torch.empty(0, 8), stream=0)


def test_layer_descriptor_is_checked_on_the_host(lib):
    d = M.MoELayerDesc(T=64, H=256, E=8, k=2, I=128, dtype=M.MOE_BF16, renormalize=1,
                       n_groups=1, topk_groups=1, W_gate=256, bias=None, w13=512, w2=768)
    n = lib.moe_layer_workspace_bytes(ctypes.byref(d))
    # two copies each of x and out, the packed buffers, fp16 y_packed, the workspaces
    assert n >= 4 * 64 * 256 * 2 + 128 * 256 * 2 + 128 * 128 * 2 + 128 * 256 * 2
    f = M.MoELayerDesc.from_buffer_copy(d)
    f.y_f32 = 1                                 # fp32 y_packed: 2 more bytes per element
    assert lib.moe_layer_workspace_bytes(ctypes.byref(f)) >= n + 128 * 256 * 2
    for field, bad in (("I", 100), ("k", 9), ("E", 0), ("dtype", 7), ("H", 200)):
        b = M.MoELayerDesc.from_buffer_copy(d)
        setattr(b, field, bad)
        assert lib.moe_layer_workspace_bytes(ctypes.byref(b)) == 0, field
    g = M.MoELayerDesc.from_buffer_copy(d)
    g.n_groups, g.topk_groups = 4, 1            # k = 2 <= 1 * 8 / 4: fine
    assert lib.moe_layer_workspace_bytes(ctypes.byref(g)) == n
    g.n_groups, g.topk_groups = 8, 1            # k = 2 > 1 * 8 / 8
    assert lib.moe_layer_workspace_bytes(ctypes.byref(g)) == 0
    h = ctypes.c_void_p()
    assert lib.moe_layer_create(ctypes.byref(d), None, n, None, ctypes.byref(h)) == M.MOE_ERR_INVALID_ARG
    assert "workspace" in M.moe_last_error()
    assert lib.moe_layer_create(ctypes.byref(d), ctypes.c_void_p(4096 + 16), n, None,
                                ctypes.byref(h)) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_forward(None, P, P, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_destroy(None) == M.MOE_OK


def test_new_entry_points_reject_bad_arguments_on_the_host(lib):
    B = M.MOE_BF16
    # group-limited router: groups must divide E, at most 32, enough experts kept
    assert lib.moe_route_grouped(P, P, NULL, 4, 64, 12, 2, 1, 5, 1, B, P, P, P, NULL, NULL) == M.MOE_ERR_INVALID_ARG
    assert "n_groups must divide E" in M.moe_last_error()
    assert lib.moe_route_grouped(P, P, NULL, 4, 64, 64, 2, 1, 64, 2, B, P, P, P, NULL, NULL) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_route_grouped(P, P, NULL, 4, 64, 16, 8, 1, 8, 3, B, P, P, P, NULL, NULL) == M.MOE_ERR_INVALID_ARG
    assert "topk_groups * E / n_groups" in M.moe_last_error()
    assert lib.moe_route_grouped(P, P, NULL, 4, 64, 16, 2, 1, 8, 9, B, P, P, P, NULL, NULL) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_route_grouped(P, P, NULL, 4, 64, 16, 2, 1, 0, 1, B, P, P, P, NULL, NULL) == M.MOE_ERR_INVALID_ARG
    # range gather / merge: 0 <= start <= end <= E
    assert lib.moe_gather(P, P, P, 8, 3, 9, 16, 64, B, P, NULL, NULL) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_gather(P, P, P, 8, 5, 4, 16, 64, B, P, NULL, NULL) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_combine_range(P, M.MOE_F16, P, P, 8, -1, 4, 4, 64, 2, NULL, NULL, M.MOE_F32, P, NULL, NULL) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_finalize(NULL, 4, 64, B, P, NULL) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_finalize(P, 4, 60, B, P, NULL) == M.MOE_ERR_INVALID_ARG
    # owner ids: at most one rank per expert
    assert lib.moe_ep_owner(P, 8, 4, 5, P, NULL, NULL) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_pack_ids(P, P, P, 8, 4, 0, P, NULL) == M.MOE_ERR_INVALID_ARG
    # routing table: the page's panics, and a missing workspace for a large table
    assert lib.moe_ep_partition(P, 3, P, 4, 2, 2, 0, 256, P, P, P, P, P, P, P, NULL, 0, NULL) == M.MOE_ERR_INVALID_ARG
    assert M.moe_last_error() == "gate_indices length mismatch"
    assert lib.moe_ep_partition(P, 4, P, 3, 2, 2, 0, 256, P, P, P, P, P, P, P, NULL, 0, NULL) == M.MOE_ERR_INVALID_ARG
    assert M.moe_last_error() == "gate_weights length mismatch"
    assert lib.moe_ep_partition(P, 8000, P, 8000, 1000, 8, 0, 4, P, P, P, P, P, P, P, NULL, 0, NULL) == M.MOE_ERR_INVALID_ARG
    assert M.moe_ep_partition_workspace_bytes(1000, 8) >= 4 * 4
    # dispatch takes repeated ids (all-to-all by owner) but still k <= 8
    assert lib.moe_dispatch(P, P, NULL, 4, 0, 2, 9, B, P, P, P, P, P, P, NULL, P, 256, NULL, NULL) == M.MOE_ERR_INVALID_ARG
    # the testing hook's bounds
    assert lib.moe_test_set_wait_budget_ns(10) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_test_set_wait_budget_ns(0) == M.MOE_OK


def test_route_gated_rejects_bad_arguments_on_the_host(lib):
    # x, W, bias, w_sg, T, H, E, k, renorm, G, Mg, dtype, logits, ids, w, sg_logit, status, stream
    args = [P, P, NULL, P, 4, 64, 8, 2, 1, 1, 1, M.MOE_BF16, P, P, P, P, NULL, NULL]
    a = list(args); a[3] = NULL           # no gate row
    assert lib.moe_route_gated(*a) == M.MOE_ERR_INVALID_ARG and "w_gate_shared" in _err(lib)
    a = list(args); a[15] = NULL          # nowhere to put its logit
    assert lib.moe_route_gated(*a) == M.MOE_ERR_INVALID_ARG and "shared_gate_logit" in _err(lib)
    a = list(args); a[3] = ctypes.c_void_p(24)   # gate row not 16-byte aligned
    assert lib.moe_route_gated(*a) == M.MOE_ERR_INVALID_ARG and "aligned" in _err(lib)
    a = list(args); a[9] = 3              # the routed part's checks apply as well
    assert lib.moe_route_gated(*a) == M.MOE_ERR_INVALID_ARG and "n_groups" in _err(lib)
