"""Dispatcher parity: GPU moe_dispatch against the oracle, bit for bit.

Fed the same ids and weights, counts / offsets / perm / inv_perm /
packed_tok must be identical to the oracle's stable counting sort, packed_w
identical (a copy), and x_packed byte-identical to x gathered by packed_tok.
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_44_b200 as M
import oracle.moe_oracle as O
from tests.gpu_util import DEV, dev, ids_with_counts, rand_ids

pytestmark = pytest.mark.gpu


def _alloc(T, k, E, H, dtype):
    N = T * k
    i32 = dict(dtype=torch.int32, device=DEV)
    return dict(
        counts=torch.full((E,), -7, **i32), offsets=torch.full((E + 1,), -7, **i32),
        perm=torch.full((N,), -7, **i32), inv_perm=torch.full((N,), -7, **i32),
        packed_tok=torch.full((N,), -7, **i32), packed_w=torch.full((N,), -7.0, device=DEV),
        x_packed=torch.zeros(N, H, dtype=dtype, device=DEV),
        ws=torch.empty(M.moe_dispatch_workspace_bytes(T, k, E), dtype=torch.uint8, device=DEV),
        status=torch.zeros(1, **i32))


def _run(ids, w, x, E):
    T, k = ids.shape
    H = x.shape[1]
    b = _alloc(T, k, E, H, x.dtype)
    M.moe_dispatch(dev(ids), dev(w), dev(x), E, b["counts"], b["offsets"], b["perm"],
                   b["inv_perm"], b["packed_tok"], b["packed_w"], b["x_packed"], b["ws"],
                   b["status"])
    torch.cuda.synchronize()
    return {key: v.cpu() for key, v in b.items()}


def _check(ids, w, x, E):
    g = _run(ids, w, x, E)
    o = O.dispatch(ids.numpy(), w.numpy().astype(np.float64), E)
    assert int(g["status"][0]) == 0
    for key in ("counts", "offsets", "perm", "inv_perm", "packed_tok"):
        np.testing.assert_array_equal(g[key].numpy(), o[key], err_msg=key)
    # packed_w is a copy of fp32 weights: identical bits
    np.testing.assert_array_equal(g["packed_w"].numpy(), w.numpy().reshape(-1)[o["perm"]])
    want = x[torch.as_tensor(o["packed_tok"])]
    assert torch.equal(g["x_packed"].contiguous().view(torch.uint8), want.contiguous().view(torch.uint8))
    return g


@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (1, 2, 8), (5, 3, 4), (64, 2, 8), (300, 4, 60),
                                   (1000, 8, 128), (4096, 2, 64), (2049, 1, 3), (700, 8, 256),
                                   (2000, 8, 256), (10000, 1, 1), (4097, 2, 64), (1024, 2, 16),
                                   (256, 8, 256)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_dispatch_random(T, k, E, dtype):
    rng = np.random.default_rng(T * 31 + k * 7 + E)
    ids = rand_ids(rng, T, k, E)
    w = torch.tensor(rng.random((T, k)), dtype=torch.float32)
    x = torch.randn(T, 64, generator=torch.Generator().manual_seed(T)).to(dtype)
    _check(ids, w, x, E)


def test_dispatch_empty_and_dominant_experts():
    rng = np.random.default_rng(1)
    # 16 experts, half empty, one taking every token (spans many CTAs of the count pass)
    counts = [4000, 0, 700, 0, 0, 1, 0, 130, 0, 3, 0, 0, 3165, 0, 1, 0]
    ids = ids_with_counts(counts, 2, rng)
    T = ids.shape[0]
    w = torch.tensor(rng.random((T, 2)), dtype=torch.float32)
    x = torch.randn(T, 128).to(torch.bfloat16)
    g = _check(ids, w, x, 16)
    assert g["counts"].tolist() == counts


def test_dispatch_qwen3_scale():
    rng = np.random.default_rng(2)
    p = np.arange(1, 129, dtype=np.float64) ** -1.1
    p[-8:] = 0
    p /= p.sum()
    ids = rand_ids(rng, 16384, 8, 128, counts_bias=p)
    w = torch.tensor(rng.random((16384, 8)), dtype=torch.float32)
    x = torch.randn(16384, 2048).to(torch.bfloat16)
    _check(ids, w, x, 128)


def test_dispatch_bad_ids_are_reported_and_skipped():
    ids = torch.tensor([[0, 1], [3, 7], [2, -1], [1, 2]], dtype=torch.int32)   # 7, -1 invalid for E=4
    w = torch.rand(4, 2)
    x = torch.randn(4, 64)
    g = _run(ids, w, x, 4)
    assert int(g["status"][0]) == M.MOE_ERR_BAD_INDEX
    assert g["inv_perm"][3].item() == -1 and g["inv_perm"][5].item() == -1
    assert g["offsets"][4].item() == 6
    assert g["counts"].tolist() == [1, 2, 2, 1]
    valid = ids.clone()
    # the six valid assignments keep the stable order of the oracle
    flat = valid.reshape(-1).tolist()
    order = sorted([f for f in range(8) if 0 <= flat[f] < 4], key=lambda f: (flat[f], f))
    assert g["perm"][:6].tolist() == order


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_dispatch_bad_ids_on_the_multi_block_path(dtype):
    # 5000 tokens x top-2 = 10000 assignments: the count / scan / scatter kernels
    # (2048 assignments per block) and the bulk-copy gather; out-of-range ids in
    # several blocks, including the last, partial one.
    rng = np.random.default_rng(21)
    T, k, E, H = 5000, 2, 64, 96
    ids = rand_ids(rng, T, k, E)
    flat = ids.view(-1)
    bad = {5: 64, 2047: -1, 2048: 1000, 4100: -7, 9000: 64, 9999: 2 ** 31 - 1}
    for f, e in bad.items():
        flat[f] = e
    w = torch.tensor(rng.random((T, k)), dtype=torch.float32)
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(21)).to(dtype)
    g = _run(ids, w, x, E)
    assert int(g["status"][0]) == M.MOE_ERR_BAD_INDEX
    # expected: the stable order (expert, then flat index) of the valid assignments only
    fl = flat.numpy().astype(np.int64)
    valid = np.nonzero((fl >= 0) & (fl < E))[0]
    nv = len(valid)
    order = valid[np.lexsort((valid, fl[valid]))]
    counts = np.bincount(fl[valid], minlength=E)
    np.testing.assert_array_equal(g["counts"].numpy(), counts)
    np.testing.assert_array_equal(g["offsets"].numpy(), np.concatenate([[0], np.cumsum(counts)]))
    assert g["offsets"][E].item() == nv == T * k - len(bad)
    np.testing.assert_array_equal(g["perm"][:nv].numpy(), order)
    inv = np.full(T * k, -1)
    inv[order] = np.arange(nv)
    np.testing.assert_array_equal(g["inv_perm"].numpy(), inv)
    np.testing.assert_array_equal(g["packed_tok"][:nv].numpy(), order // k)
    np.testing.assert_array_equal(g["packed_w"][:nv].numpy(), w.numpy().reshape(-1)[order])
    want = x[torch.as_tensor(order // k)]
    assert torch.equal(g["x_packed"][:nv].contiguous().view(torch.uint8),
                       want.contiguous().view(torch.uint8))
    # rows past the valid ones are left as they were
    assert (g["perm"][nv:] == -7).all() and (g["packed_tok"][nv:] == -7).all()
