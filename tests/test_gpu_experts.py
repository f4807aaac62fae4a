"""Executor parity: GPU moe_experts against the oracle's experts().

Same x_packed, offsets and packed_w on both sides.  bf16 path (tcgen05):
h and y_packed within 2e-2 of the fp64 oracle (max |err| / rms; a bf16
tensor beyond its own final rounding), and y_packed within 1e-3 of the
oracle's second product fed the GPU's own h (only the fp32 accumulation
separates them); y_packed is checked both as fp16 (the default) and as fp32,
and an fp16 value beyond the fp16 range must be reported.
fp32 path: both within 1e-5.  Shapes span several tiles, ragged tails, empty
experts and rows beyond the last expert's range (which must stay untouched).
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_44_b200 as M
import oracle.moe_oracle as O
from tests.gpu_util import DEV, TOL, dev, err_bf16_out, err_stored, rel

pytestmark = pytest.mark.gpu


def _make(counts, H, I, dtype, seed=0, N=None, with_w=True):
    g = torch.Generator().manual_seed(seed)
    E = len(counts)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    N = int(offs[-1]) if N is None else N
    x = torch.randn(N, H, generator=g).to(dtype)
    w13 = (torch.randn(E, 2 * I, H, generator=g) / H ** 0.5).to(dtype)
    w2 = (torch.randn(E, H, I, generator=g) / I ** 0.5).to(dtype)
    pw = torch.rand(N, generator=g) if with_w else None
    return x, torch.tensor(offs), pw, w13, w2


def _ws(x, w13):
    N, H = x.shape
    I = w13.shape[1] // 2
    code = M.MOE_BF16 if x.dtype == torch.bfloat16 else M.MOE_F32
    return torch.zeros(max(16, M.moe_experts_workspace_bytes(N, H, I, w13.shape[0], code)),
                       dtype=torch.uint8, device=DEV)


def _bits(t):
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


def _staged(y, ref):
    return err_stored(y, ref)


def _run(x, offs, pw, w13, w2, canary=True, ws="zeros", y_dtype=None):
    N, H = x.shape
    I = w13.shape[1] // 2
    fill = 1536.0 if canary else 0.0
    if y_dtype is None:          # the default: fp16 for bf16 layers
        y_dtype = torch.float16 if x.dtype == torch.bfloat16 else torch.float32
    h = torch.full((N, I), fill, dtype=x.dtype, device=DEV)
    y = torch.full((N, H), fill, dtype=y_dtype, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    if isinstance(ws, str):
        ws = _ws(x, w13)
    M.moe_experts(dev(x), dev(offs), dev(pw), dev(w13), dev(w2), h, y, ws=ws, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    if ws is not None:       # the split-K arrival counters are back at zero
        assert int(ws[:4096 * 4].view(torch.int32).abs().sum().item()) == 0
    return h.cpu(), y.cpu()


def _check(x, offs, pw, w13, w2, tol, ws="zeros", y_dtype=None):
    h, y = _run(x, offs, pw, w13, w2, ws=ws, y_dtype=y_dtype)
    hn = int(offs[-1])
    pwn = None if pw is None else pw[:hn]
    ho, yo = O.experts(x[:hn], offs.numpy(), pwn, w13, w2)
    eh = err_bf16_out(h[:hn], ho) if h.dtype == torch.bfloat16 else rel(h[:hn], ho)
    assert eh <= tol, eh
    assert y.dtype == (y_dtype or (torch.float16 if x.dtype == torch.bfloat16 else torch.float32))
    assert _staged(y[:hn], yo) <= tol, _staged(y[:hn], yo)
    if x.dtype == torch.bfloat16:
        # the second product alone, fed the GPU's own h
        ys = O.experts_down(h[:hn], offs.numpy(), pwn, w2)
        assert _staged(y[:hn], ys) <= 1e-3, _staged(y[:hn], ys)
    # rows outside every expert's range are untouched
    assert (h[hn:].float() == 1536.0).all() and (y[hn:].float() == 1536.0).all()
    return h, y


@pytest.mark.parametrize("counts,H,I", [
    ([0, 1, 127, 300], 256, 128),            # empty, single row, one short of a tile, ragged
    ([200], 512, 256),                       # one expert, K loop wraps the 4-stage ring
    ([0, 0, 5], 256, 128),                   # N below one tile: TMA zero-fills past N
    ([128, 128, 256, 0, 129], 768, 384),     # exact tiles, then one row over
])
@pytest.mark.parametrize("y_dtype", [torch.float16, torch.float32])
def test_experts_bf16_tiles(counts, H, I, y_dtype):
    _check(*_make(counts, H, I, torch.bfloat16, seed=sum(counts)), tol=TOL["bf16"],
           y_dtype=y_dtype)


def test_experts_bf16_many_tiles_per_cta():
    rng = np.random.default_rng(0)
    counts = rng.multinomial(16384, rng.dirichlet(np.ones(8)))
    _check(*_make(list(counts), 512, 512, torch.bfloat16, seed=1), tol=TOL["bf16"])


def test_experts_bf16_rows_beyond_last_expert_untouched():
    x, offs, pw, w13, w2 = _make([40, 0, 250], 256, 128, torch.bfloat16, seed=3, N=300)
    _check(x, offs, pw, w13, w2, tol=TOL["bf16"])


def test_experts_bf16_unit_weights_for_a_shared_expert():
    x, offs, _, w13, w2 = _make([333], 256, 256, torch.bfloat16, seed=4, with_w=False)
    _check(x, offs, None, w13, w2, tol=TOL["bf16"])


def test_experts_bf16_qwen3_shape_slice():
    # I = 768, H = 2048 (the Qwen3-30B-A3B expert shape) with a skewed split
    counts = [900, 0, 37, 260, 1, 0, 0, 130]
    _check(*_make(counts, 2048, 768, torch.bfloat16, seed=5), tol=TOL["bf16"])


@pytest.mark.parametrize("counts,H,I", [
    ([10, 30, 0, 24, 16, 8, 40, 0], 128, 256),   # the tiny fp32 workload's shape
    ([65, 0, 3], 72, 40),                        # ragged H, I vs the 64 x 64 x 16 tiles
    ([1], 8, 8),
])
def test_experts_f32_simt(counts, H, I):
    _check(*_make(counts, H, I, torch.float32, seed=sum(counts) + H), tol=TOL["f32"])


@pytest.mark.parametrize("y_dtype", [torch.float16, torch.float32])
def test_experts_deterministic(y_dtype):
    args = _make([300, 17, 0, 500], 512, 256, torch.bfloat16, seed=7)
    h1, y1 = _run(*args, y_dtype=y_dtype)
    h2, y2 = _run(*args, y_dtype=y_dtype)
    assert torch.equal(h1.view(torch.int16), h2.view(torch.int16))
    assert torch.equal(_bits(y1), _bits(y2))


# Few tiles: the kernels split K across CTAs and reduce the partials in order.
@pytest.mark.parametrize("counts,H,I", [
    ([1, 0, 0, 0, 0, 1, 0, 0], 512, 1024),      # decode: one row for each of two experts
    ([0, 3, 9, 2], 1024, 512),                  # a few rows, long K for w13
    ([32], 512, 2048),                          # a shared expert at a decode batch: K = 2048 for w2
    ([300, 5, 0, 1], 1024, 256),                # full + ragged token tiles under a split
])
@pytest.mark.parametrize("y_dtype", [torch.float16, torch.float32])
def test_experts_bf16_split_k(counts, H, I, y_dtype):
    _check(*_make(counts, H, I, torch.bfloat16, seed=11 + sum(counts)), tol=TOL["bf16"],
           y_dtype=y_dtype)


def test_experts_bf16_split_k_matches_unsplit_and_is_deterministic():
    args = _make([2, 0, 7, 1], 1024, 512, torch.bfloat16, seed=12)
    h1, y1 = _run(*args)
    h2, y2 = _run(*args)
    assert torch.equal(h1.view(torch.int16), h2.view(torch.int16))
    assert torch.equal(_bits(y1), _bits(y2))
    h0, y0 = _run(*args, ws=None, y_dtype=torch.float32)   # no workspace: one unit per tile
    hn = int(args[1][-1])
    # different fp32 summation order: h may round to a neighbouring bf16 value,
    # and y (fp16) may too beyond its own rounding
    assert err_stored(y1[:hn], O.to_f64(y0[:hn])) <= 1e-3
    assert err_bf16_out(h1[:hn], O.to_f64(h0[:hn])) <= 1e-2


def test_experts_bf16_without_workspace():
    _check(*_make([1, 0, 3], 512, 512, torch.bfloat16, seed=13), tol=TOL["bf16"], ws=None)


@pytest.mark.parametrize("counts,H,I,T,Is", [
    ([2, 0, 3, 2, 5, 4, 0, 1], 512, 256, 8, 512),     # decode: split-K over both groups
    ([300, 0, 129, 40], 256, 128, 200, 384),          # prefill-like: no split
    ([0, 0, 0, 1], 256, 128, 130, 256),               # shared rows span two token tiles
])
@pytest.mark.parametrize("y_dtype", [torch.float16, torch.float32])
def test_experts_shared_matches_separate_calls(counts, H, I, T, Is, y_dtype):
    x_packed, offs, pw, w13, w2 = _make(counts, H, I, torch.bfloat16, seed=T + Is)
    g = torch.Generator().manual_seed(T)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    w13s = (torch.randn(2 * Is, H, generator=g) / H ** 0.5).to(torch.bfloat16)
    w2s = (torch.randn(H, Is, generator=g) / Is ** 0.5).to(torch.bfloat16)
    N = x_packed.shape[0]
    h = torch.full((N, I), 1536.0, dtype=torch.bfloat16, device=DEV)
    y = torch.full((N, H), 1536.0, dtype=y_dtype, device=DEV)
    hs = torch.full((T, Is), 1536.0, dtype=torch.bfloat16, device=DEV)
    ys = torch.full((T, H), 1536.0, dtype=y_dtype, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = _ws(x_packed, w13)
    M.moe_experts_shared(dev(x_packed), dev(offs), dev(pw), dev(w13), dev(w2), h, y, dev(x),
                         dev(w13s), dev(w2s), hs, ys, ws=ws, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert int(ws[:4096 * 4].view(torch.int32).abs().sum().item()) == 0
    # routed part against the oracle, as moe_experts
    ho, yo = O.experts(x_packed, offs.numpy(), pw, w13, w2)
    assert err_bf16_out(h.cpu(), ho) <= TOL["bf16"] and _staged(y.cpu(), yo) <= TOL["bf16"]
    assert _staged(y.cpu(), O.experts_down(h.cpu(), offs.numpy(), pw, w2)) <= 1e-3
    # shared part: every row of x through the dense SwiGLU MLP
    hso, yso = O.experts(x, np.array([0, T]), None, w13s.unsqueeze(0), w2s.unsqueeze(0))
    assert err_bf16_out(hs.cpu(), hso) <= TOL["bf16"] and _staged(ys.cpu(), yso) <= TOL["bf16"]
    one = np.array([0, T])
    assert _staged(ys.cpu(), O.experts_down(hs.cpu(), one, None, w2s.unsqueeze(0))) <= 1e-3
    np.testing.assert_allclose(ys.cpu().float().numpy(), O.shared_expert(x, w13s, w2s), rtol=0,
                               atol=TOL["bf16"] * float(np.sqrt(np.mean(yso ** 2))))
    # the same launch twice gives the same bits
    y2 = torch.empty_like(y); ys2 = torch.empty_like(ys)
    M.moe_experts_shared(dev(x_packed), dev(offs), dev(pw), dev(w13), dev(w2), h, y2, dev(x),
                         dev(w13s), dev(w2s), hs, ys2, ws=ws, status=status)
    torch.cuda.synchronize()
    assert torch.equal(y2, y) and torch.equal(ys2, ys)


def test_experts_fp16_y_overflow_is_reported_not_faulted():
    # activations and w2 scaled so that some outputs exceed the fp16 range
    x, offs, pw, w13, w2 = _make([40, 0, 90], 256, 128, torch.bfloat16, seed=21)
    x = (x.float() * 16).to(torch.bfloat16)
    w2 = (w2.float() * 128).to(torch.bfloat16)
    N, H = x.shape
    I = w13.shape[1] // 2
    for y_dtype, want in ((torch.float16, M.MOE_ERR_OVERFLOW), (torch.float32, 0)):
        h = torch.empty(N, I, dtype=torch.bfloat16, device=DEV)
        y = torch.empty(N, H, dtype=y_dtype, device=DEV)
        st = torch.zeros(1, dtype=torch.int32, device=DEV)
        M.moe_experts(dev(x), dev(offs), dev(pw), dev(w13), dev(w2), h, y, ws=_ws(x, w13),
                      status=st)
        torch.cuda.synchronize()
        # the second product fed the GPU's own h
        ys = O.experts_down(h.cpu(), offs.numpy(), pw, w2)
        assert np.abs(ys).max() > 65520.0 * 1.5          # the case is real
        assert int(st.item()) == want, y_dtype
        yc = y.cpu()
        if y_dtype == torch.float16:
            big = torch.as_tensor(np.abs(ys) > 65520.0 * 1.01)   # these round to inf
            assert torch.isinf(yc[big]).all()
            ok = torch.as_tensor(np.abs(ys) < 60000.0)
            assert err_stored(yc[ok], ys[ok.numpy()]) <= 1e-3
        else:
            assert rel(yc, ys) <= 1e-3


# Experts with several token tiles beside single-tile and empty ones, K not
# split: without a workspace (static units) and with one when there are enough
# tiles (dynamic units).
@pytest.mark.parametrize("counts,H,I,ws", [
    ([300, 5, 0, 700, 60, 1, 200, 40], 512, 512, None),
    ([2000, 5, 3000, 1, 90, 0, 700, 33], 512, 1024, "zeros"),
])
def test_experts_mixed_sizes_unsplit(counts, H, I, ws):
    _check(*_make(counts, H, I, torch.bfloat16, seed=sum(counts) + I), tol=TOL["bf16"], ws=ws)
