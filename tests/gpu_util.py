"""Helpers shared by the GPU parity tests (device plumbing only)."""
import numpy as np
import torch

import oracle.moe_oracle as O

DEV = "cuda"

# Tolerances (max |gpu - oracle| / rms(oracle)); see the comparison rules in
# the parity tests: fp32 outputs 1e-5, bf16 outputs 2e-2.
TOL = {"f32": 1e-5, "bf16": 2e-2}


def dev(t):
    return None if t is None else t.to(DEV, non_blocking=False).contiguous()


def params_to(params: dict) -> dict:
    return {k: dev(v) for k, v in params.items()}


def rand_ids(rng, T, k, E, counts_bias=None):
    """Distinct expert ids per token (row-major [T,k]) as int32."""
    ids = np.stack([rng.choice(E, size=k, replace=False, p=counts_bias) for _ in range(T)])
    return torch.tensor(ids, dtype=torch.int32)


def ids_with_counts(counts, k, rng):
    """ids [T,k] (distinct per token) whose per-expert counts equal ``counts``.

    Assignments are dealt round-robin over tokens in expert order so that a
    token never gets the same expert twice (requires max(counts) <= T)."""
    counts = list(counts)
    N = sum(counts)
    assert N % k == 0
    T = N // k
    assert max(counts) <= T
    flat = np.concatenate([np.full(c, e) for e, c in enumerate(counts) if c]) if N else np.zeros(0)
    ids = np.empty((T, k), dtype=np.int64)
    # slot i goes to token i % T, column i // T: equal experts land in distinct tokens
    for i, e in enumerate(flat):
        ids[i % T, i // T] = e
    perm = rng.permutation(T)
    return torch.tensor(ids[perm], dtype=torch.int32)


def check_flips(l_oracle: np.ndarray, ids_gpu: np.ndarray, ids_oracle: np.ndarray, gap=1e-5):
    """Top-k flips are allowed only where the oracle's logit gap is below ``gap``.
    Returns the number of tokens whose selection differs."""
    diff = np.nonzero((ids_gpu != ids_oracle).any(axis=1))[0]
    for t in diff:
        for j in np.nonzero(ids_gpu[t] != ids_oracle[t])[0]:
            a = l_oracle[t, ids_gpu[t, j]]
            b = l_oracle[t, ids_oracle[t, j]]
            assert abs(a - b) < gap, (t, j, a, b)
    return len(diff)


def rel(got, want):
    return O.rel_err_rms(got, want)


def bf16_half_ulp(a: np.ndarray) -> np.ndarray:
    """Half a bf16 ulp at |a| (8 significant bits): the most a correctly
    rounded bf16 store can move a value."""
    a = np.abs(a)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 8)


def err_bf16_out(got, want) -> float:
    """Error of a bf16 OUTPUT against the fp64 oracle, normalised by rms(oracle):
    max over elements of |got - want| minus the output's own final rounding
    (half an ulp of the larger magnitude).  The exactly rounded oracle itself
    scores 0 here, while it would score ~2e-2 on the plain max |err| / rms."""
    g = O.to_f64(got)
    w = O.to_f64(want)
    rms = float(np.sqrt(np.mean(w * w)))
    excess = np.maximum(np.abs(g - w) - bf16_half_ulp(np.maximum(np.abs(g), np.abs(w))), 0.0)
    return float(excess.max()) / rms if g.size else 0.0


def f16_half_ulp(a: np.ndarray) -> np.ndarray:
    """Half an fp16 ulp at |a| (11 significant bits; below 2^-14 the
    subnormal spacing 2^-24): the most a correctly rounded fp16 store can
    move a value inside the fp16 range."""
    a = np.abs(a)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return 2.0 ** (e - 11)


def err_stored(got, want) -> float:
    """Error of a STORED tensor against its fp64 reference, normalised by
    rms(reference): beyond the store's own final rounding for bf16 and fp16
    tensors (half an ulp of the larger magnitude), plain for fp32."""
    if got.dtype == torch.bfloat16:
        return err_bf16_out(got, want)
    if got.dtype != torch.float16:
        return rel(got, want)
    g = O.to_f64(got)
    w = O.to_f64(want)
    rms = float(np.sqrt(np.mean(w * w)))
    excess = np.maximum(np.abs(g - w) - f16_half_ulp(np.maximum(np.abs(g), np.abs(w))), 0.0)
    return float(excess.max()) / rms if g.size else 0.0
