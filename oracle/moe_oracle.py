"""fp64 CPU oracle for the forward pass of one Mixture-of-Experts layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or
call this module.  The CUDA library never uses it and shares no code with it.

It is the plain definition of the layer, written from the stage contracts of
the DWDP-Triton-MoE-Inference-Engine README ("Router Module", "Dispatcher
Module", "Executor Module", "Merger Module", "Runtime Integration Layer"),
the diffulex.moe API reference (``diffulex.moe.topk``: ``NaiveTopKRouter``;
``diffulex.moe.layer``: ``NaiveFusedMoE``, ``SharedExpertMLP``), the fused
``w13`` layout of the modelexpress-client test
``test_reshard_refit_moe_experts.py`` (``FusedMoEModel``: gate w1 in the low
half, up w3 in the high half of ``[E, 2*I, H]``) and the flat assignment
order of metrale's ``ep_dispatch.rs`` (``build_ep_routing_table``: entry
``token * top_k + k`` of a row-major ``[num_tokens, top_k]`` table).

Everything is float64.  bf16 / fp32 inputs are converted exactly first.  No
blocking, fusion or reordering beyond the definitions below.  Readings of
points the pages leave open (tie-break, selection on logits, offsets length,
where routing weights are applied, the shared-expert gate) are stated at each
function.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "to_f64", "router_logits", "softmax_rows", "topk_experts", "topk_experts_grouped",
    "routing_weights",
    "route", "route_from_logits", "dispatch", "gather_rows", "silu", "w13_halves",
    "expert_hidden", "expert_output", "experts", "experts_down", "combine", "shared_expert",
    "shared_gate_logit", "moe_forward", "moe_forward_tokens", "ep_partition",
    "expert_ranges", "expert_owner", "tp_slice", "moe_forward_tokens_ep",
    "moe_forward_tokens_tp", "rel_err_rms",
]


def to_f64(t) -> np.ndarray:
    """Exact conversion of a torch tensor (bf16 / fp32 / int) or array to float64 numpy."""
    if t is None:
        return None
    if hasattr(t, "detach"):                      # torch tensor, any device
        t = t.detach()
        if t.device.type != "cpu":
            t = t.cpu()
        if t.is_floating_point():
            return t.double().numpy()
        return t.numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def _ints(t) -> np.ndarray:
    if hasattr(t, "detach"):
        t = t.detach().cpu().numpy()
    return np.asarray(t).astype(np.int64)


# ---------------------------------------------------------------- Router ---

def router_logits(x, W_gate, bias=None) -> np.ndarray:
    """Router logits l[t,e] = sum_h x[t,h] * W_gate[e,h] (+ bias[e]).

    DWDP README, "Router Module": the router produces router logits.  W_gate is
    stored [E, H] (Linear convention, pages silent); the per-expert bias, when a
    workload has one, is added to the logits before softmax and selection.
    """
    l = to_f64(x) @ to_f64(W_gate).T
    if bias is not None:
        l = l + to_f64(bias)[None, :]
    return l


def softmax_rows(l: np.ndarray) -> np.ndarray:
    """Routing probabilities p = softmax(l) over all E experts of each token
    (DWDP README, "Router Module": routing probabilities).  The row max is
    subtracted first, which is exact in real arithmetic."""
    z = l - l.max(axis=1, keepdims=True)
    ez = np.exp(z)
    return ez / ez.sum(axis=1, keepdims=True)


def topk_experts(l: np.ndarray, k: int) -> np.ndarray:
    """Top-k expert indices (DWDP README, "Router Module"; diffulex.moe.topk,
    ``NaiveTopKRouter``: standard top-k router).

    Experts are ordered by the key (-logit, expert id) and the first k are
    taken, in that order: equal logits go to the lower expert id, and the k ids
    of a token are listed by descending logit.  Selection uses logits, which
    picks the same set as selection on softmax probabilities (softmax is
    strictly increasing) without ties made by rounding p.
    """
    # argsort of -l with a stable sort keeps ascending expert id among equal keys.
    order = np.argsort(-l, axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


def topk_experts_grouped(l: np.ndarray, k: int, n_groups: int, topk_groups: int) -> np.ndarray:
    """Group-limited top-k (diffulex.moe API reference, ``diffulex.moe.topk``:
    ``GroupLimitedTopKRouter``, "router with group-limited expert selection";
    the page gives no formula, so the plainest reading is taken):

    1. the E experts form ``n_groups`` equal groups of consecutive ids,
       group g = experts [g*E/G, (g+1)*E/G);
    2. a group's score is the largest logit among its experts;
    3. the ``topk_groups`` groups with the highest scores are kept (equal
       scores -> lower group id first);
    4. the k experts are chosen among the kept groups' experts exactly as
       topk_experts chooses them among all (key (-logit, expert id)).
    The routing weights stay the softmax over all E experts (routing_weights).
    """
    T, E = l.shape
    gs = E // n_groups
    out = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        score = [max(l[t, g * gs:(g + 1) * gs]) for g in range(n_groups)]
        groups = sorted(range(n_groups), key=lambda g: (-score[g], g))[:topk_groups]
        cand = [e for g in sorted(groups) for e in range(g * gs, (g + 1) * gs)]
        cand.sort(key=lambda e: (-l[t, e], e))
        out[t] = cand[:k]
    return out


def routing_weights(l: np.ndarray, ids: np.ndarray, renormalize: bool) -> np.ndarray:
    """Routing weights of the selected experts (DWDP README, "Router Module":
    normalized routing weights).

    w[t,j] = p[t, ids[t,j]] with p = softmax over all E.  When the workload
    renormalises, the k weights are divided by their sum, so they sum to 1.
    """
    p = softmax_rows(l)
    w = np.take_along_axis(p, ids, axis=1)
    if renormalize:
        w = w / w.sum(axis=1, keepdims=True)
    return w


def route(x, W_gate, bias, k: int, renormalize: bool):
    """Full router: (logits [T,E], ids [T,k], weights [T,k])."""
    l = router_logits(x, W_gate, bias)
    ids = topk_experts(l, k)
    return l, ids, routing_weights(l, ids, renormalize)


def route_from_logits(logits, k: int, renormalize: bool, n_groups: int = 1,
                      topk_groups: int = 1):
    """Selection and weights from given logits (e.g. fp32 logits made elsewhere);
    n_groups > 1 selects group-limited (topk_experts_grouped)."""
    l = to_f64(logits)
    if n_groups > 1:
        ids = topk_experts_grouped(l, k, n_groups, topk_groups)
    else:
        ids = topk_experts(l, k)
    return ids, routing_weights(l, ids, renormalize)


# ------------------------------------------------------------ Dispatcher ---

def dispatch(ids, w, E: int) -> dict:
    """Token-major to expert-major layout (DWDP README, "Dispatcher Module":
    per-expert counts, expert offsets, token permutation, inverse
    permutation, packed token indices, packed routing weights).

    Assignment f = t*k + j is entry j of token t in the row-major [T, k] table
    (metrale ep_dispatch.rs, ``build_ep_routing_table``).  Readings:
      counts[e]   = number of assignments to expert e;
      offsets     = E+1 entries, offsets[0] = 0, offsets[e+1] = offsets[e] + counts[e];
      position    p(f) = offsets[e(f)] + #{f' < f : e(f') = e(f)}  (stable:
                    inside an expert, assignments keep their given order, as
                    the ep_dispatch.rs buckets do);
      perm[p]     = f (expert-major position -> assignment);
      inv_perm[f] = p;
      packed_tok[p] = f // k (the token, not the assignment);
      packed_w[p]   = w_flat[f].
    """
    ids = _ints(ids)
    T, k = ids.shape
    N = T * k
    ids_flat = ids.reshape(N)
    w_flat = to_f64(w).reshape(N)
    counts = np.zeros(E, dtype=np.int64)
    for f in range(N):
        counts[ids_flat[f]] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    seen = np.zeros(E, dtype=np.int64)
    perm = np.empty(N, dtype=np.int64)
    inv_perm = np.empty(N, dtype=np.int64)
    for f in range(N):
        e = ids_flat[f]
        p = offsets[e] + seen[e]
        seen[e] += 1
        perm[p] = f
        inv_perm[f] = p
    packed_tok = perm // k
    packed_w = w_flat[perm]
    return dict(counts=counts, offsets=offsets, perm=perm, inv_perm=inv_perm,
                packed_tok=packed_tok, packed_w=packed_w)


def gather_rows(x, packed_tok) -> np.ndarray:
    """Gather token activations into expert-major order (DWDP README,
    "Executor Module": gather token activations for scheduled expert ranges):
    x_packed[p] = x[packed_tok[p]]."""
    return to_f64(x)[_ints(packed_tok)]


# -------------------------------------------------------------- Executor ---

def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z / (1 + exp(-z))."""
    return z / (1.0 + np.exp(-z))


def w13_halves(w13_e, I: int):
    """Split one expert's fused [2I, H] slot into (gate w1, up w3).

    modelexpress-client test_reshard_refit_moe_experts.py, ``FusedMoEModel``:
    the fused buffer stacks gate (w1) then up (w3); member 0 (w1) occupies rows
    [0, I) and member 1 (w3) rows [I, 2I) of the expert's slot.
    """
    return w13_e[:I], w13_e[I:2 * I]


def expert_hidden(x_rows: np.ndarray, w13_e, I: int) -> np.ndarray:
    """SwiGLU hidden h = silu(x W1^T) * (x W3^T) for rows of one expert."""
    W1, W3 = w13_halves(to_f64(w13_e), I)
    return silu(x_rows @ W1.T) * (x_rows @ W3.T)


def expert_output(x_rows: np.ndarray, w13_e, w2_e, I: int) -> np.ndarray:
    """One SwiGLU expert applied to rows: (silu(x W1^T) * (x W3^T)) W2^T, W2 [H, I]."""
    return expert_hidden(x_rows, w13_e, I) @ to_f64(w2_e).T


def experts_down(h, offsets, packed_w, w2):
    """The Executor's second product alone, fed a given hidden h [N, I]: for
    each expert e and position p in its range, y_packed[p] = packed_w[p] *
    (h[p] W2e^T).  experts() is expert_hidden followed by this step; fed the
    hidden of a device, it checks that device's second product by itself."""
    hh = to_f64(h)
    offs = _ints(offsets)
    E = len(offs) - 1
    N = hh.shape[0]
    H = w2.shape[1]
    y = np.zeros((N, H))
    pw = np.ones(N) if packed_w is None else to_f64(packed_w)
    for e in range(E):
        a, b = offs[e], offs[e + 1]
        if b == a:
            continue
        y[a:b] = pw[a:b, None] * (hh[a:b] @ to_f64(w2[e]).T)
    return y


def experts(x_packed, offsets, packed_w, w13, w2):
    """Expert execution over expert-major ranges (DWDP README, "Executor
    Module": execute expert modules, apply routing weights, write packed
    expert outputs).

    For each expert e and each position p in [offsets[e], offsets[e+1]):
    h[p] = silu(x_p W1e^T) * (x_p W3e^T) and y_packed[p] = packed_w[p] * (h[p] W2e^T).
    Routing weights are applied here, once; the merger then only sums (the
    README lets the merger apply them "optionally"; the sum is the same).
    ``packed_w=None`` means every weight is 1.  Returns (h, y_packed).
    """
    xp = to_f64(x_packed)
    offs = _ints(offsets)
    E = len(offs) - 1
    N = xp.shape[0]
    I = w13.shape[1] // 2
    H = w2.shape[1]
    h = np.zeros((N, I))
    for e in range(E):
        a, b = offs[e], offs[e + 1]
        if b == a:
            continue
        h[a:b] = expert_hidden(xp[a:b], w13[e], I)
    return h, experts_down(h, offs, packed_w, w2)


# ---------------------------------------------------------------- Merger ---

def shared_expert(x, w13s, w2s) -> np.ndarray:
    """Always-on shared SwiGLU expert (diffulex.moe.layer, ``SharedExpertMLP``),
    same fused gate/up layout as the routed experts."""
    Is = w13s.shape[0] // 2
    return expert_output(to_f64(x), w13s, w2s, Is)


def shared_gate_logit(x, w_sg) -> np.ndarray:
    """Scalar gate logit per token, x_t . w_sg (no bias); the merger scales the
    shared expert's output by sigmoid of it."""
    return to_f64(x) @ to_f64(w_sg)


def combine(y_packed, inv_perm, T: int, k: int, shared=None, shared_gate=None) -> np.ndarray:
    """Merge back to token order (DWDP README, "Merger Module": restore
    token-major assignment order, accumulate top-k expert outputs, reshape to
    the token layout).

    out[t] = sum_{j<k} y_packed[inv_perm[t*k + j]]; with a shared expert,
    out[t] += sigmoid(shared_gate[t]) * shared[t].
    """
    y = to_f64(y_packed)
    ip = _ints(inv_perm)
    H = y.shape[1]
    out = np.zeros((T, H))
    for j in range(k):
        out += y[ip[np.arange(T) * k + j]]
    if shared is not None:
        g = 1.0 / (1.0 + np.exp(-to_f64(shared_gate)))
        out += g[:, None] * to_f64(shared)
    return out


# ---------------------------------------------------------- whole layer ---

def moe_forward(params: dict, k: int, renormalize: bool, ids=None, logits=None) -> dict:
    """Staged forward, stage by stage in the runtime's order (DWDP README,
    "Runtime Integration Layer": Router -> Dispatcher -> ... -> Executor ->
    Merger).  ``logits`` (e.g. a device's fp32 logits) replaces the router GEMM;
    ``ids`` replaces the selection.  Returns every intermediate."""
    x = params["x"]
    E = params["W_gate"].shape[0]
    T = x.shape[0]
    if logits is None:
        l = router_logits(x, params["W_gate"], params.get("bias"))
    else:
        l = to_f64(logits)
    sel = topk_experts(l, k) if ids is None else _ints(ids)
    w = routing_weights(l, sel, renormalize)
    d = dispatch(sel, w, E)
    xp = gather_rows(x, d["packed_tok"])
    h, y = experts(xp, d["offsets"], d["packed_w"], params["w13"], params["w2"])
    shared = sg = None
    if params.get("w13s") is not None:
        shared = shared_expert(x, params["w13s"], params["w2s"])
        sg = shared_gate_logit(x, params["w_sg"])
    out = combine(y, d["inv_perm"], T, k, shared, sg)
    return dict(logits=l, ids=sel, w=w, x_packed=xp, h=h, y_packed=y,
                shared=shared, shared_gate=sg, out=out, **d)


def moe_forward_tokens(params: dict, tokens, ids, w) -> np.ndarray:
    """Direct per-token form for a subset of tokens, given their routing:
    out[t] = sum_j w[t,j] * SwiGLU_{ids[t,j]}(x_t) (+ sigmoid(x_t.w_sg) * SwiGLU_s(x_t)).

    diffulex.moe.layer, ``NaiveFusedMoE`` (reference fused MoE): each token's
    output is the routing-weighted sum of its selected experts.  ``ids`` and
    ``w`` are [len(tokens), k].  Rows of the same expert are batched into one
    matmul (a library primitive); nothing else is reordered.
    """
    tokens = _ints(tokens)
    ids = _ints(ids)
    w = to_f64(w)
    xs = to_f64(params["x"])[tokens]
    I = params["w13"].shape[1] // 2
    H = params["w2"].shape[1]
    out = np.zeros((len(tokens), H))
    for e in np.unique(ids):
        rows, cols = np.nonzero(ids == e)
        y = expert_output(xs[rows], params["w13"][int(e)], params["w2"][int(e)], I)
        np.add.at(out, rows, w[rows, cols][:, None] * y)
    if params.get("w13s") is not None:
        s = shared_expert(xs, params["w13s"], params["w2s"])
        g = 1.0 / (1.0 + np.exp(-shared_gate_logit(xs, params["w_sg"])))
        out += g[:, None] * s
    return out


# ------------------------------------------------- expert-parallel split ---

def ep_partition(gate_indices, gate_weights, num_tokens: int, top_k: int,
                 local_start: int, local_end: int) -> dict:
    """Split the row-major [num_tokens, top_k] assignments into a local bucket
    (expert id in [local_start, local_end)) and a remote bucket, each in the
    order the assignments were given (metrale ep_dispatch.rs,
    ``EpRoutingTable`` / ``build_ep_routing_table``).  A length other than
    num_tokens * top_k raises ValueError (the Rust code panics)."""
    total = num_tokens * top_k
    if len(gate_indices) != total:
        raise ValueError("gate_indices length mismatch")
    if len(gate_weights) != total:
        raise ValueError("gate_weights length mismatch")
    b = {f"{side}_{what}": [] for side in ("local", "remote")
         for what in ("token_indices", "expert_ids", "weights")}
    for t in range(num_tokens):
        for j in range(top_k):
            f = t * top_k + j
            e = int(gate_indices[f])
            side = "local" if local_start <= e < local_end else "remote"
            b[f"{side}_token_indices"].append(t)
            b[f"{side}_expert_ids"].append(e)
            b[f"{side}_weights"].append(gate_weights[f])
    return b


# ------------------------------------- expert / tensor parallel forms ---

def expert_ranges(E: int, world: int):
    """Contiguous expert ranges of ``world`` ranks: rank q owns
    [floor(E*q/world), floor(E*(q+1)/world)) -- the local_expert_start ..
    local_expert_end of metrale's build_ep_routing_table, one range per rank,
    every expert on exactly one rank (the pages leave the split open; this is
    the plain even split)."""
    return [(E * q // world, E * (q + 1) // world) for q in range(world)]


def expert_owner(expert_ids, E: int, world: int) -> np.ndarray:
    """Owning rank of each expert id: the range of expert_ranges() holding it,
    found by a plain search."""
    ids = _ints(expert_ids)
    ranges = expert_ranges(E, world)
    out = np.empty(ids.shape, dtype=np.int64)
    for i, e in np.ndenumerate(ids):
        out[i] = next(q for q, (a, b) in enumerate(ranges) if a <= e < b)
    return out


def tp_slice(w13_e, w2_e, rank: int, tp: int):
    """One expert's tensor-parallel slice (modelexpress refit test,
    ``FusedMoEModel._expert_loader``: take this rank's slice of the source --
    rows [rank*I/tp, (rank+1)*I/tp) -- of w1 and of w3, and store them w1 low,
    w3 high in the rank's [2*I/tp, H] slot).  The down projection w2 [H, I]
    keeps the same I columns (the pages show only w13; splitting w2 along its
    input dimension is the reading under which the ranks' outputs add up).
    Returns (w13 slot [2*I/tp, H], w2 slice [H, I/tp]) in float64."""
    w13_e = to_f64(w13_e)
    w2_e = to_f64(w2_e)
    I = w13_e.shape[0] // 2
    it = I // tp
    w1, w3 = w13_halves(w13_e, I)
    slot = np.empty((2 * it, w13_e.shape[1]))
    slot[0:it] = w1[rank * it:(rank + 1) * it]          # member 0 (w1): low half
    slot[it:2 * it] = w3[rank * it:(rank + 1) * it]     # member 1 (w3): high half
    return slot, w2_e[:, rank * it:(rank + 1) * it]


def moe_forward_tokens_ep(params: dict, tokens, ids, w, start: int, end: int,
                          with_shared: bool) -> np.ndarray:
    """Masked-local partial of an expert-parallel rank owning experts
    [start, end) (metrale ep_dispatch.rs, module doc: "masked-local plus
    all-reduce"): out[t] = sum over j with start <= ids[t,j] < end of
    w[t,j] * SwiGLU_{ids[t,j]}(x_t), plus the shared term on the one rank that
    holds the shared expert.  The ranks' partials add up to the layer."""
    tokens = _ints(tokens)
    ids = _ints(ids)
    w = to_f64(w)
    xs = to_f64(params["x"])[tokens]
    I = params["w13"].shape[1] // 2
    H = params["w2"].shape[1]
    out = np.zeros((len(tokens), H))
    for e in np.unique(ids):
        if not start <= e < end:
            continue                                   # another rank's expert
        rows, cols = np.nonzero(ids == e)
        y = expert_output(xs[rows], params["w13"][int(e)], params["w2"][int(e)], I)
        np.add.at(out, rows, w[rows, cols][:, None] * y)
    if with_shared and params.get("w13s") is not None:
        s = shared_expert(xs, params["w13s"], params["w2s"])
        g = 1.0 / (1.0 + np.exp(-shared_gate_logit(xs, params["w_sg"])))
        out += g[:, None] * s
    return out


def moe_forward_tokens_tp(params: dict, tokens, ids, w, rank: int, tp: int) -> np.ndarray:
    """Partial of tensor-parallel rank ``rank`` of ``tp``: every selected
    expert (and the shared one) run on the rank's I-slice (tp_slice); the
    ranks' partials add up to the layer."""
    tokens = _ints(tokens)
    ids = _ints(ids)
    w = to_f64(w)
    xs = to_f64(params["x"])[tokens]
    H = params["w2"].shape[1]
    out = np.zeros((len(tokens), H))
    for e in np.unique(ids):
        rows, cols = np.nonzero(ids == e)
        slot, w2r = tp_slice(params["w13"][int(e)], params["w2"][int(e)], rank, tp)
        y = expert_output(xs[rows], slot, w2r, slot.shape[0] // 2)
        np.add.at(out, rows, w[rows, cols][:, None] * y)
    if params.get("w13s") is not None:
        slot, w2r = tp_slice(params["w13s"], params["w2s"], rank, tp)
        s = expert_output(xs, slot, w2r, slot.shape[0] // 2)
        g = 1.0 / (1.0 + np.exp(-shared_gate_logit(xs, params["w_sg"])))
        out += g[:, None] * s
    return out


# ------------------------------------------------------------- metrics ---

def rel_err_rms(got, want) -> float:
    """max |got - want| / rms(want): the error measure the tolerances use."""
    g = to_f64(got)
    w = to_f64(want)
    rms = float(np.sqrt(np.mean(w * w)))
    if rms == 0.0:
        return float(np.max(np.abs(g - w))) if g.size else 0.0
    return float(np.max(np.abs(g - w))) / rms if g.size else 0.0
