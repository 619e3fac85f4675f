"""Oracle for the MoE-layer forward pass: plain, slow, fp64, CPU only.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run
this module. The product path (the CUDA library and its Python binding) never
calls it, and this module imports nothing from the product package.

Every function states the plain definition of one step of the layer, in
float64, with numpy (and ``scipy.special.erfc``) as the only library
primitives. Inputs are taken at their exact stored values (fp32 or bf16
widened to fp64; bf16 arrives here already widened to fp32 by the caller,
which is exact). Sources, by page and section:

* EC-DiT: Scaling Diffusion Transformers with Adaptive Expert-Choice Routing
  (ByteDance), section 3 "core formulas": token-choice routing (each token
  picks its top-k experts), expert-choice routing (each expert picks its
  top tokens), the "Expert-Choice routing formula" (router affinity
  A = softmax over the E experts of x'.W_r) and the "capacity factor"
  (Capacity = f_c * S / E, f_c = 2.0).
* DICE: Staleness-Centric Optimizations for Parallel Diffusion MoE
  Inference, "Conditional Communication": the layer output is the
  routing-score weighted sum of the expert outputs.
* Dynamic Expert Sharing: Decoupling Memory from Parallelism in
  Mixture-of-Experts Diffusion LLMs, section 2.3 "DES-Seq" (the core set is
  the union of every token's top-k_local), section 2.4 "DES-Vote" (filter
  to the own top-K, vote with the routing weights, elect the M_core most
  voted),
  section 3.1 (M_core = beta * M) and section 4.3 (tokens re-activate
  experts from the core set at their original per-token count).
* MMOE: Modernizing Diffusion Transformers with Efficient Expert Design,
  "Methodology": MoE++ expert layer (heavy MLP experts plus identity, zero
  and constant zero-computation experts), gate-residual routing (the
  previous expert layer's gate logits are carried into the router) and an
  always-active shared expert.

Where the pages are silent the reading taken is stated at the function and
listed with the others in the design notes (readings R1-R20).

Every function here is pinned by tests/test_oracle_pins.py against closed
forms, brute force on tiny inputs and invariants the pages fix.
"""

from __future__ import annotations

import math

import numpy as np
from scipy.special import erfc as _erfc

# Expert kinds (MMOE page, "MoE++ expert layer").
HEAVY, IDENTITY, ZERO, CONST = 0, 1, 2, 3

# DES vote fixed point: a vote q(p) = rint(p * 2**40) as an int64 (reading R8).
VOTE_SCALE_LOG2 = 40


def _f64(a):
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------
# Router (EC-DiT page, "Expert-Choice routing formula"; MMOE page,
# "gate-residual routing").
# --------------------------------------------------------------------------
def router_logits(x, W_r, logit_bias=None, z_prev=None, z_prev_scale=0.0):
    """z = x . W_r (+ b) (+ lambda * z_prev), fp64.

    ``x`` is [T, d]; ``W_r`` is stored [E, d] (row e holds expert e's router
    weights, i.e. the transpose of the pages' d x E matrix). ``logit_bias``
    [E] is an optional per-expert bias (used only to skew synthetic
    workloads). ``z_prev`` [T, E] is the previous expert layer's gate
    logits, added with weight ``z_prev_scale`` before the softmax
    (gate-residual routing, reading R16).
    """
    z = _f64(x) @ _f64(W_r).T
    if logit_bias is not None:
        z = z + _f64(logit_bias)[None, :]
    if z_prev is not None:
        z = z + float(z_prev_scale) * _f64(z_prev)
    return z


def softmax_rows(z):
    """A[s, i] = exp(z[s, i]) / sum_j exp(z[s, j]) (EC-DiT affinity A).

    The row maximum is subtracted first; that leaves the quotient unchanged
    and keeps exp in range.
    """
    z = _f64(z)
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    return e / e.sum(axis=1, keepdims=True)


# --------------------------------------------------------------------------
# Selection.
# --------------------------------------------------------------------------
def _order_desc(keys, ids):
    """Indices sorting by (key descending, id ascending) (reading R6).

    numpy compares -0.0 == +0.0, so those are a tie and the lower id wins.
    """
    keys = _f64(keys)
    return np.lexsort((np.asarray(ids), -keys))


def topk_token_choice(z, k):
    """Token choice: every token keeps its k highest-affinity experts.

    EC-DiT page, "Token-Choice routing": each token selects its top-k
    experts; dropless (no capacity, reading R3). Ranking key is the logit z
    (softmax is monotone; reading R7); ties go to the lower expert id.
    Returns idx [T, k] int32 in rank order.
    """
    z = _f64(z)
    T, E = z.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    ids = np.arange(E)
    idx = np.empty((T, k), dtype=np.int32)
    for s in range(T):
        idx[s] = _order_desc(z[s], ids)[:k]
    return idx


def gather_weights(A, idx):
    """Routing weight of each selected pair: w = A[s, idx[s, j]] (reading R2)."""
    A = _f64(A)
    return np.take_along_axis(A, np.asarray(idx, dtype=np.int64), axis=1)


def renormalize(w):
    """Optional variant: weights renormalised over the selected set."""
    w = _f64(w)
    return w / w.sum(axis=1, keepdims=True)


def capacity(S, E, f_c):
    """EC-DiT page, "capacity factor": Capacity = f_c * S / E.

    Non-integers are floored and the result is clamped to [1, S]
    (reading R4).
    """
    c = math.floor(float(f_c) * S / E)
    return max(1, min(S, c))


def expert_choice(A, group_size, C):
    """Expert choice: each expert picks the C tokens with highest affinity.

    EC-DiT page, "Expert-Choice routing" and "capacity factor". The routing
    group is one sequence of ``group_size`` tokens (the router sees the
    whole sequence; reading R5); A is ranked per expert column within the
    group, ties to the lower token id (R6, R7).

    Returns ``tok`` [G, E, C] int32 of GLOBAL token ids in ascending order
    within each (group, expert), and ``w`` [G, E, C] = A[tok, e].
    """
    A = _f64(A)
    T, E = A.shape
    S = int(group_size)
    if T % S != 0:
        raise ValueError("T must be a multiple of the group size")
    if not 1 <= C <= S:
        raise ValueError("need 1 <= C <= S")
    G = T // S
    tok = np.empty((G, E, C), dtype=np.int32)
    w = np.empty((G, E, C), dtype=np.float64)
    local = np.arange(S)
    for g in range(G):
        block = A[g * S:(g + 1) * S]
        for e in range(E):
            chosen = np.sort(_order_desc(block[:, e], local)[:C])
            tok[g, e] = g * S + chosen
            w[g, e] = block[chosen, e]
    return tok, w


def vote_quantum(p):
    """q(p) = round-half-even(p * 2**40) as int64 (reading R8).

    Multiplying by a power of two is exact in binary floating point, so for
    any fp32 or fp64 p the only rounding is the final rint.
    """
    return np.rint(_f64(p) * float(2 ** VOTE_SCALE_LOG2)).astype(np.int64)


def des_vote(P, K, M_core):
    """DES-Vote core set and restricted re-routing.

    Dynamic Expert Sharing page, section 2.4 "DES-Vote":
      (i)   filter: every token n keeps only its own top-K experts;
      (ii)  vote: the kept experts' routing weights are summed over tokens;
      (iii) elect: the M_core experts with the highest total form the core set.
    Section 3.1: M_core = beta * M. Section 4.3: tokens then re-activate
    experts from the core set at their original per-token count K
    (reading R11: each token takes its K largest P over the core set).

    ``P`` is [N, M] routing probabilities. Votes are int64 fixed point
    (R8); ties go to the lower expert id everywhere (R6); the core set
    always holds exactly M_core experts (R10). Weights are P itself (R9).

    Returns votes [M] int64, core [M_core] int32 ascending, idx [N, K] int32
    (rank order), w [N, K].
    """
    P = _f64(P)
    N, M = P.shape
    if not 1 <= K <= M:
        raise ValueError("need 1 <= K <= M")
    if not K <= M_core <= M:
        raise ValueError("need K <= M_core <= M")
    ids = np.arange(M)
    votes = np.zeros(M, dtype=np.int64)
    for n in range(N):
        for e in _order_desc(P[n], ids)[:K]:
            votes[e] += vote_quantum(P[n, e])
    elected = np.lexsort((ids, -votes))[:M_core]
    core = np.sort(elected).astype(np.int32)
    idx = np.empty((N, K), dtype=np.int32)
    for n in range(N):
        order = _order_desc(P[n, core], core)[:K]
        idx[n] = core[order]
    w = np.take_along_axis(P, idx.astype(np.int64), axis=1)
    return votes, core, idx, w


def des_seq(P, K, k_local):
    """DES-Seq core set and restricted re-routing.

    Dynamic Expert Sharing page, section 2.3 "DES-Seq": every token n of the
    block selects its k_local most salient experts (its top-k_local by P);
    the core set is the union of these local selections. Section 2.2: the
    tokens' expert selection is then restricted to the core set; section
    4.3: at the original per-token count K. Reading: each token takes its
    min(K, |core|) largest P over the core set, in rank order (ties to the
    lower id, R6); when the core holds fewer than K experts the remaining
    slots are empty (expert -1, weight 0). Weights are P itself (R9).

    Returns core [|core|] int32 ascending, idx [N, K] int32, w [N, K].
    """
    P = _f64(P)
    N, M = P.shape
    if not 1 <= K <= M:
        raise ValueError("need 1 <= K <= M")
    if not 1 <= k_local <= M:
        raise ValueError("need 1 <= k_local <= M")
    ids = np.arange(M)
    in_core = np.zeros(M, dtype=bool)
    for n in range(N):
        in_core[_order_desc(P[n], ids)[:k_local]] = True
    core = np.nonzero(in_core)[0].astype(np.int32)
    idx = np.full((N, K), -1, dtype=np.int32)
    w = np.zeros((N, K))
    take = min(K, core.shape[0])
    for n in range(N):
        order = _order_desc(P[n, core], core)[:take]
        idx[n, :take] = core[order]
        w[n, :take] = P[n, core[order]]
    return core, idx, w


def des_core_size(M, beta):
    """Dynamic Expert Sharing page, section 3.1: M_core = beta * M (floored)."""
    return int(math.floor(float(beta) * M))


# --------------------------------------------------------------------------
# Dispatch: a stable permutation into per-expert groups.
# --------------------------------------------------------------------------
def dispatch(a_tok, a_exp, n_heavy, n_tokens):
    """Group the heavy assignments by expert, stably.

    ``a_tok[a]``, ``a_exp[a]`` describe assignment a in slot order (token
    choice: a = s*k + j; expert choice: a = (g*E + e)*C + c; DES: a = n*K + j).
    Only experts with id < n_heavy get rows. Rows are ordered by
    (expert ascending, assignment ascending), which is ascending token
    within each expert for all three routings.

    Returns
      offsets  [n_heavy + 1] int32: rows of expert e are offsets[e]:offsets[e+1]
      perm     [n_rows] int32: token of each row (x_perm[r] = x[perm[r]])
      row_of   [n_assign] int32: row of assignment a, -1 when not heavy
      tok_ptr  [n_tokens + 1] int32, tok_assign [n_assign] int32: the
               assignments of each token, in slot order (a CSR by token).
    """
    a_tok = np.asarray(a_tok, dtype=np.int64)
    a_exp = np.asarray(a_exp, dtype=np.int64)
    n_assign = a_tok.shape[0]
    counts = np.zeros(n_heavy, dtype=np.int64)
    for a in range(n_assign):
        if 0 <= a_exp[a] < n_heavy:  # -1: an empty slot (DES-Seq), no row
            counts[a_exp[a]] += 1
    offsets = np.zeros(n_heavy + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    fill = offsets[:-1].copy()
    perm = np.empty(int(offsets[-1]), dtype=np.int32)
    row_of = np.full(n_assign, -1, dtype=np.int32)
    for a in range(n_assign):
        e = a_exp[a]
        if 0 <= e < n_heavy:
            r = fill[e]
            fill[e] += 1
            perm[r] = a_tok[a]
            row_of[a] = r
    tcount = np.zeros(n_tokens, dtype=np.int64)
    for a in range(n_assign):
        tcount[a_tok[a]] += 1
    tok_ptr = np.zeros(n_tokens + 1, dtype=np.int64)
    tok_ptr[1:] = np.cumsum(tcount)
    tfill = tok_ptr[:-1].copy()
    tok_assign = np.empty(n_assign, dtype=np.int32)
    for a in range(n_assign):
        t = a_tok[a]
        tok_assign[tfill[t]] = a
        tfill[t] += 1
    return (offsets.astype(np.int32), perm, row_of,
            tok_ptr.astype(np.int32), tok_assign)


# --------------------------------------------------------------------------
# Experts (MMOE page, "MoE++ expert layer"; reading R1 for GELU).
# --------------------------------------------------------------------------
def gelu_erf(u):
    """GELU(u) = u * Phi(u) = 0.5 * u * (1 + erf(u / sqrt(2))).

    Phi is evaluated as 0.5 * erfc(-u / sqrt(2)), the same function written
    without the cancellation of 1 + erf in the negative tail.
    """
    u = _f64(u)
    return 0.5 * u * _erfc(-u / math.sqrt(2.0))


def silu(u):
    """SiLU(u) = u / (1 + exp(-u))."""
    u = _f64(u)
    return u / (1.0 + np.exp(-u))


def mlp_gelu(X, W1, W2):
    """Heavy expert, standard MLP: W2 . GELU(W1 . x) per row of X.

    ``W1`` is [h, d], ``W2`` is [d, h]; no biases (reading R18).
    """
    H = gelu_erf(_f64(X) @ _f64(W1).T)
    return H @ _f64(W2).T


def mlp_swiglu(X, Wg, Wu, Wd):
    """Heavy expert, SwiGLU: Wd . (silu(Wg . x) * (Wu . x)) per row of X.

    ``Wg``, ``Wu`` are [h, d]; ``Wd`` is [d, h] (reading R20).
    """
    X = _f64(X)
    H = silu(X @ _f64(Wg).T) * (X @ _f64(Wu).T)
    return H @ _f64(Wd).T


def zero_compute_expert(kind, X, v=None, Wc=None):
    """MMOE zero-computation experts: identity -> x, zero -> 0, constant -> v.

    The constant expert returns its learned vector v [d] for every token
    (reading R14). Mixture variant (MMOE page, "Methodology": a constant
    expert mixes with a learned vector; reading R24): with learned mixing
    weights Wc [2, d], E(x) = a0(x) * x + a1(x) * v where
    (a0, a1) = softmax(Wc . x).
    """
    X = _f64(X)
    if kind == IDENTITY:
        return X.copy()
    if kind == ZERO:
        return np.zeros_like(X)
    if kind == CONST:
        v = _f64(v)
        if Wc is None:
            return np.broadcast_to(v[None, :], X.shape).copy()
        a = softmax_rows(X @ _f64(Wc).T)  # [rows, 2]
        return a[:, :1] * X + a[:, 1:2] * v[None, :]
    raise ValueError("not a zero-computation kind")


def heavy_expert(act, X, W1e, W2e, h):
    """One heavy expert on rows X. ``W1e`` is [h, d] (GELU) or [2h, d]
    holding gate rows then up rows (SwiGLU); ``W2e`` is [d, h]."""
    if act == "gelu":
        return mlp_gelu(X, W1e, W2e)
    if act == "swiglu":
        W1e = _f64(W1e)
        return mlp_swiglu(X, W1e[:h], W1e[h:2 * h], W2e)
    raise ValueError(act)


# --------------------------------------------------------------------------
# Combine (DICE page, "Conditional Communication": the output is the
# routing-score weighted sum of the expert outputs; MMOE page, "shared
# experts": always active; reading R17 for the residual).
# --------------------------------------------------------------------------
def combine(tokens, a_tok, a_exp, a_w, expert_out, residual=None,
            shared_out=None, d=None):
    """y_s = r_s + shared(x_s) + sum over the assignments a of s of w_a * E_{e_a}(x_s).

    ``expert_out(a)`` returns the [d] output of assignment a's expert on
    its token. Returns y for the requested ``tokens`` (in that order). A
    token with no residual, no shared output and no expert (expert choice
    can leave a token unpicked) sums nothing: its row is 0, which needs the
    model width ``d`` when no other row shows it.
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    a_tok = np.asarray(a_tok, dtype=np.int64)
    rows = []
    for i, s in enumerate(tokens):
        acc = None
        if residual is not None:
            acc = _f64(residual[s]).copy()
        if shared_out is not None:
            acc = shared_out[i].copy() if acc is None else acc + shared_out[i]
        for a in np.nonzero(a_tok == s)[0]:
            if a_exp is not None and a_exp[a] < 0:
                continue  # an empty slot (DES-Seq) contributes nothing
            term = float(a_w[a]) * expert_out(a)
            acc = term if acc is None else acc + term
        rows.append(acc)
    if d is None:
        widths = [r.shape[0] for r in rows if r is not None]
        if not widths:
            raise ValueError("no token has a term: pass the model width d")
        d = widths[0]
    return np.stack([np.zeros(d) if r is None else r for r in rows])


# --------------------------------------------------------------------------
# Whole layer.
# --------------------------------------------------------------------------
def assignments_from_selection(cfg, sel):
    """Flatten a selection into the slot-ordered assignment list.

    Token choice / DES: a = s*k + j. Expert choice: a = (g*E + e)*C + c.
    """
    if cfg["routing"] in ("token_topk", "des_vote", "des_seq"):
        idx = np.asarray(sel["idx"])
        T, k = idx.shape
        a_tok = np.repeat(np.arange(T), k)
        a_exp = idx.reshape(-1).astype(np.int64)
        a_w = _f64(sel["w"]).reshape(-1)
    elif cfg["routing"] == "expert_choice":
        tok = np.asarray(sel["tok"])
        G, E, C = tok.shape
        a_tok = tok.reshape(-1).astype(np.int64)
        a_exp = np.tile(np.repeat(np.arange(E), C), G)
        a_w = _f64(sel["w"]).reshape(-1)
    else:
        raise ValueError(cfg["routing"])
    return a_tok, a_exp, a_w


def route(cfg, x, W_r, logit_bias=None, z_prev=None):
    """Router + selection in fp64 (the oracle's own routing)."""
    z = router_logits(x, W_r, logit_bias, z_prev, cfg.get("gate_residual_scale", 0.0))
    A = softmax_rows(z)
    r = cfg["routing"]
    if r == "token_topk":
        idx = topk_token_choice(z, cfg["k"])
        w = gather_weights(A, idx)
        if cfg.get("renorm", 0):
            w = renormalize(w)
        return {"z": z, "A": A, "idx": idx, "w": w}
    if r == "expert_choice":
        tok, w = expert_choice(A, cfg["group_size"], cfg["capacity"])
        return {"z": z, "A": A, "tok": tok, "w": w}
    if r == "des_vote":
        votes, core, idx, w = des_vote(A, cfg["k"], cfg["M_core"])
        return {"z": z, "A": A, "votes": votes, "core": core, "idx": idx, "w": w}
    if r == "des_seq":
        core, idx, w = des_seq(A, cfg["k"], cfg["k_local"])
        return {"z": z, "A": A, "core": core, "idx": idx, "w": w}
    raise ValueError(r)


def forward(cfg, x, W1, W2, sel, kinds=None, const_vecs=None, Ws1=None,
            Ws2=None, residual=None, tokens=None):
    """Layer output y for ``tokens`` (default: all) given a selection.

    ``W1`` [E_h, h, d] (GELU) or [E_h, 2h, d] (SwiGLU, gate then up rows),
    ``W2`` [E_h, d, h]. ``kinds`` [E] gives each expert's kind (heavy ids
    come first); ``const_vecs`` [n_const, d] holds the constant experts'
    vectors in id order, or [n_const, 3, d] (v, then the two rows of the
    mixing weights Wc) when ``cfg["const_mix"]`` is set. Shared experts
    arrive concatenated along the hidden dimension: ``Ws1`` [n_sh*h_sh, d],
    ``Ws2`` [d, n_sh*h_sh]; for GELU
    this is the sum of the individual shared experts exactly (the hidden
    units of different experts never mix).

    Each expert is evaluated only on the requested tokens that it serves;
    the result for a token depends only on its own selection, so a subset
    of tokens gives exactly the rows of the full output.
    """
    x = np.asarray(x)
    T = x.shape[0]
    tokens = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    E = cfg["E"]
    kinds = np.zeros(E, dtype=np.int64) if kinds is None else np.asarray(kinds)
    h = cfg["h"]
    a_tok, a_exp, a_w = assignments_from_selection(cfg, sel)
    wanted = np.zeros(T, dtype=bool)
    wanted[tokens] = True
    const_slot = {}
    for e in range(E):
        if kinds[e] == CONST:
            const_slot[e] = len(const_slot)
    out = {}
    live = np.nonzero(wanted[a_tok] & (a_exp >= 0))[0]  # -1: empty slot
    for e in np.unique(a_exp[live]):
        rows_a = live[a_exp[live] == e]
        X = _f64(x[a_tok[rows_a]])
        if kinds[e] == HEAVY:
            Y = heavy_expert(cfg["act"], X, W1[e], W2[e], h)
        elif kinds[e] == CONST:
            cv = const_vecs[const_slot[e]]
            if cfg.get("const_mix"):
                Y = zero_compute_expert(CONST, X, cv[0], cv[1:3])
            else:
                Y = zero_compute_expert(CONST, X, cv)
        else:
            Y = zero_compute_expert(int(kinds[e]), X)
        for i, a in enumerate(rows_a):
            out[int(a)] = Y[i]
    shared = None
    if Ws1 is not None:
        shared = mlp_gelu(_f64(x[tokens]), Ws1, Ws2)
    return combine(tokens, a_tok, a_exp, a_w, lambda a: out[int(a)],
                   residual=residual, shared_out=shared, d=x.shape[1])


def dense_masked_forward(cfg, x, W1, W2, A, mask, kinds=None,
                         const_vecs=None, Ws1=None, Ws2=None, residual=None):
    """Independent formulation of the layer for small inputs:
    y = r + shared(x) + sum_e mask[:, e] * A[:, e] * E_e(x), with EVERY
    expert evaluated on EVERY token. Used as a pin of ``forward``.
    """
    x64 = _f64(x)
    T = x64.shape[0]
    E = cfg["E"]
    kinds = np.zeros(E, dtype=np.int64) if kinds is None else np.asarray(kinds)
    y = np.zeros_like(x64) if residual is None else _f64(residual).copy()
    if Ws1 is not None:
        y = y + mlp_gelu(x64, Ws1, Ws2)
    ci = 0
    for e in range(E):
        if kinds[e] == HEAVY:
            Ye = heavy_expert(cfg["act"], x64, W1[e], W2[e], cfg["h"])
        elif kinds[e] == CONST:
            cv = const_vecs[ci]
            Ye = (zero_compute_expert(CONST, x64, cv[0], cv[1:3]) if cfg.get("const_mix")
                  else zero_compute_expert(CONST, x64, cv))
            ci += 1
        else:
            Ye = zero_compute_expert(int(kinds[e]), x64)
        y = y + (_f64(mask[:, e]) * _f64(A[:, e]))[:, None] * Ye
    return y
