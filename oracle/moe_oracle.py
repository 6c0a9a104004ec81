"""CPU oracle for the skew-aware MoE forward layer.

TEST INFRASTRUCTURE ONLY. This is the plain, slow, obviously correct statement of what the
layer computes, used to check the CUDA library. It shares no code with the library and
imports nothing from it. Only the tests, the package smoke check and the benchmark's CPU
baseline leg may import or run it; the product path never does.

Sources (cited by page title and section; the pages print no code and no worked example):
  [MF]  "MegaFlux" summary (picx.dev/p/e4jAzZ):
          - "Routing Skew Problem": the skew measure kappa and its uniform case kappa = 1;
          - Methodology 1, "Problem Formulation": token blocks of at most beta rows,
            b_e = ceil(c_e / beta), the planner objective min_q max_r l_r with
            l_r = sum_e q_er, the constraints sum_r q_er = b_e and
            sum_{e: h(e) != r} 1[q_er > 0] <= s;
          - Methodology 1, "Bounded Greedy Search": four greedy searches from the
            no-replica assignment toward tau = ceil(sum_e b_e / P), donor priority
            (total overload | largest remaining home-expert load) x fan-out (one new copy
            per expert per round | several); the reduction-aware proxy
            C_lambda(q) = max_r (l_r + lambda n_r), n_r = remote replicas of experts owned
            by r, lambda = 12;
          - Methodology 2, expert-computation equation: Z_e = X_e W1_e, Z_e = [G_e, U_e],
            A_e = SiLU(G_e) * U_e, O_e = A_e W2_e, y_t = sum_{e in S_t} p_{t,e} O_e[t];
          - Methodology 2, "Backward gradients": dA_e = D_e W2_e^T, dX_e = dZ_e W1_e^T,
            dW2_e = A_e^T D_e, dW1_e = X_e^T dZ_e; Backward item 3: token-axis D_e and
            dZ_e are requantized;
          - Summary and "Theoretical Contributions" 1: router outputs, token counts,
            expert selections and routing weights are preserved.
  [UE]  "UltraEP: Exact Load Balancing for Rack-Scale MoE" reading notes, section 4
        ("The Quota-Driven Planning Solver", Algorithm 1 "joint solving"): binary search
        for the smallest load threshold tau a greedy feasibility oracle satisfies; excess
        exc_r = max(l_r - tau, 0) and slack slk_r = max(tau - l_r, 0); overloaded ranks by
        descending excess, their hot experts by descending load; receiver t* = the rank
        with the most slack that does not host the expert; delta = min(exc_r, slk_t*,
        remaining load of e), transferred only if delta >= the quota floor u_min.  The
        receiver rule also serves the bounded greedy search (R4).
  [TE]  TopoEP abstract: plans are deterministic and bitwise identical.

Readings where the pages leave a step open (each is also listed in the design notes):
  R1  top-k order is by descending logit, ties to the lower expert id; gates are the
      softmax over the k chosen logits (= full softmax renormalised over the top-k),
      evaluated in fp64 and rounded to fp32.
  R2  kappa = E * S / N^2 with S = sum_e c_e^2 and N = sum_e c_e, exact integers, one
      fp64 rounding; kappa = 0.0 when N = 0 (no routed rows).
  R3  owner map h(e) = floor(e * P / E) (contiguous equal ranges of experts per slot).
  R4  the bounded greedy rule of `plan_variant` (donor order, expert order, receiver
      choice, move size, rounds, stop rule) and the best-variant choice of `plan`.
  R5  dispatch is a stable counting sort of the (t, j) pairs by expert, token-ascending
      inside an expert; expert e's i-th row goes to padded row beta*block_off[e] + i.
  R6  the FFN is evaluated in fp32 from the exact bf16 input values; A is kept in fp32.
  R7  the combine sums j = 0..k-1 in ascending order in fp32.
  R13 the quota solver of `plan_quota` (variant 4) in this block formulation: ranks are
      the P slots, the load of expert e is b_e blocks, N_slot = s; the search runs over
      integer tau in [ceil(B / P), max_r home load] exactly as printed (while lo < hi,
      tau = floor((lo + hi) / 2); the target coefficient beta does not enter the printed
      loop and is not used); the oracle makes one transfer per hot expert (as printed),
      receivers are ranks other than the donor with slack > 0 and a free replica slot
      (rep_t < s), ties of slack to the lower rank; u_min is counted in blocks (default 1);
      the plan is the oracle's quota table at the tau the search ends on.
  R14 the reduction-aware variant (C_lambda) keeps each greedy search's moves and returns
      the plan, among the search's start and the plan after each move, of least C_lambda
      (the earliest on ties; n_r grows by one whenever a move opens a copy of one of r's
      experts); the quota solver's plan is scored as it ends; the best variant is then
      the least (C_lambda, makespan, replicas, variant index).
  R15 backward: D = dL/dO on row r is row_gate[r] * dy[row_token[r]] (zero on padding
      rows); the weights are stored w1 [2f, d], w2 [d, f], so each page formula is taken
      with that transpose (dA = D w2, dX = dZ w1, dW2 = D^T A, dW1 = dZ^T X);
      dZ = [dA * U * SiLU'(G), dA * SiLU(G)]; D and dZ are requantized to bf16
      (round to nearest even) before they enter a product, everything else is fp32;
      with `saved_bf16` the activations the forward keeps for the backward (A, computed
      from fp32 G and U, and Z = [G, U]) enter it rounded to bf16, as they are stored;
      dx_t = sum_j dX[tok_row[t, j]], j ascending.  The gate gradient (router backward)
      is not part of the expert computation and is left out.
"""
from __future__ import annotations

import numpy as np

VARIANT_NAMES = ("over/one", "over/multi", "hot/one", "hot/multi", "quota")
QUOTA_VARIANT = 4
GREEDY_VARIANTS = 0xF
ALL_VARIANTS = 0x1F


# --------------------------------------------------------------------------- routing
def route_topk(logits: np.ndarray, k: int) -> tuple[np.ndarray, np.ndarray]:
    """S_t and p_{t,e} per token: the k largest logits and their renormalised softmax.

    [MF] Summary (router outputs are fixed inputs); reading R1.
    Returns ids int32 [T, k] (descending logit, ties to the lower id) and gates fp32 [T, k].
    """
    logits = np.asarray(logits, dtype=np.float32)
    if not np.all(np.isfinite(logits)):
        raise ValueError("router logits must be finite")
    T, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    # a stable ascending sort of -logit keeps equal logits in expert-id order
    ids = np.argsort(-logits, axis=1, kind="stable")[:, :k].astype(np.int32)
    sel = np.take_along_axis(logits, ids, axis=1).astype(np.float64)
    w = np.exp(sel - sel[:, :1])          # sel[:, 0] is the row's largest chosen logit
    gates = (w / w.sum(axis=1, keepdims=True)).astype(np.float32)
    return ids, gates


def expert_counts(ids: np.ndarray, E: int) -> np.ndarray:
    """c_e: number of routed (t, j) pairs with ids[t, j] = e.  [MF] Routing Skew Problem."""
    ids = np.asarray(ids).ravel()
    if ids.size and (ids.min() < 0 or ids.max() >= E):
        raise ValueError("expert id out of range")
    return np.bincount(ids, minlength=E).astype(np.int64)


def skew_kappa(counts) -> tuple[int, float]:
    """(S, kappa): S = sum_e c_e^2 and kappa = E * sum_e (c_e / sum_j c_j)^2.

    [MF] "Routing Skew Problem" equation; reading R2. Written as E*S/N^2 over exact
    integers, so the single rounding is Python's correctly rounded int/int division.
    """
    c = [int(v) for v in counts]
    E = len(c)
    S = sum(v * v for v in c)
    N = sum(c)
    if N == 0:
        return 0, 0.0
    return S, (E * S) / (N * N)


# --------------------------------------------------------------------------- blocks
def block_counts(counts, beta: int) -> list[int]:
    """b_e = ceil(c_e / beta) (0 for an idle expert).  [MF] Problem Formulation."""
    return [-(-int(c) // beta) for c in counts]


def block_offsets(b) -> list[int]:
    """Exclusive prefix sum of b_e, E+1 entries; block_off[E] = B = sum_e b_e."""
    off = [0]
    for v in b:
        off.append(off[-1] + int(v))
    return off


def owner(e: int, E: int, P: int) -> int:
    """h(e), the home slot of expert e.  Reading R3: contiguous equal ranges."""
    return e * P // E


# --------------------------------------------------------------------------- planner
def reduction_cost(q, P: int, lam: int) -> int:
    """[MF] C_lambda(q) = max_r (l_r + lambda n_r), n_r = the remote replicas of experts
    owned by r: #{(e, t) : h(e) = r, t != r, q_et > 0}."""
    q = np.asarray(q)
    E = q.shape[0]
    n = [0] * P
    for e in range(E):
        h = owner(e, E, P)
        n[h] += sum(1 for t in range(P) if t != h and q[e, t] > 0)
    loads = q.sum(axis=0)
    return max(int(loads[r]) + lam * n[r] for r in range(P)) if P else 0


def plan_variant(b, P: int, s: int, v: int, lam: int | None = None) -> dict:
    """One bounded greedy search of [MF] "Bounded Greedy Search"; reading R4 (and with
    `lam`, the reduction-aware variant of reading R14).

    Variant v = 2*D + F with donor priority D (0: decreasing total overload l_r,
    1: largest remaining home-expert load max_{h(e)=r} q_er) and fan-out F (0: at most
    one new copy of an expert per round, 1: several copies per round).

    Start: the no-replica assignment q[e][h(e)] = b_e.  Target: tau = ceil(B / P).
    A round visits the donors (slots with l_r > tau) in priority order (ties to the
    lower slot); a donor offers its home experts in order of q[e][r] descending (ties to
    the lower id); a home expert keeps moving blocks while its donor is above tau:
      receivers = slots t != r with l_t < tau that either already hold a copy of e
                  (q[e][t] > 0) or may open one (rep_t < s, and under fan-out "one" e has
                  not been copied yet in this round);
      receiver  = the one with the most slack, i.e. least l_t, ties to the lower slot
                  ([UE] Algorithm 1's receiver rule);
      move      = min(l_r - tau, tau - l_t, q[e][r]) blocks, the largest that keeps both
                  ends on their side of tau.
    The search stops when max_r l_r <= tau or a round moves nothing (bounded: every move
    lowers the total overload by at least one block).
    """
    E = len(b)
    b = [int(x) for x in b]
    D, F = v >> 1, v & 1
    h = [owner(e, E, P) for e in range(E)]
    q = [[0] * P for _ in range(E)]
    for e in range(E):
        q[e][h[e]] = b[e]
    load = [0] * P
    for e in range(E):
        load[h[e]] += b[e]
    rep = [0] * P
    B = sum(b)
    tau = -(-B // P)
    rounds = 0
    # reading R14: the least C_lambda along the search (start, then after every move)
    best = None
    if lam is not None:
        best = {"cost": reduction_cost(q, P, lam), "q": [row[:] for row in q],
                "load": load[:], "rep": rep[:], "rounds": 0}
    while max(load) > tau:
        rounds += 1
        newcopies = [0] * E
        progress = False
        donors = [r for r in range(P) if load[r] > tau]
        if D == 0:
            donors.sort(key=lambda r: (-load[r], r))
        else:
            donors.sort(key=lambda r: (-max([q[e][r] for e in range(E) if h[e] == r],
                                              default=0), r))
        for r in donors:
            home = sorted((e for e in range(E) if h[e] == r), key=lambda e: (-q[e][r], e))
            for e in home:
                while load[r] > tau and q[e][r] > 0:
                    cand = [t for t in range(P)
                            if t != r and load[t] < tau
                            and (q[e][t] > 0
                                 or (rep[t] < s and (F == 1 or newcopies[e] == 0)))]
                    if not cand:
                        break
                    t = min(cand, key=lambda t: (load[t], t))
                    delta = min(load[r] - tau, tau - load[t], q[e][r])
                    if q[e][t] == 0:
                        rep[t] += 1
                        newcopies[e] += 1
                    q[e][r] -= delta
                    q[e][t] += delta
                    load[r] -= delta
                    load[t] += delta
                    progress = True
                    if best is not None:
                        c = reduction_cost(q, P, lam)
                        if c < best["cost"]:
                            best = {"cost": c, "q": [row[:] for row in q], "load": load[:],
                                    "rep": rep[:], "rounds": rounds}
        if not progress:
            break
    out = {"q": np.array(q, dtype=np.int32).reshape(E, P), "load": load,
           "makespan": max(load) if P else 0, "replicas": sum(rep), "tau": tau,
           "B": B, "variant": v, "rounds": rounds}
    if best is not None:
        out.update(q=np.array(best["q"], dtype=np.int32).reshape(E, P), load=best["load"],
                   makespan=max(best["load"]) if P else 0, replicas=sum(best["rep"]),
                   rounds=best["rounds"], cost=best["cost"])
    return out


def quota_feasible(b, P: int, s: int, u_min: int, tau: int) -> dict:
    """[UE] Algorithm 1's greedy feasibility oracle at one threshold tau; reading R13.

    Start from the home placement q[e][h(e)] = b_e.  exc_r = max(l_r - tau, 0) and
    slk_r = max(tau - l_r, 0).  Overloaded ranks in order of descending excess (ties to the
    lower rank); for each, its hot experts (h(e) = r, b_e > 0) in order of descending load
    (ties to the lower id): t* = the rank != r with the most slack among those with slack
    left and a free replica slot (ties to the lower rank); delta = min(exc_r, slk_t*,
    q[e][r]); if delta >= u_min the quota moves to t*, which then hosts a replica of e.
    Feasible when no rank keeps an excess."""
    E = len(b)
    h = [owner(e, E, P) for e in range(E)]
    q = [[0] * P for _ in range(E)]
    load = [0] * P
    for e in range(E):
        q[e][h[e]] = int(b[e])
        load[h[e]] += int(b[e])
    exc = [max(load[r] - tau, 0) for r in range(P)]
    slk = [max(tau - load[r], 0) for r in range(P)]
    rep = [0] * P
    for r in sorted((r for r in range(P) if exc[r] > 0), key=lambda r: (-exc[r], r)):
        hot = sorted((e for e in range(E) if h[e] == r and b[e] > 0), key=lambda e: (-b[e], e))
        for e in hot:
            cand = [t for t in range(P) if t != r and q[e][t] == 0 and slk[t] > 0 and rep[t] < s]
            if not cand:
                continue
            t = min(cand, key=lambda t: (-slk[t], t))
            delta = min(exc[r], slk[t], q[e][r])
            if delta >= u_min:
                q[e][r] -= delta
                q[e][t] += delta
                exc[r] -= delta
                slk[t] -= delta
                load[r] -= delta
                load[t] += delta
                rep[t] += 1
    return {"feasible": all(x == 0 for x in exc), "q": q, "load": load, "rep": rep}


def plan_quota(b, P: int, s: int, u_min: int = 1) -> dict:
    """[UE] Algorithm 1 (joint solving): binary search for the smallest tau that
    `quota_feasible` satisfies, on [ceil(B / P), max_r home load]; the plan is the quota
    table at that tau.  Reading R13.  'rounds' counts the search iterations."""
    E = len(b)
    b = [int(x) for x in b]
    u_min = max(int(u_min), 1)
    B = sum(b)
    lo = -(-B // P)
    home = [0] * P
    for e in range(E):
        home[owner(e, E, P)] += b[e]
    hi = max(home) if P else 0
    rounds = 0
    while lo < hi:
        rounds += 1
        tau = (lo + hi) // 2
        if quota_feasible(b, P, s, u_min, tau)["feasible"]:
            hi = tau
        else:
            lo = tau + 1
    res = quota_feasible(b, P, s, u_min, hi)
    load = res["load"]
    return {"q": np.array(res["q"], dtype=np.int32).reshape(E, P), "load": load,
            "makespan": max(load) if P else 0, "replicas": sum(res["rep"]),
            "tau": -(-B // P), "tau_star": hi, "B": B, "variant": QUOTA_VARIANT,
            "rounds": rounds}


def fixed_makespan(b, P: int) -> int:
    """Largest slot load of the no-replica (fixed placement) assignment."""
    E = len(b)
    load = [0] * P
    for e in range(E):
        load[owner(e, E, P)] += int(b[e])
    return max(load)


def plan(b, P: int, s: int, variant_mask: int = GREEDY_VARIANTS, u_min: int = 1,
         lam: int | None = None) -> dict:
    """Run the enabled variants (bits 0..3: the greedy searches, bit 4: the quota solver;
    0 means the four greedy searches, the method's planner) and keep the best.  Reading
    R4: the best is the lexicographic minimum of (makespan, total replicas, variant
    index); with `lam` (reading R14), of (C_lambda, makespan, replicas, variant index)."""
    mask = variant_mask & ALL_VARIANTS or GREEDY_VARIANTS
    results = [plan_variant(b, P, s, v, lam) for v in range(4) if mask >> v & 1]
    if mask >> QUOTA_VARIANT & 1:
        results.append(plan_quota(b, P, s, u_min))
        if lam is not None:
            results[-1]["cost"] = reduction_cost(results[-1]["q"], P, lam)
    if lam is None:
        best = min(results, key=lambda r: (r["makespan"], r["replicas"], r["variant"]))
    else:
        best = min(results, key=lambda r: (r["cost"], r["makespan"], r["replicas"],
                                           r["variant"]))
    out = dict(best)
    out["all"] = {r["variant"]: r for r in results}
    out["fixed_makespan"] = fixed_makespan(b, P)
    return out


def block_list(q: np.ndarray) -> tuple[list[tuple[int, int]], list[int]]:
    """Expand q into the per-slot block list and its slot offsets.

    Slot r lists its experts in ascending order; expert e's slot-r share is the run of
    block indices j in [sum_{r' < r} q[e][r'], + q[e][r]).
    Returns (blocks [(e, j)], slot_off [P+1]).
    """
    q = np.asarray(q)
    E, P = q.shape
    blocks: list[tuple[int, int]] = []
    slot_off = [0]
    for r in range(P):
        for e in range(E):
            j0 = int(q[e, :r].sum())
            for j in range(j0, j0 + int(q[e, r])):
                blocks.append((e, j))
        slot_off.append(len(blocks))
    return blocks, slot_off


# --------------------------------------------------------------------------- dispatch
def dispatch(ids: np.ndarray, gates: np.ndarray, block_off, beta: int):
    """Tile-aligned dispatch; reading R5.

    Visits the (t, j) pairs in t-major order; the next free row of expert e (starting at
    beta * block_off[e]) receives the pair.  Returns row_token int32 [R] (-1 on padding
    rows), row_gate fp32 [R] (0 on padding rows) and tok_row int32 [T, k], with
    R = beta * block_off[E].
    """
    ids = np.asarray(ids)
    T, k = ids.shape
    E = len(block_off) - 1
    R = beta * int(block_off[E])
    row_token = np.full(R, -1, dtype=np.int32)
    row_gate = np.zeros(R, dtype=np.float32)
    tok_row = np.empty((T, k), dtype=np.int32)
    nxt = [beta * int(block_off[e]) for e in range(E)]
    for t in range(T):
        for j in range(k):
            e = int(ids[t, j])
            r = nxt[e]
            nxt[e] += 1
            if r >= beta * int(block_off[e + 1]):
                raise ValueError("expert overflows its blocks")
            row_token[r] = t
            row_gate[r] = gates[t, j]
            tok_row[t, j] = r
    return row_token, row_gate, tok_row


def gather_rows(x: np.ndarray, row_token: np.ndarray) -> np.ndarray:
    """Xp: x[row_token[r]] on valid rows, zeros on padding rows."""
    xp = np.zeros((len(row_token), x.shape[1]), dtype=x.dtype)
    valid = row_token >= 0
    xp[valid] = x[row_token[valid]]
    return xp


# --------------------------------------------------------------------------- FFN
def silu(g: np.ndarray) -> np.ndarray:
    """SiLU(g) = g / (1 + exp(-g))."""
    with np.errstate(over="ignore"):
        return g / (g.dtype.type(1.0) + np.exp(-g))


def silu_grad(g: np.ndarray) -> np.ndarray:
    """d SiLU(g) / dg = s + g s (1 - s) with s = 1 / (1 + exp(-g))."""
    one = g.dtype.type(1.0)
    with np.errstate(over="ignore"):
        sg = one / (one + np.exp(-g))
    return sg * (one + g * (one - sg))


def round_bf16(a: np.ndarray) -> np.ndarray:
    """fp32 -> nearest bf16 value (ties to even), returned as fp32 (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    u = (u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) & np.uint32(0xFFFF0000)
    return u.view(np.float32)


def expert_ffn(x_rows: np.ndarray, w1: np.ndarray, w2: np.ndarray,
               dtype=np.float32) -> np.ndarray:
    """O_e = (SiLU(G_e) * U_e) W2_e for rows of one expert; [MF] expert-computation
    equation; reading R6.  Shapes: x_rows [n, d], w1 [2f, d] (rows: G then U),
    w2 [d, f]; all fp32 (fp64 with dtype=np.float64).  Returns O [n, d]."""
    x_rows = np.asarray(x_rows, dtype=dtype)
    f = w1.shape[0] // 2
    Z = x_rows @ np.asarray(w1, dtype=dtype).T
    G, U = Z[:, :f], Z[:, f:]
    A = silu(G) * U
    return A @ np.asarray(w2, dtype=dtype).T


def expert_ffn_backward(x_rows, w1, w2, d_rows, dtype=np.float32, requant=True,
                        saved_bf16=False) -> dict:
    """[MF] "Backward gradients" for the rows of one expert, reading R15.  x_rows [n, d],
    w1 [2f, d], w2 [d, f], d_rows = dL/dO [n, d].  Recomputes Z, G, U, A, then
        dA = D w2,  dG = dA * U * SiLU'(G),  dU = dA * SiLU(G),  dZ = [dG, dU],
        dX = dZ w1,  dW2 = D^T A  [d, f],  dW1 = dZ^T X  [2f, d];
    with `requant`, D and dZ are rounded to bf16 before their products, and with
    `saved_bf16`, A and Z are taken as bf16-rounded copies (fp32 only)."""
    X = np.asarray(x_rows, dtype=dtype)
    W1 = np.asarray(w1, dtype=dtype)
    W2 = np.asarray(w2, dtype=dtype)
    D = np.asarray(d_rows, dtype=dtype)
    if requant:
        D = round_bf16(D)
    f = W1.shape[0] // 2
    Z = X @ W1.T
    G, U = Z[:, :f], Z[:, f:]
    A = silu(G) * U
    if saved_bf16:
        A = round_bf16(A)
        Z = round_bf16(Z)
        G, U = Z[:, :f], Z[:, f:]
    dA = D @ W2
    dZ = np.concatenate([dA * U * silu_grad(G), dA * silu(G)], axis=1)
    if requant:
        dZ = round_bf16(dZ)
    return {"Z": Z, "A": A, "D": D, "dA": dA, "dZ": dZ, "dX": dZ @ W1,
            "dW2": D.T @ A, "dW1": dZ.T @ X}


def combine(O_rows: np.ndarray, tok_row: np.ndarray, gates: np.ndarray) -> np.ndarray:
    """y_t = sum_j p_{t,j} O[tok_row[t, j]], j ascending in fp32; reading R7."""
    T, k = tok_row.shape
    y = np.zeros((T, O_rows.shape[1]), dtype=np.float32)
    for j in range(k):
        y += gates[:, j:j + 1].astype(np.float32) * O_rows[tok_row[:, j]]
    return y


def moe_forward(logits, x, get_expert, k: int, beta: int, P: int, s: int,
                variant_mask: int = GREEDY_VARIANTS) -> dict:
    """The whole forward layer: route, histogram + kappa, blocks, plan, dispatch,
    per-expert FFN, combine.  `x` is [T, d] fp32 holding bf16 values; `get_expert(e)`
    returns (w1 [2f, d], w2 [d, f]) as fp32 arrays holding bf16 values."""
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    ids, gates = route_topk(logits, k)
    counts = expert_counts(ids, E)
    S, kappa = skew_kappa(counts)
    b = block_counts(counts, beta)
    boff = block_offsets(b)
    pl = plan(b, P, s, variant_mask)
    row_token, row_gate, tok_row = dispatch(ids, gates, boff, beta)
    d = x.shape[1]
    O = np.zeros((len(row_token), d), dtype=np.float32)
    for e in range(E):
        if counts[e] == 0:
            continue
        r0 = beta * boff[e]
        rows = slice(r0, r0 + int(counts[e]))
        w1, w2 = get_expert(e)
        O[rows] = expert_ffn(x[row_token[rows]], w1, w2)
    y = combine(O, tok_row, gates)
    return {"ids": ids, "gates": gates, "counts": counts, "sumsq": S, "kappa": kappa,
            "b": b, "block_off": boff, "plan": pl, "row_token": row_token,
            "row_gate": row_gate, "tok_row": tok_row, "O": O, "y": y}


def moe_backward(logits, x, get_expert, dy, k: int, beta: int, dtype=np.float32,
                 requant=True, saved_bf16=False) -> dict:
    """Backward of the expert computation for upstream gradient dy = dL/dy [T, d]
    (reading R15): D rows = row_gate * dy[row_token] in the dispatched row order, each
    expert's rows through `expert_ffn_backward`, dx_t = sum_j dX[tok_row[t, j]].  Returns
    dx [T, d], per-expert dW1 [E, 2f, d] and dW2 [E, d, f] (zero for idle experts), and
    the row-wise D, Z, A, dZ, dX (zero on padding rows)."""
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    ids, gates = route_topk(logits, k)
    counts = expert_counts(ids, E)
    boff = block_offsets(block_counts(counts, beta))
    row_token, row_gate, tok_row = dispatch(ids, gates, boff, beta)
    x = np.asarray(x, dtype=dtype)
    dy = np.asarray(dy, dtype=dtype)
    d = x.shape[1]
    w1_0, _ = get_expert(0)
    f = w1_0.shape[0] // 2
    R = len(row_token)
    out = {name: np.zeros((R, n), dtype=dtype) for name, n in
           (("D", d), ("Z", 2 * f), ("A", f), ("dZ", 2 * f), ("dX", d))}
    dW1 = np.zeros((E, 2 * f, d), dtype=dtype)
    dW2 = np.zeros((E, d, f), dtype=dtype)
    for e in range(E):
        if counts[e] == 0:
            continue
        r0 = beta * boff[e]
        rows = slice(r0, r0 + int(counts[e]))
        w1, w2 = get_expert(e)
        Drows = row_gate[rows, None].astype(dtype) * dy[row_token[rows]]
        g = expert_ffn_backward(x[row_token[rows]], w1, w2, Drows, dtype, requant, saved_bf16)
        for name in ("D", "Z", "A", "dZ", "dX"):
            out[name][rows] = g[name]
        dW1[e] = g["dW1"]
        dW2[e] = g["dW2"]
    dx = np.zeros((T, d), dtype=dtype)
    for j in range(k):
        dx += out["dX"][tok_row[:, j]]
    out.update(dx=dx, dW1=dW1, dW2=dW2, row_token=row_token, row_gate=row_gate,
               tok_row=tok_row, block_off=boff, counts=counts)
    return out


def token_output(x_t: np.ndarray, experts, gates_t, get_expert) -> np.ndarray:
    """y_t for one token from its chosen experts and gates (rows of the FFN are
    independent, so any single token can be checked on its own at full size)."""
    y = np.zeros(x_t.shape[-1], dtype=np.float32)
    for e, g in zip(experts, gates_t):
        w1, w2 = get_expert(int(e))
        y += np.float32(g) * expert_ffn(x_t[None, :], w1, w2)[0]
    return y
