// Token blocks and the replica-budgeted block planner, on one CTA.
//
// "MegaFlux" summary, Methodology 1: "Problem Formulation" (b_e = ceil(c_e / beta); find
// q in Z^{E x P} minimising max_r sum_e q_er with sum_r q_er = b_e and at most s remote
// experts per slot) and "Bounded Greedy Search" (four searches from the no-replica
// assignment toward tau = ceil(B / P): donor priority x fan-out).  The receiver of a move
// is the slot with the most slack, as in the quota solver of the UltraEP notes
// (section 4, Algorithm 1); that solver is also a one-SM kernel with its load matrix in
// shared memory.  Plans are deterministic (TopoEP: bitwise-identical plans).
//
// The greedy rule (the same rule the CPU oracle states; no code is shared):
//   start  q[e][h(e)] = b_e, h(e) = floor(e P / E); loads l_r; replicas rep_r = 0.
//   round  while max_r l_r > tau: donors = {r : l_r > tau} ordered by (key desc, r asc)
//          with key = l_r (variant D = 0) or max_{h(e)=r} q[e][r] (D = 1), taken at the
//          start of the round; a donor's home experts in order (q[e][r] desc, e asc);
//          while the donor is above tau and the expert still has home blocks:
//            receivers t != r with l_t < tau and (q[e][t] > 0 or (rep_t < s and
//            (F = 1 or no copy of e was opened this round)));
//            t = the receiver of least (l_t, t); move min(l_r - tau, tau - l_t, q[e][r]).
//          A round that moves nothing ends the search.
//   best   least (makespan, total replicas, variant index) among enabled variants.
//
// Variant 4 is the quota solver of the UltraEP notes (section 4, Algorithm 1): a binary
// search over integer thresholds tau in [ceil(B / P), max_r home load] (tau = floor((lo +
// hi) / 2); feasible -> hi = tau, else lo = tau + 1) around a greedy feasibility oracle:
// from the home placement, overloaded slots by (excess desc, r asc), each one's loaded
// home experts by (b_e desc, e asc), one transfer per expert to the slot t != r of most
// slack among those with slack left and a free replica slot (rep_t < s; ties to the lower
// slot), of delta = min(excess, slack, b_e) blocks, made only if delta >= u_min; tau is
// feasible when no excess is left.  The plan is the oracle's quota table at the final tau.
//
// Reduction-aware selection (the summary's proxy for backward, C_lambda(q) = max_r (l_r +
// lambda n_r), n_r = remote copies of slot r's experts): each greedy search keeps its
// moves and returns the plan of least C_lambda among its start and the plan after each
// move (the earliest on ties; found by tracking C_lambda, then replaying the search up to
// that move); the quota solver's plan is scored as it ends; the best variant is the least
// (C_lambda, makespan, replicas, variant).
//
// One warp runs one variant: slot-parallel work (candidate test, arg-min, maxima) uses
// lanes 0..P-1 and warp shuffles; expert-parallel work strides the lanes over experts.
// Lane 0 applies each move; __syncwarp() orders it against the next read.
#include <climits>

#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kVariants = 5;       // 4 greedy variants + the quota solver, one warp each
constexpr int kPlanThreads = 32 * kVariants;
constexpr int kQuota = 4;          // variant index of the quota solver
constexpr int kTileRows = 256;     // rows of one execution tile of the FFN
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ int home_lo(int r, int E, int P) { return (r * E + P - 1) / P; }

__device__ __forceinline__ int warp_max(int v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = max(v, __shfl_xor_sync(kFull, v, off));
  return v;
}
__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
  return v;
}
// exclusive prefix sum over lanes
__device__ __forceinline__ int warp_excl_scan(int v, int lane) {
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(kFull, incl, off);
    if (lane >= off) incl += y;
  }
  return incl - v;
}

struct VariantState {
  int* q;      // [E * P] blocks of expert e on slot r
  int* load;   // [P] final slot loads (written at the end)
  int* order;  // [E] home experts of the current donor, in visiting order
  int* donors; // [P]
};

// min over lanes 0..7 of a key (lanes >= 8 hold INT_MAX), broadcast to the warp
__device__ __forceinline__ int min8(int v) {
  v = min(v, __shfl_xor_sync(kFull, v, 4));
  v = min(v, __shfl_xor_sync(kFull, v, 2));
  v = min(v, __shfl_xor_sync(kFull, v, 1));
  return __shfl_sync(kFull, v, 0);
}

// Runs greedy variant v on the calling warp; returns (makespan, replicas, rounds) in lane 0.
// Lane t < P holds slot t's load and replica count in registers; q lives in shared memory
// and, while one expert moves, each lane touches only its own slot's entry.
// lam >= 0 (the reduction-aware proxy C = max_r (l_r + lam n_r), n_r = remote copies of
// slot r's experts): also tracks C after every move and returns the least C seen, the move
// count and round where it was first reached (start: 0, 0).  max_moves >= 0: the search
// stops before move max_moves + 1, leaving the plan after max_moves moves in q.
__device__ void greedy_variant(int v, int E, int P, int s, int tau, const int* b,
                               VariantState st, int lam, int max_moves, int* out_makespan,
                               int* out_replicas, int* out_rounds, int* out_best_cost,
                               int* out_best_moves, int* out_best_rounds) {
  const int lane = threadIdx.x & 31;
  const int D = v >> 1, F = v & 1;
  int* q = st.q;

  for (int i = lane; i < E * P; i += 32) q[i] = 0;
  __syncwarp();
  for (int e = lane; e < E; e += 32) q[e * P + e * P / E] = b[e];
  int load = 0, rep = 0;  // lane t < P: slot t
  if (lane < P)
    for (int e = home_lo(lane, E, P); e < home_lo(lane + 1, E, P); ++e) load += b[e];
  __syncwarp();

  int rounds = 0, moves = 0, nown = 0;  // nown, lane r: remote copies of r's experts
  int best_cost = lam >= 0 ? warp_max(lane < P ? load : INT_MIN) : 0;
  int best_moves = 0, best_rounds = 0;
  bool halt = false;
  while (!halt) {
    const int maxload = warp_max(lane < P ? load : INT_MIN);
    if (maxload <= tau) break;
    ++rounds;

    // donor order, keys taken at the start of the round
    const bool is_donor = lane < P && load > tau;
    int key = 0;
    if (lane < P) {
      if (D == 0) {
        key = load;
      } else {
        for (int e = home_lo(lane, E, P); e < home_lo(lane + 1, E, P); ++e)
          key = max(key, q[e * P + lane]);
      }
    }
    const unsigned dmask = __ballot_sync(kFull, is_donor);
    const int ndon = __popc(dmask);
    int rank = 0;
    for (int r2 = 0; r2 < P; ++r2) {
      const int k2 = __shfl_sync(kFull, key, r2);
      if (is_donor && (dmask >> r2 & 1u) && (k2 > key || (k2 == key && r2 < lane))) ++rank;
    }
    if (is_donor) st.donors[rank] = lane;
    __syncwarp();

    bool progress = false;
    for (int di = 0; di < ndon && !halt; ++di) {
      const int r = st.donors[di];
      const int lo = home_lo(r, E, P), n = home_lo(r + 1, E, P) - lo;
      // home experts by (q[e][r] desc, e asc)
      for (int i = lane; i < n; i += 32) {
        const int e = lo + i, qe = q[e * P + r];
        int rk = 0;
        for (int i2 = 0; i2 < n; ++i2) {
          const int q2 = q[(lo + i2) * P + r];
          rk += (q2 > qe) || (q2 == qe && i2 < i);
        }
        st.order[rk] = e;
      }
      __syncwarp();
      int lr = __shfl_sync(kFull, load, r);  // donor load, warp-uniform
      for (int oi = 0; oi < n && lr > tau && !halt; ++oi) {
        const int e = st.order[oi];
        int qer = q[e * P + r];              // donor's blocks of e, warp-uniform
        int qt = lane < P ? q[e * P + lane] : 0;
        int newc = 0;                        // copies of e opened in this round
        while (lr > tau && qer > 0) {
          if (moves == max_moves) {
            halt = true;
            break;
          }
          int ck = INT_MAX;
          if (lane < P && lane != r && load < tau &&
              (qt > 0 || (rep < s && (F || newc == 0))))
            ck = (load << 4) | lane;
          ck = min8(ck);
          if (ck == INT_MAX) break;
          const int t = ck & 15, lt = ck >> 4;
          const int delta = min(min(lr - tau, tau - lt), qer);
          const bool opened = __shfl_sync(kFull, qt == 0, t);
          if (lane == t) {
            load += delta;
            rep += opened ? 1 : 0;
            qt += delta;
          }
          if (lane == r) {
            load -= delta;
            qt -= delta;
            nown += opened ? 1 : 0;  // r owns e: only home blocks move
          }
          newc += opened ? 1 : 0;
          lr -= delta;
          qer -= delta;
          progress = true;
          ++moves;
          if (lam >= 0) {
            const int c = warp_max(lane < P ? load + lam * nown : INT_MIN);
            if (c < best_cost) {
              best_cost = c;
              best_moves = moves;
              best_rounds = rounds;
            }
          }
        }
        if (lane < P) q[e * P + lane] = qt;
        __syncwarp();
      }
      __syncwarp();
    }
    if (!progress) break;
  }
  const int mk = warp_max(lane < P ? load : 0);
  const int reps = warp_sum(lane < P ? rep : 0);
  if (lane < P) st.load[lane] = load;
  if (lane == 0) {
    *out_makespan = mk;
    *out_replicas = reps;
    *out_rounds = rounds;
    *out_best_cost = best_cost;
    *out_best_moves = lam >= 0 ? best_moves : moves;
    *out_best_rounds = lam >= 0 ? best_rounds : rounds;
  }
  __syncwarp();
}

// Orders the lanes 0..P-1 flagged in `is_donor` by (key desc, lane asc) into donors[].
__device__ __forceinline__ int order_donors(bool is_donor, int key, int P, int* donors) {
  const int lane = threadIdx.x & 31;
  const unsigned dmask = __ballot_sync(kFull, is_donor);
  int rank = 0;
  for (int r2 = 0; r2 < P; ++r2) {
    const int k2 = __shfl_sync(kFull, key, r2);
    if (is_donor && (dmask >> r2 & 1u) && (k2 > key || (k2 == key && r2 < lane))) ++rank;
  }
  if (is_donor) donors[rank] = lane;
  __syncwarp();
  return __popc(dmask);
}

// Runs the quota solver on the calling warp; the plan lands in st.q.  Lane t < P holds
// slot t's home load, and during an oracle pass its load and replica count.
__device__ void quota_variant(int E, int P, int s, int u_min, int B, const int* b,
                              VariantState st, int lam, int* out_makespan, int* out_replicas,
                              int* out_rounds, int* out_tau, int* out_cost) {
  const int lane = threadIdx.x & 31;
  constexpr int kBig = 1 << 26;  // slack < B < 2^17; (kBig - slack) << 4 | slot fits an int
  // each slot's home experts by (b_e desc, e asc), at st.order[home_lo(r) ..)
  for (int r = 0; r < P; ++r) {
    const int lo = home_lo(r, E, P), n = home_lo(r + 1, E, P) - lo;
    for (int i = lane; i < n; i += 32) {
      const int be = b[lo + i];
      int rk = 0;
      for (int i2 = 0; i2 < n; ++i2) {
        const int b2 = b[lo + i2];
        rk += (b2 > be) || (b2 == be && i2 < i);
      }
      st.order[lo + rk] = lo + i;
    }
  }
  int home = 0;
  if (lane < P)
    for (int e = home_lo(lane, E, P); e < home_lo(lane + 1, E, P); ++e) home += b[e];
  __syncwarp();

  // One oracle pass at tau: returns feasibility; load / rep end in the lanes' registers;
  // with `write`, the transfers are applied to st.q (which then holds the home placement).
  int nown = 0;  // lane r: transfers of r's experts (remote copies), counted in each pass
  auto oracle = [&](int tau, bool write, int& load, int& rep) -> bool {
    load = lane < P ? home : 0;
    rep = 0;
    nown = 0;
    const int ndon = order_donors(lane < P && load > tau, load, P, st.donors);
    bool stuck = false;  // no slot can receive any more
    for (int di = 0; di < ndon && !stuck; ++di) {
      const int r = st.donors[di];
      int exc = __shfl_sync(kFull, load, r) - tau;  // warp-uniform
      for (int oi = home_lo(r, E, P); oi < home_lo(r + 1, E, P) && exc > 0; ++oi) {
        const int e = st.order[oi], be = b[e];
        if (be == 0) break;  // the rest of this slot's experts carry no load
        const int slk = lane < P ? max(tau - load, 0) : 0;
        int ck = INT_MAX;
        if (lane < P && lane != r && slk > 0 && rep < s) ck = ((kBig - slk) << 4) | lane;
        ck = min8(ck);
        if (ck == INT_MAX) {  // slack and free slots only shrink: nobody can receive later
          stuck = true;
          break;
        }
        const int t = ck & 15, slk_t = kBig - (ck >> 4);
        const int delta = min(min(exc, slk_t), be);
        if (delta >= u_min) {
          if (lane == t) {
            load += delta;
            rep += 1;
          }
          if (lane == r) {
            load -= delta;
            nown += 1;
          }
          exc -= delta;
          if (write && lane == 0) {
            st.q[e * P + r] -= delta;
            st.q[e * P + t] += delta;
          }
        }
        __syncwarp();
      }
    }
    return warp_max(lane < P ? load : INT_MIN) <= tau;
  };

  int lo = P > 0 ? (B + P - 1) / P : 0;
  int hi = warp_max(lane < P ? home : 0);
  int rounds = 0, load = 0, rep = 0;
  while (lo < hi) {
    ++rounds;
    const int tau = (lo + hi) / 2;
    if (oracle(tau, false, load, rep)) hi = tau;
    else lo = tau + 1;
  }
  for (int i = lane; i < E * P; i += 32) st.q[i] = 0;
  __syncwarp();
  for (int e = lane; e < E; e += 32) st.q[e * P + e * P / E] = b[e];
  __syncwarp();
  oracle(hi, true, load, rep);
  __syncwarp();
  const int mk = warp_max(lane < P ? load : 0);
  const int reps = warp_sum(lane < P ? rep : 0);
  const int cost = lam >= 0 ? warp_max(lane < P ? load + lam * nown : INT_MIN) : -1;
  if (lane < P) st.load[lane] = load;
  if (lane == 0) {
    *out_makespan = mk;
    *out_replicas = reps;
    *out_rounds = rounds;
    *out_tau = hi;
    *out_cost = cost;
  }
  __syncwarp();
}

// b_e = ceil(c_e / beta) and the exclusive scan block_off on one warp (lane l owns a
// contiguous chunk of experts), as the planner's first step computes them.
__global__ void __launch_bounds__(32, 1)
block_offsets_kernel(const int32_t* __restrict__ counts, int E, int beta,
                     int32_t* __restrict__ block_off) {
  const int lane = threadIdx.x;
  const int C = (E + 31) / 32;
  const int e0 = min(lane * C, E), e1 = min(e0 + C, E);
  int local = 0;
  for (int e = e0; e < e1; ++e) local += (max(counts[e], 0) + beta - 1) / beta;
  int run = warp_excl_scan(local, lane);
  for (int e = e0; e < e1; ++e) {
    block_off[e] = run;
    run += (max(counts[e], 0) + beta - 1) / beta;
  }
  if (lane == 31) block_off[E] = run;
}

__global__ void __launch_bounds__(kPlanThreads, 1)
plan_kernel(const int32_t* __restrict__ counts, int E, int P, int s, int beta,
            unsigned mask, int u_min, int lam, int b_max, int32_t* __restrict__ block_off, int32_t* __restrict__ q_out,
            int32_t* __restrict__ slot_load, int32_t* __restrict__ slot_off,
            int32_t* __restrict__ blocks, int32_t* __restrict__ tiles,
            int32_t* __restrict__ plan_info, int32_t* __restrict__ status) {
  extern __shared__ int sm[];
  int* b = sm;                          // E
  int* boff = b + E;                    // E + 1
  int* qv = boff + E + 1;               // 5 * E * P
  int* loadv = qv + kVariants * E * P;  // 5 * 8
  int* order = loadv + kVariants * kMaxP;  // 5 * E
  int* donors = order + kVariants * E;  // 5 * 8
  // res: makespan[5], replicas[5], rounds[5], quota tau*, C_lambda[5], 3 spare, then per
  // greedy warp (C_lambda, moves, round) at its least C_lambda
  int* res = donors + kVariants * kMaxP;  // 40
  int* misc = res + 40;                 // [0] B, [1] tau, [2] best, [3..3+P] slot tile offsets
                                        // [12..12+P] slot_off, [24..] fixed loads (P)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // ---- b_e and the exclusive scan block_off (warp 0; lane owns a chunk of experts)
  if (warp == 0) {
    const int C = (E + 31) / 32;
    const int e0 = min(lane * C, E), e1 = min(e0 + C, E);
    int local = 0;
    for (int e = e0; e < e1; ++e) {
      const int c = max(counts[e], 0);
      const int be = (c + beta - 1) / beta;
      b[e] = be;
      local += be;
    }
    int run = warp_excl_scan(local, lane);
    for (int e = e0; e < e1; ++e) {
      boff[e] = run;
      block_off[e] = run;
      run += b[e];
    }
    const int B = __shfl_sync(kFull, run, 31);
    if (lane == 31) {
      boff[E] = B;
      block_off[E] = B;
      misc[0] = B;
      misc[1] = (B + P - 1) / P;
    }
  }
  __syncthreads();
  const int B = misc[0], tau = misc[1];

  // ---- four greedy variants and the quota solver, one per warp
  {
    VariantState st;
    st.q = qv + warp * E * P;
    st.load = loadv + warp * kMaxP;
    st.order = order + warp * E;
    st.donors = donors + warp * kMaxP;
    int* cost = res + 16;
    if (!(mask >> warp & 1u)) {
      if (lane == 0) {
        res[warp] = INT_MAX;
        res[kVariants + warp] = INT_MAX;
        res[2 * kVariants + warp] = 0;
        cost[warp] = INT_MAX;
        if (warp == kQuota) res[3 * kVariants] = -1;
      }
    } else if (warp == kQuota) {
      quota_variant(E, P, s, u_min, B, b, st, lam, &res[warp], &res[kVariants + warp],
                    &res[2 * kVariants + warp], &res[3 * kVariants], &cost[warp]);
    } else {
      int* aux = res + 24 + 3 * warp;
      greedy_variant(warp, E, P, s, tau, b, st, lam, -1, &res[warp], &res[kVariants + warp],
                     &res[2 * kVariants + warp], &aux[0], &aux[1], &aux[2]);
      if (lam >= 0) {
        // replay the search up to its least C_lambda (the plan after aux[1] moves)
        const int bc = aux[0], bm = aux[1], br = aux[2];
        __syncwarp();
        greedy_variant(warp, E, P, s, tau, b, st, -1, bm, &res[warp], &res[kVariants + warp],
                       &aux[0], &aux[0], &aux[1], &aux[2]);
        if (lane == 0) {
          res[2 * kVariants + warp] = br;
          cost[warp] = bc;
        }
      } else if (lane == 0) {
        cost[warp] = -1;
      }
      __syncwarp();
    }
  }
  __syncthreads();

  // ---- best variant: least (makespan, replicas, v), or (C_lambda, makespan, replicas, v)
  if (tid == 0) {
    const int* cost = res + 16;
    int best = -1;
    for (int v = 0; v < kVariants; ++v) {
      if (!(mask >> v & 1u)) continue;
      if (best < 0) {
        best = v;
        continue;
      }
      if (lam >= 0 && cost[v] != cost[best]) {
        if (cost[v] < cost[best]) best = v;
        continue;
      }
      if (res[v] < res[best] ||
          (res[v] == res[best] && res[kVariants + v] < res[kVariants + best]))
        best = v;
    }
    misc[2] = best;
  }
  __syncthreads();
  const int best = misc[2];
  const int* qb = qv + best * E * P;
  const int* lb = loadv + best * kMaxP;

  for (int i = tid; i < E * P; i += blockDim.x) q_out[i] = qb[i];

  // ---- per-slot tile counts, slot offsets (thread 0; P <= 8)
  if (tid < P) {
    const int r = tid;
    int nt = 0;
    for (int e = 0; e < E; ++e) {
      const int qer = qb[e * P + r];
      nt += (qer * beta + kTileRows - 1) / kTileRows;
    }
    misc[3 + r] = nt;  // temporarily the count
    int fixed = 0;
    for (int e = home_lo(r, E, P); e < home_lo(r + 1, E, P); ++e) fixed += b[e];
    misc[24 + r] = fixed;
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0, tacc = 0, fixed_max = 0;
    for (int r = 0; r < P; ++r) {
      slot_load[r] = lb[r];
      slot_off[r] = acc;
      misc[12 + r] = acc;
      acc += lb[r];
      const int nt = misc[3 + r];
      misc[3 + r] = tacc;
      tacc += nt;
      fixed_max = max(fixed_max, misc[24 + r]);
    }
    slot_off[P] = acc;
    misc[12 + P] = acc;
    misc[3 + P] = tacc;
    if (B > b_max) set_status(status, MOE_STATUS_PLAN);
    plan_info[MOE_PI_B] = B;
    plan_info[MOE_PI_TAU] = tau;
    plan_info[MOE_PI_MAKESPAN] = res[best];
    plan_info[MOE_PI_VARIANT] = best;
    plan_info[MOE_PI_NTILES] = min(tacc, b_max);
    plan_info[MOE_PI_FIXED_MAKESPAN] = fixed_max;
    plan_info[MOE_PI_REPLICAS] = res[kVariants + best];
    plan_info[MOE_PI_ROUNDS] = res[2 * kVariants + best];
    for (int r = 0; r <= kMaxP; ++r)
      plan_info[MOE_PI_SLOT_TILE_OFF + r] = r <= P ? min(misc[3 + r], b_max) : min(tacc, b_max);
    for (int v = 0; v < kVariants; ++v) {
      const bool on = mask >> v & 1u;
      plan_info[MOE_PI_VAR_MAKESPAN + v] = on ? res[v] : -1;
      plan_info[MOE_PI_VAR_REPLICAS + v] = on ? res[kVariants + v] : -1;
      plan_info[MOE_PI_VAR_ROUNDS + v] = on ? res[2 * kVariants + v] : -1;
    }
    plan_info[MOE_PI_QUOTA_TAU] = res[3 * kVariants];
    plan_info[MOE_PI_COST] = lam >= 0 ? res[16 + best] : -1;
    for (int v = 0; v < kVariants; ++v)
      plan_info[MOE_PI_VAR_COST + v] = (lam >= 0 && (mask >> v & 1u)) ? res[16 + v] : -1;
    for (int i = MOE_PI_VAR_COST + kVariants; i < MOE_PI_LEN; ++i) plan_info[i] = 0;
  }
  __syncthreads();

  // ---- block list and tile list: warp w expands slots w, w + 5
  for (int r = warp; r < P; r += kVariants) {
    const int C = (E + 31) / 32;
    const int e0 = min(lane * C, E), e1 = min(e0 + C, E);
    int nb = 0, nt = 0;
    for (int e = e0; e < e1; ++e) {
      const int qer = qb[e * P + r];
      nb += qer;
      nt += (qer * beta + kTileRows - 1) / kTileRows;
    }
    int pb = misc[12 + r] + warp_excl_scan(nb, lane);
    int pt = misc[3 + r] + warp_excl_scan(nt, lane);
    for (int e = e0; e < e1; ++e) {
      const int qer = qb[e * P + r];
      int j0 = 0;
      for (int r2 = 0; r2 < r; ++r2) j0 += qb[e * P + r2];
      for (int i = 0; i < qer; ++i, ++pb) {
        if (pb < b_max) {
          blocks[2 * pb] = e;
          blocks[2 * pb + 1] = j0 + i;
        }
      }
      const int rows = qer * beta;
      for (int i = 0; i < rows; i += kTileRows, ++pt) {
        if (pt < b_max) {
          tiles[4 * pt + 0] = e;
          tiles[4 * pt + 1] = beta * (boff[e] + j0) + i;
          tiles[4 * pt + 2] = min(kTileRows, rows - i);
          tiles[4 * pt + 3] = r;
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_block_offsets(const moe_cfg& c, const int32_t* counts, int32_t* block_off,
                                 cudaStream_t st) {
  block_offsets_kernel<<<1, 32, 0, st>>>(counts, c.E, c.beta, block_off);
  return cudaGetLastError();
}

cudaError_t launch_plan(const moe_cfg& c, const int32_t* counts, uint32_t mask,
                        int32_t* block_off, int32_t* q, int32_t* slot_load,
                        int32_t* slot_off, int32_t* blocks, int32_t* tiles,
                        int32_t* plan_info, int32_t* status, cudaStream_t st) {
  const int E = c.E, P = c.P;
  const size_t words = (size_t)E + (E + 1) + kVariants * ((size_t)E * P + kMaxP + E + kMaxP) +
                       40 + 40;
  const size_t bytes = words * sizeof(int);
  // allow the largest configuration once per device (E = 256 experts, P = 8 slots)
  static OncePerDevice attr_once;
  cudaError_t err = once_per_device(attr_once, [](int&) {
    const size_t most = (size_t)kMaxE + (kMaxE + 1) +
                        kVariants * ((size_t)kMaxE * kMaxP + kMaxP + kMaxE + kMaxP) + 40 + 40;
    return cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(most * sizeof(int)));
  });
  if (err != cudaSuccess) return err;
  const unsigned all = (1u << kVariants) - 1u;
  const unsigned m = (mask & all) ? (mask & all) : 0xFu;  // default: the four greedy searches
  const int u_min = (mask >> 8 & 0xFFu) ? (int)(mask >> 8 & 0xFFu) : 1;
  const int lam = !(mask >> 5 & 1u) ? -1 : (mask >> 16 & 0xFFu) ? (int)(mask >> 16 & 0xFFu) : 12;
  plan_kernel<<<1, kPlanThreads, bytes, st>>>(counts, E, P, c.s, c.beta, m, u_min, lam,
                                              (int)max_blocks(c), block_off, q, slot_load,
                                              slot_off, blocks, tiles, plan_info, status);
  return cudaGetLastError();
}

}  // namespace moe
