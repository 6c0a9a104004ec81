/*
 * moeskew.h - C ABI of the skew-aware MoE forward layer on one NVIDIA B200 (sm_100a).
 *
 * The layer follows the "MegaFlux" summary (picx.dev): routing skew kappa ("Routing Skew
 * Problem"), tile-aligned token blocks and the replica-budgeted block planner
 * (Methodology 1, "Problem Formulation" and "Bounded Greedy Search"), and the SwiGLU
 * expert computation with the gate-weighted combine (Methodology 2, expert-computation
 * equation).  On one GPU the P "GPUs" of the planner are P virtual execution slots.
 *
 * Conventions shared by every entry point
 *   - Every array argument is a DEVICE pointer owned by the caller; the library never
 *     allocates, frees or keeps a pointer after the call returns.  Arrays must be 16-byte
 *     aligned.  bf16 data is passed as uint16_t bit patterns.
 *   - Every call is asynchronous on `stream` (a cudaStream_t / CUstream handle; NULL is
 *     the legacy default stream) and never synchronises the host.  Inputs are const and
 *     never modified.
 *   - The return value is MOE_OK or a negative host-detected error; on error nothing has
 *     been enqueued.  Problems only the device can see (an expert id out of range, more
 *     rows than the blocks hold, a non-finite logit, a bounded wait that ran out) are
 *     OR-ed into the caller's int32 `status` word in device memory as MOE_STATUS_* bits;
 *     the caller clears it before and reads it after its own synchronisation.  When a bit
 *     is set the outputs of that call are unspecified (but every write stayed inside the
 *     caller's buffers).
 *   - There is no mutable global state: calls on different streams with different
 *     buffers may run concurrently.
 *
 * Sizes: N = T*k routed rows; b_e = ceil(c_e/beta) blocks of expert e; B = sum_e b_e;
 * B_max = floor((N + min(E,N)*(beta-1)) / beta) bounds B for every routing; R_max =
 * beta*B_max bounds the padded rows.  moe_workspace_size() returns both, and the byte size
 * of the FFN's scratch buffer.
 */
#ifndef MOESKEW_H
#define MOESKEW_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* moe_stream_t;   /* == cudaStream_t */

/* Layer configuration, validated by every call.
 *   T tokens; d model width; E experts (1..256); k experts per token (1..min(E,8));
 *   f expert FFN width (FC1 has 2f outputs: f gate columns G then f up columns U);
 *   beta rows per token block (64 or 128); P virtual slots (1..8); s replica budget
 *   per slot (>= 0).  N = T*k must not exceed 2^22.
 *   The FFN needs d % 256 == 0 and f % 128 == 0; dispatch and combine need d % 8 == 0. */
typedef struct moe_cfg {
  int32_t T, d, E, k, f, beta, P, s;
} moe_cfg;

/* host-detected errors (return values) */
enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1, /* NULL pointer, k > E, k > 8, beta not 64/128, P > 8, ... */
  MOE_ERR_UNSUPPORTED = -2, /* shape outside what the kernels take, misaligned pointer */
  MOE_ERR_CUDA = -3,        /* a launch or a CUDA call failed */
  MOE_ERR_TOO_LARGE = -4    /* moe_expert_ffn_noalloc: A would not fit its fixed array */
};

/* device-detected problems (bits OR-ed into *status) */
enum {
  MOE_STATUS_BAD_ID = 1,     /* an expert id outside [0, E) */
  MOE_STATUS_OVERFLOW = 2,   /* an expert has more rows than its blocks hold */
  MOE_STATUS_NONFINITE = 4,  /* a router logit is NaN or infinite */
  MOE_STATUS_TIMEOUT = 8,    /* a bounded wait inside a kernel ran out */
  MOE_STATUS_PLAN = 16       /* the block plan does not fit B_max (inconsistent counts) */
};

/* moe_workspace_size(which) */
enum {
  MOE_WS_ROWS = 0,
  MOE_WS_BLOCKS = 1,
  MOE_WS_FFN_SCRATCH = 2,
  MOE_WS_FFN_SCRATCH_Z = 3,  /* a_scratch of moe_expert_ffn with MOE_FFN_SAVE_Z */
  MOE_WS_BWD_SCRATCH = 4,    /* bwd_scratch of moe_expert_ffn_backward */
  MOE_WS_FFN_RECORD = 5      /* byte offset in a_scratch of the slot record written with
                                MOE_FFN_RECORD_SLOTS (int32 [B_max]) */
};

/* plan_info layout (int32[MOE_PI_LEN]) written by moe_plan_blocks */
enum {
  MOE_PI_B = 0,              /* B = sum_e b_e */
  MOE_PI_TAU = 1,            /* tau = ceil(B / P) */
  MOE_PI_MAKESPAN = 2,       /* max_r l_r of the chosen plan */
  MOE_PI_VARIANT = 3,        /* chosen variant (0..3 greedy, 4 quota solver) */
  MOE_PI_NTILES = 4,         /* number of execution tiles (up to 256 rows each) */
  MOE_PI_FIXED_MAKESPAN = 5, /* max_r l_r of the no-replica (fixed placement) plan */
  MOE_PI_REPLICAS = 6,       /* total replicas of the chosen plan */
  MOE_PI_ROUNDS = 7,         /* greedy rounds (quota solver: search iterations) of the
                                chosen plan */
  MOE_PI_SLOT_TILE_OFF = 8,  /* P+1 entries: first tile of each slot */
  MOE_PI_VAR_MAKESPAN = 17,  /* 5 entries: makespan per variant, -1 when disabled */
  MOE_PI_VAR_REPLICAS = 22,  /* 5 entries */
  MOE_PI_VAR_ROUNDS = 27,    /* 5 entries */
  MOE_PI_QUOTA_TAU = 32,     /* threshold the quota solver's search ended on (-1: off) */
  MOE_PI_COST = 33,          /* C_lambda of the chosen plan (-1: not reduction-aware) */
  MOE_PI_VAR_COST = 34,      /* 5 entries: C_lambda per variant (-1: off) */
  MOE_PI_LEN = 40
};

/* moe_expert_ffn modes */
enum {
  MOE_FFN_FUSED_COMBINE = 0, /* out = y fp32 [T, d]; the call zeroes y, then FC2's
                                epilogue adds row_gate * O into y[row_token] */
  MOE_FFN_WRITE_O = 1,       /* out = O bf16 [R_max, d]; moe_combine reduces it */
  MOE_FFN_STRICT_SLOTS = 2,  /* flag: execution unit u (an SM pair, or an SM) only runs
                                slot (u mod P)'s tiles, so the layer time follows the
                                plan's makespan (one GPU standing in for P); without it
                                every unit takes tiles of any slot.  The call returns
                                MOE_ERR_UNSUPPORTED when the GPU has fewer than P units */
  MOE_FFN_SM_PAIR = 4,       /* flag: run each tile on a pair of SMs (a cluster of two
                                CTAs, tcgen05 cta_group::2, M = 256) instead of each
                                128-row half on one SM (cta_group::1, the default) */
  MOE_FFN_SAVE_Z = 16,       /* flag: FC1 also stores Z = [G, U] (bf16 [R_max, 2f]) after
                                A and the counters in a_scratch, which must then hold
                                moe_workspace_size(cfg, MOE_WS_FFN_SCRATCH_Z) bytes; the
                                backward pass reads A and Z from there */
  MOE_FFN_ONE_LAUNCH = 32,   /* flag: FC1 and FC2 in one persistent launch; FC2's work on
                                a tile half starts once FC1's epilogues have published all
                                of its A rows (per-half counters, bounded waits).  With the
                                fused combine, single-SM tiles and Xp only: combined with
                                WRITE_O, STRICT_SLOTS, SM_PAIR or GATHER_X the call returns
                                MOE_ERR_INVALID_ARG.  Without this flag or
                                MOE_FFN_TWO_LAUNCHES, a fused single-SM Xp call takes one
                                launch when FC1 has at most 2 work items (128 x 128 tiles,
                                padding aside) per SM, two launches otherwise */
  MOE_FFN_TWO_LAUNCHES = 64, /* flag: FC1 and FC2 as two launches (never one) */
  MOE_FFN_TEST_WAIT_TIMEOUT = 128, /* test hook for failure detection, not for production:
                                runs the one-launch FFN with FC2's readiness target one
                                above what FC1's epilogues reach and every wait limited to
                                10 ms, so FC2's producers give up: the call leaves
                                MOE_STATUS_TIMEOUT in status (out is then undefined) and
                                the context stays usable */
  MOE_FFN_FC1_M128 = 256,    /* flag: run FC1 on 128-row halves of the tiles (the tile-half
                                kernel, M = 128 per SM) instead of on whole tiles of up to
                                256 rows (two M = 128 MMAs sharing each weight stage, the
                                two-launch default).  The one-launch FFN, SM pairs, rows
                                gathered from x and MOE_FFN_SAVE_Z always use tile halves */
  MOE_FFN_FC2_WHOLE = 512,   /* flag: run the fused-combine FC2 on whole tiles (two M = 128
                                MMAs sharing each weight stage) instead of on tile halves.
                                Whole tiles need a third less L2 traffic per MMA, but both
                                256-column accumulators then fill TMEM and the fp32
                                reductions of an item no longer overlap the next item's
                                MMAs; on the layers measured halves are as fast or faster,
                                so this is off by default.  With MOE_FFN_WRITE_O the
                                two-launch FFN's FC2 always runs whole tiles (its O rows
                                leave through TMA stores); SM pairs and the one-launch FFN
                                always use tile halves */
  MOE_FFN_RECORD_SLOTS = 1024, /* diagnostic flag: the call also records which virtual
                                slots' execution units ran each execution tile: int32 word
                                m of the slot record (at byte offset
                                moe_workspace_size(cfg, MOE_WS_FFN_RECORD) of a_scratch,
                                zeroed by the call) gets bit (u mod P) when unit u (an SM,
                                or an SM pair) ran one of tile m's FC1 items and bit
                                8 + (u mod P) for FC2.  With MOE_FFN_STRICT_SLOTS tile m
                                then holds exactly its slot's two bits */
  MOE_FFN_GATHER_X = 8       /* flag: the `xp` argument is x itself (bf16 [T, d]); FC1
                                gathers each tile's rows x[row_token[r]] straight into
                                shared memory (TMA row gather), so the dispatched copy
                                Xp is never written (moe_dispatch_permute with
                                xp = NULL).  Padding rows of A (and of O) then hold
                                unspecified finite values instead of zeros. */
};

/* Upper bounds: which = MOE_WS_ROWS -> R_max rows (Xp, A, O, row_token, row_gate);
 * MOE_WS_BLOCKS -> B_max entries (blocks, tiles); MOE_WS_FFN_SCRATCH -> bytes of the
 * a_scratch buffer of moe_expert_ffn (A, bf16 [R_max, f], rounded up to 256 bytes, then
 * 256 bytes of tile-scheduler counters, then 2 * B_max int32 readiness counters rounded
 * up to 256 bytes, then the B_max int32 slot record rounded up to 256 bytes);
 * MOE_WS_FFN_RECORD -> the byte offset of that slot record; MOE_WS_FFN_SCRATCH_Z -> the
 * same scratch followed by
 * Z (bf16 [R_max, 2f], rounded up to 256 bytes); MOE_WS_BWD_SCRATCH -> bytes of the
 * bwd_scratch buffer of moe_expert_ffn_backward (dZ, bf16 [R_max, 2f], rounded up to 256
 * bytes, then 256 bytes of counters).  Returns 0 for an invalid cfg. */
MOE_API size_t moe_workspace_size(const moe_cfg* cfg, int which);

/* Router top-k, expert histogram and skew ("Routing Skew Problem"; router outputs of the
 * expert-computation equation).
 *   logits     fp32 [T, E] row-major, read only.
 *   topk_ids   int32 [T, k]: the k largest logits of each row, descending, ties to the
 *              lower expert id.
 *   topk_gates fp32 [T, k]: softmax over the k chosen logits (= the full softmax
 *              renormalised over the top-k).
 *   counts     int32 [E]: c_e = #{(t, j) : topk_ids[t, j] = e}.
 *   sumsq      int64 [1]: S = sum_e c_e^2.
 *   kappa      fp64 [1]: E * S / N^2 (one rounding, exact integers); 0 when N = 0.
 * A non-finite logit sets MOE_STATUS_NONFINITE. */
MOE_API int moe_route_hist(const moe_cfg* cfg, const float* logits, int32_t* topk_ids,
                   float* topk_gates, int32_t* counts, int64_t* sumsq, double* kappa,
                   int32_t* status, moe_stream_t stream);

/* Token blocks on their own ("Problem Formulation": b_e = ceil(c_e / beta)) and their
 * exclusive prefix sum block_off int32 [E+1], from counts int32 [E] (moe_route_hist).
 * moe_plan_blocks writes the same values; the dispatch needs nothing else from the plan,
 * so with this call it can run on another stream while the planner searches. */
MOE_API int moe_block_offsets(const moe_cfg* cfg, const int32_t* counts, int32_t* block_off,
                              moe_stream_t stream);

/* Token blocks and the block planner ("Problem Formulation", "Bounded Greedy Search").
 *   counts       int32 [E] (from moe_route_hist).
 *   variant_mask bits 0..3 enable greedy variants v = 2*D + F (D donor priority:
 *                0 total overload, 1 largest home-expert load; F fan-out: 0 one new copy
 *                per expert per round, 1 several); bit 4 enables variant 4, the quota
 *                solver ("UltraEP" notes, section 4, Algorithm 1: binary search on the
 *                threshold with a greedy feasibility oracle); bits 0..4 all clear means
 *                the four greedy variants (the method's planner; 0x1F runs all five).
 *                Bit 5: reduction-aware selection for backward with the proxy
 *                C_lambda(q) = max_r (l_r + lambda n_r), n_r = remote copies of slot r's
 *                experts ("Methodology" 1): each greedy search returns its plan of least
 *                C_lambda (its start or the plan after some move) and the variant of least
 *                (C_lambda, makespan, replicas, v) wins.  Bits 8..15: the quota solver's
 *                floor u_min in blocks (0 means 1).  Bits 16..23: lambda (0 means 12).
 *                Other bits are invalid.
 *   block_off    int32 [E+1]: exclusive prefix sum of b_e = ceil(c_e / beta).
 *   q            int32 [E, P] row-major: blocks of expert e run by slot r, of the best
 *                enabled variant (least makespan, then fewest replicas, then lowest v).
 *   slot_load    int32 [P]: l_r = sum_e q[e, r].
 *   slot_off     int32 [P+1]: exclusive prefix sum of slot_load.
 *   blocks       int32 [B_max, 2]: (e, j) pairs; slot r's run is
 *                [slot_off[r], slot_off[r+1]), experts ascending, expert e's share being
 *                block indices j in [sum_{r'<r} q[e, r'], + q[e, r]).
 *   tiles        int32 [B_max, 4]: execution tiles of the FFN (e, first padded row, rows
 *                in the tile, slot): each slot's run of expert e (q[e, r] consecutive
 *                blocks) cut into tiles of 256 rows (the last may be shorter), in the same
 *                slot/expert order.
 *   plan_info    int32 [MOE_PI_LEN]: see MOE_PI_*.
 * The owner of expert e is slot h(e) = floor(e * P / E).  The plan is deterministic and
 * bit-identical across calls.  Runs on one CTA. */
MOE_API int moe_plan_blocks(const moe_cfg* cfg, const int32_t* counts, uint32_t variant_mask,
                    int32_t* block_off, int32_t* q, int32_t* slot_load, int32_t* slot_off,
                    int32_t* blocks, int32_t* tiles, int32_t* plan_info, int32_t* status,
                    moe_stream_t stream);

/* Tile-aligned dispatch: a stable counting sort of the (t, j) pairs by expert.
 *   x          bf16 [T, d]; topk_ids, topk_gates [T, k]; block_off [E+1].
 *   xp         bf16 [R_max, d]: row beta*block_off[e] + i holds x[t] of expert e's i-th
 *              pair in token order; padding rows of each expert's blocks are zero; rows at
 *              or beyond beta*B are not written.  May be NULL: then only the row maps
 *              below are written (for moe_expert_ffn with MOE_FFN_GATHER_X).
 *   row_token  int32 [R_max]: t on valid rows, -1 on padding rows.
 *   row_gate   fp32 [R_max]: topk_gates[t, j] on valid rows, 0 on padding rows.
 *   tok_row    int32 [T, k]: the padded row of pair (t, j).
 * Ids outside [0, E) set MOE_STATUS_BAD_ID; rows beyond an expert's blocks set
 * MOE_STATUS_OVERFLOW and are dropped. */
MOE_API int moe_dispatch_permute(const moe_cfg* cfg, const uint16_t* x, const int32_t* topk_ids,
                         const float* topk_gates, const int32_t* block_off, uint16_t* xp,
                         int32_t* row_token, float* row_gate, int32_t* tok_row,
                         int32_t* status, moe_stream_t stream);

/* Grouped SwiGLU expert FFN over the planner's tiles (expert-computation equation):
 * for each tile of expert e, Z = Xp[rows] W1_e^T (fp32 accumulate on the tensor cores),
 * A = SiLU(G) * U rounded to bf16 into a_scratch, then O = A W2_e^T.
 *   xp         bf16 [R_max, d] from moe_dispatch_permute, or with MOE_FFN_GATHER_X the
 *              token rows x bf16 [T, d] (Xp[r] = x[row_token[r]] is then read in place).
 *   w1         bf16 [E, 2f, d] (rows 0..f-1 = G, f..2f-1 = U; K-major).
 *   w2         bf16 [E, d, f] (K-major).
 *   tiles, plan_info from moe_plan_blocks; row_token, row_gate from moe_dispatch_permute.
 *   a_scratch  caller-owned scratch of moe_workspace_size(cfg, MOE_WS_FFN_SCRATCH)
 *              bytes: A (bf16 [R_max, f]) then the tile-scheduler counters, which the
 *              call zeroes itself.
 *   out        MOE_FFN_FUSED_COMBINE: y fp32 [T, d], zeroed by the call, then
 *              y[row_token[r]] += row_gate[r] * O[r] for every valid row (fp32 atomic
 *              adds: the summation order, and so the last bits, may vary run to run).
 *              MOE_FFN_WRITE_O: O bf16 [R_max, d] (rows of the plan's tiles).
 *   mode       MOE_FFN_FUSED_COMBINE or MOE_FFN_WRITE_O, optionally | MOE_FFN_STRICT_SLOTS,
 *              | MOE_FFN_SM_PAIR and | MOE_FFN_GATHER_X.
 * Two persistent kernels (FC1+SwiGLU, then FC2) of one CTA per SM (in clusters of two
 * CTAs with MOE_FFN_SM_PAIR); every wait inside them is bounded and sets
 * MOE_STATUS_TIMEOUT instead of hanging. */
MOE_API int moe_expert_ffn(const moe_cfg* cfg, const uint16_t* xp, const uint16_t* w1,
                   const uint16_t* w2, const int32_t* tiles, const int32_t* plan_info,
                   const int32_t* row_token, const float* row_gate, int mode,
                   uint16_t* a_scratch, void* out, int32_t* status, moe_stream_t stream);

/* Deterministic gate-weighted combine (expert-computation equation):
 * y[t] = sum_{j=0..k-1} topk_gates[t, j] * O[tok_row[t, j]], in that order, fp32.
 *   o bf16 [R_max, d]; tok_row, topk_gates [T, k]; y fp32 [T, d] (overwritten). */
MOE_API int moe_combine(const moe_cfg* cfg, const uint16_t* o, const int32_t* tok_row,
                const float* topk_gates, float* y, int32_t* status, moe_stream_t stream);

/* Size of the library's fixed FC1-output array used by moe_expert_ffn_noalloc. */
#define MOE_NOALLOC_SCRATCH_BYTES (64u << 20)

/* moe_expert_ffn without the caller's scratch buffer, for callers that cannot allocate
 * device memory (a plugin or custom operator that its host framework hands only inputs
 * and outputs, or a deployment that forbids cudaMalloc after start-up).  The pages have no
 * counterpart: this is a deployment variant of the FFN entry point above.
 *   Arguments, outputs and device status are those of moe_expert_ffn, without a_scratch:
 *   its contents (A, the tile-scheduler counters, the one-launch FFN's readiness counters
 *   and the slot record, together moe_workspace_size(cfg, MOE_WS_FFN_SCRATCH) bytes) live
 *   in a library-owned array of MOE_NOALLOC_SCRATCH_BYTES, which they must not exceed, else
 *   the call returns MOE_ERR_TOO_LARGE and enqueues nothing.  The modes are those of
 *   moe_expert_ffn except MOE_FFN_SAVE_Z (Z for a backward pass needs the caller's
 *   scratch) and MOE_FFN_RECORD_SLOTS (the caller could not read the record back): both
 *   return MOE_ERR_INVALID_ARG.
 *   The call allocates nothing.  The array is reserved on every GPU where the library's
 *   device code is loaded, until the process exits.  The first call on a device looks up
 *   the array's device address (cudaGetSymbolAddress, with that device current) and caches
 *   it with the current CUDA context, so make that first call before any stream capture; a
 *   call under a different context of the device (after cudaDeviceReset) looks it up
 *   again, so it too must come before any capture.
 *   All calls share the array and it keeps the last call's contents; every call zeroes the
 *   counters that must start at zero.  Calls whose kernels overlap on the GPU (e.g. on two
 *   streams) race on the array and must be serialised. */
MOE_API int moe_expert_ffn_noalloc(const moe_cfg* cfg, const uint16_t* xp, const uint16_t* w1,
                                   const uint16_t* w2, const int32_t* tiles,
                                   const int32_t* plan_info, const int32_t* row_token,
                                   const float* row_gate, int mode, void* out,
                                   int32_t* status, moe_stream_t stream);

/* Backward, step 1: the gradient rows of the expert outputs ("MegaFlux" summary,
 * Methodology 2, backward gradients: D_e = dL/dO_e; Backward item 3: D_e is requantized).
 *   dy         fp32 [T, d]: dL/dy.
 *   row_token, row_gate from moe_dispatch_permute; plan_info from moe_plan_blocks.
 *   d_rows     bf16 [R_max, d]: row r < beta * B holds bf16(row_gate[r] * dy[row_token[r]])
 *              (round to nearest even), zeros on padding rows.
 * A token index outside [0, T) sets MOE_STATUS_BAD_ID and gives a zero row. */
MOE_API int moe_dispatch_grad(const moe_cfg* cfg, const float* dy, const int32_t* row_token,
                              const float* row_gate, const int32_t* plan_info,
                              uint16_t* d_rows, int32_t* status, moe_stream_t stream);

/* Backward, step 2: the expert computation's gradients (same section; the weights are
 * stored w1 [E, 2f, d] and w2 [E, d, f], so each of the pages' products is taken with that
 * transpose), on the tensor cores, bf16 operands and fp32 accumulation:
 *   dA = D w2_e, dZ = [dA * U * SiLU'(G), dA * SiLU(G)] (bf16, requantized), dX = dZ w1_e,
 *   dx[t] = sum over t's rows of dX (fp32 atomic adds; the order of the adds, and so the
 *   last bits, may vary), dW2_e = D^T A and dW1_e = dZ^T Xp over expert e's rows.
 *   xp         bf16 [R_max, d] from moe_dispatch_permute (zero padding rows).
 *   w1, w2, tiles, plan_info, block_off, row_token as for the forward.
 *   d_rows     from moe_dispatch_grad.
 *   saved      the a_scratch of the forward moe_expert_ffn call made with MOE_FFN_SAVE_Z
 *              (A and Z of the same rows).
 *   bwd_scratch moe_workspace_size(cfg, MOE_WS_BWD_SCRATCH) bytes: dZ then counters.
 *   dx         fp32 [T, d], zeroed by the call.
 *   dw1        fp32 [E, 2f, d] and dw2 fp32 [E, d, f]: written in full (zero for idle
 *              experts).
 * Four persistent kernels (dA + SwiGLU backward, dX, dW2, dW1) of one CTA per SM; every
 * wait is bounded and sets MOE_STATUS_TIMEOUT instead of hanging.  Needs d % 256 == 0 and
 * f % 128 == 0. */
MOE_API int moe_expert_ffn_backward(const moe_cfg* cfg, const uint16_t* xp, const uint16_t* w1,
                                    const uint16_t* w2, const int32_t* tiles,
                                    const int32_t* plan_info, const int32_t* block_off,
                                    const int32_t* row_token, const uint16_t* d_rows,
                                    const uint16_t* saved, uint16_t* bwd_scratch, float* dx,
                                    float* dw1, float* dw2, int32_t* status,
                                    moe_stream_t stream);

/* Static text for a return code (negative) or a status bit mask (positive). */
MOE_API const char* moe_status_string(int code);

#ifdef __cplusplus
}
#endif
#endif /* MOESKEW_H */
