// Grouped SwiGLU expert FFN on the sm_100a tensor cores (tcgen05 + TMEM, fed by TMA).
//
// "MegaFlux" summary, Methodology 2, expert-computation equation:
//   Z_e = X_e W1_e,  Z_e = [G_e, U_e],  A_e = SiLU(G_e) * U_e,  O_e = A_e W2_e,
//   y_t = sum_{e in S_t} p_{t,e} O_e[t].
// The pages' forward megakernel runs FC1, then FC2 on each token block ("Executor:
// Pipelined Expert Replication", Forward); here the blocks form the planner's tiles (up to
// 256 rows of one expert), and the GEMMs run as two persistent launches over the tile list,
// or as one (FC2 on a tile half starts once FC1 wrote its rows) for small layers.
//
// Two variants of one kernel template:
//   single SM (default): one CTA runs one 128-row half of a tile with
//     tcgen05.mma.cta_group::1 (M=128, N=256).
//   SM pair (MOE_FFN_SM_PAIR): a cluster of two CTAs on two SMs runs one 256-row tile.  Each CTA
//     loads its own 128 rows of the A tile and half of the B tile (128 of its 256 rows)
//     into its shared memory; CTA 0 issues tcgen05.mma.cta_group::2 (M=256, N=256), whose
//     accumulator lands in both CTAs' TMEM (each CTA: its 128 rows x 256 columns).  Each SM
//     therefore moves 32 KB per K step instead of 48 KB, and six stages fit where four did.
//     A tile of at most 128 rows runs as an M=128 pair MMA (64 rows per CTA; each CTA's
//     TMEM then holds its rows' first N/2 columns in lanes 0..63 and the other N/2 in
//     lanes 64..127), so no tensor work is spent on an empty half.  On the MoE workloads
//     measured here the two variants are within a few per cent; single SM is the default.
// Roles in every CTA (192 threads, one CTA per SM, persistent):
//   warp 0      TMA producer: A [128 x 64] and B [128 or 256 x 64] bf16 tiles per K step
//               into a ring of shared-memory stages (128-byte swizzle).  In a pair, both
//               CTAs' copies signal CTA 0's stage barrier.  With MOE_FFN_GATHER_X, FC1's A
//               tile is gathered from x itself (rows x[row_token[row]]), so the dispatched
//               copy Xp is never written.  Single SM: the warp's lanes copy the tile with
//               16-byte cp.async (8 lanes per 128-byte row segment, written at its
//               128-byte-swizzled place; padding rows copy token 0's row), each lane's copies
//               counted on the stage barrier by a cp.async mbarrier arrive; the MMA thread
//               fences the generic and async proxies before reading the stage.  SM pair:
//               lane l copies rows 4l..4l+3 with one TMA row-gather (tile::gather4) per K
//               step (fewer instructions for the warp, but the TMA unit takes ~1.8x longer
//               per stage than the MMAs need, so this variant is slower).
//   warp 1      MMA issuer (CTA 0 of a pair): one thread issues the MMAs of a stage into a
//               TMEM accumulator; tcgen05.commit frees the stage (in both CTAs of a pair)
//               and, after the last K step, hands the accumulator to the epilogue.
//   warps 2..5  epilogue: tcgen05.ld of the fp32 accumulator (warp w reads TMEM lanes
//               32*(w%4)..+31, i.e. 32 rows), then
//                 FC1: A = SiLU(G) * U rounded to bf16 -> scratch (the B tile stacks 128 rows
//                      of W1_e's G half over the matching 128 rows of its U half, so G and U
//                      of an output column sit 128 accumulator columns apart);
//                 FC2: y[row_token] += row_gate * O (fused combine): each 32 x 32 chunk is
//                      transposed through shared memory so that one 16-byte vector reduction
//                      instruction covers four whole 128-byte row segments; or O rounded to
//                      bf16 (unfused path).
//   TMEM holds two 256-column accumulators (512 columns): the epilogue of one work item
//   overlaps the MMAs of the next.
// Work items (tile, n-tile) are handed out in increasing order by a global atomic counter
// (the producer draws the next item when it is ready for it, so fast SMs take more) and
// passed to the other roles, and in a pair to the other CTA, through a small ring in
// shared memory.  All n-tiles of a tile are in flight together and consecutive tiles
// belong to the same expert, so each expert's weights stream from HBM about once.  With
// MOE_FFN_STRICT_SLOTS, unit u (a CTA, or a pair) draws from slot (u mod P)'s counter.
// Every mbarrier wait is bounded (globaltimer); on expiry the kernel sets
// MOE_STATUS_TIMEOUT, lets the other roles drop out, waits (bounded) for its own copies
// and MMAs in flight, frees its TMEM and returns.
#include "tc_util.cuh"

namespace moe {
namespace {

constexpr int BM = 128;   // A rows per CTA = TMEM lanes
constexpr int BK = 64;    // K per stage: 64 bf16 = 128 bytes = one swizzle span
constexpr int BN = 256;   // MMA N (FC1: 128 G + 128 U columns; FC2: 256 output columns)
constexpr int A_BYTES = BM * BK * 2;
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 2 * BN;
constexpr int RING = 8;                 // work items in flight between roles
constexpr int STG_STRIDE = 36;          // floats per staged row of the FC2 combine
constexpr int STG_BYTES = 4 * 32 * STG_STRIDE * 4;
constexpr int META_BYTES = 2048;        // barriers, ring, per-row tokens
constexpr unsigned long long kTimeoutNs = 2000000000ull;  // 2 s per wait
constexpr unsigned long long kTestTimeoutNs = 10000000ull;  // MOE_FFN_TEST_WAIT_TIMEOUT

template <int PHASE, bool PAIR>
struct Geo {
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;  // B rows held by one CTA
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = PAIR ? 6 : 4;
  static constexpr int TX_BYTES = PAIR ? 2 * STAGE_BYTES : STAGE_BYTES;  // per stage
  static constexpr int M = PAIR ? 2 * BM : BM;
  // kind::f16 instruction descriptor: D fp32 (bits 4-5 = 1), A bf16 (bits 7-9 = 1),
  // B bf16 (bits 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 at bit 17, M >> 4 at 24.
  static constexpr uint32_t idesc(int m) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
           ((uint32_t)(m >> 4) << 24);
  }
  static constexpr uint32_t IDESC = idesc(M);
  static constexpr uint32_t IDESC_M128 = idesc(BM);  // SM pair: a tile of at most 128 rows
  static constexpr int NBARS = 2 * STAGES + 5 + 2 * RING;
  static constexpr int STG = PHASE >= 2 ? STG_BYTES : 0;  // FC2 combine staging
  static constexpr int SMEM = STAGES * STAGE_BYTES + STG + META_BYTES + 1024;
};
static_assert(Geo<1, true>::SMEM <= 227 * 1024 && Geo<2, true>::SMEM <= 227 * 1024 &&
                  Geo<1, false>::SMEM <= 227 * 1024 && Geo<2, false>::SMEM <= 227 * 1024 &&
                  Geo<3, false>::SMEM <= 227 * 1024,
              "smem");
static_assert(Geo<1, true>::NBARS * 8 + 4 * (2 + RING) + 4 * 128 <= META_BYTES, "meta");

struct FfnArgs {
  int32_t* sched;           // this launch's counters: [0], or [slot] (strict); zeroed
  const int32_t* tiles;
  const int32_t* plan_info;
  const int32_t* row_token;
  const float* row_gate;
  void* out;
  int32_t* status;
  long long r_max;
  int T, d, f, E, P;
  int n_k;       // K steps of 64
  int n_n;       // n-tiles per tile
  int out_ld;    // output row length (elements)
  int write_o;   // FC2: store O (1) or fused combine (0)
  uint16_t* z;   // FC1 with MOE_FFN_SAVE_Z: Z = [G, U] bf16 [r_max, 2f] (else null)
  const void* x; // the token rows x bf16 [T, d] (gather)
  // PHASE 3 (FC1 and FC2 in one launch): FC2's K steps, n-tiles, output and row length,
  // and the per-(tile, half) readiness counters FC1's epilogue raises to ready_target
  int n_k2, n_n2, out_ld2;
  void* out2;
  int32_t* ready;
  int ready_target;
  int strict;
  int n_group;   // n-tiles per group of the item order (see Sched); n_n: no grouping
  int32_t* slot_rec;  // MOE_FFN_RECORD_SLOTS: per tile, bit (u mod P) [+ 8 for FC2] of every
                      // unit u that ran one of its items; else null
  unsigned long long timeout_ns;
};

// the slot record: unit u (an SM, or an SM pair) ran an item of tile m of GEMM gp
__device__ __forceinline__ void record_slot(const FfnArgs& a, int m, int gp, int unit) {
  if (a.slot_rec) atomicOr(a.slot_rec + m, 1 << ((unit % a.P) + (gp == 2 ? 8 : 0)));
}

// ------------------------------------------------------------------ work schedule
// Item L of a unit's range -> tile m, n-tile n and (single SM) the tile half.  Items come in
// groups of n_group n-tiles (column stripes of the output): group by group, within a group
// row by row (a row = a tile half, or a tile), within a row its n-tiles.  With
// n_group = n_n that is row by row with all n-tiles of a row together.
struct Sched {
  int32_t* counter;  // global counter this unit draws items from
  long long total;   // items in its range
  long long total1;  // PHASE 3: the first total1 items are FC1's, the rest FC2's
  int m_base, n_n, n_n2, halves;
  int rows;          // rows (tile halves, or tiles) in the unit's range
  int n_group;
  __device__ void decode(int L, int& m, int& n, int& half) const {
    const int per_group = rows * n_group;
    const int g = L / per_group;
    const int r = L - g * per_group;
    const int width = min(n_group, n_n - g * n_group);  // the last group may be narrower
    const int t = r / width;
    n = g * n_group + (r - t * width);
    m = m_base + t / halves;
    half = t % halves;
  }
  // PHASE 3: also which GEMM the item belongs to (1: FC1, 2: FC2)
  __device__ int decode_phase(int L, int& m, int& n, int& half) const {
    if (L < total1) {
      decode(L, m, n, half);
      return 1;
    }
    const int L2 = (int)(L - total1);
    n = L2 % n_n2;
    const int t = L2 / n_n2;
    m = t / halves;
    half = t % halves;
    return 2;
  }
};

template <bool PAIR>
__device__ Sched make_sched(const FfnArgs& a) {
  Sched s;
  s.n_n = a.n_n;
  s.halves = PAIR ? 1 : 2;
  const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int* pi = a.plan_info;
  s.n_n2 = a.n_n2;
  s.total1 = 1LL << 62;
  // grouping only for a plain FC2 launch (PHASE 3 decodes its FC2 items separately)
  s.n_group = (a.n_group > 0 && a.n_group < a.n_n && a.n_n2 == 0) ? a.n_group : a.n_n;
  if (!a.strict) {
    s.counter = a.sched;
    s.rows = max(pi[MOE_PI_NTILES], 0) * s.halves;
    s.total = (long long)s.rows * a.n_n;
    s.m_base = 0;
    if (a.n_n2 > 0) {  // PHASE 3: FC2's items after FC1's
      s.total1 = s.total;
      s.total += (long long)max(pi[MOE_PI_NTILES], 0) * a.n_n2 * s.halves;
    }
  } else {
    const int r = unit % a.P;
    const int lo = pi[MOE_PI_SLOT_TILE_OFF + r], hi = pi[MOE_PI_SLOT_TILE_OFF + r + 1];
    s.counter = a.sched + r;
    s.rows = max(hi - lo, 0) * s.halves;
    s.total = (long long)s.rows * a.n_n;
    s.m_base = lo;
  }
  return s;
}

struct TileInfo {
  int e, row0, nrows;  // row0 / nrows of this CTA's share of the tile
  int a_row;           // A rows this CTA loads (moved inside the buffer when empty)
  bool ok;             // a well-formed tile (all roles of both CTAs agree)
  bool run;            // this work item is executed (single SM: its half has rows)
  bool m128;           // SM pair: the tile has at most 128 rows, so the pair runs an M = 128
                       // MMA and each CTA holds 64 of them
};
// `part`: single SM, the 128-row half; SM pair, the CTA's rank
template <bool PAIR>
__device__ __forceinline__ TileInfo read_tile(const FfnArgs& a, int m, int part) {
  TileInfo t;
  const int4 v = __ldg(reinterpret_cast<const int4*>(a.tiles) + m);
  t.e = v.x;
  t.ok = v.x >= 0 && v.x < a.E && v.y >= 0 && (long long)v.y < a.r_max && v.z > 0 &&
         v.z <= 2 * BM;
  t.m128 = PAIR && v.z <= BM;
  const int share = t.m128 ? BM / 2 : BM;  // rows per CTA
  t.row0 = v.y + share * part;
  t.nrows = min(v.z - share * part, share);
  t.run = t.ok && (PAIR || t.nrows > 0);
  t.a_row = t.nrows > 0 ? t.row0 : (int)max(a.r_max - share, 0LL);
  return t;
}

// ------------------------------------------------------------------ the kernel
// PHASE 1: FC1 + SwiGLU, 2: FC2 (+ combine); GATHER (FC1 only): A rows read from x itself
template <int PHASE, bool PAIR, bool GATHER>
__global__ void __launch_bounds__(THREADS, 1)
ffn_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const __grid_constant__ CUtensorMap tmA64, const __grid_constant__ CUtensorMap tmA2,
           const __grid_constant__ CUtensorMap tmB2, const FfnArgs a) {
  using G = Geo<PHASE, PAIR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* stg = reinterpret_cast<float*>(smem + G::STAGES * G::STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G::STAGES * G::STAGE_BYTES + G::STG);
  // bars: full[S], empty[S], tmem_full[2], tmem_empty[2], drain, item_full[R], item_empty[R]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + G::NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ring = reinterpret_cast<volatile int*>(tmem_slot + 2);  // [RING] items
  int* s_tok = reinterpret_cast<int*>(tmem_slot + 2 + RING);           // [4][32] tokens

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool mma_cta = rank == 0;  // single SM: always; pair: CTA 0 issues the MMAs
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + G::STAGES + s); };
  auto tfull_bar = [&](int b) { return smem_u32(bars + 2 * G::STAGES + b); };
  auto tempty_bar = [&](int b) { return smem_u32(bars + 2 * G::STAGES + 2 + b); };
  const uint32_t drain_bar = smem_u32(bars + 2 * G::STAGES + 4);
  auto ifull_bar = [&](int i) { return smem_u32(bars + 2 * G::STAGES + 5 + i); };
  auto iempty_bar = [&](int i) { return smem_u32(bars + 2 * G::STAGES + 5 + RING + i); };
  auto sA = [&](int s) { return smem_u32(smem + s * G::STAGE_BYTES); };
  auto sB = [&](int s) { return smem_u32(smem + s * G::STAGE_BYTES + A_BYTES); };

  // single-SM FC1 gathering A with cp.async: every producer lane arrives on the stage
  static_assert(PHASE == 1 || !GATHER, "only FC1 reads rows from x");
  constexpr bool lsu_gather = GATHER && !PAIR;
  if (threadIdx.x == 0) {
    for (int s = 0; s < G::STAGES; ++s) {
      // the MMA CTA's producer (expect_tx), plus the 32 lanes' cp.async arrivals
      mbar_init(full_bar(s), lsu_gather ? 33 : 1);
      mbar_init(empty_bar(s), 1);  // the MMA thread's commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), PAIR ? 8 : 4);  // every epilogue warp (of both CTAs)
    }
    mbar_init(drain_bar, 1);
    for (int i = 0; i < RING; ++i) {
      mbar_init(ifull_bar(i), 1);
      // consumers of an item: MMA thread + 4 epilogue warps (+ the other CTA's producer
      // and 4 epilogue warps)
      mbar_init(iempty_bar(i), PAIR ? 10 : 5);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (PAIR) prefetch_tmap(&tmA64);
    if (PHASE == 3) {
      prefetch_tmap(&tmA2);
      prefetch_tmap(&tmB2);
    }
  }
  if (warp == 1) tmem_alloc<PAIR, TMEM_COLS>(smem_u32(tmem_slot));
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const Sched sch = make_sched<PAIR>(a);

  if (warp == 0 && !GATHER) {
    // ------------------------------------------------------------ TMA producer
    // One thread, item by item: draw the next item, pass it on, then issue its K steps.
    // (Drawing items ahead with the whole warp, as the row-gather producer below does,
    // measured 5-15 % slower on this path.)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t pending = 0, pend_parity = 0;
      bool bad_tile = false;
      for (int it = 0;; ++it) {
        const int slot = it % RING;
        const uint32_t ph = (uint32_t)(it / RING) & 1u;
        int L;
        if (mma_cta) {
          if (!mbar_wait(iempty_bar(slot), ph ^ 1u, abort_flag, a.status, a.timeout_ns, true))
            break;
          const long long v = atomicAdd(sch.counter, 1);
          L = v < sch.total ? (int)v : -1;
          ring[slot] = L;
          if constexpr (PAIR) {
            st_remote_u32(mapa(smem_u32((const void*)(ring + slot)), 1), (uint32_t)L);
            mbar_arrive_remote(mapa(ifull_bar(slot), 1));
          }
          mbar_arrive(ifull_bar(slot));
        } else {
          if (!mbar_wait(ifull_bar(slot), ph, abort_flag, a.status, a.timeout_ns, true)) break;
          L = ring[slot];
          mbar_arrive_remote(mapa(iempty_bar(slot), 0));
        }
        if (L < 0) break;
        int m, n, half;
        const int gp = PHASE == 3 ? sch.decode_phase(L, m, n, half) : (sch.decode(L, m, n, half), PHASE);
        const TileInfo ti = read_tile<PAIR>(a, m, PAIR ? (int)rank : half);
        if (!ti.ok) bad_tile = true;
        if (!ti.run) continue;
        if (mma_cta) record_slot(a, m, gp, PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x);
        // FC1 B rows: single SM, the n-tile's 128 G rows over its 128 U rows; SM pair, CTA
        // `rank` holds G rows [64 rank, +64) of the n-tile over the matching U rows
        int brow;
        if (gp == 1) brow = ti.e * 2 * a.f + n * (BN / 2) + (PAIR ? (int)rank * (BN / 4) : 0);
        else brow = ti.e * a.d + n * BN + (PAIR ? (int)rank * (BN / 2) : 0);
        uint32_t tx = G::TX_BYTES;
        if (PAIR && ti.m128) tx = 2 * (A_BYTES / 2 + G::B_BYTES);  // 64 A rows per CTA
        const CUtensorMap* mapA = (PHASE == 3 && gp == 2) ? &tmA2 : &tmA;
        const CUtensorMap* mapB = (PHASE == 3 && gp == 2) ? &tmB2 : &tmB;
        const int nk = (PHASE == 3 && gp == 2) ? a.n_k2 : a.n_k;
        if (PHASE == 3 && gp == 2) {
          // FC2 reads A rows of this tile half: wait until FC1 wrote all of them
          if (!wait_count(a.ready + (2 * m + half), a.ready_target, abort_flag, a.status,
                          a.timeout_ns))
            break;
          fence_proxy_async_global();
        }
        bool stop = false;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.status, a.timeout_ns,
                         true)) {
            stop = true;
            break;
          }
          if (mma_cta) mbar_expect_tx(full_bar(stage), tx);
          if constexpr (PAIR) {
            const uint32_t fb = mapa(full_bar(stage), 0);
            tma_load_2d_pair(sA(stage), ti.m128 ? &tmA64 : &tmA, fb, kb * BK, ti.a_row);
            tma_load_2d_pair(sB(stage), &tmB, fb, kb * BK, brow);
            if (PHASE == 1)
              tma_load_2d_pair(sB(stage) + G::B_BYTES / 2, &tmB, fb, kb * BK, brow + a.f);
          } else {
            tma_load_2d(sA(stage), mapA, full_bar(stage), kb * BK, ti.a_row);
            tma_load_2d(sB(stage), mapB, full_bar(stage), kb * BK, brow);
            if (gp == 1)
              tma_load_2d(sB(stage) + G::B_BYTES / 2, mapB, full_bar(stage), kb * BK,
                          brow + a.f);
          }
          pending |= 1u << stage;
          pend_parity = (pend_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == G::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (stop) break;
      }
      if (bad_tile && mma_cta) set_status(a.status, MOE_STATUS_PLAN);
      if (*abort_flag && mma_cta) {
        // let the copies already armed land before shared memory goes away
        for (int s = 0; s < G::STAGES; ++s)
          if (pending >> s & 1u)
            mbar_wait(full_bar(s), pend_parity >> s & 1u, abort_flag, a.status, a.timeout_ns,
                      false);
      }
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer, FC1 from x
    // The whole warp walks the items; lane 0 alone draws items and handles the barriers,
    // and broadcasts what the other lanes need.  Item it+1 is drawn, located and its row
    // tokens loaded while item it's K steps are issued, so the counter, tile and token
    // round trips stay off the critical path between items.
    constexpr bool gather = true;
    int stage = 0;
    uint32_t phase = 0;
    uint32_t pending = 0, pend_parity = 0;
    bool bad_tile = false;
    long long drawn = 0;  // lane 0 of the MMA CTA: the counter value taken for the next item
    // lane 0 of the MMA CTA: wait until item it's ring slot is free, then take a number
    auto take = [&](int it) -> bool {
      if (!mbar_wait(iempty_bar(it % RING), ((uint32_t)(it / RING) & 1u) ^ 1u, abort_flag,
                     a.status, a.timeout_ns, true))
        return false;
      drawn = atomicAdd(sch.counter, 1);
      return true;
    };
    // hand item it to the other roles (MMA CTA) or receive it (other CTA of a pair);
    // returns the item number, or -1 when the work is done or a wait gave up
    auto publish = [&](int it, bool took) -> int {
      const int slot = it % RING;
      int L = -1;
      if (lane == 0) {
        if (mma_cta) {
          if (took) {
            L = drawn < sch.total ? (int)drawn : -1;
            ring[slot] = L;
            if constexpr (PAIR) {
              st_remote_u32(mapa(smem_u32((const void*)(ring + slot)), 1), (uint32_t)L);
              mbar_arrive_remote(mapa(ifull_bar(slot), 1));
            }
            mbar_arrive(ifull_bar(slot));
          }
        } else if (mbar_wait(ifull_bar(slot), (uint32_t)(it / RING) & 1u, abort_flag, a.status,
                             a.timeout_ns, true)) {
          L = ring[slot];
          mbar_arrive_remote(mapa(iempty_bar(slot), 0));
        }
      }
      return __shfl_sync(0xffffffffu, L, 0);
    };
    struct Item {
      int L;        // item number, -1: none
      int m;        // tile
      int brow;     // first B row
      TileInfo ti;
      int mt[4];    // cp.async gather: tokens of rows lane + 32q (padding rows: token 0)
      int4 tok;     // row gather: tokens of rows 4 lane .. 4 lane + 3
    };
    auto locate = [&](Item& w) {
      int m, n, half;
      sch.decode(w.L, m, n, half);
      w.m = m;
      w.ti = read_tile<PAIR>(a, m, PAIR ? (int)rank : half);
      // FC1 B rows: single SM, the n-tile's 128 G rows over its 128 U rows; SM pair, CTA
      // `rank` holds G rows [64 rank, +64) of the n-tile over the matching U rows, so that
      // in both accumulator layouts (M = 256 and M = 128) a row's G and U sit in one lane
      if (PHASE == 1) w.brow = w.ti.e * 2 * a.f + n * (BN / 2) + (PAIR ? (int)rank * (BN / 4) : 0);
      else w.brow = w.ti.e * a.d + n * BN + (PAIR ? (int)rank * (BN / 2) : 0);
    };
    // rows outside the tile and padding rows read token 0's row; their results are dropped
    auto load_tokens = [&](Item& w) {
      if (!gather || !w.ti.run) return;
      if (lsu_gather) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = 32 * q + lane;
          const long long r = (long long)w.ti.row0 + i;
          const int t = (i < w.ti.nrows && r < a.r_max) ? __ldg(a.row_token + r) : 0;
          w.mt[q] = (t >= 0 && t < a.T) ? t : 0;
        }
      } else {
        const int i0 = 4 * lane;
        const long long r0 = (long long)w.ti.row0 + i0;
        int4 t = make_int4(0, 0, 0, 0);
        // r_max and row0 are multiples of 64, so the four rows are all in range or none is
        if (i0 < w.ti.nrows && r0 + 3 < a.r_max)
          t = __ldg(reinterpret_cast<const int4*>(a.row_token + r0));
        t.x = (i0 + 0 < w.ti.nrows && t.x >= 0 && t.x < a.T) ? t.x : 0;
        t.y = (i0 + 1 < w.ti.nrows && t.y >= 0 && t.y < a.T) ? t.y : 0;
        t.z = (i0 + 2 < w.ti.nrows && t.z >= 0 && t.z < a.T) ? t.z : 0;
        t.w = (i0 + 3 < w.ti.nrows && t.w >= 0 && t.w < a.T) ? t.w : 0;
        w.tok = t;
      }
    };
    // cp.async gather: copy j (0..31) of a K step moves 16-byte chunk c = lane & 7 of tile
    // row 4j + rl (rl = lane >> 3) to its 128-byte-swizzled place: chunk c ^ (row & 7),
    // where row & 7 = 4 (j & 1) + rl
    const int rl = lane >> 3, ck = lane & 7;
    const uint32_t off_even = 128 * rl + ((ck ^ rl) << 4);
    const uint32_t off_odd = 128 * rl + ((ck ^ (rl + 4)) << 4);
    const int k_pub = min(2, a.n_k - 1), k_tok = min(4, a.n_k - 1);  // n_k >= 2

    Item cur, nxt;
    bool took = lane == 0 && mma_cta ? take(0) : true;
    cur.L = publish(0, took);
    if (cur.L >= 0) {
      locate(cur);
      load_tokens(cur);
    }
    for (int it = 0; cur.L >= 0; ++it) {
      if (!cur.ti.ok) bad_tile = true;
      if (cur.ti.run && lane == 0 && mma_cta)
        record_slot(a, cur.m, PHASE, PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x);
      bool drew = false, located = false, loaded = false;
      took = true;
      nxt.L = -1;
      bool stop = false;
      if (cur.ti.run) {
        int tj[32];  // cp.async gather: token of row 4j + rl
        if (lsu_gather) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            tj[j] = __shfl_sync(0xffffffffu, cur.mt[j >> 3], (4 * j + rl) & 31);
        }
        for (int kb = 0; kb < a.n_k; ++kb) {
          int ready = 1;
          if (lane == 0) {
            ready = mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.status, a.timeout_ns,
                              true);
            if (ready) {
              if (mma_cta) {
                uint32_t tx = lsu_gather ? G::TX_BYTES - A_BYTES : G::TX_BYTES;
                if (PAIR && cur.ti.m128) tx = 2 * (A_BYTES / 2 + G::B_BYTES);  // 64 A rows
                mbar_expect_tx(full_bar(stage), tx);
              }
              // B first: the weights come from the farthest memory
              if constexpr (PAIR) {
                const uint32_t fb = mapa(full_bar(stage), 0);
                if (PHASE == 1) {
                  tma_load_2d_pair(sB(stage), &tmB, fb, kb * BK, cur.brow);
                  tma_load_2d_pair(sB(stage) + G::B_BYTES / 2, &tmB, fb, kb * BK,
                                   cur.brow + a.f);
                } else {
                  tma_load_2d_pair(sB(stage), &tmB, fb, kb * BK, cur.brow);
                }
                if (!gather)
                  tma_load_2d_pair(sA(stage), cur.ti.m128 ? &tmA64 : &tmA, fb, kb * BK,
                                   cur.ti.a_row);
              } else {
                tma_load_2d(sB(stage), &tmB, full_bar(stage), kb * BK, cur.brow);
                if (PHASE == 1)
                  tma_load_2d(sB(stage) + G::B_BYTES / 2, &tmB, full_bar(stage), kb * BK,
                              cur.brow + a.f);
                if (!gather) tma_load_2d(sA(stage), &tmA, full_bar(stage), kb * BK, cur.ti.a_row);
              }
            }
          }
          if (!__shfl_sync(0xffffffffu, ready, 0)) {
            stop = true;
            break;
          }
          if constexpr (PAIR) {
            if (gather && lane < (cur.ti.m128 ? 16 : 32))
              tma_gather4_pair(sA(stage) + lane * 512, &tmA, mapa(full_bar(stage), 0), kb * BK,
                               cur.tok);
          } else if (lsu_gather) {
            const uint32_t a0 = sA(stage);
            const __nv_bfloat16* xk =
                reinterpret_cast<const __nv_bfloat16*>(a.x) + kb * BK + 8 * ck;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              cp_async16(a0 + 512 * j + ((j & 1) ? off_odd : off_even),
                         xk + (long long)tj[j] * a.d);
            cp_async_arrive(full_bar(stage));
          }
          pending |= 1u << stage;
          pend_parity = (pend_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == G::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          // the next item, overlapped with this one's copies
          if (kb == 0) {
            if (lane == 0 && mma_cta) took = take(it + 1);
            drew = true;
          }
          if (kb == k_pub) {
            nxt.L = publish(it + 1, took);
            if (nxt.L >= 0) locate(nxt);
            located = true;
          }
          if (kb == k_tok) {
            if (nxt.L >= 0) load_tokens(nxt);
            loaded = true;
          }
        }
        if (stop) break;
      }
      if (!drew && lane == 0 && mma_cta) took = take(it + 1);
      if (!located) {
        nxt.L = publish(it + 1, took);
        if (nxt.L >= 0) locate(nxt);
      }
      if (!loaded && nxt.L >= 0) load_tokens(nxt);
      cur = nxt;
    }
    if (lane == 0) {
      if (bad_tile && mma_cta) set_status(a.status, MOE_STATUS_PLAN);
      if (*abort_flag && mma_cta) {
        // let the copies already armed land before shared memory goes away
        for (int s = 0; s < G::STAGES; ++s)
          if (pending >> s & 1u)
            mbar_wait(full_bar(s), pend_parity >> s & 1u, abort_flag, a.status, a.timeout_ns,
                      false);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && mma_cta) {
      int stage = 0;
      uint32_t phase = 0;
      int acc_it = 0;
      bool issued = false;
      for (int it = 0;; ++it) {
        const int slot = it % RING;
        const uint32_t ph = (uint32_t)(it / RING) & 1u;
        if (!mbar_wait(ifull_bar(slot), ph, abort_flag, a.status, a.timeout_ns, true)) break;
        const int L = ring[slot];
        mbar_arrive(iempty_bar(slot));
        if (L < 0) break;
        int m, n, half;
        const int gp = PHASE == 3 ? sch.decode_phase(L, m, n, half) : (sch.decode(L, m, n, half), PHASE);
        const TileInfo ti = read_tile<PAIR>(a, m, PAIR ? 0 : half);
        if (!ti.run) continue;
        const int nk = (PHASE == 3 && gp == 2) ? a.n_k2 : a.n_k;
        const int buf = acc_it & 1;
        const uint32_t use = (uint32_t)(acc_it >> 1) & 1u;
        if (!mbar_wait(tempty_bar(buf), use ^ 1u, abort_flag, a.status, a.timeout_ns, true))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        const uint32_t idesc = ti.m128 ? G::IDESC_M128 : G::IDESC;
        bool stop = false;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, a.status, a.timeout_ns, true)) {
            stop = true;
            break;
          }
          tc_fence_after();
          if (lsu_gather) fence_proxy_async();  // A arrived through the generic proxy
          const uint32_t a0 = sA(stage), b0 = sB(stage);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_bf16<PAIR>(d_tmem, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), idesc,
                            (kb | kk) != 0);
          issued = true;
          umma_commit_all<PAIR>(empty_bar(stage));
          if (++stage == G::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (stop) break;
        umma_commit_all<PAIR>(tfull_bar(buf));
        ++acc_it;
      }
      if (issued) {
        // every MMA this thread issued has completed once the drain barrier fires
        umma_commit_local<PAIR>(drain_bar);
        mbar_wait(drain_bar, 0, abort_flag, a.status, a.timeout_ns, false);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;         // TMEM lanes this warp may read: 32*quarter ..
    const int rit = quarter * 32 + lane;  // row inside this CTA's half
    const int ew = warp - 2;              // staging slot of this warp
    int acc_it = 0;
    for (int it = 0;; ++it) {
      const int slot = it % RING;
      const uint32_t ph = (uint32_t)(it / RING) & 1u;
      const bool have =
          mbar_wait(ifull_bar(slot), ph, abort_flag, a.status, a.timeout_ns, true);
      if (!__all_sync(0xffffffffu, have)) break;
      const int L = ring[slot];
      __syncwarp();
      if (lane == 0) {
        if (mma_cta) mbar_arrive(iempty_bar(slot));
        else mbar_arrive_remote(mapa(iempty_bar(slot), 0));
      }
      if (L < 0) break;
      int m, n, half;
      const int gp = PHASE == 3 ? sch.decode_phase(L, m, n, half) : (sch.decode(L, m, n, half), PHASE);
      const TileInfo ti = read_tile<PAIR>(a, m, PAIR ? (int)rank : half);
      if (!ti.run) continue;
      void* const outp = (PHASE == 3 && gp == 2) ? a.out2 : a.out;
      const int out_ld = (PHASE == 3 && gp == 2) ? a.out_ld2 : a.out_ld;
      const int buf = acc_it & 1;
      const uint32_t use = (uint32_t)(acc_it >> 1) & 1u;
      const bool got =
          mbar_wait(tfull_bar(buf), use, abort_flag, a.status, a.timeout_ns, true);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      // Accumulator layout in TMEM.  Single SM, or SM pair with M = 256: lane 32 quarter + i
      // holds row 32 quarter + i of this CTA's rows, all N columns.  SM pair with M = 128:
      // lanes 0..63 hold the CTA's 64 rows with columns [0, N/2), lanes 64..127 the same rows
      // with columns [N/2, N), both at TMEM columns [0, N/2).
      const bool m128 = PAIR && ti.m128;
      const int lrow = m128 ? 32 * (quarter & 1) + lane : rit;
      const int chalf = m128 ? (quarter >> 1) : 0;  // accumulator column half of this warp
      const long long row = (long long)ti.row0 + lrow;
      const bool valid = lrow < ti.nrows && row < a.r_max;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
      if (gp == 1) {
        // chunk cc: G at TMEM column gcol, U at ucol, giving A columns [ocol, ocol + 32) of
        // the n-tile.  Single SM: B held the n-tile's 128 G rows over its 128 U rows.  SM
        // pair: CTA r's B half held G rows [64 r, +64) over the matching U rows, so
        // accumulator columns [128 r, +64) are G and [128 r + 64, +64) are U.
        __nv_bfloat16* A = reinterpret_cast<__nv_bfloat16*>(outp) + row * out_ld + n * (BN / 2);
        const int ncc = m128 ? 2 : 4;
#pragma unroll 1
        for (int cc = 0; cc < ncc; ++cc) {
          int gcol, ucol, ocol;
          if (!PAIR) {
            gcol = 32 * cc;
            ucol = BN / 2 + 32 * cc;
            ocol = 32 * cc;
          } else if (!m128) {
            gcol = 128 * (cc >> 1) + 32 * (cc & 1);
            ucol = gcol + 64;
            ocol = 64 * (cc >> 1) + 32 * (cc & 1);
          } else {
            gcol = 32 * cc;
            ucol = 64 + 32 * cc;
            ocol = 64 * chalf + 32 * cc;
          }
          uint32_t g[32], u[32];
          tmem_ld32(taddr + gcol, g);
          tmem_ld32(taddr + ucol, u);
          tmem_wait_ld();
          uint32_t p[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a0 = silu(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
            const float a1 = silu(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
            p[i] = pack_bf16(a0, a1);
          }
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(A + ocol);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
            if (a.z) {  // keep Z = [G, U] for the backward pass
              uint4* zg = reinterpret_cast<uint4*>(a.z + row * 2 * a.f + n * (BN / 2) + ocol);
              uint4* zu = reinterpret_cast<uint4*>(a.z + row * 2 * a.f + a.f + n * (BN / 2) + ocol);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                zg[i] = make_uint4(
                    pack_bf16(__uint_as_float(g[8 * i + 0]), __uint_as_float(g[8 * i + 1])),
                    pack_bf16(__uint_as_float(g[8 * i + 2]), __uint_as_float(g[8 * i + 3])),
                    pack_bf16(__uint_as_float(g[8 * i + 4]), __uint_as_float(g[8 * i + 5])),
                    pack_bf16(__uint_as_float(g[8 * i + 6]), __uint_as_float(g[8 * i + 7])));
                zu[i] = make_uint4(
                    pack_bf16(__uint_as_float(u[8 * i + 0]), __uint_as_float(u[8 * i + 1])),
                    pack_bf16(__uint_as_float(u[8 * i + 2]), __uint_as_float(u[8 * i + 3])),
                    pack_bf16(__uint_as_float(u[8 * i + 4]), __uint_as_float(u[8 * i + 5])),
                    pack_bf16(__uint_as_float(u[8 * i + 6]), __uint_as_float(u[8 * i + 7])));
              }
            }
          }
        }
        if (PHASE == 3) {
          // publish this warp's A rows of the tile half to FC2's producers (other CTAs
          // read them with TMA, through the async proxy)
          fence_proxy_async_global();
          __threadfence();
          __syncwarp();
          if (lane == 0) atomicAdd(a.ready + (2 * m + half), 1);
        }
      } else if (a.write_o) {
        // chunk c: TMEM columns [32 c, +32) = output columns n BN + ocol0 + 32 c ..
        const int ncc = m128 ? 4 : 8, ocol0 = 128 * chalf;
        __nv_bfloat16* O = reinterpret_cast<__nv_bfloat16*>(outp);
        uint4* dst = reinterpret_cast<uint4*>(O + row * out_ld + n * BN + ocol0);
#pragma unroll 1
        for (int c = 0; c < ncc; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[c * 4 + i] = make_uint4(
                  pack_bf16(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1])),
                  pack_bf16(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3])),
                  pack_bf16(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5])),
                  pack_bf16(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7])));
          }
        }
      } else {
        // fused combine: y[token] += gate * O, staged per 32 x 32 chunk so that lanes
        // 8q..8q+7 of one reduction cover a whole 128-byte segment of one row
        const int ncc = m128 ? 4 : 8, ocol0 = 128 * chalf;
        int tok = -1;
        float gate = 0.f;
        if (valid) {
          tok = __ldg(a.row_token + row);
          gate = __ldg(a.row_gate + row);
          if (tok >= a.T) tok = -1;
        }
        s_tok[ew * 32 + lane] = tok;
        float* my_row = stg + (ew * 32 + lane) * STG_STRIDE;
        float* y = reinterpret_cast<float*>(outp) + n * BN + ocol0 + 4 * (lane & 7);
        __syncwarp();
#pragma unroll 1
        for (int c = 0; c < ncc; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4*>(my_row + 4 * j) = make_float4(
                gate * __uint_as_float(v[4 * j]), gate * __uint_as_float(v[4 * j + 1]),
                gate * __uint_as_float(v[4 * j + 2]), gate * __uint_as_float(v[4 * j + 3]));
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = 4 * i + (lane >> 3);
            const int tk = s_tok[ew * 32 + r];
            if (tk >= 0) {
              const float4 x = *reinterpret_cast<const float4*>(
                  stg + (ew * 32 + r) * STG_STRIDE + 4 * (lane & 7));
              red_add_v4(y + (long long)tk * out_ld + c * 32, x);
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (mma_cta) mbar_arrive(tempty_bar(buf));
        else mbar_arrive_remote(mapa(tempty_bar(buf), 0));
      }
      ++acc_it;
    }
  }

  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<PAIR, TMEM_COLS>(tmem_base);
  }
}

// ------------------------------------------------------------------ host side
template <int PHASE, bool PAIR, bool GATHER = false>
cudaError_t launch_one(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& ta64,
                       const CUtensorMap& ta2, const CUtensorMap& tb2, const FfnArgs& args,
                       cudaStream_t st) {
  auto kern = ffn_kernel<PHASE, PAIR, GATHER>;
  static OncePerDevice attr_once;
  cudaError_t err = once_per_device(attr_once, [&](int&) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Geo<PHASE, PAIR>::SMEM);
  });
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = Geo<PHASE, PAIR>::SMEM;
  cfg.stream = st;
  if (PAIR) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(2);
    int clusters = 0;
    static OncePerDevice occ_once;
    err = once_per_device(occ_once, [&](int& n) {
      return cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    }, &clusters);
    if (err != cudaSuccess) return err;
    if (clusters < 1) return cudaErrorInvalidConfiguration;
    cfg.gridDim = dim3(2 * clusters);
  } else {
    cfg.gridDim = dim3(num_sms());
  }
  // strict slots need one unit per slot at least (checked by the caller before anything is
  // enqueued; a unit u >= units would never exist to run slot u's tiles)
  const int units = PAIR ? (int)cfg.gridDim.x / 2 : (int)cfg.gridDim.x;
  if (args.strict && units < args.P) return cudaErrorInvalidConfiguration;
  return cudaLaunchKernelEx(&cfg, kern, ta, tb, ta64, ta2, tb2, args);
}

}  // namespace

// Whether a mode without a launch-count flag runs FC1 and FC2 as one launch: tiny layers
// only (one launch saves a launch and overlaps FC1's tail with FC2's start; from a few items
// per SM on, two launches with FC1 on whole 256-row tiles are faster, about 10 % on the
// 4096-token layer with 14 FC1 half-tile items per SM)
bool ffn_auto_one_launch(const moe_cfg& c, int mode) {
  if (mode & (kOneLaunchExcludes | MOE_FFN_ONE_LAUNCH | MOE_FFN_TEST_WAIT_TIMEOUT)) return false;
  const long long fc1_items = (long long)c.T * c.k / BM * (c.f / (BN / 2));
  return fc1_items <= 2LL * num_sms();
}

cudaError_t launch_ffn(const moe_cfg& c, const uint16_t* xp, const uint16_t* w1,
                       const uint16_t* w2, const int32_t* tiles, const int32_t* plan_info,
                       const int32_t* row_token, const float* row_gate, int mode,
                       uint16_t* a_scratch, void* out, int32_t* status, cudaStream_t st) {
  const bool write_o = (mode & MOE_FFN_WRITE_O) != 0;
  const bool pair = (mode & MOE_FFN_SM_PAIR) != 0;
  const long long r_max = max_rows(c);
  cudaError_t err;
  // y is zeroed for the fused combine: by the whole-tile FC1 kernel beside its work when it
  // runs (two launches), else by a memset first
  const bool one_launch_forced = (mode & (MOE_FFN_ONE_LAUNCH | MOE_FFN_TEST_WAIT_TIMEOUT)) != 0;
  const bool zero_in_fc1 = !write_o && c.T > 0 && r_max > 0 && fc1_wide_supported(mode) &&
                           !one_launch_forced && !ffn_auto_one_launch(c, mode);
  if (!write_o && c.T > 0 && !zero_in_fc1) {
    err = cudaMemsetAsync(out, 0, sizeof(float) * (size_t)c.T * c.d, st);
    if (err != cudaSuccess) return err;
  }
  if (r_max == 0) return cudaSuccess;
  // scheduler counters after A in the scratch buffer: [0, 8) FC1, [8, 16) FC2
  int32_t* sched = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(a_scratch) +
                                              ffn_a_bytes(c));
  err = cudaMemsetAsync(sched, 0, 16 * sizeof(int32_t), st);
  if (err != cudaSuccess) return err;
  int32_t* slot_rec = nullptr;
  if (mode & MOE_FFN_RECORD_SLOTS) {
    slot_rec = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(a_scratch) +
                                          ffn_record_offset(c));
    err = cudaMemsetAsync(slot_rec, 0, (size_t)ffn_record_bytes(c), st);
    if (err != cudaSuccess) return err;
  }

  const bool gather = (mode & MOE_FFN_GATHER_X) != 0;
  // A maps: boxes of 128 rows, and of 64 rows for the SM pair's tiles of at most 128 rows;
  // B maps: one CTA's share of the n-tile (FC1 on a pair: 64 G rows, then 64 U rows)
  CUtensorMap tm_xp, tm_xp64, tm_w1, tm_a, tm_a64, tm_w2;
  // gather: `xp` is x [T, d], read one row per box by the row-gather copies
  if (!(gather ? encode_2d(&tm_xp, xp, c.d, (uint64_t)c.T, 1)
               : encode_2d(&tm_xp, xp, c.d, r_max, BM)) ||
      !(gather ? encode_2d(&tm_xp64, xp, c.d, (uint64_t)c.T, 1)
               : encode_2d(&tm_xp64, xp, c.d, r_max, BM / 2)) ||
      !encode_2d(&tm_w1, w1, c.d, (uint64_t)c.E * 2 * c.f, pair ? BN / 4 : BN / 2) ||
      !encode_2d(&tm_a, a_scratch, c.f, r_max, BM) ||
      !encode_2d(&tm_a64, a_scratch, c.f, r_max, BM / 2) ||
      !encode_2d(&tm_w2, w2, c.f, (uint64_t)c.E * c.d, pair ? BN / 2 : BN))
    return cudaErrorInvalidValue;

  FfnArgs a1{};
  a1.tiles = tiles;
  a1.plan_info = plan_info;
  a1.row_token = row_token;
  a1.row_gate = row_gate;
  a1.status = status;
  a1.r_max = r_max;
  a1.T = c.T;
  a1.d = c.d;
  a1.f = c.f;
  a1.E = c.E;
  a1.P = c.P;
  a1.strict = (mode & MOE_FFN_STRICT_SLOTS) != 0;
  a1.slot_rec = slot_rec;
  a1.timeout_ns = kTimeoutNs;

  a1.n_group = 0;  // FC1: no grouping
  FfnArgs a2 = a1;
  a1.sched = sched;
  a1.out = a_scratch;
  a1.n_k = c.d / BK;
  a1.n_n = c.f / (BN / 2);
  a1.out_ld = c.f;
  a1.write_o = 0;
  a1.x = gather ? xp : nullptr;
  // Z after A, the scheduler counters and the readiness counters in the scratch buffer
  a1.z = (mode & MOE_FFN_SAVE_Z)
             ? reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(a_scratch) +
                                           ffn_scratch_bytes(c))
             : nullptr;
  a2.sched = sched + 8;
  a2.out = out;
  a2.n_k = c.f / BK;
  a2.n_n = c.d / BN;
  a2.n_group = write_o ? a2.n_n : fc2_n_group(c);
  a2.out_ld = c.d;
  a2.write_o = write_o;

  const bool test_timeout = (mode & MOE_FFN_TEST_WAIT_TIMEOUT) != 0;
  const bool one_launch = one_launch_forced || ffn_auto_one_launch(c, mode);
  if (one_launch) {
    // FC1 items, then FC2 items, in one persistent launch; FC2 waits per tile half
    int32_t* ready = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(a_scratch) +
                                                ffn_a_bytes(c) + kSchedBytes);
    err = cudaMemsetAsync(ready, 0, (size_t)ffn_ready_bytes(c), st);
    if (err != cudaSuccess) return err;
    FfnArgs a3 = a1;
    a3.n_k2 = a2.n_k;
    a3.n_n2 = a2.n_n;
    a3.out2 = out;
    a3.out_ld2 = a2.out_ld;
    a3.ready = ready;
    a3.ready_target = 4 * a1.n_n;  // four epilogue warps per FC1 n-tile of the half
    if (test_timeout) {            // a target nothing reaches, and short waits
      a3.ready_target += 1;
      a3.timeout_ns = kTestTimeoutNs;
    }
    return launch_one<3, false>(tm_xp, tm_w1, tm_xp64, tm_a, tm_w2, a3, st);
  }
  if (fc1_wide_supported(mode))
    err = launch_fc1_wide(c, xp, w1, tiles, plan_info, a_scratch, sched, status, a1.strict != 0,
                          slot_rec, zero_in_fc1 ? static_cast<float*>(out) : nullptr, st);
  else if (gather)
    err = pair ? launch_one<1, true, true>(tm_xp, tm_w1, tm_xp64, tm_a, tm_w2, a1, st)
               : launch_one<1, false, true>(tm_xp, tm_w1, tm_xp64, tm_a, tm_w2, a1, st);
  else
    err = pair ? launch_one<1, true>(tm_xp, tm_w1, tm_xp64, tm_a, tm_w2, a1, st)
               : launch_one<1, false>(tm_xp, tm_w1, tm_xp64, tm_a, tm_w2, a1, st);
  if (err != cudaSuccess) return err;
  if (fc2_wide_supported(mode))
    return launch_fc2_wide(c, a_scratch, w2, tiles, plan_info, row_token, row_gate, out,
                           write_o, a2.sched, status, a2.strict != 0, slot_rec, st);
  return pair ? launch_one<2, true>(tm_a, tm_w2, tm_a64, tm_a, tm_w2, a2, st)
              : launch_one<2, false>(tm_a, tm_w2, tm_a64, tm_a, tm_w2, a2, st);
}

int fc2_n_group(const moe_cfg& c) {
  // FC2's fused combine adds into y (T x d fp32).  When y is larger than what stays in L2,
  // its lines are written back and fetched again between a token's k contributions (the
  // sweep layer's 134 MB y cost 2 GB of DRAM traffic in FC2, about 10 y).  Items taken in
  // groups of n-tiles keep only the group's y columns live (T x 256 x 4 bytes per n-tile),
  // at the price of reading A once per group.  Estimated DRAM bytes: A x groups, plus y x 2
  // when the group's columns fit in 64 MB of L2 and y x 10 when they do not; the group
  // count with the least estimate wins (ties: fewer groups), groups of equal width.
  const int n_n = c.d / BN;
  const double stripe = (double)c.T * BN * 4;
  const double y_bytes = stripe * n_n;
  const double a_bytes = (double)max_rows(c) * c.f * 2;
  const double live_cap = 64.0 * 1024 * 1024;
  int best = n_n;
  double best_cost = 0;
  for (int groups = 1; groups <= n_n; ++groups) {
    const int width = (n_n + groups - 1) / groups;
    if ((n_n + width - 1) / width != groups) continue;  // same as a smaller group count
    const double cost = a_bytes * groups + (stripe * width <= live_cap ? 2.0 : 10.0) * y_bytes;
    if (groups == 1 || cost < best_cost) {
      best_cost = cost;
      best = width;
    }
  }
  return best;
}

int ffn_units(int mode) {
  if (!(mode & MOE_FFN_SM_PAIR)) return num_sms();
  // clusters of two CTAs that fit at once (the pair launches' grid)
  auto kern = ffn_kernel<2, true, false>;
  static OncePerDevice occ_once;
  int clusters = 0;
  cudaError_t err = once_per_device(occ_once, [&](int& n) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Geo<2, true>::SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = Geo<2, true>::SMEM;
    return cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
  }, &clusters);
  return err == cudaSuccess ? clusters : 0;
}

}  // namespace moe
