// The grouped expert FFN on whole 256-row tiles (tcgen05 + TMEM, fed by TMA): FC1 + SwiGLU,
// and FC2 with the gate-weighted combine fused into its epilogue.  These are the two-launch
// FFN's default kernels.
//
// "MegaFlux" summary, Methodology 2, expert-computation equation:
//   Z_e = X_e W1_e,  Z_e = [G_e, U_e],  A_e = SiLU(G_e) * U_e,  O_e = A_e W2_e,
//   y_t = sum_{e in S_t} p_{t,e} O_e[t].
// A work item is one planner tile (up to 256 rows of one expert) times one n-tile: 128
// output columns of A for FC1 (the B tile stacks the n-tile's 128 G rows of W1_e over its
// 128 U rows), 256 output columns of y for FC2.
//
// Why a 256-row tile on one SM: a K step of 64 then moves A (256 rows, 32 KB) and B (256
// rows, 32 KB) for 2 x 128x256x64 MMAs, i.e. 64 bytes per tensor-core clock of the SM, where
// a 128-row tile moves 48 KB per 128x256x64 MMA (96 B/clk).  On B200 an SM takes in about
// 69 B/clk from L2 (copies from L2 plus, for a cta_group::2 pair, the partner's B half), so
// the 128-row tile is capped near 0.73 of the tensor rate and the 256-row tile is not (0.98
// measured with operands in L2).  The price: the two 128x256 fp32 accumulators fill all 512
// TMEM columns, so the next item cannot start in a spare accumulator.  Instead the epilogue
// frees the accumulator half by half: the next item's MMAs for rows 0..127 start as soon as
// the first half has been read, and its MMAs for rows 128..255 may lag them by up to the
// three pipeline stages while the second half is still being read (1.8 % faster on the
// DeepSeek-V3-shaped layer, 14 % on the 4096-token layer than freeing both at once).  The
// epilogue itself is kept short:
//   FC1: SiLU(g) = g/2 + (g/2) tanh(g/2) with the tanh.approx instruction (one MUFU op); the
//        warps that read TMEM never touch global memory (a warp's pending global stores
//        hold up its later instructions, TMEM loads included): they write A, rounded to
//        bf16, into a shared-memory staging buffer laid out as 32-row x 64-column boxes with
//        the 128-byte swizzle, and a store warp writes the boxes to A with TMA stores.
//   FC2, fused combine: each warp scales its 32 rows by the gates, transposes 32 x 32 chunks
//        through a swizzled 4 KB shared-memory slot and adds them into y with 16-byte vector
//        reductions, each instruction covering four whole 128-byte row segments.
//   FC2, O rows (MOE_FFN_WRITE_O): O rounded to bf16 leaves like FC1's A, through the
//        staging buffer and TMA stores (256 columns per item: two 128-column rounds per half);
//        moe_combine then adds each token's k rows in order.  Each warp first reads its 128
//        columns of a half into registers (64 bf16 pairs) and frees the half, then stages
//        them: the TMA stores share the SM's copy engine with the operand loads and take
//        about 1300 clocks per 32 KB round, which the next item's MMAs no longer wait for
//        (9 % faster FC2 + combine on the 16384-token sweep layers, 2 % on the
//        DeepSeek-V3-shaped layer).
// The fused-combine FC2 on whole tiles is an option (MOE_FFN_FC2_WHOLE): its reductions,
// about 2 TB/s of fp32 adds into y competing with the operand copies for L2, cannot overlap
// the next item's MMAs here, and the tile-half FC2 (double-buffered accumulators) is as fast
// or faster on the layers measured.
//
// Roles (384 threads, one CTA per SM, persistent):
//   warp 0      TMA producer: draws items from the global (or, strict slots, the slot's)
//               counter, passes them through a ring in shared memory, and loads per K step
//               the A rows [row0, row0 + 256) (the second 128-row box only when the tile
//               has more than 128 rows) and the item's 256 B rows into a 3-stage ring
//               (128-byte swizzle).
//   warp 1      MMA issuer: per K step tcgen05.mma.cta_group::1.kind::f16 M=128 N=256 for
//               rows 0..127 into TMEM columns [0, 256), and for rows 128..255 into
//               [256, 512) (queued for up to three stages until the epilogue has read the
//               previous item's second half); commit frees the stage; after the last K step
//               the accumulators go to the epilogue.
//   warps 2..9  epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 (32 rows of each half)
//               and half of the accumulator columns ((w - 2) / 4 picks which).
//   warp 10     store warp (FC1, and FC2 with O rows): TMA stores of the staged boxes whose
//               rows are in the tile (tile sizes are multiples of 64 rows), then frees the
//               staging buffer once the copies have read it.  Idle in the fused combine.
//   warp 11     FC1 only, when asked: zeroes the CTA's share of y (16-byte stores), which the
//               following fused-combine FC2 adds into, while FC1 computes; without it the
//               host writes y with a memset before FC1 (470 MB at T = 16384, d = 7168).
// Every wait is bounded (globaltimer); on expiry the kernel sets MOE_STATUS_TIMEOUT, the
// other roles drop out, copies and MMAs in flight are waited for, TMEM is freed.
#include "tc_util.cuh"

namespace moe {
namespace {

constexpr int WM = 256;                 // rows per item
constexpr int HM = 128;                 // rows per MMA (TMEM lanes)
constexpr int WK = 64;                  // K per stage: one 128-byte swizzle span of bf16
constexpr int WN = 256;                 // MMA N (FC1: 128 G + 128 U columns)
constexpr int W_ST = 3;                 // stages
constexpr int W_A_BYTES = WM * WK * 2;  // 32 KB
constexpr int W_B_BYTES = WN * WK * 2;  // 32 KB
constexpr int W_STAGE = W_A_BYTES + W_B_BYTES;
constexpr int W_HALF_A = HM * WK * 2;   // one 128-row box
constexpr int W_STG_BYTES = 32768;      // 128 rows x 128 bf16 (one store round); FC2 fused: 8 x 4 KB
constexpr int W_RING = 8;
constexpr int W_EPI_WARPS = 8;          // two per TMEM lane quadrant
constexpr int W_THREADS = 32 * (4 + W_EPI_WARPS);
constexpr int W_ZERO_WARP = 3 + W_EPI_WARPS;
// full[ST], empty[ST], drain, tfull, tfree[2], staged, stgfree, ifull[RING], iempty[RING]
constexpr int W_NBARS = 2 * W_ST + 6 + 2 * W_RING;
constexpr int W_META = 512;
constexpr int W_SMEM = W_ST * W_STAGE + W_STG_BYTES + W_META + 1024;
static_assert(W_SMEM <= 227 * 1024, "shared memory");
static_assert(W_NBARS * 8 + 4 * (2 + W_RING) <= W_META, "meta");
static_assert(W_EPI_WARPS * 4096 <= W_STG_BYTES, "FC2 transpose slots");
// kind::f16: D fp32, A and B bf16, both K-major, N = 256, M = 128
constexpr uint32_t W_IDESC =
    (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(WN >> 3) << 17) | ((uint32_t)(HM >> 4) << 24);

struct WideArgs {
  int32_t* sched;  // item counters: [0], or [slot] with strict slots; zeroed by the host
  const int32_t* tiles;
  const int32_t* plan_info;
  const int32_t* row_token;  // FC2
  const float* row_gate;     // FC2
  float* y;                  // FC2: y fp32 [T, d], zeroed by the host
  int32_t* status;
  long long r_max;
  int T, d, E, P, f;
  int n_k, n_n;     // K steps of 64, n-tiles per tile
  int n_group;      // n-tiles per group of the item order (n_n: no grouping)
  int brows_per_e;  // B rows per expert: FC1 2f, FC2 d
  int strict;
  int32_t* slot_rec;  // MOE_FFN_RECORD_SLOTS: per tile, bit (unit mod P) [+ 8 for FC2]
  uint4* zero;        // FC1: y to zero for the fused combine (16-byte units), or null
  long long zero_n16;
  unsigned long long timeout_ns;
};

// Items come in groups of n_group n-tiles (column stripes of the output): group by group,
// within a group tile by tile, within a tile its n-tiles.
struct WideSched {
  int32_t* counter;
  long long total;
  int m_base, n_n, n_group, tiles;
};

__device__ WideSched wide_sched(const WideArgs& a) {
  WideSched s;
  s.n_n = a.n_n;
  s.n_group = (a.n_group > 0 && a.n_group < a.n_n) ? a.n_group : a.n_n;
  const int* pi = a.plan_info;
  if (!a.strict) {
    s.counter = a.sched;
    s.tiles = max(pi[MOE_PI_NTILES], 0);
    s.m_base = 0;
  } else {
    const int r = (int)blockIdx.x % a.P;
    const int lo = pi[MOE_PI_SLOT_TILE_OFF + r], hi = pi[MOE_PI_SLOT_TILE_OFF + r + 1];
    s.counter = a.sched + r;
    s.tiles = max(hi - lo, 0);
    s.m_base = lo;
  }
  s.total = (long long)s.tiles * a.n_n;
  return s;
}

struct WideTile {
  int m, e, row0, nrows, n;
  bool ok;
};
__device__ __forceinline__ WideTile wide_tile(const WideArgs& a, const WideSched& s, int L) {
  WideTile t;
  const int per_group = s.tiles * s.n_group;
  const int g = L / per_group;
  const int r = L - g * per_group;
  const int width = min(s.n_group, s.n_n - g * s.n_group);  // the last group may be narrower
  const int mt = r / width;
  t.n = g * s.n_group + (r - mt * width);
  const int m = s.m_base + mt;
  t.m = m;
  const int4 v = __ldg(reinterpret_cast<const int4*>(a.tiles) + m);
  t.e = v.x;
  t.row0 = v.y;
  t.nrows = v.z;
  // tiles hold whole 64-row blocks; a 32-row store box is then all in the tile or all out
  t.ok = v.x >= 0 && v.x < a.E && v.y >= 0 && (long long)v.y < a.r_max && v.z > 0 &&
         v.z <= WM && (v.z & 31) == 0;
  return t;
}

// SiLU(g) = g * sigmoid(g) = g/2 + (g/2) tanh(g/2)
__device__ __forceinline__ float silu_tanh(float g) {
  const float h = 0.5f * g;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
  return fmaf(h, t, h);
}

// What an item's epilogue produces
enum { EPI_SWIGLU = 1, EPI_COMBINE = 2, EPI_STORE_O = 3 };

// KIND EPI_SWIGLU: FC1 + SwiGLU -> A (tmO = A's store map); EPI_COMBINE: FC2 + fused
// combine -> y; EPI_STORE_O: FC2 -> O bf16 (tmO = O's store map)
template <int KIND>
__global__ void __launch_bounds__(W_THREADS, 1)
wide_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
            const __grid_constant__ CUtensorMap tmO, const WideArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stg = smem + W_ST * W_STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg + W_STG_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + W_NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ring = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + W_ST + s); };
  const uint32_t drain_bar = smem_u32(bars + 2 * W_ST);
  const uint32_t tfull_bar = smem_u32(bars + 2 * W_ST + 1);
  // tfree[h]: the epilogue has read accumulator half h (TMEM columns [256 h, +256))
  auto tfree_bar = [&](int h) { return smem_u32(bars + 2 * W_ST + 2 + h); };
  const uint32_t staged_bar = smem_u32(bars + 2 * W_ST + 4);
  const uint32_t stgfree_bar = smem_u32(bars + 2 * W_ST + 5);
  auto ifull_bar = [&](int i) { return smem_u32(bars + 2 * W_ST + 6 + i); };
  auto iempty_bar = [&](int i) { return smem_u32(bars + 2 * W_ST + 6 + W_RING + i); };
  auto sA = [&](int s) { return smem_u32(smem + s * W_STAGE); };
  auto sB = [&](int s) { return smem_u32(smem + s * W_STAGE + W_A_BYTES); };
  constexpr int PHASE = KIND == EPI_SWIGLU ? 1 : 2;
  constexpr bool STORE_WARP = KIND != EPI_COMBINE;

  if (threadIdx.x == 0) {
    for (int s = 0; s < W_ST; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(drain_bar, 1);
    mbar_init(tfull_bar, 1);
    mbar_init(tfree_bar(0), W_EPI_WARPS);
    mbar_init(tfree_bar(1), W_EPI_WARPS);
    mbar_init(staged_bar, W_EPI_WARPS);
    mbar_init(stgfree_bar, 1);
    for (int i = 0; i < W_RING; ++i) {
      mbar_init(ifull_bar(i), 1);
      // MMA thread, epilogue warps (and the store thread)
      mbar_init(iempty_bar(i), 1 + W_EPI_WARPS + (STORE_WARP ? 1 : 0));
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmW);
    if (STORE_WARP) prefetch_tmap(&tmO);
  }
  if (warp == 1) tmem_alloc<false, 512>(smem_u32(tmem_slot));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WideSched sch = wide_sched(a);

  // consumers: the item of ring position `it`, -1 when the work is done, -2 when the wait
  // gave up
  auto take_item = [&](int it) -> int {
    const int slot = it % W_RING;
    if (!mbar_wait(ifull_bar(slot), (uint32_t)(it / W_RING) & 1u, abort_flag, a.status,
                   a.timeout_ns, true))
      return -2;
    return ring[slot];
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, pending = 0, pend_parity = 0;
      bool bad_tile = false;
      for (int it = 0;; ++it) {
        const int slot = it % W_RING;
        if (!mbar_wait(iempty_bar(slot), ((uint32_t)(it / W_RING) & 1u) ^ 1u, abort_flag,
                       a.status, a.timeout_ns, true))
          break;
        const long long v = atomicAdd(sch.counter, 1);
        const int L = v < sch.total ? (int)v : -1;
        ring[slot] = L;
        mbar_arrive(ifull_bar(slot));
        if (L < 0) break;
        const WideTile t = wide_tile(a, sch, L);
        if (!t.ok) {
          bad_tile = true;
          continue;
        }
        if (a.slot_rec)
          atomicOr(a.slot_rec + t.m, 1 << ((int)(blockIdx.x % a.P) + (PHASE == 2 ? 8 : 0)));
        const bool two = t.nrows > HM;
        // B rows: FC1 the n-tile's G rows (its U rows f further on), FC2 256 rows of W2_e
        const int brow = t.e * a.brows_per_e + t.n * (PHASE == 1 ? WN / 2 : WN);
        const int brow2 = PHASE == 1 ? brow + a.f : brow + WN / 2;
        const uint32_t tx = (two ? 2 : 1) * W_HALF_A + W_B_BYTES;
        bool stop = false;
        for (int kb = 0; kb < a.n_k; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.status, a.timeout_ns,
                         true)) {
            stop = true;
            break;
          }
          mbar_expect_tx(full_bar(stage), tx);
          // B first: the weights come from the farthest memory
          tma_load_2d(sB(stage), &tmW, full_bar(stage), kb * WK, brow);
          tma_load_2d(sB(stage) + W_B_BYTES / 2, &tmW, full_bar(stage), kb * WK, brow2);
          tma_load_2d(sA(stage), &tmX, full_bar(stage), kb * WK, t.row0);
          if (two) tma_load_2d(sA(stage) + W_HALF_A, &tmX, full_bar(stage), kb * WK, t.row0 + HM);
          pending |= 1u << stage;
          pend_parity = (pend_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == W_ST) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (stop) break;
      }
      if (bad_tile) set_status(a.status, MOE_STATUS_PLAN);
      if (*abort_flag) {
        // let the copies already armed land before shared memory goes away
        for (int s = 0; s < W_ST; ++s)
          if (pending >> s & 1u)
            mbar_wait(full_bar(s), pend_parity >> s & 1u, abort_flag, a.status, a.timeout_ns,
                      false);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc_it = 0;
      bool issued = false;
      for (int it = 0;; ++it) {
        const int L = take_item(it);
        if (L == -2) break;
        mbar_arrive(iempty_bar(it % W_RING));
        if (L < 0) break;
        const WideTile t = wide_tile(a, sch, L);
        if (!t.ok) continue;
        const bool two = t.nrows > HM;
        const uint32_t par = ((uint32_t)acc_it & 1u) ^ 1u;  // the previous item's phase
        // the previous item's first accumulator half has been read out
        if (!mbar_wait(tfree_bar(0), par, abort_flag, a.status, a.timeout_ns, true)) break;
        tc_fence_after();
        // second-half MMAs may lag the first half's by up to W_ST stages while the
        // epilogue still reads the previous item's second half
        bool m1_ready = false, stop = false;
        // queued stages are consecutive: the first one, its K step, and how many
        int pend_stage = 0, pend_kb = 0, npend = 0;
        auto issue_m1 = [&](int st, int kb) {
          const uint32_t a0 = sA(st), b0 = sB(st);
#pragma unroll
          for (int kk = 0; kk < WK / 16; ++kk)
            umma_bf16<false>(tmem_base + WN, sw128_desc(a0 + W_HALF_A + kk * 32),
                             sw128_desc(b0 + kk * 32), W_IDESC, (kb | kk) != 0);
          umma_commit_all<false>(empty_bar(st));
        };
        for (int kb = 0; kb < a.n_k; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, a.status, a.timeout_ns, true)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = sA(stage), b0 = sB(stage);
#pragma unroll
          for (int kk = 0; kk < WK / 16; ++kk)
            umma_bf16<false>(tmem_base, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32),
                             W_IDESC, (kb | kk) != 0);
          issued = true;
          if (!two) {
            umma_commit_all<false>(empty_bar(stage));
          } else {
            if (!m1_ready && mbar_try_wait(tfree_bar(1), par)) {
              m1_ready = true;
              tc_fence_after();
            }
            if (!m1_ready) {
              if (npend == 0) {
                pend_stage = stage;
                pend_kb = kb;
              }
              ++npend;
              if (npend == W_ST || kb == a.n_k - 1) {
                if (!mbar_wait(tfree_bar(1), par, abort_flag, a.status, a.timeout_ns, true)) {
                  stop = true;
                  break;
                }
                m1_ready = true;
                tc_fence_after();
                for (int i = 0; i < npend; ++i)
                  issue_m1((pend_stage + i) % W_ST, pend_kb + i);
                npend = 0;
              }
            } else {
              for (int i = 0; i < npend; ++i) issue_m1((pend_stage + i) % W_ST, pend_kb + i);
              npend = 0;
              issue_m1(stage, kb);
            }
          }
          if (++stage == W_ST) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (stop) break;
        if (!two && !mbar_wait(tfree_bar(1), par, abort_flag, a.status, a.timeout_ns, true))
          break;  // keep one phase of each half's barrier per item
        umma_commit_all<false>(tfull_bar);
        ++acc_it;
      }
      if (issued) {
        umma_commit_local<false>(drain_bar);
        mbar_wait(drain_bar, 0, abort_flag, a.status, a.timeout_ns, false);
      }
    }
  } else if (warp < 2 + W_EPI_WARPS) {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    const int quarter = warp & 3;    // TMEM lanes 32 quarter .. +31 = rows of each half
    const int ch = (warp - 2) >> 2;  // accumulator column half (FC1: of G and of U)
    int acc_it = 0, staged_n = 0;
    for (int it = 0;; ++it) {
      const int L = take_item(it);
      if (!__all_sync(0xffffffffu, L != -2)) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(iempty_bar(it % W_RING));
      if (L < 0) break;
      const WideTile t = wide_tile(a, sch, L);
      if (!t.ok) continue;
      const int halves = t.nrows > HM ? 2 : 1;
      const bool got = wait_inl(tfull_bar, (uint32_t)acc_it & 1u, abort_flag, a.status,
                                a.timeout_ns);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16);
      bool ok = true;
      if constexpr (KIND != EPI_COMBINE) {
        // A store round fills the staging buffer: quarter q's rows hold two 32-row x 128-byte
        // boxes (columns 0..63 and 64..127 of the round), box ch written by this warp, its
        // 16-byte chunk c of row `lane` at position c ^ (lane & 7) (128-byte swizzle).
        uint8_t* my_box = stg + quarter * 8192 + ch * 4096 + lane * 128;
#pragma unroll 1
        for (int h = 0; h < halves; ++h) {
          if constexpr (KIND == EPI_SWIGLU) {
            // one round per half: the item's 128 A columns, this warp's 64 from its 64 G and
            // 64 U columns (G at accumulator columns [256 h, +128), U at [256 h + 128, +128)),
            // each 32-column chunk written to its box row as soon as it is converted
            const bool fr = wait_inl(stgfree_bar, ((uint32_t)staged_n & 1u) ^ 1u, abort_flag,
                                     a.status, a.timeout_ns);
            if (!__all_sync(0xffffffffu, fr)) {
              ok = false;
              break;
            }
#pragma unroll 1
            for (int cc = 0; cc < 2; ++cc) {
              uint32_t g[32], u[32], p[16];
              const int col = 64 * ch + 32 * cc;
              tmem_ld32(taddr + h * WN + col, g);
              tmem_ld32(taddr + h * WN + WN / 2 + col, u);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i)
                p[i] = pack_bf16(silu_tanh(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]),
                                 silu_tanh(__uint_as_float(g[2 * i + 1])) *
                                     __uint_as_float(u[2 * i + 1]));
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int c = cc * 4 + i;
                *reinterpret_cast<uint4*>(my_box + ((c ^ (lane & 7)) << 4)) =
                    make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
              }
            }
            // accumulator half h has been read: the next item's MMAs for it may start (a
            // single-half item frees the unused second half at the same time, so that each
            // item completes one phase of both barriers)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(tfree_bar(h));
              if (halves == 1) mbar_arrive(tfree_bar(1));
            }
            fence_proxy_async();  // make the staging writes visible to the TMA engine
            __syncwarp();
            if (lane == 0) mbar_arrive(staged_bar);
            ++staged_n;
          } else {
            // O rows: the warp first reads all 128 of its accumulator columns of the half
            // (64 ch + 128 r .. +64 for the rounds r = 0, 1) into registers as bf16 and frees
            // the half, so that the next item's MMAs restart after the TMEM reads alone; the
            // two store rounds then go out of registers while those MMAs run
            uint32_t p[64];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              uint32_t v[32];
              tmem_ld32(taddr + h * WN + 128 * (k >> 1) + 64 * ch + 32 * (k & 1), v);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i)
                p[16 * k + i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(tfree_bar(h));
              if (halves == 1) mbar_arrive(tfree_bar(1));
            }
#pragma unroll
            for (int rnd = 0; rnd < 2; ++rnd) {
              // the staging buffer is free once the store warp's copies have read the last
              // round
              const bool fr = wait_inl(stgfree_bar, ((uint32_t)staged_n & 1u) ^ 1u, abort_flag,
                                       a.status, a.timeout_ns);
              if (!__all_sync(0xffffffffu, fr)) {
                ok = false;
                break;
              }
#pragma unroll
              for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(my_box + ((c ^ (lane & 7)) << 4)) =
                    make_uint4(p[32 * rnd + 4 * c], p[32 * rnd + 4 * c + 1],
                               p[32 * rnd + 4 * c + 2], p[32 * rnd + 4 * c + 3]);
              fence_proxy_async();  // make the staging writes visible to the TMA engine
              __syncwarp();
              if (lane == 0) mbar_arrive(staged_bar);
              ++staged_n;
            }
            if (!ok) break;
          }
        }
      } else {
        // fused combine: y[token] += gate * O over columns [256 n + 128 ch, +128) for this
        // warp's 32 rows of each half.  Each 32 x 32 chunk is staged in this warp's 4 KB slot
        // (row r's 16-byte group j at position j ^ (r & 7)); then lanes 8q..8q+7 of a vector
        // reduction take one 128-byte row segment.
        float* slot_f = reinterpret_cast<float*>(stg + (warp - 2) * 4096);
#pragma unroll 1
        for (int h = 0; h < halves; ++h) {
          const int rit = HM * h + 32 * quarter + lane;  // row inside the tile
          const long long row = (long long)t.row0 + rit;
          int tok = -1;
          float gate = 0.f;
          if (rit < t.nrows && row < a.r_max) {
            tok = __ldg(a.row_token + row);
            gate = __ldg(a.row_gate + row);
            if (tok >= a.T) tok = -1;
          }
          float* ybase = a.y + (long long)t.n * WN + 128 * ch + 4 * (lane & 7);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t v[32];
            tmem_ld32(taddr + h * WN + 128 * ch + 32 * c, v);
            tmem_wait_ld();
            if (c == 3) {
              // accumulator half h has been read (a single-half item also frees the second)
              tc_fence_before();
              __syncwarp();
              if (lane == 0) {
                mbar_arrive(tfree_bar(h));
                if (halves == 1) mbar_arrive(tfree_bar(1));
              }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<float4*>(slot_f + 32 * lane + 4 * (j ^ (lane & 7))) =
                  make_float4(gate * __uint_as_float(v[4 * j]),
                              gate * __uint_as_float(v[4 * j + 1]),
                              gate * __uint_as_float(v[4 * j + 2]),
                              gate * __uint_as_float(v[4 * j + 3]));
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int r = 4 * i + (lane >> 3);
              const int tk = __shfl_sync(0xffffffffu, tok, r);
              if (tk >= 0) {
                const float4 x = *reinterpret_cast<const float4*>(
                    slot_f + 32 * r + 4 * ((lane & 7) ^ (r & 7)));
                red_add_v4(ybase + (long long)tk * a.d + 32 * c, x);
              }
            }
            __syncwarp();
          }
        }
      }
      if (!ok) break;
      ++acc_it;
    }
  } else if (warp == W_ZERO_WARP) {
    // ------------------------------------------------------------ y zeroing (warp 11)
    if (a.zero) {
      const uint4 z = make_uint4(0, 0, 0, 0);
      for (long long i = (long long)blockIdx.x * 32 + lane; i < a.zero_n16;
           i += (long long)gridDim.x * 32)
        a.zero[i] = z;
    }
  } else if (STORE_WARP) {
    // ------------------------------------------------------------ store warp (warp 10)
    if (lane == 0) {
      constexpr int ROUNDS = KIND == EPI_SWIGLU ? 1 : 2;
      constexpr int OCOLS = 128 * ROUNDS;  // output columns per item
      int staged_n = 0;
      for (int it = 0;; ++it) {
        const int L = take_item(it);
        if (L == -2) break;
        mbar_arrive(iempty_bar(it % W_RING));
        if (L < 0) break;
        const WideTile t = wide_tile(a, sch, L);
        if (!t.ok) continue;
        const int halves = t.nrows > HM ? 2 : 1;
        bool stop = false;
        for (int hr = 0; hr < halves * ROUNDS; ++hr) {
          const int h = hr / ROUNDS, rnd = hr % ROUNDS;
          if (!mbar_wait(staged_bar, (uint32_t)staged_n & 1u, abort_flag, a.status,
                         a.timeout_ns, true)) {
            stop = true;
            break;
          }
          const int rows = min(t.nrows - HM * h, HM);
          const int x0 = t.n * OCOLS + 128 * rnd;
          for (int q = 0; q < 4; ++q) {
            if (32 * q >= rows) break;
            const uint32_t src = smem_u32(stg + q * 8192);
            const int y = t.row0 + HM * h + 32 * q;
            tma_store_2d(&tmO, src, x0, y);
            tma_store_2d(&tmO, src + 4096, x0 + 64, y);
          }
          bulk_commit();
          bulk_wait_read();  // the copies have read the staging buffer
          mbar_arrive(stgfree_bar);
          ++staged_n;
        }
        if (stop) break;
      }
      bulk_wait_all();  // the output is written before the CTA's shared memory goes away
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<false, 512>(tmem_base);
  }
}

template <int KIND>
cudaError_t launch_wide(const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& to,
                        const WideArgs& a, cudaStream_t st) {
  static OncePerDevice attr_once;
  cudaError_t err = once_per_device(attr_once, [&](int&) {
    return cudaFuncSetAttribute(wide_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                W_SMEM);
  });
  if (err != cudaSuccess) return err;
  wide_kernel<KIND><<<num_sms(), W_THREADS, W_SMEM, st>>>(tx, tw, to, a);
  return cudaGetLastError();
}

WideArgs wide_args(const moe_cfg& c, const int32_t* tiles, const int32_t* plan_info,
                   int32_t* sched, int32_t* status, bool strict, int32_t* slot_rec) {
  WideArgs a{};
  a.sched = sched;
  a.tiles = tiles;
  a.plan_info = plan_info;
  a.status = status;
  a.r_max = max_rows(c);
  a.T = c.T;
  a.d = c.d;
  a.E = c.E;
  a.P = c.P;
  a.f = c.f;
  a.strict = strict ? 1 : 0;
  a.slot_rec = slot_rec;
  a.timeout_ns = 2000000000ull;
  return a;
}

}  // namespace

bool fc1_wide_supported(int mode) {
  return !(mode & (MOE_FFN_SM_PAIR | MOE_FFN_GATHER_X | MOE_FFN_SAVE_Z | MOE_FFN_FC1_M128));
}
bool fc2_wide_supported(int mode) {
  if (mode & MOE_FFN_SM_PAIR) return false;
  return (mode & (MOE_FFN_WRITE_O | MOE_FFN_FC2_WHOLE)) != 0;
}

cudaError_t launch_fc1_wide(const moe_cfg& c, const uint16_t* xp, const uint16_t* w1,
                            const int32_t* tiles, const int32_t* plan_info, uint16_t* a_out,
                            int32_t* sched, int32_t* status, bool strict, int32_t* slot_rec,
                            float* y_zero, cudaStream_t st) {
  const long long r_max = max_rows(c);
  CUtensorMap tm_x, tm_w, tm_a;
  // Xp: 128-row boxes; W1: the n-tile's 128 G (or U) rows; A: 32-row store boxes
  if (!encode_2d(&tm_x, xp, c.d, r_max, HM) ||
      !encode_2d(&tm_w, w1, c.d, (uint64_t)c.E * 2 * c.f, WN / 2) ||
      !encode_2d(&tm_a, a_out, c.f, r_max, 32))
    return cudaErrorInvalidValue;
  WideArgs a = wide_args(c, tiles, plan_info, sched, status, strict, slot_rec);
  a.n_k = c.d / WK;
  a.n_n = c.f / 128;
  a.n_group = a.n_n;
  a.brows_per_e = 2 * c.f;
  if (y_zero) {  // T * d fp32, d % 256 == 0: whole 16-byte units
    a.zero = reinterpret_cast<uint4*>(y_zero);
    a.zero_n16 = (long long)c.T * c.d / 4;
  }
  return launch_wide<EPI_SWIGLU>(tm_x, tm_w, tm_a, a, st);
}

cudaError_t launch_fc2_wide(const moe_cfg& c, const uint16_t* a_in, const uint16_t* w2,
                            const int32_t* tiles, const int32_t* plan_info,
                            const int32_t* row_token, const float* row_gate, void* out,
                            bool write_o, int32_t* sched, int32_t* status, bool strict,
                            int32_t* slot_rec, cudaStream_t st) {
  const long long r_max = max_rows(c);
  CUtensorMap tm_a, tm_w, tm_o;
  // A: 128-row boxes; W2: 128-row boxes (two per 256-row n-tile); O: 32-row store boxes
  if (!encode_2d(&tm_a, a_in, c.f, r_max, HM) ||
      !encode_2d(&tm_w, w2, c.f, (uint64_t)c.E * c.d, WN / 2) ||
      (write_o && !encode_2d(&tm_o, out, c.d, r_max, 32)))
    return cudaErrorInvalidValue;
  WideArgs a = wide_args(c, tiles, plan_info, sched, status, strict, slot_rec);
  a.row_token = row_token;
  a.row_gate = row_gate;
  a.n_k = c.f / WK;
  a.n_n = c.d / WN;
  a.brows_per_e = c.d;
  if (write_o) {
    a.n_group = a.n_n;
    return launch_wide<EPI_STORE_O>(tm_a, tm_w, tm_o, a, st);
  }
  a.y = static_cast<float*>(out);
  a.n_group = fc2_n_group(c);
  return launch_wide<EPI_COMBINE>(tm_a, tm_w, tm_a, a, st);
}

}  // namespace moe
