// Grouped SwiGLU expert FFN on the sm_100a tensor cores (tcgen05 + TMEM, fed by TMA).
//
// "MegaFlux" summary, Methodology 2, expert-computation equation:
//   Z_e = X_e W1_e,  Z_e = [G_e, U_e],  A_e = SiLU(G_e) * U_e,  O_e = A_e W2_e,
//   y_t = sum_{e in S_t} p_{t,e} O_e[t].
// The pages' forward megakernel runs FC1, then FC2 on each token block ("Executor:
// Pipelined Expert Replication", Forward); here the blocks are the planner's 128-row tiles
// and the two GEMMs are two persistent launches over the same tile list.
//
// Kernel shape (one CTA per SM, 192 threads, persistent over (m-tile, n-tile) work items):
//   warp 0      TMA producer: A tile [128 x 64] and B tile [256 x 64] bf16 per K step into
//               a 4-stage shared-memory ring (128-byte swizzle), one mbarrier per stage.
//   warp 1      MMA issuer: one thread issues tcgen05.mma.cta_group::1.kind::f16 (M=128,
//               N=256, K=16 x 4 per stage) into a TMEM accumulator; tcgen05.commit frees
//               the smem stage and, after the last K step, hands the accumulator over.
//   warps 2..5  epilogue: tcgen05.ld of the fp32 accumulator (each warp reads its own 32
//               TMEM lanes = 32 rows), then
//                 FC1: A = SiLU(G) * U rounded to bf16 -> a_scratch (the B tile stacks
//                      128 rows of W1_e's G half over the matching 128 rows of its U half,
//                      so G and U of the same output column sit 128 TMEM columns apart);
//                 FC2: y[row_token] += row_gate * O with 16-byte fp32 vector reductions
//                      (fused combine), or O rounded to bf16 (unfused path).
//   TMEM holds two 256-column accumulators (512 columns), so the epilogue of one work item
//   overlaps the MMAs of the next.
// Work items: item L -> m-tile L / n_n, n-tile L % n_n, handed out in increasing L by a
// global atomic counter (the producer thread draws the next item when it is ready for
// it, so faster SMs take more items) and passed to the MMA and epilogue warps through a
// small shared-memory ring.  All n-tiles of a block are in flight together, and
// consecutive blocks belong to the same expert, so each expert's weights stream from HBM
// about once.  With MOE_FFN_STRICT_SLOTS, CTA c draws from slot (c mod P)'s counter and
// only runs that slot's tiles.
// Every mbarrier wait is bounded (globaltimer); on expiry the kernel sets
// MOE_STATUS_TIMEOUT, lets the other roles drop out, waits (bounded) for its own copies
// and MMAs in flight, frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <mutex>

#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int BM = 128;   // rows per tile (M)
constexpr int BK = 64;    // K per stage: 64 bf16 = 128 bytes = one swizzle span
constexpr int BN = 256;   // MMA N (FC1: 128 G + 128 U columns; FC2: 256 output columns)
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 2 * BN;
constexpr int RING = 8;   // work items in flight between the producer and the consumers
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 512;  // + alignment slack, barriers
constexpr unsigned long long kTimeoutNs = 2000000000ull;  // 2 s per wait

// kind::f16 instruction descriptor: D fp32 (bits 4-5 = 1), A bf16 (bits 7-9 = 1),
// B bf16 (bits 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 at bit 17, M >> 4 at 24.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                            ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

struct FfnArgs {
  int32_t* sched;           // this launch's counters: [0] or [slot] (strict), zeroed
  const int32_t* tiles;
  const int32_t* plan_info;
  const int32_t* row_token;
  const float* row_gate;
  void* out;
  int32_t* status;
  long long r_max;
  int T, d, f, E, P;
  int n_k;       // K steps of 64
  int n_n;       // n-tiles per m-tile
  int out_ld;    // output row length (elements)
  int write_o;   // FC2: store O (1) or fused combine (0)
  int strict;
  unsigned long long timeout_ns;
};

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; "
      "selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait for the phase of `parity` to complete.  Returns false if another role
// raised `abort_flag` (when honour_abort) or if the wait ran out (then raises it).
__device__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                          int32_t* status, unsigned long long timeout_ns, bool honour_abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((spin & 31u) == 0) {
      if (honour_abort && *abort_flag) return false;
      if (globaltimer() - t0 > timeout_ns) {
        *abort_flag = 1;
        set_status(status, MOE_STATUS_TIMEOUT);
        return false;
      }
    }
  }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}
// Shared-memory matrix descriptor of a K-major tile written by TMA with the 128-byte
// swizzle: start address >> 4 (bits 0-13), leading offset unused for this layout (1),
// stride offset = 1024 bytes between 8-row groups (bits 32-45), descriptor version 1
// (bit 46), swizzle mode 2 = 128-byte (bits 61-63).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(kIdesc), "r"(accumulate));
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float silu(float g) { return g / (1.0f + __expf(-g)); }

// ------------------------------------------------------------------ work schedule
struct Sched {
  int32_t* counter;   // global counter this CTA draws items from
  long long total;    // items in its range
  int m_base, n_n;
  __device__ void decode(int L, int& m, int& n) const {
    m = m_base + L / n_n;
    n = L % n_n;
  }
};

__device__ Sched make_sched(const FfnArgs& a) {
  Sched s;
  s.n_n = a.n_n;
  const int* pi = a.plan_info;
  if (!a.strict) {
    s.counter = a.sched;
    s.total = (long long)max(pi[MOE_PI_NTILES], 0) * a.n_n;
    s.m_base = 0;
  } else {
    const int r = blockIdx.x % a.P;
    const int lo = pi[MOE_PI_SLOT_TILE_OFF + r], hi = pi[MOE_PI_SLOT_TILE_OFF + r + 1];
    s.counter = a.sched + r;
    s.total = (long long)max(hi - lo, 0) * a.n_n;
    s.m_base = lo;
  }
  return s;
}

struct TileInfo {
  int e, row0, nrows;
  bool ok;
};
__device__ __forceinline__ TileInfo read_tile(const FfnArgs& a, int m) {
  TileInfo t;
  const int4 v = __ldg(reinterpret_cast<const int4*>(a.tiles) + m);
  t.e = v.x;
  t.row0 = v.y;
  t.nrows = v.z;
  t.ok = v.x >= 0 && v.x < a.E && v.y >= 0 && (long long)v.y < a.r_max && v.z > 0 && v.z <= BM;
  return t;
}

// ------------------------------------------------------------------ the kernel
template <int PHASE>  // 1: FC1 + SwiGLU, 2: FC2 (+ combine)
__global__ void __launch_bounds__(THREADS, 1)
ffn_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const FfnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  // bars: full[STAGES], empty[STAGES], tmem_full[2], tmem_empty[2], drain,
  //       item_full[RING], item_empty[RING]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5 + 2 * RING);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ring = reinterpret_cast<volatile int*>(tmem_slot + 2);  // [RING] items

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  auto tfull_bar = [&](int b) { return smem_u32(bars + 2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return smem_u32(bars + 2 * STAGES + 2 + b); };
  const uint32_t drain_bar = smem_u32(bars + 2 * STAGES + 4);
  auto ifull_bar = [&](int i) { return smem_u32(bars + 2 * STAGES + 5 + i); };
  auto iempty_bar = [&](int i) { return smem_u32(bars + 2 * STAGES + 5 + RING + i); };
  auto sA = [&](int s) { return smem_u32(smem + s * STAGE_BYTES); };
  auto sB = [&](int s) { return smem_u32(smem + s * STAGE_BYTES + A_BYTES); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 4 * 32);
    }
    mbar_init(drain_bar, 1);
    for (int i = 0; i < RING; ++i) {
      mbar_init(ifull_bar(i), 1);
      mbar_init(iempty_bar(i), 1 + 4);  // the MMA thread and the four epilogue warps
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const Sched sch = make_sched(a);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t pending = 0, pend_parity = 0;
      bool bad_tile = false;
      for (int it = 0;; ++it) {
        const int slot = it % RING;
        const uint32_t ph = (uint32_t)(it / RING) & 1u;
        if (!mbar_wait(iempty_bar(slot), ph ^ 1u, abort_flag, a.status, a.timeout_ns, true))
          break;
        const long long L = atomicAdd(sch.counter, 1);
        ring[slot] = L < sch.total ? (int)L : -1;
        mbar_arrive(ifull_bar(slot));
        if (L >= sch.total) break;
        int m, n;
        sch.decode((int)L, m, n);
        const TileInfo ti = read_tile(a, m);
        if (!ti.ok) {
          bad_tile = true;
          continue;
        }
        const int brow = PHASE == 1 ? ti.e * 2 * a.f + n * (BN / 2) : ti.e * a.d + n * BN;
        bool stop = false;
        for (int kb = 0; kb < a.n_k; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.status, a.timeout_ns, true)) {
            stop = true;
            break;
          }
          mbar_expect_tx(full_bar(stage), STAGE_BYTES);
          tma_load_2d(sA(stage), &tmA, full_bar(stage), kb * BK, ti.row0);
          if (PHASE == 1) {
            tma_load_2d(sB(stage), &tmB, full_bar(stage), kb * BK, brow);
            tma_load_2d(sB(stage) + B_BYTES / 2, &tmB, full_bar(stage), kb * BK, brow + a.f);
          } else {
            tma_load_2d(sB(stage), &tmB, full_bar(stage), kb * BK, brow);
          }
          pending |= 1u << stage;
          pend_parity = (pend_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (stop) break;
      }
      if (bad_tile) set_status(a.status, MOE_STATUS_PLAN);
      if (*abort_flag) {
        // let the copies already issued land before the CTA's shared memory goes away
        for (int s = 0; s < STAGES; ++s)
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
        const int slot = it % RING;
        const uint32_t ph = (uint32_t)(it / RING) & 1u;
        if (!mbar_wait(ifull_bar(slot), ph, abort_flag, a.status, a.timeout_ns, true)) break;
        const int L = ring[slot];
        mbar_arrive(iempty_bar(slot));
        if (L < 0) break;
        int m, n;
        sch.decode(L, m, n);
        const TileInfo ti = read_tile(a, m);
        if (!ti.ok) continue;
        const int buf = acc_it & 1;
        const uint32_t use = (uint32_t)(acc_it >> 1) & 1u;
        if (!mbar_wait(tempty_bar(buf), use ^ 1u, abort_flag, a.status, a.timeout_ns, true)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        bool stop = false;
        for (int kb = 0; kb < a.n_k; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, a.status, a.timeout_ns, true)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = sA(stage), b0 = sB(stage);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            umma_bf16(d_tmem, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32),
                      (kb | kk) != 0);
          }
          issued = true;
          umma_commit(empty_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (stop) break;
        umma_commit(tfull_bar(buf));
        ++acc_it;
      }
      if (issued) {
        // every MMA this thread issued has completed once the drain barrier fires
        umma_commit(drain_bar);
        mbar_wait(drain_bar, 0, abort_flag, a.status, a.timeout_ns, false);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;  // TMEM lanes this warp may read: 32*quarter ..
    const int rit = quarter * 32 + lane;  // row inside the tile
    int acc_it = 0;
    for (int it = 0;; ++it) {
      const int slot = it % RING;
      const uint32_t ph = (uint32_t)(it / RING) & 1u;
      const bool have =
          mbar_wait(ifull_bar(slot), ph, abort_flag, a.status, a.timeout_ns, true);
      if (!__all_sync(0xffffffffu, have)) break;
      const int L = ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(iempty_bar(slot));
      if (L < 0) break;
      int m, n;
      sch.decode(L, m, n);
      const TileInfo ti = read_tile(a, m);
      if (!ti.ok) continue;
      const int buf = acc_it & 1;
      const uint32_t use = (uint32_t)(acc_it >> 1) & 1u;
      const bool got =
          mbar_wait(tfull_bar(buf), use, abort_flag, a.status, a.timeout_ns, true);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const long long row = (long long)ti.row0 + rit;
      const bool valid = rit < ti.nrows && row < a.r_max;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
      if (PHASE == 1) {
        __nv_bfloat16* A = reinterpret_cast<__nv_bfloat16*>(a.out);
        uint4* dst = reinterpret_cast<uint4*>(A + row * a.out_ld + n * (BN / 2));
#pragma unroll 1
        for (int c = 0; c < (BN / 2) / 32; ++c) {
          uint32_t g[32], u[32];
          tmem_ld32(taddr + c * 32, g);
          tmem_ld32(taddr + BN / 2 + c * 32, u);
          tmem_wait_ld();
          uint32_t p[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a0 = silu(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
            const float a1 = silu(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
            p[i] = pack_bf16(a0, a1);
          }
          if (valid) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[c * 4 + i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
          }
        }
      } else if (a.write_o) {
        __nv_bfloat16* O = reinterpret_cast<__nv_bfloat16*>(a.out);
        uint4* dst = reinterpret_cast<uint4*>(O + row * a.out_ld + n * BN);
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
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
        int tok = -1;
        float gate = 0.f;
        if (valid) {
          tok = __ldg(a.row_token + row);
          gate = __ldg(a.row_gate + row);
          if (tok >= a.T) tok = -1;
        }
        float* y = reinterpret_cast<float*>(a.out) + (long long)(tok < 0 ? 0 : tok) * a.out_ld +
                   n * BN;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_wait_ld();
          if (tok >= 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              red_add_v4(y + c * 32 + 4 * i, gate * __uint_as_float(v[4 * i]),
                         gate * __uint_as_float(v[4 * i + 1]),
                         gate * __uint_as_float(v[4 * i + 2]),
                         gate * __uint_as_float(v[4 * i + 3]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(buf));
      ++acc_it;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS));
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor [outer, inner] (inner contiguous), box [box_outer, 64], 128-byte swizzle.
bool encode_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
               uint32_t box_outer) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_ffn(const moe_cfg& c, const uint16_t* xp, const uint16_t* w1,
                       const uint16_t* w2, const int32_t* tiles, const int32_t* plan_info,
                       const int32_t* row_token, const float* row_gate, int mode,
                       uint16_t* a_scratch, void* out, int32_t* status, cudaStream_t st) {
  const bool write_o = (mode & MOE_FFN_WRITE_O) != 0;
  const long long r_max = max_rows(c);
  cudaError_t err;
  if (!write_o && c.T > 0) {
    err = cudaMemsetAsync(out, 0, sizeof(float) * (size_t)c.T * c.d, st);
    if (err != cudaSuccess) return err;
  }
  if (r_max == 0) return cudaSuccess;

  // scheduler counters after A in the scratch buffer: [0, 8) FC1, [8, 16) FC2
  int32_t* sched = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(a_scratch) +
                                              ffn_a_bytes(c));
  err = cudaMemsetAsync(sched, 0, 16 * sizeof(int32_t), st);
  if (err != cudaSuccess) return err;

  CUtensorMap tm_xp, tm_w1, tm_a, tm_w2;
  if (!encode_2d(&tm_xp, xp, c.d, r_max, BM) ||
      !encode_2d(&tm_w1, w1, c.d, (uint64_t)c.E * 2 * c.f, BN / 2) ||
      !encode_2d(&tm_a, a_scratch, c.f, r_max, BM) ||
      !encode_2d(&tm_w2, w2, c.f, (uint64_t)c.E * c.d, BN))
    return cudaErrorInvalidValue;

  err = cudaFuncSetAttribute(ffn_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(ffn_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES);
  if (err != cudaSuccess) return err;

  const int grid = num_sms();
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
  a1.strict = (mode & MOE_FFN_STRICT_SLOTS) && grid >= c.P;
  a1.timeout_ns = kTimeoutNs;

  FfnArgs a2 = a1;
  a1.sched = sched;
  a2.sched = sched + 8;
  a1.out = a_scratch;
  a1.n_k = c.d / BK;
  a1.n_n = c.f / (BN / 2);
  a1.out_ld = c.f;
  a1.write_o = 0;
  ffn_kernel<1><<<grid, THREADS, SMEM_BYTES, st>>>(tm_xp, tm_w1, a1);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;

  a2.out = out;
  a2.n_k = c.f / BK;
  a2.n_n = c.d / BN;
  a2.out_ld = c.d;
  a2.write_o = write_o;
  ffn_kernel<2><<<grid, THREADS, SMEM_BYTES, st>>>(tm_a, tm_w2, a2);
  return cudaGetLastError();
}

}  // namespace moe
