// Backward of the grouped SwiGLU expert FFN on the sm_100a tensor cores: the dispatch of the
// output gradient, the launch sequence of the four gradient products, and the tile-half
// kernels for the two products whose N is f (dA and dW2) when f is not a multiple of 256.
// Every other product runs on the whole-tile kernels of ffn_bwd_wide.cu.
//
// "MegaFlux" summary, Methodology 2, backward gradients, with this library's weight layouts
// w1 [E, 2f, d] and w2 [E, d, f] (each of the pages' products is taken with that transpose):
//   D   = row_gate * dy[row_token]                 moe_dispatch_grad (bf16, zero padding)
//   dA  = D w2_e; dZ = [dA U SiLU'(G), dA SiLU(G)]  kind DGRAD_A: GEMM + SwiGLU backward
//   dX  = dZ w1_e; dx[row_token] += dX              kind DGRAD_X (whole tiles only)
//   dW2_e = D^T A                                   kind WGRAD_2: per expert, K = its rows
//   dW1_e = dZ^T Xp                                 kind WGRAD_1 (whole tiles only)
// Backward item 3 requantizes D and dZ: both are stored bf16 and enter the products so.
//
// Operand layouts.  K-major operands (D and dZ as A of the DGrad kinds) are copied as in
// the forward: boxes of 64 K (128 bytes) x 128 rows, 128-byte swizzle.  MN-major operands
// (the weights as B of the DGrad kinds, and both operands of the WGrad kinds, whose K is
// the token rows) are copied in boxes of 64 MN elements (128 bytes) x 64 K rows, box j of
// a stage 8 KB after box j-1; their MMA descriptors describe the MN-major swizzled layout:
// leading offset 8 KB (between 64-element MN chunks), stride offset 1 KB (between 8-row K
// groups), and a K step of 16 advances 2 KB.  The instruction descriptor marks such an
// operand MN-major (bit 15 for A, bit 16 for B).
//
// Roles (192 threads, one CTA per SM, persistent), scheduling and bounded waits are those
// of the forward kernels: warp 0 issues the TMA copies, one thread of warp 1 the MMAs into
// two TMEM accumulators, warps 2..5 drain them; work items come from a global counter in
// increasing order through a ring in shared memory.  DGrad items are (128-row half of a
// planner tile, n-tile), so each expert's weights stream about once; WGrad items are
// (expert, m-tile, n-tile) with the expert's padded rows as K (an idle expert's items just
// write zeros).
#include "tc_util.cuh"

namespace moe {
namespace {

constexpr int kBM = 128, kBK = 64;
constexpr int kThreads = 192;
constexpr int kRing = 8;
constexpr int kStgStride = 36;
constexpr int kMetaBytes = 2048;
constexpr unsigned long long kWaitNs = 2000000000ull;

enum Kind { DGRAD_A = 1, DGRAD_X = 2, WGRAD_2 = 3, WGRAD_1 = 4 };

template <int KIND, int BN>
struct BGeo {
  static constexpr bool A_MN = KIND == WGRAD_2 || KIND == WGRAD_1;  // A read MN-major
  static constexpr bool B_MN = true;                                // B always MN-major
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = STAGE_BYTES <= 32 * 1024 ? 6 : 4;
  static constexpr int STG = 4 * 32 * kStgStride * 4;  // epilogue staging, 32 x 32 per warp
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int NBARS = 2 * STAGES + 5 + 2 * kRing;
  static constexpr int SMEM = STAGES * STAGE_BYTES + STG + kMetaBytes + 1024;
  // kind::f16: D fp32, A and B bf16, A / B major bits, N >> 3 at bit 17, M >> 4 at bit 24
  static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) |
                                    ((A_MN ? 1u : 0u) << 15) | ((B_MN ? 1u : 0u) << 16) |
                                    ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
};
static_assert(BGeo<DGRAD_A, 128>::SMEM <= 227 * 1024 && BGeo<WGRAD_2, 128>::SMEM <= 227 * 1024,
              "smem");
static_assert(BGeo<DGRAD_A, 128>::NBARS * 8 + 4 * (2 + kRing) + 4 * 128 <= kMetaBytes, "meta");

struct BwdArgs {
  int32_t* sched;  // this launch's work counter (zeroed by the launcher)
  const int32_t* tiles;
  const int32_t* plan_info;
  const int32_t* block_off;
  const int32_t* row_token;
  const uint16_t* z;  // DGRAD_A: saved Z = [G, U] bf16 [r_max, 2f]
  uint16_t* dz;       // DGRAD_A: dZ bf16 [r_max, 2f]
  float* dw;          // WGRAD: dW2 [E, d, f] or dW1 [E, 2f, d]
  int32_t* status;
  long long r_max;
  int T, d, f, E, beta;
  int n_k;        // DGrad: K steps of 64
  int n_n;        // n-tiles (N / BN)
  int n_m;        // WGrad: m-tiles per expert (M / 128)
  int n_out;      // WGrad: row length of dW (N); DGrad: unused
  int k_rows;     // DGrad: first B row of expert e is e * k_rows (d for w2, 2f for w1)
  unsigned long long timeout_ns;
};


struct BItem {
  bool run;    // work to do (a DGrad half with rows, or any WGrad item)
  bool zero;   // WGrad item of an idle expert: no K, the output tile is zero
  bool ok;     // a well-formed tile
  int e, row0, nrows, nk, m0, n0;
};

template <int KIND, int BN>
__device__ __forceinline__ BItem decode_item(const BwdArgs& a, int L) {
  BItem it;
  const int n = L % a.n_n;
  const int t = L / a.n_n;
  it.n0 = n * BN;
  if (KIND == DGRAD_A || KIND == DGRAD_X) {
    const int m = t >> 1, half = t & 1;
    const int4 v = __ldg(reinterpret_cast<const int4*>(a.tiles) + m);
    it.e = v.x;
    it.ok = v.x >= 0 && v.x < a.E && v.y >= 0 && (long long)v.y < a.r_max && v.z > 0 &&
            v.z <= 2 * kBM;
    it.row0 = v.y + kBM * half;
    it.nrows = min(v.z - kBM * half, kBM);
    it.run = it.ok && it.nrows > 0;
    it.zero = false;
    it.nk = a.n_k;
    it.m0 = 0;
  } else {
    it.e = t / a.n_m;
    it.m0 = (t % a.n_m) * kBM;
    const int b0 = __ldg(a.block_off + it.e), b1 = __ldg(a.block_off + it.e + 1);
    it.row0 = a.beta * b0;
    it.nrows = a.beta * (b1 - b0);
    it.ok = b0 >= 0 && b1 >= b0 && (long long)a.beta * b1 <= a.r_max;
    it.nk = it.ok ? it.nrows / kBK : 0;
    it.run = true;
    it.zero = it.nk == 0;
  }
  return it;
}

template <int KIND, int BN>
__global__ void __launch_bounds__(kThreads, 1)
bwd_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const BwdArgs a) {
  using G = BGeo<KIND, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* stg = reinterpret_cast<float*>(smem + G::STAGES * G::STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G::STAGES * G::STAGE_BYTES + G::STG);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + G::NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ring = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + G::STAGES + s); };
  auto tfull_bar = [&](int b) { return smem_u32(bars + 2 * G::STAGES + b); };
  auto tempty_bar = [&](int b) { return smem_u32(bars + 2 * G::STAGES + 2 + b); };
  const uint32_t drain_bar = smem_u32(bars + 2 * G::STAGES + 4);
  auto ifull_bar = [&](int i) { return smem_u32(bars + 2 * G::STAGES + 5 + i); };
  auto iempty_bar = [&](int i) { return smem_u32(bars + 2 * G::STAGES + 5 + kRing + i); };
  auto sA = [&](int s) { return smem_u32(smem + s * G::STAGE_BYTES); };
  auto sB = [&](int s) { return smem_u32(smem + s * G::STAGE_BYTES + G::A_BYTES); };

  long long total;
  if (KIND == DGRAD_A || KIND == DGRAD_X)
    total = (long long)max(a.plan_info[MOE_PI_NTILES], 0) * 2 * a.n_n;
  else
    total = (long long)a.E * a.n_m * a.n_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < G::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 4);
    }
    mbar_init(drain_bar, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(ifull_bar(i), 1);
      mbar_init(iempty_bar(i), 5);  // MMA thread + 4 epilogue warps
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) tmem_alloc<false, G::TMEM_COLS>(smem_u32(tmem_slot));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, pending = 0, pend_parity = 0;
      bool bad = false;
      for (int it = 0;; ++it) {
        const int slot = it % kRing;
        const uint32_t ph = (uint32_t)(it / kRing) & 1u;
        if (!mbar_wait(iempty_bar(slot), ph ^ 1u, abort_flag, a.status, a.timeout_ns, true))
          break;
        const long long v = atomicAdd(a.sched, 1);
        const int L = v < total ? (int)v : -1;
        ring[slot] = L;
        mbar_arrive(ifull_bar(slot));
        if (L < 0) break;
        const BItem w = decode_item<KIND, BN>(a, L);
        if (!w.ok) bad = true;
        if (!w.run || w.zero) continue;
        bool stop = false;
        for (int kb = 0; kb < w.nk; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.status, a.timeout_ns,
                         true)) {
            stop = true;
            break;
          }
          mbar_expect_tx(full_bar(stage), G::STAGE_BYTES);
          const int krow = KIND == DGRAD_A || KIND == DGRAD_X ? w.e * a.k_rows + kb * kBK
                                                              : w.row0 + kb * kBK;
#pragma unroll
          for (int j = 0; j < BN / 64; ++j)
            tma_load_2d(sB(stage) + j * 8192, &tmB, full_bar(stage), w.n0 + 64 * j, krow);
          if (G::A_MN) {
#pragma unroll
            for (int j = 0; j < kBM / 64; ++j)
              tma_load_2d(sA(stage) + j * 8192, &tmA, full_bar(stage), w.m0 + 64 * j, krow);
          } else {
            tma_load_2d(sA(stage), &tmA, full_bar(stage), kb * kBK, w.row0);
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
      if (bad) set_status(a.status, MOE_STATUS_PLAN);
      if (*abort_flag) {
        for (int s = 0; s < G::STAGES; ++s)
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
        const int slot = it % kRing;
        const uint32_t ph = (uint32_t)(it / kRing) & 1u;
        if (!mbar_wait(ifull_bar(slot), ph, abort_flag, a.status, a.timeout_ns, true)) break;
        const int L = ring[slot];
        mbar_arrive(iempty_bar(slot));
        if (L < 0) break;
        const BItem w = decode_item<KIND, BN>(a, L);
        if (!w.run || w.zero) continue;
        const int buf = acc_it & 1;
        const uint32_t use = (uint32_t)(acc_it >> 1) & 1u;
        if (!mbar_wait(tempty_bar(buf), use ^ 1u, abort_flag, a.status, a.timeout_ns, true))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        bool stop = false;
        for (int kb = 0; kb < w.nk; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, a.status, a.timeout_ns, true)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = sA(stage), b0 = sB(stage);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = G::A_MN ? sw128_mn_desc(a0 + kk * 2048) : sw128_desc(a0 + kk * 32);
            const uint64_t bd = sw128_mn_desc(b0 + kk * 2048);
            umma_bf16<false>(d_tmem, ad, bd, G::IDESC, (kb | kk) != 0);
          }
          issued = true;
          umma_commit_all<false>(empty_bar(stage));
          if (++stage == G::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (stop) break;
        umma_commit_all<false>(tfull_bar(buf));
        ++acc_it;
      }
      if (issued) {
        umma_commit_local<false>(drain_bar);
        mbar_wait(drain_bar, 0, abort_flag, a.status, a.timeout_ns, false);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;
    const int ew = warp - 2;
    int acc_it = 0;
    for (int it = 0;; ++it) {
      const int slot = it % kRing;
      const uint32_t ph = (uint32_t)(it / kRing) & 1u;
      const bool have =
          mbar_wait(ifull_bar(slot), ph, abort_flag, a.status, a.timeout_ns, true);
      if (!__all_sync(0xffffffffu, have)) break;
      const int L = ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(iempty_bar(slot));
      if (L < 0) break;
      const BItem w = decode_item<KIND, BN>(a, L);
      if (!w.run) continue;
      if (KIND == WGRAD_2 || KIND == WGRAD_1) {
        if (w.zero) {  // idle expert: its gradient is zero (the warp's 32 rows, coalesced)
          float* out0 =
              a.dw + ((long long)w.e * a.n_m * kBM + w.m0 + quarter * 32) * a.n_out + w.n0;
          const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int r = 0; r < 32; ++r)
            for (int i = lane; i < BN / 4; i += 32)
              reinterpret_cast<float4*>(out0 + (long long)r * a.n_out)[i] = z4;
          continue;
        }
      }
      const int buf = acc_it & 1;
      const uint32_t use = (uint32_t)(acc_it >> 1) & 1u;
      const bool got =
          mbar_wait(tfull_bar(buf), use, abort_flag, a.status, a.timeout_ns, true);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
      if (KIND == DGRAD_A) {
        // dZ = [dA * U * SiLU'(G), dA * SiLU(G)] for the n-tile's BN columns of G and U.
        // Each 32 x 32 chunk of dA goes through shared memory; then lanes 8q..8q+7 take
        // four columns each of one row, so a warp's loads of G and U and stores of dG and
        // dU each cover four whole 64-byte row segments.
        float* my_row = stg + (ew * 32 + lane) * kStgStride;
        const int rq = lane >> 3, cq = 4 * (lane & 7);
        bool rvalid[8];
        long long rrow[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = quarter * 32 + 4 * i + rq;
          rrow[i] = (long long)w.row0 + r;
          rvalid[i] = r < w.nrows && rrow[i] < a.r_max;
        }
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4*>(my_row + 4 * j) =
                make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                            __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
          __syncwarp();
          const int col = w.n0 + 32 * c + cq;
          // all sixteen loads of the chunk in flight at once (rows outside the tile read the
          // tile's first row and store nothing)
          uint2 gzs[8], uzs[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint16_t* zrow = a.z + (rvalid[i] ? rrow[i] : (long long)w.row0) * 2 * a.f;
            gzs[i] = __ldg(reinterpret_cast<const uint2*>(zrow + col));
            uzs[i] = __ldg(reinterpret_cast<const uint2*>(zrow + a.f + col));
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (!rvalid[i]) continue;
            const float4 da = *reinterpret_cast<const float4*>(
                stg + (ew * 32 + 4 * i + rq) * kStgStride + cq);
            const uint2 gz = gzs[i], uz = uzs[i];
            const float2 g01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gz.x));
            const float2 g23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gz.y));
            const float2 u01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uz.x));
            const float2 u23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uz.y));
            const float gs[4] = {g01.x, g01.y, g23.x, g23.y};
            const float us[4] = {u01.x, u01.y, u23.x, u23.y};
            const float ds[4] = {da.x, da.y, da.z, da.w};
            float dg[4], du[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float sg = 1.0f / (1.0f + __expf(-gs[q]));
              dg[q] = ds[q] * us[q] * (sg * (1.0f + gs[q] * (1.0f - sg)));
              du[q] = ds[q] * gs[q] * sg;
            }
            uint16_t* dzrow = a.dz + rrow[i] * 2 * a.f;
            *reinterpret_cast<uint2*>(dzrow + col) =
                make_uint2(pack_bf16(dg[0], dg[1]), pack_bf16(dg[2], dg[3]));
            *reinterpret_cast<uint2*>(dzrow + a.f + col) =
                make_uint2(pack_bf16(du[0], du[1]), pack_bf16(du[2], du[3]));
          }
          __syncwarp();
        }
      } else {
        // WGrad: rows m0 + 32 quarter .. of expert e's gradient, BN fp32 columns; each
        // 32 x 32 chunk goes through shared memory so that one store instruction writes
        // four whole 128-byte row segments
        float* my_row = stg + (ew * 32 + lane) * kStgStride;
        float* out0 = a.dw + ((long long)w.e * a.n_m * kBM + w.m0 + quarter * 32) * a.n_out +
                      w.n0 + 4 * (lane & 7);
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4*>(my_row + 4 * j) =
                make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                            __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = 4 * i + (lane >> 3);
            *reinterpret_cast<float4*>(out0 + (long long)r * a.n_out + 32 * c) =
                *reinterpret_cast<const float4*>(stg + (ew * 32 + r) * kStgStride +
                                                 4 * (lane & 7));
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(buf));
      ++acc_it;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<false, G::TMEM_COLS>(tmem_base);
  }
}

// D[r] = bf16(row_gate[r] * dy[row_token[r]]) on rows of the plan, zero on padding rows:
// one warp per row, 16-byte loads.
__global__ void __launch_bounds__(256)
dispatch_grad_kernel(const float4* __restrict__ dy, const int32_t* __restrict__ row_token,
                     const float* __restrict__ row_gate, const int32_t* __restrict__ plan_info,
                     int beta, int T, long long r_max, int d4, uint2* __restrict__ d_rows,
                     int32_t* __restrict__ status) {
  const long long rows = min((long long)beta * max(plan_info[MOE_PI_B], 0), r_max);
  const int lane = threadIdx.x & 31;
  bool bad = false;
  for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += (long long)gridDim.x * (blockDim.x >> 5)) {
    int t = __ldg(row_token + r);
    const float gt = __ldg(row_gate + r);
    if (t >= T) {
      bad = true;
      t = -1;
    }
    uint2* dst = d_rows + r * d4;
    if (t < 0) {
      for (int i = lane; i < d4; i += 32) dst[i] = make_uint2(0u, 0u);
    } else {
      const float4* src = dy + (long long)t * d4;
      for (int i = lane; i < d4; i += 32) {
        const float4 v = __ldg(src + i);
        dst[i] = make_uint2(pack_bf16(gt * v.x, gt * v.y), pack_bf16(gt * v.z, gt * v.w));
      }
    }
  }
  if (bad) set_status(status, MOE_STATUS_BAD_ID);
}

template <int KIND, int BN>
cudaError_t launch_bwd(const CUtensorMap& ta, const CUtensorMap& tb, const BwdArgs& args,
                       cudaStream_t st) {
  auto kern = bwd_kernel<KIND, BN>;
  static OncePerDevice attr_once;
  cudaError_t err = once_per_device(attr_once, [&](int&) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                BGeo<KIND, BN>::SMEM);
  });
  if (err != cudaSuccess) return err;
  kern<<<num_sms(), kThreads, BGeo<KIND, BN>::SMEM, st>>>(ta, tb, args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dispatch_grad(const moe_cfg& c, const float* dy, const int32_t* row_token,
                                 const float* row_gate, const int32_t* plan_info,
                                 uint16_t* d_rows, int32_t* status, cudaStream_t st) {
  const long long r_max = max_rows(c);
  if (r_max == 0) return cudaSuccess;
  dispatch_grad_kernel<<<num_sms() * 8, 256, 0, st>>>(
      reinterpret_cast<const float4*>(dy), row_token, row_gate, plan_info, c.beta, c.T, r_max,
      c.d / 4, reinterpret_cast<uint2*>(d_rows), status);
  return cudaGetLastError();
}

cudaError_t launch_ffn_backward(const moe_cfg& c, const uint16_t* xp, const uint16_t* w1,
                                const uint16_t* w2, const int32_t* tiles,
                                const int32_t* plan_info, const int32_t* block_off,
                                const int32_t* row_token, const uint16_t* d_rows,
                                const uint16_t* saved, uint16_t* bwd_scratch, float* dx,
                                float* dw1, float* dw2, int32_t* status, cudaStream_t st) {
  const long long r_max = max_rows(c);
  cudaError_t err;
  if (c.T > 0) {
    err = cudaMemsetAsync(dx, 0, sizeof(float) * (size_t)c.T * c.d, st);
    if (err != cudaSuccess) return err;
  }
  if (r_max == 0) {  // no rows: the weight gradients are zero
    err = cudaMemsetAsync(dw1, 0, sizeof(float) * (size_t)c.E * 2 * c.f * c.d, st);
    if (err != cudaSuccess) return err;
    return cudaMemsetAsync(dw2, 0, sizeof(float) * (size_t)c.E * c.d * c.f, st);
  }
  uint16_t* dz = bwd_scratch;
  int32_t* sched = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(bwd_scratch) +
                                              ffn_z_bytes(c));
  err = cudaMemsetAsync(sched, 0, 4 * sizeof(int32_t), st);
  if (err != cudaSuccess) return err;
  const uint16_t* a_saved = saved;
  const uint16_t* z_saved = reinterpret_cast<const uint16_t*>(
      reinterpret_cast<const uint8_t*>(saved) + ffn_scratch_bytes(c));

  // K-major A operands: boxes of 128 rows; MN-major operands: boxes of 64 rows
  CUtensorMap m_d_k, m_w2, m_d_mn, m_a_mn;
  if (!encode_2d(&m_d_k, d_rows, c.d, r_max, kBM) ||
      !encode_2d(&m_w2, w2, c.f, (uint64_t)c.E * c.d, kBK) ||
      !encode_2d(&m_d_mn, d_rows, c.d, r_max, kBK) ||
      !encode_2d(&m_a_mn, a_saved, c.f, r_max, kBK))
    return cudaErrorInvalidValue;

  BwdArgs base{};
  base.tiles = tiles;
  base.plan_info = plan_info;
  base.block_off = block_off;
  base.row_token = row_token;
  base.status = status;
  base.r_max = r_max;
  base.T = c.T;
  base.d = c.d;
  base.f = c.f;
  base.E = c.E;
  base.beta = c.beta;
  base.timeout_ns = kWaitNs;

  // Each product runs on whole 256-row tiles (ffn_bwd_wide.cu) where its shape allows: dX and
  // dW1 always, dA and dW2 when f is a multiple of 256; else on 128-row tile halves (N = 128).
  // dA = D w2 (N = f, K = d) with the SwiGLU backward -> dZ
  if (bwd_wide_supported(c, BWD_DGRAD_A)) {
    err = launch_bwd_wide(c, BWD_DGRAD_A, d_rows, w2, dz, tiles, plan_info, block_off,
                          row_token, z_saved, sched + 0, status, st);
  } else {
    BwdArgs g1 = base;
    g1.sched = sched + 0;
    g1.z = z_saved;
    g1.dz = dz;
    g1.n_k = c.d / kBK;
    g1.k_rows = c.d;
    g1.n_n = c.f / 128;
    err = launch_bwd<DGRAD_A, 128>(m_d_k, m_w2, g1, st);
  }
  if (err != cudaSuccess) return err;
  // dX = dZ w1 (N = d, K = 2f), reduced into dx
  err = launch_bwd_wide(c, BWD_DGRAD_X, dz, w1, dx, tiles, plan_info, block_off, row_token,
                        nullptr, sched + 1, status, st);
  if (err != cudaSuccess) return err;
  // dW2_e [d, f] = D^T A (M = d, N = f, K = the expert's rows)
  if (bwd_wide_supported(c, BWD_WGRAD_2)) {
    err = launch_bwd_wide(c, BWD_WGRAD_2, d_rows, a_saved, dw2, tiles, plan_info, block_off,
                          row_token, nullptr, sched + 2, status, st);
  } else {
    BwdArgs g3 = base;
    g3.sched = sched + 2;
    g3.dw = dw2;
    g3.n_m = c.d / kBM;
    g3.n_out = c.f;
    g3.n_n = c.f / 128;
    err = launch_bwd<WGRAD_2, 128>(m_d_mn, m_a_mn, g3, st);
  }
  if (err != cudaSuccess) return err;
  // dW1_e [2f, d] = dZ^T Xp (M = 2f, N = d, K = the expert's rows)
  return launch_bwd_wide(c, BWD_WGRAD_1, dz, xp, dw1, tiles, plan_info, block_off, row_token,
                         nullptr, sched + 3, status, st);
}

}  // namespace moe
