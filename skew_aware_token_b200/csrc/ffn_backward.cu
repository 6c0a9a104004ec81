// Backward of the grouped SwiGLU expert FFN on the sm_100a tensor cores: the dispatch of the
// output gradient, the launch sequence of the four gradient products, and a weight-gradient
// kernel on 128-row tiles for dW2 when f is not a multiple of 256.  The products themselves
// run on the whole-tile kernels of ffn_bwd_wide.cu.
//
// "MegaFlux" summary, Methodology 2, backward gradients, with this library's weight layouts
// w1 [E, 2f, d] and w2 [E, d, f] (each of the pages' products is taken with that transpose):
//   D   = row_gate * dy[row_token]                 moe_dispatch_grad (bf16, zero padding)
//   dA  = D w2_e; dZ = [dA U SiLU'(G), dA SiLU(G)]  GEMM + SwiGLU backward
//   dX  = dZ w1_e; dx[row_token] += dX              GEMM + reduction into dx
//   dW2_e = D^T A                                   per expert, K = its rows
//   dW1_e = dZ^T Xp                                 per expert, K = its rows
// Backward item 3 requantizes D and dZ: both are stored bf16 and enter the products so.
//
// The 128-row weight-gradient kernel: items (expert, m-tile of 128 dW2 rows, n-tile of 128
// columns) with the expert's padded rows as K (an idle expert's items just write zeros).
// Both operands are MN-major, copied in boxes of 64 MN elements (128 bytes) x 64 K rows, box
// j of a stage 8 KB after box j-1; their MMA descriptors describe the MN-major swizzled
// layout: leading offset 8 KB (between 64-element MN chunks), stride offset 1 KB (between
// 8-row K groups), and a K step of 16 advances 2 KB; the instruction descriptor marks both
// operands MN-major (bits 15 and 16).  Roles (192 threads, one CTA per SM, persistent): warp
// 0 issues the TMA copies, one thread of warp 1 the MMAs into two TMEM accumulators, warps
// 2..5 drain them; work items come from a global counter in increasing order through a ring
// in shared memory; every wait is bounded.
#include "tc_util.cuh"

namespace moe {
namespace {

constexpr int kBM = 128, kBK = 64;
constexpr int kThreads = 192;
constexpr int kRing = 8;
constexpr int kStgStride = 36;
constexpr int kMetaBytes = 2048;
constexpr unsigned long long kWaitNs = 2000000000ull;

template <int BN>
struct BGeo {
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
                                    (1u << 15) | (1u << 16) |
                                    ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
};
static_assert(BGeo<128>::SMEM <= 227 * 1024, "smem");
static_assert(BGeo<128>::NBARS * 8 + 4 * (2 + kRing) <= kMetaBytes, "meta");

struct BwdArgs {
  int32_t* sched;  // this launch's work counter (zeroed by the launcher)
  const int32_t* block_off;
  float* dw;  // dW2 [E, d, f]
  int32_t* status;
  long long r_max;
  int E, beta;
  int n_n;    // n-tiles (N / BN)
  int n_m;    // m-tiles per expert (M / 128)
  int n_out;  // row length of dW (N)
  unsigned long long timeout_ns;
};


struct BItem {
  bool zero;   // item of an idle expert: no K, the output tile is zero
  bool ok;     // a well-formed tile
  int e, row0, nrows, nk, m0, n0;
};

template <int BN>
__device__ __forceinline__ BItem decode_item(const BwdArgs& a, int L) {
  BItem it;
  const int n = L % a.n_n;
  const int t = L / a.n_n;
  it.n0 = n * BN;
  it.e = t / a.n_m;
  it.m0 = (t % a.n_m) * kBM;
  const int b0 = __ldg(a.block_off + it.e), b1 = __ldg(a.block_off + it.e + 1);
  it.row0 = a.beta * b0;
  it.nrows = a.beta * (b1 - b0);
  it.ok = b0 >= 0 && b1 >= b0 && (long long)a.beta * b1 <= a.r_max;
  it.nk = it.ok ? it.nrows / kBK : 0;
  it.zero = it.nk == 0;
  return it;
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
bwd_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const BwdArgs a) {
  using G = BGeo<BN>;
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

  const long long total = (long long)a.E * a.n_m * a.n_n;

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
        const BItem w = decode_item<BN>(a, L);
        if (!w.ok) bad = true;
        if (w.zero) continue;
        bool stop = false;
        for (int kb = 0; kb < w.nk; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, a.status, a.timeout_ns,
                         true)) {
            stop = true;
            break;
          }
          mbar_expect_tx(full_bar(stage), G::STAGE_BYTES);
          const int krow = w.row0 + kb * kBK;
#pragma unroll
          for (int j = 0; j < BN / 64; ++j)
            tma_load_2d(sB(stage) + j * 8192, &tmB, full_bar(stage), w.n0 + 64 * j, krow);
#pragma unroll
          for (int j = 0; j < kBM / 64; ++j)
            tma_load_2d(sA(stage) + j * 8192, &tmA, full_bar(stage), w.m0 + 64 * j, krow);
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
        const BItem w = decode_item<BN>(a, L);
        if (w.zero) continue;
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
            const uint64_t ad = sw128_mn_desc(a0 + kk * 2048);
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
      const BItem w = decode_item<BN>(a, L);
      if (w.zero) {  // idle expert: its gradient is zero (the warp's 32 rows, coalesced)
        float* out0 =
            a.dw + ((long long)w.e * a.n_m * kBM + w.m0 + quarter * 32) * a.n_out + w.n0;
        const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < 32; ++r)
          for (int i = lane; i < BN / 4; i += 32)
            reinterpret_cast<float4*>(out0 + (long long)r * a.n_out)[i] = z4;
        continue;
      }
      const int buf = acc_it & 1;
      const uint32_t use = (uint32_t)(acc_it >> 1) & 1u;
      const bool got =
          mbar_wait(tfull_bar(buf), use, abort_flag, a.status, a.timeout_ns, true);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
      {
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

template <int BN>
cudaError_t launch_bwd(const CUtensorMap& ta, const CUtensorMap& tb, const BwdArgs& args,
                       cudaStream_t st) {
  auto kern = bwd_kernel<BN>;
  static OncePerDevice attr_once;
  cudaError_t err = once_per_device(attr_once, [&](int&) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                BGeo<BN>::SMEM);
  });
  if (err != cudaSuccess) return err;
  kern<<<num_sms(), kThreads, BGeo<BN>::SMEM, st>>>(ta, tb, args);
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

  // dA = D w2 (N = f, K = d) with the SwiGLU backward -> dZ
  err = launch_bwd_wide(c, BWD_DGRAD_A, d_rows, w2, dz, tiles, plan_info, block_off, row_token,
                        z_saved, sched + 0, status, st);
  if (err != cudaSuccess) return err;
  // dX = dZ w1 (N = d, K = 2f), reduced into dx
  err = launch_bwd_wide(c, BWD_DGRAD_X, dz, w1, dx, tiles, plan_info, block_off, row_token,
                        nullptr, sched + 1, status, st);
  if (err != cudaSuccess) return err;
  // dW2_e [d, f] = D^T A (M = d, N = f, K = the expert's rows): whole tiles when f is a
  // multiple of 256, else the 128-row kernel above (n-tiles of 128)
  if (bwd_wide_supported(c, BWD_WGRAD_2)) {
    err = launch_bwd_wide(c, BWD_WGRAD_2, d_rows, a_saved, dw2, tiles, plan_info, block_off,
                          row_token, nullptr, sched + 2, status, st);
  } else {
    // MN-major operands: boxes of 64 rows
    CUtensorMap m_d_mn, m_a_mn;
    if (!encode_2d(&m_d_mn, d_rows, c.d, r_max, kBK) ||
        !encode_2d(&m_a_mn, a_saved, c.f, r_max, kBK))
      return cudaErrorInvalidValue;
    BwdArgs g3{};
    g3.sched = sched + 2;
    g3.block_off = block_off;
    g3.dw = dw2;
    g3.status = status;
    g3.r_max = r_max;
    g3.E = c.E;
    g3.beta = c.beta;
    g3.n_m = c.d / kBM;
    g3.n_out = c.f;
    g3.n_n = c.f / 128;
    g3.timeout_ns = kWaitNs;
    err = launch_bwd<128>(m_d_mn, m_a_mn, g3, st);
  }
  if (err != cudaSuccess) return err;
  // dW1_e [2f, d] = dZ^T Xp (M = 2f, N = d, K = the expert's rows)
  return launch_bwd_wide(c, BWD_WGRAD_1, dz, xp, dw1, tiles, plan_info, block_off, row_token,
                         nullptr, sched + 3, status, st);
}

}  // namespace moe
