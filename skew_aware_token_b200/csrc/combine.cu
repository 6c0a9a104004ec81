// Deterministic gate-weighted combine back to token order.
//
// "MegaFlux" summary, Methodology 2, expert-computation equation:
// y_t = sum_{e in S_t} p_{t,e} O_e[t].  The k terms of a token are added in the order
// j = 0..k-1 in fp32, so the result does not depend on scheduling.
//
// One warp per token; each lane owns 8-column groups of the row (16-byte bf16 loads of
// the k expert rows, two 16-byte fp32 stores), two groups per iteration so that 2k loads
// are in flight per lane before the first add.  O rows are read once, so the loads bypass
// L1 (ld.global.nc.L1::no_allocate).  Rows outside the caller's O buffer are skipped and
// reported (MOE_STATUS_BAD_ID), never read.
#include <cuda_bf16.h>

#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kCombineThreads = 256;
constexpr int kGroups = 2;  // 8-column groups per lane per iteration

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void bf16x8_fma(const uint4 v, float g, float* acc) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __uint_as_float(w[i] << 16);
    const float hi = __uint_as_float(w[i] & 0xffff0000u);
    acc[2 * i] = fmaf(g, lo, acc[2 * i]);
    acc[2 * i + 1] = fmaf(g, hi, acc[2 * i + 1]);
  }
}

__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const uint4* __restrict__ o, const int32_t* __restrict__ tok_row,
               const float* __restrict__ gates, int T, int k, long long r_max, int d8,
               float4* __restrict__ y, int32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  bool bad = false;
  for (long long t = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T;
       t += warps) {
    int rows[kMaxK];
    float g[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k) {
        rows[j] = __ldg(tok_row + t * k + j);
        g[j] = __ldg(gates + t * k + j);
        if (rows[j] < 0 || rows[j] >= r_max) {
          bad = true;
          rows[j] = -1;
        }
      }
    }
    for (int c0 = lane; c0 < d8; c0 += 32 * kGroups) {
      uint4 v[kGroups][kMaxK];
#pragma unroll
      for (int u = 0; u < kGroups; ++u) {
        const int c = c0 + 32 * u;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
          v[u][j] = (j < k && rows[j] >= 0 && c < d8)
                        ? ld_stream(o + (long long)rows[j] * d8 + c)
                        : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kGroups; ++u) {
        const int c = c0 + 32 * u;
        if (c >= d8) break;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
          if (j < k && rows[j] >= 0) bf16x8_fma(v[u][j], g[j], acc);
        float4* dst = y + (t * d8 + c) * 2;
        dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      }
    }
  }
  if (bad) set_status(status, MOE_STATUS_BAD_ID);
}

}  // namespace

cudaError_t launch_combine(const moe_cfg& c, const uint16_t* o, const int32_t* tok_row,
                           const float* gates, float* y, int32_t* status, cudaStream_t st) {
  if (c.T == 0) return cudaSuccess;
  const int warps = kCombineThreads / 32;
  long long want = ((long long)c.T + warps - 1) / warps;
  long long cap = (long long)num_sms() * 8;
  const int grid = (int)(want < cap ? want : cap);
  combine_kernel<<<grid, kCombineThreads, 0, st>>>(
      reinterpret_cast<const uint4*>(o), tok_row, gates, c.T, c.k, max_rows(c), c.d / 8,
      reinterpret_cast<float4*>(y), status);
  return cudaGetLastError();
}

}  // namespace moe
