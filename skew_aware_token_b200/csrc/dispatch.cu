// Tile-aligned dispatch: a stable counting sort of the routed (t, j) pairs by expert, then
// a gather of the token rows into the padded, block-aligned activation matrix Xp.
//
// "MegaFlux" summary, Methodology 1 "Problem Formulation": each expert's routed rows are
// cut into blocks of at most beta rows matching the kernel tile; the Summary and
// "Theoretical Contributions" 1: token counts, expert selections and routing weights are
// preserved (every pair lands on exactly one row, with its own gate).
//
// Pass 1 (rank): one CTA per expert scans the flattened topk_ids in pair order
// i = t*k + j, sixteen consecutive ids per thread per pass (16-byte loads), and ranks its
// matches with a warp-shuffle scan plus a CTA scan of the 32 warp totals; the running
// total carries the order across passes, so ranks follow the pair order (stable).  It writes row_token,
// row_gate and tok_row, then marks the expert's padding rows.
// Pass 2 (gather): one warp per padded row copies x[row_token] (or zeros) with 16-byte
// vector loads (eight in flight per lane) and stores; the grid strides over the rows of
// the plan (read on device).  Skipped when the caller passes no Xp: the expert FFN can
// gather the rows itself.
#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kRankThreads = 1024;
constexpr int kIdsPerThread = 16;  // consecutive pairs ranked by one thread per pass
constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = 8;   // 16-byte loads in flight per lane before the stores
constexpr unsigned kFull = 0xffffffffu;

__global__ void __launch_bounds__(kRankThreads)
dispatch_rank_kernel(const int32_t* __restrict__ ids, const float* __restrict__ gates,
                     const int32_t* __restrict__ block_off, int N, int k, int E, int beta,
                     long long r_max, int32_t* __restrict__ row_token,
                     float* __restrict__ row_gate, int32_t* __restrict__ tok_row,
                     int32_t* __restrict__ status) {
  __shared__ int warp_tot[32];
  const int e = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long base = (long long)beta * block_off[e];
  // rows this expert may fill: its blocks, clipped to the caller's buffers
  long long cap = (long long)beta * (block_off[e + 1] - block_off[e]);
  if (base < 0 || base > r_max) cap = 0;
  else if (base + cap > r_max) cap = r_max - base;
  long long running = 0;
  bool overflow = false, bad = false;
  for (int chunk = 0; chunk < N; chunk += kIdsPerThread * kRankThreads) {
    const int i0 = chunk + kIdsPerThread * threadIdx.x;
    int id[kIdsPerThread];
    if (i0 + kIdsPerThread <= N) {
#pragma unroll
      for (int q = 0; q < kIdsPerThread / 4; ++q) {
        const int4 v = __ldg(reinterpret_cast<const int4*>(ids + i0) + q);
        id[4 * q] = v.x; id[4 * q + 1] = v.y; id[4 * q + 2] = v.z; id[4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < kIdsPerThread; ++j) id[j] = i0 + j < N ? __ldg(ids + i0 + j) : -1;
    }
    uint32_t match = 0;
#pragma unroll
    for (int j = 0; j < kIdsPerThread; ++j) {
      match |= (uint32_t)(id[j] == e) << j;
      if (blockIdx.x == 0 && i0 + j < N && (id[j] < 0 || id[j] >= E)) bad = true;
    }
    const int cnt = __popc(match);
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = warp_tot[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(kFull, w, off);
        if (lane >= off) w += y;
      }
      warp_tot[lane] = w;
    }
    __syncthreads();
    long long pos = running + (warp ? warp_tot[warp - 1] : 0) + incl - cnt;
    const int total = warp_tot[31];
    while (match) {
      const int j = __ffs(match) - 1;
      match &= match - 1;
      const int i = i0 + j;
      if (pos < cap) {
        const long long row = base + pos;
        row_token[row] = i / k;
        row_gate[row] = __ldg(gates + i);
        tok_row[i] = (int32_t)row;
      } else {
        overflow = true;
      }
      ++pos;
    }
    running += total;
    __syncthreads();  // warp_tot is rewritten by the next pass
  }
  for (long long i = running + threadIdx.x; i < cap; i += blockDim.x) {
    row_token[base + i] = -1;
    row_gate[base + i] = 0.f;
  }
  if (overflow) set_status(status, MOE_STATUS_OVERFLOW);
  if (bad) set_status(status, MOE_STATUS_BAD_ID);
}

__global__ void __launch_bounds__(kGatherThreads)
dispatch_gather_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ row_token,
                       const int32_t* __restrict__ block_off, int E, int beta, int T,
                       long long r_max, int d8, uint4* __restrict__ xp) {
  const long long R = min((long long)beta * block_off[E], r_max);
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < R;
       r += warps) {
    const int t = row_token[r];
    uint4* dst = xp + r * d8;
    const bool copy = t >= 0 && t < T;
    const uint4* src = x + (long long)(copy ? t : 0) * d8;
    for (int c0 = lane; c0 < d8; c0 += 32 * kGatherUnroll) {
      uint4 v[kGatherUnroll];
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int c = c0 + 32 * u;
        v[u] = (copy && c < d8) ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int c = c0 + 32 * u;
        if (c < d8) dst[c] = v[u];
      }
    }
  }
}

}  // namespace

cudaError_t launch_dispatch(const moe_cfg& c, const uint16_t* x, const int32_t* ids,
                            const float* gates, const int32_t* block_off, uint16_t* xp,
                            int32_t* row_token, float* row_gate, int32_t* tok_row,
                            int32_t* status, cudaStream_t st) {
  const int N = c.T * c.k;
  if (N == 0) return cudaSuccess;
  dispatch_rank_kernel<<<c.E, kRankThreads, 0, st>>>(ids, gates, block_off, N, c.k, c.E,
                                                     c.beta, max_rows(c), row_token,
                                                     row_gate, tok_row, status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess || xp == nullptr) return err;
  const int grid = num_sms() * 8;
  dispatch_gather_kernel<<<grid, kGatherThreads, 0, st>>>(
      reinterpret_cast<const uint4*>(x), row_token, block_off, c.E, c.beta, c.T,
      max_rows(c), c.d / 8, reinterpret_cast<uint4*>(xp));
  return cudaGetLastError();
}

}  // namespace moe
