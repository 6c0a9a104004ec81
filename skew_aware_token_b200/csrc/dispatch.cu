// Tile-aligned dispatch: a stable counting sort of the routed (t, j) pairs by expert, then
// a gather of the token rows into the padded, block-aligned activation matrix Xp.
//
// "MegaFlux" summary, Methodology 1 "Problem Formulation": each expert's routed rows are
// cut into blocks of at most beta rows matching the kernel tile; the Summary and
// "Theoretical Contributions" 1: token counts, expert selections and routing weights are
// preserved (every pair lands on exactly one row, with its own gate).
//
// The sort reads the ids a constant number of times (O(N) work and traffic), in three
// kernels over chunks of kChunk consecutive pairs (pair i = t*k + j; the last chunk also
// takes the remainder, so every chunk holds at least kChunk >= E pairs):
//   count   CTA c counts each expert's pairs in its chunk (shared-memory histogram) and
//           writes the E counts into tok_row[c * kChunk + e], i.e. inside its own chunk's
//           range of tok_row, which nothing else reads or writes before the rank kernel;
//   prefix  one thread per expert turns its column of counts into exclusive prefixes over
//           the chunks, in place;
//   rank    CTA c first reads its prefix row into shared memory, then ranks its pairs: in
//           groups of 32 consecutive pairs a warp finds equal ids with __match_any_sync, a
//           pair's rank is the number of equal ids before it in its group, plus those in the
//           warp's earlier groups (per-warp counts in shared memory), in earlier warps of the
//           pass (exclusive scan over the warps) and in earlier chunks (the prefix row).
//           Ranks therefore follow the pair order (stable).  It writes row_token, row_gate
//           and tok_row (overwriting its own prefix row); the last CTA, which then knows
//           every expert's total, marks the padding rows.
// With one chunk the count and prefix kernels are skipped.
// Pass 2 (gather): one warp per padded row copies x[row_token] (or zeros) with 16-byte
// vector loads (eight in flight per lane) and stores; the grid strides over the rows of
// the plan (read on device).  Skipped when the caller passes no Xp: the expert FFN can
// gather the rows itself.
#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kChunk = 1024;        // pairs per chunk (>= the largest E)
constexpr int kRankThreads = 256;   // 8 warps; one pass = 8 warps x 4 groups x 32 pairs
constexpr int kRankWarps = kRankThreads / 32;
constexpr int kGroupsPerWarp = kChunk / (kRankThreads);  // 4
constexpr int kCountThreads = 256;
constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = 8;   // 16-byte loads in flight per lane before the stores
constexpr unsigned kFull = 0xffffffffu;
static_assert(kChunk >= kMaxE, "a chunk must hold an expert count per expert");
static_assert(kRankWarps * kGroupsPerWarp * 32 == kChunk, "one pass per chunk");

__device__ __forceinline__ void chunk_range(int c, int C, int N, int& i0, int& i1) {
  i0 = c * kChunk;
  i1 = c == C - 1 ? N : i0 + kChunk;
}

__global__ void __launch_bounds__(kCountThreads)
dispatch_count_kernel(const int32_t* __restrict__ ids, int N, int E, int C,
                      int32_t* __restrict__ table, int32_t* __restrict__ status) {
  __shared__ int hist[kMaxE];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  int i0, i1;
  chunk_range(blockIdx.x, C, N, i0, i1);
  bool bad = false;
  for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
    const int id = __ldg(ids + i);
    if (id >= 0 && id < E) atomicAdd(&hist[id], 1);
    else bad = true;
  }
  __syncthreads();
  // this chunk's counts go into its own range of tok_row (kChunk >= E entries)
  for (int e = threadIdx.x; e < E; e += blockDim.x) table[(long long)blockIdx.x * kChunk + e] = hist[e];
  if (bad) set_status(status, MOE_STATUS_BAD_ID);
}

__global__ void dispatch_prefix_kernel(int32_t* __restrict__ table, int E, int C) {
  constexpr int kBatch = 8;  // chunk counts loaded ahead of the running sum
  const int e = threadIdx.x;
  if (e >= E) return;
  int run = 0;
  for (int c0 = 0; c0 < C; c0 += kBatch) {
    int v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      v[u] = c0 + u < C ? table[(long long)(c0 + u) * kChunk + e] : 0;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (c0 + u < C) table[(long long)(c0 + u) * kChunk + e] = run;
      run += v[u];
    }
  }
}

__global__ void __launch_bounds__(kRankThreads)
dispatch_rank_kernel(const int32_t* __restrict__ ids, const float* __restrict__ gates,
                     const int32_t* __restrict__ block_off, int N, int k, int E, int beta,
                     int C, long long r_max, int32_t* __restrict__ row_token,
                     float* __restrict__ row_gate, int32_t* __restrict__ tok_row,
                     int32_t* __restrict__ status) {
  __shared__ int run[kMaxE];                 // pairs of each expert before the current pass
  __shared__ int hist[kRankWarps][kMaxE];    // per-warp counts of the pass, then offsets
  __shared__ long long base[kMaxE], cap[kMaxE];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    run[e] = C > 1 ? tok_row[(long long)c * kChunk + e] : 0;
    // rows this expert may fill: its blocks, clipped to the caller's buffers
    const long long b = (long long)beta * block_off[e];
    long long cp = (long long)beta * (block_off[e + 1] - block_off[e]);
    if (b < 0 || b > r_max) cp = 0;
    else if (b + cp > r_max) cp = r_max - b;
    base[e] = b;
    cap[e] = cp;
  }
  __syncthreads();  // the prefix row is read before this CTA overwrites its tok_row range
  int i0, i1;
  chunk_range(c, C, N, i0, i1);
  bool overflow = false, bad = false;
  const unsigned lt = (1u << lane) - 1u;
  for (int p0 = i0; p0 < i1; p0 += kChunk) {
    for (int e = lane; e < E; e += 32) hist[warp][e] = 0;
    __syncwarp();
    int my_e[kGroupsPerWarp], my_r[kGroupsPerWarp];
#pragma unroll
    for (int j = 0; j < kGroupsPerWarp; ++j) {
      const int i = p0 + (warp * kGroupsPerWarp + j) * 32 + lane;
      const int id = i < i1 ? __ldg(ids + i) : -1;
      const bool in = id >= 0 && id < E;
      if (i < i1 && !in) bad = true;
      const unsigned peers = __match_any_sync(kFull, in ? id : -1);
      const int before = in ? hist[warp][id] : 0;
      __syncwarp();
      if (in && (peers & lt) == 0) hist[warp][id] = before + __popc(peers);
      __syncwarp();
      my_e[j] = in ? id : -1;
      my_r[j] = before + __popc(peers & lt);
    }
    __syncthreads();
    // per expert: exclusive offsets over the warps of this pass, on top of earlier passes
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      int r = run[e];
#pragma unroll
      for (int w = 0; w < kRankWarps; ++w) {
        const int v = hist[w][e];
        hist[w][e] = r;
        r += v;
      }
      run[e] = r;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kGroupsPerWarp; ++j) {
      const int e = my_e[j];
      if (e < 0) continue;
      const int i = p0 + (warp * kGroupsPerWarp + j) * 32 + lane;
      const long long pos = (long long)hist[warp][e] + my_r[j];
      if (pos < cap[e]) {
        const long long row = base[e] + pos;
        row_token[row] = i / k;
        row_gate[row] = __ldg(gates + i);
        tok_row[i] = (int32_t)row;
      } else {
        overflow = true;
      }
    }
    __syncthreads();  // hist is rewritten by the next pass
  }
  if (c == C - 1) {
    // every expert's total is now known: one thread per expert marks its padding rows
    // (fewer than beta of them unless the counts and blocks disagree)
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      for (long long r = run[e]; r < cap[e]; ++r) {
        row_token[base[e] + r] = -1;
        row_gate[base[e] + r] = 0.f;
      }
    }
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
  const int C = N / kChunk > 1 ? N / kChunk : 1;  // chunks; the last takes the remainder
  if (C > 1) {
    dispatch_count_kernel<<<C, kCountThreads, 0, st>>>(ids, N, c.E, C, tok_row, status);
    dispatch_prefix_kernel<<<1, (c.E + 31) / 32 * 32, 0, st>>>(tok_row, c.E, C);
  }
  dispatch_rank_kernel<<<C, kRankThreads, 0, st>>>(ids, gates, block_off, N, c.k, c.E, c.beta,
                                                   C, max_rows(c), row_token, row_gate,
                                                   tok_row, status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess || xp == nullptr) return err;
  const int grid = num_sms() * 8;
  dispatch_gather_kernel<<<grid, kGatherThreads, 0, st>>>(
      reinterpret_cast<const uint4*>(x), row_token, block_off, c.E, c.beta, c.T,
      max_rows(c), c.d / 8, reinterpret_cast<uint4*>(xp));
  return cudaGetLastError();
}

}  // namespace moe
