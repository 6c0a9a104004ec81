// Router top-k, expert histogram and the skew measure kappa.
//
// "MegaFlux" summary: the router outputs S_t (k experts) and p_{t,e} (gates) of the
// expert-computation equation, and "Routing Skew Problem": c_e and
// kappa = E * sum_e (c_e / sum_j c_j)^2.
//
// One warp per token row.  Lane l holds logits l, l+32, ... of the row (coalesced 128-byte
// loads); k rounds of a warp arg-max (larger value first, ties to the lower expert id)
// pick the top-k in descending order.  Gates are the softmax over the k chosen logits.
// Each CTA counts its tokens' choices in a shared-memory histogram and merges the non-zero
// bins into `counts` with one global atomic each; a one-CTA kernel then forms S and kappa.
#include <cfloat>
#include <climits>

#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kRouteThreads = 256;

template <int EPL>  // experts per lane = ceil(E / 32)
__global__ void __launch_bounds__(kRouteThreads)
route_topk_hist_kernel(const float* __restrict__ logits, int T, int E, int k,
                       int32_t* __restrict__ topk_ids, float* __restrict__ topk_gates,
                       int32_t* __restrict__ counts, int32_t* __restrict__ status) {
  __shared__ int32_t hist[kMaxE];
  for (int i = threadIdx.x; i < E; i += blockDim.x) hist[i] = 0;
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  bool bad = false;
  for (long long t = (long long)blockIdx.x * warps + (threadIdx.x >> 5); t < T;
       t += (long long)gridDim.x * warps) {
    const float* row = logits + t * E;
    float v[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      float x = e < E ? __ldg(row + e) : -INFINITY;
      if (e < E && !isfinite(x)) {
        bad = true;
        if (x != x) x = -INFINITY;  // NaN never wins; the status bit reports it
      }
      v[i] = x;
    }
    uint32_t taken = 0;
    float selv[kMaxK];
    int seli[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k) {
        float bv = -INFINITY;
        int bi = INT_MAX;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const int e = lane + 32 * i;
          if (e < E && !(taken >> i & 1u) && (v[i] > bv || (v[i] == bv && e < bi))) {
            bv = v[i];
            bi = e;
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
          if (ov > bv || (ov == bv && oi < bi)) {
            bv = ov;
            bi = oi;
          }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        selv[j] = bv;
        seli[j] = bi;
      }
    }
    // gates: softmax over the chosen logits; selv[0] is the largest
    float w[kMaxK];
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k) {
        w[j] = expf(selv[j] - selv[0]);
        sum += w[j];
      }
    }
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k && lane == j) {
        topk_ids[t * k + j] = seli[j];
        topk_gates[t * k + j] = w[j] / sum;
        atomicAdd(&hist[seli[j]], 1);
      }
    }
  }
  if (bad) set_status(status, MOE_STATUS_NONFINITE);
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x) {
    const int c = hist[i];
    if (c) atomicAdd(&counts[i], c);
  }
}

// S = sum_e c_e^2 and kappa = E * S / N^2 with N = sum_e c_e, both exact integers below
// 2^53 (N <= 2^22, E <= 256), so the fp64 quotient is the correctly rounded value.
__global__ void __launch_bounds__(256)
kappa_kernel(const int32_t* __restrict__ counts, int E, int64_t* __restrict__ sumsq,
             double* __restrict__ kappa) {
  __shared__ long long s_sq[8], s_n[8];
  long long sq = 0, n = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const long long c = counts[e];
    sq += c * c;
    n += c;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    sq += __shfl_xor_sync(0xffffffffu, sq, off);
    n += __shfl_xor_sync(0xffffffffu, n, off);
  }
  if ((threadIdx.x & 31) == 0) {
    s_sq[threadIdx.x >> 5] = sq;
    s_n[threadIdx.x >> 5] = n;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    long long S = 0, N = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
      S += s_sq[w];
      N += s_n[w];
    }
    *sumsq = S;
    *kappa = N == 0 ? 0.0 : (double)((long long)E * S) / (double)(N * N);
  }
}

template <int EPL>
cudaError_t launch_epl(const moe_cfg& c, const float* logits, int32_t* ids, float* gates,
                       int32_t* counts, int32_t* status, cudaStream_t st) {
  const int warps = kRouteThreads / 32;
  long long want = ((long long)c.T + warps - 1) / warps;
  // two CTAs per SM: each warp ranks a few rows, and few per-CTA histograms contend on
  // the global counters
  long long cap = (long long)num_sms() * 2;
  int grid = (int)(want < cap ? want : cap);
  if (grid < 1) grid = 1;
  route_topk_hist_kernel<EPL><<<grid, kRouteThreads, 0, st>>>(logits, c.T, c.E, c.k, ids,
                                                               gates, counts, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route_hist(const moe_cfg& c, const float* logits, int32_t* ids,
                              float* gates, int32_t* counts, int64_t* sumsq, double* kappa,
                              int32_t* status, cudaStream_t st) {
  cudaError_t err = cudaMemsetAsync(counts, 0, sizeof(int32_t) * c.E, st);
  if (err != cudaSuccess) return err;
  if (c.T > 0) {
    const int epl = (c.E + 31) / 32;
    switch (epl) {
      case 1: err = launch_epl<1>(c, logits, ids, gates, counts, status, st); break;
      case 2: err = launch_epl<2>(c, logits, ids, gates, counts, status, st); break;
      case 3: err = launch_epl<3>(c, logits, ids, gates, counts, status, st); break;
      case 4: err = launch_epl<4>(c, logits, ids, gates, counts, status, st); break;
      case 5: err = launch_epl<5>(c, logits, ids, gates, counts, status, st); break;
      case 6: err = launch_epl<6>(c, logits, ids, gates, counts, status, st); break;
      case 7: err = launch_epl<7>(c, logits, ids, gates, counts, status, st); break;
      default: err = launch_epl<8>(c, logits, ids, gates, counts, status, st); break;
    }
    if (err != cudaSuccess) return err;
  }
  kappa_kernel<<<1, 256, 0, st>>>(counts, c.E, sumsq, kappa);
  return cudaGetLastError();
}

}  // namespace moe
