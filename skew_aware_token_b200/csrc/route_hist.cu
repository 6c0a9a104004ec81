// Router top-k, expert histogram and the skew measure kappa.
//
// "MegaFlux" summary: the router outputs S_t (k experts) and p_{t,e} (gates) of the
// expert-computation equation, and "Routing Skew Problem": c_e and
// kappa = E * sum_e (c_e / sum_j c_j)^2.
//
// One warp ranks a few token rows together.  Lane l holds logits l, l+32, ... of each row
// (coalesced 128-byte loads); k rounds of a warp arg-max (larger value first, ties to the
// lower expert id) pick the top-k in descending order, the rows' shuffle chains
// interleaved.  Lane j keeps the j-th choice; gates are the softmax over the k chosen
// logits, normalised with a warp sum.
// Each CTA counts its tokens' choices in a shared-memory histogram and merges the non-zero
// bins into `counts` with one global atomic each; a one-CTA kernel then forms S and kappa.
#include <cfloat>
#include <climits>

#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kRouteThreads = 256;

// EPL experts per lane = ceil(E / 32); TPW token rows ranked together by one warp, so the
// shuffle chains of different rows interleave.
template <int EPL, int TPW>
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
  for (long long t0 = ((long long)blockIdx.x * warps + (threadIdx.x >> 5)) * TPW; t0 < T;
       t0 += (long long)gridDim.x * warps * TPW) {
    float v[TPW][EPL];
#pragma unroll
    for (int u = 0; u < TPW; ++u) {
      const long long t = t0 + u;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        float x = (t < T && e < E) ? __ldg(logits + t * E + e) : -INFINITY;
        if (t < T && e < E && !isfinite(x)) {
          bad = true;
          if (x != x) x = -INFINITY;  // NaN never wins; the status bit reports it
        }
        v[u][i] = x;
      }
    }
    uint32_t taken[TPW];
    float myv[TPW], top[TPW];  // lane j keeps the j-th choice; top = the largest logit
    int myi[TPW];
#pragma unroll
    for (int u = 0; u < TPW; ++u) {
      taken[u] = 0;
      myv[u] = -INFINITY;
      top[u] = 0.f;
      myi[u] = 0;
    }
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k) {
        float bv[TPW];
        int bi[TPW];
#pragma unroll
        for (int u = 0; u < TPW; ++u) {
          bv[u] = -INFINITY;
          bi[u] = INT_MAX;
#pragma unroll
          for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !(taken[u] >> i & 1u) &&
                (v[u][i] > bv[u] || (v[u][i] == bv[u] && e < bi[u]))) {
              bv[u] = v[u][i];
              bi[u] = e;
            }
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
          for (int u = 0; u < TPW; ++u) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv[u], off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi[u], off);
            if (ov > bv[u] || (ov == bv[u] && oi < bi[u])) {
              bv[u] = ov;
              bi[u] = oi;
            }
          }
        }
#pragma unroll
        for (int u = 0; u < TPW; ++u) {
          if ((bi[u] & 31) == lane) taken[u] |= 1u << (bi[u] >> 5);
          if (lane == j) {
            myv[u] = bv[u];
            myi[u] = bi[u];
          }
          if (j == 0) top[u] = bv[u];
        }
      }
    }
    // gates: softmax over the chosen logits (lanes 0..k-1 hold them, in order)
    float w[TPW], sum[TPW];
#pragma unroll
    for (int u = 0; u < TPW; ++u) {
      w[u] = lane < k ? expf(myv[u] - top[u]) : 0.f;
      sum[u] = w[u];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
      for (int u = 0; u < TPW; ++u) sum[u] += __shfl_xor_sync(0xffffffffu, sum[u], off);
    }
#pragma unroll
    for (int u = 0; u < TPW; ++u) {
      const long long t = t0 + u;
      if (t < T && lane < k) {
        topk_ids[t * k + lane] = myi[u];
        topk_gates[t * k + lane] = w[u] / sum[u];
        atomicAdd(&hist[myi[u]], 1);
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
  constexpr int TPW = EPL <= 4 ? 4 : 2;
  const int rows_per_cta = (kRouteThreads / 32) * TPW;
  long long want = ((long long)c.T + rows_per_cta - 1) / rows_per_cta;
  long long cap = (long long)num_sms() * 4;
  int grid = (int)(want < cap ? want : cap);
  if (grid < 1) grid = 1;
  route_topk_hist_kernel<EPL, TPW><<<grid, kRouteThreads, 0, st>>>(logits, c.T, c.E, c.k,
                                                                    ids, gates, counts,
                                                                    status);
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
