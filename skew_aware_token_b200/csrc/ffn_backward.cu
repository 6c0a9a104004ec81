// Backward of the grouped SwiGLU expert FFN: the dispatch of the output gradient, and the
// launch sequence of the four gradient products, which run on the whole-tile kernels of
// ffn_bwd_wide.cu.
//
// "MegaFlux" summary, Methodology 2, backward gradients, with this library's weight layouts
// w1 [E, 2f, d] and w2 [E, d, f] (each of the pages' products is taken with that transpose):
//   D   = row_gate * dy[row_token]                 moe_dispatch_grad (bf16, zero padding)
//   dA  = D w2_e; dZ = [dA U SiLU'(G), dA SiLU(G)]  GEMM + SwiGLU backward
//   dX  = dZ w1_e; dx[row_token] += dX              GEMM + reduction into dx
//   dW2_e = D^T A                                   per expert, K = its rows
//   dW1_e = dZ^T Xp                                 per expert, K = its rows
// Backward item 3 requantizes D and dZ: both are stored bf16 and enter the products so.
#include "tc_util.cuh"

namespace moe {
namespace {

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
  // dW2_e [d, f] = D^T A (M = d, N = f, K = the expert's rows)
  err = launch_bwd_wide(c, BWD_WGRAD_2, d_rows, a_saved, dw2, tiles, plan_info, block_off,
                        row_token, nullptr, sched + 2, status, st);
  if (err != cudaSuccess) return err;
  // dW1_e [2f, d] = dZ^T Xp (M = 2f, N = d, K = the expert's rows)
  return launch_bwd_wide(c, BWD_WGRAD_1, dz, xp, dw1, tiles, plan_info, block_off, row_token,
                         nullptr, sched + 3, status, st);
}

}  // namespace moe
