// Shared definitions of the moeskew CUDA library (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include <mutex>

#include "moeskew.h"

namespace moe {

constexpr int kMaxE = 256;
constexpr int kMaxK = 8;
constexpr int kMaxP = 8;
constexpr long long kMaxN = 1LL << 22;
// every flag moe_expert_ffn accepts
constexpr int kFfnModes = MOE_FFN_WRITE_O | MOE_FFN_STRICT_SLOTS | MOE_FFN_SM_PAIR |
                          MOE_FFN_GATHER_X | MOE_FFN_SAVE_Z | MOE_FFN_ONE_LAUNCH |
                          MOE_FFN_TWO_LAUNCHES | MOE_FFN_TEST_WAIT_TIMEOUT |
                          MOE_FFN_FC1_M128 | MOE_FFN_FC2_WHOLE | MOE_FFN_RECORD_SLOTS;
// flags the one-launch FFN does not combine with
constexpr int kOneLaunchExcludes = MOE_FFN_WRITE_O | MOE_FFN_STRICT_SLOTS | MOE_FFN_SM_PAIR |
                                   MOE_FFN_GATHER_X | MOE_FFN_TWO_LAUNCHES;

// Bound on the number of token blocks over every routing of N rows into E experts:
// sum_e ceil(c_e / beta) <= (N + min(E, N) * (beta - 1)) / beta.
inline long long max_blocks(const moe_cfg& c) {
  const long long N = (long long)c.T * c.k;
  const long long nz = N < c.E ? N : c.E;
  return (N + nz * (c.beta - 1)) / c.beta;
}
inline long long max_rows(const moe_cfg& c) { return max_blocks(c) * c.beta; }

// FFN scratch: A (bf16 [R_max, f]) rounded up to 256 bytes, then the tile-scheduler
// counters (kSchedBytes), then the one-launch FFN's readiness counters, then the slot record.
constexpr long long kSchedBytes = 256;
inline long long ffn_a_bytes(const moe_cfg& c) {
  return (max_rows(c) * c.f * 2 + 255) / 256 * 256;
}
// readiness counters of the one-launch FFN: one per (tile, 128-row half), tiles <= B_max
inline long long ffn_ready_bytes(const moe_cfg& c) {
  return (2 * max_blocks(c) * 4 + 255) / 256 * 256;
}
// slot record of MOE_FFN_RECORD_SLOTS: one int32 per execution tile (tiles <= B_max)
inline long long ffn_record_bytes(const moe_cfg& c) {
  return (max_blocks(c) * 4 + 255) / 256 * 256;
}
inline long long ffn_record_offset(const moe_cfg& c) {
  return ffn_a_bytes(c) + kSchedBytes + ffn_ready_bytes(c);
}
inline long long ffn_scratch_bytes(const moe_cfg& c) {
  return ffn_record_offset(c) + ffn_record_bytes(c);
}
// Z = [G, U] (bf16 [R_max, 2f]) or dZ, rounded up to 256 bytes
inline long long ffn_z_bytes(const moe_cfg& c) {
  return (max_rows(c) * 2 * c.f * 2 + 255) / 256 * 256;
}
// with MOE_FFN_SAVE_Z: A, the counters, then Z
inline long long ffn_scratch_z_bytes(const moe_cfg& c) {
  return ffn_scratch_bytes(c) + ffn_z_bytes(c);
}
// backward scratch: dZ, then the counters of its four launches
inline long long bwd_scratch_bytes(const moe_cfg& c) { return ffn_z_bytes(c) + kSchedBytes; }

// Once per device for one call site: `f(int& value)` runs on the first call made with that
// device current, and every later call returns its result (and value).  Used for kernel
// attributes and occupancy queries, so that a launch sequence can be captured into a CUDA
// graph with nothing but stream work inside it.
constexpr int kMaxDevices = 64;
struct OncePerDevice {
  std::mutex m;
  bool done[kMaxDevices] = {};
  cudaError_t err[kMaxDevices] = {};
  int value[kMaxDevices] = {};
};
template <class F>
cudaError_t once_per_device(OncePerDevice& o, F&& f, int* value = nullptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) {
    int v = 0;
    e = f(v);
    if (value) *value = v;
    return e;
  }
  std::lock_guard<std::mutex> lock(o.m);
  if (!o.done[dev]) {
    o.err[dev] = f(o.value[dev]);
    o.done[dev] = true;
  }
  if (value) *value = o.value[dev];
  return o.err[dev];
}

__device__ __forceinline__ void set_status(int32_t* status, int bits) {
  atomicOr(status, bits);
}

// ---- launchers (one per kernel family), called by the C ABI after validation ----
cudaError_t launch_route_hist(const moe_cfg& c, const float* logits, int32_t* ids,
                              float* gates, int32_t* counts, int64_t* sumsq, double* kappa,
                              int32_t* status, cudaStream_t st);
cudaError_t launch_block_offsets(const moe_cfg& c, const int32_t* counts, int32_t* block_off,
                                 cudaStream_t st);
cudaError_t launch_plan(const moe_cfg& c, const int32_t* counts, uint32_t mask,
                        int32_t* block_off, int32_t* q, int32_t* slot_load,
                        int32_t* slot_off, int32_t* blocks, int32_t* tiles,
                        int32_t* plan_info, int32_t* status, cudaStream_t st);
cudaError_t launch_dispatch(const moe_cfg& c, const uint16_t* x, const int32_t* ids,
                            const float* gates, const int32_t* block_off, uint16_t* xp,
                            int32_t* row_token, float* row_gate, int32_t* tok_row,
                            int32_t* status, cudaStream_t st);
cudaError_t launch_ffn(const moe_cfg& c, const uint16_t* xp, const uint16_t* w1,
                       const uint16_t* w2, const int32_t* tiles, const int32_t* plan_info,
                       const int32_t* row_token, const float* row_gate, int mode,
                       uint16_t* a_scratch, void* out, int32_t* status, cudaStream_t st);
// FC1 + SwiGLU on whole 256-row tiles (ffn_wide.cu): the two-launch FFN's FC1 unless the
// mode asks for SM pairs, rows gathered from x, Z kept for the backward, or 128-row halves
bool fc1_wide_supported(int mode);
// y_zero: y (T x d fp32) for the kernel to zero beside FC1's work, or null
cudaError_t launch_fc1_wide(const moe_cfg& c, const uint16_t* xp, const uint16_t* w1,
                            const int32_t* tiles, const int32_t* plan_info, uint16_t* a_out,
                            int32_t* sched, int32_t* status, bool strict, int32_t* slot_rec,
                            float* y_zero, cudaStream_t st);
// FC2 on whole 256-row tiles: the two-launch FFN's FC2 with O rows (unless on SM pairs), and
// with the fused combine when the mode asks for MOE_FFN_FC2_WHOLE
bool fc2_wide_supported(int mode);
cudaError_t launch_fc2_wide(const moe_cfg& c, const uint16_t* a_in, const uint16_t* w2,
                            const int32_t* tiles, const int32_t* plan_info,
                            const int32_t* row_token, const float* row_gate, void* out,
                            bool write_o, int32_t* sched, int32_t* status, bool strict,
                            int32_t* slot_rec, cudaStream_t st);
// n-tiles of 256 output columns per group of FC2's item order (ffn_tcgen05.cu)
int fc2_n_group(const moe_cfg& c);
// execution units of the FFN launches for this mode (SMs, or SM pairs): strict slots need
// at least P of them
int ffn_units(int mode);
cudaError_t launch_combine(const moe_cfg& c, const uint16_t* o, const int32_t* tok_row,
                           const float* gates, float* y, int32_t* status, cudaStream_t st);
cudaError_t launch_dispatch_grad(const moe_cfg& c, const float* dy, const int32_t* row_token,
                                 const float* row_gate, const int32_t* plan_info,
                                 uint16_t* d_rows, int32_t* status, cudaStream_t st);
cudaError_t launch_ffn_backward(const moe_cfg& c, const uint16_t* xp, const uint16_t* w1,
                                const uint16_t* w2, const int32_t* tiles,
                                const int32_t* plan_info, const int32_t* block_off,
                                const int32_t* row_token, const uint16_t* d_rows,
                                const uint16_t* saved, uint16_t* bwd_scratch, float* dx,
                                float* dw1, float* dw2, int32_t* status, cudaStream_t st);
// The four gradient products on whole 256-row tiles (ffn_bwd_wide.cu); kinds as below.
// a_src / b_src: the product's A and B operands, out: dZ (DGRAD_A), dx (DGRAD_X, zeroed by
// the caller), dW2 or dW1 (fp32).
enum BwdKind { BWD_DGRAD_A = 1, BWD_DGRAD_X = 2, BWD_WGRAD_2 = 3, BWD_WGRAD_1 = 4 };
bool bwd_wide_supported(const moe_cfg& c, int kind);
cudaError_t launch_bwd_wide(const moe_cfg& c, int kind, const uint16_t* a_src,
                            const uint16_t* b_src, void* out, const int32_t* tiles,
                            const int32_t* plan_info, const int32_t* block_off,
                            const int32_t* row_token, const uint16_t* z, int32_t* sched,
                            int32_t* status, cudaStream_t st);

int num_sms();

}  // namespace moe
