// C ABI of the moeskew library: argument validation, then the stage launchers.
// Nothing is enqueued when validation fails; see include/moeskew.h for the contract.
#include <cstdint>

#include "moe_common.cuh"

namespace moe {

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 1;
  return n > 0 ? n : 1;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Checks shared by every stage.
int check_cfg(const moe_cfg* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->E < 1 || c->k < 1 || c->k > c->E || c->k > kMaxK || c->P < 1 ||
      c->P > kMaxP || c->s < 0 || (c->beta != 64 && c->beta != 128) || c->d < 1 || c->f < 1)
    return MOE_ERR_INVALID_ARG;
  if (c->E > kMaxE || (long long)c->T * c->k > kMaxN) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

int check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps) {
    if (!p) return MOE_ERR_INVALID_ARG;
    if (!aligned16(p)) return MOE_ERR_UNSUPPORTED;
  }
  return MOE_OK;
}

int cuda_result(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_size(const moe_cfg* cfg, int which) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  if (which == MOE_WS_ROWS) return (size_t)max_rows(*cfg);
  if (which == MOE_WS_BLOCKS) return (size_t)max_blocks(*cfg);
  if (which == MOE_WS_FFN_SCRATCH) return (size_t)ffn_scratch_bytes(*cfg);
  if (which == MOE_WS_FFN_SCRATCH_Z) return (size_t)ffn_scratch_z_bytes(*cfg);
  if (which == MOE_WS_BWD_SCRATCH) return (size_t)bwd_scratch_bytes(*cfg);
  if (which == MOE_WS_FFN_RECORD) return (size_t)ffn_record_offset(*cfg);
  return 0;
}

int moe_route_hist(const moe_cfg* cfg, const float* logits, int32_t* topk_ids,
                   float* topk_gates, int32_t* counts, int64_t* sumsq, double* kappa,
                   int32_t* status, moe_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  rc = check_ptrs({logits, topk_ids, topk_gates, counts, sumsq, kappa, status});
  if (rc != MOE_OK) return rc;
  return cuda_result(launch_route_hist(*cfg, logits, topk_ids, topk_gates, counts, sumsq,
                                       kappa, status, (cudaStream_t)stream));
}

int moe_block_offsets(const moe_cfg* cfg, const int32_t* counts, int32_t* block_off,
                      moe_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  rc = check_ptrs({counts, block_off});
  if (rc != MOE_OK) return rc;
  return cuda_result(launch_block_offsets(*cfg, counts, block_off, (cudaStream_t)stream));
}

int moe_plan_blocks(const moe_cfg* cfg, const int32_t* counts, uint32_t variant_mask,
                    int32_t* block_off, int32_t* q, int32_t* slot_load, int32_t* slot_off,
                    int32_t* blocks, int32_t* tiles, int32_t* plan_info, int32_t* status,
                    moe_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  if (variant_mask & ~0xFFFF3Fu) return MOE_ERR_INVALID_ARG;  // variants, C_lambda, u_min, lambda
  rc = check_ptrs({counts, block_off, q, slot_load, slot_off, blocks, tiles, plan_info, status});
  if (rc != MOE_OK) return rc;
  return cuda_result(launch_plan(*cfg, counts, variant_mask, block_off, q, slot_load, slot_off,
                                 blocks, tiles, plan_info, status, (cudaStream_t)stream));
}

int moe_dispatch_permute(const moe_cfg* cfg, const uint16_t* x, const int32_t* topk_ids,
                         const float* topk_gates, const int32_t* block_off, uint16_t* xp,
                         int32_t* row_token, float* row_gate, int32_t* tok_row,
                         int32_t* status, moe_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  if (cfg->d % 8) return MOE_ERR_UNSUPPORTED;
  rc = check_ptrs({x, topk_ids, topk_gates, block_off, row_token, row_gate, tok_row, status});
  if (rc == MOE_OK && xp) rc = check_ptrs({xp});  // NULL: row maps only
  if (rc != MOE_OK) return rc;
  return cuda_result(launch_dispatch(*cfg, x, topk_ids, topk_gates, block_off, xp, row_token,
                                     row_gate, tok_row, status, (cudaStream_t)stream));
}

int moe_expert_ffn(const moe_cfg* cfg, const uint16_t* xp, const uint16_t* w1,
                   const uint16_t* w2, const int32_t* tiles, const int32_t* plan_info,
                   const int32_t* row_token, const float* row_gate, int mode,
                   uint16_t* a_scratch, void* out, int32_t* status, moe_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  if (mode & ~kFfnModes) return MOE_ERR_INVALID_ARG;
  if ((mode & (MOE_FFN_ONE_LAUNCH | MOE_FFN_TEST_WAIT_TIMEOUT)) && (mode & kOneLaunchExcludes))
    return MOE_ERR_INVALID_ARG;
  if (cfg->d % 256 || cfg->f % 128) return MOE_ERR_UNSUPPORTED;
  rc = check_ptrs({xp, w1, w2, tiles, plan_info, row_token, row_gate, a_scratch, out, status});
  if (rc != MOE_OK) return rc;
  if ((mode & MOE_FFN_STRICT_SLOTS) && ffn_units(mode) < cfg->P) return MOE_ERR_UNSUPPORTED;
  return cuda_result(launch_ffn(*cfg, xp, w1, w2, tiles, plan_info, row_token, row_gate, mode,
                                a_scratch, out, status, (cudaStream_t)stream));
}

int moe_dispatch_grad(const moe_cfg* cfg, const float* dy, const int32_t* row_token,
                      const float* row_gate, const int32_t* plan_info, uint16_t* d_rows,
                      int32_t* status, moe_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  if (cfg->d % 8) return MOE_ERR_UNSUPPORTED;
  rc = check_ptrs({dy, row_token, row_gate, plan_info, d_rows, status});
  if (rc != MOE_OK) return rc;
  return cuda_result(launch_dispatch_grad(*cfg, dy, row_token, row_gate, plan_info, d_rows,
                                          status, (cudaStream_t)stream));
}

int moe_expert_ffn_backward(const moe_cfg* cfg, const uint16_t* xp, const uint16_t* w1,
                            const uint16_t* w2, const int32_t* tiles, const int32_t* plan_info,
                            const int32_t* block_off, const int32_t* row_token,
                            const uint16_t* d_rows, const uint16_t* saved,
                            uint16_t* bwd_scratch, float* dx, float* dw1, float* dw2,
                            int32_t* status, moe_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  if (cfg->d % 256 || cfg->f % 128) return MOE_ERR_UNSUPPORTED;
  rc = check_ptrs({xp, w1, w2, tiles, plan_info, block_off, row_token, d_rows, saved,
                   bwd_scratch, dx, dw1, dw2, status});
  if (rc != MOE_OK) return rc;
  return cuda_result(launch_ffn_backward(*cfg, xp, w1, w2, tiles, plan_info, block_off,
                                         row_token, d_rows, saved, bwd_scratch, dx, dw1, dw2,
                                         status, (cudaStream_t)stream));
}

int moe_combine(const moe_cfg* cfg, const uint16_t* o, const int32_t* tok_row,
                const float* topk_gates, float* y, int32_t* status, moe_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  if (cfg->d % 8) return MOE_ERR_UNSUPPORTED;
  rc = check_ptrs({o, tok_row, topk_gates, y, status});
  if (rc != MOE_OK) return rc;
  return cuda_result(
      launch_combine(*cfg, o, tok_row, topk_gates, y, status, (cudaStream_t)stream));
}

const char* moe_status_string(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or misaligned pointer";
    case MOE_ERR_CUDA: return "CUDA launch or call failed";
    case MOE_ERR_TOO_LARGE: return "problem too large for the fixed scratch of moe_expert_ffn_noalloc";
    case MOE_STATUS_BAD_ID: return "expert id out of range";
    case MOE_STATUS_OVERFLOW: return "expert rows exceed their blocks";
    case MOE_STATUS_NONFINITE: return "non-finite router logit";
    case MOE_STATUS_TIMEOUT: return "bounded wait in a kernel ran out";
    case MOE_STATUS_PLAN: return "block plan exceeds its bound";
    default: return code > 0 ? "several device status bits" : "unknown code";
  }
}

}  // extern "C"
