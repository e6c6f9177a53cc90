// launch.h -- internal launch entry points of libattn.so (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sdpa {

struct FwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* cu_q;   // TND only
  const int32_t* cu_kv;  // TND only
  int B, Sq, Skv, Nq, Nkv, D;
  int Dv;  // value / output head size (== D except through attn_fwd_masked)
  float scale;
  int mask_mode, layout, dtype;
  int pre, next;               // band limits (mask_mode ATTN_MASK_BAND), clamped to +-2^30
  const uint8_t* mask;         // explicit mask, 1 = excluded (null: none)
  int64_t mask_bs, mask_rs;    // its batch and row strides in bytes
  bool mask_vec;               // mask, mask_bs and mask_rs all 16-byte aligned
  int acc_mode;  // 0: plain output; 1: overwrite an accumulator; 2: merge into it
  void* out;     // output, or the accumulator's output (merge layouts) when acc_mode != 0
  float* smax;   // statistics (may be null with ssum when acc_mode == 0), or the accumulator's
  float* ssum;   // [.., 8]-lane statistics when acc_mode != 0
  int* status;  // device status word
  int num_sms;
};

struct CsrArgs {
  const float* q;
  const float* k;
  const float* v;
  const int32_t* offset;
  const int32_t* columns;
  int B, H, S, D;
  int64_t nnz_cap;
  bool cols_vec;  // columns 16-byte aligned and nnz_cap % 4 == 0: read 4 indices at a time
  float* out;
  int* status;
  int num_sms;   // SMs of the device (the tiled kernel sizes its blocks to fill whole rounds)
};

struct CsrTcArgs {  // attn_sparse_csr_tc: 16-bit q, k, v, out [B, H, S, D]
  const void* q;
  const void* k;
  const void* v;
  const int32_t* offset;   // unused with a plan
  const int32_t* columns;  // unused with a plan
  const uint8_t* plan;     // a plan of the pattern (csr_plan.cuh), or null: build per block
  int B, H, S, D, dtype;
  int64_t nnz_cap;
  bool cols_vec;  // columns 16-byte aligned and nnz_cap % 4 == 0: read 4 indices at a time
  void* out;
  int* status;
};

struct CsrPlanArgs {  // attn_csr_plan: the pattern of a CSR call and the plan buffer to fill
  const int32_t* offset;
  const int32_t* columns;
  int B, H, S;
  int64_t nnz_cap;
  bool cols_vec;
  uint8_t* plan;
  int* status;
};

struct MergeArgs {
  const void* prev_out;
  const float* prev_max;
  const float* prev_sum;
  const void* cur_out;
  const float* cur_max;
  const float* cur_sum;
  int S, B, N, D, dtype, layout;
  const int64_t* seq_qlen;  // TND only, may be null
  void* out;
  float* out_max;
  float* out_sum;
  int* status;
};

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t st);
cudaError_t launch_fwd_f32(const FwdArgs& a, cudaStream_t st);
cudaError_t launch_fwd_bf16(const FwdArgs& a, cudaStream_t st);
cudaError_t launch_sparse_csr(const CsrArgs& a, cudaStream_t st);
bool sparse_csr_tiled_supported(const CsrArgs& a);
cudaError_t launch_sparse_csr_tiled(const CsrArgs& a, cudaStream_t st);
cudaError_t launch_sparse_csr_tc(const CsrTcArgs& a, cudaStream_t st);
cudaError_t launch_csr_plan(const CsrPlanArgs& a, cudaStream_t st);

}  // namespace sdpa
