// csr_plan.cuh -- layout of a CSR pattern plan, shared by the kernel that builds it
// (csr_plan.cu) and the tensor-core CSR kernel that reads it (csr_tc_sm100.cu).
//
// "paddle.nn.functional.sparse_attention" (Paddle 2.3 API doc), 参数: per (b, h) the pattern is a
// row pointer offset [S+1] and columns [nnz]. A plan holds, for every block of 128 query rows of
// every (b, h), what the tiled kernels otherwise rebuild on every call:
//   * the sorted union of the columns the block's rows store (U entries, each key once);
//   * per row and per tile of 128 union columns, 128 bits that say which of those columns the
//     row stores (its "marks");
//   * which rows are bad (a row pointer or column out of range, or a column stored twice).
// A plan depends on the pattern only, so one plan serves every call with the same pattern
// (every layer and step of a model with a fixed sparsity pattern).
//
// Block record (one per (b, h, row block), in that order, kBlockHeader + 20 * ucap bytes):
//   [0, 64)                 header: magic, S, ucap, U, bad-row bits [4 words]
//   [64, 64 + 4 ucap)       int32 union columns, U used
//   [64 + 4 ucap, ...)      marks: uint4 [ucap / 128 tiles][128 rows], bit c of word x of tile t,
//                           row r = row r stores union column t*128 + 32x + c
// ucap = min(S, nnz_cap) rounded up to 128: no block's union can be larger.
#pragma once

#include <stdint.h>

namespace sdpa {

constexpr int kPlanRows = 128;                 // query rows per block
constexpr int64_t kPlanHeader = 64;            // bytes of a block record's header
constexpr uint32_t kPlanMagic = 0x43535250u;   // "PRSC": a record the plan kernel wrote

struct PlanHeader {
  uint32_t magic;
  int32_t S;
  int32_t ucap;
  int32_t U;
  uint32_t bad[4];  // bit r%32 of word r/32: row r of the block is bad (zeros, ATTN_ERR_DATA)
  uint32_t pad[8];
};
static_assert(sizeof(PlanHeader) == kPlanHeader, "plan header is 64 bytes");

__host__ __device__ inline int64_t plan_ucap(int S, int64_t nnz_cap) {
  const int64_t u = nnz_cap < S ? nnz_cap : (int64_t)S;
  return (u + kPlanRows - 1) / kPlanRows * kPlanRows;
}
__host__ __device__ inline int64_t plan_block_bytes(int S, int64_t nnz_cap) {
  return kPlanHeader + 20 * plan_ucap(S, nnz_cap);
}
__host__ __device__ inline int plan_row_blocks(int S) { return (S + kPlanRows - 1) / kPlanRows; }
// Bytes of the whole plan, or -1 if it would not fit in int64.
__host__ __device__ inline int64_t plan_bytes(int B, int H, int S, int64_t nnz_cap) {
  const int64_t blocks = (int64_t)B * H * plan_row_blocks(S);
  const int64_t per = plan_block_bytes(S, nnz_cap);
  if (blocks > 0 && per > INT64_MAX / blocks) return -1;
  return blocks * per;
}

}  // namespace sdpa
