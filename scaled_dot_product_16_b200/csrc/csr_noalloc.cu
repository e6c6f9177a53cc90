// csr_noalloc.cu -- attn_sparse_csr_tc_noalloc: the tensor-core CSR attention for callers that
// cannot allocate device memory.
//
// attn_sparse_csr_tc_planned is the fastest form of the CSR call, but it reads a plan of the
// pattern from a buffer the caller allocates. Some callers have no way to do that: code that runs
// inside a host application which owns the GPU's memory through its own pool and gives its
// plugins no workspace, or a latency-critical path where cudaMalloc (which can synchronise the
// device and can fail once the pool holds all the memory) is not acceptable. For them this file
// keeps one fixed scratch array in the library itself, and the entry point builds the plan there
// and runs the planned kernel, allocating nothing.
//
// The array is a file-scope __device__ variable: every GPU on which the library's code for this
// file is loaded holds its kScratchBytes until the process exits. In host code its name is only
// a host-side stand-in, not a device address, so its device address is looked up once per device
// (with that device current) and passed to the kernels.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "attn.h"
#include "csr_plan.cuh"

namespace {

constexpr int64_t kScratchBytes = int64_t(48) << 20;  // 48 MiB: the largest plan this call takes

static __device__ __align__(256) uint8_t g_csr_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint8_t* g_scratch[kMaxDevices] = {};

// The scratch array's device address on the current device, looked up on the first call there.
int scratch_on_current_device(uint8_t** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_csr_scratch) != cudaSuccess || p == nullptr) return ATTN_ERR_CUDA;
    g_scratch[dev] = static_cast<uint8_t*>(p);
  }
  *ptr = g_scratch[dev];
  return ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

int attn_sparse_csr_tc_noalloc(const void* q, const void* k, const void* v,
                               const int32_t* csr_offset, const int32_t* csr_columns, int B, int H,
                               int S, int D, int64_t nnz_cap, int dtype, void* out, void* stream) {
  // every argument is checked before anything is launched (the rules of attn_sparse_csr_tc)
  if (dtype != ATTN_BF16 && dtype != ATTN_F16) return ATTN_ERR_INVALID;
  if (B < 0 || H < 0 || S < 0 || nnz_cap < 0 || D < 1) return ATTN_ERR_INVALID;
  if ((int64_t)B * H * S == 0) return ATTN_OK;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || csr_offset == nullptr)
    return ATTN_ERR_INVALID;
  if (nnz_cap > 0 && csr_columns == nullptr) return ATTN_ERR_INVALID;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (S > 32768) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATTN_ERR_INVALID;
  int64_t need = 0;
  int rc = attn_csr_plan_size(B, H, S, nnz_cap, &need);
  if (rc != ATTN_OK) return rc;
  if (need > kScratchBytes) return ATTN_ERR_UNSUPPORTED;  // the plan does not fit the scratch
  uint8_t* scratch = nullptr;
  rc = scratch_on_current_device(&scratch);
  if (rc != ATTN_OK) return rc;
  // the plan kernel writes every byte the planned kernel reads (headers, the union entries in
  // use, the mark tiles in use), so the scratch needs no clearing between calls
  rc = attn_csr_plan(csr_offset, csr_columns, B, H, S, nnz_cap, scratch, kScratchBytes, stream);
  if (rc != ATTN_OK) return rc;
  return attn_sparse_csr_tc_planned(q, k, v, scratch, kScratchBytes, B, H, S, D, nnz_cap, dtype, out,
                                    stream);
}

}  // extern "C"
