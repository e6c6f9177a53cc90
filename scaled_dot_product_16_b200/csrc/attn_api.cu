// attn_api.cu -- the C ABI of libattn.so: argument checks, the device status word, dispatch.
//
// Argument limits follow the constraints of "aclnnFlashAttentionVarLenScore" (CANN 8.5 API
// doc, 约束说明): Nq/Nkv a nonzero integer with 1 <= Nq <= 256, head dim at most 768, at most
// 1M packed tokens and 2K cumulative-length entries. The host never reads device data, so
// data-dependent checks happen in the kernels, which record them in the status word below.
#include <cuda_runtime.h>
#include <stdint.h>

#include <math.h>

#include <mutex>

#include "attn.h"
#include "csr_plan.cuh"
#include "launch.h"

namespace {

// One status word per device; kernels record the first device-side error here. Beside it, the
// slot attn_get_last_error reads the word into (exchanging it for 0 in one atomic step).
__device__ int g_status_word;
__device__ int g_status_read;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
std::mutex g_read_mu[kMaxDevices];  // one status reader at a time per device (the read slot)
int* g_status_ptr[kMaxDevices] = {};
int* g_read_ptr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

// Device addresses of this device's status word and read slot, and its SM count (looked up
// once per device, with that device current).
int device_state(int** status, int* num_sms, int** read_slot = nullptr, int* device = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_status_ptr[dev] == nullptr) {
    void* p = nullptr;
    void* r = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return ATTN_ERR_CUDA;
    if (cudaGetSymbolAddress(&r, g_status_read) != cudaSuccess) return ATTN_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    g_read_ptr[dev] = static_cast<int*>(r);
    g_num_sms[dev] = sms;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  *status = g_status_ptr[dev];
  *num_sms = g_num_sms[dev];
  if (read_slot != nullptr) *read_slot = g_read_ptr[dev];
  if (device != nullptr) *device = dev;
  return ATTN_OK;
}

// Reads the status word and clears it in one step, so an error a kernel on another stream
// records meanwhile is kept for the next read instead of being lost between a read and a clear.
__global__ void read_and_clear_status(int* word, int* slot) { *slot = atomicExch(word, 0); }

constexpr int64_t kMaxTokens = 1 << 20;  // "1M"
constexpr int kMaxCu = 2048;             // "2K" cumulative-length entries

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

int attn_abi_version(void) { return (1 << 16) | 3; }  // 1.3: CSR plans (attn_csr_plan, ..._planned)

const char* attn_status_string(int s) {
  switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported by this library";
    case ATTN_ERR_CUDA: return "CUDA runtime error";
    case ATTN_ERR_DATA: return "bad device data (cumulative lengths or CSR indices)";
    case ATTN_ERR_TIMEOUT: return "pipeline wait timed out";
    default: return "unknown status";
  }
}

}  // extern "C"

namespace {

// The masked-call extras of fwd_impl (band limits, explicit mask, value head size).
struct Extras {
  bool allow_band = false;
  int Dv = -1;  // -1: same as D
  int64_t pre = 0, next = 0;
  const uint8_t* mask = nullptr;
  int64_t mask_bs = 0, mask_rs = 0;
};

int clamp30(int64_t x) {
  const int64_t lim = int64_t(1) << 30;
  return (int)(x < -lim ? -lim : (x > lim ? lim : x));
}

int fwd_impl(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
             const int32_t* cu_seqlens_kv, int B, int Sq, int Skv, int Nq, int Nkv, int D,
             float scale, int mask_mode, int dtype, int layout, void* out, float* softmax_max,
             float* softmax_sum, int acc_mode, void* stream, const Extras& x = Extras()) {
  if (layout != ATTN_BHSD && layout != ATTN_TND) return ATTN_ERR_INVALID;
  if (dtype != ATTN_BF16 && dtype != ATTN_F32 && dtype != ATTN_F16) return ATTN_ERR_INVALID;
  const int max_mode = x.allow_band ? ATTN_MASK_BAND : ATTN_MASK_CAUSAL_BOTTOMRIGHT;
  if (mask_mode < ATTN_MASK_NONE || mask_mode > max_mode) return ATTN_ERR_INVALID;
  if (mask_mode == ATTN_MASK_BAND && clamp30(x.pre) + clamp30(x.next) < 0) return ATTN_ERR_INVALID;
  const int Dv = x.Dv < 0 ? D : x.Dv;
  if (Dv < 1 || Dv > D) return ATTN_ERR_INVALID;
  if (x.mask != nullptr && (x.mask_bs < 0 || x.mask_rs < 0)) return ATTN_ERR_INVALID;
  if (x.mask != nullptr && layout == ATTN_BHSD && x.mask_rs < Skv) return ATTN_ERR_INVALID;
  if (B < 0 || Sq < 0 || Skv < 0) return ATTN_ERR_INVALID;
  if (Nq < 1 || Nq > 256 || Nkv < 1 || Nq % Nkv != 0) return ATTN_ERR_INVALID;
  if (D < 1 || D > 768) return ATTN_ERR_INVALID;
  if (!(scale > 0.f) || scale == INFINITY) return ATTN_ERR_INVALID;  // finite and positive
  if ((softmax_max == nullptr) != (softmax_sum == nullptr)) return ATTN_ERR_INVALID;
  if (acc_mode != 0 && softmax_max == nullptr) return ATTN_ERR_INVALID;
  if (layout == ATTN_TND) {
    if (B > kMaxCu || Sq > kMaxTokens || Skv > kMaxTokens) return ATTN_ERR_INVALID;
    if (B > 0 && (cu_seqlens_q == nullptr || cu_seqlens_kv == nullptr)) return ATTN_ERR_INVALID;
  } else if (cu_seqlens_q != nullptr || cu_seqlens_kv != nullptr) {
    return ATTN_ERR_INVALID;
  }
  const bool empty_q = B == 0 || Sq == 0;
  if (empty_q) return ATTN_OK;
  if (q == nullptr || out == nullptr) return ATTN_ERR_INVALID;
  if (Skv > 0 && (k == nullptr || v == nullptr)) return ATTN_ERR_INVALID;
  if (dtype == ATTN_F32 && D > 256) return ATTN_ERR_UNSUPPORTED;
  if (dtype == ATTN_BF16 || dtype == ATTN_F16) {
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (Dv != D && !(D == 128 && Dv == 64)) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATTN_ERR_INVALID;
  }

  sdpa::FwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.cu_q = cu_seqlens_q;
  a.cu_kv = cu_seqlens_kv;
  a.B = B;
  a.Sq = Sq;
  a.Skv = Skv;
  a.Nq = Nq;
  a.Nkv = Nkv;
  a.D = D;
  a.Dv = Dv;
  a.scale = scale;
  a.mask_mode = mask_mode;
  a.pre = clamp30(x.pre);
  a.next = clamp30(x.next);
  a.mask = x.mask;
  a.mask_bs = x.mask_bs;
  a.mask_rs = x.mask_rs;
  a.mask_vec = x.mask != nullptr && aligned16(x.mask) && (x.mask_bs & 15) == 0 && (x.mask_rs & 15) == 0;
  a.layout = layout;
  a.dtype = dtype;
  a.acc_mode = acc_mode;
  a.out = out;
  a.smax = softmax_max;
  a.ssum = softmax_sum;
  int rc = device_state(&a.status, &a.num_sms);
  if (rc != ATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = dtype == ATTN_F32 ? sdpa::launch_fwd_f32(a, st) : sdpa::launch_fwd_bf16(a, st);
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
             const int32_t* cu_seqlens_kv, int B, int Sq, int Skv, int Nq, int Nkv, int D,
             float scale, int mask_mode, int dtype, int layout, void* out, float* softmax_max,
             float* softmax_sum, void* stream) {
  return fwd_impl(q, k, v, cu_seqlens_q, cu_seqlens_kv, B, Sq, Skv, Nq, Nkv, D, scale, mask_mode,
                  dtype, layout, out, softmax_max, softmax_sum, 0, stream);
}

int attn_fwd_accumulate(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                        const int32_t* cu_seqlens_kv, int B, int Sq, int Skv, int Nq, int Nkv,
                        int D, float scale, int mask_mode, int dtype, int layout, int first,
                        void* acc_out, float* acc_max, float* acc_sum, void* stream) {
  if (acc_out == nullptr || acc_max == nullptr || acc_sum == nullptr) return ATTN_ERR_INVALID;
  if (first != 0 && first != 1) return ATTN_ERR_INVALID;
  // the tensor-core epilogue moves a row's 8 statistic lanes as two 16-byte vectors
  if ((dtype == ATTN_BF16 || dtype == ATTN_F16) && (!aligned16(acc_max) || !aligned16(acc_sum)))
    return ATTN_ERR_INVALID;
  return fwd_impl(q, k, v, cu_seqlens_q, cu_seqlens_kv, B, Sq, Skv, Nq, Nkv, D, scale, mask_mode,
                  dtype, layout, acc_out, acc_max, acc_sum, first ? 1 : 2, stream);
}

int attn_fwd_masked(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                    const int32_t* cu_seqlens_kv, int B, int Sq, int Skv, int Nq, int Nkv, int Dqk,
                    int Dv, float scale, int mask_mode, int64_t pre_tokens, int64_t next_tokens,
                    const uint8_t* atten_mask, int64_t mask_batch_stride, int64_t mask_row_stride,
                    int dtype, int layout, void* out, float* softmax_max, float* softmax_sum,
                    void* stream) {
  Extras x;
  x.allow_band = true;
  x.Dv = Dv < 1 ? 0 : Dv;  // 0 is rejected as out of range
  x.pre = pre_tokens;
  x.next = next_tokens;
  x.mask = atten_mask;
  x.mask_bs = mask_batch_stride;
  x.mask_rs = mask_row_stride;
  return fwd_impl(q, k, v, cu_seqlens_q, cu_seqlens_kv, B, Sq, Skv, Nq, Nkv, Dqk, scale, mask_mode,
                  dtype, layout, out, softmax_max, softmax_sum, 0, stream, x);
}

int attn_sparse_csr(const float* q, const float* k, const float* v, const int32_t* csr_offset,
                    const int32_t* csr_columns, int B, int H, int S, int D, int64_t nnz_cap,
                    float* out, void* stream) {
  if (B < 0 || H < 0 || S < 0 || nnz_cap < 0) return ATTN_ERR_INVALID;
  if (D < 1) return ATTN_ERR_INVALID;
  if ((int64_t)B * H * S == 0) return ATTN_OK;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || csr_offset == nullptr)
    return ATTN_ERR_INVALID;
  if (nnz_cap > 0 && csr_columns == nullptr) return ATTN_ERR_INVALID;
  if (D > 256) return ATTN_ERR_UNSUPPORTED;
  sdpa::CsrArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.offset = csr_offset;
  a.columns = csr_columns;
  a.B = B;
  a.H = H;
  a.S = S;
  a.D = D;
  a.nnz_cap = nnz_cap;
  a.cols_vec = csr_columns != nullptr && aligned16(csr_columns) && nnz_cap % 4 == 0;
  a.out = out;
  int rc = device_state(&a.status, &a.num_sms);
  if (rc != ATTN_OK) return rc;
  // D = 64 or 128 with 16-byte aligned tensors: tiled over each block's union of columns;
  // otherwise a warp per row gathering its own entries
  const cudaError_t e = sdpa::sparse_csr_tiled_supported(a)
                            ? sdpa::launch_sparse_csr_tiled(a, static_cast<cudaStream_t>(stream))
                            : sdpa::launch_sparse_csr(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_sparse_csr_tc(const void* q, const void* k, const void* v, const int32_t* csr_offset,
                       const int32_t* csr_columns, int B, int H, int S, int D, int64_t nnz_cap,
                       int dtype, void* out, void* stream) {
  if (dtype != ATTN_BF16 && dtype != ATTN_F16) return ATTN_ERR_INVALID;
  if (B < 0 || H < 0 || S < 0 || nnz_cap < 0) return ATTN_ERR_INVALID;
  if (D < 1) return ATTN_ERR_INVALID;
  if ((int64_t)B * H * S == 0) return ATTN_OK;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || csr_offset == nullptr)
    return ATTN_ERR_INVALID;
  if (nnz_cap > 0 && csr_columns == nullptr) return ATTN_ERR_INVALID;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (S > 32768) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATTN_ERR_INVALID;
  sdpa::CsrTcArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.offset = csr_offset;
  a.columns = csr_columns;
  a.B = B;
  a.H = H;
  a.S = S;
  a.D = D;
  a.dtype = dtype;
  a.nnz_cap = nnz_cap;
  a.cols_vec = csr_columns != nullptr && aligned16(csr_columns) && nnz_cap % 4 == 0;
  a.out = out;
  int sms = 0;
  int rc = device_state(&a.status, &sms);
  if (rc != ATTN_OK) return rc;
  const cudaError_t e = sdpa::launch_sparse_csr_tc(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_csr_plan_size(int B, int H, int S, int64_t nnz_cap, int64_t* bytes) {
  if (bytes == nullptr || B < 0 || H < 0 || S < 0 || nnz_cap < 0) return ATTN_ERR_INVALID;
  if (S > 32768) return ATTN_ERR_UNSUPPORTED;
  const int64_t n = sdpa::plan_bytes(B, H, S, nnz_cap);
  if (n < 0) return ATTN_ERR_UNSUPPORTED;
  *bytes = n;
  return ATTN_OK;
}

int attn_csr_plan(const int32_t* csr_offset, const int32_t* csr_columns, int B, int H, int S,
                  int64_t nnz_cap, void* plan, int64_t plan_bytes, void* stream) {
  int64_t need = 0;
  const int rc0 = attn_csr_plan_size(B, H, S, nnz_cap, &need);
  if (rc0 != ATTN_OK) return rc0;
  if ((int64_t)B * H * S == 0) return ATTN_OK;
  if (csr_offset == nullptr || plan == nullptr) return ATTN_ERR_INVALID;
  if (nnz_cap > 0 && csr_columns == nullptr) return ATTN_ERR_INVALID;
  if (plan_bytes < need || !aligned16(plan)) return ATTN_ERR_INVALID;
  sdpa::CsrPlanArgs a{};
  a.offset = csr_offset;
  a.columns = csr_columns;
  a.B = B;
  a.H = H;
  a.S = S;
  a.nnz_cap = nnz_cap;
  a.cols_vec = csr_columns != nullptr && aligned16(csr_columns) && nnz_cap % 4 == 0;
  a.plan = static_cast<uint8_t*>(plan);
  int sms = 0;
  int rc = device_state(&a.status, &sms);
  if (rc != ATTN_OK) return rc;
  const cudaError_t e = sdpa::launch_csr_plan(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_sparse_csr_tc_planned(const void* q, const void* k, const void* v, const void* plan,
                               int64_t plan_bytes, int B, int H, int S, int D, int64_t nnz_cap,
                               int dtype, void* out, void* stream) {
  if (dtype != ATTN_BF16 && dtype != ATTN_F16) return ATTN_ERR_INVALID;
  int64_t need = 0;
  const int rc0 = attn_csr_plan_size(B, H, S, nnz_cap, &need);
  if (rc0 != ATTN_OK) return rc0;
  if (D < 1) return ATTN_ERR_INVALID;
  if ((int64_t)B * H * S == 0) return ATTN_OK;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || plan == nullptr)
    return ATTN_ERR_INVALID;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (plan_bytes < need || !aligned16(plan)) return ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATTN_ERR_INVALID;
  sdpa::CsrTcArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.plan = static_cast<const uint8_t*>(plan);
  a.B = B;
  a.H = H;
  a.S = S;
  a.D = D;
  a.dtype = dtype;
  a.nnz_cap = nnz_cap;
  a.out = out;
  int sms = 0;
  int rc = device_state(&a.status, &sms);
  if (rc != ATTN_OK) return rc;
  const cudaError_t e = sdpa::launch_sparse_csr_tc(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_merge(const void* prev_out, const float* prev_max, const float* prev_sum,
               const void* cur_out, const float* cur_max, const float* cur_sum, int S, int B,
               int N, int D, int dtype, int layout, const int64_t* actual_seq_qlen, void* out,
               float* out_max, float* out_sum, void* stream) {
  if (dtype != ATTN_BF16 && dtype != ATTN_F32 && dtype != ATTN_F16) return ATTN_ERR_INVALID;
  if (layout != ATTN_BHSD && layout != ATTN_TND) return ATTN_ERR_INVALID;
  if (S < 0 || B < 0 || N < 1 || D < 1) return ATTN_ERR_INVALID;
  if (layout == ATTN_BHSD && actual_seq_qlen != nullptr) return ATTN_ERR_INVALID;
  if (layout == ATTN_TND && actual_seq_qlen != nullptr && (B < 1 || B > kMaxCu)) return ATTN_ERR_INVALID;
  const int64_t rows = layout == ATTN_TND ? (int64_t)S * N : (int64_t)S * B;
  if (rows == 0) return ATTN_OK;
  if (layout == ATTN_BHSD && ((int64_t)B * N > 0x7fffffffLL || S > 65535LL * 8)) return ATTN_ERR_UNSUPPORTED;
  if (layout == ATTN_TND && rows > 0x7fffffffLL * 8) return ATTN_ERR_UNSUPPORTED;
  if (!prev_out || !prev_max || !prev_sum || !cur_out || !cur_max || !cur_sum || !out ||
      !out_max || !out_sum)
    return ATTN_ERR_INVALID;
  sdpa::MergeArgs a{};
  a.prev_out = prev_out;
  a.prev_max = prev_max;
  a.prev_sum = prev_sum;
  a.cur_out = cur_out;
  a.cur_max = cur_max;
  a.cur_sum = cur_sum;
  a.S = S;
  a.B = B;
  a.N = N;
  a.D = D;
  a.dtype = dtype;
  a.layout = layout;
  a.seq_qlen = actual_seq_qlen;
  a.out = out;
  a.out_max = out_max;
  a.out_sum = out_sum;
  int sms = 0;
  int rc = device_state(&a.status, &sms);
  if (rc != ATTN_OK) return rc;
  const cudaError_t e = sdpa::launch_merge(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_get_last_error(void* stream, int* device_status) {
  if (device_status == nullptr) return ATTN_ERR_INVALID;
  int* word = nullptr;
  int* slot = nullptr;
  int sms = 0, dev = 0;
  int rc = device_state(&word, &sms, &slot, &dev);
  if (rc != ATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lk(g_read_mu[dev]);
  int host = 0;
  read_and_clear_status<<<1, 1, 0, st>>>(word, slot);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemcpyAsync(&host, slot, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return ATTN_ERR_CUDA;
  *device_status = host;
  return ATTN_OK;
}

}  // extern "C"
