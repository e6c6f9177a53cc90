// csr_plan.cu -- builds the plan of a CSR pattern (layout in csr_plan.cuh) on the device.
//
// "paddle.nn.functional.sparse_attention" (Paddle 2.3 API doc), 参数: offset is a row pointer
// [S+1] per (b, h) and columns [nnz] per (b, h). The plan is the pattern bookkeeping of the
// tiled CSR kernels (the union of a block's columns and each row's marks), done once for a
// pattern instead of once per call; "aclnnFlashAttentionVarLenScore" (CANN 8.5 API doc), 函数原型,
// likewise splits its call into a sizing step and an execution that takes caller-owned memory.
//
// One block of 512 threads per (b, h, 128-row block):
//   1. the union of the rows' columns (csr_union.cuh): a byte per column from one streamed
//      pass over the block's column indices, packed into a bitmap with a popcount prefix;
//   2. the union list: a thread per bitmap word writes the columns of its set bits in order;
//   3. the marks, 2,048 union columns at a time: a warp per row, each lane a contiguous run of
//      the row's columns, ORs the bits of their union indices into register words and those
//      into shared memory (csr_mark_row in csr_union.cuh); the window is then written out as a uint4 per
//      (tile, row), and a row whose set bits number fewer than its entries stored a column
//      twice, which marks cannot hold: it is flagged bad (ATTN_ERR_DATA);
//   4. the header: magic, S, ucap, U and the bad-row bits.
#include "common.cuh"
#include "csr_plan.cuh"
#include "csr_union.cuh"
#include "launch.h"

namespace sdpa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxS = 32768;
constexpr int kWin = 2048;                    // union columns whose marks are held at once
constexpr int kWinWords = kWin / 32;
constexpr int kMarkStride = kWinWords + 1;    // padded row: a warp reading 32 rows' word hits 32 banks
constexpr int kMarkBytes = kPlanRows * kMarkStride * 4;
// the marks reuse the union's byte-per-column region once the union is packed
constexpr int kRegion = kMaxS > kMarkBytes ? kMaxS : kMarkBytes;
constexpr int kBitmapOff = kRegion;
constexpr int kPrefixOff = kBitmapOff + kMaxS / 8;
constexpr int kRowOff = kPrefixOff + kMaxS / 8;     // c0, c1, bad, count per row
constexpr int kMiscOff = kRowOff + 4 * kPlanRows * 4;
constexpr int kSmemBytes = kMiscOff + 16;

__global__ void __launch_bounds__(kThreads) csr_plan_kernel(CsrPlanArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* bytes = smem;
  uint32_t* marks = reinterpret_cast<uint32_t*>(smem);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + kBitmapOff);
  uint32_t* wpre = reinterpret_cast<uint32_t*>(smem + kPrefixOff);
  int* row_c0 = reinterpret_cast<int*>(smem + kRowOff);
  int* row_c1 = row_c0 + kPlanRows;
  int* row_bad = row_c1 + kPlanRows;
  int* row_cnt = row_bad + kPlanRows;
  int* misc = reinterpret_cast<int*>(smem + kMiscOff);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = a.S;
  const int tiles_q = plan_row_blocks(S);
  const int64_t bh = blockIdx.x / tiles_q;
  const int r0 = (int)(blockIdx.x - bh * tiles_q) * kPlanRows;
  const int32_t* off = a.offset + bh * (int64_t)(S + 1);
  const int32_t* cols = a.columns + bh * a.nnz_cap;
  const int64_t ucap = plan_ucap(S, a.nnz_cap);
  uint8_t* rec = a.plan + (int64_t)blockIdx.x * plan_block_bytes(S, a.nnz_cap);
  PlanHeader* hdr = reinterpret_cast<PlanHeader*>(rec);
  int32_t* ucol = reinterpret_cast<int32_t*>(rec + kPlanHeader);
  uint4* mk = reinterpret_cast<uint4*>(rec + kPlanHeader + 4 * ucap);
  const int nw = (S + 31) >> 5;

  for (int w = tid; w < nw * 8; w += kThreads) reinterpret_cast<uint32_t*>(bytes)[w] = 0u;
  for (int x = tid; x < kPlanRows; x += kThreads) row_bad[x] = 0;
  __syncthreads();
  const CsrUnion un{bitmap, wpre, bytes, row_c0, row_c1, row_bad, misc};
  const int U = csr_block_union<kThreads, kPlanRows>(un, off, cols, S, r0, a.nnz_cap, a.cols_vec, a.status);

  // the union list: union column u is the u-th set bit of the bitmap
  for (int w = tid; w < nw; w += kThreads) {
    uint32_t bits = bitmap[w];
    int u = (int)wpre[w];
    while (bits != 0u) {
      ucol[u++] = w * 32 + (__ffs(bits) - 1);
      bits &= bits - 1u;
    }
  }

  for (int W0 = 0; W0 < U; W0 += kWin) {
    for (int x = tid; x < kPlanRows * kMarkStride; x += kThreads) marks[x] = 0u;
    __syncthreads();
    for (int rr = warp; rr < kPlanRows; rr += kWarps) {
      const int n = csr_mark_row(marks + rr * kMarkStride, bitmap, wpre, cols, row_c0[rr], row_c1[rr], S, W0, kWin);
      if (lane == 0) row_cnt[rr] = n;
    }
    __syncthreads();
    const int t0 = W0 / 128;                              // first tile of the window
    const int nt = (min(kWin, U - W0) + 127) / 128;       // tiles of the window holding union columns
    for (int x = tid; x < nt * kPlanRows; x += kThreads) {
      const int tl = x / kPlanRows, r = x - tl * kPlanRows;
      const uint32_t* m = marks + r * kMarkStride + 4 * tl;
      mk[(int64_t)(t0 + tl) * kPlanRows + r] = make_uint4(m[0], m[1], m[2], m[3]);
    }
    if (tid < kPlanRows) {
      int set = 0;
      for (int w = 0; w < kWinWords; ++w) set += __popc(marks[tid * kMarkStride + w]);
      if (set != row_cnt[tid] && row_bad[tid] == 0) {  // a column stored twice in this row
        row_bad[tid] = 1;
        report(a.status, ATTN_ERR_DATA);
      }
    }
    __syncthreads();
  }

  if (warp < kPlanRows / 32) {
    const unsigned bad = __ballot_sync(0xffffffffu, row_bad[tid] != 0);
    if (lane == 0) hdr->bad[warp] = bad;
  }
  if (tid == 0) {
    hdr->S = S;
    hdr->ucap = (int32_t)ucap;
    hdr->U = U;
    hdr->magic = kPlanMagic;
  }
}

}  // namespace

cudaError_t launch_csr_plan(const CsrPlanArgs& a, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(csr_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)a.B * a.H * plan_row_blocks(a.S);
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  csr_plan_kernel<<<(unsigned)blocks, kThreads, kSmemBytes, st>>>(a);
  return cudaGetLastError();
}

}  // namespace sdpa
