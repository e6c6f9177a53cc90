// common.cuh -- small device helpers shared by the kernels of libattn.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "attn.h"

namespace sdpa {

// Record a device-side error in the status word; the first recorded error is kept.
__device__ __forceinline__ void report(int* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// Start token and length of sequence b from cumulative lengths without a leading zero
// ("aclnnFlashAttentionVarLenScore", constraints on actualSeqQLenOptional).
__device__ __forceinline__ void seq_span(const int32_t* cu, int b, int* start, int* len) {
  const int lo = b == 0 ? 0 : __ldg(cu + b - 1);
  *start = lo;
  *len = __ldg(cu + b) - lo;
}

// Keys visible to query row i under the mode are visible_begin(i) .. visible_end(i) - 1: a
// prefix for the causal modes, a window i - pre .. i + next for the band (both limits within
// +-2^30, so the sums below stay in int range).
__device__ __forceinline__ int visible_end(int mask_mode, int i, int sq, int sk, int next = 0) {
  if (mask_mode == ATTN_MASK_NONE) return sk;
  const int last = mask_mode == ATTN_MASK_CAUSAL_TOPLEFT ? i
                   : mask_mode == ATTN_MASK_BAND         ? i + next
                                                         : i + sk - sq;
  return last < 0 ? 0 : (last + 1 < sk ? last + 1 : sk);
}
__device__ __forceinline__ int visible_begin(int mask_mode, int i, int pre) {
  if (mask_mode != ATTN_MASK_BAND) return 0;
  return i - pre > 0 ? i - pre : 0;
}

// Find which query tile of a packed batch this block owns. Sequence b contributes
// ceil(len_b / tile) tiles, in sequence order. Run by one full warp; all lanes get the answer.
// Returns false if `x` is past the last tile. Also validates the cumulative lengths
// (non-decreasing, last entry == total) and reports ATTN_ERR_DATA if they are not.
__device__ __forceinline__ bool warp_find_tile(const int32_t* cu, int B, int total, int tile, int x,
                                               int* seq, int* tile_in_seq, int* status, bool* bad) {
  const int lane = threadIdx.x & 31;
  int base = 0;       // tiles before the current chunk of 32 sequences
  int prev_end = 0;   // cu of the sequence before the chunk
  *bad = false;
  for (int c0 = 0; c0 < B; c0 += 32) {
    const int b = c0 + lane;
    int end = b < B ? __ldg(cu + b) : 0;
    int start = __shfl_up_sync(0xffffffffu, end, 1);
    if (lane == 0) start = prev_end;
    const int len = b < B ? end - start : 0;
    const bool wrong = (b < B) && (len < 0 || end > total || (b == B - 1 && end != total));
    if (__any_sync(0xffffffffu, wrong)) {
      if (lane == 0) report(status, ATTN_ERR_DATA);
      *bad = true;
      return false;
    }
    int n = len > 0 ? (len + tile - 1) / tile : 0;
    // inclusive scan of tile counts across the warp
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, b < B && x < base + incl);
    if (hit) {
      const int src = __ffs(hit) - 1;
      const int excl = __shfl_sync(0xffffffffu, incl - n, src);
      *seq = c0 + src;
      *tile_in_seq = x - base - excl;
      return true;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
    prev_end = __shfl_sync(0xffffffffu, end, 31);
  }
  return false;
}

}  // namespace sdpa
