// sparse_csr.cu -- CSR-sparse attention forward in float32.
//
// "paddle.nn.functional.sparse_attention" (Paddle 2.3 API doc), formula and 参数: for every
// (b, h, i) the softmax of q_i . k_j / sqrt(D) runs over the stored entries of row i of that
// (b, h) slice (offset = row pointer [B,H,S+1], columns [B,H,nnz]) and weights the rows v_j.
//
// Design (gather-bound, not a dense contraction, so no tensor cores):
//   * one warp per query row; the warp is split into 4 groups of 8 lanes and each group owns
//     one stored entry at a time, so a warp has 4 key rows (and 4 value rows) in flight;
//   * inside a group the head dimension is split across the 8 lanes in 16-byte pieces, so a
//     key row is read as whole 32-byte sectors and the q.k dot needs 3 shuffles;
//   * each group keeps its own online-softmax state (max, sum, partial output) and the four
//     states are combined once at the end of the row;
//   * the 8 warps of a block take 8 consecutive rows of the same (b, h): for window-shaped
//     patterns their key/value rows overlap and come from L1/L2.
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace sdpa {
namespace {

constexpr int kWarps = 8;
constexpr int kGroup = 8;            // lanes per stored entry
constexpr int kGroups = 32 / kGroup; // entries in flight per warp

// VEC4: D % 4 == 0 and 16-byte aligned rows -> float4 pieces; otherwise scalar pieces.
// NP: pieces per lane (float4 pieces when VEC4, else scalars), >= ceil(D / (4 or 1) / 8).
template <bool VEC4, int NP>
__global__ void __launch_bounds__(kWarps * 32) csr_kernel(CsrArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane / kGroup, sub = lane % kGroup;
  const int64_t row = (int64_t)blockIdx.x * kWarps + warp;  // (b*H + h)*S + i
  const int64_t nrows = (int64_t)a.B * a.H * a.S;
  if (row >= nrows) return;
  const int S = a.S, D = a.D;
  const int64_t bh = row / S;
  const int i = (int)(row - bh * S);
  const int32_t* off = a.offset + bh * (S + 1);
  const int32_t* col = a.columns + bh * a.nnz_cap;
  const float* Kb = a.k + bh * (int64_t)S * D;
  const float* Vb = a.v + bh * (int64_t)S * D;
  const float* q = a.q + row * D;
  float* o = a.out + row * D;
  const float scale = 1.0f / sqrtf((float)D);

  constexpr int W = VEC4 ? 4 : 1;  // floats per piece
  const int npieces = (D + W - 1) / W;

  // ---- row pointer checks ---------------------------------------------------------------
  const int c0 = __ldg(off + i), c1 = __ldg(off + i + 1);
  bool bad = c0 < 0 || c1 < c0 || (int64_t)c1 > a.nnz_cap || (i == 0 && c0 != 0);

  // q pieces of this lane (same for the 4 groups)
  float qv[NP][W];
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int pc = sub + p * kGroup;
#pragma unroll
    for (int w = 0; w < W; ++w) qv[p][w] = 0.f;
    if (pc < npieces) {
      if constexpr (VEC4) {
        const float4 t = __ldg(reinterpret_cast<const float4*>(q) + pc);
        qv[p][0] = t.x * scale;
        qv[p][1] = t.y * scale;
        qv[p][2] = t.z * scale;
        qv[p][3] = t.w * scale;
      } else {
        qv[p][0] = __ldg(q + pc) * scale;
      }
    }
  }

  float m = -INFINITY, l = 0.f;
  float acc[NP][W];
#pragma unroll
  for (int p = 0; p < NP; ++p)
#pragma unroll
    for (int w = 0; w < W; ++w) acc[p][w] = 0.f;

  if (!bad) {
    for (int c = c0 + grp; c < c1 + grp; c += kGroups) {
      const bool live = c < c1;
      int j = live ? __ldg(col + c) : 0;
      bad = __any_sync(0xffffffffu, live && (j < 0 || j >= S));
      if (bad) break;
      float kv[NP][W], vv[NP][W];
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const int pc = sub + p * kGroup;
        if (live && pc < npieces) {
          if constexpr (VEC4) {
            const float4 tk = __ldg(reinterpret_cast<const float4*>(Kb + (int64_t)j * D) + pc);
            const float4 tv = __ldg(reinterpret_cast<const float4*>(Vb + (int64_t)j * D) + pc);
            kv[p][0] = tk.x; kv[p][1] = tk.y; kv[p][2] = tk.z; kv[p][3] = tk.w;
            vv[p][0] = tv.x; vv[p][1] = tv.y; vv[p][2] = tv.z; vv[p][3] = tv.w;
          } else {
            kv[p][0] = __ldg(Kb + (int64_t)j * D + pc);
            vv[p][0] = __ldg(Vb + (int64_t)j * D + pc);
          }
        } else {
#pragma unroll
          for (int w = 0; w < W; ++w) kv[p][w] = vv[p][w] = 0.f;
        }
      }
      float s = 0.f;
#pragma unroll
      for (int p = 0; p < NP; ++p)
#pragma unroll
        for (int w = 0; w < W; ++w) s = fmaf(qv[p][w], kv[p][w], s);
#pragma unroll
      for (int x = kGroup / 2; x > 0; x >>= 1) s += __shfl_xor_sync(0xffffffffu, s, x);
      if (live) {
        const float mnew = fmaxf(m, s);
        const float corr = expf(m - mnew);  // m = -inf on the first entry gives 0
        const float pe = expf(s - mnew);
        l = l * corr + pe;
        m = mnew;
#pragma unroll
        for (int p = 0; p < NP; ++p)
#pragma unroll
          for (int w = 0; w < W; ++w) acc[p][w] = fmaf(pe, vv[p][w], acc[p][w] * corr);
      }
    }
  }
  if (bad) {
    if (lane == 0) report(a.status, ATTN_ERR_DATA);
    m = -INFINITY;
    l = 0.f;
#pragma unroll
    for (int p = 0; p < NP; ++p)
#pragma unroll
      for (int w = 0; w < W; ++w) acc[p][w] = 0.f;
  }

  // ---- combine the 4 group states (lanes sub, sub+8, sub+16, sub+24 hold the same pieces)
  float mt = m;
#pragma unroll
  for (int x = kGroup; x < 32; x <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, x));
  const float f = (m == -INFINITY) ? 0.f : expf(m - mt);
  float lt = l * f;
#pragma unroll
  for (int x = kGroup; x < 32; x <<= 1) lt += __shfl_xor_sync(0xffffffffu, lt, x);
  const float inv = lt > 0.f ? 1.f / lt : 0.f;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
#pragma unroll
    for (int w = 0; w < W; ++w) {
      float t = acc[p][w] * f;
#pragma unroll
      for (int x = kGroup; x < 32; x <<= 1) t += __shfl_xor_sync(0xffffffffu, t, x);
      acc[p][w] = t * inv;
    }
  }
  if (grp == 0) {
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const int pc = sub + p * kGroup;
      if (pc < npieces) {
        if constexpr (VEC4) {
          reinterpret_cast<float4*>(o)[pc] = make_float4(acc[p][0], acc[p][1], acc[p][2], acc[p][3]);
        } else {
          o[pc] = acc[p][0];
        }
      }
    }
  }
}

template <bool VEC4, int NP>
cudaError_t go(const CsrArgs& a, cudaStream_t st) {
  const int64_t rows = (int64_t)a.B * a.H * a.S;
  const int64_t blocks = (rows + kWarps - 1) / kWarps;
  if (blocks == 0) return cudaSuccess;
  csr_kernel<VEC4, NP><<<(unsigned)blocks, kWarps * 32, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_csr(const CsrArgs& a, cudaStream_t st) {
  const bool aligned = ((uintptr_t)a.q % 16 == 0) && ((uintptr_t)a.k % 16 == 0) &&
                       ((uintptr_t)a.v % 16 == 0) && ((uintptr_t)a.out % 16 == 0);
  if (a.D % 4 == 0 && aligned) {
    const int pieces = a.D / 4;  // float4 pieces per row, <= 64
    if (pieces <= 8) return go<true, 1>(a, st);
    if (pieces <= 16) return go<true, 2>(a, st);
    if (pieces <= 32) return go<true, 4>(a, st);
    return go<true, 8>(a, st);
  }
  if (a.D <= 64) return go<false, 8>(a, st);
  if (a.D <= 128) return go<false, 16>(a, st);
  return go<false, 32>(a, st);
}

}  // namespace sdpa
