// csr_f32_tiled.cu -- CSR-sparse attention forward in float32 on the CUDA cores, tiled over the
// union of a block's columns (the attn_sparse_csr path for D = 64 or 128).
//
// "paddle.nn.functional.sparse_attention" (Paddle 2.3 API doc), formula and 参数: for every
// (b, h, i) the softmax of q_i . k_j / sqrt(D) runs over the stored entries of row i of that
// (b, h) slice and weights the rows v_j; a column stored c times in a row counts c times.
//
// Design: a block owns 128 query rows of one (b, h) (256 threads). It takes the union of its
// rows' columns (csr_union.cuh), then walks the union 32 keys at a time: the key and value rows
// are gathered once into shared memory and serve all 128 rows, instead of every row gathering
// its own ~300 key/value rows through L1/L2 (which bounds the row-per-warp kernel). Scores are
// a 128x32 register-tiled product on the FMA pipe (4 rows x 4 keys per thread, Q transposed and
// pre-scaled in shared memory); each row counts how often it stores each union column (a byte
// per row and union column, 256-column windows, built by the row's own thread), so a score
// enters the online softmax with weight count * exp(s - m), or not at all. P goes through
// shared memory to the P.V product (4 rows x D/8 columns per thread). All arithmetic is fp32
// FMA with expf, as the row-per-warp kernel does. A row that stores one column more than 255
// times in a window (a count a byte cannot hold) is recomputed exactly by a row-per-warp pass
// at the end.
#include <math.h>

#include "common.cuh"
#include "csr_union.cuh"
#include "launch.h"

namespace sdpa {
namespace {

constexpr int kRows = 128;                   // query rows per block
constexpr int kKeys = 32;                    // union keys per tile
constexpr int kThreads = 256;
constexpr int kWin = 256;                    // union columns whose per-row counts are held at once
constexpr int kWinStride = kWin + 16;        // padded row of the counts
constexpr int kMaxS = 32768;
constexpr int kPStride = kKeys + 1;          // padded row of P

template <int D>
struct F32Cfg {
  static constexpr int kQtOff = 0;                                  // float Qt[D][kRows]
  static constexpr int kKtOff = kQtOff + D * kRows * 4;             // float Kt[D][kKeys]
  static constexpr int kVsOff = kKtOff + D * kKeys * 4;             // float Vs[kKeys][D]
  static constexpr int kPsOff = kVsOff + kKeys * D * 4;             // float Ps[kRows][kPStride]
  static constexpr int kBitmapOff = kPsOff + kRows * kPStride * 4;
  static constexpr int kPrefixOff = kBitmapOff + kMaxS / 8;
  static constexpr int kBytesOff = kPrefixOff + kMaxS / 8;
  static constexpr int kBytesSize = kMaxS > kRows * kWinStride ? kMaxS : kRows * kWinStride;
  static constexpr int kColOff = kBytesOff + kBytesSize;
  static constexpr int kRowOff = kColOff + kKeys * 4;               // c0, c1, bad, heavy per row
  static constexpr int kMiscOff = kRowOff + 4 * kRows * 4;
  static constexpr int kSmemBytes = kMiscOff + 16;
  static_assert(kSmemBytes <= 232448, "227 KB of shared memory per block");
};

template <int D>
__global__ void __launch_bounds__(kThreads, D == 64 ? 2 : 1) csr_f32_tiled_kernel(CsrArgs a) {
  using C = F32Cfg<D>;
  extern __shared__ __align__(16) uint8_t smem[];
  float* Qt = reinterpret_cast<float*>(smem + C::kQtOff);
  float* Kt = reinterpret_cast<float*>(smem + C::kKtOff);
  float* Vs = reinterpret_cast<float*>(smem + C::kVsOff);
  float* Ps = reinterpret_cast<float*>(smem + C::kPsOff);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + C::kBitmapOff);
  uint32_t* wpre = reinterpret_cast<uint32_t*>(smem + C::kPrefixOff);
  uint8_t* bytes = smem + C::kBytesOff;
  int* kcol = reinterpret_cast<int*>(smem + C::kColOff);
  int* row_c0 = reinterpret_cast<int*>(smem + C::kRowOff);
  int* row_c1 = row_c0 + kRows;
  int* row_bad = row_c1 + kRows;
  int* row_heavy = row_bad + kRows;
  int* misc = reinterpret_cast<int*>(smem + C::kMiscOff);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = a.S;
  const int tiles_q = (S + kRows - 1) / kRows;
  const int64_t bh = blockIdx.x / tiles_q;
  const int r0 = (int)(blockIdx.x - bh * tiles_q) * kRows;
  const int32_t* off = a.offset + bh * (int64_t)(S + 1);
  const int32_t* cols = a.columns + bh * a.nnz_cap;
  const float* Qb = a.q + bh * (int64_t)S * D;
  const float* Kb = a.k + bh * (int64_t)S * D;
  const float* Vb = a.v + bh * (int64_t)S * D;
  const int nw = (S + 31) >> 5;
  const float scale = 1.0f / sqrtf((float)D);

  for (int w = tid; w < nw * 8; w += kThreads) reinterpret_cast<uint32_t*>(bytes)[w] = 0u;
  for (int x = tid; x < kRows; x += kThreads) {
    row_bad[x] = 0;
    row_heavy[x] = 0;
  }
  __syncthreads();
  const CsrUnion un{bitmap, wpre, bytes, row_c0, row_c1, row_bad, misc};
  const int U = csr_block_union<kThreads, kRows>(un, off, cols, S, r0, a.nnz_cap, a.cols_vec, a.status);
  const int T = (U + kKeys - 1) / kKeys;

  // Q, transposed and scaled: Qt[d][r] = q[r0 + r][d] / sqrt(D); rows past S are zero
  for (int x = tid; x < kRows * (D / 4); x += kThreads) {
    const int rr = x % kRows, c4 = x / kRows;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + rr < S) v = __ldg(reinterpret_cast<const float4*>(Qb + (int64_t)(r0 + rr) * D) + c4);
    Qt[(4 * c4 + 0) * kRows + rr] = v.x * scale;
    Qt[(4 * c4 + 1) * kRows + rr] = v.y * scale;
    Qt[(4 * c4 + 2) * kRows + rr] = v.z * scale;
    Qt[(4 * c4 + 3) * kRows + rr] = v.w * scale;
  }

  const int rg = tid >> 3;  // rows 4rg .. 4rg+3
  const int kg = tid & 7;   // keys 4kg .. 4kg+3 of a tile; columns kg*D/8 .. of the output
  constexpr int kCols = D / 8;
  float m[4], l[4], o[4][kCols];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int c = 0; c < kCols; ++c) o[i][c] = 0.f;
  }

  for (int t = 0; t < T; ++t) {
    if ((t * kKeys) % kWin == 0) {
      // each row's counts for union columns [t*32, t*32 + kWin), built by the row's thread
      __syncthreads();
      if (tid < kRows) {
        const int base = t * kKeys;
        uint8_t* row = bytes + tid * kWinStride;
#pragma unroll
        for (int x = 0; x < kWin / 16; ++x) reinterpret_cast<uint4*>(row)[x] = make_uint4(0u, 0u, 0u, 0u);
        const int e1 = row_c1[tid];
        for (int e0 = row_c0[tid]; e0 < e1; e0 += kUnionBatch) {
          int jj[kUnionBatch];
#pragma unroll
          for (int b = 0; b < kUnionBatch; ++b) jj[b] = e0 + b < e1 ? __ldg(cols + e0 + b) : -1;
#pragma unroll
          for (int b = 0; b < kUnionBatch; ++b) {
            const int j = jj[b];
            if (j >= 0 && j < S) {  // bad columns are already flagged; the row is zeroed
              const int u = csr_union_index(bitmap, wpre, j);
              if (u >= base && u < base + kWin) {
                const uint8_t c = row[u - base];
                if (c == 255) row_heavy[tid] = 1;
                else row[u - base] = (uint8_t)(c + 1);
              }
            }
          }
        }
      }
      __syncthreads();
    }
    // the tile's union columns, then their key rows (transposed) and value rows
    if (warp == 0) {
      const int u = t * kKeys + lane;
      kcol[lane] = u < U ? csr_union_col(bitmap, wpre, nw, u) : -1;
    }
    __syncthreads();
    // key rows: lane = key, so the transposed stores of a warp fall in 32 different banks
    for (int x = tid; x < kKeys * (D / 4); x += kThreads) {
      const int k = x % kKeys, c4 = x / kKeys, col = kcol[k];
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f);
      if (col >= 0) kv = __ldg(reinterpret_cast<const float4*>(Kb + (int64_t)col * D) + c4);
      Kt[(4 * c4 + 0) * kKeys + k] = kv.x;
      Kt[(4 * c4 + 1) * kKeys + k] = kv.y;
      Kt[(4 * c4 + 2) * kKeys + k] = kv.z;
      Kt[(4 * c4 + 3) * kKeys + k] = kv.w;
    }
    // value rows: lanes along the row, so every row is one contiguous 16-byte-per-lane store
    for (int x = tid; x < kKeys * (D / 4); x += kThreads) {
      const int k = x / (D / 4), c4 = x % (D / 4), col = kcol[k];
      float4 vv = make_float4(0.f, 0.f, 0.f, 0.f);
      if (col >= 0) vv = __ldg(reinterpret_cast<const float4*>(Vb + (int64_t)col * D) + c4);
      reinterpret_cast<float4*>(Vs + k * D)[c4] = vv;
    }
    __syncthreads();

    // scores of rows 4rg.. against keys 4kg..
    float sc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) sc[i][j] = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; ++d) {
      const float4 qa = *reinterpret_cast<const float4*>(Qt + d * kRows + 4 * rg);
      const float4 kb = *reinterpret_cast<const float4*>(Kt + d * kKeys + 4 * kg);
      const float qv[4] = {qa.x, qa.y, qa.z, qa.w}, kvv[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) sc[i][j] = fmaf(qv[i], kvv[j], sc[i][j]);
    }
    // online softmax per row over the 8 lanes that share it
    float corr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t cw = *reinterpret_cast<const uint32_t*>(bytes + (4 * rg + i) * kWinStride +
                                                            (t * kKeys) % kWin + 4 * kg);
      float cnt[4], tmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        cnt[j] = (float)((cw >> (8 * j)) & 0xffu);
        if (cnt[j] > 0.f) tmax = fmaxf(tmax, sc[i][j]);
      }
#pragma unroll
      for (int x = 1; x < 8; x <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, x));
      const float mnew = fmaxf(m[i], tmax);
      float p[4] = {0.f, 0.f, 0.f, 0.f}, rs = 0.f;
      corr[i] = 1.f;
      if (mnew != -INFINITY) {
        corr[i] = m[i] == -INFINITY ? 0.f : expf(m[i] - mnew);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          p[j] = cnt[j] > 0.f ? cnt[j] * expf(sc[i][j] - mnew) : 0.f;
          rs += p[j];
        }
      }
#pragma unroll
      for (int x = 1; x < 8; x <<= 1) rs += __shfl_xor_sync(0xffffffffu, rs, x);
      l[i] = l[i] * corr[i] + rs;
      m[i] = mnew;
#pragma unroll
      for (int j = 0; j < 4; ++j) Ps[(4 * rg + i) * kPStride + 4 * kg + j] = p[j];
    }
    __syncthreads();
    // O = O * corr + P V for rows 4rg.. and columns kg*D/8 ..
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int c = 0; c < kCols; ++c) o[i][c] *= corr[i];
#pragma unroll 4
    for (int k = 0; k < kKeys; ++k) {
      float pk[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) pk[i] = Ps[(4 * rg + i) * kPStride + k];
#pragma unroll
      for (int c4 = 0; c4 < kCols / 4; ++c4) {
        const float4 vv = reinterpret_cast<const float4*>(Vs + k * D + kg * kCols)[c4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          o[i][4 * c4 + 0] = fmaf(pk[i], vv.x, o[i][4 * c4 + 0]);
          o[i][4 * c4 + 1] = fmaf(pk[i], vv.y, o[i][4 * c4 + 1]);
          o[i][4 * c4 + 2] = fmaf(pk[i], vv.z, o[i][4 * c4 + 2]);
          o[i][4 * c4 + 3] = fmaf(pk[i], vv.w, o[i][4 * c4 + 3]);
        }
      }
    }
    __syncthreads();  // the next tile overwrites Kt, Vs and Ps
  }
  __syncthreads();

  // ---- epilogue: O / l; bad rows are zeros, heavy rows are redone below -----------------------
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = 4 * rg + i, ii = r0 + rr;
    if (ii >= S || row_heavy[rr]) continue;
    const float f = (row_bad[rr] == 0 && l[i] > 0.f) ? 1.f / l[i] : 0.f;
    float* dst = a.out + (bh * (int64_t)S + ii) * D + kg * kCols;
#pragma unroll
    for (int c4 = 0; c4 < kCols / 4; ++c4)
      reinterpret_cast<float4*>(dst)[c4] =
          make_float4(o[i][4 * c4] * f, o[i][4 * c4 + 1] * f, o[i][4 * c4 + 2] * f, o[i][4 * c4 + 3] * f);
  }

  // ---- rows that store a column more than 255 times: a row per warp, entry by entry ----------
  for (int rr = warp; rr < kRows; rr += kThreads / 32) {
    if (!row_heavy[rr] || r0 + rr >= S) continue;
    constexpr int kPer = D / 32;  // columns per lane
    const float* qrow = Qb + (int64_t)(r0 + rr) * D;
    float qv[kPer], acc[kPer], mm = -INFINITY, ll = 0.f;
#pragma unroll
    for (int c = 0; c < kPer; ++c) {
      qv[c] = __ldg(qrow + lane + 32 * c) * scale;
      acc[c] = 0.f;
    }
    const int e1 = row_c1[rr];
    for (int e = row_c0[rr]; e < e1; ++e) {
      const int j = __ldg(cols + e);
      if (j < 0 || j >= S) continue;  // flagged already; the row is zeroed below
      float sd = 0.f;
#pragma unroll
      for (int c = 0; c < kPer; ++c) sd = fmaf(qv[c], __ldg(Kb + (int64_t)j * D + lane + 32 * c), sd);
#pragma unroll
      for (int x = 16; x > 0; x >>= 1) sd += __shfl_xor_sync(0xffffffffu, sd, x);
      const float mnew = fmaxf(mm, sd);
      const float cr = mm == -INFINITY ? 0.f : expf(mm - mnew);
      const float pe = expf(sd - mnew);
      ll = ll * cr + pe;
      mm = mnew;
#pragma unroll
      for (int c = 0; c < kPer; ++c) acc[c] = fmaf(pe, __ldg(Vb + (int64_t)j * D + lane + 32 * c), acc[c] * cr);
    }
    const float f = (row_bad[rr] == 0 && ll > 0.f) ? 1.f / ll : 0.f;
    float* dst = a.out + (bh * (int64_t)S + r0 + rr) * D;
#pragma unroll
    for (int c = 0; c < kPer; ++c) dst[lane + 32 * c] = acc[c] * f;
  }
}

template <int D>
cudaError_t launch_d(const CsrArgs& a, cudaStream_t st) {
  using C = F32Cfg<D>;
  cudaError_t e = cudaFuncSetAttribute(csr_f32_tiled_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)a.B * a.H * ((a.S + kRows - 1) / kRows);
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  csr_f32_tiled_kernel<D><<<(unsigned)blocks, kThreads, C::kSmemBytes, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

bool sparse_csr_tiled_supported(const CsrArgs& a) {
  const bool aligned = ((uintptr_t)a.q % 16 == 0) && ((uintptr_t)a.k % 16 == 0) &&
                       ((uintptr_t)a.v % 16 == 0) && ((uintptr_t)a.out % 16 == 0);
  return aligned && (a.D == 64 || a.D == 128) && a.S <= kMaxS;
}

cudaError_t launch_sparse_csr_tiled(const CsrArgs& a, cudaStream_t st) {
  return a.D == 128 ? launch_d<128>(a, st) : launch_d<64>(a, st);
}

}  // namespace sdpa
