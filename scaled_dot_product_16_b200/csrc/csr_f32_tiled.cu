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
// its own ~300 key/value rows through L1/L2 (which bounds the row-per-warp kernel).
//  * The gathers are cp.async copies into two buffers: tile t+1's rows are in flight while
//    tile t is multiplied, and a tile costs one block barrier (the P rows a thread's softmax
//    writes are read back only by the 8 lanes of its own warp that share those rows).
//  * For each window of 512 union columns, every row's thread marks which of them its row
//    stores (a bit per row and union column) from its own column list, merging runs of
//    neighbouring columns in registers. The window's union columns are listed once, a thread
//    per bitmap word, so no tile searches for its columns.
//  * Scores are a 128x32 register-tiled product on the FMA pipe (4 rows x 4 keys per thread,
//    keys kg, kg+8, kg+16, kg+24, so the 16-byte reads of 8 neighbouring threads fall in 8
//    different bank groups); an unmarked score is left out of the online softmax.
//  * P goes through shared memory to the P.V product (4 rows x D/8 columns per thread, columns
//    4kg + 32c, so 8 neighbouring threads read 128 contiguous bytes of a value row).
// All arithmetic is fp32 FMA. The softmax works in log2 units (Q is staged pre-scaled by
// log2(e) / sqrt(D)), so each probability is one subtraction and one ex2.approx (relative error
// about 2^-22, far inside the fp32 tolerance) instead of an expf. A row that stores some
// column more than once (each copy weighs once, which a bit cannot hold) is recomputed exactly
// by a row-per-warp pass at the end.
#include <math.h>

#include <atomic>

#include "common.cuh"
#include "csr_union.cuh"
#include "launch.h"

namespace sdpa {
namespace {

constexpr int kKeys = 32;                    // union keys per tile
constexpr int kWin = 512;                    // union columns whose row marks are held at once
constexpr int kWinTiles = kWin / kKeys;
constexpr int kWinWords = kWin / 32;         // mark words per row
constexpr int kMaskStride = kWinWords + 1;   // padded row of the marks: a warp's 4 rows, 4 banks apart
constexpr int kMaxS = 32768;

// A block owns ROWS query rows (a multiple of 16: a warp per 16 rows, two threads per row);
// the host picks ROWS per call so that the blocks fill whole rounds of the GPU's block slots.
template <int D, int ROWS>
struct F32Cfg {
  static constexpr int kRows = ROWS;
  static constexpr int kThreads = 2 * ROWS;
  static constexpr int kPtStride = ROWS + 4;  // padded key row of P^T: a warp's 16-byte stores spread over banks
  static_assert(ROWS % 16 == 0 && ROWS <= 128, "a warp per 16 rows, at most 8 warps");
  static constexpr int kKStride = D + 4;  // floats per staged key row (16-byte groups: key k -> k mod 8)
  static constexpr int kQsOff = 0;                                    // float Qt[D][kRows], scaled
  static constexpr int kKsOff = kQsOff + kRows * D * 4;               // float Ks[2][kKeys][kKStride]
  static constexpr int kVsOff = kKsOff + 2 * kKeys * kKStride * 4;    // float Vs[2][kKeys][D]
  static constexpr int kPsOff = kVsOff + 2 * kKeys * D * 4;           // float Pt[kKeys][kPtStride]
  static constexpr int kMaskOff = kPsOff + kKeys * kPtStride * 4;     // uint32 marks[kRows][kMaskStride]
  static constexpr int kKcolOff = kMaskOff + kRows * kMaskStride * 4; // int kcol[kWin]
  static constexpr int kBitmapOff = kKcolOff + kWin * 4;
  static constexpr int kPrefixOff = kBitmapOff + kMaxS / 8;
  static constexpr int kRowOff = kPrefixOff + kMaxS / 8;              // c0, c1, bad, heavy, count per row
  static constexpr int kMiscOff = kRowOff + 5 * kRows * 4;
  static constexpr int kSmemBytes = kMiscOff + 16;
  // the union's byte per column lives in the K/V buffers until the union is packed
  static_assert(kPsOff - kKsOff >= kMaxS, "the union's column bytes fit the K/V buffers");
  static_assert(kSmemBytes <= 232448, "227 KB of shared memory per block");
  static_assert(D != 64 || kSmemBytes <= 112 * 1024, "two blocks per SM at D = 64");
  static_assert((kPtStride % 32) % 8 == 4, "16-byte P^T stores of 8 consecutive keys on distinct banks");
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Starts the copies of the key and value rows of kcol[0 .. nk) into one buffer pair (key row k
// at ks + k * kKStride floats, value row k at vs + k * D floats); rows nk .. kKeys-1 are zeroed.
template <int D, int ROWS>
__device__ __forceinline__ void stage_tile(uint32_t ks, uint32_t vs, const int* kcol, int nk, const float* Kb,
                                           const float* Vb) {
  using C = F32Cfg<D, ROWS>;
  constexpr int kChunks = D / 4;  // 16-byte chunks per row
  for (int x = threadIdx.x; x < kKeys * kChunks; x += C::kThreads) {
    const int k = x / kChunks, c = x % kChunks;
    const bool valid = k < nk;
    const int64_t col = valid ? kcol[k] : 0;  // row 0 is a readable address for a zero fill
    cp_async16(ks + (uint32_t)(k * C::kKStride + 4 * c) * 4u, Kb + col * D + 4 * c, valid);
    cp_async16(vs + (uint32_t)(k * D + 4 * c) * 4u, Vb + col * D + 4 * c, valid);
  }
}

// Marks for rows of the block: bit u - W0 of row x's words is set when row x stores union column
// u (W0 <= u < W0 + kWin), built a warp per row (csr_mark_row in csr_union.cuh). A row that
// stores some column twice sets fewer bits than it has entries in the window: it is marked heavy.
// Every thread of the block calls this; it ends with the marks complete.
template <int ROWS>
__device__ __forceinline__ void build_marks(uint32_t* marks, const CsrUnion& un, int* row_heavy,
                                            int* row_cnt, const int32_t* cols, int S, int W0) {
  constexpr int kThreads = 2 * ROWS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int x = threadIdx.x; x < ROWS * kMaskStride; x += kThreads) marks[x] = 0u;
  __syncthreads();
  // a warp takes its rows two at a time (the rows are a multiple of 16, the warps ROWS / 16)
  constexpr int kWarps = kThreads / 32;
  for (int rr = warp; rr < ROWS; rr += 2 * kWarps) {
    const int r2 = rr + kWarps;
    int na, nb;
    csr_mark_row2(marks + rr * kMaskStride, marks + r2 * kMaskStride, un.bitmap, un.wpre, cols, un.row_c0[rr],
                  un.row_c1[rr], un.row_c0[r2], un.row_c1[r2], S, W0, kWin, na, nb);
    if (lane == 0) {
      row_cnt[rr] = na;
      row_cnt[r2] = nb;
    }
  }
  __syncthreads();
  if (threadIdx.x < ROWS) {
    const int x = threadIdx.x;
    int set = 0;
#pragma unroll
    for (int w = 0; w < kWinWords; ++w) set += __popc(marks[x * kMaskStride + w]);
    if (set != row_cnt[x]) row_heavy[x] = 1;
  }
}

// kcol[u - W0] = the column of union index u, for W0 <= u < min(U, W0 + kWin): a thread per
// bitmap word walks its set bits.
template <int THREADS>
__device__ __forceinline__ void list_window_columns(int* kcol, const CsrUnion& un, int nw, int W0) {
  for (int w = threadIdx.x; w < nw; w += THREADS) {
    uint32_t bits = un.bitmap[w];
    int u = (int)un.wpre[w];
    if (u >= W0 + kWin || u + __popc(bits) <= W0) continue;
    while (bits != 0u) {
      const int pos = __ffs(bits) - 1;
      bits &= bits - 1u;
      if (u >= W0 && u < W0 + kWin) kcol[u - W0] = w * 32 + pos;
      ++u;
    }
  }
}

template <int D, int ROWS>
__global__ void __launch_bounds__(2 * ROWS, D == 64 ? 2 : 1) csr_f32_tiled_kernel(CsrArgs a) {
  using C = F32Cfg<D, ROWS>;
  constexpr int kRows = C::kRows, kThreads = C::kThreads, kPtStride = C::kPtStride;
  extern __shared__ __align__(16) uint8_t smem[];
  float* Qt = reinterpret_cast<float*>(smem + C::kQsOff);
  float* Ks = reinterpret_cast<float*>(smem + C::kKsOff);
  float* Vs = reinterpret_cast<float*>(smem + C::kVsOff);
  float* Pt = reinterpret_cast<float*>(smem + C::kPsOff);
  uint32_t* marks = reinterpret_cast<uint32_t*>(smem + C::kMaskOff);
  int* kcol = reinterpret_cast<int*>(smem + C::kKcolOff);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + C::kBitmapOff);
  uint32_t* wpre = reinterpret_cast<uint32_t*>(smem + C::kPrefixOff);
  uint8_t* bytes = smem + C::kKsOff;  // the union's byte per column, before any K/V row lands
  int* row_c0 = reinterpret_cast<int*>(smem + C::kRowOff);
  int* row_c1 = row_c0 + kRows;
  int* row_bad = row_c1 + kRows;
  int* row_heavy = row_bad + kRows;
  int* row_cnt = row_heavy + kRows;
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
  const float scale2 = scale * 1.4426950408889634f;  // scores in log2 units for the tiles

  for (int w = tid; w < nw * 8; w += kThreads) reinterpret_cast<uint32_t*>(bytes)[w] = 0u;
  for (int x = tid; x < kRows; x += kThreads) {
    row_bad[x] = 0;
    row_heavy[x] = 0;
  }
  __syncthreads();
  const CsrUnion un{bitmap, wpre, bytes, row_c0, row_c1, row_bad, misc};
  const int U = csr_block_union<kThreads, kRows>(un, off, cols, S, r0, a.nnz_cap, a.cols_vec, a.status);
  const int T = (U + kKeys - 1) / kKeys;

  // Q, scaled and transposed: Qt[d][r] = q[r0 + r][d] * log2(e) / sqrt(D); rows past S are zero. With d
  // outermost, the 4 rows a thread multiplies are one 16-byte read, and the 16 rows a warp reads
  // at one d are 64 contiguous bytes (one wavefront; row-major, they were 4 bank-conflicting ones)
  for (int x = tid; x < kRows * (D / 4); x += kThreads) {
    const int rr = x % kRows, c4 = x / kRows;  // consecutive threads: consecutive rows (no conflict)
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + rr < S) v = __ldg(reinterpret_cast<const float4*>(Qb + (int64_t)(r0 + rr) * D) + c4);
    Qt[(4 * c4 + 0) * kRows + rr] = v.x * scale2;
    Qt[(4 * c4 + 1) * kRows + rr] = v.y * scale2;
    Qt[(4 * c4 + 2) * kRows + rr] = v.z * scale2;
    Qt[(4 * c4 + 3) * kRows + rr] = v.w * scale2;
  }

  const int rg = tid >> 3;  // rows 4rg .. 4rg+3
  const int kg = tid & 7;   // keys kg + 8j of a tile; output columns 4kg + 32c .. +3
  constexpr int kV4 = D / 32;
  constexpr uint32_t kKsBuf = kKeys * C::kKStride * 4, kVsBuf = kKeys * D * 4;
  const uint32_t ks0 = smem_addr(Ks), vs0 = smem_addr(Vs);
  float m[4], l[4], o[4][kV4 * 4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int c = 0; c < kV4 * 4; ++c) o[i][c] = 0.f;
  }

  int W0 = 0;
  for (int t = 0; t < T; ++t) {
    const int b = t & 1;
    if (t % kWinTiles == 0) {
      __syncthreads();  // the last window's marks, columns and buffers are read no more
      W0 = t * kKeys;
      build_marks<ROWS>(marks, un, row_heavy, row_cnt, cols, S, W0);
      list_window_columns<kThreads>(kcol, un, nw, W0);
      __syncthreads();
      stage_tile<D, ROWS>(ks0 + b * kKsBuf, vs0 + b * kVsBuf, kcol, min(kKeys, U - W0), Kb, Vb);
    }
    cp_async_wait_all();
    __syncthreads();  // tile t has landed for every thread; tile t-1's reads of K, V and P are done
    if (t + 1 < T && (t + 1) % kWinTiles != 0)
      stage_tile<D, ROWS>(ks0 + (b ^ 1) * kKsBuf, vs0 + (b ^ 1) * kVsBuf, kcol + (t + 1) * kKeys - W0,
                    min(kKeys, U - (t + 1) * kKeys), Kb, Vb);
    const float* Kt = Ks + b * (kKeys * C::kKStride);
    const float* Vt = Vs + b * (kKeys * D);
    // A warp whose 16 rows store none of this tile's 32 union columns has nothing to add: it
    // skips the tile's products (its softmax state and output stay as they are).
    const uint32_t wmark = marks[(16 * warp + (lane & 15)) * kMaskStride + t % kWinTiles];
    if (!__any_sync(0xffffffffu, wmark != 0u)) continue;

    // scores of rows 4rg.. against keys kg + 8j
    float sc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) sc[i][j] = 0.f;
#pragma unroll 8  // (2, 4 and 16 measured slower)
    for (int d = 0; d < D; d += 4) {
      float4 kk[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) kk[j] = *reinterpret_cast<const float4*>(Kt + (kg + 8 * j) * C::kKStride + d);
      float4 qq[4];  // qq[dd] = rows 4rg .. 4rg+3 at d + dd
#pragma unroll
      for (int dd = 0; dd < 4; ++dd) qq[dd] = *reinterpret_cast<const float4*>(Qt + (d + dd) * kRows + 4 * rg);
      // rows (4rg, 4rg+1) and (4rg+2, 4rg+3) as fp32 pairs: one packed FMA for two scores
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float kd[4] = {kk[j].x, kk[j].y, kk[j].z, kk[j].w};
#pragma unroll
        for (int dd = 0; dd < 4; ++dd) {
          const float2 k2 = make_float2(kd[dd], kd[dd]);
          float2 lo = __ffma2_rn(make_float2(qq[dd].x, qq[dd].y), k2, make_float2(sc[0][j], sc[1][j]));
          float2 hi = __ffma2_rn(make_float2(qq[dd].z, qq[dd].w), k2, make_float2(sc[2][j], sc[3][j]));
          sc[0][j] = lo.x;
          sc[1][j] = lo.y;
          sc[2][j] = hi.x;
          sc[3][j] = hi.y;
        }
      }
    }
    // Online softmax per row over the 8 lanes that share it. The max in use is raised only when
    // some stored score of the tile exceeds it by more than 2^kLazyLog2 (log2 units, as the
    // scores are): only then is the tile's row max reduced over the 8 lanes and O and the sum
    // rescaled. Otherwise P is taken against the max in use (each P at most 2^kLazyLog2, and
    // the same max for the row's P, sum and O, so the result is unchanged).
    constexpr float kLazyLog2 = 8.f;
    float corr[4], p[4][4], lmax[4];
    bool has[4][4];
    bool need = false;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t mw = marks[(4 * rg + i) * kMaskStride + t % kWinTiles] >> kg;
      lmax[i] = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        has[i][j] = ((mw >> (8 * j)) & 1u) != 0u;
        if (has[i][j]) lmax[i] = fmaxf(lmax[i], sc[i][j]);
      }
      need |= lmax[i] > m[i] + kLazyLog2;  // also true for the first finite score of a row
    }
    const bool bump = __any_sync(0xffffffffu, need);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      corr[i] = 1.f;
      if (bump) {
        float tmax = lmax[i];
#pragma unroll
        for (int x = 1; x < 8; x <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, x));
        if (tmax > m[i] + kLazyLog2) {  // the same on the row's 8 lanes
          corr[i] = m[i] == -INFINITY ? 0.f : ex2_approx(m[i] - tmax);
          m[i] = tmax;
        }
      }
      float rs = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        p[i][j] = has[i][j] && m[i] != -INFINITY ? ex2_approx(sc[i][j] - m[i]) : 0.f;
        rs += p[i][j];
      }
      // this lane's part of the row sum: the 8 lanes of a row share its max (so its rescale
      // factor), and their parts are added once, after the last tile
      l[i] = l[i] * corr[i] + rs;
    }
    // P transposed: key kg + 8j's 4 rows 4rg.. as one 16-byte store, read back below as one
    // 16-byte load per key by the same 8 lanes of this warp
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<float4*>(Pt + (kg + 8 * j) * kPtStride + 4 * rg) = make_float4(p[0][j], p[1][j], p[2][j], p[3][j]);
    __syncwarp();
    // O = O * corr + P V for rows 4rg.. and columns 4kg + 32c .. (the rescale only after a bump)
    if (bump) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < kV4 * 4; ++c) o[i][c] *= corr[i];
    }
    // keys in groups of 8; a group that none of this warp's 16 rows stores is skipped
    const uint32_t kmask = __reduce_or_sync(0xffffffffu, wmark);
#pragma unroll 1
    for (int g = 0; g < kKeys / 8; ++g) {
    if (((kmask >> (8 * g)) & 0xffu) == 0u) continue;
#pragma unroll
    for (int k = 8 * g; k < 8 * g + 8; ++k) {
      const float4 p4 = *reinterpret_cast<const float4*>(Pt + k * kPtStride + 4 * rg);
      const float pk[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
      for (int c = 0; c < kV4; ++c) {
        const float4 vv = *reinterpret_cast<const float4*>(Vt + k * D + 4 * kg + 32 * c);
        // output columns (4kg + 32c, +1) and (+2, +3) as fp32 pairs
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 p2 = make_float2(pk[i], pk[i]);
          const float2 lo = __ffma2_rn(p2, make_float2(vv.x, vv.y), make_float2(o[i][4 * c + 0], o[i][4 * c + 1]));
          const float2 hi = __ffma2_rn(p2, make_float2(vv.z, vv.w), make_float2(o[i][4 * c + 2], o[i][4 * c + 3]));
          o[i][4 * c + 0] = lo.x;
          o[i][4 * c + 1] = lo.y;
          o[i][4 * c + 2] = hi.x;
          o[i][4 * c + 3] = hi.y;
        }
      }
    }
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int x = 1; x < 8; x <<= 1) l[i] += __shfl_xor_sync(0xffffffffu, l[i], x);

  // ---- epilogue: O / l; bad rows are zeros, heavy rows are redone below -----------------------
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = 4 * rg + i, ii = r0 + rr;
    if (ii >= S || row_heavy[rr]) continue;
    const float f = (row_bad[rr] == 0 && l[i] > 0.f) ? 1.f / l[i] : 0.f;
    float* dst = a.out + (bh * (int64_t)S + ii) * D + 4 * kg;
#pragma unroll
    for (int c = 0; c < kV4; ++c)
      reinterpret_cast<float4*>(dst + 32 * c)[0] =
          make_float4(o[i][4 * c] * f, o[i][4 * c + 1] * f, o[i][4 * c + 2] * f, o[i][4 * c + 3] * f);
  }

  // ---- rows that store a column more than once: a row per warp, entry by entry ---------------
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

template <int D, int ROWS>
cudaError_t launch_rows(const CsrArgs& a, cudaStream_t st) {
  using C = F32Cfg<D, ROWS>;
  const int64_t blocks = (int64_t)a.B * a.H * ((a.S + ROWS - 1) / ROWS);
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  csr_f32_tiled_kernel<D, ROWS><<<(unsigned)blocks, C::kThreads, C::kSmemBytes, st>>>(a);
  return cudaGetLastError();
}

// Blocks of one instantiation resident on an SM at once (0 on error), looked up once per device.
template <int D, int ROWS>
int resident_blocks() {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> cached[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  int n = cached[dev].load(std::memory_order_acquire);
  if (n > 0) return n;
  using C = F32Cfg<D, ROWS>;
  if (cudaFuncSetAttribute(csr_f32_tiled_kernel<D, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::kSmemBytes) != cudaSuccess)
    return 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, csr_f32_tiled_kernel<D, ROWS>, C::kThreads,
                                                    C::kSmemBytes) != cudaSuccess || n <= 0)
    return 0;
  cached[dev].store(n, std::memory_order_release);
  return n;
}

// Rows per block: the blocks of a call run in rounds of (resident blocks per SM x SMs), and a
// round takes about as long as one block. A block's time is a fixed part (taking the union of its
// rows' columns and their marks: latency-bound, a warp per 16 rows, about as long as the tile
// loop of kFixedRows rows on the window-and-stride pattern of 4,096 keys) plus its tile loop, in
// proportion to its rows. The choice minimises rounds x (kFixedRows + ROWS) among the block sizes
// that fit as many blocks on an SM as 128-row blocks do (fewer rows per block with more blocks per
// SM would change the sharing the estimate assumes); on a tie the larger blocks win. On the
// 148-SM B200 and 2 x 8 heads of 4,096 rows this picks 112 rows: 592 blocks, exactly two rounds of
// 2 x 148, where 128-row blocks make 512 and leave 68 SMs with a fourth block after the others
// are done (0.2936 -> 0.2875 ms measured).
constexpr int kFixedRows = 74;

template <int D>
cudaError_t launch_d(const CsrArgs& a, cudaStream_t st, int num_sms) {
  struct Cand {
    int rows;
    int resident;
  };
  const Cand cands[] = {{128, resident_blocks<D, 128>()}, {112, resident_blocks<D, 112>()},
                        {96, resident_blocks<D, 96>()},   {80, resident_blocks<D, 80>()},
                        {64, resident_blocks<D, 64>()}};
  // candidates that cannot be resident at all are skipped; the 128-row block's residency is the
  // reference (if it cannot run, the first size that can sets it)
  int ref = -1, best = -1;
  int64_t best_cost = 0;
  for (int c = 0; c < 5; ++c) {
    if (cands[c].resident <= 0) continue;
    if (ref < 0) ref = c;
    if (cands[c].resident != cands[ref].resident) continue;
    const int64_t blocks = (int64_t)a.B * a.H * ((a.S + cands[c].rows - 1) / cands[c].rows);
    const int64_t slots = (int64_t)cands[c].resident * (num_sms > 0 ? num_sms : 1);
    const int64_t rounds = (blocks + slots - 1) / slots;
    const int64_t cost = rounds * (kFixedRows + cands[c].rows);
    if (best < 0 || cost < best_cost) {
      best = c;
      best_cost = cost;
    }
  }
  if (best < 0) return cudaErrorInvalidConfiguration;
  switch (cands[best].rows) {
    case 128: return launch_rows<D, 128>(a, st);
    case 112: return launch_rows<D, 112>(a, st);
    case 96: return launch_rows<D, 96>(a, st);
    case 80: return launch_rows<D, 80>(a, st);
    default: return launch_rows<D, 64>(a, st);
  }
}

}  // namespace

bool sparse_csr_tiled_supported(const CsrArgs& a) {
  const bool aligned = ((uintptr_t)a.q % 16 == 0) && ((uintptr_t)a.k % 16 == 0) &&
                       ((uintptr_t)a.v % 16 == 0) && ((uintptr_t)a.out % 16 == 0);
  return aligned && (a.D == 64 || a.D == 128) && a.S <= kMaxS;
}

cudaError_t launch_sparse_csr_tiled(const CsrArgs& a, cudaStream_t st) {
  return a.D == 128 ? launch_d<128>(a, st, a.num_sms) : launch_d<64>(a, st, a.num_sms);
}

}  // namespace sdpa
