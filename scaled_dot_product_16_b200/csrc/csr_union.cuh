// csr_union.cuh -- the union of the columns stored by a block of CSR rows, for the tiled CSR
// kernels ("paddle.nn.functional.sparse_attention", 参数: offset is a row pointer [S+1] per
// (b, h), columns [nnz] per (b, h)).
//
// A block owns ROWS consecutive query rows of one (b, h). The union of the columns those rows
// store is kept as a bitmap over the S keys with an exclusive prefix of its words' popcounts,
// so union column u is the u-th set bit: the union is sorted and each key appears once.
// Building it: thread x < ROWS checks row r0 + x; when every row pointer is good the block's
// entries are one contiguous span of the column array and all threads stream it, 32 indices
// deep (16-byte loads when the array allows), writing a plain byte per column that is packed
// into the bitmap afterwards, so no update is a read-modify-write. Otherwise, or when a column
// is out of range, a slow pass goes a row per warp at a time and flags the offending rows.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace sdpa {

struct CsrUnion {
  uint32_t* bitmap;  // [S/32 rounded up] words
  uint32_t* wpre;    // exclusive prefix of the words' popcounts
  uint8_t* bytes;    // S bytes, zero on entry (a byte per column while the union is taken)
  int* row_c0;       // [ROWS] first entry of each row (0 for a bad row)
  int* row_c1;       // [ROWS] one past its last entry (0 for a bad row)
  int* row_bad;      // [ROWS] zero on entry; 1 for a bad row pointer or column
  int* misc;         // [2] scratch words of the block
};

constexpr int kUnionBatch = 32;  // column indices each thread loads before using any (16 and 64 measured slower)

// Builds the union for rows r0 .. r0 + ROWS - 1 (rows past S are empty). Every thread of the
// block must call it. Returns the number of union columns U. Bad rows report ATTN_ERR_DATA.
template <int THREADS, int ROWS>
__device__ __forceinline__ int csr_block_union(const CsrUnion& m, const int32_t* off, const int32_t* cols,
                                               int S, int r0, int64_t nnz_cap, bool cols_vec,
                                               int* status) {
  static_assert(THREADS >= ROWS, "a thread per row");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = (S + 31) >> 5;
  const int nrows = min(ROWS, S - r0);
  bool good_x = true;
  if (threadIdx.x < ROWS) {
    const int x = threadIdx.x, ii = r0 + x;
    int c0 = 0, c1 = 0;
    if (ii < S) {
      c0 = __ldg(off + ii);
      c1 = __ldg(off + ii + 1);
      good_x = !(c0 < 0 || c1 < c0 || (int64_t)c1 > nnz_cap || (ii == 0 && c0 != 0));
    } else {
      c0 = c1 = __ldg(off + S);  // past the end: empty rows at the span's end
    }
    m.row_c0[x] = good_x ? c0 : 0;
    m.row_c1[x] = good_x ? c1 : 0;
    if (!good_x) {
      m.row_bad[x] = 1;
      report(status, ATTN_ERR_DATA);
    }
  }
  if (threadIdx.x == 0) m.misc[1] = 0;
  const bool all_good = __syncthreads_and(good_x) != 0;
  if (all_good) {
    const int E0 = m.row_c0[0], E1 = m.row_c1[ROWS - 1];
    bool col_bad = false;
    if (cols_vec) {
      // 16 bytes (4 indices) per load from the aligned quad holding E0 on; quads end at
      // nnz_cap, a multiple of 4, so none reads past this (b, h)'s columns
      for (int q0 = E0 >> 2; q0 * 4 < E1; q0 += THREADS * (kUnionBatch / 4)) {
        int4 jj[kUnionBatch / 4];
#pragma unroll
        for (int b = 0; b < kUnionBatch / 4; ++b) {
          const int q = q0 + b * THREADS + (int)threadIdx.x;
          jj[b] = q * 4 < E1 ? __ldg(reinterpret_cast<const int4*>(cols) + q) : make_int4(0, 0, 0, 0);
        }
#pragma unroll
        for (int b = 0; b < kUnionBatch / 4; ++b) {
          const int e = (q0 + b * THREADS + (int)threadIdx.x) * 4;
          const int js[4] = {jj[b].x, jj[b].y, jj[b].z, jj[b].w};
#pragma unroll
          for (int z = 0; z < 4; ++z) {
            if (e + z >= E0 && e + z < E1) {
              if (js[z] >= 0 && js[z] < S) m.bytes[js[z]] = 1;
              else col_bad = true;
            }
          }
        }
      }
    } else {
      for (int base = E0; base < E1; base += THREADS * kUnionBatch) {
        int jj[kUnionBatch];
#pragma unroll
        for (int b = 0; b < kUnionBatch; ++b) {
          const int e = base + b * THREADS + (int)threadIdx.x;
          jj[b] = e < E1 ? __ldg(cols + e) : 0;
        }
#pragma unroll
        for (int b = 0; b < kUnionBatch; ++b) {
          const int e = base + b * THREADS + (int)threadIdx.x, j = jj[b];
          if (e < E1) {
            if (j >= 0 && j < S) m.bytes[j] = 1;
            else col_bad = true;
          }
        }
      }
    }
    if (col_bad) m.misc[1] = 1;
  }
  __syncthreads();
  if (!all_good || m.misc[1] != 0) {
    // slow pass: a row per warp, good rows only; rows holding a bad column are flagged
    for (int rr = warp; rr < nrows; rr += THREADS / 32) {
      const int c0 = m.row_c0[rr], c1 = m.row_c1[rr];
      bool col_bad = false;
      for (int e = (m.row_bad[rr] ? c1 : c0) + lane; e < c1; e += 32) {
        const int j = __ldg(cols + e);
        if (j >= 0 && j < S) m.bytes[j] = 1;
        else col_bad = true;
      }
      if (__any_sync(0xffffffffu, col_bad) && lane == 0) {
        m.row_bad[rr] = 1;
        report(status, ATTN_ERR_DATA);
      }
    }
  }
  __syncthreads();
  // pack the column bytes into bitmap words (byte b of a 32-bit group -> bit b)
  for (int w = threadIdx.x; w < nw; w += THREADS) {
    const uint32_t* g = reinterpret_cast<const uint32_t*>(m.bytes) + w * 8;
    uint32_t bits = 0;
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const uint32_t v = g[x];
      bits |= ((v & 1u) | ((v >> 7) & 2u) | ((v >> 14) & 4u) | ((v >> 21) & 8u)) << (4 * x);
    }
    m.bitmap[w] = bits;
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive prefix of the popcounts, 32 words at a time
    uint32_t carry = 0;
    for (int w0 = 0; w0 < nw; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t c = w < nw ? (uint32_t)__popc(m.bitmap[w]) : 0u;
      uint32_t x = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (w < nw) m.wpre[w] = carry + x - c;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) m.misc[0] = (int)carry;
  }
  __syncthreads();
  return m.misc[0];
}

// Union index of column j (0 <= j < S).
__device__ __forceinline__ int csr_union_index(const uint32_t* bitmap, const uint32_t* wpre, int j) {
  return (int)wpre[j >> 5] + __popc(bitmap[j >> 5] & ((1u << (j & 31)) - 1u));
}

// Column of union index u (0 <= u < U): the word holding the u-th set bit (the largest w with
// wpre[w] <= u), then the bit of that rank inside it.
__device__ __forceinline__ int csr_union_col(const uint32_t* bitmap, const uint32_t* wpre, int nw, int u) {
  int lo = 0, hi = nw - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int)wpre[mid] <= u) lo = mid;
    else hi = mid - 1;
  }
  uint32_t bits = bitmap[lo];
  for (int z = u - (int)wpre[lo]; z > 0; --z) bits &= bits - 1;
  return lo * 32 + (__ffs(bits) - 1);
}

// One warp marks which union columns in [W0, W0 + win) row entries c0 .. c1-1 store: bit
// u - W0 of mrow. Lane L takes a contiguous run of ceil((c1 - c0) / 32) entries, loads them
// kMarkBatch at a time, and ORs the bits of consecutive entries into a register word, writing a
// word out (an atomic OR in shared memory: the runs of two lanes can end in the same word) only
// when it moves to another word. A row's columns are mostly consecutive, so a lane writes one or two
// words where an atomic per entry would serialise the 32 lanes of a warp on one word. Columns
// outside [0, S) are skipped (their rows are flagged by the union pass). Returns, to every lane,
// the number of the row's entries that fall in the window.
constexpr int kMarkBatch = 16;  // a lane's column indices in flight at once (8 measured 1% slower)

struct MarkRun {
  int n = 0;          // entries of the run that fall in the window
  int cur_w = -1;     // word the register bits belong to
  uint32_t cur = 0u;  // bits of word cur_w not yet written out
};

// One entry j of a lane's run: its union index's bit goes into the register word (written out,
// by an atomic OR, when the run moves to another word).
__device__ __forceinline__ void csr_mark_one(MarkRun& m, uint32_t* mrow, const uint32_t* bitmap,
                                             const uint32_t* wpre, int j, int S, int W0, int win) {
  if (j >= 0 && j < S) {
    const int u = csr_union_index(bitmap, wpre, j) - W0;
    if (u >= 0 && u < win) {
      const int w = u >> 5;
      if (w != m.cur_w) {
        if (m.cur_w >= 0) atomicOr(mrow + m.cur_w, m.cur);
        m.cur_w = w;
        m.cur = 0u;
      }
      m.cur |= 1u << (u & 31);
      ++m.n;
    }
  }
}

__device__ __forceinline__ int csr_mark_row(uint32_t* mrow, const uint32_t* bitmap, const uint32_t* wpre,
                                            const int32_t* cols, int c0, int c1, int S, int W0, int win) {
  const int lane = threadIdx.x & 31;
  const int per = (c1 - c0 + 31) >> 5;
  const int e0 = c0 + lane * per, e1 = min(c1, e0 + per);
  MarkRun m;
  for (int eb = e0; eb < e1; eb += kMarkBatch) {
    int jj[kMarkBatch];
#pragma unroll
    for (int z = 0; z < kMarkBatch; ++z) jj[z] = eb + z < e1 ? __ldg(cols + eb + z) : -1;
#pragma unroll
    for (int z = 0; z < kMarkBatch; ++z) csr_mark_one(m, mrow, bitmap, wpre, jj[z], S, W0, win);
  }
  if (m.cur_w >= 0) atomicOr(mrow + m.cur_w, m.cur);
  int n = m.n;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
  return n;
}

// Two rows at once (rows A and B of a warp): the same as csr_mark_row for each, with both rows'
// first batches of column indices in flight together, so that one row's load latency hides the
// other's. Returns the two counts through na and nb (to every lane).
__device__ __forceinline__ void csr_mark_row2(uint32_t* mrow_a, uint32_t* mrow_b, const uint32_t* bitmap,
                                              const uint32_t* wpre, const int32_t* cols, int c0a, int c1a,
                                              int c0b, int c1b, int S, int W0, int win, int& na, int& nb) {
  const int lane = threadIdx.x & 31;
  const int pa = (c1a - c0a + 31) >> 5, pb = (c1b - c0b + 31) >> 5;
  const int ea0 = c0a + lane * pa, ea1 = min(c1a, ea0 + pa);
  const int eb0 = c0b + lane * pb, eb1 = min(c1b, eb0 + pb);
  MarkRun ma, mb;
  int ja[kMarkBatch], jb[kMarkBatch];
#pragma unroll
  for (int z = 0; z < kMarkBatch; ++z) {
    ja[z] = ea0 + z < ea1 ? __ldg(cols + ea0 + z) : -1;
    jb[z] = eb0 + z < eb1 ? __ldg(cols + eb0 + z) : -1;
  }
#pragma unroll
  for (int z = 0; z < kMarkBatch; ++z) csr_mark_one(ma, mrow_a, bitmap, wpre, ja[z], S, W0, win);
#pragma unroll
  for (int z = 0; z < kMarkBatch; ++z) csr_mark_one(mb, mrow_b, bitmap, wpre, jb[z], S, W0, win);
  // entries past the first batch (rows longer than 32 x kMarkBatch), one row after the other
  for (int e = ea0 + kMarkBatch; e < ea1; e += kMarkBatch) {
#pragma unroll
    for (int z = 0; z < kMarkBatch; ++z) ja[z] = e + z < ea1 ? __ldg(cols + e + z) : -1;
#pragma unroll
    for (int z = 0; z < kMarkBatch; ++z) csr_mark_one(ma, mrow_a, bitmap, wpre, ja[z], S, W0, win);
  }
  for (int e = eb0 + kMarkBatch; e < eb1; e += kMarkBatch) {
#pragma unroll
    for (int z = 0; z < kMarkBatch; ++z) jb[z] = e + z < eb1 ? __ldg(cols + e + z) : -1;
#pragma unroll
    for (int z = 0; z < kMarkBatch; ++z) csr_mark_one(mb, mrow_b, bitmap, wpre, jb[z], S, W0, win);
  }
  if (ma.cur_w >= 0) atomicOr(mrow_a + ma.cur_w, ma.cur);
  if (mb.cur_w >= 0) atomicOr(mrow_b + mb.cur_w, mb.cur);
  na = ma.n;
  nb = mb.n;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    na += __shfl_xor_sync(0xffffffffu, na, o);
    nb += __shfl_xor_sync(0xffffffffu, nb, o);
  }
}

}  // namespace sdpa
