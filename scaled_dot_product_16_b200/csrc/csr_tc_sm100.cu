// csr_tc_sm100.cu -- CSR-sparse attention forward on the tcgen05 tensor cores (bf16 / fp16).
//
// "paddle.nn.functional.sparse_attention" (Paddle 2.3 API doc), formula and 参数: for every
// (b, h, i) the softmax of q_i . k_j / sqrt(D) runs over the stored entries of row i of that
// (b, h) slice (offset = row pointer [B,H,S+1], columns [B,H,nnz]) and weights the rows v_j.
//
// Design (tiles of the CSR pattern, gathered):
//   * a block owns 128 query rows of one (b, h); row r is TMEM lane r and softmax thread r;
//   * the block first takes the union of the columns its rows store (csr_union.cuh): a bitmap
//     over the S keys with an exclusive prefix of its words' popcounts, built from one streamed
//     pass over the block's column indices. Union column u is the u-th set bit, so the union
//     is sorted and each key appears once;
//   * two producer warps gather the union's key and value rows, 128 per tile, with 16-byte
//     cp.async into the 128-byte-swizzled K-major layout the MMA descriptors expect (the same
//     layout a TMA load with 128-byte swizzle gives), zero-filling past the union's end;
//   * one thread issues S = Q K_t^T (both operands in shared memory) into one of two TMEM score
//     buffers, and O += P_t V_t with P read from TMEM; S_{t+1} overlaps the softmax of tile t;
//   * each row keeps a byte per union column of the current window (512 columns at D = 64, 256
//     at D = 128) that says whether the column is one of its entries, built by the row's own
//     softmax thread from its own columns, 16 loads deep; the softmax sets the other scores to
//     -inf, so every row sums over exactly its own entries, with the online (streaming) update
//     and a lazy rescale;
//   * P is written to TMEM as a 16-bit high part and a 16-bit remainder, and O accumulates both
//     (two MMAs per key step): rows with few entries put large weights on few values, where a
//     single 16-bit P would cost up to 2^-9 of |v| on top of the output's own rounding;
//   * every wait is bounded; a timeout records ATTN_ERR_TIMEOUT and the block drains and exits.
// A column stored twice in one row would be counted once by the byte mask, so a repeated
// column is reported as ATTN_ERR_DATA and that row is written as zeros.
#include <math.h>

#include "common.cuh"
#include "csr_plan.cuh"
#include "csr_union.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace sdpa {
namespace {

using namespace sm100;

constexpr int kRows = 128;       // query rows per block
constexpr int kKeys = 128;       // gathered keys per tile
constexpr int kMmaWarp = 4;
constexpr int kProdWarp = 5;     // warps 5 and 6 gather
constexpr int kThreads = 7 * 32;
constexpr int kMaxS = 32768;
constexpr int kTmemCols = 512;   // S0 [0,128), S1 [128,256), O [256, 256+D)
constexpr int kRescaleThreshold = 8;
constexpr uint64_t kWaitLimitNs = 200ull * 1000 * 1000;
constexpr uint32_t kSuspendNs = 20000;

template <int HD, bool F16>
struct CsrCfg {
  static constexpr int kTileBytes = kKeys * HD * 2;       // a Q, K or V tile
  static constexpr int kStages = HD == 64 ? 4 : 2;        // K/V ring depth (even: fixed owner warp)
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = kTileBytes;               // stage s: K, then V
  static constexpr int kBitmapOff = kKVOff + 2 * kStages * kTileBytes;
  static constexpr int kPrefixOff = kBitmapOff + kMaxS / 8;
  // union columns whose per-row bytes are held at once, and the padded row of those bytes
  // (16-byte reads of consecutive rows then fall in different banks)
  static constexpr int kWin = HD == 64 ? 512 : 256;
  static constexpr int kWinStride = kWin + 16;
  // a byte per column while the union is taken, then the rows' byte masks [kRows][kWinStride]
  static constexpr int kBytesOff = kPrefixOff + kMaxS / 8;
  static constexpr int kBytesSize = kMaxS > kRows * kWinStride ? kMaxS : kRows * kWinStride;
  static constexpr int kColOff = kBytesOff + kBytesSize;
  static constexpr int kRowOff = kColOff + kStages * kKeys * 4;  // c0, c1, bad flag per row
  static constexpr int kMiscOff = kRowOff + 3 * kRows * 4;
  static constexpr int kBarOff = kMiscOff + 16;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;
  static_assert(kSmemBytes <= 232448, "227 KB of shared memory per block");
  static constexpr uint32_t kFmt = F16 ? 0u : 1u;
  static constexpr uint32_t kIdescQK = idesc_f16_f32(kRows, kKeys, 0, 0, kFmt);
  static constexpr uint32_t kIdescPV = idesc_f16_f32(kRows, HD, 0, 1, kFmt);
};

struct CsrBarriers {
  uint64_t full[4];
  uint64_t empty[4];
  uint64_t q_full;
  uint64_t s_full[2];
  uint64_t p_ready[2];
  uint64_t pv_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort,
                                         int* status, bool heed_abort = true) {
  if (mbar_try_wait_sleep(bar, parity, kSuspendNs)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, kSuspendNs)) return true;
    if (heed_abort && *abort) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort = 1;
      report(status, ATTN_ERR_TIMEOUT);
      return false;
    }
  }
}

constexpr int kRowBatch = 16;   // a row's column indices its thread loads before using any

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Copy 128 rows of HD 16-bit elements into a 128-byte-swizzled K-major tile: row k, 16-byte
// chunk c of 64-element atom x lands at x*16KB + k*128 + ((c ^ (k & 7)) * 16). Row k comes from
// src_row(k), or is zero-filled when that is null (any_row is a valid address nothing reads).
template <int HD, typename RowFn>
__device__ __forceinline__ void gather_tile(uint32_t dst, RowFn src_row, const uint16_t* any_row, int lane) {
  constexpr int kChunks = HD / 8;  // 16-byte chunks per row
  for (int x = lane; x < kKeys * kChunks; x += 32) {
    const int k = x / kChunks, c = x % kChunks;
    const int atom = c >> 3, cc = c & 7;
    const uint16_t* row = src_row(k);
    const uint32_t d = dst + atom * (kKeys * 128) + k * 128 + ((cc ^ (k & 7)) << 4);
    cp_async16(d, row != nullptr ? row + c * 8 : any_row, row != nullptr);  // zero-filled if null
  }
}

// PLANNED: the union list, the rows' marks and the bad rows come from a plan of the pattern
// (csr_plan.cuh) instead of being built here; the block then only gathers and multiplies.
template <int HD, bool F16, bool PLANNED>
__global__ void __launch_bounds__(kThreads, 1) csr_tc_kernel(CsrTcArgs a, float scale_log2) {
  using C = CsrCfg<HD, F16>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + C::kBitmapOff);
  uint32_t* wpre = reinterpret_cast<uint32_t*>(smem + C::kPrefixOff);
  uint8_t* bytes = smem + C::kBytesOff;
  int* kcol = reinterpret_cast<int*>(smem + C::kColOff);
  int* misc = reinterpret_cast<int*>(smem + C::kMiscOff);
  int* row_c0 = reinterpret_cast<int*>(smem + C::kRowOff);
  int* row_c1 = row_c0 + kRows;
  int* row_bad = row_c1 + kRows;
  CsrBarriers* bars = reinterpret_cast<CsrBarriers*>(smem + C::kBarOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.S;
  const int tiles_q = (S + kRows - 1) / kRows;
  const int64_t bh = blockIdx.x / tiles_q;
  const int r0 = (int)(blockIdx.x - bh * tiles_q) * kRows;
  const int32_t* off = PLANNED ? nullptr : a.offset + bh * (int64_t)(S + 1);
  const int32_t* cols = PLANNED ? nullptr : a.columns + bh * a.nnz_cap;
  const uint16_t* Qb = static_cast<const uint16_t*>(a.q) + bh * (int64_t)S * HD;
  const uint16_t* Kb = static_cast<const uint16_t*>(a.k) + bh * (int64_t)S * HD;
  const uint16_t* Vb = static_cast<const uint16_t*>(a.v) + bh * (int64_t)S * HD;
  const int nw = (S + 31) >> 5;

  // ---- setup: barriers, TMEM, empty bitmap ---------------------------------------------------
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 32);  // every lane of the filling warp
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->q_full), 32);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bars->s_full[b]), 1);
      mbar_init(smem_u32(&bars->p_ready[b]), 4);
    }
    mbar_init(smem_u32(&bars->pv_done), 1);
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if constexpr (!PLANNED)
    for (int w = threadIdx.x; w < nw * 8; w += kThreads) reinterpret_cast<uint32_t*>(bytes)[w] = 0u;
  for (int x = threadIdx.x; x < kRows; x += kThreads) row_bad[x] = 0;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  // ---- the union of the block's rows' columns (csr_union.cuh), or the plan's ------------------
  const int r = warp * 32 + lane;
  const int i = r0 + r;
  const int32_t* plan_cols = nullptr;  // PLANNED: the block's union list
  const uint4* plan_marks = nullptr;   // PLANNED: [tile][row] marks
  int U;
  if constexpr (PLANNED) {
    const int64_t ucap = plan_ucap(S, a.nnz_cap);
    const uint8_t* rec = a.plan + (int64_t)blockIdx.x * plan_block_bytes(S, a.nnz_cap);
    plan_cols = reinterpret_cast<const int32_t*>(rec + kPlanHeader);
    plan_marks = reinterpret_cast<const uint4*>(rec + kPlanHeader + 4 * ucap);
    if (threadIdx.x < kRows) {
      const PlanHeader* h = reinterpret_cast<const PlanHeader*>(rec);
      // a record that is not a plan of this shape gives zeros and ATTN_ERR_DATA, and nothing
      // it holds is used as an index
      const bool valid = h->magic == kPlanMagic && h->S == S && h->ucap == (int32_t)ucap &&
                         h->U >= 0 && h->U <= ucap;
      row_bad[threadIdx.x] = !valid || ((h->bad[threadIdx.x >> 5] >> (threadIdx.x & 31)) & 1u);
      if (threadIdx.x == 0) {
        misc[0] = valid ? h->U : 0;
        if (!valid) report(a.status, ATTN_ERR_DATA);
      }
    }
    __syncthreads();
    U = misc[0];
  } else {
    const CsrUnion un{bitmap, wpre, bytes, row_c0, row_c1, row_bad, misc};
    U = csr_block_union<kThreads, kRows>(un, off, cols, S, r0, a.nnz_cap, a.cols_vec, a.status);
  }
  const int T = (U + kKeys - 1) / kKeys;  // gathered key tiles

  const uint32_t sQ = smem_u32(smem + C::kQOff);
  auto sK = [&](int s) { return smem_u32(smem + C::kKVOff + 2 * s * C::kTileBytes); };
  auto sV = [&](int s) { return smem_u32(smem + C::kKVOff + (2 * s + 1) * C::kTileBytes); };

  if (warp >= kProdWarp) {
    // =============================== gather producers ====================================
    const int p = warp - kProdWarp;
    auto union_col = [&](int u) { return csr_union_col(bitmap, wpre, nw, u); };
    bool ok = true;
    if (p == 0 && T > 0) {
      gather_tile<HD>(sQ, [&](int k) { return r0 + k < S ? Qb + (int64_t)(r0 + k) * HD : nullptr; }, Qb, lane);
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&bars->q_full));
    }
    for (int t = p; ok && t < T; t += 2) {
      const int s = t % C::kStages;
      if (t >= C::kStages &&
          !(ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&bars->empty[s]), ((t / C::kStages) - 1) & 1, abort, a.status))))
        break;
      int* kc = kcol + s * kKeys;
#pragma unroll
      for (int m = 0; m < kKeys / 32; ++m) {
        const int u = t * kKeys + m * 32 + lane;
        if constexpr (PLANNED) {
          int c = u < U ? __ldg(plan_cols + u) : -1;
          if (c >= S) {  // not a column of this pattern: the plan was built for another one
            report(a.status, ATTN_ERR_DATA);
            c = -1;
          }
          kc[m * 32 + lane] = c;
        } else {
          kc[m * 32 + lane] = u < U ? union_col(u) : -1;
        }
      }
      __syncwarp();
      gather_tile<HD>(sK(s), [&](int k) { return kc[k] >= 0 ? Kb + (int64_t)kc[k] * HD : nullptr; }, Kb, lane);
      gather_tile<HD>(sV(s), [&](int k) { return kc[k] >= 0 ? Vb + (int64_t)kc[k] * HD : nullptr; }, Vb, lane);
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&bars->full[s]));
    }
    cp_async_wait_all();
  } else if (warp == kMmaWarp) {
    // =============================== MMA issue ============================================
    if (lane == 0 && T > 0) {
      const uint32_t Sb[2] = {tmem, tmem + 128};
      const uint32_t O = tmem + 256;
      const uint64_t dq = smem_desc_sw128(sQ, 16, 1024);
      auto issue_s = [&](int t) {
        const int s = t % C::kStages;
        const uint64_t dk = smem_desc_sw128(sK(s), 16, 1024);
        if constexpr (HD == 128)
          mma_ss_chain8(Sb[t & 1], dq, dk, C::kIdescQK, 0u);
        else
          mma_ss_chain4(Sb[t & 1], dq, dk, C::kIdescQK, 0u);
        mma_commit(smem_u32(&bars->s_full[t & 1]));
      };
      auto full = [&](int t) {
        return wait_bar(smem_u32(&bars->full[t % C::kStages]), (t / C::kStages) & 1, abort, a.status);
      };
      bool ok = wait_bar(smem_u32(&bars->q_full), 0, abort, a.status);
      if (ok && (ok = full(0))) {
        tc_fence_after();
        issue_s(0);
      }
      if (ok && T > 1 && (ok = full(1))) {
        tc_fence_after();
        issue_s(1);
      }
      for (int t = 0; ok && t < T; ++t) {
        if (!(ok = wait_bar(smem_u32(&bars->p_ready[t & 1]), (t >> 1) & 1, abort, a.status))) break;
        tc_fence_after();
        const int s = t % C::kStages;
        const uint64_t dv = smem_desc_sw128(sV(s), kKeys * 128, 1024);
        mma_ts_chain8(O, Sb[t & 1], dv, C::kIdescPV, t > 0 ? 1u : 0u);
        mma_ts_chain8(O, Sb[t & 1] + 64, dv, C::kIdescPV, 1u);  // the remainder of P
        mma_commit(smem_u32(&bars->pv_done));
        mma_commit(smem_u32(&bars->empty[s]));
        if (t + 2 < T) {
          if (!(ok = full(t + 2))) break;
          tc_fence_after();
          issue_s(t + 2);
        }
      }
      if (!ok) *abort = 1;
      mma_commit(smem_u32(&bars->drain));
      wait_bar(smem_u32(&bars->drain), 0, abort, a.status, false);
    }
  } else {
    // =============================== softmax + epilogue ===================================
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t O = tmem + lane_off + 256;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      uint4 pmark = make_uint4(0u, 0u, 0u, 0u);
      if constexpr (PLANNED) pmark = __ldg(plan_marks + (int64_t)t * kRows + r);  // before the waits
      if (!PLANNED && (t * kKeys) % C::kWin == 0) {
        // this row's bytes for union columns [t*128, t*128 + kWin): the thread reads its own
        // row's columns (16 at a time) and marks its own bytes, so no other thread is involved
        const int base = t * kKeys;
        uint8_t* row = bytes + r * C::kWinStride;
#pragma unroll
        for (int x = 0; x < C::kWin / 16; ++x) reinterpret_cast<uint4*>(row)[x] = make_uint4(0u, 0u, 0u, 0u);
        const int e1 = row_c1[r];
        int hits = 0;
        for (int e0 = row_c0[r]; e0 < e1; e0 += kRowBatch) {
          int jj[kRowBatch];
#pragma unroll
          for (int b = 0; b < kRowBatch; ++b) jj[b] = e0 + b < e1 ? __ldg(cols + e0 + b) : -1;
#pragma unroll
          for (int b = 0; b < kRowBatch; ++b) {
            const int j = jj[b];
            if (j >= 0 && j < S) {  // bad columns are already flagged; the row is zeroed
              const int u = csr_union_index(bitmap, wpre, j);
              if (u >= base && u < base + C::kWin) {
                row[u - base] = 1;
                ++hits;
              }
            }
          }
        }
        // distinct columns <=> as many marked bytes as entries in the window
        int set = 0;
#pragma unroll 4
        for (int x = 0; x < C::kWin / 16; ++x) {
          const uint4 v = reinterpret_cast<const uint4*>(row)[x];
          set += (__popc(__vcmpne4(v.x, 0u)) + __popc(__vcmpne4(v.y, 0u)) + __popc(__vcmpne4(v.z, 0u)) +
                  __popc(__vcmpne4(v.w, 0u))) / 8;
        }
        if (set != hits && row_bad[r] == 0) {  // the same column stored twice in this row
          row_bad[r] = 1;
          report(a.status, ATTN_ERR_DATA);
        }
      }
      if (ok) ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&bars->s_full[t & 1]), (t >> 1) & 1, abort, a.status));
      if (ok && t > 0)
        ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&bars->pv_done), (t - 1) & 1, abort, a.status));
      if (!ok) break;
      tc_fence_after();
      const uint32_t Sa = tmem + lane_off + (t & 1) * 128;
      float s[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32f(Sa + c * 32, s[c]);
      tmem_wait_ld();
      if constexpr (PLANNED) {
        // this row's marks for the tile's 128 union columns: bit c of word x = column 32x + c
        const uint32_t wd[4] = {pmark.x, pmark.y, pmark.z, pmark.w};
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (((wd[x] >> c) & 1u) == 0u) s[x][c] = -INFINITY;
      } else {
        // this row's bytes for the tile's 128 union columns
        const uint4* mb = reinterpret_cast<const uint4*>(bytes + r * C::kWinStride + (t * kKeys) % C::kWin);
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const uint4 v = mb[x];
          const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int y = 0; y < 16; ++y)
            if (((wd[y >> 2] >> (8 * (y & 3))) & 0xffu) == 0u) s[(x * 16 + y) >> 5][(x * 16 + y) & 31] = -INFINITY;
        }
      }
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int x = 0; x < 32; x += 2) tmax = fmax3(tmax, s[c][x], s[c][x + 1]);
      const float tmax2 = tmax * scale_log2;
      const bool bump = tmax2 > m + kRescaleThreshold;  // also true for the first finite max
      float corr = 1.f;
      if (bump) {
        corr = (m == -INFINITY) ? 0.f : ex2(m - tmax2);
        m = tmax2;
        l *= corr;
      }
      const float muse = m == -INFINITY ? 0.f : m;
      uint32_t pk[2][32], pl[2][32];  // P's 16-bit high part and remainder
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < kKeys; c += 2) {
        const float p0 = ex2(fmaf(s[c >> 5][c & 31], scale_log2, -muse));
        const float p1 = ex2(fmaf(s[c >> 5][(c + 1) & 31], scale_log2, -muse));
        rs += p0 + p1;
        const uint32_t hi = pack16x2<F16>(p0, p1);
        const float2 h = unpack16x2<F16>(hi);
        pk[c >> 6][(c >> 1) & 31] = hi;
        pl[c >> 6][(c >> 1) & 31] = pack16x2<F16>(p0 - h.x, p1 - h.y);
      }
      l += rs;
      // rescale O (complete through tile t-1: pv_done was waited for above)
      if (__any_sync(0xffffffffu, bump && t > 0)) {
        const float f = (bump && t > 0) ? corr : 1.f;
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(O + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * f);
          tmem_st32(O + c * 32, o);
        }
      }
      tmem_st32(Sa, pk[0]);
      tmem_st32(Sa + 32, pk[1]);
      tmem_st32(Sa + 64, pl[0]);
      tmem_st32(Sa + 96, pl[1]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->p_ready[t & 1]));
    }
    // ---- epilogue: O / l -> 16-bit output row ----------------------------------------------
    if (ok && T > 0)
      ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&bars->pv_done), (T - 1) & 1, abort, a.status));
    tc_fence_after();
    {
      // the TMEM loads are warp-wide: every lane loads, rows past the end do not store
      const bool row_ok = i < S && row_bad[r] == 0;
      const float f = (ok && row_ok && l > 0.f) ? 1.f / l : 0.f;
      uint16_t* out = static_cast<uint16_t*>(a.out) + (bh * (int64_t)S + i) * HD;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t o[32];
        if (ok && T > 0) {
          tmem_ld32(O + c * 32, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = 0u;
        }
        if (i < S) {
          uint32_t pkd[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const float v0 = f == 0.f ? 0.f : __uint_as_float(o[2 * x]) * f;
            const float v1 = f == 0.f ? 0.f : __uint_as_float(o[2 * x + 1]) * f;
            pkd[x] = pack16x2<F16>(v0, v1);
          }
          uint4* dst = reinterpret_cast<uint4*>(out + c * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x)
            dst[x] = make_uint4(pkd[4 * x], pkd[4 * x + 1], pkd[4 * x + 2], pkd[4 * x + 3]);
        }
      }
    }
  }

  // ---- teardown -----------------------------------------------------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int HD, bool F16, bool PLANNED>
cudaError_t launch_hd(const CsrTcArgs& a, cudaStream_t st) {
  using C = CsrCfg<HD, F16>;
  auto kernel = csr_tc_kernel<HD, F16, PLANNED>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)a.B * a.H * ((a.S + kRows - 1) / kRows);
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const float scale_log2 = (1.0f / sqrtf((float)HD)) * 1.4426950408889634f;
  kernel<<<(unsigned)blocks, kThreads, C::kSmemBytes, st>>>(a, scale_log2);
  return cudaGetLastError();
}

template <bool PLANNED>
cudaError_t launch_tc(const CsrTcArgs& a, cudaStream_t st) {
  const bool f16 = a.dtype == ATTN_F16;
  if (a.D == 128) return f16 ? launch_hd<128, true, PLANNED>(a, st) : launch_hd<128, false, PLANNED>(a, st);
  return f16 ? launch_hd<64, true, PLANNED>(a, st) : launch_hd<64, false, PLANNED>(a, st);
}

}  // namespace

cudaError_t launch_sparse_csr_tc(const CsrTcArgs& a, cudaStream_t st) {
  return a.plan != nullptr ? launch_tc<true>(a, st) : launch_tc<false>(a, st);
}

}  // namespace sdpa
