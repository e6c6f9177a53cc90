// fwd_f32.cu -- attention forward in float32 on the CUDA cores (the ATTN_F32 path).
//
// O = softmax(scale * Q K^T + mask) V with per-row max / sum statistics, for dense BHSD or
// packed TND batches, GQA/MQA and causal masks ("aclnnFlashAttentionVarLenScore", 功能说明
// and 约束说明; formula of "paddle.nn.functional.sparse_attention"). The torch.nn.attention
// blog notes that fp32 inputs leave the fast flash path; here fp32 keeps full fp32 FMA
// arithmetic (no TF32), so the result stays within 1e-5 of the exact value.
//
// Tiling: a block owns 32 query rows of one (sequence, head); its 4 warps own 8 rows each.
// Key/value tiles of 32 rows are staged in shared memory; lane = key for the scores and
// lane = head-dim column for the P.V accumulation. The softmax is the online (streaming)
// form: the running maximum and sum are rescaled when the maximum grows.
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace sdpa {
namespace {

constexpr int kBM = 32;       // query rows per block
constexpr int kBN = 32;       // keys per tile
constexpr int kWarps = 4;
constexpr int kRowsPerWarp = kBM / kWarps;

template <int DMAX>
__global__ void __launch_bounds__(kWarps * 32) fwd_f32_kernel(FwdArgs a, int tiles_per_seq) {
  extern __shared__ float smem[];
  const int D = a.D, Dv = a.Dv;
  const int ldk = D + 1;  // padded row of the K tile: lane-strided reads avoid bank conflicts
  float* sQ = smem;                       // [kBM][D]
  float* sK = sQ + kBM * D;               // [kBN][D+1]
  float* sV = sK + kBN * ldk;             // [kBN][Dv]
  float* sP = sV + kBN * Dv;              // [kWarps][kRowsPerWarp][kBN]
  __shared__ int s_info[4];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int g = h / (a.Nq / a.Nkv);

  // ---- which (sequence, query tile) this block owns -------------------------------------
  if (warp == 0) {
    int b, t, ok;
    if (a.layout == ATTN_BHSD) {
      b = blockIdx.x / tiles_per_seq;
      t = blockIdx.x - b * tiles_per_seq;
      ok = 1;
    } else {
      bool bad;
      ok = warp_find_tile(a.cu_q, a.B, a.Sq, kBM, blockIdx.x, &b, &t, a.status, &bad);
      if (!ok && !bad && blockIdx.y == 0) {
        // a block past the last tile checks the key-side lengths for everyone
        int seq, tis;
        bool bad2;
        warp_find_tile(a.cu_kv, a.B, a.Skv, 1 << 30, 1 << 30, &seq, &tis, a.status, &bad2);
      }
    }
    if (lane == 0) {
      s_info[0] = ok;
      s_info[1] = b;
      s_info[2] = t;
    }
  }
  __syncthreads();
  if (!s_info[0]) return;
  const int b = s_info[1], qt = s_info[2];

  int q0, sq, k0, sk;  // token offsets and lengths of this sequence
  if (a.layout == ATTN_BHSD) {
    q0 = 0;
    sq = a.Sq;
    k0 = 0;
    sk = a.Skv;
  } else {
    seq_span(a.cu_q, b, &q0, &sq);
    seq_span(a.cu_kv, b, &k0, &sk);
    if (k0 < 0 || sk < 0 || k0 + sk > a.Skv) {
      if (threadIdx.x == 0) report(a.status, ATTN_ERR_DATA);
      return;
    }
  }
  const float* Q = (const float*)a.q;
  const float* K = (const float*)a.k;
  const float* V = (const float*)a.v;
  // element (token i of this sequence, head, d)
  auto qoff = [&](int i) -> int64_t {
    return a.layout == ATTN_BHSD ? (((int64_t)b * a.Nq + h) * a.Sq + i) * D
                                 : ((int64_t)(q0 + i) * a.Nq + h) * D;
  };
  auto kvoff = [&](int j) -> int64_t {
    return a.layout == ATTN_BHSD ? (((int64_t)b * a.Nkv + g) * a.Skv + j) * D
                                 : ((int64_t)(k0 + j) * a.Nkv + g) * D;
  };
  // value rows and output rows have Dv columns
  auto voff = [&](int j) -> int64_t {
    return a.layout == ATTN_BHSD ? (((int64_t)b * a.Nkv + g) * a.Skv + j) * Dv
                                 : ((int64_t)(k0 + j) * a.Nkv + g) * Dv;
  };
  auto ooff = [&](int i) -> int64_t {
    return a.layout == ATTN_BHSD ? (((int64_t)b * a.Nq + h) * a.Sq + i) * Dv
                                 : ((int64_t)(q0 + i) * a.Nq + h) * Dv;
  };
  const uint8_t* mrow0 = a.mask != nullptr ? a.mask + (int64_t)b * a.mask_bs : nullptr;

  const int row0 = qt * kBM;
  const int nrows = min(kBM, sq - row0);
  // stage Q (rows past the sequence end are zero-filled)
  for (int x = threadIdx.x; x < kBM * D; x += blockDim.x) {
    const int r = x / D, d = x - r * D;
    sQ[x] = r < nrows ? Q[qoff(row0 + r) + d] : 0.f;
  }

  // keys needed by the tile: from the first row's first visible key to the last row's last
  const int kv_end = visible_end(a.mask_mode, row0 + nrows - 1, sq, sk, a.next);
  const int kv_begin = visible_begin(a.mask_mode, row0, a.pre) / kBN * kBN;

  constexpr int DT = DMAX / 32;  // head-dim columns per lane
  float acc[kRowsPerWarp][DT];
  float m[kRowsPerWarp], l[kRowsPerWarp];
  int vbeg[kRowsPerWarp], vend[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
    const int i = row0 + warp * kRowsPerWarp + r;
    vend[r] = i < sq ? visible_end(a.mask_mode, i, sq, sk, a.next) : 0;
    vbeg[r] = visible_begin(a.mask_mode, i, a.pre);
#pragma unroll
    for (int t = 0; t < DT; ++t) acc[r][t] = 0.f;
  }

  for (int j0 = kv_begin; j0 < kv_end; j0 += kBN) {
    __syncthreads();  // previous tile fully consumed (and Q staged on the first pass)
    for (int x = threadIdx.x; x < kBN * D; x += blockDim.x) {
      const int r = x / D, d = x - r * D;
      const bool in = j0 + r < sk;
      sK[r * ldk + d] = in ? K[kvoff(j0 + r) + d] : 0.f;
    }
    for (int x = threadIdx.x; x < kBN * Dv; x += blockDim.x) {
      const int r = x / Dv, d = x - r * Dv;
      sV[x] = j0 + r < sk ? V[voff(j0 + r) + d] : 0.f;
    }
    __syncthreads();

    // scores: lane = key j0 + lane, one value per row of this warp
    float s[kRowsPerWarp];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) s[r] = 0.f;
    const float* kr = sK + lane * ldk;
    const float* qr = sQ + warp * kRowsPerWarp * D;
    for (int d = 0; d < D; ++d) {
      const float kv = kr[d];
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) s[r] = fmaf(qr[r * D + d], kv, s[r]);
    }
    const int j = j0 + lane;
    float* pw = sP + warp * kRowsPerWarp * kBN;
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int i = row0 + warp * kRowsPerWarp + r;
      bool vis = j >= vbeg[r] && j < vend[r];
      if (vis && mrow0 != nullptr) vis = mrow0[(int64_t)i * a.mask_rs + j] == 0;
      const float sc = vis ? s[r] * a.scale : -INFINITY;
      float mx = sc;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float mnew = fmaxf(m[r], mx);
      float p = 0.f, corr = 1.f;
      if (mnew != -INFINITY) {
        p = vis ? expf(sc - mnew) : 0.f;
        corr = m[r] == -INFINITY ? 0.f : expf(m[r] - mnew);
      }
      float ps = p;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      l[r] = l[r] * corr + ps;
      m[r] = mnew;
#pragma unroll
      for (int t = 0; t < DT; ++t) acc[r][t] *= corr;
      pw[r * kBN + lane] = p;
    }
    __syncwarp();
    // P.V: lane owns head-dim columns lane, lane+32, ...
    for (int jj = 0; jj < kBN; ++jj) {
      const float* vr = sV + jj * Dv;
      float vv[DT];
#pragma unroll
      for (int t = 0; t < DT; ++t) vv[t] = (lane + 32 * t) < Dv ? vr[lane + 32 * t] : 0.f;
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) {
        const float p = pw[r * kBN + jj];
#pragma unroll
        for (int t = 0; t < DT; ++t) acc[r][t] = fmaf(p, vv[t], acc[r][t]);
      }
    }
    __syncwarp();
  }

  // ---- epilogue ---------------------------------------------------------------------------
  float* O = (float*)a.out;
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int i = row0 + warp * kRowsPerWarp + r;
    if (i >= sq) continue;  // warp-uniform
    const bool any = l[r] > 0.f;
    const float m_loc = any ? m[r] : -INFINITY;
    const float l_loc = l[r];
    float f_o = any ? 1.f / l[r] : 0.f;
    float f_prev = 0.f;
    int64_t o;
    if (a.acc_mode == 0) {
      o = ooff(i);
      if (lane == 0 && a.smax != nullptr) {
        const int64_t so = a.layout == ATTN_BHSD ? ((int64_t)b * a.Nq + h) * a.Sq + i
                                                 : (int64_t)(q0 + i) * a.Nq + h;
        a.smax[so] = m_loc;
        a.ssum[so] = l_loc;
      }
    } else {
      // accumulator in the merge layouts: BHSD -> output [Sq, B, Nq*D] (SBH), statistics
      // [B, Nq, Sq, 8]; TND -> output [T, Nq*D], statistics [T, Nq, 8]. Lanes 0-7 update the
      // 8 statistic lanes ("npu_ring_attention_update", 小算子等价计算逻辑); lane 0's factors
      // rescale the output row.
      o = a.layout == ATTN_BHSD ? (((int64_t)i * a.B + b) * a.Nq + h) * D : qoff(i);
      const int64_t so = (a.layout == ATTN_BHSD ? ((int64_t)b * a.Nq + h) * a.Sq + i
                                                : (int64_t)(q0 + i) * a.Nq + h) * 8;
      float ps2 = 0.f, cs2 = 0.f, nl = 0.f;
      if (lane < 8) {
        if (a.acc_mode == 1) {
          a.smax[so + lane] = m_loc;
          a.ssum[so + lane] = l_loc;
          cs2 = l_loc;
          nl = l_loc;
        } else {
          const float pm = a.smax[so + lane], ps = a.ssum[so + lane];
          const float mk = fmaxf(pm, m_loc);
          if (mk != -INFINITY) {
            ps2 = ps * expf(pm - mk);
            cs2 = l_loc * expf(m_loc - mk);
          }
          nl = ps2 + cs2;
          a.smax[so + lane] = mk;
          a.ssum[so + lane] = nl;
        }
      }
      ps2 = __shfl_sync(0xffffffffu, ps2, 0);
      cs2 = __shfl_sync(0xffffffffu, cs2, 0);
      nl = __shfl_sync(0xffffffffu, nl, 0);
      const float inv = nl != 0.f ? 1.f / nl : 0.f;
      f_prev = a.acc_mode == 1 ? 0.f : ps2 * inv;
      f_o = a.acc_mode == 1 ? f_o : f_o * cs2 * inv;
    }
#pragma unroll
    for (int t = 0; t < DT; ++t) {
      const int d = lane + 32 * t;
      if (d < Dv) {
        float v = acc[r][t] * f_o;
        if (a.acc_mode == 2) v = fmaf(O[o + d], f_prev, v);
        O[o + d] = v;
      }
    }
  }
}

template <int DMAX>
cudaError_t launch_dmax(const FwdArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(float) * (size_t)(kBM * a.D + kBN * (a.D + 1) + kBN * a.Dv +
                                              kWarps * kRowsPerWarp * kBN);
  cudaError_t e = cudaFuncSetAttribute(fwd_f32_kernel<DMAX>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int tiles_per_seq = 0;
  int64_t gx;
  if (a.layout == ATTN_BHSD) {
    tiles_per_seq = (a.Sq + kBM - 1) / kBM;
    gx = (int64_t)a.B * tiles_per_seq;
  } else {
    gx = (a.Sq + kBM - 1) / kBM + a.B;  // upper bound on the tiles of a packed batch
  }
  if (gx <= 0) return cudaSuccess;
  dim3 grid((unsigned)gx, a.Nq);
  fwd_f32_kernel<DMAX><<<grid, kWarps * 32, smem, st>>>(a, tiles_per_seq);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_f32(const FwdArgs& a, cudaStream_t st) {
  if (a.D <= 64) return launch_dmax<64>(a, st);
  if (a.D <= 128) return launch_dmax<128>(a, st);
  return launch_dmax<256>(a, st);
}

}  // namespace sdpa
