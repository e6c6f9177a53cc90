// merge.cu -- merge of two partial attention results from their softmax statistics.
//
// "npu_ring_attention_update" (MindSpeed op doc), 小算子等价计算逻辑: per statistic lane,
//   m = max(pm, cm), ps' = ps * exp(pm - m), cs' = cs * exp(cm - m), l = ps' + cs',
// and out = prev * (ps'_0 / l_0) + cur * (cs'_0 / l_0) with lane 0 of each (b, n, s) row.
//
// SBH layout: outputs [S, B, N*D]; statistics [B, N, S, 8] fp32. TND layout: outputs
// [T, N*D]; statistics [T, N, 8] fp32 (rows t*N + n, contiguous in both).
//
// The kernel is HBM-bound (about 1 GB moved per call at S=8192, B=4, N=32, D=128), so the
// design is about access shape and bytes in flight only:
//   * one block owns a few consecutive s of one (b, n): its statistics are rows*8 contiguous
//     floats per array (one coalesced load per thread), and every output row is D contiguous
//     elements (D*2 = 256 B for bf16, D = 128);
//   * every thread issues all of its output loads before the statistics phase, so the block
//     barrier that hands over the lane-0 scales overlaps the bulk loads;
//   * blocks are small (8 rows, 64 threads): in a sweep of block shapes on B200 this reached
//     79 % of the measured copy bandwidth, against 67 % for 64-row blocks, because many small
//     independent blocks keep more requests in flight;
//   * the outputs move as 32-byte accesses that do not allocate in L1 when every output base
//     is 32-byte aligned (one load per input and one store per thread and row chunk, against
//     two 16-byte ones): 0.162 against 0.176 ms for SBH 8192 x 4 x 32 x 128 bf16, 95 % of the
//     measured copy bandwidth.
#include <cuda_fp16.h>

#include "common.cuh"
#include "launch.h"

namespace sdpa {
namespace {

constexpr int kRows = 32;     // s rows per block (generic path)
constexpr int kThreads = 256;
// Vectorised path block shape: rows per block, threads, 16-byte vectors per thread and input.
#ifndef SDPA_MERGE_ROWS
#define SDPA_MERGE_ROWS 8
#endif
#ifndef SDPA_MERGE_THREADS
#define SDPA_MERGE_THREADS 64
#endif
#ifndef SDPA_MERGE_PER
#define SDPA_MERGE_PER 2
#endif

template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int n = 8;
};
template <>
struct Vec16<float> {
  static constexpr int n = 4;
};
template <>
struct Vec16<__half> {
  static constexpr int n = 8;
};

__device__ __forceinline__ void unpack(const uint4& u, float* f, __nv_bfloat16*) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void unpack(const uint4& u, float* f, __half*) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void unpack(const uint4& u, float* f, float*) {
  f[0] = __uint_as_float(u.x);
  f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z);
  f[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ uint4 pack(const float* f, __nv_bfloat16*) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return u;
}
__device__ __forceinline__ uint4 pack(const float* f, __half*) {
  uint4 u;
  __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
  return u;
}
__device__ __forceinline__ uint4 pack(const float* f, float*) {
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                    __float_as_uint(f[3]));
}

__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
__device__ __forceinline__ void from_f(float x, __half* p) { *p = __float2half_rn(x); }
__device__ __forceinline__ void from_f(float x, __nv_bfloat16* p) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ void from_f(float x, float* p) { *p = x; }

// 32-byte global accesses that do not allocate in L1 (every byte of the merge is touched once).
__device__ __forceinline__ void ld32_na(const void* p, uint4& lo, uint4& hi) {
  asm volatile("ld.global.L1::no_allocate.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
               : "l"(p));
}
__device__ __forceinline__ void st32_na(void* p, const uint4& lo, const uint4& hi) {
  asm volatile("st.global.L1::no_allocate.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(lo.x),
               "r"(lo.y), "r"(lo.z), "r"(lo.w), "r"(hi.x), "r"(hi.y), "r"(hi.z), "r"(hi.w)
               : "memory");
}

// Lane-wise statistics update; returns the lane's scaled partial sums.
__device__ __forceinline__ void merge_lane(float pm, float ps, float cm, float cs, float* m,
                                           float* ps2, float* cs2) {
  const float mx = fmaxf(pm, cm);
  if (mx == -INFINITY) {  // both partials empty
    *m = mx;
    *ps2 = 0.f;
    *cs2 = 0.f;
    return;
  }
  *m = mx;
  *ps2 = ps * expf(pm - mx);
  *cs2 = cs * expf(cm - mx);
}

// Generic path: a block of ROWS = 32 rows loads the statistics, then the outputs.
// VEC: true when D is a multiple of the 16-byte vector width and the row bases stay aligned.
template <typename T, bool VEC, bool FLAT>
__global__ void __launch_bounds__(kThreads) merge_sbh_kernel(
    const T* prev_out, const float* prev_max, const float* prev_sum,  // may alias the outputs
    const T* __restrict__ cur_out,
    const float* __restrict__ cur_max, const float* __restrict__ cur_sum, int S, int B, int N,
    int D, T* out, float* out_max, float* out_sum) {
  __shared__ float s_po[kRows], s_co[kRows];
  // SBH: block (b*N + n, s-block); FLAT (TND): block = kRows consecutive rows t*N + n
  const int bn = FLAT ? 0 : blockIdx.x;
  const int b = FLAT ? 0 : bn / N, n = FLAT ? 0 : bn - b * N;
  const int64_t s0 = FLAT ? (int64_t)blockIdx.x * kRows : (int64_t)blockIdx.y * kRows;
  const int64_t nrow_all = FLAT ? (int64_t)S * N : (int64_t)S;
  const int rows = (int)min((int64_t)kRows, nrow_all - s0);

  // ---- statistics: ROWS * 8 contiguous floats per array, one per thread ----------------
  {
    const int t = threadIdx.x;  // t = row * 8 + lane
    const int64_t base = FLAT ? s0 * 8 : ((int64_t)bn * S + s0) * 8;
    if (t < rows * 8) {
      const float pm = prev_max[base + t], ps = prev_sum[base + t];
      const float cm = cur_max[base + t], cs = cur_sum[base + t];
      float m, ps2, cs2;
      merge_lane(pm, ps, cm, cs, &m, &ps2, &cs2);
      const float l = ps2 + cs2;
      out_max[base + t] = m;
      out_sum[base + t] = l;
      if ((t & 7) == 0) {
        const float inv = l != 0.f ? 1.f / l : 0.f;
        s_po[t >> 3] = ps2 * inv;
        s_co[t >> 3] = cs2 * inv;
      }
    }
  }
  __syncthreads();

  // ---- outputs: SBH row s is D contiguous elements at ((s*B + b)*N + n)*D; FLAT row r at r*D
  const int64_t row_stride = FLAT ? (int64_t)D : (int64_t)B * N * D;
  const int64_t row0 = FLAT ? s0 * D : ((int64_t)s0 * B + b) * N * D + (int64_t)n * D;
  if constexpr (VEC) {
    constexpr int V = Vec16<T>::n;
    const int vpr = D / V;                  // vectors per row
    const int total = rows * vpr;
    constexpr int kPer = 4;                 // vectors per thread in flight
    for (int base = 0; base < total; base += kThreads * kPer) {
      uint4 pv[kPer], cv[kPer];
      int idx[kPer];
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        idx[u] = base + u * kThreads + threadIdx.x;
        if (idx[u] < total) {
          const int r = idx[u] / vpr, c = idx[u] - r * vpr;
          const int64_t off = row0 + r * row_stride + (int64_t)c * V;
          pv[u] = *reinterpret_cast<const uint4*>(prev_out + off);
          cv[u] = *reinterpret_cast<const uint4*>(cur_out + off);
        }
      }
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        if (idx[u] < total) {
          const int r = idx[u] / vpr, c = idx[u] - r * vpr;
          const int64_t off = row0 + r * row_stride + (int64_t)c * V;
          float a[V], bb[V], o[V];
          unpack(pv[u], a, (T*)nullptr);
          unpack(cv[u], bb, (T*)nullptr);
          const float po = s_po[r], co = s_co[r];
#pragma unroll
          for (int i = 0; i < V; ++i) o[i] = fmaf(a[i], po, bb[i] * co);
          *reinterpret_cast<uint4*>(out + off) = pack(o, (T*)nullptr);
        }
      }
    }
  } else {
    const int total = rows * D;
    for (int i = threadIdx.x; i < total; i += kThreads) {
      const int r = i / D, d = i - r * D;
      const int64_t off = row0 + r * row_stride + d;
      const float o = fmaf(to_f(prev_out[off]), s_po[r], to_f(cur_out[off]) * s_co[r]);
      from_f(o, out + off);
    }
  }
}

// Vectorised path (D a multiple of the 16-byte vector width, aligned rows). A block owns ROWS
// consecutive s of one (b, n). Every thread first issues all of its 16-byte loads of the two
// partial outputs (PER vectors each; they do not depend on the statistics), then the block
// merges the lane-wise statistics (ROWS * 8 contiguous floats per array, one per thread, each
// element read and written by the same thread, so the outputs may alias prev_*) and hands
// the lane-0 output scales through shared memory. The barrier therefore overlaps the bulk
// loads instead of preceding them.
// W32: 32-byte accesses (two 16-byte vectors each) when every row base is 32-byte aligned.
template <typename T, int ROWS, int THREADS, int PER, bool FLAT, bool W32>
__global__ void __launch_bounds__(THREADS) merge_sbh_vec_kernel(
    const T* prev_out, const float* prev_max, const float* prev_sum,  // may alias the outputs
    const T* __restrict__ cur_out, const float* __restrict__ cur_max,
    const float* __restrict__ cur_sum, int S, int B, int N, int D, T* out, float* out_max,
    float* out_sum) {
  constexpr int V16 = Vec16<T>::n;        // elements per 16-byte vector
  constexpr int H = W32 ? 2 : 1;           // 16-byte vectors per access
  constexpr int V = V16 * H;               // elements per access
  __shared__ float s_po[ROWS], s_co[ROWS];
  // SBH: block (b*N + n, s-block); FLAT (TND): block = ROWS consecutive rows t*N + n
  const int bn = FLAT ? 0 : blockIdx.x;
  const int b = FLAT ? 0 : bn / N, n = FLAT ? 0 : bn - b * N;
  const int64_t s0 = FLAT ? (int64_t)blockIdx.x * ROWS : (int64_t)blockIdx.y * ROWS;
  const int64_t nrow_all = FLAT ? (int64_t)S * N : (int64_t)S;
  const int rows = (int)min((int64_t)ROWS, nrow_all - s0);
  const int vpr = D / V;  // vectors per row
  const int total = rows * vpr;
  const int64_t row_stride = FLAT ? (int64_t)D : (int64_t)B * N * D;
  const int64_t row0 = FLAT ? s0 * D : ((int64_t)s0 * B + b) * N * D + (int64_t)n * D;

  // 1. bulk loads of the partial outputs, all in flight at once
  uint4 pv[PER][H], cv[PER][H];
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int idx = u * THREADS + threadIdx.x;
    if (idx < total) {
      const int r = idx / vpr, c = idx - r * vpr;
      const int64_t off = row0 + r * row_stride + (int64_t)c * V;
      if constexpr (W32) {
        ld32_na(prev_out + off, pv[u][0], pv[u][H - 1]);
        ld32_na(cur_out + off, cv[u][0], cv[u][H - 1]);
      } else {
        pv[u][0] = *reinterpret_cast<const uint4*>(prev_out + off);
        cv[u][0] = *reinterpret_cast<const uint4*>(cur_out + off);
      }
    }
  }
  // 2. lane-wise statistics, one (row, lane) element per thread
  const int64_t st0 = FLAT ? s0 * 8 : ((int64_t)bn * S + s0) * 8;
  for (int t = threadIdx.x; t < rows * 8; t += THREADS) {
    const float pm = prev_max[st0 + t], ps = prev_sum[st0 + t];
    const float cm = cur_max[st0 + t], cs = cur_sum[st0 + t];
    float m, ps2, cs2;
    merge_lane(pm, ps, cm, cs, &m, &ps2, &cs2);
    const float l = ps2 + cs2;
    out_max[st0 + t] = m;
    out_sum[st0 + t] = l;
    if ((t & 7) == 0) {
      const float inv = l != 0.f ? 1.f / l : 0.f;
      s_po[t >> 3] = ps2 * inv;
      s_co[t >> 3] = cs2 * inv;
    }
  }
  __syncthreads();
  // 3. outputs
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int idx = u * THREADS + threadIdx.x;
    if (idx < total) {
      const int r = idx / vpr, c = idx - r * vpr;
      const int64_t off = row0 + r * row_stride + (int64_t)c * V;
      const float po = s_po[r], co = s_co[r];
      uint4 res[H];
#pragma unroll
      for (int h = 0; h < H; ++h) {
        float a[V16], bb[V16], o[V16];
        unpack(pv[u][h], a, (T*)nullptr);
        unpack(cv[u][h], bb, (T*)nullptr);
#pragma unroll
        for (int i = 0; i < V16; ++i) o[i] = fmaf(a[i], po, bb[i] * co);
        res[h] = pack(o, (T*)nullptr);
      }
      if constexpr (W32)
        st32_na(out + off, res[0], res[H - 1]);
      else
        *reinterpret_cast<uint4*>(out + off) = res[0];
    }
  }
}

template <typename T, int ROWS, int THREADS, int PER, bool FLAT, bool W32 = false>
void launch_vec(const MergeArgs& a, cudaStream_t st) {
  const dim3 grid = FLAT ? dim3((unsigned)(((int64_t)a.S * a.N + ROWS - 1) / ROWS), 1)
                         : dim3(a.B * a.N, (a.S + ROWS - 1) / ROWS);
  merge_sbh_vec_kernel<T, ROWS, THREADS, PER, FLAT, W32><<<grid, THREADS, 0, st>>>(
      (const T*)a.prev_out, a.prev_max, a.prev_sum, (const T*)a.cur_out, a.cur_max, a.cur_sum,
      a.S, a.B, a.N, a.D, (T*)a.out, a.out_max, a.out_sum);
}

template <typename T, bool FLAT>
void launch_generic(const MergeArgs& a, bool vec, cudaStream_t st) {
  const dim3 grid = FLAT ? dim3((unsigned)(((int64_t)a.S * a.N + kRows - 1) / kRows), 1)
                         : dim3(a.B * a.N, (a.S + kRows - 1) / kRows);
  if (vec)
    merge_sbh_kernel<T, true, FLAT><<<grid, kThreads, 0, st>>>(
        (const T*)a.prev_out, a.prev_max, a.prev_sum, (const T*)a.cur_out, a.cur_max, a.cur_sum,
        a.S, a.B, a.N, a.D, (T*)a.out, a.out_max, a.out_sum);
  else
    merge_sbh_kernel<T, false, FLAT><<<grid, kThreads, 0, st>>>(
        (const T*)a.prev_out, a.prev_max, a.prev_sum, (const T*)a.cur_out, a.cur_max, a.cur_sum,
        a.S, a.B, a.N, a.D, (T*)a.out, a.out_max, a.out_sum);
}

template <typename T, bool FLAT>
void launch_layout(const MergeArgs& a, cudaStream_t st) {
  constexpr int V = Vec16<T>::n;
  const bool vec = (a.D % V) == 0 && ((uintptr_t)a.prev_out % 16) == 0 &&
                   ((uintptr_t)a.cur_out % 16) == 0 && ((uintptr_t)a.out % 16) == 0;
  // tiny blocks (8 rows x 64 threads x 2 vectors) measured fastest: many independent blocks
  const int vpr = a.D / V;
  constexpr int R = SDPA_MERGE_ROWS, TH = SDPA_MERGE_THREADS, PR = SDPA_MERGE_PER;
  // 32-byte accesses: D a multiple of two vectors and every output base 32-byte aligned (row
  // strides are then multiples of 32 bytes too)
  const bool w32 = vec && (a.D % (2 * V)) == 0 && ((uintptr_t)a.prev_out % 32) == 0 &&
                   ((uintptr_t)a.cur_out % 32) == 0 && ((uintptr_t)a.out % 32) == 0;
  if (w32 && R * (vpr / 2) <= (PR / 2 > 0 ? PR / 2 : 1) * TH)
    launch_vec<T, R, TH, (PR / 2 > 0 ? PR / 2 : 1), FLAT, true>(a, st);
  else if (vec && R * vpr <= PR * TH)
    launch_vec<T, R, TH, PR, FLAT>(a, st);
  else if (vec && 16 * vpr <= 4 * 256)
    launch_vec<T, 16, 256, 4, FLAT>(a, st);
  else
    launch_generic<T, FLAT>(a, vec, st);
}

// Cumulative query lengths of a TND merge (int64, B entries, no leading zero): they only fix
// the token count, so the check is that they never decrease and end at T.
__global__ void check_seq_qlen_kernel(const int64_t* cu, int B, int64_t T, int* status) {
  int64_t prev_end = 0;
  bool bad = false;
  for (int c0 = 0; c0 < B; c0 += 32) {
    const int i = c0 + threadIdx.x;
    const int64_t end = i < B ? cu[i] : 0;
    int64_t start = __shfl_up_sync(0xffffffffu, end, 1);
    if (threadIdx.x == 0) start = prev_end;
    bad |= i < B && (end < start || (i == B - 1 && end != T));
    prev_end = __shfl_sync(0xffffffffu, end, 31);
  }
  if (__any_sync(0xffffffffu, bad) && threadIdx.x == 0) report(status, ATTN_ERR_DATA);
}

template <typename T>
cudaError_t launch_typed(const MergeArgs& a, cudaStream_t st) {
  if (a.layout == ATTN_TND) {
    if (a.seq_qlen != nullptr) check_seq_qlen_kernel<<<1, 32, 0, st>>>(a.seq_qlen, a.B, a.S, a.status);
    launch_layout<T, true>(a, st);
  } else {
    launch_layout<T, false>(a, st);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t st) {
  if (a.dtype == ATTN_BF16) return launch_typed<__nv_bfloat16>(a, st);
  if (a.dtype == ATTN_F16) return launch_typed<__half>(a, st);
  return launch_typed<float>(a, st);
}

}  // namespace sdpa
