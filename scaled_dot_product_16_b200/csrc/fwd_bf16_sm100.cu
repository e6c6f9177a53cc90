// fwd_bf16_sm100.cu -- fused attention forward for bf16 (and fp16) on B200 (sm_100a).
//
// O = softmax(scale * Q K^T + mask) V with per-row softmax max / sum, for dense BHSD or packed
// TND batches with GQA/MQA head ratios and causal masks ("aclnnFlashAttentionVarLenScore",
// CANN 8.5 API doc, 功能说明 and 约束说明; the formula of "paddle.nn.functional.sparse_attention").
// The pages name the FlashAttention algorithm (tiles of Q against streamed K/V tiles with an
// online softmax) but give no kernel; this is a from-scratch sm_100a design:
//
//   * one block per SM takes work items one after another; an item is two 128-row tiles Q0 and
//     Q1: the same rows of two query heads that share a KV head (GQA with an even group), else
//     256 consecutive rows of one head;
//   * K and V tiles (128 keys x D) stream through a ring of shared-memory stages, loaded by
//     TMA with 128-byte swizzle (one issuing thread, no multicast);
//   * one thread issues every tcgen05.mma: S_q = Q_q K_j^T (both operands in shared memory,
//     fp32 accumulator in tensor memory) and O_q += P_q V_j (P read from tensor memory);
//   * two softmax warpgroups (one per Q tile, one thread per row = one TMEM lane) read S with
//     tcgen05.ld, apply the mask, keep the running max / sum, write P = exp2(...) as bf16 back
//     into the first half of S's TMEM columns, and at the end normalise O and store it;
//   * while one warpgroup is in its softmax, the tensor core runs the other tile's MMAs;
//   * the running max is updated lazily: only when a row's maximum grows by more than 2^8 are
//     O and the sum rescaled (exact, because the same max is used for P, the sum and O);
//   * key tiles entirely above the causal diagonal are never loaded or multiplied, the
//     diagonal and ragged tiles are masked element by element, rows past a sequence's end are
//     never stored, and zero-length sequences produce no work.
//
// Roles (384 threads): warps 0-3 softmax Q0, warps 4-7 softmax Q1, warp 8 MMA issue,
// warp 9 TMA producer (warps 10-11 idle). TMEM: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).
//
// Every mbarrier wait is bounded in time: if a wait runs out the block records
// ATTN_ERR_TIMEOUT, stops issuing work, drains what it started and frees its TMEM.
#include <cuda.h>
#include <math.h>

#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace sdpa {
namespace {

using namespace sm100;

constexpr int kBM = 128;          // rows per Q tile (= TMEM lanes)
constexpr int kBN = 128;          // keys per K/V tile
constexpr int kRowsPerBlock = 2 * kBM;
constexpr int kThreads = 384;
constexpr int kMmaWarp = 8;
constexpr int kTmaWarp = 9;       // warps 10 and 11 only complete the producer warpgroup
// Register split: the block is launched with kRegsLaunch a thread (the limit for 384 threads,
// which the host checks before each launch); the softmax warpgroups raise theirs to
// kRegsSoftmax, the producer warpgroup lowers its own to kRegsProducer.
constexpr int kRegsLaunch = 168;
constexpr int kRegsSoftmax = 216;
constexpr int kRegsProducer = 72;
static_assert(256 * kRegsSoftmax + 128 * kRegsProducer <= kThreads * kRegsLaunch, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale when the max grows by > 2^8
// Time bounds of a barrier wait: one in the pipeline (data or a hand-off from another role),
// and one while draining work this block already issued (its TMA loads and MMAs must land
// before TMEM is freed and the block exits). The test build of the library shortens the first.
#ifndef SDPA_PIPE_WAIT_NS
#define SDPA_PIPE_WAIT_NS 200000000ull
#endif
constexpr uint64_t kPipeWaitNs = SDPA_PIPE_WAIT_NS;
constexpr uint64_t kDrainWaitNs = 200ull * 1000ull * 1000ull;  // 200 ms
// Test build only: the MMA warp first waits on a barrier that nothing arrives on, so that wait
// runs out and the timeout path (status word, abort, drains) is exercised without any fault.
#ifndef SDPA_TEST_STALL
#define SDPA_TEST_STALL 0
#endif
#ifndef SDPA_SUSPEND_NS
#define SDPA_SUSPEND_NS 20000
#endif
constexpr uint32_t kSuspendNs = SDPA_SUSPEND_NS;  // longest hardware suspension per try_wait

#ifndef SDPA_EMU_EVERY
#define SDPA_EMU_EVERY 5
#endif
// One exp2 pair in kEmuEvery goes to the FMA-pipe polynomial (0: none).
constexpr int kEmuEvery = SDPA_EMU_EVERY;
#ifndef SDPA_STAGES_D128
#define SDPA_STAGES_D128 4
#endif

// 2^x for a pair on the FMA/ALU pipes. Range reduction after Cody and Waite: x = j + f with
// j = round(x) (adding 1.5 * 2^23 rounds to nearest and leaves j in the low mantissa bits) and
// f in [-1/2, 1/2]; 2^f by a degree-3 polynomial fitted here by the Remez exchange for minimum
// relative error (csrc/fit_exp2_poly.py, max relative error 7.5e-5); 2^j is added into the
// exponent field. Inputs are clamped at -126 first (one max per lane instead of a compare and a
// select): from there down, -inf from masking included, the result is a positive value below
// 2^-125, which the callers treat as zero (rows that see no key at all are caught by their max).
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& p0, float& p1) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  constexpr float c0 = 9.999280572e-01f, c1 = 6.932609677e-01f, c2 = 2.426111251e-01f,
                  c3 = 5.517166853e-02f;
  x0 = fmaxf(x0, -126.f);
  x1 = fmaxf(x1, -126.f);
  float t0, t1, j0, j1, f0, f1, q0, q1;
  fadd2(x0, x1, kShift, kShift, t0, t1);
  fadd2(t0, t1, -kShift, -kShift, j0, j1);
  ffma2(j0, j1, -1.f, -1.f, x0, x1, f0, f1);  // f = x - j
  ffma2(c3, c3, f0, f1, c2, c2, q0, q1);
  ffma2(q0, q1, f0, f1, c1, c1, q0, q1);
  ffma2(q0, q1, f0, f1, c0, c0, q0, q1);
  p0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
  p1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}

// HD: head size of Q and K; HDV: head size of V and the output (HDV <= HD).
template <int HD, int HDV, bool F16>
struct Cfg {
  static constexpr int kBoxes = HD / 64;                 // 64-element (128-byte) TMA boxes
  static constexpr int kBoxesV = HDV / 64;
  static constexpr int kTileBytes = kBM * HD * 2;        // one Q or K tile; a K/V ring slot
  static constexpr int kTileBytesV = kBN * HDV * 2;      // one V tile
  static constexpr int kStages = HD == 128 ? SDPA_STAGES_D128 : 6;  // K/V ring depth
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
  // output staging for the TMA stores: 4 KB (32 rows x 64 columns, 128-byte swizzle) per softmax warp
  static constexpr int kStageOff = kBarOff + 1024;
  static constexpr int kSmemBytes = kStageOff + 8 * 4096 + 1024;  // + 1 KB for alignment
  static_assert(kStages >= 2 && kStages <= 8, "barrier arrays hold 8 stages");
  static_assert(kSmemBytes <= 232448, "227 KB of shared memory per block");
  static constexpr uint32_t kFmt = F16 ? 0u : 1u;  // instruction-descriptor operand format
  static constexpr uint32_t kIdescQK = idesc_f16_f32(kBM, kBN, 0, 0, kFmt);
  static constexpr uint32_t kIdescPV = idesc_f16_f32(kBM, HDV, 0, 1, kFmt);
  static_assert(HDV <= HD && HDV % 64 == 0, "value head size");
};

// Work counters of the persistent grid, a pair per slot: the next item to hand out (counted
// past the first gridDim.x items, which block x takes without asking) and the blocks finished.
// A launch draws its items from one slot with atomicAdd; its last block to finish puts both back
// to 0, so the next launch that uses the slot starts from 0. The host gives every stream its own
// slot (launches on one stream run one after another), and launches that cannot be given one
// divide the items statically instead.
constexpr int kSchedSlots = 256;
__device__ int g_sched[kSchedSlots * 2];

// One work item decoded: two 128-row Q tiles of sequence b (see pair_heads: the same rows of
// query heads h and h + 1, or 256 consecutive rows of head h).
struct Unit {
  int b, h;          // sequence and (first) query head; b < 0 marks the end of the block's work
  int q0, sq, sk;    // first query token and query length of the sequence; its key length
  int row0;          // first row (within the sequence) of Q0
  int rows0, rows1;  // rows of Q0 and Q1 (rows1 <= 0: no second tile)
  int jlo;           // first key tile (the band's first tile for row0; 0 otherwise)
  int n0, n1;        // key tiles from jlo up to Q0's / Q1's last visible key (n1 >= n0)
  int s1;            // Q1's first key tile, counted from jlo (0 except with the band)
};

constexpr int kUnitSlots = 4;    // decoded items the TMA warp may run ahead
constexpr int kUnitReaders = 9;  // the MMA warp and the eight softmax warps read each item

struct Barriers {
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint64_t q_full;
  uint64_t q_empty;  // the last S MMAs of an item have run: Q may be overwritten
  uint64_t s_full[2];
  uint64_t p_ready[2];
  uint64_t o_done[2];
  uint64_t drain;
  uint64_t stall;  // never arrived on (the test build waits on it)
  uint64_t unit_full[kUnitSlots];   // an item (or the end mark) is in the slot
  uint64_t unit_empty[kUnitSlots];  // every reader has taken the slot's item
  Unit units[kUnitSlots];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Barriers) <= 512, "the barrier area of the shared-memory layout");

// Bounded wait on an mbarrier phase. Returns false (after recording a timeout, or when another
// role of this block already gave up) instead of waiting forever.
// With heed_abort = false (used when draining work already issued) only the drain's time
// bound applies.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort,
                                         int* status, bool heed_abort = true) {
  if (mbar_try_wait_sleep(bar, parity, kSuspendNs)) return true;
  const uint64_t t0 = globaltimer_ns();
  const uint64_t limit = heed_abort ? kPipeWaitNs : kDrainWaitNs;
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, kSuspendNs)) return true;
    if (heed_abort && *abort) return false;
    if (globaltimer_ns() - t0 > limit) {
      *abort = 1;
      report(status, ATTN_ERR_TIMEOUT);
      return false;
    }
  }
}

constexpr int kAccNone = 0, kAccFirst = 1, kAccMerge = 2;

// Fold one row's result (max m_loc, sum l_loc, output o = O * f_o) into an accumulator row
// with the lane-wise update of "npu_ring_attention_update" (小算子等价计算逻辑): for each of the
// 8 statistic lanes m = max(pm, m_loc), ps' = ps e^(pm - m), cs' = l_loc e^(m_loc - m),
// l = ps' + cs'; the output becomes prev * ps'_0 / l_0 + o * cs'_0 / l_0. On the first chunk the
// accumulator is simply overwritten. Returns the two output factors.
__device__ __forceinline__ void merge_into_stats(const FwdArgs& a, int64_t so, float m_loc, float l_loc,
                                                 float* f_prev, float* f_o) {
  float4* mx = reinterpret_cast<float4*>(a.smax + so);
  float4* sm = reinterpret_cast<float4*>(a.ssum + so);
  if (a.acc_mode == kAccFirst) {
    const float4 mv = make_float4(m_loc, m_loc, m_loc, m_loc), lv = make_float4(l_loc, l_loc, l_loc, l_loc);
    mx[0] = mv; mx[1] = mv; sm[0] = lv; sm[1] = lv;
    *f_prev = 0.f;
    return;
  }
  float pm[8], ps[8];
  *reinterpret_cast<float4*>(pm) = mx[0];
  *reinterpret_cast<float4*>(pm + 4) = mx[1];
  *reinterpret_cast<float4*>(ps) = sm[0];
  *reinterpret_cast<float4*>(ps + 4) = sm[1];
  float nm[8], nl[8], ps0 = 0.f, cs0 = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float mk = fmaxf(pm[k], m_loc);
    float a1 = 0.f, a2 = 0.f;
    if (mk != -INFINITY) {
      a1 = ps[k] * expf(pm[k] - mk);
      a2 = l_loc * expf(m_loc - mk);
    }
    nm[k] = mk;
    nl[k] = a1 + a2;
    if (k == 0) {
      ps0 = a1;
      cs0 = a2;
    }
  }
  mx[0] = *reinterpret_cast<float4*>(nm);
  mx[1] = *reinterpret_cast<float4*>(nm + 4);
  sm[0] = *reinterpret_cast<float4*>(nl);
  sm[1] = *reinterpret_cast<float4*>(nl + 4);
  const float inv = nl[0] != 0.f ? 1.f / nl[0] : 0.f;
  *f_prev = ps0 * inv;
  *f_o *= cs0 * inv;
}

// The two Q tiles of an item: with an even number of query heads per KV head (GQA), the same 128
// rows of two query heads of one group (h, h + 1), which need exactly the same key tiles and read
// the same K/V; otherwise 256 consecutive rows of one head (Q1 the second 128).
__host__ __device__ __forceinline__ bool pair_heads(const FwdArgs& a) {
  return a.Nkv > 0 && (a.Nq / a.Nkv) % 2 == 0;
}
__host__ __device__ __forceinline__ int rows_per_item(const FwdArgs& a) {
  return pair_heads(a) ? kBM : kRowsPerBlock;
}

// Decodes item x. Items run query-head (pair) fastest; for BHSD the row blocks go by level (the
// last row block of every sequence first), for TND sequence by sequence with each sequence's last
// row block first, so that the heaviest items of a sequence come first. Run by one full warp;
// every lane gets the result. Returns false for an item past the last row block (an item there
// with h == 0 checks the key-side cumulative lengths) and for a sequence whose keys lie outside
// [0, Skv), recording ATTN_ERR_DATA for bad lengths.
template <int EXT>
__device__ __forceinline__ bool decode_unit(const FwdArgs& a, int units_per_seq, int x, Unit& U, int& k0) {
  const int lane = threadIdx.x & 31;
  const bool pair = pair_heads(a);
  const int rows = rows_per_item(a);
  const int heads = pair ? a.Nq / 2 : a.Nq;  // items per row block
  const int h = pair ? 2 * (x % heads) : x % heads;
  const int y = x / heads;
  int b = 0, u = 0;
  bool ok = true;
  if (a.layout == ATTN_BHSD) {
    const int level = y / a.B;  // 0 = last row block of every sequence
    b = y - level * a.B;
    u = units_per_seq - 1 - level;
    ok = u >= 0;
  } else {
    bool bad;
    int t;
    ok = warp_find_tile(a.cu_q, a.B, a.Sq, rows, y, &b, &t, a.status, &bad);
    if (ok) {
      int qs, ql;
      seq_span(a.cu_q, b, &qs, &ql);
      u = (ql + rows - 1) / rows - 1 - t;
    } else if (!bad && h == 0) {
      int sb, st;
      bool bad2;
      warp_find_tile(a.cu_kv, a.B, a.Skv, 1 << 30, 1 << 30, &sb, &st, a.status, &bad2);
    }
  }
  if (!ok) return false;
  U.b = b;
  U.h = h;
  U.row0 = u * rows;
  if (a.layout == ATTN_BHSD) {
    U.q0 = 0;
    U.sq = a.Sq;
    k0 = 0;
    U.sk = a.Skv;
  } else {
    seq_span(a.cu_q, b, &U.q0, &U.sq);
    seq_span(a.cu_kv, b, &k0, &U.sk);
    if (k0 < 0 || U.sk < 0 || k0 + U.sk > a.Skv) {
      if (lane == 0) report(a.status, ATTN_ERR_DATA);
      return false;
    }
  }
  U.rows0 = min(kBM, U.sq - U.row0);
  U.rows1 = pair ? U.rows0 : min(kBM, U.sq - U.row0 - kBM);
  const bool has1 = U.rows1 > 0;
  const int r1 = pair ? U.row0 : U.row0 + kBM;  // Q1's first row
  // Key tiles run from jlo to the tile holding each Q tile's last visible key; n0 and n1 count
  // tiles from jlo. With the band, Q1 starts at its own first tile: s1 tiles after jlo.
  U.jlo = EXT >= 1 ? visible_begin(a.mask_mode, U.row0, a.pre) / kBN : 0;
  const int kv_end0 = visible_end(a.mask_mode, U.row0 + U.rows0 - 1, U.sq, U.sk, a.next);
  const int kv_end1 = has1 ? visible_end(a.mask_mode, r1 + U.rows1 - 1, U.sq, U.sk, a.next) : 0;
  U.n0 = max((kv_end0 + kBN - 1) / kBN, U.jlo) - U.jlo;
  U.n1 = has1 ? max((kv_end1 + kBN - 1) / kBN, U.jlo) - U.jlo : U.n0;
  U.s1 = EXT >= 1 && has1 ? visible_begin(a.mask_mode, r1, a.pre) / kBN - U.jlo : 0;
  return true;
}

// EXT: the masked-call features. 0: plain calls, whose softmax loop carries none of their code;
// 1: the band's lower edge; 2: the band and an explicit mask (its bytes take registers that the
// band alone does not need).
//
// Persistent: each block (one per SM) takes items one after another, from the scheduler slot
// `sched` when there is one, else x = blockIdx.x + k * gridDim.x. The TMA warp decodes each item
// and hands it to the MMA warp and the softmax warps through a ring of kUnitSlots shared-memory
// slots; its loads of item u+1 (the first K/V tiles, then Q once the last S of item u has run)
// overlap the last softmax, P.V and epilogue of item u, and the block's setup is paid once.
template <int HD, int HDV, bool F16, int EXT>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    FwdArgs a, int units_per_seq,
                    float scale_log2, int n_items, int* sched) {
  using C = Cfg<HD, HDV, F16>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Barriers* bars = reinterpret_cast<Barriers*>(smem + C::kBarOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar_addr = [&](const uint64_t* p) { return smem_u32(p); };

  // ---- setup (once per block): barriers, TMEM ----------------------------------------------
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar_addr(&bars->kv_full[s]), 1);
      mbar_init(bar_addr(&bars->kv_empty[s]), 1);
    }
    mbar_init(bar_addr(&bars->q_full), 1);
    mbar_init(bar_addr(&bars->q_empty), 1);
    mbar_init(bar_addr(&bars->drain), 1);
    mbar_init(bar_addr(&bars->stall), 1);
    for (int q = 0; q < 2; ++q) {
      mbar_init(bar_addr(&bars->s_full[q]), 1);
      mbar_init(bar_addr(&bars->p_ready[q]), 4);  // one arrival per softmax warp
      mbar_init(bar_addr(&bars->o_done[q]), 1);
    }
    for (int s = 0; s < kUnitSlots; ++s) {
      mbar_init(bar_addr(&bars->unit_full[s]), 1);
      mbar_init(bar_addr(&bars->unit_empty[s]), kUnitReaders);
    }
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  const uint32_t sQ = smem_u32(smem + C::kQOff);
  const uint32_t sKV = smem_u32(smem + C::kKVOff);

  if (warp >= 8) {
    // the producer warpgroup gives registers to the softmax warpgroups (each branch sets its own
    // count first, so that the code after it is compiled for that count)
    setmaxnreg_dec<kRegsProducer>();
    if (warp == kTmaWarp) {
      // =============================== TMA producer (and item decoder) ===========================
      const bool bhsd = a.layout == ATTN_BHSD;
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
      }
      auto load_tile = [&](const CUtensorMap* map, uint32_t dst, uint32_t bar, int tok, int head, int boxes) {
        for (int x = 0; x < boxes; ++x) {
          if (bhsd)
            tma_load_3d(dst + x * (kBM * 128), map, bar, x * 64, tok, head);
          else
            tma_load_3d(dst + x * (kBM * 128), map, bar, x * 64, head, tok);
        }
      };
      uint32_t it = 0;  // K/V tiles issued by this block: position in the ring
      int qn = 0;       // Q loads issued
      int k = 0;        // items handed out
      bool ok = true;
      int64_t x = blockIdx.x;
      for (;;) {
        Unit U;
        int k0 = 0;
        const bool end = x >= n_items;
        const bool live = !end && decode_unit<EXT>(a, units_per_seq, (int)x, U, k0);
        if (end || live) {
          // hand the item (or the end mark) to the other roles through slot k % kUnitSlots
          if (lane == 0) {
            const int slot = k % kUnitSlots;
            if (k >= kUnitSlots)
              ok = wait_bar(bar_addr(&bars->unit_empty[slot]), ((k / kUnitSlots) - 1) & 1, abort, a.status);
            if (ok) {
              if (end) bars->units[slot].b = -1;
              else bars->units[slot] = U;
              mbar_arrive(bar_addr(&bars->unit_full[slot]));  // releases the slot's contents
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
          ++k;
          if (!ok || end) break;
          if (lane == 0 && U.n1 > 0) {
            const int g = U.h / (a.Nq / a.Nkv);
            const int qhead = bhsd ? U.b * a.Nq + U.h : U.h;
            const int khead = bhsd ? U.b * a.Nkv + g : g;
            const int nl = 2 * U.n1;
            // K0, V0, K1, V1, ... through the ring; Q once the previous item's last S has run
            auto load_kv = [&](int i) {
              const uint32_t s = it % C::kStages, r = it / C::kStages;
              if (r > 0 && !wait_bar(bar_addr(&bars->kv_empty[s]), (r - 1) & 1, abort, a.status)) return false;
              const uint32_t fb = bar_addr(&bars->kv_full[s]);
              mbar_arrive_expect_tx(fb, (i & 1) ? C::kTileBytesV : C::kTileBytes);
              load_tile((i & 1) ? &tm_v : &tm_k, sKV + s * C::kTileBytes, fb, k0 + (U.jlo + (i >> 1)) * kBN, khead,
                        (i & 1) ? C::kBoxesV : C::kBoxes);
              ++it;
              return true;
            };
            const int first = min(2, nl);
            for (int i = 0; ok && i < first; ++i) ok = load_kv(i);
            if (ok && qn > 0) ok = wait_bar(bar_addr(&bars->q_empty), (qn - 1) & 1, abort, a.status);
            if (ok) {
              const bool has1 = U.rows1 > 0;
              const uint32_t qbar = bar_addr(&bars->q_full);
              mbar_arrive_expect_tx(qbar, (has1 ? 2 : 1) * C::kTileBytes);
              load_tile(&tm_q, sQ, qbar, U.q0 + U.row0, qhead, C::kBoxes);
              if (has1) {
                if (pair_heads(a))
                  load_tile(&tm_q, sQ + C::kTileBytes, qbar, U.q0 + U.row0, qhead + 1, C::kBoxes);
                else
                  load_tile(&tm_q, sQ + C::kTileBytes, qbar, U.q0 + U.row0 + kBM, qhead, C::kBoxes);
              }
              ++qn;
            }
            for (int i = first; ok && i < nl; ++i) ok = load_kv(i);
          }
          ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
          if (!ok) break;
        }
        int64_t nx = 0;
        if (lane == 0) nx = sched != nullptr ? (int64_t)gridDim.x + atomicAdd(sched, 1) : x + gridDim.x;
        x = __shfl_sync(0xffffffffu, nx, 0);
      }
      if (lane == 0) {
        // drain: every load this thread issued must have landed before the block exits
        for (uint32_t i = it > (uint32_t)C::kStages ? it - C::kStages : 0u; i < it; ++i)
          wait_bar(bar_addr(&bars->kv_full[i % C::kStages]), (i / C::kStages) & 1, abort, a.status, false);
        if (qn > 0) wait_bar(bar_addr(&bars->q_full), (qn - 1) & 1, abort, a.status, false);
      }
    } else if (warp == kMmaWarp) {
      // =============================== MMA issue ==========================================
      if (lane == 0) {
        const uint32_t S0 = tmem, S1 = tmem + 128, O0 = tmem + 256, O1 = tmem + 256 + HDV;
        // Descriptors are built once. K-step kk of an operand adds a constant to the start
        // address field (shared-memory addresses stay below 256 KB, so the 14-bit field never
        // carries), which keeps the issue loop at a few instructions per MMA.
        const uint64_t dq0 = smem_desc_sw128(sQ, 16, 1024);
        const uint64_t dq1 = dq0 + (uint64_t)(C::kTileBytes >> 4);
        const uint64_t dk0 = smem_desc_sw128(sKV, 16, 1024);
        const uint64_t dv0 = smem_desc_sw128(sKV, kBN * 128, 1024);
        const uint32_t kvfull0 = bar_addr(&bars->kv_full[0]), kvempty0 = bar_addr(&bars->kv_empty[0]);
        auto full = [&](uint32_t i) {
          return wait_bar(kvfull0 + 8 * (i % C::kStages), (i / C::kStages) & 1, abort, a.status);
        };
        auto release = [&](uint32_t i) { mma_commit(kvempty0 + 8 * (i % C::kStages)); };
        auto issue_qk = [&](uint32_t d, uint64_t dq, uint32_t i) {
          const uint64_t dk = dk0 + (uint64_t)(((i % C::kStages) * C::kTileBytes) >> 4);
          if constexpr (HD == 128)
            mma_ss_chain8(d, dq, dk, C::kIdescQK, 0u);
          else
            mma_ss_chain4(d, dq, dk, C::kIdescQK, 0u);
        };
        auto issue_pv = [&](uint32_t d, uint32_t p_tmem, uint32_t i, bool acc) {
          const uint64_t dv = dv0 + (uint64_t)(((i % C::kStages) * C::kTileBytes) >> 4);
          mma_ts_chain8(d, p_tmem, dv, C::kIdescPV, acc ? 1u : 0u);
        };
        bool ok = true;
        if constexpr (SDPA_TEST_STALL != 0) ok = wait_bar(bar_addr(&bars->stall), 0, abort, a.status);
        uint32_t it = 0;        // K/V tiles consumed (the same sequence the TMA warp issues)
        int qn = 0;             // Q loads consumed
        uint32_t pc0 = 0, pc1 = 0;  // P hand-offs taken from each softmax warpgroup
        for (int k = 0; ok; ++k) {
          const int slot = k % kUnitSlots;
          if (!(ok = wait_bar(bar_addr(&bars->unit_full[slot]), (k / kUnitSlots) & 1, abort, a.status))) break;
          const Unit* us = &bars->units[slot];
          const int ub = us->b, n0 = us->n0, n1 = us->n1, s1 = us->s1;
          const bool has1 = us->rows1 > 0;
          mbar_arrive(bar_addr(&bars->unit_empty[slot]));
          if (ub < 0) break;
          if (n1 <= 0) continue;
          // Q1 works on key tiles s1 .. n1-1 (s1 = 0 except with the band)
          auto act1 = [&](int j) { return has1 && j >= s1; };
          // after the S MMAs of the item's last key tile: Q may be overwritten once they have run
          auto after_s = [&](int t) {
            if (t == n1 - 1) mma_commit(bar_addr(&bars->q_empty));
          };
          ok = wait_bar(bar_addr(&bars->q_full), qn & 1, abort, a.status);
          ++qn;
          if (ok) ok = full(it);
          if (!ok) break;
          tc_fence_after();
          if (n0 > 0) {
            issue_qk(S0, dq0, it);
            mma_commit(bar_addr(&bars->s_full[0]));
          }
          if (act1(0)) {
            issue_qk(S1, dq1, it);
            mma_commit(bar_addr(&bars->s_full[1]));
          }
          after_s(0);
          release(it);
          for (int j = 0; ok && j < n1; ++j) {
            const uint32_t iv = it + 2 * j + 1, ik = it + 2 * j + 2;
            if (!(ok = full(iv))) break;
            tc_fence_after();
            if (j < n0) {
              if (!(ok = wait_bar(bar_addr(&bars->p_ready[0]), pc0 & 1, abort, a.status))) break;
              ++pc0;
              tc_fence_after();
              issue_pv(O0, S0, iv, j > 0);
              if (j == n0 - 1) mma_commit(bar_addr(&bars->o_done[0]));
            }
            const bool next = j + 1 < n1;
            if (next) {
              if (!(ok = full(ik))) break;
              tc_fence_after();
              if (j + 1 < n0) {
                issue_qk(S0, dq0, ik);
                mma_commit(bar_addr(&bars->s_full[0]));
              }
            }
            if (act1(j)) {
              if (!(ok = wait_bar(bar_addr(&bars->p_ready[1]), pc1 & 1, abort, a.status))) break;
              ++pc1;
              tc_fence_after();
              issue_pv(O1, S1, iv, j > s1);
              if (j == n1 - 1) mma_commit(bar_addr(&bars->o_done[1]));
            }
            release(iv);
            if (next) {
              if (act1(j + 1)) {
                issue_qk(S1, dq1, ik);
                mma_commit(bar_addr(&bars->s_full[1]));
              }
              after_s(j + 1);
              release(ik);
            }
          }
          it += 2 * n1;
        }
        if (!ok) *abort = 1;
        // every MMA and commit issued above must have completed before TMEM is freed
        mma_commit(bar_addr(&bars->drain));
        wait_bar(bar_addr(&bars->drain), 0, abort, a.status, false);
      }
    }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // =============================== softmax + epilogue ================================
    const int q = warp >> 2;                       // Q tile of this warpgroup
    const int quarter = warp & 3;                  // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;             // row within the Q tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t S = tmem + lane_off + q * 128;
    const uint32_t O = tmem + lane_off + 256 + q * HDV;
    uint32_t sfc = 0;  // S hand-offs taken, over all of the block's items
    uint32_t odc = 0;  // final-O hand-offs taken
    for (int k = 0;; ++k) {
      const int slot = k % kUnitSlots;
      if (!__all_sync(0xffffffffu, wait_bar(bar_addr(&bars->unit_full[slot]), (k / kUnitSlots) & 1, abort, a.status)))
        break;
      // the item stays in its slot until this warp is done with it (fields are read as needed)
      const Unit& w = bars->units[slot];
      if (w.b < 0) break;
      const bool has1 = w.rows1 > 0;
      const int jlo = w.jlo;
      const int j0 = q == 0 ? 0 : w.s1;              // this Q tile's key tiles: j0 .. n-1
      const int n = q == 0 ? w.n0 : (has1 ? w.n1 : 0);
      const bool pair = pair_heads(a);
      const int i = w.row0 + (pair ? 0 : q * kBM) + r;  // row within the sequence
      const int hq = w.h + (pair ? q : 0);              // query head of this Q tile
      const int lim = i < w.sq ? visible_end(a.mask_mode, i, w.sq, w.sk, a.next) : w.sk;
      const int lo = EXT >= 1 && i < w.sq ? visible_begin(a.mask_mode, i, a.pre) : 0;
      // explicit mask row of this query (rows past the sequence read none)
      const uint8_t* mrow = nullptr;
      if constexpr (EXT == 2)
        if (i < w.sq && a.mask != nullptr) mrow = a.mask + (int64_t)w.b * a.mask_bs + (int64_t)i * a.mask_rs;

      float m = -INFINITY;        // running max used for P (log2 units, lazily updated)
      float mraw = -INFINITY;     // true max of the raw scores q.k
      float l = 0.f;
      bool ok = true;
      if (q == 0 || has1) {
        for (int j = j0; j < n; ++j) {
          ok = __all_sync(0xffffffffu, wait_bar(bar_addr(&bars->s_full[q]), sfc & 1, abort, a.status));
          ++sfc;
          if (!ok) break;
          tc_fence_after();
          const int kbase = (jlo + j) * kBN;
          uint4 mk[EXT == 2 ? 8 : 1];
          if constexpr (EXT == 2) {
            // the mask bytes of this row's 128 keys (16 at a time when aligned and whole);
            // issued before the TMEM loads so the two latencies overlap
            if (mrow == nullptr) {
              // band only, or a row past the sequence: nothing to read
            } else if (a.mask_vec && kbase + kBN <= w.sk) {
              const uint4* src = reinterpret_cast<const uint4*>(mrow + kbase);
#pragma unroll
              for (int x = 0; x < 8; ++x) mk[x] = __ldg(src + x);
            } else {
#pragma unroll
              for (int x = 0; x < 8; ++x) {
                uint32_t wd[4];
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                  uint32_t word = 0;
#pragma unroll
                  for (int z = 0; z < 4; ++z) {
                    const int c = x * 16 + y * 4 + z;
                    const uint32_t byte = kbase + c < w.sk ? mrow[kbase + c] : 0u;
                    word |= (byte != 0u ? 1u : 0u) << (8 * z);
                  }
                  wd[y] = word;
                }
                mk[x] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
              }
            }
          }
          float s[4][32];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32f(S + c * 32, s[c]);
          tmem_wait_ld();
          if constexpr (EXT == 0) {
            if (kbase + kBN > lim) {
              const int hi = lim - kbase;  // this row's first masked column of the tile
#pragma unroll
              for (int c = 0; c < kBN; ++c)
                if (c >= hi) s[c >> 5][c & 31] = -INFINITY;
            }
          } else if constexpr (EXT == 1) {
            // each edge on its own: a tile of a band wider than a tile holds at most one of them
            if (kbase + kBN > lim) {
              const int hi = lim - kbase;
#pragma unroll
              for (int c = 0; c < kBN; ++c)
                if (c >= hi) s[c >> 5][c & 31] = -INFINITY;
            }
            if (kbase < lo) {
              const int first = lo - kbase;  // this row's first visible column of the tile
#pragma unroll
              for (int c = 0; c < kBN; ++c)
                if (c < first) s[c >> 5][c & 31] = -INFINITY;
            }
          } else {
            if (kbase + kBN > lim || kbase < lo) {
#pragma unroll
              for (int c = 0; c < kBN; ++c)
                if (kbase + c >= lim || kbase + c < lo) s[c >> 5][c & 31] = -INFINITY;
            }
            if (EXT == 2 && mrow != nullptr) {
#pragma unroll
            for (int c = 0; c < kBN; ++c) {
              const uint4 v4 = mk[c >> 4];
              const uint32_t wd = ((c >> 2) & 3) == 0 ? v4.x : ((c >> 2) & 3) == 1 ? v4.y
                                : ((c >> 2) & 3) == 2 ? v4.z : v4.w;
              if ((wd >> (8 * (c & 3))) & 0xffu) s[c >> 5][c & 31] = -INFINITY;
            }
            }
          }
          // row max: a tree of 3-input maxima over the 128 scores
          float mx[8];
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const float* v = &s[x >> 1][(x & 1) * 16];
            const float a0 = fmax3(v[0], v[1], v[2]), a1 = fmax3(v[3], v[4], v[5]);
            const float a2 = fmax3(v[6], v[7], v[8]), a3 = fmax3(v[9], v[10], v[11]);
            const float a4 = fmax3(v[12], v[13], v[14]);
            mx[x] = fmax3(fmax3(a0, a1, a2), fmax3(a3, a4, v[15]), a0);
          }
          const float tmax = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                                   fmaxf(mx[6], mx[7]));
          mraw = fmaxf(mraw, tmax);
          const float tmax2 = tmax * scale_log2;
          bool bump = tmax2 > m + kRescaleThreshold;  // also true for the first finite max
          float corr = 1.f;
          if (bump) {
            corr = (m == -INFINITY) ? 0.f : ex2(m - tmax2);
            m = tmax2;
            l *= corr;
          }
          const float muse = m == -INFINITY ? 0.f : m;
          // P = 2^(s * scale_log2 - m) with packed (two-lane) FMA and add; exp2 on the MUFU unit
          // (and, for one pair in kEmuEvery, on the FMA pipe).
          float2 rs[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
          const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(-muse, -muse);
          uint32_t pk[2][32];
#pragma unroll
          for (int c = 0; c < kBN; c += 2) {
            const float2 x = __ffma2_rn(make_float2(s[c >> 5][c & 31], s[c >> 5][(c + 1) & 31]), sc2, nm2);
            float p0, p1;
            if (kEmuEvery > 0 && ((c >> 1) % (kEmuEvery > 0 ? kEmuEvery : 1)) == kEmuEvery - 1) {
              exp2_poly2(x.x, x.y, p0, p1);
            } else {
              p0 = ex2(x.x);
              p1 = ex2(x.y);
            }
            rs[(c >> 1) & 3] = __fadd2_rn(rs[(c >> 1) & 3], make_float2(p0, p1));
            pk[c >> 6][(c >> 1) & 31] = pack16x2<F16>(p0, p1);
            // the first 64 keys' P go to TMEM (over S columns already read) as soon as they
            // are packed, so that half of P need not stay in registers
            if (c == 62) tmem_st32(S, pk[0]);
          }
          l += ((rs[0].x + rs[0].y) + (rs[1].x + rs[1].y)) + ((rs[2].x + rs[2].y) + (rs[3].x + rs[3].y));
          // rescale O (complete up to tile j-1: the S_j commit covers every earlier MMA)
          if (__any_sync(0xffffffffu, bump && j > j0)) {
            const float f = (bump && j > j0) ? corr : 1.f;
#pragma unroll
            for (int c = 0; c < HDV / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(O + c * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * f);
              tmem_st32(O + c * 32, o);
            }
          }
          tmem_st32(S + 32, pk[1]);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_addr(&bars->p_ready[q]));
        }
      }
      // ---- epilogue: O / l -> bf16, statistics ------------------------------------------------
      const bool have_o = ok && n > j0 && (q == 0 || has1);
      if (have_o) {
        ok = __all_sync(0xffffffffu, wait_bar(bar_addr(&bars->o_done[q]), odc & 1, abort, a.status));
        ++odc;
      }
      tc_fence_after();
      if (q == 0 || has1) {
        const bool store = r < (q == 0 ? w.rows0 : w.rows1);
        const bool bhsd = a.layout == ATTN_BHSD;
        uint16_t* out = static_cast<uint16_t*>(a.out);  // bf16 or f16 bit patterns
        // this row's own result: o = O / l, max and sum in natural-log units
        // a row that saw no key keeps mraw = -inf (its sum holds only the polynomial's tiny
        // values for masked scores) and gives a zero output, max -inf and sum 0
        const bool any = mraw > -INFINITY && l > 0.f && ok;
        const float m_loc = any ? mraw * a.scale : -INFINITY;
        const float l_loc = any ? l * ex2(m - mraw * scale_log2) : 0.f;
        float f_o = any ? __frcp_rn(l) : 0.f;  // factor on the unnormalised O in TMEM
        float f_prev = 0.f;               // factor on the accumulator's previous output row
        int64_t orow, so;
        if (a.acc_mode == kAccNone) {
          orow = bhsd ? (((int64_t)w.b * a.Nq + hq) * a.Sq + i) * HDV : ((int64_t)(w.q0 + i) * a.Nq + hq) * HDV;
          so = bhsd ? ((int64_t)w.b * a.Nq + hq) * a.Sq + i : (int64_t)(w.q0 + i) * a.Nq + hq;
          if (store && a.smax != nullptr) {
            a.smax[so] = m_loc;
            a.ssum[so] = l_loc;
          }
        } else {
          // accumulator in the merge layouts: BHSD -> output [Sq, B, Nq*D] (SBH), statistics
          // [B, Nq, Sq, 8]; TND -> output [T, Nq*D], statistics [T, Nq, 8]
          orow = bhsd ? (((int64_t)i * a.B + w.b) * a.Nq + hq) * HDV : ((int64_t)(w.q0 + i) * a.Nq + hq) * HDV;
          so = (bhsd ? ((int64_t)w.b * a.Nq + hq) * a.Sq + i : (int64_t)(w.q0 + i) * a.Nq + hq) * 8;
          if (store) merge_into_stats(a, so, m_loc, l_loc, &f_prev, &f_o);
        }
        // A warp whose 32 rows all lie in the sequence writes its plain output through its
        // shared-memory slot, 64 columns at a time, with a TMA store of the 32 x 64 box (the
        // layout the tensor map's 128-byte swizzle expects); otherwise each thread stores its row.
        const bool tma_out = a.acc_mode == kAccNone && __all_sync(0xffffffffu, store);
        const uint32_t stg = smem_u32(smem + C::kStageOff) + (uint32_t)warp * 4096u;
        const int wrow0 = i - lane;  // the warp's first row within the sequence
        // the output row leaves TMEM 64 columns per round trip (two loads, then one wait)
        uint32_t oc[2][32];
#pragma unroll
        for (int c = 0; c < HDV / 32; ++c) {
          if ((c & 1) == 0) {
            if (have_o && ok) {
              tmem_ld32(O + c * 32, oc[0]);
              tmem_ld32(O + (c + 1) * 32, oc[1]);
              tmem_wait_ld();
            } else {
#pragma unroll
              for (int x = 0; x < 32; ++x) oc[0][x] = oc[1][x] = 0u;
            }
            if (tma_out) {
              // the slot's previous TMA store (the last 64 columns, or the previous item's) must
              // have read it; that wait overlaps the TMEM loads above
              if (lane == 0) bulk_wait_read0();
              __syncwarp();
            }
          }
          const uint32_t (&o)[32] = oc[c & 1];
          if (store) {
            uint4* dst = reinterpret_cast<uint4*>(out + orow + c * 32);
            uint32_t prev[16];
            if (a.acc_mode == kAccMerge) {
#pragma unroll
              for (int x = 0; x < 4; ++x) {
                const uint4 t = dst[x];
                prev[4 * x] = t.x;
                prev[4 * x + 1] = t.y;
                prev[4 * x + 2] = t.z;
                prev[4 * x + 3] = t.w;
              }
            }
            // O is finite, so a row that saw no key (f_o = 0) gives zeros
            uint32_t pkd[16];
            if (a.acc_mode == kAccMerge) {
#pragma unroll
              for (int x = 0; x < 16; ++x) {
                const float2 pv = unpack16x2<F16>(prev[x]);
                pkd[x] = pack16x2<F16>(fmaf(pv.x, f_prev, __uint_as_float(o[2 * x]) * f_o),
                                       fmaf(pv.y, f_prev, __uint_as_float(o[2 * x + 1]) * f_o));
              }
            } else {
#pragma unroll
              for (int x = 0; x < 16; ++x)
                pkd[x] = pack16x2<F16>(__uint_as_float(o[2 * x]) * f_o, __uint_as_float(o[2 * x + 1]) * f_o);
            }
            if (tma_out) {
#pragma unroll
              for (int x = 0; x < 4; ++x) {
                const uint32_t chunk = (uint32_t)(((c & 1) * 4 + x) ^ (lane & 7));
                st_shared_v4(stg + (uint32_t)lane * 128u + chunk * 16u, pkd[4 * x], pkd[4 * x + 1], pkd[4 * x + 2],
                             pkd[4 * x + 3]);
              }
            } else {
#pragma unroll
              for (int x = 0; x < 4; ++x)
                dst[x] = make_uint4(pkd[4 * x], pkd[4 * x + 1], pkd[4 * x + 2], pkd[4 * x + 3]);
            }
          }
          if (tma_out && (c & 1) == 1) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (bhsd)
                tma_store_3d(&tm_o, stg, 64 * (c >> 1), wrow0, w.b * a.Nq + hq);
              else
                tma_store_3d(&tm_o, stg, 64 * (c >> 1), hq, w.q0 + wrow0);
              bulk_commit();
            }
          }
        }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_addr(&bars->unit_empty[slot]));
      }
      if (lane == 0) bulk_wait0();  // this warp's output stores are complete before it exits
    }

  // ---- teardown ----------------------------------------------------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (sched != nullptr && threadIdx.x == 0) {
    // the last block to finish puts the slot's counters back to 0 for the next launch using it
    __threadfence();
    if (atomicAdd(sched + 1, 1) == (int)gridDim.x - 1) {
      atomicExch(sched, 0);
      atomicExch(sched + 1, 0);
    }
  }
}

// ------------------------------------------------------------------------------------------------
// host side: tensor maps and launch
// ------------------------------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D map over a 16-bit tensor viewed as (D, dim1, dim2), box (64, box1, box2), 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t D, uint64_t dim1, uint64_t dim2,
              uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box1, uint32_t box2,
              bool f16) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {D, dim1, dim2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {64, box1, box2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
            const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The scheduler slot (g_sched) for a launch on stream `st`, or null: static division of the
// items. Every stream of every device gets a slot of its own on first use (launches on one
// stream run one after another, so they can share it). A launch gets none when its stream is
// being captured into a graph (a graph may be replayed on any stream, next to other launches),
// for the per-thread default stream (one handle, a different stream in every thread), and once
// all slots of the device are taken.
cudaError_t sched_slot(cudaStream_t st, int** out) {
  *out = nullptr;
  if (st == cudaStreamPerThread) return cudaSuccess;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(st, &cap);
  if (e != cudaSuccess) return e;
  if (cap != cudaStreamCaptureStatusNone) return cudaSuccess;
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  constexpr int kMaxDevices = 64;
  if (dev < 0 || dev >= kMaxDevices) return cudaSuccess;
  static std::mutex mu;
  static int* base[kMaxDevices] = {};
  static int used[kMaxDevices] = {};
  static std::map<std::pair<int, cudaStream_t>, int> slot_of;
  std::lock_guard<std::mutex> lk(mu);
  if (base[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_sched);
    if (e != cudaSuccess) return e;
    base[dev] = static_cast<int*>(p);
  }
  const auto key = std::make_pair(dev, st);
  auto f = slot_of.find(key);
  int slot;
  if (f != slot_of.end()) {
    slot = f->second;
  } else {
    if (used[dev] >= kSchedSlots) return cudaSuccess;
    slot = used[dev]++;
    slot_of.emplace(key, slot);
  }
  *out = base[dev] + 2 * slot;
  return cudaSuccess;
}

template <int HD, int HDV, bool F16>
cudaError_t launch_hd(const FwdArgs& a, cudaStream_t st) {
  using C = Cfg<HD, HDV, F16>;
  CUtensorMap tq, tk, tv;
  const uint64_t D = HD, Dv = HDV;
  bool ok;
  if (a.layout == ATTN_BHSD) {
    // (d, s, b*h): rows of a head are contiguous
    ok = make_map(&tq, a.q, D, a.Sq, (uint64_t)a.B * a.Nq, D * 2, (uint64_t)a.Sq * D * 2, kBM, 1, F16) &&
         make_map(&tk, a.k, D, a.Skv, (uint64_t)a.B * a.Nkv, D * 2, (uint64_t)a.Skv * D * 2, kBN, 1, F16) &&
         make_map(&tv, a.v, Dv, a.Skv, (uint64_t)a.B * a.Nkv, Dv * 2, (uint64_t)a.Skv * Dv * 2, kBN, 1, F16);
  } else {
    // (d, head, token): a tile is 128 tokens of one head
    const uint64_t tq_rows = a.Sq > 0 ? a.Sq : 1, tk_rows = a.Skv > 0 ? a.Skv : 1;
    ok = make_map(&tq, a.q, D, a.Nq, tq_rows, D * 2, (uint64_t)a.Nq * D * 2, 1, kBM, F16) &&
         make_map(&tk, a.k, D, a.Nkv, tk_rows, D * 2, (uint64_t)a.Nkv * D * 2, 1, kBN, F16) &&
         make_map(&tv, a.v, Dv, a.Nkv, tk_rows, Dv * 2, (uint64_t)a.Nkv * Dv * 2, 1, kBN, F16);
  }
  // the plain output has Q's layout with the value head size; the TMA stores write 32-row boxes
  CUtensorMap to = tq;  // not read by the kernel when the output is an accumulator
  if (ok && a.acc_mode == 0) {
    if (a.layout == ATTN_BHSD)
      ok = make_map(&to, a.out, Dv, a.Sq, (uint64_t)a.B * a.Nq, Dv * 2, (uint64_t)a.Sq * Dv * 2, 32, 1, F16);
    else
      ok = make_map(&to, a.out, Dv, a.Nq, a.Sq > 0 ? a.Sq : 1, Dv * 2, (uint64_t)a.Nq * Dv * 2, 1, 32, F16);
  }
  if (!ok) return cudaErrorInvalidValue;
  auto kernel = a.mask != nullptr                 ? fwd_bf16_kernel<HD, HDV, F16, 2>
                : a.mask_mode == ATTN_MASK_BAND ? fwd_bf16_kernel<HD, HDV, F16, 1>
                                                : fwd_bf16_kernel<HD, HDV, F16, 0>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  // The register split inside the kernel (softmax warpgroups up to kRegsSoftmax, the producer
  // warpgroup down to kRegsProducer) waits for registers the block must have been launched with:
  // refuse to launch a build whose kernel holds fewer than kRegsLaunch a thread.
  {
    static std::atomic<int> checked[3] = {};
    const int which = kernel == fwd_bf16_kernel<HD, HDV, F16, 2> ? 2 : kernel == fwd_bf16_kernel<HD, HDV, F16, 1> ? 1 : 0;
    if (checked[which].load(std::memory_order_acquire) == 0) {
      cudaFuncAttributes fa;
      e = cudaFuncGetAttributes(&fa, kernel);
      if (e != cudaSuccess) return e;
      if (fa.numRegs < kRegsLaunch || fa.maxThreadsPerBlock < kThreads) return cudaErrorInvalidConfiguration;
      checked[which].store(1, std::memory_order_release);
    }
  }
  int units_per_seq = 0;
  int64_t units;
  if (a.layout == ATTN_BHSD) {
    units_per_seq = (a.Sq + rows_per_item(a) - 1) / rows_per_item(a);
    units = (int64_t)a.B * units_per_seq;
  } else {
    units = (a.Sq + rows_per_item(a) - 1) / rows_per_item(a) + a.B;
  }
  const int64_t items = units * (pair_heads(a) ? a.Nq / 2 : a.Nq);
  if (items <= 0) return cudaSuccess;
  if (items > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const float scale_log2 = a.scale * 1.4426950408889634f;
  // one persistent block per SM (fewer when there are fewer items)
  const int64_t grid = items < a.num_sms ? items : (a.num_sms > 0 ? a.num_sms : 1);
  int* sched = nullptr;
  cudaError_t se = sched_slot(st, &sched);
  if (se != cudaSuccess) return se;
  kernel<<<(unsigned)grid, kThreads, C::kSmemBytes, st>>>(tq, tk, tv, to, a, units_per_seq, scale_log2, (int)items,
                                                           sched);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_bf16(const FwdArgs& a, cudaStream_t st) {
  const bool f16 = a.dtype == ATTN_F16;
  if (a.D == 128 && a.Dv == 64) return f16 ? launch_hd<128, 64, true>(a, st) : launch_hd<128, 64, false>(a, st);
  if (a.D == 128) return f16 ? launch_hd<128, 128, true>(a, st) : launch_hd<128, 128, false>(a, st);
  return f16 ? launch_hd<64, 64, true>(a, st) : launch_hd<64, 64, false>(a, st);
}

}  // namespace sdpa
