// Persistent causal forward for sm_100a (tcgen05 + TMEM + TMA).
//
// Article "Lightning Attention-2 新一代注意力机制", section
// "Lightning Attention-2简介", point 2 (Fig. 3): a block's output is the masked
// left product inside the block plus the right product of its queries with the
// KV state accumulated over the earlier blocks; point 3: tiles go HBM -> on-chip
// -> HBM once.
//
// Work decomposition. The B*H sequences are laid end to end as one list of
// (sequence, block) tasks of Bk rows. The host cuts that list into R contiguous
// ranges (about one per SM, balanced by a cost model) and CTA j runs ranges
// j, j+G, ... A range may cross sequence boundaries; it is processed as
// segments, one per sequence it touches. A segment that starts at block 0
// starts from a zero state. The first segment of a range may start inside a
// sequence; its initial state is either
//   * rebuilt by a pre-pass over the sequence's earlier blocks (K and V only,
//     KV += K^T V, no output) - one launch, no workspace; or
//   * the sum of the per-range states that a state-only launch of the same
//     kernel (KIND_AGG) wrote for the earlier ranges of that sequence; the
//     three consumer warpgroups add them up at CTA start.
// The host picks the cheaper of the two from a cost model (plan_ranges).
//
// Per main block (one CTA, warp-specialised):
//   S   = Q K^T           tcgen05 M=Bk N=Bk K=d          TMEM
//   P   = bf16(S ⊙ M_B)   mask warpgroup                  SMEM (K-major)
//   KV += K^T V           tcgen05 M=d N=dv K=Bk          TMEM (fp32 state)
//   O   = Q bf16(KV_old)  tcgen05 M=Bk N=dv K=d          TMEM (snapshot taken before the update)
//   O  += P V             tcgen05 M=Bk N=dv K=Bk
// One warp issues the MMAs (one elected lane per instruction) in the order
// S; Q bf16(KV_old) once the snapshot of the old state is in SMEM; the KV
// update; P V once the mask warpgroup has written P. The state warpgroup turns
// the updated state into the next snapshot while P V and the next block's S
// run. At Bk=64 O leaves through a swizzled staging tile and TMA stores.
#pragma once

#include "la2_sm100.cuh"

namespace la2 {
namespace sm100 {

// Optional per-step timestamps of CTA 0 (globaltimer, ns) for pipeline
// studies: build with -DLA2_TRACE and read them with la2_trace_read().
// Per-step events are those of CTA LA2_TRACE_CTA (default 0); LA2_TRACE_CTA_POINT
// stamps one event per CTA (start, first main step, end).
#ifdef LA2_TRACE
#ifndef LA2_TRACE_CTA
#define LA2_TRACE_CTA 0
#endif
constexpr int kTraceEvents = 16, kTraceSteps = 512, kTraceCtas = 160;
__device__ unsigned long long g_trace[kTraceEvents][kTraceSteps];
__device__ unsigned long long g_trace_cta[4][kTraceCtas];
#define LA2_TRACE_POINT(ev, idx)                                                             \
  do {                                                                                       \
    if (blockIdx.x == LA2_TRACE_CTA && (idx) < kTraceSteps) g_trace[ev][idx] = globaltimer_ns(); \
  } while (0)
#define LA2_TRACE_CTA_POINT(ev)                                                   \
  do {                                                                            \
    if (blockIdx.x < kTraceCtas) g_trace_cta[ev][blockIdx.x] = globaltimer_ns(); \
  } while (0)
#else
#define LA2_TRACE_POINT(ev, idx) \
  do {                           \
  } while (0)
#define LA2_TRACE_CTA_POINT(ev) \
  do {                          \
  } while (0)
#endif

constexpr int kMaxRanges = 160;  // the range table travels as a kernel parameter (< 4 KB)

struct RangeTable {
  int32_t R;            // number of ranges
  int32_t prefix_mode;  // 0: pre-pass rebuilds a mid-sequence start; 1: sum of range states
  int64_t T;            // blocks per sequence
  int64_t starts[kMaxRanges + 1];  // range r = tasks [starts[r], starts[r+1])
};

struct CausalParams {
  __nv_bfloat16* o;  // [BH][N][DV]
  float* agg;        // range states [R][D*DV] (prefix_mode 1, or KIND_AGG output); see agg_f4
  int64_t N;
  int64_t spin_limit;
  int32_t H, G;      // query heads per batch, query heads per K/V head (kv_seq)
};

enum Kind : int { KIND_MAIN = 0, KIND_AGG = 1 };

struct Step {
  int64_t bh;
  int32_t blk;
  int32_t range;
  uint8_t pre;        // K/V-only state step (pre-pass or range state)
  uint8_t pre_first;  // first state step of a fresh state
  uint8_t pre_last;   // last state step (its state is consumed next)
  uint8_t seg_first;  // first main step of a segment
  uint8_t seg_last;   // last main step of a segment
  uint8_t init;       // seg_first: 0 zero state, 1 state from the pre-pass, 2 from range states
};

// Deterministic walk of this CTA's steps; every role runs its own copy.
template <int KIND>
struct StepIter {
  const RangeTable* rt;
  // Task indices fit in 32 bits (the host rejects larger task lists).
  int32_t r;
  int32_t f, fend;      // KIND_MAIN: next task / end of the current range
  int32_t seg_end;      // end of the open segment (0 when none is open)
  int32_t seg_lo;
  int32_t bh;           // sequence of task f
  int32_t blk;          // block of task f inside its sequence
  uint8_t seg_init;
  int32_t pre_bh;
  int32_t pre_blk, pre_end, pre_lo;

  __device__ __forceinline__ void begin(const RangeTable* t) {
    rt = t;
    r = static_cast<int32_t>(blockIdx.x) - static_cast<int32_t>(gridDim.x);
    f = fend = 0;
    seg_end = 0;
    seg_lo = 0;
    bh = blk = 0;
    seg_init = 0;
    pre_bh = 0;
    pre_blk = pre_end = pre_lo = 0;
  }

  // Next step of this CTA; false when its ranges are exhausted. No recursion
  // and one division per range, so every role can call it each step.
  __device__ __forceinline__ bool next(Step& s) {
    const int32_t T = static_cast<int32_t>(rt->T);
    if (pre_blk >= pre_end) {
      if (KIND == KIND_AGG) {
        // One state pass per range whose end falls inside a sequence.
        bool found = false;
        while (!found) {
          r += static_cast<int32_t>(gridDim.x);
          if (r >= rt->R - 1) return false;  // the last range's state is never needed
          const int32_t e = static_cast<int32_t>(rt->starts[r + 1]);
          const int32_t hb = (e - 1) / T;
          if (e - hb * T == T) continue;  // ends on a sequence boundary
          const int32_t lo = max(static_cast<int32_t>(rt->starts[r]), hb * T);
          pre_bh = hb;
          pre_lo = lo - hb * T;
          pre_blk = pre_lo;
          pre_end = e - hb * T;
          found = true;
        }
      } else {
        if (f >= fend) {
          do {
            r += static_cast<int32_t>(gridDim.x);
            if (r >= rt->R) return false;
            f = static_cast<int32_t>(rt->starts[r]);
            fend = static_cast<int32_t>(rt->starts[r + 1]);
          } while (f >= fend);
          seg_end = 0;
          bh = f / T;
          blk = f - bh * T;
        }
        bool main_now = true;
        if (seg_end == 0) {  // a segment opens at f
          seg_lo = f;
          seg_end = min(fend, f + (T - blk));
          if (blk == 0) {
            seg_init = 0;
          } else if (rt->prefix_mode == 0) {
            seg_init = 1;  // pre-pass over the sequence's earlier blocks first
            pre_bh = bh;
            pre_lo = 0;
            pre_blk = 0;
            pre_end = static_cast<int32_t>(blk);
            main_now = false;
          } else {
            seg_init = 2;
          }
        }
        if (main_now) {
          s.bh = bh;
          s.blk = static_cast<int32_t>(blk);
          s.range = r;
          s.pre = 0;
          s.pre_first = s.pre_last = 0;
          s.seg_first = f == seg_lo;
          s.seg_last = f == seg_end - 1;
          s.init = seg_init;
          ++f;
          if (++blk == T) {
            blk = 0;
            ++bh;
          }
          if (f == seg_end) seg_end = 0;
          return true;
        }
      }
    }
    s.bh = pre_bh;
    // The state launch walks each range from its last block down: when it
    // ends, L2 still holds the K and V it read last, the first blocks of the
    // ranges, which the main launch reads first. (The state is a sum.)
    s.blk = KIND == KIND_AGG ? pre_lo + pre_end - 1 - pre_blk : pre_blk;
    s.range = r;
    s.pre = 1;
    s.pre_first = pre_blk == pre_lo;
    s.pre_last = pre_blk == pre_end - 1;
    s.seg_first = s.seg_last = 0;
    s.init = 0;
    ++pre_blk;
    return true;
  }
};

template <int BK, int D, int DV, int KIND = KIND_MAIN>
struct CCfg {
  // The state-only pass (KIND_AGG) holds no Q, P, snapshot or O tiles and
  // spends that space on a deeper K/V ring: its loads are latency-bound.
  static constexpr bool AGG = KIND == KIND_AGG;
  // Bk=128: P lives in tensor memory (the P V MMA reads its A operand there)
  // and O has one TMEM buffer; the shared memory a P tile would take carries a
  // second Q slot instead, so Q rides with K and V in a 2-deep ring and the
  // next block's Q arrives while the current block computes.
  static constexpr bool P_TMEM = BK == 128 && !AGG;
  static constexpr int QS = BK == 64 ? 3 : 2;
  static constexpr int KS = AGG ? (BK == 64 ? 6 : 3) : (BK == 64 ? 3 : 2);
  static constexpr int NSB = BK == 64 ? 2 : 1;    // S buffers (TMEM)
  static constexpr int NPB = BK == 64 ? 2 : 1;    // P buffers (SMEM at Bk=64, TMEM at Bk=128)
  static constexpr int NOB = P_TMEM ? 1 : 2;      // O buffers (TMEM)
  // One snapshot buffer suffices: the state role writes snapshot m+1 only after
  // update(m) completed, and update(m) is issued after QKV(m) read snapshot m.
  static constexpr int NSNAP = 1;
  // Bk=64: O leaves through a swizzled staging tile and per-warp TMA stores
  // (plain row stores from the epilogue crowd the SM's memory-instruction
  // queue that the MMA warp's barrier and tcgen05 instructions also use).
  static constexpr bool TMA_STORE = BK == 64 && !AGG;
  static constexpr int OSTAGE = TMA_STORE ? 2 : 0;
  // Bk=128: O(m) is staged in Q(m)'s tile (dead once P V(m) completed; same
  // size and swizzled layout) and leaves by TMA stores; the epilogue, not the
  // MMA warp, then releases the Q slot, after its stores have read the tile.
  static constexpr bool O_IN_Q = BK == 128 && !AGG;
  // Q rides in the K/V ring (one barrier per step) when the rings are as deep
  // and the MMA warp releases Q.
  static constexpr bool QWITHKV = QS == KS && !O_IN_Q;
  // With as many P as O buffers the P-free signal is the O-full commit of the
  // block that read the P buffer (P V is the last MMA writing that O).
  static constexpr bool MERGE_OP = NPB == NOB;
  static constexpr int DP = D / 64;
  static constexpr int VP = DV / 64;
  static constexpr int QTILE = BK * D * 2;
  static constexpr int KTILE = BK * D * 2;
  static constexpr int VTILE = BK * DV * 2;
  static constexpr int PTILE = BK * BK * 2;
  static constexpr int SNAP = D * DV * 2;
  static constexpr int OTILE = BK * DV * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + (AGG ? 0 : QS * QTILE);
  static constexpr int OFF_V = OFF_K + KS * KTILE;
  static constexpr int OFF_P = OFF_V + KS * VTILE;
  static constexpr int OFF_SNAP = OFF_P + ((AGG || P_TMEM) ? 0 : NPB * PTILE);
  static constexpr int OFF_OST = OFF_SNAP + (AGG ? 0 : NSNAP * SNAP);
  static constexpr int OFF_BAR = OFF_OST + OSTAGE * OTILE;
  static constexpr int NBAR = 2 * QS + 2 * KS + 19;  // rings + 8 pairs + 3 singles
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  static constexpr uint32_t COL_KV = 0;
  static constexpr uint32_t COL_O = 128;  // NOB buffers of 128 columns
  static constexpr uint32_t COL_P = 256;  // P_TMEM: BK rows x BK bf16 (BK / 2 columns)
  static constexpr uint32_t COL_S = 384;  // NSB buffers of BK columns
  // Bk=64: O is accumulated transposed, O^T = KV^T Q^T + V^T P^T (M = dv = 128
  // rows of the tensor datapath instead of M = Bk = 64: the two O products at
  // full rate), BK columns per buffer; the epilogue transposes while staging.
  static constexpr bool OT = BK == 64 && !AGG;
  static constexpr uint32_t O_COLS = OT ? BK : 128;  // TMEM columns of one O buffer
  static constexpr uint32_t ID_S = make_idesc(BK, BK, false, false);
  static constexpr uint32_t ID_QKV = OT ? make_idesc(DV, BK, true, false) : make_idesc(BK, DV, false, true);
  static constexpr uint32_t ID_UPD = make_idesc(D, DV, true, true);
  static constexpr uint32_t ID_PV = OT ? make_idesc(DV, BK, true, false) : make_idesc(BK, DV, false, true);
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(COL_S + NSB * BK <= kTmemCols, "TMEM budget");
  static_assert(COL_O + NOB * O_COLS <= (P_TMEM ? COL_P : COL_S) && COL_P + BK / 2 <= COL_S,
                "TMEM columns of O, P and S overlap");
};

template <int D>
__device__ __forceinline__ void put_snap_row(uint32_t sbase, int r, const uint32_t* v, int col0) {
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    const int col = col0 + q4 * 8;
    const int panel = col >> 6, cj = (col & 63) >> 3;
    st_shared_v4(sbase + panel * D * 128 + r * 128 + ((cj ^ (r & 7)) << 4),
                 pack_bf16x2(__uint_as_float(v[q4 * 8 + 0]), __uint_as_float(v[q4 * 8 + 1])),
                 pack_bf16x2(__uint_as_float(v[q4 * 8 + 2]), __uint_as_float(v[q4 * 8 + 3])),
                 pack_bf16x2(__uint_as_float(v[q4 * 8 + 4]), __uint_as_float(v[q4 * 8 + 5])),
                 pack_bf16x2(__uint_as_float(v[q4 * 8 + 6]), __uint_as_float(v[q4 * 8 + 7])));
  }
}

// Row r of the state: sum over the earlier ranges of this sequence of their
// range states (fp32, HBM), written to TMEM (fp32) and, rounded to bf16, to
// the snapshot at `sbase`. Cold path (once per range), kept out of line.
// A range state (D x DV fp32) is stored column-chunk-major: float4 j (columns
// 4j..4j+3) of row r at float4 index j*D + r. The 32 threads of a warp own 32
// consecutive rows, so each 16-byte access of the warp covers 512 contiguous
// bytes (row-major rows would put the warp's accesses 4*DV bytes apart).
template <int D>
__device__ __forceinline__ int64_t agg_f4(int r, int j) {
  return static_cast<int64_t>(j) * D + r;
}

template <int D, int DV>
__device__ __noinline__ void init_from_ranges(const float* agg, const RangeTable& rt, int32_t range,
                                              int64_t head0, int r, uint32_t tKV, uint32_t sbase) {
#pragma unroll 1
  for (int c32 = 0; c32 < DV / 32; ++c32) {
    float acc[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) acc[j] = 0.f;
    if (r >= 0) {
      for (int rr = range - 1; rr >= 0 && rt.starts[rr + 1] > head0; --rr) {
        const float4* src = reinterpret_cast<const float4*>(agg + static_cast<int64_t>(rr) * D * DV);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const float4 x = src[agg_f4<D>(r, c32 * 8 + q4)];
          acc[4 * q4] += x.x;
          acc[4 * q4 + 1] += x.y;
          acc[4 * q4 + 2] += x.z;
          acc[4 * q4 + 3] += x.w;
        }
      }
    }
    uint32_t u[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(acc[j]);
    tmem_st32(tKV + c32 * 32, u);
    if (r >= 0) put_snap_row<D>(sbase, r, u, c32 * 32);
  }
  tmem_st_wait();
}

// Initial state of the CTA's first range when it starts inside a sequence
// (range-state mode): the sum of the states of the sequence's earlier ranges.
// Run once at CTA start by the three consumer warpgroups together; warp w4 of
// each owns TMEM lanes (state rows) 32*w4 .. 32*w4+31 and warpgroup `part`
// (0..2) sums the 32-column chunks {0, 3}, {1} or {2} of those rows, two
// ranges' loads in flight per round.
template <int D, int DV>
__device__ __noinline__ void init_state_coop(const float* agg, const RangeTable& rt, int32_t range,
                                             int64_t head0, int part, int w4, int lane,
                                             uint32_t tKV, uint32_t sbase) {
  static_assert(D == 128 && DV == 128, "one TMEM lane per state row, four column chunks");
  int nprev = 0;
  while (range - 1 - nprev >= 0 && rt.starts[range - nprev] > head0) ++nprev;
  const int r = 32 * w4 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(32 * w4) << 16;
  for (int c = part; c < DV / 32; c += 3) {
    float acc[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) acc[j] = 0.f;
    int i = 0;
    for (; i + 2 <= nprev; i += 2) {
      const float4* s0 = reinterpret_cast<const float4*>(agg + static_cast<int64_t>(range - 1 - i) * D * DV);
      const float4* s1 = s0 - static_cast<int64_t>(D) * DV / 4;
      float4 x[8], y[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        x[q] = s0[agg_f4<D>(r, c * 8 + q)];
        y[q] = s1[agg_f4<D>(r, c * 8 + q)];
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        acc[4 * q] += x[q].x + y[q].x;
        acc[4 * q + 1] += x[q].y + y[q].y;
        acc[4 * q + 2] += x[q].z + y[q].z;
        acc[4 * q + 3] += x[q].w + y[q].w;
      }
    }
    if (i < nprev) {
      const float4* s0 = reinterpret_cast<const float4*>(agg + static_cast<int64_t>(range - 1 - i) * D * DV);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 x = s0[agg_f4<D>(r, c * 8 + q)];
        acc[4 * q] += x.x;
        acc[4 * q + 1] += x.y;
        acc[4 * q + 2] += x.z;
        acc[4 * q + 3] += x.w;
      }
    }
    uint32_t u[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(acc[j]);
    tmem_st32(tKV + lane_off + c * 32, u);
    put_snap_row<D>(sbase, r, u, c * 32);
  }
  tmem_st_wait();
}

template <int BK, int D, int DV, int KIND>
__global__ void __launch_bounds__(kThreads, 1)
la2_causal_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_o,
                        const __grid_constant__ RangeTable rt, const CausalParams prm) {
  using CF = CCfg<BK, D, DV, KIND>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int wg = warp >> 2;
  const int w4 = warp & 3;

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + CF::OFF_BAR);
  uint64_t* q_full = bar;
  uint64_t* q_empty = q_full + CF::QS;
  uint64_t* kv_full = q_empty + CF::QS;
  uint64_t* kv_empty = kv_full + CF::KS;
  uint64_t* s_full = kv_empty + CF::KS;
  uint64_t* p_full = s_full + 2;
  uint64_t* p_empty = p_full + 2;
  uint64_t* snap_full = p_empty + 2;
  uint64_t* snap_free = snap_full + 2;
  uint64_t* o_full = snap_free + 2;
  uint64_t* o_empty = o_full + 2;
  uint64_t* kv_updated = o_empty + 2;
  uint64_t* seg_ack = kv_updated + 1;
  uint64_t* drain = seg_ack + 1;
  uint64_t* stage_free = drain + 1;       // [2] transposing epilogue: staging tile free
  uint64_t* stage_full = stage_free + 2;  // [2] transposing epilogue: staging tile written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stage_full + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < CF::QS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], CF::O_IN_Q ? 4 : 1);  // O_IN_Q: one arrival per epilogue warp
    }
    for (int s = 0; s < CF::KS; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&p_empty[s], 1);
      mbar_init(&snap_full[s], 128);
      mbar_init(&snap_free[s], 1);
      mbar_init(&o_full[s], 1);
      mbar_init(&o_empty[s], 128);
    }
    mbar_init(kv_updated, 1);
    mbar_init(seg_ack, 128);
    mbar_init(drain, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&stage_free[s], 1);
      mbar_init(&stage_full[s], 128);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kWarpProducer && lane == 0) {
    if (KIND == KIND_MAIN) tma_prefetch(&tm_q);
    if (KIND == KIND_MAIN && (CF::TMA_STORE || CF::O_IN_Q)) tma_prefetch(&tm_o);
    tma_prefetch(&tm_k);
    tma_prefetch(&tm_v);
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t lim = prm.spin_limit;
  // Everything above touches only this CTA's shared memory, TMEM and kernel
  // parameters; from here on global memory is read and written.
  pdl_launch_dependents();
  pdl_wait();
  if (threadIdx.x == 0) LA2_TRACE_CTA_POINT(0);

  // Range-state mode: a CTA's range (at most one per CTA) that starts inside
  // a sequence gets its initial state from the consumer warpgroups before
  // they take up their roles. The producer warp holds its first loads until
  // then: behind a full TMA ring the state loads would queue for microseconds.
  bool first_init_ready = false;
  if (KIND == KIND_MAIN && rt.prefix_mode == 1 && static_cast<int32_t>(blockIdx.x) < rt.R) {
    const int64_t f0 = rt.starts[blockIdx.x];
    const int64_t head0 = (f0 / rt.T) * rt.T;
    if (f0 != head0 && (wg >= 1 || warp == kWarpProducer)) {
      if (wg >= 1) {
        init_state_coop<D, DV>(prm.agg, rt, static_cast<int32_t>(blockIdx.x), head0, wg - 1, w4,
                               lane, tmem + CF::COL_KV, smem_u32(smem + CF::OFF_SNAP));
        first_init_ready = true;
        fence_proxy_async();
        tc_fence_before();
      }
      named_bar_sync(1, 416);  // warps 4..15 and the producer warp
      tc_fence_after();
    }
  }

  uint8_t* sQ = smem + CF::OFF_Q;
  uint8_t* sK = smem + CF::OFF_K;
  uint8_t* sV = smem + CF::OFF_V;
  uint8_t* sP = smem + CF::OFF_P;
  uint8_t* sSnap = smem + CF::OFF_SNAP;

  if (warp == kWarpProducer) {
    // ================================================================ TMA
    if (lane == 0) {
      StepIter<KIND> it;
      it.begin(&rt);
      Step st;
      uint32_t g = 0, m = 0;
      int issued_kv = 0, issued_q = 0;
      bool ok = true;
      while (ok && it.next(st)) {
        const int row = st.blk * BK;
        const int zz = static_cast<int>(st.bh);                               // Q (and O)
        const int zkv = static_cast<int>(kv_seq(st.bh, prm.H, prm.G));        // K, V
        const int ks = g % CF::KS;
        if (!wait_bar(&kv_empty[ks], ((g / CF::KS) & 1) ^ 1, lim, abort_flag, 101)) { ok = false; break; }
        LA2_TRACE_POINT(0, g);
        const bool q_here = CF::QWITHKV && !st.pre;
        mbar_expect_tx(&kv_full[ks], CF::KTILE + CF::VTILE + (q_here ? CF::QTILE : 0));
        for (int p = 0; p < CF::DP; ++p)
          tma_load_3d(sK + ks * CF::KTILE + p * BK * 128, &tm_k, &kv_full[ks], 64 * p, row, zkv);
        for (int p = 0; p < CF::VP; ++p)
          tma_load_3d(sV + ks * CF::VTILE + p * BK * 128, &tm_v, &kv_full[ks], 64 * p, row, zkv);
        if (q_here)
          for (int p = 0; p < CF::DP; ++p)
            tma_load_3d(sQ + ks * CF::QTILE + p * BK * 128, &tm_q, &kv_full[ks], 64 * p, row, zz);
        ++issued_kv;
        ++g;
        if (!CF::QWITHKV && !st.pre) {
          const int qs = m % CF::QS;
          if (!wait_bar(&q_empty[qs], ((m / CF::QS) & 1) ^ 1, lim, abort_flag, 102)) { ok = false; break; }
          LA2_TRACE_POINT(1, m);
          mbar_expect_tx(&q_full[qs], CF::QTILE);
          for (int p = 0; p < CF::DP; ++p)
            tma_load_3d(sQ + qs * CF::QTILE + p * BK * 128, &tm_q, &q_full[qs], 64 * p, row, zz);
          ++issued_q;
          ++m;
        }
      }
      if (!ok) {
        for (int j = max(0, issued_kv - CF::KS); j < issued_kv; ++j)
          drain_wait(&kv_full[j % CF::KS], (j / CF::KS) & 1);
        for (int j = max(0, issued_q - CF::QS); j < issued_q; ++j)
          drain_wait(&q_full[j % CF::QS], (j / CF::QS) & 1);
      }
    }
  } else if (warp == kWarpMma) {
    // ================================================================ MMA
    // The whole warp runs the issue loop (warp-uniform bookkeeping); one
    // elected lane issues each tcgen05 instruction.
    {
      const uint32_t tKV = tmem + CF::COL_KV;
      StepIter<KIND> it;
      it.begin(&rt);
      Step st, nx;
      bool have = it.next(st);
      uint32_t g = 0, m = 0, sn = 0, acks = 0;
      bool ack_pending = false, s_ready = false, ok = true;
      auto wait_w = [&](uint64_t* b, uint32_t par, int where) -> bool {
        return __all_sync(0xffffffffu, wait_bar(b, par, lim, abort_flag, where));
      };

      auto wait_ack = [&]() -> bool {
        if (!ack_pending) return true;
        if (!wait_w(seg_ack, acks & 1, 110)) return false;
        ++acks;
        ack_pending = false;
        return true;
      };
      // Descriptor templates (start address 0); a tile's descriptor is the
      // template plus its address >> 4, and a k-step adds its byte offset >> 4.
      const uint64_t dK_mn = make_desc(0, BK * 128, 1024);   // MN-major, panels of BK rows
      const uint64_t dKm = make_desc(0, 16, 1024);           // K-major
      const uint64_t dSnap = make_desc(0, D * 128, 1024);    // MN-major, panels of D rows
      const uint32_t sK0 = smem_u32(sK), sV0 = smem_u32(sV), sQ0 = smem_u32(sQ);
      const uint32_t sP0 = smem_u32(sP), sS0 = smem_u32(sSnap);
      auto update = [&](uint32_t slot, bool accumulate) {
        const uint64_t a = dK_mn + ((sK0 + slot * CF::KTILE) >> 4);
        const uint64_t b = dK_mn + ((sV0 + slot * CF::VTILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          mma_bf16_ss_warp(tKV, a + kk * (2048 >> 4), b + kk * (2048 >> 4), CF::ID_UPD,
                      (accumulate || kk > 0) ? 1u : 0u);
      };
      auto qslot = [](uint32_t mm, uint32_t gg) -> uint32_t {
        return CF::QWITHKV ? gg % CF::KS : mm % CF::QS;
      };
      // S(mm) = Q K^T into S buffer mm % NSB; Q slot qslot(mm, gg), K slot gg % KS.
      auto issue_s = [&](uint32_t mm, uint32_t gg) -> bool {
        LA2_TRACE_POINT(5, mm);
        if (!CF::QWITHKV && !wait_w(&q_full[mm % CF::QS], (mm / CF::QS) & 1, 111)) return false;
        if (!wait_w(&kv_full[gg % CF::KS], (gg / CF::KS) & 1, 112)) return false;
        LA2_TRACE_POINT(15, mm);
        // S buffer mm % NSB is free: the mask role read S(mm - NSB) before it
        // arrived on p_full(mm - 1), which this warp waited for before PV(mm - 1).
        tc_fence_after();
        const uint64_t a = dKm + ((sQ0 + qslot(mm, gg) * CF::QTILE) >> 4);
        const uint64_t b = dKm + ((sK0 + (gg % CF::KS) * CF::KTILE) >> 4);
        const uint32_t tS = tmem + CF::COL_S + (mm % CF::NSB) * BK;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * BK * 128 + (kk & 3) * 32) >> 4;
          mma_bf16_ss_warp(tS, a + off, b + off, CF::ID_S, kk > 0);
        }
        mma_commit_warp(&s_full[mm % CF::NSB]);
        LA2_TRACE_POINT(6, mm);
        return true;
      };

      while (have && ok) {
        const bool have_nx = it.next(nx);
        const uint32_t ks = g % CF::KS;
        if (st.pre) {
          if (!wait_w(&kv_full[ks], (g / CF::KS) & 1, 114)) { ok = false; break; }
          if (!wait_ack()) { ok = false; break; }
          LA2_TRACE_POINT(1, g);
          tc_fence_after();
          update(ks, !st.pre_first);
          if (st.pre_last) {
            mma_commit_warp(kv_updated);
            if (KIND == KIND_AGG) ack_pending = true;
          }
          mma_commit_warp(&kv_empty[ks]);
        } else {
          if (m == 0 && lane == 0) LA2_TRACE_CTA_POINT(1);
          if (!s_ready && !issue_s(m, g)) { ok = false; break; }
          s_ready = false;
          const bool needs_snap = !(st.seg_first && st.init == 0);
          const uint32_t sb = sn % CF::NSNAP;
          if (needs_snap &&
              !wait_w(&snap_full[sb], (sn / CF::NSNAP) & 1, 115)) { ok = false; break; }
          if (!wait_ack()) { ok = false; break; }
          LA2_TRACE_POINT(2, m);
          const uint32_t ob = m % CF::NOB;
          const uint32_t tO = tmem + CF::COL_O + ob * CF::O_COLS;
          if (!wait_w(&o_empty[ob], ((m / CF::NOB) & 1) ^ 1, 116)) { ok = false; break; }
          LA2_TRACE_POINT(13, m);
          tc_fence_after();
          if (needs_snap) {
            const uint64_t q = dKm + ((sQ0 + qslot(m, g) * CF::QTILE) >> 4);
            const uint64_t kv = dSnap + ((sS0 + sb * CF::SNAP) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * BK * 128 + (kk & 3) * 32) >> 4;
              if constexpr (CF::OT)  // O^T += KV^T Q^T: A = snapshot (MN-major), B = Q (K-major)
                mma_bf16_ss_warp(tO, kv + kk * (2048 >> 4), q + off, CF::ID_QKV, kk > 0);
              else
                mma_bf16_ss_warp(tO, q + off, kv + kk * (2048 >> 4), CF::ID_QKV, kk > 0);
            }
            mma_commit_warp(&snap_free[sb]);
            ++sn;
          }
          if (!CF::QWITHKV && !CF::O_IN_Q) mma_commit_warp(&q_empty[m % CF::QS]);
          update(ks, needs_snap);
          mma_commit_warp(kv_updated);
          if (st.seg_last) ack_pending = true;
          const uint32_t pb = m % CF::NPB;
          LA2_TRACE_POINT(3, m);
          if (!wait_w(&p_full[pb], (m / CF::NPB) & 1, 117)) { ok = false; break; }
          LA2_TRACE_POINT(4, m);
          tc_fence_after();
          if constexpr (CF::P_TMEM) {
            // A = P from TMEM: the k-th 16-column slice of P is 8 TMEM columns in
            const uint64_t b = dK_mn + ((sV0 + ks * CF::VTILE) >> 4);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              mma_bf16_ts_warp(tO, tmem + CF::COL_P + kk * 8, b + kk * (2048 >> 4), CF::ID_PV,
                               (needs_snap || kk > 0) ? 1u : 0u);
          } else {
            const uint64_t pp = dKm + ((sP0 + pb * CF::PTILE) >> 4);
            const uint64_t vv = dK_mn + ((sV0 + ks * CF::VTILE) >> 4);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * BK * 128 + (kk & 3) * 32) >> 4;
              if constexpr (CF::OT)  // O^T += V^T P^T: A = V (MN-major), B = P (K-major)
                mma_bf16_ss_warp(tO, vv + kk * (2048 >> 4), pp + off, CF::ID_PV,
                                 (needs_snap || kk > 0) ? 1u : 0u);
              else
                mma_bf16_ss_warp(tO, pp + off, vv + kk * (2048 >> 4), CF::ID_PV,
                                 (needs_snap || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit_warp(&o_full[ob]);
          if (!CF::MERGE_OP) mma_commit_warp(&p_empty[pb]);
          mma_commit_warp(&kv_empty[ks]);
          LA2_TRACE_POINT(14, m);
          ++m;
        }
        ++g;
        st = nx;
        have = have_nx;
      }
      mma_commit_warp(drain);
      drain_wait(drain, 0);
    }
  } else if (wg == kWgMask) {
    // ================================================ mask + convert S -> P
    if (KIND == KIND_MAIN) {
      const int r = acc_row<BK>(w4, lane);
      const uint32_t lane_off = static_cast<uint32_t>(32 * w4) << 16;
      StepIter<KIND> it;
      it.begin(&rt);
      Step st;
      uint32_t m = 0;
      while (it.next(st)) {
        if (st.pre) continue;
        const uint32_t sbuf = m % CF::NSB, pb = m % CF::NPB;
        const uint32_t tS = tmem + CF::COL_S + sbuf * BK + lane_off;
        if (!__all_sync(0xffffffffu, wait_bar(&s_full[sbuf], (m / CF::NSB) & 1, lim, abort_flag, 120))) break;
        if (threadIdx.x % 128 == 0) LA2_TRACE_POINT(7, m);
        // P buffer pb is free once PV(m - NPB) completed (o_full doubles as the signal).
        uint64_t* p_free = CF::MERGE_OP ? o_full : p_empty;
        if (!__all_sync(0xffffffffu, wait_bar(&p_free[pb], ((m / CF::NPB) & 1) ^ 1, lim, abort_flag, 121))) break;
        tc_fence_after();
        if constexpr (CF::P_TMEM) {
          // P rows into TMEM next to S: lane r, column j holds bf16 P[r][2j], P[r][2j+1]
          const uint32_t tP = tmem + CF::COL_P + lane_off;
#pragma unroll
          for (int c32 = 0; c32 < BK / 32; ++c32) {
            uint32_t v[32];
            tmem_ld32(tS + c32 * 32, v);
            tmem_ld_wait();
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int col = c32 * 32 + 2 * e;
              const float a = (col <= r) ? __uint_as_float(v[2 * e]) : 0.f;
              const float bb = (col + 1 <= r) ? __uint_as_float(v[2 * e + 1]) : 0.f;
              w[e] = pack_bf16x2(a, bb);
            }
            tmem_st16(tP + c32 * 16, w);
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&p_full[pb]);
          if (threadIdx.x % 128 == 0) LA2_TRACE_POINT(8, m);
          ++m;
          continue;
        }
        const uint32_t pbase = smem_u32(sP + pb * CF::PTILE);
#pragma unroll
        for (int c32 = 0; c32 < BK / 32; ++c32) {
          uint32_t v[32];
          tmem_ld32(tS + c32 * 32, v);
          tmem_ld_wait();
          if (r >= 0) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int col = c32 * 32 + q4 * 8 + 2 * e;
                const float a = (col <= r) ? __uint_as_float(v[q4 * 8 + 2 * e]) : 0.f;
                const float bb = (col + 1 <= r) ? __uint_as_float(v[q4 * 8 + 2 * e + 1]) : 0.f;
                w[e] = pack_bf16x2(a, bb);
              }
              const int ch = c32 * 4 + q4;
              const int panel = ch >> 3, cj = ch & 7;
              st_shared_v4(pbase + panel * BK * 128 + r * 128 + ((cj ^ (r & 7)) << 4), w[0], w[1],
                           w[2], w[3]);
            }
          }
        }
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(&p_full[pb]);
        if (threadIdx.x % 128 == 0) LA2_TRACE_POINT(8, m);
        ++m;
      }
    }
  } else if (wg == kWgState) {
    // ==================================================== KV state (snapshot)
    const int r = acc_row<D>(w4, lane);  // state row
    const uint32_t lane_off = static_cast<uint32_t>(32 * w4) << 16;
    const uint32_t tKV = tmem + CF::COL_KV + lane_off;
    StepIter<KIND> it;
    it.begin(&rt);
    Step st;
    uint32_t sn = 0, kvu = 0;
    bool ok = true;

    auto wait_kvu = [&]() -> bool {
      const bool w = __all_sync(0xffffffffu, wait_bar(kv_updated, kvu & 1, lim, abort_flag, 130));
      ++kvu;
      if (w) tc_fence_after();
      return w;
    };
    auto snap_from_tmem = [&]() -> bool {
      const uint32_t sb = sn % CF::NSNAP;
      const uint32_t sbase = smem_u32(sSnap + sb * CF::SNAP);
#pragma unroll
      for (int c32 = 0; c32 < DV / 32; ++c32) {
        uint32_t v[32];
        tmem_ld32(tKV + c32 * 32, v);
        tmem_ld_wait();
        if (c32 == 0 &&
            !__all_sync(0xffffffffu,
                        wait_bar(&snap_free[sb], ((sn / CF::NSNAP) & 1) ^ 1, lim, abort_flag, 131)))
          return false;
        if (r >= 0) put_snap_row<D>(sbase, r, v, c32 * 32);
      }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(&snap_full[sb]);
      ++sn;
      return true;
    };
    // Initial state = sum of the states of the earlier ranges of this sequence.
    auto snap_from_ranges = [&](const Step& s) -> bool {
      const uint32_t sb = sn % CF::NSNAP;
      if (!__all_sync(0xffffffffu,
                      wait_bar(&snap_free[sb], ((sn / CF::NSNAP) & 1) ^ 1, lim, abort_flag, 132)))
        return false;
      init_from_ranges<D, DV>(prm.agg, rt, s.range, s.bh * rt.T, r, tKV,
                              smem_u32(sSnap + sb * CF::SNAP));
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(&snap_full[sb]);
      ++sn;
      return true;
    };

    while (ok && it.next(st)) {
      if (KIND == KIND_AGG) {
        if (!st.pre_last) continue;
        if (!wait_kvu()) break;
        float* dst = prm.agg + static_cast<int64_t>(st.range) * D * DV;
#pragma unroll
        for (int c32 = 0; c32 < DV / 32; ++c32) {
          uint32_t v[32];
          tmem_ld32(tKV + c32 * 32, v);
          tmem_ld_wait();
          if (r >= 0) {
            float4* p4 = reinterpret_cast<float4*>(dst);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              p4[agg_f4<D>(r, c32 * 8 + q4)] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                   __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
          }
        }
        tc_fence_before();
        mbar_arrive(seg_ack);
        continue;
      }
      if (st.pre) continue;
      if (st.seg_first) {
        if (st.init == 1) {
          if (!wait_kvu() || !snap_from_tmem()) break;
        } else if (st.init == 2) {
          if (first_init_ready) {  // built at CTA start into TMEM and snapshot 0
            first_init_ready = false;
            tc_fence_before();
            mbar_arrive(&snap_full[sn % CF::NSNAP]);
            ++sn;
          } else if (!snap_from_ranges(st)) {
            break;
          }
        }
      } else {
        if (!wait_kvu()) break;
        if (threadIdx.x % 128 == 0) LA2_TRACE_POINT(9, sn);
        if (!snap_from_tmem()) break;
        if (threadIdx.x % 128 == 0) LA2_TRACE_POINT(10, sn - 1);
      }
      if (st.seg_last) {
        if (!wait_kvu()) break;
        tc_fence_before();
        mbar_arrive(seg_ack);
      }
    }
  } else if (wg == kWgEpilogue) {
    // ========================================== O: TMEM -> bf16 -> HBM
    if (KIND == KIND_MAIN) {
      const int r = acc_row<BK>(w4, lane);
      const uint32_t lane_off = static_cast<uint32_t>(32 * w4) << 16;
      StepIter<KIND> it;
      it.begin(&rt);
      Step st;
      uint32_t m = 0;
      while (it.next(st)) {
        if (st.pre) continue;
        const uint32_t ob = m % CF::NOB;
        const uint32_t tO = tmem + CF::COL_O + ob * CF::O_COLS + lane_off;
        if (!__all_sync(0xffffffffu, wait_bar(&o_full[ob], (m / CF::NOB) & 1, lim, abort_flag, 140))) break;
        if (threadIdx.x % 128 == 0) LA2_TRACE_POINT(11, m);
        tc_fence_after();
        if constexpr (CF::OT) {
          // Thread (w4, lane) holds column e = 32 w4 + lane of O for the BK rows of
          // the block (TMEM lane e, one column per row). It writes them into the
          // staging tile in the TMA layout (128B-swizzled 64-column panels, rows =
          // tokens); thread 0 then stores the whole tile.
          // The four epilogue warps meet on mbarriers (bounded waits, so an
          // abort elsewhere cannot leave a warp waiting for ever).
          const int e = 32 * w4 + lane;
          const uint32_t sb = m & 1, sph = (m >> 1) & 1;
          uint8_t* stage = smem + CF::OFF_OST + sb * CF::OTILE;
          if (threadIdx.x % 128 == 0) {
            bulk_wait_group_read<1>();  // block m-2's store has read this tile
            mbar_arrive(&stage_free[sb]);
          }
          if (!__all_sync(0xffffffffu, wait_bar(&stage_free[sb], sph, lim, abort_flag, 141))) break;
          const uint32_t col_base = smem_u32(stage + (e >> 6) * BK * 128) + (e & 7) * 2;
          const int chunk = (e & 63) >> 3;
#pragma unroll
          for (int c32 = 0; c32 < BK / 32; ++c32) {
            uint32_t v[32];
            tmem_ld32(tO + c32 * 32, v);
            tmem_ld_wait();
            if (c32 == BK / 32 - 1) {  // every TMEM read of O(m) is done
              tc_fence_before();
              mbar_arrive(&o_empty[ob]);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int t = c32 * 32 + j;  // token row of the block
              st_shared_u16(col_base + t * 128 + ((chunk ^ (t & 7)) << 4),
                            bf16_bits(__uint_as_float(v[j])));
            }
          }
          fence_proxy_async();
          mbar_arrive(&stage_full[sb]);
          if (w4 == 0) {  // the first epilogue warp stores the tile (warp-uniform wait)
            if (!__all_sync(0xffffffffu, wait_bar(&stage_full[sb], sph, lim, abort_flag, 142))) break;
            if (lane == 0) {
              const int64_t y = static_cast<int64_t>(st.blk) * BK;
#pragma unroll
              for (int p = 0; p < DV / 64; ++p)  // rows past N are clipped by the tensor map
                tma_store_3d(&tm_o, stage + p * BK * 128, 64 * p, static_cast<int>(y),
                             static_cast<int>(st.bh));
              bulk_commit_group();
            }
          }
          if (threadIdx.x % 128 == 0) LA2_TRACE_POINT(12, m);
          ++m;
          continue;
        }
        if constexpr (CF::TMA_STORE) {
          // Warp w4 owns rows 16*w4 .. 16*w4+15 of the block: it stages them
          // (128B-swizzled, panels of 64 columns) and stores them itself.
          uint8_t* stage = smem + CF::OFF_OST + ob * CF::OTILE + w4 * 16 * 128;
          if (lane == 0) bulk_wait_group_read<1>();  // this warp's store of block m-2 has read it
          __syncwarp();
          const int rl = lane & 15;
#pragma unroll
          for (int c32 = 0; c32 < DV / 32; ++c32) {
            uint32_t v[32];
            tmem_ld32(tO + c32 * 32, v);
            tmem_ld_wait();
            if (r >= 0) {
              const uint32_t base = smem_u32(stage + (c32 >> 1) * BK * 128) + rl * 128;
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int cj = (c32 & 1) * 4 + q;
                st_shared_v4(base + ((cj ^ (rl & 7)) << 4),
                             pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                             pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                             pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                             pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
              }
            }
          }
          tc_fence_before();
          mbar_arrive(&o_empty[ob]);
          fence_proxy_async();
          __syncwarp();
          const int64_t y = static_cast<int64_t>(st.blk) * BK + 16 * w4;
          if (lane == 0) {
            if (y < prm.N) {  // rows past N are clipped by the tensor map
#pragma unroll
              for (int p = 0; p < DV / 64; ++p)
                tma_store_3d(&tm_o, stage + p * BK * 128, 64 * p, static_cast<int>(y),
                             static_cast<int>(st.bh));
            }
            // One bulk group per block, empty when every row of this warp lies
            // past N: the wait above counts groups, and a skipped group would
            // let block m reuse the staging tile that block m-2's store may
            // still be reading (a range can run on into the next sequence).
            bulk_commit_group();
          }
          if (threadIdx.x % 128 == 0) LA2_TRACE_POINT(12, m);
          ++m;
          continue;
        }
        const int64_t row = static_cast<int64_t>(st.blk) * BK + r;
        const bool valid = r >= 0 && row < prm.N;
        uint4* dst = reinterpret_cast<uint4*>(prm.o + (st.bh * prm.N + (valid ? row : 0)) * DV);
        if constexpr (CF::O_IN_Q) {
          // One O buffer: read the whole row out of TMEM (packed to bf16) and
          // release the buffer to the next block's Q KV first; then stage the
          // row in Q(m)'s tile (128B-swizzled 64-column panels, as TMA wrote Q)
          // and store this warp's 32 rows with TMA.
          (void)valid;
          (void)dst;
          const uint32_t qs = m % CF::QS;
          uint8_t* stage = sQ + qs * CF::QTILE;
#pragma unroll
          for (int c32 = 0; c32 < DV / 32; ++c32) {
            uint32_t v[32];
            tmem_ld32(tO + c32 * 32, v);
            tmem_ld_wait();
            if (c32 == DV / 32 - 1) {  // every TMEM read of O(m) is done
              tc_fence_before();
              mbar_arrive(&o_empty[ob]);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // 16-byte chunk ch of row r
              const int ch = c32 * 4 + q;
              const int panel = ch >> 3, cj = ch & 7;
              st_shared_v4(smem_u32(stage + panel * BK * 128) + r * 128 + ((cj ^ (r & 7)) << 4),
                           pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                           pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                           pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                           pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
            }
          }
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            const int64_t y = static_cast<int64_t>(st.blk) * BK + 32 * w4;
            if (y < prm.N) {  // rows past N are clipped by the tensor map
#pragma unroll
              for (int p = 0; p < DV / 64; ++p)
                tma_store_3d(&tm_o, stage + p * BK * 128 + 32 * w4 * 128, 64 * p,
                             static_cast<int>(y), static_cast<int>(st.bh));
            }
            bulk_commit_group();
            bulk_wait_group_read<0>();  // the tile may take Q(m + QS) once read
            mbar_arrive(&q_empty[qs]);
          }
          if (threadIdx.x % 128 == 0) LA2_TRACE_POINT(12, m);
          ++m;
          continue;
        }
#pragma unroll
        for (int c32 = 0; c32 < DV / 32; ++c32) {
          uint32_t v[32];
          tmem_ld32(tO + c32 * 32, v);
          tmem_ld_wait();
          if (valid) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[c32 * 4 + q] = make_uint4(
                  pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                  pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                  pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                  pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
          }
        }
        tc_fence_before();
        mbar_arrive(&o_empty[ob]);
        if (threadIdx.x % 128 == 0) LA2_TRACE_POINT(12, m);
        ++m;
      }
      if ((CF::TMA_STORE || CF::O_IN_Q) && lane == 0) bulk_wait_group<0>();  // stores done before exit
      if (threadIdx.x % 128 == 0) LA2_TRACE_CTA_POINT(2);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace sm100

// ------------------------------------------------------------------ host side

// Cost model of the range split, in units of one main block. Under load a
// pre-pass step takes 0.42-0.54 us against 1.38-1.63 us for a main step
// (per-step timelines of a CTA with a pre-pass at Bk=64; its K and V mostly
// come from L2, read at the same time by the CTA whose range holds them). A
// sweep of the cost on B4 H16 N2K, B1 H32 N1K and N4K (Bk 64 and 128) put the
// best single value at 0.4: 0.5 kept ranges that start at block 0 too long
// (N1K Bk=64: 16.4 -> 14.5 us per step at 0.4), while 0.35 and below split
// B4 H16 N2K into ranges that span two sequences (35.3 -> 36.5 us).
constexpr double kPrepassCost = 0.4;
constexpr double kRangeStateCost = 0.5;  // separate state launch, per block
// Extra launch + initial-state sum, in Bk=64 main blocks: fitted so that the
// plans follow measured winners (B1 H32 N4K Bk=64: range states over ranges
// aligned to the sequences 43.9 us, pre-pass 46.5 us per step; B4 H16 N2K,
// B1 H32 N1K and B2 H32 N8K: pre-pass, 17-50 % faster than range states).
constexpr double kLaunchCost = 4.0;

struct RangePlan {
  int R = 0;
  int prefix_mode = 0;
  int64_t T = 0;
  std::vector<int64_t> starts;
  double makespan = 0.0;
};

// Greedy split of `total` tasks into ranges of cost <= tau; a range that
// starts at block b of a sequence pays b pre-pass blocks. Returns the count,
// or kMaxRanges + 1 when tau is infeasible (a range would have to start where
// its pre-pass alone leaves no room for one main block).
inline int greedy_ranges(int64_t total, int64_t T, double tau, std::vector<int64_t>* starts) {
  int64_t f = 0;
  int n = 0;
  if (starts) starts->clear();
  while (f < total) {
    const int64_t blk = f % T;
    const double budget = tau - static_cast<double>(blk) * kPrepassCost;
    if (budget < 1.0) return sm100::kMaxRanges + 1;
    const int64_t take = static_cast<int64_t>(budget);
    if (starts) starts->push_back(f);
    f = std::min(total, f + take);
    ++n;
    if (n > sm100::kMaxRanges) return n;
  }
  if (starts) starts->push_back(total);
  return n;
}

inline RangePlan plan_ranges(int64_t BH, int64_t N, int block, int sms, int64_t forced_len) {
  RangePlan p;
  const int64_t T = (N + block - 1) / block;
  const int64_t total = BH * T;
  p.T = T;
  if (forced_len > 0) {
    // fixed ranges of forced_len rows, never crossing a sequence; states from range sums
    const int64_t per = std::max<int64_t>(1, forced_len / block);
    p.prefix_mode = 1;
    for (int64_t h = 0; h < BH; ++h)
      for (int64_t b = 0; b < T; b += per) p.starts.push_back(h * T + b);
    p.starts.push_back(total);
    p.R = static_cast<int>(p.starts.size()) - 1;
    return p;
  }
  const int G = std::max(1, sms);
  // (a) pre-pass plan: smallest makespan tau whose greedy split fits in G ranges
  double lo = std::max(1.0, static_cast<double>(total) / G), hi = static_cast<double>(total) + T;
  for (int it = 0; it < 40; ++it) {
    const double mid = 0.5 * (lo + hi);
    if (greedy_ranges(total, T, mid, nullptr) <= G) hi = mid;
    else lo = mid;
  }
  std::vector<int64_t> pre_starts;
  const int n_pre = greedy_ranges(total, T, hi, &pre_starts);
  const double tau_pre = hi;
  // (b) range-state plan: equal split; a separate launch computes range states.
  // With a few ranges per sequence (at most 8) the ranges are aligned to the
  // sequences (the same count in each), when that leaves at least 3/4 of the
  // SMs busy: no range then holds the end of one sequence and the start of
  // the next, and every sequence's last range (1/k of the K/V) needs no
  // state. Measured against the split over all SMs: B1 H32 N4K and N16K at
  // Bk=128 2-4 % faster, N64K Bk=128 2.6 %, N64K Bk=64 unchanged. With many
  // ranges per sequence the saving is small and the SMs left idle cost more
  // (B1 H8 N512K: 144 ranges up to 3 % slower than 148 under the power cap).
  int n_eq = static_cast<int>(std::min<int64_t>(G, total));
  if (BH <= G && G / BH <= 8) {
    const int64_t aligned = BH * (G / BH);
    if (4 * aligned >= 3 * static_cast<int64_t>(G) && aligned <= total) n_eq = static_cast<int>(aligned);
  }
  // the launch cost is a time: in units of this block size's main block
  const double launch = kLaunchCost * 64.0 / static_cast<double>(block);
  const double tau_eq = static_cast<double>(total) / n_eq * (1.0 + kRangeStateCost) + launch;
  if (tau_pre <= tau_eq && n_pre <= sm100::kMaxRanges) {
    p.prefix_mode = 0;
    p.starts = pre_starts;
    p.R = n_pre;
    p.makespan = tau_pre;
  } else {
    p.prefix_mode = 1;
    p.starts.resize(n_eq + 1);
    for (int j = 0; j <= n_eq; ++j) p.starts[j] = total * j / n_eq;
    p.R = n_eq;
    p.makespan = tau_eq;
  }
  return p;
}

inline bool fill_range_table(const RangePlan& p, sm100::RangeTable* t) {
  if (p.R < 1 || p.R > sm100::kMaxRanges) return false;
  if (p.starts.back() > 0x7fffffff) return false;  // task indices are 32-bit on the device
  t->R = p.R;
  t->prefix_mode = p.prefix_mode;
  t->T = p.T;
  for (int i = 0; i <= p.R; ++i) t->starts[i] = p.starts[i];
  return true;
}

template <int BK, int D, int DV, int KIND>
inline la2_status launch_causal_sm100(const CUtensorMap& tq, const CUtensorMap& tk,
                                      const CUtensorMap& tv, const CUtensorMap& to,
                                      const sm100::RangeTable& rt,
                                      const sm100::CausalParams& p, int grid, cudaStream_t st) {
  using CF = sm100::CCfg<BK, D, DV, KIND>;
  auto kern = sm100::la2_causal_sm100_kernel<BK, D, DV, KIND>;
  static bool attr_done[128];  // one per template instantiation
  if (!smem_attribute_set(kern, CF::SMEM, attr_done)) return LA2_ERR_CUDA;
  // Programmatic stream serialization: this grid may begin launching while
  // the previous kernel of the stream finishes; the kernel waits for it
  // (griddepcontrol.wait) before it touches global memory.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(sm100::kThreads);
  cfg.dynamicSmemBytes = CF::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, to, rt, p) != cudaSuccess) return LA2_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? LA2_OK : LA2_ERR_CUDA;
}

}  // namespace la2
