// libla2: host side of the C ABI declared in include/la2.h.
//
// Argument validation, the chunk plan, workspace carving, kernel launches and
// the optional per-kernel event timing. Every kernel of the library is in this
// translation unit (the .cuh files below), so the device error word is one
// symbol.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "la2.h"
#include "la2_common.cuh"
#include "la2_decode.cuh"
#include "la2_simt.cuh"
#include "la2_sm100.cuh"
#include "la2_sm100_causal.cuh"
#include "la2_sm100_bwd.cuh"

namespace la2 {

// ------------------------------------------------------------------ profiler

enum KernelId : int {
  K_CHUNK_STATE = 0,
  K_CHUNK_SCAN,
  K_FWD_SIMT,
  K_BWD_DQ_SIMT,
  K_BWD_DKDV_SIMT,
  K_FWD_TC,
  K_STATE_TC,
  K_BWD_DQ_TC,
  K_BWD_DKDV_TC,
  K_DECODE,
  K_STATE_ACC,
  K_REVERSE,
  K_COUNT
};

static const char* kKernelNames[K_COUNT] = {
    "la2_chunk_state_simt", "la2_chunk_scan",      "la2_fwd_simt",
    "la2_bwd_dq_simt",      "la2_bwd_dkdv_simt",   "la2_fwd_sm100",
    "la2_chunk_state_sm100", "la2_bwd_dq_sm100",   "la2_bwd_dkdv_sm100",
    "la2_decode_step",      "la2_state_accumulate", "la2_reverse_rows"};

struct EventRecord {
  int kernel;
  cudaEvent_t start, stop;
};

struct Profiler {
  bool on = false;
  std::vector<EventRecord> pool;  // events are reused across enable() calls
  size_t used = 0;
};
static Profiler g_prof;

struct LaunchTimer {
  EventRecord* rec = nullptr;
  cudaStream_t stream;
  LaunchTimer(int kernel, cudaStream_t s) : stream(s) {
    if (!g_prof.on) return;
    if (g_prof.used == g_prof.pool.size()) {
      EventRecord r{};
      if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess) return;
      g_prof.pool.push_back(r);
    }
    rec = &g_prof.pool[g_prof.used++];
    rec->kernel = kernel;
    cudaEventRecord(rec->start, stream);
  }
  ~LaunchTimer() {
    if (rec) cudaEventRecord(rec->stop, stream);
  }
};

// ------------------------------------------------------------------ settings

static int64_t g_chunk_len = 0;           // 0: automatic
static int64_t g_spin_limit = 0;          // 0: default
constexpr int64_t kDefaultSpinLimit = int64_t(1) << 31;

static int64_t spin_limit() { return g_spin_limit > 0 ? g_spin_limit : kDefaultSpinLimit; }

constexpr int kMaxDevices = 128;

static int device_sm_count() {
  static int cached[kMaxDevices];
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < kMaxDevices && cached[dev] > 0) return cached[dev];
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < kMaxDevices) cached[dev] = sms;
  return sms;
}

// ------------------------------------------------------------------ planning

struct Plan {
  int64_t L = 0;        // chunk length (rows), multiple of block
  int64_t C = 1;        // chunks per (b, h)
  bool tc = false;      // tensor-core (sm_100a) path
  bool need_states = false;
  size_t ws_bytes = 0;
  bool ranges = false;  // persistent range split (tensor-core causal forward)
  bool dq_ranges = false;  // tensor-core causal backward: dQ through the range split
  // Tensor-core causal backward, dK/dV in two chunks per K/V sequence, rows
  // [0, dk_split) and [dk_split, N): the first builds its suffix state in the
  // kernel (no suffix-state pass, no scan). 0: chunks of L rows.
  int64_t dk_split = 0;
  RangePlan rp;
};

static bool is_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Shape checks shared by every entry point. Returns LA2_OK or an error.
static la2_status check_shape(int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv, int causal,
                              int block, la2_dtype dt, bool is_bwd, int64_t Hkv = -1) {
  if (Hkv < 0) Hkv = H;  // plain layout: one K/V head per query head
  if (B < 0 || H < 0 || N < 0 || d < 1 || dv < 1) return LA2_ERR_INVALID_ARG;
  // grouped heads: Hkv >= 1 divides H (an empty H takes any Hkv >= 0)
  if (H > 0 && (Hkv < 1 || H % Hkv != 0)) return LA2_ERR_INVALID_ARG;
  if (H > 0x7fffffff) return LA2_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return LA2_ERR_INVALID_ARG;
  if (dt != LA2_F32 && dt != LA2_BF16) return LA2_ERR_INVALID_ARG;
  if (block < 1) return LA2_ERR_INVALID_ARG;
  // int64 overflow guard on the largest index the kernels form.
  const double elems = double(B) * double(H) * double(N) * double(std::max(d, dv));
  if (elems > 9.0e18) return LA2_ERR_INVALID_ARG;
  if (dt == LA2_BF16) {
    if ((d != 64 && d != 128) || (dv != 64 && dv != 128)) return LA2_ERR_UNSUPPORTED;
    if (block != 64 && block != 128) return LA2_ERR_UNSUPPORTED;
  } else {
    if (d > 128 || dv > 128) return LA2_ERR_UNSUPPORTED;
    if (block != 16 && block != 32 && block != 64 && block != 128) return LA2_ERR_UNSUPPORTED;
  }
  const size_t es = dt == LA2_BF16 ? 2 : 4;
  const size_t smem = is_bwd ? std::max(bwd_dq_simt_smem((int)d, (int)dv, block, es),
                                        bwd_dkdv_simt_smem((int)d, (int)dv, block, es))
                             : fwd_simt_smem((int)d, (int)dv, block, es);
  const bool tc = (dt == LA2_BF16) && sm100_supports(d, dv, block, is_bwd);
  if (!tc && smem > 227 * 1024) return LA2_ERR_UNSUPPORTED;
  if (!tc && is_bwd && !bwd_dkdv_simt_fits((int)d, (int)dv, block)) return LA2_ERR_UNSUPPORTED;
  return LA2_OK;
}

static Plan make_plan_uncached(int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t d, int64_t dv,
                               int causal, int block, la2_dtype dt, bool is_bwd, int sms, bool sp) {
  Plan p;
  const int64_t BH = B * H;
  const int64_t BHkv = B * Hkv;
  const int64_t T = (N + block - 1) / block;
  // The backward's heaviest pass (dK, dV) runs one unit per K/V sequence and chunk.
  const int64_t BHu = is_bwd ? BHkv : BH;
  p.tc = (dt == LA2_BF16) && sm100_supports(d, dv, block, is_bwd);
  int64_t L;
  if (g_chunk_len > 0) {
    L = ((g_chunk_len + block - 1) / block) * block;
  } else {
    // Enough (b, h, chunk) units for about two per SM, chunks no shorter than
    // four blocks so the chunk-state pass stays a small fraction of the work.
    // Tensor-core non-causal forward: about one wave, since the map pass sums
    // a sequence's chunk states itself.
    const bool one_wave = p.tc && !causal && !is_bwd;
    const int64_t target = (one_wave ? 1 : 2) * (int64_t)std::max(sms, 1);
    int64_t C = one_wave ? std::max<int64_t>(1, target / std::max<int64_t>(BHu, 1))
                         : std::max<int64_t>(1, (target + BHu - 1) / std::max<int64_t>(BHu, 1));
    C = std::min<int64_t>(C, std::max<int64_t>(1, T / 4));
    if (p.tc && is_bwd) {
      // The dK/dV pass runs one CTA per (sequence, chunk), in waves of `sms`
      // CTAs: pick the chunk count whose waves times chunk length (plus a fixed
      // cost per chunk: initial state, pipeline fill) is smallest, so that a
      // nearly empty last wave does not stretch the pass (64 sequences x 5
      // chunks on 148 SMs ran 3 waves where 2 chunks run in one).
      constexpr double kChunkCost = 3.0;  // blocks
      const int64_t G = std::max(sms, 1), cmax = std::max<int64_t>(1, T / 4);
      double best = 0.0;
      for (int64_t c = 1; c <= cmax; ++c) {
        const int64_t units = BHu * c;
        const double cost = static_cast<double>((units + G - 1) / G) *
                            (static_cast<double>((T + c - 1) / c) + kChunkCost);
        if (c == 1 || cost < best) {
          best = cost;
          C = c;
        }
      }
    }
    L = ((T + C - 1) / C) * block;
  }
  L = std::max<int64_t>(L, block);
  const size_t state_bytes = (size_t)d * (size_t)dv * sizeof(float);
  // The range split runs when its table holds the ranges (always for the
  // automatic plan; a forced split of many sequences can exceed it) and its
  // task indices fit in 32 bits. Otherwise the chunk path below runs, for the
  // forward as for the backward's dQ pass.
  bool range_fits = false;
  // A part of a longer sequence (sequence parallelism) starts from the states
  // of the other parts: the chunk path, whose state scan takes them as a base.
  if (p.tc && causal && !sp) {
    p.rp = plan_ranges(BH, N, block, sms, g_chunk_len);
    range_fits = p.rp.R >= 1 && p.rp.R <= sm100::kMaxRanges && BH * T <= 0x7fffffff;
    p.ranges = range_fits;
    if (!is_bwd && range_fits) {
      p.need_states = p.rp.prefix_mode == 1;
      p.ws_bytes = p.need_states ? (size_t)p.rp.R * state_bytes : 0;
      return p;
    }
  }
  p.L = L;
  p.C = std::max<int64_t>(1, (N + L - 1) / L);
  p.need_states = (p.C > 1) || !causal || sp;
  // chunk states belong to K/V sequences (shared by a group's query heads)
  const size_t one = (size_t)BHkv * (size_t)p.C * state_bytes;
  p.ws_bytes = p.need_states ? one * (is_bwd ? 2 : 1) : 0;
  if (p.tc && causal && is_bwd) {
    // Workspace: [U chunk states | K^T V chunk states or the dQ pass's range
    // states, whichever is larger]. The dQ pass takes the range split when
    // its table can hold the ranges, else the chunk path.
    p.dq_ranges = range_fits;
    const size_t agg = p.dq_ranges && p.rp.prefix_mode == 1 ? (size_t)p.rp.R * state_bytes : 0;
    const size_t kv = p.need_states ? one : 0;
    p.ws_bytes = (p.need_states ? one : 0) + std::max(agg, kv);
    // dK/dV split in two with the suffix state built in the kernel, when one
    // wave holds both chunks of every K/V sequence and the model prefers it.
    // Costs in dK/dV block steps (one query head of one block): a chunk of c
    // blocks costs c G + kChunkCost; the suffix-state pass costs kUPass per
    // block it reads; an in-kernel pre-pass step kPrePass. The first chunk
    // takes the share a of the blocks that balances a + kPrePass (T - a)
    // against T - a.
    constexpr double kChunkCost = 3.0, kUPass = 0.38, kPrePass = 0.25;
    const int64_t G = std::max<int64_t>(1, H / std::max<int64_t>(1, Hkv));
    // (64-row dK/dV tiles only: their two-stage ring keeps the pre-pass loads
    // in flight; the 128-row kernel has one stage)
    const bool tiles64 = block == 64 || G > 1;
    if (p.dq_ranges && tiles64 && T >= 2 && 2 * BHkv <= sms && g_chunk_len == 0) {
      const int64_t waves = (BHkv * p.C + sms - 1) / sms;
      const double per = static_cast<double>((T + p.C - 1) / p.C);
      // (one chunk per sequence needs no suffix states)
      const double cost_a = static_cast<double>(waves) *
                            (per * G * (1.0 + (p.C > 1 ? kUPass : 0.0)) + kChunkCost);
      const int64_t a = std::min<int64_t>(
          T - 1, std::max<int64_t>(1, std::llround(static_cast<double>(T) * (1.0 - kPrePass) /
                                                    (2.0 - kPrePass))));
      const double cost_b = std::max(static_cast<double>(a) + kPrePass * static_cast<double>(T - a),
                                     static_cast<double>(T - a)) * G + kChunkCost;
      if (cost_b < cost_a) {
        p.dk_split = a * block;
        p.C = 2;
        p.L = a * block;
        p.need_states = false;
        p.ws_bytes = agg;
      }
    }
  }
  return p;
}

// Plans are pure functions of the arguments, the split override and the SM
// count; the range split is a small search, so recent plans are kept.
struct PlanKey {
  int64_t B, H, Hkv, N, d, dv, chunk_len;
  int causal, block, dt, is_bwd, sms, sp;
  bool operator==(const PlanKey& o) const {
    return B == o.B && H == o.H && Hkv == o.Hkv && N == o.N && d == o.d && dv == o.dv &&
           chunk_len == o.chunk_len && causal == o.causal && block == o.block && dt == o.dt &&
           is_bwd == o.is_bwd && sms == o.sms && sp == o.sp;
  }
};

static Plan make_plan(int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv, int causal, int block,
                      la2_dtype dt, bool is_bwd, int sms, int64_t Hkv = -1, bool sp = false) {
  if (Hkv < 0) Hkv = H;
  constexpr int kSlots = 16;
  static PlanKey keys[kSlots];
  static Plan plans[kSlots];
  static int used = 0, next_slot = 0;
  static std::mutex mu;
  const PlanKey k{B, H, Hkv, N, d, dv, g_chunk_len, causal, block, static_cast<int>(dt), is_bwd ? 1 : 0,
                  sms, sp ? 1 : 0};
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
      if (keys[i] == k) return plans[i];
  }
  Plan p = make_plan_uncached(B, H, Hkv, N, d, dv, causal, block, dt, is_bwd, sms, sp);
  std::lock_guard<std::mutex> lock(mu);
  keys[next_slot] = k;
  plans[next_slot] = p;
  next_slot = (next_slot + 1) % kSlots;
  used = used < kSlots ? used + 1 : kSlots;
  return p;
}

// ------------------------------------------------------------------ launches

static la2_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LA2_OK : LA2_ERR_CUDA;
}

// Query and K/V head counts of a call: H query heads per batch entry, G query
// heads per K/V head (G = 1 for the plain layout).
struct Heads {
  int64_t BH;    // query sequences
  int64_t BHkv;  // K/V sequences
  int32_t H, G;
};

// States of the other parts of each sequence (sequence parallelism): the sum
// of n_pre states [n_pre][nseq][d][dv] before this part (the causal prefix,
// K^T V) and of n_suf states after it (sum Q^T dO, the backward's suffix).
struct Ext {
  const float* pre = nullptr;
  int64_t n_pre = 0;
  const float* suf = nullptr;
  int64_t n_suf = 0;
  bool on = false;
};

template <typename T>
static la2_status run_chunk_states(const void* a, const void* b, float* out, int64_t nseq, int64_t N,
                                   int da, int db, const Plan& p, cudaStream_t st, int32_t H = 1,
                                   int32_t G = 1, int group = 1, const float* lam = nullptr,
                                   int decay = 0) {
  const size_t smem = chunk_state_smem(da, db);
  LaunchTimer t(K_CHUNK_STATE, st);
  chunk_state_kernel<T><<<(unsigned)(nseq * p.C), kSimtThreads, smem, st>>>(
      static_cast<const T*>(a), static_cast<const T*>(b), out, N, da, db, p.L, p.C, H, G, group,
      lam, decay);
  return launch_status();
}

static la2_status run_scan(float* s, int64_t nseq, int nel, const Plan& p, int mode, cudaStream_t st,
                           const float* ext = nullptr, int64_t n_ext = 0, int d = 0, int dv = 0,
                           int f4_layout = 0, const float* lam = nullptr, int H = 1) {
  dim3 grid((nel + kSimtThreads - 1) / kSimtThreads, (unsigned)nseq);
  LaunchTimer t(K_CHUNK_SCAN, st);
  if (launch_pdl(chunk_scan_kernel, grid, dim3(kSimtThreads), 0, st, s, p.C, nel, mode,
                 n_ext > 0 ? ext : nullptr, n_ext, nseq, d, dv, f4_layout, lam, H, p.L) != cudaSuccess)
    return LA2_ERR_CUDA;
  return launch_status();
}

template <typename T>
static la2_status forward_simt(const void* q, const void* k, const void* v, void* o, const Heads& hd,
                               int64_t N, int d, int dv, int causal, int block, float* states,
                               const Plan& p, cudaStream_t st, const float* lam = nullptr) {
  const size_t smem = fwd_simt_smem(d, dv, block, sizeof(T), lam != nullptr);
  if (cudaFuncSetAttribute(fwd_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return LA2_ERR_CUDA;
  LaunchTimer t(K_FWD_SIMT, st);
  fwd_simt_kernel<T><<<(unsigned)(hd.BH * p.C), kSimtThreads, smem, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
      static_cast<T*>(o), states, N, d, dv, block, p.L, p.C, causal, hd.H, hd.G, lam);
  return launch_status();
}

template <typename T>
static la2_status backward_simt(const void* q, const void* k, const void* v, const void* dout,
                                void* dq, void* dk, void* dvv, const Heads& hd, int64_t N, int d,
                                int dv, int causal, int block, float* s_kv, float* s_u,
                                const Plan& p, cudaStream_t st, const float* lam = nullptr) {
  const size_t smem_q = bwd_dq_simt_smem(d, dv, block, sizeof(T), lam != nullptr);
  const size_t smem_kv = bwd_dkdv_simt_smem(d, dv, block, sizeof(T), lam != nullptr);
  if (cudaFuncSetAttribute(bwd_dq_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem_q) != cudaSuccess ||
      cudaFuncSetAttribute(bwd_dkdv_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem_kv) != cudaSuccess)
    return LA2_ERR_CUDA;
  {
    LaunchTimer t(K_BWD_DQ_SIMT, st);
    bwd_dq_simt_kernel<T><<<(unsigned)(hd.BH * p.C), kSimtThreads, smem_q, st>>>(
        static_cast<const T*>(k), static_cast<const T*>(v), static_cast<const T*>(dout),
        static_cast<T*>(dq), s_kv, N, d, dv, block, p.L, p.C, causal, hd.H, hd.G, lam);
  }
  la2_status s = launch_status();
  if (s != LA2_OK) return s;
  {
    LaunchTimer t(K_BWD_DKDV_SIMT, st);
    bwd_dkdv_simt_kernel<T><<<(unsigned)(hd.BHkv * p.C), kSimtThreads, smem_kv, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
        static_cast<const T*>(dout), static_cast<T*>(dk), static_cast<T*>(dvv), s_u, N, d, dv,
        block, p.L, p.C, causal, hd.H, hd.G, lam);
  }
  return launch_status();
}

// Causal O = ((Q K^T) ⊙ M) V on the persistent range-split kernel: the
// (b, h, block) task list cut into at most one range per SM; a range that
// starts inside a sequence gets its initial state from a pre-pass over the
// sequence's earlier blocks or from the range states of a separate pass.
// Also the dQ pass of the backward, with (dO, V, K) in the (Q, K, V) slots.
// The K and V slots hold hd.BHkv sequences, read through the head map.
template <int BK>
static la2_status causal_range_split(const void* q, const void* k, const void* v, void* o,
                                     const Heads& hd, int64_t N, float* range_states,
                                     const RangePlan& rp, int64_t spin, cudaStream_t st,
                                     int kid_states, int kid_main) {
  constexpr int D = 128, DV = 128;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_3d(&tq, q, hd.BH, N, D, BK) || !make_tmap_3d(&tk, k, hd.BHkv, N, D, BK) ||
      !make_tmap_3d(&tv, v, hd.BHkv, N, DV, BK))
    return LA2_ERR_CUDA;
  sm100::RangeTable rt;
  if (!fill_range_table(rp, &rt)) return LA2_ERR_UNSUPPORTED;
  // O tiles leave through per-warp TMA stores: 16 rows a warp at Bk=64, 32 at Bk=128.
  CUtensorMap to = tq;
  using CF = sm100::CCfg<BK, D, DV>;
  // (Bk=64 with O transposed in TMEM: one store of the whole 64-row tile.)
  if ((CF::TMA_STORE || CF::O_IN_Q) &&
      !make_tmap_3d(&to, o, hd.BH, N, DV, CF::O_IN_Q ? 32 : (CF::OT ? BK : 16)))
    return LA2_ERR_CUDA;
  sm100::CausalParams cp{};
  cp.o = static_cast<__nv_bfloat16*>(o);
  cp.agg = range_states;
  cp.N = N;
  cp.spin_limit = spin;
  cp.H = hd.H;
  cp.G = hd.G;
  const int sms = device_sm_count();
  const int grid = std::max(1, std::min(rp.R, sms));
  if (rp.prefix_mode == 1) {
    LaunchTimer t(kid_states, st);
    const la2_status s = launch_causal_sm100<BK, D, DV, sm100::KIND_AGG>(tq, tk, tv, to, rt, cp, grid, st);
    if (s != LA2_OK) return s;
  }
  LaunchTimer t(kid_main, st);
  return launch_causal_sm100<BK, D, DV, sm100::KIND_MAIN>(tq, tk, tv, to, rt, cp, grid, st);
}

// Non-causal: up to this many chunk states per sequence are added up inside
// the map pass (no scan launch); more are scanned into slot 0 first.
constexpr int64_t kSumInKernel = 8;

// K^T V chunk states of every K/V sequence (MODE_STATE, one unit per K/V
// sequence and chunk; tk and tv hold hd.BHkv sequences).
template <int BK>
static la2_status kv_chunk_states(const CUtensorMap& tk, const CUtensorMap& tv, float* states,
                                  const Heads& hd, int64_t N, const Plan& p, int64_t spin,
                                  cudaStream_t st) {
  sm100::Params ps{};
  ps.N = N;
  ps.L = p.L;
  ps.C = p.C;
  ps.units_per_seq = p.C;
  ps.out_states = states;
  ps.spin_limit = spin;
  ps.H = hd.H;
  ps.G = hd.G;
  ps.state_group = 1;
  LaunchTimer t(K_STATE_TC, st);
  return launch_fwd_sm100<BK, 128, 128, sm100::MODE_STATE>(tk, tk, tv, tk, ps, hd.BHkv * p.C, st);
}

// Tensor-core forward. Causal: the range split above (or, for splits the
// range table cannot hold, chunk states, their prefix, and the chunk loops).
// Non-causal: chunk states, their total, then every block against the total.
template <int BK>
static la2_status forward_sm100_bk(const void* q, const void* k, const void* v, void* o,
                                   const Heads& hd, int64_t N, int causal, float* states,
                                   const Plan& p, int64_t spin, cudaStream_t st, const Ext& ext) {
  if (causal && p.ranges)
    return causal_range_split<BK>(q, k, v, o, hd, N, states, p.rp, spin, st, K_STATE_TC, K_FWD_TC);
  constexpr int D = 128, DV = 128;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_3d(&tq, q, hd.BH, N, D, BK) || !make_tmap_3d(&tk, k, hd.BHkv, N, D, BK) ||
      !make_tmap_3d(&tv, v, hd.BHkv, N, DV, BK))
    return LA2_ERR_CUDA;
  sm100::Params prm{};
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.N = N;
  prm.L = p.L;
  prm.C = p.C;
  prm.spin_limit = spin;
  prm.H = hd.H;
  prm.G = hd.G;
  prm.state_group = 1;
  la2_status s = LA2_OK;
  const int nel = D * DV;
  CUtensorMap to_c = tq;
  if (sm100::Cfg<BK, D, DV>::TMA_STORE && !make_tmap_3d(&to_c, o, hd.BH, N, DV, 16)) return LA2_ERR_CUDA;
  if (causal) {
    // A split the range table cannot hold: chunk states, their exclusive
    // prefix per sequence, then every chunk's block loop from its prefix.
    if (p.need_states) {
      s = kv_chunk_states<BK>(tk, tv, states, hd, N, p, spin, st);
      if (s != LA2_OK) return s;
      s = run_scan(states, hd.BHkv, nel, p, 0, st, ext.pre, ext.n_pre, D, DV, 1);
      if (s != LA2_OK) return s;
    }
    prm.init_states = p.need_states ? states : nullptr;
    prm.init_all = ext.on ? 1 : 0;
    prm.units_per_seq = p.C;
    LaunchTimer t(K_FWD_TC, st);
    return launch_fwd_sm100<BK, D, DV, sm100::MODE_CAUSAL>(tq, tk, tv, to_c, prm, hd.BH * p.C, st);
  }
  s = kv_chunk_states<BK>(tk, tv, states, hd, N, p, spin, st);
  if (s != LA2_OK) return s;
  // A few chunk states: the map pass adds them up itself; many: scan first.
  prm.init_count = p.C <= kSumInKernel ? p.C : 1;
  if (p.C > kSumInKernel) {
    s = run_scan(states, hd.BHkv, nel, p, 2, st);
    if (s != LA2_OK) return s;
  }
  prm.init_states = states;
  prm.units_per_seq = p.C;
  LaunchTimer t(K_FWD_TC, st);
  return launch_fwd_sm100<BK, D, DV, sm100::MODE_NONCAUSAL>(tq, tk, tv, to_c, prm, hd.BH * p.C, st);
}

// The dK/dV pass: one unit per K/V sequence and chunk, reverse block order,
// the group's query heads walked per block (tiles of TB rows).
template <int TB>
static la2_status dkdv_sm100(const void* q, const void* k, const void* v, const void* dout, void* dk,
                             void* dvv, const Heads& hd, int64_t N, int causal, const float* s_u,
                             const Plan& p, int64_t spin, cudaStream_t st, bool init_all,
                             bool sum_states) {
  constexpr int D = 128, DV = 128;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_tmap_3d(&tq, q, hd.BH, N, D, TB) || !make_tmap_3d(&tk, k, hd.BHkv, N, D, TB) ||
      !make_tmap_3d(&tv, v, hd.BHkv, N, DV, TB) || !make_tmap_3d(&tdo, dout, hd.BH, N, DV, TB))
    return LA2_ERR_CUDA;
  sm100::BwdParams pb{};
  pb.dk = static_cast<__nv_bfloat16*>(dk);
  pb.dv = static_cast<__nv_bfloat16*>(dvv);
  pb.init_u = s_u;
  pb.N = N;
  pb.L = p.L;
  pb.C = p.C;
  pb.spin_limit = spin;
  pb.causal = causal;
  pb.H = hd.H;
  pb.G = hd.G;
  pb.init_all = init_all ? 1 : 0;
  pb.sum_states = sum_states ? 1 : 0;
  pb.split = causal ? p.dk_split : 0;
  CUtensorMap tdk = tq, tdv = tq;
  using BC = sm100::BCfg<TB, D, DV>;
  const int srows = BC::OT ? TB : 16;  // transposed accumulators: one store of the whole tile
  if (BC::TMA_STORE &&
      (!make_tmap_3d(&tdk, dk, hd.BHkv, N, D, srows) || !make_tmap_3d(&tdv, dvv, hd.BHkv, N, DV, srows)))
    return LA2_ERR_CUDA;
  LaunchTimer t(K_BWD_DKDV_TC, st);
  return launch_bwd_dkdv_sm100<TB>(tq, tk, tv, tdo, tdk, tdv, pb, hd.BHkv * p.C, st);
}

// Tensor-core backward: chunk states K^T V (prefix for dQ) and Q^T dO
// (suffix for dK, dV; summed over a group's query heads), their scans, then
// the dQ pass (the block loop with dO, V, K in the Q, K, V slots) and the
// reverse dK/dV pass.
template <int BK>
static la2_status backward_sm100_bk(const void* q, const void* k, const void* v, const void* dout,
                                    void* dq, void* dk, void* dvv, const Heads& hd, int64_t N,
                                    int causal, float* s_kv, float* s_u, const Plan& p,
                                    int64_t spin, cudaStream_t st, const Ext& ext) {
  constexpr int D = 128, DV = 128;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_tmap_3d(&tq, q, hd.BH, N, D, BK) || !make_tmap_3d(&tk, k, hd.BHkv, N, D, BK) ||
      !make_tmap_3d(&tv, v, hd.BHkv, N, DV, BK) || !make_tmap_3d(&tdo, dout, hd.BH, N, DV, BK))
    return LA2_ERR_CUDA;
  la2_status s = LA2_OK;
  const int nel = D * DV;
  const bool states = p.need_states;
  const bool dq_split = causal && p.dq_ranges;
  const bool u_summed = states && !ext.on && p.C <= kSumInKernel;
  if (dq_split) {
    // dQ = ((dO V^T) ⊙ M) K: the causal forward with (dO, V, K) as (Q, K, V).
    s = causal_range_split<BK>(dout, v, k, dq, hd, N, s_kv, p.rp, spin, st, K_STATE_TC, K_BWD_DQ_TC);
    if (s != LA2_OK) return s;
  }
  if (states) {  // (a dK/dV split builds its suffix state in the kernel: no states)
    if (!dq_split) {
      s = kv_chunk_states<BK>(tk, tv, s_kv, hd, N, p, spin, st);  // K^T V per chunk
      if (s != LA2_OK) return s;
    }
    {
      // Q^T dO per chunk of each K/V sequence, summed over its group's query heads
      sm100::Params ps{};
      ps.N = N;
      ps.L = p.L;
      ps.C = p.C;
      ps.units_per_seq = p.C;
      ps.spin_limit = spin;
      ps.out_states = s_u;
      ps.H = hd.H;
      ps.G = hd.G;
      ps.state_group = hd.G;
      LaunchTimer t(K_STATE_TC, st);
      s = launch_fwd_sm100<BK, D, DV, sm100::MODE_STATE>(tq, tq, tdo, tq, ps, hd.BHkv * p.C, st);
    }
    if (s != LA2_OK) return s;
    if (!dq_split && (causal || p.C > kSumInKernel)) {
      s = run_scan(s_kv, hd.BHkv, nel, p, causal ? 0 : 2, st, ext.pre, ext.n_pre, D, DV, 1);
      if (s != LA2_OK) return s;
    }
    // A few chunk states per sequence: the dK/dV pass adds up the later (or,
    // without the mask, all) chunks' states itself; many, or with external
    // states of other parts: scan first.
    if (!u_summed) {
      s = run_scan(s_u, hd.BHkv, nel, p, causal ? 1 : 2, st, ext.suf, ext.n_suf, D, DV, 1);
      if (s != LA2_OK) return s;
    }
  }
  // Otherwise (non-causal, or a forced split beyond the range table) the
  // block loop over chunks from the scanned K^T V prefix (or total) states.
  if (!dq_split) {
    sm100::Params pq{};
    pq.o = static_cast<__nv_bfloat16*>(dq);
    pq.init_states = states ? s_kv : nullptr;
    pq.N = N;
    pq.L = p.L;
    pq.C = p.C;
    pq.units_per_seq = p.C;
    pq.init_count = p.C <= kSumInKernel ? p.C : 1;  // non-causal dQ: summed here or scanned
    pq.spin_limit = spin;
    pq.H = hd.H;
    pq.G = hd.G;
    pq.state_group = 1;
    pq.init_all = ext.on ? 1 : 0;
    CUtensorMap tdq = tq;
    if (sm100::Cfg<BK, D, DV>::TMA_STORE && !make_tmap_3d(&tdq, dq, hd.BH, N, D, 16)) return LA2_ERR_CUDA;
    {
      LaunchTimer t(K_BWD_DQ_TC, st);
      s = causal
              ? launch_fwd_sm100<BK, D, DV, sm100::MODE_CAUSAL, true>(tdo, tv, tk, tdq, pq, hd.BH * p.C, st)
              : launch_fwd_sm100<BK, D, DV, sm100::MODE_NONCAUSAL, true>(tdo, tv, tk, tdq, pq,
                                                                        hd.BH * p.C, st);
    }
    if (s != LA2_OK) return s;
  }
  // A group of query heads accumulates into one dK, dV: the scores of each
  // head need their own TMEM columns, which 64-row tiles leave free.
  if (hd.G > 1 && BK == 128 && causal)
    return dkdv_sm100<64>(q, k, v, dout, dk, dvv, hd, N, causal, states ? s_u : nullptr, p, spin, st,
                          ext.on, u_summed);
  return dkdv_sm100<BK>(q, k, v, dout, dk, dvv, hd, N, causal, states ? s_u : nullptr, p, spin, st,
                        ext.on, u_summed);
}

static la2_status forward_sm100(const void* q, const void* k, const void* v, void* o, const Heads& hd,
                                int64_t N, int causal, int block, float* states, const Plan& p,
                                int64_t spin, cudaStream_t st, const Ext& ext) {
  return block == 64 ? forward_sm100_bk<64>(q, k, v, o, hd, N, causal, states, p, spin, st, ext)
                     : forward_sm100_bk<128>(q, k, v, o, hd, N, causal, states, p, spin, st, ext);
}

}  // namespace la2

using namespace la2;

// ====================================================================== C ABI

extern "C" {

size_t la2_workspace_size_gqa(int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t d, int64_t dv,
                              int causal, int block, la2_dtype dt, int is_backward) {
  if (check_shape(B, H, N, d, dv, causal, block, dt, is_backward != 0, Hkv) != LA2_OK) return (size_t)-1;
  if (B == 0 || H == 0 || N == 0) return 0;
  const int sms = device_sm_count();
  if (sms <= 0) return (size_t)-1;
  return make_plan(B, H, N, d, dv, causal, block, dt, is_backward != 0, sms, Hkv).ws_bytes;
}

size_t la2_workspace_size(int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv, int causal,
                          int block, la2_dtype dt, int is_backward) {
  return la2_workspace_size_gqa(B, H, H, N, d, dv, causal, block, dt, is_backward);
}

int64_t la2_plan_ranges(int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv, int causal,
                        int block, la2_dtype dt, int is_backward, int64_t* starts, int64_t cap) {
  if (check_shape(B, H, N, d, dv, causal, block, dt, is_backward != 0) != LA2_OK) return -1;
  if (B == 0 || H == 0 || N == 0) return 0;
  const int sms = device_sm_count();
  if (sms <= 0) return -1;
  const Plan p = make_plan(B, H, N, d, dv, causal, block, dt, is_backward != 0, sms);
  const int64_t T = (N + block - 1) / block;
  std::vector<int64_t> v;
  if (p.ranges) {
    v = p.rp.starts;
  } else {
    const int64_t per = p.L / block;
    for (int64_t h = 0; h < B * H; ++h)
      for (int64_t c = 0; c < p.C; ++c) v.push_back(h * T + c * per);
    v.push_back(B * H * T);
  }
  const int64_t R = static_cast<int64_t>(v.size()) - 1;
  if (starts && cap >= R + 1)
    for (int64_t i = 0; i <= R; ++i) starts[i] = v[i];
  return R;
}

la2_status la2_set_chunk_len(int64_t chunk_len) {
  if (chunk_len < 0) return LA2_ERR_INVALID_ARG;
  g_chunk_len = chunk_len;
  return LA2_OK;
}

la2_status la2_set_spin_limit(int64_t iterations) {
  if (iterations < 0) return LA2_ERR_INVALID_ARG;
  g_spin_limit = iterations;
  return LA2_OK;
}

size_t la2_kv_state_workspace_size(int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv,
                                   la2_dtype dt) {
  if (check_shape(B, H, N, d, dv, 0, 64, dt, false) != LA2_OK) return (size_t)-1;
  if (B == 0 || H == 0 || N == 0) return 0;
  const int sms = device_sm_count();
  if (sms <= 0) return (size_t)-1;
  return make_plan(B, H, N, d, dv, 0, 64, dt, false, sms).ws_bytes;
}

la2_status la2_kv_state(const void* k, const void* v, float* state, int64_t B, int64_t H, int64_t N,
                        int64_t d, int64_t dv, la2_dtype dt, void* workspace,
                        size_t workspace_bytes, la2_stream_t stream) {
  la2_status s = check_shape(B, H, N, d, dv, 0, 64, dt, false);
  if (s != LA2_OK) return s;
  if (B == 0 || H == 0 || N == 0) return LA2_OK;
  if (!k || !v || !state) return LA2_ERR_INVALID_ARG;
  if (!is_aligned(k, 16) || !is_aligned(v, 16) || !is_aligned(state, 16)) return LA2_ERR_INVALID_ARG;
  const size_t es = dt == LA2_BF16 ? 2 : 4;
  const int64_t BH = B * H;
  const size_t nk = (size_t)BH * N * d * es, nv = (size_t)BH * N * dv * es;
  const size_t ns = (size_t)BH * d * dv * sizeof(float);
  if (overlaps(state, ns, k, nk) || overlaps(state, ns, v, nv)) return LA2_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  if (sms <= 0) return LA2_ERR_CUDA;
  // The non-causal plan: per-chunk states K_c^T V_c, then their sum per sequence.
  const Plan p = make_plan(B, H, N, d, dv, 0, 64, dt, false, sms);
  if (!workspace || workspace_bytes < p.ws_bytes) return LA2_ERR_WORKSPACE;
  if (!is_aligned(workspace, 256)) return LA2_ERR_INVALID_ARG;
  if (overlaps(workspace, p.ws_bytes, state, ns)) return LA2_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* chunks = static_cast<float*>(workspace);
  if (p.tc) {
    CUtensorMap tk, tv;
    if (!make_tmap_3d(&tk, k, BH, N, 128, 64) || !make_tmap_3d(&tv, v, BH, N, 128, 64))
      return LA2_ERR_CUDA;
    sm100::Params ps{};
    ps.N = N;
    ps.L = p.L;
    ps.C = p.C;
    ps.units_per_seq = p.C;
    ps.out_states = chunks;
    ps.spin_limit = spin_limit();
    ps.H = 1;
    ps.G = 1;
    ps.state_group = 1;
    LaunchTimer t(K_STATE_TC, st);
    s = launch_fwd_sm100<64, 128, 128, sm100::MODE_STATE>(tk, tk, tv, tk, ps, BH * p.C, st);
  } else {
    s = dt == LA2_BF16 ? run_chunk_states<__nv_bfloat16>(k, v, chunks, BH, N, (int)d, (int)dv, p, st)
                       : run_chunk_states<float>(k, v, chunks, BH, N, (int)d, (int)dv, p, st);
  }
  if (s != LA2_OK) return s;
  const int nel = (int)(d * dv);
  LaunchTimer t(K_STATE_ACC, st);
  if (launch_pdl(state_accumulate_kernel, dim3((unsigned)((nel + 255) / 256), (unsigned)BH),
                 dim3(256), 0, st, static_cast<const float*>(chunks), state, p.C, (int)d, (int)dv,
                 p.tc ? 1 : 0) != cudaSuccess)
    return LA2_ERR_CUDA;
  return launch_status();
}

la2_status la2_decode_step(const void* q, const void* k, const void* v, void* o, float* state,
                           int64_t B, int64_t H, int64_t d, int64_t dv, la2_dtype dt,
                           la2_stream_t stream) {
  if (B < 0 || H < 0 || d < 1 || dv < 1) return LA2_ERR_INVALID_ARG;
  if (dt != LA2_F32 && dt != LA2_BF16) return LA2_ERR_INVALID_ARG;
  if (double(B) * double(H) * double(d) * double(dv) > 9.0e18) return LA2_ERR_INVALID_ARG;
  if (B == 0 || H == 0) return LA2_OK;
  if (!q || !k || !v || !o || !state) return LA2_ERR_INVALID_ARG;
  const size_t es = dt == LA2_BF16 ? 2 : 4;
  if (!is_aligned(q, es) || !is_aligned(k, es) || !is_aligned(v, es) || !is_aligned(o, es) ||
      !is_aligned(state, 4))
    return LA2_ERR_INVALID_ARG;
  const int64_t BH = B * H;
  if (BH > 0x7fffffff || (dv + 31) / 32 > 65535) return LA2_ERR_UNSUPPORTED;
  const size_t nq = (size_t)BH * d * es, nv = (size_t)BH * dv * es;
  const size_t ns = (size_t)BH * d * dv * sizeof(float);
  if (overlaps(o, nv, q, nq) || overlaps(o, nv, k, nq) || overlaps(o, nv, v, nv) ||
      overlaps(o, nv, state, ns) || overlaps(state, ns, q, nq) || overlaps(state, ns, k, nq) ||
      overlaps(state, ns, v, nv))
    return LA2_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  LaunchTimer t(K_DECODE, st);
  // Four columns per lane when rows of the state, v and o allow 16-, 8- or
  // 16-byte vector accesses and every row of a thread fits in its registers.
  const dim3 block(32 * kDecodeWarps);
  cudaError_t e;
  if (dv % 4 == 0 && d <= kDecodeWarps * kRows && is_aligned(state, 16) && is_aligned(v, 4 * es) &&
      is_aligned(o, es)) {
    const dim3 grid4((unsigned)BH, (unsigned)((dv + 127) / 128));
    if (dt == LA2_BF16)
      e = launch_pdl(decode_step_v4_kernel<__nv_bfloat16>, grid4, block, 0, st,
                     static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                     static_cast<const __nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(o), state,
                     (int)d, (int)dv);
    else
      e = launch_pdl(decode_step_v4_kernel<float>, grid4, block, 0, st,
                     static_cast<const float*>(q), static_cast<const float*>(k),
                     static_cast<const float*>(v), static_cast<float*>(o), state, (int)d, (int)dv);
  } else {
    const dim3 grid((unsigned)BH, (unsigned)((dv + 31) / 32));
    if (dt == LA2_BF16)
      e = launch_pdl(decode_step_kernel<__nv_bfloat16>, grid, block, 0, st,
                     static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                     static_cast<const __nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(o), state,
                     (int)d, (int)dv);
    else
      e = launch_pdl(decode_step_kernel<float>, grid, block, 0, st, static_cast<const float*>(q),
                     static_cast<const float*>(k), static_cast<const float*>(v),
                     static_cast<float*>(o), state, (int)d, (int)dv);
  }
  if (e != cudaSuccess) return LA2_ERR_CUDA;
  return launch_status();
}

}  // extern "C"

namespace la2 {

static bool ext_ok(const float* p, int64_t n, size_t one, const void* out, size_t nout) {
  if (n < 0) return false;
  if (n == 0) return true;
  if (!p || !is_aligned(p, 16)) return false;
  return !overlaps(p, (size_t)n * one, out, nout);
}

static la2_status forward_impl(const void* q, const void* k, const void* v, void* o, int64_t B,
                               int64_t H, int64_t Hkv, int64_t N, int64_t d, int64_t dv, int causal,
                               int block, la2_dtype dt, void* workspace, size_t workspace_bytes,
                               la2_stream_t stream, const Ext& ext) {
  la2_status s = check_shape(B, H, N, d, dv, causal, block, dt, false, Hkv);
  if (s != LA2_OK) return s;
  if (B == 0 || H == 0 || N == 0) return LA2_OK;
  if (!q || !k || !v || !o) return LA2_ERR_INVALID_ARG;
  if (!is_aligned(q, 16) || !is_aligned(k, 16) || !is_aligned(v, 16) || !is_aligned(o, 16))
    return LA2_ERR_INVALID_ARG;
  const size_t es = dt == LA2_BF16 ? 2 : 4;
  const size_t nq = (size_t)B * H * N * d * es, no = (size_t)B * H * N * dv * es;
  const size_t nk = (size_t)B * Hkv * N * d * es, nv = (size_t)B * Hkv * N * dv * es;
  if (overlaps(o, no, q, nq) || overlaps(o, no, k, nk) || overlaps(o, no, v, nv))
    return LA2_ERR_INVALID_ARG;
  if (!ext_ok(ext.pre, ext.n_pre, (size_t)B * Hkv * d * dv * sizeof(float), o, no))
    return LA2_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  if (sms <= 0) return LA2_ERR_CUDA;
  const Plan p = make_plan(B, H, N, d, dv, causal, block, dt, false, sms, Hkv, ext.on);
  const Heads hd{B * H, B * Hkv, static_cast<int32_t>(H), static_cast<int32_t>(H / Hkv)};
  if (p.ws_bytes > 0) {
    if (!workspace || workspace_bytes < p.ws_bytes) return LA2_ERR_WORKSPACE;
    if (!is_aligned(workspace, 256)) return LA2_ERR_INVALID_ARG;
    if (overlaps(workspace, p.ws_bytes, o, no)) return LA2_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* states = p.need_states ? static_cast<float*>(workspace) : nullptr;
  const int nel = (int)(d * dv);
  if (p.tc) return forward_sm100(q, k, v, o, hd, N, causal, block, states, p, spin_limit(), st, ext);
  if (p.need_states) {  // K^T V chunk states of the K/V sequences, then their prefix / total
    s = dt == LA2_BF16
            ? run_chunk_states<__nv_bfloat16>(k, v, states, hd.BHkv, N, (int)d, (int)dv, p, st)
            : run_chunk_states<float>(k, v, states, hd.BHkv, N, (int)d, (int)dv, p, st);
    if (s != LA2_OK) return s;
    s = run_scan(states, hd.BHkv, nel, p, causal ? 0 : 2, st, ext.pre, ext.n_pre, (int)d, (int)dv, 0);
    if (s != LA2_OK) return s;
  }
  return dt == LA2_BF16
             ? forward_simt<__nv_bfloat16>(q, k, v, o, hd, N, (int)d, (int)dv, causal, block,
                                           states, p, st)
             : forward_simt<float>(q, k, v, o, hd, N, (int)d, (int)dv, causal, block, states, p,
                                   st);
}

}  // namespace la2

extern "C" {

la2_status la2_forward_gqa(const void* q, const void* k, const void* v, void* o, int64_t B,
                           int64_t H, int64_t Hkv, int64_t N, int64_t d, int64_t dv, int causal,
                           int block, la2_dtype dt, void* workspace, size_t workspace_bytes,
                           la2_stream_t stream) {
  return forward_impl(q, k, v, o, B, H, Hkv, N, d, dv, causal, block, dt, workspace, workspace_bytes,
                      stream, Ext{});
}

la2_status la2_forward_sp(const void* q, const void* k, const void* v, void* o,
                          const float* prefix_states, int64_t n_prefix, int64_t B, int64_t H,
                          int64_t N, int64_t d, int64_t dv, int block, la2_dtype dt,
                          void* workspace, size_t workspace_bytes, la2_stream_t stream) {
  Ext ext;
  ext.pre = prefix_states;
  ext.n_pre = n_prefix;
  ext.on = true;
  return forward_impl(q, k, v, o, B, H, H, N, d, dv, 1, block, dt, workspace, workspace_bytes, stream,
                      ext);
}

size_t la2_workspace_size_sp(int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv, int block,
                             la2_dtype dt, int is_backward) {
  if (check_shape(B, H, N, d, dv, 1, block, dt, is_backward != 0) != LA2_OK) return (size_t)-1;
  if (B == 0 || H == 0 || N == 0) return 0;
  const int sms = device_sm_count();
  if (sms <= 0) return (size_t)-1;
  return make_plan(B, H, N, d, dv, 1, block, dt, is_backward != 0, sms, H, true).ws_bytes;
}

la2_status la2_forward(const void* q, const void* k, const void* v, void* o, int64_t B, int64_t H,
                       int64_t N, int64_t d, int64_t dv, int causal, int block, la2_dtype dt,
                       void* workspace, size_t workspace_bytes, la2_stream_t stream) {
  return la2_forward_gqa(q, k, v, o, B, H, H, N, d, dv, causal, block, dt, workspace,
                         workspace_bytes, stream);
}

}  // extern "C"

namespace la2 {

static la2_status backward_impl(const void* q, const void* k, const void* v, const void* dout,
                                void* dq, void* dk, void* dvv, int64_t B, int64_t H, int64_t Hkv,
                                int64_t N, int64_t d, int64_t dv, int causal, int block,
                                la2_dtype dt, void* workspace, size_t workspace_bytes,
                                la2_stream_t stream, const Ext& ext) {
  la2_status s = check_shape(B, H, N, d, dv, causal, block, dt, true, Hkv);
  if (s != LA2_OK) return s;
  if (B == 0 || H == 0 || N == 0) return LA2_OK;
  const void* ins[4] = {q, k, v, dout};
  void* outs[3] = {dq, dk, dvv};
  for (const void* p : ins)
    if (!p || !is_aligned(p, 16)) return LA2_ERR_INVALID_ARG;
  for (void* p : outs)
    if (!p || !is_aligned(p, 16)) return LA2_ERR_INVALID_ARG;
  const size_t es = dt == LA2_BF16 ? 2 : 4;
  const size_t nq = (size_t)B * H * N * d * es, nod = (size_t)B * H * N * dv * es;
  const size_t nk = (size_t)B * Hkv * N * d * es, nv = (size_t)B * Hkv * N * dv * es;
  const size_t in_sz[4] = {nq, nk, nv, nod};
  const size_t out_sz[3] = {nq, nk, nv};
  for (int i = 0; i < 3; ++i) {
    for (int j = 0; j < 4; ++j)
      if (overlaps(outs[i], out_sz[i], ins[j], in_sz[j])) return LA2_ERR_INVALID_ARG;
    for (int j = i + 1; j < 3; ++j)
      if (overlaps(outs[i], out_sz[i], outs[j], out_sz[j])) return LA2_ERR_INVALID_ARG;
  }
  const size_t one = (size_t)B * Hkv * d * dv * sizeof(float);
  for (int i = 0; i < 3; ++i)
    if (!ext_ok(ext.pre, ext.n_pre, one, outs[i], out_sz[i]) ||
        !ext_ok(ext.suf, ext.n_suf, one, outs[i], out_sz[i]))
      return LA2_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  if (sms <= 0) return LA2_ERR_CUDA;
  const Plan p = make_plan(B, H, N, d, dv, causal, block, dt, true, sms, Hkv, ext.on);
  if (p.ws_bytes > 0) {
    if (!workspace || workspace_bytes < p.ws_bytes) return LA2_ERR_WORKSPACE;
    if (!is_aligned(workspace, 256)) return LA2_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i)
      if (overlaps(workspace, p.ws_bytes, outs[i], out_sz[i])) return LA2_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Heads hd{B * H, B * Hkv, static_cast<int32_t>(H), static_cast<int32_t>(H / Hkv)};
  const int nel = (int)(d * dv);
  // chunk states of the K/V sequences: [K^T V | Q^T dO summed over each group]
  float* s_kv = p.need_states ? static_cast<float*>(workspace) : nullptr;
  float* s_u = p.need_states ? s_kv + (size_t)hd.BHkv * p.C * nel : nullptr;
  if (p.tc) {
    float* second = nullptr;  // K^T V chunk states, or the dQ pass's range states
    if (p.need_states) {
      s_u = static_cast<float*>(workspace);
      second = s_u + (size_t)hd.BHkv * p.C * nel;
    } else if (p.ws_bytes > 0) {
      second = static_cast<float*>(workspace);
    }
    return block == 64 ? backward_sm100_bk<64>(q, k, v, dout, dq, dk, dvv, hd, N, causal, second,
                                                s_u, p, spin_limit(), st, ext)
                       : backward_sm100_bk<128>(q, k, v, dout, dq, dk, dvv, hd, N, causal, second,
                                                 s_u, p, spin_limit(), st, ext);
  }
  if (p.need_states) {
    const bool bf = dt == LA2_BF16;
    s = bf ? run_chunk_states<__nv_bfloat16>(k, v, s_kv, hd.BHkv, N, (int)d, (int)dv, p, st)
           : run_chunk_states<float>(k, v, s_kv, hd.BHkv, N, (int)d, (int)dv, p, st);
    if (s != LA2_OK) return s;
    s = bf ? run_chunk_states<__nv_bfloat16>(q, dout, s_u, hd.BHkv, N, (int)d, (int)dv, p, st,
                                             hd.H, hd.G, hd.G)
           : run_chunk_states<float>(q, dout, s_u, hd.BHkv, N, (int)d, (int)dv, p, st, hd.H, hd.G,
                                     hd.G);
    if (s != LA2_OK) return s;
    s = run_scan(s_kv, hd.BHkv, nel, p, causal ? 0 : 2, st, ext.pre, ext.n_pre, (int)d, (int)dv, 0);
    if (s != LA2_OK) return s;
    s = run_scan(s_u, hd.BHkv, nel, p, causal ? 1 : 2, st, ext.suf, ext.n_suf, (int)d, (int)dv, 0);
    if (s != LA2_OK) return s;
  }
  return dt == LA2_BF16
             ? backward_simt<__nv_bfloat16>(q, k, v, dout, dq, dk, dvv, hd, N, (int)d, (int)dv,
                                            causal, block, s_kv, s_u, p, st)
             : backward_simt<float>(q, k, v, dout, dq, dk, dvv, hd, N, (int)d, (int)dv, causal,
                                    block, s_kv, s_u, p, st);
}

// ------------------------------------------------------------------ decayed form

// Time reversal of up to four [S, N, 16 * kRevVecs bytes] row-major tensors
// (blockIdx.y picks the tensor): dst[s][N-1-t] = src[s][t]. With src == dst the
// reversal is in place: a thread swaps rows t and N-1-t of one 16-byte column
// for t < N/2 (the middle row of an odd N stays). Row index 32-bit: S * N
// <= INT32_MAX (checked by the caller). Each thread moves kRevUnroll columns a
// grid-stride step, all loads before the stores.
constexpr int kRevVecs = 16;  // 256-byte rows: 128 bf16
constexpr int kRevUnroll = 4;
struct RevArgs {
  const uint4* src[4];
  uint4* dst[4];
};

__global__ void __launch_bounds__(256) reverse_rows_kernel(RevArgs a, uint32_t N, uint32_t S) {
  pdl_launch_dependents();
  pdl_wait();
  const uint4* src = a.src[blockIdx.y];  // may be dst itself: no __restrict__
  uint4* dst = a.dst[blockIdx.y];
  const bool in_place = static_cast<const void*>(src) == static_cast<const void*>(dst);
  const uint32_t rows = in_place ? N / 2 : N;
  const uint64_t total = static_cast<uint64_t>(S) * rows * kRevVecs;
  const uint64_t step = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t e0 = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e0 < total;
       e0 += step * kRevUnroll) {
    uint64_t i[kRevUnroll], j[kRevUnroll];
    uint4 x[kRevUnroll], z[kRevUnroll];
#pragma unroll
    for (int u = 0; u < kRevUnroll; ++u) {
      const uint64_t e = e0 + u * step;
      if (e >= total) break;
      const uint32_t r = static_cast<uint32_t>(e / kRevVecs), c = static_cast<uint32_t>(e % kRevVecs);
      const uint32_t sq = r / rows, t = r - sq * rows;
      const uint64_t base = static_cast<uint64_t>(sq) * N;
      i[u] = (base + t) * kRevVecs + c;
      j[u] = (base + (N - 1 - t)) * kRevVecs + c;
      x[u] = src[i[u]];
      if (in_place) z[u] = dst[j[u]];
    }
#pragma unroll
    for (int u = 0; u < kRevUnroll; ++u) {
      if (e0 + u * step >= total) break;
      dst[j[u]] = x[u];
      if (in_place) dst[i[u]] = z[u];
    }
  }
}

// Reverses n (<= 4) bf16 [S, N, 128] tensors (src[i] == dst[i]: in place).
static la2_status reverse_rows(const void* const* src, void* const* dst, int n, int64_t S, int64_t N,
                               int sms, cudaStream_t st) {
  RevArgs a{};
  for (int i = 0; i < n; ++i) {
    a.src[i] = static_cast<const uint4*>(src[i]);
    a.dst[i] = static_cast<uint4*>(dst[i]);
  }
  const int64_t per = S * N * kRevVecs, threads = 256;
  const int64_t want = (per + threads * kRevUnroll - 1) / (threads * kRevUnroll);
  const unsigned blocks = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(want, 8LL * sms / n)));
  LaunchTimer t(K_REVERSE, st);
  if (launch_pdl(reverse_rows_kernel, dim3(blocks, static_cast<unsigned>(n)), dim3(threads), 0, st, a,
                 static_cast<uint32_t>(N), static_cast<uint32_t>(S)) != cudaSuccess)
    return LA2_ERR_CUDA;
  return LA2_OK;
}

// The decayed form on tensor cores: bf16, d = dv = 128, block 64 or 128.
static bool decay_tc(int64_t d, int64_t dv, int block, la2_dtype dt) {
  return dt == LA2_BF16 && sm100_supports(d, dv, block, false);
}

// Plan of the decayed form: chunks of L rows, chunk states decayed to a chunk
// edge and their decayed scan when a sequence has more than one chunk. The
// chunk count is chosen by waves of SMs (one CTA per (b, h, chunk)): the
// fewest waves times (chunk blocks + a fixed cost of 3 blocks), chunks of at
// least four blocks (B4 H16 N2K: 2 chunks, 128 CTAs in one wave, where 5 ran
// three waves). The tensor-core backward keeps one set of chunk states (its
// three passes run one after another) and the four time-reversed inputs.
static Plan plan_decay(int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv, int block,
                       bool is_bwd, bool tc, int sms) {
  Plan p;
  const int64_t BH = B * H, T = (N + block - 1) / block;
  int64_t L;
  if (g_chunk_len > 0) {
    L = ((g_chunk_len + block - 1) / block) * block;
  } else {
    const int64_t G = std::max(sms, 1), cmax = std::max<int64_t>(1, T / 4);
    int64_t C = 1;
    double best = 0.0;
    for (int64_t c = 1; c <= cmax; ++c) {
      const double cost = static_cast<double>((BH * c + G - 1) / G) *
                          (static_cast<double>((T + c - 1) / c) + 3.0);
      if (c == 1 || cost < best) {
        best = cost;
        C = c;
      }
    }
    L = ((T + C - 1) / C) * block;
  }
  p.L = std::max<int64_t>(L, block);
  p.C = std::max<int64_t>(1, (N + p.L - 1) / p.L);
  p.need_states = p.C > 1;
  const size_t states = p.need_states ? (size_t)BH * p.C * d * dv * sizeof(float) : 0;
  if (is_bwd && tc)
    p.ws_bytes = states + 4 * (size_t)BH * N * d * sizeof(__nv_bfloat16);
  else
    p.ws_bytes = states * (is_bwd ? 2 : 1);
  return p;
}

template <int BK>
static la2_status decay_forward_tc(const void* q, const void* k, const void* v, void* o,
                                  const float* lam, int64_t BH, int64_t H, int64_t N,
                                  float* states, const Plan& p, cudaStream_t st) {
  constexpr int D = 128, DV = 128;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_3d(&tq, q, BH, N, D, BK) || !make_tmap_3d(&tk, k, BH, N, D, BK) ||
      !make_tmap_3d(&tv, v, BH, N, DV, BK))
    return LA2_ERR_CUDA;
  sm100::Params prm{};
  prm.N = N;
  prm.L = p.L;
  prm.C = p.C;
  prm.units_per_seq = p.C;
  prm.spin_limit = spin_limit();
  prm.H = static_cast<int32_t>(H);
  prm.G = 1;
  prm.state_group = 1;
  prm.lam = lam;
  la2_status s = LA2_OK;
  if (p.need_states) {
    sm100::Params ps = prm;
    ps.out_states = states;
    {
      LaunchTimer t(K_STATE_TC, st);
      s = launch_fwd_sm100<BK, D, DV, sm100::MODE_STATE, false, true>(tk, tk, tv, tk, ps, BH * p.C, st);
    }
    if (s != LA2_OK) return s;
    // A few chunks a sequence: each chunk adds up the earlier chunks' states
    // itself (decay-weighted, no scan launch); many: their decayed prefix first.
    if (p.C > kSumInKernel) {
      s = run_scan(states, BH, D * DV, p, 3, st, nullptr, 0, D, DV, 0, lam, static_cast<int>(H));
      if (s != LA2_OK) return s;
    } else {
      prm.decay_sum = 1;
    }
  }
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.init_states = p.need_states ? states : nullptr;
  CUtensorMap to = tq;
  if (sm100::Cfg<BK, D, DV>::TMA_STORE && !make_tmap_3d(&to, o, BH, N, DV, 16)) return LA2_ERR_CUDA;
  LaunchTimer t(K_FWD_TC, st);
  return launch_fwd_sm100<BK, D, DV, sm100::MODE_CAUSAL, false, true>(tq, tk, tv, to, prm, BH * p.C, st);
}

// Gradients of the decayed form from three decayed forwards (bf16, d = dv =
// 128). dQ_t = sum_{s<=t} lam^(t-s) (dO_t . v_s) k_s is the forward with dO,
// V, K in the places of Q, K, V. dK_s = sum_{t>=s} lam^(t-s) (dO_t . v_s) q_t
// and dV_s = sum_{t>=s} lam^(t-s) (q_t . k_s) dO_t run over later rows: on
// the time-reversed sequences (row t at N-1-t) they are the causal forwards
// dK~ = F(V~, dO~, Q~) and dV~ = F(K~, Q~, dO~), written into dk / dvv and
// reversed there in place. `rev`: room for the four reversed inputs.
template <int BK>
static la2_status decay_backward_tc(const void* q, const void* k, const void* v, const void* dout,
                                    void* dq, void* dk, void* dvv, const float* lam, int64_t BH,
                                    int64_t H, int64_t N, float* states, void* rev, const Plan& p,
                                    int sms, cudaStream_t st) {
  la2_status s = decay_forward_tc<BK>(dout, v, k, dq, lam, BH, H, N, states, p, st);
  if (s != LA2_OK) return s;
  const size_t n = (size_t)BH * N * 128;
  __nv_bfloat16* qr = static_cast<__nv_bfloat16*>(rev);
  __nv_bfloat16 *kr = qr + n, *vr = kr + n, *dor = vr + n;
  const void* src[4] = {q, k, v, dout};
  void* dst[4] = {qr, kr, vr, dor};
  s = reverse_rows(src, dst, 4, BH, N, sms, st);
  if (s != LA2_OK) return s;
  s = decay_forward_tc<BK>(kr, qr, dor, dvv, lam, BH, H, N, states, p, st);
  if (s != LA2_OK) return s;
  s = decay_forward_tc<BK>(vr, dor, qr, dk, lam, BH, H, N, states, p, st);
  if (s != LA2_OK) return s;
  void* outs[2] = {dk, dvv};
  s = reverse_rows(outs, outs, 2, BH, N, sms, st);
  if (s != LA2_OK) return s;
  return launch_status();
}

static la2_status check_decay_shape(int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv,
                                    int block, la2_dtype dt, bool is_bwd) {
  const la2_status s = check_shape(B, H, N, d, dv, 1, block, dt, is_bwd);
  if (s != LA2_OK) return s;
  // tensor cores both ways; the backward's time reversal indexes rows in 32 bits
  if (decay_tc(d, dv, block, dt))
    return is_bwd && double(B) * double(H) * double(N) > 2147483647.0 ? LA2_ERR_UNSUPPORTED : LA2_OK;
  const size_t es = dt == LA2_BF16 ? 2 : 4, lim = 227 * 1024;
  if (fwd_simt_smem((int)d, (int)dv, block, es, true) > lim) return LA2_ERR_UNSUPPORTED;
  if (is_bwd && (bwd_dq_simt_smem((int)d, (int)dv, block, es, true) > lim ||
                 bwd_dkdv_simt_smem((int)d, (int)dv, block, es, true) > lim ||
                 !bwd_dkdv_simt_fits((int)d, (int)dv, block)))
    return LA2_ERR_UNSUPPORTED;
  return LA2_OK;
}

static la2_status decay_impl(const void* q, const void* k, const void* v, const void* dout, void* o,
                             void* dq, void* dk, void* dvv, const float* lam, int64_t B, int64_t H,
                             int64_t N, int64_t d, int64_t dv, int block, la2_dtype dt,
                             void* workspace, size_t workspace_bytes, la2_stream_t stream,
                             bool is_bwd) {
  la2_status s = check_decay_shape(B, H, N, d, dv, block, dt, is_bwd);
  if (s != LA2_OK) return s;
  if (B == 0 || H == 0 || N == 0) return LA2_OK;
  const size_t es = dt == LA2_BF16 ? 2 : 4;
  const size_t nq = (size_t)B * H * N * d * es, nv = (size_t)B * H * N * dv * es;
  const void* ins[4] = {q, k, v, is_bwd ? dout : q};
  const size_t in_sz[4] = {nq, nq, nv, is_bwd ? nv : nq};
  void* outs[3] = {is_bwd ? dq : o, is_bwd ? dk : nullptr, is_bwd ? dvv : nullptr};
  const size_t out_sz[3] = {is_bwd ? nq : nv, nq, nv};
  const int nout = is_bwd ? 3 : 1;
  for (const void* x : ins)
    if (!x || !is_aligned(x, 16)) return LA2_ERR_INVALID_ARG;
  if (!lam || !is_aligned(lam, 4)) return LA2_ERR_INVALID_ARG;
  const size_t nl = (size_t)H * sizeof(float);
  for (int i = 0; i < nout; ++i) {
    if (!outs[i] || !is_aligned(outs[i], 16)) return LA2_ERR_INVALID_ARG;
    for (int j = 0; j < 4; ++j)
      if (overlaps(outs[i], out_sz[i], ins[j], in_sz[j])) return LA2_ERR_INVALID_ARG;
    for (int j = i + 1; j < nout; ++j)
      if (overlaps(outs[i], out_sz[i], outs[j], out_sz[j])) return LA2_ERR_INVALID_ARG;
    if (overlaps(outs[i], out_sz[i], lam, nl)) return LA2_ERR_INVALID_ARG;
  }
  const int sms = device_sm_count();
  if (sms <= 0) return LA2_ERR_CUDA;
  const bool tc = decay_tc(d, dv, block, dt);
  const Plan p = plan_decay(B, H, N, d, dv, block, is_bwd, tc, sms);
  if (p.ws_bytes > 0) {
    if (!workspace || workspace_bytes < p.ws_bytes) return LA2_ERR_WORKSPACE;
    if (!is_aligned(workspace, 256)) return LA2_ERR_INVALID_ARG;
    for (int i = 0; i < nout; ++i)
      if (overlaps(workspace, p.ws_bytes, outs[i], out_sz[i])) return LA2_ERR_INVALID_ARG;
    for (int j = 0; j < 4; ++j)
      if (overlaps(workspace, p.ws_bytes, ins[j], in_sz[j])) return LA2_ERR_INVALID_ARG;
    if (overlaps(workspace, p.ws_bytes, lam, nl)) return LA2_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t BH = B * H;
  const Heads hd{BH, BH, static_cast<int32_t>(H), 1};
  const int nel = (int)(d * dv);
  const bool bf = dt == LA2_BF16;
  float* s_kv = p.need_states ? static_cast<float*>(workspace) : nullptr;
  float* s_u = p.need_states && is_bwd ? s_kv + (size_t)BH * p.C * nel : nullptr;
  // The tensor-core shapes: the chunk kernels with the decayed form (chunk
  // states decayed to their last row, their decayed prefix, then every chunk's
  // block loop from it); the backward as three such forwards.
  if (tc && !is_bwd)
    return block == 64 ? decay_forward_tc<64>(q, k, v, o, lam, BH, H, N, s_kv, p, st)
                       : decay_forward_tc<128>(q, k, v, o, lam, BH, H, N, s_kv, p, st);
  if (tc) {
    const size_t states = p.need_states ? (size_t)BH * p.C * nel * sizeof(float) : 0;
    void* rev = static_cast<char*>(workspace) + states;
    return block == 64
               ? decay_backward_tc<64>(q, k, v, dout, dq, dk, dvv, lam, BH, H, N, s_kv, rev, p, sms, st)
               : decay_backward_tc<128>(q, k, v, dout, dq, dk, dvv, lam, BH, H, N, s_kv, rev, p, sms, st);
  }
  if (p.need_states) {
    // K^T V of each chunk decayed to its last row, then their decayed prefix
    s = bf ? run_chunk_states<__nv_bfloat16>(k, v, s_kv, BH, N, (int)d, (int)dv, p, st, (int)H, 1, 1, lam, 1)
           : run_chunk_states<float>(k, v, s_kv, BH, N, (int)d, (int)dv, p, st, (int)H, 1, 1, lam, 1);
    if (s != LA2_OK) return s;
    s = run_scan(s_kv, BH, nel, p, 3, st, nullptr, 0, (int)d, (int)dv, 0, lam, (int)H);
    if (s != LA2_OK) return s;
    if (is_bwd) {  // Q^T dO of each chunk decayed to its first row, then their decayed suffix
      s = bf ? run_chunk_states<__nv_bfloat16>(q, dout, s_u, BH, N, (int)d, (int)dv, p, st, (int)H, 1, 1, lam, 2)
             : run_chunk_states<float>(q, dout, s_u, BH, N, (int)d, (int)dv, p, st, (int)H, 1, 1, lam, 2);
      if (s != LA2_OK) return s;
      s = run_scan(s_u, BH, nel, p, 4, st, nullptr, 0, (int)d, (int)dv, 0, lam, (int)H);
      if (s != LA2_OK) return s;
    }
  }
  if (!is_bwd)
    return bf ? forward_simt<__nv_bfloat16>(q, k, v, o, hd, N, (int)d, (int)dv, 1, block, s_kv, p, st, lam)
              : forward_simt<float>(q, k, v, o, hd, N, (int)d, (int)dv, 1, block, s_kv, p, st, lam);
  return bf ? backward_simt<__nv_bfloat16>(q, k, v, dout, dq, dk, dvv, hd, N, (int)d, (int)dv, 1,
                                           block, s_kv, s_u, p, st, lam)
            : backward_simt<float>(q, k, v, dout, dq, dk, dvv, hd, N, (int)d, (int)dv, 1, block,
                                   s_kv, s_u, p, st, lam);
}

}  // namespace la2

extern "C" {

size_t la2_workspace_size_decay(int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv, int block,
                                la2_dtype dt, int is_backward) {
  if (check_decay_shape(B, H, N, d, dv, block, dt, is_backward != 0) != LA2_OK) return (size_t)-1;
  if (B == 0 || H == 0 || N == 0) return 0;
  const int sms = device_sm_count();
  if (sms <= 0) return (size_t)-1;
  return plan_decay(B, H, N, d, dv, block, is_backward != 0, decay_tc(d, dv, block, dt), sms).ws_bytes;
}

la2_status la2_forward_decay(const void* q, const void* k, const void* v, void* o, const float* lambda,
                             int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv, int block,
                             la2_dtype dt, void* workspace, size_t workspace_bytes,
                             la2_stream_t stream) {
  return decay_impl(q, k, v, nullptr, o, nullptr, nullptr, nullptr, lambda, B, H, N, d, dv, block, dt,
                    workspace, workspace_bytes, stream, false);
}

la2_status la2_backward_decay(const void* q, const void* k, const void* v, const void* dout, void* dq,
                              void* dk, void* dvv, const float* lambda, int64_t B, int64_t H,
                              int64_t N, int64_t d, int64_t dv, int block, la2_dtype dt,
                              void* workspace, size_t workspace_bytes, la2_stream_t stream) {
  return decay_impl(q, k, v, dout, nullptr, dq, dk, dvv, lambda, B, H, N, d, dv, block, dt, workspace,
                    workspace_bytes, stream, true);
}

la2_status la2_backward_gqa(const void* q, const void* k, const void* v, const void* dout, void* dq,
                            void* dk, void* dvv, int64_t B, int64_t H, int64_t Hkv, int64_t N,
                            int64_t d, int64_t dv, int causal, int block, la2_dtype dt,
                            void* workspace, size_t workspace_bytes, la2_stream_t stream) {
  return backward_impl(q, k, v, dout, dq, dk, dvv, B, H, Hkv, N, d, dv, causal, block, dt, workspace,
                       workspace_bytes, stream, Ext{});
}

la2_status la2_backward_sp(const void* q, const void* k, const void* v, const void* dout, void* dq,
                           void* dk, void* dvv, const float* prefix_states, int64_t n_prefix,
                           const float* suffix_states, int64_t n_suffix, int64_t B, int64_t H,
                           int64_t N, int64_t d, int64_t dv, int block, la2_dtype dt,
                           void* workspace, size_t workspace_bytes, la2_stream_t stream) {
  Ext ext;
  ext.pre = prefix_states;
  ext.n_pre = n_prefix;
  ext.suf = suffix_states;
  ext.n_suf = n_suffix;
  ext.on = true;
  return backward_impl(q, k, v, dout, dq, dk, dvv, B, H, H, N, d, dv, 1, block, dt, workspace,
                       workspace_bytes, stream, ext);
}

la2_status la2_backward(const void* q, const void* k, const void* v, const void* dout, void* dq,
                        void* dk, void* dvv, int64_t B, int64_t H, int64_t N, int64_t d,
                        int64_t dv, int causal, int block, la2_dtype dt, void* workspace,
                        size_t workspace_bytes, la2_stream_t stream) {
  return la2_backward_gqa(q, k, v, dout, dq, dk, dvv, B, H, H, N, d, dv, causal, block, dt,
                          workspace, workspace_bytes, stream);
}

la2_status la2_check(la2_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return LA2_ERR_CUDA;
  int code = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&code, g_error_code, sizeof(int)) != cudaSuccess) return LA2_ERR_CUDA;
  if (code != 0) {
    if (cudaMemcpyToSymbol(g_error_code, &zero, sizeof(int)) != cudaSuccess) return LA2_ERR_CUDA;
    return code == DEV_ERR_TIMEOUT ? LA2_ERR_TIMEOUT : LA2_ERR_CUDA;
  }
  return LA2_OK;
}

const char* la2_status_string(la2_status s) {
  switch (s) {
    case LA2_OK: return "LA2_OK";
    case LA2_ERR_INVALID_ARG: return "LA2_ERR_INVALID_ARG: invalid argument";
    case LA2_ERR_UNSUPPORTED: return "LA2_ERR_UNSUPPORTED: unsupported dtype/shape/block";
    case LA2_ERR_WORKSPACE: return "LA2_ERR_WORKSPACE: workspace missing or too small";
    case LA2_ERR_CUDA: return "LA2_ERR_CUDA: CUDA call or launch failed";
    case LA2_ERR_TIMEOUT: return "LA2_ERR_TIMEOUT: a device-side wait gave up";
  }
  return "LA2: unknown status";
}

la2_status la2_profile_enable(int on) {
  if (on < 0 || on > 2) return LA2_ERR_INVALID_ARG;
  g_prof.on = on != 0;
  if (on == 1) g_prof.used = 0;
  return LA2_OK;
}

int la2_profile_num_kernels(void) { return K_COUNT; }

const char* la2_profile_kernel_name(int kernel) {
  return (kernel >= 0 && kernel < K_COUNT) ? kKernelNames[kernel] : nullptr;
}

la2_status la2_profile_collect(int kernel, int64_t* launches, double* total_ms) {
  if (kernel < 0 || kernel >= K_COUNT || !launches || !total_ms) return LA2_ERR_INVALID_ARG;
  int64_t n = 0;
  double ms = 0.0;
  for (size_t i = 0; i < g_prof.used; ++i) {
    EventRecord& r = g_prof.pool[i];
    if (r.kernel != kernel) continue;
    if (cudaEventSynchronize(r.stop) != cudaSuccess) return LA2_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) return LA2_ERR_CUDA;
    ms += t;
    ++n;
  }
  *launches = n;
  *total_ms = ms;
  return LA2_OK;
}

int la2_version(void) { return (0 << 16) | 1; }

#ifdef LA2_TRACE
// Copies the per-step timestamps of CTA 0 of the last traced launch (16 x 512 u64).
LA2_API int la2_trace_read(unsigned long long* dst) {
  return cudaMemcpyFromSymbol(dst, sm100::g_trace, sizeof(sm100::g_trace)) == cudaSuccess ? 0 : 1;
}
// Copies the per-CTA stamps (start, first main step, end) of the last traced launch (4 x 160 u64).
LA2_API int la2_trace_cta_read(unsigned long long* dst) {
  return cudaMemcpyFromSymbol(dst, sm100::g_trace_cta, sizeof(sm100::g_trace_cta)) == cudaSuccess ? 0 : 1;
}
#endif

}  // extern "C"

// ============================================ forward without caller workspace
//
// For callers that cannot allocate device memory when they call the op: the
// chunk states live in one array compiled into this library instead of a
// caller-provided workspace. Host code cannot use the array's name as a device
// address (it is only a host-side handle), so each device's address is looked
// up once with cudaGetSymbolAddress, with that device current.

namespace la2 {

static __device__ __align__(256) unsigned char g_noalloc_scratch[LA2_NOALLOC_SCRATCH_BYTES];

constexpr int kNoallocMaxDevices = 128;
static void* g_noalloc_ptr[kNoallocMaxDevices];
static std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device (set-up on first
// use per device), or nullptr if the lookup fails.
static void* noalloc_scratch_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace la2

extern "C" la2_status la2_forward_noalloc(const void* q, const void* k, const void* v, void* o,
                                          int64_t B, int64_t H, int64_t N, int64_t d, int64_t dv,
                                          int causal, int block, la2_dtype dt,
                                          la2_stream_t stream) {
  const size_t need = la2_workspace_size(B, H, N, d, dv, causal, block, dt, 0);
  if (need == static_cast<size_t>(-1))  // let the regular entry point name the argument error
    return la2_forward(q, k, v, o, B, H, N, d, dv, causal, block, dt, nullptr, 0, stream);
  if (need > static_cast<size_t>(LA2_NOALLOC_SCRATCH_BYTES)) return LA2_ERR_WORKSPACE;
  void* ws = nullptr;
  if (need > 0) {
    ws = noalloc_scratch_current_device();
    if (!ws) return LA2_ERR_CUDA;
  }
  return la2_forward(q, k, v, o, B, H, N, d, dv, causal, block, dt, ws,
                     static_cast<size_t>(LA2_NOALLOC_SCRATCH_BYTES), stream);
}
