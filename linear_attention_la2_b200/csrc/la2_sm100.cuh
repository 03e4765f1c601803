// Tensor-core kernels of libla2 for sm_100a: TMA-staged tiles in shared
// memory, tcgen05 MMAs with fp32 accumulators in tensor memory (TMEM), and a
// warp-specialised pipeline.
//
// Article "Lightning Attention-2 新一代注意力机制", section
// "Lightning Attention-2简介": point 1 (the left product ((QK^T)⊙M)V, the right
// product Q(K^T V) without the mask), point 2 (Fig. 3: blocks; intra-block left
// product, inter-block right product with a KV state accumulated block by
// block, the two added), point 3 (tiles moved from HBM to on-chip memory,
// computed there, the output written back).
//
// Per block i of Bk rows (one CTA owns one chunk of one (b, h) sequence):
//   S_i  = Q_i K_i^T                    tcgen05, M=Bk N=Bk K=d   -> TMEM (fp32)
//   P_i  = bf16(S_i ⊙ M_B)               mask warpgroup, TMEM -> SMEM
//   O_i  = Q_i * bf16(KV)                tcgen05, M=Bk N=dv K=d   -> TMEM (fp32)
//   KV  += K_i^T V_i                    tcgen05, M=d  N=dv K=Bk  -> TMEM (fp32 state)
//   O_i += P_i V_i                      tcgen05, M=Bk N=dv K=Bk
//   O_i  -> bf16 -> HBM                 epilogue warpgroup
// The state never leaves the SM: it is accumulated in TMEM, and a bf16 copy
// (the "snapshot") is written to SMEM each block as the B operand of Q_i*KV.
//
// Warp roles (16 warps): 0 TMA producer, 1 MMA issuer (the whole warp runs the
// loop, one elected lane issues; + TMEM allocation), 4-7 mask/convert S -> P,
// 8-11 KV snapshot, 12-15 epilogue O -> HBM (Bk=64: swizzled staging tile and
// TMA stores).
//
// Every wait is bounded (iteration count and a wall-clock deadline); on
// expiry the waiting role records LA2_ERR_TIMEOUT in the device error word,
// raises a CTA-wide abort flag, and the CTA drains its own in-flight TMA
// loads and MMAs (again bounded) before it frees TMEM and exits.
#pragma once

#include <cuda.h>

#include "la2.h"
#include "la2_common.cuh"

namespace la2 {
namespace sm100 {

// ------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}



__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_prefetch(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// 3-D tiled TMA load global -> shared, completion counted on `bar` in bytes.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 3-D tiled TMA store shared -> global; completion tracked by bulk groups of
// the issuing thread. Coordinates are never negative here (tile origins).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y,
                                             int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(map),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N committed groups still read their shared-memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until at most N committed groups are still in flight (writes done).
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// Barrier `id` (1..15) over `n` threads (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem], bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Warp-wide forms: every lane of a converged warp executes the call and one
// elected lane issues the instruction. The warp's descriptor arithmetic then
// stays warp-uniform, which keeps the issuing loop short.
__device__ __forceinline__ void mma_bf16_ss_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                 uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p, e;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]: the A operand (M rows in TMEM lanes, two
// bf16 of consecutive k per 32-bit column) is read from tensor memory.
__device__ __forceinline__ void mma_bf16_ts_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                 uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p, e;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit_warp(uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation issued so far by this thread completes.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

#define LA2_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), \
                  "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
// Thread t of the warp reads TMEM lane (lane field of taddr) + t, 32 consecutive columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : LA2_R8(0), LA2_R8(8), LA2_R8(16), LA2_R8(24)
      : "r"(taddr));
}
#undef LA2_R8
#define LA2_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), \
                  "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
          taddr),
      LA2_W8(0), LA2_W8(8), LA2_W8(16), LA2_W8(24)
      : "memory");
}
#undef LA2_W8
// Thread t writes 16 consecutive 32-bit columns of TMEM lane (lane field of taddr) + t.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t x) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(x) : "memory");
}
__device__ __forceinline__ uint16_t bf16_bits(float x) {
  const __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<const uint16_t*>(&b);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c,
                                             uint32_t& d) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr)
               : "memory");
}

// Multiplies row r of a [ROWS x 128] bf16 operand tile (two 64-column panels
// of ROWS 128-byte rows, 128B-swizzled as TMA writes them) by f, in place.
template <int ROWS>
__device__ __forceinline__ void scale_tile_row(uint32_t base, int r, float f) {
#pragma unroll
  for (int ch = 0; ch < 16; ++ch) {
    const int panel = ch >> 3, cj = ch & 7;
    const uint32_t addr = base + panel * ROWS * 128 + r * 128 + ((cj ^ (r & 7)) << 4);
    uint32_t x[4];
    ld_shared_v4(addr, x[0], x[1], x[2], x[3]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&x[e]);
      x[e] = pack_bf16x2(__low2float(h) * f, __high2float(h) * f);
    }
    st_shared_v4(addr, x[0], x[1], x[2], x[3]);
  }
}

// ------------------------------------------------------ operand descriptors
//
// Shared-memory matrix descriptor (tcgen05): start address, leading and stride
// byte offsets (all >> 4), version 1, layout SWIZZLE_128B. Every operand tile
// here is stored as 128-byte rows in 1024-byte-aligned panels with the 128B
// swizzle (16-byte chunk j of row r sits at chunk j ^ (r % 8)), which is what
// a TMA box with a 128-byte inner extent and CU_TENSOR_MAP_SWIZZLE_128B writes.
//  * K-major (rows = M or N, contiguous along K): SBO = 1024 (8-row groups),
//    LBO unused (16). The k-th 16-element slice starts 32*k bytes into the row
//    (128-byte panel p holds K elements [64p, 64p+64)).
//  * MN-major (rows = K, contiguous along M or N): SBO = 1024 (8 K-rows),
//    LBO = byte distance between 64-element M/N panels; the k-th 16-row slice
//    starts 2048*k bytes in.
__device__ __forceinline__ uint64_t make_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version for tcgen05
  d |= static_cast<uint64_t>(2) << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, dense.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                                   // D format: f32
         | (1u << 7)                                 // A format: bf16
         | (1u << 10)                                // B format: bf16
         | ((a_mn_major ? 1u : 0u) << 15)            // A major
         | ((b_mn_major ? 1u : 0u) << 16)            // B major
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// ------------------------------------------------------------ kernel config

enum Mode : int { MODE_CAUSAL = 0, MODE_NONCAUSAL = 1, MODE_STATE = 2 };

constexpr int kThreads = 512;
constexpr int kWarpProducer = 0;
constexpr int kWarpMma = 1;
constexpr int kWgMask = 1;      // warps 4-7
constexpr int kWgState = 2;     // warps 8-11
constexpr int kWgEpilogue = 3;  // warps 12-15
constexpr uint32_t kTmemCols = 512;

template <int BK, int D, int DV>
struct Cfg {
  static constexpr int QS = BK == 64 ? 3 : 1;   // Q ring depth
  static constexpr int KS = BK == 64 ? 3 : 2;   // K/V ring depth
  static constexpr int DP = D / 64;             // 128-byte panels of a d-wide row
  static constexpr int VP = DV / 64;
  static constexpr int QTILE = BK * D * 2;      // bytes
  static constexpr int KTILE = BK * D * 2;
  static constexpr int VTILE = BK * DV * 2;
  static constexpr int PTILE = BK * BK * 2;
  static constexpr int SNAP = D * DV * 2;
  // shared-memory carve-up (offsets from a 1024-aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QS * QTILE;
  static constexpr int OFF_V = OFF_K + KS * KTILE;
  static constexpr int OFF_P = OFF_V + KS * VTILE;
  static constexpr int OFF_SNAP = OFF_P + PTILE;
  // Bk=64: O leaves through two swizzled staging tiles and per-warp TMA stores.
  static constexpr bool TMA_STORE = BK == 64;
  static constexpr int OTILE = BK * DV * 2;
  static constexpr int OFF_OST = OFF_SNAP + SNAP;
  static constexpr int OFF_BAR = OFF_OST + (TMA_STORE ? 2 * OTILE : 0);
  static constexpr int NBAR = 2 * QS + 2 * KS + 20;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;  // + alignment slack
  // TMEM columns
  static constexpr uint32_t COL_KV = 0;
  static constexpr uint32_t COL_O0 = 128;
  static constexpr uint32_t COL_O1 = 256;
  static constexpr uint32_t COL_S0 = 384;
  static constexpr uint32_t COL_S1 = BK == 64 ? 448 : 384;  // one S buffer at Bk=128
  static constexpr int NSB = BK == 64 ? 2 : 1;
  // instruction descriptors
  static constexpr uint32_t ID_S = make_idesc(BK, BK, false, false);
  static constexpr uint32_t ID_QKV = make_idesc(BK, DV, false, true);
  static constexpr uint32_t ID_QKV_KMAJOR = make_idesc(BK, DV, false, false);
  static constexpr uint32_t ID_UPD = make_idesc(D, DV, true, true);
  static constexpr uint32_t ID_PV = make_idesc(BK, DV, false, true);
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

struct Params {
  __nv_bfloat16* o;           // [BH][N][DV] (forward modes)
  const float* init_states;   // [BH][C][D*DV] (state_f4): scanned prefix (causal); non-causal:
                              // slots 0..init_count-1 of the sequence, summed by the kernel
  int64_t init_count;         // non-causal: chunk states to add up (1 after a total scan)
  float* out_states;          // MODE_STATE output [BH][C][D][DV]
  int64_t N;
  int64_t L;                  // chunk length (multiple of BK)
  int64_t C;                  // chunks per sequence
  int64_t units_per_seq;      // C (forward) or the number of chunks whose state is needed
  int64_t spin_limit;
  // Grouped K/V heads: query heads per batch and query heads per K/V head.
  // Block loops (MODE_CAUSAL, MODE_NONCAUSAL) run one unit per query sequence
  // and read K, V and the initial states of its K/V sequence (kv_seq).
  // MODE_STATE runs one unit per state sequence; with state_group > 1 that is
  // a K/V sequence whose state sums the tiles of its group's state_group query
  // sequences (the K and V slots then hold Q and dO: the dK/dV pass's U).
  int32_t H, G;
  int32_t state_group;
  // MODE_CAUSAL: every chunk, the first included, starts from its slot of
  // init_states (a sequence part whose earlier parts are summarised there).
  int32_t init_all;
  // Decayed form (kernels built with DEC): one rate per query head, lam[bh % H].
  const float* lam;
  // DEC, MODE_CAUSAL: init_states hold the sequence's raw chunk states (each
  // decayed to its chunk's last row, no scan ran); chunk c adds the first c of
  // them, state c' weighted by lam^(L (c-1-c')).
  int32_t decay_sum;
};

// Shared state of one CTA.
struct Bars {
  uint64_t* q_full;
  uint64_t* q_empty;
  uint64_t* kv_full;
  uint64_t* kv_empty;
  uint64_t* s_full;      // [2]
  uint64_t* s_empty;     // [2]
  uint64_t* p_full;
  uint64_t* p_empty;
  uint64_t* snap_full;
  uint64_t* kv_updated;
  uint64_t* o_full;      // [2]
  uint64_t* o_empty;     // [2]
  uint64_t* drain;
  uint64_t* qk_ready;    // decayed form: Q and K rows of the block scaled
  uint64_t* k_scaled;    // [2] decayed chunk state: K rows of block i scaled (slot i % 2)
  uint64_t* k_free;      // [2] ... and the update that read them done
  uint32_t* tmem_base;
  volatile int* abort_flag;
};

// Bounded wait. Returns false (after recording a timeout and raising the
// CTA abort flag) when the limit is reached or another role aborted. The
// common case - the phase has already completed - stays inline; the spin loop
// and its timeout bookkeeping live out of line to keep every role's hot loop
// small in the instruction cache.
__device__ __noinline__ bool wait_bar_slow(uint64_t* bar, uint32_t parity, int64_t limit,
                                           volatile int* abort_flag, int where) {
  int64_t n = 0;
  uint64_t deadline = 0;
  while (!mbar_try_wait(bar, parity)) {
    ++n;
    bool expired = n >= limit;
    if ((n & 63) == 0) {
      if (*abort_flag) return false;
      const uint64_t now = globaltimer_ns();
      if (deadline == 0) deadline = now + 20ull * 1000ull * 1000ull * 1000ull;  // 20 s
      expired = expired || now > deadline;
    }
    if (expired) {
      record_error(DEV_ERR_TIMEOUT, where);
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, int64_t limit,
                                         volatile int* abort_flag, int where) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_bar_slow(bar, parity, limit, abort_flag, where);
}

// Drain wait used after an abort: bounded by a fixed budget, never records.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t deadline = globaltimer_ns() + 2ull * 1000ull * 1000ull * 1000ull;  // 2 s
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() > deadline) return;
  }
}

// A fp32 state (D x DV) in HBM is stored column-chunk-major: float4 j
// (columns 4j..4j+3) of row r at float4 index j*D + r. The 32 threads of a
// warp own 32 consecutive rows of a TMEM accumulator, so each of their
// 16-byte accesses covers 512 contiguous bytes.
template <int D>
__device__ __forceinline__ int64_t state_f4(int r, int j) {
  return static_cast<int64_t>(j) * D + r;
}

// Row of an M-row accumulator held by thread `t` of warpgroup-warp `w4`
// (tcgen05.ld 32x32b), or -1. M=128: lane = row. M=64: rows 16w..16w+15
// live in lanes 32w..32w+15 of the warp's TMEM sub-partition.
template <int M>
__device__ __forceinline__ int acc_row(int w4, int t) {
  if (M == 128) return 32 * w4 + t;
  return t < 16 ? 16 * w4 + t : -1;
}

// ------------------------------------------------------------------- kernel

// DQ = true turns the block loop into the dQ pass of the backward
// (d = dv): the Q, K, V slots hold dO, V, K, so S = dO V^T, the masked
// product P K gives the intra-block part of dQ, the state update is
// KV += K^T V from the swapped slots, and the inter-block part is dO KV^T
// (the bf16 snapshot read K-major).
// DEC = true (MODE_STATE, MODE_CAUSAL forward) is the decayed form with rate
// lam = prm.lam[bh % H]: KV_t = lam KV_{t-1} + k_t^T v_t. MODE_STATE scales the
// K rows of its chunk by lam^(t1-1-s) (the chunk's state decayed to its last
// row), one block ahead of the update MMA (k_scaled / k_free, two slots). MODE_CAUSAL keeps KV decayed to the row before the block and, per block:
// once S has read Q and K unscaled, the mask warpgroup scales, in shared
// memory, Q's rows by lam^(t+1) and K's by lam^(Bk-1-j) (qk_ready), then weights
// S by lam^(t-j) into P; the MMA warp issues Q KV and the update on qk_ready,
// while P is made, and P V on p_full; the state warpgroup writes lam^Bk KV back
// to TMEM beside each snapshot, so the update adds onto the decayed state.
template <int BK, int D, int DV, int MODE, bool DQ = false, bool DEC = false>
__global__ void __launch_bounds__(kThreads, 1)
la2_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_o, const Params prm) {
  using CF = Cfg<BK, D, DV>;
  static_assert(!DEC || (!DQ && MODE != MODE_NONCAUSAL), "decayed form: forward, causal");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int wg = warp >> 2;   // warpgroup
  const int w4 = warp & 3;    // TMEM sub-partition of this warp

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + CF::OFF_BAR);
  Bars b;
  b.q_full = bars;
  b.q_empty = b.q_full + CF::QS;
  b.kv_full = b.q_empty + CF::QS;
  b.kv_empty = b.kv_full + CF::KS;
  b.s_full = b.kv_empty + CF::KS;
  b.s_empty = b.s_full + 2;
  b.p_full = b.s_empty + 2;
  b.p_empty = b.p_full + 1;
  b.snap_full = b.p_empty + 1;
  b.kv_updated = b.snap_full + 1;
  b.o_full = b.kv_updated + 1;
  b.o_empty = b.o_full + 2;
  b.drain = b.o_empty + 2;
  b.qk_ready = b.drain + 1;
  b.k_scaled = b.qk_ready + 1;
  b.k_free = b.k_scaled + 2;
  b.tmem_base = reinterpret_cast<uint32_t*>(b.k_free + 2);
  b.abort_flag = reinterpret_cast<volatile int*>(b.tmem_base + 1);

  // ---- unit of work
  const int64_t unit = blockIdx.x;
  const int64_t bh = unit / prm.units_per_seq;
  const int64_t c = unit % prm.units_per_seq;
  const int64_t t0 = c * prm.L;
  const int64_t t1 = min(prm.N, t0 + prm.L);
  const int nblk = static_cast<int>((t1 - t0 + BK - 1) / BK);
  // K/V sequence of this unit's loads (a state unit is its own sequence)
  const int64_t bkv = MODE == MODE_STATE ? bh : kv_seq(bh, prm.H, prm.G);
  const int sgroup = (MODE == MODE_STATE && prm.state_group > 1) ? prm.state_group : 1;
  const int nsteps = MODE == MODE_STATE ? nblk * sgroup : nblk;
  const bool has_init = (MODE == MODE_NONCAUSAL) ||
                        (MODE == MODE_CAUSAL && prm.init_states && (c > 0 || prm.init_all));
  const float* init = nullptr;
  if (MODE == MODE_NONCAUSAL) init = prm.init_states + bkv * prm.C * (int64_t)(D * DV);
  else if (DEC && prm.decay_sum && has_init) init = prm.init_states + bkv * prm.C * (int64_t)(D * DV);
  else if (has_init) init = prm.init_states + (bkv * prm.C + c) * (int64_t)(D * DV);

  // ---- setup
  if (threadIdx.x == 0) {
    for (int s = 0; s < CF::QS; ++s) { mbar_init(&b.q_full[s], 1); mbar_init(&b.q_empty[s], 1); }
    for (int s = 0; s < CF::KS; ++s) { mbar_init(&b.kv_full[s], 1); mbar_init(&b.kv_empty[s], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&b.s_full[s], 1);
      mbar_init(&b.s_empty[s], 128);
      mbar_init(&b.o_full[s], 1);
      mbar_init(&b.o_empty[s], 128);
    }
    mbar_init(b.p_full, 128);
    mbar_init(b.p_empty, 1);
    mbar_init(b.snap_full, 128);
    mbar_init(b.kv_updated, 1);
    mbar_init(b.drain, 1);
    mbar_init(b.qk_ready, 128);
    for (int s = 0; s < 2; ++s) { mbar_init(&b.k_scaled[s], 128); mbar_init(&b.k_free[s], 1); }
    *b.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kWarpProducer && lane == 0) {
    tma_prefetch(&tm_q);
    tma_prefetch(&tm_k);
    tma_prefetch(&tm_v);
    if (MODE != MODE_STATE && CF::TMA_STORE) tma_prefetch(&tm_o);
  }
  if (warp == kWarpMma) {
    tmem_alloc(b.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *b.tmem_base;
  const int64_t lim = prm.spin_limit;
  pdl_launch_dependents();  // global memory is touched only after this point
  pdl_wait();

  uint8_t* sQ = smem + CF::OFF_Q;
  uint8_t* sK = smem + CF::OFF_K;
  uint8_t* sV = smem + CF::OFF_V;
  uint8_t* sP = smem + CF::OFF_P;
  uint8_t* sSnap = smem + CF::OFF_SNAP;

  if (warp == kWarpProducer) {
    // ================================================================ TMA
    if (lane == 0) {
      int issued_kv = 0, issued_q = 0;
      bool ok = true;
      for (int i = 0; i < nsteps && ok; ++i) {
        // a state unit of a group walks the blocks of each query sequence in turn
        const int blk = MODE == MODE_STATE ? i % nblk : i;
        const int zkv = MODE == MODE_STATE && sgroup > 1
                            ? static_cast<int>(q_seq0(bh, prm.H, prm.G) + i / nblk)
                            : static_cast<int>(bkv);
        const int row = static_cast<int>(t0 + static_cast<int64_t>(blk) * BK);
        if (MODE != MODE_NONCAUSAL) {
          const int s = i % CF::KS;
          if (!wait_bar(&b.kv_empty[s], ((i / CF::KS) & 1) ^ 1, lim, b.abort_flag, 1)) { ok = false; break; }
          mbar_expect_tx(&b.kv_full[s], CF::KTILE + CF::VTILE);
          for (int p = 0; p < CF::DP; ++p)
            tma_load_3d(sK + s * CF::KTILE + p * BK * 128, &tm_k, &b.kv_full[s], 64 * p, row, zkv);
          for (int p = 0; p < CF::VP; ++p)
            tma_load_3d(sV + s * CF::VTILE + p * BK * 128, &tm_v, &b.kv_full[s], 64 * p, row, zkv);
          ++issued_kv;
        }
        if (MODE != MODE_STATE) {
          const int s = i % CF::QS;
          if (!wait_bar(&b.q_empty[s], ((i / CF::QS) & 1) ^ 1, lim, b.abort_flag, 2)) { ok = false; break; }
          mbar_expect_tx(&b.q_full[s], CF::QTILE);
          for (int p = 0; p < CF::DP; ++p)
            tma_load_3d(sQ + s * CF::QTILE + p * BK * 128, &tm_q, &b.q_full[s], 64 * p, row, (int)bh);
          ++issued_q;
        }
      }
      if (!ok) {
        // Let every load this thread issued land before the CTA exits.
        for (int j = max(0, issued_kv - CF::KS); j < issued_kv; ++j)
          drain_wait(&b.kv_full[j % CF::KS], (j / CF::KS) & 1);
        for (int j = max(0, issued_q - CF::QS); j < issued_q; ++j)
          drain_wait(&b.q_full[j % CF::QS], (j / CF::QS) & 1);
      }
    }
  } else if (warp == kWarpMma) {
    // ================================================================ MMA
    // The whole warp runs the issue loop; one elected lane issues each
    // tcgen05 instruction (warp-uniform bookkeeping).
    {
      auto wait_w = [&](uint64_t* bar, uint32_t par, int where) -> bool {
        return __all_sync(0xffffffffu, wait_bar(bar, par, lim, b.abort_flag, where));
      };
      const uint32_t tKV = tmem + CF::COL_KV;
      int snap_ph = 0;
      bool ok = true;
      for (int i = 0; i < nsteps && ok; ++i) {
        const int qs = i % CF::QS, ks = i % CF::KS;
        const uint32_t qa = smem_u32(sQ + qs * CF::QTILE);
        const uint32_t ka = smem_u32(sK + ks * CF::KTILE);
        const uint32_t va = smem_u32(sV + ks * CF::VTILE);
        if constexpr (MODE == MODE_STATE) {
          if (!wait_w(&b.kv_full[ks], (i / CF::KS) & 1, 10)) { ok = false; break; }
          if (DEC && !wait_w(&b.k_scaled[i & 1], (i >> 1) & 1, 17)) { ok = false; break; }  // K rows scaled
          tc_fence_after();
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16_ss_warp(tKV, make_desc(ka + kk * 2048, BK * 128, 1024),
                        make_desc(va + kk * 2048, BK * 128, 1024), CF::ID_UPD, (i > 0 || kk > 0));
          if (DEC) mma_commit_warp(&b.k_free[i & 1]);
          mma_commit_warp(&b.kv_empty[ks]);
          continue;
        }
        if (!wait_w(&b.q_full[qs], (i / CF::QS) & 1, 11)) { ok = false; break; }
        if (MODE == MODE_CAUSAL &&
            !wait_w(&b.kv_full[ks], (i / CF::KS) & 1, 12)) { ok = false; break; }
        tc_fence_after();
        const int sb = CF::NSB == 2 ? (i & 1) : 0;
        const int s_use = CF::NSB == 2 ? (i >> 1) : i;
        const uint32_t tS = tmem + (sb ? CF::COL_S1 : CF::COL_S0);
        if (MODE == MODE_CAUSAL) {
          // S_i = Q_i K_i^T
          if (!wait_w(&b.s_empty[sb], (s_use & 1) ^ 1, 13)) { ok = false; break; }
          tc_fence_after();
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * BK * 128 + (kk & 3) * 32;
            mma_bf16_ss_warp(tS, make_desc(qa + off, 16, 1024), make_desc(ka + off, 16, 1024), CF::ID_S,
                        kk > 0);
          }
          mma_commit_warp(&b.s_full[sb]);
        }
        // Decayed form: the scaled Q and K rows before Q KV and the update
        if (DEC && !wait_w(b.qk_ready, i & 1, 18)) { ok = false; break; }
        // O_i = Q_i * bf16(KV)
        const int ob = i & 1;
        const uint32_t tO = tmem + (ob ? CF::COL_O1 : CF::COL_O0);
        if (!wait_w(&b.o_empty[ob], ((i >> 1) & 1) ^ 1, 14)) { ok = false; break; }
        const bool have_snap = (i > 0) || has_init;
        if (have_snap && (MODE == MODE_CAUSAL || i == 0)) {
          if (!wait_w(b.snap_full, snap_ph, 15)) { ok = false; break; }
          snap_ph ^= 1;
        }
        tc_fence_after();
        if (have_snap) {
          const uint32_t sa = smem_u32(sSnap);
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * BK * 128 + (kk & 3) * 32;
            if constexpr (DQ)  // B[n=c][k=e] = KV[c][e]: snapshot rows read K-major
              mma_bf16_ss_warp(tO, make_desc(qa + off, 16, 1024),
                          make_desc(sa + (kk >> 2) * D * 128 + (kk & 3) * 32, 16, 1024),
                          CF::ID_QKV_KMAJOR, kk > 0);
            else
              mma_bf16_ss_warp(tO, make_desc(qa + off, 16, 1024), make_desc(sa + kk * 2048, D * 128, 1024),
                          CF::ID_QKV, kk > 0);
          }
        }
        mma_commit_warp(&b.q_empty[qs]);
        if constexpr (MODE == MODE_NONCAUSAL) {
          mma_commit_warp(&b.o_full[ob]);
          continue;
        }
        // KV += K_i^T V_i (after the snapshot of the old state was taken)
        for (int kk = 0; kk < BK / 16; ++kk)
          mma_bf16_ss_warp(tKV, make_desc((DQ ? va : ka) + kk * 2048, BK * 128, 1024),
                      make_desc((DQ ? ka : va) + kk * 2048, BK * 128, 1024), CF::ID_UPD,
                      (have_snap || kk > 0) ? 1u : 0u);
        mma_commit_warp(b.kv_updated);
        // O_i += P_i V_i
        if (!wait_w(b.p_full, i & 1, 16)) { ok = false; break; }
        tc_fence_after();
        const uint32_t pa = smem_u32(sP);
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint32_t off = (kk >> 2) * BK * 128 + (kk & 3) * 32;
          mma_bf16_ss_warp(tO, make_desc(pa + off, 16, 1024), make_desc(va + kk * 2048, BK * 128, 1024),
                      CF::ID_PV, (have_snap || kk > 0) ? 1u : 0u);
        }
        mma_commit_warp(&b.o_full[ob]);
        mma_commit_warp(b.p_empty);
        mma_commit_warp(&b.kv_empty[ks]);
      }
      if (MODE == MODE_STATE && ok) mma_commit_warp(b.kv_updated);
      // All MMAs issued by this thread must finish before TMEM is released.
      mma_commit_warp(b.drain);
      drain_wait(b.drain, 0);
    }
  } else if (wg == kWgMask) {
    // ================================================ mask + convert S -> P
    const float lam = DEC ? prm.lam[bh % prm.H] : 1.f;
    if (DEC && MODE == MODE_STATE) {
      // Scale row r of each K tile by lam^(t1-1-s), s its row in the sequence.
      // Two hand-off slots: block i+1's rows are scaled while the update of
      // block i runs (a slot is reused once the update two blocks back is done).
      const int r = threadIdx.x % 128;
      for (int i = 0; i < nblk; ++i) {
        const int ks = i % CF::KS;
        if (!__all_sync(0xffffffffu, wait_bar(&b.kv_full[ks], (i / CF::KS) & 1, lim, b.abort_flag, 22))) break;
        if (!__all_sync(0xffffffffu, wait_bar(&b.k_free[i & 1], ((i >> 1) & 1) ^ 1, lim, b.abort_flag, 23))) break;
        if (r < BK) {
          const int64_t srow = t0 + static_cast<int64_t>(i) * BK + r;
          const int64_t e = t1 - 1 - srow;  // rows past the chunk end are zero (past N)
          scale_tile_row<BK>(smem_u32(sK + ks * CF::KTILE), r, e >= 0 ? powf(lam, static_cast<float>(e)) : 0.f);
        }
        fence_proxy_async();
        mbar_arrive(&b.k_scaled[i & 1]);
      }
    }
    if (MODE == MODE_CAUSAL) {
      const int t = lane;
      const int r = acc_row<BK>(w4, t);
      const uint32_t lane_off = static_cast<uint32_t>(32 * w4) << 16;
      const uint32_t pbase = smem_u32(sP);
      for (int i = 0; i < nblk; ++i) {
        const int sb = CF::NSB == 2 ? (i & 1) : 0;
        const int s_use = CF::NSB == 2 ? (i >> 1) : i;
        const uint32_t tS = tmem + (sb ? CF::COL_S1 : CF::COL_S0) + lane_off;
        if (!__all_sync(0xffffffffu, wait_bar(&b.s_full[sb], s_use & 1, lim, b.abort_flag, 20))) break;
        if constexpr (DEC) {
          // S(i) has completed (s_full): its Q and K tiles can take their
          // scales now, ahead of P (which waits for P V of the block before)
          if (r >= 0) {
            scale_tile_row<BK>(smem_u32(sQ + (i % CF::QS) * CF::QTILE), r, powf(lam, static_cast<float>(r + 1)));
            scale_tile_row<BK>(smem_u32(sK + (i % CF::KS) * CF::KTILE), r,
                               powf(lam, static_cast<float>(BK - 1 - r)));
          }
          fence_proxy_async();
          mbar_arrive(b.qk_ready);
        }
        if (!__all_sync(0xffffffffu, wait_bar(b.p_empty, (i & 1) ^ 1, lim, b.abort_flag, 21))) break;
        tc_fence_after();
#pragma unroll
        for (int c32 = 0; c32 < BK / 32; ++c32) {
          uint32_t v[32];
          tmem_ld32(tS + c32 * 32, v);
          tmem_ld_wait();
          if (r >= 0) {
            if constexpr (DEC) {
              // D_B: column col gets lam^(r - col); walk down from the last
              // kept column of this chunk, multiplying by lam (no division)
              const int c0 = c32 * 32, hi = min(r, c0 + 31);
              float wgt = hi >= c0 ? powf(lam, static_cast<float>(r - hi)) : 0.f;
#pragma unroll
              for (int jj = 31; jj >= 0; --jj) {
                if (c0 + jj <= hi) {
                  v[jj] = __float_as_uint(__uint_as_float(v[jj]) * wgt);
                  wgt *= lam;
                }
              }
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {  // 16-byte chunks (8 columns) of row r
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
              const uint32_t addr = pbase + panel * BK * 128 + r * 128 + ((cj ^ (r & 7)) << 4);
              st_shared_v4(addr, w[0], w[1], w[2], w[3]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&b.s_empty[sb]);
        fence_proxy_async();
        mbar_arrive(b.p_full);
      }
    }
  } else if (wg == kWgState) {
    // ============================================ KV state snapshot (bf16)
    const int t = lane;
    const int r = acc_row<D>(w4, t);  // state row c
    const uint32_t lane_off = static_cast<uint32_t>(32 * w4) << 16;
    const uint32_t tKV = tmem + CF::COL_KV + lane_off;
    const uint32_t sbase = smem_u32(sSnap);
    auto write_snap_row = [&](const float* vals, int col0) {
      // 32 fp32 values of row r, columns col0..col0+31 -> 4 swizzled 16B chunks
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int col = col0 + q4 * 8;
        const int panel = col >> 6, cj = (col & 63) >> 3;
        const uint32_t addr = sbase + panel * D * 128 + r * 128 + ((cj ^ (r & 7)) << 4);
        st_shared_v4(addr, pack_bf16x2(vals[q4 * 8 + 0], vals[q4 * 8 + 1]),
                     pack_bf16x2(vals[q4 * 8 + 2], vals[q4 * 8 + 3]),
                     pack_bf16x2(vals[q4 * 8 + 4], vals[q4 * 8 + 5]),
                     pack_bf16x2(vals[q4 * 8 + 6], vals[q4 * 8 + 7]));
      }
    };
    // Decayed form: the state the next update adds onto is lam^Bk times the one
    // the snapshot shows (every block of a chunk but its last has Bk rows).
    const float decay_bk = DEC ? powf(prm.lam[bh % prm.H], static_cast<float>(BK)) : 1.f;
    if (MODE == MODE_STATE) {
      // Chunk state out: TMEM (fp32) -> HBM, column-chunk-major (state_f4).
      if (__all_sync(0xffffffffu, wait_bar(b.kv_updated, 0, lim, b.abort_flag, 30))) {
        tc_fence_after();
        float* dst = prm.out_states + (bh * prm.C + c) * (int64_t)(D * DV);
#pragma unroll
        for (int c32 = 0; c32 < DV / 32; ++c32) {
          uint32_t v[32];
          tmem_ld32(tKV + c32 * 32, v);
          tmem_ld_wait();
          if (r >= 0) {
            float4* p4 = reinterpret_cast<float4*>(dst);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              p4[state_f4<D>(r, c32 * 8 + q4)] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                   __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
          }
        }
      }
    } else {
      if (has_init) {
        // Initial state (prefix or total) from HBM: into TMEM (causal) and the snapshot.
#pragma unroll
        for (int c32 = 0; c32 < DV / 32; ++c32) {
          float vals[32];
          uint32_t u[32];
          if (r >= 0) {
            // Non-causal: the total is the sum of the sequence's first
            // init_count chunk states, added here in chunk order (a few chunk
            // states: no separate scan launch; many: scanned into slot 0).
            const bool dsum = DEC && prm.decay_sum;
            const int64_t nsum = MODE == MODE_NONCAUSAL ? prm.init_count : (dsum ? c : 1);
#pragma unroll
            for (int j = 0; j < 32; ++j) vals[j] = 0.f;
            for (int64_t cc = 0; cc < nsum; ++cc) {
              const float4* src = reinterpret_cast<const float4*>(init + cc * (int64_t)(D * DV));
              const float wc = dsum ? powf(prm.lam[bh % prm.H], static_cast<float>(prm.L * (c - 1 - cc))) : 1.f;
#pragma unroll
              for (int q4 = 0; q4 < 8; ++q4) {
                const float4 x = src[state_f4<D>(r, c32 * 8 + q4)];
                vals[4 * q4] = fmaf(wc, x.x, vals[4 * q4]);
                vals[4 * q4 + 1] = fmaf(wc, x.y, vals[4 * q4 + 1]);
                vals[4 * q4 + 2] = fmaf(wc, x.z, vals[4 * q4 + 2]);
                vals[4 * q4 + 3] = fmaf(wc, x.w, vals[4 * q4 + 3]);
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) vals[j] = 0.f;
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(DEC ? decay_bk * vals[j] : vals[j]);
          if (MODE == MODE_CAUSAL) tmem_st32(tKV + c32 * 32, u);
          if (r >= 0) write_snap_row(vals, c32 * 32);
        }
        if (MODE == MODE_CAUSAL) tmem_st_wait();
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(b.snap_full);
      }
      if (MODE == MODE_CAUSAL) {
        for (int i = 0; i + 1 < nblk; ++i) {
          if (!__all_sync(0xffffffffu, wait_bar(b.kv_updated, i & 1, lim, b.abort_flag, 31))) break;
          tc_fence_after();
#pragma unroll
          for (int c32 = 0; c32 < DV / 32; ++c32) {
            uint32_t v[32];
            tmem_ld32(tKV + c32 * 32, v);
            tmem_ld_wait();
            if (r >= 0) {
              float vals[32];
#pragma unroll
              for (int j = 0; j < 32; ++j) vals[j] = __uint_as_float(v[j]);
              write_snap_row(vals, c32 * 32);
            }
            if constexpr (DEC) {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(decay_bk * __uint_as_float(v[j]));
              tmem_st32(tKV + c32 * 32, v);
            }
          }
          if (DEC) tmem_st_wait();
          fence_proxy_async();
          tc_fence_before();
          mbar_arrive(b.snap_full);
        }
      }
    }
  } else if (wg == kWgEpilogue) {
    // ========================================== O: TMEM -> bf16 -> HBM
    if (MODE != MODE_STATE) {
      const int t = lane;
      const int r = acc_row<BK>(w4, t);
      const uint32_t lane_off = static_cast<uint32_t>(32 * w4) << 16;
      __nv_bfloat16* ob = prm.o + bh * prm.N * DV;
      for (int i = 0; i < nblk; ++i) {
        const int buf = i & 1;
        const uint32_t tO = tmem + (buf ? CF::COL_O1 : CF::COL_O0) + lane_off;
        if (!__all_sync(0xffffffffu, wait_bar(&b.o_full[buf], (i >> 1) & 1, lim, b.abort_flag, 40))) break;
        tc_fence_after();
        if constexpr (CF::TMA_STORE) {
          // Warp w4 stages its 16 rows (128B-swizzled 64-column panels) and
          // stores them with TMA; rows past the chunk end are not written.
          uint8_t* stage = smem + CF::OFF_OST + buf * CF::OTILE + w4 * 16 * 128;
          if (lane == 0) bulk_wait_group_read<1>();  // this warp's store of block i-2 has read it
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
          mbar_arrive(&b.o_empty[buf]);
          fence_proxy_async();
          __syncwarp();
          const int64_t y = t0 + static_cast<int64_t>(i) * BK + 16 * w4;
          // A chunk ends on a block boundary or at N, so the tensor map's
          // bound at N is the only clip needed.
          if (lane == 0) {
            if (y < t1) {
#pragma unroll
              for (int p = 0; p < DV / 64; ++p)
                tma_store_3d(&tm_o, stage + p * BK * 128, 64 * p, static_cast<int>(y),
                             static_cast<int>(bh));
            }
            bulk_commit_group();  // one group per block (empty past the end): see the wait above
          }
          continue;
        }
        const int64_t row = t0 + static_cast<int64_t>(i) * BK + r;
        const bool valid = r >= 0 && row < t1;
        uint4* dst = reinterpret_cast<uint4*>(ob + (valid ? row : 0) * DV);
#pragma unroll
        for (int c32 = 0; c32 < DV / 32; ++c32) {
          uint32_t v[32];
          tmem_ld32(tO + c32 * 32, v);
          tmem_ld_wait();
          if (valid) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[c32 * 4 + q] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                                            pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                                            pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                                            pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
          }
        }
        tc_fence_before();
        mbar_arrive(&b.o_empty[buf]);
      }
      if (CF::TMA_STORE && lane == 0) bulk_wait_group<0>();  // stores done before exit
    }
  }

  // ---- teardown: every role has left its loop; free TMEM.
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace sm100

// --------------------------------------------------------------- host side

inline bool sm100_supports(int64_t d, int64_t dv, int block, bool is_bwd) {
  (void)is_bwd;
  return d == 128 && dv == 128 && (block == 64 || block == 128);
}

// Raises a kernel's dynamic shared-memory limit once per device (the
// attribute is per function and per device context). `done` must be a
// per-kernel flag array: every launcher below passes its own static one.
template <typename Kernel>
inline bool smem_attribute_set(Kernel kern, int bytes, bool (&done)[128]) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev >= 0 && dev < 128 && done[dev]) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  if (dev >= 0 && dev < 128) done[dev] = true;
  return true;
}

using PFN_encodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                     const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                     const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline PFN_encodeTiled get_encode_fn() {
  static PFN_encodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  }
  return fn;
}

// [BH][N][W] bf16 tensor, boxes of 64 columns (128 B) x `box_rows` rows, 128B swizzle.
inline bool make_tmap_3d(CUtensorMap* m, const void* base, int64_t BH, int64_t N, int W,
                         int box_rows) {
  PFN_encodeTiled enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(W), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(W) * 2,
                                 static_cast<cuuint64_t>(N) * W * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BK, int D, int DV, int MODE, bool DQ = false, bool DEC = false>
inline la2_status launch_fwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk,
                                   const CUtensorMap& tv, const CUtensorMap& to,
                                   const sm100::Params& p, int64_t units, cudaStream_t st) {
  using CF = sm100::Cfg<BK, D, DV>;
  auto kern = sm100::la2_fwd_sm100_kernel<BK, D, DV, MODE, DQ, DEC>;
  static bool attr_done[128];  // one per template instantiation
  if (!smem_attribute_set(kern, CF::SMEM, attr_done)) return LA2_ERR_CUDA;
  if (launch_pdl(kern, dim3(static_cast<unsigned>(units)), dim3(sm100::kThreads), CF::SMEM, st, tq,
                 tk, tv, to, p) != cudaSuccess)
    return LA2_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? LA2_OK : LA2_ERR_CUDA;
}

}  // namespace la2
