// dK / dV pass of the backward on sm_100a (tcgen05 + TMEM + TMA).
//
// Gradients of L = <dO, O> for O = ((Q K^T) ⊙ M) V (article "Lightning
// Attention-2 新一代注意力机制", section "Lightning Attention-2简介", point 1;
// the article names its backward algorithm without printing it). Split along
// the blocks of point 2, with U = sum over later blocks l of Q_l^T dO_l
// (d x dv, fp32, kept in TMEM) walking the blocks of a chunk in reverse:
//   S^T = K_i Q_i^T,  A^T = V_i dO_i^T            (masked: query t >= key j)
//   dV_i = K_i U + (S^T ⊙ M)  dO_i
//   dK_i = V_i U^T + (A^T ⊙ M) Q_i
//   U   += Q_i^T dO_i                             (after U was read for block i)
// Non-causal: dV_i = K_i U, dK_i = V_i U^T with U = Q^T dO over the sequence.
//
// One CTA per (b, h, chunk); 512 threads: warp 0 TMA, warp 1 MMA issuer
// (+ TMEM), warps 4-7 mask S^T, A^T -> bf16 P^T, Pd^T (SMEM), warps 8-11 the
// bf16 snapshot of U, warps 12-15 dK, dV -> HBM. A^T lives in the columns of
// the dK accumulator until the mask warpgroup has read it (Bk=128).
//
// Grouped K/V heads (G query heads per K/V head): a K/V head's dK and dV add
// up over its query heads h, and so do their suffix states: with
// U = sum_h sum_{l>i} Q_{h,l}^T dO_{h,l} one state serves the whole group,
//   dV_i = K_i U + sum_h (S_h^T ⊙ M) dO_{h,i},  dK_i = V_i U^T + sum_h (A_h^T ⊙ M) Q_{h,i},
//   U   += sum_h Q_{h,i}^T dO_{h,i}.
// The CTA then runs G steps per block (causal), one per query head, loading
// (Q_h, K, V, dO_h) each time; dK and dV leave once per block. G > 1 needs
// A^T in its own columns (Bk=64 tiles).
#pragma once

#include "la2_sm100.cuh"

namespace la2 {
namespace sm100 {

template <int BK, int D, int DV>
struct BCfg {
  static_assert(D == 128 && DV == 128, "tensor-core backward: d = dv = 128");
  static constexpr int NS = BK == 64 ? 2 : 1;  // stages of (Q, K, V, dO)
  static constexpr int TILE = BK * 128 * 2;    // one [BK x 128] bf16 tile
  static constexpr int STAGE = 4 * TILE;
  static constexpr int PTILE = BK * BK * 2;
  static constexpr int SNAP = D * DV * 2;
  static constexpr int OFF_ST = 0;
  static constexpr int OFF_PT = OFF_ST + NS * STAGE;
  static constexpr int OFF_PDT = OFF_PT + PTILE;
  static constexpr int OFF_SNAP = OFF_PDT + PTILE;
  // Bk=64: dV and dK leave through one swizzled staging tile each and
  // per-warp TMA stores.
  static constexpr bool TMA_STORE = BK == 64;
  static constexpr int OFF_OST = OFF_SNAP + SNAP;
  static constexpr int OFF_BAR = OFF_OST + (TMA_STORE ? 2 * TILE : 0);
  static constexpr int NBAR = 2 * NS + 13;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  // Bk=64: dV and dK are accumulated transposed, dV^T = U^T K^T + dO^T P and
  // dK^T = U V^T + Q^T Pd (M = dv = d = 128 rows of the tensor datapath instead of
  // M = Bk = 64: four of the block's products at full rate); the epilogue
  // transposes while staging each tile for one TMA store.
  static constexpr bool OT = BK == 64;
  // TMEM columns: U, dV, dK, S^T, A^T
  static constexpr uint32_t COL_U = 0;
  static constexpr uint32_t G_COLS = OT ? BK : 128;  // columns of one dV or dK accumulator
  static constexpr uint32_t COL_DV = 128, COL_DK = COL_DV + G_COLS, COL_ST = COL_DK + G_COLS;
  // Bk=64: A^T gets its own columns, so the next block's S^T and A^T need
  // not wait for the epilogue to read dK; Bk=128: A^T aliases dK.
  static constexpr bool AT_OWN = BK == 64;
  static constexpr uint32_t COL_AT = AT_OWN ? COL_ST + BK : COL_DK;
  static_assert(COL_ST + BK + (AT_OWN ? BK : 0) <= 512, "TMEM columns");
  static constexpr uint32_t ID_ST = make_idesc(BK, BK, false, false);   // K Q^T, V dO^T
  static constexpr uint32_t ID_MN = make_idesc(BK, 128, false, true);   // X[K-major] * Y[MN-major]
  static constexpr uint32_t ID_KM = make_idesc(BK, 128, false, false);  // X[K-major] * Y[K-major]
  static constexpr uint32_t ID_UPD = make_idesc(D, DV, true, true);     // Q^T dO
  static constexpr uint32_t ID_T_MK = make_idesc(128, BK, true, false);   // X[MN-major] * Y[K-major]
  static constexpr uint32_t ID_T_KK = make_idesc(128, BK, false, false);  // X[K-major] * Y[K-major]
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

struct BwdParams {
  __nv_bfloat16* dk;       // [BHkv][N][D]
  __nv_bfloat16* dv;       // [BHkv][N][DV]
  const float* init_u;     // [BHkv][C][D*DV] (state_f4 layout): suffix (causal) or total in slot 0
  int64_t N, L, C;
  int64_t spin_limit;
  int causal;
  int32_t H, G;            // query heads per batch; query heads per K/V head (q_seq0)
  int32_t init_all;        // causal: the last chunk too starts from its slot of init_u
  // 1: init_u holds the raw chunk states (no scan ran); a chunk adds up the
  // states of the later chunks of its sequence (causal) or all of them.
  int32_t sum_states;
  // Causal, C = 2: chunk 0 is rows [0, split), chunk 1 rows [split, N), and
  // chunk 0 builds U itself by a pre-pass over the blocks of chunk 1 (U +=
  // Q^T dO, Q and dO loads only) before its own blocks: no suffix states are
  // read (init_u unused). 0: chunks of L rows, U from init_u.
  int64_t split;
};

template <int BK, int D, int DV>
__global__ void __launch_bounds__(kThreads, 1)
la2_bwd_dkdv_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_do,
                          const __grid_constant__ CUtensorMap tm_dk,
                          const __grid_constant__ CUtensorMap tm_dv, const BwdParams prm) {
  using CF = BCfg<BK, D, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, wg = warp >> 2, w4 = warp & 3;

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + CF::OFF_BAR);
  uint64_t* st_full = bar;
  uint64_t* st_empty = st_full + CF::NS;
  uint64_t* s_full = st_empty + CF::NS;   // S^T and A^T written
  uint64_t* s_read = s_full + 1;          // mask warpgroup has read both
  uint64_t* p_full = s_read + 1;          // P^T and Pd^T written
  uint64_t* p_empty = p_full + 1;
  uint64_t* snap_full = p_empty + 1;
  uint64_t* u_updated = snap_full + 1;
  uint64_t* g_full = u_updated + 1;       // dK, dV complete
  uint64_t* g_empty = g_full + 1;
  uint64_t* drain = g_empty + 1;
  uint64_t* stage_free = drain + 1;       // transposing epilogue: staging tiles free
  uint64_t* stage_full = stage_free + 1;  // transposing epilogue: staging tiles written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + CF::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int64_t unit = blockIdx.x;
  const int64_t bh = unit / prm.C, c = unit % prm.C;  // bh: the K/V sequence
  const bool causal = prm.causal != 0;
  const bool split = causal && prm.split > 0;
  const int64_t t0 = split ? (c == 0 ? 0 : prm.split) : c * prm.L;
  const int64_t t1 = split ? (c == 0 ? prm.split : prm.N) : min(prm.N, t0 + prm.L);
  const int nblk = static_cast<int>((t1 - t0 + BK - 1) / BK);
  // query heads walked per block (the non-causal form needs only K, V and U)
  const int gq = causal && prm.G > 1 ? prm.G : 1;
  const int nsteps = nblk * gq;
  const int64_t q0 = q_seq0(bh, prm.H, prm.G);
  // In-kernel suffix state: chunk 0 of a split walks the later blocks first
  // (t1 is a multiple of BK there), from the last block of the sequence down.
  // Its steps need only Q and dO: two of them share a stage of the ring
  // (tiles 0, 3 and 1, 2), so twice as many of their loads are in flight.
  const int64_t nblk_seq = (prm.N + BK - 1) / BK;
  const int npre = split && c == 0 ? static_cast<int>(nblk_seq - t1 / BK) * gq : 0;
  const int npair = (npre + 1) / 2;  // ring steps of the pre-pass
  const bool has_init = !causal || (!split && prm.init_u && (c + 1 < prm.C || prm.init_all));
  const bool has_u0 = has_init || npre > 0;  // U is non-zero before the first own block
  const float* init = nullptr;
  // states added at init: one scanned slot, or the raw states of chunks
  // [c0, C) of the sequence (the later chunks, or all of them without the mask)
  int64_t c0 = 0, nsum = 1;
  if (!causal) {
    init = prm.init_u + bh * prm.C * static_cast<int64_t>(D * DV);
    nsum = prm.sum_states ? prm.C : 1;
  } else if (has_init) {
    c0 = prm.sum_states ? c + 1 : c;
    nsum = prm.sum_states ? prm.C - c - 1 : 1;
    init = prm.init_u + (bh * prm.C + c0) * static_cast<int64_t>(D * DV);
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < CF::NS; ++s) { mbar_init(&st_full[s], 1); mbar_init(&st_empty[s], 1); }
    mbar_init(s_full, 1);
    mbar_init(s_read, 128);
    mbar_init(p_full, 128);
    mbar_init(p_empty, 1);
    mbar_init(snap_full, 128);
    mbar_init(u_updated, 1);
    mbar_init(g_full, 1);
    mbar_init(g_empty, 128);
    mbar_init(drain, 1);
    mbar_init(stage_free, 1);
    mbar_init(stage_full, 128);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kWarpProducer && lane == 0) {
    tma_prefetch(&tm_q);
    tma_prefetch(&tm_k);
    tma_prefetch(&tm_v);
    tma_prefetch(&tm_do);
    if (CF::TMA_STORE) {
      tma_prefetch(&tm_dk);
      tma_prefetch(&tm_dv);
    }
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
  pdl_launch_dependents();  // global memory is touched only after this point
  pdl_wait();
  uint8_t* sStage = smem + CF::OFF_ST;
  uint8_t* sPT = smem + CF::OFF_PT;
  uint8_t* sPdT = smem + CF::OFF_PDT;
  uint8_t* sSnap = smem + CF::OFF_SNAP;
  // tile t of stage s: 0 = Q, 1 = K, 2 = V, 3 = dO ([BK rows x 128], two 64-column panels)
  auto tile = [&](int s, int t) { return sStage + s * CF::STAGE + t * CF::TILE; };

  if (warp == kWarpProducer) {
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      for (int s = 0; s < npair + nsteps && ok; ++s) {
        const int slot = s % CF::NS;
        if (!wait_bar(&st_empty[slot], ((s / CF::NS) & 1) ^ 1, lim, abort_flag, 201)) { ok = false; break; }
        if (s < npair) {  // suffix pre-pass: Q and dO of one or two later (block, head) steps
          const int n2 = min(2, npre - 2 * s);
          mbar_expect_tx(&st_full[slot], 2 * n2 * CF::TILE);
          for (int e = 0; e < n2; ++e) {
            const int sp = 2 * s + e;
            const int hq = static_cast<int>(q0 + sp % gq);
            const int row = static_cast<int>((nblk_seq - 1 - sp / gq) * BK);
            const int tq = e == 0 ? 0 : 1, tdo = e == 0 ? 3 : 2;
            for (int p = 0; p < 2; ++p) {
              tma_load_3d(tile(slot, tq) + p * BK * 128, &tm_q, &st_full[slot], 64 * p, row, hq);
              tma_load_3d(tile(slot, tdo) + p * BK * 128, &tm_do, &st_full[slot], 64 * p, row, hq);
            }
          }
          ++issued;
          continue;
        }
        const int sm = s - npair;
        const int hq = static_cast<int>(q0 + sm % gq);  // query sequence of Q and dO
        const int row = static_cast<int>(t0 + static_cast<int64_t>(nblk - 1 - sm / gq) * BK);  // reverse order
        mbar_expect_tx(&st_full[slot], causal ? 4 * CF::TILE : 2 * CF::TILE);
        const CUtensorMap* maps[4] = {&tm_q, &tm_k, &tm_v, &tm_do};
        for (int t = 0; t < 4; ++t) {
          if (!causal && (t == 0 || t == 3)) continue;  // non-causal needs only K and V
          const int z = (t == 0 || t == 3) ? hq : static_cast<int>(bh);
          for (int p = 0; p < 2; ++p)
            tma_load_3d(tile(slot, t) + p * BK * 128, maps[t], &st_full[slot], 64 * p, row, z);
        }
        ++issued;
      }
      if (!ok)
        for (int j = max(0, issued - CF::NS); j < issued; ++j) drain_wait(&st_full[j % CF::NS], (j / CF::NS) & 1);
    }
  } else if (warp == kWarpMma) {
    // The whole warp runs the issue loop; one elected lane issues each
    // tcgen05 instruction.
    {
      auto wait_w = [&](uint64_t* b, uint32_t par, int where) -> bool {
        return __all_sync(0xffffffffu, wait_bar(b, par, lim, abort_flag, where));
      };
      const uint64_t dKm = make_desc(0, 16, 1024);
      const uint64_t dMN = make_desc(0, BK * 128, 1024);
      const uint64_t dSnapMN = make_desc(0, D * 128, 1024);
      const uint32_t tU = tmem + CF::COL_U, tDV = tmem + CF::COL_DV, tDK = tmem + CF::COL_DK;
      const uint32_t tST = tmem + CF::COL_ST, tAT = tmem + CF::COL_AT;
      const uint32_t snap0 = smem_u32(sSnap), pt0 = smem_u32(sPT), pdt0 = smem_u32(sPdT);
      int snap_ph = 0;
      bool ok = true;
      // Suffix pre-pass: U = sum of Q^T dO over the later blocks (fresh U on
      // the first step); its completion is the first u_updated phase.
      for (int s = 0; s < npair && ok; ++s) {
        const int slot = s % CF::NS;
        if (!wait_w(&st_full[slot], (s / CF::NS) & 1, 217)) { ok = false; break; }
        tc_fence_after();
        const int n2 = min(2, npre - 2 * s);
        for (int e = 0; e < n2; ++e) {
          const uint32_t aq = smem_u32(tile(slot, e == 0 ? 0 : 1));
          const uint32_t ado = smem_u32(tile(slot, e == 0 ? 3 : 2));
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16_ss_warp(tU, dMN + (aq >> 4) + kk * (2048 >> 4), dMN + (ado >> 4) + kk * (2048 >> 4),
                             CF::ID_UPD, (s > 0 || e > 0 || kk > 0) ? 1u : 0u);
        }
        if (s == npair - 1) mma_commit_warp(u_updated);
        mma_commit_warp(&st_empty[slot]);
      }
      for (int sm = 0; sm < nsteps && ok; ++sm) {
        const int s = sm;                       // own-block step (mask and P barriers)
        const int gs = npair + sm;              // step of the stage ring
        const int slot = gs % CF::NS;
        const int blk = s / gq;                 // block counter (reverse order)
        const bool first = s % gq == 0;         // first query head of the block
        const bool last = s % gq == gq - 1;     // last query head of the block
        const uint32_t aq = smem_u32(tile(slot, 0)), ak = smem_u32(tile(slot, 1));
        const uint32_t av = smem_u32(tile(slot, 2)), ado = smem_u32(tile(slot, 3));
        if (!wait_w(&st_full[slot], (gs / CF::NS) & 1, 210)) { ok = false; break; }
        // A^T aliasing dK: the epilogue must have read the last block's dK
        if (!CF::AT_OWN && !wait_w(g_empty, (blk & 1) ^ 1, 211)) { ok = false; break; }
        const bool have_u = blk > 0 || has_u0;
        if (causal) {
          if (!wait_w(s_read, (s & 1) ^ 1, 212)) { ok = false; break; }
          tc_fence_after();
          // S^T = K Q^T and A^T = V dO^T (both K-major operands, K = 128)
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = ((kk >> 2) * BK * 128 + (kk & 3) * 32) >> 4;
            mma_bf16_ss_warp(tST, dKm + (ak >> 4) + off, dKm + (aq >> 4) + off, CF::ID_ST, kk > 0);
          }
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = ((kk >> 2) * BK * 128 + (kk & 3) * 32) >> 4;
            mma_bf16_ss_warp(tAT, dKm + (av >> 4) + off, dKm + (ado >> 4) + off, CF::ID_ST, kk > 0);
          }
          mma_commit_warp(s_full);
        }
        // the dK/dV accumulators must be free (the epilogue read the last block's)
        if (CF::AT_OWN && first && !wait_w(g_empty, (blk & 1) ^ 1, 216)) { ok = false; break; }
        if (have_u && first && (causal || s == 0)) {
          if (!wait_w(snap_full, snap_ph, 213)) { ok = false; break; }
          snap_ph ^= 1;
        }
        tc_fence_after();
        if (have_u && first) {
          // dV = K U: A = K (K-major, K = d), B[n=e][k=c] = U[c][e] (snapshot, MN-major);
          // transposed: dV^T = U^T K^T, A[m=e][k=c] = U[c][e] (MN-major), B = K (K-major)
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = ((kk >> 2) * BK * 128 + (kk & 3) * 32) >> 4;
            if constexpr (CF::OT)
              mma_bf16_ss_warp(tDV, dSnapMN + (snap0 >> 4) + kk * (2048 >> 4), dKm + (ak >> 4) + off,
                               CF::ID_T_MK, kk > 0);
            else
              mma_bf16_ss_warp(tDV, dKm + (ak >> 4) + off, dSnapMN + (snap0 >> 4) + kk * (2048 >> 4),
                               CF::ID_MN, kk > 0);
          }
        }
        if (causal) {
          // U += Q^T dO (after the snapshot of the old U was taken)
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16_ss_warp(tU, dMN + (aq >> 4) + kk * (2048 >> 4), dMN + (ado >> 4) + kk * (2048 >> 4),
                        CF::ID_UPD, (have_u || !first || kk > 0) ? 1u : 0u);
          // A^T aliasing dK: the mask warpgroup must have read it
          if (!CF::AT_OWN) {
            if (!wait_w(s_read, s & 1, 214)) { ok = false; break; }
            tc_fence_after();
          }
        }
        if (have_u && first) {
          // dK = V U^T: A = V (K-major, K = dv), B[n=c][k=e] = U[c][e] (snapshot, K-major)
          // transposed: dK^T = U V^T, A[m=c][k=e] = U[c][e] (K-major), B = V (K-major)
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = ((kk >> 2) * BK * 128 + (kk & 3) * 32) >> 4;
            const uint32_t soff = ((kk >> 2) * D * 128 + (kk & 3) * 32) >> 4;
            if constexpr (CF::OT)
              mma_bf16_ss_warp(tDK, dKm + (snap0 >> 4) + soff, dKm + (av >> 4) + off, CF::ID_T_KK, kk > 0);
            else
              mma_bf16_ss_warp(tDK, dKm + (av >> 4) + off, dKm + (snap0 >> 4) + soff, CF::ID_KM, kk > 0);
          }
        }
        // U is updated (by every query head of the block) and no issued MMA
        // reads the snapshot any more: the state warpgroup may take the next one
        if (causal && last) mma_commit_warp(u_updated);
        if (causal) {
          if (!wait_w(p_full, s & 1, 215)) { ok = false; break; }
          tc_fence_after();
          const uint32_t acc0 = (have_u || !first) ? 1u : 0u;
          // dV += P^T dO ; dK += Pd^T Q  (A = masked tiles, K-major, K = BK; B MN-major);
          // transposed: dV^T += dO^T P, dK^T += Q^T Pd (A MN-major, B = masked tiles)
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * BK * 128 + (kk & 3) * 32) >> 4;
            const uint32_t acc = (acc0 || kk > 0) ? 1u : 0u;
            if constexpr (CF::OT)
              mma_bf16_ss_warp(tDV, dMN + (ado >> 4) + kk * (2048 >> 4), dKm + (pt0 >> 4) + off,
                               CF::ID_T_MK, acc);
            else
              mma_bf16_ss_warp(tDV, dKm + (pt0 >> 4) + off, dMN + (ado >> 4) + kk * (2048 >> 4),
                               CF::ID_MN, acc);
          }
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * BK * 128 + (kk & 3) * 32) >> 4;
            const uint32_t acc = (acc0 || kk > 0) ? 1u : 0u;
            if constexpr (CF::OT)
              mma_bf16_ss_warp(tDK, dMN + (aq >> 4) + kk * (2048 >> 4), dKm + (pdt0 >> 4) + off,
                               CF::ID_T_MK, acc);
            else
              mma_bf16_ss_warp(tDK, dKm + (pdt0 >> 4) + off, dMN + (aq >> 4) + kk * (2048 >> 4),
                               CF::ID_MN, acc);
          }
          mma_commit_warp(p_empty);
        }
        if (last) mma_commit_warp(g_full);
        mma_commit_warp(&st_empty[slot]);
      }
      mma_commit_warp(drain);
      drain_wait(drain, 0);
    }
  } else if (wg == kWgMask) {
    // S^T, A^T (TMEM, rows = keys j, columns = queries t) -> keep t >= j -> bf16 P^T, Pd^T
    if (causal) {
      const int r = acc_row<BK>(w4, lane);
      const uint32_t lane_off = static_cast<uint32_t>(32 * w4) << 16;
      const uint32_t bases[2] = {smem_u32(sPT), smem_u32(sPdT)};
      const uint32_t srcs[2] = {tmem + CF::COL_ST + lane_off, tmem + CF::COL_AT + lane_off};
      for (int s = 0; s < nsteps; ++s) {
        if (!__all_sync(0xffffffffu, wait_bar(s_full, s & 1, lim, abort_flag, 220))) break;
        if (!__all_sync(0xffffffffu, wait_bar(p_empty, (s & 1) ^ 1, lim, abort_flag, 221))) break;
        tc_fence_after();
        for (int which = 0; which < 2; ++which) {
#pragma unroll
          for (int c32 = 0; c32 < BK / 32; ++c32) {
            uint32_t v[32];
            tmem_ld32(srcs[which] + c32 * 32, v);
            tmem_ld_wait();
            if (r >= 0) {
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int col = c32 * 32 + q4 * 8 + 2 * e;
                  const float a = (col >= r) ? __uint_as_float(v[q4 * 8 + 2 * e]) : 0.f;
                  const float b = (col + 1 >= r) ? __uint_as_float(v[q4 * 8 + 2 * e + 1]) : 0.f;
                  w[e] = pack_bf16x2(a, b);
                }
                const int ch = c32 * 4 + q4;
                const int panel = ch >> 3, cj = ch & 7;
                st_shared_v4(bases[which] + panel * BK * 128 + r * 128 + ((cj ^ (r & 7)) << 4), w[0],
                             w[1], w[2], w[3]);
              }
            }
          }
        }
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(s_read);
        mbar_arrive(p_full);
      }
    }
  } else if (wg == kWgState) {
    // bf16 snapshot of U (rows c, 64-column panels); initial U from HBM
    const int r = acc_row<D>(w4, lane);
    const uint32_t lane_off = static_cast<uint32_t>(32 * w4) << 16;
    const uint32_t tU = tmem + CF::COL_U + lane_off;
    const uint32_t sbase = smem_u32(sSnap);
    auto put_row = [&](const uint32_t* v, int col0) {
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
    };
    if (has_init) {
#pragma unroll 1
      for (int c32 = 0; c32 < DV / 32; ++c32) {
        float acc[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = 0.f;
        for (int64_t cc = 0; cc < nsum; ++cc) {  // chunk states in chunk order
          const float4* src = reinterpret_cast<const float4*>(init + cc * static_cast<int64_t>(D * DV));
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 x = src[state_f4<D>(r, c32 * 8 + q4)];
            acc[4 * q4] += x.x;
            acc[4 * q4 + 1] += x.y;
            acc[4 * q4 + 2] += x.z;
            acc[4 * q4 + 3] += x.w;
          }
        }
        uint32_t u[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(acc[j]);
        if (causal) tmem_st32(tU + c32 * 32, u);
        put_row(u, c32 * 32);
      }
      if (causal) tmem_st_wait();
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(snap_full);
    }
    bool ok_pre = true;
    if (npre > 0) {  // U from the suffix pre-pass: snapshot it once it is complete
      ok_pre = __all_sync(0xffffffffu, wait_bar(u_updated, 0, lim, abort_flag, 231));
      if (ok_pre) {
        tc_fence_after();
#pragma unroll
        for (int c32 = 0; c32 < DV / 32; ++c32) {
          uint32_t v[32];
          tmem_ld32(tU + c32 * 32, v);
          tmem_ld_wait();
          put_row(v, c32 * 32);
        }
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(snap_full);
      }
    }
    if (causal && ok_pre) {
      const int ph0 = npre > 0 ? 1 : 0;  // the pre-pass took the first u_updated phase
      for (int s = 0; s + 1 < nblk; ++s) {
        if (!__all_sync(0xffffffffu, wait_bar(u_updated, (s + ph0) & 1, lim, abort_flag, 230))) break;
        // the snapshot buffer is free: every MMA reading it was issued before
        // the update whose completion u_updated reports
        tc_fence_after();
#pragma unroll
        for (int c32 = 0; c32 < DV / 32; ++c32) {
          uint32_t v[32];
          tmem_ld32(tU + c32 * 32, v);
          tmem_ld_wait();
          put_row(v, c32 * 32);
        }
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(snap_full);
      }
    }
  } else if (wg == kWgEpilogue) {
    // dV, dK (TMEM, fp32) -> bf16 -> HBM rows
    const int r = acc_row<BK>(w4, lane);
    const uint32_t lane_off = static_cast<uint32_t>(32 * w4) << 16;
    for (int s = 0; s < nblk; ++s) {
      const int i = nblk - 1 - s;
      if (!__all_sync(0xffffffffu, wait_bar(g_full, s & 1, lim, abort_flag, 240))) break;
      tc_fence_after();
      if constexpr (CF::OT) {
        // Thread (w4, lane) holds column x = 32 w4 + lane of dV and of dK for the
        // BK rows of the block (TMEM lane x, one column per row). It writes them
        // into the two staging tiles in the TMA layout (128B-swizzled 64-column
        // panels, rows = keys); the first warp then stores both tiles. The four
        // warps meet on mbarriers with bounded waits.
        const int x = 32 * w4 + lane;
        const uint32_t ph = s & 1;
        if (threadIdx.x % 128 == 0) {
          bulk_wait_group_read<0>();  // the last block's stores have read the tiles
          mbar_arrive(stage_free);
        }
        if (!__all_sync(0xffffffffu, wait_bar(stage_free, ph, lim, abort_flag, 241))) break;
        const int chunk = (x & 63) >> 3;
        for (int which = 0; which < 2; ++which) {
          const uint32_t src = tmem + (which == 0 ? CF::COL_DV : CF::COL_DK) + lane_off;
          const uint32_t col_base =
              smem_u32(smem + CF::OFF_OST + which * CF::TILE + (x >> 6) * BK * 128) + (x & 7) * 2;
#pragma unroll
          for (int c32 = 0; c32 < BK / 32; ++c32) {
            uint32_t v[32];
            tmem_ld32(src + c32 * 32, v);
            tmem_ld_wait();
            if (which == 1 && c32 == BK / 32 - 1) {  // every TMEM read of this block is done
              tc_fence_before();
              mbar_arrive(g_empty);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int t = c32 * 32 + j;  // key row of the block
              st_shared_u16(col_base + t * 128 + ((chunk ^ (t & 7)) << 4),
                            bf16_bits(__uint_as_float(v[j])));
            }
          }
        }
        fence_proxy_async();
        mbar_arrive(stage_full);
        if (w4 == 0) {
          if (!__all_sync(0xffffffffu, wait_bar(stage_full, ph, lim, abort_flag, 242))) break;
          if (lane == 0) {
            // chunks end on block boundaries or at N (the tensor maps clip at N)
            const int64_t y = t0 + static_cast<int64_t>(i) * BK;
            for (int which = 0; which < 2; ++which) {
              uint8_t* stage = smem + CF::OFF_OST + which * CF::TILE;
              const CUtensorMap* map = which == 0 ? &tm_dv : &tm_dk;
#pragma unroll
              for (int p = 0; p < 2; ++p)
                tma_store_3d(map, stage + p * BK * 128, 64 * p, static_cast<int>(y),
                             static_cast<int>(bh));
            }
            bulk_commit_group();
          }
        }
        continue;
      }
      if constexpr (CF::TMA_STORE) {
        // Warp w4 stages its 16 rows of dV and dK (128B-swizzled 64-column
        // panels) and stores them with TMA.
        if (lane == 0) bulk_wait_group_read<0>();  // this warp's stores of the last block have read
        __syncwarp();
        const int rl = lane & 15;
        for (int which = 0; which < 2; ++which) {
          uint8_t* stage = smem + CF::OFF_OST + which * CF::TILE + w4 * 16 * 128;
          const uint32_t src = tmem + (which == 0 ? CF::COL_DV : CF::COL_DK) + lane_off;
#pragma unroll
          for (int c32 = 0; c32 < 128 / 32; ++c32) {
            uint32_t v[32];
            tmem_ld32(src + c32 * 32, v);
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
        }
        tc_fence_before();
        mbar_arrive(g_empty);
        fence_proxy_async();
        __syncwarp();
        // chunks end on block boundaries or at N (the tensor maps clip at N)
        const int64_t y = t0 + static_cast<int64_t>(i) * BK + 16 * w4;
        if (lane == 0) {
          if (y < t1) {
            for (int which = 0; which < 2; ++which) {
              uint8_t* stage = smem + CF::OFF_OST + which * CF::TILE + w4 * 16 * 128;
              const CUtensorMap* map = which == 0 ? &tm_dv : &tm_dk;
#pragma unroll
              for (int p = 0; p < 2; ++p)
                tma_store_3d(map, stage + p * BK * 128, 64 * p, static_cast<int>(y),
                             static_cast<int>(bh));
            }
          }
          bulk_commit_group();  // one group per block, empty past the end
        }
        continue;
      }
      const int64_t row = t0 + static_cast<int64_t>(i) * BK + r;
      const bool valid = r >= 0 && row < t1;
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* outp = which == 0 ? prm.dv : prm.dk;
        const int W = which == 0 ? DV : D;
        const uint32_t src = tmem + (which == 0 ? CF::COL_DV : CF::COL_DK) + lane_off;
        uint4* dst = reinterpret_cast<uint4*>(outp + (bh * prm.N + (valid ? row : 0)) * W);
#pragma unroll
        for (int c32 = 0; c32 < 128 / 32; ++c32) {
          uint32_t v[32];
          tmem_ld32(src + c32 * 32, v);
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
      }
      tc_fence_before();
      mbar_arrive(g_empty);
    }
    if (CF::TMA_STORE && lane == 0) bulk_wait_group<0>();  // stores done before exit
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace sm100

template <int BK>
inline la2_status launch_bwd_dkdv_sm100(const CUtensorMap& tq, const CUtensorMap& tk,
                                        const CUtensorMap& tv, const CUtensorMap& tdo,
                                        const CUtensorMap& tdk, const CUtensorMap& tdv,
                                        const sm100::BwdParams& p, int64_t units, cudaStream_t st) {
  using CF = sm100::BCfg<BK, 128, 128>;
  auto kern = sm100::la2_bwd_dkdv_sm100_kernel<BK, 128, 128>;
  static bool attr_done[128];
  if (!smem_attribute_set(kern, CF::SMEM, attr_done)) return LA2_ERR_CUDA;
  if (launch_pdl(kern, dim3(static_cast<unsigned>(units)), dim3(sm100::kThreads), CF::SMEM, st, tq,
                 tk, tv, tdo, tdk, tdv, p) != cudaSuccess)
    return LA2_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? LA2_OK : LA2_ERR_CUDA;
}

}  // namespace la2
